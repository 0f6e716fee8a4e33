"""Attention-fidelity diagnostics on the GPU against the oracle.

Per query row the CUDA path returns both log-sum-exps, the cached mass of the reference and the
quantised softmax, KL(P_ref || P_q), top-1 agreement (token drift, pchao.org 'QuantWM', section
实验如何设计) and top-5 recall (gist.science, 'Statistical Inference and Quality Measures of KV Cache
Quantisations Inspired by TurboQuant', section Métricas de Avaliação), plus both top-5 key lists.

Tolerances, from the fp32 arithmetic of the kernel (each score a 4-way split fp32 dot product, then
running fp32 sums): a score is within ~1e-5 of its fp64 value on these inputs, so LSEs and masses
agree to 2e-4 and the KL to 2e-4 + 1e-3 KL. Top lists are decided in fp32: where the oracle's
(fp64) top-6 scores are separated by more than the score tolerance the lists must be identical;
otherwise every listed key must hold, by the oracle's scores, the rank it is listed at (within the
tolerance), and agreement / recall must be those of the returned lists.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from quantized_kv_cache_19_b200 import api
from quantized_kv_cache_19_b200.workloads import WORKLOADS, make_inputs, sample_rows

from parity_utils import build_gpu_cache, np32, sub_problem

pytestmark = pytest.mark.gpu

LSE_TOL = 2e-4
MASS_TOL = 2e-4
KL_ABS, KL_REL = 2e-4, 1e-3
FULL_LSE_TOL = 1e-3          # sums over up to ~1e5 keys per row at the full sizes


def _score_tol(s):
    return 1e-4 + 1e-5 * np.abs(s)


def run_gpu(w, x, cache, correct, with_top=True):
    K_ref = x["K_src"] if w.Lc else None
    K_cur = x["K_cur"] if w.Lcur else None
    st, top = api.attention_fidelity(x["Q"], cache, K_ref, K_cur, correct=correct, causal=w.causal,
                                     with_top=with_top)
    torch.cuda.synchronize()
    return st, top


def oracle_rows(w, x, b, h, correct, rows, key_block=0):
    """The oracle on packed rows `rows` (head_in_group * Lq + i) of (batch b, KV head h)."""
    sub = sub_problem(x, w, b, h)
    d = w.d
    group = 1 if key_block else w.group
    if w.Lc:
        c = oracle.build_cache(sub["K_src"], sub["V_src"], w.bits, w.group, w.meta, key_block=key_block)
        kh, _, ks = oracle.cache_rows(c, 0, 0)
        k_ref = sub["K_src"][0, 0]
    else:
        kh, ks, k_ref = np.zeros((0, d)), np.zeros((0, d // group)), np.zeros((0, d))
    k_cur = sub["K_cur"][0, 0] if w.Lcur else np.zeros((0, d))
    rows = np.asarray(rows)
    q = sub["Q"][0][rows // w.Lq, rows % w.Lq]
    return oracle.fidelity_rows(q, rows % w.Lq, k_ref, kh, ks, group, k_cur, correct, w.causal,
                                1.0 / math.sqrt(d), w.Lq, return_scores=True)


def gpu_rows(w, st, top, b, h, rows):
    r = w.Hq // w.Hkv
    rows = np.asarray(rows)
    hq = torch.as_tensor(h * r + rows // w.Lq)
    qi = torch.as_tensor(rows % w.Lq)
    return np32(st[b, hq, qi]).astype(np.float64), top[b, hq, qi].cpu().numpy()


def _check_list(s, got, want, what):
    vis = np.isfinite(s)
    n = int(min(5, vis.sum()))
    assert np.all(got[n:] == -1), f"{what}: padding {got}"
    idx = got[:n]
    assert len(set(idx.tolist())) == n and np.all((idx >= 0) & (idx < s.size)) and np.all(vis[idx]), \
        f"{what}: invalid list {got}"
    best = np.sort(s[vis])[::-1]
    assert np.all(np.abs(s[idx] - best[:n]) <= _score_tol(best[:n])), f"{what}: ranks {got} vs {want}"
    top6 = best[:n + 1]
    unique = np.all(-np.diff(top6) > 2 * _score_tol(top6[1:])) if top6.size > 1 else True
    if unique:
        assert np.array_equal(idx, want[:n]), f"{what}: {got} vs {want}"
    return unique


def compare(st, top, f, what, lse_tol=LSE_TOL):
    fin = np.isfinite(f["lse_ref"])
    assert np.array_equal(np.isfinite(st[:, 0]), fin), f"{what}: rows without keys differ"
    assert np.array_equal(np.isfinite(st[:, 1]), np.isfinite(f["lse_q"]))
    errs = {
        "lse_ref": np.max(np.abs(st[fin, 0] - f["lse_ref"][fin]), initial=0.0),
        "lse_q": np.max(np.abs(st[fin, 1] - f["lse_q"][fin]), initial=0.0),
        "mass_ref": np.max(np.abs(st[:, 2] - f["mass_ref"]), initial=0.0),
        "mass_q": np.max(np.abs(st[:, 3] - f["mass_q"]), initial=0.0),
    }
    assert errs["lse_ref"] <= lse_tol and errs["lse_q"] <= lse_tol, f"{what}: {errs}"
    assert errs["mass_ref"] <= MASS_TOL and errs["mass_q"] <= MASS_TOL, f"{what}: {errs}"
    kl_err = np.abs(st[:, 4] - f["kl"]) - KL_REL * f["kl"]
    assert np.max(kl_err, initial=0.0) <= KL_ABS, f"{what}: KL error {np.max(kl_err):.3e}"
    assert np.all(st[:, 7] == 0)
    for i in range(st.shape[0]):
        u_r = _check_list(f["s_ref"][i], top[i, 0], f["top_ref"][i], f"{what} row {i} ref")
        u_q = _check_list(f["s_q"][i], top[i, 1], f["top_q"][i], f"{what} row {i} quant")
        r_list = top[i, 0][top[i, 0] >= 0]
        agree = 1.0 if r_list.size == 0 else float(top[i, 0, 0] == top[i, 1, 0])
        recall = 1.0 if r_list.size == 0 else np.isin(r_list, top[i, 1]).sum() / r_list.size
        assert st[i, 5] == agree and st[i, 6] == pytest.approx(recall, abs=1e-7), f"{what} row {i}"
        if u_r and u_q:
            assert st[i, 5] == f["top1_agree"][i] and st[i, 6] == pytest.approx(f["recall"][i], abs=1e-7)
    return errs


def chan_cache(w, K, V, T):
    cache = api.KVCache(w.B, w.Hkv, w.d, w.bits, w.group, api.round_capacity(w.Lc), w.meta,
                        device=K.device, key_block=T)
    if w.Lc:
        api.kv_quantize_append(cache, K, V)
    return cache


def check_all_rows(w, correct, seed=None, key_block=0):
    x = make_inputs(w, device="cuda", seed=seed)
    if key_block:
        cache = chan_cache(w, x["K_src"], x["V_src"], key_block)
    else:
        cache = build_gpu_cache(w, x["K_src"], x["V_src"])
    st, top = run_gpu(w, x, cache, correct)
    rows = np.arange(w.rows_per_kv_head)
    for b in range(w.B):
        for h in range(w.Hkv):
            f = oracle_rows(w, x, b, h, correct, rows, key_block)
            s, t = gpu_rows(w, st, top, b, h, rows)
            compare(s, t, f, f"{w.name} b{b} h{h} correct={correct}")
    assert api.device_status() == 0
    return x, cache, st


SMALL = {
    "tiny_f32": WORKLOADS["tiny_f32"],
    "bf16_int4": WORKLOADS["bf16_int4"].with_(Hq=2, Hkv=2, Lq=100, Lcur=100, Lc=300),
    "bf16_int2": WORKLOADS["bf16_int2"].with_(Hq=2, Hkv=2, Lq=100, Lcur=100, Lc=300),
    "long_video": WORKLOADS["long_video"].with_(Hq=2, Hkv=2, Lq=70, Lcur=70, Lc=500),
    "prefill_gqa": WORKLOADS["prefill_gqa"].with_(B=2, Hq=8, Hkv=2, Lq=45, Lcur=45, Lc=333),
}


@pytest.mark.parametrize("name", sorted(SMALL))
@pytest.mark.parametrize("correct", [0, 1, 2])
def test_every_row(name, correct):
    check_all_rows(SMALL[name], correct)


def test_empty_cache_and_empty_current_chunk():
    w = SMALL["bf16_int2"]
    check_all_rows(w.with_(Lc=0), 1)
    check_all_rows(w.with_(Lcur=0), 1)


def test_rows_without_keys():
    # no cache and a causal current chunk shorter than the query chunk: the first rows see nothing
    w = SMALL["prefill_gqa"].with_(Lc=0, Lcur=20, causal=True)
    x, _, st = check_all_rows(w, 1)
    s = np32(st)
    empty = s[:, :, : w.Lq - w.Lcur]
    assert np.all(np.isneginf(empty[..., 0])) and np.all(empty[..., 2:5] == 0) and np.all(empty[..., 5:7] == 1)


def test_equal_scores_list_lower_index_first():
    # every cached key repeated four times: equal codes, equal fp32 scores, ties broken by index
    w = SMALL["bf16_int2"].with_(Lc=64, Lcur=0)
    x = make_inputs(w, device="cuda")
    x["K_src"] = x["K_src"][:, :, :16].repeat_interleave(4, dim=2).contiguous()
    cache = build_gpu_cache(w, x["K_src"], x["V_src"])
    st, top = run_gpu(w, x, cache, 1)
    t = top.cpu().numpy()
    for lst in (t[..., 0, :], t[..., 1, :]):
        assert np.all(lst[..., 0] % 4 == 0) and np.all(lst[..., 1:4] - lst[..., :1] == [1, 2, 3])
    rows = np.arange(w.rows_per_kv_head)
    for h in range(w.Hkv):
        f = oracle_rows(w, x, 0, h, 1, rows)
        s_, t_ = gpu_rows(w, st, top, 0, h, rows)
        compare(s_, t_, f, f"ties h{h}")


def test_lse_q_matches_corrected_attention():
    """P_q is the corrected attention's distribution: the fidelity LSE_q and corrected_attention's LSE
    agree within the attention kernel's own tolerance (bf16 operands there, fp32 here)."""
    w = SMALL["prefill_gqa"]
    x = make_inputs(w, device="cuda")
    cache = build_gpu_cache(w, x["K_src"], x["V_src"])
    for correct in (0, 1, 2):
        st, _ = run_gpu(w, x, cache, correct, with_top=False)
        _, lse = api.corrected_attention(x["Q"], cache, x["K_cur"], x["V_cur"], correct=correct, causal=True)
        torch.cuda.synchronize()
        assert torch.max(torch.abs(st[..., 1] - lse)).item() <= 2e-3


@pytest.mark.parametrize("name,heads", [
    ("bf16_int2", [(0, 0), (0, 11)]),
    ("bf16_int4", [(0, 5)]),
    ("video_dit", [(0, 0), (0, 17)]),
    ("long_video", [(0, 3), (0, 39)]),
    ("prefill_gqa", [(0, 0), (3, 7)]),
])
def test_full_size_sampled_rows(name, heads):
    """The full workload in one launch; 64 sampled rows of a few (batch, KV head) pairs."""
    w = WORKLOADS[name]
    x = make_inputs(w, device="cuda")
    cache = build_gpu_cache(w, x["K_src"], x["V_src"], chunk=w.Lcur)
    st, top = run_gpu(w, x, cache, 1)
    rows = sample_rows(w, 64).numpy()
    for b, h in heads:
        f = oracle_rows(w, x, b, h, 1, rows)
        s, t = gpu_rows(w, st, top, b, h, rows)
        compare(s, t, f, f"{name} b{b} h{h}", lse_tol=FULL_LSE_TOL)
    assert api.device_status() == 0


def test_correction_restores_cached_mass_full_bf16_int2():
    """Over every row of the bf16 INT2 workload: quantised keys take extra cached mass, the correction
    gives most of it back and lowers the mean KL; the GPU's means match the oracle's on two heads."""
    w = WORKLOADS["bf16_int2"]
    x = make_inputs(w, device="cuda")
    cache = build_gpu_cache(w, x["K_src"], x["V_src"])
    s0, _ = run_gpu(w, x, cache, 0, with_top=False)
    s1, _ = run_gpu(w, x, cache, 1, with_top=False)
    gap0 = (s0[..., 3] - s0[..., 2]).mean().item()
    gap1 = (s1[..., 3] - s1[..., 2]).mean().item()
    assert gap0 > 0.1 and abs(gap1) < 0.5 * gap0
    assert s1[..., 4].mean().item() < s0[..., 4].mean().item()
    rows = np.arange(w.rows_per_kv_head)
    for h in (2, 9):
        for s, c in ((s0, 0), (s1, 1)):
            f = oracle_rows(w, x, 0, h, c, rows)
            g = np32(s[0, h])
            assert abs(g[:, 3].mean() - f["mass_q"].mean()) < 1e-5
            assert abs(g[:, 4].mean() - f["kl"].mean()) < 1e-4
            assert abs(g[:, 5].mean() - f["top1_agree"].mean()) < 0.01


@pytest.mark.parametrize("name", ["tiny_f32", "bf16_int2", "long_video", "prefill_gqa"])
@pytest.mark.parametrize("correct", [0, 1, 2])
def test_every_row_per_channel_keys(name, correct):
    """Caches with per-channel key blocks (32 positions): the correction uses each key's block steps."""
    check_all_rows(SMALL[name], correct, key_block=32)


def test_full_size_sampled_rows_per_channel_keys():
    w = WORKLOADS["bf16_int2"]
    x = make_inputs(w, device="cuda")
    cache = chan_cache(w, x["K_src"], x["V_src"], 32)
    st, top = run_gpu(w, x, cache, 1)
    rows = sample_rows(w, 64).numpy()
    for b, h in [(0, 1), (0, 14)]:
        f = oracle_rows(w, x, b, h, 1, rows, key_block=32)
        s, t = gpu_rows(w, st, top, b, h, rows)
        compare(s, t, f, f"bf16_int2 per-channel b{b} h{h}", lse_tol=FULL_LSE_TOL)
    assert api.device_status() == 0
