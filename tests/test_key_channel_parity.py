"""Per-channel keys along tokens (KIVI-style key blocks of T cache positions) on the GPU against the
oracle: the quantiser bit-exact, the correction term, and corrected attention on every row of small
workloads and on sampled rows at full size."""
import math

import numpy as np
import pytest
import torch

import oracle
from quantized_kv_cache_19_b200 import api
from quantized_kv_cache_19_b200.workloads import WORKLOADS, make_inputs, sample_rows

from parity_utils import BIAS_REL_TOL, compare, np32, sub_problem

pytestmark = pytest.mark.gpu


def build_chan_cache(w, K, V, T, chunk=None):
    L = K.shape[2]
    cache = api.KVCache(w.B, w.Hkv, w.d, w.bits, w.group, api.round_capacity(L), w.meta,
                        device=K.device, key_block=T)
    step = chunk or max(L, 1)
    assert step % T == 0 or step >= L
    for t0 in range(0, L, step):
        api.kv_quantize_append(cache, K[:, :, t0:t0 + step].contiguous(), V[:, :, t0:t0 + step].contiguous())
    assert cache.length == L
    return cache


SMALL = {
    "tiny_f32": WORKLOADS["tiny_f32"],
    "bf16_int4": WORKLOADS["bf16_int4"].with_(Hq=2, Hkv=2, Lq=100, Lcur=100, Lc=300),
    "bf16_int2": WORKLOADS["bf16_int2"].with_(Hq=2, Hkv=2, Lq=100, Lcur=100, Lc=300),
    "long_video": WORKLOADS["long_video"].with_(Hq=2, Hkv=2, Lq=70, Lcur=70, Lc=500),
    "prefill_gqa": WORKLOADS["prefill_gqa"].with_(B=2, Hq=8, Hkv=2, Lq=45, Lcur=45, Lc=333),
}


def check_quantiser(w, x, cache, T):
    Lc = w.Lc
    K, V = np32(x["K_src"]), np32(x["V_src"])
    kc, ks, kz = oracle.quantize_tokens(K, w.bits, T, w.meta)
    nb = ks.shape[2]
    got_kc = cache.codes("k")[:, :, :Lc].cpu().numpy()
    got_km = cache.meta_view("k")[:, :, :nb].cpu().numpy()
    np.testing.assert_array_equal(got_kc, oracle.pack_codes(kc, w.bits), err_msg=f"{w.name} T{T} key codes")
    np.testing.assert_array_equal(got_km[..., 0], ks, err_msg=f"{w.name} T{T} key steps")
    np.testing.assert_array_equal(got_km[..., 1], kz, err_msg=f"{w.name} T{T} key zero-points")
    vc, vs, vz = oracle.quantize(V, w.bits, w.group, w.meta)
    np.testing.assert_array_equal(cache.codes("v")[:, :, :Lc].cpu().numpy(), oracle.pack_codes(vc, w.bits))
    got_vm = cache.meta_view("v")[:, :, :Lc].cpu().numpy()
    np.testing.assert_array_equal(got_vm[..., 0], vs)
    np.testing.assert_array_equal(got_vm[..., 1], vz)


@pytest.mark.parametrize("name", sorted(SMALL))
@pytest.mark.parametrize("T", [32, 64, 128])
def test_quantiser_bit_exact(name, T):
    w = SMALL[name]
    x = make_inputs(w, device="cuda")
    cache = build_chan_cache(w, x["K_src"], x["V_src"], T, chunk=2 * T)     # ragged last block
    torch.cuda.synchronize()
    check_quantiser(w, x, cache, T)
    assert api.device_status() == 0


def oracle_head(w, sub, T, correct, rows=None):
    cache = oracle.build_cache(sub["K_src"], sub["V_src"], w.bits, w.group, w.meta, key_block=T) if w.Lc else None
    return oracle.corrected_attention(sub["Q"], cache, sub["K_cur"], sub["V_cur"], correct=correct,
                                      causal=w.causal, scale=1.0 / math.sqrt(w.d), rows=rows)


def check_every_row(w, T, correct, mode="auto"):
    """mode: "auto" (key split when the shape asks for it), "unsplit" (no workspace) or "noalloc"."""
    x = make_inputs(w, device="cuda")
    cache = build_chan_cache(w, x["K_src"], x["V_src"], T)
    Kc = x["K_cur"] if w.Lcur else None
    Vc = x["V_cur"] if w.Lcur else None
    if mode == "noalloc":
        O, LSE = api.corrected_attention_noalloc(x["Q"], cache, Kc, Vc, correct=correct, causal=w.causal)
    else:
        O, LSE = api.corrected_attention(x["Q"], cache, Kc, Vc, correct=correct, causal=w.causal,
                                         workspace="auto" if mode == "auto" else None)
    torch.cuda.synchronize()
    r = w.Hq // w.Hkv
    for b in range(w.B):
        for h in range(w.Hkv):
            O_ref, L_ref = oracle_head(w, sub_problem(x, w, b, h), T, correct)
            compare(np32(O[b:b + 1, h * r:(h + 1) * r]).astype(np.float64), O_ref,
                    np32(LSE[b:b + 1, h * r:(h + 1) * r]).astype(np.float64), L_ref,
                    f"{w.name} T{T} b{b} h{h} correct={correct}")
    assert api.device_status() == 0
    return O, LSE


@pytest.mark.parametrize("name", sorted(SMALL))
@pytest.mark.parametrize("correct", [0, 1, 2])
def test_attention_every_row(name, correct):
    check_every_row(SMALL[name], 32, correct)


@pytest.mark.parametrize("T", [64, 128])
def test_attention_other_block_sizes(T):
    check_every_row(SMALL["bf16_int2"], T, 1)
    check_every_row(SMALL["long_video"], T, 2)


def test_attention_edge_cases():
    w = SMALL["prefill_gqa"]
    check_every_row(w.with_(Lcur=0), 32, 1)                  # cache only
    check_every_row(w.with_(Lc=0), 32, 1)                    # current chunk only
    check_every_row(w.with_(Lq=1, Lcur=1), 64, 1)            # one query row per head
    check_every_row(w.with_(Lc=32 * 5, Lq=33, Lcur=20), 32, 2)   # whole blocks, short current chunk


def test_noalloc_entry_point_serves_per_channel_keys():
    """The allocation-free entry point runs per-channel caches unsplit: the same result as the
    workspace-free call."""
    w = SMALL["prefill_gqa"].with_(Lq=4, Lcur=4)
    O1, L1 = check_every_row(w, 32, 1, mode="noalloc")
    O2, L2 = check_every_row(w, 32, 1, mode="unsplit")
    assert torch.equal(O1, O2) and torch.equal(L1, L2)


@pytest.mark.parametrize("Lq,causal", [(1, True), (4, False), (16, True)])
def test_key_split_every_row_and_against_unsplit(Lq, causal):
    """Few query rows per KV head: the bf16 path splits the cached keys over CTAs and merges the
    partials. Every row against the oracle, and the split against the unsplit kernel."""
    w = SMALL["prefill_gqa"].with_(Lq=Lq, Lcur=Lq, Lc=32 * 40 + 9, causal=causal)
    cache = api.KVCache(w.B, w.Hkv, w.d, w.bits, w.group, api.round_capacity(w.Lc), w.meta, key_block=32)
    cache.length = w.Lc
    assert api.attention_workspace_bytes(cache, w.Hq, w.Lq, w.Lcur) > 0
    O1, L1 = check_every_row(w, 32, 1, mode="auto")
    O2, L2 = check_every_row(w, 32, 1, mode="unsplit")
    compare(np32(O1).astype(np.float64), np32(O2).astype(np.float64), np32(L1).astype(np.float64),
            np32(L2).astype(np.float64), f"per-channel split vs unsplit Lq={Lq}")


@pytest.mark.parametrize("name", ["tiny_f32", "bf16_int2", "long_video"])
def test_correction_term(name):
    w = SMALL[name]
    T = 32
    x = make_inputs(w, device="cuda")
    cache = build_chan_cache(w, x["K_src"], x["V_src"], T)
    bias = api.jensen_bias(x["Q"], cache)
    torch.cuda.synchronize()
    oc = oracle.build_cache(np32(x["K_src"]), np32(x["V_src"]), w.bits, w.group, w.meta, key_block=T)
    scale = 1.0 / math.sqrt(w.d)
    r = w.Hq // w.Hkv
    for b in range(w.B):
        for hq in range(w.Hq):
            _, _, ks = oracle.cache_rows(oc, b, hq // r)
            want = oracle.jensen_bias_taylor(np32(x["Q"][b, hq]).astype(np.float64), ks, 1, scale)
            got = np32(bias[b, hq]).astype(np.float64)
            err = np.max(np.abs(got - want) / np.maximum(np.abs(want), 1e-30))
            assert err <= BIAS_REL_TOL, f"{name} b{b} hq{hq}: {err:.2e}"


@pytest.mark.parametrize("name,T,heads", [
    ("bf16_int2", 32, [(0, 0), (0, 13)]),
    ("prefill_gqa", 64, [(0, 0), (3, 7)]),
])
def test_full_size_sampled_rows(name, T, heads):
    """The full workload, the cache appended chunk by chunk; 64 sampled rows of a few heads."""
    w = WORKLOADS[name]
    x = make_inputs(w, device="cuda")
    cache = build_chan_cache(w, x["K_src"], x["V_src"], T, chunk=w.Lcur)
    O, LSE = api.corrected_attention(x["Q"], cache, x["K_cur"], x["V_cur"], correct=1, causal=w.causal)
    torch.cuda.synchronize()
    rows = sample_rows(w, 64).numpy()
    r = w.Hq // w.Hkv
    for b, h in heads:
        O_ref, L_ref = oracle_head(w, sub_problem(x, w, b, h), T, 1, rows=rows)
        hq = torch.as_tensor(h * r + rows // w.Lq)
        qi = torch.as_tensor(rows % w.Lq)
        compare(np32(O[b, hq, qi])[None, None].astype(np.float64), O_ref,
                np32(LSE[b, hq, qi])[None, None].astype(np.float64), L_ref, f"{name} T{T} b{b} h{h}")
    assert api.device_status() == 0
