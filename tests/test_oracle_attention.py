"""Pins of the oracle's corrected attention (no GPU).

Scores are q.k/sqrt(d) (pchao.org, 'QuantWM', eq. (5)); the Jensen correction is subtracted from the
scores of cached (quantised) keys only, then one softmax runs over cached and current keys
(agents-report.net, 'KV-Cache 量化導致的 Jensen 偏差', sections 方法 and 為何校正有效).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from quantized_kv_cache_19_b200.workloads import WORKLOADS, make_inputs


def _rand_problem(seed, B=1, Hq=2, Hkv=1, d=16, Lq=5, Lcur=6, Lc=9, bits=2, group=8, meta="f32"):
    rng = np.random.default_rng(seed)
    Q = rng.standard_normal((B, Hq, Lq, d)).astype(np.float32)
    K = (rng.standard_normal((B, Hkv, Lc, d)) * rng.uniform(0.5, 3, (1, Hkv, 1, d))).astype(np.float32)
    V = rng.standard_normal((B, Hkv, Lc, d)).astype(np.float32)
    Kc = rng.standard_normal((B, Hkv, Lcur, d)).astype(np.float32)
    Vc = rng.standard_normal((B, Hkv, Lcur, d)).astype(np.float32)
    cache = oracle.build_cache(K, V, bits, group, meta)
    return Q, K, V, Kc, Vc, cache


def _sdpa_reference(Q, cache, Kc, Vc, causal, scale, bias_fn=None):
    """torch float64 scaled_dot_product_attention over [dequantised cache ; current]."""
    B, Hq, Lq, d = Q.shape
    Hkv = Kc.shape[1]; r = Hq // Hkv
    O = np.zeros(Q.shape)
    for b in range(B):
        for hq in range(Hq):
            h = hq // r
            kh, vh, ks = oracle.cache_rows(cache, b, h)
            k = torch.from_numpy(np.concatenate([kh, Kc[b, h].astype(np.float64)]))
            v = torch.from_numpy(np.concatenate([vh, Vc[b, h].astype(np.float64)]))
            q = torch.from_numpy(Q[b, hq].astype(np.float64))
            Lc, Lcur = kh.shape[0], Kc.shape[2]
            mask = torch.zeros(Lq, Lc + Lcur, dtype=torch.float64)
            if bias_fn is not None:
                mask[:, :Lc] -= torch.from_numpy(bias_fn(Q[b, hq], ks))
            if causal:
                i = torch.arange(Lq)[:, None]; j = torch.arange(Lcur)[None, :]
                mask[:, Lc:] = mask[:, Lc:].masked_fill(j > i + (Lcur - Lq), float("-inf"))
            o = torch.nn.functional.scaled_dot_product_attention(
                q[None, None], k[None, None], v[None, None], attn_mask=mask[None, None], scale=scale)
            O[b, hq] = o[0, 0].numpy()
    return O


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("correct", [0, 1])
def test_matches_torch_sdpa(causal, correct):
    Q, K, V, Kc, Vc, cache = _rand_problem(1, B=2, Hq=4, Hkv=2, Lq=7, Lcur=7, Lc=11)
    scale = 1 / math.sqrt(16)
    O, LSE = oracle.corrected_attention(Q, cache, Kc, Vc, correct=correct, causal=causal)
    bias_fn = (lambda q, ks: oracle.jensen_bias_taylor(q, ks, 8, scale)) if correct else None
    O_ref = _sdpa_reference(Q, cache, Kc, Vc, causal, scale, bias_fn)
    np.testing.assert_allclose(O, O_ref, rtol=1e-12, atol=1e-12)
    # LSE against torch.logsumexp of the score matrix
    for b in range(2):
        for hq in range(4):
            kh, _, ks = oracle.cache_rows(cache, b, hq // 2)
            q = torch.from_numpy(Q[b, hq].astype(np.float64))
            s_c = scale * q @ torch.from_numpy(kh).T
            if correct:
                s_c = s_c - torch.from_numpy(oracle.jensen_bias_taylor(Q[b, hq], ks, 8, scale))
            s_n = scale * q @ torch.from_numpy(Kc[b, hq // 2].astype(np.float64)).T
            if causal:
                i = torch.arange(7)[:, None]; j = torch.arange(7)[None, :]
                s_n = s_n.masked_fill(j > i, float("-inf"))
            lse = torch.logsumexp(torch.cat([s_c, s_n], 1), 1).numpy()
            np.testing.assert_allclose(LSE[b, hq], lse, rtol=1e-13, atol=1e-13)


def test_brute_force_loops_tiny():
    """Pure-Python loops with math.exp on a tiny case, causal with Lq < Lcur, GQA r = 2."""
    Q, K, V, Kc, Vc, cache = _rand_problem(3, B=1, Hq=2, Hkv=1, d=4, Lq=2, Lcur=3, Lc=3, group=2)
    scale = 0.5
    O, LSE = oracle.corrected_attention(Q, cache, Kc, Vc, correct=1, causal=True, scale=scale)
    kh, vh, ks = oracle.cache_rows(cache, 0, 0)
    for hq in range(2):
        for i in range(2):
            q = [float(t) for t in Q[0, hq, i]]
            scores, vals = [], []
            for j in range(3):
                s = scale * sum(q[c] * kh[j, c] for c in range(4))
                b = scale * scale / 24 * sum(q[c] ** 2 * ks[j, c // 2] ** 2 for c in range(4))
                scores.append(s - b); vals.append(vh[j])
            for j in range(3):
                if j <= i + (3 - 2):
                    scores.append(scale * sum(q[c] * float(Kc[0, 0, j, c]) for c in range(4)))
                    vals.append(Vc[0, 0, j].astype(np.float64))
            m = max(scores)
            e = [math.exp(s - m) for s in scores]
            l = sum(e)
            o = [sum(e[k] * vals[k][c] for k in range(len(e))) / l for c in range(4)]
            assert np.allclose(O[0, hq, i], o, rtol=1e-13, atol=1e-13)
            assert LSE[0, hq, i] == pytest.approx(m + math.log(l), rel=1e-13)


def test_empty_cache_is_plain_attention():
    Q, K, V, Kc, Vc, cache = _rand_problem(4)
    O, LSE = oracle.corrected_attention(Q, None, Kc, Vc, correct=1)
    q = torch.from_numpy(Q.astype(np.float64))
    k = torch.from_numpy(Kc.astype(np.float64)).repeat_interleave(2, 1)
    v = torch.from_numpy(Vc.astype(np.float64)).repeat_interleave(2, 1)
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v).numpy()
    np.testing.assert_allclose(O, ref, rtol=1e-12, atol=1e-12)


def test_zero_step_makes_correction_vanish():
    Q, K, V, Kc, Vc, _ = _rand_problem(5)
    Kconst = np.repeat(K[:, :, :, :1], K.shape[-1], axis=-1)    # every group constant -> step 0
    cache = oracle.build_cache(Kconst, V, 2, 8, "f32")
    assert np.all(cache["k_step"] == 0)
    O1, L1 = oracle.corrected_attention(Q, cache, Kc, Vc, correct=1)
    O0, L0 = oracle.corrected_attention(Q, cache, Kc, Vc, correct=0)
    np.testing.assert_array_equal(O1, O0)
    np.testing.assert_array_equal(L1, L0)


def test_rows_sum_to_one_and_permutation_invariance():
    Q, K, V, Kc, Vc, cache = _rand_problem(6, Lc=13)
    ones = dict(cache)
    ones["v_codes"] = np.zeros_like(cache["v_codes"])
    ones["v_step"] = np.zeros_like(cache["v_step"])
    ones["v_zp"] = np.ones_like(cache["v_zp"])
    O, _ = oracle.corrected_attention(Q, ones, Kc, np.ones_like(Vc), correct=1, causal=True)
    np.testing.assert_allclose(O, 1.0, rtol=0, atol=1e-14)
    perm = np.random.default_rng(0).permutation(13)
    pc = {k: (v[:, :, perm] if isinstance(v, np.ndarray) else v) for k, v in cache.items()}
    Oa, La = oracle.corrected_attention(Q, cache, Kc, Vc, correct=1)
    Ob, Lb = oracle.corrected_attention(Q, pc, Kc, Vc, correct=1)
    np.testing.assert_allclose(Oa, Ob, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(La, Lb, rtol=1e-13, atol=1e-13)


def test_split_merge_equals_unsplit():
    Q, K, V, Kc, Vc, cache = _rand_problem(7, Lc=20)
    kh, vh, ks = oracle.cache_rows(cache, 0, 0)
    q = Q[0, 1].astype(np.float64); pos = np.arange(5); s = 0.25
    full = oracle.attention_rows(q, pos, kh, vh, ks, 8, Kc[0, 0], Vc[0, 0], 1, True, s, 5)
    e = np.zeros((0, 16))
    p1 = oracle.attention_rows(q, pos, kh[:8], vh[:8], ks[:8], 8, e, e, 1, True, s, 5)
    p2 = oracle.attention_rows(q, pos, kh[8:], vh[8:], ks[8:], 8, e, e, 1, True, s, 5)
    p3 = oracle.attention_rows(q, pos, kh[:0], vh[:0], ks[:0], 8, Kc[0, 0], Vc[0, 0], 1, True, s, 5)
    o, lse = oracle.merge_partials([p1, p2, p3])
    np.testing.assert_allclose(o, full[0], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, full[1], rtol=1e-13)


def test_gqa_head_mapping():
    Q, K, V, Kc, Vc, cache = _rand_problem(8, B=1, Hq=4, Hkv=2)
    O, L = oracle.corrected_attention(Q, cache, Kc, Vc, correct=1, causal=True)
    rep = {k: (np.repeat(v, 2, axis=1) if isinstance(v, np.ndarray) else v) for k, v in cache.items()}
    O2, L2 = oracle.corrected_attention(Q, rep, np.repeat(Kc, 2, 1), np.repeat(Vc, 2, 1), correct=1, causal=True)
    np.testing.assert_array_equal(O, O2)
    np.testing.assert_array_equal(L, L2)


def test_row_sample_matches_full():
    Q, K, V, Kc, Vc, cache = _rand_problem(9, B=2, Hq=4, Hkv=2, Lq=6, Lcur=6)
    O, L = oracle.corrected_attention(Q, cache, Kc, Vc, correct=1, causal=True)
    rows = np.array([0, 3, 5, 6, 11])            # packed row = (hq % r) * Lq + i
    Os, Ls = oracle.corrected_attention(Q, cache, Kc, Vc, correct=1, causal=True, rows=rows)
    for b in range(2):
        for h in range(2):
            for k, R in enumerate(rows):
                hq, i = h * 2 + R // 6, R % 6
                np.testing.assert_allclose(Os[b, h, k], O[b, hq, i], rtol=1e-13, atol=1e-14)
                assert Ls[b, h, k] == pytest.approx(L[b, hq, i], rel=1e-14)


def test_correction_removes_expected_inflation_under_uniform_noise():
    """With exact b and noise e ~ U(+-Delta/2): E_e[sum_j exp(s_j + delta_j - b_j)] = sum_j exp(s_j)."""
    rng = np.random.default_rng(12)
    d, group, Lc, n = 32, 16, 6, 100_000
    scale = 1 / math.sqrt(d)
    q = rng.standard_normal(d) * 1.5
    k = rng.standard_normal((Lc, d))
    step = rng.uniform(0.5, 2.0, (Lc, 2))
    s = scale * k @ q
    b = oracle.jensen_bias_exact(q[None], step, group, scale)[0]
    e = (rng.random((n, Lc, d)) - 0.5) * np.repeat(step, group, axis=-1)[None]
    delta = scale * e @ q
    corrected = np.exp(s + delta - b).sum(1)
    raw = np.exp(s + delta).sum(1)
    se = corrected.std() / math.sqrt(n)
    assert abs(corrected.mean() - np.exp(s).sum()) < 4 * se
    assert raw.mean() - np.exp(s).sum() > 20 * se     # uncorrected mass is inflated


def test_mass_restoration_on_tiny_workload():
    """The point of the method: quantised cached keys gain softmax mass; the correction gives it back.
    Cached mass per row = exp(LSE over cache - LSE over cache and current), averaged over 64 seeds."""
    w = WORKLOADS["tiny_f32"]
    gaps_q, gaps_c = [], []
    for seed in range(64):
        x = {k: v.numpy() for k, v in make_inputs(w, seed=5000 + seed).items()}
        cache = oracle.build_cache(x["K_src"], x["V_src"], w.bits, w.group, w.meta)
        scale = 1 / math.sqrt(w.d)
        for h in range(w.Hkv):
            kh, vh, ks = oracle.cache_rows(cache, 0, h)
            q = x["Q"][0, h].astype(np.float64); pos = np.arange(w.Lq)
            e = np.zeros((0, w.d))
            kf = x["K_src"][0, h].astype(np.float64); vf = x["V_src"][0, h].astype(np.float64)
            kc, vc = x["K_cur"][0, h], x["V_cur"][0, h]

            def mass(kk, vv, corr):
                lc = oracle.attention_rows(q, pos, kk, vv, ks, w.group, e, e, corr, False, scale, w.Lq)[1]
                la = oracle.attention_rows(q, pos, kk, vv, ks, w.group, kc, vc, corr, False, scale, w.Lq)[1]
                return np.exp(lc - la)

            m_ref = mass(kf, vf, 0)
            gaps_q.append(mass(kh, vh, 0) - m_ref)
            gaps_c.append(mass(kh, vh, 1) - m_ref)
    gq = np.mean(gaps_q); gc = np.mean(gaps_c)
    assert gq > 0
    assert abs(gc) < 0.25 * gq
