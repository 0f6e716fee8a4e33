"""Pins of the oracle's attention-fidelity diagnostics (no GPU).

Token drift (top-1 agreement) follows pchao.org, 'QuantWM', section 实验如何设计; the KL divergence
between the reference and the quantised softmax distributions and top-5 recall follow gist.science,
'Statistical Inference and Quality Measures of KV Cache Quantisations Inspired by TurboQuant',
section Métricas de Avaliação; the cached-mass gain of quantised keys and its removal by the
correction follow agents-report.net, 'KV-Cache 量化導致的 Jensen 偏差', section 為何校正有效.
"""
import math

import numpy as np
import pytest
from scipy.stats import entropy

import oracle
from quantized_kv_cache_19_b200.workloads import WORKLOADS, make_inputs


def _problem(seed, d=16, group=8, Lq=6, Lcur=7, Lc=11, bits=2):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((Lq, d)) * 1.5
    k = rng.standard_normal((Lc, d)) * rng.uniform(0.5, 3, (1, d))
    kc = rng.standard_normal((Lcur, d))
    cache = oracle.build_cache(k[None, None].astype(np.float32), k[None, None].astype(np.float32), bits, group)
    kh, _, ks = oracle.cache_rows(cache, 0, 0)
    return q, k.astype(np.float32).astype(np.float64), kh, ks, kc


@pytest.mark.parametrize("correct", [0, 1, 2, 3])
@pytest.mark.parametrize("causal", [False, True])
def test_against_probabilities_from_one_hot_values(correct, causal):
    """With one-hot value rows the attention output IS the probability row, so the pinned attention
    oracle gives P_ref and P_q; scipy's entropy gives the KL and a plain sort the top keys."""
    q, k, kh, ks, kc = _problem(10 + correct + 5 * causal)
    Lq, d = q.shape
    Lc, Lcur = k.shape[0], kc.shape[0]
    pos = np.arange(Lq)
    scale = 1 / math.sqrt(d)
    eye = np.eye(Lc + Lcur)
    P_ref, L_ref = oracle.attention_rows(q, pos, k, eye[:Lc], ks, 8, kc, eye[Lc:], 0, causal, scale, Lq)
    P_q, L_q = oracle.attention_rows(q, pos, kh, eye[:Lc], ks, 8, kc, eye[Lc:], correct, causal, scale, Lq)
    f = oracle.fidelity_rows(q, pos, k, kh, ks, 8, kc, correct, causal, scale, Lq)
    np.testing.assert_allclose(f["lse_ref"], L_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(f["lse_q"], L_q, rtol=0, atol=1e-12)
    np.testing.assert_allclose(f["mass_ref"], P_ref[:, :Lc].sum(1), rtol=0, atol=1e-12)
    np.testing.assert_allclose(f["mass_q"], P_q[:, :Lc].sum(1), rtol=0, atol=1e-12)
    np.testing.assert_allclose(f["kl"], entropy(P_ref.T, P_q.T), rtol=1e-9, atol=1e-14)
    for i in range(Lq):
        want_r = np.argsort(-P_ref[i], kind="stable")[:5]
        want_q = np.argsort(-P_q[i], kind="stable")[:5]
        assert list(f["top_ref"][i]) == list(want_r)
        assert list(f["top_q"][i]) == list(want_q)
        assert f["top1_agree"][i] == float(want_r[0] == want_q[0])
        assert f["recall"][i] == len(set(want_r) & set(want_q)) / 5


def test_two_keys_closed_form():
    """One cached and one current key: the masses are logistic functions of the score gap and the KL
    is that of two Bernoulli distributions."""
    d, group, scale = 2, 2, 0.5
    q = np.array([[1.5, -0.5]])
    k_ref = np.array([[0.8, 0.2]])
    k_hat = np.array([[1.0, 0.0]])
    step = np.array([[0.4]])
    kc = np.array([[0.3, 0.9]])
    f = oracle.fidelity_rows(q, np.array([0]), k_ref, k_hat, step, group, kc, 1, False, scale, 1)
    s_ref = scale * (1.5 * 0.8 - 0.5 * 0.2)
    s_q = scale * 1.5 - (scale ** 2 / 24) * (1.5 ** 2 + 0.5 ** 2) * 0.4 ** 2
    s_c = scale * (1.5 * 0.3 - 0.5 * 0.9)
    p = 1 / (1 + math.exp(s_c - s_ref))
    pq = 1 / (1 + math.exp(s_c - s_q))
    assert f["mass_ref"][0] == pytest.approx(p, abs=1e-15)
    assert f["mass_q"][0] == pytest.approx(pq, abs=1e-15)
    kl = p * math.log(p / pq) + (1 - p) * math.log((1 - p) / (1 - pq))
    assert f["kl"][0] == pytest.approx(kl, rel=1e-12)
    assert f["lse_ref"][0] == pytest.approx(math.log(math.exp(s_ref) + math.exp(s_c)), abs=1e-15)
    assert list(f["top_ref"][0]) == [0, 1, -1, -1, -1]
    assert list(f["top_q"][0]) == [0, 1, -1, -1, -1]
    assert f["recall"][0] == 1.0


def test_grid_keys_uncorrected_is_exact_and_correction_moves_mass_off_the_cache():
    """Keys already on the quantisation grid are reproduced exactly by the cache: uncorrected, the two
    distributions coincide. The correction only lowers cached scores: cached mass goes down."""
    rng = np.random.default_rng(3)
    d, group, Lc = 16, 8, 9
    # dyadic steps and zero-points: (max - min) / 3 gives the step back exactly in fp32
    zp = (rng.integers(-8, 9, (Lc, d // group)) / 8).astype(np.float32)
    st = (rng.integers(1, 9, (Lc, d // group)) / 8).astype(np.float32)
    codes = rng.integers(0, 4, (Lc, d))
    codes[:, 0] = 0; codes[:, 1] = 3; codes[:, 8] = 0; codes[:, 9] = 3   # min and max in every group
    k = (np.repeat(zp, group, 1).astype(np.float64) + np.repeat(st, group, 1) * codes).astype(np.float32)
    cache = oracle.build_cache(k[None, None], k[None, None], 2, group)
    kh, _, ks = oracle.cache_rows(cache, 0, 0)
    np.testing.assert_array_equal(kh, k.astype(np.float64))
    q = rng.standard_normal((5, d)) * 2
    kc = rng.standard_normal((4, d))
    args = (q, np.arange(5), k.astype(np.float64), kh, ks, group, kc)
    f0 = oracle.fidelity_rows(*args, 0, False, 0.25, 5)
    assert np.all(f0["kl"] == 0) and np.array_equal(f0["mass_ref"], f0["mass_q"])
    assert np.all(f0["top1_agree"] == 1) and np.all(f0["recall"] == 1)
    assert np.array_equal(f0["lse_ref"], f0["lse_q"])
    for corr in (1, 2, 3):
        f = oracle.fidelity_rows(*args, corr, False, 0.25, 5)
        assert np.all(f["kl"] > 0)
        assert np.all(f["mass_q"] < f["mass_ref"])
        assert np.all(f["lse_q"] < f["lse_ref"])


def test_equal_scores_rank_lower_index_first():
    d = 8
    k = np.tile(np.arange(d, dtype=np.float64) / d, (7, 1))     # seven identical cached keys
    q = np.ones((1, d))
    f = oracle.fidelity_rows(q, np.array([0]), k, k, np.zeros((7, 1)), d, np.zeros((0, d)), 1, False,
                             0.3, 1)
    assert list(f["top_ref"][0]) == [0, 1, 2, 3, 4]
    assert list(f["top_q"][0]) == [0, 1, 2, 3, 4]
    assert f["mass_ref"][0] == pytest.approx(1.0, abs=1e-15) and f["kl"][0] == 0.0


def test_rows_without_keys_and_causal_visibility():
    """Lc = 0 and a causal current chunk shorter than the query chunk: the first rows see no key."""
    rng = np.random.default_rng(4)
    d, Lq, Lcur = 8, 5, 3
    q = rng.standard_normal((Lq, d))
    kc = rng.standard_normal((Lcur, d))
    e = np.zeros((0, d))
    f = oracle.fidelity_rows(q, np.arange(Lq), e, e, np.zeros((0, 1)), d, kc, 1, True, 0.3, Lq)
    seen = np.arange(Lq) + (Lcur - Lq) + 1      # current keys seen by each row
    for i in range(Lq):
        n = max(0, min(Lcur, seen[i]))
        if n == 0:
            assert f["lse_ref"][i] == -np.inf and f["lse_q"][i] == -np.inf
            assert f["mass_ref"][i] == 0 and f["kl"][i] == 0
            assert list(f["top_ref"][i]) == [-1] * 5 and f["top1_agree"][i] == 1 and f["recall"][i] == 1
        else:
            assert set(f["top_ref"][i][f["top_ref"][i] >= 0]) == set(range(n))
            assert f["kl"][i] == 0 and f["mass_ref"][i] == 0      # no cached keys, same current keys


def test_permuting_cached_tokens_permutes_indices_only():
    q, k, kh, ks, kc = _problem(21)
    perm = np.random.default_rng(5).permutation(k.shape[0])
    inv = np.argsort(perm)
    pos = np.arange(q.shape[0])
    f = oracle.fidelity_rows(q, pos, k, kh, ks, 8, kc, 1, True, 0.25, q.shape[0])
    g = oracle.fidelity_rows(q, pos, k[perm], kh[perm], ks[perm], 8, kc, 1, True, 0.25, q.shape[0])
    for key in ("lse_ref", "lse_q", "mass_ref", "mass_q", "kl", "top1_agree", "recall"):
        np.testing.assert_allclose(g[key], f[key], rtol=1e-12, atol=1e-14)
    Lc = k.shape[0]
    mapped = np.where((g["top_ref"] >= 0) & (g["top_ref"] < Lc), perm[np.clip(g["top_ref"], 0, Lc - 1)], g["top_ref"])
    assert np.array_equal(mapped, f["top_ref"])
    assert np.array_equal(inv[perm], np.arange(Lc))


def test_correction_restores_cached_mass_and_lowers_kl_on_tiny_workload():
    """Over 64 seeds of the tiny fp32 workload: quantised keys inflate the cached mass; the correction
    removes at least three quarters of that gain, and the mean KL to the reference drops."""
    w = WORKLOADS["tiny_f32"]
    scale = 1 / math.sqrt(w.d)
    gap_q, gap_c, kl_q, kl_c = [], [], [], []
    for seed in range(64):
        x = {k: v.numpy() for k, v in make_inputs(w, seed=5000 + seed).items()}
        cache = oracle.build_cache(x["K_src"], x["V_src"], w.bits, w.group, w.meta)
        for h in range(w.Hkv):
            kh, _, ks = oracle.cache_rows(cache, 0, h)
            args = (x["Q"][0, h], np.arange(w.Lq), x["K_src"][0, h], kh, ks, w.group, x["K_cur"][0, h])
            f0 = oracle.fidelity_rows(*args, 0, False, scale, w.Lq)
            f1 = oracle.fidelity_rows(*args, 1, False, scale, w.Lq)
            assert np.all(f0["kl"] >= 0) and np.all(f1["kl"] >= 0)
            gap_q.append(np.mean(f0["mass_q"] - f0["mass_ref"]))
            gap_c.append(np.mean(f1["mass_q"] - f1["mass_ref"]))
            kl_q.append(f0["kl"].mean()); kl_c.append(f1["kl"].mean())
    assert np.mean(gap_q) > 0
    assert abs(np.mean(gap_c)) < 0.25 * np.mean(gap_q)
    assert np.mean(kl_c) < np.mean(kl_q)
