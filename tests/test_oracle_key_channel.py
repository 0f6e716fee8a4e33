"""Pins of the oracle's per-channel key quantisation along tokens (KIVI's key grouping, named in
agents-report.net, 'KV-Cache 量化導致的 Jensen 偏差', section 跨主題對比分析; grouping along the sequence
axis in the hotelren.com blog, section 3.1) and of corrected attention over such a cache (no GPU).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from quantized_kv_cache_19_b200.workloads import WORKLOADS, make_inputs


def _x(seed, shape, scale_chan=True):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal(shape)
    if scale_chan:
        x = x * rng.uniform(0.5, 3, shape[:-2] + (1, shape[-1]))
    return x.astype(np.float32)


@pytest.mark.parametrize("bits", [2, 4])
@pytest.mark.parametrize("meta", ["f32", "f16"])
@pytest.mark.parametrize("T", [4, 32])
def test_equals_the_per_token_quantiser_on_the_transposed_block(bits, meta, T):
    """Along tokens per channel is the (pinned) per-token quantiser applied to the transpose, with
    group = T, whenever the length is a whole number of blocks."""
    x = _x(1, (2, 3, 4 * T, 16))
    c, s, z = oracle.quantize_tokens(x, bits, T, meta)
    ct, st, zt = oracle.quantize(np.swapaxes(x, -1, -2), bits, T, meta)
    np.testing.assert_array_equal(c, np.swapaxes(ct, -1, -2))
    np.testing.assert_array_equal(s, np.swapaxes(st, -1, -2))
    np.testing.assert_array_equal(z, np.swapaxes(zt, -1, -2))


def test_partial_last_block_uses_only_its_own_tokens():
    x = _x(2, (1, 2, 3 * 32 + 7, 8))
    c, s, z = oracle.quantize_tokens(x, 2, 32, "f32")
    assert s.shape == (1, 2, 4, 8)
    c_head, s_head, z_head = oracle.quantize_tokens(x[..., :96, :], 2, 32, "f32")
    c_tail, s_tail, z_tail = oracle.quantize_tokens(x[..., 96:, :], 2, 32, "f32")
    np.testing.assert_array_equal(c[..., :96, :], c_head)
    np.testing.assert_array_equal(c[..., 96:, :], c_tail)
    np.testing.assert_array_equal(s[..., :3, :], s_head)
    np.testing.assert_array_equal(s[..., 3:, :], s_tail)
    np.testing.assert_array_equal(z[..., 3:, :], z_tail)


@pytest.mark.parametrize("bits", [2, 4])
def test_block_extremes_and_error_bound(bits):
    T = 16
    x = _x(3, (1, 1, 5 * T, 12))
    c, s, z = oracle.quantize_tokens(x, bits, T, "f32")
    for k in range(5):
        xb = x[0, 0, k * T:(k + 1) * T]
        cb = c[0, 0, k * T:(k + 1) * T]
        for ch in range(12):
            assert cb[np.argmin(xb[:, ch]), ch] == 0
            assert cb[np.argmax(xb[:, ch]), ch] == (1 << bits) - 1
        xh = z[0, 0, k].astype(np.float64) + s[0, 0, k].astype(np.float64) * cb
        assert np.all(np.abs(xh - xb) <= s[0, 0, k] / 2 * (1 + 1e-6))


def test_cache_rows_expand_each_block_over_its_tokens():
    x = _x(4, (1, 1, 70, 8))
    cache = oracle.build_cache(x, x, 2, 8, "f32", key_block=32)
    kh, _, ks = oracle.cache_rows(cache, 0, 0)
    assert ks.shape == (70, 8) and oracle.key_step_group(cache, 8) == 1
    for j in (0, 31, 32, 63, 64, 69):
        k = j // 32
        np.testing.assert_array_equal(ks[j], cache["k_step"][0, 0, k].astype(np.float64))
        want = cache["k_zp"][0, 0, k].astype(np.float64) + cache["k_step"][0, 0, k].astype(np.float64) * cache["k_codes"][0, 0, j]
        np.testing.assert_allclose(kh[j], want, rtol=0, atol=0)


def test_one_token_blocks_are_exact_and_need_no_correction():
    """T = 1: every block is one token, every step is 0, the cache reproduces the keys exactly and the
    corrected attention is plain attention over them (torch SDPA in fp64 as a second opinion)."""
    rng = np.random.default_rng(5)
    d, Lq, Lc, Lcur = 16, 6, 9, 5
    Q = rng.standard_normal((1, 2, Lq, d))
    K = rng.standard_normal((1, 1, Lc, d)).astype(np.float32)
    V = rng.standard_normal((1, 1, Lc, d)).astype(np.float32)
    Kc = rng.standard_normal((1, 1, Lcur, d))
    Vc = rng.standard_normal((1, 1, Lcur, d))
    cache = oracle.build_cache(K, V, 2, 8, "f32", key_block=1)
    assert np.all(cache["k_step"] == 0)
    O, L = oracle.corrected_attention(Q, cache, Kc, Vc, correct=1, causal=False)
    kh, vh, _ = oracle.cache_rows(cache, 0, 0)
    np.testing.assert_array_equal(kh, K[0, 0].astype(np.float64))
    k = torch.from_numpy(np.concatenate([kh, Kc[0, 0]]))
    v = torch.from_numpy(np.concatenate([vh, Vc[0, 0]]))
    for hq in range(2):
        want = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(Q[0, hq])[None], k[None], v[None])[0].numpy()
        np.testing.assert_allclose(O[0, hq], want, rtol=1e-12, atol=1e-12)


def test_per_channel_exact_correction_unbiased_by_monte_carlo():
    """The correction with each key's own per-channel steps (group 1) makes the expected softmax
    denominator over uniformly perturbed keys equal the unperturbed one."""
    rng = np.random.default_rng(6)
    d, Lc, n = 16, 5, 200_000
    scale = 1 / math.sqrt(d)
    q = rng.standard_normal(d) * 1.5
    k = rng.standard_normal((Lc, d))
    step = rng.uniform(0.2, 2.0, (Lc, d))               # a different step per key and channel
    s = scale * k @ q
    b = oracle.jensen_bias_exact(q[None], step, 1, scale)[0]
    e = (rng.random((n, Lc, d)) - 0.5) * step[None]
    corrected = np.exp(s + scale * e @ q - b).sum(1)
    se = corrected.std() / math.sqrt(n)
    assert abs(corrected.mean() - np.exp(s).sum()) < 4 * se
    bt = oracle.jensen_bias_taylor(q[None], step, 1, scale)[0]
    a = 0.5 * scale * q[None, :] * step
    assert np.all(bt >= b) and np.all(bt - b <= (a ** 4 / 180).sum(1) * (1 + 1e-9))


def test_attention_over_a_per_channel_cache_matches_sdpa_with_the_bias_as_a_mask():
    """Corrected attention = SDPA in fp64 over the dequantised keys with -b as an additive mask, b
    from each key's block steps per channel."""
    rng = np.random.default_rng(7)
    d, Lq, Lc, Lcur, T = 16, 5, 40, 6, 8
    Q = rng.standard_normal((1, 2, Lq, d))
    K = _x(8, (1, 1, Lc, d))
    V = _x(9, (1, 1, Lc, d), False)
    Kc = rng.standard_normal((1, 1, Lcur, d))
    Vc = rng.standard_normal((1, 1, Lcur, d))
    cache = oracle.build_cache(K, V, 2, 8, "f32", key_block=T)
    scale = 1 / math.sqrt(d)
    O, L = oracle.corrected_attention(Q, cache, Kc, Vc, correct=1, causal=True)
    kh, vh, _ = oracle.cache_rows(cache, 0, 0)
    kst = cache["k_step"][0, 0].astype(np.float64)
    k = torch.from_numpy(np.concatenate([kh, Kc[0, 0]]))
    v = torch.from_numpy(np.concatenate([vh, Vc[0, 0]]))
    for hq in range(2):
        q = Q[0, hq]
        mask = np.zeros((Lq, Lc + Lcur))
        for i in range(Lq):
            for j in range(Lc):
                mask[i, j] = -(scale ** 2 / 24) * sum(q[i, c] ** 2 * kst[j // T, c] ** 2 for c in range(d))
            for t in range(Lcur):
                if t > i + (Lcur - Lq):
                    mask[i, Lc + t] = -np.inf
        want = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q)[None], k[None], v[None], attn_mask=torch.from_numpy(mask)[None])[0].numpy()
        np.testing.assert_allclose(O[0, hq], want, rtol=1e-11, atol=1e-12)


def test_correction_restores_cached_mass_with_per_channel_keys():
    """Over 64 seeds of the tiny workload with 32-token key blocks at INT2: quantised keys inflate
    the cached mass and the correction removes at least three quarters of the gain."""
    w = WORKLOADS["tiny_f32"]
    scale = 1 / math.sqrt(w.d)
    gq, gc = [], []
    for seed in range(64):
        x = {k: v.numpy() for k, v in make_inputs(w, seed=5000 + seed).items()}
        cache = oracle.build_cache(x["K_src"], x["V_src"], 2, w.group, w.meta, key_block=32)
        for h in range(w.Hkv):
            kh, _, ks = oracle.cache_rows(cache, 0, h)
            args = (x["Q"][0, h], np.arange(w.Lq), x["K_src"][0, h], kh, ks, 1, x["K_cur"][0, h])
            f0 = oracle.fidelity_rows(*args, 0, False, scale, w.Lq)
            f1 = oracle.fidelity_rows(*args, 1, False, scale, w.Lq)
            gq.append(np.mean(f0["mass_q"] - f0["mass_ref"]))
            gc.append(np.mean(f1["mass_q"] - f1["mass_ref"]))
    assert np.mean(gq) > 0
    assert abs(np.mean(gc)) < 0.25 * np.mean(gq)
