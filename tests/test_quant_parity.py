"""GPU quantise-append against the oracle: codes bit-exact, (step, zero-point) identical."""
import numpy as np
import pytest
import torch

import oracle
from quantized_kv_cache_19_b200 import api
from quantized_kv_cache_19_b200.workloads import WORKLOADS, make_inputs

from parity_utils import build_gpu_cache, np32

pytestmark = pytest.mark.gpu


def _compare_rows(w, cache, K, V, idx_bht):
    """idx_bht: int array [n][3] of (b, h, t) token-head rows to check."""
    b, h, t = (torch.as_tensor(idx_bht[:, k]) for k in range(3))
    for which, src in (("k", K), ("v", V)):
        x = np32(src[b, h, t])                                        # [n][d]
        codes, step, zp = oracle.quantize(x, w.bits, w.group, w.meta)
        packed = oracle.pack_codes(codes, w.bits)
        got_codes = cache.codes(which)[b, h, t].cpu().numpy()
        got_meta = cache.meta_view(which)[b, h, t].cpu().numpy()       # [n][n_g][2]
        np.testing.assert_array_equal(got_codes, packed, err_msg=f"{w.name} {which} codes")
        np.testing.assert_array_equal(got_meta[..., 0], step, err_msg=f"{w.name} {which} step")
        np.testing.assert_array_equal(got_meta[..., 1], zp, err_msg=f"{w.name} {which} zero-point")


@pytest.mark.parametrize("name", ["tiny_f32", "bf16_int4", "bf16_int2"])
def test_whole_cache_bit_exact(name):
    w = WORKLOADS[name]
    x = make_inputs(w, device="cuda")
    cache = build_gpu_cache(w, x["K_src"], x["V_src"], chunk=1000)      # ragged chunks
    torch.cuda.synchronize()
    B, H, L = w.B, w.Hkv, w.Lc
    idx = np.stack(np.meshgrid(np.arange(B), np.arange(H), np.arange(L), indexing="ij"), -1).reshape(-1, 3)
    _compare_rows(w, cache, x["K_src"], x["V_src"], idx)
    assert api.device_status() == 0


@pytest.mark.parametrize("name", ["video_dit", "long_video", "prefill_gqa"])
def test_full_size_sampled_rows(name):
    """The whole cache of the workload built chunk by chunk at full size; 4096 random rows checked."""
    w = WORKLOADS[name]
    x = make_inputs(w, device="cuda")
    cache = build_gpu_cache(w, x["K_src"], x["V_src"], chunk=w.Lcur)
    torch.cuda.synchronize()
    rng = np.random.default_rng(17)
    n = 4096
    idx = np.stack([rng.integers(0, w.B, n), rng.integers(0, w.Hkv, n), rng.integers(0, w.Lc, n)], -1)
    idx[:8, 2] = [0, 1, w.Lcur - 1, w.Lcur, w.Lc - w.Lcur, w.Lc - 2, w.Lc - 1, w.Lc // 2]  # chunk edges
    _compare_rows(w, cache, x["K_src"], x["V_src"], idx)
    assert api.device_status() == 0


def test_append_writes_only_its_rows_and_advances_length():
    w = WORKLOADS["bf16_int2"].with_(Hq=2, Hkv=2, Lc=300)
    x = make_inputs(w, device="cuda")
    cache = api.KVCache(w.B, w.Hkv, w.d, w.bits, w.group, 384, w.meta)
    cache.k_codes.fill_(0xAB)
    cache.k_meta.fill_(-7.0)
    cache.length = 100
    K = x["K_src"][:, :, :37].contiguous()
    V = x["V_src"][:, :, :37].contiguous()
    api.kv_quantize_append(cache, K, V)
    assert cache.length == 137
    torch.cuda.synchronize()
    codes = cache.codes("k").cpu().numpy()
    meta = cache.meta_view("k").cpu().numpy()
    assert np.all(codes[:, :, :100] == 0xAB) and np.all(codes[:, :, 137:] == 0xAB)
    assert np.all(meta[:, :, :100] == -7.0) and np.all(meta[:, :, 137:] == -7.0)
    c_ref, s_ref, z_ref = oracle.quantize(np32(K), w.bits, w.group, w.meta)
    np.testing.assert_array_equal(codes[:, :, 100:137], oracle.pack_codes(c_ref, w.bits))
    np.testing.assert_array_equal(meta[:, :, 100:137, :, 0], s_ref)
    # overflow is rejected before anything is enqueued; L_new = 0 is a no-op
    big = x["K_src"][:, :, :248].contiguous()
    with pytest.raises(api.QkvError) as e:
        api.kv_quantize_append(cache, big, big)
    assert e.value.status == api.QKV_ERR_CAPACITY and cache.length == 137
    api.kv_quantize_append(cache, K[:, :, :0].contiguous(), V[:, :, :0].contiguous())
    assert cache.length == 137
    assert api.device_status() == 0


@pytest.mark.parametrize("bits,group,meta,dtype", [(2, 32, "f16", "f32"), (4, 128, "f16", "bf16"),
                                                   (4, 32, "f32", "f32"), (2, 128, "f32", "bf16")])
def test_other_codecs(bits, group, meta, dtype):
    w = WORKLOADS["bf16_int2"].with_(Hq=3, Hkv=3, Lc=257, bits=bits, group=group, meta=meta, dtype=dtype)
    x = make_inputs(w, device="cuda")
    cache = build_gpu_cache(w, x["K_src"], x["V_src"], chunk=100)
    torch.cuda.synchronize()
    idx = np.stack(np.meshgrid(np.arange(1), np.arange(3), np.arange(257), indexing="ij"), -1).reshape(-1, 3)
    _compare_rows(w, cache, x["K_src"], x["V_src"], idx)


@pytest.mark.parametrize("bits,meta,d,group", [(2, "f32", 128, 64), (4, "f32", 64, 32),
                                                (2, "f16", 64, 64), (4, "f16", 128, 128)])
def test_exact_ties_round_to_even(bits, meta, d, group):
    """Groups laid on a half-step grid, so that (x - min) / step is exactly k + 1/2 for about half of
    the channels; rint must pick the even code there (oracle: round half to even)."""
    levels = (1 << bits) - 1
    rows, n_g = 96, d // group
    rng = np.random.default_rng(11 + bits)
    h = rng.integers(0, 2 * levels + 1, size=(rows, n_g, group))
    h[:, :, 0], h[:, :, 1] = 0, 2 * levels                      # min and max present in every group
    for r in range(rows):                                       # shuffle each group's channels
        for g in range(n_g):
            rng.shuffle(h[r, g])
    base = rng.integers(-8, 8, size=(rows, n_g, 1)) * 0.25      # zero-point, exact in bf16
    scale = 2.0 ** rng.integers(-3, 1, size=(rows, n_g, 1))     # step: a power of two
    x = (base + scale * h / 2).reshape(1, 1, rows, d)
    K = torch.tensor(x, dtype=torch.bfloat16, device="cuda")
    assert torch.equal(K.float().cpu(), torch.tensor(x, dtype=torch.float32))   # exact in bf16
    V = (-K).contiguous()
    w = WORKLOADS["bf16_int2"].with_(Hq=1, Hkv=1, d=d, Lc=rows, bits=bits, group=group, meta=meta)
    cache = api.KVCache(1, 1, d, bits, group, 128, meta)
    api.kv_quantize_append(cache, K, V)
    torch.cuda.synchronize()
    ties = (np.asarray(h) % 2 == 1).mean()
    assert ties > 0.3
    idx = np.stack([np.zeros(rows, int), np.zeros(rows, int), np.arange(rows)], -1)
    _compare_rows(w, cache, K, V, idx)
