"""The Python binding's own checks, which fail before any device work (no GPU needed): layouts the
library does not serve, CPU tensors (there is no CPU path), and shape or dtype mismatches."""
import pytest
import torch

from quantized_kv_cache_19_b200 import api


def test_round_capacity_is_a_multiple_of_the_cache_tile():
    assert api.round_capacity(0) == api.CACHE_TILE
    assert api.round_capacity(1) == api.CACHE_TILE
    assert api.round_capacity(128) == 128
    assert api.round_capacity(129) == 256
    assert api.round_capacity(4680) % api.CACHE_TILE == 0 and api.round_capacity(4680) >= 4680


@pytest.mark.parametrize("kw,status", [
    (dict(key_block=16), api.QKV_ERR_UNSUPPORTED),     # key blocks of 32, 64 or 128 positions
    (dict(bits=3), api.QKV_ERR_UNSUPPORTED),
    (dict(group=48), api.QKV_ERR_UNSUPPORTED),
    (dict(capacity=100), api.QKV_ERR_INVALID_ARG),     # not a multiple of the cache tile
])
def test_cache_layouts_the_library_does_not_serve_are_refused_before_allocation(kw, status):
    args = dict(B=1, H_kv=2, d=128, bits=2, group=64, capacity=256, meta="f32", device="cpu")
    args.update(kw)
    with pytest.raises(api.QkvError) as err:
        api.KVCache(**args)
    assert err.value.status == status


def test_cpu_tensors_are_refused():
    q = torch.zeros(1, 2, 4, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        api.corrected_attention(q, None, q, q)
    with pytest.raises(ValueError, match="CUDA"):
        api.attention_fidelity(q, None, q, q)
    with pytest.raises(ValueError, match="CUDA"):
        api.jensen_bias(q, None)


def test_packed_bytes_follow_the_layout():
    """Bytes of codes and (step, zero-point) per token for both key layouts, from the layout sizes
    the library reports (the buffers live on the CPU here; nothing is launched)."""
    c = api.KVCache(1, 2, 128, 2, 64, 256, "f32", device="cpu")
    assert c.packed_bytes(100) == 2 * 2 * 100 * (32 + 2 * 2 * 4)
    k = api.KVCache(1, 2, 128, 2, 64, 256, "f16", device="cpu", key_block=32)
    # keys: 32 B of codes per token + one (step, zero-point) pair per channel per started block
    assert k.packed_bytes(100) == 2 * (100 * (2 * 32 + 2 * 2 * 2) + 4 * 128 * 2 * 2)
    assert k.meta_view("k").shape == (1, 2, 256 // 32, 128, 2)
    assert k.meta_view("v").shape == (1, 2, 256, 2, 2)
