"""Few query rows per KV head (decoding, small chunks): the cached keys are split over CTAs and the
partial results merged. Every row against the oracle, and the split against the unsplit kernel."""
import numpy as np
import pytest
import torch

from quantized_kv_cache_19_b200 import api
from quantized_kv_cache_19_b200.workloads import WORKLOADS, make_inputs

from parity_utils import build_gpu_cache, check_full, compare, np32

pytestmark = pytest.mark.gpu


def _decode(Lq, **kw):
    # GQA with four query heads per KV head, as in the chunked-prefill shape; a ragged cache length.
    return WORKLOADS["prefill_gqa"].with_(B=2, Hq=8, Hkv=2, Lq=Lq, Lcur=Lq, Lc=8192 + 77, seed=400 + Lq, **kw)


@pytest.mark.parametrize("Lq", [1, 4, 16])
@pytest.mark.parametrize("correct", [0, 1, 2])
def test_split_keys_every_row(Lq, correct):
    w = _decode(Lq)
    cache = api.KVCache(w.B, w.Hkv, w.d, w.bits, w.group, api.round_capacity(w.Lc), w.meta)
    cache.length = w.Lc
    assert api.attention_workspace_bytes(cache, w.Hq, w.Lq, w.Lcur) > 0   # this shape is split
    check_full(w, correct)


@pytest.mark.parametrize("Lq,causal", [(1, True), (16, True), (16, False)])
def test_split_matches_unsplit(Lq, causal):
    w = _decode(Lq, causal=causal)
    x = make_inputs(w, device="cuda")
    cache = build_gpu_cache(w, x["K_src"], x["V_src"])
    O1, L1 = api.corrected_attention(x["Q"], cache, x["K_cur"], x["V_cur"], correct=1, causal=causal)
    O2, L2 = api.corrected_attention(x["Q"], cache, x["K_cur"], x["V_cur"], correct=1, causal=causal,
                                     workspace=None)
    torch.cuda.synchronize()
    # two evaluations of the same sums in different orders: agreement well inside the oracle bar
    compare(np32(O1).astype(np.float64), np32(O2).astype(np.float64), np32(L1).astype(np.float64),
            np32(L2).astype(np.float64), f"split vs unsplit Lq={Lq}")
    assert api.device_status() == 0


def test_split_with_one_key_tile_per_split_and_empty_current():
    # a cache of a few tiles (every split gets one) and no current chunk
    w = _decode(4).with_(Lc=3 * 128 + 5, Lcur=0)
    check_full(w, 1)


def test_workspace_too_small_falls_back_to_unsplit():
    w = _decode(4)
    x = make_inputs(w, device="cuda")
    cache = build_gpu_cache(w, x["K_src"], x["V_src"])
    need = api.attention_workspace_bytes(cache, w.Hq, w.Lq, w.Lcur)
    small = torch.empty(need // 2, dtype=torch.uint8, device="cuda")
    O1, L1 = api.corrected_attention(x["Q"], cache, x["K_cur"], x["V_cur"], correct=1, causal=True,
                                     workspace=small)
    O2, L2 = api.corrected_attention(x["Q"], cache, x["K_cur"], x["V_cur"], correct=1, causal=True,
                                     workspace=None)
    torch.cuda.synchronize()
    assert torch.equal(O1, O2) and torch.equal(L1, L2)   # both took the unsplit kernel


@pytest.mark.parametrize("Lq", [1, 16])
def test_full_size_decode_cache(Lq):
    """The chunked-prefill workload's whole 131072-token cache with a decode-sized query chunk; every
    row of two (batch, KV head) pairs against the oracle."""
    from parity_utils import oracle_head, sub_problem
    w = WORKLOADS["prefill_gqa"].with_(Lq=Lq, Lcur=Lq)
    x = make_inputs(w, device="cuda")
    cache = build_gpu_cache(w, x["K_src"], x["V_src"], chunk=8192)
    assert api.attention_workspace_bytes(cache, w.Hq, w.Lq, w.Lcur) > 0
    O, LSE = api.corrected_attention(x["Q"], cache, x["K_cur"], x["V_cur"], correct=1, causal=True)
    torch.cuda.synchronize()
    r = w.Hq // w.Hkv
    for b, h in [(0, 0), (3, 7)]:
        O_ref, L_ref = oracle_head(w, sub_problem(x, w, b, h), 1)
        compare(np32(O[b:b + 1, h * r:(h + 1) * r]).astype(np.float64), O_ref,
                np32(LSE[b:b + 1, h * r:(h + 1) * r]).astype(np.float64), L_ref, f"decode Lq={Lq} b{b} h{h}")
    assert api.device_status() == 0
