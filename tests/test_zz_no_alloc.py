"""The entry point for callers that cannot allocate device memory (corrected_attention_noalloc).

It takes its key-split scratch from an array the library holds itself, instead of a workspace the
caller allocates. Checked here through the C ABI against corrected_attention with a workspace, on
two calls in a row, within the tolerances of the other attention tests. Between those calls another
shape, split more ways, fills the shared array with other values, so that a split which failed to
write its part of the partials would be caught. This file is collected last on purpose."""
import numpy as np
import pytest
import torch

from quantized_kv_cache_19_b200 import api
from quantized_kv_cache_19_b200.workloads import WORKLOADS, make_inputs

from parity_utils import build_gpu_cache, compare, np32

pytestmark = pytest.mark.gpu

STATIC_SCRATCH_BYTES = 8 << 20


def _run(w, fn, x, cache, **kw):
    O, L = fn(x["Q"], cache, x["K_cur"], x["V_cur"], correct=1, causal=w.causal, **kw)
    torch.cuda.synchronize()
    return np32(O).astype(np.float64), np32(L).astype(np.float64)


def _problem(w):
    x = make_inputs(w, device="cuda")
    return x, build_gpu_cache(w, x["K_src"], x["V_src"])


@pytest.mark.parametrize("Lq", [1, 16])
def test_noalloc_matches_workspace_entry_point_on_two_calls(Lq):
    # few query rows per KV head, so that the cached keys are split and the scratch is used
    w = WORKLOADS["prefill_gqa"].with_(B=2, Hq=8, Hkv=2, Lq=Lq, Lcur=Lq, Lc=8192 + 77, seed=900 + Lq)
    x, cache = _problem(w)
    need = api.attention_workspace_bytes(cache, w.Hq, w.Lq, w.Lcur)
    assert 0 < need <= STATIC_SCRATCH_BYTES
    # another shape with more splits (one KV head, one query row: the grid is split the most ways)
    # and other values, to run between the two checked calls
    w2 = WORKLOADS["prefill_gqa"].with_(B=1, Hq=4, Hkv=1, Lq=1, Lcur=1, Lc=16384 + 5, seed=950 + Lq)
    x2, cache2 = _problem(w2)
    assert api.attention_workspace_bytes(cache2, w2.Hq, w2.Lq, w2.Lcur) > 0
    O_ref, L_ref = _run(w, api.corrected_attention, x, cache)
    O2_ref, L2_ref = _run(w2, api.corrected_attention, x2, cache2)
    for call in range(2):
        O, L = _run(w, api.corrected_attention_noalloc, x, cache)
        compare(O, O_ref, L, L_ref, f"noalloc call {call} Lq={Lq}")
        O2, L2 = _run(w2, api.corrected_attention_noalloc, x2, cache2)
        compare(O2, O2_ref, L2, L2_ref, f"noalloc other shape, call {call} Lq={Lq}")
    assert api.device_status() == 0


def test_noalloc_splits_fewer_ways_when_the_workspace_split_does_not_fit():
    # 2 KV heads, 256 query rows each (one CTA pair per KV head): the workspace split (32 ways)
    # needs 8.45 MB of partials, more than the 8 MiB array; the allocation-free call then splits
    # 31 ways, with the same results
    w = WORKLOADS["prefill_gqa"].with_(B=1, Hq=8, Hkv=2, Lq=64, Lcur=64, Lc=4096 + 40, seed=901)
    x, cache = _problem(w)
    assert api.attention_workspace_bytes(cache, w.Hq, w.Lq, w.Lcur) > STATIC_SCRATCH_BYTES
    O_ref, L_ref = _run(w, api.corrected_attention, x, cache)
    for call in range(2):
        O, L = _run(w, api.corrected_attention_noalloc, x, cache)
        compare(O, O_ref, L, L_ref, f"noalloc reduced split, call {call}")
    assert api.device_status() == 0
