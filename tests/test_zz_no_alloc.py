"""The entry point for callers that cannot allocate device memory (corrected_attention_noalloc).

It takes its key-split scratch from an array the library holds itself, instead of a workspace the
caller allocates. Checked here through the C ABI against corrected_attention with a workspace, on
two calls in a row (the second call finds the first call's values in the shared array), within the
tolerances of the other attention tests. This file is collected last on purpose."""
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


@pytest.mark.parametrize("Lq", [1, 16])
def test_noalloc_matches_workspace_entry_point_on_two_calls(Lq):
    # few query rows per KV head, so that the cached keys are split and the scratch is used
    w = WORKLOADS["prefill_gqa"].with_(B=2, Hq=8, Hkv=2, Lq=Lq, Lcur=Lq, Lc=8192 + 77, seed=900 + Lq)
    x = make_inputs(w, device="cuda")
    cache = build_gpu_cache(w, x["K_src"], x["V_src"])
    need = api.attention_workspace_bytes(cache, w.Hq, w.Lq, w.Lcur)
    assert 0 < need <= STATIC_SCRATCH_BYTES
    O_ref, L_ref = _run(w, api.corrected_attention, x, cache)
    for call in range(2):
        O, L = _run(w, api.corrected_attention_noalloc, x, cache)
        compare(O, O_ref, L, L_ref, f"noalloc call {call} Lq={Lq}")
    assert api.device_status() == 0


def test_noalloc_rejects_a_split_larger_than_its_scratch():
    # 4 x 8 KV heads, 128 query rows each: split 4 ways, 8.45 MB of partials > 8 MiB
    w = WORKLOADS["prefill_gqa"].with_(Lq=32, Lcur=32, Lc=512, seed=901)
    x = make_inputs(w, device="cuda")
    cache = build_gpu_cache(w, x["K_src"], x["V_src"])
    assert api.attention_workspace_bytes(cache, w.Hq, w.Lq, w.Lcur) > STATIC_SCRATCH_BYTES
    with pytest.raises(api.QkvError) as err:
        api.corrected_attention_noalloc(x["Q"], cache, x["K_cur"], x["V_cur"], correct=1, causal=True)
    assert err.value.status == api.QKV_ERR_UNSUPPORTED and "static scratch" in str(err.value)
