"""The attention kernels' bounded waits: with the bound lowered to one cycle every wait that does
not succeed at once gives up, the kernel drains its own copies and tensor-core operations, frees
its tensor memory and returns; the device status word then reads QKV_ERR_TIMEOUT, the context
stays usable, and the next call with the default bound passes parity on the same device.

No GPU fault is involved: the waits are made to run out by their bound, not by a fault."""
import pytest
import torch

from quantized_kv_cache_19_b200 import api
from quantized_kv_cache_19_b200.workloads import WORKLOADS, make_inputs

from parity_utils import build_gpu_cache, check_full

pytestmark = pytest.mark.gpu

CASES = {
    # several key tiles per CTA, cached and current
    "prefill_tiles": dict(Hq=4, Hkv=2, Lq=256, Lcur=256, Lc=1024 + 40, causal=True),
    # few query rows per KV head: the cached keys are split over CTAs and merged afterwards
    "split_keys": dict(Hq=8, Hkv=2, Lq=1, Lcur=1, Lc=4096 + 3),
}


@pytest.mark.parametrize("case", sorted(CASES))
def test_wait_bound_runs_out_then_next_call_passes(case):
    w = WORKLOADS["bf16_int2"].with_(seed=313, **CASES[case])
    assert api.device_status(reset=True) == 0
    prev = api.set_wait_limit(1)
    try:
        x = make_inputs(w, device="cuda")
        cache = build_gpu_cache(w, x["K_src"], x["V_src"])
        api.corrected_attention(x["Q"], cache, x["K_cur"], x["V_cur"], correct=1, causal=w.causal)
        torch.cuda.synchronize()
    finally:
        api.set_wait_limit(prev)
    assert api.device_status(reset=True) == api.QKV_ERR_TIMEOUT
    assert api.device_status(reset=True) == 0
    # same device, default bound: every row against the oracle
    check_full(w, correct=1)


@pytest.mark.parametrize("Lq", [45, 1])
def test_wait_bound_runs_out_per_channel_keys(Lq):
    """The same for the tensor-core kernel of caches with per-channel key blocks (unsplit, and with
    its cached keys split over CTAs for a one-row chunk)."""
    from test_key_channel_parity import SMALL, build_chan_cache, check_every_row
    w = SMALL["prefill_gqa"].with_(seed=317, Lq=Lq, Lcur=Lq, Lc=32 * 40 + 9 if Lq == 1 else 333)
    assert api.device_status(reset=True) == 0
    prev = api.set_wait_limit(1)
    try:
        x = make_inputs(w, device="cuda")
        cache = build_chan_cache(w, x["K_src"], x["V_src"], 32)
        api.corrected_attention(x["Q"], cache, x["K_cur"], x["V_cur"], correct=1, causal=w.causal,
                                workspace="auto")
        torch.cuda.synchronize()
    finally:
        api.set_wait_limit(prev)
    assert api.device_status(reset=True) == api.QKV_ERR_TIMEOUT
    assert api.device_status(reset=True) == 0
    check_every_row(w, 32, 1)
