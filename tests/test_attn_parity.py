"""GPU corrected attention against the oracle: O max relative error <= 1e-2 per head, LSE absolute
error <= 2e-3, the correction term relative error <= 1e-5."""
import math

import numpy as np
import pytest
import torch

import oracle
from quantized_kv_cache_19_b200 import api
from quantized_kv_cache_19_b200.workloads import WORKLOADS, make_inputs

from parity_utils import (BIAS_REL_TOL, build_gpu_cache, check_full, check_sampled, compare, np32,
                          oracle_head, sub_problem)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("correct", [0, 1, 2])
@pytest.mark.parametrize("name", ["tiny_f32", "bf16_int4", "bf16_int2"])
def test_small_workloads_every_row(name, correct):
    check_full(WORKLOADS[name], correct)


@pytest.mark.parametrize("correct", [0, 1, 2])
@pytest.mark.parametrize("name,heads", [
    ("video_dit", [(0, 0), (0, 11), (0, 23)]),
    ("long_video", [(0, 0), (0, 39)]),
    ("prefill_gqa", [(0, 0), (3, 7), (2, 4)]),
])
def test_full_size_sampled_rows(name, heads, correct):
    check_sampled(WORKLOADS[name], correct, heads)


EDGE = {
    # name: overrides of the small bf16 INT2 workload
    "empty_cache": dict(Lc=0),
    "empty_current": dict(Lcur=0, Lq=96),
    "ragged_all": dict(Lc=300, Lq=77, Lcur=45),
    "one_query": dict(Lq=1, Lcur=1, Lc=129),
    "gqa_rows_cross_heads": dict(Hq=8, Hkv=2, Lq=100, Lcur=100, Lc=260, causal=True),
    "causal_short_queries": dict(Lq=40, Lcur=200, Lc=128, causal=True),
    "causal_long_queries_no_cache": dict(Lq=200, Lcur=40, Lc=0, causal=True),
    "causal_long_queries": dict(Lq=200, Lcur=40, Lc=64, causal=True),
    "int4_g32_d128": dict(bits=4, group=32, Lc=256),
    "int2_g128_f16": dict(group=128, meta="f16", Lc=384),
    "d64_int4_g64": dict(d=64, bits=4, group=64, Lc=200),
    "d64_bf16_g32": dict(d=64, group=32, Lc=333, Lq=130),
    "f32_inputs_d128": dict(dtype="f32", Lc=256),
}


@pytest.mark.parametrize("correct", [0, 1, 2])
@pytest.mark.parametrize("case", sorted(EDGE))
def test_edge_cases(case, correct):
    base = WORKLOADS["bf16_int2"].with_(Hq=2, Hkv=2, Lq=64, Lcur=64, Lc=256, seed=77)
    check_full(base.with_(**EDGE[case]), correct)


def test_correction_term_matches_oracle():
    w = WORKLOADS["bf16_int2"].with_(Hq=4, Hkv=2, Lq=50, Lc=300)
    x = make_inputs(w, device="cuda")
    cache = build_gpu_cache(w, x["K_src"], x["V_src"])
    bias = api.jensen_bias(x["Q"], cache).cpu().numpy()
    scale = 1 / math.sqrt(w.d)
    for b in range(w.B):
        for hq in range(w.Hq):
            h = hq // 2
            step = cache.meta_view("k")[b, h, :w.Lc, :, 0].cpu().numpy().astype(np.float64)
            ref = oracle.jensen_bias_taylor(np32(x["Q"][b, hq]), step, w.group, scale)
            rel = np.abs(bias[b, hq] - ref) / np.maximum(np.abs(ref), 1e-30)
            assert rel.max() <= BIAS_REL_TOL, rel.max()
    assert api.device_status() == 0


def test_values_one_gives_rows_summing_to_one():
    """V = 1 everywhere (cache and current): every output must be exactly representable 1."""
    w = WORKLOADS["video_dit"].with_(Hq=4, Hkv=4, Lq=600, Lcur=600, Lc=1000)
    x = make_inputs(w, device="cuda")
    ones = torch.ones_like(x["V_src"])
    cache = build_gpu_cache(w, x["K_src"], ones)
    O, LSE = api.corrected_attention(x["Q"], cache, x["K_cur"], torch.ones_like(x["V_cur"]), correct=1)
    torch.cuda.synchronize()
    assert torch.all((O.float() - 1).abs() <= 1e-2)
    assert torch.isfinite(LSE).all()
    assert api.device_status() == 0


def test_repeated_calls_are_deterministic():
    w = WORKLOADS["bf16_int2"]
    x = make_inputs(w, device="cuda")
    cache = build_gpu_cache(w, x["K_src"], x["V_src"])
    O1, L1 = api.corrected_attention(x["Q"], cache, x["K_cur"], x["V_cur"], correct=1)
    O2, L2 = api.corrected_attention(x["Q"], cache, x["K_cur"], x["V_cur"], correct=1)
    torch.cuda.synchronize()
    assert torch.equal(O1, O2) and torch.equal(L1, L2)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_fourth_order_term_is_applied(dtype):
    """correct = 2 matches the oracle's fourth-order form and differs from the second-order one by
    far more than the tolerance on keys with outlier channels (large steps)."""
    w = WORKLOADS["bf16_int2"].with_(Hq=2, Hkv=2, Lq=64, Lcur=64, Lc=512, dtype=dtype, seed=78)
    x = make_inputs(w, device="cuda")
    cache = build_gpu_cache(w, x["K_src"], x["V_src"])
    O, L = api.corrected_attention(x["Q"], cache, x["K_cur"], x["V_cur"], correct=2)
    torch.cuda.synchronize()
    sub = sub_problem(x, w, 0, 1)
    O4, L4 = oracle_head(w, sub, 2)
    O2, L2 = oracle_head(w, sub, 1)
    Lg = np32(L[0:1, 1:2]).astype(np.float64)
    compare(np32(O[0:1, 1:2]).astype(np.float64), O4, Lg, L4, f"fourth order {dtype}")
    assert np.max(np.abs(L4 - L2)) > 10 * 2e-3
    assert api.device_status() == 0
