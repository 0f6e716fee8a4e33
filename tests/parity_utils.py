"""Shared helpers of the GPU parity tests: run the CUDA path, run the oracle on the same bytes."""
from __future__ import annotations

import math
from typing import Dict, Optional, Sequence

import numpy as np
import torch

import oracle
from quantized_kv_cache_19_b200 import api
from quantized_kv_cache_19_b200.workloads import Workload, make_inputs

# Agreement criteria for the attention output and LSE (bf16 operands, fp32 accumulation).
O_REL_TOL = 1e-2
LSE_ABS_TOL = 2e-3
BIAS_REL_TOL = 1e-5


def np32(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()


def build_gpu_cache(w: Workload, K: torch.Tensor, V: torch.Tensor, chunk: Optional[int] = None,
                    capacity: Optional[int] = None) -> api.KVCache:
    """Quantise-append K, V [B][Hkv][L][d] chunk by chunk into a fresh device cache."""
    L = K.shape[2]
    cache = api.KVCache(w.B, w.Hkv, w.d, w.bits, w.group, capacity or api.round_capacity(L), w.meta,
                        device=K.device)
    step = chunk or max(L, 1)
    for t0 in range(0, L, step):
        api.kv_quantize_append(cache, K[:, :, t0:t0 + step].contiguous(), V[:, :, t0:t0 + step].contiguous())
    assert cache.length == L
    return cache


def sub_problem(x: Dict[str, torch.Tensor], w: Workload, b: int, h: int) -> Dict[str, np.ndarray]:
    """The oracle's inputs for one (batch, KV head): arrays shaped [1][r or 1][L][d]."""
    r = w.Hq // w.Hkv
    return {
        "Q": np32(x["Q"][b:b + 1, h * r:(h + 1) * r]),
        "K_src": np32(x["K_src"][b:b + 1, h:h + 1]),
        "V_src": np32(x["V_src"][b:b + 1, h:h + 1]),
        "K_cur": np32(x["K_cur"][b:b + 1, h:h + 1]),
        "V_cur": np32(x["V_cur"][b:b + 1, h:h + 1]),
    }


def oracle_head(w: Workload, sub: Dict[str, np.ndarray], correct: int, rows=None):
    cache = oracle.build_cache(sub["K_src"], sub["V_src"], w.bits, w.group, w.meta) if w.Lc else None
    return oracle.corrected_attention(sub["Q"], cache, sub["K_cur"], sub["V_cur"], correct=correct,
                                      causal=w.causal, scale=1.0 / math.sqrt(w.d), rows=rows)


def compare(O: np.ndarray, O_ref: np.ndarray, L: np.ndarray, L_ref: np.ndarray, what: str):
    """O [..., n, d] per head group: max|O-O_ref| / max|O_ref| <= 1e-2; |LSE - LSE_ref| <= 2e-3."""
    fin = np.isfinite(L_ref)
    assert np.array_equal(np.isfinite(L), fin), f"{what}: rows without keys differ"
    assert np.all(O[~fin] == 0), f"{what}: rows without keys must be 0"
    lse_err = float(np.max(np.abs(L[fin] - L_ref[fin]), initial=0.0))
    num = np.max(np.abs(O - O_ref), axis=(-1, -2))
    den = np.maximum(np.max(np.abs(O_ref), axis=(-1, -2)), 1e-30)
    o_err = float(np.max(num / den))
    assert o_err <= O_REL_TOL, f"{what}: O max relative error {o_err:.3e}"
    assert lse_err <= LSE_ABS_TOL, f"{what}: LSE max abs error {lse_err:.3e}"
    return o_err, lse_err


def run_gpu(w: Workload, x: Dict[str, torch.Tensor], correct: int, cache: Optional[api.KVCache] = None):
    if cache is None:
        cache = build_gpu_cache(w, x["K_src"], x["V_src"])
    Kc = x["K_cur"] if w.Lcur else None
    Vc = x["V_cur"] if w.Lcur else None
    O, LSE = api.corrected_attention(x["Q"], cache, Kc, Vc, correct=correct, causal=w.causal)
    torch.cuda.synchronize()
    return cache, O, LSE


def check_full(w: Workload, correct: int, seed: Optional[int] = None):
    """Every output row of every head against the oracle (small workloads)."""
    x = make_inputs(w, device="cuda", seed=seed)
    cache, O, LSE = run_gpu(w, x, correct)
    r = w.Hq // w.Hkv
    worst = (0.0, 0.0)
    for b in range(w.B):
        for h in range(w.Hkv):
            sub = sub_problem(x, w, b, h)
            O_ref, L_ref = oracle_head(w, sub, correct)
            Og = np32(O[b:b + 1, h * r:(h + 1) * r]).astype(np.float64)
            Lg = np32(LSE[b:b + 1, h * r:(h + 1) * r]).astype(np.float64)
            e = compare(Og, O_ref, Lg, L_ref, f"{w.name} b{b} h{h} correct={correct}")
            worst = (max(worst[0], e[0]), max(worst[1], e[1]))
    assert api.device_status() == 0
    return worst


def check_sampled(w: Workload, correct: int, heads: Sequence[tuple], n_rows: int = 64):
    """Full-size launch; sampled packed rows of a few (batch, KV head) pairs against the oracle."""
    from quantized_kv_cache_19_b200.workloads import sample_rows
    x = make_inputs(w, device="cuda")
    chunk = w.Lcur if w.Lcur else None
    cache = build_gpu_cache(w, x["K_src"], x["V_src"], chunk=chunk)
    _, O, LSE = run_gpu(w, x, correct, cache)
    rows = sample_rows(w, n_rows).numpy()
    r = w.Hq // w.Hkv
    worst = (0.0, 0.0)
    for (b, h) in heads:
        sub = sub_problem(x, w, b, h)
        O_ref, L_ref = oracle_head(w, sub, correct, rows=rows)
        hq = h * r + rows // w.Lq
        qi = rows % w.Lq
        Og = np32(O[b, torch.as_tensor(hq), torch.as_tensor(qi)])[None, None].astype(np.float64)
        Lg = np32(LSE[b, torch.as_tensor(hq), torch.as_tensor(qi)])[None, None].astype(np.float64)
        e = compare(Og, O_ref, Lg, L_ref, f"{w.name} b{b} h{h} correct={correct}")
        worst = (max(worst[0], e[0]), max(worst[1], e[1]))
    assert api.device_status() == 0
    return worst
