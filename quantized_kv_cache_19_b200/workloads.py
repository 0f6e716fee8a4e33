"""Seeded synthetic workloads for chunk-wise attention over a low-bit KV cache.

This module only draws random tensors with the shapes and value distributions of
the five workloads below; it holds none of the method's arithmetic (no
quantisation, no attention, no correction). Both the CUDA path (tests, bench)
and the CPU oracle (tests) receive the bytes it produces.

Shapes follow the chunk-wise autoregressive video-diffusion setting of
"Quantized Keys Steal Attention: Bias Correction for KV-Cache Compression in
Video Diffusion" (abstract): the current chunk's queries attend over a cache of
previous chunks plus the unquantised current chunk. The model weights, prompts
and videos of that paper are not available, so standard-normal tensors with the
per-channel key structure named in each workload stand in for real activations.

Layouts (all contiguous, row-major):
  Q      [B][Hq][Lq][d]
  K_src  [B][Hkv][Lc][d]    keys of the previous chunks, before quantisation
  V_src  [B][Hkv][Lc][d]
  K_cur  [B][Hkv][Lcur][d]  the current (unquantised) chunk
  V_cur  [B][Hkv][Lcur][d]
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    Lq: int
    Lcur: int
    Lc: int
    bits: int
    group: int
    meta: str          # "f32" or "f16": storage type of the per-group (step, zero-point)
    dtype: str         # "f32" or "bf16": type of Q, K, V
    causal: bool       # causal mask inside the current chunk
    k_style: str       # per-channel key structure, see _key_structure
    k_frac: float = 0.0
    k_param: float = 0.0
    seed: int = 0

    @property
    def n_groups(self) -> int:
        return self.d // self.group

    @property
    def rows_per_kv_head(self) -> int:
        return (self.Hq // self.Hkv) * self.Lq

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads. Where a workload leaves a count open (outlier or heavy-tail
# channel count) it is round(frac * d), at least one channel, chosen per KV head
# by a seeded permutation; the same channels are used in the cached and the
# current keys.
WORKLOADS: Dict[str, Workload] = {
    "tiny_f32": Workload("tiny_f32", B=1, Hq=2, Hkv=2, d=64, Lq=64, Lcur=64, Lc=256,
                         bits=2, group=32, meta="f32", dtype="f32", causal=False,
                         k_style="chan_uniform", k_frac=0.0, k_param=0.0, seed=1001),
    "bf16_int4": Workload("bf16_int4", B=1, Hq=16, Hkv=16, d=128, Lq=1024, Lcur=1024, Lc=4096,
                          bits=4, group=64, meta="f32", dtype="bf16", causal=False,
                          k_style="outlier", k_frac=0.05, k_param=8.0, seed=1002),
    "bf16_int2": Workload("bf16_int2", B=1, Hq=16, Hkv=16, d=128, Lq=1024, Lcur=1024, Lc=4096,
                          bits=2, group=64, meta="f32", dtype="bf16", causal=False,
                          k_style="outlier", k_frac=0.05, k_param=8.0, seed=1002),
    "video_dit": Workload("video_dit", B=1, Hq=24, Hkv=24, d=128, Lq=4680, Lcur=4680, Lc=28080,
                          bits=2, group=64, meta="f32", dtype="bf16", causal=False,
                          k_style="lognormal", k_frac=0.0, k_param=0.7, seed=1003),
    "long_video": Workload("long_video", B=1, Hq=40, Hkv=40, d=128, Lq=1560, Lcur=1560, Lc=99840,
                           bits=2, group=128, meta="f16", dtype="bf16", causal=False,
                           k_style="student_t", k_frac=0.05, k_param=3.0, seed=1004),
    "prefill_gqa": Workload("prefill_gqa", B=4, Hq=32, Hkv=8, d=128, Lq=512, Lcur=512, Lc=131072,
                            bits=2, group=64, meta="f32", dtype="bf16", causal=True,
                            k_style="outlier", k_frac=0.02, k_param=10.0, seed=1005),
}

TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}


def _channel_pick(gen: torch.Generator, Hkv: int, d: int, frac: float, device) -> torch.Tensor:
    """Boolean mask [Hkv][d] of the structured channels of each KV head."""
    count = max(1, int(round(frac * d)))
    mask = torch.zeros(Hkv, d, dtype=torch.bool, device=device)
    for h in range(Hkv):
        perm = torch.randperm(d, generator=gen, device=device)
        mask[h, perm[:count]] = True
    return mask


def _key_structure(w: Workload, gen: torch.Generator, device):
    """Per-(KV head, channel) key structure: ('scale', s[Hkv][d]) or ('student_t', mask)."""
    if w.k_style == "none":
        return ("scale", torch.ones(w.Hkv, w.d, device=device))
    if w.k_style == "chan_uniform":      # channels scaled by U(0.5, 3)
        u = torch.rand(w.Hkv, w.d, generator=gen, device=device)
        return ("scale", 0.5 + 2.5 * u)
    if w.k_style == "outlier":           # a fraction of channels multiplied by k_param
        m = _channel_pick(gen, w.Hkv, w.d, w.k_frac, device)
        return ("scale", torch.where(m, torch.tensor(w.k_param, device=device),
                                     torch.tensor(1.0, device=device)))
    if w.k_style == "lognormal":         # per-channel scale exp(sigma * N(0,1))
        z = torch.randn(w.Hkv, w.d, generator=gen, device=device)
        return ("scale", torch.exp(w.k_param * z))
    if w.k_style == "student_t":         # a fraction of channels drawn from Student-t(nu)
        return ("student_t", _channel_pick(gen, w.Hkv, w.d, w.k_frac, device))
    raise ValueError(w.k_style)


def _student_t(shape, nu: int, gen: torch.Generator, device) -> torch.Tensor:
    """Student-t(nu) for integer nu: z0 / sqrt(chi2_nu / nu), chi2_nu a sum of nu squared normals."""
    z0 = torch.randn(shape, generator=gen, device=device)
    chi2 = torch.zeros(shape, device=device)
    for _ in range(nu):
        chi2 += torch.randn(shape, generator=gen, device=device) ** 2
    return z0 / torch.sqrt(chi2 / nu)


def _keys(w: Workload, L: int, struct, gen: torch.Generator, device) -> torch.Tensor:
    k = torch.randn(w.B, w.Hkv, L, w.d, generator=gen, device=device)
    kind, val = struct
    if kind == "scale":
        k *= val[None, :, None, :]
    else:
        t = _student_t((w.B, w.Hkv, L, w.d), int(w.k_param), gen, device)
        k = torch.where(val[None, :, None, :], t, k)
    return k


def make_inputs(w: Workload, device: str = "cpu", seed: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """Draw Q, K_src, V_src, K_cur, V_cur for workload `w` on `device`.

    The generator lives on `device`, so a given seed yields the same bytes for
    every call on the same kind of device; the oracle is given copies of exactly
    these tensors.
    """
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed if seed is None else seed)
    dt = TORCH_DTYPE[w.dtype]
    struct = _key_structure(w, gen, device)
    out = {
        "Q": torch.randn(w.B, w.Hq, w.Lq, w.d, generator=gen, device=device).to(dt),
        "K_src": _keys(w, w.Lc, struct, gen, device).to(dt),
        "V_src": torch.randn(w.B, w.Hkv, w.Lc, w.d, generator=gen, device=device).to(dt),
        "K_cur": _keys(w, w.Lcur, struct, gen, device).to(dt),
        "V_cur": torch.randn(w.B, w.Hkv, w.Lcur, w.d, generator=gen, device=device).to(dt),
    }
    return {k: v.contiguous() for k, v in out.items()}


def sample_rows(w: Workload, n: int, seed: int = 7) -> torch.Tensor:
    """Seeded sample of n distinct packed query rows of one KV head (row = head_in_group * Lq + i)."""
    gen = torch.Generator().manual_seed(seed)
    total = w.rows_per_kv_head
    n = min(n, total)
    return torch.randperm(total, generator=gen)[:n].sort().values
