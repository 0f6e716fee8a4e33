"""Splitting one attention problem over ranks by (batch, KV head), with no exchange.

Every (batch b, KV head h) pair is an independent problem: its packed cache rows, the query heads
that read it (h * r .. h * r + r - 1 with r = Hq / Hkv, the GQA map of the kernels), its slice of
the current chunk and its slice of the outputs. In the row-major layouts of the library these are
contiguous ranges of the flattened index i = b * Hkv + h:

    Q, O          [B][Hq][Lq][d]     -> [B*Hkv][r][Lq][d]
    LSE           [B][Hq][Lq]        -> [B*Hkv][r][Lq]
    K_*, V_*      [B][Hkv][L][d]     -> [B*Hkv][1][L][d]
    cache arrays  [B][Hkv][cap][...] -> [B*Hkv][1][cap][...]

so rank k of n takes the pairs [start, stop) of a balanced contiguous partition and runs them as a
problem with B' = stop - start, Hkv' = 1 and Hq' = r. Putting the ranks' outputs back in order along
the flattened index gives the outputs of the whole problem. Host logic only (no arithmetic of the
method): it slices and concatenates arrays.
"""
from __future__ import annotations

from typing import Dict, List, Sequence, Tuple


def pair_ranges(n_pairs: int, world: int) -> List[Tuple[int, int]]:
    """Balanced contiguous partition of n_pairs (batch, KV head) pairs over `world` ranks: rank k
    takes [k * n // world, (k + 1) * n // world). Ranks beyond n_pairs get an empty range."""
    if n_pairs < 0 or world < 1:
        raise ValueError("n_pairs >= 0 and world >= 1")
    return [(k * n_pairs // world, (k + 1) * n_pairs // world) for k in range(world)]


def shard_inputs(x: Dict, B: int, Hq: int, Hkv: int, start: int, stop: int) -> Dict:
    """The sub-problem of pairs [start, stop) of inputs x (Q, K_src, V_src, K_cur, V_cur; torch
    tensors or numpy arrays), as arrays of B' = stop - start batches, r query heads and 1 KV head."""
    r = Hq // Hkv
    out = {}
    for k, t in x.items():
        if k == "Q":
            out[k] = t.reshape((B * Hkv, r) + tuple(t.shape[2:]))[start:stop]
        else:
            out[k] = t.reshape((B * Hkv, 1) + tuple(t.shape[2:]))[start:stop]
    return out


def stitch(parts: Sequence[Tuple[int, int, object]], B: int, Hq: int, Hkv: int, concat):
    """Outputs of the whole problem from per-rank outputs [(start, stop, array [stop-start][r][...])],
    with `concat` the array library's concatenation along axis 0. The ranges must cover
    [0, B * Hkv) exactly once."""
    parts = sorted(parts, key=lambda p: p[0])
    pos = 0
    for start, stop, _ in parts:
        if start != pos:
            raise ValueError(f"pairs [{pos}, {start}) missing or overlapping")
        pos = stop
    if pos != B * Hkv:
        raise ValueError(f"pairs cover [0, {pos}) of [0, {B * Hkv})")
    arrs = [a for start, stop, a in parts if stop > start]
    full = concat(arrs)
    r = Hq // Hkv
    return full.reshape((B, Hkv * r) + tuple(full.shape[2:]))
