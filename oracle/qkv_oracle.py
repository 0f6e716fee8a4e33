"""Oracle: plain numpy restatement of the corrected low-bit KV-cache attention.

TEST INFRASTRUCTURE ONLY (see the package docstring). Nothing here is blocked,
fused or reordered beyond what the definitions state; a library matmul serves as
the dot-product step.

Sources (cited by page title and section):
  [JB]   agents-report.net, "KV-Cache 量化導致的 Jensen 偏差：以每分數校正恢復影片擴散品質"
         (summary of Tuncer, Becker, Pfeil, arXiv 2605.26266), sections
         「問題：量化後的注意力偏移與 Jensen 偏差」 (problem), 「方法：逐分數的偏差校正與實作近似」
         (method: b_i = log E[e^{delta_i}] and its Taylor form), 「為何校正有效？」 (why it works:
         subtract b_i from quantised-key scores before the softmax), 「限制與邊界情況」 (limits).
  [ABS]  fugumt.com, "Quantized Keys Steal Attention: Bias Correction for KV-Cache Compression
         in Video Diffusion", Abstract (correction from step sizes and query norm, no extra memory).
  [QWM]  pchao.org, "QuantWM：保住时间一致性的两比特键值缓存量化", eq. (5): logits are Q K^T / sqrt(d);
         section 实验如何设计 (token drift: top-1 attended token differing from the BF16 one).
  [SIQ]  gist.science, "Statistical Inference and Quality Measures of KV Cache Quantisations
         Inspired by TurboQuant", section Métricas de Avaliação (KL divergence between reference and
         quantised softmax distributions, top-5 recall).

Readings taken where the pages are silent (each one is also listed in the design notes):
  * Quantiser: asymmetric min-max per (token, head, group of `group` consecutive channels);
    step = (max - min) / (2^bits - 1) and zero-point = min, both computed in IEEE fp32 and
    then stored in the meta dtype (fp32 or fp16, round to nearest even). Codes use the STORED
    step and zero-point: code = clamp(rint((x - zp) * (1/step)), 0, 2^bits - 1), every
    operation a single correctly rounded fp32 operation, ties to even; a zero step gives code 0.
  * Packing: the codes of one (token, head) row form a little-endian bit string, channel c at
    bit c*bits, i.e. byte (c*bits)//8, bit (c*bits)%8.
  * Per-channel keys (optional, key_block = T): every T consecutive cache positions (aligned to
    position 0; the last block may be shorter) of one channel share a step and zero-point, by the
    same fp32 arithmetic; codes are packed per token as above; values keep per-token groups.
    The correction then uses each key's own per-channel steps.
  * Score scale: s = scale * q.k with scale = 1/sqrt(d) unless given; the correction is in the
    same scaled-score units. For a general scale the Taylor term is (scale^2/24) sum_c q_c^2
    Delta_c^2, which is the page's (1/(24 d)) sum_c q_c^2 Delta_{i,c}^2 at scale = 1/sqrt(d).
  * Correction modes: 0 none, 1 the second-order Taylor form of [JB] 方法, 2 the series of the exact
    form to fourth order (a^2/6 - a^4/180 per channel), 3 the exact form (oracle only).
  * Exact correction (not printed on the pages, called numerically unfavourable in [JB] 方法):
    uniform rounding noise e_c ~ U(-Delta_c/2, Delta_c/2) gives E[e^{a u}] = sinh(a)/a, so
    b = sum_c log(sinh(a_c)/a_c), a_c = scale * q_c * Delta_c / 2.
  * Only cached (quantised) keys get the correction; current-chunk keys get none ([JB] 為何).
  * V is quantised with the same quantiser; no correction is applied on the value side.
  * Causal mask (optional) acts inside the current chunk only, bottom-right aligned: query i
    (of Lq) sees current key j (of Lcur) iff j <= i + (Lcur - Lq). The cache is always visible.
  * GQA: query head hq reads KV head hq // (Hq // Hkv).
  * LSE is the natural-log log-sum-exp of the corrected scores of each query row.
  * Fidelity diagnostics: the reference distribution is the softmax over the cached keys as they
    were before quantisation (in the input precision) and the current keys; the quantised one is
    the corrected attention's softmax. Top-k lists break equal scores by the lower key index;
    recall counts over min(k, visible keys) keys; the top-k size is 5 ([SIQ]).
"""
from __future__ import annotations

import math
from typing import Dict, Optional, Sequence, Tuple

import numpy as np

__all__ = [
    "META_DTYPES", "levels", "quantize", "pack_codes", "unpack_codes", "dequantize",
    "build_cache", "cache_rows", "log_sinhc", "jensen_bias_taylor", "jensen_bias_exact",
    "attention_rows", "corrected_attention", "merge_partials", "jensen_bias_taylor4",
    "FIDELITY_TOPK", "fidelity_rows", "quantize_tokens", "key_step_group",
]

META_DTYPES = {"f32": np.float32, "f16": np.float16}


def levels(bits: int) -> int:
    """Largest code of a `bits`-bit unsigned integer code ([JB] 問題: INT4 / INT2 keys and values)."""
    return (1 << bits) - 1


# --------------------------------------------------------------------------------------------
# Quantiser ([JB] 問題 "low-bit integer quantisation"; step Delta and zero-point as in [ABS]).
# --------------------------------------------------------------------------------------------
def quantize(x: np.ndarray, bits: int, group: int, meta: str = "f32"
             ) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Group-wise asymmetric min-max quantisation of the last axis.

    x: [..., d] (converted to fp32; bf16 / fp32 inputs are exact in fp32).
    Returns codes uint8 [..., d] (unpacked), step [..., d/group] and zero-point [..., d/group]
    in the meta dtype. All arithmetic is single fp32 IEEE operations in the order written.
    """
    x = np.asarray(x, dtype=np.float32)
    d = x.shape[-1]
    if d % group:
        raise ValueError("d must be a multiple of group")
    mt = META_DTYPES[meta]
    xg = x.reshape(x.shape[:-1] + (d // group, group))
    mn = xg.min(axis=-1)
    mx = xg.max(axis=-1)
    step32 = (mx - mn) / np.float32(levels(bits))          # fp32 subtract, fp32 divide
    step = step32.astype(mt)                               # stored step (RN to meta dtype)
    zp = mn.astype(mt)                                     # stored zero-point
    stepf = step.astype(np.float32)                        # values the codes are taken against
    zpf = zp.astype(np.float32)
    pos = stepf > 0
    inv = np.zeros_like(stepf)
    inv[pos] = np.float32(1.0) / stepf[pos]                # fp32 reciprocal, RN
    t = (xg - zpf[..., None]) * inv[..., None]             # fp32 subtract then fp32 multiply
    code = np.clip(np.rint(t), 0, levels(bits))            # ties to even, clamp to the code range
    code = np.where(pos[..., None], code, 0).astype(np.uint8)
    return code.reshape(x.shape), step, zp


def pack_codes(codes: np.ndarray, bits: int) -> np.ndarray:
    """Pack codes [..., d] into bytes [..., d*bits/8]: channel c at bit c*bits, LSB first."""
    codes = np.asarray(codes, dtype=np.uint8)
    per = 8 // bits
    d = codes.shape[-1]
    c = codes.reshape(codes.shape[:-1] + (d // per, per))
    out = np.zeros(c.shape[:-1], dtype=np.uint8)
    for k in range(per):
        out |= (c[..., k] << np.uint8(k * bits)).astype(np.uint8)
    return out


def unpack_codes(packed: np.ndarray, bits: int) -> np.ndarray:
    """Inverse of pack_codes."""
    packed = np.asarray(packed, dtype=np.uint8)
    per = 8 // bits
    mask = np.uint8(levels(bits))
    parts = [(packed >> np.uint8(k * bits)) & mask for k in range(per)]
    return np.stack(parts, axis=-1).reshape(packed.shape[:-1] + (packed.shape[-1] * per,))


def dequantize(codes: np.ndarray, step: np.ndarray, zp: np.ndarray, group: int) -> np.ndarray:
    """x_hat = zp + step * code per group, in fp64 from the stored (meta-dtype) step and zero-point."""
    n_g = step.shape[-1]
    c = np.asarray(codes, dtype=np.float64).reshape(codes.shape[:-1] + (n_g, group))
    xh = zp.astype(np.float64)[..., None] + step.astype(np.float64)[..., None] * c
    return xh.reshape(codes.shape)


def quantize_tokens(x: np.ndarray, bits: int, block: int, meta: str = "f32"
                    ) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Per-channel asymmetric min-max quantisation along the token axis (KIVI's key grouping, named
    in [JB] 跨主題對比分析; [BLOG] groups along the sequence axis): tokens [k*block, (k+1)*block)
    of one channel share one step and zero-point; the last block may be shorter.

    x: [..., L, d]. Returns codes uint8 [..., L, d] (unpacked), step and zero-point
    [..., ceil(L/block), d] in the meta dtype. The arithmetic of each (block, channel) is that of
    `quantize` for one group: single fp32 IEEE operations in the same order.
    """
    x = np.asarray(x, dtype=np.float32)
    L, d = x.shape[-2], x.shape[-1]
    nb = -(-L // block)
    mt = META_DTYPES[meta]
    codes = np.zeros(x.shape, dtype=np.uint8)
    step = np.zeros(x.shape[:-2] + (nb, d), dtype=mt)
    zp = np.zeros(x.shape[:-2] + (nb, d), dtype=mt)
    for k in range(nb):
        xb = x[..., k * block:(k + 1) * block, :]
        mn = xb.min(axis=-2)
        mx = xb.max(axis=-2)
        step32 = (mx - mn) / np.float32(levels(bits))
        step[..., k, :] = step32.astype(mt)
        zp[..., k, :] = mn.astype(mt)
        stepf = step[..., k, :].astype(np.float32)
        zpf = zp[..., k, :].astype(np.float32)
        pos = stepf > 0
        inv = np.zeros_like(stepf)
        inv[pos] = np.float32(1.0) / stepf[pos]
        t = (xb - zpf[..., None, :]) * inv[..., None, :]
        code = np.clip(np.rint(t), 0, levels(bits))
        codes[..., k * block:(k + 1) * block, :] = np.where(pos[..., None, :], code, 0).astype(np.uint8)
    return codes, step, zp


def build_cache(K: np.ndarray, V: np.ndarray, bits: int, group: int, meta: str = "f32",
                key_block: int = 0) -> Dict:
    """Quantise previous-chunk keys and values [B][Hkv][L][d] into the oracle's cache record.

    key_block = 0: keys in groups of `group` channels per token, like values. key_block = T > 0: keys
    per channel over blocks of T tokens (`quantize_tokens`); values stay per token.
    """
    if key_block:
        kc, ks, kz = quantize_tokens(K, bits, key_block, meta)
    else:
        kc, ks, kz = quantize(K, bits, group, meta)
    vc, vs, vz = quantize(V, bits, group, meta)
    return {"bits": bits, "group": group, "meta": meta, "key_block": key_block,
            "k_codes": kc, "k_step": ks, "k_zp": kz,
            "v_codes": vc, "v_step": vs, "v_zp": vz}


def key_step_group(cache: Optional[Dict], d: int) -> int:
    """Channels that share one key step within a key, as `cache_rows` returns the steps: `group` for
    per-token key groups, 1 for per-channel keys."""
    if cache is None:
        return d
    return 1 if cache.get("key_block") else cache["group"]


def cache_rows(cache: Dict, b: int, h: int) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Dequantised keys, values [Lc][d] (fp64) and key steps of one (batch, KV head): [Lc][n_g] for
    per-token key groups, [Lc][d] (each key's own per-channel steps) for per-channel keys."""
    g = cache["group"]
    T = cache.get("key_block", 0)
    if T:
        codes = cache["k_codes"][b, h]
        Lc = codes.shape[0]
        ks = np.repeat(cache["k_step"][b, h].astype(np.float64), T, axis=0)[:Lc]
        kz = np.repeat(cache["k_zp"][b, h].astype(np.float64), T, axis=0)[:Lc]
        kh = kz + ks * codes.astype(np.float64)
    else:
        kh = dequantize(cache["k_codes"][b, h], cache["k_step"][b, h], cache["k_zp"][b, h], g)
        ks = cache["k_step"][b, h].astype(np.float64)
    vh = dequantize(cache["v_codes"][b, h], cache["v_step"][b, h], cache["v_zp"][b, h], g)
    return kh, vh, ks


# --------------------------------------------------------------------------------------------
# Jensen-bias correction ([JB] 方法, [ABS]).
# --------------------------------------------------------------------------------------------
_SERIES = (1.0 / 6.0, -1.0 / 180.0, 1.0 / 2835.0, -1.0 / 37800.0, 1.0 / 467775.0)


def log_sinhc(a: np.ndarray) -> np.ndarray:
    """log(sinh(a)/a) = log E[exp(a u)], u ~ U(-1, 1); even in a, 0 at a = 0.

    Small |a| (< 0.1): the Maclaurin series sum_n 2^{2n} B_{2n} a^{2n} / (2n (2n)!) to a^10.
    Otherwise: |a| + log(-expm1(-2|a|)) - log(2|a|), which has no cancellation there.
    """
    a = np.abs(np.asarray(a, dtype=np.float64))
    out = np.empty_like(a)
    small = a < 0.1
    s2 = a[small] ** 2
    acc = np.zeros_like(s2)
    for coef in reversed(_SERIES):
        acc = (acc + coef) * s2
    out[small] = acc
    L = a[~small]
    out[~small] = L + np.log(-np.expm1(-2.0 * L)) - np.log(2.0 * L)
    return out


def _per_channel(step: np.ndarray, group: int) -> np.ndarray:
    """Delta_{j,c}: the step of the group that channel c belongs to (channel c is in group c // group)."""
    return np.repeat(np.asarray(step, dtype=np.float64), group, axis=-1)


def jensen_bias_taylor(q: np.ndarray, step: np.ndarray, group: int, scale: float) -> np.ndarray:
    """Second-order correction b_ij = (scale^2 / 24) sum_c q_ic^2 Delta_{j,c}^2.

    q: [n, d] queries, step: [Lc, d/group] key steps. Returns [n, Lc]. At scale = 1/sqrt(d) this
    is the (1/(24 d)) sum_c q_c^2 Delta_{i,c}^2 of [JB] 方法.
    """
    dc = _per_channel(step, group)
    q = np.asarray(q, dtype=np.float64)
    return (scale * scale / 24.0) * ((q * q) @ (dc * dc).T)


def jensen_bias_taylor4(q: np.ndarray, step: np.ndarray, group: int, scale: float) -> np.ndarray:
    """Correction to fourth order: b_ij = sum_c (a^2/6 - a^4/180), a = scale q_ic Delta_{j,c} / 2.

    The first two terms of the series of log(sinh a / a) (the exact form below). The a^2 term is
    the second-order correction of [JB] 方法; the a^4 term is
    -(scale^4 / 2880) sum_c q_ic^4 Delta_{j,c}^4, again a sum over channel groups of a per-query
    power sum times a per-key step power.
    """
    dc = _per_channel(step, group)
    q = np.asarray(q, dtype=np.float64)
    q2 = q * q
    return jensen_bias_taylor(q, step, group, scale) - (scale ** 4 / 2880.0) * ((q2 * q2) @ (dc ** 4).T)


def jensen_bias_exact(q: np.ndarray, step: np.ndarray, group: int, scale: float) -> np.ndarray:
    """Exact correction for uniform rounding noise: b_ij = sum_c log(sinh(a)/a), a = scale q_ic Delta_{j,c} / 2."""
    dc = _per_channel(step, group)
    q = np.asarray(q, dtype=np.float64)
    out = np.empty((q.shape[0], dc.shape[0]))
    for i in range(q.shape[0]):
        a = 0.5 * scale * q[i][None, :] * dc
        out[i] = log_sinhc(a).sum(axis=-1)
    return out


# --------------------------------------------------------------------------------------------
# Corrected attention over [cache ; current] ([JB] 為何: subtract b_i from the scores of the
# quantised cached keys, then softmax over cached and current keys; [QWM] eq. (5) for the scale).
# --------------------------------------------------------------------------------------------
def attention_rows(q: np.ndarray, q_pos: np.ndarray, k_hat: np.ndarray, v_hat: np.ndarray,
                   k_step: np.ndarray, group: int, k_cur: np.ndarray, v_cur: np.ndarray,
                   correct: int, causal: bool, scale: float, Lq: int
                   ) -> Tuple[np.ndarray, np.ndarray]:
    """Attention of query rows q [n, d] (positions q_pos in the chunk of Lq queries).

    k_hat, v_hat [Lc, d]: dequantised cache; k_step [Lc, n_g]; k_cur, v_cur [Lcur, d].
    correct: 0 none, 1 second-order Taylor (the paper's), 2 fourth-order Taylor, 3 exact (oracle only).
    Returns O [n, d] and LSE [n] (natural log), fp64.
    """
    q = np.asarray(q, dtype=np.float64)
    k_cur = np.asarray(k_cur, dtype=np.float64)
    v_cur = np.asarray(v_cur, dtype=np.float64)
    n, Lc, Lcur = q.shape[0], k_hat.shape[0], k_cur.shape[0]
    s_cache = scale * (q @ k_hat.T)
    if correct == 1 and Lc:
        s_cache = s_cache - jensen_bias_taylor(q, k_step, group, scale)
    elif correct == 2 and Lc:
        s_cache = s_cache - jensen_bias_taylor4(q, k_step, group, scale)
    elif correct == 3 and Lc:
        s_cache = s_cache - jensen_bias_exact(q, k_step, group, scale)
    s_cur = scale * (q @ k_cur.T)
    if causal and Lcur:
        lim = np.asarray(q_pos)[:, None] + (Lcur - Lq)
        s_cur = np.where(np.arange(Lcur)[None, :] <= lim, s_cur, -np.inf)
    s = np.concatenate([s_cache, s_cur], axis=1)
    v = np.concatenate([v_hat, v_cur], axis=0)
    m = s.max(axis=1, initial=-np.inf)
    m_safe = np.where(np.isfinite(m), m, 0.0)
    p = np.exp(s - m_safe[:, None])
    l = p.sum(axis=1)
    with np.errstate(invalid="ignore", divide="ignore"):
        o = (p @ v) / l[:, None]
        lse = m_safe + np.log(l)
    o = np.where(l[:, None] > 0, o, 0.0)
    return o, lse


def corrected_attention(Q: np.ndarray, cache: Optional[Dict], K_cur: np.ndarray, V_cur: np.ndarray,
                        correct: int = 1, causal: bool = False, scale: Optional[float] = None,
                        rows: Optional[Sequence[int]] = None) -> Tuple[np.ndarray, np.ndarray]:
    """Full corrected attention. Q [B][Hq][Lq][d]; K_cur, V_cur [B][Hkv][Lcur][d].

    cache: record from build_cache over [B][Hkv][Lc][d] (None means an empty cache).
    rows: optional packed-row sample per KV head (row = (hq % r) * Lq + i); then the outputs are
    O [B][Hkv][len(rows)][d] and LSE [B][Hkv][len(rows)] for those rows only.
    Without rows: O [B][Hq][Lq][d], LSE [B][Hq][Lq].
    """
    Q = np.asarray(Q, dtype=np.float64)
    B, Hq, Lq, d = Q.shape
    Hkv = K_cur.shape[1]
    r = Hq // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    group = key_step_group(cache, d)
    if rows is None:
        O = np.zeros((B, Hq, Lq, d))
        LSE = np.zeros((B, Hq, Lq))
    else:
        rows = np.asarray(rows)
        O = np.zeros((B, Hkv, len(rows), d))
        LSE = np.zeros((B, Hkv, len(rows)))
    for b in range(B):
        for h in range(Hkv):
            if cache is not None:
                kh, vh, ks = cache_rows(cache, b, h)
            else:
                kh, vh, ks = np.zeros((0, d)), np.zeros((0, d)), np.zeros((0, 1))
            if rows is None:
                for j in range(r):
                    hq = h * r + j
                    o, lse = attention_rows(Q[b, hq], np.arange(Lq), kh, vh, ks, group,
                                            K_cur[b, h], V_cur[b, h], correct, causal, scale, Lq)
                    O[b, hq], LSE[b, hq] = o, lse
            else:
                hq = h * r + rows // Lq
                pos = rows % Lq
                o, lse = attention_rows(Q[b, hq, pos], pos, kh, vh, ks, group,
                                        K_cur[b, h], V_cur[b, h], correct, causal, scale, Lq)
                O[b, h], LSE[b, h] = o, lse
    return O, LSE


def merge_partials(parts: Sequence[Tuple[np.ndarray, np.ndarray]]) -> Tuple[np.ndarray, np.ndarray]:
    """Combine attention results over disjoint key sets: LSE = logsumexp_k LSE_k, O = sum_k e^{LSE_k - LSE} O_k."""
    lses = np.stack([p[1] for p in parts])
    m = lses.max(axis=0)
    w = np.exp(lses - m)
    lse = m + np.log(w.sum(axis=0))
    o = sum(np.exp(p[1] - lse)[..., None] * p[0] for p in parts)
    return o, lse


# --------------------------------------------------------------------------------------------
# Attention-fidelity diagnostics: how far the softmax over the quantised cache is from the one
# over the unquantised keys. [QWM] 实验如何设计 defines the token drift rate as the share of
# positions whose top-1 attended token under the quantised cache differs from the BF16 one;
# [SIQ] Métricas de Avaliação uses the KL divergence between the reference and the quantised
# softmax distributions and the recall of the reference's top-5 keys; [JB] 為何校正有效 and the
# [ABS] title describe the quantised keys' excess ("stolen") attention mass on the cached segment.
# --------------------------------------------------------------------------------------------
FIDELITY_TOPK = 5


def _top_keys(s: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest finite scores of each row, largest first, the lower index first on
    equal scores; -1 where a row has fewer than k visible keys."""
    n = s.shape[0]
    out = np.full((n, k), -1, dtype=np.int64)
    for i in range(n):
        vis = np.flatnonzero(np.isfinite(s[i]))
        order = vis[np.argsort(-s[i, vis], kind="stable")]
        out[i, :min(k, order.size)] = order[:k]
    return out


def fidelity_rows(q: np.ndarray, q_pos: np.ndarray, k_ref: np.ndarray, k_hat: np.ndarray,
                  k_step: np.ndarray, group: int, k_cur: np.ndarray, correct: int, causal: bool,
                  scale: float, Lq: int, topk: int = FIDELITY_TOPK,
                  return_scores: bool = False) -> Dict[str, np.ndarray]:
    """Per query row q [n, d] (positions q_pos in the chunk of Lq queries), fp64:

    P_ref: softmax of scale q.k over [k_ref ; k_cur] (k_ref [Lc, d]: the cached keys unquantised);
    P_q:   softmax over [k_hat ; k_cur] of scale q.k minus the correction of mode `correct` on the
           cached keys (the scores of `attention_rows`).
    Returns lse_ref, lse_q (natural log), mass_ref, mass_q (total probability of the Lc cached keys),
    kl = KL(P_ref || P_q) = sum_j P_ref,j (log P_ref,j - log P_q,j), top_ref / top_q [n, topk] (the
    `_top_keys` of each score row; key index j < Lc is cached key j, Lc + t is current key t),
    top1_agree (1.0 where the two top-1 keys coincide) and recall (share of the reference's top
    keys that are among the quantised ones, over min(topk, visible keys) keys).
    A row that sees no key: lse -inf, masses 0, kl 0, top -1, top1_agree 1, recall 1.
    With return_scores, also s_ref and s_q [n, Lc + Lcur] (-inf where a key is masked).
    """
    q = np.asarray(q, dtype=np.float64)
    k_ref = np.asarray(k_ref, dtype=np.float64)
    k_cur = np.asarray(k_cur, dtype=np.float64)
    n, Lc, Lcur = q.shape[0], k_hat.shape[0], k_cur.shape[0]
    s_ref_cache = scale * (q @ k_ref.T)
    s_q_cache = scale * (q @ k_hat.T)
    if correct == 1 and Lc:
        s_q_cache = s_q_cache - jensen_bias_taylor(q, k_step, group, scale)
    elif correct == 2 and Lc:
        s_q_cache = s_q_cache - jensen_bias_taylor4(q, k_step, group, scale)
    elif correct == 3 and Lc:
        s_q_cache = s_q_cache - jensen_bias_exact(q, k_step, group, scale)
    s_cur = scale * (q @ k_cur.T)
    if causal and Lcur:
        lim = np.asarray(q_pos)[:, None] + (Lcur - Lq)
        s_cur = np.where(np.arange(Lcur)[None, :] <= lim, s_cur, -np.inf)
    s_ref = np.concatenate([s_ref_cache, s_cur], axis=1)
    s_q = np.concatenate([s_q_cache, s_cur], axis=1)

    def log_softmax(s):
        m = s.max(axis=1, initial=-np.inf)
        m_safe = np.where(np.isfinite(m), m, 0.0)
        with np.errstate(divide="ignore", invalid="ignore"):
            lse = m_safe + np.log(np.exp(s - m_safe[:, None]).sum(axis=1))
            return s - lse[:, None], lse

    logp_ref, lse_ref = log_softmax(s_ref)
    logp_q, lse_q = log_softmax(s_q)
    p_ref, p_q = np.exp(logp_ref), np.exp(logp_q)
    vis = np.isfinite(s_ref)
    kl = np.where(vis, p_ref * (np.where(vis, logp_ref, 0.0) - np.where(vis, logp_q, 0.0)), 0.0).sum(axis=1)
    top_ref = _top_keys(s_ref, topk)
    top_q = _top_keys(s_q, topk)
    agree = np.ones(n)
    recall = np.ones(n)
    for i in range(n):
        r = top_ref[i][top_ref[i] >= 0]
        if r.size:
            agree[i] = float(top_ref[i, 0] == top_q[i, 0])
            recall[i] = np.isin(r, top_q[i]).sum() / r.size
    out = {"lse_ref": lse_ref, "lse_q": lse_q,
           "mass_ref": p_ref[:, :Lc].sum(axis=1), "mass_q": p_q[:, :Lc].sum(axis=1),
           "kl": kl, "top_ref": top_ref, "top_q": top_q, "top1_agree": agree, "recall": recall}
    if return_scores:
        out["s_ref"], out["s_q"] = s_ref, s_q
    return out
