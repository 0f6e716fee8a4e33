"""Thin ctypes binding of libqkv (include/qkv.h): argument marshalling only.

Every step of the quantise-append and corrected-attention path runs in the library's CUDA
kernels; torch provides device memory and the current stream. There is no CPU fallback: if the
library is missing or a tensor is not on a CUDA device, these functions raise.
"""
from __future__ import annotations

import ctypes
import math
import os
import re
from typing import Optional, Tuple

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libqkv.so")
HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "qkv.h")

QKV_OK, QKV_ERR_INVALID_ARG, QKV_ERR_UNSUPPORTED, QKV_ERR_CAPACITY, QKV_ERR_CUDA, QKV_ERR_TIMEOUT = \
    0, -1, -2, -3, -4, -5
QKV_F32, QKV_BF16, QKV_F16 = 0, 1, 2
CACHE_TILE = 128

_DTYPE = {torch.float32: QKV_F32, torch.bfloat16: QKV_BF16, torch.float16: QKV_F16}
_META = {"f32": (QKV_F32, torch.float32), "f16": (QKV_F16, torch.float16)}


class QkvCacheDesc(ctypes.Structure):
    """Mirror of the C struct qkv_cache."""
    _fields_ = [("B", ctypes.c_int32), ("H_kv", ctypes.c_int32), ("d", ctypes.c_int32),
                ("bits", ctypes.c_int32), ("group", ctypes.c_int32), ("meta_dtype", ctypes.c_int32),
                ("capacity", ctypes.c_int64), ("length", ctypes.c_int64),
                ("k_codes", ctypes.c_void_p), ("v_codes", ctypes.c_void_p),
                ("k_meta", ctypes.c_void_p), ("v_meta", ctypes.c_void_p),
                ("key_block", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class QkvError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{message} (status {status})")
        self.status = status


_lib = None
_P = ctypes.c_void_p
_SIGS = {
    "qkv_abi_version": (ctypes.c_int32, []),
    "qkv_status_string": (ctypes.c_char_p, [ctypes.c_int32]),
    "qkv_last_error": (ctypes.c_char_p, []),
    "qkv_cache_bytes": (ctypes.c_int, [ctypes.c_int32] * 6 + [ctypes.c_int64, ctypes.POINTER(ctypes.c_size_t),
                                                             ctypes.POINTER(ctypes.c_size_t)]),
    "qkv_cache_layout_bytes": (ctypes.c_int, [ctypes.POINTER(QkvCacheDesc)] + [ctypes.POINTER(ctypes.c_size_t)] * 4),
    "kv_quantize_append": (ctypes.c_int, [ctypes.POINTER(QkvCacheDesc), _P, _P, ctypes.c_int32,
                                          ctypes.c_int64, _P]),
    "corrected_attention_workspace_bytes": (ctypes.c_int, [ctypes.POINTER(QkvCacheDesc), ctypes.c_int32,
                                                           ctypes.c_int64, ctypes.c_int64,
                                                           ctypes.POINTER(ctypes.c_size_t)]),
    "corrected_attention": (ctypes.c_int, [_P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int64,
                                           ctypes.POINTER(QkvCacheDesc), _P, _P, ctypes.c_int64,
                                           ctypes.c_int32, ctypes.c_int32, ctypes.c_float, _P, _P, _P,
                                           ctypes.c_size_t, _P]),
    "corrected_attention_noalloc": (ctypes.c_int, [_P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int64,
                                                   ctypes.POINTER(QkvCacheDesc), _P, _P, ctypes.c_int64,
                                                   ctypes.c_int32, ctypes.c_int32, ctypes.c_float, _P, _P,
                                                   _P]),
    "qkv_jensen_bias": (ctypes.c_int, [_P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int64,
                                       ctypes.POINTER(QkvCacheDesc), ctypes.c_float, _P, _P]),
    "attention_fidelity": (ctypes.c_int, [_P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int64,
                                          ctypes.POINTER(QkvCacheDesc), _P, _P, ctypes.c_int64,
                                          ctypes.c_int32, ctypes.c_int32, ctypes.c_float, _P, _P, _P]),
    "qkv_device_status": (ctypes.c_int, [ctypes.c_int32, ctypes.POINTER(ctypes.c_int32)]),
    "qkv_set_wait_limit": (ctypes.c_int, [ctypes.c_int64, ctypes.POINTER(ctypes.c_int64)]),
}


def load_library():
    """Load libqkv.so from this package directory (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m quantized_kv_cache_19_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(lib, name)
            f.restype = res
            f.argtypes = args
        _lib = lib
    return _lib


def header_functions():
    """Names of the functions include/qkv.h declares."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:qkv_status|const char\s*\*|int32_t)\s+(\w+)\s*\(", text, flags=re.M)))


def _check(status: int):
    if status != QKV_OK:
        lib = load_library()
        msg = lib.qkv_last_error().decode() or lib.qkv_status_string(status).decode()
        raise QkvError(status, msg)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _need_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors (there is no CPU path)")


def round_capacity(tokens: int) -> int:
    return max(CACHE_TILE, -(-tokens // CACHE_TILE) * CACHE_TILE)


class KVCache:
    """Device buffers of a packed INT2/INT4 cache plus the C descriptor that points at them."""

    def __init__(self, B: int, H_kv: int, d: int, bits: int, group: int, capacity: int,
                 meta: str = "f32", device="cuda", key_block: int = 0):
        """key_block = T > 0: keys quantised per channel over blocks of T positions (values stay per
        token in groups of `group` channels)."""
        lib = load_library()
        mcode, self.meta_torch = _META[meta]
        shape = QkvCacheDesc(B, H_kv, d, bits, group, mcode, capacity, 0, None, None, None, None,
                             key_block, 0)
        kc, vc, km, vm = (ctypes.c_size_t() for _ in range(4))
        _check(lib.qkv_cache_layout_bytes(ctypes.byref(shape), ctypes.byref(kc), ctypes.byref(vc),
                                          ctypes.byref(km), ctypes.byref(vm)))
        self.device = torch.device(device)
        self.B, self.H_kv, self.d, self.bits, self.group, self.capacity, self.meta = \
            B, H_kv, d, bits, group, capacity, meta
        self.key_block = key_block
        self.n_groups = d // group
        isz = self.meta_torch.itemsize
        self.k_codes = torch.zeros(kc.value, dtype=torch.uint8, device=self.device)
        self.v_codes = torch.zeros(vc.value, dtype=torch.uint8, device=self.device)
        self.k_meta = torch.zeros(km.value // isz, dtype=self.meta_torch, device=self.device)
        self.v_meta = torch.zeros(vm.value // isz, dtype=self.meta_torch, device=self.device)
        self.desc = QkvCacheDesc(B, H_kv, d, bits, group, mcode, capacity, 0,
                                 self.k_codes.data_ptr(), self.v_codes.data_ptr(),
                                 self.k_meta.data_ptr(), self.v_meta.data_ptr(), key_block, 0)

    @property
    def length(self) -> int:
        return int(self.desc.length)

    @length.setter
    def length(self, n: int):
        if not 0 <= n <= self.capacity:
            raise ValueError("length outside [0, capacity]")
        self.desc.length = n

    def codes(self, which: str) -> torch.Tensor:
        t = self.k_codes if which == "k" else self.v_codes
        return t.view(self.B, self.H_kv, self.capacity, self.d * self.bits // 8)

    def meta_view(self, which: str) -> torch.Tensor:
        """[B][H_kv][capacity][d/group][2]; per-channel keys: [B][H_kv][capacity/T][d][2]."""
        if which == "k" and self.key_block:
            return self.k_meta.view(self.B, self.H_kv, self.capacity // self.key_block, self.d, 2)
        t = self.k_meta if which == "k" else self.v_meta
        return t.view(self.B, self.H_kv, self.capacity, self.n_groups, 2)

    def packed_bytes(self, tokens: Optional[int] = None) -> int:
        """Bytes of codes + (step, zero-point) for `tokens` tokens of K and V."""
        n = self.length if tokens is None else tokens
        codes = self.d * self.bits // 8
        v_meta = self.n_groups * 2 * self.meta_torch.itemsize
        if self.key_block:
            k_meta = -(-n // self.key_block) * self.d * 2 * self.meta_torch.itemsize
            return self.B * self.H_kv * (n * (2 * codes + v_meta) + k_meta)
        return 2 * self.B * self.H_kv * n * (codes + v_meta)


def kv_quantize_append(cache: KVCache, K: torch.Tensor, V: torch.Tensor) -> None:
    """Quantise K, V [B][H_kv][L_new][d] (fp32 or bf16) into the cache at its current length."""
    _need_cuda(K, V)
    if K.shape != V.shape or K.dim() != 4 or K.shape[0] != cache.B or K.shape[1] != cache.H_kv \
            or K.shape[3] != cache.d or K.dtype != V.dtype:
        raise ValueError("K, V must both be [B][H_kv][L_new][d] of one dtype")
    lib = load_library()
    _check(lib.kv_quantize_append(ctypes.byref(cache.desc), _ptr(K), _ptr(V), _DTYPE[K.dtype],
                                  K.shape[2], _stream(K.device)))


def corrected_attention(Q: torch.Tensor, cache: KVCache, K_cur: Optional[torch.Tensor],
                        V_cur: Optional[torch.Tensor], correct: int = 1, causal: bool = False,
                        scale: float = 0.0, out: Optional[torch.Tensor] = None,
                        lse: Optional[torch.Tensor] = None,
                        workspace="auto") -> Tuple[torch.Tensor, torch.Tensor]:
    """O [B][H_q][L_q][d] (Q's dtype) and LSE [B][H_q][L_q] (fp32) of the corrected attention.

    workspace: "auto" allocates the scratch the library asks for (a key split for shapes with few
    query rows per KV head); None runs without it (no split); a uint8 CUDA tensor is used as is.
    """
    _need_cuda(Q, K_cur, V_cur, out, lse)
    B, Hq, Lq, d = Q.shape
    Lcur = 0 if K_cur is None else K_cur.shape[2]
    if K_cur is not None and (K_cur.dtype != Q.dtype or V_cur.dtype != Q.dtype):
        raise ValueError("K_cur, V_cur must have Q's dtype")
    if out is None:
        out = torch.empty_like(Q)
    if lse is None:
        lse = torch.empty(B, Hq, Lq, dtype=torch.float32, device=Q.device)
    lib = load_library()
    ws = ctypes.c_size_t()
    _check(lib.corrected_attention_workspace_bytes(ctypes.byref(cache.desc), Hq, Lq, Lcur, ctypes.byref(ws)))
    if isinstance(workspace, torch.Tensor):
        _need_cuda(workspace)
        work, nbytes = workspace, workspace.numel() * workspace.element_size()
    elif workspace == "auto" and ws.value:
        work, nbytes = torch.empty(ws.value, dtype=torch.uint8, device=Q.device), ws.value
    else:
        work, nbytes = None, 0
    _check(lib.corrected_attention(_ptr(Q), _DTYPE[Q.dtype], Hq, Lq, ctypes.byref(cache.desc),
                                   _ptr(K_cur), _ptr(V_cur), Lcur, int(correct), int(bool(causal)),
                                   float(scale), _ptr(out), _ptr(lse), _ptr(work), nbytes,
                                   _stream(Q.device)))
    return out, lse


def corrected_attention_noalloc(Q: torch.Tensor, cache: KVCache, K_cur: Optional[torch.Tensor],
                                V_cur: Optional[torch.Tensor], correct: int = 1, causal: bool = False,
                                scale: float = 0.0, out: Optional[torch.Tensor] = None,
                                lse: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """corrected_attention through the entry point that allocates nothing (library-owned scratch).

    For callers that may not allocate device memory; only O and LSE are allocated here when not
    given. Calls that overlap on the GPU share the library's scratch and must not run concurrently.
    """
    _need_cuda(Q, K_cur, V_cur, out, lse)
    B, Hq, Lq, d = Q.shape
    Lcur = 0 if K_cur is None else K_cur.shape[2]
    if K_cur is not None and (K_cur.dtype != Q.dtype or V_cur.dtype != Q.dtype):
        raise ValueError("K_cur, V_cur must have Q's dtype")
    if out is None:
        out = torch.empty_like(Q)
    if lse is None:
        lse = torch.empty(B, Hq, Lq, dtype=torch.float32, device=Q.device)
    lib = load_library()
    _check(lib.corrected_attention_noalloc(_ptr(Q), _DTYPE[Q.dtype], Hq, Lq, ctypes.byref(cache.desc),
                                           _ptr(K_cur), _ptr(V_cur), Lcur, int(correct), int(bool(causal)),
                                           float(scale), _ptr(out), _ptr(lse), _stream(Q.device)))
    return out, lse


def attention_workspace_bytes(cache: KVCache, Hq: int, Lq: int, Lcur: int) -> int:
    """Scratch bytes with which corrected_attention splits the cached keys (0: no split)."""
    lib = load_library()
    ws = ctypes.c_size_t()
    _check(lib.corrected_attention_workspace_bytes(ctypes.byref(cache.desc), Hq, Lq, Lcur, ctypes.byref(ws)))
    return int(ws.value)


FIDELITY_FIELDS = ("lse_ref", "lse_q", "mass_ref", "mass_q", "kl", "top1_agree", "recall")


def attention_fidelity(Q: torch.Tensor, cache: KVCache, K_ref: Optional[torch.Tensor],
                       K_cur: Optional[torch.Tensor], correct: int = 1, causal: bool = False,
                       scale: float = 0.0, with_top: bool = True
                       ) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Per-row fidelity of the quantised attention against the unquantised keys.

    K_ref [B][H_kv][cache.length][d] (Q's dtype): the cached keys before quantisation.
    Returns stats fp32 [B][H_q][L_q][8] (columns named by FIDELITY_FIELDS, the last one 0) and, with
    with_top, top int32 [B][H_q][L_q][2][5]: the reference's and the quantised softmax's five
    highest-scoring key indices (cached keys first, then current keys; -1 pads).
    """
    _need_cuda(Q, K_ref, K_cur)
    B, Hq, Lq, d = Q.shape
    Lcur = 0 if K_cur is None else K_cur.shape[2]
    for t in (K_ref, K_cur):
        if t is not None and t.dtype != Q.dtype:
            raise ValueError("K_ref, K_cur must have Q's dtype")
    if K_ref is not None and tuple(K_ref.shape) != (B, cache.H_kv, cache.length, d):
        raise ValueError("K_ref must be [B][H_kv][cache.length][d]")
    stats = torch.empty(B, Hq, Lq, 8, dtype=torch.float32, device=Q.device)
    top = torch.empty(B, Hq, Lq, 2, 5, dtype=torch.int32, device=Q.device) if with_top else None
    lib = load_library()
    _check(lib.attention_fidelity(_ptr(Q), _DTYPE[Q.dtype], Hq, Lq, ctypes.byref(cache.desc),
                                  _ptr(K_ref), _ptr(K_cur), Lcur, int(correct), int(bool(causal)),
                                  float(scale), _ptr(stats), _ptr(top), _stream(Q.device)))
    return stats, top


def jensen_bias(Q: torch.Tensor, cache: KVCache, scale: float = 0.0) -> torch.Tensor:
    """bias [B][H_q][L_q][length] fp32: the correction term the attention subtracts."""
    _need_cuda(Q)
    B, Hq, Lq, d = Q.shape
    out = torch.empty(B, Hq, Lq, cache.length, dtype=torch.float32, device=Q.device)
    lib = load_library()
    _check(lib.qkv_jensen_bias(_ptr(Q), _DTYPE[Q.dtype], Hq, Lq, ctypes.byref(cache.desc),
                               float(scale), _ptr(out), _stream(Q.device)))
    return out


def device_status(reset: bool = True) -> int:
    """The library's device status word (0 = no kernel reported an error); synchronises."""
    lib = load_library()
    code = ctypes.c_int32()
    _check(lib.qkv_device_status(int(reset), ctypes.byref(code)))
    return int(code.value)


def set_wait_limit(cycles: int) -> int:
    """Bound, in SM clock cycles, of the internal waits of kernels launched from now on (0 restores
    the default of 2e9); returns the previous bound. For tests of the timeout path."""
    lib = load_library()
    prev = ctypes.c_int64()
    _check(lib.qkv_set_wait_limit(int(cycles), ctypes.byref(prev)))
    return int(prev.value)


def attention_flops(B: int, Hq: int, Lq: int, Lc: int, Lcur: int, d: int, causal: bool = False) -> float:
    """Algorithmic tensor FLOPs: 4 d per (query, visible key) pair (QK^T and PV)."""
    if causal:
        vis_cur = sum(min(Lcur, max(0, i + 1 + Lcur - Lq)) for i in range(Lq))
    else:
        vis_cur = Lq * Lcur
    return 4.0 * d * B * Hq * (Lq * Lc + vis_cur)


def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)
