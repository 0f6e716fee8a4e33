"""The C-ABI library loads without a GPU, exports what include/qkv.h declares, and rejects bad
arguments on the host (no CUDA call is made on any path exercised here)."""
import ctypes

import pytest

from quantized_kv_cache_19_b200 import api


def test_exports_every_header_function(lib):
    names = api.header_functions()
    assert {"kv_quantize_append", "corrected_attention", "qkv_jensen_bias", "qkv_cache_bytes",
            "corrected_attention_workspace_bytes", "qkv_device_status", "qkv_status_string",
            "qkv_last_error", "qkv_abi_version"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n
    assert lib.qkv_abi_version() == 2


def test_status_strings(lib):
    assert lib.qkv_status_string(0) == b"ok"
    assert lib.qkv_status_string(-3) == b"cache capacity exceeded"
    assert lib.qkv_status_string(-5) == b"device wait timed out"


@pytest.mark.parametrize("args,codes,meta", [
    ((1, 2, 64, 2, 32, api.QKV_F32, 256), 2 * 256 * 16, 2 * 256 * 2 * 2 * 4),
    ((1, 16, 128, 4, 64, api.QKV_F32, 5120), 16 * 5120 * 64, 16 * 5120 * 2 * 2 * 4),
    ((1, 40, 128, 2, 128, api.QKV_F16, 99840), 40 * 99840 * 32, 40 * 99840 * 1 * 2 * 2),
    ((4, 8, 128, 2, 64, api.QKV_F32, 131072), 32 * 131072 * 32, 32 * 131072 * 2 * 2 * 4),
])
def test_cache_bytes(lib, args, codes, meta):
    cb, mb = ctypes.c_size_t(), ctypes.c_size_t()
    assert lib.qkv_cache_bytes(*args, ctypes.byref(cb), ctypes.byref(mb)) == 0
    assert (cb.value, mb.value) == (codes, meta)


@pytest.mark.parametrize("args,status", [
    ((1, 2, 64, 3, 32, api.QKV_F32, 256), api.QKV_ERR_UNSUPPORTED),     # 3-bit codes
    ((1, 2, 96, 2, 32, api.QKV_F32, 256), api.QKV_ERR_UNSUPPORTED),     # head dim
    ((1, 2, 64, 2, 128, api.QKV_F32, 256), api.QKV_ERR_INVALID_ARG),    # group > d
    ((1, 2, 64, 2, 32, api.QKV_F32, 200), api.QKV_ERR_INVALID_ARG),     # capacity not a tile multiple
    ((0, 2, 64, 2, 32, api.QKV_F32, 256), api.QKV_ERR_INVALID_ARG),
    ((1, 2, 64, 2, 32, api.QKV_BF16, 256), api.QKV_ERR_UNSUPPORTED),    # meta must be f32 / f16
])
def test_cache_bytes_rejects(lib, args, status):
    cb, mb = ctypes.c_size_t(), ctypes.c_size_t()
    assert lib.qkv_cache_bytes(*args, ctypes.byref(cb), ctypes.byref(mb)) == status
    assert lib.qkv_last_error() != b""


def _fake_cache(**kw):
    c = dict(B=1, H_kv=2, d=128, bits=2, group=64, meta_dtype=api.QKV_F32, capacity=256, length=0,
             k_codes=0x10000, v_codes=0x20000, k_meta=0x30000, v_meta=0x40000)
    c.update(kw)
    return api.QkvCacheDesc(**c)


def test_append_rejections(lib):
    c = _fake_cache(length=200)
    s = lib.kv_quantize_append(ctypes.byref(c), ctypes.c_void_p(0x50000), ctypes.c_void_p(0x60000),
                               api.QKV_BF16, 57, None)
    assert s == api.QKV_ERR_CAPACITY and c.length == 200
    assert b"exceed" in lib.qkv_last_error() or b"append" in lib.qkv_last_error()
    assert lib.kv_quantize_append(ctypes.byref(c), ctypes.c_void_p(0x50000), ctypes.c_void_p(0x60000),
                                  api.QKV_F16, 8, None) == api.QKV_ERR_UNSUPPORTED
    assert lib.kv_quantize_append(ctypes.byref(c), ctypes.c_void_p(0x50008), ctypes.c_void_p(0x60000),
                                  api.QKV_BF16, 8, None) == api.QKV_ERR_INVALID_ARG
    assert lib.kv_quantize_append(ctypes.byref(c), None, None, api.QKV_BF16, 0, None) == 0  # no-op
    assert c.length == 200
    bad = _fake_cache(k_meta=0x30004)
    assert lib.kv_quantize_append(ctypes.byref(bad), ctypes.c_void_p(0x50000), ctypes.c_void_p(0x60000),
                                  api.QKV_BF16, 8, None) == api.QKV_ERR_INVALID_ARG
    assert lib.kv_quantize_append(None, None, None, api.QKV_BF16, 8, None) == api.QKV_ERR_INVALID_ARG


def test_attention_rejections(lib):
    c = _fake_cache(length=0)
    P = ctypes.c_void_p
    q, o, l = P(0x70000), P(0x80000), P(0x90000)
    call = lambda **kw: lib.corrected_attention(
        kw.get("Q", q), kw.get("dt", api.QKV_BF16), kw.get("Hq", 4), kw.get("Lq", 16), ctypes.byref(kw.get("c", c)),
        kw.get("K", P(0xA0000)), kw.get("V", P(0xB0000)), kw.get("Lcur", 0), kw.get("corr", 1), 0,
        kw.get("scale", 0.0), o, l, None, 0, None)
    assert call() == api.QKV_ERR_INVALID_ARG                         # no keys at all
    c2 = _fake_cache(length=100)
    assert call(c=c2, Hq=3) == api.QKV_ERR_INVALID_ARG               # H_q not a multiple of H_kv
    assert call(c=c2, dt=api.QKV_F16) == api.QKV_ERR_UNSUPPORTED
    assert call(c=c2, corr=3) == api.QKV_ERR_UNSUPPORTED             # exact correction is oracle-only
    assert call(c=c2, corr=-1) == api.QKV_ERR_UNSUPPORTED
    assert call(c=c2, Q=P(0x70002)) == api.QKV_ERR_INVALID_ARG       # misaligned
    assert call(c=c2, Lcur=8, K=None) == api.QKV_ERR_INVALID_ARG
    assert call(c=c2, scale=float("nan")) == api.QKV_ERR_INVALID_ARG
    assert call(c=c2, Lq=0) == 0                                     # empty query chunk: no-op
    ws = ctypes.c_size_t(1)
    assert lib.corrected_attention_workspace_bytes(ctypes.byref(c2), 4, 16, 8, ctypes.byref(ws)) == 0
    assert lib.qkv_jensen_bias(q, api.QKV_BF16, 3, 16, ctypes.byref(c2), 0.0, P(0xC0000), None) == \
        api.QKV_ERR_INVALID_ARG


def test_fidelity_rejections(lib):
    c = _fake_cache(length=0)
    P = ctypes.c_void_p
    q, st = P(0x70000), P(0x80000)
    call = lambda **kw: lib.attention_fidelity(
        kw.get("Q", q), kw.get("dt", api.QKV_BF16), kw.get("Hq", 4), kw.get("Lq", 16), ctypes.byref(kw.get("c", c)),
        kw.get("Kref", P(0xA0000)), kw.get("K", P(0xB0000)), kw.get("Lcur", 0), kw.get("corr", 1),
        kw.get("causal", 0), kw.get("scale", 0.0), kw.get("stats", st), kw.get("top", None), None)
    assert call() == api.QKV_ERR_INVALID_ARG                         # no keys at all
    c2 = _fake_cache(length=100)
    assert call(c=c2, Hq=3) == api.QKV_ERR_INVALID_ARG
    assert call(c=c2, dt=api.QKV_F16) == api.QKV_ERR_UNSUPPORTED
    assert call(c=c2, corr=3) == api.QKV_ERR_UNSUPPORTED
    assert call(c=c2, causal=2) == api.QKV_ERR_INVALID_ARG
    assert call(c=c2, Kref=None) == api.QKV_ERR_INVALID_ARG          # cached keys need K_ref
    assert call(c=c2, Lcur=8, K=None) == api.QKV_ERR_INVALID_ARG
    assert call(c=c2, stats=None) == api.QKV_ERR_INVALID_ARG
    assert call(c=c2, top=P(0x90004)) == api.QKV_ERR_INVALID_ARG     # misaligned
    assert call(c=c2, Kref=P(0xA0008)) == api.QKV_ERR_INVALID_ARG
    assert call(c=c2, scale=float("inf")) == api.QKV_ERR_INVALID_ARG
    assert call(c=c2, Lcur=2 ** 31) == api.QKV_ERR_UNSUPPORTED       # key indices are int32
    assert call(c=c2, Lq=0) == 0                                     # empty query chunk: no-op


def test_descriptor_size_matches_the_header():
    # 6 int32, 2 int64, 4 pointers, key_block and reserved
    assert ctypes.sizeof(api.QkvCacheDesc) == 6 * 4 + 2 * 8 + 4 * 8 + 2 * 4


@pytest.mark.parametrize("key_block,meta,k_meta", [
    (0, api.QKV_F32, 2 * 256 * 2 * 2 * 4),            # per-token: [B][H][cap][d/group][2]
    (32, api.QKV_F32, 2 * (256 // 32) * 128 * 2 * 4),  # per-channel: [B][H][cap/T][d][2]
    (128, api.QKV_F16, 2 * (256 // 128) * 128 * 2 * 2),
])
def test_layout_bytes(lib, key_block, meta, k_meta):
    c = _fake_cache(key_block=key_block, meta_dtype=meta)
    out = [ctypes.c_size_t() for _ in range(4)]
    assert lib.qkv_cache_layout_bytes(ctypes.byref(c), *[ctypes.byref(o) for o in out]) == 0
    kc, vc, km, vm = (o.value for o in out)
    msz = 4 if meta == api.QKV_F32 else 2
    assert kc == vc == 2 * 256 * 32
    assert vm == 2 * 256 * 2 * 2 * msz
    assert km == k_meta


def test_key_block_rejections(lib):
    P = ctypes.c_void_p
    out = [ctypes.c_size_t() for _ in range(4)]
    bad = _fake_cache(key_block=16)
    assert lib.qkv_cache_layout_bytes(ctypes.byref(bad), *[ctypes.byref(o) for o in out]) == \
        api.QKV_ERR_UNSUPPORTED
    assert lib.kv_quantize_append(ctypes.byref(bad), P(0x50000), P(0x60000), api.QKV_BF16, 8, None) == \
        api.QKV_ERR_UNSUPPORTED
    # appends must start on a block boundary; the cache is left unchanged
    c = _fake_cache(key_block=32, length=40)
    assert lib.kv_quantize_append(ctypes.byref(c), P(0x50000), P(0x60000), api.QKV_BF16, 8, None) == \
        api.QKV_ERR_UNSUPPORTED
    assert c.length == 40 and b"key_block" in lib.qkv_last_error()
    # a decode-sized query chunk over per-channel keys asks for a key split: n partial rows of d + 1
    c2 = _fake_cache(key_block=64, length=256, capacity=256)
    ws = ctypes.c_size_t(0)
    assert lib.corrected_attention_workspace_bytes(ctypes.byref(c2), 2, 1, 1, ctypes.byref(ws)) == 0
    rows_all = 1 * 2 * 1
    assert ws.value > 0 and ws.value % (rows_all * (128 + 1) * 4) == 0
    # the fidelity diagnostics accept per-channel caches (an empty query chunk: no launch)
    st = P(0x80000)
    assert lib.attention_fidelity(P(0x70000), api.QKV_BF16, 2, 0, ctypes.byref(c2), P(0xA0000), None, 0,
                                  1, 0, 0.0, st, None, None) == 0


def test_symbol_address_cache_policy(tmp_path):
    """The remembered device addresses of the library's own device variables (the status word and
    the allocation-free entry point's scratch) are reused only in the CUDA context they were looked
    up in, and the cache is safe across host threads: a host-only C++ test of the helper."""
    import os
    import shutil
    import subprocess
    gxx = shutil.which("g++")
    if gxx is None:
        pytest.skip("g++ not available")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    exe = str(tmp_path / "symbol_cache_test")
    subprocess.run([gxx, "-std=c++17", "-O1", "-pthread",
                    "-I" + os.path.join(root, "quantized_kv_cache_19_b200", "csrc"),
                    os.path.join(root, "tests", "native", "symbol_cache_test.cpp"), "-o", exe],
                   check=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout + r.stderr
