// C ABI of libqkv: argument validation, dispatch to the kernels, error reporting.
// The declarations, layouts and error behaviour are documented in include/qkv.h.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <algorithm>
#include <atomic>
#include <mutex>
#include <string>

#include "../../include/qkv.h"
#include "channel.h"
#include "fidelity.h"
#include "qkv_internal.h"
#include "symbol_cache.h"

#define QKV_API extern "C" __attribute__((visibility("default")))

namespace qkv {

// Device status word of this library: 0 = ok, else a negative qkv_status set by a kernel.
__device__ int g_device_status;

// Bound of the progress waits of kernels launched from now on, in SM clock cycles.
static std::atomic<long long> g_wait_limit{kDefaultWaitLimitCycles};

namespace {

thread_local std::string t_last_error;

qkv_status fail(qkv_status s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
qkv_status fail(qkv_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  t_last_error = buf;
  return s;
}

qkv_status cuda_fail(cudaError_t e, const char* what) {
  return fail(QKV_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Unique id of the current CUDA context (0 if there is none, or if the driver cannot say). The
// driver calls are reached through the runtime's entry-point query, so the library does not link
// the driver library itself.
unsigned long long current_context_id() {
  using GetCurrent = int (*)(void**);
  using GetId = int (*)(void*, unsigned long long*);
  static GetCurrent get_current = nullptr;
  static GetId get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrent>(f);
    f = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetId>(f);
    cudaGetLastError();
  });
  if (!get_current || !get_id) return 0;
  void* ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != 0 || ctx == nullptr || get_id(ctx, &id) != 0) return 0;
  return id;
}

// Device address of one of the library's __device__ variables on the current device, looked up
// again whenever the current context is not the one the remembered address was taken in.
template <class T>
void* symbol_address(SymbolAddressCache& cache, const T& symbol, cudaError_t* err) {
  int dev = 0;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return nullptr;
  unsigned long long ctx = current_context_id();
  if (ctx == 0) {
    // No context yet on this thread: the runtime creates the device's primary context on the
    // first call that needs one, such as this lookup; then its id can be read.
    void* p = nullptr;
    *err = cudaGetSymbolAddress(&p, symbol);
    if (*err != cudaSuccess) return nullptr;
    ctx = current_context_id();
  }
  void* out = nullptr;
  cudaError_t lookup_err = cudaSuccess;
  const int rc = cache.get(dev, ctx, [&](void** p) {
    lookup_err = cudaGetSymbolAddress(p, symbol);
    return lookup_err == cudaSuccess ? 0 : 1;
  }, &out);
  if (rc != 0) {
    *err = rc == -1 ? cudaErrorInvalidDevice : lookup_err;
    return nullptr;
  }
  *err = cudaSuccess;
  return out;
}

SymbolAddressCache g_status_addr;

// Address of g_device_status on the current device, in the current context.
int* status_word(cudaError_t* err) {
  return static_cast<int*>(symbol_address(g_status_addr, g_device_status, err));
}

qkv_status check_shape(int32_t B, int32_t H_kv, int32_t d, int32_t bits, int32_t group,
                       int32_t meta_dtype, int64_t capacity) {
  if (B < 1 || H_kv < 1) return fail(QKV_ERR_INVALID_ARG, "B and H_kv must be >= 1");
  if (capacity < QKV_CACHE_TILE || capacity % QKV_CACHE_TILE)
    return fail(QKV_ERR_INVALID_ARG, "capacity must be a positive multiple of %d", QKV_CACHE_TILE);
  if (d != 64 && d != 128) return fail(QKV_ERR_UNSUPPORTED, "head dim %d not supported (64, 128)", d);
  if (bits != 2 && bits != 4) return fail(QKV_ERR_UNSUPPORTED, "bits %d not supported (2, 4)", bits);
  if (group != 32 && group != 64 && group != 128)
    return fail(QKV_ERR_UNSUPPORTED, "group %d not supported (32, 64, 128)", group);
  if (d % group) return fail(QKV_ERR_INVALID_ARG, "group %d does not divide d %d", group, d);
  if (meta_dtype != QKV_F32 && meta_dtype != QKV_F16)
    return fail(QKV_ERR_UNSUPPORTED, "meta dtype must be QKV_F32 or QKV_F16");
  return QKV_OK;
}

qkv_status check_key_block(int32_t key_block) {
  if (key_block != 0 && key_block != 32 && key_block != 64 && key_block != 128)
    return fail(QKV_ERR_UNSUPPORTED, "key_block %d not supported (0, 32, 64, 128)", key_block);
  return QKV_OK;
}

qkv_status check_cache(const qkv_cache* c) {
  if (c == nullptr) return fail(QKV_ERR_INVALID_ARG, "cache is NULL");
  qkv_status s = check_shape(c->B, c->H_kv, c->d, c->bits, c->group, c->meta_dtype, c->capacity);
  if (s != QKV_OK) return s;
  if (c->length < 0 || c->length > c->capacity)
    return fail(QKV_ERR_INVALID_ARG, "cache length %lld outside [0, capacity]",
                static_cast<long long>(c->length));
  if (!c->k_codes || !c->v_codes || !c->k_meta || !c->v_meta)
    return fail(QKV_ERR_INVALID_ARG, "cache buffer is NULL");
  if (!aligned16(c->k_codes) || !aligned16(c->v_codes) || !aligned16(c->k_meta) ||
      !aligned16(c->v_meta))
    return fail(QKV_ERR_INVALID_ARG, "cache buffers must be 16-byte aligned");
  return check_key_block(c->key_block);
}

bool in_dtype_ok(int32_t dt) { return dt == QKV_F32 || dt == QKV_BF16; }

}  // namespace
}  // namespace qkv

using namespace qkv;

QKV_API int32_t qkv_abi_version(void) { return QKV_ABI_VERSION; }

QKV_API const char* qkv_status_string(int32_t s) {
  switch (s) {
    case QKV_OK: return "ok";
    case QKV_ERR_INVALID_ARG: return "invalid argument";
    case QKV_ERR_UNSUPPORTED: return "unsupported configuration";
    case QKV_ERR_CAPACITY: return "cache capacity exceeded";
    case QKV_ERR_CUDA: return "CUDA error";
    case QKV_ERR_TIMEOUT: return "device wait timed out";
    default: return "unknown status";
  }
}

QKV_API const char* qkv_last_error(void) { return t_last_error.c_str(); }

QKV_API qkv_status qkv_cache_bytes(int32_t B, int32_t H_kv, int32_t d, int32_t bits, int32_t group,
                                   int32_t meta_dtype, int64_t capacity, size_t* codes_bytes_each,
                                   size_t* meta_bytes_each) {
  t_last_error.clear();
  qkv_status s = check_shape(B, H_kv, d, bits, group, meta_dtype, capacity);
  if (s != QKV_OK) return s;
  if (!codes_bytes_each || !meta_bytes_each) return fail(QKV_ERR_INVALID_ARG, "NULL output");
  const size_t tokens = static_cast<size_t>(B) * H_kv * static_cast<size_t>(capacity);
  *codes_bytes_each = tokens * (d * bits / 8);
  *meta_bytes_each = tokens * (d / group) * 2 * (meta_dtype == QKV_F16 ? 2 : 4);
  return QKV_OK;
}

QKV_API qkv_status qkv_cache_layout_bytes(const qkv_cache* c, size_t* k_codes, size_t* v_codes,
                                          size_t* k_meta, size_t* v_meta) {
  t_last_error.clear();
  if (c == nullptr) return fail(QKV_ERR_INVALID_ARG, "cache is NULL");
  qkv_status s = check_shape(c->B, c->H_kv, c->d, c->bits, c->group, c->meta_dtype, c->capacity);
  if (s != QKV_OK) return s;
  s = check_key_block(c->key_block);
  if (s != QKV_OK) return s;
  if (!k_codes || !v_codes || !k_meta || !v_meta) return fail(QKV_ERR_INVALID_ARG, "NULL output");
  const size_t tokens = static_cast<size_t>(c->B) * c->H_kv * static_cast<size_t>(c->capacity);
  const size_t mb = c->meta_dtype == QKV_F16 ? 2 : 4;
  *k_codes = *v_codes = tokens * (c->d * c->bits / 8);
  *v_meta = tokens * (c->d / c->group) * 2 * mb;
  *k_meta = c->key_block ? tokens / c->key_block * c->d * 2 * mb : *v_meta;
  return QKV_OK;
}

QKV_API qkv_status kv_quantize_append(qkv_cache* cache, const void* K, const void* V,
                                      int32_t in_dtype, int64_t L_new, void* stream) {
  t_last_error.clear();
  qkv_status s = check_cache(cache);
  if (s != QKV_OK) return s;
  if (!in_dtype_ok(in_dtype)) return fail(QKV_ERR_UNSUPPORTED, "input dtype must be F32 or BF16");
  if (L_new < 0) return fail(QKV_ERR_INVALID_ARG, "L_new must be >= 0");
  if (L_new > cache->capacity - cache->length)
    return fail(QKV_ERR_CAPACITY, "append of %lld tokens to a cache holding %lld of %lld",
                static_cast<long long>(L_new), static_cast<long long>(cache->length),
                static_cast<long long>(cache->capacity));
  if (L_new == 0) return QKV_OK;
  if (!K || !V) return fail(QKV_ERR_INVALID_ARG, "K or V is NULL");
  if (!aligned16(K) || !aligned16(V)) return fail(QKV_ERR_INVALID_ARG, "K and V must be 16-byte aligned");
  QuantAppendParams p;
  p.K = K; p.V = V;
  p.k_codes = cache->k_codes; p.v_codes = cache->v_codes;
  p.k_meta = cache->k_meta; p.v_meta = cache->v_meta;
  p.BH = static_cast<int64_t>(cache->B) * cache->H_kv;
  p.L_new = L_new;
  p.capacity = cache->capacity;
  p.start = cache->length;
  p.d = cache->d;
  p.group = cache->group;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cache->key_block) {
    // Keys per channel over blocks of key_block positions: an append starts a new block.
    if (cache->length % cache->key_block)
      return fail(QKV_ERR_UNSUPPORTED,
                  "per-channel key blocks: the cache length %lld is not a multiple of key_block %d "
                  "(only the last append may end inside a block)",
                  static_cast<long long>(cache->length), cache->key_block);
    ChanQuantParams kp;
    kp.K = K; kp.k_codes = cache->k_codes; kp.k_meta = cache->k_meta;
    kp.BH = p.BH; kp.L_new = L_new; kp.capacity = cache->capacity; kp.start = cache->length;
    kp.d = cache->d; kp.T = cache->key_block;
    if (kp.BH > 65535 || (L_new + kp.T - 1) / kp.T > 2147483647LL)
      return fail(QKV_ERR_UNSUPPORTED, "grid too large");
    p.K = nullptr;                    // the per-token kernel quantises V only
    cudaError_t e = launch_quantize_keys_channel(kp, in_dtype, cache->meta_dtype, cache->bits, st);
    if (e != cudaSuccess) return cuda_fail(e, "kv_quantize_append (keys) launch");
  }
  cudaError_t e = launch_quantize_append(p, in_dtype, cache->meta_dtype, cache->bits, st);
  if (e != cudaSuccess) return cuda_fail(e, "kv_quantize_append launch");
  cache->length += L_new;
  return QKV_OK;
}

// Splits of the cached keys for the tensor-core kernels: used only when the (row tile, batch * KV
// head) grid of 128-row CTAs would leave more than half of the SMs idle (few query rows per KV
// head, e.g. decoding). The kernels run one CTA per SM, so the split count is the one whose grid
// fills whole waves of the SMs best (the smallest such), at most 32 (the merge's limit) and at most
// one split per key tile of `tile` keys. 1 = no split.
static int wave_splits(const qkv_cache* c, int32_t H_q, int64_t L_q, int tile) {
  if (L_q <= 0 || c->length <= 0) return 1;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    sms = 148;
  }
  const int64_t rows = static_cast<int64_t>(H_q / c->H_kv) * L_q;
  const int64_t ctas = (rows + 127) / 128 * c->B * c->H_kv;
  const int64_t tiles = (c->length + tile - 1) / tile;
  if (ctas * 2 > sms || tiles < 2) return 1;
  int best = 1;
  double best_fill = -1.0;
  for (int n = 1; n <= 32 && n <= tiles; ++n) {
    const int64_t grid = ctas * n;
    const double fill = static_cast<double>(grid) / static_cast<double>(((grid + sms - 1) / sms) * sms);
    if (fill > best_fill + 1e-9) {
      best_fill = fill;
      best = n;
    }
  }
  return best;
}

static int attention_splits(const qkv_cache* c, int32_t H_q, int64_t L_q) {
  return wave_splits(c, H_q, L_q, attention_tile_keys(c->d / c->group));
}

// Splits of the cached keys for the per-channel-key kernels (bf16 inputs). The tensor-core kernel
// (`tc`) splits like the per-token one. The CUDA-core kernel splits only when the (row tile,
// batch * KV head) grid would leave more than half of the SMs idle, into as many splits as fit one
// wave: splitting fuller grids was measured slower, as that kernel gains nothing from a second CTA
// on an SM. 1 = no split.
static int channel_splits(const qkv_cache* c, int32_t H_q, int64_t L_q, bool tc) {
  if (tc) return wave_splits(c, H_q, L_q, kChanTcTileKeys);
  if (L_q <= 0 || c->length <= 0) return 1;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    sms = 148;
  }
  const int64_t rows = static_cast<int64_t>(H_q / c->H_kv) * L_q;
  const int64_t rpc = channel_rows_per_cta();
  const int64_t ctas = (rows + rpc - 1) / rpc * c->B * c->H_kv;
  const int64_t tiles = (c->length + channel_tile_keys() - 1) / channel_tile_keys();
  if (ctas * 2 > sms || tiles < 2) return 1;
  int64_t n = sms / ctas;
  if (n > tiles) n = tiles;
  if (n > 32) n = 32;
  return n < 1 ? 1 : static_cast<int>(n);
}

static size_t split_workspace_bytes(const qkv_cache* c, int32_t H_q, int64_t L_q, int n) {
  if (n <= 1) return 0;
  const size_t rows_all = static_cast<size_t>(c->B) * H_q * L_q;
  return static_cast<size_t>(n) * rows_all * (static_cast<size_t>(c->d) + 1) * sizeof(float);
}

QKV_API qkv_status corrected_attention_workspace_bytes(const qkv_cache* cache, int32_t H_q,
                                                       int64_t L_q, int64_t L_cur, size_t* bytes) {
  t_last_error.clear();
  qkv_status s = check_cache(cache);
  if (s != QKV_OK) return s;
  if (!bytes) return fail(QKV_ERR_INVALID_ARG, "NULL output");
  if (H_q < 1 || H_q % cache->H_kv || L_q < 0 || L_cur < 0)
    return fail(QKV_ERR_INVALID_ARG, "bad H_q / L_q / L_cur");
  // The per-channel-key kernels split only bf16 inputs; this size covers both of them (the
  // tensor-core one serves correct <= 1, the CUDA-core one the rest; fp32 inputs ignore it).
  int n = attention_splits(cache, H_q, L_q);
  if (cache->key_block) {
    n = channel_splits(cache, H_q, L_q, false);
    if (chan_tc_serves(cache->d, 0, 0)) n = std::max(n, channel_splits(cache, H_q, L_q, true));
  }
  *bytes = split_workspace_bytes(cache, H_q, L_q, n);
  return QKV_OK;
}

QKV_API qkv_status corrected_attention(const void* Q, int32_t dtype, int32_t H_q, int64_t L_q,
                                       const qkv_cache* cache, const void* K_cur,
                                       const void* V_cur, int64_t L_cur, int32_t correct,
                                       int32_t causal_cur, float scale, void* O, float* LSE,
                                       void* workspace, size_t workspace_bytes, void* stream) {
  t_last_error.clear();
  qkv_status s = check_cache(cache);
  if (s != QKV_OK) return s;
  if (!in_dtype_ok(dtype)) return fail(QKV_ERR_UNSUPPORTED, "dtype must be F32 or BF16");
  if (H_q < 1 || H_q % cache->H_kv)
    return fail(QKV_ERR_INVALID_ARG, "H_q %d must be a positive multiple of H_kv %d", H_q,
                cache->H_kv);
  if (L_q < 0 || L_cur < 0) return fail(QKV_ERR_INVALID_ARG, "negative length");
  if (correct < 0 || correct > 2) return fail(QKV_ERR_UNSUPPORTED, "correct must be 0, 1 or 2");
  if (causal_cur != 0 && causal_cur != 1) return fail(QKV_ERR_INVALID_ARG, "causal_cur must be 0 or 1");
  if (L_cur == 0 && cache->length == 0) return fail(QKV_ERR_INVALID_ARG, "no keys: empty cache and L_cur = 0");
  if (!(std::isfinite(scale))) return fail(QKV_ERR_INVALID_ARG, "scale is not finite");
  if (L_q == 0) return QKV_OK;
  if (!Q || !O || !LSE) return fail(QKV_ERR_INVALID_ARG, "Q, O or LSE is NULL");
  if (L_cur > 0 && (!K_cur || !V_cur)) return fail(QKV_ERR_INVALID_ARG, "K_cur or V_cur is NULL");
  if (!aligned16(Q) || !aligned16(O) || !aligned16(LSE) || (L_cur > 0 && (!aligned16(K_cur) || !aligned16(V_cur))))
    return fail(QKV_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
  const int64_t rows = static_cast<int64_t>(H_q / cache->H_kv) * L_q;
  if ((rows + 127) / 128 > 2147483647LL || static_cast<int64_t>(cache->B) * cache->H_kv > 65535)
    return fail(QKV_ERR_UNSUPPORTED, "grid too large");
  cudaError_t e;
  int* status = status_word(&e);
  if (!status) return cuda_fail(e, "device status word");
  const float sc = scale > 0.f ? scale : 1.0f / std::sqrt(static_cast<float>(cache->d));
  const float log2e = 1.4426950408889634f;
  AttnParams p;
  p.Q = Q; p.K_cur = K_cur; p.V_cur = V_cur; p.O = O; p.LSE = LSE;
  p.k_codes = cache->k_codes; p.v_codes = cache->v_codes;
  p.k_meta = cache->k_meta; p.v_meta = cache->v_meta;
  p.status = status;
  p.Lq = L_q; p.Lc = cache->length; p.Lcur = L_cur; p.capacity = cache->capacity;
  p.B = cache->B; p.Hq = H_q; p.Hkv = cache->H_kv; p.r = H_q / cache->H_kv;
  p.group = cache->group; p.n_groups = cache->d / cache->group;
  p.correct = correct; p.causal = causal_cur;
  p.in_f32 = dtype == QKV_F32; p.meta_f16 = cache->meta_dtype == QKV_F16;
  p.scale_log2 = sc * log2e;
  p.wcoef_log2 = sc * sc / 24.0f * log2e;
  p.inv_scale_log2 = 1.0f / (sc * log2e);
  p.ucoef_log2 = correct == 2 ? sc * sc * sc * sc / 2880.0f * log2e : 0.0f;
  p.n_split = 1;
  p.rows_all = static_cast<int64_t>(cache->B) * H_q * L_q;
  p.ws_o = nullptr;
  p.ws_lse = nullptr;
  p.wait_limit = g_wait_limit.load(std::memory_order_relaxed);
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cache->key_block) {
    // bf16 inputs split the cached keys when the caller gave the workspace for it.
    const bool tc = chan_tc_serves(cache->d, dtype == QKV_F32, correct);
    const int n = dtype == QKV_BF16 ? channel_splits(cache, H_q, L_q, tc) : 1;
    const size_t need = split_workspace_bytes(cache, H_q, L_q, n);
    if (n > 1 && workspace && workspace_bytes >= need && aligned16(workspace)) {
      p.n_split = n;
      p.ws_o = static_cast<float*>(workspace);
      p.ws_lse = p.ws_o + static_cast<size_t>(n) * p.rows_all * cache->d;
    }
    e = launch_attention_channel(p, cache->d, cache->bits, cache->key_block, st);
    if (e != cudaSuccess) return cuda_fail(e, "corrected_attention launch");
    if (p.n_split > 1) {
      e = launch_split_merge(p.ws_o, p.ws_lse, p.n_split, p.rows_all, cache->d, O, LSE, st);
      if (e != cudaSuccess) return cuda_fail(e, "corrected_attention merge launch");
    }
    return QKV_OK;
  }
  if (dtype == QKV_F32) {
    e = launch_attention_f32(p, cache->d, cache->bits, st);
    if (e != cudaSuccess) return cuda_fail(e, "corrected_attention launch");
    return QKV_OK;
  }
  // Split over the cached keys when the caller gave the workspace for it; without it the same
  // result comes from the unsplit kernel.
  const int n = attention_splits(cache, H_q, L_q);
  const size_t need = split_workspace_bytes(cache, H_q, L_q, n);
  if (n > 1 && workspace && workspace_bytes >= need && aligned16(workspace)) {
    p.n_split = n;
    p.ws_o = static_cast<float*>(workspace);
    p.ws_lse = p.ws_o + static_cast<size_t>(n) * p.rows_all * cache->d;
  }
  e = launch_attention_bf16(p, cache->d, cache->bits, st);
  if (e != cudaSuccess) return cuda_fail(e, "corrected_attention launch");
  if (p.n_split > 1) {
    e = launch_split_merge(p.ws_o, p.ws_lse, p.n_split, p.rows_all, cache->d, O, LSE, st);
    if (e != cudaSuccess) return cuda_fail(e, "corrected_attention merge launch");
  }
  return QKV_OK;
}

QKV_API qkv_status qkv_jensen_bias(const void* Q, int32_t dtype, int32_t H_q, int64_t L_q,
                                   const qkv_cache* cache, float scale, float* bias, void* stream) {
  t_last_error.clear();
  qkv_status s = check_cache(cache);
  if (s != QKV_OK) return s;
  if (!in_dtype_ok(dtype)) return fail(QKV_ERR_UNSUPPORTED, "dtype must be F32 or BF16");
  if (H_q < 1 || H_q % cache->H_kv) return fail(QKV_ERR_INVALID_ARG, "bad H_q");
  if (L_q < 0) return fail(QKV_ERR_INVALID_ARG, "negative L_q");
  if (!(std::isfinite(scale))) return fail(QKV_ERR_INVALID_ARG, "scale is not finite");
  if (L_q == 0 || cache->length == 0) return QKV_OK;
  if (!Q || !bias) return fail(QKV_ERR_INVALID_ARG, "Q or bias is NULL");
  if (!aligned16(Q) || !aligned16(bias)) return fail(QKV_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
  if ((cache->length + 255) / 256 > 65535 ||
      static_cast<int64_t>(cache->B) * H_q * L_q > 2147483647LL)
    return fail(QKV_ERR_UNSUPPORTED, "bias grid too large");
  const float sc = scale > 0.f ? scale : 1.0f / std::sqrt(static_cast<float>(cache->d));
  BiasParams p;
  p.Q = Q; p.k_meta = cache->k_meta; p.bias = bias;
  p.Lq = L_q; p.Lc = cache->length; p.capacity = cache->capacity;
  p.B = cache->B; p.Hq = H_q; p.Hkv = cache->H_kv; p.r = H_q / cache->H_kv;
  p.d = cache->d; p.group = cache->group; p.n_groups = cache->d / cache->group;
  p.in_f32 = dtype == QKV_F32; p.meta_f16 = cache->meta_dtype == QKV_F16;
  p.wcoef = sc * sc / 24.0f;
  cudaError_t e = cache->key_block
                      ? launch_jensen_bias_channel(p, cache->key_block, static_cast<cudaStream_t>(stream))
                      : launch_jensen_bias(p, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "qkv_jensen_bias launch");
  return QKV_OK;
}

QKV_API qkv_status attention_fidelity(const void* Q, int32_t dtype, int32_t H_q, int64_t L_q,
                                      const qkv_cache* cache, const void* K_ref, const void* K_cur,
                                      int64_t L_cur, int32_t correct, int32_t causal_cur, float scale,
                                      float* stats, int32_t* top, void* stream) {
  t_last_error.clear();
  qkv_status s = check_cache(cache);
  if (s != QKV_OK) return s;
  if (!in_dtype_ok(dtype)) return fail(QKV_ERR_UNSUPPORTED, "dtype must be F32 or BF16");
  if (H_q < 1 || H_q % cache->H_kv)
    return fail(QKV_ERR_INVALID_ARG, "H_q %d must be a positive multiple of H_kv %d", H_q,
                cache->H_kv);
  if (L_q < 0 || L_cur < 0) return fail(QKV_ERR_INVALID_ARG, "negative length");
  if (correct < 0 || correct > 2) return fail(QKV_ERR_UNSUPPORTED, "correct must be 0, 1 or 2");
  if (causal_cur != 0 && causal_cur != 1) return fail(QKV_ERR_INVALID_ARG, "causal_cur must be 0 or 1");
  if (L_cur == 0 && cache->length == 0) return fail(QKV_ERR_INVALID_ARG, "no keys: empty cache and L_cur = 0");
  if (cache->length + L_cur >= 2147483647LL)
    return fail(QKV_ERR_UNSUPPORTED, "length + L_cur must be below 2^31 - 1");
  if (!(std::isfinite(scale))) return fail(QKV_ERR_INVALID_ARG, "scale is not finite");
  if (L_q == 0) return QKV_OK;
  if (!Q || !stats) return fail(QKV_ERR_INVALID_ARG, "Q or stats is NULL");
  if (cache->length > 0 && !K_ref) return fail(QKV_ERR_INVALID_ARG, "K_ref is NULL");
  if (L_cur > 0 && !K_cur) return fail(QKV_ERR_INVALID_ARG, "K_cur is NULL");
  if (!aligned16(Q) || !aligned16(stats) || (top && !aligned16(top)) ||
      (cache->length > 0 && !aligned16(K_ref)) || (L_cur > 0 && !aligned16(K_cur)))
    return fail(QKV_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
  const int64_t rows = static_cast<int64_t>(H_q / cache->H_kv) * L_q;
  const int rpc = fidelity_rows_per_cta();
  if ((rows + rpc - 1) / rpc > 2147483647LL || static_cast<int64_t>(cache->B) * cache->H_kv > 65535)
    return fail(QKV_ERR_UNSUPPORTED, "grid too large");
  const float sc = scale > 0.f ? scale : 1.0f / std::sqrt(static_cast<float>(cache->d));
  FidelityParams p;
  p.Q = Q; p.K_ref = K_ref; p.K_cur = K_cur;
  p.k_codes = cache->k_codes; p.k_meta = cache->k_meta;
  p.stats = stats; p.top = top;
  p.Lq = L_q; p.Lc = cache->length; p.Lcur = L_cur; p.capacity = cache->capacity;
  p.B = cache->B; p.Hq = H_q; p.Hkv = cache->H_kv; p.r = H_q / cache->H_kv;
  p.bits = cache->bits; p.group = cache->group; p.n_groups = cache->d / cache->group;
  p.key_block = cache->key_block;
  p.correct = correct; p.causal = causal_cur;
  p.in_f32 = dtype == QKV_F32; p.meta_f16 = cache->meta_dtype == QKV_F16;
  p.scale = sc;
  p.wcoef = sc * sc / 24.0f;
  p.ucoef = correct == 2 ? sc * sc * sc * sc / 2880.0f : 0.0f;
  cudaError_t e = launch_attention_fidelity(p, cache->d, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "attention_fidelity launch");
  return QKV_OK;
}

QKV_API qkv_status qkv_set_wait_limit(int64_t cycles, int64_t* previous) {
  t_last_error.clear();
  if (cycles < 0) return fail(QKV_ERR_INVALID_ARG, "wait limit must be >= 0 (0 restores the default)");
  const long long v = cycles == 0 ? kDefaultWaitLimitCycles : static_cast<long long>(cycles);
  const long long old = g_wait_limit.exchange(v, std::memory_order_relaxed);
  if (previous) *previous = old;
  return QKV_OK;
}

QKV_API qkv_status qkv_device_status(int32_t reset, int32_t* code) {
  t_last_error.clear();
  if (!code) return fail(QKV_ERR_INVALID_ARG, "NULL output");
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "synchronise");
  int* addr = status_word(&e);
  if (!addr) return cuda_fail(e, "device status word");
  int v = 0;
  e = cudaMemcpy(&v, addr, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "read device status");
  if (reset && v != 0) {
    const int zero = 0;
    e = cudaMemcpy(addr, &zero, sizeof(int), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_fail(e, "reset device status");
  }
  *code = v;
  return QKV_OK;
}

// ------------------------------------------------------------------ allocation-free attention
// Some callers cannot allocate device memory at all: a host runtime whose device memory belongs to
// another allocator and forbids allocations outside it, or a service that must not allocate once
// it has started. For them corrected_attention_noalloc takes its key-split scratch from one
// fixed-size array that the library itself owns in device memory (a file-scope __device__ array,
// reserved on every GPU that loads the library until the process exits), so the call needs no
// workspace argument and allocates nothing.
//
// In host code the array's name is only a host-side stand-in, not a device address: a kernel given
// it would fault or, where the GPU can reach host memory, silently use the wrong memory. Its device
// address is therefore looked up with cudaGetSymbolAddress, with that device current, on the entry
// point's first call on the device that needs the scratch (and again if the device's context has
// been re-created since), and passed to the kernels.
static constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;   // 8 MiB
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchBytes / sizeof(float)];

static SymbolAddressCache g_scratch_addr;

static float* noalloc_scratch(cudaError_t* err) {
  return static_cast<float*>(symbol_address(g_scratch_addr, g_noalloc_scratch, err));
}

QKV_API qkv_status corrected_attention_noalloc(const void* Q, int32_t dtype, int32_t H_q, int64_t L_q,
                                               const qkv_cache* cache, const void* K_cur,
                                               const void* V_cur, int64_t L_cur, int32_t correct,
                                               int32_t causal_cur, float scale, void* O, float* LSE,
                                               void* stream) {
  t_last_error.clear();
  qkv_status s = check_cache(cache);
  if (s != QKV_OK) return s;
  if (!in_dtype_ok(dtype)) return fail(QKV_ERR_UNSUPPORTED, "dtype must be F32 or BF16");
  if (H_q < 1 || H_q % cache->H_kv)
    return fail(QKV_ERR_INVALID_ARG, "H_q %d must be a positive multiple of H_kv %d", H_q,
                cache->H_kv);
  if (L_q < 0 || L_cur < 0) return fail(QKV_ERR_INVALID_ARG, "negative length");
  if (correct < 0 || correct > 2) return fail(QKV_ERR_UNSUPPORTED, "correct must be 0, 1 or 2");
  if (causal_cur != 0 && causal_cur != 1) return fail(QKV_ERR_INVALID_ARG, "causal_cur must be 0 or 1");
  if (L_cur == 0 && cache->length == 0) return fail(QKV_ERR_INVALID_ARG, "no keys: empty cache and L_cur = 0");
  if (!(std::isfinite(scale))) return fail(QKV_ERR_INVALID_ARG, "scale is not finite");
  if (L_q == 0) return QKV_OK;
  if (!Q || !O || !LSE) return fail(QKV_ERR_INVALID_ARG, "Q, O or LSE is NULL");
  if (L_cur > 0 && (!K_cur || !V_cur)) return fail(QKV_ERR_INVALID_ARG, "K_cur or V_cur is NULL");
  if (!aligned16(Q) || !aligned16(O) || !aligned16(LSE) || (L_cur > 0 && (!aligned16(K_cur) || !aligned16(V_cur))))
    return fail(QKV_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
  const int64_t rows = static_cast<int64_t>(H_q / cache->H_kv) * L_q;
  if ((rows + 127) / 128 > 2147483647LL || static_cast<int64_t>(cache->B) * cache->H_kv > 65535)
    return fail(QKV_ERR_UNSUPPORTED, "grid too large");
  // The key split this shape takes, cut down to as many splits as the library's array holds the
  // partials of; fewer than two run unsplit (the same result, with fewer CTAs sharing the reads).
  int n = dtype == QKV_BF16 && !cache->key_block ? attention_splits(cache, H_q, L_q) : 1;
  if (n > 1) {
    const size_t per_split = split_workspace_bytes(cache, H_q, L_q, 2) / 2;
    const size_t fit = kNoAllocScratchBytes / per_split;
    if (fit < static_cast<size_t>(n)) n = fit >= 2 ? static_cast<int>(fit) : 1;
  }
  cudaError_t e;
  int* status = status_word(&e);
  if (!status) return cuda_fail(e, "device status word");
  float* scratch = nullptr;
  if (n > 1) {
    scratch = noalloc_scratch(&e);
    if (!scratch) return cuda_fail(e, "address of the static scratch");
  }
  const float sc = scale > 0.f ? scale : 1.0f / std::sqrt(static_cast<float>(cache->d));
  const float log2e = 1.4426950408889634f;
  AttnParams p;
  p.Q = Q; p.K_cur = K_cur; p.V_cur = V_cur; p.O = O; p.LSE = LSE;
  p.k_codes = cache->k_codes; p.v_codes = cache->v_codes;
  p.k_meta = cache->k_meta; p.v_meta = cache->v_meta;
  p.status = status;
  p.Lq = L_q; p.Lc = cache->length; p.Lcur = L_cur; p.capacity = cache->capacity;
  p.B = cache->B; p.Hq = H_q; p.Hkv = cache->H_kv; p.r = H_q / cache->H_kv;
  p.group = cache->group; p.n_groups = cache->d / cache->group;
  p.correct = correct; p.causal = causal_cur;
  p.in_f32 = dtype == QKV_F32; p.meta_f16 = cache->meta_dtype == QKV_F16;
  p.scale_log2 = sc * log2e;
  p.wcoef_log2 = sc * sc / 24.0f * log2e;
  p.inv_scale_log2 = 1.0f / (sc * log2e);
  p.ucoef_log2 = correct == 2 ? sc * sc * sc * sc / 2880.0f * log2e : 0.0f;
  p.n_split = n;
  p.rows_all = static_cast<int64_t>(cache->B) * H_q * L_q;
  p.ws_o = scratch;
  p.ws_lse = scratch ? scratch + static_cast<size_t>(n) * p.rows_all * cache->d : nullptr;
  p.wait_limit = g_wait_limit.load(std::memory_order_relaxed);
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  e = cache->key_block ? launch_attention_channel(p, cache->d, cache->bits, cache->key_block, st)
      : dtype == QKV_F32 ? launch_attention_f32(p, cache->d, cache->bits, st)
                         : launch_attention_bf16(p, cache->d, cache->bits, st);
  if (e != cudaSuccess) return cuda_fail(e, "corrected_attention_noalloc launch");
  if (n > 1) {
    e = launch_split_merge(p.ws_o, p.ws_lse, n, p.rows_all, cache->d, O, LSE, st);
    if (e != cudaSuccess) return cuda_fail(e, "corrected_attention_noalloc merge launch");
  }
  return QKV_OK;
}
