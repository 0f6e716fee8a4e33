/*
 * qkv.h — C ABI of libqkv: a low-bit (INT2/INT4) group-quantised KV cache and
 * Jensen-bias-corrected chunk-wise attention over it, for NVIDIA B200 (sm_100a).
 *
 * Method: "Quantized Keys Steal Attention: Bias Correction for KV-Cache Compression
 * in Video Diffusion" (Tuncer, Becker, Pfeil), as summarised on agents-report.net
 * ("KV-Cache 量化導致的 Jensen 偏差：以每分數校正恢復影片擴散品質") and in the abstract on
 * fugumt.com. The current chunk's queries attend over the quantised cache of the previous
 * chunks plus the unquantised current chunk; every cached-key score has the correction
 * b = (1/(24 d)) sum_c q_c^2 Delta_c^2 subtracted before the softmax (summary, section 方法).
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller, 16-byte aligned, contiguous
 *    row-major. The library never allocates, frees or synchronises: work is enqueued on the
 *    caller's CUDA stream (`stream` is a cudaStream_t; NULL means the legacy default stream).
 *  - Arguments are validated on the host before anything is enqueued. A rejected call returns
 *    QKV_ERR_INVALID_ARG, QKV_ERR_UNSUPPORTED or QKV_ERR_CAPACITY and changes nothing.
 *  - A launch failure returns QKV_ERR_CUDA. qkv_last_error() gives a message (per host thread).
 *  - Kernels bound every internal wait. A wait that runs out sets a word in device memory and
 *    the kernel returns early; qkv_device_status() reads that word (it synchronises the device).
 *  - There is no CPU fallback and no other backend: every combination that is not compiled
 *    returns QKV_ERR_UNSUPPORTED.
 *  - Calls that touch the same cache must be ordered by the caller (e.g. one stream).
 */
#ifndef QKV_H
#define QKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define QKV_ABI_VERSION 2
/* Tokens per cache tile; a cache's capacity must be a multiple of it. */
#define QKV_CACHE_TILE 128

typedef enum {
  QKV_OK = 0,
  QKV_ERR_INVALID_ARG = -1, /* null/misaligned pointer, bad size or shape */
  QKV_ERR_UNSUPPORTED = -2, /* valid request that no compiled kernel serves */
  QKV_ERR_CAPACITY = -3,    /* append would exceed the cache capacity */
  QKV_ERR_CUDA = -4,        /* CUDA runtime or launch error */
  QKV_ERR_TIMEOUT = -5      /* a kernel's bounded wait ran out (from qkv_device_status) */
} qkv_status;

typedef enum { QKV_F32 = 0, QKV_BF16 = 1, QKV_F16 = 2 } qkv_dtype;

/*
 * Packed KV cache (plain descriptor; the caller owns all four buffers).
 *
 * Quantiser (summary, section 問題 "INT4/INT2 integer quantisation"; abstract "quantisation step
 * sizes"): for each (batch b, KV head h, token t) and each group g of `group` consecutive
 * channels, asymmetric min-max: step = (max - min) / (2^bits - 1) and zero-point = min, both in
 * IEEE fp32, then stored in `meta_dtype` (round to nearest even). Codes are taken against the
 * STORED values: code = clamp(rint((x - zp) * (1/step)), 0, 2^bits - 1), each operation one
 * correctly rounded fp32 operation, ties to even; a zero step gives code 0.
 *
 *  k_codes, v_codes : uint8 [B][H_kv][capacity][d*bits/8]; channel c of a token at bit c*bits of
 *                     the row's little-endian bit string (byte c*bits/8, bit c*bits%8).
 *  k_meta, v_meta   : meta_dtype [B][H_kv][capacity][d/group][2]; element 0 = step, 1 = zero-point.
 *  length           : tokens currently held per (b, h) (positions 0..length-1 are valid).
 *  capacity         : tokens the buffers hold per (b, h); a positive multiple of QKV_CACHE_TILE.
 * Supported: d in {64, 128}; bits in {2, 4}; group in {32, 64, 128} dividing d;
 * meta_dtype in {QKV_F32, QKV_F16}.
 *
 * key_block = T in {32, 64, 128} selects per-channel keys along tokens instead (KIVI's key
 * grouping, named in the summary's section 跨主題對比分析; the hotelren.com blog, section 3.1, groups
 * along the sequence axis): the T cache positions [k T, (k+1) T) of one channel share one step and
 * zero-point, computed over those tokens with the arithmetic above; codes are packed per token as
 * above; values keep per-token groups.
 *  k_meta (key_block = T) : meta_dtype [B][H_kv][capacity / T][d][2].
 * Every append must then start at a multiple of T (an append may end inside a block; that block's
 * meta comes from the tokens appended), and the correction uses each key's per-channel steps.
 * key_block = 0 is the per-token layout; zero-initialise the field (and `reserved`).
 */
typedef struct {
  int32_t B, H_kv, d, bits, group;
  int32_t meta_dtype;
  int64_t capacity;
  int64_t length;
  uint8_t* k_codes;
  uint8_t* v_codes;
  void* k_meta;
  void* v_meta;
  int32_t key_block;
  int32_t reserved;
} qkv_cache;

/*
 * Bytes of each of the four buffers of the cache described by `shape` (its shape fields and
 * key_block; pointers and length are ignored). Host only.
 */
qkv_status qkv_cache_layout_bytes(const qkv_cache* shape, size_t* k_codes_bytes, size_t* v_codes_bytes,
                                  size_t* k_meta_bytes, size_t* v_meta_bytes);

/* Bytes of ONE codes buffer and of ONE meta buffer for the per-token layout (host only). */
qkv_status qkv_cache_bytes(int32_t B, int32_t H_kv, int32_t d, int32_t bits, int32_t group,
                           int32_t meta_dtype, int64_t capacity, size_t* codes_bytes_each,
                           size_t* meta_bytes_each);

/*
 * Quantise a finished chunk and append it to the cache (QuantWM page on pchao.org, 方法概览:
 * each cache block is quantised once, after it is built).
 *  K, V     : in_dtype [B][H_kv][L_new][d] (QKV_F32 or QKV_BF16), device, 16-byte aligned.
 *  L_new    : tokens to append, >= 0 (0 is a no-op).
 * Writes codes and (step, zero-point) for positions length .. length+L_new-1 and, once the
 * kernel is enqueued, advances cache->length by L_new. Returns QKV_ERR_CAPACITY (and enqueues
 * nothing) if length + L_new > capacity.
 */
qkv_status kv_quantize_append(qkv_cache* cache, const void* K, const void* V, int32_t in_dtype,
                              int64_t L_new, void* stream);

/*
 * Device workspace with which corrected_attention splits the cached keys of each (batch, KV head)
 * over several CTAs (0 when the shape fills the GPU without a split). A split is chosen when the
 * query rows of a KV head fill few 128-row tiles (few query rows per KV head, e.g. decoding), so
 * that more SMs share the cache reads; its partial results, n_split * B * H_q * L_q * (d + 1) fp32
 * values, are then merged by a second kernel. The size depends on the GPU's SM count.
 */
qkv_status corrected_attention_workspace_bytes(const qkv_cache* cache, int32_t H_q, int64_t L_q,
                                               int64_t L_cur, size_t* bytes);

/*
 * Corrected chunk attention (summary, sections 方法 and 為何校正有效; scores q.k*scale as in the
 * QuantWM page, eq. (5)). For each query row, one softmax runs over the cache's first
 * cache->length keys followed by the L_cur current keys. Cached-key scores have the Jensen
 * correction subtracted when correct = 1:
 *     b_j = (scale^2 / 24) * sum_c q_c^2 * step_{j, c/group}^2   (= (1/(24 d)) ... at scale 1/sqrt(d)).
 *  Q            : dtype [B][H_q][L_q][d]; dtype QKV_F32 or QKV_BF16. H_q % H_kv == 0; query head
 *                 hq reads KV head hq / (H_q / H_kv).
 *  K_cur, V_cur : dtype [B][H_kv][L_cur][d], the unquantised current chunk (may be NULL if L_cur=0).
 *  correct      : 0 = plain attention over the dequantised cache, 1 = Taylor correction (the
 *                 summary's second-order form), 2 = the series of the exact correction
 *                 sum_c log(sinh(a_c)/a_c), a_c = scale*q_c*step/2, to fourth order:
 *                 b_j = sum_c (a_c^2/6 - a_c^4/180), i.e. the term above minus
 *                 (scale^4 / 2880) * sum_c q_c^4 * step_{j, c/group}^4.
 *  causal_cur   : 1 = query i sees current key j only if j <= i + (L_cur - L_q); the cache is
 *                 always fully visible.
 *  scale        : score scale; <= 0 means 1/sqrt(d).
 *  O            : dtype [B][H_q][L_q][d] (same type as Q). LSE: fp32 [B][H_q][L_q], natural log
 *                 of the row's softmax denominator (-inf and O = 0 for a row that sees no key).
 *  workspace    : device scratch of corrected_attention_workspace_bytes() bytes, 16-byte aligned,
 *                 owned by the caller; NULL (or too small) runs the same attention without the
 *                 key split. Calls on one stream may reuse it; concurrent calls need their own.
 * L_cur = 0 and cache->length = 0 together are rejected (no keys at all).
 * A cache with per-channel keys (key_block > 0) is served, for bf16 inputs with d = 128 and
 * correct <= 1, by a tensor-core kernel that dequantises the keys into bf16 high and low parts, and
 * otherwise (fp32 inputs, d = 64, correct = 2) by an fp32 CUDA-core kernel. With bf16 inputs both
 * split the cached keys over CTAs for decode-sized query chunks (when the unsplit grid would leave
 * more than half of the SMs idle) and then use the workspace the same way; fp32 inputs run unsplit
 * and ignore the workspace. corrected_attention_workspace_bytes() covers either kernel.
 */
qkv_status corrected_attention(const void* Q, int32_t dtype, int32_t H_q, int64_t L_q,
                               const qkv_cache* cache, const void* K_cur, const void* V_cur,
                               int64_t L_cur, int32_t correct, int32_t causal_cur, float scale,
                               void* O, float* LSE, void* workspace, size_t workspace_bytes,
                               void* stream);

/*
 * corrected_attention for callers that cannot allocate device memory. (The pages have no
 * counterpart: this is an interface of this library.) Same arguments and results as
 * corrected_attention, without the workspace: when the shape splits its cached keys, the partial
 * results go to a scratch array that the library itself holds in device memory, 8 MiB on every GPU
 * that loads the library, kept until the process exits. No call allocates or frees memory.
 *  - A shape whose split needs more than 8 MiB of scratch (corrected_attention_workspace_bytes()
 *    larger than 8 MiB) splits its cached keys fewer ways, as many as the 8 MiB hold the partials
 *    of, or runs unsplit when fewer than two fit: the results are the same, only the number of
 *    CTAs that share the cache reads differs. Caches with per-channel keys (key_block > 0) run
 *    unsplit here and need no scratch.
 *  - The first call on a device that needs the scratch looks up the array's device address (with
 *    that device current), and looks it up again after the device's context has been re-created
 *    (e.g. after cudaDeviceReset); make that first call before any stream capture.
 *  - All calls share the one array: every value a call reads from it was written by the same call,
 *    but two calls that overlap on the GPU (different streams, or different host threads) race on
 *    it and must be serialised by the caller.
 */
qkv_status corrected_attention_noalloc(const void* Q, int32_t dtype, int32_t H_q, int64_t L_q,
                                       const qkv_cache* cache, const void* K_cur, const void* V_cur,
                                       int64_t L_cur, int32_t correct, int32_t causal_cur, float scale,
                                       void* O, float* LSE, void* stream);

/*
 * The correction term alone, for checking: bias fp32 [B][H_q][L_q][cache->length] with
 * bias[b][hq][i][j] = (scale^2/24) * sum_c Q[b][hq][i][c]^2 * step_{j, c/group}^2, computed by
 * the same device functions corrected_attention uses (fp32). With per-channel keys (key_block > 0)
 * step_{j,c} is the step of channel c in key j's block.
 */
qkv_status qkv_jensen_bias(const void* Q, int32_t dtype, int32_t H_q, int64_t L_q,
                           const qkv_cache* cache, float scale, float* bias, void* stream);

/*
 * Attention-fidelity diagnostics: per query row, how far the corrected softmax over the quantised
 * cache is from the softmax over the same keys before quantisation.
 *   Token drift: pchao.org, "QuantWM：保住时间一致性的两比特键值缓存量化", section 实验如何设计
 *   (share of positions whose top-1 attended token differs from the BF16 one).
 *   KL and top-5 recall: gist.science, "Statistical Inference and Quality Measures of KV Cache
 *   Quantisations Inspired by TurboQuant", section Métricas de Avaliação.
 *   Cached mass: agents-report.net, "KV-Cache 量化導致的 Jensen 偏差", section 為何校正有效.
 * P_ref is the softmax of scale * q.k over [K_ref ; K_cur]; P_q is corrected_attention's softmax
 * (the same Q, cache, K_cur, correct, causal_cur and scale). V is not involved.
 *  K_ref  : dtype [B][H_kv][cache->length][d], the cached keys as they were before quantisation
 *           (may be NULL when cache->length = 0).
 *  stats  : fp32 [B][H_q][L_q][8] = { LSE_ref, LSE_q, cached mass under P_ref, cached mass under
 *           P_q, KL(P_ref || P_q), top-1 agreement (1 or 0), top-5 recall, 0 }. A row that sees no
 *           key gets LSE -inf, masses and KL 0, agreement and recall 1.
 *  top    : int32 [B][H_q][L_q][2][5] or NULL: the five highest-scoring keys of P_ref, then of
 *           P_q, highest first, the lower index first on equal scores; key j < length is cached
 *           key j, length + t is current key t; -1 pads rows that see fewer than 5 keys. Recall
 *           counts the reference list's keys found in the quantised list, over min(5, keys seen).
 * Every score is fp32 (CUDA cores). Pointers are device pointers, 16-byte aligned, caller-owned;
 * nothing is allocated. length + L_cur must be below 2^31 - 1. Caches with per-channel keys
 * (key_block > 0) are supported. Errors as corrected_attention.
 */
qkv_status attention_fidelity(const void* Q, int32_t dtype, int32_t H_q, int64_t L_q,
                              const qkv_cache* cache, const void* K_ref, const void* K_cur,
                              int64_t L_cur, int32_t correct, int32_t causal_cur, float scale,
                              float* stats, int32_t* top, void* stream);

/*
 * Bound of every internal wait of the kernels launched from now on by this process, in SM clock
 * cycles (default 2e9, about a second; 0 restores the default); *previous (if not NULL) receives
 * the bound in force before. For tests of the timeout path: with a bound of a few cycles the
 * attention kernel's waits give up at once, the kernel returns early with its outputs undefined,
 * and qkv_device_status() reports QKV_ERR_TIMEOUT. The waits on the way out of a kernel (for its
 * own copies and tensor-core operations in flight) keep the default bound. Host only.
 */
qkv_status qkv_set_wait_limit(int64_t cycles, int64_t* previous);

/*
 * Reads the library's device status word (0 = no error, else a qkv_status such as
 * QKV_ERR_TIMEOUT) into *code; clears it when reset != 0. Synchronises the current device.
 */
qkv_status qkv_device_status(int32_t reset, int32_t* code);

const char* qkv_status_string(int32_t status);
/* Message of the last failed call on this host thread ("" if none). */
const char* qkv_last_error(void);
int32_t qkv_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* QKV_H */
