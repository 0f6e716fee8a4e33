// fp32-input corrected attention on CUDA cores, and the correction term alone.
//
// Tensor cores have no fp32 mode, and rounding fp32 queries or keys to bf16 moves the
// log-sum-exp by ~1e-2, so fp32 inputs take this CUDA-core path: every score, exponential and
// accumulation is fp32. Same method as the bf16 kernel (agents-report.net, "KV-Cache 量化導致的
// Jensen 偏差", sections 方法 / 為何校正有效): scores q . x_hat * scale over the dequantised cache
// minus the Jensen term b, then over the current chunk, one online softmax, O and LSE.
//
// One CTA of 128 threads per (128 packed query rows, batch * KV head); one thread per query row.
// Keys are staged 32 at a time in shared memory as fp32 (cached keys dequantised with one fp32
// FMA, zp + step * code), and every thread walks them in order.
//
// The same kernel serves caches whose keys are quantised per channel along tokens (KIVI's key
// grouping, agents-report.net, section 跨主題對比分析; hotelren.com blog, section 3.1): every T
// cache positions of a channel share one step. There the correction of [JB] 方法,
// (scale^2 / 24) sum_c q_c^2 Delta_{j,c}^2, is the same for all keys of a block, so it is taken once
// per row and 32-key tile (T is a multiple of 32) from the block's squared steps; inputs may be
// bf16 or fp32 and O has the input type.
#include <cuda_bf16.h>

#include "channel.h"
#include "qkv_common.cuh"
#include "qkv_internal.h"
#include "qkv_jensen.cuh"

namespace qkv {
namespace {

constexpr int kRows = 128;
constexpr int kKT = 32;         // keys per shared-memory tile

__device__ __forceinline__ int code_at(const uint8_t* row, int c, int bits) {
  const int bit = c * bits;
  return (row[bit >> 3] >> (bit & 7)) & ((1 << bits) - 1);
}

template <bool kF32In>
__device__ __forceinline__ float ld_in(const void* base, int64_t i) {
  if (kF32In) return static_cast<const float*>(base)[i];
  return __bfloat162float(static_cast<const __nv_bfloat16*>(base)[i]);
}

// kChan: keys quantised per channel over blocks of T positions (meta [BH][capacity/T][D][2]);
// otherwise per token in groups of p.group channels. kF32In: Q, K_cur, V_cur and O are fp32 (else bf16).
template <int D, bool kChan, bool kF32In>
__global__ void __launch_bounds__(kRows) attention_f32_kernel(const AttnParams p, int bits, int T) {
  extern __shared__ float sm[];
  float* q_s = sm;                              // [128][D + 1]
  float* k_s = q_s + kRows * (D + 1);           // [kKT][D]
  float* v_s = k_s + kKT * D;                   // [kKT][D]
  float* d2_s = v_s + kKT * D;                  // [kKT][4]; per-channel keys: [D] squared steps
  const int t = threadIdx.x;
  const int m_tile = blockIdx.x;
  const int bh = blockIdx.y;
  const int b = bh / p.Hkv;
  const int h = bh - b * p.Hkv;
  const int64_t rows_total = static_cast<int64_t>(p.r) * p.Lq;
  const int64_t R = static_cast<int64_t>(m_tile) * kRows + t;
  const bool valid_row = R < rows_total;
  const int64_t hq = static_cast<int64_t>(h) * p.r + (valid_row ? R / p.Lq : 0);
  const int64_t qi = valid_row ? R % p.Lq : 0;
  const int64_t out_row = (static_cast<int64_t>(b) * p.Hq + hq) * p.Lq + qi;
  const float scale = p.scale_log2 * 0.69314718055994530942f;   // natural units here
  const float wcoef = p.wcoef_log2 * 0.69314718055994530942f;
  const int G = p.group, NG = p.n_groups;
  const int row_codes = D * bits / 8;

  const float ucoef = p.ucoef_log2 * 0.69314718055994530942f;
  float w[kMaxGroups] = {0.f, 0.f, 0.f, 0.f};
  float u[kMaxGroups] = {0.f, 0.f, 0.f, 0.f};
  const uint8_t* qrow = static_cast<const uint8_t*>(p.Q) + out_row * D * (kF32In ? 4 : 2);
  if (valid_row) {
    if (!kChan && p.correct) query_group_powers<D>(qrow, kF32In, G, wcoef, ucoef, w, u);
    for (int c = 0; c < D; ++c) q_s[t * (D + 1) + c] = ld_in<kF32In>(qrow, c);
  } else {
    for (int c = 0; c < D; ++c) q_s[t * (D + 1) + c] = 0.f;
  }
  float o[D];
#pragma unroll
  for (int c = 0; c < D; ++c) o[c] = 0.f;
  float m = -INFINITY, l = 0.f;
  const int64_t lim_cur = p.causal ? qi + (p.Lcur - p.Lq) + 1 : p.Lcur;   // current keys this row sees

  // Keys [k_begin, total) of this CTA. With a split over the cached keys (n_split > 1, grid z),
  // split z takes the 32-key cached tiles [z T / n, (z+1) T / n) and the last split also the
  // current chunk; the partial O (normalised) and LSE go to the workspace for the merge.
  int64_t k_begin = 0, total = p.Lc + p.Lcur;
  if (p.n_split > 1) {
    const int64_t tiles = (p.Lc + kKT - 1) / kKT;
    const int z = blockIdx.z;
    k_begin = tiles * z / p.n_split * kKT;
    if (z + 1 < p.n_split) total = tiles * (z + 1) / p.n_split * kKT;
  }
  for (int64_t k0 = k_begin; k0 < total; k0 += kKT) {
    __syncthreads();
    for (int e = t; e < kKT * D; e += kRows) {
      const int kk = e / D, c = e % D;
      const int64_t key = k0 + kk;
      float kv = 0.f, vv = 0.f;
      if (key < p.Lc) {
        const int64_t row = static_cast<int64_t>(bh) * p.capacity + key;
        const int g = c / G;
        // key meta: per (token, group), or per (block of T tokens, channel)
        const int64_t kmi = kChan ? ((static_cast<int64_t>(bh) * (p.capacity / T) + key / T) * D + c) * 2
                                  : (row * NG + g) * 2;
        float ks, kz, vs, vz;
        if (p.meta_f16) {
          const __half* km = static_cast<const __half*>(p.k_meta) + kmi;
          const __half* vm = static_cast<const __half*>(p.v_meta) + (row * NG + g) * 2;
          ks = __half2float(km[0]); kz = __half2float(km[1]);
          vs = __half2float(vm[0]); vz = __half2float(vm[1]);
        } else {
          const float* km = static_cast<const float*>(p.k_meta) + kmi;
          const float* vm = static_cast<const float*>(p.v_meta) + (row * NG + g) * 2;
          ks = km[0]; kz = km[1]; vs = vm[0]; vz = vm[1];
        }
        kv = fmaf(ks, static_cast<float>(code_at(p.k_codes + row * row_codes, c, bits)), kz);
        vv = fmaf(vs, static_cast<float>(code_at(p.v_codes + row * row_codes, c, bits)), vz);
        if (kChan) {
          if (kk == 0) d2_s[c] = ks * ks;        // the tile lies in one key block (T % 32 == 0)
        } else if (c % G == 0) {
          d2_s[kk * 4 + g] = ks * ks;
        }
      } else if (key < total) {
        const int64_t row = static_cast<int64_t>(bh) * p.Lcur + (key - p.Lc);
        kv = ld_in<kF32In>(p.K_cur, row * D + c);
        vv = ld_in<kF32In>(p.V_cur, row * D + c);
      }
      k_s[kk * D + c] = kv;
      v_s[kk * D + c] = vv;
    }
    __syncthreads();
    // Per-channel keys: the tile's correction for this row, sum_c w_c Delta_c^2 (minus the fourth-
    // order term sum_c u_c Delta_c^4 when correct = 2), one pass over the block's squared steps.
    float tile_b = 0.f;
    if (kChan && p.correct && k0 < p.Lc) {
      for (int c = 0; c < D; ++c) {
        const float q2 = q_s[t * (D + 1) + c] * q_s[t * (D + 1) + c];
        const float d2 = d2_s[c];
        tile_b = fmaf(wcoef * q2, d2, tile_b);
        if (p.correct == 2) tile_b = fmaf(-ucoef * (q2 * q2), d2 * d2, tile_b);
      }
    }
    for (int kk = 0; kk < kKT; ++kk) {
      const int64_t key = k0 + kk;
      if (key >= total) break;
      const bool cached = key < p.Lc;
      if (!cached && (key - p.Lc) >= lim_cur) continue;
      float s = 0.f;
      for (int c = 0; c < D; ++c) s = fmaf(q_s[t * (D + 1) + c], k_s[kk * D + c], s);
      s *= scale;
      if (kChan) {
        if (cached) s -= tile_b;
      } else if (cached && p.correct) {
        float d2[kMaxGroups] = {0.f, 0.f, 0.f, 0.f};
        for (int g = 0; g < NG; ++g) d2[g] = d2_s[kk * 4 + g];
        s -= jensen_term(w, d2, NG);
        if (p.correct == 2) {
          for (int g = 0; g < NG; ++g) s = fmaf(u[g], d2[g] * d2[g], s);
        }
      }
      if (s > m) {
        const float a = expf(m - s);       // 0 when m = -inf
        l *= a;
#pragma unroll
        for (int c = 0; c < D; ++c) o[c] *= a;
        m = s;
      }
      const float pk = expf(s - m);
      l += pk;
#pragma unroll
      for (int c = 0; c < D; ++c) o[c] = fmaf(pk, v_s[kk * D + c], o[c]);
    }
  }
  if (valid_row && p.n_split > 1) {
    const int64_t prow = static_cast<int64_t>(blockIdx.z) * p.rows_all + out_row;
    const float inv = l > 0.f ? 1.f / l : 0.f;
    float* orow = p.ws_o + prow * D;
#pragma unroll
    for (int c = 0; c < D; ++c) orow[c] = o[c] * inv;
    p.ws_lse[prow] = l > 0.f ? m + logf(l) : -INFINITY;
  } else if (valid_row) {
    const float inv = l > 0.f ? 1.f / l : 0.f;
    if (kF32In) {
      float* orow = static_cast<float*>(p.O) + out_row * D;
#pragma unroll
      for (int c = 0; c < D; ++c) orow[c] = o[c] * inv;
    } else {
      __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.O) + out_row * D;
#pragma unroll
      for (int c = 0; c < D; ++c) orow[c] = __float2bfloat16_rn(o[c] * inv);
    }
    p.LSE[out_row] = l > 0.f ? m + logf(l) : -INFINITY;
  }
}

// Correction term alone: bias[b][hq][i][j] with the same device functions as the attention.
template <int D>
__global__ void __launch_bounds__(256) jensen_bias_kernel(const BiasParams p) {
  const int64_t qrow = blockIdx.x;                          // over B * Hq * Lq
  const int64_t j = static_cast<int64_t>(blockIdx.y) * blockDim.x + threadIdx.x;
  if (j >= p.Lc) return;
  const int64_t bhq = qrow / p.Lq;
  const int64_t b = bhq / p.Hq, hq = bhq % p.Hq;
  const int64_t hkv = hq / p.r;
  const size_t esz = p.in_f32 ? 4 : 2;
  float w[kMaxGroups];
  query_group_weights<D>(static_cast<const uint8_t*>(p.Q) + qrow * D * esz, p.in_f32 != 0, p.group,
                         p.wcoef, w);
  const int64_t key = (b * p.Hkv + hkv) * p.capacity + j;
  float d2[kMaxGroups] = {0.f, 0.f, 0.f, 0.f};
  for (int g = 0; g < p.n_groups; ++g) {
    const float s = p.meta_f16
                        ? __half2float(static_cast<const __half*>(p.k_meta)[(key * p.n_groups + g) * 2])
                        : static_cast<const float*>(p.k_meta)[(key * p.n_groups + g) * 2];
    d2[g] = s * s;
  }
  p.bias[qrow * p.Lc + j] = jensen_term(w, d2, p.n_groups);
}

// Correction term alone for per-channel keys: b = (scale^2 / 24) sum_c q_c^2 Delta_{block(j), c}^2.
template <int D, bool kF32In>
__global__ void __launch_bounds__(256) jensen_bias_channel_kernel(const BiasParams p, int T) {
  const int64_t qrow = blockIdx.x;
  const int64_t j = static_cast<int64_t>(blockIdx.y) * blockDim.x + threadIdx.x;
  if (j >= p.Lc) return;
  const int64_t bhq = qrow / p.Lq;
  const int64_t b = bhq / p.Hq, hq = bhq % p.Hq;
  const int64_t hkv = hq / p.r;
  const int64_t blk = (b * p.Hkv + hkv) * (p.capacity / T) + j / T;
  float acc = 0.f;
  for (int c = 0; c < D; ++c) {
    const float q = ld_in<kF32In>(p.Q, qrow * D + c);
    const float s = p.meta_f16 ? __half2float(static_cast<const __half*>(p.k_meta)[(blk * D + c) * 2])
                               : static_cast<const float*>(p.k_meta)[(blk * D + c) * 2];
    acc = fmaf(p.wcoef * (q * q), s * s, acc);
  }
  p.bias[qrow * p.Lc + j] = acc;
}

template <int D, bool kChan, bool kF32In>
cudaError_t launch_f32(const AttnParams& p, int bits, int T, cudaStream_t stream) {
  const size_t smem = (kRows * (D + 1) + 2 * kKT * D + (kChan ? D : kKT * 4)) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(attention_f32_kernel<D, kChan, kF32In>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int64_t rows = static_cast<int64_t>(p.r) * p.Lq;
  dim3 grid(static_cast<unsigned>((rows + kRows - 1) / kRows), static_cast<unsigned>(p.B * p.Hkv),
            static_cast<unsigned>(p.n_split > 1 ? p.n_split : 1));
  attention_f32_kernel<D, kChan, kF32In><<<grid, kRows, smem, stream>>>(p, bits, T);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention_f32(const AttnParams& p, int d, int bits, cudaStream_t stream) {
  return d == 128 ? launch_f32<128, false, true>(p, bits, 0, stream)
                  : launch_f32<64, false, true>(p, bits, 0, stream);
}

int channel_rows_per_cta() { return kRows; }
int channel_tile_keys() { return kKT; }

cudaError_t launch_attention_channel(const AttnParams& p, int d, int bits, int T, cudaStream_t stream) {
  if (p.in_f32) {
    return d == 128 ? launch_f32<128, true, true>(p, bits, T, stream)
                    : launch_f32<64, true, true>(p, bits, T, stream);
  }
  return d == 128 ? launch_f32<128, true, false>(p, bits, T, stream)
                  : launch_f32<64, true, false>(p, bits, T, stream);
}

cudaError_t launch_jensen_bias_channel(const BiasParams& p, int T, cudaStream_t stream) {
  dim3 grid(static_cast<unsigned>(p.B * p.Hq * p.Lq), static_cast<unsigned>((p.Lc + 255) / 256));
  if (p.d == 128) {
    if (p.in_f32) jensen_bias_channel_kernel<128, true><<<grid, 256, 0, stream>>>(p, T);
    else jensen_bias_channel_kernel<128, false><<<grid, 256, 0, stream>>>(p, T);
  } else {
    if (p.in_f32) jensen_bias_channel_kernel<64, true><<<grid, 256, 0, stream>>>(p, T);
    else jensen_bias_channel_kernel<64, false><<<grid, 256, 0, stream>>>(p, T);
  }
  return cudaGetLastError();
}

cudaError_t launch_jensen_bias(const BiasParams& p, cudaStream_t stream) {
  dim3 grid(static_cast<unsigned>(p.B * p.Hq * p.Lq), static_cast<unsigned>((p.Lc + 255) / 256));
  if (p.d == 128) jensen_bias_kernel<128><<<grid, 256, 0, stream>>>(p);
  else jensen_bias_kernel<64><<<grid, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace qkv
