// fp32-input corrected attention on CUDA cores, and the correction term alone.
//
// Tensor cores have no fp32 mode, and rounding fp32 queries or keys to bf16 moves the
// log-sum-exp by ~1e-2, so fp32 inputs take this CUDA-core path: every score, exponential and
// accumulation is fp32. Same method as the bf16 kernel (agents-report.net, "KV-Cache 量化導致的
// Jensen 偏差", sections 方法 / 為何校正有效): scores q . x_hat * scale over the dequantised cache
// minus the Jensen term b, then over the current chunk, one online softmax, O and LSE.
//
// One CTA of 256 threads per (128 packed query rows, batch * KV head); two threads per query row,
// one on the even and one on the odd keys of each tile. Keys are staged 32 at a time in shared
// memory as fp32 (cached keys dequantised with one fp32 FMA, zp + step * code); a row's q is read
// from shared memory in 16-byte pieces, keys and values as broadcasts, and the dot products and the
// P.V update use packed fp32x2 FMAs.
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
constexpr int kThreads = 2 * kRows;   // two threads per query row
constexpr int kKT = 32;         // keys per shared-memory tile

template <bool kF32In>
__device__ __forceinline__ float ld_in(const void* base, int64_t i) {
  if (kF32In) return static_cast<const float*>(base)[i];
  return __bfloat162float(static_cast<const __nv_bfloat16*>(base)[i]);
}

// Codes of 4 consecutive channels c4*4 .. c4*4+3 of a packed row.
__device__ __forceinline__ void codes4(const uint8_t* row, int c4, int bits, float (&c)[4]) {
  if (bits == 2) {
    const uint32_t v = row[c4];
    c[0] = static_cast<float>(v & 3u); c[1] = static_cast<float>((v >> 2) & 3u);
    c[2] = static_cast<float>((v >> 4) & 3u); c[3] = static_cast<float>(v >> 6);
  } else {
    const uint32_t v = *reinterpret_cast<const uint16_t*>(row + 2 * c4);
    c[0] = static_cast<float>(v & 15u); c[1] = static_cast<float>((v >> 4) & 15u);
    c[2] = static_cast<float>((v >> 8) & 15u); c[3] = static_cast<float>(v >> 12);
  }
}

template <bool kF32In>
__device__ __forceinline__ float4 ld_in4(const void* base, int64_t i) {
  if (kF32In) return *reinterpret_cast<const float4*>(static_cast<const float*>(base) + i);
  const uint2 u = *reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(base) + i);
  return make_float4(bf16_lo(u.x), bf16_hi(u.x), bf16_lo(u.y), bf16_hi(u.y));
}

// A cached key's score minus the correction from its per-group squared steps d2[g] (plus the
// fourth-order term u_g d2_g^2 when correct = 2).
__device__ __forceinline__ float corrected(float s, const float (&w)[kMaxGroups], const float (&u)[kMaxGroups],
                                           const float* d2s, int NG, int correct) {
  float d2[kMaxGroups] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int g = 0; g < kMaxGroups; ++g)
    if (g < NG) d2[g] = d2s[g];
  s -= jensen_term(w, d2, NG);
  if (correct == 2) {
#pragma unroll
    for (int g = 0; g < kMaxGroups; ++g)
      if (g < NG) s = fmaf(u[g], d2[g] * d2[g], s);
  }
  return s;
}

// kChan: keys quantised per channel over blocks of T positions (meta [BH][capacity/T][D][2]);
// otherwise per token in groups of p.group channels. kF32In: Q, K_cur, V_cur and O are fp32 (else bf16).
// Two threads per query row (threads t and t + 128): each takes the even or the odd keys of every
// 32-key tile with its own running max, sum and O, merged through shared memory at the end.
template <int D, bool kChan, bool kF32In>
__global__ void __launch_bounds__(kThreads) attention_f32_kernel(const AttnParams p, int bits, int T) {
  constexpr int kPitch = D + 4;                 // 16-byte rows; 8 lanes' rows hit distinct banks
  extern __shared__ float sm[];
  float* q_s = sm;                              // [128][kPitch]
  float* k_s = q_s + kRows * kPitch;            // [kKT][D]
  float* v_s = k_s + kKT * D;                   // [kKT][D]
  float* d2_s = v_s + kKT * D;                  // [kKT][4]; per-channel keys: [D] squared steps
  const int t = threadIdx.x;
  const int rt = t & (kRows - 1);               // row within the tile
  const int par = t / kRows;                    // key parity this thread takes
  const int bh = blockIdx.y;
  const int b = bh / p.Hkv;
  const int h = bh - b * p.Hkv;
  const int64_t rows_total = static_cast<int64_t>(p.r) * p.Lq;
  const int64_t R = static_cast<int64_t>(blockIdx.x) * kRows + rt;
  const bool valid_row = R < rows_total;
  const int64_t hq = static_cast<int64_t>(h) * p.r + (valid_row ? R / p.Lq : 0);
  const int64_t qi = valid_row ? R % p.Lq : 0;
  const int64_t out_row = (static_cast<int64_t>(b) * p.Hq + hq) * p.Lq + qi;
  const float scale = p.scale_log2 * 0.69314718055994530942f;   // natural units here
  const float wcoef = p.wcoef_log2 * 0.69314718055994530942f;
  const float ucoef = p.ucoef_log2 * 0.69314718055994530942f;
  const int G = p.group, NG = p.n_groups;
  const int row_codes = D * bits / 8;

  float w[kMaxGroups] = {0.f, 0.f, 0.f, 0.f};
  float u[kMaxGroups] = {0.f, 0.f, 0.f, 0.f};
  const uint8_t* qrow = static_cast<const uint8_t*>(p.Q) + out_row * D * (kF32In ? 4 : 2);
  if (!kChan && valid_row && p.correct) query_group_powers<D>(qrow, kF32In, G, wcoef, ucoef, w, u);
  // The row's q in shared memory: fp32, or for bf16 inputs as bf16 (exact), 8 channels per 16 bytes.
  if (par == 0) {
    if (kF32In) {
      for (int c4 = 0; c4 < D / 4; ++c4) {
        const float4 x = valid_row ? ld_in4<kF32In>(qrow, 4 * c4) : make_float4(0.f, 0.f, 0.f, 0.f);
        *reinterpret_cast<float4*>(q_s + rt * kPitch + 4 * c4) = x;
      }
    } else {
      for (int c8 = 0; c8 < D / 8; ++c8) {
        const uint4 v = valid_row ? reinterpret_cast<const uint4*>(qrow)[c8] : make_uint4(0u, 0u, 0u, 0u);
        reinterpret_cast<uint4*>(q_s + rt * kPitch)[c8] = v;
      }
    }
  }
  float2 o[D / 2];
#pragma unroll
  for (int c = 0; c < D / 2; ++c) o[c] = make_float2(0.f, 0.f);
  float m = -INFINITY, l = 0.f;
  const int64_t lim_cur = p.causal ? qi + (p.Lcur - p.Lq) + 1 : p.Lcur;   // current keys this row sees
  const float4* q4 = reinterpret_cast<const float4*>(q_s + rt * kPitch);      // fp32 q
  const uint4* qb8 = reinterpret_cast<const uint4*>(q_s + rt * kPitch);       // bf16 q

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
    for (int e = t; e < kKT * (D / 4); e += kThreads) {
      const int kk = e / (D / 4), c4 = e % (D / 4);
      const int64_t key = k0 + kk;
      float4 kv = make_float4(0.f, 0.f, 0.f, 0.f), vv = kv;
      if (key < p.Lc) {
        const int64_t row = static_cast<int64_t>(bh) * p.capacity + key;
        const int g = (4 * c4) / G;
        const int64_t vmi = (row * NG + g) * 2;
        float ks[4], kz[4], vs, vz;
        if (kChan) {
          const int64_t kmi = ((static_cast<int64_t>(bh) * (p.capacity / T) + key / T) * D + 4 * c4) * 2;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            if (p.meta_f16) {
              ks[i] = __half2float(static_cast<const __half*>(p.k_meta)[kmi + 2 * i]);
              kz[i] = __half2float(static_cast<const __half*>(p.k_meta)[kmi + 2 * i + 1]);
            } else {
              ks[i] = static_cast<const float*>(p.k_meta)[kmi + 2 * i];
              kz[i] = static_cast<const float*>(p.k_meta)[kmi + 2 * i + 1];
            }
          }
        } else {
          const int64_t kmi = (row * NG + g) * 2;
          float s0, z0;
          if (p.meta_f16) {
            s0 = __half2float(static_cast<const __half*>(p.k_meta)[kmi]);
            z0 = __half2float(static_cast<const __half*>(p.k_meta)[kmi + 1]);
          } else {
            s0 = static_cast<const float*>(p.k_meta)[kmi];
            z0 = static_cast<const float*>(p.k_meta)[kmi + 1];
          }
#pragma unroll
          for (int i = 0; i < 4; ++i) { ks[i] = s0; kz[i] = z0; }
        }
        if (p.meta_f16) {
          vs = __half2float(static_cast<const __half*>(p.v_meta)[vmi]);
          vz = __half2float(static_cast<const __half*>(p.v_meta)[vmi + 1]);
        } else {
          vs = static_cast<const float*>(p.v_meta)[vmi];
          vz = static_cast<const float*>(p.v_meta)[vmi + 1];
        }
        float kc[4], vc[4];
        codes4(p.k_codes + row * row_codes, c4, bits, kc);
        codes4(p.v_codes + row * row_codes, c4, bits, vc);
        kv = make_float4(fmaf(ks[0], kc[0], kz[0]), fmaf(ks[1], kc[1], kz[1]),
                         fmaf(ks[2], kc[2], kz[2]), fmaf(ks[3], kc[3], kz[3]));
        vv = make_float4(fmaf(vs, vc[0], vz), fmaf(vs, vc[1], vz), fmaf(vs, vc[2], vz), fmaf(vs, vc[3], vz));
        if (kChan) {
          if (kk == 0) {                          // the tile lies in one key block (T % 32 == 0)
#pragma unroll
            for (int i = 0; i < 4; ++i) d2_s[4 * c4 + i] = ks[i] * ks[i];
          }
        } else if ((4 * c4) % G == 0) {
          d2_s[kk * 4 + g] = ks[0] * ks[0];
        }
      } else if (key < total) {
        const int64_t row = static_cast<int64_t>(bh) * p.Lcur + (key - p.Lc);
        kv = ld_in4<kF32In>(p.K_cur, row * D + 4 * c4);
        vv = ld_in4<kF32In>(p.V_cur, row * D + 4 * c4);
      }
      *reinterpret_cast<float4*>(k_s + kk * D + 4 * c4) = kv;
      *reinterpret_cast<float4*>(v_s + kk * D + 4 * c4) = vv;
    }
    __syncthreads();
    // Per-channel keys: the tile's correction for this row, sum_c w_c Delta_c^2 (minus the fourth-
    // order term sum_c u_c Delta_c^4 when correct = 2), one pass over the block's squared steps.
    float tile_b = 0.f;
    if (kChan && p.correct && k0 < p.Lc) {
      float2 s2 = make_float2(0.f, 0.f), s4 = s2;
      const float4* d4 = reinterpret_cast<const float4*>(d2_s);
#pragma unroll
      for (int c4 = 0; c4 < D / 4; ++c4) {
        float4 x;
        if (kF32In) {
          x = q4[c4];
        } else {
          const uint2 u = reinterpret_cast<const uint2*>(qb8)[c4];
          x = make_float4(bf16_lo(u.x), bf16_hi(u.x), bf16_lo(u.y), bf16_hi(u.y));
        }
        const float4 d = d4[c4];
        const float2 t0 = __fmul2_rn(__fmul2_rn(make_float2(x.x, x.y), make_float2(x.x, x.y)), make_float2(d.x, d.y));
        const float2 t1 = __fmul2_rn(__fmul2_rn(make_float2(x.z, x.w), make_float2(x.z, x.w)), make_float2(d.z, d.w));
        s2 = __fadd2_rn(s2, __fadd2_rn(t0, t1));
        s4 = __ffma2_rn(t0, t0, __ffma2_rn(t1, t1, s4));
      }
      tile_b = wcoef * (s2.x + s2.y);
      if (p.correct == 2) tile_b = fmaf(-ucoef, s4.x + s4.y, tile_b);
    }
    for (int kk = par; kk < kKT; kk += 2) {
      const int64_t key = k0 + kk;
      if (key >= total) break;
      const bool cached = key < p.Lc;
      if (!cached && (key - p.Lc) >= lim_cur) continue;
      const float4* k4 = reinterpret_cast<const float4*>(k_s + kk * D);
      float2 a0 = make_float2(0.f, 0.f), a1 = a0;
      if (kF32In) {
#pragma unroll
        for (int c4 = 0; c4 < D / 4; ++c4) {
          const float4 x = q4[c4], y = k4[c4];
          a0 = __ffma2_rn(make_float2(x.x, x.y), make_float2(y.x, y.y), a0);
          a1 = __ffma2_rn(make_float2(x.z, x.w), make_float2(y.z, y.w), a1);
        }
      } else {
#pragma unroll
        for (int c8 = 0; c8 < D / 8; ++c8) {
          const uint4 u = qb8[c8];
          const float4 y = k4[2 * c8], z = k4[2 * c8 + 1];
          a0 = __ffma2_rn(make_float2(bf16_lo(u.x), bf16_hi(u.x)), make_float2(y.x, y.y), a0);
          a1 = __ffma2_rn(make_float2(bf16_lo(u.y), bf16_hi(u.y)), make_float2(y.z, y.w), a1);
          a0 = __ffma2_rn(make_float2(bf16_lo(u.z), bf16_hi(u.z)), make_float2(z.x, z.y), a0);
          a1 = __ffma2_rn(make_float2(bf16_lo(u.w), bf16_hi(u.w)), make_float2(z.z, z.w), a1);
        }
      }
      float s = ((a0.x + a0.y) + (a1.x + a1.y)) * scale;
      if (kChan) {
        if (cached) s -= tile_b;
      } else if (cached && p.correct) {
        s = corrected(s, w, u, d2_s + kk * 4, NG, p.correct);
      }
      if (s > m) {
        const float a = expf(m - s);       // 0 when m = -inf
        l *= a;
        const float2 a2 = make_float2(a, a);
#pragma unroll
        for (int c = 0; c < D / 2; ++c) o[c] = __fmul2_rn(o[c], a2);
        m = s;
      }
      const float pk = expf(s - m);
      l += pk;
      const float2 p2 = make_float2(pk, pk);
      const float4* v4 = reinterpret_cast<const float4*>(v_s + kk * D);
#pragma unroll
      for (int c4 = 0; c4 < D / 4; ++c4) {
        const float4 y = v4[c4];
        o[2 * c4] = __ffma2_rn(p2, make_float2(y.x, y.y), o[2 * c4]);
        o[2 * c4 + 1] = __ffma2_rn(p2, make_float2(y.z, y.w), o[2 * c4 + 1]);
      }
    }
  }
  // Merge the odd-key half of each row into the even-key half (q_s is free now).
  __syncthreads();
  float* mg = q_s + rt * kPitch;                // [D] partial O, then m and l
  if (par == 1) {
#pragma unroll
    for (int c = 0; c < D / 2; ++c) *reinterpret_cast<float2*>(mg + 2 * c) = o[c];
    mg[D] = m;
    mg[D + 1] = l;
  }
  __syncthreads();
  if (par == 1 || !valid_row) return;
  {
    const float m2 = mg[D], l2 = mg[D + 1];
    const float mn = fmaxf(m, m2);
    if (mn != -INFINITY) {
      const float f1 = expf(m - mn), f2 = expf(m2 - mn);
      l = l * f1 + l2 * f2;
      const float2 f1v = make_float2(f1, f1), f2v = make_float2(f2, f2);
#pragma unroll
      for (int c = 0; c < D / 2; ++c)
        o[c] = __ffma2_rn(f2v, *reinterpret_cast<const float2*>(mg + 2 * c), __fmul2_rn(o[c], f1v));
      m = mn;
    }
  }
  const float inv = l > 0.f ? 1.f / l : 0.f;
  if (p.n_split > 1) {
    const int64_t prow = static_cast<int64_t>(blockIdx.z) * p.rows_all + out_row;
    float* orow = p.ws_o + prow * D;
#pragma unroll
    for (int c = 0; c < D / 2; ++c) *reinterpret_cast<float2*>(orow + 2 * c) = make_float2(o[c].x * inv, o[c].y * inv);
    p.ws_lse[prow] = l > 0.f ? m + logf(l) : -INFINITY;
  } else {
    if (kF32In) {
      float* orow = static_cast<float*>(p.O) + out_row * D;
#pragma unroll
      for (int c = 0; c < D / 2; ++c) *reinterpret_cast<float2*>(orow + 2 * c) = make_float2(o[c].x * inv, o[c].y * inv);
    } else {
      __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.O) + out_row * D;
#pragma unroll
      for (int c = 0; c < D / 2; ++c)
        *reinterpret_cast<__nv_bfloat162*>(orow + 2 * c) = __floats2bfloat162_rn(o[c].x * inv, o[c].y * inv);
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
  const size_t smem = (kRows * (D + 4) + 2 * kKT * D + (kChan ? D : kKT * 4)) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(attention_f32_kernel<D, kChan, kF32In>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int64_t rows = static_cast<int64_t>(p.r) * p.Lq;
  dim3 grid(static_cast<unsigned>((rows + kRows - 1) / kRows), static_cast<unsigned>(p.B * p.Hkv),
            static_cast<unsigned>(p.n_split > 1 ? p.n_split : 1));
  attention_f32_kernel<D, kChan, kF32In><<<grid, kThreads, smem, stream>>>(p, bits, T);
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
  if (chan_tc_serves(d, p.in_f32, p.correct)) return launch_attention_channel_tc(p, bits, T, stream);
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
