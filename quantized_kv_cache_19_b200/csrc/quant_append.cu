// Quantise-and-append: packs a finished chunk's K and V into the low-bit cache.
//
// Method: per (token, head, group of `group` channels) asymmetric min-max quantisation to INT2 /
// INT4 (agents-report.net, "KV-Cache 量化導致的 Jensen 偏差", section 問題; the per-token step sizes
// of the fugumt.com abstract of "Quantized Keys Steal Attention"), once per finished chunk (QuantWM
// page on pchao.org, 方法概览). Every fp32 operation is one correctly rounded IEEE operation in a
// fixed order, so the codes are bit-exact against any other IEEE implementation of the same steps:
//   step = (max - min) / (2^bits - 1)  -> stored in the meta dtype (RN)
//   zp   = min                          -> stored in the meta dtype (RN)
//   code = clamp(rint((x - zp_stored) * (1 / step_stored)), 0, 2^bits - 1), ties to even; 0 if step = 0
//
// HBM-bound. Each thread owns 8 consecutive channels of four token-head rows (one 16-byte load of
// bf16 per row, two of fp32, all issued before any arithmetic); the min / max of a group is a
// butterfly of warp shuffles over the group's group/8 lanes; 8 codes are packed into 2 (INT2) or
// 4 (INT4) bytes and stored coalesced with the neighbouring lanes; one lane per group stores
// (step, zero-point). Blocks index (token range, batch * KV head, K or V) directly, so there is
// no integer division on the path.
#include "qkv_common.cuh"
#include "qkv_internal.h"

#include <type_traits>

namespace qkv {
namespace {

__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&x)[8]) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  x[0] = bf16_lo(u.x); x[1] = bf16_hi(u.x);
  x[2] = bf16_lo(u.y); x[3] = bf16_hi(u.y);
  x[4] = bf16_lo(u.z); x[5] = bf16_hi(u.z);
  x[6] = bf16_lo(u.w); x[7] = bf16_hi(u.w);
}
__device__ __forceinline__ void load8(const float* p, float (&x)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
  x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}

template <typename M> struct MetaOps;
template <> struct MetaOps<float> {
  __device__ static float store(float v) { return v; }
  __device__ static float load(float v) { return v; }
  __device__ static void put_pair(void* dst, float a, float b) {
    *reinterpret_cast<float2*>(dst) = make_float2(a, b);
  }
};
template <> struct MetaOps<__half> {
  __device__ static __half store(float v) { return __float2half_rn(v); }
  __device__ static float load(__half v) { return __half2float(v); }
  __device__ static void put_pair(void* dst, __half a, __half b) {
    *reinterpret_cast<__half2*>(dst) = __halves2half2(a, b);
  }
};

__device__ __forceinline__ float fmin3(float a, float b, float c) {
  float y;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(y) : "f"(a), "f"(b), "f"(c));
  return y;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float y;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(y) : "f"(a), "f"(b), "f"(c));
  return y;
}

// Adding 1.5 * 2^23 to a float of magnitude below 2^22 rounds it to an integer (to nearest, ties
// to even) and leaves that integer in the low mantissa bits.
constexpr float kRoundMagic = 12582912.0f;

// Codes of 8 channels, packed LSB-first into 8 * BITS bits:
//   code_k = clamp(rint((x_k - zp) * inv), 0, levels)
// (x - zp) and (* inv) are single IEEE operations as in the definition; rint is the magic-number
// add and subtract (exact, ties to even). The packed value sum_k code_k * 2^(k * BITS) is then
// formed in fp32 FMAs: every partial sum is an integer below 2^16, so each step is exact. With an
// fp32 zero-point x - zp >= 0 and (x - zp) * inv <= levels + a few ulps, so no clamp is needed;
// an fp16 zero-point or step can move either end, and is clamped. A zero step has inv = 0 and
// gives code 0. Non-finite inputs give unspecified codes for their 8 channels.
template <int BITS, bool kClamp>
__device__ __forceinline__ uint32_t pack_codes8(const float (&x)[8], float zp, float inv) {
  constexpr float kLevels = static_cast<float>((1 << BITS) - 1);
  const float2 nzp = make_float2(-zp, -zp);
  const float2 pm = make_float2(kRoundMagic, kRoundMagic), nm = make_float2(-kRoundMagic, -kRoundMagic);
  float2 acc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
  for (int k = 0; k < 8; k += 2) {
    // The product stays a separately rounded multiply (__fmul_rn is never merged into an FMA): a
    // fused multiply-add with the rounding constant would round exact ties the wrong way. (The
    // pair form __fmul2_rn changed the codes of exact ties, so the two products stay scalar.)
    const float2 dx = __fadd2_rn(make_float2(x[k], x[k + 1]), nzp);
    float2 v = make_float2(__fmul_rn(dx.x, inv), __fmul_rn(dx.y, inv));
    if (kClamp) {
      v.x = fminf(fmaxf(v.x, 0.f), kLevels);
      v.y = fminf(fmaxf(v.y, 0.f), kLevels);
    }
    const float2 r = __fadd2_rn(__fadd2_rn(v, pm), nm);
    // INT2: one 16-bit sum; INT4: channels 0-3 and 4-7 in two 16-bit sums
    const int h = (BITS == 4 && k >= 4) ? 1 : 0;
    const int sh = (k - 4 * h) * BITS;
    acc[h] = __ffma2_rn(r, make_float2(static_cast<float>(1 << sh), static_cast<float>(1 << (sh + BITS))), acc[h]);
  }
  const uint32_t lo = __float_as_uint(__fadd_rn(__fadd_rn(acc[0].x, acc[0].y), kRoundMagic));
  if (BITS == 2) return lo & 0xFFFFu;
  const uint32_t hi = __float_as_uint(__fadd_rn(__fadd_rn(acc[1].x, acc[1].y), kRoundMagic));
  return __byte_perm(lo, hi, 0x5410);
}

// One block: kRowsPerBlock consecutive tokens of one (batch, KV head) of one tensor (z = 0: K,
// z = 1: V). D/8 lanes per token row, 8 channels per lane, kPasses rows per thread loaded ahead.
template <typename InT, typename MetaT, int BITS, int D, int G>
__global__ void __launch_bounds__(256) quantize_append_kernel(const QuantAppendParams p) {
  constexpr int kLevels = (1 << BITS) - 1;
  constexpr int kTpr = D / 8;                 // lanes per token row
  constexpr int kTpg = G / 8;                 // lanes per group
  constexpr int kNG = D / G;
  constexpr int kRowsPerPass = 256 / kTpr;
  constexpr int kPasses = 4;
  constexpr int kRowsPerBlock = kRowsPerPass * kPasses;
  static_assert(kTpg >= kPasses, "each row's step is computed by its own lane of the group");
  const int tensor = blockIdx.z;
  if (tensor == 0 && p.K == nullptr) return;  // keys quantised per channel by another kernel
  const int lr = threadIdx.x % kTpr;          // lane within the row: channels 8*lr .. 8*lr+7
  const int pr = threadIdx.x / kTpr;          // row within the pass
  const InT* src_base = static_cast<const InT*>(tensor ? p.V : p.K);
  uint8_t* codes_base = tensor ? p.v_codes : p.k_codes;
  MetaT* meta_base = static_cast<MetaT*>(tensor ? p.v_meta : p.k_meta);
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kRowsPerBlock + pr;

  for (int64_t bh = blockIdx.y; bh < p.BH; bh += gridDim.y) {
    // This thread's first row and channels of the block; row u of the passes is u * kRowsPerPass
    // rows further on (constant strides).
    const InT* src = src_base + (bh * p.L_new + t0) * D + lr * 8;
    const int64_t dst_row0 = bh * p.capacity + p.start + t0;
    float x[kPasses][8];
#pragma unroll
    for (int u = 0; u < kPasses; ++u) {
      const int64_t t = t0 + u * kRowsPerPass;
      if (t < p.L_new) {
        load8(src + u * kRowsPerPass * D, x[u]);
      } else {
#pragma unroll
        for (int k = 0; k < 8; ++k) x[u][k] = 0.f;
      }
    }
    // Group min/max of every row, reduced over the group's lanes (all of them get the result).
    float mn[kPasses], mx[kPasses];
#pragma unroll
    for (int u = 0; u < kPasses; ++u) {
      mn[u] = fmin3(fmin3(x[u][0], x[u][1], x[u][2]), fmin3(x[u][3], x[u][4], x[u][5]), fminf(x[u][6], x[u][7]));
      mx[u] = fmax3(fmax3(x[u][0], x[u][1], x[u][2]), fmax3(x[u][3], x[u][4], x[u][5]), fmaxf(x[u][6], x[u][7]));
#pragma unroll
      for (int off = 1; off < kTpg; off <<= 1) {
        mn[u] = fminf(mn[u], __shfl_xor_sync(0xffffffffu, mn[u], off));
        mx[u] = fmaxf(mx[u], __shfl_xor_sync(0xffffffffu, mx[u], off));
      }
    }
    // Step, zero-point and reciprocal of a group: lane j of the group (kTpg >= kPasses lanes)
    // computes them for row j % kPasses only, writes that row's meta, and the group's lanes read
    // them back with shuffles. The arithmetic is the same single IEEE operations for every row.
    const int jg = lr % kTpg;                    // lane within the group
    const int uo = jg % kPasses;                 // the row this lane takes
    float mn_o = mn[0], mx_o = mx[0];
#pragma unroll
    for (int u = 1; u < kPasses; ++u)
      if (uo == u) { mn_o = mn[u]; mx_o = mx[u]; }
    const float step32 = __fdiv_rn(__fsub_rn(mx_o, mn_o), static_cast<float>(kLevels));
    const MetaT step_m = MetaOps<MetaT>::store(step32);
    const MetaT zp_m = MetaOps<MetaT>::store(mn_o);
    const float step_o = MetaOps<MetaT>::load(step_m);
    const float zp_o = MetaOps<MetaT>::load(zp_m);
    const float inv_o = step_o > 0.f ? __frcp_rn(step_o) : 0.f;
    {
      const int64_t t = t0 + uo * kRowsPerPass;
      if (jg < kPasses && t < p.L_new) {
        const int64_t dst_row = dst_row0 + uo * kRowsPerPass;
        MetaOps<MetaT>::put_pair(meta_base + (dst_row * kNG + lr / kTpg) * 2, step_m, zp_m);
      }
    }
    const int lane0 = (threadIdx.x & 31) - jg;  // first lane of this group in the warp
#pragma unroll
    for (int u = 0; u < kPasses; ++u) {
      const float zp = __shfl_sync(0xffffffffu, zp_o, lane0 + u);
      const float inv = __shfl_sync(0xffffffffu, inv_o, lane0 + u);
      const int64_t t = t0 + u * kRowsPerPass;
      if (t >= p.L_new) continue;
      const uint32_t packed = pack_codes8<BITS, !std::is_same<MetaT, float>::value>(x[u], zp, inv);
      uint8_t* codes = codes_base + (dst_row0 + u * kRowsPerPass) * (D * BITS / 8) + lr * BITS;
      if (BITS == 2) {
        *reinterpret_cast<uint16_t*>(codes) = static_cast<uint16_t>(packed);
      } else {
        *reinterpret_cast<uint32_t*>(codes) = packed;
      }
    }
  }
}

template <typename InT, typename MetaT, int BITS, int D, int G>
cudaError_t launch(const QuantAppendParams& p, cudaStream_t stream) {
  constexpr int kRowsPerBlock = (256 / (D / 8)) * 4;
  const int64_t bx = (p.L_new + kRowsPerBlock - 1) / kRowsPerBlock;
  if (bx > 0x7fffffffLL) return cudaErrorInvalidValue;
  const dim3 grid(static_cast<unsigned>(bx), static_cast<unsigned>(p.BH < 65535 ? p.BH : 65535), 2);
  quantize_append_kernel<InT, MetaT, BITS, D, G><<<grid, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

template <typename InT, typename MetaT, int BITS>
cudaError_t launch_dg(const QuantAppendParams& p, cudaStream_t stream) {
  if (p.d == 128) {
    if (p.group == 32) return launch<InT, MetaT, BITS, 128, 32>(p, stream);
    if (p.group == 64) return launch<InT, MetaT, BITS, 128, 64>(p, stream);
    return launch<InT, MetaT, BITS, 128, 128>(p, stream);
  }
  if (p.group == 32) return launch<InT, MetaT, BITS, 64, 32>(p, stream);
  return launch<InT, MetaT, BITS, 64, 64>(p, stream);
}

}  // namespace

cudaError_t launch_quantize_append(const QuantAppendParams& p, int in_dtype, int meta_dtype,
                                   int bits, cudaStream_t stream) {
  const bool f32 = in_dtype == kF32;
  const bool m16 = meta_dtype == kF16;
  if (bits == 2) {
    if (f32) return m16 ? launch_dg<float, __half, 2>(p, stream) : launch_dg<float, float, 2>(p, stream);
    return m16 ? launch_dg<__nv_bfloat16, __half, 2>(p, stream)
               : launch_dg<__nv_bfloat16, float, 2>(p, stream);
  }
  if (f32) return m16 ? launch_dg<float, __half, 4>(p, stream) : launch_dg<float, float, 4>(p, stream);
  return m16 ? launch_dg<__nv_bfloat16, __half, 4>(p, stream)
             : launch_dg<__nv_bfloat16, float, 4>(p, stream);
}

}  // namespace qkv
