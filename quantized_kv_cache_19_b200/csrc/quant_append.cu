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
// HBM-bound. Each thread owns 8 consecutive channels of one token-head row (one 16-byte load of
// bf16, two of fp32); the min / max of a group is a butterfly of warp shuffles over the
// group's group/8 lanes; 8 codes are packed into 2 (INT2) or 4 (INT4) bytes and stored
// coalesced with the neighbouring lanes; one lane per group stores (step, zero-point).
#include "qkv_common.cuh"
#include "qkv_internal.h"

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

template <typename InT, typename MetaT, int BITS>
__global__ void __launch_bounds__(256) quantize_append_kernel(const QuantAppendParams p) {
  constexpr int kLevels = (1 << BITS) - 1;
  const int tpr = p.d >> 3;        // lanes per token-head row
  const int tpg = p.group >> 3;    // lanes per group
  const int n_g = p.d / p.group;
  const int64_t per_tensor = p.rows * tpr;
  const int64_t total = 2 * per_tensor;
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) - lane;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;

  // The loop bound is warp-uniform so every lane reaches every shuffle.
  for (int64_t base = warp0; base < total; base += stride) {
    const int64_t idx = base + lane;
    const bool active = idx < total;
    const int tensor = active ? static_cast<int>(idx / per_tensor) : 0;
    const int64_t rem = active ? idx - tensor * per_tensor : 0;
    const int64_t row = rem / tpr;
    const int chunk = static_cast<int>(rem - row * tpr);

    float x[8];
    if (active) {
      const InT* src = static_cast<const InT*>(tensor ? p.V : p.K) + row * p.d + chunk * 8;
      load8(src, x);
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) x[k] = 0.f;
    }
    float mn = x[0], mx = x[0];
#pragma unroll
    for (int k = 1; k < 8; ++k) { mn = fminf(mn, x[k]); mx = fmaxf(mx, x[k]); }
    for (int off = 1; off < tpg; off <<= 1) {
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    }
    if (!active) continue;

    const float step32 = __fdiv_rn(__fsub_rn(mx, mn), static_cast<float>(kLevels));
    const MetaT step_m = MetaOps<MetaT>::store(step32);
    const MetaT zp_m = MetaOps<MetaT>::store(mn);
    const float step = MetaOps<MetaT>::load(step_m);
    const float zp = MetaOps<MetaT>::load(zp_m);
    const bool pos = step > 0.f;
    const float inv = pos ? __frcp_rn(step) : 0.f;

    uint32_t packed = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      int c = 0;
      if (pos) {
        c = __float2int_rn(__fmul_rn(__fsub_rn(x[k], zp), inv));
        c = min(max(c, 0), kLevels);
      }
      packed |= static_cast<uint32_t>(c) << (k * BITS);
    }

    const int64_t bh = row / p.L_new;
    const int64_t t = row - bh * p.L_new;
    const int64_t dst_row = bh * p.capacity + p.start + t;
    uint8_t* codes = (tensor ? p.v_codes : p.k_codes) + dst_row * (p.d * BITS / 8) + chunk * BITS;
    if (BITS == 2) {
      *reinterpret_cast<uint16_t*>(codes) = static_cast<uint16_t>(packed);
    } else {
      *reinterpret_cast<uint32_t*>(codes) = packed;
    }
    if ((chunk % tpg) == 0) {
      MetaT* meta = static_cast<MetaT*>(tensor ? p.v_meta : p.k_meta) +
                    (dst_row * n_g + chunk / tpg) * 2;
      MetaOps<MetaT>::put_pair(meta, step_m, zp_m);
    }
  }
}

template <typename InT, typename MetaT, int BITS>
cudaError_t launch(const QuantAppendParams& p, cudaStream_t stream) {
  const int64_t total = 2 * p.rows * (p.d / 8);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t want = (total + 255) / 256;
  const int grid = static_cast<int>(want < sms * 8LL ? want : sms * 8LL);
  quantize_append_kernel<InT, MetaT, BITS><<<grid, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quantize_append(const QuantAppendParams& p, int in_dtype, int meta_dtype,
                                   int bits, cudaStream_t stream) {
  const bool f32 = in_dtype == kF32;
  const bool m16 = meta_dtype == kF16;
  if (bits == 2) {
    if (f32) return m16 ? launch<float, __half, 2>(p, stream) : launch<float, float, 2>(p, stream);
    return m16 ? launch<__nv_bfloat16, __half, 2>(p, stream)
               : launch<__nv_bfloat16, float, 2>(p, stream);
  }
  if (f32) return m16 ? launch<float, __half, 4>(p, stream) : launch<float, float, 4>(p, stream);
  return m16 ? launch<__nv_bfloat16, __half, 4>(p, stream)
             : launch<__nv_bfloat16, float, 4>(p, stream);
}

}  // namespace qkv
