// Per-channel key quantisation along tokens (KIVI's key grouping, named in agents-report.net,
// "KV-Cache 量化導致的 Jensen 偏差", section 跨主題對比分析; the hotelren.com blog, section 3.1, groups
// along the sequence axis).
//
// Every T consecutive cache positions of one (batch, KV head, channel) share one step and zero-point:
//   step = (max - min) / (2^bits - 1), zero-point = min over the block's tokens (IEEE fp32, then
//   stored in the meta dtype), code = clamp(rint((x - zp) * (1 / step)), 0, 2^bits - 1) from the
//   stored values, each operation one correctly rounded fp32 operation; 0 for a zero step.
// The codes of a token are packed as in the per-token layout (channel c at bit c * bits).
//
// One CTA of 256 threads per (key block, batch * KV head): D/8 channel octets x (256 / (D/8)) token
// lanes. Pass 1 takes each lane's min/max over its tokens and reduces them through shared memory;
// pass 2 re-reads the block (from L1/L2), codes it and writes 8 channels' codes per thread.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "channel.h"
#include "qkv_common.cuh"

namespace qkv {
namespace {

constexpr int kThreadsQ = 256;

__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&x)[8]) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  x[0] = bf16_lo(u.x); x[1] = bf16_hi(u.x); x[2] = bf16_lo(u.y); x[3] = bf16_hi(u.y);
  x[4] = bf16_lo(u.z); x[5] = bf16_hi(u.z); x[6] = bf16_lo(u.w); x[7] = bf16_hi(u.w);
}

__device__ __forceinline__ void load8(const float* p, float (&x)[8]) {
  const float4 a = reinterpret_cast<const float4*>(p)[0];
  const float4 b = reinterpret_cast<const float4*>(p)[1];
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}

__device__ __forceinline__ void store_meta(float* m, float step, float zp, float& step_f, float& zp_f) {
  m[0] = step;
  m[1] = zp;
  step_f = step;
  zp_f = zp;
}

__device__ __forceinline__ void store_meta(__half* m, float step, float zp, float& step_f, float& zp_f) {
  const __half s = __float2half_rn(step), z = __float2half_rn(zp);
  m[0] = s;
  m[1] = z;
  step_f = __half2float(s);
  zp_f = __half2float(z);
}

template <typename InT, typename MetaT, int BITS, int D>
__global__ void __launch_bounds__(kThreadsQ) quantize_keys_channel_kernel(const ChanQuantParams p) {
  constexpr int kLevels = (1 << BITS) - 1;
  constexpr int kOct = D / 8;                     // channel octets per token
  constexpr int kLanes = kThreadsQ / kOct;        // token lanes
  __shared__ float red_mn[kLanes][D];
  __shared__ float red_mx[kLanes][D];
  __shared__ float s_zp[D];
  __shared__ float s_inv[D];

  const int oct = threadIdx.x % kOct;
  const int lane = threadIdx.x / kOct;
  const int64_t bh = blockIdx.y;
  const int64_t first = static_cast<int64_t>(blockIdx.x) * p.T;      // within the appended tokens
  const int nt = static_cast<int>(min(static_cast<int64_t>(p.T), p.L_new - first));
  const InT* src = static_cast<const InT*>(p.K) + (bh * p.L_new + first) * D + 8 * oct;

  float mn[8], mx[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) { mn[k] = INFINITY; mx[k] = -INFINITY; }
  for (int t = lane; t < nt; t += kLanes) {
    float x[8];
    load8(src + static_cast<int64_t>(t) * D, x);
#pragma unroll
    for (int k = 0; k < 8; ++k) { mn[k] = fminf(mn[k], x[k]); mx[k] = fmaxf(mx[k], x[k]); }
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) { red_mn[lane][8 * oct + k] = mn[k]; red_mx[lane][8 * oct + k] = mx[k]; }
  __syncthreads();
  if (threadIdx.x < D) {
    const int c = threadIdx.x;
    float a = red_mn[0][c], b = red_mx[0][c];
    for (int l = 1; l < kLanes; ++l) { a = fminf(a, red_mn[l][c]); b = fmaxf(b, red_mx[l][c]); }
    const float step32 = __fdiv_rn(__fsub_rn(b, a), static_cast<float>(kLevels));
    const int64_t blk = p.start / p.T + blockIdx.x;
    MetaT* m = static_cast<MetaT*>(p.k_meta) + ((bh * (p.capacity / p.T) + blk) * D + c) * 2;
    float step_f, zp_f;
    store_meta(m, step32, a, step_f, zp_f);
    s_zp[c] = zp_f;
    s_inv[c] = step_f > 0.f ? __frcp_rn(step_f) : 0.f;     // a zero step codes everything as 0
  }
  __syncthreads();

  float zp[8], inv[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) { zp[k] = s_zp[8 * oct + k]; inv[k] = s_inv[8 * oct + k]; }
  constexpr int kRowBytes = D * BITS / 8;
  uint8_t* dst = p.k_codes + (bh * p.capacity + p.start + first) * kRowBytes + oct * BITS;
  for (int t = lane; t < nt; t += kLanes) {
    float x[8];
    load8(src + static_cast<int64_t>(t) * D, x);
    uint32_t word = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float v = rintf(__fmul_rn(__fsub_rn(x[k], zp[k]), inv[k]));
      const float cl = fminf(fmaxf(v, 0.f), static_cast<float>(kLevels));
      word |= static_cast<uint32_t>(cl) << (k * BITS);
    }
    uint8_t* row = dst + static_cast<int64_t>(t) * kRowBytes;
    if (BITS == 2) *reinterpret_cast<uint16_t*>(row) = static_cast<uint16_t>(word);
    else *reinterpret_cast<uint32_t*>(row) = word;
  }
}

template <typename InT, typename MetaT, int BITS>
cudaError_t launch_q(const ChanQuantParams& p, cudaStream_t stream) {
  const dim3 grid(static_cast<unsigned>((p.L_new + p.T - 1) / p.T), static_cast<unsigned>(p.BH));
  if (p.d == 128) quantize_keys_channel_kernel<InT, MetaT, BITS, 128><<<grid, kThreadsQ, 0, stream>>>(p);
  else quantize_keys_channel_kernel<InT, MetaT, BITS, 64><<<grid, kThreadsQ, 0, stream>>>(p);
  return cudaGetLastError();
}

template <typename InT, typename MetaT>
cudaError_t launch_qb(const ChanQuantParams& p, int bits, cudaStream_t stream) {
  return bits == 2 ? launch_q<InT, MetaT, 2>(p, stream) : launch_q<InT, MetaT, 4>(p, stream);
}

template <typename InT>
cudaError_t launch_qm(const ChanQuantParams& p, int meta_dtype, int bits, cudaStream_t stream) {
  return meta_dtype == kF16 ? launch_qb<InT, __half>(p, bits, stream) : launch_qb<InT, float>(p, bits, stream);
}

}  // namespace

cudaError_t launch_quantize_keys_channel(const ChanQuantParams& p, int in_dtype, int meta_dtype,
                                         int bits, cudaStream_t stream) {
  return in_dtype == kF32 ? launch_qm<float>(p, meta_dtype, bits, stream)
                          : launch_qm<__nv_bfloat16>(p, meta_dtype, bits, stream);
}

}  // namespace qkv
