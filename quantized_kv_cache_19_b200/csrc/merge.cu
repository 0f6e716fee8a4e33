// Merge of split-over-keys partial attention results.
//
// When the cached keys of a (batch, KV head) are split over several CTAs, each split s produces,
// for every query row, the softmax-normalised output O_s over its keys and the log-sum-exp L_s of
// its (corrected) scores. The row's result over all keys is the softmax-weighted combination
//     L = log sum_s exp(L_s),   O = sum_s exp(L_s - L) * O_s,
// the same online-softmax identity the attention kernel applies tile by tile (a split with no
// visible key has L_s = -inf and weight 0; a row without any key gets O = 0, L = -inf).
//
// HBM-bound: one warp per row reads n_split * (d + 1) floats and writes d bf16 values and one
// float; the log-sum-exps of the row are held one per lane (n_split <= 32).
#include "qkv_common.cuh"
#include "qkv_internal.h"

namespace qkv {
namespace {

template <int D>
__global__ void __launch_bounds__(256) split_merge_kernel(const float* __restrict__ ws_o,
                                                          const float* __restrict__ ws_lse,
                                                          int n_split, int64_t rows_all,
                                                          __nv_bfloat16* __restrict__ O,
                                                          float* __restrict__ LSE) {
  constexpr int kPerLane = D / 32;
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (row >= rows_all) return;
  const float l_s = lane < n_split ? ws_lse[static_cast<int64_t>(lane) * rows_all + row] : -INFINITY;
  float m = l_s;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  __nv_bfloat16* orow = O + row * D;
  if (m == -INFINITY) {
#pragma unroll
    for (int k = 0; k < kPerLane; ++k) orow[lane * kPerLane + k] = __float2bfloat16_rn(0.f);
    if (lane == 0) LSE[row] = -INFINITY;
    return;
  }
  const float w = lane < n_split ? expf(l_s - m) : 0.f;
  float wsum = w;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, off);
  float acc[kPerLane];
#pragma unroll
  for (int k = 0; k < kPerLane; ++k) acc[k] = 0.f;
  for (int s = 0; s < n_split; ++s) {
    const float ws = __shfl_sync(0xffffffffu, w, s);
    const float* o = ws_o + (static_cast<int64_t>(s) * rows_all + row) * D + lane * kPerLane;
    if (ws != 0.f) {
#pragma unroll
      for (int k = 0; k < kPerLane; ++k) acc[k] = fmaf(ws, o[k], acc[k]);
    }
  }
  const float inv = 1.f / wsum;
#pragma unroll
  for (int k = 0; k < kPerLane; ++k) orow[lane * kPerLane + k] = __float2bfloat16_rn(acc[k] * inv);
  if (lane == 0) LSE[row] = m + logf(wsum);
}

}  // namespace

cudaError_t launch_split_merge(const float* ws_o, const float* ws_lse, int n_split, int64_t rows_all,
                               int d, void* O, float* LSE, cudaStream_t stream) {
  if (n_split < 1 || n_split > 32) return cudaErrorInvalidValue;
  const int64_t blocks = (rows_all + 7) / 8;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  if (d == 128)
    split_merge_kernel<128><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        ws_o, ws_lse, n_split, rows_all, static_cast<__nv_bfloat16*>(O), LSE);
  else
    split_merge_kernel<64><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        ws_o, ws_lse, n_split, rows_all, static_cast<__nv_bfloat16*>(O), LSE);
  return cudaGetLastError();
}

}  // namespace qkv
