// Host-side declarations of the per-channel key layout (keys grouped along tokens), not part of
// the public ABI.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "qkv_internal.h"

namespace qkv {

// Keys [BH][L_new][d] quantised per channel over blocks of T cache positions: block k holds
// positions [k T, (k+1) T); meta [BH][capacity / T][d][2] = (step, zero-point). `start` (the cache
// length before the append) is a multiple of T; a last block may be partial.
struct ChanQuantParams {
  const void* K;
  uint8_t* k_codes;
  void* k_meta;
  int64_t BH;
  int64_t L_new;
  int64_t capacity;
  int64_t start;
  int d, T;
};
cudaError_t launch_quantize_keys_channel(const ChanQuantParams& p, int in_dtype, int meta_dtype,
                                         int bits, cudaStream_t stream);

// Corrected attention over a cache with per-channel key blocks of T positions (fp32 CUDA cores,
// bf16 or fp32 inputs; O in the input type). With p.n_split > 1 (bf16 inputs only) the cached keys
// are split over grid z and the normalised partials written to p.ws_o / p.ws_lse for the merge.
cudaError_t launch_attention_channel(const AttnParams& p, int d, int bits, int T, cudaStream_t stream);
// Query rows per CTA and keys per shared-memory tile of that kernel.
int channel_rows_per_cta();
int channel_tile_keys();

// The tensor-core kernel for per-channel key blocks (attention_chan.cu) serves d = 128, bf16
// inputs and correct <= 1; launch_attention_channel routes those calls to it. It takes 128 query
// rows per CTA and 128-key tiles; with p.n_split > 1 it splits the 128-key tiles of the cache.
bool chan_tc_serves(int d, int in_f32, int correct);
constexpr int kChanTcTileKeys = 128;
cudaError_t launch_attention_channel_tc(const AttnParams& p, int bits, int T, cudaStream_t stream);

// Correction term alone over per-channel key blocks: bias[B][Hq][Lq][Lc].
cudaError_t launch_jensen_bias_channel(const BiasParams& p, int T, cudaStream_t stream);

}  // namespace qkv
