// Host-side declarations of the attention-fidelity diagnostic (not part of the public ABI).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace qkv {

constexpr int kFidelityTopK = 5;      // length of each top-key list
constexpr int kFidelityStats = 8;     // floats per query row in the statistics output

// Per query row: the softmax over the unquantised cached keys and the current keys (reference)
// against the corrected softmax over the quantised cache and the current keys.
struct FidelityParams {
  const void* Q;          // [B][Hq][Lq][d], fp32 or bf16
  const void* K_ref;      // [B][Hkv][Lc][d], Q's dtype: the cached keys before quantisation
  const void* K_cur;      // [B][Hkv][Lcur][d], Q's dtype
  const uint8_t* k_codes;
  const void* k_meta;
  float* stats;           // [B][Hq][Lq][kFidelityStats]
  int32_t* top;           // [B][Hq][Lq][2][kFidelityTopK] or null
  int64_t Lq, Lc, Lcur, capacity;
  int B, Hq, Hkv, r;
  int bits, group, n_groups;
  int key_block;          // 0: key groups per token; T: keys per channel over blocks of T positions
  int correct, causal;
  int in_f32, meta_f16;
  float scale;            // score scale (natural units)
  float wcoef;            // scale^2 / 24
  float ucoef;            // scale^4 / 2880 when correct = 2, else 0
};
cudaError_t launch_attention_fidelity(const FidelityParams& p, int d, cudaStream_t stream);
// Query rows of one CTA of the fidelity kernel.
int fidelity_rows_per_cta();

}  // namespace qkv
