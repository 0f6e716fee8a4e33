// Host-side declarations shared by the translation units of libqkv (not part of the public ABI).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace qkv {

enum : int { kF32 = 0, kBF16 = 1, kF16 = 2 };

// Default bound of a kernel's progress waits, in SM clock cycles (about a second at 1.9 GHz).
constexpr long long kDefaultWaitLimitCycles = 2000000000LL;

// Quantise-and-append: K and V [B][H_kv][L_new][d] into the cache at positions start..start+L_new-1.
struct QuantAppendParams {
  const void* K;
  const void* V;
  uint8_t* k_codes;
  uint8_t* v_codes;
  void* k_meta;
  void* v_meta;
  int64_t BH;        // B * H_kv
  int64_t L_new;
  int64_t capacity;
  int64_t start;
  int d, group;
};
cudaError_t launch_quantize_append(const QuantAppendParams& p, int in_dtype, int meta_dtype,
                                   int bits, cudaStream_t stream);

// Corrected attention: one CTA per (128 packed query rows, batch * KV head).
struct AttnParams {
  const void* Q;
  const void* K_cur;
  const void* V_cur;
  void* O;
  float* LSE;
  const uint8_t* k_codes;
  const uint8_t* v_codes;
  const void* k_meta;
  const void* v_meta;
  int* status;
  int64_t Lq, Lc, Lcur, capacity;
  int B, Hq, Hkv, r;
  int group, n_groups;
  int correct, causal;
  int in_f32, meta_f16;
  float scale_log2;   // score scale * log2(e)
  float wcoef_log2;   // scale^2 / 24 * log2(e): Jensen-correction coefficient in log2 units
  float inv_scale_log2;  // 1 / (scale * log2(e))
  float ucoef_log2;   // scale^4 / 2880 * log2(e): fourth-order coefficient (correct = 2), else 0
  // Split over the cached keys (n_split > 1): CTA z takes cached tiles [z * T / n, (z+1) * T / n)
  // (the last one also the current chunk) and writes its row's normalised partial output and
  // log-sum-exp to ws_o [n_split][rows_all][d] and ws_lse [n_split][rows_all] (fp32).
  int n_split;
  int64_t rows_all;     // B * Hq * Lq
  float* ws_o;
  float* ws_lse;
  long long wait_limit;   // bound of the kernel's progress waits, SM clock cycles
};
// bf16 inputs: tcgen05 kernel. fp32 inputs: CUDA-core fp32 kernel.
cudaError_t launch_attention_bf16(const AttnParams& p, int d, int bits, cudaStream_t stream);
// Key tiles of one (batch, KV head) in the bf16 kernel (128 keys, or 64 with four groups).
int attention_tile_keys(int n_groups);
// Merge of split partials: O (bf16) and LSE from ws_o / ws_lse.
cudaError_t launch_split_merge(const float* ws_o, const float* ws_lse, int n_split, int64_t rows_all,
                               int d, void* O, float* LSE, cudaStream_t stream);
cudaError_t launch_attention_f32(const AttnParams& p, int d, int bits, cudaStream_t stream);

// Jensen-correction term alone: bias[B][Hq][Lq][Lc] (natural units).
struct BiasParams {
  const void* Q;
  const void* k_meta;
  float* bias;
  int64_t Lq, Lc, capacity;
  int B, Hq, Hkv, r;
  int d, group, n_groups;
  int in_f32, meta_f16;
  float wcoef;        // scale^2 / 24
};
cudaError_t launch_jensen_bias(const BiasParams& p, cudaStream_t stream);

}  // namespace qkv
