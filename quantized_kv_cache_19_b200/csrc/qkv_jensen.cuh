// Per-query-row quantities of the Jensen correction, shared by the attention kernels and the
// correction-only kernel so that all of them evaluate the term the same way.
//
// Correction (agents-report.net, "KV-Cache 量化導致的 Jensen 偏差", section 方法):
//   b_ij = (scale^2 / 24) * sum_c q_ic^2 * Delta_{j, c/group}^2 = sum_g w_ig * Delta_jg^2,
//   w_ig = (scale^2 / 24) * sum_{c in group g} q_ic^2.
#pragma once

#include "qkv_common.cuh"

namespace qkv {

constexpr int kMaxGroups = 4;   // d <= 128 and group >= 32

// Loads 8 consecutive channels of a query row as fp32 (fp32 or bf16 storage).
__device__ __forceinline__ void load_q8(const uint8_t* qrow, bool f32, int c8, float (&x)[8]) {
  if (f32) {
    const float4 a = reinterpret_cast<const float4*>(qrow)[2 * c8];
    const float4 b = reinterpret_cast<const float4*>(qrow)[2 * c8 + 1];
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  } else {
    const uint4 u = reinterpret_cast<const uint4*>(qrow)[c8];
    x[0] = bf16_lo(u.x); x[1] = bf16_hi(u.x); x[2] = bf16_lo(u.y); x[3] = bf16_hi(u.y);
    x[4] = bf16_lo(u.z); x[5] = bf16_hi(u.z); x[6] = bf16_lo(u.w); x[7] = bf16_hi(u.w);
  }
}

// w[g] = coef * sum_{c in g} q_c^2, accumulated in fp32 in channel order (8 channels at a time).
template <int D>
__device__ __forceinline__ void query_group_weights(const uint8_t* qrow, bool f32, int group,
                                                    float coef, float (&w)[kMaxGroups]) {
#pragma unroll
  for (int g = 0; g < kMaxGroups; ++g) w[g] = 0.f;
#pragma unroll
  for (int c8 = 0; c8 < D / 8; ++c8) {
    float x[8];
    load_q8(qrow, f32, c8, x);
    float acc = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) acc = fmaf(x[k], x[k], acc);
    const int g = (c8 * 8) / group;
#pragma unroll
    for (int gg = 0; gg < kMaxGroups; ++gg)
      if (gg == g) w[gg] += acc;
  }
#pragma unroll
  for (int g = 0; g < kMaxGroups; ++g) w[g] *= coef;
}

// Second- and fourth-order weights in one pass over the row: w[g] = coef2 * sum_{c in g} q_c^2 and
// u[g] = coef4 * sum_{c in g} q_c^4 (the a^4 / 180 term of the series of log(sinh a / a),
// a = scale q_c Delta / 2, is (scale^4 / 2880) q_c^4 Delta^4).
template <int D>
__device__ __forceinline__ void query_group_powers(const uint8_t* qrow, bool f32, int group, float coef2,
                                                   float coef4, float (&w)[kMaxGroups],
                                                   float (&u)[kMaxGroups]) {
#pragma unroll
  for (int g = 0; g < kMaxGroups; ++g) { w[g] = 0.f; u[g] = 0.f; }
#pragma unroll
  for (int c8 = 0; c8 < D / 8; ++c8) {
    float x[8];
    load_q8(qrow, f32, c8, x);
    float a2 = 0.f, a4 = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float x2 = x[k] * x[k];
      a2 += x2;
      a4 = fmaf(x2, x2, a4);
    }
    const int g = (c8 * 8) / group;
#pragma unroll
    for (int gg = 0; gg < kMaxGroups; ++gg)
      if (gg == g) { w[gg] += a2; u[gg] += a4; }
  }
#pragma unroll
  for (int g = 0; g < kMaxGroups; ++g) { w[g] *= coef2; u[g] *= coef4; }
}

// The correction of one (query, key) pair from the key's squared steps: sum_g w[g] * d2[g].
__device__ __forceinline__ float jensen_term(const float (&w)[kMaxGroups],
                                             const float (&d2)[kMaxGroups], int n_groups) {
  float b = w[0] * d2[0];
#pragma unroll
  for (int g = 1; g < kMaxGroups; ++g)
    if (g < n_groups) b = fmaf(w[g], d2[g], b);
  return b;
}

}  // namespace qkv
