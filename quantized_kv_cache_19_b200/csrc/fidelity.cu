// Attention-fidelity diagnostics: how far the corrected softmax over the quantised cache is from
// the softmax over the same keys before quantisation.
//
// The measures come from the pages:
//   - pchao.org, "QuantWM", section 实验如何设计: token drift, the share of positions whose
//     top-1 attended token under the quantised cache differs from the BF16 one;
//   - gist.science, "Statistical Inference and Quality Measures of KV Cache Quantisations Inspired
//     by TurboQuant", section Métricas de Avaliação: KL divergence between the reference and the
//     quantised softmax distributions, and recall of the reference's top-5 keys;
//   - agents-report.net, "KV-Cache 量化導致的 Jensen 偏差", section 為何校正有效: quantised keys
//     gain softmax mass on the cached segment, and the correction removes that gain.
//
// Per query row, with s_ref = scale q.k over [K_ref ; K_cur] and s_q = the corrected attention's
// scores over [dequantised cache ; K_cur]:
//   stats = { LSE_ref, LSE_q, cached mass under P_ref, cached mass under P_q, KL(P_ref || P_q),
//             top-1 agreement (0 or 1), top-5 recall, 0 }
// KL uses sum_j P_ref,j (s_ref,j - s_q,j) - LSE_ref + LSE_q, accumulated online next to the two
// log-sum-exps. Every score is fp32 on CUDA cores: the KL of an INT4 cache is small enough that
// rounding dequantised keys to bf16 for tensor cores would change it.
//
// Layout of the work: a CTA of four warps takes 32 query rows of one (batch, KV head), one row per
// lane; warp w takes keys w, w + 4, ... of each 32-key shared-memory tile, so all lanes of a warp
// read the same key (a broadcast) while each keeps its row of q in registers. The dot products use
// packed fp32x2 FMAs (even and odd channels in the two halves). At the end the four warps' running
// sums and top-5 lists of each row are merged through shared memory.
#include <cuda_fp16.h>

#include "fidelity.h"
#include "qkv_common.cuh"
#include "qkv_jensen.cuh"

namespace qkv {
namespace {

constexpr int kRowsF = 32;                  // query rows per CTA
constexpr int kSlices = 4;                  // warps per CTA, each on every fourth key
constexpr int kThreadsF = kRowsF * kSlices;
constexpr int kKeysF = 32;                  // keys per shared-memory tile
constexpr int kTop = kFidelityTopK;
constexpr int kNoKey = 0x7fffffff;          // empty slot of a top list

struct TopList {
  float v[kTop];
  int ix[kTop];
};

// Descending score; the lower key index first on equal scores.
__device__ __forceinline__ bool ranks_before(float a, int ia, float b, int ib) {
  return a > b || (a == b && ia < ib);
}

__device__ __forceinline__ void top_init(TopList& t) {
#pragma unroll
  for (int i = 0; i < kTop; ++i) { t.v[i] = -INFINITY; t.ix[i] = kNoKey; }
}

__device__ __forceinline__ void top_insert(TopList& t, float s, int j) {
  if (!ranks_before(s, j, t.v[kTop - 1], t.ix[kTop - 1])) return;
  t.v[kTop - 1] = s;
  t.ix[kTop - 1] = j;
#pragma unroll
  for (int i = kTop - 1; i > 0; --i) {
    if (ranks_before(t.v[i], t.ix[i], t.v[i - 1], t.ix[i - 1])) {
      const float fv = t.v[i]; t.v[i] = t.v[i - 1]; t.v[i - 1] = fv;
      const int fi = t.ix[i]; t.ix[i] = t.ix[i - 1]; t.ix[i - 1] = fi;
    }
  }
}

// Running softmax sums of one distribution: max m, sum l = sum e^{s - m}, its cached part lc.
struct Running {
  float m, l, lc;
};

__device__ __forceinline__ float rescale_to(Running& r, float s) {
  float a = 1.f;
  if (s > r.m) {
    a = expf(r.m - s);          // 0 while nothing was seen (m = -inf)
    r.l *= a;
    r.lc *= a;
    r.m = s;
  }
  return a;
}

// Adds the running sums (m2, l2, lc2) and A2 of a disjoint key set.
__device__ __forceinline__ void merge_running(Running& r, float& A, float m2, float l2, float lc2, float A2) {
  const float m = fmaxf(r.m, m2);
  if (m == -INFINITY) return;
  const float f1 = expf(r.m - m), f2 = expf(m2 - m);
  r.l = r.l * f1 + l2 * f2;
  r.lc = r.lc * f1 + lc2 * f2;
  A = A * f1 + A2 * f2;
  r.m = m;
}

// Four consecutive channels of a key row (fp32 or bf16 storage) as fp32.
__device__ __forceinline__ float4 load_key4(const void* base, int64_t elem, bool f32) {
  if (f32) return *reinterpret_cast<const float4*>(static_cast<const float*>(base) + elem);
  const uint2 u = *reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(base) + elem);
  return make_float4(bf16_lo(u.x), bf16_hi(u.x), bf16_lo(u.y), bf16_hi(u.y));
}

// One 4-channel chunk e of the key tile starting at k0: the reference key (K_ref, or K_cur past the
// cache) and the dequantised key zp + step * code in fp32, plus the squared steps of the tile's
// cached keys (per group and key; per channel for the block with per-channel keys).
template <int D, bool kChan>
__device__ __forceinline__ void fill_key_chunk(const FidelityParams& p, int e, int64_t k0, int64_t total,
                                               int bh, bool f32, float* kr_s, float* kq_s, float* d2_s) {
  constexpr int kPitch = D + 4;
  const int kk = e / (D / 4), c4 = e - kk * (D / 4);
  const int64_t key = k0 + kk;
  float4 xr = make_float4(0.f, 0.f, 0.f, 0.f), xq = xr;
  if (key < p.Lc) {
    xr = load_key4(p.K_ref, (static_cast<int64_t>(bh) * p.Lc + key) * D + 4 * c4, f32);
    const int64_t crow = static_cast<int64_t>(bh) * p.capacity + key;
    const int g = (4 * c4) / p.group;
    // (step, zero-point) of the 4 channels: one group's pair, or each channel's own pair
    float st[4], zp[4];
    if (kChan) {
      const int64_t mi = ((static_cast<int64_t>(bh) * (p.capacity / p.key_block) + key / p.key_block) * D + 4 * c4) * 2;
      if (p.meta_f16) {
        const uint4 u = *reinterpret_cast<const uint4*>(static_cast<const __half*>(p.k_meta) + mi);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          st[i] = __half2float(__ushort_as_half(static_cast<unsigned short>(w[i] & 0xFFFFu)));
          zp[i] = __half2float(__ushort_as_half(static_cast<unsigned short>(w[i] >> 16)));
        }
      } else {
        const float4 a = *reinterpret_cast<const float4*>(static_cast<const float*>(p.k_meta) + mi);
        const float4 b = *reinterpret_cast<const float4*>(static_cast<const float*>(p.k_meta) + mi + 4);
        st[0] = a.x; zp[0] = a.y; st[1] = a.z; zp[1] = a.w;
        st[2] = b.x; zp[2] = b.y; st[3] = b.z; zp[3] = b.w;
      }
    } else {
      const int64_t mi = (crow * p.n_groups + g) * 2;
      float s0, z0;
      if (p.meta_f16) {
        const __half* m = static_cast<const __half*>(p.k_meta) + mi;
        s0 = __half2float(m[0]);
        z0 = __half2float(m[1]);
      } else {
        const float* m = static_cast<const float*>(p.k_meta) + mi;
        s0 = m[0];
        z0 = m[1];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) { st[i] = s0; zp[i] = z0; }
    }
    const uint8_t* cr = p.k_codes + crow * (D * p.bits / 8);
    uint32_t c0, c1, c2, c3;
    if (p.bits == 2) {
      const uint32_t v = cr[c4];
      c0 = v & 3u; c1 = (v >> 2) & 3u; c2 = (v >> 4) & 3u; c3 = v >> 6;
    } else {
      const uint32_t v = *reinterpret_cast<const uint16_t*>(cr + 2 * c4);
      c0 = v & 15u; c1 = (v >> 4) & 15u; c2 = (v >> 8) & 15u; c3 = v >> 12;
    }
    xq = make_float4(fmaf(st[0], static_cast<float>(c0), zp[0]), fmaf(st[1], static_cast<float>(c1), zp[1]),
                     fmaf(st[2], static_cast<float>(c2), zp[2]), fmaf(st[3], static_cast<float>(c3), zp[3]));
    if (kChan) {
      if (kk == 0) {
#pragma unroll
        for (int i = 0; i < 4; ++i) d2_s[4 * c4 + i] = st[i] * st[i];
      }
    } else if ((4 * c4) % p.group == 0) {
      d2_s[kk * kMaxGroups + g] = st[0] * st[0];
    }
  } else if (key < total) {
    xr = load_key4(p.K_cur, (static_cast<int64_t>(bh) * p.Lcur + (key - p.Lc)) * D + 4 * c4, f32);
    xq = xr;
  }
  *reinterpret_cast<float4*>(kr_s + kk * kPitch + 4 * c4) = xr;
  *reinterpret_cast<float4*>(kq_s + kk * kPitch + 4 * c4) = xq;
}

// Partial sums over channel quarter W of one row: (sum q_c^2 Delta_c^2, sum q_c^4 Delta_c^4), from
// the row's q pairs and the block's squared steps, in fp32x2.
template <int D, int W>
__device__ __forceinline__ float2 tile_partial(const float2 (&q)[D / 2], const float* d2_s) {
  const float2* d2p = reinterpret_cast<const float2*>(d2_s);
  float2 s2 = make_float2(0.f, 0.f), s4 = s2;
#pragma unroll
  for (int i = 0; i < D / 8; ++i) {
    const int c2 = (D / 8) * W + i;
    const float2 qq = __fmul2_rn(q[c2], q[c2]);
    const float2 t = __fmul2_rn(qq, d2p[c2]);
    s2 = __fadd2_rn(s2, t);
    s4 = __ffma2_rn(t, t, s4);
  }
  return make_float2(s2.x + s2.y, s4.x + s4.y);
}

// kChan: keys quantised per channel over blocks of p.key_block positions (a multiple of the 32-key
// tile, so a tile lies in one block): the correction of a row is the same for all cached keys of a
// tile, sum_c w_c Delta_c^2 (minus sum_c u_c Delta_c^4 for correct = 2), taken once per tile.
template <int D, bool kChan>
__global__ void __launch_bounds__(kThreadsF, 2) attention_fidelity_kernel(const FidelityParams p) {
  constexpr int kPitch = D + 4;
  __shared__ __align__(16) float tiles[2 * kKeysF * kPitch];
  __shared__ __align__(8) float d2_s[kChan ? D : kKeysF * kMaxGroups];  // squared steps of the cached keys
  __shared__ float2 part_s[kChan ? kSlices * kRowsF : 1];  // per-channel keys: partial corrections
  float* kr_s = tiles;                                    // reference (or current) keys
  float* kq_s = tiles + kKeysF * kPitch;                  // dequantised cached keys
  static_assert(2 * kKeysF * kPitch >= kSlices * kRowsF * (8 + 4 * kTop), "merge area");

  const int t = threadIdx.x;
  const int slice = t >> 5;          // warp: key slice
  const int lane = t & 31;           // query row within the CTA
  const int bh = blockIdx.y;
  const int b = bh / p.Hkv;
  const int h = bh - b * p.Hkv;
  const int64_t rows_total = static_cast<int64_t>(p.r) * p.Lq;
  const int64_t R = static_cast<int64_t>(blockIdx.x) * kRowsF + lane;
  const bool valid_row = R < rows_total;
  const int64_t hq = static_cast<int64_t>(h) * p.r + (valid_row ? R / p.Lq : 0);
  const int64_t qi = valid_row ? R % p.Lq : 0;
  const int64_t out_row = (static_cast<int64_t>(b) * p.Hq + hq) * p.Lq + qi;
  const bool f32 = p.in_f32 != 0;
  const int G = p.group, NG = p.n_groups;
  const int64_t total = p.Lc + p.Lcur;
  const int64_t lim_cur = p.causal ? qi + (p.Lcur - p.Lq) + 1 : p.Lcur;

  float2 q[D / 2];                   // (channel 2k, channel 2k + 1)
  float w[kMaxGroups] = {0.f, 0.f, 0.f, 0.f};
  float u[kMaxGroups] = {0.f, 0.f, 0.f, 0.f};
  {
    const uint8_t* qrow = static_cast<const uint8_t*>(p.Q) + out_row * D * (f32 ? 4 : 2);
#pragma unroll
    for (int c8 = 0; c8 < D / 8; ++c8) {
      float x[8];
      if (valid_row) {
        load_q8(qrow, f32, c8, x);
      } else {
#pragma unroll
        for (int k = 0; k < 8; ++k) x[k] = 0.f;
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) q[4 * c8 + k] = make_float2(x[2 * k], x[2 * k + 1]);
    }
    if (!kChan && valid_row && p.correct) query_group_powers<D>(qrow, f32, G, p.wcoef, p.ucoef, w, u);
  }

  Running ref{-INFINITY, 0.f, 0.f}, qnt{-INFINITY, 0.f, 0.f};
  float A = 0.f;                    // sum over keys of e^{s_ref - m_ref} (s_ref - s_q)
  TopList top_r, top_q;
  top_init(top_r);
  top_init(top_q);

  for (int64_t k0 = 0; k0 < total; k0 += kKeysF) {
    __syncthreads();
    if (kChan) {
#pragma unroll 1
      for (int e = t; e < kKeysF * (D / 4); e += kThreadsF)
        fill_key_chunk<D, kChan>(p, e, k0, total, bh, f32, kr_s, kq_s, d2_s);
    } else {
      for (int e = t; e < kKeysF * (D / 4); e += kThreadsF)
        fill_key_chunk<D, kChan>(p, e, k0, total, bh, f32, kr_s, kq_s, d2_s);
    }
    __syncthreads();
    // Per-channel keys: this row's correction for the tile, sum_c q_c^2 Delta_c^2 (and the fourth-
    // order sum_c q_c^4 Delta_c^4), each warp over a quarter of the channels, combined in smem.
    float tile_b = 0.f;
    if (kChan && p.correct && k0 < p.Lc) {
      float2 part;
      switch (slice) {
        case 0: part = tile_partial<D, 0>(q, d2_s); break;
        case 1: part = tile_partial<D, 1>(q, d2_s); break;
        case 2: part = tile_partial<D, 2>(q, d2_s); break;
        default: part = tile_partial<D, 3>(q, d2_s); break;
      }
      part_s[slice * kRowsF + lane] = part;
      __syncthreads();
      float s2 = 0.f, s4 = 0.f;
#pragma unroll
      for (int w = 0; w < kSlices; ++w) {
        s2 += part_s[w * kRowsF + lane].x;
        s4 += part_s[w * kRowsF + lane].y;
      }
      tile_b = p.wcoef * s2;
      if (p.correct == 2) tile_b = fmaf(-p.ucoef, s4, tile_b);
    }
#pragma unroll 1
    for (int kk = slice; kk < kKeysF; kk += kSlices) {
      const int64_t key = k0 + kk;
      if (key >= total) break;
      const bool cached = key < p.Lc;
      if (!cached && key - p.Lc >= lim_cur) continue;
      const float4* xr4 = reinterpret_cast<const float4*>(kr_s + kk * kPitch);
      float sr, sq;
      if (cached) {
        const float4* xq4 = reinterpret_cast<const float4*>(kq_s + kk * kPitch);
        float2 a0 = make_float2(0.f, 0.f), a1 = a0, b0 = a0, b1 = a0;
#pragma unroll
        for (int c4 = 0; c4 < D / 4; ++c4) {
          const float4 x = xr4[c4];
          const float4 y = xq4[c4];
          a0 = __ffma2_rn(q[2 * c4], make_float2(x.x, x.y), a0);
          a1 = __ffma2_rn(q[2 * c4 + 1], make_float2(x.z, x.w), a1);
          b0 = __ffma2_rn(q[2 * c4], make_float2(y.x, y.y), b0);
          b1 = __ffma2_rn(q[2 * c4 + 1], make_float2(y.z, y.w), b1);
        }
        sr = ((a0.x + a0.y) + (a1.x + a1.y)) * p.scale;
        sq = ((b0.x + b0.y) + (b1.x + b1.y)) * p.scale;
        if (kChan) {
          sq -= tile_b;
        } else if (p.correct) {
          float d2[kMaxGroups] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int g = 0; g < kMaxGroups; ++g)
            if (g < NG) d2[g] = d2_s[kk * kMaxGroups + g];
          sq -= jensen_term(w, d2, NG);
          if (p.correct == 2) {
#pragma unroll
            for (int g = 0; g < kMaxGroups; ++g)
              if (g < NG) sq = fmaf(u[g], d2[g] * d2[g], sq);
          }
        }
      } else {
        float2 a0 = make_float2(0.f, 0.f), a1 = a0;
#pragma unroll
        for (int c4 = 0; c4 < D / 4; ++c4) {
          const float4 x = xr4[c4];
          a0 = __ffma2_rn(q[2 * c4], make_float2(x.x, x.y), a0);
          a1 = __ffma2_rn(q[2 * c4 + 1], make_float2(x.z, x.w), a1);
        }
        sr = ((a0.x + a0.y) + (a1.x + a1.y)) * p.scale;
        sq = sr;
      }
      A *= rescale_to(ref, sr);
      const float pr = expf(sr - ref.m);
      ref.l += pr;
      if (cached) ref.lc += pr;
      A = fmaf(pr, sr - sq, A);
      rescale_to(qnt, sq);
      const float pq = expf(sq - qnt.m);
      qnt.l += pq;
      if (cached) qnt.lc += pq;
      const int j = static_cast<int>(key);
      top_insert(top_r, sr, j);
      top_insert(top_q, sq, j);
    }
  }

  // Merge the four warps' partial results of each row through shared memory (the key tiles are
  // no longer needed): per (slice, row) 8 floats of running sums, then both top lists.
  __syncthreads();
  float* mf = tiles;                                      // [kSlices][kRowsF][8]
  float* mv = tiles + kSlices * kRowsF * 8;               // [kSlices][kRowsF][2][kTop] scores
  int* mi = reinterpret_cast<int*>(mv + kSlices * kRowsF * 2 * kTop);   // same shape, indices
  if (slice != 0) {
    float* f = mf + (slice * kRowsF + lane) * 8;
    f[0] = ref.m; f[1] = ref.l; f[2] = ref.lc; f[3] = A;
    f[4] = qnt.m; f[5] = qnt.l; f[6] = qnt.lc;
    const int o = (slice * kRowsF + lane) * 2 * kTop;
#pragma unroll
    for (int i = 0; i < kTop; ++i) {
      mv[o + i] = top_r.v[i]; mi[o + i] = top_r.ix[i];
      mv[o + kTop + i] = top_q.v[i]; mi[o + kTop + i] = top_q.ix[i];
    }
  }
  __syncthreads();
  if (slice != 0) return;
#pragma unroll 1
  for (int sl = 1; sl < kSlices; ++sl) {
    const float* f = mf + (sl * kRowsF + lane) * 8;
    merge_running(ref, A, f[0], f[1], f[2], f[3]);
    float unused = 0.f;
    merge_running(qnt, unused, f[4], f[5], f[6], 0.f);
    const int o = (sl * kRowsF + lane) * 2 * kTop;
#pragma unroll
    for (int i = 0; i < kTop; ++i) {
      top_insert(top_r, mv[o + i], mi[o + i]);
      top_insert(top_q, mv[o + kTop + i], mi[o + kTop + i]);
    }
  }

  if (!valid_row) return;
  const bool any = ref.l > 0.f;
  float4 s0, s1;
  s0.x = any ? ref.m + logf(ref.l) : -INFINITY;
  s0.y = qnt.l > 0.f ? qnt.m + logf(qnt.l) : -INFINITY;
  s0.z = any ? ref.lc / ref.l : 0.f;
  s0.w = qnt.l > 0.f ? qnt.lc / qnt.l : 0.f;
  s1.x = any ? A / ref.l + (qnt.m - ref.m) + logf(qnt.l / ref.l) : 0.f;
  s1.y = top_r.ix[0] == top_q.ix[0] ? 1.f : 0.f;
  int n = 0, hit = 0;
#pragma unroll
  for (int i = 0; i < kTop; ++i) {
    if (top_r.ix[i] == kNoKey) continue;
    ++n;
#pragma unroll
    for (int k = 0; k < kTop; ++k) hit += top_r.ix[i] == top_q.ix[k];
  }
  s1.z = n ? static_cast<float>(hit) / static_cast<float>(n) : 1.f;
  s1.w = 0.f;
  float4* so = reinterpret_cast<float4*>(p.stats + out_row * kFidelityStats);
  so[0] = s0;
  so[1] = s1;
  if (p.top) {
    int32_t* to = p.top + out_row * 2 * kTop;
#pragma unroll
    for (int i = 0; i < kTop; ++i) {
      to[i] = top_r.ix[i] == kNoKey ? -1 : top_r.ix[i];
      to[kTop + i] = top_q.ix[i] == kNoKey ? -1 : top_q.ix[i];
    }
  }
}

template <int D>
cudaError_t launch_fid(const FidelityParams& p, cudaStream_t stream) {
  const int64_t rows = static_cast<int64_t>(p.r) * p.Lq;
  dim3 grid(static_cast<unsigned>((rows + kRowsF - 1) / kRowsF), static_cast<unsigned>(p.B * p.Hkv));
  if (p.key_block) attention_fidelity_kernel<D, true><<<grid, kThreadsF, 0, stream>>>(p);
  else attention_fidelity_kernel<D, false><<<grid, kThreadsF, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

int fidelity_rows_per_cta() { return kRowsF; }

cudaError_t launch_attention_fidelity(const FidelityParams& p, int d, cudaStream_t stream) {
  return d == 128 ? launch_fid<128>(p, stream) : launch_fid<64>(p, stream);
}

}  // namespace qkv
