// Jensen-bias-corrected chunk attention over the packed low-bit KV cache (sm_100a).
//
// Method (agents-report.net, "KV-Cache 量化導致的 Jensen 偏差", sections 方法 and 為何校正有效; the
// fugumt.com abstract of "Quantized Keys Steal Attention"): each query row attends, in one softmax,
// over the dequantised cached keys and the unquantised current chunk. Every cached-key score has
//     b_j = (scale^2 / 24) * sum_c q_c^2 * step_{j, c/group}^2
// subtracted before the softmax (the page's (1/(24 d)) sum_c q_c^2 Delta_{i,c}^2 at scale 1/sqrt d).
// The page asks for the dequantisation to be fused into the attention (hotelren.com blog, §4.3:
// unfused dequantisation cost latency and memory); here it happens tile by tile in shared memory.
//
// One CTA computes 128 packed query rows (the Hq/Hkv query heads of one KV head, row =
// head_in_group * Lq + i) against every key of its (batch, KV head). Warp roles:
//   warp 0     one lane issues bulk (TMA-engine) copies of packed cache tiles (codes and
//              step/zero-point of 128 keys, K and V) into a 2-stage ring;
//   warp 1     allocates tensor memory; one lane issues tcgen05.mma:
//                S = Q K^T   (A = Q bf16 in TMEM, B = K tile bf16 in smem, K-major, 128B swizzle)
//                O += P V    (A = P bf16 in TMEM, aliasing S; B = V tile in smem, MN-major)
//              and tcgen05.commit to the mbarriers below;
//   warps 2-5  dequantise packed tiles (or convert current-chunk tiles) into the bf16 K / V
//              operand tiles (2-slot rings, 128-byte swizzle) and write step^2 per (key, group);
//   warps 6-9  one query row per thread: load Q (fp32 group norms for the correction, bf16 copy
//              into TMEM), then per tile: read S from TMEM, scale, subtract the correction,
//              online softmax in base 2 with lazy rescaling of O, write P (bf16) back to TMEM;
//              finally O / l and LSE to global memory.
// Tensor memory (512 columns): O [0, d), Q [128, 128 + d/2), S0/P0 [256, 384), S1/P1 [384, 512).
// Every mbarrier wait is bounded; on timeout the CTA records QKV_ERR_TIMEOUT, drains its copies
// and MMAs, frees tensor memory and returns.
#include "qkv_common.cuh"
#include "qkv_internal.h"

namespace qkv {
namespace {

constexpr int kBM = 128;           // query rows per CTA (MMA M)
constexpr int kBN = 128;           // keys per tile (MMA N of S, K of PV)
constexpr int kThreads = 320;
constexpr int kStages = 2;         // packed-tile ring
constexpr float kRescaleThreshold = 8.0f;   // log2 units: O is rescaled only when the max grows by more
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0, kColQ = 128, kColS = 256;

// mbarrier indices
enum {
  B_PK_FULL = 0, B_PK_EMPTY = B_PK_FULL + kStages,
  B_KH_FULL = B_PK_EMPTY + kStages, B_KH_EMPTY = B_KH_FULL + 2,
  B_VH_FULL = B_KH_EMPTY + 2, B_VH_EMPTY = B_VH_FULL + 2,
  B_D2_FULL = B_VH_EMPTY + 2, B_D2_EMPTY = B_D2_FULL + 2,
  B_S_FULL = B_D2_EMPTY + 2, B_P_FULL = B_S_FULL + 2,
  B_PV_DONE = B_P_FULL + 2, B_Q_FULL = B_PV_DONE + 1, B_DRAIN = B_Q_FULL + 1,
  B_COUNT = B_DRAIN + 1
};

struct Layout {
  uint32_t kh, vh, pk, d2, bars, misc, total;
  uint32_t tile_bytes, stage_bytes, codes_bytes, meta_bytes;
};

__host__ __device__ inline Layout make_layout(int d, int bits, int n_groups, int meta_bytes) {
  Layout L;
  L.tile_bytes = kBN * d * 2;                                  // bf16 operand tile
  L.codes_bytes = kBN * d * bits / 8;                          // packed codes of one tile
  L.meta_bytes = kBN * n_groups * 2 * meta_bytes;              // (step, zp) of one tile
  L.stage_bytes = (2 * (L.codes_bytes + L.meta_bytes) + 127) & ~127u;
  L.kh = 0;
  L.vh = L.kh + 2 * L.tile_bytes;
  L.pk = L.vh + 2 * L.tile_bytes;
  L.d2 = L.pk + kStages * L.stage_bytes;
  L.bars = L.d2 + 2 * kBN * 4 * 4;
  L.misc = L.bars + B_COUNT * 8;
  L.total = L.misc + 16;
  return L;
}

// Group squared norms of one query row, times `coef`: w[g] = coef * sum_{c in g} q_c^2 (fp32, in
// channel order). Shared with the correction-only kernel below.
template <int D>
__device__ __forceinline__ void query_group_weights(const void* qrow, bool f32, int group,
                                                    float coef, float (&w)[4]) {
#pragma unroll
  for (int g = 0; g < 4; ++g) w[g] = 0.f;
#pragma unroll
  for (int c8 = 0; c8 < D / 8; ++c8) {
    float x[8];
    if (f32) {
      const float4 a = reinterpret_cast<const float4*>(qrow)[2 * c8];
      const float4 b = reinterpret_cast<const float4*>(qrow)[2 * c8 + 1];
      x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
    } else {
      const uint4 u = reinterpret_cast<const uint4*>(qrow)[c8];
      x[0] = bf16_lo(u.x); x[1] = bf16_hi(u.x); x[2] = bf16_lo(u.y); x[3] = bf16_hi(u.y);
      x[4] = bf16_lo(u.z); x[5] = bf16_hi(u.z); x[6] = bf16_lo(u.w); x[7] = bf16_hi(u.w);
    }
    const int g = (c8 * 8) / group;
    float acc = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) acc = fmaf(x[k], x[k], acc);
#pragma unroll
    for (int gg = 0; gg < 4; ++gg)
      if (gg == g) w[gg] += acc;
  }
#pragma unroll
  for (int g = 0; g < 4; ++g) w[g] *= coef;
}

// The correction of one (query, key) pair: sum_g w[g] * step_g^2.
__device__ __forceinline__ float jensen_term(const float (&w)[4], const float4 d2, int n_groups) {
  float b = w[0] * d2.x;
  if (n_groups > 1) b = fmaf(w[1], d2.y, b);
  if (n_groups > 2) {
    b = fmaf(w[2], d2.z, b);
    b = fmaf(w[3], d2.w, b);
  }
  return b;
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Dequantises 32 consecutive channels of one key: 8 (INT2) or 16 (INT4) code bytes -> 16 bf16x2.
// x_hat = zp + step * code, evaluated as one fp32 FMA on a float whose mantissa holds the code
// (1 + code * 2^-k) so no integer-to-float conversion is needed, then rounded to bf16.
template <int BITS>
__device__ __forceinline__ void dequant32(const uint8_t* codes, float step, float zp,
                                          uint32_t (&out)[16]) {
  if constexpr (BITS == 2) {
    const uint2 w2 = *reinterpret_cast<const uint2*>(codes);
    const float s16 = step * 16.f, s4 = step * 4.f;
    const float c16 = zp - s16, c4 = zp - s4;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t w = h ? w2.y : w2.x;   // 16 codes, code k at bits 2k
#pragma unroll
      for (int p = 0; p < 8; ++p) {
        const int sh = 19 - 4 * p;          // low code of the pair -> bits 19-20, high -> 21-22
        const uint32_t s = sh >= 0 ? (w << sh) : (w >> (-sh));
        const float lo = __uint_as_float((s & (3u << 19)) | 0x3F800000u);   // 1 + c/16
        const float hi = __uint_as_float((s & (3u << 21)) | 0x3F800000u);   // 1 + c/4
        out[h * 8 + p] = pack_bf16x2(fmaf(s16, lo, c16), fmaf(s4, hi, c4));
      }
    }
  } else {
    const uint4 w4 = *reinterpret_cast<const uint4*>(codes);
    const float s256 = step * 256.f, s16 = step * 16.f;
    const float c256 = zp - s256, c16 = zp - s16;
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const uint32_t w = h == 0 ? w4.x : h == 1 ? w4.y : h == 2 ? w4.z : w4.w;  // 8 codes at 4k
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const int sh = 15 - 8 * p;          // low code -> bits 15-18, high -> 19-22
        const uint32_t s = sh >= 0 ? (w << sh) : (w >> (-sh));
        const float lo = __uint_as_float((s & (0xFu << 15)) | 0x3F800000u);  // 1 + c/256
        const float hi = __uint_as_float((s & (0xFu << 19)) | 0x3F800000u);  // 1 + c/16
        out[h * 4 + p] = pack_bf16x2(fmaf(s256, lo, c256), fmaf(s16, hi, c16));
      }
    }
  }
}

// Stores 32 channels (16 bf16x2) of key `key` at channel block `blk` into a [d/64][128][64]
// bf16 tile with the 128-byte swizzle.
template <int D>
__device__ __forceinline__ void store32(uint8_t* tile, int key, int blk, const uint32_t (&v)[16]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int c = blk * 4 + i;               // 16-byte chunk of the row (8 channels)
    uint8_t* dst = tile + (c >> 3) * (kBN * 128) + sw128_offset(key, c & 7);
    *reinterpret_cast<uint4*>(dst) = make_uint4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
  }
}

// Dequantises one packed tile (128 keys) into a bf16 operand tile; keys >= valid are zero.
// When d2 is given, also writes step^2 for every (key, group) (0 beyond valid).
template <int D, int BITS>
__device__ __forceinline__ void dequant_tile(const uint8_t* codes, const uint8_t* meta,
                                             bool meta_f16, int group, int n_groups,
                                             uint8_t* tile, int valid, float* d2, int t) {
  constexpr int kTPK = D / 32;               // threads per key
  constexpr int kKPP = 128 / kTPK;           // keys per pass
  const int blk = t % kTPK;
  const int g = (blk * 32) / group;
  const bool first_of_group = ((blk * 32) % group) == 0;
#pragma unroll 1
  for (int pass = 0; pass < kBN / kKPP; ++pass) {
    const int key = pass * kKPP + t / kTPK;
    uint32_t v[16];
    float step = 0.f;
    if (key < valid) {
      float zp;
      if (meta_f16) {
        const __half2 m = reinterpret_cast<const __half2*>(meta)[key * n_groups + g];
        step = __low2float(m);
        zp = __high2float(m);
      } else {
        const float2 m = reinterpret_cast<const float2*>(meta)[key * n_groups + g];
        step = m.x;
        zp = m.y;
      }
      dequant32<BITS>(codes + key * (D * BITS / 8) + blk * (32 * BITS / 8), step, zp, v);
    } else {
#pragma unroll
      for (int k = 0; k < 16; ++k) v[k] = 0u;
    }
    store32<D>(tile, key, blk, v);
    if (d2 != nullptr && first_of_group) d2[key * 4 + g] = step * step;
  }
}

// Converts one current-chunk tile (rows t0.., `valid` of them) into a bf16 operand tile.
template <int D>
__device__ __forceinline__ void convert_tile(const void* src_rows, bool f32, uint8_t* tile,
                                             int valid, int t) {
  constexpr int kTPK = D / 32;
  constexpr int kKPP = 128 / kTPK;
  const int blk = t % kTPK;
#pragma unroll 1
  for (int pass = 0; pass < kBN / kKPP; ++pass) {
    const int key = pass * kKPP + t / kTPK;
    uint32_t v[16];
    if (key < valid) {
      if (f32) {
        const float4* s = reinterpret_cast<const float4*>(src_rows) + (key * D + blk * 32) / 4;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float4 a = s[i];
          v[2 * i] = pack_bf16x2(a.x, a.y);
          v[2 * i + 1] = pack_bf16x2(a.z, a.w);
        }
      } else {
        const uint4* s = reinterpret_cast<const uint4*>(src_rows) + (key * D + blk * 32) / 8;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint4 a = s[i];
          v[4 * i] = a.x; v[4 * i + 1] = a.y; v[4 * i + 2] = a.z; v[4 * i + 3] = a.w;
        }
      }
    } else {
#pragma unroll
      for (int k = 0; k < 16; ++k) v[k] = 0u;
    }
    store32<D>(tile, key, blk, v);
  }
}

template <int D, int BITS>
__global__ void __launch_bounds__(kThreads, 1) corrected_attention_kernel(const AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const Layout L = make_layout(D, BITS, p.n_groups, p.meta_f16 ? 2 : 4);
  const uint32_t bar0 = smem_u32(smem + L.bars);
  auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L.misc);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L.misc + 4);
  float* d2s = reinterpret_cast<float*>(smem + L.d2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m_tile = blockIdx.x;
  const int bh = blockIdx.y;
  const int b = bh / p.Hkv;
  const int h = bh - b * p.Hkv;
  const int64_t rows_total = static_cast<int64_t>(p.r) * p.Lq;

  // Tiles: cached ones first, then current ones (causal: only those some row of this CTA sees).
  const int Tc = static_cast<int>((p.Lc + kBN - 1) / kBN);
  int64_t cur_keys = p.Lcur;
  if (p.causal) {
    const int64_t R0 = static_cast<int64_t>(m_tile) * kBM;
    const int64_t R1 = (R0 + kBM < rows_total ? R0 + kBM : rows_total) - 1;
    const int64_t max_i = (R0 / p.Lq != R1 / p.Lq) ? p.Lq - 1 : R1 % p.Lq;
    const int64_t lim = max_i + 1 + (p.Lcur - p.Lq);
    cur_keys = lim < 0 ? 0 : (lim < p.Lcur ? lim : p.Lcur);
  }
  const int Tn = static_cast<int>((cur_keys + kBN - 1) / kBN);
  const int T = Tc + Tn;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int i = 0; i < B_COUNT; ++i) {
      uint32_t cnt = 1;
      if (i == B_PK_EMPTY || i == B_PK_EMPTY + 1 || i == B_KH_FULL || i == B_KH_FULL + 1 ||
          i == B_VH_FULL || i == B_VH_FULL + 1 || i == B_D2_FULL || i == B_D2_FULL + 1 ||
          i == B_D2_EMPTY || i == B_D2_EMPTY + 1 || i == B_P_FULL || i == B_P_FULL + 1 ||
          i == B_Q_FULL)
        cnt = 4;   // one arrival per warp of a 4-warp group
      mbar_init(bar(i), cnt);
    }
    mbar_init_fence();
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------------- bulk-copy producer
    if (lane == 0) {
      const int64_t row_codes = D * BITS / 8;
      const int64_t row_meta = static_cast<int64_t>(p.n_groups) * 2 * (p.meta_f16 ? 2 : 4);
      int issued = 0;
      for (int jc = 0; jc < Tc; ++jc) {
        const int s = jc % kStages, k = jc / kStages;
        if (!mbar_wait(bar(B_PK_EMPTY + s), (k & 1) ^ 1, abort_flag, p.status)) break;
        const uint32_t dst = smem_u32(smem + L.pk + s * L.stage_bytes);
        const int64_t row0 = static_cast<int64_t>(bh) * p.capacity + static_cast<int64_t>(jc) * kBN;
        mbar_arrive_expect_tx(bar(B_PK_FULL + s), 2 * (L.codes_bytes + L.meta_bytes));
        bulk_g2s(dst, p.k_codes + row0 * row_codes, L.codes_bytes, bar(B_PK_FULL + s));
        bulk_g2s(dst + L.codes_bytes,
                 static_cast<const uint8_t*>(p.k_meta) + row0 * row_meta, L.meta_bytes,
                 bar(B_PK_FULL + s));
        bulk_g2s(dst + L.codes_bytes + L.meta_bytes, p.v_codes + row0 * row_codes, L.codes_bytes,
                 bar(B_PK_FULL + s));
        bulk_g2s(dst + 2 * L.codes_bytes + L.meta_bytes,
                 static_cast<const uint8_t*>(p.v_meta) + row0 * row_meta, L.meta_bytes,
                 bar(B_PK_FULL + s));
        ++issued;
      }
      // Never leave the CTA with copies in flight: wait for the last use of every stage.
      for (int s = 0; s < kStages && s < issued; ++s) {
        const int last = ((issued - 1 - s) / kStages) * kStages + s;
        mbar_wait_drain(bar(B_PK_FULL + s), (last / kStages) & 1);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kBM, kBN, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kBM, D, 0, 1);
      const uint32_t tm_q = tmem + kColQ, tm_o = tmem + kColO;
      auto issue_pv = [&](int i) -> bool {
        const int sb = i & 1, n = i >> 1;
        if (!mbar_wait(bar(B_P_FULL + sb), n & 1, abort_flag, p.status)) return false;
        if (!mbar_wait(bar(B_VH_FULL + sb), n & 1, abort_flag, p.status)) return false;
        tc_fence_after();
        const uint32_t vbase = smem_u32(smem + L.vh + sb * L.tile_bytes);
        const uint32_t tm_p = tmem + kColS + 128u * sb;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          // V tile [d/64][128 keys][64] with the 128B swizzle, MN-major: 16 keys per step
          // (2 x 1024-byte atoms), LBO = next 64 channels, SBO = next 8 keys.
          const uint64_t desc = smem_desc_sw128(vbase + kk * 2048u, kBN * 128u, 1024u);
          mma_ts(tm_o, tm_p + kk * 8u, desc, idesc_pv, (i > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(bar(B_VH_EMPTY + sb));
        tc_commit(bar(B_PV_DONE));
        return true;
      };
      bool ok = T > 0 && mbar_wait(bar(B_Q_FULL), 0, abort_flag, p.status);
      if (ok) {
        tc_fence_after();
        for (int j = 0; j < T && ok; ++j) {
          const int sb = j & 1, n = j >> 1;
          if (!mbar_wait(bar(B_KH_FULL + sb), n & 1, abort_flag, p.status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t kbase = smem_u32(smem + L.kh + sb * L.tile_bytes);
          const uint32_t tm_s = tmem + kColS + 128u * sb;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            // K tile [d/64][128 keys][64] with the 128B swizzle, K-major: 16 channels per step
            // (32 bytes inside the swizzle row), SBO = next 8 keys.
            const uint32_t addr = kbase + (kk >> 2) * (kBN * 128u) + (kk & 3) * 32u;
            const uint64_t desc = smem_desc_sw128(addr, 16u, 1024u);
            mma_ts(tm_s, tm_q + kk * 8u, desc, idesc_qk, kk > 0 ? 1u : 0u);
          }
          tc_commit(bar(B_KH_EMPTY + sb));
          tc_commit(bar(B_S_FULL + sb));
          if (j >= 1) ok = issue_pv(j - 1);
        }
        if (ok) issue_pv(T - 1);
      }
      // Never free tensor memory under a running MMA.
      tc_commit(bar(B_DRAIN));
      mbar_wait_drain(bar(B_DRAIN), 0);
    }
  } else if (warp < 6) {
    // ---------------------------------------------------------------- dequantise / convert
    const int t = threadIdx.x - 64;
    const bool f32 = p.in_f32 != 0;
    for (int j = 0; j < T; ++j) {
      const int sb = j & 1, n = j >> 1;
      uint8_t* kt = smem + L.kh + sb * L.tile_bytes;
      uint8_t* vt = smem + L.vh + sb * L.tile_bytes;
      if (j < Tc) {
        const int s = j % kStages, k = j / kStages;
        const int valid = static_cast<int>(p.Lc - static_cast<int64_t>(j) * kBN < kBN
                                               ? p.Lc - static_cast<int64_t>(j) * kBN
                                               : kBN);
        const uint8_t* st = smem + L.pk + s * L.stage_bytes;
        if (!warp_wait(bar(B_PK_FULL + s), k & 1, abort_flag, p.status)) break;
        if (!warp_wait(bar(B_KH_EMPTY + sb), (n & 1) ^ 1, abort_flag, p.status)) break;
        float* d2 = nullptr;
        if (p.correct) {
          if (!warp_wait(bar(B_D2_EMPTY + sb), (n & 1) ^ 1, abort_flag, p.status)) break;
          d2 = d2s + sb * (kBN * 4);
        }
        dequant_tile<D, BITS>(st, st + L.codes_bytes, p.meta_f16, p.group, p.n_groups, kt, valid,
                              d2, t);
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(bar(B_KH_FULL + sb));
          if (p.correct) mbar_arrive(bar(B_D2_FULL + sb));
        }
        if (!warp_wait(bar(B_VH_EMPTY + sb), (n & 1) ^ 1, abort_flag, p.status)) break;
        dequant_tile<D, BITS>(st + L.codes_bytes + L.meta_bytes, st + 2 * L.codes_bytes + L.meta_bytes,
                              p.meta_f16, p.group, p.n_groups, vt, valid, nullptr, t);
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(bar(B_VH_FULL + sb));
          mbar_arrive(bar(B_PK_EMPTY + s));
        }
      } else {
        const int64_t t0 = static_cast<int64_t>(j - Tc) * kBN;
        const int valid = static_cast<int>(cur_keys - t0 < kBN ? cur_keys - t0 : kBN);
        const size_t esz = f32 ? 4 : 2;
        const int64_t row0 = static_cast<int64_t>(bh) * p.Lcur + t0;
        if (!warp_wait(bar(B_KH_EMPTY + sb), (n & 1) ^ 1, abort_flag, p.status)) break;
        convert_tile<D>(static_cast<const uint8_t*>(p.K_cur) + row0 * D * esz, f32, kt, valid, t);
        fence_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_KH_FULL + sb));
        if (!warp_wait(bar(B_VH_EMPTY + sb), (n & 1) ^ 1, abort_flag, p.status)) break;
        convert_tile<D>(static_cast<const uint8_t*>(p.V_cur) + row0 * D * esz, f32, vt, valid, t);
        fence_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_VH_FULL + sb));
      }
    }
  } else {
    // ---------------------------------------------------------------- softmax / epilogue
    const int quad = warp & 3;                 // TMEM lane quadrant of this warp
    const int row = quad * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const int64_t R = static_cast<int64_t>(m_tile) * kBM + row;
    const bool valid_row = R < rows_total;
    const int64_t hq = static_cast<int64_t>(h) * p.r + (valid_row ? R / p.Lq : 0);
    const int64_t qi = valid_row ? R % p.Lq : 0;
    const int64_t out_row = (static_cast<int64_t>(b) * p.Hq + hq) * p.Lq + qi;
    const bool f32 = p.in_f32 != 0;
    const size_t esz = f32 ? 4 : 2;

    // Q row: fp32 group weights for the correction (log2 units) and a bf16 copy into TMEM.
    float w[4] = {0.f, 0.f, 0.f, 0.f};
    {
      uint32_t qp[D / 2];
      const uint8_t* qrow = static_cast<const uint8_t*>(p.Q) + out_row * D * esz;
      if (valid_row) {
        query_group_weights<D>(qrow, f32, p.group, p.wcoef_log2, w);
#pragma unroll
        for (int c8 = 0; c8 < D / 8; ++c8) {
          if (f32) {
            const float4 a = reinterpret_cast<const float4*>(qrow)[2 * c8];
            const float4 bq = reinterpret_cast<const float4*>(qrow)[2 * c8 + 1];
            qp[4 * c8] = pack_bf16x2(a.x, a.y); qp[4 * c8 + 1] = pack_bf16x2(a.z, a.w);
            qp[4 * c8 + 2] = pack_bf16x2(bq.x, bq.y); qp[4 * c8 + 3] = pack_bf16x2(bq.z, bq.w);
          } else {
            const uint4 u = reinterpret_cast<const uint4*>(qrow)[c8];
            qp[4 * c8] = u.x; qp[4 * c8 + 1] = u.y; qp[4 * c8 + 2] = u.z; qp[4 * c8 + 3] = u.w;
          }
        }
      } else {
#pragma unroll
        for (int k = 0; k < D / 2; ++k) qp[k] = 0u;
      }
#pragma unroll
      for (int c = 0; c < D / 2; c += 32) {
        uint32_t chunk[32];
#pragma unroll
        for (int k = 0; k < 32; ++k) chunk[k] = qp[c + k];
        tmem_st32(tmem + lane_off + kColQ + c, chunk);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_Q_FULL));
    }

    float m_run = -INFINITY;   // max used for the exponentials so far (log2 units)
    float l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < T && ok; ++j) {
      const int sb = j & 1, n = j >> 1;
      const bool cached = j < Tc;
      if (!warp_wait(bar(B_S_FULL + sb), n & 1, abort_flag, p.status)) { ok = false; break; }
      tc_fence_after();
      const uint32_t tm_s = tmem + lane_off + kColS + 128u * sb;
      float s[kBN];
#pragma unroll
      for (int c = 0; c < kBN; c += 32) {
        uint32_t r[32];
        tmem_ld32(tm_s + c, r);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 32; ++k) s[c + k] = __uint_as_float(r[k]);
      }
      float m_tile = -INFINITY;
      if (cached) {
        const int valid = static_cast<int>(p.Lc - static_cast<int64_t>(j) * kBN < kBN
                                               ? p.Lc - static_cast<int64_t>(j) * kBN
                                               : kBN);
        if (p.correct) {
          if (!warp_wait(bar(B_D2_FULL + sb), n & 1, abort_flag, p.status)) { ok = false; break; }
          const float4* d2 = reinterpret_cast<const float4*>(d2s + sb * (kBN * 4));
#pragma unroll
          for (int k = 0; k < kBN; ++k) {
            const float tk = fmaf(s[k], p.scale_log2, -jensen_term(w, d2[k], p.n_groups));
            s[k] = k < valid ? tk : -INFINITY;
            m_tile = fmaxf(m_tile, s[k]);
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(B_D2_EMPTY + sb));
        } else {
#pragma unroll
          for (int k = 0; k < kBN; ++k) {
            s[k] = k < valid ? s[k] * p.scale_log2 : -INFINITY;
            m_tile = fmaxf(m_tile, s[k]);
          }
        }
      } else {
        const int64_t t0 = static_cast<int64_t>(j - Tc) * kBN;
        int64_t lim = cur_keys - t0;                       // keys of this tile that exist
        if (p.causal) {
          const int64_t c = qi + (p.Lcur - p.Lq) - t0 + 1;  // keys this row may see
          lim = c < lim ? c : lim;
        }
        const int valid = static_cast<int>(lim < 0 ? 0 : (lim < kBN ? lim : kBN));
#pragma unroll
        for (int k = 0; k < kBN; ++k) {
          s[k] = k < valid ? s[k] * p.scale_log2 : -INFINITY;
          m_tile = fmaxf(m_tile, s[k]);
        }
      }
      // Lazy rescaling: keep the old max unless the new one exceeds it by the threshold.
      const bool need = (m_tile > m_run + kRescaleThreshold) ||
                        (m_run == -INFINITY && m_tile > -INFINITY);
      float factor = 1.f;
      if (need) {
        factor = ex2(m_run - m_tile);    // 0 when m_run = -inf
        l_run *= factor;
        m_run = m_tile;
      }
      const float m_use = m_run == -INFINITY ? 0.f : m_run;
      float psum = 0.f;
#pragma unroll
      for (int c = 0; c < kBN; c += 64) {
        uint32_t pk[32];
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          const float p0 = ex2(s[c + 2 * k] - m_use);
          const float p1 = ex2(s[c + 2 * k + 1] - m_use);
          psum += p0 + p1;
          pk[k] = pack_bf16x2(p0, p1);
        }
        tmem_st32(tm_s + c / 2, pk);
      }
      l_run += psum;
      if (j > 0) {
        // O must not be touched while the previous P.V is in flight.
        if (!warp_wait(bar(B_PV_DONE), (j - 1) & 1, abort_flag, p.status)) { ok = false; break; }
        tc_fence_after();
        if (__any_sync(0xffffffffu, need)) {
          const uint32_t tm_o = tmem + lane_off + kColO;
#pragma unroll
          for (int c = 0; c < D; c += 32) {
            uint32_t r[32];
            tmem_ld32(tm_o + c, r);
            tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 32; ++k) r[k] = __float_as_uint(__uint_as_float(r[k]) * factor);
            tmem_st32(tm_o + c, r);
          }
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_P_FULL + sb));
    }

    // Epilogue: O / l and LSE.
    bool have_o = false;
    if (ok && T > 0) {
      have_o = warp_wait(bar(B_PV_DONE), (T - 1) & 1, abort_flag, p.status);
      tc_fence_after();
    }
    const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
    uint8_t* orow = static_cast<uint8_t*>(p.O) + out_row * D * esz;
#pragma unroll
    for (int c = 0; c < D; c += 32) {
      uint32_t r[32];
      if (have_o) {
        tmem_ld32(tmem + lane_off + kColO + c, r);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int k = 0; k < 32; ++k) r[k] = 0u;
      }
      if (valid_row) {
        if (f32) {
          float4* dst = reinterpret_cast<float4*>(orow) + c / 4;
#pragma unroll
          for (int k = 0; k < 8; ++k)
            dst[k] = make_float4(__uint_as_float(r[4 * k]) * inv_l, __uint_as_float(r[4 * k + 1]) * inv_l,
                                 __uint_as_float(r[4 * k + 2]) * inv_l, __uint_as_float(r[4 * k + 3]) * inv_l);
        } else {
          uint4* dst = reinterpret_cast<uint4*>(orow) + c / 8;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            uint32_t o4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
              o4[e] = pack_bf16x2(__uint_as_float(r[8 * k + 2 * e]) * inv_l,
                                  __uint_as_float(r[8 * k + 2 * e + 1]) * inv_l);
            dst[k] = make_uint4(o4[0], o4[1], o4[2], o4[3]);
          }
        }
      }
    }
    if (valid_row) {
      const float m_use = m_run == -INFINITY ? 0.f : m_run;
      p.LSE[out_row] = l_run > 0.f ? (m_use + __log2f(l_run)) * 0.69314718055994530942f : -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
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
  float w[4];
  query_group_weights<D>(static_cast<const uint8_t*>(p.Q) + qrow * D * esz, p.in_f32 != 0, p.group,
                         p.wcoef, w);
  const int64_t key = (b * p.Hkv + hkv) * p.capacity + j;
  float st[4] = {0.f, 0.f, 0.f, 0.f};
  for (int g = 0; g < p.n_groups; ++g) {
    const float s = p.meta_f16
                        ? __half2float(static_cast<const __half*>(p.k_meta)[(key * p.n_groups + g) * 2])
                        : static_cast<const float*>(p.k_meta)[(key * p.n_groups + g) * 2];
    st[g] = s * s;
  }
  p.bias[qrow * p.Lc + j] = jensen_term(w, make_float4(st[0], st[1], st[2], st[3]), p.n_groups);
}

template <int D, int BITS>
cudaError_t launch_impl(const AttnParams& p, cudaStream_t stream) {
  const size_t smem = attention_smem_bytes(D, BITS, p.n_groups, p.meta_f16 ? 2 : 4);
  cudaError_t e = cudaFuncSetAttribute(corrected_attention_kernel<D, BITS>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int64_t rows = static_cast<int64_t>(p.r) * p.Lq;
  dim3 grid(static_cast<unsigned>((rows + kBM - 1) / kBM), static_cast<unsigned>(p.B * p.Hkv));
  corrected_attention_kernel<D, BITS><<<grid, kThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

// At least 116 KB so that two CTAs never share an SM: each holds all 512 tensor-memory columns.
size_t attention_smem_bytes(int d, int bits, int n_groups, int meta_bytes) {
  const size_t need = make_layout(d, bits, n_groups, meta_bytes).total + 1024;
  return need > 116u * 1024u ? need : 116u * 1024u;
}

cudaError_t launch_attention(const AttnParams& p, int d, int bits, cudaStream_t stream) {
  if (d == 128) return bits == 2 ? launch_impl<128, 2>(p, stream) : launch_impl<128, 4>(p, stream);
  return bits == 2 ? launch_impl<64, 2>(p, stream) : launch_impl<64, 4>(p, stream);
}

cudaError_t launch_jensen_bias(const BiasParams& p, cudaStream_t stream) {
  dim3 grid(static_cast<unsigned>(p.B * p.Hq * p.Lq), static_cast<unsigned>((p.Lc + 255) / 256));
  if (p.d == 128) jensen_bias_kernel<128><<<grid, 256, 0, stream>>>(p);
  else jensen_bias_kernel<64><<<grid, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace qkv
