// Jensen-bias-corrected chunk attention over a cache whose keys are quantised per channel along
// tokens (KIVI's key grouping, named in agents-report.net, "KV-Cache 量化導致的 Jensen 偏差", section
// 跨主題對比分析; the hotelren.com blog, section 3.1, groups along the sequence axis), on the tensor
// cores, bf16 inputs, d = 128, sm_100a.
//
// Every T consecutive cache positions of one (batch, KV head, channel) share one step and
// zero-point, so the per-token code-domain identity of the 128-row kernel does not apply (its scale
// a_jg multiplies a whole group of one key; here every channel has its own). The keys are therefore
// dequantised in fp32, x_hat = zp_c + step_c * code, and split into two bf16 tiles, high and low
// (x_hat = hi + lo to ~2^-14 relative): S = Q K_hi^T + Q K_lo^T in one fp32 accumulator, two
// chains of eight 128 x 128 x 16 MMAs with both operands in shared memory. The correction of the
// Jensen-bias pages (agents-report.net, section 方法) is the same for all keys of a block:
// b = (scale^2 / 24) sum_c q_c^2 step_c^2, taken for the 128 / T blocks of a tile by MMAs of
// N = 16: q^2 as an exact pair of bf16 parts (in tensor memory) against the blocks' scaled squared
// steps, also split in two (rows blk and 4 + blk of the operand), so that b is accurate to ~2^-16
// relative; a single bf16 rounding of each factor moved the log-sum-exp by up to 3e-3 on inputs
// with outlier channels. The softmax forms scale * S - b with one FMA per score; the rest (online
// softmax over the cached and current keys, P.V with V dequantised per token, O / l, LSE) is the
// 128-row kernel's.
//
// One CTA per 128 packed query rows (row = head_in_group * Lq + i) of one (batch, KV head), 128-key
// tiles; warp roles as in the 128-row kernel:
//   warp 0       tensor memory, and one thread issuing S_j (hi and lo chains, the correction chain)
//                and then P_{j-1} V_{j-1}.
//   warps 1-3, WG4  K hi / lo tiles (natural channel order), one buffer, and the scaled squared steps
//                of the tile's blocks; for current tiles a copy of K_cur (lo = 0, no correction).
//   WG1, WG2     softmax: Q into shared memory, q^2 into tensor memory; per tile S and the
//                correction, online
//                softmax in base 2 with lazy rescaling, P (bf16) into tensor memory; O / l, LSE.
//   WG3          V tiles, dequantised per token; one lane issues the bulk copies of packed tiles.
// Tensor memory: O [0, 128), q^2 high part [128, 192), P [192, 256), S [256, 384), q^2 low part
// [384, 448), correction [448, 464). Q is an operand in shared memory so that both parts of q^2 fit.
// Every mbarrier wait is bounded (QKV_ERR_TIMEOUT), as in the 128-row kernel.
#include "channel.h"
#include "qkv_common.cuh"
#include "qkv_internal.h"
#include "tile_ops.cuh"

namespace qkv {
namespace {

constexpr int D = 128;
constexpr int kBM = 128;                      // query rows per CTA (MMA M)
constexpr int kN = 128;                       // keys per tile
constexpr int kThreads = 640;
constexpr int kKThreads = 224;                // K producers: warps 1-3 and warpgroup 4
// Registers per thread after setmaxnreg: 2 * 128 * 128 + 3 * 128 * 72 = 60416 <= 640 * 96, the
// block's allocation at launch (the producers' dequantisation spills at 64).
constexpr int kRegProducer = 72, kRegSoftmax = 128;
constexpr int kStagesMax = 3;                // packed-tile ring (INT2: 3 stages, INT4: 2)
constexpr float kRescaleThreshold = 8.0f;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0, kColQ2H = 128, kColP = 192, kColS = 256, kColQ2L = 384, kColC = 448;
// Rows of the squared-step operand: blk (high part), 4 + blk (low part), the rest zero.
constexpr int kCRows = 16;

enum {
  B_PK_FULL = 0, B_PK_EMPTY = B_PK_FULL + kStagesMax,
  B_KH_FULL = B_PK_EMPTY + kStagesMax, B_KH_EMPTY = B_KH_FULL + 2,   // per 64-channel half
  B_VH_FULL = B_KH_EMPTY + 2, B_VH_EMPTY = B_VH_FULL + 2,
  B_S_FULL = B_VH_EMPTY + 2, B_S_FREE = B_S_FULL + 1,
  B_P_FULL = B_S_FREE + 1, B_PV_DONE = B_P_FULL + 1,
  B_Q_FULL = B_PV_DONE + 1, B_DRAIN = B_Q_FULL + 1,
  B_COUNT = B_DRAIN + 1
};

template <int BITS, int NGV>
struct CCfg {
  static constexpr int GV = D / NGV;                      // value channels per group
  static constexpr uint32_t kTile = kN * D * 2;           // bf16 operand tile
  static constexpr uint32_t kCodes = kN * D * BITS / 8;   // packed codes of one tile
  static constexpr uint32_t kDblk = kN * 128;             // bytes between 64-channel blocks
  static constexpr uint32_t kCTile = kCRows * D * 2;      // squared steps [D/64][16][64]
  static constexpr int kStages = BITS == 2 ? 3 : 2;       // packed-tile ring
};

struct CLayout {
  uint32_t khi, klo, vt, qs, ct, pk, xc, bars, misc, total, stage, kmeta, vmeta;
};

template <int BITS, int NGV>
__host__ __device__ inline CLayout make_clayout(int meta_bytes, int T) {
  using C = CCfg<BITS, NGV>;
  CLayout L;
  L.kmeta = (kN / T) * D * 2 * meta_bytes;               // (step, zp) per channel of each block
  L.vmeta = kN * NGV * 2 * meta_bytes;                   // per token and value group
  L.stage = (2 * C::kCodes + L.kmeta + L.vmeta + 127) & ~127u;
  L.khi = 0;
  L.klo = L.khi + C::kTile;
  L.vt = L.klo + C::kTile;
  L.qs = L.vt + 2 * C::kTile;                             // Q [D/64][128 rows][64], 128B swizzle
  L.ct = L.qs + kBM * D * 2;
  L.pk = L.ct + C::kCTile;
  L.xc = L.pk + C::kStages * L.stage;          // row-max exchange [2][2][128] and row-sum [2][128]
  L.bars = L.xc + (4 + 2) * kBM * 4;
  L.misc = L.bars + B_COUNT * 8;
  L.total = L.misc + 16;
  return L;
}

// (step, zero-point) of 8 consecutive channels of a block's meta [D][2].
template <bool F16>
__device__ __forceinline__ void meta8(const uint8_t* meta, int c0, float (&st)[8], float (&zp)[8]) {
  if (F16) {
    const uint4 a = *reinterpret_cast<const uint4*>(meta + c0 * 4);
    const uint4 b = *reinterpret_cast<const uint4*>(meta + c0 * 4 + 16);
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const __half2 h = *reinterpret_cast<const __half2*>(&w[k]);
      st[k] = __low2float(h);
      zp[k] = __high2float(h);
    }
  } else {
    const float4* m = reinterpret_cast<const float4*>(meta + c0 * 8);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float4 v = m[k];
      st[2 * k] = v.x; zp[2 * k] = v.y; st[2 * k + 1] = v.z; zp[2 * k + 1] = v.w;
    }
  }
}

// Dequantisation of one 8-channel chunk of a key block, x = zp + step * code, in the form
// x = s' * (1 + code * 2^-k) + c' with s' = 2^k step and c' = zp - s': after one shift of the packed
// codes word, the codes of a channel pair sit in the mantissa of 1.0 at bits 19-20 and 21-22 (INT2:
// k = 4 and 2) or 15-18 and 19-22 (INT4: k = 8 and 4), so a pair is two masks and one paired FMA.
struct ChunkScale {
  float2 s[4], c[4];
};
template <int BITS, bool F16>
__device__ __forceinline__ void chunk_scale(const uint8_t* meta, int c0, ChunkScale& cs);
template <int BITS>
__device__ __forceinline__ void dequant8_split(uint32_t w, const ChunkScale& cs, uint32_t (&hw)[4],
                                               uint32_t (&lw)[4]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t a, b;
    if (BITS == 2) {
      const uint32_t sh = w << (19 - 4 * q);
      a = (sh & (3u << 19)) | 0x3F800000u;
      b = (sh & (3u << 21)) | 0x3F800000u;
    } else {
      const int k = 15 - 8 * q;
      const uint32_t sh = k >= 0 ? (w << k) : (w >> (-k));
      a = (sh & (0xFu << 15)) | 0x3F800000u;
      b = (sh & (0xFu << 19)) | 0x3F800000u;
    }
    const float2 x = __ffma2_rn(cs.s[q], make_float2(__uint_as_float(a), __uint_as_float(b)), cs.c[q]);
    // hi = x truncated to bf16 (the upper halves of the two words), lo = the exact remainder x - hi
    // truncated again: x = hi + lo to 2^-14 relative, with byte permutes and masks on the integer
    // pipes instead of float-to-bf16 conversions.
    const uint32_t ux = __float_as_uint(x.x), uy = __float_as_uint(x.y);
    const float2 r = __fadd2_rn(x, make_float2(-__uint_as_float(ux & 0xFFFF0000u), -__uint_as_float(uy & 0xFFFF0000u)));
    hw[q] = __byte_perm(ux, uy, 0x7632);
    lw[q] = __byte_perm(__float_as_uint(r.x), __float_as_uint(r.y), 0x7632);
  }
}

// One 16-byte chunk (8 channels) of row `row` into a [D/64][rows][64] bf16 tile, 128-byte swizzle.
template <int ROWS>
__device__ __forceinline__ void store_chunk(uint8_t* tile, int row, int chunk, uint4 v) {
  *reinterpret_cast<uint4*>(tile + (chunk >> 3) * (ROWS * 128) + sw128_offset(row, chunk & 7)) = v;
}

template <int BITS, bool F16>
__device__ __forceinline__ void chunk_scale(const uint8_t* meta, int c0, ChunkScale& cs) {
  float st[8], zp[8];
  meta8<F16>(meta, c0, st, zp);
  constexpr float kA = BITS == 2 ? 16.f : 256.f, kB = BITS == 2 ? 4.f : 16.f;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    cs.s[q] = make_float2(st[2 * q] * kA, st[2 * q + 1] * kB);
    cs.c[q] = make_float2(zp[2 * q] - cs.s[q].x, zp[2 * q + 1] - cs.s[q].y);
  }
}

template <int BITS, int NGV>
__global__ void __launch_bounds__(kThreads, 1) chan_attention_kernel(const AttnParams p, int T) {
  using C = CCfg<BITS, NGV>;
  constexpr int kStages = C::kStages;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const CLayout L = make_clayout<BITS, NGV>(p.meta_f16 ? 2 : 4, T);
  const uint32_t bar0 = smem_u32(smem + L.bars);
  auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L.misc);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L.misc + 4);
  float* xmax = reinterpret_cast<float*>(smem + L.xc);        // [tile parity][half][row]
  float* xsum = xmax + 4 * kBM;                                // [half][row]
  auto wait1 = [&](int i, uint32_t parity) -> bool {
    return mbar_wait(bar(i), parity, abort_flag, p.status, p.wait_limit);
  };
  auto waitw = [&](int i, uint32_t parity) -> bool {
    return warp_wait(bar(i), parity, abort_flag, p.status, p.wait_limit);
  };

  const int warp = threadIdx.x >> 5;
  const int wg = warp >> 2;
  const int lane = threadIdx.x & 31;
  const int m_tile = blockIdx.x;
  const int bh = blockIdx.y;
  const int b = bh / p.Hkv;
  const int h = bh - b * p.Hkv;
  const int64_t rows_total = static_cast<int64_t>(p.r) * p.Lq;
  const int nblk = kN / T;                     // key blocks per tile

  const int Tc_all = static_cast<int>((p.Lc + kN - 1) / kN);
  const int split = blockIdx.z;
  const int c0 = static_cast<int>(static_cast<int64_t>(split) * Tc_all / gridDim.z);
  const int Tc = static_cast<int>(static_cast<int64_t>(split + 1) * Tc_all / gridDim.z) - c0;
  const bool last_split = split == static_cast<int>(gridDim.z) - 1;
  int64_t cur_keys = p.Lcur;
  if (p.causal) {
    const int64_t R0 = static_cast<int64_t>(m_tile) * kBM;
    const int64_t R1 = (R0 + kBM < rows_total ? R0 + kBM : rows_total) - 1;
    const int64_t max_i = (R0 / p.Lq != R1 / p.Lq) ? p.Lq - 1 : R1 % p.Lq;
    const int64_t lim = max_i + 1 + (p.Lcur - p.Lq);
    cur_keys = lim < 0 ? 0 : (lim < p.Lcur ? lim : p.Lcur);
  }
  const int Tn = last_split ? static_cast<int>((cur_keys + kN - 1) / kN) : 0;
  const int T_all = Tc + Tn;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int i = 0; i < B_COUNT; ++i) {
      uint32_t cnt = 1;
      if (i == B_KH_FULL || i == B_KH_FULL + 1) cnt = kKThreads / 32;
      if (i == B_VH_FULL || i == B_VH_FULL + 1) cnt = 4;
      if (i == B_S_FREE || i == B_P_FULL || i == B_Q_FULL) cnt = 8;   // both softmax warpgroups
      if (i >= B_PK_EMPTY && i < B_PK_EMPTY + kStages) cnt = kKThreads / 32 + 4;
      mbar_init(bar(i), cnt);
    }
    mbar_init_fence();
  }
  // Rows of the squared-step operand beyond a tile's blocks stay zero.
  for (uint32_t i = threadIdx.x; i < C::kCTile / 16; i += kThreads)
    reinterpret_cast<uint4*>(smem + L.ct)[i] = make_uint4(0u, 0u, 0u, 0u);
  if (warp == 0) tmem_alloc(smem_u32(tmem_slot), kTmemCols);
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegProducer));
    if (lane == 0) {
      // -------------------------------------------- MMA issue loop (one thread)
      constexpr uint32_t idesc_s = idesc_bf16_f32(kBM, kN, 0, 0);
      constexpr uint32_t idesc_c = idesc_bf16_f32(kBM, kCRows, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kBM, D, 0, 1);
      const uint64_t qdesc = smem_desc_sw128(smem_u32(smem + L.qs), 16u, 1024u);
      const uint64_t hdesc = smem_desc_sw128(smem_u32(smem + L.khi), 16u, 1024u);
      const uint64_t ldesc = smem_desc_sw128(smem_u32(smem + L.klo), 16u, 1024u);
      const uint64_t cdesc = smem_desc_sw128(smem_u32(smem + L.ct), 16u, 1024u);
      const uint64_t vdesc0 = smem_desc_sw128(smem_u32(smem + L.vt), C::kDblk, 1024u);
      auto vdesc = [&](int bb) { return vdesc0 + static_cast<uint64_t>(bb) * (C::kTile >> 4); };
      // 16 channels of a K tile (128 rows) or of the squared-step tile (16 rows).
      auto kofs = [](int ch) { return static_cast<uint64_t>(((ch >> 6) * C::kDblk + ((ch & 63) >> 4) * 32u) >> 4); };
      auto cofs = [](int ch) { return static_cast<uint64_t>(((ch >> 6) * (kCRows * 128u) + ((ch & 63) >> 4) * 32u) >> 4); };
      auto issue_pv = [&](int i) -> bool {
        const int vb = i & 1;
        if (!wait1(B_P_FULL, i & 1)) return false;
        if (!wait1(B_VH_FULL + vb, (i >> 1) & 1)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kN / 16; ++kk)
          mma_ts(tmem + kColO, tmem + kColP + kk * 8u, vdesc(vb) + kk * (2048u >> 4), idesc_pv,
                 (i > 0 || kk > 0) ? 1u : 0u);
        tc_commit(bar(B_VH_EMPTY + vb));
        tc_commit(bar(B_PV_DONE));
        return true;
      };
      bool ok = T_all > 0 && wait1(B_Q_FULL, 0);
      if (ok) tc_fence_after();
      for (int j = 0; j < T_all && ok; ++j) {
        const bool cached = j < Tc;
        // Each 64-channel half of the K tiles as soon as it is written: the producers write the
        // second half of tile j while the first half's MMAs run.
        for (int h = 0; h < 2 && ok; ++h) {
          if (!wait1(B_KH_FULL + h, j & 1)) { ok = false; break; }
          if (h == 0 && j >= 1 && !wait1(B_S_FREE, (j - 1) & 1)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int kk = 4 * h; kk < 4 * h + 4; ++kk)
            mma_ss(tmem + kColS, qdesc + kofs(kk * 16), hdesc + kofs(kk * 16), idesc_s, kk > 0 ? 1u : 0u);
          if (cached) {
#pragma unroll
            for (int kk = 4 * h; kk < 4 * h + 4; ++kk)
              mma_ss(tmem + kColS, qdesc + kofs(kk * 16), ldesc + kofs(kk * 16), idesc_s, 1u);
          }
          if (h == 0) tc_commit(bar(B_KH_EMPTY));
        }
        if (!ok) break;
        if (cached) {
          if (p.correct) {
            // (q2_hi + q2_lo) x (rows blk: d2_hi, rows 4 + blk: d2_lo)
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
              mma_ts(tmem + kColC, tmem + kColQ2H + kk * 8u, cdesc + cofs(kk * 16), idesc_c, kk > 0 ? 1u : 0u);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
              mma_ts(tmem + kColC, tmem + kColQ2L + kk * 8u, cdesc + cofs(kk * 16), idesc_c, 1u);
          }
        }
        tc_commit(bar(B_KH_EMPTY + 1));
        tc_commit(bar(B_S_FULL));
        if (j >= 1) ok = issue_pv(j - 1);
      }
      if (ok) issue_pv(T_all - 1);
      tc_commit(bar(B_DRAIN));
      mbar_wait_drain(bar(B_DRAIN), 0);
    }
    __syncwarp();
  } else if (wg == 0 || wg == 4) {
    // ---------------------------------------------------------------- K hi / lo tiles
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegProducer));
    const int t = wg == 0 ? threadIdx.x - 32 : threadIdx.x - 512 + 96;   // 0 .. kKThreads - 1
    // Half h of a tile is channels [64 h, 64 h + 64) of its hi and lo tiles. Thread t of warp
    // w = t / 32 takes chunk cl of the half (8 channels) for the four keys of key lane
    // 4 w + ks, [4 (4 w + ks), +4), which lie in one key block (T is a multiple of 4), in the order
    // (i + ks) mod 4; threads of warps 0-3 also take one of the keys 112-127. A quarter-warp holds
    // chunks {2 q, 2 q + 1} of four key lanes, so that its four rows and two chunks cover the eight
    // 16-byte bank groups in every store of the swizzled tiles and in every load of the scales, and
    // at INT2 its code loads fall in distinct banks. The four keys share one set of scales and no
    // branch, so that their dequantisations interleave.
    constexpr int kKeysA = 4;                   // 28 key lanes x 4 = 112 keys, then 16 x 1
    static_assert((kKThreads / 8) * kKeysA + 128 / 8 == kN, "key lanes must cover a tile");
    const int w7 = t >> 5, ks = (t & 7) >> 1;
    const int cl = 2 * ((t & 31) >> 3) + (t & 1);
    const int key0 = 4 * (4 * w7 + ks);
    const int keyB = (kKThreads / 8) * kKeysA + 2 * ks + 8 * (w7 & 1) + (w7 >> 1);
    const bool has_b = w7 < 4;
    auto key_a = [&](int i) { return key0 + ((i + ks) & 3); };
    const int tshift = __ffs(T) - 1;            // T is a power of two
    const int64_t row_codes = D * BITS / 8;
    uint8_t* khi = smem + L.khi;
    uint8_t* klo = smem + L.klo;
    bool kok = true;
    for (int j = 0; j < T_all && kok; ++j) {
      const bool cached = j < Tc;
      const int s = j % kStages;
      int valid;
      if (cached) {
        const int64_t rem = p.Lc - static_cast<int64_t>(c0 + j) * kN;
        valid = static_cast<int>(rem < kN ? rem : kN);
      } else {
        const int64_t t0 = static_cast<int64_t>(j - Tc) * kN;
        valid = static_cast<int>(cur_keys - t0 < kN ? cur_keys - t0 : kN);
      }
      const uint8_t* kcodes = smem + L.pk + s * L.stage;
      const uint8_t* kmeta = kcodes + 2 * C::kCodes;            // [blocks][D][2]
      const int blk_bytes = D * 2 * (p.meta_f16 ? 2 : 4);
      for (int h = 0; h < 2; ++h) {
        if (!waitw(B_KH_EMPTY + h, (j & 1) ^ 1)) { kok = false; break; }
        const int chunk = h * 8 + cl;
        if (cached) {
          if (h == 0 && !waitw(B_PK_FULL + s, (j / kStages) & 1)) { kok = false; break; }
          auto load_code = [&](int key) -> uint32_t {
            if (key >= valid) return 0u;
            if (BITS == 2) return *reinterpret_cast<const uint16_t*>(kcodes + key * row_codes + chunk * 2);
            return *reinterpret_cast<const uint32_t*>(kcodes + key * row_codes + chunk * 4);
          };
          auto scale_of = [&](int key, ChunkScale& cs) {
            const uint8_t* m = kmeta + (key >> tshift) * blk_bytes;
            if (p.meta_f16) chunk_scale<BITS, true>(m, chunk * 8, cs);
            else chunk_scale<BITS, false>(m, chunk * 8, cs);
          };
          auto put = [&](int key, const uint32_t (&hw)[4], const uint32_t (&lw)[4]) {
            const bool v = key < valid;          // keys past the cache end become zero
            store_chunk<kN>(khi, key, chunk, v ? make_uint4(hw[0], hw[1], hw[2], hw[3]) : make_uint4(0u, 0u, 0u, 0u));
            store_chunk<kN>(klo, key, chunk, v ? make_uint4(lw[0], lw[1], lw[2], lw[3]) : make_uint4(0u, 0u, 0u, 0u));
          };
          {
            uint32_t w[kKeysA];
#pragma unroll
            for (int i = 0; i < kKeysA; ++i) w[i] = load_code(key_a(i));
            ChunkScale cs;
            scale_of(key0, cs);
#pragma unroll
            for (int i = 0; i < kKeysA; ++i) {
              uint32_t hw[4], lw[4];
              dequant8_split<BITS>(w[i], cs, hw, lw);
              put(key_a(i), hw, lw);
            }
          }
          if (has_b) {
            const uint32_t wb = load_code(keyB);
            ChunkScale cs;
            scale_of(keyB, cs);
            uint32_t hw[4], lw[4];
            dequant8_split<BITS>(wb, cs, hw, lw);
            put(keyB, hw, lw);
          }
          // The tile's blocks' squared steps, scaled to the correction in log2 units, as hi and lo
          // parts (rows blk and 4 + blk), with the second half (read by the same MMAs).
          // (Threads t >= 160, which have no fifth key.)
          const int tc = t - (kKThreads - 64);
          if (h == 1 && p.correct && tc >= 0 && tc < nblk * (D / 8)) {
            const int blk = tc / (D / 8), ch = tc % (D / 8);
            float st[8], zp[8];
            if (p.meta_f16) meta8<true>(kmeta + blk * blk_bytes, ch * 8, st, zp);
            else meta8<false>(kmeta + blk * blk_bytes, ch * 8, st, zp);
            uint32_t dh[4], dl[4];
#pragma unroll
            for (int k = 0; k < 8; k += 2) {
              const float2 d2 = __fmul2_rn(__fmul2_rn(make_float2(st[k], st[k + 1]), make_float2(st[k], st[k + 1])),
                                           make_float2(p.wcoef_log2, p.wcoef_log2));
              dh[k / 2] = pack_bf16x2(d2.x, d2.y);
              const float2 r = __fadd2_rn(d2, make_float2(-bf16_lo(dh[k / 2]), -bf16_hi(dh[k / 2])));
              dl[k / 2] = pack_bf16x2(r.x, r.y);
            }
            store_chunk<kCRows>(smem + L.ct, blk, ch, make_uint4(dh[0], dh[1], dh[2], dh[3]));
            store_chunk<kCRows>(smem + L.ct, 4 + blk, ch, make_uint4(dl[0], dl[1], dl[2], dl[3]));
          }
        } else {
          const int64_t t0 = static_cast<int64_t>(j - Tc) * kN;
          const uint4* src = reinterpret_cast<const uint4*>(p.K_cur) + (static_cast<int64_t>(bh) * p.Lcur + t0) * (D / 8);
#pragma unroll 1
          for (int i = 0; i <= kKeysA; ++i) {
            if (i == kKeysA && !has_b) break;
            const int key = i < kKeysA ? key_a(i) : keyB;
            const uint4 v = key < valid ? src[key * (D / 8) + chunk] : make_uint4(0u, 0u, 0u, 0u);
            store_chunk<kN>(khi, key, chunk, v);
          }
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_KH_FULL + h));
      }
      if (kok && cached) {
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_PK_EMPTY + s));
      }
    }
  } else if (wg == 3) {
    // ---------------------------------------------------------------- V tiles (per token)
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegProducer));
    const int t = threadIdx.x - 384;
    constexpr int kItems = kN * (D / 32);
    constexpr int kItersV = kItems / 128;
    // This thread's items t, t + 128, ...: one channel block, keys 32 apart.
    constexpr int kKeyStepV = 128 * 32 / D;
    const int vkey0 = item_key<D>(t), vblk0 = item_blk<D>(t);
    uint32_t vso[4];
    chunk_offsets<kN>(vkey0, vblk0, vso);
    const bool loader = t == 0;
    const int64_t row_codes = D * BITS / 8;
    const int64_t vrow_meta = static_cast<int64_t>(NGV) * 2 * (p.meta_f16 ? 2 : 4);
    const int64_t kblk_meta = static_cast<int64_t>(D) * 2 * (p.meta_f16 ? 2 : 4);
    int next_load = 0;
    auto issue_load = [&]() -> bool {
      const int s = next_load % kStages, k = next_load / kStages;
      if (!wait1(B_PK_EMPTY + s, (k & 1) ^ 1)) return false;
      const uint32_t dst = smem_u32(smem + L.pk + s * L.stage);
      const int64_t tok0 = static_cast<int64_t>(c0 + next_load) * kN;
      const int64_t row0 = static_cast<int64_t>(bh) * p.capacity + tok0;
      const int64_t blk0 = static_cast<int64_t>(bh) * (p.capacity / T) + tok0 / T;
      const uint32_t fb = bar(B_PK_FULL + s);
      mbar_arrive_expect_tx(fb, 2 * C::kCodes + L.kmeta + L.vmeta);
      bulk_g2s(dst, p.k_codes + row0 * row_codes, C::kCodes, fb);
      bulk_g2s(dst + C::kCodes, p.v_codes + row0 * row_codes, C::kCodes, fb);
      bulk_g2s(dst + 2 * C::kCodes, static_cast<const uint8_t*>(p.k_meta) + blk0 * kblk_meta, L.kmeta, fb);
      bulk_g2s(dst + 2 * C::kCodes + L.kmeta, static_cast<const uint8_t*>(p.v_meta) + row0 * vrow_meta,
               L.vmeta, fb);
      ++next_load;
      return true;
    };
    bool load_ok = true;
    if (loader)
      while (load_ok && next_load < Tc && next_load < kStages) load_ok = issue_load();
    for (int j = 0; j < T_all; ++j) {
      const int sb = j & 1, n = j >> 1;
      uint8_t* vt = smem + L.vt + sb * C::kTile;
      if (!waitw(B_VH_EMPTY + sb, (n & 1) ^ 1)) break;
      if (j < Tc) {
        const int s = j % kStages, k = j / kStages;
        const int64_t rem = p.Lc - static_cast<int64_t>(c0 + j) * kN;
        const int valid = static_cast<int>(rem < kN ? rem : kN);
        const uint8_t* vcodes = smem + L.pk + s * L.stage + C::kCodes;
        const uint8_t* vmeta = smem + L.pk + s * L.stage + 2 * C::kCodes + L.kmeta;
        if (!waitw(B_PK_FULL + s, k & 1)) break;
        using CodeVec = typename CodeVecT<BITS>::type;
        const uint8_t* csrc = vcodes + vkey0 * row_codes + vblk0 * (4 * BITS);
        const int mb2 = p.meta_f16 ? 4 : 8;
        const uint8_t* msrc = vmeta + (vkey0 * NGV + (vblk0 * 32) / C::GV) * mb2;
#pragma unroll 1
        for (int i = 0; i < kItersV; ++i) {
          const int key = vkey0 + kKeyStepV * i;
          uint32_t v[16];
          if (key < valid) {
            const CodeVec cv = *reinterpret_cast<const CodeVec*>(csrc + i * (kKeyStepV * row_codes));
            float st, zp;
            if (p.meta_f16) load_meta<true>(msrc + i * (kKeyStepV * NGV * mb2), 0, st, zp);
            else load_meta<false>(msrc + i * (kKeyStepV * NGV * mb2), 0, st, zp);
            dequant32(cv, st, zp, v);
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) v[e] = 0u;
          }
          store_chunks(vt + (vkey0 + kKeyStepV * i) * 128, vso, v);
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(bar(B_VH_FULL + sb));
          mbar_arrive(bar(B_PK_EMPTY + s));
        }
        if (loader && load_ok && next_load < Tc) load_ok = issue_load();
      } else {
        const int64_t t0 = static_cast<int64_t>(j - Tc) * kN;
        const int valid = static_cast<int>(cur_keys - t0 < kN ? cur_keys - t0 : kN);
#pragma unroll 1
        for (int i = 0; i < kItersV; ++i) {
          const int it = t + 128 * i, key = item_key<D>(it), blk = item_blk<D>(it);
          uint32_t v[16];
          if (key < valid) {
            const uint4* src = reinterpret_cast<const uint4*>(p.V_cur) +
                               (static_cast<int64_t>(bh) * p.Lcur + t0 + key) * (D / 8) + blk * 4;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const uint4 x = src[e];
              v[4 * e] = x.x; v[4 * e + 1] = x.y; v[4 * e + 2] = x.z; v[4 * e + 3] = x.w;
            }
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) v[e] = 0u;
          }
          store32<kN>(vt, key, blk, v);
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_VH_FULL + sb));
      }
    }
    if (loader) {
      for (int s = 0; s < kStages && s < next_load; ++s) {
        const int last = ((next_load - 1 - s) / kStages) * kStages + s;
        mbar_wait_drain(bar(B_PK_FULL + s), (last / kStages) & 1);
      }
    }
  } else {
    // ---------------------------------------------------------------- softmax / epilogue (WG1, WG2)
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegSoftmax));
    constexpr int NH = kN / 2;
    const int half = wg - 1;
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const int64_t R = static_cast<int64_t>(m_tile) * kBM + row;
    const bool valid_row = R < rows_total;
    const int64_t hq = static_cast<int64_t>(h) * p.r + (valid_row ? R / p.Lq : 0);
    const int64_t qi = valid_row ? R % p.Lq : 0;
    const int64_t out_row = (static_cast<int64_t>(b) * p.Hq + hq) * p.Lq + qi;
    const int kbase_h = half * NH;
    {
      // This half's channels of Q (natural order) into shared memory, and of q^2 as two bf16 parts
      // (exact: q is bf16, so q^2 has at most 16 significant bits) into tensor memory.
      const uint8_t* qrow = static_cast<const uint8_t*>(p.Q) + out_row * D * 2;
#pragma unroll
      for (int g = 0; g < 2; ++g) {             // 32 channels (16 columns) at a time
        uint32_t q2h[16], q2l[16];
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          const int c = 4 * g + c4;
          uint4 u = make_uint4(0u, 0u, 0u, 0u);
          if (valid_row) u = reinterpret_cast<const uint4*>(qrow)[half * (D / 16) + c];
          store_chunk<kBM>(smem + L.qs, row, half * (D / 16) + c, u);
          const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 a = __fmul2_rn(make_float2(bf16_lo(w[e]), bf16_hi(w[e])), make_float2(bf16_lo(w[e]), bf16_hi(w[e])));
            const uint32_t hi = pack_bf16x2(a.x, a.y);
            const float2 r = __fadd2_rn(a, make_float2(-bf16_lo(hi), -bf16_hi(hi)));
            q2h[4 * c4 + e] = hi;
            q2l[4 * c4 + e] = pack_bf16x2(r.x, r.y);
          }
        }
        tmem_st16(tmem + lane_off + kColQ2H + half * (D / 4) + 16 * g, q2h);
        tmem_st16(tmem + lane_off + kColQ2L + half * (D / 4) + 16 * g, q2l);
      }
      fence_async_smem();
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_Q_FULL));
    }
    float m_run = -INFINITY;
    float l_run = 0.f;
    const float2 scale2 = make_float2(p.scale_log2, p.scale_log2);
    // As in the 128-row kernel: a warp whose wait failed skips the rest of the tile, and the eight
    // softmax warps leave the loop together at the next row-max exchange.
    bool ok = true;
    for (int j = 0; j < T_all; ++j) {
      const bool cached = j < Tc;
      if (ok && !waitw(B_S_FULL, j & 1)) ok = false;
      tc_fence_after();
      const uint32_t tm_s = tmem + lane_off + kColS + kbase_h;
      int valid;
      if (cached) {
        const int64_t rem = p.Lc - static_cast<int64_t>(c0 + j) * kN;
        valid = static_cast<int>(rem < kN ? rem : kN);
      } else {
        const int64_t t0 = static_cast<int64_t>(j - Tc) * kN;
        int64_t lim = cur_keys - t0;
        if (p.causal) {
          const int64_t c = qi + (p.Lcur - p.Lq) - t0 + 1;
          lim = c < lim ? c : lim;
        }
        valid = static_cast<int>(lim < 0 ? 0 : (lim < kN ? lim : kN));
      }
      // The correction of each block of the tile (log2 units), for cached tiles.
      // Scores relative to the maximum in use so far (0 before the first key), as in the
      // per-token kernel: no subtraction in the exponentials unless the maximum moves.
      const float m_prev = m_run == -INFINITY ? 0.f : m_run;
      float corr[4] = {0.f, 0.f, 0.f, 0.f};
      if (cached && p.correct) {
        uint32_t cr[8];
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                     : "=r"(cr[0]), "=r"(cr[1]), "=r"(cr[2]), "=r"(cr[3]),
                       "=r"(cr[4]), "=r"(cr[5]), "=r"(cr[6]), "=r"(cr[7])
                     : "r"(tmem + lane_off + kColC)
                     : "memory");
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 4; ++k) corr[k] = __uint_as_float(cr[k]) + __uint_as_float(cr[4 + k]);
      }
      float2 s2[NH / 2];
#pragma unroll
      for (int cc = 0; cc < NH; cc += 32) {
        uint32_t r[32];
        tmem_ld32(tm_s + cc, r);
        tmem_wait_ld();
        // 32 keys of one block (T is a multiple of 32).
        const int bk = (kbase_h + cc) / T;
        const float cb = bk == 0 ? corr[0] : (bk == 1 ? corr[1] : (bk == 2 ? corr[2] : corr[3]));
        const float2 nc = make_float2(-cb - m_prev, -cb - m_prev);
#pragma unroll
        for (int q = 0; q < 16; ++q)
          s2[cc / 2 + q] = __ffma2_rn(scale2, make_float2(__uint_as_float(r[2 * q]), __uint_as_float(r[2 * q + 1])), nc);
      }
      tc_fence_before();
      __syncwarp();
      if (ok && lane == 0) mbar_arrive(bar(B_S_FREE));
      if (valid < kbase_h + NH) {
#pragma unroll
        for (int q = 0; q < NH / 2; ++q) {
          if (kbase_h + 2 * q >= valid) s2[q].x = -INFINITY;
          if (kbase_h + 2 * q + 1 >= valid) s2[q].y = -INFINITY;
        }
      }
      float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
#pragma unroll
      for (int q = 0; q < NH / 2; q += 4) {
        m0 = fmax3(m0, s2[q].x, s2[q].y);
        m1 = fmax3(m1, s2[q + 1].x, s2[q + 1].y);
        m2 = fmax3(m2, s2[q + 2].x, s2[q + 2].y);
        m3 = fmax3(m3, s2[q + 3].x, s2[q + 3].y);
      }
      const float m_half = fmax3(fmaxf(m0, m1), m2, m3);
      xmax[((j & 1) * 2 + half) * kBM + row] = m_half;
      if (named_sync_or(1, 256, !ok)) { ok = false; break; }
      const float m_tile = fmaxf(m_half, xmax[((j & 1) * 2 + (half ^ 1)) * kBM + row]) + m_prev;
      const bool need = (m_tile > m_run + kRescaleThreshold) || (m_run == -INFINITY && m_tile > -INFINITY);
      float factor = 1.f;
      if (need) {
        factor = ex2(m_run - m_tile);
        l_run *= factor;
        m_run = m_tile;
      }
      const float m_use = m_run == -INFINITY ? 0.f : m_run;
      const bool any_need = __any_sync(0xffffffffu, need);
      // O is rescaled after the previous P.V has finished; P is rewritten after it too (one buffer).
      if (j > 0) {
        if (!waitw(B_PV_DONE, (j - 1) & 1)) { ok = false; continue; }
        tc_fence_after();
        if (any_need) {
          const uint32_t tm_o = tmem + lane_off + kColO + half * (D / 2);
          const float2 f2 = make_float2(factor, factor);
#pragma unroll 1
          for (int c = 0; c < D / 2; c += 32) {
            uint32_t r[32];
            tmem_ld32(tm_o + c, r);
            tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 32; k += 2) {
              const float2 o2 = __fmul2_rn(make_float2(__uint_as_float(r[k]), __uint_as_float(r[k + 1])), f2);
              r[k] = __float_as_uint(o2.x);
              r[k + 1] = __float_as_uint(o2.y);
            }
            tmem_st32(tm_o + c, r);
          }
        }
      }
      if (any_need) {
        const float2 d2 = make_float2(m_prev - m_use, m_prev - m_use);
#pragma unroll
        for (int k = 0; k < NH / 2; ++k) s2[k] = __fadd2_rn(s2[k], d2);
      }
      float2 psum = make_float2(0.f, 0.f);
      uint32_t pk[NH / 2];
#pragma unroll
      for (int k = 0; k < NH / 2; ++k) {
        const float2 e = s2[k];
        const float2 pp = make_float2(ex2(e.x), ex2(e.y));
        psum = __fadd2_rn(psum, pp);
        pk[k] = pack_bf16x2(pp.x, pp.y);
      }
      tmem_st<NH / 2>(tmem + lane_off + kColP + kbase_h / 2, pk);
      l_run += psum.x + psum.y;
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_P_FULL));
    }

    bool have_o = false;
    if (ok && T_all > 0) {
      have_o = waitw(B_PV_DONE, (T_all - 1) & 1);
      tc_fence_after();
    }
    xsum[half * kBM + row] = l_run;
    named_sync(1, 256);
    const float l_tot = l_run + xsum[(half ^ 1) * kBM + row];
    const float inv_l = l_tot > 0.f ? 1.f / l_tot : 0.f;
    uint8_t* orow = static_cast<uint8_t*>(p.O) + out_row * D * 2 + half * D;
    const bool partial = gridDim.z > 1;
    float* prow = partial ? p.ws_o + (static_cast<int64_t>(split) * p.rows_all + out_row) * D + half * (D / 2) : nullptr;
#pragma unroll
    for (int c = 0; c < D / 2; c += 32) {
      uint32_t r[32];
      if (have_o) {
        tmem_ld32(tmem + lane_off + kColO + half * (D / 2) + c, r);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int k = 0; k < 32; ++k) r[k] = 0u;
      }
      if (valid_row && partial) {
        float4* dst = reinterpret_cast<float4*>(prow + c);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          dst[k] = make_float4(__uint_as_float(r[4 * k]) * inv_l, __uint_as_float(r[4 * k + 1]) * inv_l,
                               __uint_as_float(r[4 * k + 2]) * inv_l, __uint_as_float(r[4 * k + 3]) * inv_l);
      } else if (valid_row) {
        uint4* dst = reinterpret_cast<uint4*>(orow) + c / 8;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          uint32_t o4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            o4[e] = pack_bf16x2(__uint_as_float(r[8 * k + 2 * e]) * inv_l, __uint_as_float(r[8 * k + 2 * e + 1]) * inv_l);
          dst[k] = make_uint4(o4[0], o4[1], o4[2], o4[3]);
        }
      }
    }
    if (valid_row && half == 0) {
      const float m_use = m_run == -INFINITY ? 0.f : m_run;
      const float lse = l_tot > 0.f ? (m_use + __log2f(l_tot)) * 0.69314718055994530942f : -INFINITY;
      if (partial) p.ws_lse[static_cast<int64_t>(split) * p.rows_all + out_row] = lse;
      else p.LSE[out_row] = lse;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int BITS, int NGV>
cudaError_t launch_chan(const AttnParams& p, int T, cudaStream_t stream) {
  const CLayout L = make_clayout<BITS, NGV>(p.meta_f16 ? 2 : 4, T);
  size_t smem = L.total + 1024;
  if (smem < 116u * 1024u) smem = 116u * 1024u;
  if (smem > 227u * 1024u) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(chan_attention_kernel<BITS, NGV>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int64_t rows = static_cast<int64_t>(p.r) * p.Lq;
  dim3 grid(static_cast<unsigned>((rows + kBM - 1) / kBM), static_cast<unsigned>(p.B * p.Hkv),
            static_cast<unsigned>(p.n_split > 1 ? p.n_split : 1));
  chan_attention_kernel<BITS, NGV><<<grid, kThreads, smem, stream>>>(p, T);
  return cudaGetLastError();
}

template <int BITS>
cudaError_t launch_chan_groups(const AttnParams& p, int T, cudaStream_t stream) {
  if (p.n_groups == 1) return launch_chan<BITS, 1>(p, T, stream);
  if (p.n_groups == 2) return launch_chan<BITS, 2>(p, T, stream);
  return launch_chan<BITS, 4>(p, T, stream);
}

}  // namespace

bool chan_tc_serves(int d, int dtype_f32, int correct) { return d == 128 && !dtype_f32 && correct <= 1; }

cudaError_t launch_attention_channel_tc(const AttnParams& p, int bits, int T, cudaStream_t stream) {
  return bits == 2 ? launch_chan_groups<2>(p, T, stream) : launch_chan_groups<4>(p, T, stream);
}

}  // namespace qkv
