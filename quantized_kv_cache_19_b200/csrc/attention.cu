// Jensen-bias-corrected chunk attention over the packed low-bit KV cache, bf16 inputs, sm_100a.
//
// Method (agents-report.net, "KV-Cache 量化導致的 Jensen 偏差", sections 方法 and 為何校正有效; the
// fugumt.com abstract of "Quantized Keys Steal Attention"): each query row attends, in one softmax,
// over the cached keys and the unquantised current chunk; every cached-key score has
//     b_j = (scale^2 / 24) * sum_c q_c^2 * step_{j, c/group}^2
// subtracted before the softmax (the page's (1/(24 d)) sum_c q_c^2 Delta_{i,c}^2 at scale 1/sqrt d).
// The dequantisation is fused into the attention (hotelren.com blog, §4.3), tile by tile.
//
// Cached-key scores are computed from the integer codes, not from bf16-rounded keys: with
// x_hat = zp_g + step_g * code per group g,
//     t_ij = sum_g a_jg * [ q_ig . code_jg + qs_ig * rho_jg - w_ig * sigma_jg ]    (log2 units)
// where a = step' * scale * log2 e (step' = step, or 1 for a constant group), rho = zp / step',
// sigma = step / (scale * log2 e), qs_ig = sum_{c in g} q_ic and w_ig = (scale^2 / 24) log2 e
// sum_{c in g} q_ic^2 (so that a * w * sigma is the Jensen term b). The bracket is one tensor-core
// accumulator per group: the codes are exact small integers in bf16 (fp32 accumulate), and the
// two rank-1 terms ride on one extra 16-channel k-step per group whose operands are the row and
// key values split into three bf16 parts each (every product of parts whose orders add up to at
// most two), which keeps both terms to ~2^-24 relative. The softmax then needs one FMA per group
// per score. Rounding keys to bf16 instead would move the log-sum-exp by up to ~3e-2 on keys with
// outlier channels. Values are dequantised to bf16 (x_hat in fp32, then rounded) for P.V.
//
// One CTA computes 128 packed query rows (the Hq/Hkv query heads of one KV head; row =
// head_in_group * Lq + i) against every key of its (batch, KV head), in tiles of N = 128 keys (64
// with four groups), so that every MMA has N = 128 or four independent accumulators: a dependent
// chain of 128 x 64 x 16 MMAs into one accumulator issues at a third of the tensor rate. Five
// warpgroups, registers rebalanced with setmaxnreg:
//   WG0      warp 0: allocates tensor memory; one thread issues, in order, S_j = Q K_j^T and then
//            P_{j-1} V_{j-1} with precomputed descriptors.
//   WG0 warps 1-3 and the first 1-2 warps of WG4: K operand tiles (codes unpacked to exact bf16
//            integers, 128-byte
//            swizzle, two buffers) and the tile's per-key constants (scales a for the softmax, key
//            extras for the S MMA); for current tiles, a copy of K_cur. Channels are stored in an
//            operand order (k, k+8 interleaved inside each 16-channel block) that makes the unpack
//            three operations per channel pair; Q in tensor memory and K_cur use the same order.
//   WG1/WG2  softmax, one query row per thread, WG1 on the first half of every key tile and WG2
//            on the second: Q row statistics and a bf16 copy of Q into TMEM; per tile read S from
//            TMEM (releasing it at once), form the corrected scores, exchange the row max through
//            shared memory, online softmax in base 2 with lazy rescaling of O (each half rescales
//            half of O's columns), P (bf16) into TMEM; finally O / l and LSE.
//   WG3 and the rest of WG4: V operand tiles, dequantised to bf16; for current tiles, a copy of
//            V_cur (the split between K and V warps is in Cfg). One lane of WG3
//            also issues the bulk (TMA-engine) copies of packed tiles (codes and step/zero-point
//            of N keys, K and V) into a 2-3 stage ring.
// Tensor memory (512 columns): O [0, d), Q [128, 128 + d/2), P [192, 256), S [256, 512) (one
// buffer of groups * N columns, or two with one group). The MMA for S_{j+1} runs while the
// softmax works on tile j; the softmax waits for P_{j-1}.V_{j-1} before it writes P_j.
// Every mbarrier wait is bounded; on timeout the CTA records QKV_ERR_TIMEOUT in the library's
// device status word, drains its copies and MMAs, frees tensor memory and returns.
#include "qkv_common.cuh"
#include "qkv_internal.h"
#include "qkv_jensen.cuh"
#include "tile_ops.cuh"

#include <type_traits>

namespace qkv {
namespace {

constexpr int kBM = 128;                     // query rows per CTA (MMA M)
constexpr int kThreads = 640;                 // five warpgroups
// Registers per thread after setmaxnreg: 2 * 128 * 144 + 3 * 128 * 64 = 61440 = 640 * 96, the
// block's allocation at launch.
constexpr int kRegProducer = 64, kRegSoftmax = 144;
constexpr int kStagesMax = 3;                // packed-tile ring (INT2: 3 stages, INT4: 2)
constexpr float kRescaleThreshold = 8.0f;    // log2 units: O is rescaled only when the max grows by more
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0, kColQ = 128, kColP = 192, kColS = 256;   // P: 64 columns, S: 256

enum {
  B_PK_FULL = 0, B_PK_EMPTY = B_PK_FULL + kStagesMax,
  B_KH_FULL = B_PK_EMPTY + kStagesMax, B_KH_EMPTY = B_KH_FULL + 2,
  B_VH_FULL = B_KH_EMPTY + 2, B_VH_EMPTY = B_VH_FULL + 2,
  B_KC_FULL = B_VH_EMPTY + 2, B_KC_EMPTY = B_KC_FULL + 2,
  B_S_FULL = B_KC_EMPTY + 2, B_S_FREE = B_S_FULL + 2,
  B_P_FULL = B_S_FREE + 2, B_PV_DONE = B_P_FULL + 2,
  B_Q_FULL = B_PV_DONE + 2, B_DRAIN = B_Q_FULL + 1,
  B_COUNT = B_DRAIN + 1
};

template <int D, int BITS, int NG>
struct Cfg {
  // Keys per tile: 128, so that every MMA has N = 128 (a dependent chain of N = 64 MMAs into one
  // accumulator issues at a third of the tensor rate; at N = 128 it runs at the full rate), or 64
  // with four groups, whose four accumulators then hide the chain latency.
  static constexpr int N = NG == 4 ? 64 : 128;
  static constexpr int G = D / NG;                       // channels per group
  static constexpr uint32_t kTile = N * D * 2;           // bf16 operand tile
  static constexpr uint32_t kCodes = N * D * BITS / 8;   // packed codes of one tile
  static constexpr int NA = NG;                          // score accumulators: one per group
  static constexpr int NAH = (NA + 1) / 2;               // float4s of scales per key pair
  // per-key scales a of one tile: for each key pair, NAH float4 (acc even: x,y; acc odd: z,w)
  static constexpr uint32_t kKconst = (N / 2) * NAH * 16;
  static constexpr uint32_t kAx = NG * kBM * 32;         // row extras, [g][128 rows][16] bf16
  static constexpr uint32_t kBx = NG * N * 32;           // key extras of one tile, [g][N][16] bf16
  static constexpr int kStages = BITS == 2 ? 3 : 2;      // packed-tile ring
  static constexpr uint32_t kDblk = N * 128;             // bytes between 64-channel blocks
  static constexpr int kSCols = NA * N;                  // TMEM columns of one S buffer
  static constexpr int kSB = 256 / kSCols;               // S buffers in the 256 S columns (1 or 2)
  static constexpr int kPB = 64 / (N / 2);               // P buffers in the 64 P columns (1 or 2)
  // Producer warps: K on warps 1-3 and the first kKWarps - 3 warps of warpgroup 4, V on warpgroup 3
  // and the rest of warpgroup 4 (11 in all). Warp w issues from sub-partition w % 4: with four K
  // warps every sub-partition holds one K warp, two softmax warps and one or two V warps. Measured
  // over 4-7 K warps (one launch each, 1965 MHz): 4 was fastest with two groups (chunked prefill
  // 9.37 ms against 9.60 with 7), 5 with one group (the long-video cache 6.47 ms against 7.01);
  // the V dequantisation costs more instructions than the K unpack and per-key constants.
  static constexpr int kKWarps = NG == 1 ? 5 : 4;
  static constexpr int kVWarps = 11 - kKWarps;
  static constexpr int kKThreads = 32 * kKWarps;
  static constexpr int kVThreads = 32 * kVWarps;
};

struct Layout {
  uint32_t kt, vt, pk, kc, ax, bx, xc, bars, misc, total, stage, meta;
};

template <int D, int BITS, int NG>
__host__ __device__ inline Layout make_layout(int meta_bytes) {
  using C = Cfg<D, BITS, NG>;
  Layout L;
  L.meta = C::N * NG * 2 * meta_bytes;
  L.stage = (2 * (C::kCodes + L.meta) + 127) & ~127u;
  L.kt = 0;
  L.vt = L.kt + 2 * C::kTile;
  L.pk = L.vt + 2 * C::kTile;
  L.kc = L.pk + C::kStages * L.stage;
  L.ax = (L.kc + 4 * C::kKconst + 127) & ~127u;   // scales a (2 buffers), then step^4 (2 buffers)
  L.bx = L.ax + C::kAx;
  L.xc = L.bx + 2 * C::kBx;                // row-max exchange [2][2][128] and row-sum [2][128]
  L.bars = L.xc + (4 + 2) * kBM * 4;
  L.misc = L.bars + B_COUNT * 8;
  L.total = L.misc + 16;
  return L;
}

// Copies `valid` rows (of N) of bf16 [row][D] from global memory into a [D/64][N][64] swizzled tile;
// rows beyond `valid` become zero. NT threads, kIters (key, 32-channel block) items each.
template <int D, int N, int kIters, int NT, bool kPermute>
__device__ __forceinline__ void copy_rows(const uint4* src, uint8_t* tile, int valid, int t) {
  constexpr int kItems = N * (D / 32);
  constexpr int kBatch = 1;                  // items in flight per thread (register budget)
#pragma unroll 1
  for (int i0 = 0; i0 < kIters; i0 += kBatch) {
    uint4 a[kBatch][4];
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const int it = t + NT * (i0 + i), key = item_key<D>(it), blk = item_blk<D>(it);
#pragma unroll
      for (int e = 0; e < 4; ++e)
        a[i][e] = (i0 + i < kIters && it < kItems && key < valid) ? src[key * (D / 8) + blk * 4 + e]
                                                                  : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const int it = t + NT * (i0 + i), key = item_key<D>(it), blk = item_blk<D>(it);
      if (i0 + i >= kIters || it >= kItems) break;
      uint32_t v[16];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        v[4 * e] = a[i][e].x; v[4 * e + 1] = a[i][e].y; v[4 * e + 2] = a[i][e].z; v[4 * e + 3] = a[i][e].w;
      }
      if (kPermute) {
        uint32_t u[16];
        permute16(v, u);
        permute16(v + 8, u + 8);
        store32<N>(tile, key, blk, u);
      } else {
        store32<N>(tile, key, blk, v);
      }
    }
  }
}

template <int D, int BITS, int NG, bool kQuartic>
__global__ void __launch_bounds__(kThreads, 1) corrected_attention_kernel(const AttnParams p) {
  using C = Cfg<D, BITS, NG>;
  constexpr int kKWarps = C::kKWarps, kVWarps = C::kVWarps;
  constexpr int kKThreads = C::kKThreads, kVThreads = C::kVThreads;
  constexpr int N = C::N;
  constexpr int kStages = C::kStages;
  constexpr int NH = N / 2;                   // keys of a tile per softmax warpgroup
  constexpr int kItems = N * (D / 32);        // (key, 32-channel block) items of one tile
  constexpr int kItersV = (kItems + kVThreads - 1) / kVThreads;   // per V-producer thread
  constexpr int kItersK = (kItems + kKThreads - 1) / kKThreads;   // per K-producer thread
  extern __shared__ __align__(16) uint8_t smem_raw[];
  // 1024-byte alignment (128B-swizzle atoms) by offsetting the shared array itself, so that the
  // compiler keeps every access in the shared address space.
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const Layout L = make_layout<D, BITS, NG>(p.meta_f16 ? 2 : 4);
  const uint32_t bar0 = smem_u32(smem + L.bars);
  auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L.misc);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L.misc + 4);
  float4* kconst = reinterpret_cast<float4*>(smem + L.kc);
  uint8_t* ax = smem + L.ax;                                   // row extras (written by the softmax)
  uint8_t* bx = smem + L.bx;                                   // key extras ring (K producers)
  float* xmax = reinterpret_cast<float*>(smem + L.xc);        // [tile parity][half][row]
  float* xsum = xmax + 4 * kBM;                                // [half][row]

  const int warp = threadIdx.x >> 5;
  const int wg = warp >> 2;
  const int lane = threadIdx.x & 31;
  const int m_tile = blockIdx.x;
  const int bh = blockIdx.y;
  const int b = bh / p.Hkv;
  const int h = bh - b * p.Hkv;
  const int64_t rows_total = static_cast<int64_t>(p.r) * p.Lq;

  // Tiles: cached ones first, then current ones (causal: only those some row of this CTA sees).
  // With a split over the cached keys, this CTA takes cached tiles [c0, c0 + Tc) and, if it is the
  // last split, the current chunk.
  const int Tc_all = static_cast<int>((p.Lc + N - 1) / N);
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
  const int Tn = last_split ? static_cast<int>((cur_keys + N - 1) / N) : 0;
  const int T = Tc + Tn;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int i = 0; i < B_COUNT; ++i) {
      uint32_t cnt = 1;
      if (i == B_KH_FULL || i == B_KH_FULL + 1 || i == B_KC_FULL || i == B_KC_FULL + 1) cnt = kKWarps;
      if (i == B_VH_FULL || i == B_VH_FULL + 1) cnt = kVWarps;
      if (i == B_KC_EMPTY || i == B_KC_EMPTY + 1 || i == B_S_FREE || i == B_S_FREE + 1 ||
          i == B_P_FULL || i == B_P_FULL + 1 || i == B_Q_FULL)
        cnt = 8;                                   // both softmax warpgroups
      if (i >= B_PK_EMPTY && i < B_PK_EMPTY + kStages) cnt = kKWarps + kVWarps;  // K and V producer warps
      mbar_init(bar(i), cnt);
    }
    mbar_init_fence();
  }
  if (warp == 0) tmem_alloc(smem_u32(tmem_slot), kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (wg == 0 && warp == 0) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegProducer));
    if (lane == 0) {
      // -------------------------------------------- bulk-copy and MMA issue loop (one thread)
      constexpr uint32_t idesc_s = idesc_bf16_f32(kBM, N, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kBM, D, 0, 1);
      const uint32_t tm_q = tmem + kColQ, tm_o = tmem + kColO, tm_p = tmem + kColP;
      const uint32_t tm_s = tmem + kColS;
      // Descriptors of buffer 0; buffer 1 is the same descriptor with its start address (bits 0-13,
      // 16-byte units) advanced by the buffer size. Arithmetic, not an array indexed by the
      // buffer, which would live in local memory.
      const uint64_t kdesc0 = smem_desc_sw128(smem_u32(smem + L.kt), 16u, 1024u);
      const uint64_t vdesc0 = smem_desc_sw128(smem_u32(smem + L.vt), C::kDblk, 1024u);
      const uint64_t adesc = smem_desc_noswz(smem_u32(ax), 128u, 256u);
      const uint64_t bdesc0 = smem_desc_noswz(smem_u32(bx), 128u, 256u);
      auto kdesc = [&](int b) { return kdesc0 + static_cast<uint64_t>(b) * (C::kTile >> 4); };
      auto vdesc = [&](int b) { return vdesc0 + static_cast<uint64_t>(b) * (C::kTile >> 4); };
      auto bdesc = [&](int b) { return bdesc0 + static_cast<uint64_t>(b) * (C::kBx >> 4); };
      // O += P_i V_i once the softmax wrote P_i and V_i is in smem.
      auto issue_pv = [&](int i) -> bool {
        const int vb = i & 1, pb = i % C::kPB;
        if (!mbar_wait(bar(B_P_FULL + pb), (i / C::kPB) & 1, abort_flag, p.status, p.wait_limit)) return false;
        if (!mbar_wait(bar(B_VH_FULL + vb), (i >> 1) & 1, abort_flag, p.status, p.wait_limit)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < N / 16; ++kk)   // 16 keys = two 1024-byte atoms per step
          mma_ts(tm_o, tm_p + pb * (N / 2) + kk * 8u, vdesc(vb) + kk * (2048u >> 4), idesc_pv,
                 (i > 0 || kk > 0) ? 1u : 0u);
        tc_commit(bar(B_VH_EMPTY + vb));
        tc_commit(bar(B_PV_DONE + pb));
        return true;
      };
      bool ok = T > 0 && mbar_wait(bar(B_Q_FULL), 0, abort_flag, p.status, p.wait_limit);
      if (ok) tc_fence_after();
      // In order: S_j (once K_j is in smem and its S buffer was read by the softmax), then
      // P_{j-1}.V_{j-1}.
      for (int j = 0; j < T && ok; ++j) {
        const int kb = j & 1, sb = j % C::kSB;
        if (!mbar_wait(bar(B_KH_FULL + kb), (j >> 1) & 1, abort_flag, p.status, p.wait_limit)) { ok = false; break; }
        if (j >= C::kSB && !mbar_wait(bar(B_S_FREE + sb), ((j - C::kSB) / C::kSB) & 1, abort_flag, p.status, p.wait_limit)) { ok = false; break; }
        tc_fence_after();
        const uint32_t tm_sj = tm_s + sb * C::kSCols;
        // K tile [d/64][N keys][64], 128B swizzle, K-major: 16 channels per step (32 bytes inside
        // the swizzle row), SBO = next 8 keys; descriptor start addresses advance in 16-byte units.
        auto kofs = [](int ch) { return static_cast<uint64_t>(((ch >> 6) * C::kDblk + ((ch & 63) >> 4) * 32u) >> 4); };
        // k-steps interleaved over the group accumulators (independent chains)
#pragma unroll
        for (int kk = 0; kk < C::G / 16; ++kk)
#pragma unroll
          for (int g = 0; g < NG; ++g) {
            const int ch = g * C::G + kk * 16;
            mma_ts(tm_sj + g * N, tm_q + ch / 2, kdesc(kb) + kofs(ch), idesc_s, kk > 0 ? 1u : 0u);
          }
        if (j < Tc) {
          // zero-point and correction terms: row extras x key extras (no swizzle, K-major)
#pragma unroll
          for (int g = 0; g < NG; ++g)
            mma_ss(tm_sj + g * N, adesc + g * ((kBM * 32) >> 4), bdesc(kb) + g * ((N * 32) >> 4), idesc_s, 1u);
        }
        tc_commit(bar(B_KH_EMPTY + kb));
        tc_commit(bar(B_S_FULL + sb));
        if (j >= 1) ok = issue_pv(j - 1);
      }
      if (ok) issue_pv(T - 1);
      // Never free tensor memory under a running MMA, never leave with copies in flight.
      tc_commit(bar(B_DRAIN));
      mbar_wait_drain(bar(B_DRAIN), 0);
    }
    __syncwarp();
  } else if (wg == 0 || (wg == 4 && warp < 16 + kKWarps - 3)) {
    // ---------------------------------------------------------------- K operand tiles (warps 1-3, 16..)
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegProducer));
    const int t = wg == 0 ? threadIdx.x - 32 : threadIdx.x - 512 + 96;   // 0 .. kKThreads - 1
    // This thread's unpack items t, t + kKThreads, ...: one channel block, keys kKeyStep apart
    // (item_key / item_blk of those indices), so their code and store addresses advance by
    // constants.
    constexpr int kKeyStep = kKThreads * 32 / D;
    static_assert((kKThreads * 32) % D == 0 && kKeyStep % 8 == 0, "items of a thread share a block");
    const int key0 = item_key<D>(t), blk0 = item_blk<D>(t);
    uint32_t so[4];
    chunk_offsets<N>(key0, blk0, so);
    // Per-key-constant items t, t + kKThreads, ...: (key, group) = (e / NG, e % NG), one group,
    // keys kKeyStepC apart; the scale index and the extras row advance by constants.
    constexpr int kKeyStepC = kKThreads / NG;
    static_assert(kKThreads % NG == 0 && kKeyStepC % 8 == 0, "constant items of a thread share a group");
    const int gc = t % NG, keyc0 = t / NG;
    const int ci0 = ((keyc0 >> 1) * C::NAH + (gc >> 1)) * 4 + (gc & 1) * 2 + (keyc0 & 1);
    const int xo0 = gc * (N * 32) + (keyc0 >> 3) * 256 + (keyc0 & 7) * 16;   // store_extras layout
    for (int j = 0; j < T; ++j) {
      const int sb = j & 1, n = j >> 1;
      uint8_t* kt = smem + L.kt + sb * C::kTile;
      if (!warp_wait(bar(B_KH_EMPTY + sb), (n & 1) ^ 1, abort_flag, p.status, p.wait_limit)) break;
      if (j < Tc) {
        const int s = j % kStages, k = j / kStages;
        const int64_t rem = p.Lc - static_cast<int64_t>(c0 + j) * N;
        const int valid = static_cast<int>(rem < N ? rem : N);
        const uint8_t* kcodes = smem + L.pk + s * L.stage;
        if (!warp_wait(bar(B_PK_FULL + s), k & 1, abort_flag, p.status, p.wait_limit)) break;
        using CodeVec = typename CodeVecT<BITS>::type;
        // One item per iteration with the next item's codes already loaded (shared-memory loads
        // take ~170 cycles while the tensor core reads its operands), the loop itself not
        // unrolled: the code of all roles shares the instruction caches of each SM sub-partition.
        constexpr int kRowCodes = D * BITS / 8;
        const uint8_t* src = kcodes + key0 * kRowCodes + blk0 * (4 * BITS);
        uint8_t* row = kt + key0 * 128;
        CodeVec cv_next = *reinterpret_cast<const CodeVec*>(src);
#pragma unroll 1
        for (int key = key0; key < N; key += kKeyStep, src += kKeyStep * kRowCodes, row += kKeyStep * 128) {
          const CodeVec cv = cv_next;
          if (key + kKeyStep < N) cv_next = *reinterpret_cast<const CodeVec*>(src + kKeyStep * kRowCodes);
          uint32_t v[16];
          if (key < valid) {
            unpack_codes32(cv, v);
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) v[e] = 0u;
          }
          store_chunks(row, so, v);
        }
        // Per-key constants of the tile: scales a for the softmax (once it has read the previous
        // ones from this buffer) and the key extras of the S MMA.
        if (!warp_wait(bar(B_KC_EMPTY + sb), (n & 1) ^ 1, abort_flag, p.status, p.wait_limit)) break;
        const uint8_t* kmeta = kcodes + C::kCodes;
        float* kc = reinterpret_cast<float*>(kconst + sb * (C::kKconst / 16));
        constexpr int kItersC = (N * NG + kKThreads - 1) / kKThreads;
#pragma unroll 1
        for (int i = 0; i < kItersC; ++i) {
          const int key = keyc0 + kKeyStepC * i;
          if (key >= N) break;
          float a = 0.f, rho = 0.f, sigma = 0.f, d4 = 0.f;
          if (key < valid) {
            float step, zp;
            if (p.meta_f16) load_meta<true>(kmeta, t + kKThreads * i, step, zp);
            else load_meta<false>(kmeta, t + kKThreads * i, step, zp);
            const float sp = step > 0.f ? step : 1.f;     // a constant group has code 0 everywhere
            a = sp * p.scale_log2;
            // rho = zp / step to within 2 ulp (reciprocal and multiply): its three bf16 parts keep
            // ~24 bits, so the IEEE division's last ulp is not resolved anyway.
            rho = __fdividef(zp, sp);
            sigma = step * p.inv_scale_log2;
            const float s2 = step * step;
            d4 = s2 * s2;                                 // fourth-order term (softmax, fp32)
          }
          const int ci = ci0 + i * (kKeyStepC / 2) * C::NAH * 4;
          kc[ci] = a;
          if (kQuartic) kc[2 * (C::kKconst / 4) + ci] = d4;   // read by the softmax with correct = 2 only
          // rho and sigma split together into three bf16 parts each (hi = RN(x), mid = RN(x - hi),
          // lo = RN(x - hi - mid)), as pairs (rho part, sigma part)
          const uint32_t hp = pack_bf16x2(rho, sigma);
          const float2 r1 = make_float2(rho - bf16_lo(hp), sigma - bf16_hi(hp));
          const uint32_t mp = pack_bf16x2(r1.x, r1.y);
          const uint32_t lp = pack_bf16x2(r1.x - bf16_lo(mp), r1.y - bf16_hi(mp));
          // [rho_h, rho_m, rho_h, rho_l, rho_m, rho_h, sig_h, sig_m, sig_h, sig_l, sig_h, sig_m, 0, 0, 0, 0]
          const uint32_t sig_hm = __byte_perm(hp, mp, 0x7632);
          // the extras row of (key, group): [row / 8][2 halves][row % 8][8] (store_extras' layout)
          uint8_t* xrow = bx + sb * C::kBx + xo0 + i * ((kKeyStepC / 8) * 256);
          *reinterpret_cast<uint4*>(xrow) = make_uint4(__byte_perm(hp, mp, 0x5410), __byte_perm(hp, lp, 0x5410),
                                                       __byte_perm(mp, hp, 0x5410), sig_hm);
          *reinterpret_cast<uint4*>(xrow + 128) = make_uint4(__byte_perm(hp, lp, 0x7632), sig_hm, 0u, 0u);
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(bar(B_KH_FULL + sb));
          mbar_arrive(bar(B_KC_FULL + sb));
          mbar_arrive(bar(B_PK_EMPTY + s));
        }
      } else {
        const int64_t t0 = static_cast<int64_t>(j - Tc) * N;
        const int valid = static_cast<int>(cur_keys - t0 < N ? cur_keys - t0 : N);
        const uint4* src = reinterpret_cast<const uint4*>(p.K_cur) + (static_cast<int64_t>(bh) * p.Lcur + t0) * (D / 8);
        copy_rows<D, N, kItersK, kKThreads, true>(src, kt, valid, t);
        fence_async_smem();
        // Scales of the current tile: the plain score scale for every key and group, so that the
        // softmax forms every tile's scores the same way.
        if (!warp_wait(bar(B_KC_EMPTY + sb), (n & 1) ^ 1, abort_flag, p.status, p.wait_limit)) break;
        float* kc = reinterpret_cast<float*>(kconst + sb * (C::kKconst / 16));
#pragma unroll 1
        for (int e = t; e < static_cast<int>(C::kKconst / 4); e += kKThreads) {
          kc[e] = p.scale_log2;
          kc[2 * (C::kKconst / 4) + e] = 0.f;        // no correction on current keys
        }
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(bar(B_KH_FULL + sb));
          mbar_arrive(bar(B_KC_FULL + sb));
        }
      }
    }
  } else if (wg == 3 || wg == 4) {
    // ---------------------------------------------------------------- V operand tiles
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegProducer));
    const int t = wg == 3 ? threadIdx.x - 384 : threadIdx.x - 32 * (16 + kKWarps - 3) + 128;  // 0 .. kVThreads - 1
    // This thread's items t, t + kVThreads, ...: one channel block, keys kKeyStepV apart.
    constexpr int kKeyStepV = kVThreads * 32 / D;
    static_assert((kVThreads * 32) % D == 0 && kKeyStepV % 8 == 0, "items of a thread share a block");
    const int vkey0 = item_key<D>(t), vblk0 = item_blk<D>(t);
    uint32_t vso[4];
    chunk_offsets<N>(vkey0, vblk0, vso);
    // Lane 0 of the first V warp also issues the bulk copies of packed tiles, kStages - 1 ahead.
    const bool loader = t == 0;
    const int64_t row_codes = D * BITS / 8;
    const int64_t row_meta = static_cast<int64_t>(NG) * 2 * (p.meta_f16 ? 2 : 4);
    int next_load = 0;
    auto issue_load = [&]() -> bool {
      const int s = next_load % kStages, k = next_load / kStages;
      if (!mbar_wait(bar(B_PK_EMPTY + s), (k & 1) ^ 1, abort_flag, p.status, p.wait_limit)) return false;
      const uint32_t dst = smem_u32(smem + L.pk + s * L.stage);
      const int64_t row0 = static_cast<int64_t>(bh) * p.capacity + static_cast<int64_t>(c0 + next_load) * N;
      const uint32_t fb = bar(B_PK_FULL + s);
      mbar_arrive_expect_tx(fb, 2 * (C::kCodes + L.meta));
      bulk_g2s(dst, p.k_codes + row0 * row_codes, C::kCodes, fb);
      bulk_g2s(dst + C::kCodes, static_cast<const uint8_t*>(p.k_meta) + row0 * row_meta, L.meta, fb);
      bulk_g2s(dst + C::kCodes + L.meta, p.v_codes + row0 * row_codes, C::kCodes, fb);
      bulk_g2s(dst + 2 * C::kCodes + L.meta, static_cast<const uint8_t*>(p.v_meta) + row0 * row_meta,
               L.meta, fb);
      ++next_load;
      return true;
    };
    bool load_ok = true;
    if (loader)
      while (load_ok && next_load < Tc && next_load < kStages) load_ok = issue_load();
    for (int j = 0; j < T; ++j) {
      const int sb = j & 1, n = j >> 1;
      uint8_t* vt = smem + L.vt + sb * C::kTile;
      if (!warp_wait(bar(B_VH_EMPTY + sb), (n & 1) ^ 1, abort_flag, p.status, p.wait_limit)) break;
      if (j < Tc) {
        const int s = j % kStages, k = j / kStages;
        const int64_t rem = p.Lc - static_cast<int64_t>(c0 + j) * N;
        const int valid = static_cast<int>(rem < N ? rem : N);
        const uint8_t* vcodes = smem + L.pk + s * L.stage + C::kCodes + L.meta;
        const uint8_t* vmeta = vcodes + C::kCodes;
        if (!warp_wait(bar(B_PK_FULL + s), k & 1, abort_flag, p.status, p.wait_limit)) break;
        using CodeVec = typename CodeVecT<BITS>::type;
        // One item per iteration with the next item's codes and (step, zero-point) already loaded
        // (shared-memory loads are slow while the tensor core reads its operands); the loop itself
        // is not unrolled.
        struct VItem { CodeVec cv; float st, zp; };
        constexpr int kRowCodes = D * BITS / 8;
        const int mb2 = p.meta_f16 ? 4 : 8;                       // bytes of one (step, zero-point)
        const uint8_t* csrc = vcodes + vkey0 * kRowCodes + vblk0 * (4 * BITS);
        const uint8_t* msrc = vmeta + (vkey0 * NG + (vblk0 * 32) / C::G) * mb2;
        const int mstep = kKeyStepV * NG * mb2;
        auto load_item = [&](const uint8_t* cp, const uint8_t* mp) {
          VItem r;
          r.cv = *reinterpret_cast<const CodeVec*>(cp);
          if (p.meta_f16) load_meta<true>(mp, 0, r.st, r.zp);
          else load_meta<false>(mp, 0, r.st, r.zp);
          return r;
        };
        VItem nxt = load_item(csrc, msrc);
        uint8_t* vrow = vt + vkey0 * 128;
        // Unrolled with one group (the long-video cache: 6.22 ms against 6.46), not with two (the
        // chunked-prefill and video shapes gain nothing or lose 1%: instruction-cache pressure).
#pragma unroll (NG == 1 ? kItersV : 1)
        for (int i = 0; i < kItersV; ++i) {
          const int key = vkey0 + kKeyStepV * i;
          if (key >= N) break;
          const VItem cur = nxt;
          if (i + 1 < kItersV && key + kKeyStepV < N)
            nxt = load_item(csrc + (i + 1) * (kKeyStepV * kRowCodes), msrc + (i + 1) * mstep);
          uint32_t v[16];
          if (key < valid) {
            dequant32(cur.cv, cur.st, cur.zp, v);
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) v[e] = 0u;
          }
          store_chunks(vrow + i * (kKeyStepV * 128), vso, v);
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(bar(B_VH_FULL + sb));
          mbar_arrive(bar(B_PK_EMPTY + s));
        }
        // Tile j + kStages reuses this stage once K is done with tile j too.
        if (loader && load_ok && next_load < Tc) load_ok = issue_load();
      } else {
        const int64_t t0 = static_cast<int64_t>(j - Tc) * N;
        const int valid = static_cast<int>(cur_keys - t0 < N ? cur_keys - t0 : N);
        const uint4* src = reinterpret_cast<const uint4*>(p.V_cur) + (static_cast<int64_t>(bh) * p.Lcur + t0) * (D / 8);
        copy_rows<D, N, kItersV, kVThreads, false>(src, vt, valid, t);
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
    const int half = wg - 1;                   // which half of every key tile
    const int quad = warp & 3;                 // TMEM lane quadrant of this warp
    const int row = quad * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const int64_t R = static_cast<int64_t>(m_tile) * kBM + row;
    const bool valid_row = R < rows_total;
    const int64_t hq = static_cast<int64_t>(h) * p.r + (valid_row ? R / p.Lq : 0);
    const int64_t qi = valid_row ? R % p.Lq : 0;
    const int64_t out_row = (static_cast<int64_t>(b) * p.Hq + hq) * p.Lq + qi;
    const int kbase_h = half * NH;             // first key of this warpgroup's half of a tile

    // Q row: group sums of q (what the codes multiply), correction weights; this half's columns of
    // the bf16 copy of Q go into TMEM.
    float w[kMaxGroups] = {0.f, 0.f, 0.f, 0.f};
    float u[kMaxGroups] = {0.f, 0.f, 0.f, 0.f};   // fourth-order weights (correct = 2)
    float qs[kMaxGroups] = {0.f, 0.f, 0.f, 0.f};
    {
      const uint8_t* qrow = static_cast<const uint8_t*>(p.Q) + out_row * D * 2;
      uint32_t qp[D / 4];
      if (valid_row) {
        query_group_powers<D>(qrow, false, C::G, p.wcoef_log2, kQuartic ? p.ucoef_log2 : 0.f, w, u);
#pragma unroll
        for (int c8 = 0; c8 < D / 8; ++c8) {
          float x[8];
          load_q8(qrow, false, c8, x);
          float acc = 0.f;
#pragma unroll
          for (int k = 0; k < 8; ++k) acc += x[k];
#pragma unroll
          for (int g = 0; g < NG; ++g)
            if (g == (c8 * 8) / C::G) qs[g] += acc;
        }
#pragma unroll
        for (int c8 = 0; c8 < D / 16; c8 += 2) {   // 16 channels at a time, in operand order
          const uint4 u0 = reinterpret_cast<const uint4*>(qrow)[half * (D / 16) + c8];
          const uint4 u1 = reinterpret_cast<const uint4*>(qrow)[half * (D / 16) + c8 + 1];
          const uint32_t nat[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
          permute16(nat, qp + 4 * c8);
        }
      } else {
#pragma unroll
        for (int k = 0; k < D / 4; ++k) qp[k] = 0u;
      }
      tmem_st<D / 4>(tmem + lane_off + kColQ + half * (D / 4), qp);
      if (half == 0) {
        // row extras per group [qs_h, qs_h, qs_m, qs_h, qs_m, qs_l, nw_h, nw_h, nw_m, nw_h, nw_l, nw_m,
        // 0..] against the key extras [rho_h, rho_m, rho_h, rho_l, rho_m, rho_h, sig_h, sig_m, sig_h,
        // sig_l, sig_h, sig_m, 0..]: every product of parts whose orders add up to at most two. The
        // fourth-order term (correct = 2) is added in the softmax in fp32 instead: for keys with
        // large steps its series term grows without bound, beyond what bf16 parts resolve.
#pragma unroll
        for (int g = 0; g < NG; ++g) {
          __nv_bfloat16 qh, qm, ql, nh, nm, nl;
          split3(qs[g], qh, qm, ql);
          split3(p.correct ? -w[g] : 0.f, nh, nm, nl);
          store_extras(ax + g * (kBM * 32), row,
                       make_uint4(bf_pair(qh, qh), bf_pair(qm, qh), bf_pair(qm, ql), bf_pair(nh, nh)),
                       make_uint4(bf_pair(nm, nh), bf_pair(nl, nm), 0u, 0u));
        }
        fence_async_smem();
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_Q_FULL));
    }
    if (!p.correct) {
#pragma unroll
      for (int g = 0; g < kMaxGroups; ++g) w[g] = 0.f;
    }

    constexpr bool quartic = kQuartic;   // correct = 2: fourth-order term in the softmax
    float m_run = -INFINITY;   // max used for the exponentials so far (log2 units), same in both halves
    float l_run = 0.f;         // this half's part of the softmax denominator
    const float2 scale2 = make_float2(p.scale_log2, p.scale_log2);
    // ok turns false when one of this warp's waits gives up. The eight softmax warps share named
    // barrier 1, so none of them leaves the tile loop on its own: a failed warp skips its work and
    // the warps leave together at the next row-max exchange, which ORs their failures, so that
    // every warp executes the same sequence of barriers (one per tile, then one in the epilogue).
    bool ok = true;
    // S columns are read in chunks of kCK keys (NA * kCK registers); tcgen05.wait::ld waits for
    // every load of a chunk.
    constexpr int kCK = C::NA == 1 ? 32 : 64 / C::NA;
    for (int j = 0; j < T; ++j) {
      const int kb = j & 1, sbuf = j % C::kSB, pb = j % C::kPB;
      const bool cached = j < Tc;
      if (ok && !warp_wait(bar(B_S_FULL + sbuf), (j / C::kSB) & 1, abort_flag, p.status, p.wait_limit)) ok = false;
      tc_fence_after();
      const uint32_t tm_s = tmem + lane_off + kColS + sbuf * C::kSCols + kbase_h;
      float2 s2[NH / 2];         // scores of this half's key pairs (log2 units)
      int valid;                 // keys of the whole tile that count for this row
      if (cached) {
        const int64_t rem = p.Lc - static_cast<int64_t>(c0 + j) * N;
        valid = static_cast<int>(rem < N ? rem : N);
      } else {
        const int64_t t0 = static_cast<int64_t>(j - Tc) * N;
        int64_t lim = cur_keys - t0;                       // keys of this tile that exist
        if (p.causal) {
          const int64_t c = qi + (p.Lcur - p.Lq) - t0 + 1;  // keys this row may see
          lim = c < lim ? c : lim;
        }
        valid = static_cast<int>(lim < 0 ? 0 : (lim < N ? lim : N));
      }
      // The first group's first chunk of S is loaded from tensor memory while this warp waits for
      // the tile's per-key scales.
      uint32_t r[C::NA][kCK];
      tmem_ld<kCK>(tm_s, r[0]);
      if (ok && !warp_wait(bar(B_KC_FULL + kb), (j >> 1) & 1, abort_flag, p.status, p.wait_limit)) ok = false;
      // s = sum_g a_g * S_g: per-key group scales for cached tiles, the score scale for current ones.
      const float4* ka = kconst + kb * (C::kKconst / 16);
      const float4* kd4 = kconst + (2 + kb) * (C::kKconst / 16);
      // Scores are formed relative to the maximum in use so far (m_prev, 0 before the first key):
      // the exponentials then need no subtraction unless the maximum moves, which lazy rescaling
      // makes rare.
      const float m_prev = m_run == -INFINITY ? 0.f : m_run;
      const float2 mprev2 = make_float2(-m_prev, -m_prev);
#pragma unroll
      for (int c0 = 0; c0 < NH; c0 += kCK) {
        // (After a failed wait these loads read whatever the accumulators hold; the values are
        // dropped at the exchange below, where the warps leave the loop.)
#pragma unroll
        for (int a = 0; a < C::NA; ++a)
          if (c0 > 0 || a > 0) tmem_ld<kCK>(tm_s + a * N + c0, r[a]);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < kCK / 2; ++q) {
          const int pq = (kbase_h + c0) / 2 + q;
          float2 acc = mprev2;                    // scores relative to the running maximum
#pragma unroll
          for (int ah = 0; ah < C::NAH; ++ah) {
            const float4 a = ka[pq * C::NAH + ah];
            acc = __ffma2_rn(make_float2(a.x, a.y),
                             make_float2(__uint_as_float(r[2 * ah][2 * q]), __uint_as_float(r[2 * ah][2 * q + 1])), acc);
            if (2 * ah + 1 < C::NA)
              acc = __ffma2_rn(make_float2(a.z, a.w),
                               make_float2(__uint_as_float(r[2 * ah + 1][2 * q]),
                                           __uint_as_float(r[2 * ah + 1][2 * q + 1])), acc);
            if (quartic) {                          // + u_g * step_g^4 (fourth-order term)
              const float4 d = kd4[pq * C::NAH + ah];
              acc = __ffma2_rn(make_float2(d.x, d.y), make_float2(u[2 * ah], u[2 * ah]), acc);
              if (2 * ah + 1 < C::NA)
                acc = __ffma2_rn(make_float2(d.z, d.w), make_float2(u[2 * ah + 1], u[2 * ah + 1]), acc);
            }
          }
          s2[c0 / 2 + q] = acc;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (ok && lane == 0) {
        mbar_arrive(bar(B_S_FREE + sbuf));
        mbar_arrive(bar(B_KC_EMPTY + kb));
      }
      if (valid < kbase_h + NH) {
#pragma unroll
        for (int q = 0; q < NH / 2; ++q) {
          if (kbase_h + 2 * q >= valid) s2[q].x = -INFINITY;
          if (kbase_h + 2 * q + 1 >= valid) s2[q].y = -INFINITY;
        }
      }
      // Row max of this half (four chains of 3-input maxima), then of the tile via shared memory.
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
      const bool any_need = __any_sync(0xffffffffu, need);
      // O is rescaled only after the previous P.V has finished (rare with lazy rescaling).
      if (j > 0 && any_need) {
        if (!warp_wait(bar(B_PV_DONE + (j - 1) % C::kPB), ((j - 1) / C::kPB) & 1, abort_flag, p.status, p.wait_limit)) { ok = false; continue; }
        tc_fence_after();
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
      // P buffer pb was last read by P_{j-kPB}.V_{j-kPB}.
      if (j >= C::kPB) {
        if (!warp_wait(bar(B_PV_DONE + pb), ((j - C::kPB) / C::kPB) & 1, abort_flag, p.status, p.wait_limit)) { ok = false; continue; }
        tc_fence_after();
      }
      if (any_need) {                           // the maximum moved: scores relative to the new one
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
      tmem_st<NH / 2>(tmem + lane_off + kColP + pb * (N / 2) + kbase_h / 2, pk);
      l_run += psum.x + psum.y;
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_P_FULL + pb));
    }

    // Epilogue: combine the two halves' denominators, O / l (each half writes half the columns), LSE.
    bool have_o = false;
    if (ok && T > 0) {
      have_o = warp_wait(bar(B_PV_DONE + (T - 1) % C::kPB), ((T - 1) / C::kPB) & 1, abort_flag, p.status, p.wait_limit);
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
            o4[e] = pack_bf16x2(__uint_as_float(r[8 * k + 2 * e]) * inv_l,
                                __uint_as_float(r[8 * k + 2 * e + 1]) * inv_l);
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

template <int D, int BITS, int NG, bool kQuartic>
cudaError_t launch_impl(const AttnParams& p, cudaStream_t stream) {
  const Layout L = make_layout<D, BITS, NG>(p.meta_f16 ? 2 : 4);
  // At least 116 KB so that two CTAs never share an SM: each holds all 512 TMEM columns.
  size_t smem = L.total + 1024;
  if (smem < 116u * 1024u) smem = 116u * 1024u;
  cudaError_t e = cudaFuncSetAttribute(corrected_attention_kernel<D, BITS, NG, kQuartic>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int64_t rows = static_cast<int64_t>(p.r) * p.Lq;
  dim3 grid(static_cast<unsigned>((rows + kBM - 1) / kBM), static_cast<unsigned>(p.B * p.Hkv),
            static_cast<unsigned>(p.n_split > 1 ? p.n_split : 1));
  corrected_attention_kernel<D, BITS, NG, kQuartic><<<grid, kThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

template <int D, int BITS>
cudaError_t launch_groups(const AttnParams& p, cudaStream_t stream) {
  const bool q4 = p.correct == 2;
  if (p.n_groups == 1) return q4 ? launch_impl<D, BITS, 1, true>(p, stream) : launch_impl<D, BITS, 1, false>(p, stream);
  if (p.n_groups == 2) return q4 ? launch_impl<D, BITS, 2, true>(p, stream) : launch_impl<D, BITS, 2, false>(p, stream);
  if constexpr (D == 128) {
    if (p.n_groups == 4) return q4 ? launch_impl<D, BITS, 4, true>(p, stream) : launch_impl<D, BITS, 4, false>(p, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

int attention_tile_keys(int n_groups) { return n_groups == 4 ? 64 : 128; }

cudaError_t launch_attention_bf16(const AttnParams& p, int d, int bits, cudaStream_t stream) {
  if (d == 128) return bits == 2 ? launch_groups<128, 2>(p, stream) : launch_groups<128, 4>(p, stream);
  return bits == 2 ? launch_groups<64, 2>(p, stream) : launch_groups<64, 4>(p, stream);
}

}  // namespace qkv
