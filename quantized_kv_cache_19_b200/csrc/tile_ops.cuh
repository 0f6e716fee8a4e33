// Device helpers shared by the attention kernels on the packed cache: unpacking of code tiles into
// bf16 tensor-core operands, dequantisation of V, the 128-byte-swizzled operand layout, the
// three-part bf16 split of the key and row extras, and tensor-memory load / store helpers.
#pragma once

#include "qkv_common.cuh"

namespace qkv {

constexpr uint32_t kCodeMagic = 0x43004300u;  // bf16 pair (128 + c_lo, 128 + c_hi)

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float y;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(y) : "f"(a), "f"(b), "f"(c));
  return y;
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Splits x into bf16 parts: x ~ hi + mid + lo.
__device__ __forceinline__ void split3(float x, __nv_bfloat16& hi, __nv_bfloat16& mid, __nv_bfloat16& lo) {
  hi = __float2bfloat16_rn(x);
  const float r1 = x - __bfloat162float(hi);
  mid = __float2bfloat16_rn(r1);
  lo = __float2bfloat16_rn(r1 - __bfloat162float(mid));
}

// 16 bf16 channels of one row of an extras tile in the no-swizzle K-major core-matrix layout
// [row / 8][2 halves][row % 8][8].
__device__ __forceinline__ void store_extras(uint8_t* tile, int row, uint4 lo8, uint4 hi8) {
  uint8_t* base = tile + (row >> 3) * 256 + (row & 7) * 16;
  *reinterpret_cast<uint4*>(base) = lo8;
  *reinterpret_cast<uint4*>(base + 128) = hi8;
}
__device__ __forceinline__ uint32_t bf_pair(__nv_bfloat16 lo, __nv_bfloat16 hi) {
  return static_cast<uint32_t>(__bfloat16_as_ushort(lo)) | (static_cast<uint32_t>(__bfloat16_as_ushort(hi)) << 16);
}

// Operand order of the channels of K (and of Q, which must match it) inside every block of 16
// channels: position 2k holds channel k and position 2k + 1 holds channel k + 8 (k = 0..7). With
// codes packed LSB-first, the codes of channels k and k + 8 then sit 16 bits apart in one 32-bit
// word, and one bf16x2 operand word is a shift and a masked OR, (128 + c_k, 128 + c_{k+8}) with the
// codes in the low mantissa bits of 128.0 (bf16 0x4300), and one exact bf16x2 subtraction of 128.
__device__ __forceinline__ uint32_t sub128(uint32_t v) {
  __nv_bfloat162 x = *reinterpret_cast<__nv_bfloat162*>(&v);
  x = __hsub2(x, __floats2bfloat162_rn(128.f, 128.f));
  return *reinterpret_cast<uint32_t*>(&x);
}
template <int BITS> struct CodeVecT { using type = uint2; };   // 32 codes: 8 bytes (INT2)
template <> struct CodeVecT<4> { using type = uint4; };            // 16 bytes (INT4)

// Arguments by value: taking the address of a register copy would move it to local memory.
__device__ __forceinline__ void unpack_codes32(uint2 w2, uint32_t (&out)[16]) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {       // one word = 16 codes = one channel block, code k at bits 2k
    const uint32_t w = h ? w2.y : w2.x;
#pragma unroll
    for (int k = 0; k < 8; ++k) out[h * 8 + k] = sub128(((w >> (2 * k)) & 0x00030003u) | kCodeMagic);
  }
}
__device__ __forceinline__ void unpack_codes32(uint4 w4, uint32_t (&out)[16]) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {       // two words = 16 codes = one channel block, code k at bits 4k
    const uint32_t a = h ? w4.z : w4.x, b = h ? w4.w : w4.y;
    const uint32_t lo = __byte_perm(a, b, 0x5410);   // codes 0-3 | codes 8-11 << 16
    const uint32_t hi = __byte_perm(a, b, 0x7632);   // codes 4-7 | codes 12-15 << 16
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      out[h * 8 + k] = sub128(((lo >> (4 * k)) & 0x000F000Fu) | kCodeMagic);
      out[h * 8 + 4 + k] = sub128(((hi >> (4 * k)) & 0x000F000Fu) | kCodeMagic);
    }
  }
}

// The same channel order applied to 8 bf16x2 words (16 channels, natural order) of Q or K_cur.
__device__ __forceinline__ void permute16(const uint32_t* in, uint32_t* out) {
#pragma unroll
  for (int k = 0; k < 8; ++k) out[k] = __byte_perm(in[k >> 1], in[4 + (k >> 1)], (k & 1) ? 0x7632 : 0x5410);
}

// Dequantises 32 channels: x_hat = zp + step * code (fp32 FMA on a float whose mantissa holds the
// code, 1 + code * 2^-k, so no integer conversion is needed), rounded to bf16.
__device__ __forceinline__ void dequant32(uint2 w2, float step, float zp, uint32_t (&out)[16]) {
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
      const float2 x = __ffma2_rn(make_float2(s16, s4), make_float2(lo, hi), make_float2(c16, c4));
      out[h * 8 + p] = pack_bf16x2(x.x, x.y);
    }
  }
}
__device__ __forceinline__ void dequant32(uint4 w4, float step, float zp, uint32_t (&out)[16]) {
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
      const float2 x = __ffma2_rn(make_float2(s256, s16), make_float2(lo, hi), make_float2(c256, c16));
      out[h * 4 + p] = pack_bf16x2(x.x, x.y);
    }
  }
}

// (key, 32-channel block) of item `it` of a tile: eight consecutive items are eight consecutive
// keys of one block, so that the 16-byte stores of a quarter-warp into a 128B-swizzled tile land
// in eight different bank groups (keys of one block are 128 bytes apart, chunk c of key r sits at
// chunk position c ^ (r & 7)).
template <int D>
__device__ __forceinline__ int item_key(int it) { return (it & 7) + ((it >> 3) / (D / 32)) * 8; }
template <int D>
__device__ __forceinline__ int item_blk(int it) { return (it >> 3) % (D / 32); }

// Stores 32 channels (16 bf16x2) of row `key`, channel block `blk`, into a [d/64][N][64] bf16 tile
// with the 128-byte swizzle.
template <int N>
__device__ __forceinline__ void store32(uint8_t* tile, int key, int blk, const uint32_t (&v)[16]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int c = blk * 4 + i;               // 16-byte chunk of the row (8 channels)
    uint8_t* dst = tile + (c >> 3) * (N * 128) + sw128_offset(key, c & 7);
    *reinterpret_cast<uint4*>(dst) = make_uint4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
  }
}

// The 16-byte chunks of one (key, 32-channel block) item in a [d/64][N][64] tile with the 128-byte
// swizzle, as byte offsets from the start of the key's row (tile + key * 128; store32 writes the
// same addresses). They depend on the key only through key % 8, so a thread whose items lie a
// multiple of 8 keys apart keeps them for all its items and advances one row pointer.
template <int N>
__device__ __forceinline__ void chunk_offsets(int key, int blk, uint32_t (&o)[4]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int c = blk * 4 + i;
    o[i] = (c >> 3) * (N * 128) + (((c & 7) ^ (key & 7)) << 4);
  }
}
__device__ __forceinline__ void store_chunks(uint8_t* row, const uint32_t (&o)[4], const uint32_t (&v)[16]) {
#pragma unroll
  for (int i = 0; i < 4; ++i)
    *reinterpret_cast<uint4*>(row + o[i]) = make_uint4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
}

template <bool F16>
__device__ __forceinline__ void load_meta(const uint8_t* meta, int idx, float& step, float& zp) {
  if (F16) {
    const __half2 m = reinterpret_cast<const __half2*>(meta)[idx];
    step = __low2float(m);
    zp = __high2float(m);
  } else {
    const float2 m = reinterpret_cast<const float2*>(meta)[idx];
    step = m.x;
    zp = m.y;
  }
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t* r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
               "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}
__device__ __forceinline__ void tmem_ld16p(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}
// NC consecutive columns (a multiple of 8) of this thread's TMEM lane, from / into a register array.
template <int NC>
__device__ __forceinline__ void tmem_st(uint32_t taddr, const uint32_t* r) {
  static_assert(NC % 8 == 0, "");
#pragma unroll
  for (int c = 0; c < NC;) {
    if (c + 32 <= NC) {
      uint32_t t[32];
#pragma unroll
      for (int k = 0; k < 32; ++k) t[k] = r[c + k];
      tmem_st32(taddr + c, t);
      c += 32;
    } else if (c + 16 <= NC) {
      tmem_st16(taddr + c, r + c);
      c += 16;
    } else {
      tmem_st8(taddr + c, r + c);
      c += 8;
    }
  }
}
template <int NC>
__device__ __forceinline__ void tmem_ld(uint32_t taddr, uint32_t* r) {
  static_assert(NC % 16 == 0, "");
#pragma unroll
  for (int c = 0; c < NC;) {
    if (c + 32 <= NC) {
      tmem_ld32p(taddr + c, r + c);
      c += 32;
    } else {
      tmem_ld16p(taddr + c, r + c);
      c += 16;
    }
  }
}
__device__ __forceinline__ void named_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

}  // namespace qkv
