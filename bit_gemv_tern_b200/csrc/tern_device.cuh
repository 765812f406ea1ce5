// Device helpers shared by the sm_100a kernels of libterngemv.so.
//
// Decode of the packed layout (include/tern.h): a row stores, per 32 trits, one mask word m
// (bit = t != 0) and one sign word s (bit = t == -1) whose bit order is the mask order rotated by
// one. Merging the two words gives two words of sixteen 2-bit fields (mask bit low, sign bit high):
//   wa = (m & 0x55555555) | (s & 0xAAAAAAAA)          fields of the trits on even mask bits
//   wb = rotr((m & 0xAAAAAAAA) | (s & 0x55555555), 1) fields of the trits on odd mask bits
// A field (m, s) read as a 2-bit two's-complement number is exactly t (00 = 0, 01 = +1,
// 11 = -1), so a field moved to the top two bits of a byte is the int8 value 64*t, and a field in
// the top two bits of a 16-bit half is the bf16 (or fp16) value 2.0*t. One shift and one AND
// produce a whole tensor-core operand register: this is the add / skip / subtract rule of the
// ternary weights (origotech.dev "더 적은 비트로 계산하기", Figure I) carried out by the tensor
// cores with exact +-1 products.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace tern {

constexpr int kThreads = 256;  // 8 warps per CTA for the matrix kernels

// ---- programmatic dependent launch -----------------------------------------------------------
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---- global loads ------------------------------------------------------------------------------
// Streaming 128-bit load for data read exactly once (weights): bypasses L1 allocation.
__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}
__device__ __forceinline__ uint4 ld_nc(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

// ---- warp-level tensor-core products -------------------------------------------------------------
// D(16x8) += A(16x32, s8, row) * B(32x8, s8, col), s32 accumulate.
__device__ __forceinline__ void mma_s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                       uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// D(16x8) += A(16x16, bf16, row) * B(16x8, bf16, col), f32 accumulate.
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D(16x8) += A(16x32, u8, row) * B(32x8, s8, col), s32 accumulate.
__device__ __forceinline__ void mma_u8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// ---- decode ------------------------------------------------------------------------------------
// One three-input logic operation with an immediate truth table (lut bit (a<<2 | b<<1 | c) is the
// result for those input bits). Written out because the compiler does not always fold a merge of
// two planes under two complementary constants into a single operation.
template <uint32_t LUT>
__device__ __forceinline__ uint32_t lop3(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, %4;" : "=r"(d) : "r"(a), "r"(b), "r"(c), "n"(LUT));
  return d;
}

// Offset-binary merge: fields (m, NOT s) read as an unsigned 2-bit number equal t + 2
// (t = 0 -> 2, t = +1 -> 3, t = -1 -> 1). A field left in place at bit 2i of a byte and masked is
// the u8 value 4^i * (t + 2): one AND per tensor-core register, no shift. Sums then carry a known
// offset 2 * sum(x) that is removed exactly.
//   wa = (m & C) | (~s & ~C),  v = (m & ~C) | (~s & C),  C = 0x55555555:  one LOP3 each
__device__ __forceinline__ void merge_planes_offset(uint32_t m, uint32_t s, uint32_t& wa, uint32_t& wb) {
  wa = lop3<0xB1u>(m, s, 0x55555555u);
  const uint32_t v = lop3<0x72u>(m, s, 0x55555555u);
  wb = __funnelshift_r(v, v, 1);
}

//   wa = (m & C) | (s & ~C),  v = (m & ~C) | (s & C),  C = 0x55555555:  one LOP3 each
__device__ __forceinline__ void merge_planes(uint32_t m, uint32_t s, uint32_t& wa, uint32_t& wb) {
  wa = lop3<0xE4u>(m, s, 0x55555555u);
  const uint32_t v = lop3<0xD8u>(m, s, 0x55555555u);
  wb = __funnelshift_r(v, v, 1);
}

// int8 operand register R (0..7) of a 32-trit word: bytes hold 64*t for the four trits
//   R < 4: fields R, R+4, R+8, R+12 of wa;  R >= 4: the same fields (R-4, ...) of wb.
// In-word trit offsets of bytes 0..3: R < 4: {2R, 2R+8, 2R+1, 2R+9}; R >= 4: 16 + the same.
template <int R>
__device__ __forceinline__ uint32_t dec_i8(uint32_t wa, uint32_t wb) {
  constexpr int i = R & 3;
  return ((R < 4 ? wa : wb) << (6 - 2 * i)) & 0xC0C0C0C0u;
}

// bf16 operand register A (0..15) of a 32-trit word: low half = trit 2A, high half = trit 2A+1
// (in-word offsets), each as the bf16 value 2.0*t.
//   A < 8: fields A and A+8 of wa;  A >= 8: fields A-8 and A of wb.
template <int A>
__device__ __forceinline__ uint32_t dec_bf16(uint32_t wa, uint32_t wb) {
  constexpr int f = A & 7;
  return ((A < 8 ? wa : wb) << (14 - 2 * f)) & 0xC000C000u;
}

// int8 activations, permuted once per CTA so that activation word R of each 32-byte block holds
// the four bytes that dec_i8<R> pairs with. `lo` holds bytes 0..15 (or 16..31) of the block.
__device__ __forceinline__ uint4 permute_i8_half(uint4 lo) {
  uint4 o;
  o.x = __byte_perm(lo.x, lo.z, 0x5140);
  o.y = __byte_perm(lo.x, lo.z, 0x7362);
  o.z = __byte_perm(lo.y, lo.w, 0x5140);
  o.w = __byte_perm(lo.y, lo.w, 0x7362);
  return o;
}

// fp16 bit pattern -> float (exact).
__device__ __forceinline__ float f16_bits_to_float(uint16_t h) {
  return __half2float(__ushort_as_half(h));
}
__device__ __forceinline__ float bf16_bits_to_float(uint32_t b) { return __uint_as_float(b << 16); }

// ---- bf16 activations as exact integer limbs ----------------------------------------------------
// A group of bf16 activations with absmax < 2^E (E from frexp of the absmax; E = 0 for an all-zero
// group) becomes X = rint(x * 2^(kLimbFrac - E)), |X| <= 2^30, split into four int8 limbs
//   X = L3 * 2^24 + L2 * 2^16 + L1 * 2^8 + L0,   L0..L2 in [-128, 127], |L3| <= 64.
// Every tensor-core product with a limb is exact and every sum is an exact integer, so the only
// rounding of the bf16 paths is this encoding (|x - X * 2^(E - 30)| <= 2^(E - 31), zero for every x
// with |x| >= 2^(E - 23)) and the final conversion to fp32. Per output the encoding error is at
// most scale * K * 2^(E - 31) <= scale * K * 2^-30 * sum_k |x_k|, i.e. within 1e-4 * scale *
// sum_k |x_k| for every K up to 107,000, whatever the inputs' dynamic range.
constexpr int kLimbFrac = 30;
// 2^s for -126 <= s <= 127, from the exponent field (exact).
__device__ __forceinline__ float exp2f_i(int s) { return __int_as_float((s + 127) << 23); }
// x * 2^(kLimbFrac - E) rounded half to even: one or two exact power-of-two multiplies (the
// factor exceeds fp32's range only for E < -96, i.e. groups whose absmax is below 2^-97).
__device__ __forceinline__ int limb_fixed(float x, int E) {
  const int s = kLimbFrac - E;
  const float v = s <= 126 ? __fmul_rn(x, exp2f_i(s)) : __fmul_rn(__fmul_rn(x, exp2f_i(64)), exp2f_i(s - 64));
  return __float2int_rn(v);
}
// The group exponent E of an absmax a >= 0: a < 2^E, and 2^(E-1) <= a when a > 0.
__device__ __forceinline__ int limb_exponent(float a) {
  int E = 0;
  if (a > 0.0f) frexpf(a, &E);
  return E;
}
// Four limbs of X (top limb first) as bytes of the same position in four registers.
__device__ __forceinline__ void limbs_of(int X, int (&L)[4]) {
  L[3] = (int)(int8_t)(X & 0xFF);
  X = (X - L[3]) >> 8;
  L[2] = (int)(int8_t)(X & 0xFF);
  X = (X - L[2]) >> 8;
  L[1] = (int)(int8_t)(X & 0xFF);
  L[0] = (X - L[1]) >> 8;                 // |L[0]| <= 64
}
// The limbs of four values at once, as four operand registers: out[c] holds limb c (top first) of
// X[0..3] in bytes 0..3, the bytes limbs_of gives one value at a time. Balanced base-256 digits:
// with Y = X + 0x808080 each of Y's three low bytes is its digit plus 128 and Y's top byte is the
// top digit (|top| <= 64), so a 4 x 4 byte transpose of the Y's and a flip of bit 7 of the three
// low digits make the operands.
__device__ __forceinline__ void limbs4_of(const int (&X)[4], uint32_t (&out)[4]) {
  const uint32_t y0 = (uint32_t)X[0] + 0x00808080u, y1 = (uint32_t)X[1] + 0x00808080u;
  const uint32_t y2 = (uint32_t)X[2] + 0x00808080u, y3 = (uint32_t)X[3] + 0x00808080u;
  const uint32_t a = __byte_perm(y0, y1, 0x5140), b = __byte_perm(y0, y1, 0x7362);   // bytes 0,1 | 2,3
  const uint32_t c = __byte_perm(y2, y3, 0x5140), d = __byte_perm(y2, y3, 0x7362);
  out[3] = __byte_perm(a, c, 0x5410) ^ 0x80808080u;            // byte 0 of each: the lowest limb
  out[2] = __byte_perm(a, c, 0x7632) ^ 0x80808080u;
  out[1] = __byte_perm(b, d, 0x5410) ^ 0x80808080u;
  out[0] = __byte_perm(b, d, 0x7632);                           // byte 3: the top limb
}
// The limbs of 4·G bf16 values (packed two per word in wv, element 2i in the low half of word i)
// relative to 2^E: l[c][g] holds limb c (top first) of elements 4g .. 4g + 3, one per byte.
template <int G>
__device__ __forceinline__ void limbs_of_bf16(const uint32_t (&wv)[2 * G], int E, uint32_t (&l)[4][G]) {
#pragma unroll
  for (int g = 0; g < G; ++g) {
    int X[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t w2 = wv[2 * g + (e >> 1)];
      X[e] = limb_fixed(bf16_bits_to_float((e & 1) ? (w2 >> 16) : (w2 & 0xFFFFu)), E);
    }
    uint32_t o[4];
    limbs4_of(X, o);
#pragma unroll
    for (int c = 0; c < 4; ++c) l[c][g] = o[c];
  }
}
// Exact recombination of the four limb sums S[0] (top) .. S[3]: fits int64 for K < 2^24.
__device__ __forceinline__ long long limb_combine(long long s3, long long s2, long long s1, long long s0) {
  return s3 * 16777216LL + s2 * 65536LL + s1 * 256LL + s0;
}

// Monotone 32-bit key of a float (larger float -> larger key; -0 and +0 give the same key).
__device__ __forceinline__ uint32_t float_order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float float_from_order_key(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// ---- activation prologues ------------------------------------------------------------------------
// fp64 -> bf16 bit pattern, round to nearest, ties to even, as one correctly rounded step (never
// a double rounding): the value keeps 8 significant bits on the grid of its binade, or the
// subnormal grid 2^-133 below 2^-126, and values from halfway past the largest finite bf16 on
// become infinity. NaN maps to the canonical quiet NaN. Done through fp32 by rounding to odd
// (Boldo and Melquiond, "Emulation of FMA and correctly rounded sums: proved algorithms using
// rounding to odd", IEEE TC 2008): truncate to fp32 and set the last bit when the truncation was
// inexact, then round that to nearest even at bf16's last bit; fp32 carries 16 more bits than bf16
// and the same exponent range (subnormals included), so the result is the correctly rounded one.
__device__ __forceinline__ uint16_t bf16_rn(double v) {
  if (v != v) return 0x7FC0;
  const float f = __double2float_rz(v);                          // toward zero (fp32 max on overflow)
  uint32_t b = __float_as_uint(f);
  if ((double)f != v) b |= 1u;                                  // round to odd: the sticky bit
  b += 0x7FFFu + ((b >> 16) & 1u);                              // nearest even at bit 16
  return (uint16_t)(b >> 16);
}

// The int8 quantiser of one activation: clamp(rint(x / s), -127, 127), fp32 round-to-nearest
// division and round half to even; s = 0 (an all-zero row) gives 0.
__device__ __forceinline__ int quant_i8(float x, float s) {
  if (s == 0.0f) return 0;
  const int q = __float2int_rn(__fdiv_rn(x, s));
  return q > 127 ? 127 : (q < -127 ? -127 : q);
}

}  // namespace tern
