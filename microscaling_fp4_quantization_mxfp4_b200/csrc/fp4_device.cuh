// Device-side building blocks shared by the quantize, dequantize and GEMM
// kernels of libfp4 (sm_100a only).
//
// Formats follow the OCP MX v1.0 conventions (the pages name E2M1, E8M0-style
// power-of-two scales for MXFP4 and E4M3 scales for NVFP4 -- "FP4 All the
// Way", Abstract; "Bridging the Gap ...", Abstract -- but print no encodings).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace fp4dev {

// ---------------------------------------------------------------- bf16 -----
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ void unpack8(const uint4& v, float (&x)[8]) {
  x[0] = bf16_lo(v.x); x[1] = bf16_hi(v.x);
  x[2] = bf16_lo(v.y); x[3] = bf16_hi(v.y);
  x[4] = bf16_lo(v.z); x[5] = bf16_hi(v.z);
  x[6] = bf16_lo(v.w); x[7] = bf16_hi(v.w);
}

// ------------------------------------------------------------ E2M1 codes ---
// Eight E2M1 codes (element i in nibble i of w) -> their values as four f16 pairs, element 2k in
// the low half of h[k].
__device__ __forceinline__ void e2m1x8_to_f16x2(uint32_t w, uint32_t (&h)[4]) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
      : "r"(w));
}


// Hardware conversion: round to nearest even, saturating to +-6, sign kept.
// Element `a` lands in the low nibble, `b` in the high nibble.
__device__ __forceinline__ uint32_t e2m1x4_rn(float a0, float b0, float a1, float b1,
                                              float a2, float b2, float a3, float b3) {
  uint32_t out;
  asm("{\n\t.reg .b8 q0, q1, q2, q3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q3, %8, %7;\n\t"
      "mov.b32 %0, {q0, q1, q2, q3};\n\t}"
      : "=r"(out)
      : "f"(a0), "f"(b0), "f"(a1), "f"(b1), "f"(a2), "f"(b2), "f"(a3), "f"(b3));
  return out;
}

// 8 scaled values -> 8 packed RTN nibbles (element 2j low, 2j+1 high).
__device__ __forceinline__ uint32_t pack8_rtn(const float (&v)[8]) {
  return e2m1x4_rn(v[0], v[1], v[2], v[3], v[4], v[5], v[6], v[7]);
}

// a * b + c on the integer multiply-add path (keeps shifts-and-ors of packing
// and key arithmetic off the ALU pipe, which the stochastic-rounding kernels saturate).
__device__ __forceinline__ uint32_t mad_u32(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("mad.lo.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// Stochastic rounding of one scaled value with a 32-bit random word; returns
// the 4-bit code with the sign in bit 3.  lo <= |v| < hi adjacent grid points,
// p = (|v| - lo) / (hi - lo) (exact in fp32), round up iff r < ceil(p * 2^32);
// |v| >= 6 gives 6; sign kept.  With a = min(|v|, 6):
//  * a >= 1: the grid step is a quarter of a's binade, so p * 2^32 = f * 2^10 for
//    the low 22 significand bits f of a, and "r < f * 2^10" is "(r >> 10) < f",
//    i.e. the carry out of f + ((~r) >> 10) into bit 22.  The sum, shifted right by
//    22, is the binade and top significand bit of the rounded value, which are its
//    code plus 252: (A + 2^22 - 1 - (r >> 10) - 252 * 2^22) >> 22 for A = bits(a)
//    (codes 2 .. 7; 6 has f = 0 and never rounds up).
//  * a < 1: the step is 0.5, so with C = ceil(a * 2^33) (a * 2^33 is exact, below
//    2^33), floor(2a) = C >> 32 is the lower point's code (0 or 1) and C mod 2^32 =
//    ceil(p * 2^32) the threshold: code = (C >> 32) + (r < C mod 2^32).
__device__ __forceinline__ uint32_t e2m1_sr(float v, uint32_t r) {
  const float a = fminf(fabsf(v), 6.0f);
  const uint32_t big = (__float_as_uint(a) + (0x003FFFFFu - 0x3F000000u) - (r >> 10)) >> 22;
  const unsigned long long c = __float2ull_ru(__fmul_rn(a, 0x1p33f));
  const uint32_t small = (uint32_t)(c >> 32) + (r < (uint32_t)c ? 1u : 0u);
  return (a < 1.0f ? small : big) | ((__float_as_uint(v) >> 28) & 8u);
}

// Eight 4-bit codes, element i in nibble i, packed with multiply-adds.
__device__ __forceinline__ uint32_t pack8_nibbles(const uint32_t (&n)[8]) {
  const uint32_t a = mad_u32(n[1], 16u, n[0]), b = mad_u32(n[3], 16u, n[2]);
  const uint32_t c = mad_u32(n[5], 16u, n[4]), d = mad_u32(n[7], 16u, n[6]);
  return mad_u32(mad_u32(d, 256u, c), 65536u, mad_u32(b, 256u, a));
}

// ------------------------------------------------------- scale division -----
// x / S rounded to nearest-even, bit-identical to IEEE division, from the
// correctly rounded reciprocal y = RN(1/S) shared by a whole block:
// q0 = RN(x*y) is within 1.5 ulp of x/S; one FMA correction
// q1 = RN(q0 + (x - S*q0)*y) is faithful, and a second correction with a
// faithful quotient and y = RN(1/S) is correctly rounded (Markstein's
// theorem).  The residual is formed as -(S*q - x), which keeps the sign of a
// zero dividend through both corrections.  Valid when the residuals are exact
// and the quotient normal: |x| >= 2^-103 or x == 0, with S in
// [2^-125, 2^20] (recip_usable); callers check that per block and fall back
// to the IEEE division otherwise.  The quotient must also stay far from
// overflow (|x| * y < 2^64), or the corrections turn an infinite quotient into
// NaN; the quantizers check the block maximum.
__device__ __forceinline__ float div_by_recip(float x, float S, float y) {
  float q = __fmul_rn(x, y);
  float r = -__fmaf_rn(q, S, -x);
  q = __fmaf_rn(r, y, q);
  r = -__fmaf_rn(q, S, -x);
  return __fmaf_rn(r, y, q);
}
// x / S rounded to nearest-even through fp64: q = RN32(x * yd) with yd = RN64(1/S).
// For any fp32 x (at most 24 significant bits) and fp32 S > 0 this is the IEEE
// fp32 quotient whenever that quotient is normal: x / S cannot lie exactly on a
// rounding midpoint of fp32 (the midpoint's 25-bit odd significand would have to
// divide x's), and when it is not on one it is at least 2^-49 (relative) away
// from every midpoint (the residual x - m * S is a nonzero multiple of
// m's and S's last-place product), while x * yd in fp64 is within 2^-52 of x / S.
// Quotients below 2^-126 may round differently only at subnormal midpoints; the
// quantizers use such a quotient only through its E2M1 code (RTN: a signed zero
// either way) or its threshold ceil(|q| * 2^33) (1 for every nonzero |q| below
// 2^-33), and its zero-ness agrees: the one tie that decides it, x / S = 2^-150,
// gives RN64(a * RN64(1/a)) <= 1 (a the significand), which rounds to 0 as the
// IEEE division's tie-to-even does.  So the codes are those of IEEE division.
__device__ __forceinline__ float div_by_recip64(float x, double yd) {
  return __double2float_rn(__dmul_rn((double)x, yd));
}
// Running minimum over a block of 2*|x| - 2 as an unsigned integer (zeros wrap
// to the top): the block passes div_by_recip's |x| >= 2^-103 test iff the
// minimum is >= 2*bits(2^-103) - 2.
__device__ __forceinline__ uint32_t tiny_key(float x) { return mad_u32(__float_as_uint(x), 2u, 0xFFFFFFFEu); }
constexpr uint32_t kTinyKeyMin = (0x0C000000u << 1) - 2u;     // 2^-103 = biased exponent 24
__device__ __forceinline__ bool recip_usable(float S) { return S >= 0x1p-125f && S <= 0x1p+20f; }

// ---------------------------------------------------------------- Philox ----
// Philox4x32 with 10 rounds (Salmon, Moraes, Dror, Shaw, SC'11): two 32x32
// multiplies per round with the published multipliers, Weyl key schedule.
struct u32x4 { uint32_t x, y, z, w; };

__device__ __forceinline__ u32x4 philox4x32_10(uint32_t c0, uint32_t c1, uint32_t k0, uint32_t k1) {
  uint32_t c2 = 0u, c3 = 0u;
#pragma unroll
  for (int i = 0; i < 10; ++i) {
    const unsigned long long p0 = (unsigned long long)0xD2511F53u * c0;   // one wide multiply each
    const unsigned long long p1 = (unsigned long long)0xCD9E8D57u * c2;
    const uint32_t n0 = (uint32_t)(p1 >> 32) ^ c1 ^ k0;
    const uint32_t n2 = (uint32_t)(p0 >> 32) ^ c3 ^ k1;
    c0 = n0; c1 = (uint32_t)p1; c2 = n2; c3 = (uint32_t)p0;
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  return {c0, c1, c2, c3};
}

// The same generator with its key schedule (k0 + i * 0x9E3779B9, k1 + i * 0xBB67AE85 for round
// i = 0..9, interleaved) precomputed on the host and read from kernel parameters: the rounds then
// take their keys straight from the constant bank instead of adding them up per call.
struct PhiloxKeys {
  uint32_t k[20];
};

__device__ __forceinline__ u32x4 philox4x32_10(uint32_t c0, uint32_t c1, const PhiloxKeys& ks) {
  uint32_t c2 = 0u, c3 = 0u;
#pragma unroll
  for (int i = 0; i < 10; ++i) {
    const unsigned long long p0 = (unsigned long long)0xD2511F53u * c0;
    const unsigned long long p1 = (unsigned long long)0xCD9E8D57u * c2;
    const uint32_t n0 = (uint32_t)(p1 >> 32) ^ c1 ^ ks.k[2 * i];
    const uint32_t n2 = (uint32_t)(p0 >> 32) ^ c3 ^ ks.k[2 * i + 1];
    c0 = n0; c1 = (uint32_t)p1; c2 = n2; c3 = (uint32_t)p0;
  }
  return {c0, c1, c2, c3};
}

// Philox4x32-10 key schedule of a 64-bit seed: round i uses (lo + i * 0x9E3779B9, hi + i * 0xBB67AE85).
inline PhiloxKeys philox_keys(unsigned long long seed) {
  PhiloxKeys ks;
  uint32_t k0 = (uint32_t)seed, k1 = (uint32_t)(seed >> 32);
  for (int i = 0; i < 10; ++i) {
    ks.k[2 * i] = k0;
    ks.k[2 * i + 1] = k1;
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  return ks;
}

// Random words for 8 consecutive elements starting at linear index idx0
// (idx0 % 8 == 0): two counters, words in index order.
__device__ __forceinline__ void philox_words8(unsigned long long idx0, unsigned long long seed,
                                              uint32_t (&r)[8]) {
  const unsigned long long j = idx0 >> 2;
  const uint32_t k0 = (uint32_t)seed, k1 = (uint32_t)(seed >> 32);
  const u32x4 a = philox4x32_10((uint32_t)j, (uint32_t)(j >> 32), k0, k1);
  const u32x4 b = philox4x32_10((uint32_t)(j + 1), (uint32_t)((j + 1) >> 32), k0, k1);
  r[0] = a.x; r[1] = a.y; r[2] = a.z; r[3] = a.w;
  r[4] = b.x; r[5] = b.y; r[6] = b.z; r[7] = b.w;
}

// Random word of one element.
__device__ __forceinline__ uint32_t philox_word(unsigned long long idx, unsigned long long seed) {
  const unsigned long long j = idx >> 2;
  const u32x4 a = philox4x32_10((uint32_t)j, (uint32_t)(j >> 32), (uint32_t)seed, (uint32_t)(seed >> 32));
  const uint32_t s = (uint32_t)(idx & 3u);
  return s == 0 ? a.x : (s == 1 ? a.y : (s == 2 ? a.z : a.w));
}

// ------------------------------------------------------------ MX scales -----
// E = clamp(floor(log2 amax) - 2, -127, 127); byte = E + 127.  For a finite
// amax with biased exponent field f, floor(log2 amax) = f - 127 when f > 0,
// and E clamps to -127 for zero or subnormal amax: byte = max(f - 2, 0).
__device__ __forceinline__ uint32_t mx_scale_byte(float amax) {
  const int f = (int)((__float_as_uint(amax) >> 23) & 0xFFu);
  return (uint32_t)max(f - 2, 0);
}
// The same exponent under a clip threshold T in (4, 8]: E = floor(log2 amax) - 2, plus one when
// amax > T * 2^(floor(log2 amax) - 2), i.e. when amax's significand field exceeds
// thr = (T/4 - 1) * 2^23.  thr = 2^23 never triggers (T = 8, the rule above).
__device__ __forceinline__ uint32_t mx_scale_byte_clip(float amax, uint32_t thr) {
  const uint32_t b = __float_as_uint(amax);
  const int f = (int)((b >> 23) & 0xFFu);
  return (uint32_t)max(f - 2 + ((b & 0x7FFFFFu) > thr ? 1 : 0), 0);
}
// Significand threshold of the MSE-fitted clip T = 7.25 (T/4 = 1.8125 = 1 + 0x680000 / 2^23),
// and of the OCP rule (T = 8).
constexpr uint32_t kMxClipFitted = 0x680000u;
constexpr uint32_t kMxClipOcp = 0x800000u;
// 2^(127 - byte) = 1 / 2^E as an exact fp32 (byte <= 252 for finite bf16 input).
__device__ __forceinline__ float mx_inv_scale(uint32_t byte) {
  return __uint_as_float((254u - byte) << 23);
}
// 2^(byte - 127) exactly (byte 0 is the subnormal 2^-127).
__device__ __forceinline__ float mx_scale_value(uint32_t byte) {
  return byte == 0u ? __uint_as_float(0x00400000u) : __uint_as_float(byte << 23);
}

// ------------------------------------------------------------ NV scales -----
// E4M3 byte of min(t, 448) with round-to-nearest-even and saturation.
__device__ __forceinline__ uint32_t e4m3_rn_sat(float t) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(fminf(t, 448.0f)));
  return (uint32_t)(r & 0xFFu);
}
// Value of an E4M3 byte (non-negative; bias 7, subnormals m * 2^-9).
__device__ __forceinline__ float e4m3_value(uint32_t b) {
  const uint32_t e = (b >> 3) & 0xFu, m = b & 7u;
  if (e == 0u) return __fmul_rn((float)m, 0.001953125f);                 // m * 2^-9, exact
  return __uint_as_float(((e + 120u) << 23) | (m << 20));                // (1 + m/8) * 2^(e-7)
}

// NVFP4 block-scale argument t = RN(RN(amax_b / 6) / s_t), bit-identical to two
// IEEE divisions, from RN(1/6) and y_st = RN(1/s_t) (st_ok: recip_usable(s_t)).
__device__ __forceinline__ float nv_scale_arg(float am, float s_t, float y_st, bool st_ok) {
  const float d6 = div_by_recip(am, 6.0f, 0x1.555556p-3f);          // 0x1.555556p-3 = RN(1/6)
  const float t = div_by_recip(d6, s_t, y_st);
  const bool ok = st_ok && (am == 0.0f || (am >= 0x1p-100f && d6 >= 0x1p-100f && __fmul_rn(d6, y_st) < 0x1p64f));
  return ok ? t : __fdiv_rn(__fdiv_rn(am, 6.0f), s_t);
}

// Four-over-six candidate t4 = RN(RN(amax_b / 4) / s_t) (RN(amax_b / 4) = amax_b * 0.25, rounded).
__device__ __forceinline__ float nv_scale_arg4(float am, float s_t, float y_st, bool st_ok) {
  const float d4 = __fmul_rn(am, 0.25f);
  const float t = div_by_recip(d4, s_t, y_st);
  const bool ok = st_ok && (am == 0.0f || (d4 >= 0x1p-100f && __fmul_rn(d4, y_st) < 0x1p64f));
  return ok ? t : __fdiv_rn(d4, s_t);
}

// Four-over-six candidate t4 = RN(RN(amax_b / 4) / s_t) through the fp64 reciprocal of s_t (exact
// when amax_b / 4 is normal; smaller non-zero maxima take the IEEE division).
__device__ __forceinline__ float nv_scale_arg4_64(float am, float s_t, double yd_st) {
  const float d4 = __fmul_rn(am, 0.25f);
  if (am != 0.0f && am < 0x1p-120f) return __fdiv_rn(d4, s_t);
  return div_by_recip64(d4, yd_st);
}

// Per-CTA table of the element divisor S = RN(e4m3(b) * s_t) and RN(1/S) for
// every E4M3 byte b (b = 0 is the zero scale; its entry is unused).  A scale
// whose reciprocal is out of the fast path's range gets y = 0, which makes
// every quotient fail the `ok` test and take the IEEE division.
__device__ __forceinline__ void nv_fill_scale_table(float2* tab, float s_t) {
  for (int b = threadIdx.x; b < 128; b += blockDim.x) {
    const float S = (b == 0 || b == 127) ? 1.0f : __fmul_rn(e4m3_value((uint32_t)b), s_t);
    tab[b] = make_float2(S, recip_usable(S) ? __frcp_rn(S) : 0.0f);
  }
}

// Per-CTA table of RN64(1 / S) for S = RN32(e4m3(b) * s_t) and every E4M3 byte b (b = 0 and the
// NaN byte 127 get 0: their blocks' codes are zeroed or never produced).
__device__ __forceinline__ void nv_fill_recip64_table(double* tabd, float s_t) {
  for (int b = threadIdx.x; b < 128; b += blockDim.x) {
    const float S = (b == 0 || b == 127) ? 0.0f : __fmul_rn(e4m3_value((uint32_t)b), s_t);
    tabd[b] = S > 0.0f ? __drcp_rn((double)S) : 0.0;
  }
}

// Quotients q = x / S of one NVFP4 block through the fp64 reciprocal yd = RN64(1/S)
// (div_by_recip64); q may alias x.
template <int E>
__device__ __forceinline__ void nv_divide_block64(const float (&x)[E], double yd, float (&q)[E]) {
#pragma unroll
  for (int i = 0; i < E; ++i) q[i] = div_by_recip64(x[i], yd);
}

// NVFP4 block-scale argument t = RN(RN(amax_b / 6) / s_t) through fp64 reciprocals (yd_st =
// RN64(1/s_t)): both quotients are exact when amax_b / 6 is a normal fp32 (amax_b >= 2^-120 here);
// a subnormal t has E4M3 byte 0 either way.  Smaller non-zero maxima take the IEEE divisions.
__device__ __forceinline__ float nv_scale_arg64(float am, float s_t, double yd_st) {
  if (am != 0.0f && am < 0x1p-120f) return __fdiv_rn(__fdiv_rn(am, 6.0f), s_t);
  const float d6 = div_by_recip64(am, 0x1.5555555555555p-3);      // RN64(1/6)
  return div_by_recip64(d6, yd_st);
}

// -------------------------------------------------------- E2M1 decoding -----
__device__ __forceinline__ float e2m1_value(uint32_t c) {
  const uint32_t e = (c >> 1) & 3u, m = c & 1u;
  float mag = (e == 0u) ? (m ? 0.5f : 0.0f) : __uint_as_float(((e + 126u) << 23) | (m << 22));
  return (c & 8u) ? -mag : mag;
}

// One pair of scaled values -> their RTN codes, `a` in bits 0-3, `b` in bits 4-7.
__device__ __forceinline__ uint32_t e2m1x2_rn(float a, float b) {
  uint32_t out;
  asm("{\n\t.reg .b8 q;\n\tcvt.rn.satfinite.e2m1x2.f32 q, %2, %1;\n\tcvt.u32.u8 %0, q;\n\t}"
      : "=r"(out)
      : "f"(a), "f"(b));
  return out;
}

// ------------------------------------------------------ NVFP4 blocks -----
// Whether a block may divide by its scale S with div_by_recip (exact IEEE quotients) instead of
// __fdiv_rn.  Both need y = RN(1/S) usable (S in [2^-125, 2^20], y != 0) and quotients below
// 2^64.  Stochastic rounding uses the exact quotient of every element, so it also needs every
// |x| >= 2^-103 (or 0), where the residuals are exact.  Round-to-nearest only needs the codes:
// with S >= 2^-100 an element below 2^-103 has |x/S| < 2^-3, and div_by_recip keeps such a
// quotient below 0.13 with the sign of x, so it rounds to a signed zero code exactly like the
// correctly rounded quotient, while every larger element is divided exactly; that saves the
// per-element test.  RND: 0 round-to-nearest, 1 stochastic rounding.
template <int RND, int E>
__device__ __forceinline__ bool nv_fast_division(const float (&x)[E], float am, float S, float y) {
  if (y == 0.0f || !(__fmul_rn(am, y) < 0x1p64f)) return false;
  if (RND == 0) return S >= 0x1p-100f;
  uint32_t kmin = 0xFFFFFFFFu;
#pragma unroll
  for (int i = 0; i < E; ++i) kmin = min(kmin, tiny_key(x[i]));
  return kmin >= kTinyKeyMin;
}

// Quotients q = x / S of one NVFP4 block under the divisor S = sy.x (sy.y = RN(1/S)): div_by_recip
// when the block passes nv_fast_division's test for this rounding, IEEE division otherwise.  q may
// alias x.
template <int RND, int E>
__device__ __forceinline__ void nv_divide_block(const float (&x)[E], float am, float2 sy, float (&q)[E]) {
  if (nv_fast_division<RND, E>(x, am, sy.x, sy.y)) {
#pragma unroll
    for (int i = 0; i < E; ++i) q[i] = div_by_recip(x[i], sy.x, sy.y);
  } else {                                       // rare: tiny operands or scales
#pragma unroll
    for (int i = 0; i < E; ++i) q[i] = __fdiv_rn(x[i], sy.x);
  }
}

// Quotients of one NVFP4 block on packed fp32 pairs: div_by_recip's reciprocal and two
// corrections, each pair instruction doing two elements (5 pair instructions for two quotients,
// against 3 conversions and fp64 multiplies per quotient through div_by_recip64, 2 of them
// conversions).  The residual is formed as S*q - x and its product with y subtracted, the same
// values as div_by_recip's -(S*q - x) added (the sign of a zero dividend survives).  Under
// nv_fast_division's test for the rounding RND (round-to-nearest: per block only; stochastic
// rounding: also every |x| >= 2^-103) the quotients are those of IEEE division (tiny dividends
// under round-to-nearest: the same codes); blocks that fail it take __fdiv_rn.  sy = (S, RN(1/S)).
template <int RND, int E>
__device__ __forceinline__ void nv_divide_block2(float (&x)[E], float am, float2 sy) {
  if (nv_fast_division<RND, E>(x, am, sy.x, sy.y)) {
    const float2 S2 = make_float2(sy.x, sy.x), y2 = make_float2(sy.y, sy.y), ny2 = make_float2(-sy.y, -sy.y);
#pragma unroll
    for (int i = 0; i < E / 2; ++i) {
      const float2 xv = make_float2(x[2 * i], x[2 * i + 1]);
      const float2 nx = make_float2(-xv.x, -xv.y);
      float2 q = __fmul2_rn(xv, y2);
      float2 t = __ffma2_rn(q, S2, nx);
      q = __ffma2_rn(t, ny2, q);
      t = __ffma2_rn(q, S2, nx);
      q = __ffma2_rn(t, ny2, q);
      x[2 * i] = q.x;
      x[2 * i + 1] = q.y;
    }
  } else {                                       // rare: tiny or huge scales
#pragma unroll
    for (int i = 0; i < E; ++i) x[i] = __fdiv_rn(x[i], sy.x);
  }
}

// Round-to-nearest dequantization of two quotients: fp32(fp32(G[c] * sbv) * s_t) for each, where
// c is the E2M1 code of the quotient and g holds the block scale sbv in both halves.  G[c] * sbv
// has at most 6 significant bits and lies in [2^-10, 2688], so the f16 product is exact.
__device__ __forceinline__ float2 nv_rtn_dequant2(float q0, float q1, __half2 g, float s_t) {
  uint32_t h;
  asm("{\n\t.reg .b8 c;\n\tcvt.rn.satfinite.e2m1x2.f32 c, %2, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, c;\n\t}"
      : "=r"(h)
      : "f"(q0), "f"(q1));
  const float2 v = __half22float2(__hmul2(*reinterpret_cast<const __half2*>(&h), g));
  return __fmul2_rn(v, make_float2(s_t, s_t));
}

// -------------------------------------------------- scale-factor offsets ----
// Byte offset of the scale of (row, k-group g) in the tensor-core layout:
// 128x4 tiles, k-tile index fastest, (r%32)*16 + (r/32)*4 + g inside a tile.
__device__ __forceinline__ long long sf_mma_offset(long long row, long long g, long long g4) {
  return (((row >> 7) * g4 + (g >> 2)) << 9) + ((row & 31) << 4) + (((row >> 5) & 3) << 2) + (g & 3);
}

// ------------------------------------------------------ Hadamard (fp32) -----
// The butterflies run on packed fp32 pairs (the f32x2 add / multiply-add /
// multiply of sm_100): each half of a pair operation is the IEEE fp32 operation
// of that half alone, so a pair gives the values of the two scalar operations
// it replaces in one instruction.  A thread's E values sit in E/2 pairs
// (x[p], x[p + E/2]); a stage at a distance below E/2 combines two pairs, the
// stage at distance E/2 the two halves of each pair.
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 splat2(float v) { return make_float2(v, v); }

template <int HB>
__device__ __forceinline__ float hadamard_norm() {
  return HB == 16 ? 0.25f : HB == 32 ? 0.17677669529663687f : HB == 64 ? 0.125f : 0.08838834764831845f;
}

// One butterfly stage at distance d inside a thread's pairs P[E/2] (element e is
// P[e % H].x for e < H, P[e - H].y otherwise, H = E/2): (a, b) -> (a + b, a - b),
// or with a sign sg (chunk order, see hadamard_rotate_block) -> (a*sg + b, b*(-sg) + a).
template <int E, bool SIGNED>
__device__ __forceinline__ void butterfly_stage(float2 (&P)[E / 2], int d, float sg) {
  constexpr int H = E / 2;
  if (d < H) {
    const float2 s2 = splat2(SIGNED ? sg : 1.0f), m2 = splat2(SIGNED ? -sg : -1.0f);
#pragma unroll
    for (int p = 0; p < H; ++p) {
      if ((p & d) == 0) {
        const float2 a = P[p], b = P[p + d];
        P[p] = SIGNED ? fma2(a, s2, b) : add2(a, b);
        P[p + d] = fma2(b, m2, a);                   // a - b: one rounding, as the subtraction
      }
    }
  } else {
#pragma unroll
    for (int p = 0; p < H; ++p) {
      const float a = P[p].x, b = P[p].y;
      P[p].x = SIGNED ? __fmaf_rn(a, sg, b) : __fadd_rn(a, b);
      P[p].y = SIGNED ? __fmaf_rn(b, -sg, a) : __fsub_rn(a, b);
    }
  }
}

// A stage across lanes at lane distance ld: every element takes x * sgn + p,
// p the partner lane's element at register position e ^ flip (upper lanes
// p - x, lower ones x + p: a multiply-add by -1 or +1, exact negation, a single
// rounding, so the same value as the subtraction or addition).
template <int E>
__device__ __forceinline__ void butterfly_lanes(float2 (&P)[E / 2], int lane, int ld, int flip) {
  constexpr int H = E / 2;
  const float2 s2 = splat2((lane & ld) != 0 ? -1.0f : 1.0f);
  float2 Q[H];
#pragma unroll
  for (int p = 0; p < H; ++p) {
    const int e0 = p ^ flip, e1 = (p + H) ^ flip;
    const float v0 = e0 < H ? P[e0].x : P[e0 - H].y;
    const float v1 = e1 < H ? P[e1].x : P[e1 - H].y;
    Q[p] = make_float2(__shfl_xor_sync(0xFFFFFFFFu, v0, ld), __shfl_xor_sync(0xFFFFFFFFu, v1, ld));
  }
#pragma unroll
  for (int p = 0; p < H; ++p) P[p] = fma2(P[p], s2, Q[p]);
}

// In-register fast Walsh-Hadamard transform of a contiguous block of HB
// elements held 8 per lane by HB/8 consecutive lanes (Sylvester order:
// pairs (i, i + 2^s) -> (a + b, a - b), distances 1, 2, 4, ... in turn), then
// scaled by 1/sqrt(HB).
template <int HB>
__device__ __forceinline__ void hadamard_rotate(float (&x)[8], int lane) {
  float2 P[4];
#pragma unroll
  for (int p = 0; p < 4; ++p) P[p] = make_float2(x[p], x[p + 4]);
#pragma unroll
  for (int d = 1; d < 8; d <<= 1) butterfly_stage<8, false>(P, d, 1.0f);
#pragma unroll
  for (int ld = 1; ld < HB / 8; ld <<= 1) butterfly_lanes<8>(P, lane, ld, 0);
  const float2 s2 = splat2(hadamard_norm<HB>());
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    P[p] = mul2(P[p], s2);
    x[p] = P[p].x;
    x[p + 4] = P[p].y;
  }
}

// Same transform with one thread holding E consecutive elements (E = 16 or
// 32, a whole scale block): butterflies inside the thread for distances < E,
// then across HB/E consecutive lanes.  The stages run in the same order
// (distance 1, 2, 4, ...) with the same operand order as hadamard_rotate, so
// both layouts give bit-identical fp32 results.
//
// The block's 8-element chunks may sit in XOR order: register chunk k holding
// chunk k ^ sw, with sw = (lane >> SWS) & SWM (the order in which the streaming
// kernels read shared memory without bank conflicts; SWM = 0: plain order).
// A stage at distance 8 or 16 then pairs the same two registers, but when the
// matching bit of sw is set the lower element sits in the upper register, so
// each register takes x[i] * s + x[j] with the sign s of that bit (an exact
// sum or difference, one rounding: the values of the plain order).  A cross-lane
// stage whose partner lane has the other sw (a lane bit inside the sw field)
// exchanges the register of the flipped chunk, chosen at compile time.
template <int HB, int E, int SWS = 0, int SWM = 0>
__device__ __forceinline__ void hadamard_rotate_block(float (&x)[E], int lane, uint32_t sw = 0u) {
  constexpr int IN = HB < E ? HB : E, H = E / 2;
  float2 P[H];
#pragma unroll
  for (int p = 0; p < H; ++p) P[p] = make_float2(x[p], x[p + H]);
#pragma unroll
  for (int d = 1; d < IN; d <<= 1) {
    if (d < 8 || SWM == 0) {
      butterfly_stage<E, false>(P, d, 1.0f);
    } else {
      butterfly_stage<E, true>(P, d, ((sw >> (d == 8 ? 0 : 1)) & 1u) != 0u ? -1.0f : 1.0f);
    }
  }
#pragma unroll
  for (int ld = 1; ld < HB / E; ld <<= 1) butterfly_lanes<E>(P, lane, ld, ((ld >> SWS) & SWM) << 3);
  const float2 s2 = splat2(hadamard_norm<HB>());
#pragma unroll
  for (int p = 0; p < H; ++p) {
    P[p] = mul2(P[p], s2);
    x[p] = P[p].x;
    x[p + H] = P[p].y;
  }
}

// ------------------------------------------- bulk copies and mbarriers -----
// Thin wrappers over the sm_90+/sm_100 bulk-copy engine (cp.async.bulk, no
// tensor map, no multicast) and shared-memory mbarriers, used by the
// streaming kernels to move whole tiles with one instruction.
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_init_fence() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity, uint32_t sleep_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(sleep_ns)
      : "memory");
  return ok != 0u;
}
__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Wait for phase `parity` of an mbarrier, giving up after ~2 s.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity) {
  if (mbar_test(bar, parity, 0u)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    if (mbar_test(bar, parity, 10000u)) return true;
    if (globaltimer_ns() - t0 > 2000000000ull) return false;
  }
}
// global -> shared, completion counted on an mbarrier (addresses 16-byte aligned, size % 16 == 0).
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}
// shared -> global in a bulk group of the issuing thread.
__device__ __forceinline__ void bulk_s2g(void* dst, uint32_t src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src), "r"(bytes)
               : "memory");
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Wait until at most N of this thread's bulk groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// Order this thread's generic-proxy shared-memory writes before later bulk copies.
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

}  // namespace fp4dev
