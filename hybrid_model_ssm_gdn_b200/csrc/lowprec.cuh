// lowprec.cuh -- device-side number formats of the separate-precision mode.
//
// The recurrence checkpoint and the copy read for outputs may use different
// precisions so that the read copy's rounding never re-enters the recurrence
// ("Hybrid-model decoding has a new bottleneck", Interpretation, fourth paragraph);
// the pages name an FP16 recurrence with stochastic rounding (same page, Perspective,
// second paragraph) and NVFP4 reads (E2M1 values, an E4M3 scale per 16-element
// block).  Rounding rules, all exact integer or IEEE-fp32 procedures:
//
// * FP16 stochastic rounding of fp32 x with a 32-bit word r: with u the fp16 spacing
//   at |x| (2^(floor(log2|x|)-10), or 2^-24 below 2^-14) and |x| = (q + f) u, round
//   up to (q+1) u iff r < floor(f * 2^32); keep the sign; saturate at 65504.
// * E4M3 (OCP FP8 E4M3FN) and E2M1 (OCP FP4): round to nearest, ties to even,
//   saturating at 448 and 6.
// * FP8 checkpoint tile (64 rows x 128 columns): s = amax(tile)/448 (1 if amax = 0);
//   y = x / s rounded stochastically to the E4M3 grid with the FP16 rule and E4M3
//   spacings (2^(floor(log2|y|)-3), 2^-9 below 2^-6), saturating at 448; value = E4M3 * s.
// * NVFP4 tile (64 consecutive rows x 128 columns of one head's state), blocks of 16
//   columns: g = amax(tile)/2688 (1 if amax = 0); s_b = E4M3(amax_b / (6 g));
//   d_b = s_b g; code = sign | E2M1(|x| / d_b) (all zero if s_b = 0); value = E2M1 * d_b.
// * Two-axis NVFP4 tile (separate scales along the channel and state axes): g as above;
//   per column and group of 16 rows c = E4M3(amax_group / (6 g)), step k = c g;
//   x' = x / k (0 where k = 0); per row block s_b = E4M3(amax_b(x') / (6 * 2^-8)),
//   d_b = s_b * 2^-8; code = sign(x') | E2M1(|x'| / d_b); value = (E2M1 * d_b) * k.
// * Random words: Philox4x32-10 (Salmon, Moraes, Dror & Shaw, SC'11), counter
//   (sequence*H + head, epoch written, element/4, 0), key = the 64-bit seed; element e
//   uses output word e % 4.
#pragma once

#include <cuda_fp16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>
#include <stdint.h>

namespace rssm {

constexpr int kFp4Rows = 64;  // rows of one NVFP4 tile (one row block of a head's state)

__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    const uint32_t lo0 = 0xD2511F53u * c.x, hi0 = __umulhi(0xD2511F53u, c.x);
    const uint32_t lo1 = 0xCD9E8D57u * c.z, hi1 = __umulhi(0xCD9E8D57u, c.z);
    c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
  }
  return c;
}

// Stochastic rounding of fp32 x to fp16 with the uniform word r (see the rule above).
__device__ __forceinline__ __half fp16_sr(float x, uint32_t r) {
  const uint32_t bits = __float_as_uint(x);
  const uint32_t sign = bits >> 31;
  const int E = (int)((bits >> 23) & 0xFFu);
  if ((uint32_t)(E - 113) <= 29u) {
    // |x| in [2^-14, 2^16): the fp16 spacing leaves 13 fp32 mantissa bits F below it, and the rule rounds up
    // iff (r >> 19) < F.  Adding 2^13 - 1 - (r >> 19) = (~r) >> 19 to the magnitude's bits carries into bit 13
    // exactly then (a carry out of the mantissa moves to the next binade); truncating the 13 bits finishes it.
    const uint32_t m = ((bits & 0x7FFFFFFFu) + ((~r) >> 19)) & ~0x1FFFu;
    const float mag = fminf(__uint_as_float(m), 65504.f);
    return __float2half_rn(sign ? -mag : mag);                 // exact: the value lies on the fp16 grid
  }
  const uint32_t mant = bits & 0x7FFFFFu;
  if (E == 255) return mant ? __ushort_as_half(0x7E00) : __ushort_as_half(sign ? 0xFBFF : 0x7BFF);
  const uint32_t M = E ? (mant | 0x800000u) : mant;  // |x| = M * 2^(Eeff - 150)
  const int Eeff = E ? E : 1;
  const int s = max(13, 126 - Eeff);                  // fp32 bits below the fp16 spacing
  uint32_t q, F;
  if (s >= 24) { q = 0; F = M; } else { q = M >> s; F = M & ((1u << s) - 1u); }
  uint64_t thr;
  if (s <= 32) thr = (uint64_t)F << (32 - s);
  else if (s - 32 < 24) thr = (uint64_t)(F >> (s - 32));
  else thr = 0;
  const uint32_t up = ((uint64_t)r < thr) ? 1u : 0u;
  const int ulp_exp = max(Eeff - 127, -14) - 10;
  // exact: an integer <= 2^11 times 2^ulp_exp (ulp_exp >= -24, a normal fp32 power of two)
  float mag = (float)(q + up) * __int_as_float((ulp_exp + 127) << 23);
  mag = fminf(mag, 65504.f);
  return __float2half_rn(sign ? -mag : mag);          // exact: the value lies on the fp16 grid
}

// Stochastic rounding of fp32 y to E4M3 with the uniform word r; returns the E4M3 bit pattern
// (sign bit set only for a non-zero negative result).
__device__ __forceinline__ uint32_t fp8_sr_code(float y, uint32_t r) {
  const uint32_t bits = __float_as_uint(y);
  const uint32_t sign = bits >> 31;
  const int E = (int)((bits >> 23) & 0xFFu);
  if ((uint32_t)(E - 121) <= 14u) {
    // |y| in [2^-6, 2^9): 20 fp32 mantissa bits F lie below the E4M3 spacing; round up iff (r >> 12) < F, by
    // the same carry as the fp16 rule, then take exponent and 3 mantissa bits, saturating at 448 (0x7E)
    const uint32_t m = ((bits & 0x7FFFFFFFu) + ((~r) >> 12)) & ~0xFFFFFu;
    const uint32_t code = m > 0x43E00000u ? 0x7Eu : ((((m >> 23) - 120u) << 3) | ((m >> 20) & 7u));
    return code | (sign << 7);
  }
  const uint32_t mant = bits & 0x7FFFFFu;
  const uint32_t M = E ? (mant | 0x800000u) : mant;  // |y| = M * 2^(Eeff - 150)
  const int Eeff = E ? E : 1;
  const int s = max(20, 141 - Eeff);                  // fp32 bits below the E4M3 spacing
  uint32_t q, F;
  if (s >= 24) { q = 0; F = M; } else { q = M >> s; F = M & ((1u << s) - 1u); }
  uint64_t thr;
  if (s <= 32) thr = (uint64_t)F << (32 - s);
  else if (s - 32 < 24) thr = (uint64_t)(F >> (s - 32));
  else thr = 0;
  const uint32_t up = ((uint64_t)r < thr) ? 1u : 0u;
  const int ulp_exp = max(Eeff - 127, -6) - 3;
  const uint32_t n = q + up;                          // magnitude = n * 2^ulp_exp
  if (n == 0u) return 0u;
  uint32_t code;
  if (ulp_exp == -9 && n < 8u) {
    code = n;                                         // subnormal: mantissa n, exponent field 0
  } else {
    // normalise n * 2^ulp_exp (n <= 16) to (8 + m) * 2^(ef - 10)
    int ef = ulp_exp + 10;
    uint32_t mm = n;
    if (mm >= 16u) { mm >>= 1; ++ef; }                 // n = 16: carried into the next binade
    code = ((uint32_t)ef << 3) | (mm - 8u);
    if (code > 0x7Eu) code = 0x7Eu;                   // saturate at 448
  }
  return code | (sign << 7);
}

__device__ __forceinline__ float e4m3_signed_value(uint32_t code) {
  const uint32_t ef = (code >> 3) & 0xFu, m = code & 7u;
  const float mag = ef == 0 ? ldexpf((float)m, -9) : ldexpf((float)(8u + m), (int)ef - 10);
  return (code & 0x80u) ? -mag : mag;
}

// FP8 checkpoint tile scale from the tile's largest magnitude.
__device__ __forceinline__ float fp8_tile_scale(float amax) { return amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f; }


// Decoders for the kernels' tile reads, through the hardware pair conversions to f16x2 (every
// E4M3 and E2M1 value is exactly an f16 value).  The first element sits in the low byte / low
// nibble, as the tiles store it.
__device__ __forceinline__ float4 e4m3x4_to_float4(uint32_t w) {  // four codes, byte i = element i
  const __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w & 0xFFFFu), __NV_E4M3);
  const __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w >> 16), __NV_E4M3);
  const float2 a = __half22float2(__half2(lo)), b = __half22float2(__half2(hi));
  return make_float4(a.x, a.y, b.x, b.y);
}

__device__ __forceinline__ float e4m3_to_float(uint32_t code) {  // one unsigned code
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(code & 0xFFu), __NV_E4M3);
  return __low2float(__half2(h));
}

__device__ __forceinline__ float4 e2m1x4_to_float4(uint32_t w) {  // four codes, nibble i = element i
  const __half2_raw lo = __nv_cvt_fp4x2_to_halfraw2((__nv_fp4x2_storage_t)(w & 0xFFu), __NV_E2M1);
  const __half2_raw hi = __nv_cvt_fp4x2_to_halfraw2((__nv_fp4x2_storage_t)((w >> 8) & 0xFFu), __NV_E2M1);
  const float2 a = __half22float2(__half2(lo)), b = __half22float2(__half2(hi));
  return make_float4(a.x, a.y, b.x, b.y);
}

__device__ __forceinline__ float e4m3_value(uint32_t code) {
  const uint32_t ef = (code >> 3) & 0xFu, m = code & 7u;
  return ef == 0 ? ldexpf((float)m, -9) : ldexpf((float)(8u + m), (int)ef - 10);
}

// E2M1 magnitude index (0..7 for {0, .5, 1, 1.5, 2, 3, 4, 6}) of y >= 0, ties to even index.
__device__ __forceinline__ uint32_t e2m1_index(float y) {
  uint32_t n;
  if (y < 2.f) n = (uint32_t)rintf(y * 2.f);
  else if (y < 4.f) n = (uint32_t)rintf(y) + 2u;
  else n = (uint32_t)rintf(y * 0.5f) + 4u;
  return n > 7u ? 7u : n;
}

__device__ __forceinline__ float e2m1_value(uint32_t idx) {
  // {0, .5, 1, 1.5, 2, 3, 4, 6}
  const float lo = (float)idx * 0.5f;           // exact for idx <= 4
  return idx <= 4u ? lo : (idx == 5u ? 3.f : (idx == 6u ? 4.f : 6.f));
}

// NVFP4 tile scale from the tile's largest magnitude.
__device__ __forceinline__ float nvfp4_tile_scale(float amax) { return amax > 0.f ? __fdiv_rn(amax, 2688.f) : 1.f; }

// E4M3FN code of v >= 0, rounded to nearest even and saturating at 448 (the hardware conversion; subnormal
// spacing 2^-9).
__device__ __forceinline__ uint32_t e4m3_rn_code(float v) {
  return (uint32_t)__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3);
}

// Block scale code and the block's dequantisation step d_b = s_b * g.
__device__ __forceinline__ uint32_t nvfp4_block_scale(float amax_b, float g, float *d_b) {
  const float t = __fmul_rn(6.f, g);
  const uint32_t code = e4m3_rn_code(__fdiv_rn(amax_b, t));
  *d_b = __fmul_rn(e4m3_to_float(code), g);
  return code;
}

// 4-bit code of x in a block with step d_b (d_b == 0 when the block scale is zero).
__device__ __forceinline__ uint32_t nvfp4_code(float x, float d_b) {
  if (d_b == 0.f) return 0u;
  const uint32_t idx = e2m1_index(__fdiv_rn(fabsf(x), d_b));
  return idx | (x < 0.f ? 8u : 0u);
}

// The division for the four codes, out of line: kernels call it only for the rare element near a decision
// threshold, and keep their unrolled code loops compact.
static __device__ __noinline__ uint32_t nvfp4_code4_div(float4 x, float d_b) {
  return nvfp4_code(x.x, d_b) | (nvfp4_code(x.y, d_b) << 4) | (nvfp4_code(x.z, d_b) << 8) | (nvfp4_code(x.w, d_b) << 12);
}

// Four codes of one block (nibble i = element i), the same as nvfp4_code elementwise, without a division per
// element.  With r = 1/d_b correctly rounded, q' = |x| r lies within 2^-22 (relative) of the correctly rounded
// quotient q that nvfp4_code rounds, so q'(1 - 2^-19) < q < q'(1 + 2^-19) after rounding; the E2M1 conversion
// (round to nearest even, saturating at 6: the index rule of e2m1_index) is monotone, so where both ends of the
// bracket give the same code, q gives it too.  Elements whose bracket straddles a decision threshold, and blocks
// whose step is too small for a finite reciprocal, take the division.
__device__ __forceinline__ uint32_t nvfp4_code4(float4 x, float d_b, float r) {
  if (d_b == 0.f) return 0u;
  const uint32_t sgn = (x.x < 0.f ? 0x8u : 0u) | (x.y < 0.f ? 0x80u : 0u) | (x.z < 0.f ? 0x800u : 0u) |
                       (x.w < 0.f ? 0x8000u : 0u);
  if (d_b >= 0x1p-120f) {
    const float qx = __fmul_rn(fabsf(x.x), r), qy = __fmul_rn(fabsf(x.y), r);
    const float qz = __fmul_rn(fabsf(x.z), r), qw = __fmul_rn(fabsf(x.w), r);
    constexpr float kLo = 1.f - 0x1p-19f, kHi = 1.f + 0x1p-19f;
    const uint32_t lo = (uint32_t)__nv_cvt_float2_to_fp4x2(make_float2(qx * kLo, qy * kLo), __NV_E2M1, cudaRoundNearest) |
                        ((uint32_t)__nv_cvt_float2_to_fp4x2(make_float2(qz * kLo, qw * kLo), __NV_E2M1, cudaRoundNearest) << 8);
    const uint32_t hi = (uint32_t)__nv_cvt_float2_to_fp4x2(make_float2(qx * kHi, qy * kHi), __NV_E2M1, cudaRoundNearest) |
                        ((uint32_t)__nv_cvt_float2_to_fp4x2(make_float2(qz * kHi, qw * kHi), __NV_E2M1, cudaRoundNearest) << 8);
    if (lo == hi) return lo | sgn;
  }
  return nvfp4_code4_div(x, d_b);
}

// Two-axis copy: column-group scale code and step k = c * g from the group's largest magnitude.
__device__ __forceinline__ uint32_t nvfp4d_col_scale(float amax_grp, float g, float *k) {
  const uint32_t code = e4m3_rn_code(__fdiv_rn(amax_grp, __fmul_rn(6.f, g)));
  *k = __fmul_rn(e4m3_to_float(code), g);
  return code;
}

// Two-axis copy: row-block scale code and block step d_b = s_b * 2^-8 (exact) of the divided values.
__device__ __forceinline__ uint32_t nvfp4d_block_scale(float amax_b, float *d_b) {
  const uint32_t code = e4m3_rn_code(__fdiv_rn(amax_b, 0.0234375f));   // 6 * 2^-8
  *d_b = e4m3_to_float(code) * 0.00390625f;
  return code;
}

__device__ __forceinline__ float nvfp4_value(uint32_t code, float d_b) {
  const float v = __fmul_rn(e2m1_value(code & 7u), d_b);
  return (code & 8u) ? -v : v;
}

}  // namespace rssm
