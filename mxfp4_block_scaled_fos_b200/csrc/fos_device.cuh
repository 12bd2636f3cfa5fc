// fos_device.cuh -- device-side building blocks of the sm_100a quantizers.
//
// Element and scale codecs use the Blackwell conversion instructions
// (cvt.rn.satfinite.e2m1x2.f32, cvt.rn.satfinite.e4m3x2.f32 and the
// e2m1x2 -> f16x2 decode); binary32 arithmetic that the quantizer's
// definition fixes uses explicitly rounded intrinsics (no contraction), and
// element pairs are processed with the packed f32x2 FMA/MUL/ADD of sm_100.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

namespace fos {

constexpr float kE4M3Max = 448.0f;
constexpr float kFltMax = 3.402823466e38f;

// ---------------------------------------------------------------- bf16
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// ---------------------------------------------------------------- f32x2
// Packed binary32 pairs (sm_100 FMUL2/FADD2/FFMA2), each component rounded
// like its scalar _rn counterpart.  Measured on sm_100a with CUDA 12.9: a
// packed product that feeds a packed add may still be contracted into one
// fused instruction (also when written as mul.rn/add.rn PTX, and when the
// product is an fma with a literal -0 addend), which drops a rounding.  No
// code here lets a product feed an add; where the definition needs RN(a*b)
// followed by an add, the product is fma(a, b, z) with z = -0 passed at run
// time.
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
// a - b with one rounding: b * (-1) is exact, the sum rounds once.
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
  return __ffma2_rn(b, make_float2(-1.0f, -1.0f), a);
}

// RN(r / 6) without a division, for finite r >= 0: q0 = RN(r*y),
// y = RN(1/6); the remainder r - 6*q0 is exact as an fma and one correction
// step q0 + rem*y gives the correctly rounded quotient (P. Markstein, IBM J.
// Res. Dev. 34(1), 1990).  Equal to IEEE division for every finite r >=
// 2^-125 (tests/test_gpu_exhaustive.py runs all of them on the device).
// Below that both results are < 2^-127, far under the smallest E4M3
// subnormal (2^-9), so the E4M3 code of the quotient -- the only use here --
// is 0 either way and no fallback branch is needed.  r = inf would give NaN:
// the callers clamp r to FLT_MAX first.
__device__ __forceinline__ float div6_for_e4m3(float r) {
  const float y = 1.0f / 6.0f;
  const float q0 = __fmul_rn(r, y);
  const float rem = __fmaf_rn(-q0, 6.0f, r);
  return __fmaf_rn(rem, y, q0);
}

// L2 eviction-priority policies for the loads below (createpolicy).
__device__ __forceinline__ unsigned long long l2_policy_evict_last() {
  unsigned long long pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ unsigned long long l2_policy_evict_first() {
  unsigned long long pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// Asynchronous prefetch of [p, p + bytes) into L2 with an eviction policy
// (p and bytes multiples of 16).  No completion tracking: later loads of the
// range hit L2 or merge with the requests in flight.
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes, unsigned long long pol) {
  asm volatile("cp.async.bulk.prefetch.L2.global.L2::cache_hint [%0], %1, %2;"
               :: "l"(p), "r"(bytes), "l"(pol) : "memory");
}

// 32 bytes (one 16-element bf16 block) in one 256-bit load with an L2
// eviction policy; p must be 32-byte aligned.
__device__ __forceinline__ void ld_block256_hint(const void* p, unsigned long long pol, uint4 (&w)[2]) {
  asm("ld.global.nc.L2::cache_hint.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8], %9;"
      : "=r"(w[0].x), "=r"(w[0].y), "=r"(w[0].z), "=r"(w[0].w), "=r"(w[1].x), "=r"(w[1].y),
        "=r"(w[1].z), "=r"(w[1].w)
      : "l"(p), "l"(pol));
}

// 32 bytes (one 16-element bf16 block) in one 256-bit load; p must be
// 32-byte aligned.
__device__ __forceinline__ void ld_block256(const void* p, uint4 (&w)[2]) {
  asm("ld.global.nc.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
      : "=r"(w[0].x), "=r"(w[0].y), "=r"(w[0].z), "=r"(w[0].w), "=r"(w[1].x), "=r"(w[1].y),
        "=r"(w[1].z), "=r"(w[1].w)
      : "l"(p));
}

// ---------------------------------------------------------------- E2M1
// Eight binary32 values -> eight E2M1 nibbles (RNE, saturating at +-6);
// element 2k goes to the low nibble of byte k.
__device__ __forceinline__ uint32_t e2m1x8(float e0, float e1, float e2, float e3, float e4,
                                           float e5, float e6, float e7) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(e0), "f"(e1), "f"(e2), "f"(e3), "f"(e4), "f"(e5), "f"(e6), "f"(e7));
  return out;
}

// Two E2M1 nibbles -> f16x2 (low nibble in the low half), exact.  `byte`
// must be zero-extended (bits 8..31 clear): the conversion was measured to
// give wrong results when the upper bits of its operand register are not
// zero (bytes taken from a split 32-bit or 16-bit register).
__device__ __forceinline__ uint32_t e2m1x2_to_h2(uint32_t byte) {
  uint32_t out;
  const unsigned short t = (unsigned short)byte;
  asm("{\n\t.reg .b8 lo, hi;\n\t"
      "mov.b16 {lo, hi}, %1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, lo;\n\t}"
      : "=r"(out)
      : "h"(t));
  return out;
}

// Eight E2M1 nibbles -> four f16x2 words (h[k] holds elements 2k, 2k+1);
// each byte is extracted zero-extended with one byte permute.
__device__ __forceinline__ void e2m1x8_to_h2(uint32_t codes, uint32_t h[4]) {
  h[0] = e2m1x2_to_h2(__byte_perm(codes, 0u, 0x4440u));
  h[1] = e2m1x2_to_h2(__byte_perm(codes, 0u, 0x4441u));
  h[2] = e2m1x2_to_h2(__byte_perm(codes, 0u, 0x4442u));
  h[3] = e2m1x2_to_h2(__byte_perm(codes, 0u, 0x4443u));
}

__device__ __forceinline__ __half2 as_h2(uint32_t h) {
  __half2 r;
  memcpy(&r, &h, 4);
  return r;
}
// exact f16 -> f32 of the low / high half (no masking or shifting)
__device__ __forceinline__ float h_lo(uint32_t h) { return __low2float(as_h2(h)); }
__device__ __forceinline__ float h_hi(uint32_t h) { return __high2float(as_h2(h)); }

// ---------------------------------------------------------------- E4M3
// Two binary32 values -> (E4M3(hi) << 8) | E4M3(lo), RNE, saturating at 448.
__device__ __forceinline__ uint32_t e4m3x2(float hi, float lo) {
  unsigned short out;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(out) : "f"(hi), "f"(lo));
  return out;
}

// E4M3 code (0..255) -> binary32, exact (via the f16x2 decode).
__device__ __forceinline__ float e4m3_to_f32(uint32_t code) {
  uint32_t h;
  unsigned short c = (unsigned short)(code & 0xffu);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(c));
  return h_lo(h);
}

// ---------------------------------------------------------------- Philox
// Philox4x32-10 as published by Salmon et al. (SC'11).
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint2 k) {
#pragma unroll
  for (int i = 0; i < 10; ++i) {
    if (i) {
      k.x += 0x9E3779B9u;
      k.y += 0xBB67AE85u;
    }
    const uint32_t lo0 = 0xD2511F53u * c.x, hi0 = __umulhi(0xD2511F53u, c.x);
    const uint32_t lo1 = 0xCD9E8D57u * c.z, hi1 = __umulhi(0xCD9E8D57u, c.z);
    c = make_uint4(hi1 ^ c.y ^ k.x, lo1, hi0 ^ c.w ^ k.y, lo0);
  }
  return c;
}

__device__ __forceinline__ uint2 seed_key(unsigned long long seed) {
  return make_uint2((uint32_t)(seed & 0xffffffffull), (uint32_t)(seed >> 32));
}

// Philox output for the 16 consecutive source elements starting at g0
// (g0 % 16 == 0): byte j belongs to element g0 + j.
__device__ __forceinline__ uint4 sr_bytes16(unsigned long long seed, long long g0) {
  const unsigned long long u = (unsigned long long)g0;
  return philox4x32_10(make_uint4((uint32_t)((u >> 4) & 0xffffffffull), (uint32_t)(u >> 36), 0u, 0u),
                       seed_key(seed));
}

// 16-bit mask of the random Hadamard signs: bit i set -> element i negated.
__device__ __forceinline__ uint32_t rht_sign_mask(unsigned long long seed) {
  return philox4x32_10(make_uint4(0u, 0u, 1u, 0u), seed_key(seed)).x & 0xffffu;
}

// ---------------------------------------------------------------- SR
// Stochastic rounding of v >= 0 on the E2M1 magnitude grid: with lo <= v < hi
// the neighbouring grid values, round up iff 2*byte+1 < 512*(v-lo)/(hi-lo).
// Every step below is exact in binary32.
__device__ __forceinline__ float sr_e2m1_mag(float v, uint32_t byte) {
  if (v >= 6.0f) return 6.0f;
  const float step = v < 2.0f ? 0.5f : (v < 4.0f ? 1.0f : 2.0f);
  const float inv_step = v < 2.0f ? 2.0f : (v < 4.0f ? 1.0f : 0.5f);
  const float t = __fmul_rn(v, inv_step);
  const float fl = floorf(t);
  const float p = __fsub_rn(t, fl);
  const float lo = __fmul_rn(fl, step);
  const float thr = (float)(2u * byte + 1u);
  return (thr < __fmul_rn(512.0f, p)) ? __fadd_rn(lo, step) : lo;
}

// The same rule in integer form on the bits of v, cheaper where the bytes
// arrive one per register (the dual-orientation quantizer).  For v >= 1 the
// grid holds two points per binade (mantissa 1.0 and 1.5), so lo keeps v's
// bits down to mantissa bit 22, hi = lo + 2^22 (as bits), and 512*p =
// (bits & 0x3fffff) / 2^13: round up iff (2*byte+1) << 13 < (bits &
// 0x3fffff).  For 0.5 <= v < 1 the binade holds one point (0.5) and the next
// is 1.0: the same with 23 mantissa bits.  For v < 0.5: lo = 0, hi = 0.5,
// 512*p = 1024*v (exact).  Returns the chosen grid value, or a value >= 6
// that the saturating E2M1 encode turns into 6.  Equal to sr_e2m1_mag after
// that encode for every binary32 v in [0, 16] and infinity with every byte
// (tests/test_gpu_exhaustive.py runs all of them on the device).
__device__ __forceinline__ float sr_e2m1_mag_bits(float v, uint32_t byte) {
  const uint32_t bits = __float_as_uint(v);
  const uint32_t t13 = (byte << 14) | 0x2000u;   // (2*byte + 1) << 13
  const bool ge1 = bits >= 0x3F800000u;
  const uint32_t fmask = ge1 ? 0x3FFFFFu : 0x7FFFFFu;
  const uint32_t thr = ge1 ? t13 : (t13 << 1);
  const uint32_t qn = (bits & ~fmask) + (((bits & fmask) > thr) ? fmask + 1u : 0u);
  const float tf = __fsub_rn(__uint_as_float(0x4B000000u | (2u * byte + 1u)), 8388608.0f);
  const uint32_t qs = (__fmul_rn(v, 1024.0f) > tf) ? 0x3F000000u : 0u;
  return __uint_as_float(bits >= 0x3F000000u ? qn : qs);
}

// The same rule for a pair of magnitudes, as a ceiling.  With step the grid
// spacing at v (0.5 below 2, then 2^(e-1) for v in [2^e, 2^(e+1))), u = v /
// step (exact: a power of two) and r = (2*byte+1)/512, the result is step *
// ceil(u - r): ceil(u - r) = floor(u) + 1 exactly when frac(u) > r.  u - r
// is exact (both are multiples of the smaller of ulp(u) and 2^-9, and where
// the difference would need more than 24 bits it is negative, and any
// rounding keeps it in (-1, 0)), so one fma forms it from v.  Values >= 6
// come out as 6 or more and are clamped; +inf gives NaN at the fma, which
// the clamp (fminf) turns into 6; a -0 ceiling becomes +0 through the +0
// addend of the last fma.  R0, R1 carry the thresholds as the binary32 bits
// of 2^14 + (2*byte+1)/512 (sr_thr_bits): subtracting from 2^14 is exact.
__device__ __forceinline__ uint32_t sr_thr_bits(uint32_t byte) { return (byte << 1) | 0x46800001u; }

// byte j (0..3) of w as sr_thr_bits
__device__ __forceinline__ uint32_t sr_thr_bits_of(uint32_t w, int j) {
  return ((j ? (w >> (8 * j - 1)) : (w << 1)) & 0x1feu) | 0x46800001u;
}

__device__ __forceinline__ float2 sr_e2m1_mag2(float2 v, uint32_t R0, uint32_t R1) {
  const float2 rneg = sub2(make_float2(16384.0f, 16384.0f), make_float2(__uint_as_float(R0), __uint_as_float(R1)));
  const int s0 = max((int)(__float_as_uint(v.x) & 0x7f800000u) - 0x00800000, 0x3f000000);
  const int s1 = max((int)(__float_as_uint(v.y) & 0x7f800000u) - 0x00800000, 0x3f000000);
  const float2 inv_step = make_float2(__uint_as_float(0x7f000000u - (uint32_t)s0),
                                      __uint_as_float(0x7f000000u - (uint32_t)s1));
  const float2 t = fma2(v, inv_step, rneg);
  const float2 c = make_float2(ceilf(t.x), ceilf(t.y));
  const float2 q = fma2(c, make_float2(__int_as_float(s0), __int_as_float(s1)), make_float2(0.0f, 0.0f));
  return make_float2(fminf(q.x, 6.0f), fminf(q.y, 6.0f));
}

// ---------------------------------------------------------------- indexing
// Division by a runtime constant d >= 1 for numerators n < 2^31:
// n / d = (umulhi(n, m) + n) >> s.
struct FastDiv {
  uint32_t d, m, s;
};

__device__ __forceinline__ uint32_t fdiv(uint32_t n, const FastDiv& f) {
  return (__umulhi(n, f.m) + n) >> f.s;
}

// Byte offset of scale (r, c) of an [R][sf_cols] matrix in the tensor-core
// block-scaled layout: 512-byte tiles of 128 rows x 4 scales, tiles ordered
// row-major; inside a tile (r % 32) * 16 + ((r % 128) / 32) * 4 + c % 4.
__device__ __forceinline__ long long swz_offset(long long r, long long c, long long col_tiles) {
  return ((r >> 7) * col_tiles + (c >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (c & 3);
}

// Non-negative binary32 values compare like their bit patterns.
__device__ __forceinline__ void atomic_max_pos(uint32_t* addr, float v) {
  atomicMax(addr, __float_as_uint(v));
}

}  // namespace fos
