// fos_check.cu -- libfos_check.so: exhaustive device-side checks of the
// arithmetic shortcuts and conversion helpers that the quantizer kernels of
// libfos.so are built from.  TEST INFRASTRUCTURE: nothing in libfos.so calls
// it; tests/test_gpu_exhaustive.py does.  It includes the kernels' own
// device headers, so the functions checked here are the ones that run.
//
// Each check runs one or more kernels over a whole input domain (every
// binary32 pattern, every bf16 pair, every (value, random byte) pair) and
// counts disagreements with the plain definition of the step:
//  * div6_for_e4m3(r) against the IEEE quotient r / 6 (__fdiv_rn);
//  * the per-tensor division shortcut div_tscale (and its compile-time
//    variants) against the IEEE quotient a / S_t, through the two E4M3
//    candidate scale codes that are its only use;
//  * the integer form of the stochastic-rounding rule against the float
//    form, after the saturating E2M1 encode that follows both;
//  * the E2M1 and E4M3 encoders (cvt ... satfinite): every transition point
//    of the code over the binary32 patterns is returned for a host-side
//    comparison (a piecewise-constant, monotone function is fixed by its
//    transitions);
//  * the E2M1 nibble decoder of eight packed codes, against a 16-entry table
//    given by the host;
//  * the packed bf16 magnitude maximum, against the integer maximum of the
//    magnitude bits.
// Every kernel reads only its arguments and writes only its count words and
// bounded output arrays.
#include <stdint.h>

#include <curand_kernel.h>  // curand_Philox4x32_10: cuRAND's Philox4x32-10, called as a reference

#include "fos_check.h"
#include "fos_core.cuh"

namespace {

using namespace fos;

constexpr int kThreads = 256;
constexpr unsigned kGrid = 148 * 8;

__device__ __forceinline__ bool is_nan_bits(uint32_t u) { return (u & 0x7fffffffu) > 0x7f800000u; }

// ------------------------------------------------------------ r / 6
// counts[0]: finite r >= 2^-125 whose bits differ from IEEE r/6.
// counts[1]: any finite r >= 0 whose E4M3 code of the quotient differs.
__global__ void k_div6(unsigned long long* counts) {
  unsigned long long bad_bits = 0, bad_code = 0;
  const unsigned long long n = 0x7f800000ull;
  for (unsigned long long u = blockIdx.x * (unsigned long long)blockDim.x + threadIdx.x; u < n;
       u += (unsigned long long)gridDim.x * blockDim.x) {
    const float r = __uint_as_float((uint32_t)u);
    const float got = div6_for_e4m3(r);
    const float want = __fdiv_rn(r, 6.0f);
    if (u >= 0x01000000ull && __float_as_uint(got) != __float_as_uint(want)) ++bad_bits;  // 2^-125
    if ((e4m3x2(0.0f, got) & 0xffu) != (e4m3x2(0.0f, want) & 0xffu)) ++bad_code;
  }
  if (bad_bits) atomicAdd(counts + 0, bad_bits);
  if (bad_code) atomicAdd(counts + 1, bad_code);
}

// ------------------------------------------------------------ a / S_t
// The reference: RN(a / S_t) (0 when S_t == 0), then E4M3(RN(r/6)) and
// E4M3(RN(r/4)).
__device__ __forceinline__ void ref_scales(float a, float St, uint32_t& s6, uint32_t& s4, float& r) {
  r = (St == 0.0f) ? 0.0f : __fdiv_rn(a, St);
  const uint32_t both = e4m3x2(__fdiv_rn(r, 6.0f), __fmul_rn(r, 0.25f));
  s6 = (both >> 8) & 0x7fu;
  s4 = both & 0x7fu;
}

// One (a, S_t) case through every variant the kernels use: counts[0] scale
// code mismatches, counts[1] quotient-bit mismatches where a and the
// quotient are >= 2^-100 and the quotient is finite.
__device__ __forceinline__ void check_pair(float a, float St, unsigned long long& bad_code,
                                           unsigned long long& bad_bits) {
  uint32_t w6, w4;
  float r;
  ref_scales(a, St, w6, w4, r);
  const TScale ts = make_tscale(St);
  uint32_t s6, s4;
  cand_scales<true, -1>(a, ts, s6, s4);
  bad_code += (s6 != w6) + (s4 != w4);
  if (ts.fast) cand_scales<true, 1>(a, ts, s6, s4);
  else         cand_scales<true, 0>(a, ts, s6, s4);
  bad_code += (s6 != w6) + (s4 != w4);
  cand_scales<false, -1>(a, ts, s6, s4);
  bad_code += (s6 != w6);
  const float q = div_tscale(a, ts);
  if (a >= 7.888609052210118e-31f && r >= 7.888609052210118e-31f && r <= kFltMax &&
      __float_as_uint(q) != __float_as_uint(r))
    ++bad_bits;
}

// Every pair (a, A) of non-negative finite bf16 values (a: a block amax, A:
// a tensor amax; a > A happens with a caller-supplied amax), with
// S_t = RN(A / div) as the kernels form it.
__global__ void k_div_tscale_bf16(float div, unsigned long long* counts) {
  unsigned long long bad_code = 0, bad_bits = 0;
  const unsigned long long nv = 0x7f80ull;  // bf16 patterns 0x0000 .. 0x7f7f
  const unsigned long long n = nv * nv;
  for (unsigned long long u = blockIdx.x * (unsigned long long)blockDim.x + threadIdx.x; u < n;
       u += (unsigned long long)gridDim.x * blockDim.x) {
    const uint32_t ia = (uint32_t)(u / nv), iA = (uint32_t)(u % nv);
    const float a = __uint_as_float(ia << 16);
    const float St = __fdiv_rn(__uint_as_float(iA << 16), div);
    check_pair(a, St, bad_code, bad_bits);
  }
  if (bad_code) atomicAdd(counts + 0, bad_code);
  if (bad_bits) atomicAdd(counts + 1, bad_bits);
}

__device__ __forceinline__ uint32_t mix32(uint64_t x) {
  x ^= x >> 33;
  x *= 0xff51afd7ed558ccdull;
  x ^= x >> 33;
  x *= 0xc4ceb9fe1a85ec53ull;
  x ^= x >> 33;
  return (uint32_t)x;
}

// n random (a, S_t) pairs of positive finite binary32 values (uniform over
// the bit patterns, so over the binades): the case of a transformed (RHT)
// block, whose amax is any binary32.  Half of the S_t values are drawn near
// a / 1792 so that the quotients land in the E4M3 range.
__global__ void k_div_tscale_random(unsigned long long seed, unsigned long long n,
                                    unsigned long long* counts) {
  unsigned long long bad_code = 0, bad_bits = 0;
  for (unsigned long long u = blockIdx.x * (unsigned long long)blockDim.x + threadIdx.x; u < n;
       u += (unsigned long long)gridDim.x * blockDim.x) {
    const uint32_t ha = mix32(seed * 0x9E3779B97F4A7C15ull + 2 * u);
    const uint32_t hs = mix32(seed * 0x9E3779B97F4A7C15ull + 2 * u + 1);
    const float a = __uint_as_float(1u + ha % 0x7f7fffffu);
    float St;
    if (hs & 1u) {
      St = __uint_as_float(1u + (hs >> 1) % 0x7f7fffffu);
    } else {
      // A = a * 2^k for k in [0, 31): quotients from 1792 down to ~1e-6
      const float A = fminf(__fmul_rn(a, __uint_as_float((127u + ((hs >> 1) % 31u)) << 23)), kFltMax);
      St = __fdiv_rn(A, 1792.0f);
    }
    check_pair(a, St, bad_code, bad_bits);
  }
  if (bad_code) atomicAdd(counts + 0, bad_code);
  if (bad_bits) atomicAdd(counts + 1, bad_bits);
}

// ------------------------------------------------------------ Philox
// n seeded random (counter, key) pairs: the kernels' Philox4x32-10 against
// cuRAND's; counts[0] += output words that differ.
__global__ void k_philox_vs_curand(unsigned long long seed, unsigned long long n, unsigned long long* counts) {
  unsigned long long bad = 0;
  for (unsigned long long u = blockIdx.x * (unsigned long long)blockDim.x + threadIdx.x; u < n;
       u += (unsigned long long)gridDim.x * blockDim.x) {
    const unsigned long long h = seed * 0x9E3779B97F4A7C15ull + 8 * u;
    const uint4 c = make_uint4(mix32(h), mix32(h + 1), mix32(h + 2), mix32(h + 3));
    const uint2 k = make_uint2(mix32(h + 4), mix32(h + 5));
    const uint4 a = philox4x32_10(c, k);
    const uint4 r = curand_Philox4x32_10(c, k);
    bad += (a.x != r.x) + (a.y != r.y) + (a.z != r.z) + (a.w != r.w);
  }
  if (bad) atomicAdd(counts, bad);
}

// ------------------------------------------------------------ SR
// Every binary32 v in [0, 16] and +inf, with every byte: the E2M1 code of
// the integer-form rule and of the pair (ceiling) form vs the float-form
// rule.
__global__ void k_sr_forms(unsigned long long* counts) {
  unsigned long long bad = 0;
  const unsigned long long n = 0x41800001ull + 1;  // 0 .. 16.0, then +inf
  for (unsigned long long u = blockIdx.x * (unsigned long long)blockDim.x + threadIdx.x; u < n;
       u += (unsigned long long)gridDim.x * blockDim.x) {
    const uint32_t vb = (u == n - 1) ? 0x7f800000u : (uint32_t)u;
    const float v = __uint_as_float(vb);
    for (uint32_t byte = 0; byte < 256; byte += 2) {
      const uint32_t c1 = e2m1x8(sr_e2m1_mag(v, byte), sr_e2m1_mag(v, byte + 1), 0, 0, 0, 0, 0, 0);
      const uint32_t c2 =
          e2m1x8(sr_e2m1_mag_bits(v, byte), sr_e2m1_mag_bits(v, byte + 1), 0, 0, 0, 0, 0, 0);
      const float2 q = sr_e2m1_mag2(make_float2(v, v), sr_thr_bits(byte), sr_thr_bits(byte + 1));
      const uint32_t c3 = e2m1x8(q.x, q.y, 0, 0, 0, 0, 0, 0);
      bad += (c1 != c2) + (c1 != c3);
    }
  }
  if (bad) atomicAdd(counts, bad);
}

__global__ void k_sr_codes(const float* v, const uint8_t* bytes, long long n, int form, uint8_t* out) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const float m = form == 2 ? sr_e2m1_mag2(make_float2(v[i], 0.0f), sr_thr_bits(bytes[i]), sr_thr_bits(0)).x
                    : form ? sr_e2m1_mag_bits(v[i], bytes[i]) : sr_e2m1_mag(v[i], bytes[i]);
    out[i] = (uint8_t)(e2m1x8(m, 0, 0, 0, 0, 0, 0, 0) & 0xfu);
  }
}

// ------------------------------------------------------------ encoders
// Code of binary32 pattern u under the encoder (both lanes of the x2
// conversion; a lane disagreement is reported as code 0xffff).
template <bool E4M3>
__device__ __forceinline__ uint32_t enc_code(uint32_t u) {
  const float v = __uint_as_float(u);
  if (E4M3) {
    const uint32_t both = e4m3x2(v, v);
    return ((both >> 8) == (both & 0xffu)) ? (both & 0xffu) : 0xffffu;
  }
  const uint32_t w = e2m1x8(v, v, 0, 0, 0, 0, 0, 0) & 0xffu;
  return ((w >> 4) == (w & 0xfu)) ? (w & 0xfu) : 0xffffu;
}

// Every non-NaN binary32 pattern, in chunks of kChunk per thread: record
// (index, code before, code after) wherever the code changes from pattern
// i-1 to pattern i (both non-NaN, same sign half).
constexpr uint32_t kChunk = 4096;
template <bool E4M3>
__global__ void k_transitions(uint32_t* out, uint32_t max_out, uint32_t* count) {
  const unsigned long long nchunks = (1ull << 32) / kChunk;
  for (unsigned long long c = blockIdx.x * (unsigned long long)blockDim.x + threadIdx.x; c < nchunks;
       c += (unsigned long long)gridDim.x * blockDim.x) {
    const uint32_t i0 = (uint32_t)(c * kChunk);
    bool have = false;
    uint32_t prev = 0;
    if ((i0 & 0x7fffffffu) != 0 && !is_nan_bits(i0 - 1)) {
      prev = enc_code<E4M3>(i0 - 1);
      have = true;
    }
    for (uint32_t k = 0; k < kChunk; ++k) {
      const uint32_t i = i0 + k;
      if (is_nan_bits(i) || (i & 0x7fffffffu) == 0) {
        have = false;
        if (is_nan_bits(i)) continue;
      }
      const uint32_t cur = enc_code<E4M3>(i);
      if (have && cur != prev) {
        const uint32_t slot = atomicAdd(count, 1u);
        if (slot < max_out) {
          out[3 * slot] = i;
          out[3 * slot + 1] = prev;
          out[3 * slot + 2] = cur;
        }
      }
      prev = cur;
      have = true;
    }
  }
}

// Code of one pattern under each encoder, for the segment ends the host
// checks (both lanes agree or 0xffff).
__global__ void k_codes_at(const uint32_t* idx, long long n, int e4m3, uint32_t* out) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x)
    out[i] = e4m3 ? enc_code<true>(idx[i]) : enc_code<false>(idx[i]);
}

// ------------------------------------------------------------ decoders
// Every 32-bit word of eight E2M1 codes through e2m1x8_to_h2 vs the table
// (f16 bits of each nibble's value, from the host).
__global__ void k_e2m1_decode_words(const uint16_t* table16, unsigned long long* counts) {
  __shared__ uint16_t t[16];
  if (threadIdx.x < 16) t[threadIdx.x] = table16[threadIdx.x];
  __syncthreads();
  unsigned long long bad = 0;
  for (unsigned long long u = blockIdx.x * (unsigned long long)blockDim.x + threadIdx.x; u < (1ull << 32);
       u += (unsigned long long)gridDim.x * blockDim.x) {
    const uint32_t w = (uint32_t)u;
    uint32_t h[4];
    e2m1x8_to_h2(w, h);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t want = (uint32_t)t[(w >> (8 * k)) & 0xfu] | ((uint32_t)t[(w >> (8 * k + 4)) & 0xfu] << 16);
      bad += (h[k] != want);
    }
  }
  if (bad) atomicAdd(counts, bad);
}

__global__ void k_e4m3_decode_all(float* out) {
  const uint32_t c = threadIdx.x;
  if (c < 256) out[c] = e4m3_to_f32(c);
}

// Every pair (x, y) of bf16 patterns (NaN excluded): the magnitude bits of
// the packed max in both halves vs max(|x|, |y|) as integers.
__global__ void k_hmax_abs(unsigned long long* counts) {
  unsigned long long bad = 0;
  for (unsigned long long u = blockIdx.x * (unsigned long long)blockDim.x + threadIdx.x; u < (1ull << 32);
       u += (unsigned long long)gridDim.x * blockDim.x) {
    const uint32_t x = (uint32_t)u & 0xffffu, y = (uint32_t)(u >> 16);
    if ((x & 0x7fffu) > 0x7f80u || (y & 0x7fffu) > 0x7f80u) continue;
    const uint32_t d = hmax_abs2(x | (y << 16), y | (x << 16)) & 0x7fff7fffu;
    const uint32_t want = max(x & 0x7fffu, y & 0x7fffu);
    bad += ((d & 0xffffu) != want) + ((d >> 16) != want);
  }
  if (bad) atomicAdd(counts, bad);
}

int launched(cudaError_t e) { return (int)(e == cudaSuccess ? cudaGetLastError() : e); }

}  // namespace

extern "C" {

int fosck_div6(unsigned long long* counts, void* stream) {
  k_div6<<<kGrid, kThreads, 0, (cudaStream_t)stream>>>(counts);
  return launched(cudaSuccess);
}

int fosck_div_tscale_bf16(float divisor, unsigned long long* counts, void* stream) {
  k_div_tscale_bf16<<<kGrid, kThreads, 0, (cudaStream_t)stream>>>(divisor, counts);
  return launched(cudaSuccess);
}

int fosck_div_tscale_random(unsigned long long seed, unsigned long long n, unsigned long long* counts,
                            void* stream) {
  k_div_tscale_random<<<kGrid, kThreads, 0, (cudaStream_t)stream>>>(seed, n, counts);
  return launched(cudaSuccess);
}

int fosck_philox_vs_curand(unsigned long long seed, unsigned long long n, unsigned long long* counts,
                           void* stream) {
  k_philox_vs_curand<<<kGrid, kThreads, 0, (cudaStream_t)stream>>>(seed, n, counts);
  return launched(cudaSuccess);
}

int fosck_sr_forms(unsigned long long* counts, void* stream) {
  k_sr_forms<<<kGrid, kThreads, 0, (cudaStream_t)stream>>>(counts);
  return launched(cudaSuccess);
}

int fosck_sr_codes(const float* v, const uint8_t* bytes, long long n, int form, uint8_t* out,
                   void* stream) {
  if (n <= 0) return 0;
  k_sr_codes<<<kGrid, kThreads, 0, (cudaStream_t)stream>>>(v, bytes, n, form, out);
  return launched(cudaSuccess);
}

int fosck_transitions(int e4m3, uint32_t* out, uint32_t max_out, uint32_t* count, void* stream) {
  if (e4m3) k_transitions<true><<<kGrid, kThreads, 0, (cudaStream_t)stream>>>(out, max_out, count);
  else      k_transitions<false><<<kGrid, kThreads, 0, (cudaStream_t)stream>>>(out, max_out, count);
  return launched(cudaSuccess);
}

int fosck_codes_at(const uint32_t* idx, long long n, int e4m3, uint32_t* out, void* stream) {
  if (n <= 0) return 0;
  k_codes_at<<<kGrid, kThreads, 0, (cudaStream_t)stream>>>(idx, n, e4m3, out);
  return launched(cudaSuccess);
}

int fosck_e2m1_decode_words(const uint16_t* table16, unsigned long long* counts, void* stream) {
  k_e2m1_decode_words<<<kGrid, kThreads, 0, (cudaStream_t)stream>>>(table16, counts);
  return launched(cudaSuccess);
}

int fosck_e4m3_decode_all(float* out256, void* stream) {
  k_e4m3_decode_all<<<1, 256, 0, (cudaStream_t)stream>>>(out256);
  return launched(cudaSuccess);
}

int fosck_hmax_abs(unsigned long long* counts, void* stream) {
  k_hmax_abs<<<kGrid, kThreads, 0, (cudaStream_t)stream>>>(counts);
  return launched(cudaSuccess);
}

}  // extern "C"
