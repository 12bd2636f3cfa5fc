/*
 * fos_check.h -- C ABI of libfos_check.so, the exhaustive device-side checks
 * of the arithmetic shortcuts and conversion helpers inside libfos.so's
 * quantizer kernels.  TEST INFRASTRUCTURE: the quantizer never calls these;
 * tests/test_gpu_exhaustive.py does.  The library is compiled from the same
 * device headers as libfos.so, so the code checked is the code that runs.
 *
 * The steps checked are those of the 4/6 NVFP4 block quantizer described by
 * the Hugging Face transformers doc "Four Over Six" (introduction: block max
 * mapped to 4 or to 6) and the Ultralytics glossary "FP4" ("Como funciona
 * FP4": E4M3 block scale, FP32 tensor scale, E2M1 values; "Inferencia e
 * Treinamento FP4": stochastic rounding):
 *   r = a / S_t, s6 = E4M3(r / 6), s4 = E4M3(r / 4), the E2M1 and E4M3
 *   encoders, the E2M1 decoder and the stochastic-rounding rule.
 *
 * Conventions: every pointer is a DEVICE pointer; `stream` is a
 * cudaStream_t.  Each call only enqueues kernels and returns the launch's
 * cudaError_t value (0 = enqueued).  Count words are ADDED to (zero them
 * first); the caller synchronises before reading them.  Nothing is
 * allocated.
 */
#ifndef FOS_CHECK_H_
#define FOS_CHECK_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Every finite binary32 r >= 0 through the division-free r/6 of the block
 * scale step, against IEEE r/6.  counts[0] += quotients >= 2^-125 whose bits
 * differ; counts[1] += quotients whose E4M3 codes differ. */
int fosck_div6(unsigned long long* counts, void* stream);

/* Every pair (a, A) of non-negative finite bf16 values, S_t = RN(A/divisor)
 * (divisor 1792 for 4/6, 2688 for 6-only): the candidate scale codes of
 * every variant of the a / S_t shortcut against IEEE division.  counts[0] +=
 * scale-code mismatches; counts[1] += quotient-bit mismatches where dividend
 * and quotient are >= 2^-100 and the quotient is finite. */
int fosck_div_tscale_bf16(float divisor, unsigned long long* counts, void* stream);

/* The same on n seeded random pairs of positive finite binary32 values (the
 * transformed-block case, where a and A are any binary32). */
int fosck_div_tscale_random(unsigned long long seed, unsigned long long n,
                            unsigned long long* counts, void* stream);

/* n seeded random (counter, key) pairs through the kernels' Philox4x32-10
 * (Salmon et al., SC'11; the SR bytes and the RHT signs) and through
 * cuRAND's curand_Philox4x32_10.  counts[0] += output words that differ. */
int fosck_philox_vs_curand(unsigned long long seed, unsigned long long n, unsigned long long* counts,
                           void* stream);

/* Every binary32 v in [0, 16] and +inf with every byte 0..255: the E2M1 code
 * of the integer form and of the pair (ceiling) form of the
 * stochastic-rounding rule against the float form.  counts[0] += mismatching
 * codes. */
int fosck_sr_forms(unsigned long long* counts, void* stream);

/* out[i] = E2M1 magnitude code of the stochastic rounding of v[i] with byte
 * bytes[i] (form 0: float form, 1: integer form, 2: pair form), i < n. */
int fosck_sr_codes(const float* v, const uint8_t* bytes, long long n, int form, uint8_t* out,
                   void* stream);

/* Every non-NaN binary32 pattern through the E2M1 (e4m3 = 0) or E4M3
 * (e4m3 = 1) saturating encoder: for each pattern i whose code differs from
 * that of pattern i-1 (both non-NaN, same sign), one triple
 * (i, code of i-1, code of i) goes to out[3*slot .. 3*slot+2] for slot <
 * max_out; *count += the number of such patterns.  A code of 0xffff means
 * the two lanes of the paired conversion disagreed. */
int fosck_transitions(int e4m3, uint32_t* out, uint32_t max_out, uint32_t* count, void* stream);

/* out[i] = code of binary32 pattern idx[i] under the encoder (as above). */
int fosck_codes_at(const uint32_t* idx, long long n, int e4m3, uint32_t* out, void* stream);

/* Every 32-bit word of eight E2M1 codes through the eight-code decoder of the
 * error step, against table16 (f16 bits of each code's value).  counts[0] +=
 * mismatching f16x2 results. */
int fosck_e2m1_decode_words(const uint16_t* table16, unsigned long long* counts, void* stream);

/* out256[c] = binary32 value the kernels decode E4M3 code c to. */
int fosck_e4m3_decode_all(float* out256, void* stream);

/* Every pair of non-NaN bf16 patterns through the packed magnitude maximum
 * of the block amax step.  counts[0] += results whose magnitude bits differ
 * from the integer maximum of the magnitude bits. */
int fosck_hmax_abs(unsigned long long* counts, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FOS_CHECK_H_ */
