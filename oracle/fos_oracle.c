/*
 * fos_oracle.c -- plain CPU oracle for Four Over Six (4/6) NVFP4 block
 * quantization, its options and its comparison formats.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only tests/, __graft_entry__.smoke() and the CPU-baseline
 * leg of bench.py use it.  It shares no code, header, table or constant
 * generator with the CUDA library under mxfp4_block_scaled_fos_b200/csrc.
 *
 * Everything is written for clarity, not speed: nearest-value searches over
 * the format value sets, one block at a time, plain loops.  All arithmetic is
 * IEEE binary32 with round-to-nearest-even (build with -ffp-contract=off and
 * no fast-math), except where a comment says a step is exact and is done in
 * binary64 for clarity.  Subnormals are honoured.
 *
 * Sources ("the pages"):
 *   [FOS]  Hugging Face transformers doc "Four Over Six" (pt and ar copies),
 *          introduction: each NVFP4 block is scaled adaptively to 4 or to 6
 *          to lower the error of the values near the block maximum; usage
 *          section: options random Hadamard transform, 2D block scaling,
 *          transposed inputs, stochastic rounding.
 *   [FP4]  Ultralytics glossary "FP4": intro (E2M1 value set
 *          0, +-0.5, +-1, +-1.5, +-2, +-3, +-4, +-6), "Como funciona FP4"
 *          (block max mapped near 6; MXFP4 = 32 values + E8M0 power-of-two
 *          scale; NVFP4 = 16 values + E4M3 scale + FP32 per-tensor scale;
 *          worked example of blockwise MAE), "Inferencia e Treinamento FP4"
 *          (Hadamard transforms spread outliers, stochastic rounding for
 *          gradients).
 *   [SPEC] The benchmark spec of this library: 4/6 keeps the candidate with
 *          the lower block squared error, ties to 6; per-tensor scale
 *          tensor_amax / (4 * 448); 16-wide RHT with seeded +-1 signs;
 *          16x16 2D tiles; Philox4x32 stochastic rounding keyed on
 *          (seed, element index).
 *   Readings where the sources are silent are named R1..R20 below and are
 *   listed with their justification in the design notes of this repository.
 *
 * Pinning: every function here is checked by tests/test_oracle_pins.py
 * against something other than itself (ml_dtypes codecs, scipy's Hadamard
 * matrix, Triton's CPU Philox, the worked example's printed MAEs, invariants,
 * brute force).  Parity unpinned (fixed only by the readings and by GPU
 * parity, not by the pages): the binary32 evaluation order of the block
 * error tree (R6), of the effective scale (R5) and of the Hadamard
 * butterflies (R10).  The NVFP4 swizzled scale layout (R19) is pinned through
 * GPU parity and a cuBLAS block-scaled GEMM that consumes it.
 */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_VERSION 1

/* Mutation hooks for tests/test_oracle_mutants.py.  Building with
 * -DOR_MUTANT=k plants one plausible mistake (listed in that test); the pins
 * of tests/test_oracle_pins.py must catch every one of them.  The oracle the
 * other tests use is built without the macro and has none. */
#ifndef OR_MUTANT
#define OR_MUTANT 0
#endif

enum { OR_FMT_NVFP4_46 = 0, OR_FMT_NVFP4_6 = 1, OR_FMT_MXFP4 = 2 };
enum { OR_BLK_1X16 = 0, OR_BLK_16X16 = 1, OR_BLK_1X32 = 2 };
enum { OR_RND_RNE = 0, OR_RND_SR = 1 };
enum { OR_OK = 0, OR_NONFINITE = 1, OR_UNSUPPORTED = 2, OR_SHAPE = 3 };

typedef struct {
  int32_t fmt;          /* OR_FMT_* */
  int32_t blk;          /* OR_BLK_* */
  int32_t rnd;          /* OR_RND_* */
  int32_t rht;          /* 1 = 16-wide random Hadamard transform along cols */
  uint64_t seed;        /* Philox key for RHT signs and SR draws */
  int64_t elem_offset;  /* global linear index of element [0,0,0] (SR) */
  int32_t rht_col;      /* 1 = the same transform along rows for the colwise copy */
  int32_t pad;
} or_opts;

int or_version(void) { return OR_VERSION; }

/* ------------------------------------------------------------------ */
/* bf16 <-> fp32                                                        */
/* ------------------------------------------------------------------ */

float or_bf16_to_f32(uint16_t h) {
  uint32_t u = (uint32_t)h << 16; /* bf16 is the top half of binary32 */
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* Round a finite binary32 to the nearest bf16, ties to even (drop 16 bits). */
uint16_t or_f32_to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if (isnan(f)) return (uint16_t)((u >> 16) | 0x40);
  uint32_t lower = u & 0xFFFF0000u;   /* truncated candidate */
  uint32_t rest = u & 0x0000FFFFu;    /* discarded bits */
  uint32_t keep = lower >> 16;
  if (rest > 0x8000u || (rest == 0x8000u && (OR_MUTANT == 17 || (keep & 1u)))) keep += 1; /* up */
  return (uint16_t)keep;
}

/* ------------------------------------------------------------------ */
/* E2M1 (FP4): 1 sign, 2 exponent, 1 mantissa bit  ([FP4] intro)        */
/* R1: bit 3 = sign, magnitude code 0..7 -> 0,0.5,1,1.5,2,3,4,6.         */
/* ------------------------------------------------------------------ */

static const double E2M1_GRID[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

float or_e2m1_decode(uint8_t code) {
  double m = E2M1_GRID[code & 7];
  return (float)((code & 8) ? -m : m);
}

/* Magnitude code of the grid value nearest to |v|; on a tie the code with
 * an even mantissa bit (code & 1 == 0) wins (R2: round-to-nearest-even).
 * Every value at or above 6 is nearest to 6: the saturation of R2.  Below 6
 * the distances to the two nearest grid values are exact in binary64 (the
 * operands are binary32 values of similar magnitude), so ties are seen. */
static int e2m1_mag_rne(double m) {
  if (m >= 6.0) return 7;
  int best = 0;
  double bd = fabs(m - E2M1_GRID[0]);
  for (int c = 1; c < 8; c++) {
    double d = fabs(m - E2M1_GRID[c]);
    if (d < bd || (d == bd && (OR_MUTANT == 3 || (c & 1) == 0))) {
      best = c;
      bd = d;
    }
  }
  return best;
}

/* R2: the sign bit of the code is always signbit(v), zeros included. */
uint8_t or_e2m1_encode(float v) {
  return (uint8_t)(e2m1_mag_rne(fabs((double)v)) | (signbit(v) ? 8 : 0));
}

/* ------------------------------------------------------------------ */
/* E4M3 ("fn": bias 7, no infinities, 0x7F/0xFF = NaN, max 448)          */
/* NVFP4 block scale ([FP4] "Como funciona FP4", NVFP4 bullet).          */
/* ------------------------------------------------------------------ */

float or_e4m3_decode(uint8_t code) {
  int s = code >> 7, e = (code >> 3) & 15, m = code & 7;
  if (e == 15 && m == 7) return NAN;
  double v = (e == 0) ? ldexp((double)m, -9)          /* m/8 * 2^(1-7) */
                      : ldexp((double)(8 + m), e - 10); /* (1+m/8) * 2^(e-7) */
  return (float)(s ? -v : v);
}

/* R4: nearest E4M3 value, ties to the even code, saturating at 448. */
uint8_t or_e4m3_encode(float v) {
  double m = fabs((double)v);
  int best = 0;
  if (m >= 448.0) { /* saturation: everything from the max up maps to 448 */
    best = 0x7E;
  } else {
    double bd = m; /* distance to code 0 (= 0.0) */
    for (int c = 1; c <= 0x7E; c++) {
      double d = fabs(m - (double)or_e4m3_decode((uint8_t)c));
      if ((OR_MUTANT == 6) ? ((double)or_e4m3_decode((uint8_t)c) <= m)
                          : (d < bd || (d == bd && (c & 1) == 0))) {
        best = c;
        bd = d;
      }
    }
  }
  return (uint8_t)(best | (signbit(v) ? 0x80 : 0));
}

/* ------------------------------------------------------------------ */
/* E8M0 (MXFP4 scale, [FP4] MXFP4 bullet)                               */
/* R9: E = floor(log2 a) - 2 (E2M1's largest exponent is 2), clamped to  */
/* [-127, 127]; a == 0 gives -127.  Scale byte = E + 127.                */
/* ------------------------------------------------------------------ */

int or_e8m0_exponent(float a) {
  if (a == 0.0f) return -127;
  int ex;
  (void)frexp((double)a, &ex); /* a = f * 2^ex, f in [0.5, 1): exact */
  int e = (ex - 1) - (OR_MUTANT == 9 ? 1 : 2); /* floor(log2 a) = ex - 1 */
  if (e < -127) e = -127;
  if (e > 127) e = 127;
  return e;
}

float or_e8m0_decode(uint8_t code) {
  if (code == 0xFF) return NAN;
  return (float)ldexp(1.0, (int)code - 127);
}

/* ------------------------------------------------------------------ */
/* Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: */
/* As Easy as 1, 2, 3", SC'11): ten rounds of the 4x32 S-P network with  */
/* multipliers 0xD2511F53 / 0xCD9E8D57 and Weyl key increments           */
/* 0x9E3779B9 / 0xBB67AE85 applied between rounds.                       */
/* ------------------------------------------------------------------ */

void or_philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2],
                      uint32_t out[4]) {
  uint32_t c[4] = {ctr_in[0], ctr_in[1], ctr_in[2], ctr_in[3]};
  uint32_t k[2] = {key_in[0], key_in[1]};
  for (int round = 0; round < 10; round++) {
    if (round > 0) {
      k[0] += (OR_MUTANT == 16) ? 0x9E3779B8u : 0x9E3779B9u;
      k[1] += 0xBB67AE85u;
    }
    uint64_t p0 = (uint64_t)0xD2511F53u * (uint64_t)c[0];
    uint64_t p1 = (uint64_t)0xCD9E8D57u * (uint64_t)c[2];
    uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
    uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
    uint32_t n0 = hi1 ^ c[1] ^ k[0];
    uint32_t n1 = lo1;
    uint32_t n2 = hi0 ^ c[3] ^ k[1];
    uint32_t n3 = lo0;
    c[0] = n0; c[1] = n1; c[2] = n2; c[3] = n3;
  }
  out[0] = c[0]; out[1] = c[1]; out[2] = c[2]; out[3] = c[3];
}

static void seed_key(uint64_t seed, uint32_t key[2]) {
  key[0] = (uint32_t)(seed & 0xFFFFFFFFu);
  key[1] = (uint32_t)(seed >> 32);
}

/* R15: the stochastic-rounding byte of source element g. */
static uint8_t sr_byte(uint64_t seed, int64_t g) {
  uint32_t key[2], out[4];
  seed_key(seed, key);
  uint64_t ug = (uint64_t)g;
  uint32_t ctr[4] = {(uint32_t)((ug >> (OR_MUTANT == 18 ? 0 : 4)) & 0xFFFFFFFFu), (uint32_t)(ug >> 36),
                     0u, 0u};
  or_philox4x32_10(ctr, key, out);
  int j = (int)((ug + (OR_MUTANT == 11)) & 15);
  return (uint8_t)((out[j >> 2] >> (8 * (j & 3))) & 0xFFu);
}

/* ------------------------------------------------------------------ */
/* 16-wide random Hadamard transform ([FOS] usage; [FP4] training)       */
/* R10: y = 0.25 * H16 * (D .* x), Sylvester H16, D from Philox with     */
/* counter (0,0,1,0): bit i of output word 0 set -> D_ii = -1.           */
/* ------------------------------------------------------------------ */

uint32_t or_rht16_signs(uint64_t seed) {
  uint32_t key[2], out[4], ctr[4] = {0u, 0u, 1u, 0u};
  seed_key(seed, key);
  or_philox4x32_10(ctr, key, out);
  return out[OR_MUTANT == 7 ? 1 : 0] & 0xFFFFu;
}

void or_rht16(float x[16], uint32_t sign_mask) {
  for (int i = 0; i < 16; i++)
    if ((sign_mask >> i) & 1u) x[i] = -x[i];
  for (int h = 1; h < 16; h *= 2)          /* strides 1, 2, 4, 8 */
    for (int i = 0; i < 16; i += 2 * h)
      for (int j = i; j < i + h; j++) {
        float a = x[j], b = x[j + h];
        x[j] = a + b;
        x[j + h] = a - b;
      }
  for (int i = 0; i < 16; i++) x[i] = x[i] * 0.25f;
}

/* ------------------------------------------------------------------ */
/* NVFP4 pieces                                                          */
/* ------------------------------------------------------------------ */

/* R3: per-tensor scale.  4/6 maps the tensor max to 4 * 448 ([SPEC]);
 * 6-only maps it to 6 * 448, the usual NVFP4 reading of [FP4]'s "block
 * max near 6". */
float or_tensor_scale(float amax, int fmt) {
  if (fmt == OR_FMT_NVFP4_6) return amax / 2688.0f;
  return amax / (OR_MUTANT == 2 ? 2688.0f : 1792.0f);
}

/* R4: the two candidate scale codes of a block with amax a. */
static void candidate_scales(float a, float S_t, int fmt, uint8_t* s6, uint8_t* s4) {
  if (S_t == 0.0f) { /* R3: a zero tensor scale gives zero block scales */
    *s6 = 0;
    *s4 = 0;
    return;
  }
  float r = a / S_t;
  *s6 = or_e4m3_encode(r / 6.0f);
  *s4 = (fmt == OR_FMT_NVFP4_46) ? or_e4m3_encode(r / (OR_MUTANT == 15 ? 3.0f : 4.0f)) : 0;
}

/* R5: effective scale e = float(s) * S_t and its inverse; a zero e gives a
 * zero inverse (all magnitudes 0); an inverse that overflows is clamped to
 * FLT_MAX so that |w| * inv is never 0 * inf. */
static void effective_scale(uint8_t s, float S_t, float* e, float* inv) {
  float ek = or_e4m3_decode(s) * S_t;
  float iv = 0.0f;
  if (ek != 0.0f) {
    iv = 1.0f / ek;
    if (iv > FLT_MAX) iv = FLT_MAX;
  }
  *e = ek;
  *inv = iv;
}

/* R6: pairwise tree over contiguous indices, n a power of two. */
static float tree_sum(const float* t, int n) {
  if (n == 1) return t[0];
  float left = tree_sum(t, n / 2);
  float right = tree_sum(t + n / 2, n / 2);
  return left + right;
}

/* Quantize n values with one candidate scale by RNE: codes[i] (sign|mag) and
 * the squared-error terms t[i] = d*d with d = fma(-sign*q, e, w) (R6). */
static void candidate_rne(const float* w, int n, uint8_t s, float S_t,
                          uint8_t* codes, float* t) {
  float e, inv;
  effective_scale(s, S_t, &e, &inv);
  for (int i = 0; i < n; i++) {
    float v = fabsf(w[i]) * inv;
    int mag = e2m1_mag_rne((double)v);
    codes[i] = (uint8_t)(mag | (signbit(w[i]) ? 8 : 0));
    float q = (float)E2M1_GRID[mag];
    float sq = signbit(w[i]) ? -q : q;
    float d = fmaf((OR_MUTANT == 5) ? sq : -sq, e, w[i]);
    t[i] = (OR_MUTANT == 4 && i == n - 1) ? 0.0f : d * d;
  }
}

/* R16: stochastic rounding of v >= 0 on the E2M1 grid with one random byte. */
static int e2m1_mag_sr(float v, uint8_t byte) {
  if (v >= 6.0f) return 7;
  int lo = 0;
  for (int c = 0; c < 8; c++)
    if ((float)E2M1_GRID[c] <= v) lo = c;
  float glo = (float)E2M1_GRID[lo], ghi = (float)E2M1_GRID[lo + 1];
  float p = (v - glo) / (ghi - glo);           /* exact */
  float thresh = (float)(2 * (int)byte + 1);   /* exact */
  return ((OR_MUTANT == 8) ? (thresh <= 512.0f * p) : (thresh < 512.0f * p)) ? lo + 1 : lo; /* exact */
}

/* ------------------------------------------------------------------ */
/* Block quantizers                                                     */
/* ------------------------------------------------------------------ */

/* One NVFP4 block of n = 16 (1x16) or n = 256 (16x16 tile, row-major, the
 * error being a per-row tree then a tree over the 16 row sums).
 * g[i] is the global source index of w[i] (used only for SR).
 * Returns the chosen scale code; *pick4 = 1 when the 4-candidate won. */
static uint8_t nvfp4_block(const float* w, const int64_t* g, int n, float S_t,
                           const or_opts* o, uint8_t* codes, int* pick4) {
  float a = 0.0f;
  for (int i = 0; i < n; i++) a = fmaxf(a, fabsf(w[i]));
  uint8_t s6, s4;
  candidate_scales(a, S_t, o->fmt, &s6, &s4);

  uint8_t c6[256], c4[256];
  float t6[256], t4[256];
  float err6, err4;
  candidate_rne(w, n, s6, S_t, c6, t6);
  if (n == 16) {
    err6 = tree_sum(t6, 16);
  } else {
    float rs[16];
    for (int r = 0; r < 16; r++) rs[r] = tree_sum(t6 + 16 * r, 16);
    err6 = tree_sum(rs, 16);
  }
  int choose4 = 0;
  if (o->fmt == OR_FMT_NVFP4_46) {
    candidate_rne(w, n, s4, S_t, c4, t4);
    if (n == 16) {
      err4 = tree_sum(t4, 16);
    } else {
      float rs[16];
      for (int r = 0; r < 16; r++) rs[r] = tree_sum(t4 + 16 * r, 16);
      err4 = tree_sum(rs, 16);
    }
    choose4 = (OR_MUTANT == 1) ? (err4 <= err6) : (err4 < err6); /* R7: strictly lower wins */
  }
  uint8_t s = choose4 ? s4 : s6;
  const uint8_t* cc = choose4 ? c4 : c6;
  if (o->rnd == OR_RND_SR) { /* R13: SR re-rounds the chosen candidate */
    float e, inv;
    effective_scale(s, S_t, &e, &inv);
    for (int i = 0; i < n; i++) {
      float v = fabsf(w[i]) * inv;
      int mag = e2m1_mag_sr(v, sr_byte(o->seed, g[i]));
      codes[i] = (uint8_t)(mag | (signbit(w[i]) ? 8 : 0));
    }
  } else {
    memcpy(codes, cc, (size_t)n);
  }
  *pick4 = choose4;
  return s;
}

/* One MXFP4 block of 32 values (R9). Returns the E8M0 scale byte. */
static uint8_t mxfp4_block(const float* w, uint8_t* codes) {
  float a = 0.0f;
  for (int i = 0; i < 32; i++) a = fmaxf(a, fabsf(w[i]));
  int E = or_e8m0_exponent(a);
  for (int i = 0; i < 32; i++) {
    double v = ldexp(fabs((double)w[i]), -E); /* exact power-of-two scaling */
    codes[i] = (uint8_t)(e2m1_mag_rne((double)(float)v) | (signbit(w[i]) ? 8 : 0));
  }
  return (uint8_t)(E + 127);
}

static void put_nibble(uint8_t* buf, int64_t idx, uint8_t code) {
  uint8_t* p = buf + (idx >> 1);
  if (idx & 1) *p = (uint8_t)((*p & 0x0F) | (code << 4)); /* odd: high nibble */
  else         *p = (uint8_t)((*p & 0xF0) | (code & 0x0F)); /* even: low nibble */
}

static void set_bit(uint8_t* bits, int64_t b, int v) {
  if (!bits) return;
  if (v) bits[b >> 3] |= (uint8_t)(1u << (b & 7));
  else   bits[b >> 3] &= (uint8_t)~(1u << (b & 7));
}

/* ------------------------------------------------------------------ */
/* Tensor-level entry points                                            */
/* ------------------------------------------------------------------ */

/* Amax of |RHT16| over the 16-row column blocks of one entry: the tensor
 * amax the colwise copy takes when its blocks are transformed along rows. */
static float amax_cols_rht(const uint16_t* xb, int64_t rows, int64_t cols, uint32_t mask) {
  float a = 0.0f;
  for (int64_t c = 0; c < cols; c++)
    for (int64_t rb = 0; rb < rows / 16; rb++) {
      float w[16];
      for (int i = 0; i < 16; i++) w[i] = or_bf16_to_f32(xb[(rb * 16 + i) * cols + c]);
      if (OR_MUTANT != 20) or_rht16(w, mask);
      for (int i = 0; i < 16; i++) a = fmaxf(a, fabsf(w[i]));
    }
  return a;
}

/* Per-batch-entry amax of |x| (of the RHT output when rht != 0).
 * Returns OR_NONFINITE if any input is NaN or infinite (R18). */
int or_amax(const uint16_t* x, int64_t batch, int64_t rows, int64_t cols,
            int rht, uint64_t seed, float* amax) {
  uint32_t mask = or_rht16_signs(seed);
  for (int64_t b = 0; b < batch; b++) {
    float a = 0.0f;
    const uint16_t* xb = x + b * rows * cols;
    for (int64_t i = 0; i < rows * cols; i += 16) {
      float w[16];
      for (int j = 0; j < 16; j++) {
        w[j] = or_bf16_to_f32(xb[i + j]);
        if (!isfinite(w[j])) return OR_NONFINITE;
      }
      if (rht) or_rht16(w, mask);
      for (int j = 0; j < 16; j++) a = fmaxf(a, fabsf(w[j]));
    }
    amax[b] = a;
  }
  return OR_OK;
}

/* Quantize x [batch, rows, cols] (bf16 bits, contiguous).
 * Outputs (all contiguous, caller-allocated, NULL to skip):
 *   r_codes  [batch, rows, cols/2]  packed E2M1, element 2k in the low nibble
 *   r_scales [batch, rows, cols/bs] E4M3 (NVFP4) or E8M0 (MXFP4); in 16x16
 *            mode each tile's scale is repeated in its 16 rows
 *   r_choice bitmap, bit b = 1 when block b (linear index) chose 4
 *   c_codes  [batch, cols, rows/2]  colwise 1x16 (or the 16x16 transpose)
 *   c_scales [batch, cols, rows/16]
 *   c_choice bitmap over the colwise copy's blocks (1x16), or over the
 *            transposed copy's 16x16 tiles in its own tile row-major order
 *   tensor_scale [batch]  (NVFP4)
 *   c_tensor_scale [batch] (nullable) the colwise copy's S_t: the same as
 *            tensor_scale, except with rht_col, where the colwise blocks are
 *            transformed along rows and take the amax of the transformed
 *            columns (R21)
 * amax_in (nullable) gives the per-batch amax instead of computing it (with
 * rht_col it sets the rowwise S_t only). */
int or_quantize(const uint16_t* x, int64_t batch, int64_t rows, int64_t cols,
                const or_opts* o, const float* amax_in,
                uint8_t* r_codes, uint8_t* r_scales, uint8_t* r_choice,
                uint8_t* c_codes, uint8_t* c_scales, uint8_t* c_choice,
                float* tensor_scale, float* c_tensor_scale) {
  int mx = o->fmt == OR_FMT_MXFP4;
  if (mx != (o->blk == OR_BLK_1X32)) return OR_UNSUPPORTED;
  if (mx && (o->rnd != OR_RND_RNE || o->rht || c_codes)) return OR_UNSUPPORTED;
  if (o->rht && (o->blk != OR_BLK_1X16 || c_codes)) return OR_UNSUPPORTED;
  if (o->rht_col && (mx || o->blk != OR_BLK_1X16 || !(c_codes || c_scales))) return OR_UNSUPPORTED;
  int64_t bs = mx ? 32 : 16;
  if (cols % bs) return OR_SHAPE;
  if ((c_codes || o->blk == OR_BLK_16X16) && rows % 16) return OR_SHAPE;
  if (o->rnd == OR_RND_SR && (o->elem_offset & 15)) return OR_SHAPE;

  int64_t n = rows * cols;
  for (int64_t i = 0; i < batch * n; i++)
    if (!isfinite(or_bf16_to_f32(x[i]))) return OR_NONFINITE;

  uint32_t mask = or_rht16_signs(o->seed);
  for (int64_t b = 0; b < batch; b++) {
    const uint16_t* xb = x + b * n;
    if (mx) {
      for (int64_t r = 0; r < rows; r++)
        for (int64_t cb = 0; cb < cols / 32; cb++) {
          float w[32];
          uint8_t codes[32];
          for (int j = 0; j < 32; j++) w[j] = or_bf16_to_f32(xb[r * cols + cb * 32 + j]);
          uint8_t s = mxfp4_block(w, codes);
          if (r_scales) r_scales[(b * rows + r) * (cols / 32) + cb] = s;
          if (r_codes)
            for (int j = 0; j < 32; j++)
              put_nibble(r_codes, (b * rows + r) * cols + cb * 32 + j, codes[j]);
        }
      continue;
    }
    float A;
    if (amax_in) {
      A = amax_in[b];
    } else {
      int st = or_amax(xb, 1, rows, cols, o->rht, o->seed, &A);
      if (st) return st;
    }
    float S_t = or_tensor_scale(A, o->fmt);
    if (tensor_scale) tensor_scale[b] = S_t;
    float S_tc = o->rht_col ? or_tensor_scale(amax_cols_rht(xb, rows, cols, mask), o->fmt) : S_t;
    if (c_tensor_scale) c_tensor_scale[b] = S_tc;
    int64_t base = o->elem_offset + b * n; /* global index of x[b,0,0] */

    if (o->blk == OR_BLK_1X16) {
      for (int64_t r = 0; r < rows; r++)
        for (int64_t cb = 0; cb < cols / 16; cb++) {
          float w[16];
          int64_t g[16];
          uint8_t codes[16];
          int p4;
          for (int j = 0; j < 16; j++) {
            w[j] = or_bf16_to_f32(xb[r * cols + cb * 16 + j]);
            g[j] = base + r * cols + cb * 16 + j;
          }
          if (o->rht) or_rht16(w, mask);
          uint8_t s = nvfp4_block(w, g, 16, S_t, o, codes, &p4);
          int64_t blk = (b * rows + r) * (cols / 16) + cb;
          if (r_scales) r_scales[blk] = s;
          set_bit(r_choice, blk, p4);
          if (r_codes)
            for (int j = 0; j < 16; j++)
              put_nibble(r_codes, (b * rows + r) * cols + cb * 16 + j, codes[j]);
        }
      if (c_codes || c_scales) /* R12: colwise = independent 1x16 along rows; R21: RHT */
        for (int64_t c = 0; c < cols; c++)
          for (int64_t rb = 0; rb < rows / 16; rb++) {
            float w[16];
            int64_t g[16];
            uint8_t codes[16];
            int p4;
            for (int i = 0; i < 16; i++) {
              w[i] = or_bf16_to_f32(xb[(rb * 16 + i) * cols + c]);
              g[i] = base + (rb * 16 + i) * cols + c;
            }
            if (o->rht_col) or_rht16(w, mask);
            uint8_t s = nvfp4_block(w, g, 16, S_tc, o, codes, &p4);
            int64_t blk = (b * cols + c) * (rows / 16) + rb;
            if (c_scales) c_scales[blk] = s;
            set_bit(c_choice, blk, p4);
            if (c_codes)
              for (int i = 0; i < 16; i++)
                put_nibble(c_codes, (b * cols + c) * rows + rb * 16 + i, codes[i]);
          }
    } else { /* R11: 16x16 tiles, one scale and one choice per tile */
      for (int64_t tr = 0; tr < rows / 16; tr++)
        for (int64_t tc = 0; tc < cols / 16; tc++) {
          float w[256];
          int64_t g[256];
          uint8_t codes[256];
          int p4;
          for (int i = 0; i < 16; i++)
            for (int j = 0; j < 16; j++) {
              int64_t r = tr * 16 + i, c = tc * 16 + j;
              w[i * 16 + j] = or_bf16_to_f32(xb[r * cols + c]);
              g[i * 16 + j] = base + r * cols + c;
            }
          uint8_t s = nvfp4_block(w, g, 256, S_t, o, codes, &p4);
          /* R7: one bit per tile, in tile row-major order over each copy's
           * own [R][C]: the rowwise copy is x ([rows][cols]), the transposed
           * copy is x^T ([cols][rows]), where source tile (tr, tc) sits at
           * tile row tc, tile column tr. */
          set_bit(r_choice, (b * (rows / 16) + tr) * (cols / 16) + tc, p4);
          if (OR_MUTANT == 19) /* the transposed copy indexed like the source */
            set_bit(c_choice, (b * (rows / 16) + tr) * (cols / 16) + tc, p4);
          else
            set_bit(c_choice, (b * (cols / 16) + tc) * (rows / 16) + tr, p4);
          for (int i = 0; i < 16; i++) {
            int64_t r = tr * 16 + i;
            if (r_scales) r_scales[(b * rows + r) * (cols / 16) + tc] = s;
            for (int j = 0; j < 16; j++) {
              int64_t c = tc * 16 + j;
              if (r_codes) put_nibble(r_codes, (b * rows + r) * cols + c, codes[i * 16 + j]);
              if (c_codes) put_nibble(c_codes, (b * cols + c) * rows + r, codes[i * 16 + j]);
            }
          }
          if (c_scales)
            for (int j = 0; j < 16; j++)
              c_scales[(b * cols + tc * 16 + j) * (rows / 16) + tr] = s;
        }
    }
  }
  return OR_OK;
}

/* Dequantize codes [batch, rows, cols/2] with scales [batch, rows, cols/bs]
 * to bf16 bits y [batch, rows, cols].
 * NVFP4 (R17): y = bf16_rne((sign*q * float(s)) * S_t), first product exact.
 * MXFP4: y = bf16(sign*q * 2^(scale-127)), exact. */
int or_dequantize(const uint8_t* codes, const uint8_t* scales, const float* tensor_scale,
                  int64_t batch, int64_t rows, int64_t cols, int fmt, uint16_t* y) {
  int64_t bs = (fmt == OR_FMT_MXFP4) ? 32 : 16;
  if (cols % bs) return OR_SHAPE;
  for (int64_t b = 0; b < batch; b++)
    for (int64_t r = 0; r < rows; r++)
      for (int64_t c = 0; c < cols; c++) {
        int64_t idx = (b * rows + r) * cols + c;
        uint8_t byte = codes[idx >> 1];
        uint8_t code = (idx & 1) ? (byte >> 4) : (byte & 15);
        float sq = or_e2m1_decode(code);
        uint8_t s = scales[(b * rows + r) * (cols / bs) + c / bs];
        float out;
        if (fmt == OR_FMT_MXFP4) {
          out = (float)ldexp((double)sq, (int)s - 127);
        } else {
          float p = sq * or_e4m3_decode(s);
          out = p * (OR_MUTANT == 10 ? 1.0f : tensor_scale[b]);
        }
        y[idx] = or_f32_to_bf16(out);
      }
  return OR_OK;
}

/* R19: byte offset of scale (r, c) of a [rows, sf_cols] scale matrix in the
 * block-scaled tensor-core layout: 128x4 tiles of 512 bytes, tiles row-major
 * over (row tile, column tile), inside a tile row r%32 selects a 16-byte
 * group, (r%128)/32 a 4-byte word in it and c%4 the byte. */
int64_t or_swizzle_offset(int64_t r, int64_t c, int64_t sf_cols) {
  int64_t col_tiles = (sf_cols + 3) / 4;
  int64_t tile = (r / 128) * col_tiles + c / 4;
  return tile * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4 + (c % 4);
}

int64_t or_swizzled_size(int64_t rows, int64_t sf_cols) {
  return ((rows + 127) / 128) * 128 * ((sf_cols + 3) / 4) * 4;
}

/* Permute a linear [batch, rows, sf_cols] scale array into the swizzled
 * layout; each batch entry occupies or_swizzled_size bytes; padding is 0. */
void or_swizzle_scales(const uint8_t* lin, int64_t batch, int64_t rows, int64_t sf_cols,
                       uint8_t* out) {
  int64_t per = or_swizzled_size(rows, sf_cols);
  memset(out, 0, (size_t)(per * batch));
  for (int64_t b = 0; b < batch; b++)
    for (int64_t r = 0; r < rows; r++)
      for (int64_t c = 0; c < sf_cols; c++)
        out[b * per + or_swizzle_offset(r, c, sf_cols)] = lin[(b * rows + r) * sf_cols + c];
}

/* ------------------------------------------------------------------ */
/* Worked-example mode ([FP4] "Como funciona FP4", R20)                 */
/* fp32 input, scale = block amax / 6 in fp32 (no E4M3), nearest grid    */
/* value with ties to the lower index, dequantized = grid*sign*scale.    */
/* Returns the mean absolute error (accumulated in binary64).           */
/* ------------------------------------------------------------------ */

double or_page_example_mae(const float* x, int64_t n, int64_t block) {
  double acc = 0.0;
  for (int64_t b0 = 0; b0 < n; b0 += block) {
    float a = 0.0f;
    for (int64_t i = 0; i < block; i++) a = fmaxf(a, fabsf(x[b0 + i]));
    float scale = a / 6.0f;
    for (int64_t i = 0; i < block; i++) {
      float xi = x[b0 + i];
      float r = fabsf(xi) / scale;
      int best = 0;
      float bd = fabsf(r - (float)E2M1_GRID[0]);
      for (int c = 1; c < 8; c++) {
        float d = fabsf(r - (float)E2M1_GRID[c]);
        if (d < bd) { /* strict: ties keep the lower index */
          best = c;
          bd = d;
        }
      }
      float sgn = (xi > 0.0f) ? 1.0f : ((xi < 0.0f) ? -1.0f : 0.0f);
      float deq = (float)E2M1_GRID[best] * sgn * scale;
      acc += fabs((double)deq - (double)xi);
    }
  }
  return acc / (double)n;
}

/* ------------------------------------------------------------------ */
/* Array helpers used by the pin tests                                  */
/* ------------------------------------------------------------------ */

void or_e2m1_encode_array(const float* v, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; i++) out[i] = or_e2m1_encode(v[i]);
}

void or_e4m3_encode_array(const float* v, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; i++) out[i] = or_e4m3_encode(v[i]);
}

void or_e8m0_exponent_array(const float* v, int64_t n, int32_t* out) {
  for (int64_t i = 0; i < n; i++) out[i] = or_e8m0_exponent(v[i]);
}

void or_f32_to_bf16_array(const float* v, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; i++) out[i] = or_f32_to_bf16(v[i]);
}

void or_philox_array(const uint32_t* ctr, const uint32_t* key, int64_t n, uint32_t* out) {
  for (int64_t i = 0; i < n; i++) or_philox4x32_10(ctr + 4 * i, key + 2 * i, out + 4 * i);
}

/* Per-element SR magnitude for tests: v >= 0, one byte each. */
void or_e2m1_sr_array(const float* v, const uint8_t* bytes, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; i++) out[i] = (uint8_t)e2m1_mag_sr(v[i], bytes[i]);
}

void or_sr_bytes(uint64_t seed, const int64_t* g, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; i++) out[i] = sr_byte(seed, g[i]);
}

void or_rht16_rows(float* x, int64_t nblocks, uint64_t seed) {
  uint32_t mask = or_rht16_signs(seed);
  for (int64_t b = 0; b < nblocks; b++) or_rht16(x + 16 * b, mask);
}
