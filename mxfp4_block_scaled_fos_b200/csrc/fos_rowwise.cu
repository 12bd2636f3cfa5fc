// fos_rowwise.cu -- per-tensor amax pass and the rowwise 1x16 NVFP4 (4/6 and
// 6-only) quantizer for sm_100a.
//
// Method: Hugging Face transformers doc "Four Over Six", introduction (each
// NVFP4 block scaled so its max maps to 4 or to 6, the lower-error candidate
// kept); Ultralytics glossary "FP4", "Como funciona FP4" (NVFP4: 16 values,
// E4M3 block scale, FP32 per-tensor scale) and introduction (E2M1 values).
// Options from the "Four Over Six" usage section: random Hadamard transform
// and stochastic rounding.
//
// Design: one 16-element block per thread per step, loaded with one 256-bit
// load and carried as 8 packed f32x2 pairs, so that the scaling, the error
// fma, the squares and the error tree of a block run as sm_100 f32x2
// instructions.  A warp covers 32 consecutive blocks: 1 KB of contiguous
// input, 256 contiguous code bytes, 32 scale bytes and one 32-bit word of the
// 4/6 choice bitmap (a ballot).
#include <atomic>

#include "fos_core.cuh"

namespace fos {

namespace {

constexpr int kThreads = 256;
// Resident CTAs per SM the rowwise quantizer (k_q1x16) is compiled for (the
// register cap).  Its dense loop loads the next group's block one iteration
// ahead (FOS_K1_PREFETCH), which needs the registers of 4 CTAs per SM: 0.595
// ms against 0.618 ms (5 CTAs, no prefetch) on the 128-expert 4/6 batch.
#ifndef FOS_K1_MIN_BLOCKS
#define FOS_K1_MIN_BLOCKS 4
#endif
#ifndef FOS_K1_PREFETCH
#define FOS_K1_PREFETCH 1
#endif
// the fused amax + quantize kernel: the threads of 5 such CTAs per SM, no
// prefetch (its amax items want the CTAs; 0.729 ms against 0.747 ms with 4
// CTAs and prefetch)
#ifndef FOS_FUSED_MIN_BLOCKS
#define FOS_FUSED_MIN_BLOCKS 5
#endif
// the stochastic-rounding and Hadamard variants of both (more registers)
#ifndef FOS_K1_MIN_BLOCKS_HEAVY
#define FOS_K1_MIN_BLOCKS_HEAVY 4
#endif

// --------------------------------------------------------------------------
// K0: per-batch-entry amax of |x| (or of the RHT of x).
// grid (chunks, batch); each thread handles pairs of blocks.
template <bool RHT>
__global__ void __launch_bounds__(kThreads) k_amax(const QuantArgs a, uint32_t* amax_ws) {
  const int b = blockIdx.y;
  const uint32_t nunit = (a.nblk + 1) / 2;
  const uint32_t u0 = blockIdx.x * a.units_per_cta;
  const uint32_t u1 = min(u0 + a.units_per_cta, nunit);
  uint32_t mask16 = 0;
  if (RHT) mask16 = rht_sign_mask(a.seed);
  uint32_t m = 0;
  for (uint32_t u = u0 + threadIdx.x; u < u1; u += kThreads) {
    const uint32_t j0 = 2 * u;
    const bool has1 = j0 + 1 < a.nblk;
    uint4 wa[2], wb[2];
    load_block(a, b, j0, wa);
    if (has1) load_block(a, b, j0 + 1, wb);
    else      { wb[0] = wa[0]; wb[1] = wa[1]; }
    if (RHT) {
      rht_flip_signs(wa, mask16);
      rht_flip_signs(wb, mask16);
      float2 P[16];
      unpack_pairs(wa, wb, P);
      fwht16_pairs(P);
      uint32_t ma, mb;
      amax_bits_pairs(P, ma, mb);
      m = max(m, max(ma, mb));
    } else {
      m = max(m, max(amax_bits_bf16(wa), amax_bits_bf16(wb)));
    }
  }
  m = __reduce_max_sync(0xffffffffu, m);
  __shared__ uint32_t s_m[kThreads / 32];
  if ((threadIdx.x & 31) == 0) s_m[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    uint32_t v = threadIdx.x < kThreads / 32 ? s_m[threadIdx.x] : 0u;
    v = __reduce_max_sync(0xffffffffu, v);
    if (threadIdx.x == 0) {
      if (v >= 0x7f800000u) {
        if (a.status) atomicOr(a.status, FOS_STATUS_NONFINITE);
      } else {
        atomicMax(amax_ws + b, v);
      }
    }
  }
}

// --------------------------------------------------------------------------
// K1: rowwise 1x16 NVFP4 quantizer.  grid (chunks, batch).
// One block per thread per step: lane l of warp w takes block g + l, so a
// warp reads 1 KB of contiguous input per step, writes 256 contiguous code
// bytes and 32 scale bytes, and its ballot of 4/6 picks is one 32-bit word
// of the choice bitmap.  The block is carried as 8 split pairs
// (w_k, w_k+8): bf16 words unpack into them, E2M1 codes pack and decode from
// them without moves, and the contiguous error tree adds neighbouring pairs
// with f32x2 adds down to its last level.
// DENSE: rows are contiguous (ld == cols) and the outputs are packed
// (codes_ld == cols/2, linear scales with scales_ld == cols/16), so block j
// sits at element 16j, code byte 8j and scale byte j; x is 32-byte aligned
// and each block is one 256-bit load.
// pol != 0: L2 eviction policy for the dense 256-bit load (0: default)
template <bool DENSE>
__device__ __forceinline__ void k1_load(const QuantArgs& a, int b, uint32_t j, bool v, uint4 (&w)[2],
                                        unsigned long long pol = 0) {
  if (!v) {
    w[0] = w[1] = make_uint4(0u, 0u, 0u, 0u);
    return;
  }
  if (DENSE) {
    const uint16_t* p = a.x + (long long)b * a.x_bs + (long long)j * 16;
    if (pol) ld_block256_hint(p, pol, w);
    else     ld_block256(p, w);
  } else {
    load_block(a, b, j, w);
  }
}

template <bool SWZ, bool DENSE>
__device__ __forceinline__ void k1_store(const QuantArgs& a, int b, uint32_t j, const uint32_t (&codes)[2],
                                         uint32_t scale) {
  if (DENSE) {
    *reinterpret_cast<uint2*>(a.row.codes + (long long)b * a.row.codes_bs + (long long)j * 8) =
        make_uint2(codes[0], codes[1]);
    a.row.scales[(long long)b * a.row.scales_bs + j] = (uint8_t)scale;
  } else {
    store_block<SWZ>(a.row, b, j, a.bpr, codes, scale);
  }
}

__device__ __forceinline__ void store_choice32(const OutDesc& o, unsigned long long gbit, uint32_t word) {
  unsigned int* base = reinterpret_cast<unsigned int*>(o.choice);
  if (o.choice_aligned) {
    base[gbit >> 5] = word;
  } else if (word) {
    // only words that receive a set bit are touched
    const int sh = (int)(gbit & 31);
    const unsigned long long vv = (unsigned long long)word << sh;
    if ((uint32_t)vv) atomicOr(base + (gbit >> 5), (uint32_t)vv);
    if ((uint32_t)(vv >> 32)) atomicOr(base + (gbit >> 5) + 1, (uint32_t)(vv >> 32));
  }
}

// The per-block 4/6 step of the rowwise quantizer: w (8 bf16x2 words of one
// block) -> codes, scale byte, 4-picked flag.  FAST: the tensor scale's
// division shortcut applies (known at compile time).
template <bool F46, bool SR, bool RHT, int FAST>
__device__ __forceinline__ void rowwise_block(uint4 (&w)[2], const float4* s_tab, const TScale& ts,
                                              uint32_t mask16, float nz, unsigned long long seed,
                                              long long e0, uint32_t& bad, uint32_t (&codes)[2],
                                              uint32_t& sc, bool& pick) {
  if (RHT) {
    rht_flip_signs(w, mask16);
  }
  const uint32_t W[8] = {w[0].x, w[0].y, w[0].z, w[0].w, w[1].x, w[1].y, w[1].z, w[1].w};
  float2 P[8];
  unpack_split(W, P);
  uint32_t m;
  if (RHT) {
    fwht16_split(P);
    m = amax_bits_split(P);
  } else {
    m = amax_bits_bf16(w);
  }
  bad = max(bad, m);  // largest amax bits seen: >= 0x7f800000 means NaN/Inf
  uint32_t s6, s4;
  cand_scales<F46, FAST>(__uint_as_float(m), ts, s6, s4);
  const float4 t6 = s_tab[s6];
  const Cand1 c6 = candidate1_t<F46>(P, t6, nz);
  codes[0] = c6.c[0];
  codes[1] = c6.c[1];
  sc = s6;
  float inv = t6.x;
  pick = false;
  if (F46) {
    const float4 t4 = s_tab[s4];
    const Cand1 c4 = candidate1_t<true>(P, t4, nz);
    pick = c4.err < c6.err;   // strictly lower wins; ties keep 6
    if (pick) { codes[0] = c4.c[0]; codes[1] = c4.c[1]; sc = s4; inv = t4.x; }
  }
  if (SR) sr_block1(P, inv, sr_bytes16(seed, e0), codes);
}

// Dense rows (see k1_load): blocks [c0, c1) of entry b.  Whole warp groups
// of 32 blocks run without tail checks: the lane's input, code and scale
// addresses are 32-bit offsets from per-entry base pointers, every store is
// unconditional and the 4/6 choice word is one ballot stored by lane 0.  A
// partial last group (c1 - g < 32) runs once with a branch-free tail (a lane
// past c1 recomputes block c1 - 1 and stores nothing).  With choice bits the
// bitmap words must belong to one warp each (blocks per entry % 64 == 0,
// c0 % 32 == 0).
template <bool F46, bool SR, bool RHT, int FAST, int NT = kThreads, bool FAKE = false, bool PF = false>
__device__ __forceinline__ void rowwise_dense(const QuantArgs& a, int b, uint32_t c0, uint32_t c1,
                                              const float4* s_tab, const TScale& ts, uint32_t mask16,
                                              uint32_t& bad, unsigned long long pol) {
  const uint32_t lane = threadIdx.x & 31;
  const uint16_t* xb = a.x + (long long)b * a.x_bs;
  uint8_t* cb = a.row.codes + (long long)b * a.row.codes_bs;
  uint8_t* sb = a.row.scales + (long long)b * a.row.scales_bs;
  uint32_t* chw = (!FAKE && a.row.choice)
                      ? reinterpret_cast<uint32_t*>(a.row.choice) + (((unsigned long long)b * a.nblk) >> 5)
                      : nullptr;
  const long long g0 = SR ? a.elem_offset + (long long)b * a.x_bs : 0;
  const float nz = a.neg_zero;
  const unsigned long long seed = a.seed;
  uint32_t g = c0 + 32 * (NT == 32 ? 0u : (threadIdx.x >> 5));  // uniform per warp
  uint4 wn[2];  // PF: the next group's block, loaded one iteration ahead
  if (PF && g + 32 <= c1) ld_block256_hint(xb + (size_t)(g + lane) * 16, pol, wn);
#pragma unroll 1
  for (; g + 32 <= c1; g += NT) {
    const uint32_t j = g + lane;
    uint4 w[2];
    if (PF) {
      w[0] = wn[0];
      w[1] = wn[1];
      if (g + NT + 32 <= c1) ld_block256_hint(xb + (size_t)(j + NT) * 16, pol, wn);
    } else {
      ld_block256_hint(xb + (size_t)j * 16, pol, w);
    }
    uint32_t codes[2], sc;
    bool pick;
    rowwise_block<F46, SR, RHT, FAST>(w, s_tab, ts, mask16, nz, seed, g0 + (long long)j * 16, bad, codes,
                                      sc, pick);
    if (FAKE) {
      store_fake_block<true>(a, b, j, codes, e4m3_to_f32(sc), ts.St);
    } else {
      *reinterpret_cast<uint2*>(cb + (size_t)j * 8) = make_uint2(codes[0], codes[1]);
      sb[j] = (uint8_t)sc;
      if (F46 && chw) {
        const uint32_t word = __ballot_sync(0xffffffffu, pick);
        if (lane == 0) chw[g >> 5] = word;
      }
    }
  }
  if (g < c1) {  // the partial last group
    const uint32_t j = g + lane;
    const bool valid = j < c1;
    const uint32_t jj = valid ? j : c1 - 1;
    uint4 w[2];
    ld_block256_hint(xb + (size_t)jj * 16, pol, w);
    uint32_t codes[2], sc;
    bool pick;
    rowwise_block<F46, SR, RHT, FAST>(w, s_tab, ts, mask16, nz, seed, g0 + (long long)jj * 16, bad,
                                      codes, sc, pick);
    if (FAKE) {
      if (valid) store_fake_block<true>(a, b, j, codes, e4m3_to_f32(sc), ts.St);
    } else {
      if (valid) {
        *reinterpret_cast<uint2*>(cb + (size_t)j * 8) = make_uint2(codes[0], codes[1]);
        sb[j] = (uint8_t)sc;
      }
      if (F46 && chw) {
        const uint32_t word = __ballot_sync(0xffffffffu, pick && valid);
        if (lane == 0) chw[g >> 5] = word;
      }
    }
  }
}

// Quantize blocks [c0, c1) of batch entry b with a group of NT threads (the
// CTA, or with NT = 32 one warp): lane l of warp w takes block g + l for
// g = c0 + 32w, c0 + 32w + NT, ...  c0 must be a multiple of 32 so that each
// 32-bit word of the choice bitmap belongs to one warp.
template <bool F46, bool SR, bool RHT, bool SWZ, bool DENSE, int NT = kThreads, bool FAKE = false, bool PF = false>
__device__ __forceinline__ void rowwise_range(const QuantArgs& a, int b, uint32_t c0, uint32_t c1,
                                              const float4* s_tab, const TScale& ts, uint32_t mask16,
                                              uint32_t& bad, unsigned long long pol) {
  if (DENSE) {
    if (ts.fast) rowwise_dense<F46, SR, RHT, 1, NT, FAKE, PF>(a, b, c0, c1, s_tab, ts, mask16, bad, pol);
    else         rowwise_dense<F46, SR, RHT, 0, NT, FAKE, PF>(a, b, c0, c1, s_tab, ts, mask16, bad, pol);
    return;
  }
  const int lane = threadIdx.x & 31;
  for (uint32_t g = c0 + 32 * (NT == 32 ? 0u : (threadIdx.x >> 5)); g < c1; g += NT) {  // uniform per warp
    const uint32_t j = g + lane;
    const bool valid = j < c1;
    uint4 w[2];
    k1_load<DENSE>(a, b, j, valid, w, pol);
    uint32_t pick = 0;
    {  // computed for every lane (a missing block reads as zeros); only stores are predicated
      if (RHT) {
        rht_flip_signs(w, mask16);
      }
      const uint32_t W[8] = {w[0].x, w[0].y, w[0].z, w[0].w, w[1].x, w[1].y, w[1].z, w[1].w};
      float2 P[8];
      unpack_split(W, P);
      uint32_t m;
      if (RHT) {
        fwht16_split(P);
        m = amax_bits_split(P);
      } else {
        m = amax_bits_bf16(w);
      }
      bad = max(bad, m);  // largest amax bits seen: >= 0x7f800000 means NaN/Inf
      uint32_t s6, s4;
      cand_scales<F46>(__uint_as_float(m), ts, s6, s4);
      const float4 t6 = s_tab[s6];
      const Cand1 c6 = candidate1_t<F46>(P, t6, a.neg_zero);
      uint32_t codes[2] = {c6.c[0], c6.c[1]};
      uint32_t sc = s6;
      float inv = t6.x;
      if (F46) {
        const float4 t4 = s_tab[s4];
        const Cand1 c4 = candidate1_t<true>(P, t4, a.neg_zero);
        pick = valid && (c4.err < c6.err);   // strictly lower wins; ties keep 6
        if (pick) { codes[0] = c4.c[0]; codes[1] = c4.c[1]; sc = s4; inv = t4.x; }
      }
      if (SR) {
        const long long g0 = a.elem_offset + (long long)b * a.rows * a.cols;
        long long e0;
        if (DENSE) {
          e0 = g0 + (long long)j * 16;
        } else {
          const uint32_t row = fdiv(j, a.bpr), cb = j - row * a.bpr.d;
          e0 = g0 + (long long)row * a.cols + cb * 16;
        }
        sr_block1(P, inv, sr_bytes16(a.seed, e0), codes);
      }
      if (FAKE) {
        if (valid) store_fake_block<false>(a, b, j, codes, e4m3_to_f32(sc), ts.St);
      } else if (valid) {
        k1_store<SWZ, DENSE>(a, b, j, codes, sc);
      }
    }
    if (!FAKE && F46 && a.row.choice) {
      const uint32_t word = __ballot_sync(0xffffffffu, pick);
      if (lane == 0) store_choice32(a.row, (unsigned long long)b * a.nblk + g, word);
    }
  }
}

template <bool F46, bool SR, bool RHT, bool SWZ, bool DENSE, bool FAKE>
__global__ void __launch_bounds__(kThreads, (SR || RHT) ? FOS_K1_MIN_BLOCKS_HEAVY : FOS_K1_MIN_BLOCKS)
    k_q1x16(const QuantArgs a) {
  __shared__ float4 s_tab[128];
  const int b = blockIdx.y;
  const float St = tensor_scale_of(a, b, F46);
  build_scale_table4(s_tab, St);
  const TScale ts = make_tscale(St);
  if (blockIdx.x == 0 && threadIdx.x == 0 && a.row.tensor_scale) a.row.tensor_scale[b] = St;
  uint32_t mask16 = 0;
  if (RHT) mask16 = rht_sign_mask(a.seed);
  __syncthreads();
  const uint32_t c0 = blockIdx.x * a.units_per_cta;
  const uint32_t c1 = min(c0 + a.units_per_cta, a.nblk);
  if (DENSE && threadIdx.x < 32) {   // the CTA's input into L2 up front (bulk prefetch)
    const uint32_t nbytes = (c1 - c0) * 32u, off = threadIdx.x * 16384u;
    if (off < nbytes)
      prefetch_l2(a.x + (long long)b * a.x_bs + (long long)c0 * 16 + off / 2, min(16384u, nbytes - off),
                  l2_policy_evict_first());
  }
  uint32_t bad = 0;
  rowwise_range<F46, SR, RHT, SWZ, DENSE, kThreads, FAKE, FOS_K1_PREFETCH != 0>(a, b, c0, c1, s_tab, ts, mask16, bad,
                                                          DENSE ? l2_policy_evict_first() : 0ull);
  if (bad >= 0x7f800000u && a.status) atomicOr(a.status, FOS_STATUS_NONFINITE);
}

// --------------------------------------------------------------------------
// Fused amax + rowwise quantize for a batch of tensors with one S_t each
// (e.g. the experts of an MoE layer), as one persistent launch fed by a work
// queue.  The queue is a fixed sequence of items: phase p holds the amax
// chunks of entry p (if p < batch) followed by the quantize chunks of entry
// p - L (L = min(lag, batch)).  CTAs claim items in sequence order with one
// atomic counter.  An amax item reduces its chunk and counts in on done_a[entry]; a
// quantize item first waits until every amax chunk of its entry has counted
// in, then quantizes its chunk with that entry's S_t.  Every item an item
// waits on precedes it in the sequence and was claimed by a running CTA
// that never waits on a later item, so the queue needs no co-residency and
// cannot deadlock; the wait is bounded anyway (about a second, then
// FOS_STATUS_TIMEOUT).  Memory-bound amax chunks and compute-bound quantize
// chunks run side by side on every SM, and with the L + 1 entries in flight
// smaller than L2 (and the amax reads marked evict-last) the quantize reads
// hit L2, so HBM sees the input about once.
// Lag in entries between an entry's amax and its quantize items: measured on
// the 128 x 2880 x 2880 expert batch (lag 2, claims at item end: 0.738 ms for
// 4/6 against 0.781 ms for lag 3 with claim-ahead).
#ifndef FOS_FUSED_LAG_46
#define FOS_FUSED_LAG_46 2
#endif
#ifndef FOS_FUSED_LAG_6
#define FOS_FUSED_LAG_6 2
#endif
#ifndef FOS_FUSED_AMAX_UNROLL
#define FOS_FUSED_AMAX_UNROLL 4
#endif
// 1: a CTA claims its next item when it starts an item (the claim's latency
// hides behind the item, but twice as many items are in flight, so an entry's
// quantize items reach the queue head while its amax items are still being
// reduced unless the lag grows); 0: when it ends one
#ifndef FOS_FUSED_CLAIM_AHEAD
#define FOS_FUSED_CLAIM_AHEAD 0
#endif
// Threads per CTA and item sizes in blocks (amax, quantize) per variant.  The
// plain 4/6 kernel (round to nearest, codes out), bound by instruction issue,
// runs 128-thread CTAs so that the barrier at each item end waits on 4 warps,
// not 8: 0.722 ms against 0.729 ms (256 threads, items of 4096 / 2048 blocks)
// on the expert batch.  The others keep 256 threads: the 6-only kernel, bound
// by memory (0.472 ms against 0.481 ms with 128), and the fake-quantizing and
// Hadamard 4/6 kernels (0.872 against 0.907 ms, 0.048 against 0.052 ms).
#ifndef FOS_FUSED_SMALL_THREADS
#define FOS_FUSED_SMALL_THREADS 128
#endif
#ifndef FOS_FUSED_SMALL_ACHUNK
#define FOS_FUSED_SMALL_ACHUNK 2048
#endif
#ifndef FOS_FUSED_SMALL_QCHUNK
#define FOS_FUSED_SMALL_QCHUNK 1024
#endif
#ifndef FOS_FUSED_ACHUNK
#define FOS_FUSED_ACHUNK 4096
#endif
#ifndef FOS_FUSED_QCHUNK_46
#define FOS_FUSED_QCHUNK_46 2048
#endif
#ifndef FOS_FUSED_QCHUNK_6
#define FOS_FUSED_QCHUNK_6 1536
#endif
template <bool F46, bool SR, bool RHT, bool FAKE>
struct FusedCfg {
  static constexpr bool small = F46 && !SR && !RHT && !FAKE;
  static constexpr int threads = small ? FOS_FUSED_SMALL_THREADS : kThreads;
  static constexpr uint32_t achunk = small ? FOS_FUSED_SMALL_ACHUNK : FOS_FUSED_ACHUNK;
  static constexpr uint32_t qchunk = small ? FOS_FUSED_SMALL_QCHUNK : F46 ? FOS_FUSED_QCHUNK_46 : FOS_FUSED_QCHUNK_6;
  // resident CTAs per SM: the threads of FOS_FUSED_MIN_BLOCKS 256-thread CTAs
  // (FOS_K1_MIN_BLOCKS_HEAVY with SR or the transform)
  static constexpr int min_blocks = (SR || RHT ? FOS_K1_MIN_BLOCKS_HEAVY : FOS_FUSED_MIN_BLOCKS) * kThreads / threads;
  static_assert(threads % 32 == 0 && kThreads % threads == 0, "whole warps, a divisor of 256");
  static_assert(qchunk % 32 == 0, "quantize items hold whole choice words");
};

__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Bounded wait until *p >= target (one thread calls it): at most `limit`
// polls, then FOS_STATUS_TIMEOUT and return.
__device__ __forceinline__ void wait_at_least(const uint32_t* p, uint32_t target, uint32_t* status,
                                              uint32_t limit) {
  uint32_t it = 0;
  while (ld_acquire(p) < target) {
    if (++it > limit) {
      if (status) atomicOr(status, FOS_STATUS_TIMEOUT);
      return;
    }
    __nanosleep(128);
  }
}

// max |x| (of the RHT of x) over blocks [lo, hi) of entry b by a group of NT
// threads (t = this thread's index in the group), U loads in flight per
// thread.  Dense input without the transform keeps a running max of |x| over
// bf16 pairs (8 packed max per block) and converts it once at the end.
template <bool RHT, bool DENSE, int NT = kThreads>
__device__ __forceinline__ uint32_t slice_amax_bits(const QuantArgs& a, int b, uint32_t lo, uint32_t hi,
                                                    uint32_t mask16, unsigned long long pol, uint32_t t) {
  constexpr int U = FOS_FUSED_AMAX_UNROLL;
  if (DENSE && !RHT) {
    const uint16_t* xb = a.x + (long long)b * a.x_bs;
    uint32_t m2 = 0;  // the sign bits of this word carry no meaning (xorsign form)
    uint32_t j = lo + t;
#pragma unroll 1
    for (; j + (U - 1) * NT < hi; j += U * NT) {
      uint4 w[U][2];
#pragma unroll
      for (int u = 0; u < U; ++u) ld_block256_hint(xb + (size_t)(j + u * NT) * 16, pol, w[u]);
#pragma unroll
      for (int u = 0; u < U; ++u) m2 = hmax_abs2(m2, hmax_abs_words(w[u]));
    }
#pragma unroll 1
    for (; j < hi; j += NT) {
      uint4 w[2];
      ld_block256_hint(xb + (size_t)j * 16, pol, w);
      m2 = hmax_abs2(m2, hmax_abs_words(w));
    }
    m2 &= 0x7fff7fffu;
    return max(m2 & 0xffffu, m2 >> 16) << 16;
  }
  uint32_t m = 0;
  for (uint32_t j0 = lo + t; j0 < hi; j0 += U * NT) {
    uint4 w[U][2];
#pragma unroll
    for (int u = 0; u < U; ++u) k1_load<DENSE>(a, b, j0 + u * NT, j0 + u * NT < hi, w[u], pol);
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (RHT) {
        rht_flip_signs(w[u], mask16);
        const uint32_t W[8] = {w[u][0].x, w[u][0].y, w[u][0].z, w[u][0].w,
                               w[u][1].x, w[u][1].y, w[u][1].z, w[u][1].w};
        float2 P[8];
        unpack_split(W, P);
        fwht16_split(P);
        m = max(m, amax_bits_split(P));
      } else {
        m = max(m, amax_bits_bf16(w[u]));
      }
    }
  }
  return m;
}

// K0 on rows stored contiguously (ld == cols, 32-byte aligned entries): the
// blocks of an entry are one array, read 256 bits at a time with several
// loads in flight (the fused kernel's amax loop), marked evict-last so that
// the quantizer that follows finds part of them in L2.  grid (chunks, batch),
// units_per_cta blocks per CTA.
template <bool RHT>
__global__ void __launch_bounds__(kThreads) k_amax_dense(const QuantArgs a, uint32_t* amax_ws) {
  const int b = blockIdx.y;
  const uint32_t lo = blockIdx.x * a.units_per_cta, hi = min(lo + a.units_per_cta, a.nblk);
  const uint32_t mask16 = RHT ? rht_sign_mask(a.seed) : 0u;
  uint32_t m = slice_amax_bits<RHT, true>(a, b, lo, hi, mask16, l2_policy_evict_last(), threadIdx.x);
  m = __reduce_max_sync(0xffffffffu, m);
  __shared__ uint32_t s_m[kThreads / 32];
  if ((threadIdx.x & 31) == 0) s_m[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    uint32_t v = threadIdx.x < kThreads / 32 ? s_m[threadIdx.x] : 0u;
    v = __reduce_max_sync(0xffffffffu, v);
    if (threadIdx.x == 0) {
      if (v >= 0x7f800000u) {
        if (a.status) atomicOr(a.status, FOS_STATUS_NONFINITE);
      } else if (v) {
        atomicMax(amax_ws + b, v);
      }
    }
  }
}

// The item sequence of one launch (computed on the host).
struct FusedPlan {
  uint32_t na, nq;         // amax and quantize items per entry
  uint32_t head, mid;      // items of phases [0, L) and of phases [L, batch)
  uint32_t total;          // batch * (na + nq) < 2^31
  int L;
  FastDiv f_na, f_nq, f_ph;  // division by na, nq and na + nq
};

struct FusedItem {
  bool amax;        // amax item (else quantize item)
  int entry;
  uint32_t chunk;
};

// Position i of the item sequence (i < total) -> item.
__device__ __forceinline__ FusedItem fused_item(uint32_t i, int batch, const FusedPlan& p) {
  FusedItem it;
  if (i < p.head) {                                        // phases 0 .. L-1: amax only
    const uint32_t e = fdiv(i, p.f_na);
    it.amax = true; it.entry = (int)e; it.chunk = i - e * p.na;
  } else if (i - p.head < p.mid) {                         // phases L .. batch-1
    const uint32_t r0 = i - p.head, ph = fdiv(r0, p.f_ph);
    const uint32_t r = r0 - ph * (p.na + p.nq);
    const int e = p.L + (int)ph;
    if (r < p.na) { it.amax = true; it.entry = e; it.chunk = r; }
    else          { it.amax = false; it.entry = e - p.L; it.chunk = r - p.na; }
  } else {                                                 // phases batch .. batch+L-1
    const uint32_t r = i - p.head - p.mid, e = fdiv(r, p.f_nq);
    it.amax = false; it.entry = batch - p.L + (int)e; it.chunk = r - e * p.nq;
  }
  return it;
}

// An amax item's result m (max |x| bits of the chunk) into the entry's word,
// then the count-in (release) on done_a[entry]; one thread calls it.
__device__ __forceinline__ void amax_count_in(const QuantArgs& a, uint32_t* amax_ws, uint32_t* done_a, int e,
                                              uint32_t m) {
  if (m >= 0x7f800000u) {
    if (a.status) atomicOr(a.status, FOS_STATUS_NONFINITE);
  } else if (m) {
    atomicMax(amax_ws + e, m);
  }
  __threadfence();
  if (e != a.stall_entry) atomicAdd(done_a + e, 1u);
}

template <bool F46, bool SR, bool RHT, bool SWZ, bool DENSE, bool FAKE>
__global__ void __launch_bounds__((FusedCfg<F46, SR, RHT, FAKE>::threads), (FusedCfg<F46, SR, RHT, FAKE>::min_blocks))
    k_q1x16_fused(const QuantArgs a, int batch, const FusedPlan p, uint32_t* amax_ws, uint32_t* done_a,
                  uint32_t* queue) {
  __shared__ float4 s_tab[128];
  using Cfg = FusedCfg<F46, SR, RHT, FAKE>;
  constexpr int NT = Cfg::threads;
  __shared__ uint32_t s_red[NT / 32];
  __shared__ float s_St;
  __shared__ uint32_t s_item[2];
  const uint32_t mask16 = RHT ? rht_sign_mask(a.seed) : 0u;
  const unsigned long long pol_keep = l2_policy_evict_last();   // amax reads: keep for quantize
  const unsigned long long pol_done = l2_policy_evict_first();  // quantize reads: last use
  uint32_t bad = 0;
  int tab_entry = -1;   // entry whose scale table s_tab holds
  TScale ts{0.0f, 0.0f, false};

  if (threadIdx.x == 0) s_item[0] = atomicAdd(queue, 1u);
  __syncthreads();
  for (int k = 0;; k ^= 1) {
    const uint32_t i = s_item[k];
    if (i >= p.total) break;
#if FOS_FUSED_CLAIM_AHEAD
    if (threadIdx.x == 0) s_item[k ^ 1] = atomicAdd(queue, 1u);  // claim the next item now
#endif
    const FusedItem it = fused_item(i, batch, p);
    if (it.amax) {
      const uint32_t lo = it.chunk * Cfg::achunk, hi = min(lo + Cfg::achunk, a.nblk);
      uint32_t m = slice_amax_bits<RHT, DENSE, NT>(a, it.entry, lo, hi, mask16, pol_keep, threadIdx.x);
      m = __reduce_max_sync(0xffffffffu, m);
      if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = m;
      __syncthreads();
      if (threadIdx.x == 0) {
        uint32_t v = 0;
#pragma unroll
        for (int w = 0; w < NT / 32; ++w) v = max(v, s_red[w]);
        amax_count_in(a, amax_ws, done_a, it.entry, v);
      }
    } else {
      if (it.entry != tab_entry) {
        if (threadIdx.x == 0) {
          wait_at_least(done_a + it.entry, p.na, a.status, a.spin_limit);
          const float A = __uint_as_float(__ldcg(amax_ws + it.entry));
          s_St = __fdiv_rn(A, F46 ? 1792.0f : 2688.0f);
        }
        __syncthreads();
        ts = make_tscale(s_St);
        build_scale_table4(s_tab, ts.St);
        __syncthreads();
        tab_entry = it.entry;
      }
      if (it.chunk == 0 && threadIdx.x == 0 && a.row.tensor_scale) a.row.tensor_scale[it.entry] = ts.St;
      const uint32_t lo = it.chunk * Cfg::qchunk, hi = min(lo + Cfg::qchunk, a.nblk);
      rowwise_range<F46, SR, RHT, SWZ, DENSE, NT, FAKE>(a, it.entry, lo, hi, s_tab, ts, mask16, bad, pol_done);
    }
#if !FOS_FUSED_CLAIM_AHEAD
    if (threadIdx.x == 0) s_item[k ^ 1] = atomicAdd(queue, 1u);
#endif
    __syncthreads();  // the next item is in s_item[k ^ 1]; s_red / s_tab / s_St may be rewritten
  }
  if (bad >= 0x7f800000u && a.status) atomicOr(a.status, FOS_STATUS_NONFINITE);
}

// --------------------------------------------------------------------------
// MXFP4 1x32: E = floor(log2 amax) - 2 from the exponent bits, clamped to
// [-127, 127]; codes = E2M1_rne(w * 2^-E) (the scaling is exact).
template <bool SWZ>
__global__ void __launch_bounds__(kThreads) k_mxfp4(const QuantArgs a) {
  const int b = blockIdx.y;
  const uint32_t u0 = blockIdx.x * a.units_per_cta;
  const uint32_t u1 = min(u0 + a.units_per_cta, a.nblk);
  uint32_t bad = 0;
  for (uint32_t j = u0 + threadIdx.x; j < u1; j += kThreads) {
    const uint32_t row = fdiv(j, a.bpr);
    const uint32_t cb = j - row * a.bpr.d;
    const uint4* p = reinterpret_cast<const uint4*>(a.x + (long long)b * a.x_bs +
                                                   (long long)row * a.ld + (long long)cb * 32);
    uint4 w4[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) w4[k] = __ldg(p + k);
    const uint4 lo[2] = {w4[0], w4[1]}, hi[2] = {w4[2], w4[3]};
    const uint32_t am = max(amax_bits_bf16(lo), amax_bits_bf16(hi));
    bad = max(bad, am);
    const uint32_t ex = max(am >> 23, 2u);          // biased exponent, >= 2
    const uint32_t scale = ex - 2u;                 // E + 127 with E = ex - 129
    const float inv = __uint_as_float((256u - ex) << 23);  // 2^-E
    const float2 inv2 = make_float2(inv, inv);
    const uint32_t* w = &w4[0].x;
    float v[32];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const float2 r = mul2(make_float2(bf_lo(w[k]), bf_hi(w[k])), inv2);
      v[2 * k] = r.x;
      v[2 * k + 1] = r.y;
    }
    uint4 c;
    c.x = e2m1x8(v[0], v[1], v[2], v[3], v[4], v[5], v[6], v[7]);
    c.y = e2m1x8(v[8], v[9], v[10], v[11], v[12], v[13], v[14], v[15]);
    c.z = e2m1x8(v[16], v[17], v[18], v[19], v[20], v[21], v[22], v[23]);
    c.w = e2m1x8(v[24], v[25], v[26], v[27], v[28], v[29], v[30], v[31]);
    uint2* cp = reinterpret_cast<uint2*>(a.row.codes + (long long)b * a.row.codes_bs +
                                         (long long)row * a.row.codes_ld + (long long)cb * 16);
    cp[0] = make_uint2(c.x, c.y);
    cp[1] = make_uint2(c.z, c.w);
    long long so;
    if (SWZ) so = (long long)b * a.row.scales_bs + swz_offset(row, cb, a.row.col_tiles);
    else     so = (long long)b * a.row.scales_bs + (long long)row * a.row.scales_ld + cb;
    a.row.scales[so] = (uint8_t)scale;
  }
  if (bad >= 0x7f800000u && a.status) atomicOr(a.status, FOS_STATUS_NONFINITE);
}

// --------------------------------------------------------------------------
// Dequantize: NVFP4 y = bf16_rne((q * float(s)) * S_t); MXFP4 y = q * 2^(s-127).
// One 16-element group per thread (an NVFP4 block, or half an MXFP4 block):
// 8 code bytes in, 32 bytes of bf16 out.  DENSE: codes and y rows
// contiguous, linear scales and a 32-byte aligned y, so group j sits at code
// byte 8j and element 16j and is written with one 256-bit store (a warp
// writes 1 KB of contiguous output per store instruction).
__device__ __forceinline__ void st_global_v8(void* p, const uint32_t (&o)[8]) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};"
               :: "l"(p), "r"(o[0]), "r"(o[1]), "r"(o[2]), "r"(o[3]), "r"(o[4]), "r"(o[5]), "r"(o[6]), "r"(o[7])
               : "memory");
}

template <bool MX, bool SWZ, bool DENSE>
__global__ void __launch_bounds__(kThreads) k_dequant(const DequantArgs a) {
  const int b = blockIdx.y;
  constexpr uint32_t GPB = MX ? 2 : 1;  // 16-element groups per block
  const uint32_t ngroups = a.nblk * GPB;
  const uint32_t u0 = blockIdx.x * a.units_per_cta;
  const uint32_t u1 = min(u0 + a.units_per_cta, ngroups);
  const float St = MX ? 1.0f : a.tensor_scale[b];
  const float2 t2 = make_float2(St, St);
  for (uint32_t j = u0 + threadIdx.x; j < u1; j += kThreads) {
    const uint32_t blk = MX ? (j >> 1) : j;
    uint32_t row, cb;
    if (DENSE) {
      row = 0;
      cb = blk;
    } else {
      row = fdiv(blk, a.bpr);
      cb = blk - row * a.bpr.d;
    }
    long long so;
    if (SWZ) so = (long long)b * a.scales_bs + swz_offset(row, cb, a.col_tiles);
    else     so = (long long)b * a.scales_bs + (long long)row * a.scales_ld + cb;
    const uint32_t sc = a.scales[so];
    const float s = MX ? __uint_as_float(sc == 0 ? 0x00400000u : (sc << 23)) : e4m3_to_f32(sc);
    const long long goff = (long long)cb * (MX ? 2 : 1) + (MX ? (j & 1) : 0);  // group within the row
    const uint2 cw = *reinterpret_cast<const uint2*>(a.codes + (long long)b * a.codes_bs +
                                                     (long long)row * a.codes_ld + goff * 8);
    uint32_t h[8];
    e2m1x8_to_h2(cw.x, h);
    e2m1x8_to_h2(cw.y, h + 4);
    const float2 s2 = make_float2(s, s);
    uint32_t o[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      float2 q = mul2(make_float2(h_lo(h[k]), h_hi(h[k])), s2);
      if (!MX) q = mul2(q, t2);
      const __nv_bfloat162 r = __floats2bfloat162_rn(q.x, q.y);
      o[k] = *reinterpret_cast<const uint32_t*>(&r);
    }
    uint16_t* yp = a.y + (long long)b * a.y_bs + (long long)row * a.ldy + goff * 16;
    if (DENSE) {  // 32-byte aligned
      st_global_v8(yp, o);
    } else {      // rows only 16-byte aligned
      reinterpret_cast<uint4*>(yp)[0] = make_uint4(o[0], o[1], o[2], o[3]);
      reinterpret_cast<uint4*>(yp)[1] = make_uint4(o[4], o[5], o[6], o[7]);
    }
  }
}

// MXFP4 fake quantization: E = floor(log2 amax) - 2 per 32-block (clamped),
// codes = E2M1_rne(w * 2^-E), y = bf16(q * 2^E) (exact).  grid (chunks, batch).
__global__ void __launch_bounds__(kThreads) k_fake_mx(const QuantArgs a) {
  const int b = blockIdx.y;
  const uint32_t u0 = blockIdx.x * a.units_per_cta;
  const uint32_t u1 = min(u0 + a.units_per_cta, a.nblk);
  uint32_t bad = 0;
  for (uint32_t j = u0 + threadIdx.x; j < u1; j += kThreads) {
    const uint32_t row = fdiv(j, a.bpr);
    const uint32_t cb = j - row * a.bpr.d;
    const uint4* p = reinterpret_cast<const uint4*>(a.x + (long long)b * a.x_bs + (long long)row * a.ld +
                                                   (long long)cb * 32);
    uint4 w4[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) w4[k] = __ldg(p + k);
    const uint4 lo[2] = {w4[0], w4[1]}, hi[2] = {w4[2], w4[3]};
    const uint32_t am = max(amax_bits_bf16(lo), amax_bits_bf16(hi));
    bad = max(bad, am);
    const uint32_t ex = max(am >> 23, 2u);                     // biased exponent, >= 2
    const float inv = __uint_as_float((256u - ex) << 23);      // 2^-E, E = ex - 129
    const uint32_t sc = ex - 2u;                               // E + 127
    const float sE = __uint_as_float(sc == 0 ? 0x00400000u : (sc << 23));  // 2^E
    const float2 inv2 = make_float2(inv, inv), s2 = make_float2(sE, sE);
    const uint32_t* w = &w4[0].x;
    uint4* yp = reinterpret_cast<uint4*>(a.y + (long long)b * a.y_bs + (long long)row * a.ldy + (long long)cb * 32);
#pragma unroll
    for (int part = 0; part < 2; ++part) {
      float v[16];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float2 r = mul2(make_float2(bf_lo(w[8 * part + k]), bf_hi(w[8 * part + k])), inv2);
        v[2 * k] = r.x;
        v[2 * k + 1] = r.y;
      }
      const uint32_t c0 = e2m1x8(v[0], v[1], v[2], v[3], v[4], v[5], v[6], v[7]);
      const uint32_t c1 = e2m1x8(v[8], v[9], v[10], v[11], v[12], v[13], v[14], v[15]);
      uint32_t h[8];
      e2m1x8_to_h2(c0, h);
      e2m1x8_to_h2(c1, h + 4);
      uint32_t o[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float2 q = mul2(make_float2(h_lo(h[k]), h_hi(h[k])), s2);
        const __nv_bfloat162 r = __floats2bfloat162_rn(q.x, q.y);
        o[k] = *reinterpret_cast<const uint32_t*>(&r);
      }
      yp[2 * part] = make_uint4(o[0], o[1], o[2], o[3]);
      yp[2 * part + 1] = make_uint4(o[4], o[5], o[6], o[7]);
    }
  }
  if (bad >= 0x7f800000u && a.status) atomicOr(a.status, FOS_STATUS_NONFINITE);
}

}  // namespace

// ------------------------------------------------------------------ launchers
static constexpr int kMaxDevices = 64;

static dim3 grid_for(uint32_t units, uint32_t per_cta, int batch) {
  return dim3((units + per_cta - 1) / per_cta, (unsigned)batch, 1);
}

// Blocks per CTA for `nblk` blocks in each of `batch` entries on `slots`
// resident CTAs: at most max_units, a multiple of 32 (whole choice words),
// and spread so that the last wave of CTAs is about as full as the others
// (e.g. a 2.1 M-block tensor on 592 slots: 1792 blocks per CTA, 1.98 waves,
// instead of 2048 blocks and 1.73 waves).
static uint32_t balanced_units(uint32_t nblk, int batch, uint32_t max_units, int slots) {
  const unsigned long long total = (unsigned long long)nblk * (unsigned long long)batch;
  const unsigned long long per_wave = (unsigned long long)slots * max_units;
  const unsigned long long waves = (total + per_wave - 1) / per_wave;
  unsigned long long u = (total + waves * slots - 1) / (waves * slots);
  u = (u + 31) / 32 * 32;
  return (uint32_t)(u < 32 ? 32 : (u > max_units ? max_units : u));
}

// The dense amax kernel with 2 * units_per_cta blocks per CTA at most,
// spread over whole waves of its resident slots (looked up once per device).
template <bool RHT>
static cudaError_t launch_amax_dense(const QuantArgs& a, int batch, uint32_t* amax_ws, cudaStream_t st) {
  static std::atomic<int> slots_of[kMaxDevices];
  auto kern = k_amax_dense<RHT>;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return cudaErrorNotSupported;
  int slots = slots_of[dev].load(std::memory_order_relaxed);
  if (slots == 0) {
    int sms = 0, per_sm = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, 0) != cudaSuccess)
      return cudaErrorNotSupported;
    slots = sms * (per_sm > 0 ? per_sm : 1);
    slots_of[dev].store(slots, std::memory_order_relaxed);
  }
  QuantArgs b = a;
  b.units_per_cta = balanced_units(a.nblk, batch, 2 * a.units_per_cta, slots);
  kern<<<grid_for(a.nblk, b.units_per_cta, batch), kThreads, 0, st>>>(b, amax_ws);
  return cudaGetLastError();
}

cudaError_t launch_amax(const QuantArgs& a, int batch, bool rht, uint32_t* amax_ws,
                        cudaStream_t st) {
  if (a.ld == a.cols && (reinterpret_cast<uintptr_t>(a.x) & 31) == 0 && (a.x_bs & 15) == 0)
    return rht ? launch_amax_dense<true>(a, batch, amax_ws, st) : launch_amax_dense<false>(a, batch, amax_ws, st);
  const uint32_t nunit = (a.nblk + 1) / 2;
  const dim3 g = grid_for(nunit, a.units_per_cta, batch);
  if (rht) k_amax<true><<<g, kThreads, 0, st>>>(a, amax_ws);
  else     k_amax<false><<<g, kThreads, 0, st>>>(a, amax_ws);
  return cudaGetLastError();
}

// One k_q1x16 variant, with the work per CTA balanced over the resident
// slots (SMs x resident CTAs, looked up once per device and variant).
template <bool F46, bool SR, bool RHT, bool SWZ, bool DENSE, bool FAKE>
static cudaError_t launch_k1(const QuantArgs& a, int batch, cudaStream_t st) {
  static std::atomic<int> slots_of[kMaxDevices];
  auto kern = k_q1x16<F46, SR, RHT, SWZ, DENSE, FAKE>;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return cudaErrorNotSupported;
  int slots = slots_of[dev].load(std::memory_order_relaxed);
  if (slots == 0) {
    int sms = 0, per_sm = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, 0) != cudaSuccess)
      return cudaErrorNotSupported;
    slots = sms * (per_sm > 0 ? per_sm : 1);
    slots_of[dev].store(slots, std::memory_order_relaxed);
  }
  QuantArgs b = a;
  b.units_per_cta = balanced_units(a.nblk, batch, a.units_per_cta, slots);
  const dim3 g = grid_for(a.nblk, b.units_per_cta, batch);
  kern<<<g, kThreads, 0, st>>>(b);
  return cudaGetLastError();
}

cudaError_t launch_q1x16_rowwise(const QuantArgs& a, int batch, int fmt, bool sr, bool rht,
                                 bool swz, bool dense, cudaStream_t st, bool fake) {
  const bool f46 = fmt == 0;
  if (dense || fake) swz = false;
  if (fake) {
#define FOS_L(F, S, R, D) return launch_k1<F, S, R, false, D, true>(a, batch, st)
#define FOS_D(F, S, R) do { if (dense) FOS_L(F, S, R, true); else FOS_L(F, S, R, false); } while (0)
#define FOS_R(F, S) do { if (rht) FOS_D(F, S, true); else FOS_D(F, S, false); } while (0)
#define FOS_S(F) do { if (sr) FOS_R(F, true); else FOS_R(F, false); } while (0)
    if (f46) FOS_S(true);
    else     FOS_S(false);
#undef FOS_S
#undef FOS_R
#undef FOS_D
#undef FOS_L
  }
#define FOS_L(F, S, R, W, D) return launch_k1<F, S, R, W, D, false>(a, batch, st)
#define FOS_D(F, S, R, W) do { if (dense) FOS_L(F, S, R, W, true); else FOS_L(F, S, R, W, false); } while (0)
#define FOS_W(F, S, R) do { if (swz) FOS_D(F, S, R, true); else FOS_D(F, S, R, false); } while (0)
#define FOS_R(F, S) do { if (rht) FOS_W(F, S, true); else FOS_W(F, S, false); } while (0)
#define FOS_S(F) do { if (sr) FOS_R(F, true); else FOS_R(F, false); } while (0)
  if (f46) FOS_S(true);
  else     FOS_S(false);
#undef FOS_S
#undef FOS_R
#undef FOS_W
#undef FOS_D
#undef FOS_L
}

// Persistent launch of the fused kernel: one CTA per resident slot.  The
// grid (SMs x resident CTAs) is looked up once per device and kernel variant
// and cached; 0 = not yet known, -1 = the kernel cannot be resident.

// The item sequence for nblk blocks per entry; false when the item count does
// not fit the 31-bit positions of the queue.
static bool make_plan(FusedPlan& p, uint32_t nblk, int batch, uint32_t achunk, uint32_t qchunk, int lag) {
  if (nblk == 0 || batch < 1) return false;
  p.na = (nblk + achunk - 1) / achunk;
  p.nq = (nblk + qchunk - 1) / qchunk;
  p.L = lag < batch ? lag : batch;
  const unsigned long long total = (unsigned long long)batch * (p.na + p.nq);
  if (total >= (1ull << 31)) return false;
  p.total = (uint32_t)total;
  p.head = (uint32_t)p.L * p.na;
  p.mid = (uint32_t)(batch - p.L) * (p.na + p.nq);
  p.f_na = make_fastdiv(p.na);
  p.f_nq = make_fastdiv(p.nq);
  p.f_ph = make_fastdiv(p.na + p.nq);
  return true;
}

template <bool F46, bool SR, bool RHT, bool SWZ, bool DENSE, bool FAKE = false>
static cudaError_t launch_fused_t(const QuantArgs& a, int batch, uint32_t* amax_ws, uint32_t* done_a,
                                  uint32_t* queue, cudaStream_t st) {
  static std::atomic<int> grid_of[kMaxDevices];
  auto kern = k_q1x16_fused<F46, SR, RHT, SWZ, DENSE, FAKE>;
  FusedPlan plan;
  using Cfg = FusedCfg<F46, SR, RHT, FAKE>;
  if (!make_plan(plan, a.nblk, batch, Cfg::achunk, Cfg::qchunk, F46 ? FOS_FUSED_LAG_46 : FOS_FUSED_LAG_6))
    return cudaErrorNotSupported;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return cudaErrorNotSupported;
  int grid = grid_of[dev].load(std::memory_order_relaxed);
  if (grid == 0) {
    int sms = 0, per_sm = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, Cfg::threads, 0) != cudaSuccess)
      return cudaErrorNotSupported;
    grid = per_sm >= 1 ? sms * per_sm : -1;
    grid_of[dev].store(grid, std::memory_order_relaxed);
  }
  if (grid < 1) return cudaErrorNotSupported;
  kern<<<grid, Cfg::threads, 0, st>>>(a, batch, plan, amax_ws, done_a, queue);
  return cudaGetLastError();
}

cudaError_t launch_q1x16_fused(const QuantArgs& a, int batch, int fmt, bool sr, bool rht, bool swz,
                               bool dense, uint32_t* amax_ws, uint32_t* done_a, uint32_t* queue,
                               cudaStream_t st, bool fake) {
  const bool f46 = fmt == 0;
  if (dense || fake) swz = false;
  if (fake) {
#define FOS_L(F, S, R, D) return launch_fused_t<F, S, R, false, D, true>(a, batch, amax_ws, done_a, queue, st)
#define FOS_D(F, S, R) do { if (dense) FOS_L(F, S, R, true); else FOS_L(F, S, R, false); } while (0)
#define FOS_R(F, S) do { if (rht) FOS_D(F, S, true); else FOS_D(F, S, false); } while (0)
#define FOS_S(F) do { if (sr) FOS_R(F, true); else FOS_R(F, false); } while (0)
    if (f46) FOS_S(true);
    else     FOS_S(false);
#undef FOS_S
#undef FOS_R
#undef FOS_D
#undef FOS_L
  }
#define FOS_L(F, S, R, W, D) return launch_fused_t<F, S, R, W, D>(a, batch, amax_ws, done_a, queue, st)
#define FOS_D(F, S, R, W) do { if (dense) FOS_L(F, S, R, W, true); else FOS_L(F, S, R, W, false); } while (0)
#define FOS_W(F, S, R) do { if (swz) FOS_D(F, S, R, true); else FOS_D(F, S, R, false); } while (0)
#define FOS_R(F, S) do { if (rht) FOS_W(F, S, true); else FOS_W(F, S, false); } while (0)
#define FOS_S(F) do { if (sr) FOS_R(F, true); else FOS_R(F, false); } while (0)
  if (f46) FOS_S(true);
  else     FOS_S(false);
#undef FOS_S
#undef FOS_R
#undef FOS_W
#undef FOS_D
#undef FOS_L
}

cudaError_t launch_mxfp4(const QuantArgs& a, int batch, bool swz, cudaStream_t st) {
  const dim3 g = grid_for(a.nblk, a.units_per_cta, batch);
  if (swz) k_mxfp4<true><<<g, kThreads, 0, st>>>(a);
  else     k_mxfp4<false><<<g, kThreads, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_dequant(const DequantArgs& a, int batch, bool mx, bool swz, bool dense, cudaStream_t st) {
  const dim3 g = grid_for(a.nblk * (mx ? 2 : 1), a.units_per_cta, batch);
  if (swz) dense = false;
#define FOS_L(M, W, D) k_dequant<M, W, D><<<g, kThreads, 0, st>>>(a)
#define FOS_D(M, W) do { if (dense) FOS_L(M, W, true); else FOS_L(M, W, false); } while (0)
#define FOS_W(M) do { if (swz) FOS_D(M, true); else FOS_D(M, false); } while (0)
  if (mx) FOS_W(true);
  else    FOS_W(false);
#undef FOS_W
#undef FOS_D
#undef FOS_L
  return cudaGetLastError();
}

cudaError_t launch_fake_mx(const QuantArgs& a, int batch, cudaStream_t st) {
  const dim3 g((a.nblk + a.units_per_cta - 1) / a.units_per_cta, (unsigned)batch, 1);
  k_fake_mx<<<g, kThreads, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace fos
