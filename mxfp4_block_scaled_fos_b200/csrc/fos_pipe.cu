// fos_pipe.cu -- per-entry amax + rowwise 1x16 NVFP4 quantize of a batch of
// tensors (e.g. the experts of an MoE layer, one S_t each) in one persistent,
// cooperative launch that reads every input byte from HBM about once.
//
// Method: Hugging Face transformers doc "Four Over Six", introduction (each
// NVFP4 block scaled so its max maps to 4 or to 6, the lower-error candidate
// kept); Ultralytics glossary "FP4", "Como funciona FP4" (NVFP4: 16 values,
// E4M3 block scale, FP32 per-tensor scale S_t).  A block can only be scaled
// once its whole tensor's amax is known, so each entry is read twice: once
// for the amax, once to quantize.  This kernel overlaps the two so that the
// second read comes from L2.
//
// Schedule.  Phase p (p = 0 .. batch + L - 1) of every warp: quantize its
// slice of entry p - L, then take the amax of its slice of entry p.  The
// slices are the 32-block groups of an entry cut evenly over all warps of
// the grid; the cut rotates by one warp per phase so that the warps with one
// group more than the others change from phase to phase.  Entries p - L .. p
// + 1 are in flight (the next phase's amax slice is prefetched into L2 with
// a bulk prefetch), which is (L + 2) entries of input: 66 MB for 2880 x 2880
// bf16 entries and L = 2, well inside the 126 MB L2.
//
// Synchronisation, without CTA-wide barriers or a work queue:
//  * amax of entry p: each warp reduces its slice and folds it into a
//    per-CTA shared word (phase ring of R slots); the CTA's last warp to
//    count in folds that into the entry's global amax word and counts the CTA
//    in on the entry's global counter.  The CTA that completes the count
//    builds the entry's record in a ring of R slots in the workspace: S_t,
//    its reciprocal and the 128-entry table (inv, inv, -E, -E) of every
//    non-negative E4M3 code c, E = float(c) * S_t, inv = 1/E (0 for E = 0,
//    FLT_MAX at most); then it counts in once more to publish it.
//  * quantize of entry q: every lane polls the entry's counter with an
//    acquire load (bounded: FOS_STATUS_TIMEOUT after QuantArgs::spin_limit
//    polls) until it shows all CTAs plus the record, then the warp copies the
//    record's table into its own shared-memory slice (L2 loads, so no stale
//    L1 line of an earlier use of the ring slot is read).
//  * Every warp waits for entry p - L at phase p even when it has no group
//    of that entry, so no warp runs more than L phases ahead of the slowest
//    CTA's amax: a ring slot of phase p is reused at phase p + R only after
//    every warp has finished with it (R = L + 2).
// All CTAs must be resident at once (a warp waits on every CTA's count-in),
// which the cooperative launch guarantees; it fails rather than deadlock
// when the grid does not fit.
#include <cooperative_groups.h>

#include <atomic>

#include "fos_core.cuh"

namespace fos {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
#ifndef FOS_PIPE_LAG
#define FOS_PIPE_LAG 2
#endif
#ifndef FOS_PIPE_MIN_BLOCKS
#define FOS_PIPE_MIN_BLOCKS 5
#endif
constexpr int kLag = FOS_PIPE_LAG;
constexpr int kRing = kLag + 2;

// One entry's record in the workspace ring (16-byte aligned).
struct PipeRecord {
  float4 tab[128];  // (inv, inv, -E, -E) for E4M3 code c
  float St, y;      // S_t and RN(1 / S_t) (y = 0 when S_t < 2^-92)
  uint32_t pad[2];
};

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ float4 ld_cg_f4(const float4* p) {
  float4 v;
  asm volatile("ld.global.cg.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "l"(p));
  return v;
}

__device__ __forceinline__ float ld_cg_f32(const float* p) {
  float v;
  asm volatile("ld.global.cg.f32 %0, [%1];" : "=f"(v) : "l"(p));
  return v;
}

// Groups [g0, g1) of an entry with ng groups for the warp in rotated slot s
// of W: an even cut, 64-bit products.
__device__ __forceinline__ void slice_of(uint32_t s, uint32_t W, uint32_t ng, uint32_t& g0, uint32_t& g1) {
  g0 = (uint32_t)(((unsigned long long)s * ng) / W);
  g1 = (uint32_t)(((unsigned long long)(s + 1) * ng) / W);
}

// Quantize groups [g0, g1) (32 blocks each) of entry b with the table in
// this warp's shared slice.  One block per lane per group.
template <bool F46, bool SR, bool RHT, bool SWZ, bool DENSE, int FAST>
__device__ __forceinline__ void quant_groups(const QuantArgs& a, int b, uint32_t g0, uint32_t g1,
                                             const float4* tab, const TScale& ts, uint32_t mask16,
                                             uint32_t& badmax, unsigned long long pol) {
  const uint32_t lane = threadIdx.x & 31;
  const float nz = a.neg_zero;
  const long long gbase = SR ? a.elem_offset + (long long)b * a.rows * a.cols : 0;
  uint32_t* chw = a.row.choice ? reinterpret_cast<uint32_t*>(a.row.choice) : nullptr;
  for (uint32_t gi = g0; gi < g1; ++gi) {
    const uint32_t j = gi * 32 + lane;
    const bool valid = j < a.nblk;
    const uint32_t jj = valid ? j : a.nblk - 1;
    uint4 w[2];
    if (DENSE) ld_block256_hint(a.x + (long long)b * a.x_bs + (long long)jj * 16, pol, w);
    else       load_block(a, b, jj, w);
    if (RHT) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        (&w[0].x)[k] ^= rht_word_mask(mask16, k);
        (&w[1].x)[k] ^= rht_word_mask(mask16, k + 4);
      }
    }
    const uint32_t W8[8] = {w[0].x, w[0].y, w[0].z, w[0].w, w[1].x, w[1].y, w[1].z, w[1].w};
    float2 P[8];
    unpack_split(W8, P);
    uint32_t m;
    if (RHT) {
      fwht16_split(P);
      m = 0;
#pragma unroll
      for (int k = 0; k < 8; ++k)
        m = max(m, max(__float_as_uint(P[k].x) & 0x7fffffffu, __float_as_uint(P[k].y) & 0x7fffffffu));
    } else {
      m = amax_bits_bf16(w);
    }
    badmax = max(badmax, m);
    uint32_t s6, s4;
    cand_scales<F46, FAST>(__uint_as_float(m), ts, s6, s4);
    const float4 t6 = tab[s6];
    Cand1 c6 = candidate1_t<F46>(P, t6, nz);
    uint32_t codes[2] = {c6.c[0], c6.c[1]};
    uint32_t sc = s6;
    float inv = t6.x;
    bool pick = false;
    if (F46) {
      const float4 t4 = tab[s4];
      const Cand1 c4 = candidate1_t<true>(P, t4, nz);
      pick = c4.err < c6.err;  // strictly lower wins; ties keep 6
      if (pick) { codes[0] = c4.c[0]; codes[1] = c4.c[1]; sc = s4; inv = t4.x; }
    }
    if (SR) {
      long long e0;
      if (DENSE) {
        e0 = gbase + (long long)jj * 16;
      } else {
        const uint32_t row = fdiv(jj, a.bpr), cb = jj - row * a.bpr.d;
        e0 = gbase + (long long)row * a.cols + cb * 16;
      }
      sr_block1(P, inv, sr_bytes16(a.seed, e0), codes);
    }
    if (valid) {
      if (DENSE) {
        *reinterpret_cast<uint2*>(a.row.codes + (long long)b * a.row.codes_bs + (long long)j * 8) =
            make_uint2(codes[0], codes[1]);
        a.row.scales[(long long)b * a.row.scales_bs + j] = (uint8_t)sc;
      } else {
        store_block<SWZ>(a.row, b, j, a.bpr, codes, sc);
      }
    }
    if (F46 && chw) {
      const uint32_t word = __ballot_sync(0xffffffffu, pick && valid);
      if (lane == 0) {
        const unsigned long long gbit = (unsigned long long)b * a.nblk + gi * 32;
        if (a.row.choice_aligned) chw[gbit >> 5] = word;
        else if (word) {
          const int sh = (int)(gbit & 31);
          const unsigned long long vv = (unsigned long long)word << sh;
          if ((uint32_t)vv) atomicOr(chw + (gbit >> 5), (uint32_t)vv);
          if ((uint32_t)(vv >> 32)) atomicOr(chw + (gbit >> 5) + 1, (uint32_t)(vv >> 32));
        }
      }
    }
  }
}

// max |x| (of the RHT of x) over groups [g0, g1) of entry b, per lane.
template <bool RHT, bool DENSE>
__device__ __forceinline__ uint32_t amax_groups(const QuantArgs& a, int b, uint32_t g0, uint32_t g1,
                                                uint32_t mask16, unsigned long long pol) {
  const uint32_t lane = threadIdx.x & 31;
  uint32_t m = 0;
  uint32_t gi = g0;
  for (; gi + 2 <= g1; gi += 2) {  // two loads in flight per lane
    const uint32_t j0 = gi * 32 + lane, j1 = j0 + 32;
    uint4 w0[2], w1[2];
    const uint32_t jj0 = min(j0, a.nblk - 1), jj1 = min(j1, a.nblk - 1);
    if (DENSE) {
      ld_block256_hint(a.x + (long long)b * a.x_bs + (long long)jj0 * 16, pol, w0);
      ld_block256_hint(a.x + (long long)b * a.x_bs + (long long)jj1 * 16, pol, w1);
    } else {
      load_block(a, b, jj0, w0);
      load_block(a, b, jj1, w1);
    }
    if (RHT) {
      m = max(m, rht_block_amax(w0, mask16));
      m = max(m, rht_block_amax(w1, mask16));
    } else {
      m = max(m, max(amax_bits_bf16(w0), amax_bits_bf16(w1)));
    }
  }
  if (gi < g1) {
    const uint32_t jj = min(gi * 32 + lane, a.nblk - 1);
    uint4 w[2];
    if (DENSE) ld_block256_hint(a.x + (long long)b * a.x_bs + (long long)jj * 16, pol, w);
    else       load_block(a, b, jj, w);
    m = max(m, RHT ? rht_block_amax(w, mask16) : amax_bits_bf16(w));
  }
  return m;
}

template <bool F46, bool SR, bool RHT, bool SWZ, bool DENSE>
__global__ void __launch_bounds__(kThreads, (SR || RHT) ? 4 : FOS_PIPE_MIN_BLOCKS)
    k_q1x16_pipe(const QuantArgs a, int batch, uint32_t* amax_ws, uint32_t* cnt, PipeRecord* ring) {
  __shared__ __align__(16) float4 s_tab[kWarps][128];
  __shared__ uint32_t s_max[kRing], s_cnt[kRing];
  const uint32_t lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float4* tab = s_tab[warp];
  if (threadIdx.x < kRing) {
    s_max[threadIdx.x] = 0;
    s_cnt[threadIdx.x] = 0;
  }
  __syncthreads();  // the only CTA barrier: the ring counters start at zero

  const uint32_t W = gridDim.x * kWarps;
  const uint32_t wid = blockIdx.x * kWarps + warp;
  const uint32_t ng = (a.nblk + 31) / 32;
  const uint32_t G = gridDim.x;
  const uint32_t mask16 = RHT ? rht_sign_mask(a.seed) : 0u;
  uint32_t badmax = 0;
  bool timed_out = false;

  // L2 prefetch (evict-last) of the amax slice of entry e in rotated slot
  // `slot` (dense rows only; one bulk prefetch by lane 0)
  auto prefetch_slice = [&](int e, uint32_t slot) {
    if (!DENSE || e >= batch || lane != 0) return;
    uint32_t g0, g1;
    slice_of(slot, W, ng, g0, g1);
    if (g0 >= g1) return;
    const uint32_t j0 = g0 * 32, j1 = min(g1 * 32, a.nblk);
    const char* p = reinterpret_cast<const char*>(a.x + (long long)e * a.x_bs + (long long)j0 * 16);
    prefetch_l2(p, (j1 - j0) * 32u, l2_policy_evict_last());
  };
  prefetch_slice(0, wid % W);

  for (int p = 0; p < batch + kLag; ++p) {
    const uint32_t slot = (wid + (uint32_t)p) % W;
    uint32_t g0, g1;
    slice_of(slot, W, ng, g0, g1);
    prefetch_slice(p + 1, (wid + (uint32_t)p + 1) % W);

    // ---------------- quantize entry q = p - L
    const int q = p - kLag;
    if (q >= 0) {
      const uint32_t* c = cnt + q;
      uint32_t it = 0;
      while (ld_acquire_u32(c) < G + 1) {
        if (++it > a.spin_limit) { timed_out = true; break; }
        __nanosleep(128);
      }
      __syncwarp();
      const PipeRecord* rec = ring + (q % kRing);
#pragma unroll
      for (int k = 0; k < 4; ++k) tab[lane + 32 * k] = ld_cg_f4(&rec->tab[lane + 32 * k]);
      const float St = ld_cg_f32(&rec->St);
      __syncwarp();
      if (g0 < g1) {
        const TScale ts = make_tscale(St);
        const unsigned long long pol = l2_policy_evict_first();  // last use of the input
        if (ts.fast) quant_groups<F46, SR, RHT, SWZ, DENSE, 1>(a, q, g0, g1, tab, ts, mask16, badmax, pol);
        else         quant_groups<F46, SR, RHT, SWZ, DENSE, 0>(a, q, g0, g1, tab, ts, mask16, badmax, pol);
      }
      __syncwarp();  // the slice's table is rewritten at the next phase
    }

    // ---------------- amax of entry p
    if (p < batch) {
      uint32_t m = (g0 < g1) ? amax_groups<RHT, DENSE>(a, p, g0, g1, mask16, l2_policy_evict_last()) : 0u;
      m = __reduce_max_sync(0xffffffffu, m);
      bool last_cta = false;
      if (lane == 0) {
        const int r = p % kRing;
        if (m >= 0x7f800000u) {
          if (a.status) atomicOr(a.status, FOS_STATUS_NONFINITE);
          m = 0;
        }
        atomicMax(&s_max[r], m);
        __threadfence_block();
        if (atomicAdd(&s_cnt[r], 1u) == kWarps - 1) {  // last warp of the CTA for this phase
          __threadfence_block();
          const uint32_t v = atomicAdd(&s_max[r], 0u);
          s_max[r] = 0;
          s_cnt[r] = 0;
          if (v) atomicMax(amax_ws + p, v);
          __threadfence();
          if (p != a.stall_entry) last_cta = atomicAdd(cnt + p, 1u) == G - 1;
        }
      }
      last_cta = __shfl_sync(0xffffffffu, last_cta, 0);
      if (last_cta) {  // every CTA has counted in: build and publish entry p's record
        __threadfence();
        const float A = __uint_as_float(ld_acquire_u32(amax_ws + p));
        const float St = __fdiv_rn(A, F46 ? 1792.0f : 2688.0f);
        PipeRecord* rec = ring + (p % kRing);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t code = lane + 32 * k;
          const float E = __fmul_rn(e4m3_to_f32(code), St);
          const float inv = (E == 0.0f) ? 0.0f : fminf(__frcp_rn(E), kFltMax);
          rec->tab[code] = make_float4(inv, inv, -E, -E);
        }
        if (lane == 0) {
          rec->St = St;
          if (a.row.tensor_scale) a.row.tensor_scale[p] = St;
        }
        __syncwarp();  // every lane's stores precede lane 0's fence: a release
        if (lane == 0) {
          __threadfence();
          atomicAdd(cnt + p, 1u);
        }
      }
    }
  }
  badmax = __reduce_max_sync(0xffffffffu, badmax);
  if (lane == 0 && a.status) {
    if (badmax >= 0x7f800000u) atomicOr(a.status, FOS_STATUS_NONFINITE);
  }
  if (timed_out && a.status) atomicOr(a.status, FOS_STATUS_TIMEOUT);
}

}  // namespace

size_t pipe_ring_bytes() { return (size_t)kRing * sizeof(PipeRecord); }

// Cooperative persistent launch: one CTA per resident slot, looked up once
// per device and kernel variant.
static constexpr int kMaxDevices = 64;

template <bool F46, bool SR, bool RHT, bool SWZ, bool DENSE>
static cudaError_t launch_pipe_t(const QuantArgs& a, int batch, uint32_t* amax_ws, uint32_t* cnt,
                                 void* ring, cudaStream_t st) {
  static std::atomic<int> grid_of[kMaxDevices];
  auto kern = k_q1x16_pipe<F46, SR, RHT, SWZ, DENSE>;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return cudaErrorNotSupported;
  int grid = grid_of[dev].load(std::memory_order_relaxed);
  if (grid == 0) {
    int sms = 0, per_sm = 0, coop = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, 0) != cudaSuccess)
      return cudaErrorNotSupported;
    grid = (coop && per_sm >= 1) ? sms * per_sm : -1;
    grid_of[dev].store(grid, std::memory_order_relaxed);
  }
  if (grid < 1) return cudaErrorNotSupported;
  QuantArgs args = a;
  int b = batch;
  PipeRecord* r = reinterpret_cast<PipeRecord*>(ring);
  void* params[] = {&args, &b, &amax_ws, &cnt, &r};
  const cudaError_t e = cudaLaunchCooperativeKernel((const void*)kern, dim3(grid), dim3(kThreads), params, 0, st);
  if (e == cudaErrorCooperativeLaunchTooLarge) {
    (void)cudaGetLastError();
    return cudaErrorNotSupported;
  }
  return e;
}

cudaError_t launch_q1x16_pipe(const QuantArgs& a, int batch, int fmt, bool sr, bool rht, bool swz,
                              bool dense, uint32_t* amax_ws, uint32_t* cnt, void* ring, cudaStream_t st) {
  const bool f46 = fmt == 0;
  if (dense) swz = false;
#define FOS_L(F, S, R, W, D) return launch_pipe_t<F, S, R, W, D>(a, batch, amax_ws, cnt, ring, st)
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

}  // namespace fos
