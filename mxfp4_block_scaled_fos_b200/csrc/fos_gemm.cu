// fos_gemm.cu -- the consumer of the quantizer's output: an NVFP4
// block-scaled GEMM on the sm_100a tensor cores,
//   D[m][n] = (S_tA * S_tB) * sum_k A[m][k] * B[n][k],
// with A and B given as packed E2M1 codes and E4M3 16-element block scales
// in the tensor-core layout that fos_quantize writes with
// FOS_FLAG_SCALE_SWIZZLED, and S_t their FP32 per-tensor scales.
//
// Sources: Ultralytics glossary "FP4", "Como funciona FP4" (NVFP4: 16
// values, E4M3 block scale, FP32 tensor scale) and "Inferencia e
// Treinamento FP4" (FP4 matrix multiplication on Blackwell tensor cores);
// Hugging Face transformers doc "Four Over Six", introduction (the codes
// feed FP4 GEMMs on Blackwell).
//
// Persistent: one CTA per SM walks 128 x 256 tiles of D (128 x 128 when N
// is not a multiple of 256), grouped by 8 tile rows for L2 reuse of B, with
// 6 warps:
//   warp 0     TMA producer: per 256-wide K step, the A and B code tiles
//              (128 rows x 128 bytes each, 128-byte swizzle) as 2D tensor
//              copies and the four 512-byte scale atoms of each as one
//              2 KB bulk copy per 128 rows, into a 4-stage (6 for 128 x 128)
//              shared-memory ring;
//   warp 1     allocates the tensor memory; one thread copies the stage's
//              scale atoms into tensor memory (tcgen05.cp 32x128b.warpx4)
//              and issues the four K=64 tcgen05.mma of the stage
//              (kind::mxf4nvf4, block16, f32 accumulator in tensor memory);
//   warps 2-5  epilogue: tcgen05.ld of the accumulator (each warp its
//              32-lane quarter), scale by S_tA * S_tB, store bf16 or f32.
// Every tcgen05.mma (and every scale copy) holds the tensor pipe for about
// the same time whatever its N, so the 256-wide tile does twice the work per
// instruction: 8192^3 in 0.387 ms against 0.571 ms with 128 x 128 tiles.
// Its accumulator takes 256 of the 512 tensor-memory columns and the scale
// buffers most of the rest, so it is single-buffered: the epilogue releases
// it as soon as its last columns are in registers.  128 x 128 tiles keep two
// accumulators, so that a tile's epilogue runs while the next one's MMAs are
// issued.  The shared-memory ring and its barriers run on across tiles.
// Every mbarrier wait is bounded: after the limit the kernel sets
// FOS_STATUS_TIMEOUT, stops issuing work, waits (bounded) for its own copies
// in flight, frees its tensor memory and returns.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "fos.h"
#include "fos_internal.h"

namespace fos {

namespace {

constexpr int BM = 128, BK = 256;                // BK in FP4 elements (128 bytes)
constexpr int kTileA = BM * BK / 2;              // 16384 bytes
constexpr int kSFRowTile = 2048;                 // one 128-row tile's 4 scale atoms per K step
constexpr int kSFImage = 4096;                   // one 128 x 256-bit scale copy source (wide layout)
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr int kGroupM = 8;                       // tile rows per group of the tile order
constexpr uint32_t kWaitLimit = 1u << 22;        // polls of one mbarrier wait

// The tile shape BM x BN of one CTA and what follows from it.  BN = 256
// gives each tcgen05.mma twice the work of BN = 128 for the same issue cost
// (measured: an N = 256 MMA takes as long as an N = 128 one here), at the
// price of one accumulator buffer instead of two: 256 tensor-memory columns
// of accumulator leave room only for the scale buffers.
//
// WIDE: the scales come as copy-source images of the 128 x 256-bit
// tensor-memory copy (k_expand_sf): 6 copies per K step at BN = 256 instead
// of 12 of 32 x 128 bits, for 4 times the scale bytes in shared memory.
template <int BN, bool WIDE = false>
struct Cfg {
  static constexpr int kStages = WIDE ? (BN == 128 ? 4 : 3) : (BN == 128 ? 6 : 4);
  static constexpr int kTileB = BN * BK / 2;
  static constexpr int kSFA = WIDE ? 2 * kSFImage : kSFRowTile;                    // A scales per stage
  static constexpr int kSFB = (BN / 128) * (WIDE ? 2 * kSFImage : kSFRowTile);     // B scales per stage
  static constexpr uint32_t kStageTx = kTileA + kTileB + kSFA + kSFB;
  static constexpr int kAcc = BN == 128 ? 2 : 1;         // accumulator buffers (kAcc * BN <= 256 columns)
  // tensor memory: accumulators from column 0; A scales 256 + 16 * (k step &
  // 1) (4 columns per K-64 group); B scales 288 + (BN / 8) * (k step & 1)
  // (BN / 32 columns per K-64 group: 4 per 128 rows)
  static constexpr uint32_t kColSFA = 256, kColSFB = 288;
  static constexpr uint32_t kSFBGroup = BN / 32;
  // dynamic shared memory layout (from a 1024-byte aligned base)
  static constexpr int kOffA = 0;
  static constexpr int kOffB = kOffA + kStages * kTileA;
  static constexpr int kOffSFA = kOffB + kStages * kTileB;
  static constexpr int kOffSFB = kOffSFA + kStages * kSFA;
  static constexpr int kOffBar = kOffSFB + kStages * kSFB;  // full[S], empty[S], acc_full[2], acc_empty[2]
  static constexpr int kOffTmem = kOffBar + (2 * kStages + 4) * 8;
  static constexpr int kOffFlag = kOffTmem + 8;
  static constexpr int kSmemBytes = kOffFlag + 8 + 1024;    // + alignment slack
  // instruction descriptor: kind::mxf4nvf4, A and B E2M1, K-major, UE4M3
  // scales, M = 128, N = BN, K = 64 per instruction
  static constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                                     ((uint32_t)(BM >> 4) << 24);
  static_assert(kSmemBytes <= 227 * 1024, "shared memory");
  static_assert(kColSFB + 2 * (BN / 8) <= kTmemCols && kAcc * BN <= 256, "tensor memory");
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" :: "r"(bar), "r"(bytes) : "memory");
}

// Bounded wait for the phase with the given parity; false if it ran out.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  for (uint32_t it = 0; it < kWaitLimit; ++it) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done) : "r"(bar), "r"(parity) : "memory");
    if (done) return true;
  }
  return false;
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      :: "r"(dst), "l"(map), "r"(x), "r"(y), "r"(bar) : "memory");
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               :: "r"(dst), "l"(src), "r"(bytes), "r"(bar) : "memory");
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (tile base 1024-byte aligned).
__device__ __forceinline__ uint64_t desc_sw128(uint32_t addr) {
  return (uint64_t)((addr & 0x3FFFF) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Descriptor of one 4 KB wide copy source (128 rows of 32 bytes, no
// swizzle): the two 16-byte core-matrix columns of an 8-row group 128 bytes
// apart, 8-row groups 256 bytes apart.
__device__ __forceinline__ uint64_t desc_sf_wide(uint32_t addr) {
  return (uint64_t)((addr & 0x3FFFF) >> 4) | ((uint64_t)(128 >> 4) << 16) | ((uint64_t)(256 >> 4) << 32) |
         ((uint64_t)1 << 46);
}

// Descriptor of one 512-byte scale atom (32 rows of 16 bytes, no swizzle,
// 8-row groups 128 bytes apart) as the source of tcgen05.cp.
__device__ __forceinline__ uint64_t desc_sf(uint32_t addr) {
  return (uint64_t)((addr & 0x3FFFF) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(128 >> 4) << 32) |
         ((uint64_t)1 << 46);
}

__device__ __forceinline__ void umma(uint32_t tmem_c, uint64_t da, uint64_t db, uint32_t idesc, uint32_t tsfa,
                                     uint32_t tsfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
      :: "r"(tmem_c), "l"(da), "l"(db), "r"(idesc), "r"(accumulate), "r"(tsfa), "r"(tsfb) : "memory");
}

__device__ __forceinline__ void tmem_cp_sf(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" :: "r"(taddr), "l"(sdesc) : "memory");
}

// 128 lanes x 32 bytes from a wide copy source: lane l gets its row l.
__device__ __forceinline__ void tmem_cp_sf_wide(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.128x256b [%0], %1;" :: "r"(taddr), "l"(sdesc) : "memory");
}

// 32 bytes to global memory in one store; p 32-byte aligned.
__device__ __forceinline__ void st_global_v8(void* p, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                             uint32_t a4, uint32_t a5, uint32_t a6, uint32_t a7) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};"
               :: "l"(p), "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(a4), "r"(a5), "r"(a6), "r"(a7) : "memory");
}

__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" :: "r"(bar) : "memory");
}

struct GemmArgs {
  const uint8_t* sfa;  // swizzled scales of A (E4M3)
  const uint8_t* sfb;
  const float* sta;    // S_t of A and of B
  const float* stb;
  void* d;
  long long ldd;       // elements
  int M, N, K;
  int f32_out;
  int wide_st;         // rows of d 32-byte aligned: 256-bit stores
  long long sf_col_tiles;  // K / 64 (4-scale column tiles per 128-row tile)
  uint32_t* status;
};

// Tile t of the persistent order -> (tile row, tile column): groups of
// kGroupM tile rows, column-major inside a group.
__device__ __forceinline__ void tile_coords(int t, int ntm, int ntn, int& tm, int& tn) {
  const int per_group = kGroupM * ntn;
  const int grp = t / per_group;
  const int first = grp * kGroupM;
  const int gm = min(kGroupM, ntm - first);
  const int r = t - grp * per_group;
  tm = first + r % gm;
  tn = r / gm;
}

template <int BN, bool WIDE>
__global__ void __launch_bounds__(kThreads, 1)
    k_gemm_nvfp4(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                 const GemmArgs g) {
  using C = Cfg<BN, WIDE>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar_full = sbase + C::kOffBar, bar_empty = bar_full + 8 * S;
  const uint32_t bar_accf = bar_empty + 8 * S, bar_acce = bar_accf + 16;
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + C::kOffTmem);
  volatile uint32_t* fail = reinterpret_cast<volatile uint32_t*>(smem + C::kOffFlag);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ksteps = g.K / BK;
  const int ntm = g.M / BM, ntn = g.N / BN, ntiles = ntm * ntn;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_accf + 8 * b, 1);
      mbar_init(bar_acce + 8 * b, 4);  // one arrive per epilogue warp
    }
    *fail = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {  // tensor memory for the accumulators and the scale buffers
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 :: "r"(sbase + C::kOffTmem), "r"(kTmemCols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // producer: k step number `it` counts on across this CTA's tiles
      int it = 0;
      for (int t = blockIdx.x; t < ntiles && !*fail; t += gridDim.x) {
        int tm, tn;
        tile_coords(t, ntm, ntn, tm, tn);
        for (int kt = 0; kt < ksteps; ++kt, ++it) {
          const int s = it % S;
          if (it >= S && !mbar_wait(bar_empty + 8 * s, ((it / S) - 1) & 1)) { *fail = 1; break; }
          const uint32_t fb = bar_full + 8 * s;
          mbar_expect_tx(fb, C::kStageTx);
          tma_load_2d(sbase + C::kOffA + s * kTileA, &map_a, kt * (BK / 2), tm * BM, fb);
          tma_load_2d(sbase + C::kOffB + s * C::kTileB, &map_b, kt * (BK / 2), tn * BN, fb);
          if (WIDE) {
            // the K step's copy sources: A's of tile row tm, B's of tile column tn
            bulk_load(sbase + C::kOffSFA + s * C::kSFA, g.sfa + ((long long)tm * ksteps + kt) * C::kSFA, C::kSFA,
                      fb);
            bulk_load(sbase + C::kOffSFB + s * C::kSFB, g.sfb + ((long long)tn * ksteps + kt) * C::kSFB, C::kSFB,
                      fb);
          } else {
            // the 4 scale atoms of each 128-row tile, scale columns [16 kt, +16)
            bulk_load(sbase + C::kOffSFA + s * kSFRowTile, g.sfa + ((long long)tm * g.sf_col_tiles + 4 * kt) * 512,
                      kSFRowTile, fb);
#pragma unroll
            for (int h = 0; h < BN / 128; ++h)
              bulk_load(sbase + C::kOffSFB + s * C::kSFB + h * kSFRowTile,
                        g.sfb + ((long long)(tn * (BN / 128) + h) * g.sf_col_tiles + 4 * kt) * 512, kSFRowTile,
                        fb);
          }
        }
      }
      // before leaving, every copy this thread started must have landed
      for (int j = (it > S ? it - S : 0); j < it; ++j)
        if (!mbar_wait(bar_full + 8 * (j % S), (j / S) & 1)) *fail = 1;
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int it = 0, lt = 0;
      for (int t = blockIdx.x; t < ntiles && !*fail; t += gridDim.x, ++lt) {
        const int acc = lt % C::kAcc;
        // the epilogue must have drained this accumulator (tile lt - kAcc)
        if (lt >= C::kAcc && !mbar_wait(bar_acce + 8 * acc, ((lt / C::kAcc) - 1) & 1)) { *fail = 1; break; }
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const uint32_t tacc = tmem + (uint32_t)(acc * BN);
        for (int kt = 0; kt < ksteps; ++kt, ++it) {
          const int s = it % S;
          if (*fail || !mbar_wait(bar_full + 8 * s, (it / S) & 1)) { *fail = 1; break; }
          asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
          const uint32_t sfa = tmem + C::kColSFA + 16u * (it & 1);
          const uint32_t sfb = tmem + C::kColSFB + 4u * C::kSFBGroup * (it & 1);
          if (WIDE) {
            // a source holds two atoms side by side -> 8 columns: A's K-64
            // groups (0, 1) and (2, 3); B likewise at BN = 128, and at
            // BN = 256 group j of both 128-row tiles (columns 8 j .. 8 j + 7)
            const uint32_t src_a = sbase + C::kOffSFA + s * C::kSFA, src_b = sbase + C::kOffSFB + s * C::kSFB;
            tmem_cp_sf_wide(sfa, desc_sf_wide(src_a));
            tmem_cp_sf_wide(sfa + 8, desc_sf_wide(src_a + kSFImage));
#pragma unroll
            for (int c = 0; c < C::kSFB / kSFImage; ++c)
              tmem_cp_sf_wide(sfb + 8 * c, desc_sf_wide(src_b + c * kSFImage));
          } else {
            // scale atom j of each 128-row tile h -> 4 columns (K-64 group j);
            // B's groups hold BN / 32 columns, its row tiles 4 columns apart
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              tmem_cp_sf(sfa + 4 * j, desc_sf(sbase + C::kOffSFA + s * kSFRowTile + 512 * j));
#pragma unroll
              for (int h = 0; h < BN / 128; ++h)
                tmem_cp_sf(sfb + C::kSFBGroup * j + 4 * h,
                           desc_sf(sbase + C::kOffSFB + s * C::kSFB + h * kSFRowTile + 512 * j));
            }
          }
          const uint64_t da = desc_sw128(sbase + C::kOffA + s * kTileA);
          const uint64_t db = desc_sw128(sbase + C::kOffB + s * C::kTileB);
#pragma unroll
          for (int j = 0; j < 4; ++j)  // K = 64 (32 bytes) per instruction
            umma(tacc, da + 2 * j, db + 2 * j, C::kIdesc, sfa + 4 * j, sfb + C::kSFBGroup * j, (kt | j) != 0);
          umma_commit(bar_empty + 8 * s);  // the stage's smem is free once these MMAs are done
        }
        umma_commit(bar_accf + 8 * acc);  // this tile's accumulator is complete
      }
    }
  } else {
    // epilogue warps 2..5: TMEM lanes 32 * (warp % 4) ..
    const int q = warp & 3;
    const float alpha = __fmul_rn(g.sta[0], g.stb[0]);
    int lt = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++lt) {
      const int acc = lt % C::kAcc;
      const bool ok = mbar_wait(bar_accf + 8 * acc, (lt / C::kAcc) & 1);
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      if (!ok) *fail = 1;
      if (!ok || *fail) break;
      int tm, tn;
      tile_coords(t, ntm, ntn, tm, tn);
      const long long row = (long long)tm * BM + 32 * q + lane;
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 32) {
        uint32_t r[32];
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
            "%13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
            : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
              "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
              "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
              "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
              "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
            : "r"(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(acc * BN + c0)));
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
        if (c0 + 32 == BN) {
          // the last columns are in registers: the MMA warp may reuse the
          // accumulator while they are converted and stored
          asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
          __syncwarp();
          if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(bar_acce + 8 * acc) : "memory");
        }
        const long long col = (long long)tn * BN + c0;
        if (g.f32_out && g.wide_st) {
          // each lane's 128 bytes of its row in 4 stores of full 32-byte sectors
          float* dp = static_cast<float*>(g.d) + row * g.ldd + col;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            uint32_t o[8];
#pragma unroll
            for (int h = 0; h < 8; ++h) o[h] = __float_as_uint(__fmul_rn(__uint_as_float(r[8 * k + h]), alpha));
            st_global_v8(dp + 8 * k, o[0], o[1], o[2], o[3], o[4], o[5], o[6], o[7]);
          }
        } else if (g.f32_out) {
          float4* dp = reinterpret_cast<float4*>(static_cast<float*>(g.d) + row * g.ldd + col);
#pragma unroll
          for (int k = 0; k < 8; ++k)
            dp[k] = make_float4(__fmul_rn(__uint_as_float(r[4 * k]), alpha),
                                __fmul_rn(__uint_as_float(r[4 * k + 1]), alpha),
                                __fmul_rn(__uint_as_float(r[4 * k + 2]), alpha),
                                __fmul_rn(__uint_as_float(r[4 * k + 3]), alpha));
        } else if (g.wide_st) {
          uint16_t* dp = static_cast<uint16_t*>(g.d) + row * g.ldd + col;
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            uint32_t o[8];
#pragma unroll
            for (int h = 0; h < 8; ++h) {
              const __nv_bfloat162 b2 = __floats2bfloat162_rn(__fmul_rn(__uint_as_float(r[16 * k + 2 * h]), alpha),
                                                              __fmul_rn(__uint_as_float(r[16 * k + 2 * h + 1]), alpha));
              o[h] = *reinterpret_cast<const uint32_t*>(&b2);
            }
            st_global_v8(dp + 16 * k, o[0], o[1], o[2], o[3], o[4], o[5], o[6], o[7]);
          }
        } else {
          uint4* dp = reinterpret_cast<uint4*>(static_cast<uint16_t*>(g.d) + row * g.ldd + col);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            uint32_t o[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              const __nv_bfloat162 b2 = __floats2bfloat162_rn(__fmul_rn(__uint_as_float(r[8 * k + 2 * h]), alpha),
                                                              __fmul_rn(__uint_as_float(r[8 * k + 2 * h + 1]), alpha));
              o[h] = *reinterpret_cast<const uint32_t*>(&b2);
            }
            dp[k] = make_uint4(o[0], o[1], o[2], o[3]);
          }
        }
      }
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 1) {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem), "r"(kTmemCols) : "memory");
  }
  if (threadIdx.x == 0 && *fail && g.status) atomicOr(g.status, FOS_STATUS_TIMEOUT);
}

// The wide layout's copy sources from the swizzled scales (512-byte atoms
// of 128 rows x 4 scales, atom (t, c) at (t * col_tiles + c) * 512; row r of
// an atom holds the scales of rows r, r + 32, r + 64, r + 96).  A source is
// 4 KB: row l (32 bytes at (l >> 3) * 256 + (l & 7) * 16, second half 128
// bytes on) is row l % 32 of two atoms.  pair_tiles = 0: source (t, kt, s)
// pairs atoms (t, 4 kt + 2 s) and (t, 4 kt + 2 s + 1); pair_tiles = 1:
// source (p, kt, j) pairs atoms (2 p, 4 kt + j) and (2 p + 1, 4 kt + j).
// One thread per 16 bytes of the output, in output order; both operands'
// expansions in one launch (A's chunks first, then B's).
struct ExpandJob {
  const uint8_t* src;
  uint8_t* dst;
  long long col_tiles, ksteps;
  unsigned long long nchunks;   // 16-byte chunks of dst: images * 256
  int pair_tiles;
};

__device__ __forceinline__ void expand_chunk(const ExpandJob& j, unsigned long long q) {
  const unsigned long long img = q >> 8;
  const int w = (int)(q & 255);
  const int half = (w >> 3) & 1, l = ((w >> 4) << 3) | (w & 7);
  long long tile, ctile;
  if (!j.pair_tiles) {
    const long long r = (long long)(img >> 1), kt = r % j.ksteps;
    tile = r / j.ksteps;
    ctile = 4 * kt + 2 * (long long)(img & 1) + half;
  } else {
    const long long r = (long long)(img >> 2), kt = r % j.ksteps;
    tile = 2 * (r / j.ksteps) + half;
    ctile = 4 * kt + (long long)(img & 3);
  }
  *reinterpret_cast<uint4*>(j.dst + q * 16) =
      *reinterpret_cast<const uint4*>(j.src + (tile * j.col_tiles + ctile) * 512 + (l & 31) * 16);
}

__global__ void __launch_bounds__(256) k_expand_sf(const ExpandJob ja, const ExpandJob jb) {
  const unsigned long long n = ja.nchunks + jb.nchunks;
  for (unsigned long long q = blockIdx.x * (unsigned long long)blockDim.x + threadIdx.x; q < n;
       q += (unsigned long long)gridDim.x * blockDim.x) {
    if (q < ja.nchunks) expand_chunk(ja, q);
    else                expand_chunk(jb, q - ja.nchunks);
  }
}

// ---------------------------------------------------------------- host
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2D map over packed codes [rows][ld bytes]: boxes of 128 bytes x box_rows
// rows, 128-byte swizzle.
bool make_code_map(CUtensorMap* m, const void* codes, long long rows, long long kbytes, long long ld,
                   cuuint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)kbytes, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)ld};
  const cuuint32_t box[2] = {128, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(codes), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BN, bool WIDE = false>
cudaError_t launch_bn(const fos_qtensor* a, const fos_qtensor* b, int M, int N, int K, const GemmArgs& g,
                      cudaStream_t st) {
  CUtensorMap ma, mb;
  if (!make_code_map(&ma, a->codes, M, K / 2, a->codes_ld, BM) ||
      !make_code_map(&mb, b->codes, N, K / 2, b->codes_ld, BN))
    return cudaErrorNotSupported;
  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [] {
    attr_err = cudaFuncSetAttribute(k_gemm_nvfp4<BN, WIDE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    Cfg<BN, WIDE>::kSmemBytes);
  });
  if (attr_err != cudaSuccess) return attr_err;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
      cudaSuccess)
    return cudaErrorNotSupported;
  const int ntiles = (M / BM) * (N / BN);
  k_gemm_nvfp4<BN, WIDE><<<dim3(ntiles < sms ? ntiles : sms), kThreads, Cfg<BN, WIDE>::kSmemBytes, st>>>(ma, mb, g);
  return cudaGetLastError();
}

}  // namespace

size_t gemm_workspace_bytes(long long M, long long N, long long K) {
  return (size_t)4 * 512 * (size_t)((M / 128) * (K / 64) + (N / 128) * (K / 64));
}

static ExpandJob expand_job(const uint8_t* src, long long rows, int K, int pair_tiles, uint8_t* dst) {
  ExpandJob j;
  j.src = src;
  j.dst = dst;
  j.col_tiles = K / 64;
  j.ksteps = K / 256;
  j.nchunks = (unsigned long long)(rows / 128) * j.ksteps * 2 * 256;
  j.pair_tiles = pair_tiles;
  return j;
}

static cudaError_t expand_sf(const ExpandJob& ja, const ExpandJob& jb, cudaStream_t st) {
  const unsigned long long blocks = (ja.nchunks + jb.nchunks + 255) / 256;
  k_expand_sf<<<(unsigned)(blocks < 148 * 8 ? blocks : 148 * 8), 256, 0, st>>>(ja, jb);
  return cudaGetLastError();
}

// 128 x 256 tiles when N allows them, else 128 x 128.
cudaError_t launch_gemm_nvfp4(const fos_qtensor* a, const fos_qtensor* b, int M, int N, int K, void* d,
                              long long ldd, int f32_out, uint32_t* status, cudaStream_t st, void* workspace) {
  GemmArgs g;
  g.sfa = a->scales;
  g.sfb = b->scales;
  g.sta = a->tensor_scale;
  g.stb = b->tensor_scale;
  g.d = d;
  g.ldd = ldd;
  g.M = M;
  g.N = N;
  g.K = K;
  g.f32_out = f32_out;
  g.wide_st = (reinterpret_cast<uintptr_t>(d) % 32 == 0) && (ldd * (f32_out ? 4 : 2)) % 32 == 0;
  g.sf_col_tiles = K / 64;
  g.status = status;
  const bool bn256 = N % 256 == 0;
  if (workspace) {  // the wide layout: expand both operands' scales, then 6 or 4 copies per K step
    uint8_t* ea = static_cast<uint8_t*>(workspace);
    uint8_t* eb = ea + gemm_workspace_bytes(M, 0, K);
    const cudaError_t e = expand_sf(expand_job(a->scales, M, K, 0, ea), expand_job(b->scales, N, K, bn256 ? 1 : 0, eb),
                                    st);
    if (e != cudaSuccess) return e;
    g.sfa = ea;
    g.sfb = eb;
    return bn256 ? launch_bn<256, true>(a, b, M, N, K, g, st) : launch_bn<128, true>(a, b, M, N, K, g, st);
  }
  return bn256 ? launch_bn<256>(a, b, M, N, K, g, st) : launch_bn<128>(a, b, M, N, K, g, st);
}

}  // namespace fos
