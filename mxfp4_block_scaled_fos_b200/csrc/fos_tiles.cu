// fos_tiles.cu -- NVFP4 quantizers that need both orientations of a tile:
//   * 1x16 rowwise + colwise ("transposed inputs" option of the Hugging Face
//     transformers doc "Four Over Six", usage section): x and x^T are each
//     quantized with 16-element blocks along their rows, one read of x;
//   * 16x16 2D block scaling (same section): one scale and one 4/6 choice per
//     16x16 tile, written row-major and as its exact transpose.
//
// 1x16 rowwise + colwise (k_dual_warp): every warp takes units of 4
// adjacent 16x16 tiles, loaded straight from global memory, and transposes
// them through its own shared buffer; no CTA barrier in the loop.
// 16x16 (k_2d16x16): a CTA of 256 threads walks a strip of up to 8 sub-tiles
// of 64 rows x 128 columns (16 KB of bf16) down the tensor.  Each thread
// loads the two tile rows it quantizes straight from global memory, one
// sub-tile ahead; the transposed codes go through shared memory.
// Stochastic-rounding bytes are drawn once per 16 source elements (one Philox
// call per rowwise block) and shared by both orientations through shared
// memory.
#include <atomic>

#include "fos_core.cuh"

namespace fos {

namespace {

constexpr int kThreads = 256;
constexpr int kSubRows = 64;
constexpr int kSubCols = 128;
constexpr int kStrip = 8;  // most sub-tiles per CTA strip (512 rows: one 32-bit word
                           // of the transposed copy's choice bitmap per tile column)
#ifndef FOS_2D_MIN_BLOCKS
#define FOS_2D_MIN_BLOCKS 3
#endif

template <bool SWZ>
__device__ __forceinline__ long long scale_off(const OutDesc& o, int b, long long R, long long c) {
  if (SWZ) return (long long)b * o.scales_bs + swz_offset(R, c, o.col_tiles);
  return (long long)b * o.scales_bs + R * o.scales_ld + c;
}

__device__ __forceinline__ void store_codes8(const OutDesc& o, int b, long long R, long long byte_col,
                                             uint32_t w0, uint32_t w1) {
  *reinterpret_cast<uint2*>(o.codes + (long long)b * o.codes_bs + R * o.codes_ld + byte_col) =
      make_uint2(w0, w1);
}

// Quantize the pair P (blocks A, B) with per-block amax bits (ma, mb):
// returns codes, scale bytes and picks (SR re-rounding done by the caller).
template <bool F46>
struct PairResult {
  uint32_t ca[2], cb[2];
  uint32_t sa, sb;
  float inva, invb;
  uint32_t pa, pb;
};

template <bool F46>
__device__ __forceinline__ PairResult<F46> quant_pair(const float2 (&P)[16], uint32_t ma, uint32_t mb,
                                                      const TScale& St, const float2* tab, float nz) {
  PairResult<F46> r;
  uint32_t s6a, s4a, s6b, s4b;
  cand_scales<F46>(__uint_as_float(ma), St, s6a, s4a);
  cand_scales<F46>(__uint_as_float(mb), St, s6b, s4b);
  const float2 t6a = tab[s6a], t6b = tab[s6b];
  const Cand c6 = candidate<F46>(P, make_float2(t6a.y, t6b.y), make_float2(-t6a.x, -t6b.x), nz);
  r.ca[0] = c6.ca[0]; r.ca[1] = c6.ca[1]; r.cb[0] = c6.cb[0]; r.cb[1] = c6.cb[1];
  r.sa = s6a; r.sb = s6b; r.inva = t6a.y; r.invb = t6b.y; r.pa = 0; r.pb = 0;
  if (F46) {
    const float2 t4a = tab[s4a], t4b = tab[s4b];
    const Cand c4 = candidate<true>(P, make_float2(t4a.y, t4b.y), make_float2(-t4a.x, -t4b.x), nz);
    r.pa = c4.err.x < c6.err.x;
    r.pb = c4.err.y < c6.err.y;
    if (r.pa) { r.ca[0] = c4.ca[0]; r.ca[1] = c4.ca[1]; r.sa = s4a; r.inva = t4a.y; }
    if (r.pb) { r.cb[0] = c4.cb[0]; r.cb[1] = c4.cb[1]; r.sb = s4b; r.invb = t4b.y; }
  }
  return r;
}

// Nibbles of a (8) into the low halves of 8 bytes, b into the high halves:
// byte k = a_k | b_k << 4.
__device__ __forceinline__ unsigned long long zip_nibbles(uint32_t a, uint32_t b) {
  auto spread = [](unsigned long long x) {
    x = (x | (x << 16)) & 0x0000FFFF0000FFFFull;
    x = (x | (x << 8)) & 0x00FF00FF00FF00FFull;
    x = (x | (x << 4)) & 0x0F0F0F0F0F0F0F0Full;
    return x;
  };
  return spread(a) | (spread(b) << 4);
}

// --------------------------------------------------------------------------
// 1x16 rowwise + colwise from one read, warp-based.  grid (CTAs, batch);
// every warp takes units of 4 horizontally adjacent 16x16 tiles, 8 lanes per
// tile.  Lane i of a tile first quantizes the tile's rows 2i and 2i+1 (one
// rowwise block each); the tile then goes through this warp's shared buffer
// so that lane j quantizes its columns 2j and 2j+1 (one colwise block each).
// Blocks go one at a time through the rowwise quantizer's per-block step,
// which keeps the kernel at 3 CTAs per SM with stochastic rounding.  With stochastic rounding the Philox bytes of each rowwise block (one call
// per 16 consecutive elements) take the same way, so both orientations use
// the byte of the same source element.  Choice bits go into zeroed bitmaps
// with atomics.  No CTA barrier in the loop.
constexpr int kDwGroup = 16 * 32 + 32;   // bytes per tile in the buffer: 16 rows of
                                         // 32 bytes, padded so the 4 tiles' column
                                         // reads fall into distinct banks
constexpr int kDwRGroup = 16 * 16 + 16;  // Philox bytes per tile: 16 rows of 16,
                                         // padded so that the 4 tiles' colwise byte
                                         // reads fall into distinct banks
#ifndef FOS_DUALW_MIN_BLOCKS
#define FOS_DUALW_MIN_BLOCKS 3
#endif
#ifndef FOS_DUALW_MIN_BLOCKS_SR
#define FOS_DUALW_MIN_BLOCKS_SR 3
#endif

// 4 bits at lanes i, 8+i, 16+i, 24+i of a ballot -> bits 0..3
__device__ __forceinline__ uint32_t gather4(uint32_t bal, int i) {
  const uint32_t x = bal >> i;
  return (x & 1u) | ((x >> 7) & 2u) | ((x >> 14) & 4u) | ((x >> 21) & 8u);
}

__device__ __forceinline__ void or_bits(uint8_t* bitmap, unsigned long long bit, uint32_t v) {
  if (!v) return;
  unsigned int* wp = reinterpret_cast<unsigned int*>(bitmap) + (bit >> 5);
  const unsigned long long vv = (unsigned long long)v << (bit & 31);
  if ((uint32_t)vv) atomicOr(wp, (uint32_t)vv);
  if ((uint32_t)(vv >> 32)) atomicOr(wp + 1, (uint32_t)(vv >> 32));
}

// One rowwise block of the dual kernel: row R of the tile at tile column
// tc, words w, Philox bytes rnd of its 16 elements.  Returns the 4/6 pick.
template <bool F46, bool SR, bool SWZ>
__device__ __forceinline__ uint32_t dual_row_block(const QuantArgs& a, int b, const uint4 (&w)[2], uint4 rnd,
                                                   long long R, uint32_t tc, bool valid, const float4* s_tab,
                                                   const TScale& ts, uint32_t& badmax) {
  const uint32_t W[8] = {w[0].x, w[0].y, w[0].z, w[0].w, w[1].x, w[1].y, w[1].z, w[1].w};
  float2 P[8];
  unpack_split(W, P);
  const uint32_t m = amax_bits_bf16(w);
  badmax = max(badmax, m);
  uint32_t codes[2], sc;
  bool pick;
  float inv;
  block_step<F46>(P, m, s_tab, ts, a.neg_zero, codes, sc, pick, inv);
  if (SR) sr_block1(P, inv, rnd, codes);
  if (valid) {
    store_codes8(a.row, b, R, (long long)tc * 8, codes[0], codes[1]);
    a.row.scales[scale_off<SWZ>(a.row, b, R, tc)] = (uint8_t)sc;
  }
  return pick && valid;
}

// Amax of the 16-row column blocks after the 16-wide transform (the colwise
// copy's tensor amax with FOS_FLAG_RHT16_COL).  One thread per (16-row
// strip, column pair): 16 32-bit loads (a warp reads 128 contiguous bytes
// per row), the seeded signs by row, the butterfly on the packed column pair,
// then a warp max and one atomicMax per warp into amax_col[b] (zeroed).
__global__ void __launch_bounds__(kThreads) k_amax_cols_rht(const QuantArgs a, uint32_t* amax_col) {
  const int b = blockIdx.y;
  const uint32_t mask16 = rht_sign_mask(a.seed);
  const uint32_t npair = (uint32_t)a.cols / 2, nunits = npair * ((uint32_t)a.rows / 16);
  const uint16_t* xb = a.x + (long long)b * a.x_bs;
  uint32_t m = 0;
  for (uint32_t u = blockIdx.x * kThreads + threadIdx.x; u < nunits; u += gridDim.x * kThreads) {
    const uint32_t strip = u / npair, cp = u - strip * npair;
    const uint16_t* p = xb + (long long)strip * 16 * a.ld + 2 * cp;
    float2 T[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      const uint32_t w = __ldg(reinterpret_cast<const uint32_t*>(p + (long long)r * a.ld)) ^
                         (((mask16 >> r) & 1u) ? 0x80008000u : 0u);
      T[r] = make_float2(bf_lo(w), bf_hi(w));
    }
    fwht16_pairs(T);
    uint32_t ma, mb;
    amax_bits_pairs(T, ma, mb);
    m = max(m, max(ma, mb));
  }
  m = __reduce_max_sync(0xffffffffu, m);
  if ((threadIdx.x & 31) == 0) {
    if (m >= 0x7f800000u) {
      if (a.status) atomicOr(a.status, FOS_STATUS_NONFINITE);
    } else if (m) {
      atomicMax(amax_col + b, m);
    }
  }
}

// RHTC: the colwise blocks are transformed along rows (the 16-wide RHT with
// the seeded signs by row position) and take their own S_t, from the amax
// words amax_col_ws of the transformed columns.
template <bool F46, bool SR, bool SWZ, bool ROW, bool RHTC>
__global__ void __launch_bounds__(kThreads, RHTC ? 2 : (SR ? FOS_DUALW_MIN_BLOCKS_SR : FOS_DUALW_MIN_BLOCKS))
    k_dual_warp(const QuantArgs a, FastDiv ntc4) {
  __shared__ __align__(16) float4 s_tab[128];
  __shared__ __align__(16) float4 s_tabc[RHTC ? 128 : 1];   // the colwise copy's table (RHTC)
  __shared__ __align__(16) uint8_t s_x[kThreads / 32][4 * kDwGroup];
  __shared__ __align__(16) uint8_t s_r[SR ? kThreads / 32 : 1][SR ? 4 * kDwRGroup : 16];
  const int b = blockIdx.y;
  const float St = tensor_scale_of(a, b, F46);
  const float StC = RHTC ? __fdiv_rn(__uint_as_float(a.amax_col_ws[b]), F46 ? 1792.0f : 2688.0f) : St;
  build_scale_table4(s_tab, St);
  if (RHTC) build_scale_table4(s_tabc, StC);
  const float4* tab_c = RHTC ? s_tabc : s_tab;
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    if (ROW && a.row.tensor_scale) a.row.tensor_scale[b] = St;
    if (a.col.tensor_scale) a.col.tensor_scale[b] = StC;
  }
  __syncthreads();
  const TScale ts = make_tscale(St);
  const TScale tsc = RHTC ? make_tscale(StC) : ts;
  const uint32_t mask16 = RHTC ? rht_sign_mask(a.seed) : 0u;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 3, i = lane & 7;
  const uint32_t ntr = a.rows / 16, ntc = a.cols / 16;
  const uint32_t nunits = ntr * ntc4.d;
  const long long gbase = a.elem_offset + (long long)b * a.rows * a.cols;
  uint8_t* xb = s_x[warp] + g * kDwGroup;
  uint8_t* rbuf = SR ? s_r[warp] + g * kDwRGroup : nullptr;
  uint32_t badmax = 0;
  for (uint32_t u = blockIdx.x * (kThreads / 32) + warp; u < nunits; u += gridDim.x * (kThreads / 32)) {
    const uint32_t trow = fdiv(u, ntc4), tq = u - trow * ntc4.d;
    const uint32_t tc = tq * 4 + g;
    const bool valid = tc < ntc;
    const long long r0 = (long long)trow * 16 + 2 * i;
    uint4 wa[2], wb[2];
    if (valid) {
      const uint4* pa = reinterpret_cast<const uint4*>(a.x + (long long)b * a.x_bs + r0 * a.ld + (long long)tc * 16);
      const uint4* pb = reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(pa) + a.ld);
      wa[0] = __ldg(pa); wa[1] = __ldg(pa + 1);
      wb[0] = __ldg(pb); wb[1] = __ldg(pb + 1);
    } else {
      wa[0] = wa[1] = wb[0] = wb[1] = make_uint4(0u, 0u, 0u, 0u);
    }
    // the tile into the warp's buffer (row r at byte 32 r), for the colwise pass
    reinterpret_cast<uint4*>(xb + (2 * i) * 32)[0] = wa[0];
    reinterpret_cast<uint4*>(xb + (2 * i) * 32)[1] = wa[1];
    reinterpret_cast<uint4*>(xb + (2 * i + 1) * 32)[0] = wb[0];
    reinterpret_cast<uint4*>(xb + (2 * i + 1) * 32)[1] = wb[1];
    uint4 ra = make_uint4(0u, 0u, 0u, 0u), rb = ra;
    if (SR) {
      ra = sr_bytes16(a.seed, gbase + r0 * a.cols + (long long)tc * 16);
      rb = sr_bytes16(a.seed, gbase + (r0 + 1) * a.cols + (long long)tc * 16);
      reinterpret_cast<uint4*>(rbuf)[2 * i] = ra;
      reinterpret_cast<uint4*>(rbuf)[2 * i + 1] = rb;
    }
    // ---------------- rowwise: row 2i, then row 2i+1, one block each
    uint32_t pra = 0, prb = 0;
    if (ROW) {
      pra = dual_row_block<F46, SR, SWZ>(a, b, wa, ra, r0, tc, valid, s_tab, ts, badmax);
      prb = dual_row_block<F46, SR, SWZ>(a, b, wb, rb, r0 + 1, tc, valid, s_tab, ts, badmax);
    }
    __syncwarp();
    // ---------------- colwise: column 2i, then column 2i+1 of the tile
    uint32_t pca = 0, pcb = 0;
    {
      uint32_t w[16];  // row r of the tile's columns 2i (low half) and 2i+1 (high half)
#pragma unroll
      for (int r = 0; r < 16; ++r) w[r] = *reinterpret_cast<const uint32_t*>(xb + r * 32 + 4 * i);
      uint32_t mc[2];
      float2 T[16];   // RHTC: row r of both columns after the transform
      if (RHTC) {
#pragma unroll
        for (int r = 0; r < 16; ++r) {
          const uint32_t wr = w[r] ^ (((mask16 >> r) & 1u) ? 0x80008000u : 0u);
          T[r] = make_float2(bf_lo(wr), bf_hi(wr));
        }
        fwht16_pairs(T);
        amax_bits_pairs(T, mc[0], mc[1]);
      } else {
        uint32_t h[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) h[k] = hmax_abs2(w[2 * k], w[2 * k + 1]);
        const uint32_t m = hmax_abs2(hmax_abs2(hmax_abs2(h[0], h[1]), hmax_abs2(h[2], h[3])),
                                     hmax_abs2(hmax_abs2(h[4], h[5]), hmax_abs2(h[6], h[7]))) & 0x7fff7fffu;
        mc[0] = (m & 0xffffu) << 16;
        mc[1] = m & 0xffff0000u;
      }
      badmax = max(badmax, max(mc[0], mc[1]));
#pragma unroll
      for (int hc = 0; hc < 2; ++hc) {
        float2 P[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          if (RHTC) P[k] = hc ? make_float2(T[k].y, T[k + 8].y) : make_float2(T[k].x, T[k + 8].x);
          else      P[k] = hc ? make_float2(bf_hi(w[k]), bf_hi(w[k + 8])) : make_float2(bf_lo(w[k]), bf_lo(w[k + 8]));
        }
        uint32_t codes[2], sc;
        bool pick;
        float inv;
        block_step<F46>(P, mc[hc], tab_c, tsc, a.neg_zero, codes, sc, pick, inv);
        if (SR) sr_block1_smem(P, inv, rbuf + 2 * i + hc, 16, codes);
        const long long c = (long long)tc * 16 + 2 * i + hc;
        if (valid) {
          store_codes8(a.col, b, c, (long long)trow * 8, codes[0], codes[1]);
          a.col.scales[scale_off<SWZ>(a.col, b, c, trow)] = (uint8_t)sc;
        }
        (hc ? pcb : pca) = pick && valid;
      }
    }
    __syncwarp();  // the buffers are rewritten by the next unit
    if (F46) {
      const uint32_t nbc = a.cols / 16;
      if (ROW && a.row.choice) {  // rows r0, r0+1: 4 consecutive blocks (tiles tq*4 ..) each
        const uint32_t ba = __ballot_sync(0xffffffffu, pra), bb = __ballot_sync(0xffffffffu, prb);
        if (lane < 8) {
          or_bits(a.row.choice, ((unsigned long long)b * a.rows + r0) * nbc + (unsigned long long)tq * 4,
                  gather4(ba, i));
          or_bits(a.row.choice, ((unsigned long long)b * a.rows + r0 + 1) * nbc + (unsigned long long)tq * 4,
                  gather4(bb, i));
        }
      }
      if (a.col.choice) {  // column c: block trow of [cols][rows/16]
        const unsigned long long c0 = (unsigned long long)tc * 16 + 2 * i;
        if (pca) or_bits(a.col.choice, ((unsigned long long)b * a.cols + c0) * ntr + trow, 1u);
        if (pcb) or_bits(a.col.choice, ((unsigned long long)b * a.cols + c0 + 1) * ntr + trow, 1u);
      }
    }
  }
  badmax = __reduce_max_sync(0xffffffffu, badmax);
  if (lane == 0 && badmax >= 0x7f800000u && a.status) atomicOr(a.status, FOS_STATUS_NONFINITE);
}

// --------------------------------------------------------------------------
// 16x16 2D block scaling.  grid (ceil(cols/128), ceil(rows/512), batch).
// In a sub-tile, 8 threads own one 16x16 tile; thread i holds rows 2i, 2i+1
// as the pair (A, B), so the per-row error trees come out of the pair code
// and the tree over the 16 row sums is a horizontal add plus three
// xor-shuffles.  Each thread loads its two 32-byte tile rows itself (one
// 256-bit load each where rows are 32-byte aligned: a warp's load covers 8
// rows x 128 contiguous bytes), one sub-tile ahead; shared memory only
// carries the transposed codes.
template <bool F46, bool SR, bool SWZ, bool ROW, bool COL>
__global__ void __launch_bounds__(kThreads, SR ? 2 : FOS_2D_MIN_BLOCKS) k_2d16x16(const QuantArgs a, int nsub) {
  __shared__ __align__(16) uint8_t s_tc[COL ? kSubCols * 32 : 16];
  // scale bytes, written out as 4-byte words: the sub-tile's rowwise scales
  // [64 rows][8 tile columns] and the strip's transposed-copy scales
  // [128 columns][32 tile rows]
  __shared__ __align__(16) uint8_t s_rsc[ROW ? kSubRows * 8 : 16];
  __shared__ __align__(16) uint8_t s_csc[COL ? kSubCols * 32 : 16];
  __shared__ float2 s_tab[128];
  __shared__ uint32_t s_bits[kSubRows / 16];   // rowwise picks of a sub-tile: tile row -> 8 tile columns
  __shared__ uint32_t s_cbits[kSubCols / 16];  // transposed copy: tile column -> 32 tile rows of the strip

  const int b = blockIdx.z;
  const int c0 = blockIdx.x * kSubCols;
  const int rs0 = blockIdx.y * (kSubRows * nsub);
  const float St = tensor_scale_of(a, b, F46);
  build_scale_table(s_tab, St);
  const TScale ts = make_tscale(St);
  if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) {
    if (ROW && a.row.tensor_scale) a.row.tensor_scale[b] = St;
    if (COL && a.col.tensor_scale) a.col.tensor_scale[b] = St;
  }
  if (threadIdx.x < kSubRows / 16) s_bits[threadIdx.x] = 0;
  if (threadIdx.x < kSubCols / 16) s_cbits[threadIdx.x] = 0;

  const int t = threadIdx.x;
  const int tile = t >> 3, i = t & 7;
  const int tr = tile >> 3, tc = tile & 7;   // tile row (0..3) and column (0..7)
  const long long ntc = a.cols / 16, ntr = a.rows / 16;
  const long long gbase = a.elem_offset + (long long)b * a.rows * a.cols;
  uint32_t bad = 0;

  // rows 2i, 2i+1 of this thread's tile in the sub-tile starting at row r0
  // (zero for a tile outside the tensor: rows and cols are multiples of 16)
  const bool al32 = (reinterpret_cast<uintptr_t>(a.x) & 31) == 0 && (a.ld & 15) == 0 && (a.x_bs & 15) == 0;
  // 4 consecutive scales of a row (4-aligned) form one aligned word; the
  // transposed codes of 32 rows one aligned 16-byte run
  const bool rsc_word = (a.row.scales_bs & 3) == 0 && (SWZ || (a.row.scales_ld & 3) == 0);
  const bool csc_word = (a.col.scales_bs & 3) == 0 && (SWZ || (a.col.scales_ld & 3) == 0);
  const bool cc16 = (a.col.codes_bs & 15) == 0 && (a.col.codes_ld & 15) == 0;
  const uint16_t* xb = a.x + (long long)b * a.x_bs;
  auto load_rows = [&](int r0, uint4 (&ra)[2], uint4 (&rb)[2]) {
    const long long gr = (long long)r0 + 16 * tr + 2 * i;
    const int gc = c0 + 16 * tc;
    if (gr < a.rows && gc < a.cols) {
      const uint16_t* p = xb + gr * a.ld + gc;
      if (al32) {
        ld_block256(p, ra);
        ld_block256(p + a.ld, rb);
      } else {
        ra[0] = __ldg(reinterpret_cast<const uint4*>(p));
        ra[1] = __ldg(reinterpret_cast<const uint4*>(p) + 1);
        rb[0] = __ldg(reinterpret_cast<const uint4*>(p + a.ld));
        rb[1] = __ldg(reinterpret_cast<const uint4*>(p + a.ld) + 1);
      }
    } else {
      ra[0] = ra[1] = rb[0] = rb[1] = make_uint4(0u, 0u, 0u, 0u);
    }
  };
  uint4 na[2], nb[2];
  load_rows(rs0, na, nb);
  for (int k = 0; k < nsub; ++k) {
    const int r0 = rs0 + k * kSubRows;
    if (r0 >= a.rows) break;
    const uint4 wa[2] = {na[0], na[1]}, wb[2] = {nb[0], nb[1]};
    if (k + 1 < nsub && r0 + kSubRows < a.rows) load_rows(r0 + kSubRows, na, nb);
    __syncthreads();  // the previous sub-tile's readers of s_tc, s_bits and s_cbits are done

    const long long gtr = (r0 >> 4) + tr;      // global tile row
    const long long gtc = (c0 >> 4) + tc;      // global tile column
    const bool valid = gtr < ntr && gtc < ntc; // uniform over the 8 threads of a tile
    uint32_t pick = 0;
    if (valid) {
      const int ra = 16 * tr + 2 * i;
      float2 P[16];
      unpack_pairs(wa, wb, P);
      // the 8 lanes of one tile are all valid or all invalid: shuffle among them
      const uint32_t gmask = 0xffu << (threadIdx.x & 24);
      uint32_t m = max(amax_bits_bf16(wa), amax_bits_bf16(wb));
      m = max(m, __shfl_xor_sync(gmask, m, 1));
      m = max(m, __shfl_xor_sync(gmask, m, 2));
      m = max(m, __shfl_xor_sync(gmask, m, 4));
      bad |= m >= 0x7f800000u;
      uint32_t s6, s4;
      cand_scales<F46>(__uint_as_float(m), ts, s6, s4);
      const float2 t6 = s_tab[s6];
      const Cand c6 = candidate<F46>(P, make_float2(t6.y, t6.y), make_float2(-t6.x, -t6.x), a.neg_zero);
      uint32_t ca[2] = {c6.ca[0], c6.ca[1]}, cb[2] = {c6.cb[0], c6.cb[1]};
      uint32_t s = s6;
      float inv = t6.y;
      if (F46) {
        const float2 t4 = s_tab[s4];
        const Cand c4 = candidate<true>(P, make_float2(t4.y, t4.y), make_float2(-t4.x, -t4.x), a.neg_zero);
        // tree over the 16 row sums: (2i)+(2i+1), then across threads
        float e6 = __fadd_rn(c6.err.x, c6.err.y), e4 = __fadd_rn(c4.err.x, c4.err.y);
#pragma unroll
        for (int sh = 1; sh < 8; sh *= 2) {
          e6 = __fadd_rn(e6, __shfl_xor_sync(gmask, e6, sh));
          e4 = __fadd_rn(e4, __shfl_xor_sync(gmask, e4, sh));
        }
        pick = e4 < e6;
        if (pick) { ca[0] = c4.ca[0]; ca[1] = c4.ca[1]; cb[0] = c4.cb[0]; cb[1] = c4.cb[1]; s = s4; inv = t4.y; }
      }
      const long long grA = r0 + ra;
      if (SR) {
        sr_block(P, 0, inv, sr_bytes16(a.seed, gbase + grA * a.cols + gtc * 16), ca);
        sr_block(P, 1, inv, sr_bytes16(a.seed, gbase + (grA + 1) * a.cols + gtc * 16), cb);
      }
      if (ROW) {
        store_codes8(a.row, b, grA, gtc * 8, ca[0], ca[1]);
        store_codes8(a.row, b, grA + 1, gtc * 8, cb[0], cb[1]);
        s_rsc[ra * 8 + tc] = (uint8_t)s;
        s_rsc[(ra + 1) * 8 + tc] = (uint8_t)s;
      }
      if (COL) {
        // byte for rows (2i, 2i+1) of each of the tile's 16 columns.  In a
        // column's 32 bytes the 8-byte group of tile row tr sits at group
        // tr ^ (tc & 3): the 4 tile columns a warp covers are 512 bytes
        // apart, which would put their stores in the same banks
        // even (E) and odd (O) columns: byte k of word w is column 8 w + 2 k (+ 1),
        // (row 2i nibble) | (row 2i+1 nibble) << 4
        const uint32_t E[2] = {(ca[0] & 0x0f0f0f0fu) | ((cb[0] & 0x0f0f0f0fu) << 4),
                               (ca[1] & 0x0f0f0f0fu) | ((cb[1] & 0x0f0f0f0fu) << 4)};
        const uint32_t O[2] = {((ca[0] >> 4) & 0x0f0f0f0fu) | (cb[0] & 0xf0f0f0f0u),
                               ((ca[1] >> 4) & 0x0f0f0f0fu) | (cb[1] & 0xf0f0f0f0u)};
        const int gofs = 8 * (tr ^ (tc & 3)) + i;
#pragma unroll
        for (int w = 0; w < 2; ++w)
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            s_tc[(16 * tc + 8 * w + 2 * k) * 32 + gofs] = (uint8_t)(E[w] >> (8 * k));
            s_tc[(16 * tc + 8 * w + 2 * k + 1) * 32 + gofs] = (uint8_t)(O[w] >> (8 * k));
          }
        s_csc[(16 * tc + 2 * i) * 32 + 4 * k + tr] = (uint8_t)s;
        s_csc[(16 * tc + 2 * i + 1) * 32 + 4 * k + tr] = (uint8_t)s;
      }
      if (F46 && i == 0 && pick) {
        if (ROW && a.row.choice) atomicOr(&s_bits[tr], 1u << tc);
        if (COL && a.col.choice) atomicOr(&s_cbits[tc], 1u << (4 * k + tr));
      }
    }
    __syncthreads();
    if (COL) {
      // transposed codes: column col, 32 rows per half
      const int col = t >> 1, h = t & 1;
      const int gc = c0 + col;
      const int grow = r0 + 32 * h;
      if (gc < a.cols && grow < a.rows) {
        const int sw = (col >> 4) & 3;   // the group swizzle of this column's tile column
        const uint2 v0 = *reinterpret_cast<const uint2*>(s_tc + col * 32 + 8 * ((2 * h) ^ sw));
        const uint2 v1 = *reinterpret_cast<const uint2*>(s_tc + col * 32 + 8 * ((2 * h + 1) ^ sw));
        const long long byte_col = grow / 2;   // a multiple of 16
        if (grow + 16 < a.rows && cc16) {
          *reinterpret_cast<uint4*>(a.col.codes + (long long)b * a.col.codes_bs + gc * a.col.codes_ld + byte_col) =
              make_uint4(v0.x, v0.y, v1.x, v1.y);
        } else {
          store_codes8(a.col, b, gc, byte_col, v0.x, v0.y);
          if (grow + 16 < a.rows) store_codes8(a.col, b, gc, byte_col + 8, v1.x, v1.y);
        }
      }
    }
    if (ROW && t < kSubRows * 2) {
      // rowwise scales: row t / 2, tile columns 4 (t & 1) .. + 3 of the sub-tile
      const int row = t >> 1, hf = t & 1;
      const long long R = r0 + row, gc4 = (c0 >> 4) + 4 * hf;
      if (R < a.rows && gc4 < ntc) {
        const uint32_t v = *reinterpret_cast<const uint32_t*>(s_rsc + row * 8 + 4 * hf);
        if (rsc_word && gc4 + 4 <= ntc) {
          *reinterpret_cast<uint32_t*>(a.row.scales + scale_off<SWZ>(a.row, b, R, gc4)) = v;
        } else {
          for (int q = 0; q < 4 && gc4 + q < ntc; ++q)
            a.row.scales[scale_off<SWZ>(a.row, b, R, gc4 + q)] = (uint8_t)(v >> (8 * q));
        }
      }
    }
    // rowwise copy: one bit per tile in the tile row-major order of x, so a
    // sub-tile row of 8 tiles is one byte
    if (ROW && F46 && a.row.choice && t < kSubRows / 16) {
      const uint32_t v = s_bits[t];
      s_bits[t] = 0;
      const long long gtr2 = (r0 >> 4) + t;
      if (gtr2 < ntr) {
        const unsigned long long bit = ((unsigned long long)b * ntr + gtr2) * ntc + (c0 >> 4);
        if (a.row.choice_aligned) {
          a.row.choice[bit >> 3] = (uint8_t)v;
        } else if (v) {
          unsigned int* wp = reinterpret_cast<unsigned int*>(a.row.choice) + (bit >> 5);
          const int sh = (int)(bit & 31);
          const unsigned long long vv = (unsigned long long)v << sh;
          if ((uint32_t)vv) atomicOr(wp, (uint32_t)vv);
          if ((uint32_t)(vv >> 32)) atomicOr(wp + 1, (uint32_t)(vv >> 32));
        }
      }
    }
  }
  if (COL) {
    __syncthreads();
    // the strip's transposed-copy scales: column col holds tile rows tr0 ..
    // tr0 + 4 nk - 1, one word per sub-tile; consecutive threads take
    // consecutive words of a column
    const long long left = (a.rows - rs0 + kSubRows - 1) / kSubRows;   // sub-tiles left from rs0
    const int nk = left < nsub ? (int)left : nsub;
    const long long tr0 = rs0 >> 4;   // a multiple of 4
    for (int idx = t; idx < kSubCols * nk; idx += kThreads) {
      const int col = idx / nk, w = idx - col * nk;
      const long long c = c0 + col, trw = tr0 + 4 * w;
      if (c < a.cols && trw < ntr) {
        const uint32_t v = *reinterpret_cast<const uint32_t*>(s_csc + col * 32 + 4 * w);
        if (csc_word && trw + 4 <= ntr) {
          *reinterpret_cast<uint32_t*>(a.col.scales + scale_off<SWZ>(a.col, b, c, trw)) = v;
        } else {
          for (int q = 0; q < 4 && trw + q < ntr; ++q)
            a.col.scales[scale_off<SWZ>(a.col, b, c, trw + q)] = (uint8_t)(v >> (8 * q));
        }
      }
    }
  }
  // transposed copy: one bit per tile in the tile row-major order of x^T
  // ([cols][rows]), so source tile (gtr, gtc) is bit (b*ntc + gtc)*ntr + gtr
  // and the strip's 32 tile rows of one tile column are 32 consecutive bits
  if (COL && F46 && a.col.choice) {
    if (t < kSubCols / 16) {
      const long long gtc = (c0 >> 4) + t;
      if (gtc < ntc) {
        const uint32_t v = s_cbits[t];
        const unsigned long long bit = ((unsigned long long)b * ntc + gtc) * ntr + (rs0 >> 4);
        unsigned int* wp = reinterpret_cast<unsigned int*>(a.col.choice) + (bit >> 5);
        if (a.col.choice_aligned) {
          *wp = v;
        } else if (v) {
          const int sh = (int)(bit & 31);
          const unsigned long long vv = (unsigned long long)v << sh;
          if ((uint32_t)vv) atomicOr(wp, (uint32_t)vv);
          if ((uint32_t)(vv >> 32)) atomicOr(wp + 1, (uint32_t)(vv >> 32));
        }
      }
    }
  }
  if (bad && a.status) atomicOr(a.status, FOS_STATUS_NONFINITE);
}

}  // namespace

cudaError_t launch_q1x16_dual(const QuantArgs& a, int batch, int fmt, bool sr, bool swz,
                              bool want_row, cudaStream_t st, bool rht_col) {
  const bool f46 = fmt == 0;
  const uint32_t ntc4 = (uint32_t)((a.cols / 16 + 3) / 4);
  const uint32_t units = (uint32_t)(a.rows / 16) * ntc4;
  const FastDiv fd = make_fastdiv(ntc4);
  const dim3 g(min((units + kThreads / 32 - 1) / (kThreads / 32), 148u * 8u), (unsigned)batch);
#define FOS_L(F, S, W, R) do { if (rht_col) k_dual_warp<F, S, W, R, true><<<g, kThreads, 0, st>>>(a, fd); \
                              else k_dual_warp<F, S, W, R, false><<<g, kThreads, 0, st>>>(a, fd); } while (0)
#define FOS_R(F, S, W) do { if (want_row) FOS_L(F, S, W, true); else FOS_L(F, S, W, false); } while (0)
#define FOS_W(F, S) do { if (swz) FOS_R(F, S, true); else FOS_R(F, S, false); } while (0)
#define FOS_S(F) do { if (sr) FOS_W(F, true); else FOS_W(F, false); } while (0)
  if (f46) FOS_S(true);
  else     FOS_S(false);
#undef FOS_S
#undef FOS_W
#undef FOS_R
#undef FOS_L
  return cudaGetLastError();
}

cudaError_t launch_amax_cols_rht(const QuantArgs& a, int batch, uint32_t* amax_col, cudaStream_t st) {
  const uint32_t units = (uint32_t)(a.cols / 2) * (uint32_t)(a.rows / 16);
  const uint32_t blocks = min((units + kThreads - 1) / kThreads, 148u * 8u);
  k_amax_cols_rht<<<dim3(blocks, (unsigned)batch), kThreads, 0, st>>>(a, amax_col);
  return cudaGetLastError();
}

// The 2D kernel variant for these options.
const void* kernel_2d(bool f46, bool sr, bool swz, bool want_row, bool want_col) {
  const void* k = nullptr;
#define FOS_L(F, S, W, R, C) k = reinterpret_cast<const void*>(k_2d16x16<F, S, W, R, C>)
#define FOS_C(F, S, W, R) do { if (want_col) FOS_L(F, S, W, R, true); else FOS_L(F, S, W, R, false); } while (0)
#define FOS_R(F, S, W) do { if (want_row) FOS_C(F, S, W, true); else FOS_C(F, S, W, false); } while (0)
#define FOS_W(F, S) do { if (swz) FOS_R(F, S, true); else FOS_R(F, S, false); } while (0)
#define FOS_S(F) do { if (sr) FOS_W(F, true); else FOS_W(F, false); } while (0)
  if (f46) FOS_S(true);
  else     FOS_S(false);
#undef FOS_S
#undef FOS_W
#undef FOS_R
#undef FOS_C
#undef FOS_L
  return k;
}

constexpr int kMaxDev = 64;

// Sub-tiles per CTA strip: the n in 1..8 whose grid of column strips x
// ceil(rows / 64n) x batch CTAs, in rounds of the resident CTA slots, costs
// the least, counting each CTA as n sub-tiles plus 0.3 for its start-up; the
// longest strip on ties.  The slots come from the occupancy of the variant,
// cached per device.
int q16x16_strip(long long rows, long long cols, long long batch, int fmt, bool sr, bool swz, bool want_row,
                 bool want_col) {
  static std::atomic<int> slots_of[kMaxDev][32];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return kStrip;
  const int v = (fmt == 0) * 16 + sr * 8 + swz * 4 + want_row * 2 + want_col;
  int slots = slots_of[dev][v].load(std::memory_order_relaxed);
  if (slots <= 0) {
    int sms = 0, per_sm = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel_2d(fmt == 0, sr, swz, want_row, want_col),
                                                      kThreads, 0) != cudaSuccess ||
        sms <= 0 || per_sm <= 0) {
      (void)cudaGetLastError();
      return kStrip;
    }
    slots = sms * per_sm;
    slots_of[dev][v].store(slots, std::memory_order_relaxed);
  }
  const long long cts = (cols + kSubCols - 1) / kSubCols * batch;
  int best = kStrip;
  long long best_cost = -1;
  for (int n = kStrip; n >= 1; --n) {
    const long long ctas = cts * ((rows + kSubRows * n - 1) / (kSubRows * n));
    const long long cost = (ctas + slots - 1) / slots * (10 * n + 3);
    if (best_cost < 0 || cost < best_cost) { best = n; best_cost = cost; }
  }
  return best;
}

cudaError_t launch_q16x16(const QuantArgs& a, int batch, int fmt, bool sr, bool swz, bool want_row,
                          bool want_col, int nsub, cudaStream_t st) {
  if (nsub < 1 || nsub > kStrip) return cudaErrorInvalidValue;
  const bool f46 = fmt == 0;
  const dim3 g((a.cols + kSubCols - 1) / kSubCols, (a.rows + kSubRows * nsub - 1) / (kSubRows * nsub),
               (unsigned)batch);
#define FOS_L(F, S, W, R, C) k_2d16x16<F, S, W, R, C><<<g, kThreads, 0, st>>>(a, nsub)
#define FOS_C(F, S, W, R) do { if (want_col) FOS_L(F, S, W, R, true); else FOS_L(F, S, W, R, false); } while (0)
#define FOS_R(F, S, W) do { if (want_row) FOS_C(F, S, W, true); else FOS_C(F, S, W, false); } while (0)
#define FOS_W(F, S) do { if (swz) FOS_R(F, S, true); else FOS_R(F, S, false); } while (0)
#define FOS_S(F) do { if (sr) FOS_W(F, true); else FOS_W(F, false); } while (0)
  if (f46) FOS_S(true);
  else     FOS_S(false);
#undef FOS_S
#undef FOS_W
#undef FOS_R
#undef FOS_C
#undef FOS_L
  return cudaGetLastError();
}

}  // namespace fos
