// fos_internal.h -- launch descriptors shared by the C ABI layer and the
// kernel files of libfos.so (host side; no device code).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "fos.h"
#include "fos_device.cuh"

namespace fos {

// One output orientation as the kernels see it.
struct OutDesc {
  uint8_t* codes = nullptr;
  long long codes_ld = 0;   // bytes per row
  long long codes_bs = 0;   // bytes per batch entry
  uint8_t* scales = nullptr;
  long long scales_ld = 0;  // bytes per row (linear layout)
  long long scales_bs = 0;  // bytes per batch entry
  long long col_tiles = 0;  // swizzled layout: ceil(sf_cols / 4)
  uint8_t* choice = nullptr;
  int choice_aligned = 0;   // blocks per batch entry % 64 == 0
  float* tensor_scale = nullptr;
};

struct QuantArgs {
  const uint16_t* x = nullptr;
  long long ld = 0;          // elements per row of x
  long long x_bs = 0;        // elements per batch entry of x
  int rows = 0, cols = 0;
  uint32_t nblk = 0;         // 1x16 (or 1x32) blocks per batch entry
  FastDiv bpr{};             // blocks per row
  uint32_t units_per_cta = 0;
  const float* amax_in = nullptr;   // nullable
  const uint32_t* amax_ws = nullptr;
  const uint32_t* amax_col_ws = nullptr;  // the colwise copy's amax words (colwise transform)
  uint32_t* status = nullptr;       // nullable
  unsigned long long seed = 0;
  long long elem_offset = 0;
  // -0.0f, passed at run time: the addend of the squares in the error sums,
  // opaque to the code generator so that a square is never seen as a plain
  // product and fused into the following add
  float neg_zero = -0.0f;
  OutDesc row, col;
  // Bounded waits of the fused kernel: polls (each an L2 round trip plus a
  // 128 ns sleep, about 2^21 polls to a second and a half) before a wait
  // gives up and reports FOS_STATUS_TIMEOUT.  stall_entry >= 0 is a test
  // hook (fos_testing_quantize_stalled): that entry's amax items never count
  // in, so every wait on it runs out.
  uint32_t spin_limit = 1u << 21;
  int stall_entry = -1;
  // fake quantization (fos_fake_quantize): bf16 output y [batch][rows][ldy]
  // instead of codes and scales
  uint16_t* y = nullptr;
  long long ldy = 0, y_bs = 0;
};

FastDiv make_fastdiv(uint32_t d);

// Kernel launchers (return the launch's cudaError_t).
cudaError_t launch_amax(const QuantArgs& a, int batch, bool rht, uint32_t* amax_ws,
                        cudaStream_t st);
// fake: write the dequantized bf16 values to a.y instead of codes and scales
cudaError_t launch_q1x16_rowwise(const QuantArgs& a, int batch, int fmt, bool sr, bool rht,
                                 bool swz, bool dense, cudaStream_t st, bool fake = false);
// fused per-entry amax + rowwise quantize (one persistent launch fed by a
// work queue); amax_ws, done_a: one zeroed word per batch entry, queue: one
// zeroed counter.  Returns cudaErrorNotSupported when it cannot be launched.
cudaError_t launch_q1x16_fused(const QuantArgs& a, int batch, int fmt, bool sr, bool rht, bool swz,
                               bool dense, uint32_t* amax_ws, uint32_t* done_a, uint32_t* queue,
                               cudaStream_t st, bool fake = false);
// MXFP4 fake quantization (bf16 out); the NVFP4 one runs through the rowwise
// launchers with fake = true.
cudaError_t launch_fake_mx(const QuantArgs& a, int batch, cudaStream_t st);

// NVFP4 block-scaled GEMM on the tensor cores (fos_gemm.cu); shapes checked
// by the caller (M, N multiples of 128, K of 256).
// workspace (nullable): gemm_workspace_bytes(M, N, K) bytes for the wide
// scale layout (expanded from a's and b's swizzled scales in the call)
cudaError_t launch_gemm_nvfp4(const fos_qtensor* a, const fos_qtensor* b, int M, int N, int K, void* d,
                              long long ldd, int f32_out, uint32_t* status, cudaStream_t st,
                              void* workspace = nullptr);
size_t gemm_workspace_bytes(long long M, long long N, long long K);

// Workspace bytes of fos_quantize for `batch` entries: per-entry amax words,
// per-entry completion counters and the fused kernel's queue counter.
constexpr size_t workspace_bytes_for(long long batch) {
  return (size_t)(12 * ((batch + 63) / 64 * 64) + 256);
}

cudaError_t launch_q1x16_dual(const QuantArgs& a, int batch, int fmt, bool sr, bool swz,
                              bool want_row, cudaStream_t st, bool rht_col = false);
// amax of the 16-row column blocks after the 16-wide transform (the colwise
// copy's amax with FOS_FLAG_RHT16_COL) into zeroed words amax_col[batch]
cudaError_t launch_amax_cols_rht(const QuantArgs& a, int batch, uint32_t* amax_col, cudaStream_t st);
// sub-tiles (64 rows each) per CTA strip of the 2D kernel, 1..8; only a
// strip of 8 owns whole words of the transposed copy's choice bitmap
int q16x16_strip(long long rows, long long cols, long long batch, int fmt, bool sr, bool swz, bool want_row,
                 bool want_col);
cudaError_t launch_q16x16(const QuantArgs& a, int batch, int fmt, bool sr, bool swz,
                          bool want_row, bool want_col, int nsub, cudaStream_t st);
cudaError_t launch_mxfp4(const QuantArgs& a, int batch, bool swz, cudaStream_t st);

struct DequantArgs {
  const uint8_t* codes = nullptr;
  long long codes_ld = 0, codes_bs = 0;
  const uint8_t* scales = nullptr;
  long long scales_ld = 0, scales_bs = 0, col_tiles = 0;
  const float* tensor_scale = nullptr;
  uint16_t* y = nullptr;
  long long ldy = 0, y_bs = 0;
  int rows = 0, cols = 0;
  uint32_t nblk = 0;   // blocks per batch entry
  FastDiv bpr{};
  uint32_t units_per_cta = 0;
};

// dense: codes rows contiguous (codes_ld = cols/2), linear scales with
// scales_ld = cols/bs, y rows contiguous (ldy = cols), 32-byte aligned y
cudaError_t launch_dequant(const DequantArgs& a, int batch, bool mx, bool swz, bool dense, cudaStream_t st);

}  // namespace fos
