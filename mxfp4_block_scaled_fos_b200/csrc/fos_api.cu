// fos_api.cu -- the C ABI of libfos.so (argument checks, workspace layout,
// launch sequence).  Declarations and semantics: include/fos.h.
#include <string.h>

#include "fos.h"
#include "fos_internal.h"
#include "fos_testing.h"

namespace fos {

FastDiv make_fastdiv(uint32_t d) {
  FastDiv f;
  f.d = d;
  uint32_t s = 0;
  while ((1ull << s) < d) ++s;
  f.s = s;
  // m = floor(2^32 * (2^s - d) / d) + 1
  f.m = (uint32_t)((((1ull << s) - d) << 32) / d + 1ull);
  return f;
}

namespace {

constexpr uint32_t kUnitsQuant = 256 * 4;   // work units per CTA (tile kernels)
constexpr uint32_t kBlocksRowwise = 256 * 8; // 16-element blocks per CTA (rowwise 1x16)
constexpr uint32_t kUnitsAmax = 256 * 8;    // block pairs per CTA (amax pass)
constexpr uint32_t kUnitsMx = 256 * 4;      // 1x32 blocks per CTA
constexpr uint32_t kUnitsDeq = 256 * 4;     // blocks per CTA (dequantize)

inline bool aligned(const void* p, uintptr_t a) { return ((uintptr_t)p % a) == 0; }

long long round_up(long long v, long long m) { return (v + m - 1) / m * m; }

size_t ws_bytes(int64_t batch) { return workspace_bytes_for(batch); }

// Validate one output descriptor for a tensor of R rows and C columns.
fos_status check_out(const fos_qtensor* q, int64_t R, int64_t C, int64_t bs, bool nvfp4,
                     uint32_t flags) {
  if (!q->codes || !q->scales) return FOS_ERR_NULL;
  if (nvfp4 && !q->tensor_scale) return FOS_ERR_NULL;
  if (!aligned(q->codes, 16) || q->codes_ld % 8 != 0) return FOS_ERR_ALIGN;
  if (q->codes_ld < C / 2) return FOS_ERR_SHAPE;
  if (!(flags & FOS_FLAG_SCALE_SWIZZLED) && q->scales_ld < C / bs) return FOS_ERR_SHAPE;
  if (q->choice_bits && !aligned(q->choice_bits, 8)) return FOS_ERR_ALIGN;
  if (q->tensor_scale && !aligned(q->tensor_scale, 4)) return FOS_ERR_ALIGN;
  (void)R;
  return FOS_OK;
}

OutDesc make_out(const fos_qtensor* q, int64_t R, int64_t C, int64_t bs, uint32_t flags,
                 int64_t nblk_per_batch) {
  OutDesc o;
  o.codes = q->codes;
  o.codes_ld = q->codes_ld;
  o.codes_bs = q->codes_ld * R;
  o.scales = q->scales;
  const int64_t sfc = C / bs;
  if (flags & FOS_FLAG_SCALE_SWIZZLED) {
    o.col_tiles = (sfc + 3) / 4;
    o.scales_bs = round_up(R, 128) * o.col_tiles * 4;
  } else {
    o.scales_ld = q->scales_ld;
    o.scales_bs = q->scales_ld * R;
  }
  o.choice = q->choice_bits;
  o.choice_aligned = (nblk_per_batch % 64) == 0;
  o.tensor_scale = q->tensor_scale;
  return o;
}

size_t choice_bytes(int64_t nblocks) { return (size_t)(8 * ((nblocks + 63) / 64)); }

// nr rows of `width` bytes, `ld` apart on both sides, device to host: one
// plain copy when the rows are packed, else a pitched one.
cudaError_t rows_d2h(void* dst, const void* src, int64_t ld, int64_t width, int64_t nr, cudaStream_t st) {
  if (ld == width) return cudaMemcpyAsync(dst, src, (size_t)(width * nr), cudaMemcpyDeviceToHost, st);
  return cudaMemcpy2DAsync(dst, (size_t)ld, src, (size_t)ld, (size_t)width, (size_t)nr, cudaMemcpyDeviceToHost, st);
}

// Test hooks: the fused kernel's bounded waits (fos_testing_quantize_stalled)
// and the 2D kernel's strip length (fos_testing_quantize_2d_strip; 0 = the
// per-launch choice).
struct WaitHooks {
  uint32_t spin_limit = 1u << 21;
  int stall_entry = -1;
  int strip_2d = 0;
  bool validate_only = false;   // check the arguments, enqueue nothing
};

fos_status quantize_impl(const void* x, int64_t batch, int64_t rows, int64_t cols, int64_t ld,
                         const fos_options* opt, const float* amax_in, const fos_qtensor* rowwise,
                         const fos_qtensor* colwise, void* workspace, size_t workspace_bytes,
                         uint32_t* status, void* stream, const WaitHooks& hooks);

}  // namespace
}  // namespace fos

using namespace fos;

extern "C" {

int32_t fos_version(void) { return FOS_VERSION; }

const char* fos_status_string(int32_t s) {
  switch (s) {
    case FOS_OK: return "ok";
    case FOS_ERR_NULL: return "a required pointer is NULL";
    case FOS_ERR_ALIGN: return "a pointer or leading dimension is misaligned";
    case FOS_ERR_SHAPE: return "shape not divisible by the block, or out of range";
    case FOS_ERR_UNSUPPORTED: return "option combination not supported";
    case FOS_ERR_WORKSPACE: return "workspace missing or too small";
    case FOS_ERR_CUDA: return "CUDA launch or memset failed";
    case FOS_ERR_ARG: return "invalid enum value, flag or offset";
    default: return "unknown status";
  }
}

size_t fos_workspace_size(int64_t batch, int64_t rows, int64_t cols, const fos_options* opt) {
  (void)rows;
  (void)cols;
  (void)opt;
  return ws_bytes(batch < 1 ? 1 : batch);
}

size_t fos_scales_size(int64_t R, int64_t sf_cols, uint32_t flags) {
  if (R < 0 || sf_cols < 0) return 0;
  if (flags & FOS_FLAG_SCALE_SWIZZLED)
    return (size_t)(round_up(R, 128) * round_up(sf_cols, 4));
  return (size_t)(R * sf_cols);
}

fos_status fos_quantize(const void* x, int64_t batch, int64_t rows, int64_t cols, int64_t ld,
                        const fos_options* opt, const float* amax_in,
                        const fos_qtensor* rowwise, const fos_qtensor* colwise,
                        void* workspace, size_t workspace_bytes, uint32_t* status,
                        void* stream) {
  return quantize_impl(x, batch, rows, cols, ld, opt, amax_in, rowwise, colwise, workspace,
                       workspace_bytes, status, stream, WaitHooks());
}

fos_status fos_quantize_host(const void* x_host, int64_t batch, int64_t rows, int64_t cols,
                             const fos_options* opt, const float* amax_in, const fos_qtensor* out_host,
                             void* x_dev, const fos_qtensor* out_dev, void* workspace,
                             size_t workspace_bytes, uint32_t* status, int64_t chunk, void* stream_h2d,
                             void* stream_compute, void* stream_d2h, void* const* events) {
  if (!x_host || !opt || !out_host || !x_dev || !out_dev || !events) return FOS_ERR_NULL;
  if (chunk < 1) return FOS_ERR_ARG;
  if (opt->blk == FOS_BLOCK_16X16 || (opt->flags & (FOS_FLAG_SCALE_SWIZZLED | FOS_FLAG_RHT16_COL)) ||
      out_host->choice_bits || out_dev->choice_bits)
    return FOS_ERR_UNSUPPORTED;
  const bool mx = opt->fmt == FOS_FMT_MXFP4;
  if (!out_host->codes || !out_host->scales || (!mx && !out_host->tensor_scale)) return FOS_ERR_NULL;
  if (out_host->codes_ld != out_dev->codes_ld || out_host->scales_ld != out_dev->scales_ld) return FOS_ERR_ARG;
  if (!aligned(x_dev, 32)) return FOS_ERR_ALIGN;
  // later chunks start chunk * rows rows further: their codes stay 16-byte aligned
  if (batch > chunk && (chunk * rows * out_dev->codes_ld) % 16 != 0) return FOS_ERR_ALIGN;
  // every chunk has the shape and options of the first (the last may hold
  // fewer entries, which needs no more workspace): check them all up front
  WaitHooks check;
  check.validate_only = true;
  fos_status e = quantize_impl(x_dev, batch < chunk ? batch : chunk, rows, cols, cols, opt, amax_in, out_dev,
                               nullptr, workspace, workspace_bytes, status, stream_compute, check);
  if (e != FOS_OK) return e;
  cudaStream_t s_in = (cudaStream_t)stream_h2d, s_q = (cudaStream_t)stream_compute, s_out = (cudaStream_t)stream_d2h;
  if (batch == 0) return FOS_OK;
  if (rows == 0 || cols == 0) {   // empty entries: only S_t = 0 to deliver
    for (int64_t c0 = 0; c0 < batch; c0 += chunk) {
      const int64_t nb = batch - c0 < chunk ? batch - c0 : chunk;
      fos_qtensor q = *out_dev;
      if (!mx) q.tensor_scale += c0;
      e = quantize_impl(x_dev, nb, rows, cols, cols, opt, nullptr, &q, nullptr, workspace, workspace_bytes,
                        status, s_q, WaitHooks());
      if (e != FOS_OK) return e;
    }
    if (!mx && (cudaEventRecord((cudaEvent_t)events[1], s_q) != cudaSuccess ||
                cudaStreamWaitEvent(s_out, (cudaEvent_t)events[1], 0) != cudaSuccess ||
                cudaMemcpyAsync(out_host->tensor_scale, out_dev->tensor_scale, 4 * batch, cudaMemcpyDeviceToHost,
                                s_out) != cudaSuccess))
      return FOS_ERR_CUDA;
    return FOS_OK;
  }
  const int64_t per_entry = rows * cols;   // elements
  const int64_t code_w = cols / 2, scale_w = cols / (mx ? 32 : 16);
  for (int64_t c0 = 0, k = 0; c0 < batch; c0 += chunk, ++k) {
    const int64_t nb = batch - c0 < chunk ? batch - c0 : chunk;
    cudaEvent_t ev_in = (cudaEvent_t)events[2 * k], ev_q = (cudaEvent_t)events[2 * k + 1];
    const size_t xoff = (size_t)(c0 * per_entry) * 2;
    if (cudaMemcpyAsync((char*)x_dev + xoff, (const char*)x_host + xoff, (size_t)(nb * per_entry) * 2,
                        cudaMemcpyHostToDevice, s_in) != cudaSuccess ||
        cudaEventRecord(ev_in, s_in) != cudaSuccess || cudaStreamWaitEvent(s_q, ev_in, 0) != cudaSuccess)
      return FOS_ERR_CUDA;
    fos_options o = *opt;
    o.elem_offset = opt->elem_offset + c0 * per_entry;
    fos_qtensor q = *out_dev;
    q.codes += c0 * rows * q.codes_ld;
    q.scales += c0 * rows * q.scales_ld;
    if (!mx) q.tensor_scale += c0;
    e = quantize_impl((char*)x_dev + xoff, nb, rows, cols, cols, &o, amax_in ? amax_in + c0 : nullptr, &q,
                      nullptr, workspace, workspace_bytes, status, s_q, WaitHooks());
    if (e != FOS_OK) return e;
    if (cudaEventRecord(ev_q, s_q) != cudaSuccess || cudaStreamWaitEvent(s_out, ev_q, 0) != cudaSuccess)
      return FOS_ERR_CUDA;
    const int64_t r0 = c0 * rows, nr = nb * rows;
    if (rows_d2h(out_host->codes + r0 * out_host->codes_ld, q.codes, q.codes_ld, code_w, nr, s_out) != cudaSuccess ||
        rows_d2h(out_host->scales + r0 * out_host->scales_ld, q.scales, q.scales_ld, scale_w, nr, s_out) !=
            cudaSuccess ||
        (!mx && cudaMemcpyAsync(out_host->tensor_scale + c0, q.tensor_scale, 4 * nb, cudaMemcpyDeviceToHost,
                                s_out) != cudaSuccess))
      return FOS_ERR_CUDA;
  }
  return FOS_OK;
}

fos_status fos_testing_quantize_stalled(const void* x, int64_t batch, int64_t rows, int64_t cols,
                                        int64_t ld, const fos_options* opt,
                                        const fos_qtensor* rowwise, void* workspace,
                                        size_t workspace_bytes, uint32_t* status,
                                        int32_t stall_entry, uint32_t spin_limit, void* stream) {
  if (!opt || !rowwise) return FOS_ERR_NULL;
  if (opt->fmt == FOS_FMT_MXFP4 || opt->blk != FOS_BLOCK_1X16) return FOS_ERR_UNSUPPORTED;
  if (stall_entry < 0 || stall_entry >= batch || spin_limit < 1) return FOS_ERR_ARG;
  WaitHooks h;
  h.spin_limit = spin_limit;
  h.stall_entry = stall_entry;
  return quantize_impl(x, batch, rows, cols, ld, opt, nullptr, rowwise, nullptr, workspace,
                       workspace_bytes, status, stream, h);
}

fos_status fos_testing_quantize_2d_strip(const void* x, int64_t batch, int64_t rows, int64_t cols,
                                         int64_t ld, const fos_options* opt, const float* amax_in,
                                         const fos_qtensor* rowwise, const fos_qtensor* colwise,
                                         void* workspace, size_t workspace_bytes, uint32_t* status,
                                         int32_t nsub, void* stream) {
  if (!opt) return FOS_ERR_NULL;
  if (opt->blk != FOS_BLOCK_16X16) return FOS_ERR_UNSUPPORTED;
  if (nsub < 1 || nsub > 8) return FOS_ERR_ARG;
  WaitHooks h;
  h.strip_2d = nsub;
  return quantize_impl(x, batch, rows, cols, ld, opt, amax_in, rowwise, colwise, workspace,
                       workspace_bytes, status, stream, h);
}

}  // extern "C"

namespace fos {
namespace {

fos_status quantize_impl(const void* x, int64_t batch, int64_t rows, int64_t cols, int64_t ld,
                         const fos_options* opt, const float* amax_in, const fos_qtensor* rowwise,
                         const fos_qtensor* colwise, void* workspace, size_t workspace_bytes,
                         uint32_t* status, void* stream, const WaitHooks& hooks) {
  if (!opt || !x) return FOS_ERR_NULL;
  if (!rowwise && !colwise) return FOS_ERR_NULL;
  if (opt->fmt < 0 || opt->fmt > 2 || opt->blk < 0 || opt->blk > 2 || opt->rnd < 0 ||
      opt->rnd > 1 || (opt->flags & ~(FOS_FLAG_RHT16 | FOS_FLAG_SCALE_SWIZZLED | FOS_FLAG_RHT16_COL)))
    return FOS_ERR_ARG;
  if (batch < 0 || rows < 0 || cols < 0) return FOS_ERR_SHAPE;
  const bool mx = opt->fmt == FOS_FMT_MXFP4;
  const bool rht = (opt->flags & FOS_FLAG_RHT16) != 0;
  const bool rht_col = (opt->flags & FOS_FLAG_RHT16_COL) != 0;
  const bool swz = (opt->flags & FOS_FLAG_SCALE_SWIZZLED) != 0;
  const bool sr = opt->rnd == FOS_ROUND_SR;
  if (mx != (opt->blk == FOS_BLOCK_1X32)) return FOS_ERR_UNSUPPORTED;
  if (mx && (sr || rht || colwise)) return FOS_ERR_UNSUPPORTED;
  if (rht && (opt->blk != FOS_BLOCK_1X16 || colwise)) return FOS_ERR_UNSUPPORTED;
  if (rht_col && (mx || opt->blk != FOS_BLOCK_1X16 || !colwise)) return FOS_ERR_UNSUPPORTED;
  const int64_t bs = mx ? 32 : 16;
  if (cols % bs) return FOS_ERR_SHAPE;
  if ((colwise || opt->blk == FOS_BLOCK_16X16) && rows % 16) return FOS_ERR_SHAPE;
  if (sr && (opt->elem_offset < 0 || opt->elem_offset % 16)) return FOS_ERR_ARG;
  if (!aligned(x, 16) || ld % 8 != 0) return FOS_ERR_ALIGN;
  if (ld < cols) return FOS_ERR_SHAPE;
  if (batch > 65535) return FOS_ERR_SHAPE;
  // per-batch block counts must stay below 2^31 (32-bit block indices)
  if (rows > 0 && cols > 0 && (rows * (cols / 16)) >= (1ll << 31)) return FOS_ERR_SHAPE;
  if (colwise && rows > 0 && cols > 0 && (cols * (rows / 16)) >= (1ll << 31)) return FOS_ERR_SHAPE;
  fos_status e;
  if (rowwise && (e = check_out(rowwise, rows, cols, bs, !mx, opt->flags)) != FOS_OK) return e;
  if (colwise && (e = check_out(colwise, cols, rows, 16, !mx, opt->flags)) != FOS_OK) return e;
  const bool need_ws = !mx && (!amax_in || rht_col);
  if (need_ws) {
    if (!workspace) return FOS_ERR_WORKSPACE;
    if (workspace_bytes < ws_bytes(batch)) return FOS_ERR_WORKSPACE;
    if (!aligned(workspace, 16)) return FOS_ERR_ALIGN;
  }
  if (amax_in && !aligned(amax_in, 4)) return FOS_ERR_ALIGN;
  if (hooks.validate_only) return FOS_OK;

  cudaStream_t st = (cudaStream_t)stream;
  if (batch == 0) return FOS_OK;
  if (rows == 0 || cols == 0) {  // empty entries: S_t = 0, nothing else to write
    if (!mx) {
      if (rowwise && cudaMemsetAsync(rowwise->tensor_scale, 0, 4 * batch, st) != cudaSuccess)
        return FOS_ERR_CUDA;
      if (colwise && cudaMemsetAsync(colwise->tensor_scale, 0, 4 * batch, st) != cudaSuccess)
        return FOS_ERR_CUDA;
    }
    return FOS_OK;
  }

  QuantArgs a;
  a.x = (const uint16_t*)x;
  a.ld = ld;
  a.x_bs = rows * ld;
  a.rows = (int)rows;
  a.cols = (int)cols;
  a.nblk = (uint32_t)(rows * (cols / bs));
  a.bpr = make_fastdiv((uint32_t)(cols / bs));
  a.amax_in = amax_in;
  a.status = status;
  a.seed = opt->seed;
  a.elem_offset = opt->elem_offset;
  a.spin_limit = hooks.spin_limit;
  a.stall_entry = hooks.stall_entry;
  if (rowwise) {
    const int64_t nb = opt->blk == FOS_BLOCK_16X16 ? (rows / 16) * (cols / 16) : rows * (cols / bs);
    a.row = make_out(rowwise, rows, cols, bs, opt->flags, nb);
  }
  if (colwise) {
    const int64_t nb = opt->blk == FOS_BLOCK_16X16 ? (rows / 16) * (cols / 16) : cols * (rows / 16);
    a.col = make_out(colwise, cols, rows, 16, opt->flags, nb);
  }

  if (mx) {
    a.units_per_cta = kUnitsMx;
    return launch_mxfp4(a, (int)batch, swz, st) == cudaSuccess ? FOS_OK : FOS_ERR_CUDA;
  }

  // Which choice-bit words a CTA owns outright depends on the kernel's tiling;
  // bitmaps whose words are shared between CTAs are built with atomics on a
  // zeroed buffer.
  int nsub = 0;
  if (opt->blk == FOS_BLOCK_16X16) {
    // rowwise: a CTA writes whole bytes (8 tile columns of one tile row);
    // transposed copy: whole 32-bit words (32 tile rows of one tile column)
    // when its strips are 8 sub-tiles long
    nsub = hooks.strip_2d > 0
               ? hooks.strip_2d
               : q16x16_strip(rows, cols, batch, opt->fmt, sr, swz, rowwise != nullptr, colwise != nullptr);
    a.row.choice_aligned = (cols / 16) % 8 == 0;
    a.col.choice_aligned = (rows / 16) % 32 == 0 && nsub == 8;
  } else if (colwise) {
    // the warp-based kernel sets every bit with an atomic on a zeroed bitmap
    a.row.choice_aligned = a.col.choice_aligned = 0;
  }
  const int64_t nb_row = opt->blk == FOS_BLOCK_16X16 ? batch * (rows / 16) * (cols / 16)
                                                     : batch * rows * (cols / 16);
  const int64_t nb_col = opt->blk == FOS_BLOCK_16X16 ? nb_row : batch * cols * (rows / 16);
  if (rowwise && rowwise->choice_bits && !a.row.choice_aligned)
    if (cudaMemsetAsync(rowwise->choice_bits, 0, choice_bytes(nb_row), st) != cudaSuccess)
      return FOS_ERR_CUDA;
  if (colwise && colwise->choice_bits && !a.col.choice_aligned)
    if (cudaMemsetAsync(colwise->choice_bits, 0, choice_bytes(nb_col), st) != cudaSuccess)
      return FOS_ERR_CUDA;

  // workspace: amax words [batch], then the fused path's per-entry counts
  // [batch] and its queue counter
  uint32_t* amax_ws = (uint32_t*)workspace;
  uint32_t* done_ws = amax_ws + round_up(batch, 64);
  uint32_t* claim_ws = done_ws + round_up(batch, 64);
  a.amax_ws = amax_ws;
  cudaError_t ce;
  const bool rowwise_1x16 = opt->blk == FOS_BLOCK_1X16 && !colwise;
  // contiguous rows, packed outputs, 32-byte aligned input and choice-bitmap
  // words owned by one warp each: no index arithmetic per block and one
  // 256-bit load per block
  const bool dense = rowwise_1x16 && ld == cols && rowwise->codes_ld * 2 == cols && !swz &&
                     rowwise->scales_ld * 16 == cols && aligned(x, 32) &&
                     (!rowwise->choice_bits || a.row.choice_aligned);

  if (!amax_in && rowwise_1x16) {
    // one persistent launch: per-entry amax and quantize, pipelined so the
    // second read of each entry comes from L2
    if (cudaMemsetAsync(amax_ws, 0, 12 * round_up(batch, 64), st) != cudaSuccess) return FOS_ERR_CUDA;
    ce = launch_q1x16_fused(a, (int)batch, opt->fmt, sr, rht, swz, dense, amax_ws, done_ws, claim_ws,
                            st);
    if (ce == cudaSuccess) return FOS_OK;
    if (ce != cudaErrorNotSupported) return FOS_ERR_CUDA;
    (void)cudaGetLastError();  // fall back to the two-kernel path below
  }

  // per-tensor amax pass, unless the caller supplies the amaxes
  if (!amax_in) {
    if (cudaMemsetAsync(amax_ws, 0, 4 * batch, st) != cudaSuccess) return FOS_ERR_CUDA;
    a.units_per_cta = kUnitsAmax;
    if (launch_amax(a, (int)batch, rht, amax_ws, st) != cudaSuccess) return FOS_ERR_CUDA;
  }

  a.units_per_cta = kUnitsQuant;
  if (rowwise_1x16) a.units_per_cta = kBlocksRowwise;
  if (opt->blk == FOS_BLOCK_16X16) {
    ce = launch_q16x16(a, (int)batch, opt->fmt, sr, swz, rowwise != nullptr, colwise != nullptr, nsub, st);
  } else if (colwise) {
    if (rht_col) {  // the colwise copy's own amax, in the words the fused path uses for its counts
      if (cudaMemsetAsync(done_ws, 0, 4 * batch, st) != cudaSuccess) return FOS_ERR_CUDA;
      if (launch_amax_cols_rht(a, (int)batch, done_ws, st) != cudaSuccess) return FOS_ERR_CUDA;
      a.amax_col_ws = done_ws;
    }
    ce = launch_q1x16_dual(a, (int)batch, opt->fmt, sr, swz, rowwise != nullptr, st, rht_col);
  } else {
    ce = launch_q1x16_rowwise(a, (int)batch, opt->fmt, sr, rht, swz, dense, st);
  }
  if (ce == cudaErrorNotSupported) return FOS_ERR_UNSUPPORTED;
  return ce == cudaSuccess ? FOS_OK : FOS_ERR_CUDA;
}

}  // namespace
}  // namespace fos

extern "C" {

fos_status fos_fake_quantize(const void* x, int64_t batch, int64_t rows, int64_t cols, int64_t ld,
                             const fos_options* opt, const float* amax_in, void* y, int64_t ldy,
                             void* workspace, size_t workspace_bytes, uint32_t* status, void* stream) {
  if (!opt || !x || !y) return FOS_ERR_NULL;
  if (opt->fmt < 0 || opt->fmt > 2 || opt->blk < 0 || opt->blk > 2 || opt->rnd < 0 ||
      opt->rnd > 1 || (opt->flags & ~(FOS_FLAG_RHT16 | FOS_FLAG_SCALE_SWIZZLED)))
    return FOS_ERR_ARG;
  if (batch < 0 || rows < 0 || cols < 0 || batch > 65535) return FOS_ERR_SHAPE;
  const bool mx = opt->fmt == FOS_FMT_MXFP4;
  const bool rht = (opt->flags & FOS_FLAG_RHT16) != 0;
  const bool sr = opt->rnd == FOS_ROUND_SR;
  if (mx != (opt->blk == FOS_BLOCK_1X32)) return FOS_ERR_UNSUPPORTED;
  if (opt->blk == FOS_BLOCK_16X16) return FOS_ERR_UNSUPPORTED;
  if (mx && (sr || rht)) return FOS_ERR_UNSUPPORTED;
  const int64_t bs = mx ? 32 : 16;
  if (cols % bs) return FOS_ERR_SHAPE;
  if (sr && (opt->elem_offset < 0 || opt->elem_offset % 16)) return FOS_ERR_ARG;
  if (!aligned(x, 16) || ld % 8 != 0 || !aligned(y, 16) || ldy % 8 != 0) return FOS_ERR_ALIGN;
  if (ld < cols || ldy < cols) return FOS_ERR_SHAPE;
  if (rows > 0 && cols > 0 && rows * (cols / 16) >= (1ll << 31)) return FOS_ERR_SHAPE;
  const bool need_ws = !mx && !amax_in;
  if (need_ws) {
    if (!workspace || workspace_bytes < ws_bytes(batch)) return FOS_ERR_WORKSPACE;
    if (!aligned(workspace, 16)) return FOS_ERR_ALIGN;
  }
  if (amax_in && !aligned(amax_in, 4)) return FOS_ERR_ALIGN;
  cudaStream_t st = (cudaStream_t)stream;
  if (batch == 0 || rows == 0 || cols == 0) return FOS_OK;

  QuantArgs a;
  a.x = (const uint16_t*)x;
  a.ld = ld;
  a.x_bs = rows * ld;
  a.rows = (int)rows;
  a.cols = (int)cols;
  a.nblk = (uint32_t)(rows * (cols / bs));
  a.bpr = make_fastdiv((uint32_t)(cols / bs));
  a.amax_in = amax_in;
  a.status = status;
  a.seed = opt->seed;
  a.elem_offset = opt->elem_offset;
  a.y = (uint16_t*)y;
  a.ldy = ldy;
  a.y_bs = rows * ldy;
  if (mx) {
    a.units_per_cta = kUnitsMx;
    return launch_fake_mx(a, (int)batch, st) == cudaSuccess ? FOS_OK : FOS_ERR_CUDA;
  }
  const bool dense = ld == cols && ldy == cols && aligned(x, 32) && aligned(y, 32);
  uint32_t* amax_ws = (uint32_t*)workspace;
  a.amax_ws = amax_ws;
  if (!amax_in) {  // the fused amax + (fake) quantize kernel, as in fos_quantize
    uint32_t* done_ws = amax_ws + round_up(batch, 64);
    uint32_t* claim_ws = done_ws + round_up(batch, 64);
    if (cudaMemsetAsync(amax_ws, 0, 12 * round_up(batch, 64), st) != cudaSuccess) return FOS_ERR_CUDA;
    cudaError_t ce = launch_q1x16_fused(a, (int)batch, opt->fmt, sr, rht, false, dense, amax_ws, done_ws,
                                        claim_ws, st, true);
    if (ce == cudaSuccess) return FOS_OK;
    if (ce != cudaErrorNotSupported) return FOS_ERR_CUDA;
    (void)cudaGetLastError();  // amax pass, then the fake quantizer
    if (cudaMemsetAsync(amax_ws, 0, 4 * batch, st) != cudaSuccess) return FOS_ERR_CUDA;
    QuantArgs am = a;
    am.units_per_cta = kUnitsAmax;
    if (launch_amax(am, (int)batch, rht, amax_ws, st) != cudaSuccess) return FOS_ERR_CUDA;
  }
  a.units_per_cta = kBlocksRowwise;
  return launch_q1x16_rowwise(a, (int)batch, opt->fmt, sr, rht, false, dense, st, true) == cudaSuccess
             ? FOS_OK : FOS_ERR_CUDA;
}

fos_status fos_gemm_nvfp4(const fos_qtensor* a, const fos_qtensor* b, int64_t M, int64_t N, int64_t K,
                          void* d, int64_t ldd, int32_t out_dtype, uint32_t* status, void* stream) {
  return fos_gemm_nvfp4_ws(a, b, M, N, K, d, ldd, out_dtype, nullptr, 0, status, stream);
}

size_t fos_gemm_workspace_size(int64_t M, int64_t N, int64_t K) {
  if (M < 0 || N < 0 || K < 0) return 0;
  return gemm_workspace_bytes(M, N, K);
}

fos_status fos_gemm_nvfp4_ws(const fos_qtensor* a, const fos_qtensor* b, int64_t M, int64_t N, int64_t K,
                             void* d, int64_t ldd, int32_t out_dtype, void* workspace, size_t workspace_bytes,
                             uint32_t* status, void* stream) {
  if (!a || !b || !d) return FOS_ERR_NULL;
  if (!a->codes || !a->scales || !a->tensor_scale || !b->codes || !b->scales || !b->tensor_scale)
    return FOS_ERR_NULL;
  if (out_dtype != 0 && out_dtype != 1) return FOS_ERR_ARG;
  if (M < 0 || N < 0 || K < 0) return FOS_ERR_SHAPE;
  if (M % 128 || N % 128 || K % 256) return FOS_ERR_SHAPE;
  if (M > (1 << 24) || N > (1 << 24) || K > (1 << 24)) return FOS_ERR_SHAPE;
  if (ldd < N) return FOS_ERR_SHAPE;
  if (!aligned(a->codes, 16) || !aligned(b->codes, 16) || !aligned(a->scales, 16) || !aligned(b->scales, 16) ||
      !aligned(d, 16) || !aligned(a->tensor_scale, 4) || !aligned(b->tensor_scale, 4))
    return FOS_ERR_ALIGN;
  if (a->codes_ld < K / 2 || b->codes_ld < K / 2) return FOS_ERR_SHAPE;
  if (a->codes_ld % 16 || b->codes_ld % 16 || ldd % (out_dtype ? 4 : 8)) return FOS_ERR_ALIGN;
  if (workspace) {
    if (workspace_bytes < gemm_workspace_bytes(M, N, K)) return FOS_ERR_WORKSPACE;
    if (!aligned(workspace, 16)) return FOS_ERR_ALIGN;
  }
  if (M == 0 || N == 0) return FOS_OK;
  if (K == 0) {
    const size_t es = out_dtype ? 4 : 2;
    return cudaMemset2DAsync(d, (size_t)ldd * es, 0, (size_t)N * es, (size_t)M, (cudaStream_t)stream) == cudaSuccess
               ? FOS_OK : FOS_ERR_CUDA;
  }
  const cudaError_t e = launch_gemm_nvfp4(a, b, (int)M, (int)N, (int)K, d, ldd, out_dtype, status,
                                          (cudaStream_t)stream, workspace);
  if (e == cudaErrorNotSupported) return FOS_ERR_UNSUPPORTED;
  return e == cudaSuccess ? FOS_OK : FOS_ERR_CUDA;
}

fos_status fos_amax(const void* x, int64_t batch, int64_t rows, int64_t cols, int64_t ld,
                    const fos_options* opt, float* amax_out, uint32_t* status, void* stream) {
  if (!x || !opt || !amax_out) return FOS_ERR_NULL;
  if (opt->flags & ~(FOS_FLAG_RHT16 | FOS_FLAG_SCALE_SWIZZLED)) return FOS_ERR_ARG;
  if (batch < 0 || rows < 0 || cols < 0 || batch > 65535) return FOS_ERR_SHAPE;
  if (cols % 16) return FOS_ERR_SHAPE;
  if (!aligned(x, 16) || ld % 8 != 0 || !aligned(amax_out, 4)) return FOS_ERR_ALIGN;
  if (ld < cols) return FOS_ERR_SHAPE;
  if (rows > 0 && cols > 0 && rows * (cols / 16) >= (1ll << 31)) return FOS_ERR_SHAPE;
  cudaStream_t st = (cudaStream_t)stream;
  if (batch == 0) return FOS_OK;
  if (cudaMemsetAsync(amax_out, 0, 4 * batch, st) != cudaSuccess) return FOS_ERR_CUDA;
  if (rows == 0 || cols == 0) return FOS_OK;
  QuantArgs a;
  a.x = (const uint16_t*)x;
  a.ld = ld;
  a.x_bs = rows * ld;
  a.rows = (int)rows;
  a.cols = (int)cols;
  a.nblk = (uint32_t)(rows * (cols / 16));
  a.bpr = make_fastdiv((uint32_t)(cols / 16));
  a.status = status;
  a.seed = opt->seed;
  a.units_per_cta = kUnitsAmax;
  return launch_amax(a, (int)batch, (opt->flags & FOS_FLAG_RHT16) != 0, (uint32_t*)amax_out, st) ==
                 cudaSuccess
             ? FOS_OK
             : FOS_ERR_CUDA;
}

fos_status fos_dequantize(const fos_qtensor* q, int32_t fmt, int64_t batch, int64_t rows,
                          int64_t cols, uint32_t flags, void* y, int64_t ldy, void* stream) {
  if (!q || !y) return FOS_ERR_NULL;
  if (fmt < 0 || fmt > 2 || (flags & ~(FOS_FLAG_RHT16 | FOS_FLAG_SCALE_SWIZZLED))) return FOS_ERR_ARG;
  if (batch < 0 || rows < 0 || cols < 0 || batch > 65535) return FOS_ERR_SHAPE;
  const bool mx = fmt == FOS_FMT_MXFP4;
  const int64_t bs = mx ? 32 : 16;
  if (cols % bs) return FOS_ERR_SHAPE;
  fos_status e = check_out(q, rows, cols, bs, !mx, flags);
  if (e != FOS_OK) return e;
  if (!aligned(y, 16) || ldy % 8 != 0) return FOS_ERR_ALIGN;
  if (ldy < cols) return FOS_ERR_SHAPE;
  if (rows > 0 && cols > 0 && rows * (cols / bs) >= (1ll << 31)) return FOS_ERR_SHAPE;
  if (batch == 0 || rows == 0 || cols == 0) return FOS_OK;
  const OutDesc o = make_out(q, rows, cols, bs, flags, rows * (cols / bs));
  DequantArgs a;
  a.codes = o.codes;
  a.codes_ld = o.codes_ld;
  a.codes_bs = o.codes_bs;
  a.scales = o.scales;
  a.scales_ld = o.scales_ld;
  a.scales_bs = o.scales_bs;
  a.col_tiles = o.col_tiles;
  a.tensor_scale = q->tensor_scale;
  a.y = (uint16_t*)y;
  a.ldy = ldy;
  a.y_bs = ldy * rows;
  a.rows = (int)rows;
  a.cols = (int)cols;
  a.nblk = (uint32_t)(rows * (cols / bs));
  a.bpr = make_fastdiv((uint32_t)(cols / bs));
  a.units_per_cta = kUnitsDeq;
  const bool swz = (flags & FOS_FLAG_SCALE_SWIZZLED) != 0;
  const bool dense = !swz && q->codes_ld * 2 == cols && q->scales_ld * bs == cols && ldy == cols &&
                     aligned(y, 32);
  return launch_dequant(a, (int)batch, mx, swz, dense, (cudaStream_t)stream) == cudaSuccess ? FOS_OK
                                                                                            : FOS_ERR_CUDA;
}

}  // extern "C"
