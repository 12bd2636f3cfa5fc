/*
 * fos.h -- C ABI of libfos.so: Four Over Six (4/6) NVFP4 block quantization
 * for NVIDIA B200 (sm_100a), with its options and comparison formats.
 *
 * What the library computes (sources, by page and section):
 *  - Hugging Face transformers doc "Four Over Six", introduction: every NVFP4
 *    block is scaled adaptively so that its largest magnitude maps to 4 or to
 *    6, to cut the quantization error of the values near the block maximum.
 *    The candidate with the lower block squared error is kept; ties keep 6.
 *  - Same doc, usage section: the options random Hadamard transform, 2D
 *    block scaling, transposed inputs and stochastic rounding.
 *  - Ultralytics glossary "FP4", introduction: the E2M1 element format and
 *    its value set {0, +-0.5, +-1, +-1.5, +-2, +-3, +-4, +-6}.
 *  - Same page, "Como funciona FP4": NVFP4 = 16 values under an E4M3 scale
 *    plus an FP32 per-tensor scale; MXFP4 = 32 values under an 8-bit
 *    power-of-two (E8M0) scale; each block's largest magnitude maps near 6.
 *
 * Conventions shared by every entry point:
 *  - All data pointers are DEVICE pointers on the current CUDA device, except
 *    the option/descriptor structs, which are read on the host during the
 *    call and may be freed when it returns.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every
 *    call only enqueues work on `stream`; nothing is synchronised, allocated
 *    or freed.  Outputs are valid once the stream reaches that point.
 *  - The caller owns every buffer.  Argument errors are returned at once and
 *    nothing is enqueued.  Data errors (NaN/Inf input) are reported
 *    asynchronously by OR-ing FOS_STATUS_* bits into *status (if non-NULL);
 *    the outputs are then unspecified.
 *  - Packed E2M1 codes: element 2k in the low nibble of byte k, 2k+1 in the
 *    high nibble; bit 3 of a nibble is the sign (-0 is kept), bits 0..2 the
 *    magnitude index into {0, 0.5, 1, 1.5, 2, 3, 4, 6}.
 */
#ifndef FOS_H_
#define FOS_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define FOS_VERSION 1

typedef enum fos_status {
  FOS_OK = 0,
  FOS_ERR_NULL = 1,        /* a required pointer is NULL */
  FOS_ERR_ALIGN = 2,       /* a pointer or leading dimension breaks alignment */
  FOS_ERR_SHAPE = 3,       /* sizes not divisible by the block, or negative */
  FOS_ERR_UNSUPPORTED = 4, /* option combination not implemented */
  FOS_ERR_WORKSPACE = 5,   /* workspace missing or smaller than required */
  FOS_ERR_CUDA = 6,        /* a CUDA launch or memset failed */
  FOS_ERR_ARG = 7          /* enum value out of range, bad flag, bad offset */
} fos_status;

typedef enum fos_format {
  FOS_FMT_NVFP4_46 = 0, /* NVFP4, 4/6 adaptive block scale (the method) */
  FOS_FMT_NVFP4_6 = 1,  /* NVFP4, block max always mapped to 6 */
  FOS_FMT_MXFP4 = 2     /* MXFP4: 32-element blocks, E8M0 scale */
} fos_format;

typedef enum fos_block {
  FOS_BLOCK_1X16 = 0,  /* 16 consecutive elements of a row (NVFP4) */
  FOS_BLOCK_16X16 = 1, /* 16x16 tile: one scale and one 4/6 choice (NVFP4) */
  FOS_BLOCK_1X32 = 2   /* 32 consecutive elements of a row (MXFP4) */
} fos_block;

typedef enum fos_round {
  FOS_ROUND_RNE = 0, /* round to nearest, ties to even, saturating at 6 */
  FOS_ROUND_SR = 1   /* stochastic rounding with Philox4x32-10 bytes */
} fos_round;

/* fos_options.flags */
#define FOS_FLAG_RHT16 0x1u          /* 16-wide random Hadamard transform (1x16, rowwise only) */
#define FOS_FLAG_SCALE_SWIZZLED 0x2u /* scales in the 128x4 tensor-core tile layout */
#define FOS_FLAG_RHT16_COL 0x4u      /* the same transform along rows for the colwise copy (1x16 NVFP4) */

/* bits OR-ed into *status by the device */
#define FOS_STATUS_NONFINITE 0x1u /* a NaN or Inf was read; outputs unspecified */
#define FOS_STATUS_TIMEOUT 0x2u   /* a bounded device-side wait gave up */

typedef struct fos_options {
  int32_t fmt;         /* fos_format */
  int32_t blk;         /* fos_block: 1X16 or 16X16 for NVFP4, 1X32 for MXFP4 */
  int32_t rnd;         /* fos_round: SR needs NVFP4 */
  uint32_t flags;      /* FOS_FLAG_* */
  uint64_t seed;       /* Philox key: (seed & 0xffffffff, seed >> 32) */
  int64_t elem_offset; /* global linear index of x[0,0,0] in the full tensor,
                          for stochastic rounding of shards; multiple of 16 */
} fos_options;

/* One quantized orientation.  Layout of a tensor with R rows and C columns
 * (rowwise: R = rows, C = cols; colwise: R = cols, C = rows):
 *   codes  uint8 [batch][R][codes_ld], codes_ld >= C/2, multiple of 8 bytes;
 *          batch stride R * codes_ld.  16-byte aligned.
 *   scales uint8: linear layout [batch][R][scales_ld], scales_ld >= C/bs
 *          (bs = 16 or 32), batch stride R * scales_ld; or, with
 *          FOS_FLAG_SCALE_SWIZZLED, fos_scales_size(R, C/bs, flags) bytes per
 *          batch entry (scales_ld ignored; padding bytes are not written:
 *          zero them once, since block-scaled tensor-core GEMMs read the
 *          padded scales of partial tiles).
 *          NVFP4: E4M3 codes; MXFP4: E8M0 codes (2^(byte-127)).
 *          In 16x16 mode the tile's scale is repeated in each of its 16 rows.
 *   tensor_scale float [batch]: the FP32 per-tensor scale S_t (NVFP4; the
 *          rowwise and colwise copies get the same value; NULL allowed only
 *          for MXFP4).
 *   choice_bits uint8, nullable: bit b (byte b>>3, bit b&7) = 1 when linear
 *          block b kept the 4-candidate: blocks over [batch][R][C/16], or,
 *          in 16x16 mode, tiles over [batch][R/16][C/16] in the tile
 *          row-major order of this copy's own [R][C].  For the transposed
 *          copy (R = cols, C = rows) the source tile at tile row tr, tile
 *          column tc is therefore bit (b*(cols/16) + tc)*(rows/16) + tr.
 *          The buffer must hold 8*ceil(nblocks/64) bytes: the library
 *          clears and writes it in whole 32- and 64-bit words. */
typedef struct fos_qtensor {
  uint8_t* codes;
  uint8_t* scales;
  float* tensor_scale;
  uint8_t* choice_bits;
  int64_t codes_ld;
  int64_t scales_ld;
} fos_qtensor;

/*
 * fos_quantize -- quantize x (bf16, [batch][rows][ld], 16-byte aligned,
 * ld % 8 == 0, ld >= cols) into `rowwise` and/or `colwise` (either may be
 * NULL, not both).
 *
 *  NVFP4 4/6 (fmt NVFP4_46): S_t = A / (4*448) with A the per-batch-entry
 *    amax of |x| (of the transformed x with RHT); per block with amax a:
 *    r = a / S_t, s6 = E4M3(r/6), s4 = E4M3(r/4); both candidates are
 *    rounded to E2M1 with v = |w| * (1 / (E4M3(s)*S_t)); the candidate with
 *    the lower binary32 block squared error is kept (ties keep 6).
 *  NVFP4 6-only: S_t = A / (6*448), only the 6-candidate.
 *  MXFP4: E = floor(log2 a) - 2 clamped to [-127, 127], codes = E2M1(w*2^-E).
 *  colwise != NULL: blk 1X16 quantizes x^T independently with 16-blocks
 *    along rows (same S_t); blk 16X16 writes the exact transpose of the
 *    rowwise codes and scales.  rows % 16 == 0.
 *  FOS_FLAG_RHT16_COL (NVFP4, blk 1X16, colwise != NULL): each 16-row
 *    colwise block is transformed like a rowwise RHT block (the seeded signs
 *    by position in the block, the 16-point Walsh-Hadamard butterfly, x0.25)
 *    before it is quantized, and the colwise copy takes its own S_t from the
 *    amax of the transformed columns (written to colwise->tensor_scale).
 *    That amax is always computed in the call, so the workspace is needed
 *    even with amax_in, which then sets the rowwise S_t only.  The rowwise
 *    copy is not transformed (FOS_FLAG_RHT16 with a colwise copy is
 *    FOS_ERR_UNSUPPORTED).
 *  FOS_ROUND_SR: the 4/6 choice is made on the RNE candidates, then the kept
 *    candidate is re-rounded stochastically: with v in [lo, hi) on the grid,
 *    round up iff 2*byte+1 < 512*(v-lo)/(hi-lo), byte j = g & 15 of
 *    Philox4x32-10(counter (g>>4, g>>36, 0, 0), key seed) for global element
 *    index g = elem_offset + linear index.  Both orientations use the same
 *    byte per source element.
 *  amax_in (nullable, device float [batch]): use these amaxes instead of
 *    computing them (e.g. after an all-reduce across shards).
 *  workspace: device memory of at least fos_workspace_size(...) bytes,
 *    16-byte aligned; its contents need not be initialised and are
 *    overwritten.  It must not be shared by calls that overlap on the GPU.
 * Returns FOS_OK or an error (nothing enqueued on error).
 */
fos_status fos_quantize(const void* x, int64_t batch, int64_t rows, int64_t cols, int64_t ld,
                        const fos_options* opt, const float* amax_in,
                        const fos_qtensor* rowwise, const fos_qtensor* colwise,
                        void* workspace, size_t workspace_bytes, uint32_t* status,
                        void* stream);

/*
 * fos_quantize_host -- fos_quantize of a batch held in HOST memory, with the
 * rowwise outputs returned to HOST memory, pipelined in chunks of `chunk`
 * batch entries on three caller streams: the host-to-device copy of chunk
 * k + 1 (stream_h2d), the quantization of chunk k (stream_compute, one
 * fos_quantize per chunk) and the device-to-host copy of chunk k - 1
 * (stream_d2h) overlap.  Each batch entry has its own S_t and the
 * stochastic-rounding counters follow the global element index, so the
 * results equal one fos_quantize over the whole batch.  (The copies are
 * data movement around the method; the quantization is the method's.)
 *
 *   x_host        bf16 [batch][rows][cols], dense, in pinned host memory
 *                 (pageable memory works, without overlap).
 *   opt, amax_in  as fos_quantize; rowwise 1x16 (NVFP4) or 1x32 (MXFP4)
 *                 blocks only, linear scale layout (no FOS_FLAG_SCALE_SWIZZLED,
 *                 no RHT16_COL); amax_in: DEVICE [batch] or NULL.
 *   out_host      HOST codes, scales and (NVFP4) tensor_scale with their row
 *                 strides; choice_bits must be NULL.
 *   x_dev         DEVICE staging input, bf16 [batch][rows][cols], 32-byte
 *                 aligned (rows of every chunk stay 16-byte aligned).
 *   out_dev       DEVICE outputs in the same layout as out_host (the same
 *                 codes_ld and scales_ld); choice_bits must be NULL.  Each
 *                 chunk's codes start chunk * rows * codes_ld bytes on and
 *                 must stay 16-byte aligned (FOS_ERR_ALIGN otherwise).
 *   workspace     DEVICE, fos_workspace_size(chunk, rows, cols, opt) bytes;
 *                 the chunks use it one after another on stream_compute.
 *   status        DEVICE word or NULL, as fos_quantize.
 *   chunk         batch entries per pipeline stage, >= 1.
 *   streams       cudaStream_t stream_h2d, stream_compute, stream_d2h; the
 *                 call orders the chunks between them with `events`.
 *   events        2 * ceil(batch / chunk) cudaEvent_t created by the caller
 *                 (cudaEventDisableTiming is enough), recorded by this call.
 *
 * Ownership: every buffer, stream and event belongs to the caller; nothing
 * is allocated.  The call only enqueues work and returns: the first copy
 * waits for nothing the caller does not order (make the three streams wait
 * on earlier work first), and the outputs are in host memory once
 * stream_d2h reaches the point where the call returned.  Errors:
 * FOS_ERR_NULL, FOS_ERR_ARG (chunk < 1), FOS_ERR_UNSUPPORTED (colwise-only
 * options, 2D blocks, swizzled scales, choice bits), then fos_quantize's own
 * codes for the shape and options, all returned before anything is
 * enqueued; FOS_ERR_CUDA when a copy, record or launch fails (earlier chunks
 * may already be enqueued).
 */
fos_status fos_quantize_host(const void* x_host, int64_t batch, int64_t rows, int64_t cols,
                             const fos_options* opt, const float* amax_in, const fos_qtensor* out_host,
                             void* x_dev, const fos_qtensor* out_dev, void* workspace,
                             size_t workspace_bytes, uint32_t* status, int64_t chunk, void* stream_h2d,
                             void* stream_compute, void* stream_d2h, void* const* events);

/* fos_amax -- per-batch-entry amax of |x| (of the 16-wide RHT of x when
 * opt->flags has FOS_FLAG_RHT16) into amax_out (device float [batch]).
 * NaN/Inf input sets FOS_STATUS_NONFINITE in *status.  Only opt->flags and
 * opt->seed are read. */
fos_status fos_amax(const void* x, int64_t batch, int64_t rows, int64_t cols, int64_t ld,
                    const fos_options* opt, float* amax_out, uint32_t* status, void* stream);

/* fos_dequantize -- q (codes, scales, tensor_scale; layout as above with
 * R = rows, C = cols) back to bf16 y [batch][rows][ldy] (ldy % 8 == 0).
 *  NVFP4: y = bf16_rne((sign*q * E4M3(s)) * S_t) (the first product is exact).
 *  MXFP4: y = bf16(sign*q * 2^(s-127)) (exact).
 * flags may hold FOS_FLAG_SCALE_SWIZZLED. */
fos_status fos_dequantize(const fos_qtensor* q, int32_t fmt, int64_t batch, int64_t rows,
                          int64_t cols, uint32_t flags, void* y, int64_t ldy, void* stream);

/*
 * fos_fake_quantize -- quantize x and dequantize it again in one pass, with
 * bf16 output y [batch][rows][ldy] (16-byte aligned, ldy % 8 == 0,
 * ldy >= cols): y = fos_dequantize(fos_quantize(x)) bit for bit, without
 * writing codes or scales.  This is the simulated-FP4 path ("fake
 * quantization") that the Hugging Face transformers doc "Four Over Six"
 * names for hardware without FP4 tensor cores (introduction), and the
 * forward of quantization-aware training.
 *  NVFP4 (4/6 or 6-only): blk 1X16 rowwise, RNE or SR, with or without
 *    FOS_FLAG_RHT16 (y is then in the rotated domain, like fos_dequantize's);
 *    the per-entry amax is amax_in or computed in the call (workspace as for
 *    fos_quantize).
 *  MXFP4: blk 1X32, RNE; no workspace.
 *  16x16 tiles return FOS_ERR_UNSUPPORTED.  Other arguments and errors are
 *  those of fos_quantize; NaN/Inf input sets FOS_STATUS_NONFINITE.
 */
fos_status fos_fake_quantize(const void* x, int64_t batch, int64_t rows, int64_t cols, int64_t ld,
                             const fos_options* opt, const float* amax_in, void* y, int64_t ldy,
                             void* workspace, size_t workspace_bytes, uint32_t* status, void* stream);

/*
 * fos_gemm_nvfp4 -- the FP4 matrix product the quantized tensors are made
 * for, on the B200 tensor cores (tcgen05.mma kind::mxf4nvf4, 16-element
 * E4M3 block scales, FP32 accumulation):
 *   D[m][n] = (S_tA * S_tB) * sum_k A[m][k] * B[n][k]
 * where A (M x K) and B (N x K) are rowwise NVFP4 quantizations along K
 * from fos_quantize with FOS_FLAG_SCALE_SWIZZLED (a and b as filled by it,
 * batch 1; 6-only and 4/6 alike: the 4/6 choice is already in the scales).
 * Ultralytics glossary "FP4", "Inferencia e Treinamento FP4": FP4 matrix
 * multiplication on Blackwell tensor cores.
 *  a->codes [M][codes_ld] (codes_ld >= K/2, multiple of 16), a->scales the
 *  swizzled [M][K/16] scales (fos_scales_size(M, K/16, swizzled) bytes),
 *  a->tensor_scale one float; the same for b with N.  choice_bits unused.
 *  d: [M][ldd] bf16 (out_dtype 0) or f32 (out_dtype 1), 16-byte aligned,
 *  ldd >= N, ldd * element size a multiple of 16.
 *  M and N multiples of 128, K a multiple of 256 (FOS_ERR_SHAPE otherwise).
 *  A device-side wait that gives up sets FOS_STATUS_TIMEOUT in *status
 *  (nullable); D is then unspecified.
 */
fos_status fos_gemm_nvfp4(const fos_qtensor* a, const fos_qtensor* b, int64_t M, int64_t N, int64_t K,
                          void* d, int64_t ldd, int32_t out_dtype, uint32_t* status, void* stream);

/*
 * fos_gemm_nvfp4_ws -- fos_gemm_nvfp4 with a device workspace of
 * fos_gemm_workspace_size(M, N, K) bytes (16-byte aligned; NULL gives
 * fos_gemm_nvfp4).  The call first rewrites a's and b's swizzled scales into
 * the workspace as copy sources of the tensor core's 128 x 256-bit scale
 * copy (each 16-byte atom row four times; 4x the scale bytes), then runs the
 * product with 6 scale copies per 256-wide K step instead of 12 (4 instead
 * of 8 for 128 x 128 tiles).  Same result as fos_gemm_nvfp4, bit for bit; the
 * workspace is only read by this call's kernels and may be reused once the
 * stream has passed them.  Errors: those of fos_gemm_nvfp4, and
 * FOS_ERR_WORKSPACE / FOS_ERR_ALIGN for a small or misaligned workspace.
 */
size_t fos_gemm_workspace_size(int64_t M, int64_t N, int64_t K);
fos_status fos_gemm_nvfp4_ws(const fos_qtensor* a, const fos_qtensor* b, int64_t M, int64_t N, int64_t K,
                             void* d, int64_t ldd, int32_t out_dtype, void* workspace, size_t workspace_bytes,
                             uint32_t* status, void* stream);

/*
 * fos_quantize_static -- fos_quantize without a workspace argument, for
 * callers that cannot allocate device memory: code that runs inside a stream
 * capture (cudaMalloc cannot be captured), serving paths that must not
 * allocate because an allocation can synchronize the device, and hosts or
 * plugins whose memory is owned by another allocator that hands out no
 * scratch buffers.  The method itself has no such call; this is a deployment aid.
 *
 * Arguments, outputs and errors are those of fos_quantize.  The scratch
 * memory (per-batch-entry amax words and counters) lives in a fixed array in the
 * library, sized for FOS_STATIC_MAX_BATCH batch entries; every GPU that
 * loads the library holds it (about 49 KB) until the process exits.
 * A call that needs the scratch (NVFP4 without amax_in) with batch >
 * FOS_STATIC_MAX_BATCH returns FOS_ERR_WORKSPACE; MXFP4 calls and calls with
 * amax_in use no scratch and take any batch fos_quantize takes.  No device
 * memory is allocated or freed.
 *
 * The first call on a device looks up the array's device address (with that
 * device current) and keeps it; make that first call before any stream
 * capture.  All calls share the one array: calls that overlap on the GPU
 * (other streams, other host threads, concurrent graph launches) race and
 * give wrong results.  Each call clears the words it uses before reading
 * them, so the contents left by an earlier call do not matter.
 */
#define FOS_STATIC_MAX_BATCH 4096
fos_status fos_quantize_static(const void* x, int64_t batch, int64_t rows, int64_t cols,
                               int64_t ld, const fos_options* opt, const float* amax_in,
                               const fos_qtensor* rowwise, const fos_qtensor* colwise,
                               uint32_t* status, void* stream);

/* Bytes of workspace fos_quantize needs for this call. */
size_t fos_workspace_size(int64_t batch, int64_t rows, int64_t cols, const fos_options* opt);

/* Bytes of one batch entry's scale array for a [R][sf_cols] scale matrix:
 * R*sf_cols (linear) or 128*ceil(R/128) * 4*ceil(sf_cols/4) (swizzled). */
size_t fos_scales_size(int64_t R, int64_t sf_cols, uint32_t flags);

/* Static description of a status code. */
const char* fos_status_string(int32_t status);

/* FOS_VERSION of the built library. */
int32_t fos_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FOS_H_ */
