/*
 * fos_testing.h -- test hooks exported by libfos.so.  Not part of the
 * quantizer's interface (include/fos.h); tests use them to drive code paths
 * that valid input never reaches, without faulting or hanging the GPU.
 */
#ifndef FOS_TESTING_H_
#define FOS_TESTING_H_

#include "fos.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * fos_testing_quantize_stalled -- fos_quantize (NVFP4, 1x16, rowwise, amax
 * computed in the call, so the fused amax + quantize kernel runs) with a
 * failure planted on the host side: the amax items of batch entry
 * `stall_entry` never count in, and every bounded wait of the kernel gives
 * up after `spin_limit` polls (each an L2 round trip plus a 128 ns sleep)
 * instead of 2^21.
 *
 * The first wait on that entry runs out, sets FOS_STATUS_TIMEOUT in *status
 * (status must not be NULL to see it) and ends every other wait of the
 * launch, so the launch still ends.  The entries before the stalled one are
 * quantized exactly as by fos_quantize; the outputs of the stalled entry and
 * of the entries after it are unspecified.  Arguments
 * are those of fos_quantize; stall_entry must be in [0, batch) and
 * spin_limit >= 1 (FOS_ERR_ARG otherwise); other formats and block modes
 * return FOS_ERR_UNSUPPORTED.
 */
fos_status fos_testing_quantize_stalled(const void* x, int64_t batch, int64_t rows, int64_t cols,
                                        int64_t ld, const fos_options* opt,
                                        const fos_qtensor* rowwise, void* workspace,
                                        size_t workspace_bytes, uint32_t* status,
                                        int32_t stall_entry, uint32_t spin_limit, void* stream);

/*
 * fos_testing_quantize_2d_strip -- fos_quantize with the 16x16 2D kernel's
 * strip length forced to `nsub` sub-tiles of 64 rows (1..8) instead of the
 * length the library picks per launch to fill the GPU's resident CTA slots.
 * Tests use it to reach every strip length, and the transposed copy's
 * whole-word choice-bitmap stores that only strips of 8 take.  Arguments and
 * outputs are those of fos_quantize: the results do not depend on the strip
 * length.  opt->blk must be FOS_BLOCK_16X16 (FOS_ERR_UNSUPPORTED otherwise);
 * nsub outside 1..8 gives FOS_ERR_ARG.
 */
fos_status fos_testing_quantize_2d_strip(const void* x, int64_t batch, int64_t rows, int64_t cols,
                                         int64_t ld, const fos_options* opt, const float* amax_in,
                                         const fos_qtensor* rowwise, const fos_qtensor* colwise,
                                         void* workspace, size_t workspace_bytes, uint32_t* status,
                                         int32_t nsub, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FOS_TESTING_H_ */
