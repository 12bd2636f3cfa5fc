// fos_static.cu -- fos_quantize_static: the quantizer with its scratch
// memory in a file-scope device array instead of a caller-provided
// workspace, for callers that cannot or must not allocate device memory
// (see include/fos.h).
//
// The only scratch the quantizer needs is the per-batch-entry amax words of
// the amax pass (plus a little padding); here they live in g_scratch, sized
// for kStaticMaxBatch batch entries.  Every GPU that loads this library
// holds the array until the process exits.
#include <mutex>

#include "fos.h"
#include "fos_internal.h"

namespace {

constexpr int64_t kStaticMaxBatch = FOS_STATIC_MAX_BATCH;
// the workspace fos_quantize needs for kStaticMaxBatch entries
constexpr size_t kScratchBytes = fos::workspace_bytes_for(kStaticMaxBatch);
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_scratch[kScratchBytes];

std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_scratch on the current device.  In host code the name
// g_scratch is only a host-side stand-in, so the address is looked up once
// per device with that device current and cached.
fos_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FOS_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) return FOS_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return FOS_OK;
}

}  // namespace

extern "C" {

fos_status fos_quantize_static(const void* x, int64_t batch, int64_t rows, int64_t cols,
                               int64_t ld, const fos_options* opt, const float* amax_in,
                               const fos_qtensor* rowwise, const fos_qtensor* colwise,
                               uint32_t* status, void* stream) {
  // only calls that compute the amax use scratch (MXFP4 and calls with
  // amax_in need none): the batch limit applies to those alone
  const bool needs_scratch = opt && opt->fmt != FOS_FMT_MXFP4 && (!amax_in || (opt->flags & FOS_FLAG_RHT16_COL));
  if (needs_scratch && batch > kStaticMaxBatch) return FOS_ERR_WORKSPACE;
  void* scratch = nullptr;
  const fos_status e = scratch_address(&scratch);
  if (e != FOS_OK) return e;
  // fos_quantize clears the amax words it uses on `stream` before the amax
  // pass, so what an earlier call left in the array does not matter.
  return fos_quantize(x, batch, rows, cols, ld, opt, amax_in, rowwise, colwise, scratch,
                      kScratchBytes, status, stream);
}

}  // extern "C"
