// fos_tiles.cu -- quantizers that need both orientations of a tile:
// rowwise + colwise 1x16 and 16x16 2D block scaling.
#include "fos.h"
#include "fos_internal.h"

namespace fos {

cudaError_t launch_q1x16_dual(const QuantArgs&, int, int, bool, bool, bool, cudaStream_t) {
  return cudaErrorNotSupported;
}

cudaError_t launch_q16x16(const QuantArgs&, int, int, bool, bool, bool, bool, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace fos
