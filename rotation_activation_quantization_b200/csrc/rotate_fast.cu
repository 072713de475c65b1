// Fused fast kernels (filled in per shape). Returning cudaErrorNotSupported hands the call to the
// generic kernel.
#include "signrot_internal.h"

namespace signrot {

cudaError_t launch_rotate_fast(const RotateArgs&, const H28Masks&, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace signrot
