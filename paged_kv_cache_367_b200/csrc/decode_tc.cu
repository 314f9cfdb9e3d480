// Tensor-core PagedAttention decode (16-bit caches). Not yet built: every
// configuration goes to the CUDA-core kernel.
#include "schedule.cuh"

namespace pkv {

bool tc_supported(int, int, int, int) { return false; }

cudaError_t launch_decode_tc(const DecodeParams&, int, int, int, int, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace pkv
