// Tensor-core greedy pursuit encoder (placeholder until the sm_100a kernel
// lands): declines every shape, so sdk_encode runs the CUDA-core encoder.
#include "sdk_internal.cuh"

namespace sdk {

size_t encode_tc_scratch_bytes(int64_t, int, int) { return 0; }

sdk_status launch_encode_tc(const EncodeParams&, int, void*, size_t, cudaStream_t, bool* taken) {
  *taken = false;
  return SDK_OK;
}

}  // namespace sdk
