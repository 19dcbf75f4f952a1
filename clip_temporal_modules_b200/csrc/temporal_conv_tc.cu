// Tensor-core (tcgen05) path of the temporal convolution: not yet enabled.
#include "vi_internal.cuh"

namespace vi {

bool temporal_conv_tc_ok(int, int, int, int) { return false; }

int temporal_conv_bf16_tc(const bf16*, const bf16*, const bf16*, bf16*, int, int, int, int,
                          cudaStream_t) {
  return VI_ERR_UNSUPPORTED;
}

}  // namespace vi
