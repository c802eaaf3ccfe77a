// Shared-memory staged bf16 / head_dim 128 decode kernels (not built yet:
// every call falls through to the generic kernel).
#pragma once

#include "decode_common.cuh"

namespace pagedkv {

inline pa_status launch_staged_bf16_d128(const DecodeParams&, cudaStream_t) {
  return PA_ERR_UNSUPPORTED;
}

}  // namespace pagedkv
