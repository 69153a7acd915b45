// Full attention layer with fused block scores on the 5th-generation tensor cores.
#include "common.cuh"
#include "kernels.h"

namespace hys {

bool full_attn_tc_supported(const PrefillDims&, hys_dtype) { return false; }
size_t full_attn_tc_workspace(const PrefillDims&) { return 0; }
cudaError_t launch_full_attn_tc(const PrefillDims&, const void*, const void*, const void*, void*, float*, float*,
                                hys_reduce, bool, void*, size_t, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace hys
