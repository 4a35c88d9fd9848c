// tcgen05 grouped GEMMs (placeholder until the tensor-core kernels land).
#include "common.cuh"
#include "internal.h"

namespace moe {
bool tc_available() { return false; }
int tc_num_dS_parts(int f) { return 1; }
int tc_ffn_fwd(const FfnPtrs&, const void*, void*, void*, void*, int, cudaStream_t) {
  return fail(MOE_ERR_UNSUPPORTED, "tensor-core path not built");
}
int tc_ffn_bwd(const FfnPtrs&, const void*, const void*, const float*, const void*, void*, void*,
               float*, void*, void*, void*, void*, int, cudaStream_t) {
  return fail(MOE_ERR_UNSUPPORTED, "tensor-core path not built");
}
}  // namespace moe
