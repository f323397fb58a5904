// FP8 E4M3 block-scaled grouped GEMMs (W8A8, 128x128 weight blocks, 1x128 activation
// groups). Not built yet: the launchers report cudaErrorNotSupported and the C ABI
// answers MOE_ERR_UNSUPPORTED for MOE_DTYPE_FP8_BLOCK128 forwards.
#include "moe_device.cuh"
#include "moe_internal.h"

namespace moe {

size_t gemm_fp8_smem_bytes() { return 0; }

cudaError_t launch_gemm1_fp8(const Launch&, const CUtensorMap&, const CUtensorMap&, const GemmShape&,
                             const GemmBuffers&) {
  return cudaErrorNotSupported;
}

cudaError_t launch_gemm2_fp8(const Launch&, const CUtensorMap&, const CUtensorMap&, const GemmShape&,
                             const GemmBuffers&) {
  return cudaErrorNotSupported;
}

}  // namespace moe
