// FP8 attention (placeholder until the e4m3 kernels land).
#include "dit_device.cuh"

namespace dit {
cudaError_t launch_fp8_prologue(const Fp8Prep&, cudaStream_t) { return cudaErrorNotSupported; }
cudaError_t launch_attn_fp8(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&, const AttnOut&, const Fp8Prep&,
                            cudaStream_t) {
  return cudaErrorNotSupported;
}
}  // namespace dit
