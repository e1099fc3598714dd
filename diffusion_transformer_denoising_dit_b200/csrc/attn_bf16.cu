// BF16 joint attention: operands bf16, fp32 accumulation and softmax, bf16 output.
// Source: "FLUX 3 Image Klein / TensorRT-LLM VisualGen", section on why the
// differences arise (VANILLA BF16 attention, about 60 % of DiT GPU kernel time).
// The kernel itself is the shared template in attn_kernel.cuh.
#include "attn_kernel.cuh"

namespace dit {

cudaError_t launch_attn_bf16(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const AttnOut& out,
                             int B, int H, int d, cudaStream_t stream) {
  const AttnScales none{};
  if (d == 128) return launch_attn<false, 128>(tq, tk, tv, out, none, B, H, stream);
  if (d == 64) return launch_attn<false, 64>(tq, tk, tv, out, none, B, H, stream);
  return cudaErrorInvalidValue;
}

}  // namespace dit
