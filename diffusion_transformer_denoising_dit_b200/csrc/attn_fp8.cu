// FP8 (e4m3) joint attention over the prologue's quantised Q, smoothed K and
// V with their per-block scales: S = Q8 K8^T (kind::f8f6f4, fp32 accumulate),
// scores = S * sQ * sK(j) * scale folded into the softmax FFMA, P = exp2 in
// fp32 then P * 448 * sV(j) / sV_max cast to e4m3, O += P8 V8, and the
// epilogue multiplies by sV_max / 448 / l.
// Sources: "FLUX 3 Image Klein / TensorRT-LLM VisualGen" (cuDNN FP8 attention
// against VANILLA BF16 on B200) and "vflash / Optimization ledger", table
// "Accepted or exposed" (SageAttention2, quantised attention).
// With Q and K in symmetric int8 (the prologue's qk_int8 mode) S = Q8 K8^T is
// a kind::i8 MMA with s32 accumulation instead, scaled the same way.
// The kernel itself is the shared template in attn_kernel.cuh.
#include "attn_kernel.cuh"

namespace dit {

cudaError_t launch_attn_fp8(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const AttnOut& out,
                            const Fp8Prep& p, cudaStream_t stream) {
  AttnScales sc;
  sc.q_scale = p.q_scale;
  sc.k_scale = p.k_scale;
  sc.v_scale = p.v_scale;
  sc.v_scale_max = p.v_scale_max;
  sc.H = p.H;
  if (p.qk_int8) return launch_attn<true, 128, true>(tq, tk, tv, out, sc, p.B, p.H, stream);
  return launch_attn<true, 128>(tq, tk, tv, out, sc, p.B, p.H, stream);
}

}  // namespace dit
