// Internal launcher interface between the C ABI (capi.cu) and the kernel
// translation units.  Not part of the public header.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace dit {

// Launches `kernel` as a programmatic dependent of the grid before it on the
// stream: it may be scheduled once every CTA of that grid has called
// pdl_trigger (or exited), and it must call pdl_wait before it reads anything
// that grid writes.
template <typename... Params, typename... Args>
cudaError_t launch_dependent(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                             Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Keys per K/V tile of the attention kernels (the TMA box height of the K and V maps).
constexpr int kAttnBlockN = 128;

// Error codes written to the device error word (match dit_status).
constexpr int kErrTimeout = 6;
constexpr int kErrBounds = 7;  // debug builds only (DIT_DEBUG): an index failed its bounds check

// Gate: number of pass-1 CTAs for n elements, and its workspace (2 doubles per CTA).
int gate_num_ctas(int64_t n);

cudaError_t launch_rope_tables(const int32_t* pos, int N, int d0, int d1, int d2, double theta, float* cos_out,
                               float* sin_out, cudaStream_t stream);

// One strided [B,H,N,d] rotary job.
struct RopeJob {
  const void* x;
  void* y;
  int64_t sx[3];
  int64_t sy[3];
};

// Applies rotary embedding to njobs (1 or 2) tensors of the same shape in one launch
// (nothing when skip is non-null and *skip != 0 at execution time).
cudaError_t launch_rope_apply(const RopeJob* jobs, int njobs, int B, int H, int N, int d, const float* cos_tab,
                              const float* sin_tab, int out_fp32, cudaStream_t stream,
                              const int32_t* skip = nullptr);

cudaError_t launch_gate(const void* a, const void* b, int64_t n, float threshold, float* rel_out, int32_t* skip_out,
                        double* partials, cudaStream_t stream);
// Sharded gate: the totals (sum |a - b|, sum |b|) of one shard, and the decision
// from totals summed across shards.
cudaError_t launch_gate_sums(const void* a, const void* b, int64_t n, double* sums_out, double* partials,
                             cudaStream_t stream);
cudaError_t launch_gate_finalize(const double* sums, float threshold, float* rel_out, int32_t* skip_out,
                                 cudaStream_t stream);

// ref = cur (n bf16 elements, 16-byte aligned) unless skip is non-null and *skip != 0
// at execution time.
cudaError_t launch_gate_ref_update(const void* cur, void* ref, int64_t n, const int32_t* skip, cudaStream_t stream);

// Output description shared by the attention kernels.
struct AttnOut {
  void* o;          // bf16 [B,H,N,d]
  int64_t so[3];    // element strides {batch, head, token}
  int N;
  float scale_log2;  // softmax scale * log2(e)
  int* err;          // device error word
  // BF16 only: fp32 [N][d/2] rotary tables for Q, applied as the attention
  // kernel loads Q (both null: Q is used as given).  FP8 takes Q rotated and
  // quantised by its prologue.
  const float* rope_cos;
  const float* rope_sin;
  // when non-null and *skip != 0 at execution time the launch does nothing
  const int32_t* skip;
};

cudaError_t launch_attn_bf16(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const AttnOut& out,
                             int B, int H, int d, cudaStream_t stream);

// FP8 prologue: K channel means (fp32 [B*H][d]) of the rotated K.
struct Fp8Prep {
  const void* q;
  const void* k;
  const void* v;
  int64_t sq[3], sk[3], sv[3];
  const float* cos_tab;  // may be null (no rotary)
  const float* sin_tab;
  int B, H, N, d;
  int q_block, kv_block;
  int smooth_k;
  // 0: Q and K in e4m3 (scale amax/448); 1: Q and K in symmetric int8 (scale
  // amax/127, for the 8-bit integer Q.K^T).  V is e4m3 either way.
  int qk_int8;
  // workspace carve-out
  uint8_t* q8;      // e4m3 [B,H,N,d]
  uint8_t* k8;      // e4m3 [B,H,N,d]
  uint8_t* v8;      // e4m3 [B,H,N,d]
  float* q_scale;   // [B*H][ceil(N/q_block)]
  float* k_scale;   // [B*H][ceil(N/kv_block)]
  float* v_scale;   // [B*H][ceil(N/kv_block)]
  float* k_mean;    // [B*H][d]
  float* v_scale_max;  // [B*H]
  float* k_partial;    // [B*H][kFp8MeanChunks][128] K-mean partial sums
  int* err;            // device error word (a staged copy that timed out)
  int num_sms;         // the quantiser runs one persistent CTA per SM
};

constexpr int kFp8MeanChunks = 48;

cudaError_t launch_fp8_prologue(const Fp8Prep& p, cudaStream_t stream);

// One thread waits (bounded) on an mbarrier nothing arrives on: records kErrTimeout.
cudaError_t launch_selftest_wait(int* err, cudaStream_t stream);

// FP8 attention over the prologue's output; p.qk_int8 selects the Q.K^T form.
cudaError_t launch_attn_fp8(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const AttnOut& out,
                            const Fp8Prep& p, cudaStream_t stream);

}  // namespace dit
