// Unit-rate probes: the hardware rates the attention kernels' rooflines are
// drawn against, measured on the device they run on.
//
//   * tcgen05.mma throughput for the kernels' MMA shape (M = 128, N = 128, both
//     operands in shared memory; e4m3 kind::f8f6f4 and bf16 kind::f16): one CTA
//     per SM, one thread issuing back-to-back MMAs on zero-filled operands.
//   * ex2.approx.f32 (the softmax's exponential) and cvt.rn.satfinite.e4m3x2.f32
//     (its P conversion): eight independent chains per thread, one CTA of 32
//     warps per SM, timed between two CTA barriers.
//
// Each rate is per clock per SM, from clock64 cycle counts taken on the device, so
// it does not depend on the clock the probe happened to run at.  Every wait is the
// library's bounded mbarrier wait.
#include <cuda_runtime.h>

#include "dit.h"
#include "dit_device.cuh"

namespace dit {
namespace {

template <bool FP8>
__global__ void __launch_bounds__(128, 1) mma_rate_kernel(int reps, int* err, long long* cycles) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;              // 128 rows x 128 bytes
  uint8_t* sB = smem + 128 * 128;  // 128 rows x 128 bytes
  __shared__ uint64_t bar;
  __shared__ uint32_t slot;
  for (int i = threadIdx.x; i < 2 * 128 * 128 / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(smem)[i] = make_uint4(0u, 0u, 0u, 0u);
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  fence_proxy_async_smem();
  if (threadIdx.x < 32) {
    tmem_alloc(&slot, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = slot;
  if (threadIdx.x == 0) {
    const long long t0 = clock64();
    const uint32_t a = smem_u32(sA), b = smem_u32(sB);
    constexpr uint32_t idesc = FP8 ? make_idesc(0, 0, 0, 128, 128) : make_idesc(1, 1, 0, 128, 128);
    for (int r = 0; r < reps; ++r) {
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {  // 32 bytes of K per MMA, one 128-byte swizzle row per 4
        const uint64_t ad = smem_desc_sw128(a + kk * 32, 16, 1024), bd = smem_desc_sw128(b + kk * 32, 16, 1024);
        if constexpr (FP8)
          mma_f8_ss(tmem, ad, bd, idesc, 1u);
        else
          mma_f16_ss(tmem, ad, bd, idesc, 1u);
      }
    }
    mma_commit(&bar);
    if (mbar_wait(&bar, 0, err, kErrTimeout) && blockIdx.x == 0) *cycles = clock64() - t0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x < 32) tmem_dealloc(tmem, 128);
}

// op 0: ex2.approx.ftz.f32; op 1: cvt.rn.satfinite.e4m3x2.f32 (fed back through an
// xor so that nothing is loop-invariant)
template <int OP>
__global__ void __launch_bounds__(1024, 1) xu_rate_kernel(int reps, long long* cycles, float* sink) {
  float x[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) x[c] = -0.001f * static_cast<float>(threadIdx.x + c);
  __syncthreads();
  const long long t0 = clock64();
  for (int r = 0; r < reps; ++r) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      if constexpr (OP == 0) {
        asm volatile("ex2.approx.ftz.f32 %0, %0;" : "+f"(x[c]));
      } else {
        uint16_t h;
        asm volatile("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %1;" : "=h"(h) : "f"(x[c]));
        x[c] = __uint_as_float(__float_as_uint(x[c]) ^ h);
      }
    }
  }
  __syncthreads();  // every warp of the SM's one CTA has finished
  const long long t1 = clock64();
  float s = 0.f;
#pragma unroll
  for (int c = 0; c < 8; ++c) s += x[c];
  if (s == 12345.f) sink[0] = s;  // keeps the chains alive
  if (blockIdx.x == 0 && threadIdx.x == 0) *cycles = t1 - t0;
}

}  // namespace
}  // namespace dit

extern "C" DIT_API dit_status dit_probe_unit_rates(double* out, int n_out, dit_stream_t stream_handle) {
  if (out == nullptr || n_out < 4) return DIT_ERR_INVALID_ARG;
  int dev = -1, major = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DIT_ERR_UNSUPPORTED;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (major != 10 || sms < 1) return DIT_ERR_UNSUPPORTED;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_handle);
  int* err = nullptr;
  long long* cyc = nullptr;
  float* sink = nullptr;
  if (cudaMalloc(&err, sizeof(int)) != cudaSuccess) return DIT_ERR_LAUNCH;
  if (cudaMalloc(&cyc, sizeof(long long)) != cudaSuccess || cudaMalloc(&sink, sizeof(float)) != cudaSuccess) {
    cudaFree(err);
    cudaFree(cyc);
    return DIT_ERR_LAUNCH;
  }
  dit_status st = DIT_OK;
  long long c = 0;
  auto take = [&](double work_per_sm, double* dst) {
    c = 0;
    if (cudaMemcpyAsync(&c, cyc, sizeof(long long), cudaMemcpyDeviceToHost, stream) != cudaSuccess ||
        cudaStreamSynchronize(stream) != cudaSuccess) {
      st = DIT_ERR_LAUNCH;
      return;
    }
    *dst = c > 0 ? work_per_sm / static_cast<double>(c) : 0.0;
  };
  cudaMemsetAsync(err, 0, sizeof(int), stream);
  const int mma_reps = 20000, xu_reps = 8000;
  const int smem = 1024 + 2 * 128 * 128;
  // each MMA: 2 * 128 * 128 * K FLOP, K = 32 e4m3 or 16 bf16 elements
  for (int fp8 = 1; fp8 >= 0 && st == DIT_OK; --fp8) {
    auto k = fp8 ? dit::mma_rate_kernel<true> : dit::mma_rate_kernel<false>;
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) {
      st = DIT_ERR_LAUNCH;
      break;
    }
    cudaMemsetAsync(cyc, 0, sizeof(long long), stream);
    k<<<sms, 128, smem, stream>>>(mma_reps, err, cyc);
    if (cudaGetLastError() != cudaSuccess) st = DIT_ERR_LAUNCH;
    const double flop = 2.0 * 128 * 128 * (fp8 ? 32 : 16) * 4.0 * mma_reps;
    if (st == DIT_OK) take(flop, fp8 ? &out[0] : &out[1]);
  }
  for (int op = 0; op < 2 && st == DIT_OK; ++op) {
    auto k = op == 0 ? dit::xu_rate_kernel<0> : dit::xu_rate_kernel<1>;
    cudaMemsetAsync(cyc, 0, sizeof(long long), stream);
    k<<<sms, 1024, 0, stream>>>(xu_reps, cyc, sink);  // one CTA of 32 warps per SM
    if (cudaGetLastError() != cudaSuccess) st = DIT_ERR_LAUNCH;
    if (st == DIT_OK) take(8.0 * xu_reps * 1024, &out[2 + op]);
  }
  int herr = 0;
  if (st == DIT_OK && (cudaMemcpy(&herr, err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess || herr != 0))
    st = herr != 0 ? static_cast<dit_status>(herr) : DIT_ERR_LAUNCH;
  cudaFree(err);
  cudaFree(cyc);
  cudaFree(sink);
  return st;
}
