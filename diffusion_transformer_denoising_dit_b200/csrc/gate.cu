// First-Block-Cache gate: rel = sum|a - b| / sum|b| over two bf16 residuals,
// skip = rel < threshold.
//
// Source: unsloth studio commit "core/inference/diffusion.py", paragraph "Add
// opt-in step caching (First-Block-Cache)": the remaining blocks are skipped
// once the first block's residual barely changes between steps, under a
// threshold knob.  The relative-L1 statistic is the plain reading of
// "barely changes" (the same family as the residual-difference threshold of
// Cache-DiT on the TensorRT-LLM VisualGen page).
//
// HBM-bound: 4 bytes read per element, ~3 flops.  Pass 1 streams both inputs
// with 16-byte loads (4 per input in flight per thread) over up to 740 CTAs, fp32 per-thread partials,
// fp64 per-CTA combine; pass 2 (one CTA) combines the CTA partials in a fixed
// order, so the result is deterministic for a given n.  Pass 2 is a programmatic
// dependent launch: it is scheduled while pass 1 still runs and waits on the
// device (griddepcontrol.wait) until pass 1 has completed and its partials are
// visible, so no launch gap separates the two.  For a residual split
// across ranks, gate_pass2_sums stops at the two totals (summed across ranks by
// the caller) and gate_finalize takes the decision from the summed totals.
#include <cuda_bf16.h>

#include <cmath>
#include <mutex>

#include "dit.h"
#include "dit_device.cuh"

namespace dit {

constexpr int kGateThreads = 256;
// Pass 1 runs at most one wave: at 48 registers a thread, five 256-thread CTAs
// fit on an SM, so 148 x 5 CTAs are resident at once (eight per SM would need a
// second, partial wave; measured 5 % slower on the 16896 x 3072 pair).
constexpr int kGateMaxCtas = 148 * 5;

int gate_num_ctas(int64_t n) {
  const int64_t per_cta = static_cast<int64_t>(kGateThreads) * 8;
  int64_t g = (n + per_cta - 1) / per_cta;
  if (g < 1) g = 1;
  if (g > kGateMaxCtas) g = kGateMaxCtas;
  return static_cast<int>(g);
}

__device__ __forceinline__ void accum8(const uint4& av, const uint4& bv, float& num, float& den) {
  const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&av);
  const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&bv);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 x = __bfloat1622float2(a2[i]);
    const float2 y = __bfloat1622float2(b2[i]);
    num += fabsf(x.x - y.x) + fabsf(x.y - y.y);
    den += fabsf(y.x) + fabsf(y.y);
  }
}

__global__ void __launch_bounds__(kGateThreads) gate_pass1(const __nv_bfloat16* __restrict__ a,
                                                           const __nv_bfloat16* __restrict__ b, int64_t n,
                                                           double* __restrict__ partials) {
  // the dependent combine may be scheduled now; it waits for this grid to complete
  pdl_trigger();
  float num = 0.f, den = 0.f;
  const int64_t n8 = n / 8;
  const uint4* a8 = reinterpret_cast<const uint4*>(a);
  const uint4* b8 = reinterpret_cast<const uint4*>(b);
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  // four independent 16-byte loads of each input in flight per iteration
  for (; i + 3 * stride < n8; i += 4 * stride) {
    uint4 av[4], bv[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      av[u] = __ldcs(a8 + i + u * stride);
      bv[u] = __ldcs(b8 + i + u * stride);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) accum8(av[u], bv[u], num, den);
  }
  for (; i < n8; i += stride) accum8(__ldcs(a8 + i), __ldcs(b8 + i), num, den);
  if (blockIdx.x == 0 && threadIdx.x < n - n8 * 8) {  // ragged tail (< 8 elements)
    const int64_t t = n8 * 8 + threadIdx.x;
    const float x = __bfloat162float(a[t]);
    const float y = __bfloat162float(b[t]);
    num += fabsf(x - y);
    den += fabsf(y);
  }
  double dn = num, dd = den;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    dn += __shfl_xor_sync(0xffffffffu, dn, o);
    dd += __shfl_xor_sync(0xffffffffu, dd, o);
  }
  __shared__ double sn[kGateThreads / 32], sd[kGateThreads / 32];
  const int w = threadIdx.x / 32;
  if ((threadIdx.x & 31) == 0) {
    sn[w] = dn;
    sd[w] = dd;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double tn = 0.0, td = 0.0;
    for (int k = 0; k < kGateThreads / 32; ++k) {
      tn += sn[k];
      td += sd[k];
    }
    partials[2 * blockIdx.x] = tn;
    partials[2 * blockIdx.x + 1] = td;
  }
}

constexpr int kCombineThreads = 256;

// The per-CTA partials combined in a fixed order by one kCombineThreads CTA:
// thread t sums partials t, t + 256, ... in turn, each warp folds its 32 sums
// with a butterfly, and thread 0 adds the 8 warp sums in warp order.  Returns
// the totals in thread 0.
__device__ __forceinline__ void combine_partials(const double* __restrict__ partials, int nparts, double& tn,
                                                 double& td) {
  double n = 0.0, d = 0.0;
  for (int k = threadIdx.x; k < nparts; k += kCombineThreads) {
    n += partials[2 * k];
    d += partials[2 * k + 1];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    n += __shfl_xor_sync(0xffffffffu, n, o);
    d += __shfl_xor_sync(0xffffffffu, d, o);
  }
  __shared__ double sn[kCombineThreads / 32], sd[kCombineThreads / 32];
  if ((threadIdx.x & 31) == 0) {
    sn[threadIdx.x >> 5] = n;
    sd[threadIdx.x >> 5] = d;
  }
  __syncthreads();
  tn = 0.0, td = 0.0;
  if (threadIdx.x == 0) {
#pragma unroll
    for (int w = 0; w < kCombineThreads / 32; ++w) {
      tn += sn[w];
      td += sd[w];
    }
  }
}

// rel = num / den (0 when both are 0, +inf when only den is), skip = rel < threshold.
__device__ __forceinline__ void decide(double num, double den, float threshold, float* rel_out, int32_t* skip_out) {
  double rel;
  if (den == 0.0)
    rel = (num == 0.0) ? 0.0 : __longlong_as_double(0x7ff0000000000000ll);  // +inf
  else
    rel = num / den;
  rel_out[0] = static_cast<float>(rel);
  skip_out[0] = (rel < static_cast<double>(threshold)) ? 1 : 0;
}

// griddepcontrol.wait: pass 1 has completed and its partials are visible (a
// no-op when this grid was launched without the programmatic dependency)
__global__ void __launch_bounds__(kCombineThreads) gate_pass2(const double* __restrict__ partials, int nparts,
                                                              float threshold, float* __restrict__ rel_out,
                                                              int32_t* __restrict__ skip_out) {
  pdl_wait();
  double tn, td;
  combine_partials(partials, nparts, tn, td);
  if (threadIdx.x == 0) decide(tn, td, threshold, rel_out, skip_out);
}

// Sharded form: the shard's totals (sum |a - b|, sum |b|) in fp64, to be summed
// across ranks before gate_finalize decides.
__global__ void __launch_bounds__(kCombineThreads) gate_pass2_sums(const double* __restrict__ partials, int nparts,
                                                                   double* __restrict__ sums_out) {
  pdl_wait();
  double tn, td;
  combine_partials(partials, nparts, tn, td);
  if (threadIdx.x == 0) {
    sums_out[0] = tn;
    sums_out[1] = td;
  }
}

__global__ void gate_finalize(const double* __restrict__ sums, float threshold, float* __restrict__ rel_out,
                              int32_t* __restrict__ skip_out) {
  if (threadIdx.x == 0) decide(sums[0], sums[1], threshold, rel_out, skip_out);
}

cudaError_t launch_gate(const void* a, const void* b, int64_t n, float threshold, float* rel_out, int32_t* skip_out,
                        double* partials, cudaStream_t stream) {
  const int g = gate_num_ctas(n);
  gate_pass1<<<g, kGateThreads, 0, stream>>>(static_cast<const __nv_bfloat16*>(a),
                                             static_cast<const __nv_bfloat16*>(b), n, partials);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_dependent(gate_pass2, dim3(1), dim3(kCombineThreads), 0, stream, static_cast<const double*>(partials), g,
                          threshold, rel_out, skip_out);
}

cudaError_t launch_gate_sums(const void* a, const void* b, int64_t n, double* sums_out, double* partials,
                             cudaStream_t stream) {
  const int g = gate_num_ctas(n);
  gate_pass1<<<g, kGateThreads, 0, stream>>>(static_cast<const __nv_bfloat16*>(a),
                                             static_cast<const __nv_bfloat16*>(b), n, partials);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_dependent(gate_pass2_sums, dim3(1), dim3(kCombineThreads), 0, stream,
                          static_cast<const double*>(partials), g, sums_out);
}

cudaError_t launch_gate_finalize(const double* sums, float threshold, float* rel_out, int32_t* skip_out,
                                 cudaStream_t stream) {
  gate_finalize<<<1, 32, 0, stream>>>(sums, threshold, rel_out, skip_out);
  return cudaGetLastError();
}

// Reference residual of the gate's policies: r_ref = r_cur, unless the flag says
// the step was skipped (then the reference stays the last computed step's).
// Every CTA reads the flag once and returns at once when it is set; otherwise a
// grid-strided 16-byte copy with four loads in flight per thread (HBM-bound,
// 4 bytes moved per element).
__global__ void __launch_bounds__(kGateThreads) gate_ref_update(const uint4* __restrict__ cur, uint4* __restrict__ ref,
                                                                int64_t n8, const int32_t* __restrict__ skip) {
  if (skip != nullptr && *skip != 0) return;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  for (; i + 3 * stride < n8; i += 4 * stride) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = __ldcs(cur + i + u * stride);
#pragma unroll
    for (int u = 0; u < 4; ++u) ref[i + u * stride] = v[u];
  }
  for (; i < n8; i += stride) ref[i] = __ldcs(cur + i);
}

__global__ void gate_ref_update_tail(const __nv_bfloat16* __restrict__ cur, __nv_bfloat16* __restrict__ ref,
                                     int64_t from, int64_t n, const int32_t* __restrict__ skip) {
  if (skip != nullptr && *skip != 0) return;
  const int64_t t = from + threadIdx.x;
  if (t < n) ref[t] = cur[t];
}

cudaError_t launch_gate_ref_update(const void* cur, void* ref, int64_t n, const int32_t* skip, cudaStream_t stream) {
  const int64_t n8 = n / 8;
  if (n8 > 0) {
    gate_ref_update<<<gate_num_ctas(n), kGateThreads, 0, stream>>>(static_cast<const uint4*>(cur),
                                                                   static_cast<uint4*>(ref), n8, skip);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (n - n8 * 8 > 0) {
    gate_ref_update_tail<<<1, 32, 0, stream>>>(static_cast<const __nv_bfloat16*>(cur),
                                                static_cast<__nv_bfloat16*>(ref), n8 * 8, n, skip);
    return cudaGetLastError();
  }
  return cudaSuccess;
}

}  // namespace dit

// ---------------------------------------------------------------------------
// fbcache_gate_noalloc: the same two-pass gate, with its scratch in a fixed
// device array instead of a caller-provided workspace.
//
// For callers that cannot hand this library any device memory: a plug-in
// driven by a host runtime that owns the device allocator and exposes no
// scratch buffers, or a step loop whose rules forbid allocating while it runs.
// The scratch holds one (sum|a-b|, sum|b|) pair of doubles per pass-1 CTA.
// Pass 1 writes every pair that pass 2 reads, so nothing has to start at zero.
// ---------------------------------------------------------------------------
namespace {

// Largest scratch any n can need: 2 doubles for each of at most kGateMaxCtas CTAs.
constexpr int kNoAllocScratchDoubles = 2 * dit::kGateMaxCtas;
static __device__ __align__(256) double g_gate_scratch[kNoAllocScratchDoubles];

constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mu;
double* g_noalloc_ptr[kNoAllocMaxDevices] = {};

// Device address of g_gate_scratch on the current device (looked up once per device).
double* noalloc_scratch(dit_status* st) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoAllocMaxDevices) {
    *st = DIT_ERR_UNSUPPORTED;
    return nullptr;
  }
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (major != 10 || minor != 0) {
      *st = DIT_ERR_UNSUPPORTED;
      return nullptr;
    }
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_gate_scratch) != cudaSuccess || p == nullptr) {
      *st = DIT_ERR_LAUNCH;
      return nullptr;
    }
    g_noalloc_ptr[dev] = static_cast<double*>(p);
  }
  *st = DIT_OK;
  return g_noalloc_ptr[dev];
}

}  // namespace

extern "C" DIT_API dit_status fbcache_gate_noalloc(const void* r_cur, const void* r_prev, int64_t n, float threshold,
                                                   float* rel_out, int32_t* skip_out, dit_stream_t stream) {
  if (!r_cur || !r_prev || !rel_out || !skip_out || n < 1) return DIT_ERR_INVALID_ARG;
  if (!std::isfinite(threshold)) return DIT_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(r_cur) & 15u) || (reinterpret_cast<uintptr_t>(r_prev) & 15u) ||
      (reinterpret_cast<uintptr_t>(rel_out) & 3u) || (reinterpret_cast<uintptr_t>(skip_out) & 3u))
    return DIT_ERR_ALIGNMENT;
  // the fixed array must hold every pass-1 partial for this n
  if (2 * static_cast<int64_t>(dit::gate_num_ctas(n)) > kNoAllocScratchDoubles) return DIT_ERR_WORKSPACE;
  dit_status st;
  double* scratch = noalloc_scratch(&st);
  if (!scratch) return st;
  return dit::launch_gate(r_cur, r_prev, n, threshold, rel_out, skip_out, scratch,
                          reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? DIT_OK
             : DIT_ERR_LAUNCH;
}
