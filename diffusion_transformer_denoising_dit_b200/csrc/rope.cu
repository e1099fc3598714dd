// Rotary position embedding: table builder and a vectorised, HBM-bound apply.
//
// Source: "vflash / Optimization ledger", table "Accepted or exposed", row
// "strict Triton RoPE" (rotary embedding as a separate DiT op).  Multi-axis
// form with interleaved channel pairs; axis a's pair p turns by
// pos[a] * theta^(-2p/d_a).
#include <cuda_bf16.h>

#include "dit_device.cuh"

namespace dit {

// One thread per (token, pair): angle in fp64, cos/sin in fp64, rounded once to fp32.
__global__ void rope_tables_kernel(const int32_t* __restrict__ pos, int N, int d0, int d1, int d2, double theta,
                                   float* __restrict__ cos_out, float* __restrict__ sin_out) {
  const int half = (d0 + d1 + d2) / 2;
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<int64_t>(N) * half) return;
  const int n = static_cast<int>(idx / half);
  const int p = static_cast<int>(idx % half);
  int axis, pl, da;
  if (p < d0 / 2) {
    axis = 0; pl = p; da = d0;
  } else if (p < (d0 + d1) / 2) {
    axis = 1; pl = p - d0 / 2; da = d1;
  } else {
    axis = 2; pl = p - (d0 + d1) / 2; da = d2;
  }
  const double freq = pow(theta, -2.0 * pl / da);
  const double ang = static_cast<double>(pos[3 * n + axis]) * freq;
  double s, c;
  sincos(ang, &s, &c);
  cos_out[idx] = static_cast<float>(c);
  sin_out[idx] = static_cast<float>(s);
}

cudaError_t launch_rope_tables(const int32_t* pos, int N, int d0, int d1, int d2, double theta, float* cos_out,
                               float* sin_out, cudaStream_t stream) {
  const int64_t total = static_cast<int64_t>(N) * ((d0 + d1 + d2) / 2);
  const int threads = 256;
  const int64_t blocks = (total + threads - 1) / threads;
  rope_tables_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(pos, N, d0, d1, d2, theta, cos_out,
                                                                           sin_out);
  return cudaGetLastError();
}

struct RopeArgs {
  RopeJob job[2];
  int B, H, N, d;
  const float* cos_tab;
  const float* sin_tab;
  int out_fp32;
  const int32_t* skip;  // non-null and set: do nothing
};

// One thread per (batch, token, 8-channel chunk): it loads that chunk's cos and
// sin (16 bytes each) once and applies them to every head, four heads at a time
// (four independent 16-byte loads of x in flight per thread).  Consecutive
// threads walk consecutive 16-byte chunks of a token row, so for one head a
// warp reads 512 contiguous bytes.
__device__ __forceinline__ void rope8(const uint4& xv, const float (&cc)[4], const float (&ss)[4], float (&y)[8]) {
  const __nv_bfloat162* xp = reinterpret_cast<const __nv_bfloat162*>(&xv);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 x2 = __bfloat1622float2(xp[i]);
    y[2 * i] = x2.x * cc[i] - x2.y * ss[i];
    y[2 * i + 1] = x2.x * ss[i] + x2.y * cc[i];
  }
}

__device__ __forceinline__ void store8(void* base, int64_t off, const float (&y)[8], int out_fp32) {
  if (out_fp32) {
    float4* yp = reinterpret_cast<float4*>(static_cast<float*>(base) + off);
    yp[0] = make_float4(y[0], y[1], y[2], y[3]);
    yp[1] = make_float4(y[4], y[5], y[6], y[7]);
  } else {
    uint4 o;
    o.x = pack_bf16x2(y[0], y[1]);
    o.y = pack_bf16x2(y[2], y[3]);
    o.z = pack_bf16x2(y[4], y[5]);
    o.w = pack_bf16x2(y[6], y[7]);
    *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(base) + off) = o;
  }
}

__global__ void __launch_bounds__(256) rope_apply_kernel(RopeArgs a) {
  if (a.skip != nullptr && *a.skip != 0) return;
  const RopeJob& jb = a.job[blockIdx.y];
  const int cpr = a.d / 8;  // chunks per row
  const int64_t total = static_cast<int64_t>(a.B) * a.N * cpr;
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= total) return;
  const int c = static_cast<int>(idx % cpr);
  const int64_t row = idx / cpr;
  const int n = static_cast<int>(row % a.N);
  const int b = static_cast<int>(row / a.N);
  const float4 cv = *reinterpret_cast<const float4*>(a.cos_tab + static_cast<int64_t>(n) * (a.d / 2) + c * 4);
  const float4 sv = *reinterpret_cast<const float4*>(a.sin_tab + static_cast<int64_t>(n) * (a.d / 2) + c * 4);
  const float cc[4] = {cv.x, cv.y, cv.z, cv.w};
  const float ss[4] = {sv.x, sv.y, sv.z, sv.w};
  const __nv_bfloat16* x = static_cast<const __nv_bfloat16*>(jb.x) + b * jb.sx[0] + n * jb.sx[2] + c * 8;
  const int64_t yo = b * jb.sy[0] + n * jb.sy[2] + c * 8;
  int h = 0;
  for (; h + 4 <= a.H; h += 4) {
    uint4 xv[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) xv[u] = *reinterpret_cast<const uint4*>(x + (h + u) * jb.sx[1]);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      float y[8];
      rope8(xv[u], cc, ss, y);
      store8(jb.y, yo + (h + u) * jb.sy[1], y, a.out_fp32);
    }
  }
  for (; h < a.H; ++h) {
    float y[8];
    rope8(*reinterpret_cast<const uint4*>(x + h * jb.sx[1]), cc, ss, y);
    store8(jb.y, yo + h * jb.sy[1], y, a.out_fp32);
  }
}

cudaError_t launch_rope_apply(const RopeJob* jobs, int njobs, int B, int H, int N, int d, const float* cos_tab,
                              const float* sin_tab, int out_fp32, cudaStream_t stream, const int32_t* skip) {
  RopeArgs a;
  for (int i = 0; i < njobs; ++i) a.job[i] = jobs[i];
  if (njobs == 1) a.job[1] = jobs[0];
  a.B = B; a.H = H; a.N = N; a.d = d;
  a.cos_tab = cos_tab; a.sin_tab = sin_tab; a.out_fp32 = out_fp32;
  a.skip = skip;
  const int64_t total = static_cast<int64_t>(B) * N * (d / 8);  // threads: one per (b, n, chunk), all heads
  const int64_t blocks = (total + 255) / 256;
  if (blocks > 0x7fffffff) return cudaErrorInvalidConfiguration;  // grid.x limit; nothing launched
  dim3 grid(static_cast<unsigned>(blocks), njobs);
  rope_apply_kernel<<<grid, 256, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace dit
