// FP8 prologue: rotary embedding, K mean-smoothing and per-block e4m3
// quantisation of Q, K and V, ahead of the FP8 attention kernel.
//
// Sources: "FLUX 3 Image Klein / TensorRT-LLM VisualGen" (cuDNN FP8 attention
// against VANILLA BF16) and "vflash / Optimization ledger", table "Accepted or
// exposed" (SageAttention2: quantised attention).  Neither page fixes the
// scheme; the readings: e4m3 (RNE, saturating), one fp32 scale amax/448 per
// block of 128 (Q) or 64 (K, V) tokens of one (batch, head), K minus its
// channel mean over all N tokens after rotation (which leaves softmax
// unchanged in exact arithmetic).
//
// Pass 1 (kmean_partial): per (b,h) and one of 48 token chunks, fp32 channel sums of the
//   rotated K; also clears the per-(b,h) V scale maximum.
// Pass 1b (kmean_finalize): the partials of each (b,h) combined in a fixed order.
// Pass 2 (quantize): one CTA per (128-token block, (b,h), tensor): rotate Q
//   and K in fp32, subtract the K mean,
//   block amax, scale and cast to e4m3; write the scales.  Streams 6 B/element
//   in (bf16 Q, K, V) and 3 B/element out; HBM-bound.
// With qk_int8 (the 8-bit integer Q.K^T of SageAttention, the quantised
// attention the same ledger row names), Q and K are cast instead to symmetric
// int8: scale amax/127 per block, round to nearest even, within +-127; V stays
// e4m3.
#include <cuda_bf16.h>

#include "dit_device.cuh"

namespace dit {
namespace {

constexpr int kChunks = kFp8MeanChunks;  // token chunks of the K-mean pass per (b,h)
constexpr int kThreads = 256;  // 16 channel chunks (8 channels each) x 16 token lanes

__device__ __forceinline__ void load_rotate8(const __nv_bfloat16* __restrict__ src, const float* __restrict__ cos_tab,
                                             const float* __restrict__ sin_tab, int n, int cc, int half_d,
                                             float (&y)[8]) {
  const uint4 xv = *reinterpret_cast<const uint4*>(src);
  const __nv_bfloat162* xp = reinterpret_cast<const __nv_bfloat162*>(&xv);
  if (cos_tab) {
    const float4 cv = *reinterpret_cast<const float4*>(cos_tab + static_cast<int64_t>(n) * half_d + cc * 4);
    const float4 sv = *reinterpret_cast<const float4*>(sin_tab + static_cast<int64_t>(n) * half_d + cc * 4);
    const float c4[4] = {cv.x, cv.y, cv.z, cv.w};
    const float s4[4] = {sv.x, sv.y, sv.z, sv.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 x = __bfloat1622float2(xp[i]);
      y[2 * i] = x.x * c4[i] - x.y * s4[i];
      y[2 * i + 1] = x.x * s4[i] + x.y * c4[i];
    }
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 x = __bfloat1622float2(xp[i]);
      y[2 * i] = x.x;
      y[2 * i + 1] = x.y;
    }
  }
}

// Two floats -> two e4m3 bytes (round to nearest even, saturating); lo in the low byte.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float block_max(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float m = red[0];
#pragma unroll
  for (int w = 1; w < kThreads / 32; ++w) m = fmaxf(m, red[w]);
  return m;
}

__global__ void __launch_bounds__(kThreads) kmean_partial(Fp8Prep p, float* __restrict__ partial) {
  pdl_trigger();  // the mean's combine (and through it the quantiser) may be scheduled
  const int bh = blockIdx.y;
  const int chunk = blockIdx.x;
  if (chunk == 0 && threadIdx.x == 0) p.v_scale_max[bh] = 0.f;
  const int b = bh / p.H, h = bh % p.H;
  const int cc = threadIdx.x & 15, tl = threadIdx.x >> 4;
  const int per = (p.N + kChunks - 1) / kChunks;
  const int n0 = chunk * per, n1 = min(p.N, n0 + per);
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  if (p.smooth_k) {
    const __nv_bfloat16* kb = static_cast<const __nv_bfloat16*>(p.k) + b * p.sk[0] + h * p.sk[1];
    for (int n = n0 + tl; n < n1; n += 16) {
      float y[8];
      load_rotate8(kb + static_cast<int64_t>(n) * p.sk[2] + cc * 8, p.cos_tab, p.sin_tab, n, cc, p.d / 2, y);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] += y[i];
    }
  }
  __shared__ float red[16][128 + 4];
#pragma unroll
  for (int i = 0; i < 8; ++i) red[tl][cc * 8 + i] = acc[i];
  __syncthreads();
  if (threadIdx.x < 128) {
    float s = 0.f;
#pragma unroll
    for (int r = 0; r < 16; ++r) s += red[r][threadIdx.x];
    partial[(static_cast<int64_t>(bh) * kChunks + chunk) * 128 + threadIdx.x] = s;
  }
}

// K channel means: one CTA per (b,h), thread c sums the kChunks partials of
// channel c in a fixed order (independent loads, then the adds).
__global__ void __launch_bounds__(128) kmean_finalize(Fp8Prep p, const float* __restrict__ partial) {
  pdl_trigger();  // the quantiser may be scheduled: its Q blocks need nothing from here
  pdl_wait();     // every partial written
  const int bh = blockIdx.x;
  const int c = threadIdx.x;
  float v[kChunks];
#pragma unroll
  for (int k = 0; k < kChunks; ++k) v[k] = partial[(static_cast<int64_t>(bh) * kChunks + k) * 128 + c];
  float sum = 0.f;
#pragma unroll
  for (int k = 0; k < kChunks; ++k) sum += v[k];
  p.k_mean[bh * 128 + c] = p.smooth_k ? sum / static_cast<float>(p.N) : 0.f;
}

// Eight floats times inv (within [-127, 127]) -> eight int8 (two's complement),
// rounded to nearest even, in token-row byte order.  fma(x, inv, 1.5 * 2^23)
// rounds x * inv once to an integer (the float's unit in the last place is 1
// there), and the float's low byte is then that integer modulo 256.
__device__ __forceinline__ uint32_t s8_bits(float x, float inv) {
  return __float_as_uint(__fmaf_rn(x, inv, 12582912.0f));
}
__device__ __forceinline__ uint32_t cvt_s8x4(const float* x, float inv) {
  // byte_perm selector nibbles pick bytes of {y:x}: low bytes of the four codes, in order
  const uint32_t ab = __byte_perm(s8_bits(x[0], inv), s8_bits(x[1], inv), 0x0040);
  const uint32_t cd = __byte_perm(s8_bits(x[2], inv), s8_bits(x[3], inv), 0x0040);
  return __byte_perm(ab, cd, 0x5410);
}
__device__ __forceinline__ uint2 cvt_s8x8(const float (&x)[8], float inv) {
  return make_uint2(cvt_s8x4(x, inv), cvt_s8x4(x + 4, inv));
}

// Quantises one 128-token block of one tensor held as 8 chunks per thread:
// thread t owns channel chunk (t % 16) of tokens t/16 + 16 i, i = 0..7.  With
// two_blocks the first four tokens of a thread lie in the first 64-token block.
// int8: symmetric int8 codes and scales amax/127 instead of e4m3 and amax/448.
__device__ __forceinline__ void quantize_tile(float (&x)[8][8], bool two_blocks, int n_base, int N,
                                              uint8_t* __restrict__ dst, int cc, int tl, float* red, float* sc_out0,
                                              float* sc_out1, float* vmax, bool int8 = false) {
  float a0 = 0.f, a1 = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      if (i < 4 || !two_blocks)
        a0 = fmaxf(a0, fabsf(x[i][e]));
      else
        a1 = fmaxf(a1, fabsf(x[i][e]));
    }
  a0 = block_max(a0, red);
  if (two_blocks) a1 = block_max(a1, red + 8);
  const float qmax = int8 ? 127.f : 448.f;
  const float s0 = a0 > 0.f ? a0 / qmax : 1.f;
  const float s1 = a1 > 0.f ? a1 / qmax : 1.f;
  const float inv0 = a0 > 0.f ? qmax / a0 : 1.f;
  const float inv1 = a1 > 0.f ? qmax / a1 : 1.f;
  if (threadIdx.x == 0) {
    *sc_out0 = s0;
    if (two_blocks) *sc_out1 = s1;
    if (vmax) {
      atomicMax(reinterpret_cast<int*>(vmax), __float_as_int(s0));
      // a second block past the sequence end (all zeros, scale 1) is not a V block
      if (two_blocks && n_base + 64 < N) atomicMax(reinterpret_cast<int*>(vmax), __float_as_int(s1));
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int n = n_base + tl + 16 * i;
    if (n >= N) continue;
    const float inv = (i < 4 || !two_blocks) ? inv0 : inv1;
    uint2 w;
    if (int8) {
      w = cvt_s8x8(x[i], inv);
    } else {
      w.x = cvt_e4m3x2(x[i][0] * inv, x[i][1] * inv) | (cvt_e4m3x2(x[i][2] * inv, x[i][3] * inv) << 16);
      w.y = cvt_e4m3x2(x[i][4] * inv, x[i][5] * inv) | (cvt_e4m3x2(x[i][6] * inv, x[i][7] * inv) << 16);
    }
    *reinterpret_cast<uint2*>(dst + static_cast<int64_t>(n) * 128 + cc * 8) = w;
  }
}

// One CTA per (128-token block, (b,h), tensor): blockIdx.z = 0 quantises Q (one
// 128-token block, rotated), 1 quantises K (two 64-token blocks, rotated and
// smoothed), 2 quantises V (two 64-token blocks).  Every thread issues its eight
// 16-byte loads before any reduction, so each CTA keeps 32 KB in flight.
// INT8: Q and K as symmetric int8 (the integer Q.K^T form), V as e4m3.
template <bool INT8>
__global__ void __launch_bounds__(kThreads, 3) quantize_qkv(Fp8Prep p) {
  const int blk = blockIdx.x;  // 128-token block
  const int bh = blockIdx.y;
  const int which = blockIdx.z;
  const int b = bh / p.H, h = bh % p.H;
  // Launched as a dependent of the K-mean combine: Q blocks start at once (they
  // read only the inputs, written before the K-mean pass began), K blocks need the
  // mean and V blocks the cleared V scale maximum, so they wait for the combine
  // (which itself waited for the K-mean pass) to complete.
  if (which != 0) pdl_wait();
  const int cc = threadIdx.x & 15, tl = threadIdx.x >> 4;
  const int n_base = blk * 128;
  const int nq = (p.N + 127) / 128, nk = (p.N + 63) / 64;
  __shared__ float mean[128];
  __shared__ float red[16];
  __shared__ float unused_scale;  // sink for the second scale of a block past the sequence end
  const int64_t out_off = static_cast<int64_t>(bh) * p.N * 128;
  const __nv_bfloat16* src;
  int64_t tok_stride;
  const float* ct = nullptr;
  const float* st = nullptr;
  if (which == 0) {
    src = static_cast<const __nv_bfloat16*>(p.q) + b * p.sq[0] + h * p.sq[1];
    tok_stride = p.sq[2];
    ct = p.cos_tab;
    st = p.sin_tab;
  } else if (which == 1) {
    src = static_cast<const __nv_bfloat16*>(p.k) + b * p.sk[0] + h * p.sk[1];
    tok_stride = p.sk[2];
    ct = p.cos_tab;
    st = p.sin_tab;
  } else {
    src = static_cast<const __nv_bfloat16*>(p.v) + b * p.sv[0] + h * p.sv[1];
    tok_stride = p.sv[2];
  }
  float x[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int n = n_base + tl + 16 * i;
    if (n < p.N)
      load_rotate8(src + static_cast<int64_t>(n) * tok_stride + cc * 8, ct, st, n, cc, 64, x[i]);
    else
#pragma unroll
      for (int e = 0; e < 8; ++e) x[i][e] = 0.f;
  }
  if (which == 0) {
    quantize_tile(x, false, n_base, p.N, p.q8 + out_off, cc, tl, red, p.q_scale + bh * nq + blk, nullptr, nullptr,
                  INT8);
    pdl_trigger();  // the attention kernel may be scheduled
    return;
  }
  if (which == 1) {
    if (threadIdx.x < 128) mean[threadIdx.x] = p.k_mean[bh * 128 + threadIdx.x];
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (n_base + tl + 16 * i < p.N) {
#pragma unroll
        for (int e = 0; e < 8; ++e) x[i][e] -= mean[cc * 8 + e];
      }
    }
    float* s1 = (2 * blk + 1 < nk) ? p.k_scale + bh * nk + 2 * blk + 1 : &unused_scale;
    quantize_tile(x, true, n_base, p.N, p.k8 + out_off, cc, tl, red, p.k_scale + bh * nk + 2 * blk, s1, nullptr,
                  INT8);
    pdl_trigger();
    return;
  }
  float* s1 = (2 * blk + 1 < nk) ? p.v_scale + bh * nk + 2 * blk + 1 : &unused_scale;
  quantize_tile(x, true, n_base, p.N, p.v8 + out_off, cc, tl, red, p.v_scale + bh * nk + 2 * blk, s1,
                p.v_scale_max + bh);
  pdl_trigger();
}

}  // namespace

cudaError_t launch_fp8_prologue(const Fp8Prep& p, cudaStream_t stream) {
  float* partial = p.k_partial;
  dim3 g1(kChunks, p.B * p.H);
  kmean_partial<<<g1, kThreads, 0, stream>>>(p, partial);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = launch_dependent(kmean_finalize, dim3(p.B * p.H), dim3(128), 0, stream, p, static_cast<const float*>(partial));
  if (e != cudaSuccess) return e;
  dim3 g2((p.N + 127) / 128, p.B * p.H, 3);
  return p.qk_int8 ? launch_dependent(quantize_qkv<true>, g2, dim3(kThreads), 0, stream, p)
                   : launch_dependent(quantize_qkv<false>, g2, dim3(kThreads), 0, stream, p);
}

}  // namespace dit
