// FP8 (e4m3) joint attention on sm_100a, reading the prologue's quantised
// Q, smoothed K and V with their per-block scales.
//
// Sources: "FLUX 3 Image Klein / TensorRT-LLM VisualGen" (cuDNN FP8 attention
// against VANILLA BF16 on B200) and "vflash / Optimization ledger", table
// "Accepted or exposed" (SageAttention2: quantised attention with block
// scales and K smoothing).
//
// Same structure as the BF16 kernel (one CTA per 128-row Q tile, warps 0-3
// softmax, warp 4 TMA, warp 5 MMA + TMEM owner), with:
//   S = Q8 K8^T       tcgen05 kind::f8f6f4, 4 MMAs of K=32 over d = 128
//   scores            s_ij = S_ij * sQ * sK(j) * scale: the two K block scales
//                     of a 128-key tile fold into the softmax FFMA
//   P                 exp2 in fp32, then P * 448 * sV(j) / sV_max cast to e4m3
//                     (the V block scale folded in); the row sum uses fp32 P
//   O += P8 V8        TS MMA, P from TMEM (4 e4m3 per column), V MN-major
//   epilogue          O * sV_max / 448 / l -> bf16
// TMEM: [0,128) S0 [128,256) S1 [256,384) O [384,416) P0 [416,448) P1.
#include <cuda_bf16.h>

#include "dit_device.cuh"

namespace dit {
namespace {

constexpr int D = 128;
constexpr int BM = 128;
constexpr int BN = 128;
constexpr int NST = 4;
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256, kColP0 = 384, kColP1 = 416;
constexpr int kTileBytes = BN * D;  // e4m3: one byte per element, one 128-byte row per token
constexpr int kNumBars = 1 + 3 * NST + 2 + 2 + 2;
// P is quantised as p * 448 * sV/sV_max with p <= 2^kRescaleLog2, so e4m3's range
// (max 448) leaves no headroom for a stale max: rescale whenever the max grows.
constexpr float kRescaleLog2 = 0.f;
constexpr int kSmemBytes = 1024 + kTileBytes /*Q*/ + 2 * NST * kTileBytes + kNumBars * 8 + 16;

struct Fp8Scales {
  const float* q_scale;  // [B*H][nq]
  const float* k_scale;  // [B*H][nk]
  const float* v_scale;  // [B*H][nk]
  const float* v_scale_max;
  int H;
};

__device__ __forceinline__ uint32_t cvt_e4m3x4(float a, float b, float c, float d) {
  uint16_t lo, hi;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(b), "f"(a));
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(d), "f"(c));
  return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}

__global__ void __launch_bounds__(kThreads, 1)
    attn_fp8_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const AttnOut out, const Fp8Scales sc) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + kTileBytes;
  uint8_t* sV = sK + NST * kTileBytes;
  uint64_t* q_full = reinterpret_cast<uint64_t*>(sV + NST * kTileBytes);
  uint64_t* k_full = q_full + 1;
  uint64_t* v_full = k_full + NST;
  uint64_t* kv_empty = v_full + NST;
  uint64_t* s_full = kv_empty + NST;
  uint64_t* p_ready = s_full + 2;
  uint64_t* pv_done = p_ready + 2;  // [2]: PV(j) arrives on pv_done[j & 1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(q_full + kNumBars);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int N = out.N;
  const int nkv = (N + BN - 1) / BN;
  int* err = out.err;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < NST; ++s) {
      mbar_init(k_full + s, 1);
      mbar_init(v_full + s, 1);
      mbar_init(kv_empty + s, 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(s_full + s, 1);
      mbar_init(p_ready + s, 128);
      mbar_init(pv_done + s, 1);
    }
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(q_full, kTileBytes);
      tma_load_4d(sQ, &tmQ, q_full, 0, qt * BM, h, b);
      for (int j = 0; j < nkv; ++j) {
        const int st = j % NST;
        if (j >= NST && !mbar_wait(kv_empty + st, ((j / NST) & 1) ^ 1, err, kErrTimeout)) break;
        mbar_arrive_expect_tx(k_full + st, kTileBytes);
        tma_load_4d(sK + st * kTileBytes, &tmK, k_full + st, 0, j * BN, h, b);
        mbar_arrive_expect_tx(v_full + st, kTileBytes);
        tma_load_4d(sV + st * kTileBytes, &tmV, v_full + st, 0, j * BN, h, b);
      }
    }
  } else if (warp == 5) {
    if (lane == 0) {
      constexpr uint32_t idesc_s = make_idesc(0, 0, 0, BM, BN);  // e4m3 x e4m3, K-major both
      constexpr uint32_t idesc_o = make_idesc(0, 0, 1, BM, D);   // V MN-major
      const uint32_t tO = tmem + kColO;
      const uint32_t q_addr = smem_u32(sQ);
      bool ok = mbar_wait(q_full, 0, err, kErrTimeout);
      for (int j = 0; ok && j <= nkv; ++j) {
        if (j < nkv) {
          const int st = j % NST;
          if (!mbar_wait(k_full + st, (j / NST) & 1, err, kErrTimeout)) break;
          tc_fence_after();
          const uint32_t k_addr = smem_u32(sK + st * kTileBytes);
#pragma unroll
          for (int kk = 0; kk < D / 32; ++kk)  // 32 e4m3 = 32 bytes of the 128-byte swizzled row
            mma_f8_ss(tmem + ((j & 1) ? kColS1 : kColS0), smem_desc_sw128(q_addr + kk * 32, 16, 1024),
                      smem_desc_sw128(k_addr + kk * 32, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
          mma_commit(s_full + (j & 1));
        }
        if (j >= 1) {
          const int jj = j - 1;
          const int st = jj % NST;
          if (!mbar_wait(p_ready + (jj & 1), (jj >> 1) & 1, err, kErrTimeout)) break;
          if (!mbar_wait(v_full + st, (jj / NST) & 1, err, kErrTimeout)) break;
          tc_fence_after();
          const uint32_t v_addr = smem_u32(sV + st * kTileBytes);
#pragma unroll
          for (int kk = 0; kk < BN / 32; ++kk)  // 32 keys = 32 rows of 128 bytes; P: 8 columns of 4 e4m3
            mma_f8_ts(tO, tmem + ((jj & 1) ? kColP1 : kColP0) + kk * 8,
                      smem_desc_sw128(v_addr + kk * 32 * 128, 16384, 1024), idesc_o, (jj > 0 || kk > 0) ? 1u : 0u);
          mma_commit(pv_done + (jj & 1));
          mma_commit(kv_empty + st);
        }
      }
    }
  } else {
    const int row = threadIdx.x;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const int bh = b * sc.H + h;
    const int nq = (N + BM - 1) / BM, nk = (N + 63) / 64;
    const float* ksc = sc.k_scale + static_cast<int64_t>(bh) * nk;
    const float* vsc = sc.v_scale + static_cast<int64_t>(bh) * nk;
    const float vmax = sc.v_scale_max[bh];
    const float qs = sc.q_scale[static_cast<int64_t>(bh) * nq + qt] * out.scale_log2;
    const float vfold = 448.f / vmax;
    float m = -INFINITY;
    float l = 0.f;
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      const int bsel = j & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(s_full + bsel, (j >> 1) & 1, err, kErrTimeout));
      if (!ok) break;
      tc_fence_after();
      const int kb0 = 2 * j, kb1 = 2 * j + 1;
      const float c0 = qs * ksc[kb0];
      const float c1 = kb1 < nk ? qs * ksc[kb1] : 1.f;  // past the end: keys are -inf, keep -inf * c1 = -inf
      const float f0 = vsc[kb0] * vfold;
      const float f1 = kb1 < nk ? vsc[kb1] * vfold : 0.f;
      uint32_t s[BN];
      const uint32_t tS = tmem + (bsel ? kColS1 : kColS0) + lane_off;
#pragma unroll
      for (int c = 0; c < BN / 32; ++c) tmem_ld32(tS + c * 32, s + c * 32);
      tmem_wait_ld();
      reg_fence(s);
      const int kv0 = j * BN;
      if (kv0 + BN > N) {
#pragma unroll
        for (int c = 0; c < BN; ++c)
          if (kv0 + c >= N) s[c] = 0xff800000u;
      }
      // per-half row max of the raw scores: 4 independent chains per half
      float mxa[4], mxb[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        mxa[i] = __uint_as_float(s[i]);
        mxb[i] = __uint_as_float(s[64 + i]);
      }
#pragma unroll
      for (int c = 4; c < 64; c += 4)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          mxa[i] = fmaxf(mxa[i], __uint_as_float(s[c + i]));
          mxb[i] = fmaxf(mxb[i], __uint_as_float(s[64 + c + i]));
        }
      const float mx0 = fmaxf(fmaxf(mxa[0], mxa[1]), fmaxf(mxa[2], mxa[3]));
      const float mx1 = fmaxf(fmaxf(mxb[0], mxb[1]), fmaxf(mxb[2], mxb[3]));
      // c0, c1 > 0 for every in-range block; a block past the end is all -inf
      const float m_tile = fmaxf(mx0 * c0, kv0 + 64 < N ? mx1 * c1 : -INFINITY);
      // rescale whenever some row of the warp gets a larger max (kRescaleLog2 = 0)
      const bool grow = __any_sync(0xffffffffu, m_tile > m + kRescaleLog2);
      const float m_new = grow ? fmaxf(m, m_tile) : m;
      const float alpha = grow ? ex2(m - m_new) : 1.f;
      const float neg_m = -m_new;
      if (j >= 2) {  // P(j) goes to buffer j&1, last read by PV(j-2)
        ok = __all_sync(0xffffffffu, mbar_wait(pv_done + bsel, ((j >> 1) - 1) & 1, err, kErrTimeout));
        if (!ok) break;
        tc_fence_after();
      }
      float sum4[4] = {0.f, 0.f, 0.f, 0.f};
      const uint32_t tP = tmem + (bsel ? kColP1 : kColP0) + lane_off;
      uint32_t p[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const float cs = e < 16 ? c0 : c1;
        const float fv = e < 16 ? f0 : f1;
        float x[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          x[i] = ex2(fmaf(__uint_as_float(s[4 * e + i]), cs, neg_m));
          sum4[i] += x[i];
        }
        p[e] = cvt_e4m3x4(x[0] * fv, x[1] * fv, x[2] * fv, x[3] * fv);
      }
      tmem_st32(tP, p);
      const float sum = (sum4[0] + sum4[1]) + (sum4[2] + sum4[3]);
      if (j > 0 && grow) {
        ok = __all_sync(0xffffffffu, mbar_wait(pv_done + (bsel ^ 1), ((j - 1) >> 1) & 1, err, kErrTimeout));
        if (!ok) break;
        tc_fence_after();
        const uint32_t tO = tmem + kColO + lane_off;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + c * 32, o);
          tmem_wait_ld();
          reg_fence(o);
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(tO + c * 32, o);
        }
      }
      l = l * alpha + sum;
      m = m_new;
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(p_ready + bsel);
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(pv_done + ((nkv - 1) & 1), ((nkv - 1) >> 1) & 1, err, kErrTimeout));
    if (ok) {
      tc_fence_after();
      const float fin = vmax / 448.f / l;
      const int qrow = qt * BM + row;
      __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(out.o) + b * out.so[0] + h * out.so[1] +
                            static_cast<int64_t>(qrow) * out.so[2];
      const uint32_t tO = tmem + kColO + lane_off;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tO + c * 32, o);
        tmem_wait_ld();
        reg_fence(o);
        if (qrow < N) {
          uint4 pk[4];
          uint32_t* pw = reinterpret_cast<uint32_t*>(pk);
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pw[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * fin, __uint_as_float(o[2 * e + 1]) * fin);
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int e = 0; e < 4; ++e) dst[e] = pk[e];
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

cudaError_t launch_attn_fp8(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const AttnOut& out,
                            const Fp8Prep& p, cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(attn_fp8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  Fp8Scales sc;
  sc.q_scale = p.q_scale;
  sc.k_scale = p.k_scale;
  sc.v_scale = p.v_scale;
  sc.v_scale_max = p.v_scale_max;
  sc.H = p.H;
  dim3 grid((out.N + BM - 1) / BM, p.H, p.B);
  attn_fp8_kernel<<<grid, kThreads, kSmemBytes, stream>>>(tq, tk, tv, out, sc);
  return cudaGetLastError();
}

}  // namespace dit
