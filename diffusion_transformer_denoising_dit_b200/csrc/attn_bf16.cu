// BF16 joint attention on sm_100a: TMA -> shared memory -> tcgen05 MMA -> TMEM,
// flash-style online softmax in fp32 with exp2.
//
// Source: "FLUX 3 Image Klein / TensorRT-LLM VisualGen", section on why the
// differences arise: VANILLA BF16 attention over the joint text+image tokens
// is about 60 % of the DiT's GPU kernel time.  O = softmax(scale Q K^T) V per
// (batch, head), bidirectional, every key.
//
// One CTA owns one 128-row Q tile of one (b, h) and streams all K/V tiles of
// that head.  Warp roles (192 threads):
//   warps 0-3  softmax: thread t owns row t (TMEM lane t).  Reads S from TMEM,
//              keeps the running max m and sum l in fp32, writes P (bf16) to
//              TMEM, rescales O in TMEM when m grows, and runs the epilogue.
//   warp 4     TMA producer: Q once, then K_j / V_j into a NST-deep ring.
//   warp 5     MMA issuer (one thread) and TMEM owner:
//                S[j%2] = Q K_j^T          (SS: both operands in smem)
//                O     += P[j%2] V_j        (TS: P from TMEM, V from smem)
// TMEM (512 columns x 128 lanes x 32 bit):
//   [0,128) S0  [128,256) S1  [256,256+D) O  [384,448) P0  [448,512) P1
// Pipelining: S(j+1) runs on the tensor cores while the softmax warps
// exponentiate S(j); PV(j) runs while they exponentiate S(j+1).
#include <cuda_bf16.h>

#include "dit_device.cuh"

namespace dit {
namespace {

constexpr int BM = 128;  // query rows per CTA
constexpr int BN = 128;  // keys per tile
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256, kColP0 = 384, kColP1 = 448;
constexpr float kRescaleLog2 = 8.f;  // lazy-rescale threshold (log2 units)

template <int D>
struct Cfg {
  static constexpr int NST = (D == 128) ? 3 : 4;         // K/V ring depth
  static constexpr int kTileBytes = BN * D * 2;           // one K or V tile (bf16)
  static constexpr int kQBytes = BM * D * 2;
  static constexpr int kSubTile = BN * 128;               // [rows][64] bf16 sub-tile (128-byte rows)
  static constexpr int kNumBars = 1 + 3 * NST + 2 + 2 + 2;
  static constexpr int kSmemBytes = 1024 /*align slack*/ + kQBytes + 2 * NST * kTileBytes + kNumBars * 8 + 16;
};

struct Bars {
  uint64_t* q_full;
  uint64_t* k_full;
  uint64_t* v_full;
  uint64_t* kv_empty;
  uint64_t* s_full;   // [2]
  uint64_t* p_ready;  // [2]
  uint64_t* pv_done;  // [2]: PV(j) arrives on pv_done[j & 1]
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_bf16_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const AttnOut out) {
  using C = Cfg<D>;
  constexpr int NST = C::NST;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + C::kQBytes;
  uint8_t* sV = sK + NST * C::kTileBytes;
  uint64_t* bar_base = reinterpret_cast<uint64_t*>(sV + NST * C::kTileBytes);
  Bars bars;
  bars.q_full = bar_base;
  bars.k_full = bars.q_full + 1;
  bars.v_full = bars.k_full + NST;
  bars.kv_empty = bars.v_full + NST;
  bars.s_full = bars.kv_empty + NST;
  bars.p_ready = bars.s_full + 2;
  bars.pv_done = bars.p_ready + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_base + C::kNumBars);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int N = out.N;
  const int nkv = (N + BN - 1) / BN;
  int* err = out.err;

  if (threadIdx.x == 0) {
    mbar_init(bars.q_full, 1);
    for (int s = 0; s < NST; ++s) {
      mbar_init(bars.k_full + s, 1);
      mbar_init(bars.v_full + s, 1);
      mbar_init(bars.kv_empty + s, 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bars.s_full + s, 1);
      mbar_init(bars.p_ready + s, 128);
      mbar_init(bars.pv_done + s, 1);
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
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(bars.q_full, C::kQBytes);
#pragma unroll
      for (int c = 0; c < D / 64; ++c) tma_load_4d(sQ + c * C::kSubTile, &tmQ, bars.q_full, c * 64, qt * BM, h, b);
      for (int j = 0; j < nkv; ++j) {
        const int st = j % NST;
        if (j >= NST) {
          if (!mbar_wait(bars.kv_empty + st, ((j / NST) & 1) ^ 1, err, kErrTimeout)) break;
        }
        uint8_t* k_dst = sK + st * C::kTileBytes;
        uint8_t* v_dst = sV + st * C::kTileBytes;
        mbar_arrive_expect_tx(bars.k_full + st, C::kTileBytes);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_load_4d(k_dst + c * C::kSubTile, &tmK, bars.k_full + st, c * 64, j * BN, h, b);
        mbar_arrive_expect_tx(bars.v_full + st, C::kTileBytes);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_load_4d(v_dst + c * C::kSubTile, &tmV, bars.v_full + st, c * 64, j * BN, h, b);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = make_idesc(1, 1, 0, BM, BN);  // bf16 x bf16, K-major both
      constexpr uint32_t idesc_o = make_idesc(1, 1, 1, BM, D);   // V is MN-major (d contiguous)
      const uint32_t tO = tmem + kColO;
      const uint32_t q_addr = smem_u32(sQ);
      bool ok = mbar_wait(bars.q_full, 0, err, kErrTimeout);
      for (int j = 0; ok && j <= nkv; ++j) {
        if (j < nkv) {
          const int st = j % NST;
          if (!mbar_wait(bars.k_full + st, (j / NST) & 1, err, kErrTimeout)) break;
          tc_fence_after();
          const uint32_t k_addr = smem_u32(sK + st * C::kTileBytes);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * C::kSubTile + (kk & 3) * 32;
            mma_f16_ss(tmem + ((j & 1) ? kColS1 : kColS0), smem_desc_sw128(q_addr + off, 16, 1024), smem_desc_sw128(k_addr + off, 16, 1024),
                       idesc_s, kk > 0 ? 1u : 0u);
          }
          mma_commit(bars.s_full + (j & 1));
        }
        if (j >= 1) {
          const int jj = j - 1;
          const int st = jj % NST;
          if (!mbar_wait(bars.p_ready + (jj & 1), (jj >> 1) & 1, err, kErrTimeout)) break;
          if (!mbar_wait(bars.v_full + st, (jj / NST) & 1, err, kErrTimeout)) break;
          tc_fence_after();
          const uint32_t v_addr = smem_u32(sV + st * C::kTileBytes);
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {
            // 16 keys = 16 rows of 128 bytes; d sub-tiles 64 wide are C::kSubTile apart
            mma_f16_ts(tO, tmem + ((jj & 1) ? kColP1 : kColP0) + kk * 8, smem_desc_sw128(v_addr + kk * 16 * 128, C::kSubTile, 1024), idesc_o,
                       (jj > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(bars.pv_done + (jj & 1));
          mma_commit(bars.kv_empty + st);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ softmax warps 0..3
    const int row = threadIdx.x;                   // 0..127 = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const float sl2 = out.scale_log2;
    float m = -INFINITY;  // running max of scale*log2e*s
    float l = 0.f;
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      const int bsel = j & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(bars.s_full + bsel, (j >> 1) & 1, err, kErrTimeout));
      if (!ok) break;
      tc_fence_after();
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
          if (kv0 + c >= N) s[c] = 0xff800000u;  // -inf: key beyond the sequence
      }
      // row max of the raw scores: 8 independent chains, then a tree
      float mx8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mx8[i] = __uint_as_float(s[i]);
#pragma unroll
      for (int c = 8; c < BN; c += 8)
#pragma unroll
        for (int i = 0; i < 8; ++i) mx8[i] = fmaxf(mx8[i], __uint_as_float(s[c + i]));
      const float m_tile =
          fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])), fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]))) *
          sl2;
      // Lazy rescale: the running max moves (and O is rescaled) only when some row of
      // the warp gains more than kRescaleLog2; otherwise the stale max is kept, every
      // p stays <= 2^kRescaleLog2 and O, l remain consistent, so the result is exact.
      const bool grow = __any_sync(0xffffffffu, m_tile > m + kRescaleLog2);
      const float m_new = grow ? fmaxf(m, m_tile) : m;
      const float alpha = grow ? ex2(m - m_new) : 1.f;
      const float neg_m = -m_new;
      // P(j) goes to buffer j&1, last read by PV(j-2)
      if (j >= 2) {
        ok = __all_sync(0xffffffffu, mbar_wait(bars.pv_done + bsel, ((j >> 1) - 1) & 1, err, kErrTimeout));
        if (!ok) break;
        tc_fence_after();
      }
      float sum8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      const uint32_t tP = tmem + (bsel ? kColP1 : kColP0) + lane_off;
#pragma unroll
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t p[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float p0 = ex2(fmaf(__uint_as_float(s[c * 32 + 2 * e]), sl2, neg_m));
          const float p1 = ex2(fmaf(__uint_as_float(s[c * 32 + 2 * e + 1]), sl2, neg_m));
          sum8[e & 7] += p0 + p1;
          p[e] = pack_bf16x2(p0, p1);
        }
        tmem_st16(tP + c * 16, p);
      }
      const float sum = ((sum8[0] + sum8[1]) + (sum8[2] + sum8[3])) + ((sum8[4] + sum8[5]) + (sum8[6] + sum8[7]));
      if (j > 0 && grow) {
        // O holds PV(0..j-1) only once PV(j-1) has completed
        ok = __all_sync(0xffffffffu, mbar_wait(bars.pv_done + (bsel ^ 1), ((j - 1) >> 1) & 1, err, kErrTimeout));
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
      mbar_arrive(bars.p_ready + bsel);
    }
    // ---------------------------------------------------------- epilogue
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bars.pv_done + ((nkv - 1) & 1), ((nkv - 1) >> 1) & 1, err, kErrTimeout));
    if (ok) {
      tc_fence_after();
      const float inv_l = 1.f / l;
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
            pw[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv_l, __uint_as_float(o[2 * e + 1]) * inv_l);
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

template <int D>
cudaError_t launch_d(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const AttnOut& out, int B,
                     int H, cudaStream_t stream) {
  constexpr int smem = Cfg<D>::kSmemBytes;
  cudaError_t e = cudaFuncSetAttribute(attn_bf16_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid((out.N + BM - 1) / BM, H, B);
  attn_bf16_kernel<D><<<grid, kThreads, smem, stream>>>(tq, tk, tv, out);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_bf16(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const AttnOut& out,
                             int B, int H, int d, cudaStream_t stream) {
  if (d == 128) return launch_d<128>(tq, tk, tv, out, B, H, stream);
  if (d == 64) return launch_d<64>(tq, tk, tv, out, B, H, stream);
  return cudaErrorInvalidValue;
}

}  // namespace dit
