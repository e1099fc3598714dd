// Joint attention kernel for sm_100a, shared by the BF16 and FP8 variants:
// TMA -> shared memory -> tcgen05 MMA -> TMEM, flash-style online softmax in
// fp32 with exp2.
//
// Source: "FLUX 3 Image Klein / TensorRT-LLM VisualGen", section on why the
// differences arise: the DiT's VANILLA BF16 attention over the joint
// text+image tokens is about 60 % of its GPU kernel time, and cuDNN FP8
// attention is its quantised counterpart.  O = softmax(scale Q K^T) V per
// (batch, head), bidirectional over every key.
//
// One CTA owns two 128-row Q tiles (Q0, Q1) of one (b, h) and streams every
// K/V tile of that head once for both, halving the K/V traffic from L2 per
// FLOP compared with one tile per CTA.  384 threads:
//   warps 0-3  softmax of Q0 (thread t = row t = TMEM lane t)
//   warps 4-7  softmax of Q1
//   warp 8     TMA producer: Q0, Q1 once; K_j into a NK-deep ring, V_j into a NV-deep ring
//   warp 9     MMA issuer (one thread) and TMEM owner
//   warps 10-11 idle (they complete the third warpgroup for the register re-split)
// Registers: launched at 168 per thread; the third warpgroup drops to kRegsAux and
// the softmax warpgroups rise to kRegsSoftmax.  setmaxnreg draws on the block's
// launch registers, so 2*128*kRegsSoftmax + 128*kRegsAux (63,488) must not exceed
// 384 * 168 = 64,512; the static_assert below only bounds it by the register file,
// and a CPU test checks it against the count ptxas assigns.
// BF16: RoPE of Q happens as Q is loaded: the softmax warpgroup that owns a Q
// tile rotates the raw bf16 rows in shared memory with the cos/sin tables and
// writes them back in place before the first MMA reads them.  K is rotated once
// per head by a separate pass, since every CTA of the head re-reads each K tile.
// FP8: Q, K and V arrive rotated, smoothed (K) and quantised from one prologue
// pass (rotating and quantising Q here measured 4 % slower per tile).
// TMEM (512 columns x 128 lanes x 32 bit): S0 [0,128) S1 [128,256) O0, O1 (d
// columns each from 256).  BF16: P_i (64 columns of bf16 pairs) overwrites the
// first columns of S_i once the softmax has read S_i.  FP8: P_i is written to
// a shared-memory tile of its own (see kPSmem), and S_i is free as soon as the
// softmax has loaded it into registers.
// The BF16 MMA thread issues, per key tile j:
//     O0 += P0(j-1) V(j-1);  S0(j) = Q0 K(j)^T;  O1 += P1(j-1) V(j-1);  S1(j) = Q1 K(j)^T
// The FP8 MMA thread instead polls both warpgroups' hand-offs and issues
// whatever is ready: S_i(j) once softmax i has read S_i(j-1) (s_free_i) and
// K(j) has landed, O_i += P_i(j) V(j) once softmax i has stored P_i(j)
// (p_ready_i) and V(j) has landed; it commits each PV to pv_done_i, which
// softmax i waits for before it overwrites P_i or rescales O_i.  (The ordering
// argument below is BF16's.)
// tcgen05 MMAs from one thread are executed in issue order, so S_i(j) never
// overwrites P_i(j-1) before PV_i(j-1) has read it, and a tcgen05.commit
// tracks every MMA the thread issued before it: when softmax i sees S_i(j)
// complete, PV_i(j-1) is complete too and O_i may be rescaled in place.  K and
// V stages are freed by count-2 mbarriers with one commit after each of the two
// MMAs reading the stage.  The tensor core runs PV1(j-1), S1(j) while softmax 0
// works on S0(j), and PV0(j), S0(j+1) while softmax 1 works on S1(j); in BF16
// the two softmax warpgroups take turns on the ex2 unit (in FP8 they run
// freely).  BF16 releases P_i(j) in two 64-key halves, so the MMA thread issues
// the first half of PV_i(j) while the second half is still being
// exponentiated.  BF16's thread-to-thread hand-offs (P ready -> MMA warp, the
// ping-pong turns) use named barriers, which are far cheaper than an mbarrier
// round trip; FP8's (S free, P ready) are mbarriers, which the MMA lane can poll
// side by side and which have a tile of slack; the tensor core and the TMA unit
// signal through mbarriers in both.
#pragma once

#include <cuda_bf16.h>

#include <cfloat>

#include "dit_device.cuh"

namespace dit {

template <bool FP8, int D>
struct AttnCfg {
  static constexpr int BM = 128;                        // rows per Q tile (two per CTA)
  static constexpr int BN = kAttnBlockN;                // keys per K/V tile (128)
  static constexpr int kThreads = 384;
  static constexpr uint32_t kRegsSoftmax = 208, kRegsAux = 80;
  static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsAux <= 65536, "register re-split exceeds the register file");
  static constexpr int EB = FP8 ? 1 : 2;                // element bytes
  static constexpr int kRowBytes = D * EB;              // bytes of one token row
  static constexpr int kSub = kRowBytes / 128;          // 128-byte swizzle column blocks per row
  static constexpr int kSubBytes = BN * 128;            // one [128 rows][128 B] column block
  static constexpr int kTileBytes = BN * kRowBytes;     // one Q, K or V tile
  static constexpr int kBoxInner = 128 / EB;            // TMA box inner extent (elements)
  static constexpr int NK = (!FP8 && D == 128) ? 3 : 4;
  static constexpr int NV = (!FP8 && D == 128) ? 2 : 4;
  // FP8: P_i goes to shared memory (one [128 rows][128 keys] e4m3 tile per Q
  // tile, the same 128-byte-swizzled K-major layout as a Q tile) instead of
  // overwriting S_i in TMEM, so S_i(j+1) may be computed as soon as softmax i
  // has read S_i(j) into registers: the softmax never waits for PV_i(j) and
  // S_i(j+1) to run back to back.  BF16's P (32 KB per tile) does not fit.
  static constexpr bool kPSmem = FP8;
  static constexpr int kPTileBytes = kPSmem ? BM * BN : 0;
  static constexpr int kNumBars = 2 + 2 * NK + 2 * NV + 2 + 2 + 2 + 1 + 2 + 2;
  static constexpr int kSmemBytes =
      1024 + 2 * kTileBytes + (NK + NV) * kTileBytes + 2 * kPTileBytes + kNumBars * 8 + 32;
  static constexpr int kKStep = FP8 ? 32 : 16;          // K extent of one MMA (elements)
  static constexpr uint32_t kColS = 0, kColO = 256;     // S_i at 128 i, O_i at 256 + D i
  static constexpr uint32_t kTmemCols = 512;
  // Lazy rescale threshold tau (log2 units): O and l stay in the frame of a stale
  // max m until a row's tile max exceeds m + tau, so every p = 2^(x - m) <= 2^tau.
  // BF16: tau = 8 (a larger tau keeps the range but rounds the dominant p of a
  // near-one-hot row to bf16 in a stale frame, which costs accuracy).  FP8: e4m3 P is
  // stored as p * 2^-tau * 448 * sV / sV_max <= 448, so tau buys fewer rescales
  // at the price of smaller P codes; at tau = 4 only p < 2^-11 (relative to the
  // row max) falls below the e4m3 normal range.
  static constexpr int kTau = FP8 ? 4 : 8;
  // BF16 hands P to the MMA warp in two 64-key halves, so that the first half of
  // PV runs while the second half is exponentiated (2.3 % fewer cycles); for FP8,
  // whose PV is only four MMAs, the extra hand-off costs more than it hides (+7 %).
  static constexpr bool kSplitP = !FP8;
  // BF16: the two softmax warpgroups take turns on the ex2 unit (ping-pong); FP8,
  // whose MMAs are half as long, does better letting them exponentiate at the
  // same time (1.4 % fewer cycles).
  static constexpr bool kPingPong = !FP8;
  // Exponentials computed on the FMA pipe (ex2_poly_pair) instead of the MUFU
  // unit: bit e set = key pair e of each 32-key group (BF16, e < 16) or key quad e
  // of each 32-key group, over two groups (FP8, bits 0-15).
#ifdef DIT_POLY_MASK_BF16
  static constexpr uint32_t kPolyMaskBf16 = DIT_POLY_MASK_BF16;
#else
  static constexpr uint32_t kPolyMaskBf16 = 0u;
#endif
#ifdef DIT_POLY_MASK_FP8
  static constexpr uint32_t kPolyMaskFp8 = DIT_POLY_MASK_FP8;
#else
  static constexpr uint32_t kPolyMaskFp8 = 0u;
#endif
  static constexpr uint32_t kPolyMask = FP8 ? kPolyMaskFp8 : kPolyMaskBf16;
  static constexpr float kRescaleLog2 = static_cast<float>(kTau);
  static constexpr float kTwoTau = static_cast<float>(1ull << kTau);
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert(kRowBytes % 128 == 0, "token rows must be whole 128-byte swizzle atoms");
  static_assert(BM == BN, "Q and K/V tiles share the column-block size kSubBytes");
};

// Scales of the FP8 variant (unused by BF16).
struct AttnScales {
  const float* q_scale;      // [B*H][nq]  (128-token blocks)
  const float* k_scale;      // [B*H][nk]  (64-token blocks)
  const float* v_scale;      // [B*H][nk]
  const float* v_scale_max;  // [B*H]
  int H;
};

__device__ __forceinline__ uint32_t cvt_e4m3x4(float a, float b, float c, float d) {
  uint16_t lo, hi;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(b), "f"(a));
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(d), "f"(c));
  return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}

// Integer score -> float without a conversion instruction: for |s| < 2^22 the
// bits (s & 0x7FFFFF) ^ 0x4B400000 are the float 1.5 * 2^23 + s, exactly (one
// lop3).  The softmax works on these biased values and folds the bias into
// its scale-and-subtract constant.
constexpr float kI8Bias = 12582912.0f;  // 1.5 * 2^23
__device__ __forceinline__ uint32_t s32_biased_f32(uint32_t s) {
  uint32_t r;
  asm("lop3.b32 %0, %1, 0x007FFFFF, 0x4B400000, 0x6A;" : "=r"(r) : "r"(s));
  return r;
}

__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float lg2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t* r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]),
               "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}

// BF16 Q tile rotation by the softmax warpgroup that owns the tile (128
// threads): each row is rotated in fp32 with the cos/sin tables and written
// back in place as bf16 (the tensor-core operand, rounded once).
// Work split: thread t owns 16-byte channel chunk c = t % CPR (8 channels, 4
// rotary pairs) of rows t / CPR + RPP k, so a warp reads whole table rows (512
// contiguous bytes per load instruction).  Every table load is issued before the
// wait for the tile (the caller passes the wait in as a callable), so one L2
// round trip overlaps the TMA load; a thread-per-row split with per-chunk loads
// serialised sixteen round trips (about 16k cycles per CTA, measured).
// Out of line, so that its registers stay out of the softmax branch's allocation.
template <int D, typename Wait>
__device__ __noinline__ bool rotate_q_tile(uint8_t* q_tile, const float* rope_cos, const float* rope_sin, int qrow0,
                                           int N, Wait wait_tile, int* err) {
  constexpr int kSubBytes = 128 * 128;  // one 128-row, 128-byte column block
  constexpr int CPR = D / 8;            // 16-byte chunks per row
  constexpr int RPP = 128 / CPR;        // rows covered per pass
  constexpr int NP = 128 / RPP;         // passes (= rows per thread)
  const int t = threadIdx.x & 127;
  const int c = t % CPR, r0 = t / CPR;
  const bool rope = rope_cos != nullptr;
  float4 cv[NP], sv[NP];
#pragma unroll
  for (int k = 0; k < NP; ++k) {
    const int n = qrow0 + r0 + RPP * k;
    if (rope && n < N) {  // rows past N are zero-filled by TMA and stay 0
      cv[k] = __ldg(reinterpret_cast<const float4*>(rope_cos + static_cast<int64_t>(n) * (D / 2)) + c);
      sv[k] = __ldg(reinterpret_cast<const float4*>(rope_sin + static_cast<int64_t>(n) * (D / 2)) + c);
    } else {
      cv[k] = make_float4(1.f, 1.f, 1.f, 1.f);
      sv[k] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  const bool q_ok = wait_tile();
  if (!rope || !q_ok) return q_ok;
#pragma unroll
  for (int k = 0; k < NP; ++k) {
    // row r's chunk c sits at column block c / 8, 16-byte slot (c % 8) ^ (r % 8) (128-byte swizzle)
    const int r = r0 + RPP * k;
    const int off = r * 128 + (c >> 3) * kSubBytes + (((c & 7) ^ (r & 7)) << 4);
    if (!debug_check(off >= 0 && off + 16 <= 128 * D * 2, err)) continue;  // within the bf16 Q tile
    uint4* p = reinterpret_cast<uint4*>(q_tile + off);
    const uint4 xv = *p;
    const __nv_bfloat162* xp = reinterpret_cast<const __nv_bfloat162*>(&xv);
    const float cc[4] = {cv[k].x, cv[k].y, cv[k].z, cv[k].w}, ss[4] = {sv[k].x, sv[k].y, sv[k].z, sv[k].w};
    float y[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 x = __bfloat1622float2(xp[e]);
      y[2 * e] = x.x * cc[e] - x.y * ss[e];
      y[2 * e + 1] = x.x * ss[e] + x.y * cc[e];
    }
    uint4 o4;
    o4.x = pack_bf16x2(y[0], y[1]);
    o4.y = pack_bf16x2(y[2], y[3]);
    o4.z = pack_bf16x2(y[4], y[5]);
    o4.w = pack_bf16x2(y[6], y[7]);
    *p = o4;
  }
  return true;
}

// Named barriers of the attention kernel (0 is __syncthreads): P-ready of
// softmax warpgroup i (128 arrivals + the MMA warp's 32), the ping-pong turns
// (256), and BF16's first-half P hand-off (160).
constexpr uint32_t kBarPReady = 1, kBarTurn = 3, kBarPHalf = 5;

// The MMA warp's failure path: the rest of its named-barrier schedule from
// iteration j (every P-half and P-ready sync it would have made, without the
// MMAs), publishing its progress after each P-ready as the normal path does.
template <bool kSplitP>
__device__ __noinline__ void mma_warp_finish_schedule(int j, int nkv, uint32_t mma_done, bool leader) {
  for (; j <= nkv; ++j) {
    if constexpr (kSplitP) named_sync<kBarPHalf + 0, 160>();
    named_sync<kBarPReady + 0, 160>();
    if (leader) flag_store(mma_done, j);
    if constexpr (kSplitP) named_sync<kBarPHalf + 1, 160>();
    named_sync<kBarPReady + 1, 160>();
    if (leader) flag_store(mma_done + 4, j);
  }
}

// I8QK (FP8 only): Q and K are symmetric int8 and S = Q K^T is a kind::i8 MMA
// with s32 accumulation (exact: |S| <= 127^2 * 128 < 2^22); P.V stays e4m3.
template <bool FP8, int D, bool I8QK = false>
__global__ void __launch_bounds__(384, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const AttnOut out, const AttnScales sc) {
  static_assert(FP8 || !I8QK, "the integer Q.K^T belongs to the FP8 variant");
  using C = AttnCfg<FP8, D>;
  constexpr int NK = C::NK, NV = C::NV, BM = C::BM, BN = C::BN;
  // device-side skip (the cache gate's flag): the whole CTA leaves before any
  // barrier, TMEM allocation or load, so an early return is safe
  if (out.skip != nullptr && *out.skip != 0) return;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                        // Q0, Q1
  uint8_t* sK = sQ + 2 * C::kTileBytes;      // NK stages
  uint8_t* sV = sK + NK * C::kTileBytes;     // NV stages
  uint8_t* sP = sV + NV * C::kTileBytes;     // FP8: P0, P1
  uint64_t* q_full = reinterpret_cast<uint64_t*>(sP + 2 * C::kPTileBytes);  // [2]
  uint64_t* k_full = q_full + 2;
  uint64_t* k_empty = k_full + NK;
  uint64_t* v_full = k_empty + NK;
  uint64_t* v_empty = v_full + NV;
  uint64_t* s_full = v_empty + NV;   // [2] S_i(j) computed (and every earlier MMA)
  uint64_t* pv_done = s_full + 2;    // [2] BF16: the last PV_i computed (read by the epilogue);
                                     //     FP8: every PV_i(j) computed (one phase per tile)
  uint64_t* q_ready = pv_done + 2;   // [2] BF16: Q_i rotated in shared memory (128 arrivals)
  uint64_t* mma_drain = q_ready + 2; // failure path: every MMA the MMA thread issued has completed
  uint64_t* s_free = mma_drain + 1;  // [2] FP8: softmax i has read S_i(j) (one arrival per warp)
  uint64_t* p_ready = s_free + 2;    // [2] FP8: softmax i has stored P_i(j) (one arrival per warp)
  // named barriers: kBarPReady + i  softmax i finished tile j (128 arrive, MMA warp syncs)
  //                 kBarTurn + i    softmax i may exponentiate (128 arrive, 128 sync)
  //                 kBarPHalf + i   BF16: softmax i stored keys 0..63 of P (128 arrive, MMA warp syncs)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(q_full + C::kNumBars);
  // Raised by the first role whose bounded wait gives up; every other bounded
  // wait then gives up too.  BF16: a role that gives up still performs the rest
  // of its named-barrier schedule (arrivals and syncs, without the work between
  // them), so a partner blocked on a named barrier is always released: named
  // barriers cannot time out, and their schedule is balanced.  FP8 has no named
  // barriers: every wait in it is bounded, so a role simply leaves.
  const uint32_t abort_flag = smem_u32(tmem_slot + 1);
  // Progress counters that pace the failure path (written on every path, read only
  // on the failure path): mma_done[i] = PReady_i generations the MMA warp has
  // passed.  A warpgroup on the failure path makes an arrival only once its
  // partner has passed the previous generation of that barrier, as the data
  // dependencies ensure on the normal path, so that no arrival lands a
  // generation early (a named barrier would merge it into the current generation
  // and strand the partner).  The MMA warp's progress also bounds the ping-pong
  // partner's: it passes PReady_1(t-1) only after warpgroup 1 passed Turn_1(t-1),
  // and PReady_0(t) only after warpgroup 0 passed Turn_0(t-1).
  const uint32_t mma_done = smem_u32(tmem_slot + 2);  // [2]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int N = out.N;
  const int nkv = (N + BN - 1) / BN;
  int* err = out.err;

  if (threadIdx.x == 0) {
    flag_store(abort_flag, 0);
    flag_store(mma_done, 0);
    flag_store(mma_done + 4, 0);
    mbar_init(mma_drain, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(q_full + i, 1);
      mbar_init(s_full + i, 1);
      mbar_init(pv_done + i, 1);
      mbar_init(q_ready + i, 128);
      mbar_init(s_free + i, 4);
      mbar_init(p_ready + i, 4);
    }
    for (int s = 0; s < NK; ++s) {
      mbar_init(k_full + s, 1);
      mbar_init(k_empty + s, 2);  // one commit after each of S0, S1
    }
    for (int s = 0; s < NV; ++s) {
      mbar_init(v_full + s, 1);
      mbar_init(v_empty + s, 2);  // one commit after each of PV0, PV1
    }
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // FP8 is launched as a programmatic dependent of its prologue's quantiser:
  // everything above may overlap the quantiser's last CTAs, and nothing below reads
  // its outputs before this wait (a no-op for BF16's plain launch)
  pdl_wait();

  if (warp >= 8) {
   regs_dec<C::kRegsAux>();
   if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        mbar_arrive_expect_tx(q_full + i, C::kTileBytes);
#pragma unroll
        for (int c = 0; c < C::kSub; ++c)
          if (debug_check((c * C::kBoxInner * C::EB) % 16 == 0 && i * C::kTileBytes + (c + 1) * C::kSubBytes <=
                              2 * C::kTileBytes, err))  // 16-byte x coordinate; inside the Q tiles
            tma_load_4d(sQ + i * C::kTileBytes + c * C::kSubBytes, &tmQ, q_full + i, c * C::kBoxInner,
                        (2 * qt + i) * BM, h, b);
      }
      int nk_issued = 0, nv_issued = 0;
      for (int j = 0; j < nkv; ++j) {
        const int sk = j % NK, sv = j % NV;
        if (j >= NK && !mbar_wait(k_empty + sk, ((j / NK) & 1) ^ 1, err, kErrTimeout, abort_flag)) break;
        mbar_arrive_expect_tx(k_full + sk, C::kTileBytes);
#pragma unroll
        for (int c = 0; c < C::kSub; ++c)
          if (debug_check(sk < NK && j * BN < N && (c * C::kBoxInner * C::EB) % 16 == 0, err))
            tma_load_4d(sK + sk * C::kTileBytes + c * C::kSubBytes, &tmK, k_full + sk, c * C::kBoxInner, j * BN, h,
                        b);
        ++nk_issued;
        if (j >= NV && !mbar_wait(v_empty + sv, ((j / NV) & 1) ^ 1, err, kErrTimeout, abort_flag)) break;
        mbar_arrive_expect_tx(v_full + sv, C::kTileBytes);
#pragma unroll
        for (int c = 0; c < C::kSub; ++c)
          if (debug_check(sv < NV && j * BN < N && (c * C::kBoxInner * C::EB) % 16 == 0, err))
            tma_load_4d(sV + sv * C::kTileBytes + c * C::kSubBytes, &tmV, v_full + sv, c * C::kBoxInner, j * BN, h,
                        b);
        ++nv_issued;
      }
      // Drain: the last load issued into every stage has landed before the CTA
      // may exit (on the fault-free path they all have by the time consumers
      // finish; after a failure this bounds the wait for a load left in flight).
      const uint64_t deadline = globaltimer_ns() + kWaitLimitNs;
      for (int i = 0; i < 2; ++i) mbar_wait_until(q_full + i, 0, deadline);
      for (int st = 0; st < NK && st < nk_issued; ++st) {
        const int last = st + ((nk_issued - 1 - st) / NK) * NK;
        mbar_wait_until(k_full + st, (last / NK) & 1, deadline);
      }
      for (int st = 0; st < NV && st < nv_issued; ++st) {
        const int last = st + ((nv_issued - 1 - st) / NV) * NV;
        mbar_wait_until(v_full + st, (last / NV) & 1, deadline);
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp walks the schedule (named barriers are warp-aligned); lane 0 issues.
      constexpr uint32_t fmt = FP8 ? 0u : 1u;  // e4m3 (kind::f8f6f4) or bf16 (kind::f16)
      constexpr uint32_t idesc_s = I8QK ? make_idesc_s8(BM, BN) : make_idesc(fmt, fmt, 0, BM, BN);  // both K-major
      constexpr uint32_t idesc_o = make_idesc(fmt, fmt, 1, BM, D);   // V MN-major (d contiguous)
      const uint32_t q_addr = smem_u32(sQ);
      const uint32_t k_addr = smem_u32(sK);
      const uint32_t v_addr = smem_u32(sV);
      const uint32_t p_addr = smem_u32(sP);
      auto qk = [&](int i, int sk) {  // S_i = Q_i K^T
        const uint32_t qa = q_addr + i * C::kTileBytes, ka = k_addr + sk * C::kTileBytes;
        // S_i's columns end before O's; the K stage is one of the ring's
        if (!debug_check(i < 2 && sk < NK && C::kColS + 128 * i + BN <= C::kColO, err)) return;
#pragma unroll
        for (int kk = 0; kk < D / C::kKStep; ++kk) {
          const uint32_t off = (kk >> 2) * C::kSubBytes + (kk & 3) * 32;  // 32 bytes of K per MMA
          const uint64_t ad = smem_desc_sw128(qa + off, 16, 1024), bd = smem_desc_sw128(ka + off, 16, 1024);
          if constexpr (I8QK)
            mma_i8_ss(tmem + C::kColS + 128 * i, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
          else if constexpr (FP8)
            mma_f8_ss(tmem + C::kColS + 128 * i, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
          else
            mma_f16_ss(tmem + C::kColS + 128 * i, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
        }
      };
      // O_i (+)= P_i V over MMA steps [k0, k1) of the tile's keys; the first step
      // overwrites O_i when acc is false (first tile)
      auto pv = [&](int i, int sv, bool acc, int k0, int k1) {
        const uint32_t va = v_addr + sv * C::kTileBytes;
        // O_i inside the allocation, P inside S_i, the V stage one of the ring's
        if (!debug_check(i < 2 && sv < NV && C::kColO + D * (i + 1) <= C::kTmemCols && k1 * 8 <= BN &&
                             k0 >= 0 && (!C::kPSmem || k1 * 32 <= BN), err))
          return;
#pragma unroll
        for (int kk = k0; kk < k1; ++kk) {
          // kKStep keys = kKStep rows of 128 bytes; d column blocks are kSubBytes apart
          const uint64_t bd = smem_desc_sw128(va + kk * C::kKStep * 128, C::kSubBytes, 1024);
          if constexpr (C::kPSmem) {
            // P_i in shared memory, K-major like a Q tile: kKStep keys = 32 bytes of each row
            const uint64_t ad = smem_desc_sw128(p_addr + i * C::kPTileBytes + kk * 32, 16, 1024);
            mma_f8_ss(tmem + C::kColO + D * i, ad, bd, idesc_o, (acc || kk > k0) ? 1u : 0u);
          } else {
            const uint32_t pa = tmem + C::kColS + 128 * i + kk * 8;  // 8 columns of packed P per MMA
            if constexpr (FP8)
              mma_f8_ts(tmem + C::kColO + D * i, pa, bd, idesc_o, (acc || kk > k0) ? 1u : 0u);
            else
              mma_f16_ts(tmem + C::kColO + D * i, pa, bd, idesc_o, (acc || kk > k0) ? 1u : 0u);
          }
        }
      };
      const bool leader = lane == 0;
      uint64_t* q_in = FP8 ? q_full : q_ready;  // BF16 waits for the in-place rotation
      bool ok = mbar_wait(q_in, 0, err, kErrTimeout, abort_flag) && mbar_wait(k_full, 0, err, kErrTimeout, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        tc_fence_after();
        if (leader) {
          qk(0, 0);
          mma_commit(s_full);
          mma_commit(k_empty);
        }
        ok = __all_sync(0xffffffffu, mbar_wait(q_in + 1, 0, err, kErrTimeout, abort_flag));
      }
      if (ok) {
        tc_fence_after();
        if (leader) {
          qk(1, 0);
          mma_commit(s_full + 1);
          mma_commit(k_empty);
        }
      }
      __syncwarp();
      if constexpr (C::kPSmem) {
        // FP8: lane 0 polls four event streams and issues whatever is ready, so that
        // neither softmax warpgroup waits behind the other's hand-offs:
        //   S_i(ns_i)  once softmax i has read S_i(ns_i - 1) and K(ns_i) has landed
        //   PV_i(np_i) once softmax i has stored P_i(np_i) and V(np_i) has landed
        // Each barrier is at most one phase ahead of the parity polled (the next
        // phase needs the MMA being waited for), so every poll is unambiguous.
        // Bounded: it gives up when another role raised the abort flag, or after
        // kWaitLimitNs without progress (recording the timeout and raising the flag).
        if (leader && ok) {
          int ns[2] = {1, 1}, np[2] = {0, 0};
          uint32_t idle = 0;
          uint64_t idle_since = 0;
          while (np[0] < nkv || np[1] < nkv) {
            bool progress = false;
#pragma unroll
            for (int i = 0; i < 2; ++i) {
              const int js = ns[i], sk = js % NK;
              if (js < nkv && mbar_try_wait(smem_u32(s_free + i), (js - 1) & 1) &&
                  mbar_try_wait(smem_u32(k_full + sk), (js / NK) & 1)) {
                tc_fence_after();
                qk(i, sk);
                mma_commit(s_full + i);
                mma_commit(k_empty + sk);
                ns[i] = js + 1;
                progress = true;
              }
              const int jp = np[i], sv = jp % NV;
              if (jp < nkv && mbar_try_wait(smem_u32(p_ready + i), jp & 1) &&
                  mbar_try_wait(smem_u32(v_full + sv), (jp / NV) & 1)) {
                tc_fence_after();
                pv(i, sv, jp > 0, 0, BN / C::kKStep);
                mma_commit(pv_done + i);  // P_i may be overwritten, O_i rescaled or read
                mma_commit(v_empty + sv);
                np[i] = jp + 1;
                progress = true;
              }
            }
            if (progress) {
              idle = 0;
            } else if ((++idle & 63u) == 1u) {
              const uint64_t now = globaltimer_ns();
              if (idle == 1u) idle_since = now;
              if (flag_load(abort_flag) != 0) break;
              if (now - idle_since > kWaitLimitNs) {
                set_error(err, kErrTimeout);
                flag_store(abort_flag, 1);
                break;
              }
            }
          }
        }
        __syncwarp();
      }
      for (int j = 1; !C::kPSmem && ok && j <= nkv; ++j) {
        const int jj = j - 1, sv = jj % NV, sk = j % NK;
        // another role gave up: stop issuing.  Then TMA readiness, while the
        // softmax warpgroups are still busy
        ok = flag_load(abort_flag) == 0;
        ok = ok && mbar_wait(v_full + sv, (jj / NV) & 1, err, kErrTimeout, abort_flag);
        if (ok && j < nkv) ok = mbar_wait(k_full + sk, (j / NK) & 1, err, kErrTimeout, abort_flag);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        constexpr int NKK = BN / C::kKStep, KH = C::kSplitP ? NKK / 2 : 0;

        if constexpr (C::kSplitP) {  // first half of PV_0 while softmax 0 finishes P_0
          named_sync<kBarPHalf + 0, 160>();
          tc_fence_after();
          if (leader) pv(0, sv, jj > 0, 0, KH);
          __syncwarp();
        }
        named_sync<kBarPReady + 0, 160>();
        tc_fence_after();
        if (leader) {
          pv(0, sv, KH > 0 || jj > 0, KH, NKK);
          if (j == nkv) mma_commit(pv_done);  // the epilogue waits for the last PV only
          mma_commit(v_empty + sv);
          if (j < nkv) {
            qk(0, sk);
            mma_commit(s_full);
            mma_commit(k_empty + sk);
          }
          flag_store(mma_done, j);
        }
        __syncwarp();
        if constexpr (C::kSplitP) {
          named_sync<kBarPHalf + 1, 160>();
          tc_fence_after();
          if (leader) pv(1, sv, jj > 0, 0, KH);
          __syncwarp();
        }
        named_sync<kBarPReady + 1, 160>();
        tc_fence_after();
        if (leader) {
          pv(1, sv, KH > 0 || jj > 0, KH, NKK);
          if (j == nkv) mma_commit(pv_done + 1);  // the epilogue waits for the last PV only
          mma_commit(v_empty + sv);
          if (j < nkv) {
            qk(1, sk);
            mma_commit(s_full + 1);
            mma_commit(k_empty + sk);
          }
          flag_store(mma_done + 4, j);
        }
        __syncwarp();
      }
      // Failure path: the rest of the named-barrier schedule, no MMAs, from the first
      // iteration not completed: the one after the last progress published for
      // warpgroup 1.  (Carrying the loop index out of the loop instead cost the
      // normal path 6 % of its cycles in BF16, measured.)
      if (!C::kPSmem && !ok) mma_warp_finish_schedule<C::kSplitP>(flag_load(mma_done + 4) + 1, nkv, mma_done, leader);
   }
  } else {
    regs_inc<C::kRegsSoftmax>();
    // ------------------------------------------------------------ softmax warpgroups
    const int i = warp >> 2;                    // Q tile of this warpgroup
    const int qblk = 2 * qt + i;                // 128-row block index of this Q tile
    // ------------------------------------------------ BF16: rotate Q on load
    // First, while almost nothing is live: the per-tile loop's constants are formed
    // after it, so the preparation's registers cannot push them into local memory
    // (measured: 6 % slower per tile when it ran after them).
    bool ok = true;
    if constexpr (!FP8) {
      uint64_t* qf = q_full + i;
      auto wait_tile = [qf, err, abort_flag]() { return mbar_wait(qf, 0, err, kErrTimeout, abort_flag); };
      ok = __all_sync(0xffffffffu, rotate_q_tile<D>(sQ + i * C::kTileBytes, out.rope_cos, out.rope_sin, qblk * BM, N,
                                                    wait_tile, err));
      // the MMA reads Q through the async proxy: order the generic-proxy writes first
      fence_proxy_async_smem();
      // only a tile that came is handed on; otherwise the MMA warp's bounded wait gives up
      if (ok) mbar_arrive(q_ready + i);
    }
    const int row = threadIdx.x & 127;          // TMEM lane = row of the tile
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + C::kColS + 128 * i + lane_off;
    const uint32_t tO = tmem + C::kColO + D * i + lane_off;
    // this warp's lanes and the S_i / O_i columns inside the 512-column allocation
    debug_check((warp & 3) * 32 + 32 <= 128 && C::kColS + 128 * i + BN <= C::kColO &&
                    C::kColO + D * (i + 1) <= C::kTmemCols, err);
    const float sl2 = out.scale_log2;
    // FP8 scales: score = S * sQ * sK(j) * scale, P8 = p * 2^-tau * 448 * sV(j) / sV_max
    float qs = sl2, vfold = 1.f, fin_scale = 1.f;
    const float* ksc = nullptr;
    const float* vsc = nullptr;
    int nk = 0;
    if constexpr (FP8) {
      const int bh = b * sc.H + h;
      const int nq = (N + 127) / 128;
      nk = (N + 63) / 64;
      ksc = sc.k_scale + static_cast<int64_t>(bh) * nk;
      vsc = sc.v_scale + static_cast<int64_t>(bh) * nk;
      const float vmax = sc.v_scale_max[bh];
      qs = (qblk < nq ? sc.q_scale[static_cast<int64_t>(bh) * nq + qblk] : 1.f) * sl2;
      vfold = 448.f / (vmax * C::kTwoTau);
      fin_scale = vmax * C::kTwoTau / 448.f;
    }
    // O_i *= alpha, RC columns at a time (64 while half of the scores are still in
    // registers, all d after the tile's exps).  Called once S_i(j) is seen complete:
    // the commit behind it covers PV_i(0..j-1), so no MMA is writing O_i.
    auto rescale_o = [&](float alpha) {
      constexpr int RC = C::kSplitP ? 64 : D;
      const uint64_t a2 = f2(alpha, alpha);
#pragma unroll
      for (int hc = 0; hc < D / RC; ++hc) {
        uint32_t o[RC];
#pragma unroll
        for (int c = 0; c < RC / 32; ++c) tmem_ld32(tO + hc * RC + c * 32, o + c * 32);
        tmem_wait_ld();
        reg_fence(o);
#pragma unroll
        for (int e = 0; e < RC / 2; ++e) {
          float x, y;
          f2_split(fmul2(f2(__uint_as_float(o[2 * e]), __uint_as_float(o[2 * e + 1])), a2), x, y);
          o[2 * e] = __float_as_uint(x);
          o[2 * e + 1] = __float_as_uint(y);
        }
#pragma unroll
        for (int c = 0; c < RC / 32; ++c) tmem_st32(tO + hc * RC + c * 32, o + c * 32);
        tmem_wait_st();
        reg_fence(o);
      }
    };
    float m = -INFINITY;  // running (possibly stale) max of the scaled log2 scores
    float l = 0.f;
    // FP8: the K and V block scales of the next tile, loaded one tile ahead so that
    // their global-memory latency stays off the per-tile critical path
    float ksn0 = 1.f, ksn1 = 1.f, vsn0 = 1.f, vsn1 = 1.f;
    if constexpr (FP8) {
      ksn0 = ksc[0];
      vsn0 = vsc[0];
      if (1 < nk) {
        ksn1 = ksc[1];
        vsn1 = vsc[1];
      }
    }
    int j = 0;
    for (; ok && j < nkv; ++j) {
      ok = __all_sync(0xffffffffu, mbar_wait(s_full + i, j & 1, err, kErrTimeout, abort_flag));
      if (!ok) break;
      tc_fence_after();
      uint32_t s[BN];
#pragma unroll
      for (int c = 0; c < BN / 32; ++c) tmem_ld32(tS + c * 32, s + c * 32);
      tmem_wait_ld();
      reg_fence(s);
      if constexpr (C::kPSmem) {  // S_i is in registers: the MMA warp may compute S_i(j+1) into it
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_free + i);
      }
      if constexpr (I8QK) {
#pragma unroll
        for (int c = 0; c < BN; ++c) s[c] = s32_biased_f32(s[c]);
      }
      const int kv0 = j * BN;
      if (kv0 + BN > N) {
#pragma unroll
        for (int c = 0; c < BN; ++c)
          if (kv0 + c >= N) s[c] = 0xff800000u;  // -inf: key beyond the sequence
      }
      // per-64-key-half score multipliers (both equal for BF16)
      float c0 = sl2, c1 = sl2, f0 = 1.f, f1 = 1.f;
      if constexpr (FP8) {
        // a half past the end keeps 1: its keys are -inf (-inf * c1 = -inf) and its p are 0
        c0 = qs * ksn0;
        c1 = qs * ksn1;
        // held in the normal range, so that lg2 and the reciprocal below stay finite
        // (a V block of denormal values then contributes nothing to P.V, as it
        // would contribute nothing measurable to O)
        f0 = fmaxf(vsn0 * vfold, FLT_MIN);
        f1 = fmaxf(vsn1 * vfold, FLT_MIN);
        const int kb0 = 2 * j + 2, kb1 = 2 * j + 3;  // the next tile's blocks
        ksn0 = kb0 < nk ? ksc[kb0] : 1.f;
        vsn0 = kb0 < nk ? vsc[kb0] : 1.f;
        ksn1 = kb1 < nk ? ksc[kb1] : 1.f;
        vsn1 = kb1 < nk ? vsc[kb1] : 1.f;
      }
      // row max: two 3-input max chains per 64-key half (keys 0..3 of the half start
      // the chains, then four keys per step up to key 63 of the half)
      float ma0 = fmaxf(__uint_as_float(s[0]), __uint_as_float(s[1]));
      float ma1 = fmaxf(__uint_as_float(s[2]), __uint_as_float(s[3]));
      float mb0 = fmaxf(__uint_as_float(s[64]), __uint_as_float(s[65]));
      float mb1 = fmaxf(__uint_as_float(s[66]), __uint_as_float(s[67]));
#pragma unroll
      for (int c = 4; c < 64; c += 4) {
        ma0 = fmax3(ma0, __uint_as_float(s[c]), __uint_as_float(s[c + 1]));
        ma1 = fmax3(ma1, __uint_as_float(s[c + 2]), __uint_as_float(s[c + 3]));
        mb0 = fmax3(mb0, __uint_as_float(s[64 + c]), __uint_as_float(s[64 + c + 1]));
        mb1 = fmax3(mb1, __uint_as_float(s[64 + c + 2]), __uint_as_float(s[64 + c + 3]));
      }
      const float mx0 = fmaxf(ma0, ma1) - (I8QK ? kI8Bias : 0.f);  // exact: both within [2^23, 2^24)
      const float mx1 = fmaxf(mb0, mb1) - (I8QK ? kI8Bias : 0.f);
      // the first key of a tile is always in range; a half past the end is all -inf
      const float m_tile = fmaxf(mx0 * c0, kv0 + 64 < N ? mx1 * c1 : -INFINITY);
      const bool grow = __any_sync(0xffffffffu, m_tile > m + C::kRescaleLog2);
      const float m_new = grow ? fmaxf(m, m_tile) : m;
      const float alpha = grow ? ex2(m - m_new) : 1.f;
      // Ping-pong (BF16): the two warpgroups take turns on the ex2 unit, so one exponentiates
      // while the other's PV and next S run on the tensor core.  Softmax 0 goes first in
      // every tile; softmax 1 starts tile j once softmax 0 has finished tile j's exps.
      if constexpr (C::kPingPong) {
        if (i == 1) named_sync<kBarTurn + 1, 256>();
        else if (j > 0) named_sync<kBarTurn + 0, 256>();
      }
      // p = 2^(s * c - m): packed scale-and-subtract, ex2 per element, packed row
      // sums in 4 chains (in the shadow of the ex2 pipe), P to TMEM per 32 keys.
      // tcgen05.st reads its source registers asynchronously: every register a
      // pending store reads stays pinned (reg_fence after tcgen05.wait::st) so the
      // compiler cannot reuse it before the store has completed.
      const uint64_t nm2 = f2(-m_new, -m_new);
      // FP8: the V block scale of each 64-key half enters as an exponent offset,
      // p * f = 2^(x - m + log2 f), which saves a multiply per element.
      // I8QK: the scores in s are biased by kI8Bias; the bias times the half's
      // multiplier comes off here, once per tile, so x = s c + lf stays one FMA.
      const float lf0 = FP8 ? lg2(f0) - m_new - (I8QK ? kI8Bias * c0 : 0.f) : 0.f;
      const float lf1 = FP8 ? lg2(f1) - m_new - (I8QK ? kI8Bias * c1 : 0.f) : 0.f;
      const uint64_t nmA = f2(lf0, lf0), nmB = f2(lf1, lf1);
      uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
      constexpr int kPRegs = FP8 ? 32 : 64;  // packed P of the whole row
      uint32_t p[kPRegs];
#pragma unroll
      for (int q = 0; q < 4; ++q) {  // 32 keys per TMEM store
        const uint64_t cq = FP8 ? (q < 2 ? f2(c0, c0) : f2(c1, c1)) : f2(sl2, sl2);
        if constexpr (FP8) {  // 32 keys -> 8 columns of 4 e4m3 (V block scale folded in)
          const uint64_t nmq = q < 2 ? nmA : nmB;
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int k0 = 32 * q + 4 * e;
            const uint64_t xa = ffma2(f2(__uint_as_float(s[k0]), __uint_as_float(s[k0 + 1])), cq, nmq);
            const uint64_t xb = ffma2(f2(__uint_as_float(s[k0 + 2]), __uint_as_float(s[k0 + 3])), cq, nmq);
            float a, bq, cc, dd;
            if ((C::kPolyMask >> (8 * (q & 1) + e)) & 1u) {  // on the FMA pipe
              ex2_poly_pair(xa, a, bq);
              ex2_poly_pair(xb, cc, dd);
            } else {
              float x0, x1, x2, x3;
              f2_split(xa, x0, x1);
              f2_split(xb, x2, x3);
              a = ex2(x0), bq = ex2(x1), cc = ex2(x2), dd = ex2(x3);
            }
            // row sums per 64-key half (each carries its own V block scale)
            acc[2 * (q >> 1)] = fadd2(acc[2 * (q >> 1)], f2(a, bq));
            acc[2 * (q >> 1) + 1] = fadd2(acc[2 * (q >> 1) + 1], f2(cc, dd));
            p[8 * q + e] = cvt_e4m3x4(a, bq, cc, dd);
          }
          if constexpr (!C::kPSmem) tmem_st8(tS + 8 * q, p + 8 * q);
        } else {  // 32 keys -> 16 columns of 2 bf16
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const uint64_t xy =
                ffma2(f2(__uint_as_float(s[32 * q + 2 * e]), __uint_as_float(s[32 * q + 2 * e + 1])), cq, nm2);
            float p0, p1;
            if ((C::kPolyMask >> e) & 1u) {  // on the FMA pipe
              ex2_poly_pair(xy, p0, p1);
            } else {
              float x, y;
              f2_split(xy, x, y);
              p0 = ex2(x);
              p1 = ex2(y);
            }
            acc[e & 3] = fadd2(acc[e & 3], f2(p0, p1));
            p[16 * q + e] = pack_bf16x2(p0, p1);
          }
          tmem_st16(tS + 16 * q, p + 16 * q);
          if (C::kSplitP && q == 1) {  // keys 0..63 of P are in TMEM: PV may start on them once O is rescaled
            tmem_wait_st();
            reg_fence(p);
            if (j > 0 && grow) rescale_o(alpha);
            tc_fence_before();
            if (i == 0) named_arrive<kBarPHalf + 0, 160>();
            else named_arrive<kBarPHalf + 1, 160>();
          }
        }
      }
      // every arrive is matched by a sync of the other warpgroup
      if constexpr (C::kPingPong) {
        if (i == 0) named_arrive<kBarTurn + 1, 256>();
        else if (j + 1 < nkv) named_arrive<kBarTurn + 0, 256>();
      }
      if constexpr (C::kPSmem) {
        // PV_i(j-1) has read P_i and finished writing O_i: then P_i(j) replaces it
        if (j > 0) {
          ok = __all_sync(0xffffffffu, mbar_wait(pv_done + i, (j - 1) & 1, err, kErrTimeout, abort_flag));
          if (!ok) break;
        }
        // row `row`, 16-byte chunk c (keys 16c..16c+15) at slot c ^ (row % 8) of the row's 128 bytes
        uint8_t* prow = sP + i * C::kPTileBytes + row * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          if (debug_check(i * C::kPTileBytes + row * 128 + 128 <= 2 * C::kPTileBytes, err))
            st_shared_v4(prow + ((c ^ (row & 7)) << 4), p[4 * c], p[4 * c + 1], p[4 * c + 2], p[4 * c + 3]);
        // the MMA reads P through the async proxy: order the generic-proxy writes first
        fence_proxy_async_smem();
      } else {
        tmem_wait_st();
        reg_fence(p);
      }
      if (!C::kSplitP && j > 0 && grow) rescale_o(alpha);
      tc_fence_before();
      if constexpr (C::kPSmem) {
        __syncwarp();
        if (lane == 0) mbar_arrive(p_ready + i);
      } else if (i == 0) {
        named_arrive<kBarPReady + 0, 160>();
      } else {
        named_arrive<kBarPReady + 1, 160>();
      }
      float a0, a1;
      if constexpr (FP8) {  // divide each half's V block scale back out of its row sum
        float b0, b1;
        f2_split(fadd2(acc[0], acc[1]), a0, a1);
        f2_split(fadd2(acc[2], acc[3]), b0, b1);
        // approximate reciprocals (MUFU, relative error ~2^-23): the IEEE-rounded
        // ones cost a multi-instruction sequence twice per tile on the critical path
        l = l * alpha + ((a0 + a1) * rcp_approx(f0) + (b0 + b1) * rcp_approx(f1));
      } else {
        f2_split(fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3])), a0, a1);
        l = l * alpha + (a0 + a1);
      }
      m = m_new;
    }
    if (!C::kPSmem && !ok) {
      // Failure path: the rest of this warpgroup's named-barrier schedule (tiles j..nkv-1)
      // without the work between, so the MMA warp and the other warpgroup are never
      // left waiting on an arrival from here.  Each arrival waits (bounded) until the
      // partner has passed the previous generation of that barrier.
      const uint64_t deadline = globaltimer_ns() + kWaitLimitNs;
      const uint32_t my_mma_done = mma_done + 4 * i;
      for (; j < nkv; ++j) {
        if constexpr (C::kPingPong) {
          if (i == 1) named_sync<kBarTurn + 1, 256>();
          else if (j > 0) named_sync<kBarTurn + 0, 256>();
        }
        if (!warp_wait_flag_ge(my_mma_done, j, deadline)) break;
        if constexpr (C::kSplitP) {
          if (i == 0) named_arrive<kBarPHalf + 0, 160>();
          else named_arrive<kBarPHalf + 1, 160>();
        }
        if constexpr (C::kPingPong) {
          if (i == 0) {
            if (!warp_wait_flag_ge(mma_done + 4, j, deadline)) break;  // warpgroup 1 passed Turn_1(j-1)
            named_arrive<kBarTurn + 1, 256>();
          } else if (j + 1 < nkv) {
            if (!warp_wait_flag_ge(mma_done, j + 1, deadline)) break;  // warpgroup 0 passed Turn_0(j-1)
            named_arrive<kBarTurn + 0, 256>();
          }
        }
        if (i == 0) named_arrive<kBarPReady + 0, 160>();
        else named_arrive<kBarPReady + 1, 160>();
      }
    }
    // ---------------------------------------------------------- epilogue
    // BF16 commits pv_done once, after the last PV; FP8 once per tile
    const uint32_t pv_last = C::kPSmem ? static_cast<uint32_t>((nkv - 1) & 1) : 0u;
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(pv_done + i, pv_last, err, kErrTimeout, abort_flag));
    if (ok) {
      tc_fence_after();
      const float fin = fin_scale / l;
      const int qrow = qblk * BM + row;
      __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(out.o) + b * out.so[0] + h * out.so[1] +
                            static_cast<int64_t>(qrow) * out.so[2];
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
  if (warp == 9) {
    __syncwarp();
    tc_fence_after();
    if (flag_load(abort_flag) != 0) {
      // after a failure nobody waited for the last MMAs: wait (bounded) until every
      // MMA issued has completed, so that TMEM is not released under a running one
      if (lane == 0) mma_commit(mma_drain);
      __syncwarp();
      mbar_wait_until(mma_drain, 0, globaltimer_ns() + kWaitLimitNs);
    }
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <bool FP8, int D, bool I8QK = false>
cudaError_t launch_attn(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const AttnOut& out,
                        const AttnScales& sc, int B, int H, cudaStream_t stream) {
  constexpr int smem = AttnCfg<FP8, D>::kSmemBytes;
  cudaError_t e =
      cudaFuncSetAttribute(attn_kernel<FP8, D, I8QK>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid((out.N + 255) / 256, H, B);
  if constexpr (FP8)  // a programmatic dependent of the FP8 prologue's quantiser (see pdl_wait in the kernel)
    return launch_dependent(attn_kernel<FP8, D, I8QK>, grid, dim3(AttnCfg<FP8, D>::kThreads), smem, stream, tq, tk,
                            tv, out, sc);
  // BF16: a plain launch (as a dependent of the K rotation pass it gained nothing
  // measurable, and CUDA events around the call no longer bracketed its time)
  attn_kernel<FP8, D, I8QK><<<grid, AttnCfg<FP8, D>::kThreads, smem, stream>>>(tq, tk, tv, out, sc);
  return cudaGetLastError();
}

}  // namespace dit
