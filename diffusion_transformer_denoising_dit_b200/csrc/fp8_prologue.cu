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
    // four tokens per step, all loads issued before the adds (tokens in the same
    // order as one at a time)
    for (int n = n0 + tl; n < n1; n += 64) {
      float y[4][8];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int m = n + 16 * u;
        if (m < n1)
          load_rotate8(kb + static_cast<int64_t>(m) * p.sk[2] + cc * 8, p.cos_tab, p.sin_tab, m, cc, p.d / 2, y[u]);
        else
#pragma unroll
          for (int i = 0; i < 8; ++i) y[u][i] = 0.f;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (n + 16 * u < n1) acc[i] += y[u][i];
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

// ---------------------------------------------------------------------------
// Pass 2: the quantiser, a persistent CTA per SM.  Work item = one 128-token
// block of one (b,h): three tiles, Q, V and K, taken in that order; CTA c takes
// items c, c + G, c + 2G, ... (G CTAs), so that the CTAs together stream
// through the heads one after another.  Tiles and the rotary rows they need are
// staged in shared memory by bulk copies issued ahead of use, so the reads
// never wait on registers: three 32 KB tile slots (one per tensor; a slot is
// refilled for the next item as soon as the 16 converting warps release it) and two
// 64 KB table slots (cos and sin rows of 128 tokens, one per item in flight,
// refilled two items ahead).  A producer warp issues the copies as slots are
// released; sixteen warps convert a tile while the copies of the following
// ones are in flight.
//
// Thread t owns channel chunk cc = t % 16 (channels 8cc .. 8cc+7) of tokens
// t/16 + 32 i, i = 0..3, of the tile; for a tile of two 64-token blocks (K, V)
// tokens i = 0, 1 lie in the first block and i = 2, 3 in the second.
constexpr int kQzThreads = 512;              // converting threads
constexpr int kQzBlock = kQzThreads + 32;     // + the producer warp
constexpr int kTileBytes = 128 * 256;      // 128 tokens x 128 bf16 channels
constexpr int kTabBytes = 2 * 128 * 256;   // cos then sin rows (64 fp32 each) of 128 tokens
constexpr int kQzBarOff = 3 * kTileBytes + 2 * kTabBytes;
constexpr int kQzSmem = kQzBarOff + 512;   // + 10 mbarriers, the abort flag, two halves of warp maxima
static_assert(kQzSmem <= 227 * 1024, "the quantiser's staging exceeds a CTA's shared memory");

enum QzKind { kQzQ = 0, kQzK = 1, kQzV = 2 };

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// One warp, all lanes: stage tokens [n0, n0 + rows) of one (b,h) slab of a bf16
// tensor (token stride ts elements; a token's 128 channels contiguous and
// 16-byte aligned) into a tile slot, 256 bytes per token.
// (Debug builds: a copy whose size or alignment fails its check is not issued;
// its bytes never arrive, so the slot's wait times out after recording the error.)
__device__ __forceinline__ void stage_tile(uint8_t* slot, uint64_t* bar, const __nv_bfloat16* slab, int64_t ts,
                                           int n0, int rows, int* err) {
  const int lane = threadIdx.x & 31;
  if (lane == 0) mbar_arrive_expect_tx(bar, static_cast<uint32_t>(rows) * 256u);
  __syncwarp();
  if (ts == 128) {
    const __nv_bfloat16* src = slab + static_cast<int64_t>(n0) * 128;
    if (lane == 0 && debug_check(rows >= 1 && rows <= 128 && (reinterpret_cast<uintptr_t>(src) & 15) == 0, err))
      bulk_g2s(slot, src, static_cast<uint32_t>(rows) * 256u, bar);
  } else {
    for (int r = lane; r < rows; r += 32) {
      const __nv_bfloat16* src = slab + static_cast<int64_t>(n0 + r) * ts;
      if (debug_check(r < 128 && (reinterpret_cast<uintptr_t>(src) & 15) == 0, err))
        bulk_g2s(slot + r * 256, src, 256u, bar);
    }
  }
}

// One warp: stage the cos and sin rows of tokens [n0, n0 + rows) into a table slot.
__device__ __forceinline__ void stage_tables(uint8_t* slot, uint64_t* bar, const float* cos_tab, const float* sin_tab,
                                             int n0, int rows, int* err) {
  if ((threadIdx.x & 31) == 0) {
    const uint32_t bytes = static_cast<uint32_t>(rows) * 256u;
    mbar_arrive_expect_tx(bar, 2u * bytes);
    const float* c = cos_tab + static_cast<int64_t>(n0) * 64;
    const float* s = sin_tab + static_cast<int64_t>(n0) * 64;
    const uintptr_t a = reinterpret_cast<uintptr_t>(c) | reinterpret_cast<uintptr_t>(s);
    if (debug_check(rows >= 1 && rows <= 128 && (a & 15) == 0, err)) {
      bulk_g2s(slot, c, bytes, bar);
      bulk_g2s(slot + kTabBytes / 2, s, bytes, bar);
    }
  }
  __syncwarp();
}

// Named barrier 1 over the 16 converting warps (the producer warp is not in it),
// returning whether any of them passed true.
__device__ __forceinline__ bool converters_sync_or(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, 512, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v))
      : "memory");
  return r != 0;
}

struct QzItem {
  int bh, blk, n0, rows;
};

// item = bh * nq + blk
__device__ __forceinline__ QzItem qz_item(const Fp8Prep& p, int item, int nq) {
  QzItem r;
  r.bh = item / nq;
  r.blk = item - r.bh * nq;
  r.n0 = r.blk * 128;
  r.rows = min(128, p.N - r.n0);
  return r;
}

__device__ __forceinline__ const __nv_bfloat16* qz_slab(const Fp8Prep& p, int kind, int bh) {
  const int b = bh / p.H, h = bh - b * p.H;
  const void* base = kind == kQzQ ? p.q : kind == kQzK ? p.k : p.v;
  const int64_t* s = kind == kQzQ ? p.sq : kind == kQzK ? p.sk : p.sv;
  return static_cast<const __nv_bfloat16*>(base) + b * s[0] + h * s[1];
}

__device__ __forceinline__ int64_t qz_stride(const Fp8Prep& p, int kind) {
  return kind == kQzQ ? p.sq[2] : kind == kQzK ? p.sk[2] : p.sv[2];
}

// One tile: read the staged rows, rotate (Q, K), subtract the K mean, block
// maxima, then scale, cast and store.  Returns false when a staged copy did not
// arrive in time or the producer gave up (uniform over the converting warps).
// Each warp releases the tile slot (and, for K, the table slot: K is the last
// reader of an item's rows) with one arrival as soon as its reads are done.
// red: this tile's half of the double-buffered warp maxima (two consecutive
// tiles never share a half, so one barrier per tile suffices).
//
// A token's eight channels are held as four fp32 pairs (sm_100 f32x2
// arithmetic): ev[q] = channels (4q, 4q + 2), od[q] = (4q + 1, 4q + 3), so that
// the rotary pairs (2j, 2j + 1), j = 2q, 2q + 1, sit in matching lanes of ev and
// od, and the tables' cos and sin (j, j + 1) load as one pair each.
template <int KIND, bool INT8>
__device__ __forceinline__ bool qz_tile(const Fp8Prep& p, const QzItem& it, const uint8_t* tile, uint64_t* tile_bar,
                                        uint64_t* tile_empty, uint32_t tile_par, const uint8_t* tab,
                                        uint64_t* tab_bar, uint64_t* tab_empty, uint32_t tab_par, float* red,
                                        uint32_t abort_flag) {
  const int cc = threadIdx.x & 15, tl = threadIdx.x >> 4;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool rot = KIND != kQzV && p.cos_tab != nullptr;
  uint64_t nmean[4];  // K: minus the channel means, in the ev / od lane order
  if (KIND == kQzK) {
    const float4 m0 = *reinterpret_cast<const float4*>(p.k_mean + it.bh * 128 + cc * 8);
    const float4 m1 = *reinterpret_cast<const float4*>(p.k_mean + it.bh * 128 + cc * 8 + 4);
    nmean[0] = f2(-m0.x, -m0.z);
    nmean[1] = f2(-m0.y, -m0.w);
    nmean[2] = f2(-m1.x, -m1.z);
    nmean[3] = f2(-m1.y, -m1.w);
  }
  bool ok = mbar_wait(tile_bar, tile_par, p.err, kErrTimeout, abort_flag);
  if (rot) ok = ok && mbar_wait(tab_bar, tab_par, p.err, kErrTimeout, abort_flag);
  const uint64_t minus1 = f2(-1.f, -1.f);
  uint64_t ev[4][2], od[4][2];
  float a0 = 0.f, a1 = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int t = tl + 32 * i;
    if (ok && t < it.rows && debug_check(t < 128, p.err)) {
      const uint4 raw = *reinterpret_cast<const uint4*>(tile + t * 256 + cc * 16);
      const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};  // bf16 pairs, low half = even channel
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        ev[i][q] = f2(__uint_as_float(w[2 * q] << 16), __uint_as_float(w[2 * q + 1] << 16));
        od[i][q] = f2(__uint_as_float(w[2 * q] & 0xffff0000u), __uint_as_float(w[2 * q + 1] & 0xffff0000u));
      }
      if (rot) {
        const uint4 c = *reinterpret_cast<const uint4*>(tab + t * 256 + cc * 16);
        const uint4 s = *reinterpret_cast<const uint4*>(tab + kTabBytes / 2 + t * 256 + cc * 16);
        const uint64_t c2[2] = {f2(__uint_as_float(c.x), __uint_as_float(c.y)),
                                f2(__uint_as_float(c.z), __uint_as_float(c.w))};
        const uint64_t s2[2] = {f2(__uint_as_float(s.x), __uint_as_float(s.y)),
                                f2(__uint_as_float(s.z), __uint_as_float(s.w))};
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          // (x_e, x_o) -> (x_e c - x_o s, x_e s + x_o c)
          const uint64_t e = ev[i][q], o = od[i][q];
          ev[i][q] = ffma2(o, fmul2(s2[q], minus1), fmul2(e, c2[q]));
          od[i][q] = ffma2(o, c2[q], fmul2(e, s2[q]));
        }
      }
      if (KIND == kQzK) {
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          ev[i][q] = fadd2(ev[i][q], nmean[2 * q]);
          od[i][q] = fadd2(od[i][q], nmean[2 * q + 1]);
        }
      }
    } else {
#pragma unroll
      for (int q = 0; q < 2; ++q) ev[i][q] = od[i][q] = 0ull;
    }
    float m = 0.f;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      float e0, e1, o0, o1;
      f2_split(ev[i][q], e0, e1);
      f2_split(od[i][q], o0, o1);
      m = fmax3(m, fabsf(e0), fabsf(e1));
      m = fmax3(m, fabsf(o0), fabsf(o1));
    }
    if (KIND == kQzQ || i < 2)
      a0 = fmaxf(a0, m);
    else
      a1 = fmaxf(a1, m);
  }
  __syncwarp();  // the warp's reads of the slots are done
  if (lane == 0) {
    mbar_arrive(tile_empty);
    if (KIND == kQzK && rot) mbar_arrive(tab_empty);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    a0 = fmaxf(a0, __shfl_xor_sync(0xffffffffu, a0, o));
    if (KIND != kQzQ) a1 = fmaxf(a1, __shfl_xor_sync(0xffffffffu, a1, o));
  }
  if (lane == 0) {
    red[warp] = a0;
    red[16 + warp] = a1;
  }
  // every warp's maxima are in red
  if (converters_sync_or(!ok)) return false;
  float m = red[lane];  // lanes 0-15: first block, 16-31: second
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  const float b0 = __shfl_sync(0xffffffffu, m, 0), b1 = __shfl_sync(0xffffffffu, m, 16);
  const float qmax = (INT8 && KIND != kQzV) ? 127.f : 448.f;
  const float inv0 = b0 > 0.f ? qmax / b0 : 1.f;
  const float inv1 = (KIND != kQzQ && b1 > 0.f) ? qmax / b1 : 1.f;
  if (threadIdx.x == 0) {
    const float s0 = b0 > 0.f ? b0 / qmax : 1.f, s1 = b1 > 0.f ? b1 / qmax : 1.f;
    const int nq = (p.N + 127) / 128, nk = (p.N + 63) / 64;
    if (KIND == kQzQ) {
      p.q_scale[it.bh * nq + it.blk] = s0;
    } else {
      float* sc = (KIND == kQzK ? p.k_scale : p.v_scale) + it.bh * nk + 2 * it.blk;
      sc[0] = s0;
      const bool second = 2 * it.blk + 1 < nk;  // a second 64-token block inside the sequence
      if (second) sc[1] = s1;
      if (KIND == kQzV) {
        atomicMax(reinterpret_cast<int*>(p.v_scale_max + it.bh), __float_as_int(s0));
        if (second) atomicMax(reinterpret_cast<int*>(p.v_scale_max + it.bh), __float_as_int(s1));
      }
    }
  }
  uint8_t* dst = (KIND == kQzQ ? p.q8 : KIND == kQzK ? p.k8 : p.v8) + static_cast<int64_t>(it.bh) * p.N * 128;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int t = tl + 32 * i;
    if (t >= it.rows) continue;
    const float inv = (KIND == kQzQ || i < 2) ? inv0 : inv1;
    uint32_t wd[2];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      float e0, e1, o0, o1;  // channels 4q, 4q + 2 and 4q + 1, 4q + 3
      if (INT8 && KIND != kQzV) {
        // int8 codes: fma(x, inv, 1.5 * 2^23) rounds x * inv (within [-127, 127]) once
        // to the nearest integer, ties to even (the float's unit in the last place is 1
        // there), and the float's low byte is then that integer modulo 256, i.e. its
        // two's complement byte; byte permutes gather the four low bytes in channel order.
        const uint64_t bias = f2(12582912.0f, 12582912.0f), inv2 = f2(inv, inv);
        f2_split(ffma2(ev[i][q], inv2, bias), e0, e1);
        f2_split(ffma2(od[i][q], inv2, bias), o0, o1);
        const uint32_t lo = __byte_perm(__float_as_uint(e0), __float_as_uint(o0), 0x0040);
        const uint32_t hi = __byte_perm(__float_as_uint(e1), __float_as_uint(o1), 0x0040);
        wd[q] = __byte_perm(lo, hi, 0x5410);
      } else {
        const uint64_t inv2 = f2(inv, inv);
        f2_split(fmul2(ev[i][q], inv2), e0, e1);
        f2_split(fmul2(od[i][q], inv2), o0, o1);
        wd[q] = cvt_e4m3x2(e0, o0) | (cvt_e4m3x2(e1, o1) << 16);
      }
    }
    *reinterpret_cast<uint2*>(dst + static_cast<int64_t>(it.n0 + t) * 128 + cc * 8) = make_uint2(wd[0], wd[1]);
  }
  return true;
}

// INT8: Q and K as symmetric int8 (the integer Q.K^T form), V as e4m3.
template <bool INT8>
__global__ void __launch_bounds__(kQzBlock, 1) quantize_qkv(Fp8Prep p) {
  extern __shared__ __align__(128) uint8_t qz_smem[];
  uint8_t* tiles = qz_smem;                   // [3][kTileBytes]: slot = tensor (Q, K, V)
  uint8_t* tabs = qz_smem + 3 * kTileBytes;  // [2][kTabBytes]
  uint64_t* bars = reinterpret_cast<uint64_t*>(qz_smem + kQzBarOff);
  uint64_t* tile_full = bars;       // [3] one arrival (the producer's) + the copy's bytes
  uint64_t* tab_full = bars + 3;    // [2]
  uint64_t* tile_empty = bars + 5;  // [3] one arrival per converting warp
  uint64_t* tab_empty = bars + 8;   // [2]
  int* abort_flag = reinterpret_cast<int*>(bars + 10);
  float* red = reinterpret_cast<float*>(qz_smem + kQzBarOff + 128);  // [2][32] warp maxima
  // The attention kernel may be scheduled; it waits for this grid to complete.
  pdl_trigger();
  const int nq = (p.N + 127) / 128;
  const int items = p.B * p.H * nq;
  const int stride = gridDim.x;
  const bool rope = p.cos_tab != nullptr;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 5; ++i) mbar_init(&bars[i], 1);
    for (int i = 5; i < 10; ++i) mbar_init(&bars[i], kQzThreads / 32);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const uint32_t abort_a = smem_u32(abort_flag);
  if (threadIdx.x >= kQzThreads) {
    // Producer warp: stages item n's rows (into table slot n % 2) and its Q, V and K
    // tiles as soon as the slots' previous contents are released.
    uint32_t staged = 0, last = 0;  // per full barrier (bit b): staged at all; parity of the last phase
    bool ok = true;
    int n = 0;
    for (int item = blockIdx.x; item < items && ok; item += stride, ++n) {
      const QzItem it = qz_item(p, item, nq);
      if (rope) {
        const int ts = n & 1;
        if (n >= 2) ok = mbar_wait(&tab_empty[ts], static_cast<uint32_t>((n - 2) >> 1) & 1u, p.err, kErrTimeout,
                                   abort_a);
        if (!ok) break;
        stage_tables(tabs + ts * kTabBytes, &tab_full[ts], p.cos_tab, p.sin_tab, it.n0, it.rows, p.err);
        staged |= 1u << (3 + ts);
        last = (last & ~(1u << (3 + ts))) | ((static_cast<uint32_t>(n >> 1) & 1u) << (3 + ts));
      }
#pragma unroll
      for (int j = 0; j < 3 && ok; ++j) {
        const int kind = j == 0 ? kQzQ : j == 1 ? kQzV : kQzK;
        if (n >= 1) ok = mbar_wait(&tile_empty[kind], static_cast<uint32_t>(n - 1) & 1u, p.err, kErrTimeout, abort_a);
        if (!ok) break;
        stage_tile(tiles + kind * kTileBytes, &tile_full[kind], qz_slab(p, kind, it.bh), qz_stride(p, kind), it.n0,
                   it.rows, p.err);
        staged |= 1u << kind;
        last = (last & ~(1u << kind)) | ((static_cast<uint32_t>(n) & 1u) << kind);
      }
    }
    if ((threadIdx.x & 31) == 0) {
      // Wait, bounded, for every copy staged before the CTA's shared memory is
      // released.  Needed on every exit, not only after a failed wait of this warp:
      // the converting warps release their slots on their failure path too, which
      // can let the last stagings through after they have stopped.  On the normal
      // path the copies have landed or are about to (the converting warps wait for them).
      const uint64_t deadline = globaltimer_ns() + kWaitLimitNs;
#pragma unroll
      for (int b = 0; b < 5; ++b)
        if ((staged >> b) & 1u) mbar_wait_until(&bars[b], (last >> b) & 1u, deadline);
    }
    return;
  }
  int n = 0;
  for (int item = blockIdx.x; item < items; item += stride, ++n) {
    const QzItem it = qz_item(p, item, nq);
    const int ts = n & 1;
    const uint32_t tpar = static_cast<uint32_t>(n) & 1u, bpar = static_cast<uint32_t>(n >> 1) & 1u;
    // warp-maxima halves alternate tile by tile (Q, V, K, Q, ...: 3n, 3n + 1, 3n + 2)
    float* red_a = red + 32 * (n & 1);
    float* red_b = red + 32 * ((n + 1) & 1);
    uint8_t* tab = tabs + ts * kTabBytes;
    // Q: reads only the inputs, written before the K-mean pass began.
    bool ok = qz_tile<kQzQ, INT8>(p, it, tiles + kQzQ * kTileBytes, &tile_full[kQzQ], &tile_empty[kQzQ], tpar, tab,
                                  &tab_full[ts], &tab_empty[ts], bpar, red_a, abort_a);
    // V needs the cleared per-(b,h) scale maximum and K the channel means: both
    // from the grids this one depends on.
    if (ok && n == 0) pdl_wait();
    ok = ok && qz_tile<kQzV, INT8>(p, it, tiles + kQzV * kTileBytes, &tile_full[kQzV], &tile_empty[kQzV], tpar,
                                   nullptr, nullptr, nullptr, 0u, red_b, abort_a);
    ok = ok && qz_tile<kQzK, INT8>(p, it, tiles + kQzK * kTileBytes, &tile_full[kQzK], &tile_empty[kQzK], tpar, tab,
                                   &tab_full[ts], &tab_empty[ts], bpar, red_a, abort_a);
    if (!ok) {
      if (threadIdx.x == 0) flag_store(abort_a, 1);  // the producer stops and drains its copies
      break;
    }
  }
}

}  // namespace

cudaError_t launch_fp8_prologue(const Fp8Prep& p, cudaStream_t stream) {
  // every check before the first launch, so that an error return leaves nothing enqueued
  const int64_t items = static_cast<int64_t>(p.B) * p.H * ((p.N + 127) / 128);
  if (items > 0x7fffffff || p.num_sms < 1) return cudaErrorInvalidValue;
  const int grid = static_cast<int>(items < p.num_sms ? items : p.num_sms);  // persistent: one CTA per SM
  auto kern = p.qk_int8 ? quantize_qkv<true> : quantize_qkv<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kQzSmem);
  if (e != cudaSuccess) return e;
  float* partial = p.k_partial;
  dim3 g1(kChunks, p.B * p.H);
  kmean_partial<<<g1, kThreads, 0, stream>>>(p, partial);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = launch_dependent(kmean_finalize, dim3(p.B * p.H), dim3(128), 0, stream, p, static_cast<const float*>(partial));
  if (e != cudaSuccess) return e;
  return launch_dependent(kern, dim3(grid), dim3(kQzBlock), kQzSmem, stream, p);
}

}  // namespace dit
