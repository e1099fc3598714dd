// C ABI of the DiT joint-attention hot path (declared in include/dit.h):
// argument validation, TMA tensor-map construction, workspace carving and
// kernel launches on the caller's stream.  No allocation, no synchronisation
// (except dit_read_error), no fallback path.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>

#include <nvtx3/nvToolsExt.h>

#include "dit.h"
#include "dit_internal.h"

namespace {

// One NVTX range per call, named after the entry point, around its host work and
// launches: Nsight tools show it, and `ncu --nvtx --nvtx-include "<name>/"`
// captures one call's kernels.  Without a tool attached a push and a pop cost a
// few nanoseconds (NVTX v3, header only: a tool is loaded at the first call
// from NVTX_INJECTION64_PATH, if set).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

__device__ int g_dit_error_word;

constexpr int kMaxDevices = 64;

struct DeviceState {
  bool probed = false;
  bool sm100 = false;
  int sms = 0;         // multiprocessor count
  int* err = nullptr;  // device address of g_dit_error_word
};

std::mutex g_mu;
DeviceState g_dev[kMaxDevices];
std::atomic<PFN_cuTensorMapEncodeTiled_v12000> g_encode{nullptr};  // set once, read by make_map

// Per-device set-up on first use: architecture check and the error word's address.
const DeviceState* device_state() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceState& s = g_dev[dev];
  if (!s.probed) {
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    s.sm100 = (major == 10 && minor == 0);
    cudaDeviceGetAttribute(&s.sms, cudaDevAttrMultiProcessorCount, dev);
    if (s.sms < 1) s.sm100 = false;
    void* p = nullptr;
    if (s.sm100 && cudaGetSymbolAddress(&p, g_dit_error_word) == cudaSuccess) s.err = static_cast<int*>(p);
    if (!s.err) s.sm100 = false;
    s.probed = true;
  }
  if (!g_encode.load()) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode.store(reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn));
  }
  return &s;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// Element strides must keep every row 16-byte aligned for TMA / vector access.
bool strides_ok(const int64_t s[3], int elem_bytes) {
  for (int i = 0; i < 3; ++i)
    if (s[i] < 0 || (s[i] * elem_bytes) % 16 != 0) return false;
  return true;
}

// Every dimension of extent > 1 advances (a positive stride: neither TMA nor the
// kernels broadcast), and token rows do not overlap (token stride >= d).
bool layout_ok(const int64_t s[3], int B, int H, int N, int d) {
  return !(B > 1 && s[0] <= 0) && !(H > 1 && s[1] <= 0) && !(N > 1 && s[2] < d);
}

// 4-D tiled tensor map over [B][H][N][d] with the given element strides;
// box = {box_inner elements, box_rows tokens, 1, 1}, 128-byte swizzle.
bool make_map(CUtensorMap* map, CUtensorMapDataType dt, int elem_bytes, const void* base, int B, int H, int N, int d,
              const int64_t s[3], int box_inner, int box_rows) {
  const PFN_cuTensorMapEncodeTiled_v12000 encode = g_encode.load();
  if (!encode) return false;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(H),
                        static_cast<cuuint64_t>(B)};
  // A size-1 dimension never advances; give it a harmless legal stride.
  const int64_t tok = s[2] > 0 ? s[2] : d;
  const int64_t hs = (H == 1 || s[1] == 0) ? tok * N : s[1];
  const int64_t bs = (B == 1 || s[0] == 0) ? hs * H : s[0];
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(tok * elem_bytes), static_cast<cuuint64_t>(hs * elem_bytes),
                           static_cast<cuuint64_t>(bs * elem_bytes)};
  cuuint32_t box[4] = {static_cast<cuuint32_t>(box_inner), static_cast<cuuint32_t>(box_rows), 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = encode(map, dt, 4, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

dit_status launch_status(cudaError_t e) { return e == cudaSuccess ? DIT_OK : DIT_ERR_LAUNCH; }

bool valid_rope_tables(const float* c, const float* s) {
  if ((c == nullptr) != (s == nullptr)) return false;
  return c == nullptr || (aligned16(c) && aligned16(s));
}

}  // namespace

extern "C" {

const char* dit_status_string(dit_status s) {
  switch (s) {
    case DIT_OK: return "DIT_OK";
    case DIT_ERR_INVALID_ARG: return "DIT_ERR_INVALID_ARG";
    case DIT_ERR_UNSUPPORTED: return "DIT_ERR_UNSUPPORTED";
    case DIT_ERR_ALIGNMENT: return "DIT_ERR_ALIGNMENT";
    case DIT_ERR_WORKSPACE: return "DIT_ERR_WORKSPACE";
    case DIT_ERR_LAUNCH: return "DIT_ERR_LAUNCH";
    case DIT_ERR_TIMEOUT: return "DIT_ERR_TIMEOUT";
    case DIT_ERR_BOUNDS: return "DIT_ERR_BOUNDS";
  }
  return "DIT_ERR_UNKNOWN";
}

dit_status dit_read_error(dit_stream_t stream) {
  const NvtxRange nvtx_range("dit_read_error");
  const DeviceState* ds = device_state();
  if (!ds || !ds->sm100) return DIT_ERR_UNSUPPORTED;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return DIT_ERR_LAUNCH;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_dit_error_word, sizeof(int)) != cudaSuccess) return DIT_ERR_LAUNCH;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_dit_error_word, &zero, sizeof(int)) != cudaSuccess) return DIT_ERR_LAUNCH;
  return static_cast<dit_status>(v);
}

dit_status dit_selftest_wait_timeout(dit_stream_t stream) {
  const NvtxRange nvtx_range("dit_selftest_wait_timeout");
  const DeviceState* ds = device_state();
  if (!ds || !ds->sm100 || !ds->err) return DIT_ERR_UNSUPPORTED;
  return launch_status(dit::launch_selftest_wait(ds->err, reinterpret_cast<cudaStream_t>(stream)));
}

dit_status dit_rope_tables(const int32_t* pos, int N, int d0, int d1, int d2, double theta, float* cos_out,
                           float* sin_out, dit_stream_t stream) {
  const NvtxRange nvtx_range("dit_rope_tables");
  if (!pos || !cos_out || !sin_out || N < 1) return DIT_ERR_INVALID_ARG;
  if (d0 < 0 || d1 < 0 || d2 < 0 || (d0 | d1 | d2) & 1 || d0 + d1 + d2 < 2 || d0 + d1 + d2 > 256)
    return DIT_ERR_INVALID_ARG;
  if (!(theta > 0.0) || !std::isfinite(theta)) return DIT_ERR_INVALID_ARG;
  if (!aligned4(pos) || !aligned4(cos_out) || !aligned4(sin_out)) return DIT_ERR_ALIGNMENT;
  const DeviceState* ds = device_state();
  if (!ds || !ds->sm100) return DIT_ERR_UNSUPPORTED;
  return launch_status(dit::launch_rope_tables(pos, N, d0, d1, d2, theta, cos_out, sin_out,
                                               reinterpret_cast<cudaStream_t>(stream)));
}

dit_status rope_apply(const void* x, void* y, int B, int H, int N, int d, const int64_t sx[3], const int64_t sy[3],
                      const float* cos_tab, const float* sin_tab, int dtype, dit_stream_t stream) {
  const NvtxRange nvtx_range("rope_apply");
  if (!x || !y || !sx || !sy || !cos_tab || !sin_tab) return DIT_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || N < 1 || (dtype != 0 && dtype != 1)) return DIT_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return DIT_ERR_UNSUPPORTED;
  if (dtype == 1 && x == y) return DIT_ERR_INVALID_ARG;  // fp32 output cannot overwrite bf16 input
  if (!aligned16(x) || !aligned16(y) || !strides_ok(sx, 2) || !strides_ok(sy, dtype ? 4 : 2) ||
      !valid_rope_tables(cos_tab, sin_tab))
    return DIT_ERR_ALIGNMENT;
  if (!layout_ok(sx, B, H, N, d) || !layout_ok(sy, B, H, N, d)) return DIT_ERR_INVALID_ARG;
  if (x == y && (sx[0] != sy[0] || sx[1] != sy[1] || sx[2] != sy[2])) return DIT_ERR_INVALID_ARG;  // in place
  const DeviceState* ds = device_state();
  if (!ds || !ds->sm100) return DIT_ERR_UNSUPPORTED;
  dit::RopeJob job;
  job.x = x;
  job.y = y;
  for (int i = 0; i < 3; ++i) {
    job.sx[i] = sx[i];
    job.sy[i] = sy[i];
  }
  return launch_status(dit::launch_rope_apply(&job, 1, B, H, N, d, cos_tab, sin_tab, dtype,
                                              reinterpret_cast<cudaStream_t>(stream)));
}

size_t dit_attn_bf16_workspace_bytes(int B, int H, int N, int d, int has_rope) {
  if (!has_rope || B < 1 || H < 1 || N < 1 || d < 1) return 0;
  return align256(static_cast<size_t>(B) * H * N * d * 2);  // rotated K
}

namespace {

dit_status attn_bf16_impl(const void* q, const void* k, const void* v, void* o, int B, int H, int N, int d,
                          const int64_t sq[3], const int64_t sk[3], const int64_t sv[3], const int64_t so[3],
                          const float* rope_cos, const float* rope_sin, float softmax_scale, void* workspace,
                          size_t workspace_bytes, const int32_t* skip, dit_stream_t stream) {
  if (!q || !k || !v || !o || !sq || !sk || !sv || !so) return DIT_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || N < 1 || B > 65535 || H > 65535) return DIT_ERR_INVALID_ARG;
  if (!std::isfinite(softmax_scale)) return DIT_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return DIT_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !strides_ok(sq, 2) || !strides_ok(sk, 2) ||
      !strides_ok(sv, 2) || !strides_ok(so, 2) || !valid_rope_tables(rope_cos, rope_sin))
    return DIT_ERR_ALIGNMENT;
  if (!layout_ok(sq, B, H, N, d) || !layout_ok(sk, B, H, N, d) || !layout_ok(sv, B, H, N, d) ||
      !layout_ok(so, B, H, N, d) || o == q || o == k || o == v)
    return DIT_ERR_INVALID_ARG;
  const bool rope = rope_cos != nullptr;
  const size_t need = dit_attn_bf16_workspace_bytes(B, H, N, d, rope);
  if (need > 0 && (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u)))
    return DIT_ERR_WORKSPACE;
  const DeviceState* ds = device_state();
  if (!ds || !ds->sm100 || !g_encode.load()) return DIT_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);

  // K is rotated once per head into the workspace (every CTA of the head reads
  // each K tile); Q is rotated by the attention kernel as it loads each Q tile.
  const int64_t cs[3] = {static_cast<int64_t>(H) * N * d, static_cast<int64_t>(N) * d, d};
  const void* ka = rope ? workspace : k;
  const int64_t* ska = rope ? cs : sk;
  // Every map is built before the first launch, so an error return leaves nothing enqueued.
  CUtensorMap tq, tk, tv;
  // Q tiles are 128 tokens, K/V tiles kAttnBlockN tokens; boxes are 128 bytes wide.
  if (!make_map(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, q, B, H, N, d, sq, 64, 128) ||
      !make_map(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ka, B, H, N, d, ska, 64, dit::kAttnBlockN) ||
      !make_map(&tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, v, B, H, N, d, sv, 64, dit::kAttnBlockN))
    return DIT_ERR_ALIGNMENT;
  if (rope) {
    dit::RopeJob job;
    job.x = k;
    job.y = workspace;
    for (int i = 0; i < 3; ++i) {
      job.sx[i] = sk[i];
      job.sy[i] = cs[i];
    }
    cudaError_t e = dit::launch_rope_apply(&job, 1, B, H, N, d, rope_cos, rope_sin, 0, st, skip);
    if (e != cudaSuccess) return DIT_ERR_LAUNCH;
  }
  dit::AttnOut out{};  // value-initialised: every pointer not set below is null
  out.o = o;
  for (int i = 0; i < 3; ++i) out.so[i] = so[i];
  out.N = N;
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt(static_cast<float>(d));
  out.scale_log2 = scale * 1.4426950408889634f;
  out.err = ds->err;
  out.rope_cos = rope_cos;
  out.rope_sin = rope_sin;
  out.skip = skip;
  return launch_status(dit::launch_attn_bf16(tq, tk, tv, out, B, H, d, st));
}

}  // namespace

dit_status dit_attn_bf16(const void* q, const void* k, const void* v, void* o, int B, int H, int N, int d,
                         const int64_t sq[3], const int64_t sk[3], const int64_t sv[3], const int64_t so[3],
                         const float* rope_cos, const float* rope_sin, float softmax_scale, void* workspace,
                         size_t workspace_bytes, dit_stream_t stream) {
  const NvtxRange nvtx_range("dit_attn_bf16");
  return attn_bf16_impl(q, k, v, o, B, H, N, d, sq, sk, sv, so, rope_cos, rope_sin, softmax_scale, workspace,
                        workspace_bytes, nullptr, stream);
}

dit_status dit_attn_bf16_skippable(const void* q, const void* k, const void* v, void* o, int B, int H, int N, int d,
                                   const int64_t sq[3], const int64_t sk[3], const int64_t sv[3],
                                   const int64_t so[3], const float* rope_cos, const float* rope_sin,
                                   float softmax_scale, void* workspace, size_t workspace_bytes,
                                   const int32_t* skip, dit_stream_t stream) {
  const NvtxRange nvtx_range("dit_attn_bf16_skippable");
  if (!skip) return DIT_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(skip) & 3u) return DIT_ERR_ALIGNMENT;
  return attn_bf16_impl(q, k, v, o, B, H, N, d, sq, sk, sv, so, rope_cos, rope_sin, softmax_scale, workspace,
                        workspace_bytes, skip, stream);
}

size_t dit_attn_fp8_workspace_bytes(int B, int H, int N, int d, int q_block, int kv_block) {
  if (B < 1 || H < 1 || N < 1 || d < 1 || q_block < 1 || kv_block < 1) return 0;
  const size_t bh = static_cast<size_t>(B) * H;
  const size_t el = bh * N * d;
  const size_t nq = (N + q_block - 1) / q_block, nk = (N + kv_block - 1) / kv_block;
  return 3 * align256(el) + align256(bh * nq * 4) + 2 * align256(bh * nk * 4) + align256(bh * d * 4) +
         align256(bh * 4) + align256(bh * dit::kFp8MeanChunks * d * 4);
}

}  // extern "C"

namespace {

dit_status attn_fp8_impl(const void* q, const void* k, const void* v, void* o, int B, int H, int N, int d,
                         const int64_t sq[3], const int64_t sk[3], const int64_t sv[3], const int64_t so[3],
                         const float* rope_cos, const float* rope_sin, float softmax_scale, int q_block, int kv_block,
                         int smooth_k, void* workspace, size_t workspace_bytes, int qk_int8, dit_stream_t stream) {
  if (!q || !k || !v || !o || !sq || !sk || !sv || !so) return DIT_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || N < 1 || B > 65535 || H > 65535) return DIT_ERR_INVALID_ARG;
  if (!std::isfinite(softmax_scale)) return DIT_ERR_INVALID_ARG;
  if (d != 128 || q_block != 128 || kv_block != 64) return DIT_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(B) * H > 65535) return DIT_ERR_UNSUPPORTED;  // the prologue's grid.y is B*H
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !strides_ok(sq, 2) || !strides_ok(sk, 2) ||
      !strides_ok(sv, 2) || !strides_ok(so, 2) || !valid_rope_tables(rope_cos, rope_sin))
    return DIT_ERR_ALIGNMENT;
  if (!layout_ok(sq, B, H, N, d) || !layout_ok(sk, B, H, N, d) || !layout_ok(sv, B, H, N, d) ||
      !layout_ok(so, B, H, N, d) || o == q || o == k || o == v)
    return DIT_ERR_INVALID_ARG;
  const size_t need = dit_attn_fp8_workspace_bytes(B, H, N, d, q_block, kv_block);
  if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return DIT_ERR_WORKSPACE;
  const DeviceState* ds = device_state();
  if (!ds || !ds->sm100 || !g_encode.load()) return DIT_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);

  dit::Fp8Prep p;
  p.q = q; p.k = k; p.v = v;
  for (int i = 0; i < 3; ++i) {
    p.sq[i] = sq[i]; p.sk[i] = sk[i]; p.sv[i] = sv[i];
  }
  p.cos_tab = rope_cos; p.sin_tab = rope_sin;
  p.B = B; p.H = H; p.N = N; p.d = d; p.q_block = q_block; p.kv_block = kv_block; p.smooth_k = smooth_k != 0;
  p.qk_int8 = qk_int8;
  const size_t bh = static_cast<size_t>(B) * H;
  const size_t el = bh * N * d;
  const size_t nq = (N + q_block - 1) / q_block, nk = (N + kv_block - 1) / kv_block;
  uint8_t* w = static_cast<uint8_t*>(workspace);
  p.q8 = w; w += align256(el);
  p.k8 = w; w += align256(el);
  p.v8 = w; w += align256(el);
  p.q_scale = reinterpret_cast<float*>(w); w += align256(bh * nq * 4);
  p.k_scale = reinterpret_cast<float*>(w); w += align256(bh * nk * 4);
  p.v_scale = reinterpret_cast<float*>(w); w += align256(bh * nk * 4);
  p.k_mean = reinterpret_cast<float*>(w); w += align256(bh * d * 4);
  p.v_scale_max = reinterpret_cast<float*>(w); w += align256(bh * 4);
  p.k_partial = reinterpret_cast<float*>(w);
  p.err = ds->err;
  p.num_sms = ds->sms;

  const int64_t cs[3] = {static_cast<int64_t>(H) * N * d, static_cast<int64_t>(N) * d, d};
  // Every map is built before the first launch, so an error return leaves nothing enqueued.
  CUtensorMap tq, tk, tv;
  // 8-bit codes (e4m3, or int8 for Q and K): one 128-byte row holds all d = 128 channels of a token.
  if (!make_map(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, p.q8, B, H, N, d, cs, 128, 128) ||
      !make_map(&tk, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, p.k8, B, H, N, d, cs, 128, dit::kAttnBlockN) ||
      !make_map(&tv, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, p.v8, B, H, N, d, cs, 128, dit::kAttnBlockN))
    return DIT_ERR_ALIGNMENT;
  if (dit::launch_fp8_prologue(p, st) != cudaSuccess) return DIT_ERR_LAUNCH;
  dit::AttnOut out{};  // value-initialised: every pointer not set below is null
  out.o = o;
  for (int i = 0; i < 3; ++i) out.so[i] = so[i];
  out.N = N;
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt(static_cast<float>(d));
  out.scale_log2 = scale * 1.4426950408889634f;
  out.err = ds->err;
  out.rope_cos = nullptr;  // Q arrives rotated and quantised from the prologue
  out.rope_sin = nullptr;
  return launch_status(dit::launch_attn_fp8(tq, tk, tv, out, p, st));
}

}  // namespace

extern "C" {

dit_status dit_attn_fp8(const void* q, const void* k, const void* v, void* o, int B, int H, int N, int d,
                        const int64_t sq[3], const int64_t sk[3], const int64_t sv[3], const int64_t so[3],
                        const float* rope_cos, const float* rope_sin, float softmax_scale, int q_block, int kv_block,
                        int smooth_k, void* workspace, size_t workspace_bytes, dit_stream_t stream) {
  const NvtxRange nvtx_range("dit_attn_fp8");
  return attn_fp8_impl(q, k, v, o, B, H, N, d, sq, sk, sv, so, rope_cos, rope_sin, softmax_scale, q_block, kv_block,
                       smooth_k, workspace, workspace_bytes, 0, stream);
}

dit_status dit_attn_fp8_i8qk(const void* q, const void* k, const void* v, void* o, int B, int H, int N, int d,
                             const int64_t sq[3], const int64_t sk[3], const int64_t sv[3], const int64_t so[3],
                             const float* rope_cos, const float* rope_sin, float softmax_scale, int q_block,
                             int kv_block, int smooth_k, void* workspace, size_t workspace_bytes,
                             dit_stream_t stream) {
  const NvtxRange nvtx_range("dit_attn_fp8_i8qk");
  return attn_fp8_impl(q, k, v, o, B, H, N, d, sq, sk, sv, so, rope_cos, rope_sin, softmax_scale, q_block, kv_block,
                       smooth_k, workspace, workspace_bytes, 1, stream);
}

size_t fbcache_gate_workspace_bytes(int64_t n) {
  if (n < 1) return 0;
  return static_cast<size_t>(dit::gate_num_ctas(n)) * 2 * sizeof(double);
}

dit_status fbcache_gate(const void* r_cur, const void* r_prev, int64_t n, float threshold, float* rel_out,
                        int32_t* skip_out, void* workspace, size_t workspace_bytes, dit_stream_t stream) {
  const NvtxRange nvtx_range("fbcache_gate");
  if (!r_cur || !r_prev || !rel_out || !skip_out || n < 1) return DIT_ERR_INVALID_ARG;
  if (!std::isfinite(threshold)) return DIT_ERR_INVALID_ARG;
  if (!aligned16(r_cur) || !aligned16(r_prev) || !aligned4(rel_out) || !aligned4(skip_out)) return DIT_ERR_ALIGNMENT;
  const size_t need = fbcache_gate_workspace_bytes(n);
  if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 7u)) return DIT_ERR_WORKSPACE;
  const DeviceState* ds = device_state();
  if (!ds || !ds->sm100) return DIT_ERR_UNSUPPORTED;
  return launch_status(dit::launch_gate(r_cur, r_prev, n, threshold, rel_out, skip_out,
                                        static_cast<double*>(workspace), reinterpret_cast<cudaStream_t>(stream)));
}

dit_status fbcache_gate_sums(const void* r_cur, const void* r_prev, int64_t n, double* sums_out, void* workspace,
                             size_t workspace_bytes, dit_stream_t stream) {
  const NvtxRange nvtx_range("fbcache_gate_sums");
  if (!r_cur || !r_prev || !sums_out || n < 1) return DIT_ERR_INVALID_ARG;
  if (!aligned16(r_cur) || !aligned16(r_prev) || (reinterpret_cast<uintptr_t>(sums_out) & 7u)) return DIT_ERR_ALIGNMENT;
  const size_t need = fbcache_gate_workspace_bytes(n);
  if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 7u)) return DIT_ERR_WORKSPACE;
  const DeviceState* ds = device_state();
  if (!ds || !ds->sm100) return DIT_ERR_UNSUPPORTED;
  return launch_status(dit::launch_gate_sums(r_cur, r_prev, n, sums_out, static_cast<double*>(workspace),
                                             reinterpret_cast<cudaStream_t>(stream)));
}

dit_status fbcache_gate_ref_update(const void* r_cur, void* r_ref, int64_t n, const int32_t* skip,
                                   dit_stream_t stream) {
  const NvtxRange nvtx_range("fbcache_gate_ref_update");
  if (!r_cur || !r_ref || n < 1) return DIT_ERR_INVALID_ARG;
  if (!aligned16(r_cur) || !aligned16(r_ref) || !aligned4(skip)) return DIT_ERR_ALIGNMENT;
  if (r_cur == r_ref) return DIT_ERR_INVALID_ARG;
  const DeviceState* ds = device_state();
  if (!ds || !ds->sm100) return DIT_ERR_UNSUPPORTED;
  return launch_status(dit::launch_gate_ref_update(r_cur, r_ref, n, skip, reinterpret_cast<cudaStream_t>(stream)));
}

dit_status fbcache_gate_finalize(const double* sums, float threshold, float* rel_out, int32_t* skip_out,
                                 dit_stream_t stream) {
  const NvtxRange nvtx_range("fbcache_gate_finalize");
  if (!sums || !rel_out || !skip_out) return DIT_ERR_INVALID_ARG;
  if (!std::isfinite(threshold)) return DIT_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(sums) & 7u) || !aligned4(rel_out) || !aligned4(skip_out)) return DIT_ERR_ALIGNMENT;
  const DeviceState* ds = device_state();
  if (!ds || !ds->sm100) return DIT_ERR_UNSUPPORTED;
  return launch_status(dit::launch_gate_finalize(sums, threshold, rel_out, skip_out,
                                                 reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"
