/*
 * dit.h -- C ABI of the B200 (sm_100a) DiT joint-attention hot path.
 *
 * The operations, and the pages they are read from:
 *
 *   dit_attn_bf16    joint image+text multi-head self-attention with rotary
 *                    embedding on Q and K, BF16 operands, fp32 accumulation.
 *                    "FLUX 3 Image Klein / TensorRT-LLM VisualGen", section on
 *                    why the differences arise: the DiT's VANILLA BF16
 *                    attention takes about 60 % of its GPU kernel time.
 *   dit_attn_fp8     the same attention with e4m3 Q/K/V quantised in
 *                    per-token blocks, K mean-smoothed before quantisation.
 *                    Same page (cuDNN FP8 attention against VANILLA BF16) and
 *                    "vflash / Optimization ledger", table "Accepted or
 *                    exposed" (SageAttention2, a quantised attention).
 *   dit_attn_fp8_i8qk  the same with Q and K as symmetric int8 (8-bit integer
 *                    Q.K^T, e4m3 P.V): the SageAttention2 row of that table.
 *   dit_rope_tables  cos/sin tables of the multi-axis rotary embedding.
 *   rope_apply       rotary embedding applied to a [B,H,N,d] tensor.
 *                    "vflash / Optimization ledger", row "strict Triton RoPE".
 *   fbcache_gate     First-Block-Cache decision: relative L1 change of the
 *                    first block's residual between consecutive denoising
 *                    steps, compared with a threshold.  unsloth studio commit
 *                    "core/inference/diffusion.py", paragraph "Add opt-in step
 *                    caching (First-Block-Cache)".
 *
 * Definitions (the pages name these operations without formulas; the plain
 * textbook readings are used):
 *
 *   attention   O[b,h,i,:] = sum_j softmax_j(s_ij) V[b,h,j,:],
 *               s_ij = scale * <R_i Q[b,h,i,:], R_j K[b,h,j,:]>, every j in
 *               0..N-1 (bidirectional, no mask), scale <= 0 means 1/sqrt(d).
 *   rotary      head dim split into axis slices (d0,d1,d2), all even; pair p
 *               of axis a = channels (off_a+2p, off_a+2p+1), rotated by
 *               pos[a]*theta^(-2p/d_a):  y0 = x0 c - x1 s,  y1 = x0 s + x1 c.
 *               Tables hold c and s as fp32 [N][d/2] (pair index global).
 *   gate        rel = sum|r_cur - r_prev| / sum|r_prev| (0 if both sums are
 *               0, +inf if only the denominator is), skip = rel < threshold.
 *
 * Conventions for every entry point:
 *   - All data pointers are DEVICE pointers owned by the caller (e.g. by
 *     PyTorch).  The library never allocates, frees or synchronises, except
 *     dit_read_error which synchronises the given stream.
 *   - Tensors [B,H,N,d] are described by element strides {batch, head,
 *     token}; the channel dimension is contiguous.  Strides and base pointers
 *     must be 16-byte aligned (a TMA requirement): bf16 strides multiple of 8.
 *     A dimension of extent > 1 needs a positive stride (broadcast views are
 *     not supported) and token rows may not overlap (token stride >= d when
 *     N > 1); DIT_ERR_INVALID_ARG otherwise.  Layouts such as [B,N,H,d]
 *     (head stride d, token stride H*d) are fine.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default).
 *   - A non-DIT_OK return means nothing was enqueued.  Failures inside a
 *     kernel (a bounded wait that ran out) are recorded in a device error
 *     word that dit_read_error returns and clears.
 *   - There is no CPU fallback: every call runs the sm_100a kernels, and
 *     returns DIT_ERR_UNSUPPORTED on any other device.
 */
#ifndef DIT_H_
#define DIT_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define DIT_API __attribute__((visibility("default")))
#else
#define DIT_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* dit_stream_t; /* same type as cudaStream_t */

typedef enum {
  DIT_OK = 0,
  DIT_ERR_INVALID_ARG = 1,  /* null pointer, bad size or shape */
  DIT_ERR_UNSUPPORTED = 2,  /* d not supported, device not sm_100 */
  DIT_ERR_ALIGNMENT = 3,    /* pointer or stride not 16-byte aligned */
  DIT_ERR_WORKSPACE = 4,    /* workspace missing or too small */
  DIT_ERR_LAUNCH = 5,       /* CUDA error while enqueueing */
  DIT_ERR_TIMEOUT = 6,      /* (device error word) a bounded wait ran out */
  DIT_ERR_BOUNDS = 7        /* (device error word, debug build libdit_debug.so only) an index
                               failed a device-side bounds check; the access was skipped */
} dit_status;

/* Human-readable name of a status code (static string). */
DIT_API const char* dit_status_string(dit_status s);

/* Synchronises `stream`, then returns and clears the device error word of the
 * current device (DIT_OK if no kernel recorded a failure). */
DIT_API dit_status dit_read_error(dit_stream_t stream);

/* Failure-detection self test (no counterpart on the pages; it exercises the
 * library's own error path).  Enqueues one thread that waits, through the
 * bounded wait every kernel uses, on a barrier that nothing arrives on: after
 * the wait limit (1 s) it records DIT_ERR_TIMEOUT in the device error word and
 * ends, leaving the context usable.  dit_read_error then returns
 * DIT_ERR_TIMEOUT.  Returns DIT_ERR_UNSUPPORTED off sm_100. */
DIT_API dit_status dit_selftest_wait_timeout(dit_stream_t stream);

/* Unit-rate probes (no counterpart on the pages; they measure the hardware rates
 * the attention kernels' rooflines are drawn against).  Runs four short probes
 * on the current device, synchronously on `stream`, and writes per clock per SM
 * (from device cycle counts, so independent of the clock they ran at):
 *   out[0]  FLOP of tcgen05.mma kind::f8f6f4 (e4m3), M = 128, N = 128, both
 *           operands in shared memory (the attention kernels' Q.K^T shape)
 *   out[1]  FLOP of tcgen05.mma kind::f16 (bf16), same shape
 *   out[2]  results of ex2.approx.f32 (the softmax's exponential)
 *   out[3]  instructions of cvt.rn.satfinite.e4m3x2.f32 (two results each)
 * n_out: capacity of out, at least 4.  Allocates and frees a few bytes of
 * device memory.  Takes a few tens of milliseconds.  Returns DIT_ERR_INVALID_ARG
 * for a null out or n_out < 4, DIT_ERR_UNSUPPORTED off sm_100, DIT_ERR_TIMEOUT if
 * an MMA completion wait ran out, DIT_ERR_LAUNCH on a CUDA error. */
DIT_API dit_status dit_probe_unit_rates(double* out, int n_out, dit_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Rotary embedding                                                          */
/* ------------------------------------------------------------------------ */

/* Builds cos/sin tables, fp32 [N][d/2] each, d = d0+d1+d2, from int32
 * position ids pos[N][3] (device).  Angles are formed and evaluated in fp64
 * and rounded once to fp32.  d0,d1,d2 even and >= 0, d <= 256, N >= 1;
 * pos, cos_out, sin_out 4-byte aligned (the attention kernels read the tables
 * 16 bytes at a time, so allocate them 16-byte aligned). */
DIT_API dit_status dit_rope_tables(const int32_t* pos, int N, int d0, int d1, int d2, double theta, float* cos_out,
                           float* sin_out, dit_stream_t stream);

/* y = rotary(x) for x, y [B,H,N,d] with element strides sx/sy {batch, head,
 * token}; y may alias x exactly (in place, with sy equal to sx; a partial
 * overlap is not detected and is the caller's error).  dtype: 0 = bf16 in and out,
 * 1 = bf16 in, fp32 out.  Math in fp32, output rounded once (RNE).
 * d in {64, 128}; tables as built by dit_rope_tables. */
DIT_API dit_status rope_apply(const void* x, void* y, int B, int H, int N, int d, const int64_t sx[3], const int64_t sy[3],
                      const float* cos_tab, const float* sin_tab, int dtype, dit_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Attention                                                                 */
/* ------------------------------------------------------------------------ */

/* Workspace needed by dit_attn_bf16 (0 when has_rope == 0).  With rotary
 * tables the rotated K is staged there as contiguous bf16 [B,H,N,d] (one pass
 * per call; every Q tile reads every K tile).  Q is rotated inside the
 * attention kernel as each Q tile is loaded and needs no workspace. */
DIT_API size_t dit_attn_bf16_workspace_bytes(int B, int H, int N, int d, int has_rope);

/* O = attention(Q, K, V) in BF16 with fp32 accumulation and softmax.
 * q, k, v: bf16 [B,H,N,d] inputs; o: bf16 [B,H,N,d] output (must not alias
 * q, k or v: o equal to one of them is DIT_ERR_INVALID_ARG; a partial
 * overlap is not detected).  rope_cos/rope_sin: tables [N][d/2] or both NULL (no rotary).
 * softmax_scale <= 0 selects 1/sqrt(d).  d in {64, 128}; N >= 1.
 * workspace: device buffer of at least dit_attn_bf16_workspace_bytes, 256-byte
 * aligned (may be NULL when that size is 0). */
DIT_API dit_status dit_attn_bf16(const void* q, const void* k, const void* v, void* o, int B, int H, int N, int d,
                         const int64_t sq[3], const int64_t sk[3], const int64_t sv[3], const int64_t so[3],
                         const float* rope_cos, const float* rope_sin, float softmax_scale, void* workspace,
                         size_t workspace_bytes, dit_stream_t stream);

/* dit_attn_bf16 whose work is conditional on a device flag: when *skip != 0 at
 * the time the kernels run, both launches (the K rotation and the attention)
 * return at once and o is left as it was.  skip: device int32, 4-byte aligned,
 * typically the skip_out of fbcache_gate on the same stream, so that a
 * denoising step's remaining blocks can be enqueued without reading the gate's
 * decision on the host (the device-side form of First-Block-Cache skipping:
 * unsloth studio commit, "Add opt-in step caching (First-Block-Cache)"; the
 * decision is otherwise a graph break, as the FLUX 3 / TensorRT-LLM VisualGen
 * page's CUDA-graph note implies).  Other arguments and errors as
 * dit_attn_bf16; DIT_ERR_INVALID_ARG for a null skip, DIT_ERR_ALIGNMENT for a
 * misaligned one. */
DIT_API dit_status dit_attn_bf16_skippable(const void* q, const void* k, const void* v, void* o, int B, int H, int N,
                                           int d, const int64_t sq[3], const int64_t sk[3], const int64_t sv[3],
                                           const int64_t so[3], const float* rope_cos, const float* rope_sin,
                                           float softmax_scale, void* workspace, size_t workspace_bytes,
                                           const int32_t* skip, dit_stream_t stream);

/* Workspace needed by dit_attn_fp8: e4m3 copies of rotated Q, smoothed K
 * and V, their per-block fp32 scales and the fp32 K channel means (one
 * prologue pass rotates, smooths and quantises them before the attention
 * kernel runs). */
DIT_API size_t dit_attn_fp8_workspace_bytes(int B, int H, int N, int d, int q_block, int kv_block);

/* O = attention in FP8: Q and K rotated, K smoothed (smooth_k != 0:
 * per-(b,h) channel mean over all N tokens subtracted after rotation), then
 * quantised to e4m3 (RNE, saturating) with one fp32 scale amax/448 per block
 * of q_block (Q) or kv_block (K, V) tokens.  Scores accumulate in fp32; P is
 * e4m3 with the V block scale folded in; the row sum uses the fp32 P.
 * Supported: d = 128, q_block = 128, kv_block = 64, B * H <= 65535
 * (DIT_ERR_UNSUPPORTED otherwise).  Arguments otherwise as dit_attn_bf16. */
DIT_API dit_status dit_attn_fp8(const void* q, const void* k, const void* v, void* o, int B, int H, int N, int d,
                        const int64_t sq[3], const int64_t sk[3], const int64_t sv[3], const int64_t so[3],
                        const float* rope_cos, const float* rope_sin, float softmax_scale, int q_block, int kv_block,
                        int smooth_k, void* workspace, size_t workspace_bytes, dit_stream_t stream);

/* FP8 attention with an 8-bit integer Q.K^T: the quantised attention of
 * "vflash / Optimization ledger", table "Accepted or exposed", SageAttention2
 * row (8-bit integer Q.K^T, FP8 P.V).  As dit_attn_fp8 except that the rotated
 * Q and the rotated, smoothed K are quantised to symmetric int8 (one fp32
 * scale amax/127 per block of q_block or kv_block tokens, round to nearest
 * even, within +-127) and S = Q8 K8^T accumulates exactly in int32 on the
 * tensor cores (kind::i8) before it is scaled by sQ * sK * softmax_scale.  V,
 * P and everything after the scores are as in dit_attn_fp8.  Where a few
 * channels of Q and K carry outliers, the integer codes keep the large
 * products to within 1/254 of the block maximum where e4m3 keeps 1/16 of
 * each product, so the result stays much closer to exact attention.  The
 * workspace layout and size are dit_attn_fp8's
 * (dit_attn_fp8_workspace_bytes); same supported sizes and errors. */
DIT_API dit_status dit_attn_fp8_i8qk(const void* q, const void* k, const void* v, void* o, int B, int H, int N, int d,
                                     const int64_t sq[3], const int64_t sk[3], const int64_t sv[3],
                                     const int64_t so[3], const float* rope_cos, const float* rope_sin,
                                     float softmax_scale, int q_block, int kv_block, int smooth_k, void* workspace,
                                     size_t workspace_bytes, dit_stream_t stream);

/* ------------------------------------------------------------------------ */
/* First-Block-Cache gate                                                    */
/* ------------------------------------------------------------------------ */

/* Workspace needed by fbcache_gate for n elements (per-CTA partial sums). */
DIT_API size_t fbcache_gate_workspace_bytes(int64_t n);

/* rel_out[0] = sum|r_cur - r_prev| / sum|r_prev| over n contiguous bf16
 * elements (fp32 per-thread partials, fp64 combine in a fixed order, so the
 * result is deterministic); skip_out[0] = (rel < threshold).  rel_out and
 * skip_out are device pointers; read skip_out on the host to branch.
 * n >= 1; r_cur, r_prev 16-byte aligned; rel_out, skip_out 4-byte aligned. */
DIT_API dit_status fbcache_gate(const void* r_cur, const void* r_prev, int64_t n, float threshold, float* rel_out,
                        int32_t* skip_out, void* workspace, size_t workspace_bytes, dit_stream_t stream);

/* The gate over a residual split across ranks (sequence-parallel runs): each
 * rank computes its shard's totals, sums_out[0] = sum |r_cur - r_prev| and
 * sums_out[1] = sum |r_prev| (fp64, device, 8-byte aligned; same kernels and
 * order as fbcache_gate); the caller adds the totals across ranks (an
 * all-reduce of two doubles) and fbcache_gate_finalize decides.  Every rank
 * then holds the same rel and skip.  Workspace as fbcache_gate. */
DIT_API dit_status fbcache_gate_sums(const void* r_cur, const void* r_prev, int64_t n, double* sums_out,
                                     void* workspace, size_t workspace_bytes, dit_stream_t stream);

/* rel = sums[0] / sums[1] (0 when both are 0, +inf when only sums[1] is),
 * skip = rel < threshold, written to rel_out / skip_out (device). */
DIT_API dit_status fbcache_gate_finalize(const double* sums, float threshold, float* rel_out, int32_t* skip_out,
                                         dit_stream_t stream);

/* The gate's reference residual, for the two reference policies of the step
 * cache (unsloth studio commit "core/inference/diffusion.py", "Add opt-in step
 * caching (First-Block-Cache)": the threshold knob; which step the residual is
 * compared with is left open): r_ref = r_cur over n contiguous bf16 elements,
 * unless skip is non-NULL and *skip != 0 when the copy runs, in which case
 * r_ref is left as it is.  Called after fbcache_gate with that call's skip_out,
 * it keeps r_ref at the residual of the last step whose remaining blocks ran
 * ("last computed" policy) without a host read; with skip NULL it copies
 * unconditionally (the "consecutive" policy, previous step).  r_cur, r_ref
 * 16-byte aligned and distinct, skip 4-byte aligned; n >= 1. */
DIT_API dit_status fbcache_gate_ref_update(const void* r_cur, void* r_ref, int64_t n, const int32_t* skip,
                                           dit_stream_t stream);

/* fbcache_gate without a workspace argument (the pages have no counterpart:
 * this is a convenience of this library).  For callers that cannot give the
 * library device memory, e.g. a plug-in run by a host framework that owns the
 * device allocator, or a step loop that must not allocate while it runs.
 * Same inputs, outputs, arithmetic and result as fbcache_gate; its scratch
 * is a fixed device array of 2 * 740 doubles (11,840 bytes) inside the
 * library, held by every device that loads it until the process exits.
 * Limit: the scratch must hold 2 doubles per pass-1 CTA; the CTA count is
 * capped at 740 for any n, so every n >= 1 fits (a larger need would return
 * DIT_ERR_WORKSPACE).  Nothing in the array has to start at zero.  The first
 * call on a device looks up the array's device address (a runtime query), so
 * make that first call before capturing the stream.  All calls share the one
 * array: calls that overlap on the GPU (different streams without ordering)
 * race on it; calls on one stream are safe. */
DIT_API dit_status fbcache_gate_noalloc(const void* r_cur, const void* r_prev, int64_t n, float threshold,
                                        float* rel_out, int32_t* skip_out, dit_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* DIT_H_ */
