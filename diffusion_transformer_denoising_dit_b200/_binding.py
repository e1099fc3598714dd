"""ctypes binding over libdit.so (argument marshalling only).

Every operation runs in the library's sm_100a kernels on the caller's current
CUDA stream; this module only checks tensor metadata, passes raw device
pointers, element strides and sizes, and raises on a non-OK status.  There is
no fallback: a missing or unloadable library raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# DIT_LIB_VARIANT=debug loads the bounds-checking debug build (libdit_debug.so)
LIB_PATH = os.path.join(_PKG, "libdit_debug.so" if os.environ.get("DIT_LIB_VARIANT") == "debug" else "libdit.so")

STATUS = {0: "DIT_OK", 1: "DIT_ERR_INVALID_ARG", 2: "DIT_ERR_UNSUPPORTED", 3: "DIT_ERR_ALIGNMENT",
          4: "DIT_ERR_WORKSPACE", 5: "DIT_ERR_LAUNCH", 6: "DIT_ERR_TIMEOUT", 7: "DIT_ERR_BOUNDS"}
EXPORTS = ["dit_status_string", "dit_read_error", "dit_rope_tables", "rope_apply",
           "dit_attn_bf16_workspace_bytes", "dit_attn_bf16", "dit_attn_fp8_workspace_bytes",
           "dit_attn_fp8", "dit_attn_fp8_i8qk", "fbcache_gate_workspace_bytes", "fbcache_gate", "fbcache_gate_noalloc",
           "dit_selftest_wait_timeout", "dit_attn_bf16_skippable", "fbcache_gate_sums", "fbcache_gate_finalize",
           "fbcache_gate_ref_update", "dit_probe_unit_rates"]


class DitError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {STATUS.get(code, code)}")
        self.code = code


_lib = None

_i64x3 = ctypes.c_int64 * 3
_vp = ctypes.c_void_p
_i = ctypes.c_int
_sz = ctypes.c_size_t


def lib() -> ctypes.CDLL:
    """The loaded libdit.so; raises if it is absent (build it with build.py)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run `python -m "
                               "diffusion_transformer_denoising_dit_b200.build` (needs nvcc)")
        L = ctypes.CDLL(LIB_PATH)
        L.dit_status_string.restype = ctypes.c_char_p
        L.dit_status_string.argtypes = [_i]
        L.dit_read_error.restype = _i
        L.dit_read_error.argtypes = [_vp]
        L.dit_selftest_wait_timeout.restype = _i
        L.dit_selftest_wait_timeout.argtypes = [_vp]
        L.dit_probe_unit_rates.restype = _i
        L.dit_probe_unit_rates.argtypes = [_vp, _i, _vp]
        L.dit_rope_tables.restype = _i
        L.dit_rope_tables.argtypes = [_vp, _i, _i, _i, _i, ctypes.c_double, _vp, _vp, _vp]
        L.rope_apply.restype = _i
        L.rope_apply.argtypes = [_vp, _vp, _i, _i, _i, _i, _i64x3, _i64x3, _vp, _vp, _i, _vp]
        L.dit_attn_bf16_workspace_bytes.restype = _sz
        L.dit_attn_bf16_workspace_bytes.argtypes = [_i, _i, _i, _i, _i]
        L.dit_attn_bf16.restype = _i
        L.dit_attn_bf16.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i64x3, _i64x3, _i64x3, _i64x3,
                                    _vp, _vp, ctypes.c_float, _vp, _sz, _vp]
        L.dit_attn_bf16_skippable.restype = _i
        L.dit_attn_bf16_skippable.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i64x3, _i64x3, _i64x3, _i64x3,
                                              _vp, _vp, ctypes.c_float, _vp, _sz, _vp, _vp]
        L.dit_attn_fp8_workspace_bytes.restype = _sz
        L.dit_attn_fp8_workspace_bytes.argtypes = [_i, _i, _i, _i, _i, _i]
        L.dit_attn_fp8.restype = _i
        L.dit_attn_fp8.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i64x3, _i64x3, _i64x3, _i64x3,
                                   _vp, _vp, ctypes.c_float, _i, _i, _i, _vp, _sz, _vp]
        L.dit_attn_fp8_i8qk.restype = _i
        L.dit_attn_fp8_i8qk.argtypes = L.dit_attn_fp8.argtypes
        L.fbcache_gate_workspace_bytes.restype = _sz
        L.fbcache_gate_workspace_bytes.argtypes = [ctypes.c_int64]
        L.fbcache_gate.restype = _i
        L.fbcache_gate.argtypes = [_vp, _vp, ctypes.c_int64, ctypes.c_float, _vp, _vp, _vp, _sz, _vp]
        L.fbcache_gate_sums.restype = _i
        L.fbcache_gate_sums.argtypes = [_vp, _vp, ctypes.c_int64, _vp, _vp, _sz, _vp]
        L.fbcache_gate_finalize.restype = _i
        L.fbcache_gate_finalize.argtypes = [_vp, ctypes.c_float, _vp, _vp, _vp]
        L.fbcache_gate_ref_update.restype = _i
        L.fbcache_gate_ref_update.argtypes = [_vp, _vp, ctypes.c_int64, _vp, _vp]
        L.fbcache_gate_noalloc.restype = _i
        L.fbcache_gate_noalloc.argtypes = [_vp, _vp, ctypes.c_int64, ctypes.c_float, _vp, _vp, _vp]
        _lib = L
    return _lib


def _check(fn: str, code: int):
    if code != 0:
        raise DitError(fn, code)


def _stream(t: torch.Tensor):
    return torch.cuda.current_stream(t.device).cuda_stream


def _ptr(t):
    return None if t is None else t.data_ptr()


def _strides(t: torch.Tensor):
    """{batch, head, token} element strides of a [B,H,N,d] tensor with a contiguous last dim."""
    if t.dim() != 4:
        raise ValueError("expected a [B, H, N, d] tensor")
    if t.stride(3) != 1:
        raise ValueError("the channel (last) dimension must be contiguous")
    return _i64x3(t.stride(0), t.stride(1), t.stride(2))


def _need_cuda(*ts):
    devs = set()
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("all tensors must be CUDA tensors (there is no CPU path)")
        if t is not None:
            devs.add(t.device)
    if len(devs) > 1:
        raise ValueError(f"all tensors must be on one device, got {sorted(map(str, devs))}")


def _check_tables(cos, sin, N: int, d: int):
    """The kernels read rotary tables as fp32 [N, d/2] rows, 16 bytes at a time."""
    if (cos is None) != (sin is None):
        raise ValueError("pass both rotary tables or neither")
    for t in (cos, sin):
        if t is not None and (t.dtype != torch.float32 or tuple(t.shape) != (N, d // 2) or not t.is_contiguous()):
            raise ValueError(f"rotary tables must be contiguous float32 [{N}, {d // 2}] (as rope_tables builds them)")


def _check_out(out, shape, dtype):
    if tuple(out.shape) != tuple(shape) or out.dtype != dtype:
        raise ValueError(f"out must be {dtype} of shape {list(shape)}, got {out.dtype} {list(out.shape)}")


def _check_bytes(buf, name: str):
    if buf is not None and not buf.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def read_error(stream=None) -> int:
    """Synchronise the stream and return+clear the device error word (0 = none)."""
    s = torch.cuda.current_stream().cuda_stream if stream is None else stream
    return lib().dit_read_error(s)


def selftest_wait_timeout(stream=None) -> None:
    """Enqueue the failure-detection self test: a bounded wait that nothing
    satisfies, which gives up after its limit and records DIT_ERR_TIMEOUT
    (read it with read_error())."""
    s = torch.cuda.current_stream().cuda_stream if stream is None else stream
    _check("dit_selftest_wait_timeout", lib().dit_selftest_wait_timeout(s))


def probe_unit_rates(stream=None) -> dict:
    """The hardware rates the kernels' rooflines are drawn against, per clock per
    SM, measured on the current device (see dit_probe_unit_rates)."""
    import ctypes
    s = torch.cuda.current_stream().cuda_stream if stream is None else stream
    out = (ctypes.c_double * 4)()
    _check("dit_probe_unit_rates", lib().dit_probe_unit_rates(ctypes.cast(out, ctypes.c_void_p), 4, s))
    return {"mma_e4m3_flop": out[0], "mma_bf16_flop": out[1], "ex2_results": out[2], "cvt_e4m3x2_instructions": out[3]}


def rope_tables(pos: torch.Tensor, axes, theta: float = 10000.0):
    """fp32 cos, sin tables [N, d/2] for int32 position ids pos [N, 3] (device)."""
    _need_cuda(pos)
    if pos.dtype != torch.int32 or pos.dim() != 2 or pos.shape[1] != 3:
        raise ValueError("pos must be int32 [N, 3]")
    pos = pos.contiguous()
    N = pos.shape[0]
    d = int(sum(axes))
    c = torch.empty(N, d // 2, device=pos.device, dtype=torch.float32)
    s = torch.empty_like(c)
    _check("dit_rope_tables", lib().dit_rope_tables(pos.data_ptr(), N, int(axes[0]), int(axes[1]), int(axes[2]),
                                                    float(theta), c.data_ptr(), s.data_ptr(), _stream(pos)))
    return c, s


def rope_apply(x: torch.Tensor, cos: torch.Tensor, sin: torch.Tensor, out_dtype=torch.bfloat16, out=None):
    """Rotary embedding of x [B,H,N,d] (bf16) -> bf16 or fp32 (out may be x for in-place bf16)."""
    _need_cuda(x, cos, sin, out)
    if x.dtype != torch.bfloat16:
        raise ValueError("x must be bf16")
    B, H, N, d = x.shape
    _check_tables(cos, sin, N, d)
    if cos is None:
        raise ValueError("rope_apply needs the rotary tables")
    if out is None:
        out = torch.empty(B, H, N, d, device=x.device, dtype=out_dtype)
    if out.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("out must be bf16 or float32")
    _check_out(out, x.shape, out.dtype)
    dt = {torch.bfloat16: 0, torch.float32: 1}[out.dtype]
    _check("rope_apply", lib().rope_apply(x.data_ptr(), out.data_ptr(), B, H, N, d, _strides(x), _strides(out),
                                          cos.data_ptr(), sin.data_ptr(), dt, _stream(x)))
    return out


def attention(q, k, v, cos=None, sin=None, precision: str = "bf16", scale: float | None = None,
              out=None, workspace=None, q_block: int = 128, kv_block: int = 64, smooth_k: bool = True,
              skip=None):
    """Joint attention O [B,H,N,d] bf16 from bf16 q, k, v (+ optional rotary tables).

    precision: "bf16"; "fp8" (e4m3 Q, K, V and P); "fp8_i8qk" (symmetric int8 Q
    and K with an integer Q.K^T, e4m3 V and P).  Both 8-bit forms share one
    workspace layout.
    skip (BF16 only): a device int32 flag, e.g. FBCacheGate's output; when it is
    non-zero at the time the kernels run, the call does nothing and ``out`` keeps
    its previous contents."""
    _need_cuda(q, k, v, cos, sin, skip, out, workspace)
    if skip is not None and (precision != "bf16" or skip.dtype != torch.int32 or skip.numel() < 1):
        raise ValueError("skip must be a CUDA int32 flag and is supported for precision='bf16'")
    for t in (q, k, v):
        if t.dtype != torch.bfloat16:
            raise ValueError("q, k, v must be bf16")
    if not (q.shape == k.shape == v.shape):
        raise ValueError("q, k, v must have the same [B, H, N, d] shape")
    B, H, N, d = q.shape
    _check_tables(cos, sin, N, d)
    _check_bytes(workspace, "workspace")
    if out is None:
        out = torch.empty(B, H, N, d, device=q.device, dtype=torch.bfloat16)
    _check_out(out, q.shape, torch.bfloat16)
    sc = 0.0 if scale is None else float(scale)
    L = lib()
    if precision == "bf16":
        need = L.dit_attn_bf16_workspace_bytes(B, H, N, d, int(cos is not None))
    elif precision in ("fp8", "fp8_i8qk"):
        need = L.dit_attn_fp8_workspace_bytes(B, H, N, d, q_block, kv_block)
    else:
        raise ValueError("precision must be 'bf16', 'fp8' or 'fp8_i8qk'")
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, device=q.device, dtype=torch.uint8)
    wp = _ptr(workspace) if need else None
    wb = need if need else 0
    args = (q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, H, N, d,
            _strides(q), _strides(k), _strides(v), _strides(out), _ptr(cos), _ptr(sin), sc)
    if precision == "bf16" and skip is not None:
        _check("dit_attn_bf16_skippable", L.dit_attn_bf16_skippable(*args, wp, wb, skip.data_ptr(), _stream(q)))
    elif precision == "bf16":
        _check("dit_attn_bf16", L.dit_attn_bf16(*args, wp, wb, _stream(q)))
    elif precision == "fp8":
        _check("dit_attn_fp8", L.dit_attn_fp8(*args, q_block, kv_block, int(smooth_k), wp, wb, _stream(q)))
    else:
        _check("dit_attn_fp8_i8qk", L.dit_attn_fp8_i8qk(*args, q_block, kv_block, int(smooth_k), wp, wb, _stream(q)))
    return out


def attention_workspace(B, H, N, d, precision="bf16", rope=True, q_block=128, kv_block=64, device="cuda"):
    """Pre-allocated workspace for repeated attention calls of one shape."""
    L = lib()
    if precision not in ("bf16", "fp8", "fp8_i8qk"):
        raise ValueError("precision must be 'bf16', 'fp8' or 'fp8_i8qk'")
    need = (L.dit_attn_bf16_workspace_bytes(B, H, N, d, int(rope)) if precision == "bf16"
            else L.dit_attn_fp8_workspace_bytes(B, H, N, d, q_block, kv_block))
    return torch.empty(max(need, 1), device=device, dtype=torch.uint8)


def _a256(x: int) -> int:
    return (x + 255) // 256 * 256


def fp8_workspace_views(ws: torch.Tensor, B: int, H: int, N: int, d: int = 128, q_block: int = 128,
                        kv_block: int = 64):
    """Views into a dit_attn_fp8 / dit_attn_fp8_i8qk workspace (the layout written by the
    prologue): q8, k8, v8 (uint8 codes [B,H,N,d]: e4m3, or int8 two's complement for q8 and
    k8 of the integer Q.K^T form), q_scale, k_scale, v_scale, k_mean, v_scale_max."""
    bh = B * H
    el = bh * N * d
    nq, nk = -(-N // q_block), -(-N // kv_block)
    off = 0
    out = {}
    for name in ("q8", "k8", "v8"):
        out[name] = ws[off:off + el].view(B, H, N, d)
        off += _a256(el)
    for name, n in (("q_scale", bh * nq), ("k_scale", bh * nk), ("v_scale", bh * nk), ("k_mean", bh * d),
                    ("v_scale_max", bh)):
        out[name] = ws[off:off + 4 * n].view(torch.float32)
        off += _a256(4 * n)
    out["q_scale"] = out["q_scale"].view(B, H, nq)
    out["k_scale"] = out["k_scale"].view(B, H, nk)
    out["v_scale"] = out["v_scale"].view(B, H, nk)
    out["k_mean"] = out["k_mean"].view(B, H, d)
    out["v_scale_max"] = out["v_scale_max"].view(B, H)
    return out


def _check_flags(rel_out, skip_out):
    if rel_out is not None and (rel_out.dtype != torch.float32 or rel_out.numel() < 1):
        raise ValueError("rel_out must be a float32 tensor of at least one element")
    if skip_out is not None and (skip_out.dtype != torch.int32 or skip_out.numel() < 1):
        raise ValueError("skip_out must be an int32 tensor of at least one element")


def fbcache_gate(r_cur, r_prev, threshold: float, rel_out=None, skip_out=None, workspace=None):
    """(rel fp32 [1], skip int32 [1]) device tensors for two bf16 residuals of equal size."""
    _need_cuda(r_cur, r_prev, rel_out, skip_out, workspace)
    _check_flags(rel_out, skip_out)
    _check_bytes(workspace, "workspace")
    if r_cur.dtype != torch.bfloat16 or r_prev.dtype != torch.bfloat16:
        raise ValueError("residuals must be bf16")
    if r_cur.numel() != r_prev.numel() or not r_cur.is_contiguous() or not r_prev.is_contiguous():
        raise ValueError("residuals must be contiguous and of equal size")
    n = r_cur.numel()
    L = lib()
    need = L.fbcache_gate_workspace_bytes(n)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(need, device=r_cur.device, dtype=torch.uint8)
    if rel_out is None:
        rel_out = torch.empty(1, device=r_cur.device, dtype=torch.float32)
    if skip_out is None:
        skip_out = torch.empty(1, device=r_cur.device, dtype=torch.int32)
    _check("fbcache_gate", L.fbcache_gate(r_cur.data_ptr(), r_prev.data_ptr(), n, float(threshold),
                                          rel_out.data_ptr(), skip_out.data_ptr(), workspace.data_ptr(),
                                          workspace.numel() * workspace.element_size(), _stream(r_cur)))
    return rel_out, skip_out


def fbcache_gate_sums(r_cur, r_prev, sums_out=None, workspace=None):
    """Shard totals (sum |r_cur - r_prev|, sum |r_prev|) as a device float64 [2] tensor."""
    _need_cuda(r_cur, r_prev, sums_out, workspace)
    _check_bytes(workspace, "workspace")
    if sums_out is not None and (sums_out.dtype != torch.float64 or sums_out.numel() < 2
                                 or not sums_out.is_contiguous()):
        raise ValueError("sums_out must be a contiguous float64 tensor of at least two elements")
    if r_cur.dtype != torch.bfloat16 or r_prev.dtype != torch.bfloat16 or r_cur.shape != r_prev.shape:
        raise ValueError("r_cur, r_prev must be bf16 tensors of one shape")
    r_cur, r_prev = r_cur.contiguous(), r_prev.contiguous()
    n = r_cur.numel()
    L = lib()
    need = L.fbcache_gate_workspace_bytes(n)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(need, device=r_cur.device, dtype=torch.uint8)
    if sums_out is None:
        sums_out = torch.empty(2, device=r_cur.device, dtype=torch.float64)
    _check("fbcache_gate_sums", L.fbcache_gate_sums(r_cur.data_ptr(), r_prev.data_ptr(), n, sums_out.data_ptr(),
                                                    workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                                    _stream(r_cur)))
    return sums_out


def fbcache_gate_finalize(sums, threshold: float, rel_out=None, skip_out=None):
    """(rel, skip) device tensors from totals summed across shards."""
    _need_cuda(sums, rel_out, skip_out)
    _check_flags(rel_out, skip_out)
    if sums.dtype != torch.float64 or sums.numel() < 2:
        raise ValueError("sums must be a device float64 [2] tensor")
    if rel_out is None:
        rel_out = torch.empty(1, device=sums.device, dtype=torch.float32)
    if skip_out is None:
        skip_out = torch.empty(1, device=sums.device, dtype=torch.int32)
    _check("fbcache_gate_finalize", lib().fbcache_gate_finalize(sums.data_ptr(), float(threshold), rel_out.data_ptr(),
                                                              skip_out.data_ptr(), _stream(sums)))
    return rel_out, skip_out


def fbcache_gate_ref_update(r_cur, r_ref, skip=None):
    """r_ref <- r_cur on the device, unless the device int32 flag `skip` is set when
    the copy runs (then r_ref keeps the last computed step's residual)."""
    _need_cuda(r_cur, r_ref, skip)
    if r_cur.dtype != torch.bfloat16 or r_ref.dtype != torch.bfloat16 or r_cur.numel() != r_ref.numel():
        raise ValueError("r_cur, r_ref must be bf16 tensors of equal size")
    if not r_cur.is_contiguous() or not r_ref.is_contiguous():
        raise ValueError("r_cur, r_ref must be contiguous")
    if skip is not None and (skip.dtype != torch.int32 or skip.numel() < 1):
        raise ValueError("skip must be a CUDA int32 flag")
    _check("fbcache_gate_ref_update", lib().fbcache_gate_ref_update(r_cur.data_ptr(), r_ref.data_ptr(), r_cur.numel(),
                                                                    _ptr(skip), _stream(r_cur)))
    return r_ref


class FBCacheGate:
    """First-Block-Cache decision with its buffers allocated once.

    gate(r_cur, r_prev) enqueues the kernels for an explicit pair and returns the
    device int32 skip flag; ``.rel`` holds the relative L1 change.

    gate.step(r_cur) is the per-denoising-step form, with the reference held on
    the device: policy "consecutive" compares every step with the step before it,
    "last_computed" with the last step whose remaining blocks ran (so small
    changes add up across skipped steps); the first ``warmup`` steps (at least
    one: step 0 has nothing to compare with) are always computed.  The returned
    flag drives the skippable attention call directly; nothing is read on the
    host.  Reading it there (``bool(flag.item())``) is the one device-to-host
    crossing per step when the caller branches on the host instead.
    """

    POLICIES = ("consecutive", "last_computed")

    def __init__(self, threshold: float, numel: int, device="cuda", policy: str = "consecutive", warmup: int = 1):
        if policy not in self.POLICIES:
            raise ValueError(f"policy must be one of {self.POLICIES}")
        self.threshold = float(threshold)
        self.policy = policy
        self.warmup = max(1, int(warmup))
        self.numel = int(numel)
        self.rel = torch.empty(1, device=device, dtype=torch.float32)
        self.skip = torch.empty(1, device=device, dtype=torch.int32)
        self.never = torch.zeros(1, device=device, dtype=torch.int32)
        self.workspace = torch.empty(lib().fbcache_gate_workspace_bytes(numel), device=device, dtype=torch.uint8)
        self.ref = None
        self.t = 0

    def __call__(self, r_cur, r_prev):
        fbcache_gate(r_cur, r_prev, self.threshold, self.rel, self.skip, self.workspace)
        return self.skip

    def reset(self):
        """Start a new denoising trajectory (the next step is step 0)."""
        self.t = 0

    def step(self, r_cur):
        """Decision for this step's first-block residual r_cur: the device int32 flag
        (1 = skip the remaining blocks).  Updates the device-side reference."""
        if r_cur.numel() != self.numel:
            raise ValueError(f"r_cur must have {self.numel} elements")
        if self.ref is None:
            self.ref = torch.empty(self.numel, device=r_cur.device, dtype=torch.bfloat16)
        flat = r_cur.reshape(-1)
        if self.t < self.warmup:
            flag = self.never
            fbcache_gate_ref_update(flat, self.ref)
        else:
            fbcache_gate(flat, self.ref, self.threshold, self.rel, self.skip, self.workspace)
            flag = self.skip
            fbcache_gate_ref_update(flat, self.ref, None if self.policy == "consecutive" else flag)
        self.t += 1
        return flag
