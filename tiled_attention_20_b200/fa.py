"""Python binding of libfa (include/fa.h): argument marshalling only.

Every step of the attention forward and backward runs in the CUDA kernels
behind the C ABI; this module checks tensor properties, allocates outputs
with PyTorch (device memory is plumbing) and passes raw pointers plus the
current CUDA stream.  There is no CPU fallback: if libfa.so cannot be loaded,
every call raises.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfa.so")

FA_OK = 0
STATUS_NAMES = {
    0: "FA_OK", -1: "FA_ERR_NULL", -2: "FA_ERR_SHAPE", -3: "FA_ERR_UNSUPPORTED_D",
    -4: "FA_ERR_ALIGN", -5: "FA_ERR_WORKSPACE", -6: "FA_ERR_LAUNCH", -7: "FA_ERR_TIMEOUT",
    -8: "FA_ERR_DEVICE_ASSERT", -9: "FA_ERR_ARCH", -10: "FA_ERR_ARG",
    -11: "FA_ERR_NOALLOC_LIMIT",
}

EXPORTED = ["fa_fwd", "fa_bwd", "fa_bwd_workspace_size", "fa_strerror",
            "fa_check_device_errors", "fa_launch_shape", "fa_trace_start", "fa_trace_stop",
            "fa_trace_kernel_name", "fa_bwd_noalloc", "fa_bwd_deterministic",
            "fa_decode", "fa_decode_workspace_size", "fa_decode_plan", "fa_fwd_fp8",
            "fa_gemm", "fa_gemm_workspace_size", "fa_gemm_tiles", "fa_selftest_wait_timeout",
            "fa_fwd_schedule", "fa_trace_start_mask"]
NOALLOC_MAX_SCRATCH = 32 << 20  # FA_BWD_NOALLOC_MAX_SCRATCH
KERNEL_IDS = {0: "fa_fwd_kernel", 1: "fa_bwd_prep", 2: "fa_bwd_kernel", 3: "unused",
              4: "fa_dq_kernel", 5: "fa_decode_kernel", 6: "fa_gemm_kernel", 7: "fa_gemm_pack"}
DECODE_MAX_NQ = 8


class FAError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)} ({strerror(status)})")


_lib = None
_vp, _i, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t


def load(path: str = LIB_PATH):
    """Load libfa.so and declare its signatures.  Raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise RuntimeError(
                f"libfa.so not found at {path}: build it with "
                "`python -m tiled_attention_20_b200.build` (there is no fallback)")
        lib = ctypes.CDLL(path)
        lib.fa_fwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _vp]
        lib.fa_fwd.restype = _i
        lib.fa_bwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                               _i, _i, _i, _i, _f, _i, _vp, _sz, _i, _vp]
        lib.fa_bwd.restype = _i
        lib.fa_bwd_deterministic.argtypes = lib.fa_bwd.argtypes
        lib.fa_bwd_deterministic.restype = _i
        lib.fa_bwd_workspace_size.argtypes = [_i, _i, _i, _i]
        lib.fa_bwd_workspace_size.restype = _sz
        lib.fa_strerror.argtypes = [_i]
        lib.fa_strerror.restype = ctypes.c_char_p
        lib.fa_check_device_errors.argtypes = [_vp]
        lib.fa_check_device_errors.restype = _i
        lib.fa_launch_shape.argtypes = [_i, _i, _i, _i, _i, _i,
                                        ctypes.POINTER(_i), ctypes.POINTER(_i)]
        lib.fa_launch_shape.restype = _i
        lib.fa_trace_start.argtypes = []
        lib.fa_trace_start.restype = _i
        lib.fa_trace_start_mask.argtypes = [ctypes.c_uint]
        lib.fa_trace_start_mask.restype = _i
        lib.fa_trace_stop.argtypes = [_i, ctypes.POINTER(_i), ctypes.POINTER(ctypes.c_double)]
        lib.fa_trace_stop.restype = _i
        lib.fa_trace_kernel_name.argtypes = [_i]
        lib.fa_trace_kernel_name.restype = ctypes.c_char_p
        lib.fa_bwd_noalloc.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                       _i, _i, _i, _i, _f, _i, _i, _vp]
        lib.fa_bwd_noalloc.restype = _i
        lib.fa_selftest_wait_timeout.argtypes = [_i, _vp]
        lib.fa_selftest_wait_timeout.restype = _i
        lib.fa_gemm.argtypes = [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _sz, _vp]
        lib.fa_gemm.restype = _i
        lib.fa_gemm_workspace_size.argtypes = [_vp, _vp, _i, _i, _i, _i, _i]
        lib.fa_gemm_workspace_size.restype = _sz
        lib.fa_gemm_tiles.argtypes = [_i, _i, _i, ctypes.POINTER(_i), ctypes.POINTER(_i),
                                      ctypes.POINTER(_i)]
        lib.fa_gemm_tiles.restype = _i
        lib.fa_fwd_schedule.argtypes = [_i, _i, _i, _i, _i, ctypes.POINTER(_i),
                                         ctypes.POINTER(_i), ctypes.POINTER(_i)]
        lib.fa_fwd_schedule.restype = _i
        lib.fa_fwd_fp8.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f,
                                   _i, _vp]
        lib.fa_fwd_fp8.restype = _i
        lib.fa_decode.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i,
                                  _i, _vp, _sz, _vp]
        lib.fa_decode.restype = _i
        lib.fa_decode_workspace_size.argtypes = [_i, _i, _i, _i, _i, _i]
        lib.fa_decode_workspace_size.restype = _sz
        lib.fa_decode_plan.argtypes = [_i, _i, _i, _i, _i, _i, _i, ctypes.POINTER(_i),
                                       ctypes.POINTER(_i)]
        lib.fa_decode_plan.restype = _i
        _lib = lib
    return _lib


def strerror(status: int) -> str:
    return load().fa_strerror(int(status)).decode()


def _check(status: int, what: str):
    if status != FA_OK:
        raise FAError(status, what)


def _stream(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _check_qkv(*ts):
    q = ts[0]
    if q.dim() != 4:
        raise ValueError("expected [B, H, N, d] tensors")
    for t in ts:
        if not t.is_cuda:
            raise ValueError("tensors must be on a CUDA device (no CPU fallback)")
        if t.dtype != torch.bfloat16:
            raise ValueError("inputs must be bf16")
        if t.shape != q.shape:
            raise ValueError("all inputs must share the shape [B, H, N, d]")
        if not t.is_contiguous():
            raise ValueError("inputs must be contiguous")
        if t.device != q.device:
            raise ValueError("inputs must be on one device")


def _check_buffer(name, t, device, dtype, shape=None, min_numel=None):
    """A tensor the caller passes for the library to read or write: on
    `device`, of `dtype`, contiguous, and of `shape` (or at least `min_numel`
    elements).  Raises ValueError before anything reaches libfa."""
    if not torch.is_tensor(t):
        raise ValueError(f"{name} must be a torch tensor")
    if t.device != device:
        raise ValueError(f"{name} must be on {device} (got {t.device})")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype} (got {t.dtype})")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)} (got {tuple(t.shape)})")
    if min_numel is not None and t.numel() < min_numel:
        raise ValueError(f"{name} needs at least {min_numel} elements (got {t.numel()})")


def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)


def fwd(q, k, v, scale=None, causal=False, out=None, lse=None):
    """O [B,H,N,d] bf16 and lse [B,H,N] fp32 (natural log)."""
    _check_qkv(q, k, v)
    B, H, N, d = q.shape
    scale = default_scale(d) if scale is None else float(scale)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    _check_buffer("out", out, q.device, torch.bfloat16, q.shape)
    _check_buffer("lse", lse, q.device, torch.float32, (B, H, N))
    with torch.cuda.device(q.device):
        st = load().fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                           lse.data_ptr(), B, H, N, d, scale, int(bool(causal)), _stream(q.device))
    _check(st, "fa_fwd")
    return out, lse


def fwd_fp8(q, k, v, descale_q, descale_k, descale_v, scale=None, causal=False, out=None,
            lse=None):
    """fa_fwd_fp8: q, k, v are float8_e4m3fn [B,H,N,128] CUDA tensors and
    descale_* fp32 [B,H] per-head dequantisation factors.  Returns O bf16
    [B,H,N,128] and lse fp32 [B,H,N]."""
    if q.dim() != 4:
        raise ValueError("expected [B, H, N, d] tensors")
    for t in (q, k, v):
        if not t.is_cuda or t.dtype != torch.float8_e4m3fn or not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous float8_e4m3fn CUDA tensors")
        if t.shape != q.shape or t.device != q.device:
            raise ValueError("q, k, v must share shape and device")
    B, H, N, d = q.shape
    for t in (descale_q, descale_k, descale_v):
        if (not t.is_cuda or t.dtype != torch.float32 or t.numel() != B * H
                or not t.is_contiguous()):
            raise ValueError("descale factors must be contiguous fp32 [B, H] CUDA tensors")
    scale = default_scale(d) if scale is None else float(scale)
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    _check_buffer("out", out, q.device, torch.bfloat16, q.shape)
    _check_buffer("lse", lse, q.device, torch.float32, (B, H, N))
    with torch.cuda.device(q.device):
        st = load().fa_fwd_fp8(q.data_ptr(), k.data_ptr(), v.data_ptr(), descale_q.data_ptr(),
                               descale_k.data_ptr(), descale_v.data_ptr(), out.data_ptr(),
                               lse.data_ptr(), B, H, N, d, scale, int(bool(causal)),
                               _stream(q.device))
    _check(st, "fa_fwd_fp8")
    return out, lse


def workspace_size(B, H, N, d) -> int:
    return int(load().fa_bwd_workspace_size(B, H, N, d))


def _grad_code(grad_dtype) -> int:
    codes = {torch.bfloat16: 0, torch.float32: 1}
    if grad_dtype not in codes:
        raise ValueError("grad_dtype must be torch.bfloat16 or torch.float32")
    return codes[grad_dtype]


def _grad_buffers(q, grad_dtype, dq, dk, dv):
    """dq, dk, dv as given (checked) or freshly allocated."""
    out = []
    for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        if t is None:
            t = torch.empty(q.shape, dtype=grad_dtype, device=q.device)
        _check_buffer(name, t, q.device, grad_dtype, q.shape)
        out.append(t)
    return out


def bwd(q, k, v, o, dO, lse, scale=None, causal=False, grad_dtype=torch.bfloat16,
        workspace=None, dq=None, dk=None, dv=None, deterministic=False):
    """dQ, dK, dV [B,H,N,d] (bf16 or fp32) for the forward that produced o, lse.
    deterministic=True calls fa_bwd_deterministic (bit-reproducible dQ)."""
    _check_qkv(q, k, v, o, dO)
    B, H, N, d = q.shape
    _check_buffer("lse", lse, q.device, torch.float32, (B, H, N))
    scale = default_scale(d) if scale is None else float(scale)
    gd = _grad_code(grad_dtype)
    ws_bytes = workspace_size(B, H, N, d)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=q.device)
    _check_buffer("workspace", workspace, q.device, torch.uint8, min_numel=ws_bytes)
    dq, dk, dv = _grad_buffers(q, grad_dtype, dq, dk, dv)
    with torch.cuda.device(q.device):
        fn = load().fa_bwd_deterministic if deterministic else load().fa_bwd
        st = fn(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                dO.data_ptr(), lse.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                dv.data_ptr(), B, H, N, d, scale, int(bool(causal)),
                workspace.data_ptr(), workspace.numel(), gd, _stream(q.device))
    _check(st, "fa_bwd_deterministic" if deterministic else "fa_bwd")
    return dq, dk, dv


def bwd_noalloc(q, k, v, o, dO, lse, scale=None, causal=False, grad_dtype=torch.bfloat16,
                dq=None, dk=None, dv=None):
    """fa_bwd_noalloc: the backward with the library's fixed internal scratch
    instead of a caller workspace, for callers that cannot allocate device
    memory (the outputs here are still allocated by PyTorch for convenience;
    such a caller passes its own).  Problems needing more than
    NOALLOC_MAX_SCRATCH bytes of scratch raise FA_ERR_NOALLOC_LIMIT; calls
    that overlap on the GPU share the scratch and must not run concurrently."""
    _check_qkv(q, k, v, o, dO)
    B, H, N, d = q.shape
    _check_buffer("lse", lse, q.device, torch.float32, (B, H, N))
    scale = default_scale(d) if scale is None else float(scale)
    gd = _grad_code(grad_dtype)
    dq, dk, dv = _grad_buffers(q, grad_dtype, dq, dk, dv)
    with torch.cuda.device(q.device):
        st = load().fa_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                   dO.data_ptr(), lse.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                                   dv.data_ptr(), B, H, N, d, scale, int(bool(causal)), gd,
                                   _stream(q.device))
    _check(st, "fa_bwd_noalloc")
    return dq, dk, dv


def check_device_errors(device=None) -> None:
    """Synchronise and raise if a kernel latched a device-side error."""
    device = torch.cuda.current_device() if device is None else device
    with torch.cuda.device(device):
        _check(load().fa_check_device_errors(_stream(device)), "device status")


def launch_shape(pass_: int, B, H, N, d, causal=False):
    ctas, units = _i(0), _i(0)
    _check(load().fa_launch_shape(pass_, B, H, N, d, int(bool(causal)), ctypes.byref(ctas),
                                  ctypes.byref(units)), "fa_launch_shape")
    return ctas.value, units.value


def trace_start(kernels=None) -> None:
    """Start bracketing library launches with CUDA events: every launch, or
    only those of the kernels named in `kernels` (names of KERNEL_IDS)."""
    if kernels is None:
        _check(load().fa_trace_start(), "fa_trace_start")
        return
    ids = {name: k for k, name in KERNEL_IDS.items()}
    mask = 0
    for name in kernels:
        if name not in ids:
            raise ValueError(f"unknown kernel {name!r}")
        mask |= 1 << ids[name]
    _check(load().fa_trace_start_mask(mask), "fa_trace_start_mask")


def trace_stop() -> dict:
    """Stop tracing; {kernel name: (launches, total ms)} for kernels that ran."""
    n = len(KERNEL_IDS)
    launches = (_i * n)()
    ms = (ctypes.c_double * n)()
    _check(load().fa_trace_stop(n, launches, ms), "fa_trace_stop")
    return {load().fa_trace_kernel_name(k).decode(): (launches[k], ms[k])
            for k in range(n) if launches[k]}


def decode_plan(BH, Nq, Nk, d, num_splits=0, sms=148, ctas_per_sm=2):
    """(splits, chunk_keys) fa_decode picks for this shape on a device with
    ``sms`` SMs holding ``ctas_per_sm`` decode CTAs each (host arithmetic)."""
    sp, ck = _i(0), _i(0)
    _check(load().fa_decode_plan(BH, Nq, Nk, d, num_splits, sms, ctas_per_sm,
                                 ctypes.byref(sp), ctypes.byref(ck)), "fa_decode_plan")
    return sp.value, ck.value


def decode_workspace_size(B, H, Nq, Nk, d, num_splits=0) -> int:
    """Bytes of scratch fa_decode needs on the current device (0: none)."""
    return int(load().fa_decode_workspace_size(B, H, Nq, Nk, d, num_splits))


def decode(q, k_cache, v_cache, cache_lens=None, scale=None, causal=False, nk=None,
           num_splits=0, out=None, lse=None, workspace=None):
    """Decode-shaped attention (fa_decode): q [B,H,Nq,d] (Nq <= 8) against a
    cache k_cache, v_cache [B,H,ld,d].  nk (default ld) is the longest valid
    length; cache_lens (int32 [B] on the device, optional) the valid rows per
    batch.  Returns O [B,H,Nq,d] bf16 and lse [B,H,Nq] fp32.  ``workspace``
    (uint8, at least decode_workspace_size bytes, its first B*H int32 words
    zero) may be kept across calls; without one a zeroed buffer is made."""
    for t in (q, k_cache, v_cache):
        if not t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous() or t.dim() != 4:
            raise ValueError("q, k_cache, v_cache must be contiguous bf16 [B, H, *, d] CUDA tensors")
        if t.device != q.device:
            raise ValueError("inputs must be on one device")
    B, H, Nq, d = q.shape
    ld = k_cache.shape[2]
    if k_cache.shape != (B, H, ld, d) or v_cache.shape != k_cache.shape:
        raise ValueError("k_cache and v_cache must be [B, H, ld, d] with q's B, H, d")
    nk = ld if nk is None else int(nk)
    if cache_lens is not None:
        if (not cache_lens.is_cuda or cache_lens.dtype != torch.int32 or cache_lens.numel() != B
                or not cache_lens.is_contiguous()):
            raise ValueError("cache_lens must be a contiguous int32 [B] CUDA tensor")
    scale = default_scale(d) if scale is None else float(scale)
    if out is None:
        out = torch.empty((B, H, Nq, d), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    with torch.cuda.device(q.device):
        if workspace is None:
            ws_bytes = decode_workspace_size(B, H, Nq, nk, d, num_splits)
            workspace = torch.zeros(max(ws_bytes, 16), dtype=torch.uint8, device=q.device)
        st = load().fa_decode(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
                              out.data_ptr(), lse.data_ptr(),
                              None if cache_lens is None else cache_lens.data_ptr(),
                              B, H, Nq, nk, ld, d, scale, int(bool(causal)), int(num_splits),
                              workspace.data_ptr(), workspace.numel(), _stream(q.device))
    _check(st, "fa_decode")
    return out, lse


def gemm_tiles(M, N, sms=148):
    """(tile_n, tiles_m, tiles_n): fa_gemm's tiles are 256 x tile_n."""
    bn, tm, tn = _i(0), _i(0), _i(0)
    _check(load().fa_gemm_tiles(M, N, sms, ctypes.byref(bn), ctypes.byref(tm), ctypes.byref(tn)),
           "fa_gemm_tiles")
    return bn.value, tm.value, tn.value


def fwd_schedule(B, H, N, causal=False, sms=148):
    """(items, merged_heads, tail_shift) of fa_fwd's work-unit schedule."""
    items, merged, shift = _i(0), _i(0), _i(0)
    _check(load().fa_fwd_schedule(B, H, N, int(bool(causal)), sms, ctypes.byref(items),
                                  ctypes.byref(merged), ctypes.byref(shift)), "fa_fwd_schedule")
    return items.value, merged.value, shift.value


def _ld(t):
    if t.dim() != 2 or t.stride(1) != 1 or t.stride(0) < t.shape[1]:
        raise ValueError("expected a 2-D matrix with unit column stride (rows may be padded)")
    return t.stride(0)


def gemm(a, b, out=None, workspace=None):
    """fa_gemm: C = A B for bf16 CUDA matrices A [M, K], B [K, N] (rows may be
    strided).  Returns C bf16 [M, N]."""
    for t in (a, b):
        if not t.is_cuda or t.dtype != torch.bfloat16:
            raise ValueError("A and B must be bf16 CUDA matrices")
    M, K = a.shape
    K2, N = b.shape
    if K2 != K or b.device != a.device:
        raise ValueError("A [M, K] and B [K, N] on one device")
    lda, ldb = _ld(a), _ld(b)
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=a.device)
    ldc = _ld(out)
    with torch.cuda.device(a.device):
        need = int(load().fa_gemm_workspace_size(a.data_ptr(), b.data_ptr(), M, N, K, lda, ldb))
        if workspace is None or workspace.numel() < need:
            workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=a.device)
        st = load().fa_gemm(a.data_ptr(), b.data_ptr(), out.data_ptr(), M, N, K, lda, ldb, ldc,
                            workspace.data_ptr(), workspace.numel(), _stream(a.device))
    _check(st, "fa_gemm")
    return out


def selftest_wait_timeout(limit_ms=50, device=None):
    """Enqueue the failure-detection self-test (a bounded wait that must time
    out after limit_ms); the next check_device_errors() raises FA_ERR_TIMEOUT."""
    device = torch.cuda.current_device() if device is None else device
    with torch.cuda.device(device):
        _check(load().fa_selftest_wait_timeout(int(limit_ms), _stream(device)),
               "fa_selftest_wait_timeout")
