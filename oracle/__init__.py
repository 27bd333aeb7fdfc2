"""fp64 CPU oracle for exact attention and its gradient.

TEST INFRASTRUCTURE ONLY: the test-suite, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this package; the product path (the
CUDA library and its Python binding) never does.  It shares no code with the
CUDA kernels.

The arithmetic lives in ``attention_oracle.c`` (plain loops in double
precision, OpenMP over independent rows).  This module only marshals numpy
arrays into it.  Definitions and the readings taken where the pages are silent
are stated in the C file's header:

* forward: softmax(scale * Q K^T [+ causal mask]) V, three passes per row
  ("第17讲 Tensor Core、HBM、SRAM 与 FlashAttention", §8.1 and §8.3);
* lse = m + ln l per row (natural log of the scaled scores);
* backward: the exact gradient of sum(O * dO) (pages silent; calculus);
* ``online_fwd``: the online-softmax recurrence of the same page's §8.3;
* ``gemm``: the plain matrix product (the CS336 lecture's opening curve);
* ``decode``: the same attention for a few new queries against a key/value
  cache (the same page's §9.2–9.3), with per-batch cache lengths and the
  causal mask aligned to the newest positions.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attention_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

_dp = ctypes.POINTER(ctypes.c_double)
_ip = ctypes.POINTER(ctypes.c_int)


def compile_source(src: str, out: str) -> str:
    """gcc a copy of the oracle's C source into a shared library."""
    tmp = out + ".tmp%d" % os.getpid()
    subprocess.check_call(
        ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", tmp, src, "-lm"])
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile the oracle with gcc into ``oracle/liboracle.so``."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        compile_source(_SRC, _LIB)
    return _LIB


_lib = None


def bind(lib):
    """Declare the C signatures on a loaded copy of the oracle library."""
    lib.oracle_fwd.argtypes = [_dp, _dp, _dp, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                               ctypes.c_int, ctypes.c_double, ctypes.c_int, _dp, _dp]
    lib.oracle_fwd.restype = None
    lib.oracle_fwd_rows.argtypes = [_dp, _dp, _dp, ctypes.c_int, ctypes.c_int,
                                    ctypes.c_double, ctypes.c_int, _ip, ctypes.c_int,
                                    _dp, _dp]
    lib.oracle_fwd_rows.restype = None
    lib.oracle_probs.argtypes = [_dp, _dp, ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                 ctypes.c_int, _dp]
    lib.oracle_probs.restype = None
    lib.oracle_bwd.argtypes = [_dp, _dp, _dp, _dp, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                               ctypes.c_int, ctypes.c_double, ctypes.c_int, _dp, _dp, _dp, _dp]
    lib.oracle_bwd.restype = ctypes.c_double
    lib.oracle_online_fwd.argtypes = [_dp, _dp, _dp, ctypes.c_int, ctypes.c_int,
                                      ctypes.c_double, ctypes.c_int, ctypes.c_int, _dp, _dp]
    lib.oracle_online_fwd.restype = None
    lib.oracle_loss.argtypes = [_dp, _dp, _dp, _dp, ctypes.c_int, ctypes.c_int,
                                ctypes.c_double, ctypes.c_int]
    lib.oracle_loss.restype = ctypes.c_double
    lib.oracle_decode.argtypes = [_dp, _dp, _dp, _ip, ctypes.c_int, ctypes.c_int,
                                  ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                  ctypes.c_int, _dp, _dp]
    lib.oracle_decode.restype = None
    lib.oracle_gemm.argtypes = [_dp, _dp, _dp, ctypes.c_int, ctypes.c_int, ctypes.c_int]
    lib.oracle_gemm.restype = None
    lib.oracle_num_threads.argtypes = []
    lib.oracle_num_threads.restype = ctypes.c_int
    lib.oracle_set_num_threads.argtypes = [ctypes.c_int]
    lib.oracle_set_num_threads.restype = None
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = bind(ctypes.CDLL(build()))
    return _lib


def _f64(a) -> np.ndarray:
    """Any array-like (numpy, or a CPU torch tensor of any float dtype) as a
    C-contiguous float64 numpy array.  bf16 torch tensors are widened exactly."""
    if hasattr(a, "detach"):  # torch tensor
        a = a.detach().to("cpu")
        import torch  # local: the oracle itself never needs torch
        a = a.to(torch.float64).numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


def _p(a: np.ndarray):
    return a.ctypes.data_as(_dp)


def _shape4(q: np.ndarray):
    if q.ndim != 4:
        raise ValueError("expected [B, H, N, d]")
    return q.shape


def default_scale(d: int) -> float:
    """1/sqrt(d_k), with d_k = d (the scaling of §8.1 of the first page)."""
    return 1.0 / float(np.sqrt(d))


def fwd(q, k, v, scale=None, causal=False):
    """O [B,H,N,d] and lse [B,H,N] (natural log) in fp64."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, d = _shape4(q)
    scale = default_scale(d) if scale is None else float(scale)
    o = np.empty_like(q)
    lse = np.empty((B, H, N), dtype=np.float64)
    _load().oracle_fwd(_p(q), _p(k), _p(v), B, H, N, d, scale, int(bool(causal)), _p(o), _p(lse))
    return o, lse


def fwd_rows(q_head, k_head, v_head, rows, scale, causal=False):
    """O and lse for selected query rows of one head ([N,d] arrays)."""
    q, k, v = _f64(q_head), _f64(k_head), _f64(v_head)
    N, d = q.shape
    rows = np.ascontiguousarray(rows, dtype=np.int32)
    if rows.size and (rows.min() < 0 or rows.max() >= N):
        raise ValueError("row index out of range")
    o = np.empty((rows.size, d), dtype=np.float64)
    lse = np.empty((rows.size,), dtype=np.float64)
    _load().oracle_fwd_rows(_p(q), _p(k), _p(v), N, d, float(scale), int(bool(causal)),
                            rows.ctypes.data_as(_ip), int(rows.size), _p(o), _p(lse))
    return o, lse


def probs(q_head, k_head, scale, causal=False):
    """The N x N probability matrix of one head (small N only)."""
    q, k = _f64(q_head), _f64(k_head)
    N, d = q.shape
    P = np.empty((N, N), dtype=np.float64)
    _load().oracle_probs(_p(q), _p(k), N, d, float(scale), int(bool(causal)), _p(P))
    return P


def bwd(q, k, v, dO, scale=None, causal=False):
    """dQ, dK, dV [B,H,N,d], D [B,H,N] and the largest gap between the two
    expressions of D (sum_j P dP and dO . O)."""
    q, k, v, dO = _f64(q), _f64(k), _f64(v), _f64(dO)
    B, H, N, d = _shape4(q)
    scale = default_scale(d) if scale is None else float(scale)
    dq, dk, dv = np.empty_like(q), np.empty_like(q), np.empty_like(q)
    D = np.empty((B, H, N), dtype=np.float64)
    gap = _load().oracle_bwd(_p(q), _p(k), _p(v), _p(dO), B, H, N, d, scale,
                             int(bool(causal)), _p(dq), _p(dk), _p(dv), _p(D))
    return dq, dk, dv, D, gap


def online_fwd(q_head, k_head, v_head, scale, causal=False, tile=128):
    """The online-softmax recurrence over key tiles of ``tile`` columns."""
    q, k, v = _f64(q_head), _f64(k_head), _f64(v_head)
    N, d = q.shape
    o = np.empty((N, d), dtype=np.float64)
    lse = np.empty((N,), dtype=np.float64)
    _load().oracle_online_fwd(_p(q), _p(k), _p(v), N, d, float(scale), int(bool(causal)),
                              int(tile), _p(o), _p(lse))
    return o, lse


def decode(q, k_cache, v_cache, scale=None, causal=False, lens=None):
    """Decode-shaped attention in fp64: q [B,H,Nq,d] against a cache
    k_cache, v_cache [B,H,L,d] whose first lens[b] rows are valid (all L when
    lens is None).  Causal: query i sees keys j <= lens[b] - Nq + i.  Returns
    O [B,H,Nq,d] and lse [B,H,Nq]; a query that sees no key gets O = 0 and
    lse = -inf."""
    q, k, v = _f64(q), _f64(k_cache), _f64(v_cache)
    B, H, Nq, d = _shape4(q)
    L = k.shape[2]
    if k.shape != (B, H, L, d) or v.shape != k.shape:
        raise ValueError("k_cache and v_cache must be [B, H, L, d] with q's B, H, d")
    lp = None
    if lens is not None:
        lens = np.ascontiguousarray(lens, dtype=np.int32)
        if lens.shape != (B,) or lens.min() < 0 or lens.max() > L:
            raise ValueError("lens must be [B] with 0 <= lens[b] <= L")
        lp = lens.ctypes.data_as(_ip)
    scale = default_scale(d) if scale is None else float(scale)
    o = np.empty((B, H, Nq, d), dtype=np.float64)
    lse = np.empty((B, H, Nq), dtype=np.float64)
    _load().oracle_decode(_p(q), _p(k), _p(v), lp, B, H, Nq, L, d, scale, int(bool(causal)),
                          _p(o), _p(lse))
    return o, lse


def gemm(a, b):
    """C = A B in fp64 for A [M, K] and B [K, N] (plain triple loop)."""
    a, b = _f64(a), _f64(b)
    if a.ndim != 2 or b.ndim != 2 or a.shape[1] != b.shape[0]:
        raise ValueError("expected A [M, K] and B [K, N]")
    M, K = a.shape
    N = b.shape[1]
    c = np.empty((M, N), dtype=np.float64)
    _load().oracle_gemm(_p(a), _p(b), _p(c), M, N, K)
    return c


def loss(q_head, k_head, v_head, dO_head, scale, causal=False) -> float:
    """sum(O * dO) for one head, for finite-difference checks."""
    q, k, v, dO = _f64(q_head), _f64(k_head), _f64(v_head), _f64(dO_head)
    N, d = q.shape
    return float(_load().oracle_loss(_p(q), _p(k), _p(v), _p(dO), N, d, float(scale),
                                     int(bool(causal))))


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def set_num_threads(n: int) -> None:
    _load().oracle_set_num_threads(int(n))
