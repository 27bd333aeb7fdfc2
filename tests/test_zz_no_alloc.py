"""fa_bwd_noalloc: the backward for callers that cannot allocate device memory
(a plugin whose host framework owns all device memory, or a path where the
implicit synchronisation of cudaMalloc is not allowed).  It takes its scratch
from a fixed array inside the library instead of a caller workspace; its
results must match fa_bwd's.

This file is named to be collected last, so that a run stopping at the first
failure has already run every other test."""

import pytest
import torch

from tests.parity import TOL, max_abs
from tiled_attention_20_b200 import inputs

P = 0x10000  # fake 16-byte-aligned pointer: rejected before any device use


def _lib():
    from tiled_attention_20_b200 import build as fa_build
    fa_build.build()
    import tiled_attention_20_b200.fa as fa
    return fa, fa.load()


def test_noalloc_rejects_oversized_problem_before_launch():
    """A problem needing more scratch than the fixed maximum is refused with
    FA_ERR_NOALLOC_LIMIT, without touching the device (runs without a GPU)."""
    fa, lib = _lib()
    B, H, N, d = 2, 32, 4096, 128
    assert fa.workspace_size(B, H, N, d) > fa.NOALLOC_MAX_SCRATCH
    rc = lib.fa_bwd_noalloc(P, P, P, P, P, P, P, P, P, B, H, N, d, 0.088, 1, 0, None)
    assert rc == -11 and "fixed maximum" in fa.strerror(rc)
    rc = lib.fa_bwd_noalloc(0, P, P, P, P, P, P, P, P, 1, 1, 16, 64, 0.1, 0, 0, None)
    assert rc == -1


@pytest.mark.gpu
@pytest.mark.parametrize("causal", [False, True])
def test_noalloc_matches_workspace_backward_twice(causal):
    """Calls in a row through the C ABI, each compared with fa_bwd on the same
    inputs; no call may see an earlier call's scratch.  The third call
    repeats the first shape, so its counters sit exactly where the first
    call left its own: a counter that was not cleared would change it."""
    fa, _ = _lib()
    dev = "cuda:0"
    for call, (B, H, N, d) in enumerate([(1, 3, 300, 128), (2, 2, 777, 64), (1, 3, 300, 128)]):
        q, k, v, dO = (t.to(dev) for t in inputs.qkv_do(B, H, N, d, seed=40 + call))
        o, lse = fa.fwd(q, k, v, causal=causal)
        ref = fa.bwd(q, k, v, o, dO, lse, causal=causal)
        got = fa.bwd_noalloc(q, k, v, o, dO, lse, causal=causal)
        fa.check_device_errors()
        for name, a, b in zip(("dq", "dk", "dv"), got, ref):
            err = max_abs(a, b)
            assert err <= TOL[name], f"call {call}: {name} differs by {err:.3e}"
        # dK and dV are deterministic: the same kernels on the same inputs
        assert torch.equal(got[1], ref[1]) and torch.equal(got[2], ref[2])
