"""The Python binding rejects caller-supplied buffers that do not fit the
call (wrong device, dtype, shape, contiguity or size) with ValueError before
anything reaches libfa: a host pointer or a too-small buffer handed to a
kernel would fault or silently corrupt memory."""
import pytest
import torch

from tiled_attention_20_b200 import fa

CPU = torch.device("cpu")


def test_buffer_check_accepts_a_matching_tensor():
    fa._check_buffer("lse", torch.zeros(2, 3, 5), CPU, torch.float32, (2, 3, 5))
    fa._check_buffer("workspace", torch.zeros(64, dtype=torch.uint8), CPU, torch.uint8,
                     min_numel=64)


@pytest.mark.parametrize("bad, why", [
    (lambda: torch.zeros(2, 3, 5, dtype=torch.float64), "float32"),
    (lambda: torch.zeros(2, 3, 6), "shape"),
    (lambda: torch.zeros(5, 3, 2).permute(2, 1, 0), "contiguous"),
    (lambda: [0.0] * 30, "torch tensor"),
])
def test_buffer_check_rejects(bad, why):
    with pytest.raises(ValueError, match=why):
        fa._check_buffer("lse", bad(), CPU, torch.float32, (2, 3, 5))


def test_buffer_check_rejects_other_device():
    with pytest.raises(ValueError, match="must be on cuda:0"):
        fa._check_buffer("lse", torch.zeros(2, 3, 5), torch.device("cuda", 0), torch.float32,
                         (2, 3, 5))


def test_buffer_check_rejects_short_workspace():
    with pytest.raises(ValueError, match="at least 100"):
        fa._check_buffer("workspace", torch.zeros(99, dtype=torch.uint8), CPU, torch.uint8,
                         min_numel=100)


def test_grad_dtype_must_be_bf16_or_fp32():
    with pytest.raises(ValueError, match="grad_dtype"):
        fa._grad_code(torch.float16)


@pytest.mark.gpu
def test_public_calls_reject_bad_buffers_before_launch():
    """Every caller-supplied buffer of fwd, bwd and bwd_noalloc is checked."""
    dev = torch.device("cuda", 0)
    B, H, N, d = 1, 2, 64, 64
    q, k, v, o, dO = (torch.zeros(B, H, N, d, dtype=torch.bfloat16, device=dev) for _ in range(5))
    lse = torch.zeros(B, H, N, device=dev)
    cases = [
        lambda: fa.fwd(q, k, v, out=torch.zeros(B, H, N, d, dtype=torch.float32, device=dev)),
        lambda: fa.fwd(q, k, v, lse=torch.zeros(B, H, N)),
        lambda: fa.fwd(q, k, v, lse=torch.zeros(B, H, N + 1, device=dev)),
        lambda: fa.bwd(q, k, v, o, dO, torch.zeros(B, H, N)),
        lambda: fa.bwd(q, k, v, o, dO, lse, dq=torch.zeros(B, H, N, d, dtype=torch.bfloat16,
                                                            device=dev), grad_dtype=torch.float32),
        lambda: fa.bwd(q, k, v, o, dO, lse, dk=torch.zeros(B, H, N, d, dtype=torch.bfloat16)),
        lambda: fa.bwd(q, k, v, o, dO, lse, dv=torch.zeros(B, H, 2 * N, d, dtype=torch.bfloat16,
                                                            device=dev)),
        lambda: fa.bwd(q, k, v, o, dO, lse, workspace=torch.zeros(16, dtype=torch.uint8,
                                                                   device=dev)),
        lambda: fa.bwd_noalloc(q, k, v, o, dO, torch.zeros(B, H, N, dtype=torch.float64,
                                                            device=dev)),
        lambda: fa.bwd_noalloc(q, k, v, o, dO, lse, dq=torch.zeros(B, H, N, d, device=dev)),
    ]
    for i, call in enumerate(cases):
        with pytest.raises(ValueError):
            call()
            pytest.fail(f"case {i} was not rejected")


def test_trace_start_rejects_unknown_kernel_names():
    with pytest.raises(ValueError, match="unknown kernel"):
        fa.trace_start(["fa_no_such_kernel"])
