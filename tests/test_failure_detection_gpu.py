"""Failure detection on the GPU without a fault: a kernel whose bounded wait
on an mbarrier can never complete gives up after a short limit, latches the
timeout bit, and the host reads FA_ERR_TIMEOUT; the status is cleared by the
read and the context keeps working (a forward afterwards is correct)."""
import time

import numpy as np
import pytest
import torch

import oracle
from tiled_attention_20_b200 import inputs

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_is_reported():
    import tiled_attention_20_b200.fa as fa
    dev = torch.device("cuda:0")
    fa.check_device_errors(dev)  # start clean
    t0 = time.time()
    fa.selftest_wait_timeout(50, dev)
    with pytest.raises(fa.FAError) as e:
        fa.check_device_errors(dev)
    assert e.value.status == -7  # FA_ERR_TIMEOUT
    assert time.time() - t0 < 10.0
    fa.check_device_errors(dev)  # the read cleared the word
    q, k, v, _ = inputs.qkv_do(1, 2, 300, 64, seed=3)
    o, lse = fa.fwd(q.to(dev), k.to(dev), v.to(dev), causal=True)
    fa.check_device_errors(dev)
    o_ref, _ = oracle.fwd(q, k, v, causal=True)
    assert np.abs(o.double().cpu().numpy() - o_ref).max() <= 2e-2


def test_selftest_limit_range():
    import tiled_attention_20_b200.fa as fa
    with pytest.raises(fa.FAError):
        fa.selftest_wait_timeout(0)
    with pytest.raises(fa.FAError):
        fa.selftest_wait_timeout(5000)


@pytest.mark.parametrize("d", [64, 128])
def test_consistency_checks_stay_silent_on_tiny_ragged_shapes(d):
    """The kernels' consistency checks (every forward row's softmax
    normaliser is at least 1/2 and finite; every lse the backward reads is
    finite) hold on the smallest and most ragged shapes: nothing is latched."""
    import tiled_attention_20_b200.fa as fa
    dev = torch.device("cuda:0")
    fa.check_device_errors(dev)
    for n in (1, 2, 127, 129):
        for causal in (False, True):
            for dist in ("normal", "long_context"):
                q, k, v, dO = (t.to(dev) for t in inputs.qkv_do(2, 3, n, d, seed=n, dist=dist))
                o, lse = fa.fwd(q, k, v, causal=causal)
                fa.bwd(q, k, v, o, dO, lse, causal=causal)
                fa.check_device_errors(dev)


def test_non_finite_lse_is_reported_as_device_assert():
    """An lse that no forward can produce (+inf in one row, made on the host)
    is caught by the backward's check on the device: the host reads
    FA_ERR_DEVICE_ASSERT, the read clears it, and the next call is correct.
    Nothing faults: the bad row only yields non-finite gradients."""
    import tiled_attention_20_b200.fa as fa
    dev = torch.device("cuda:0")
    fa.check_device_errors(dev)
    q, k, v, dO = (t.to(dev) for t in inputs.qkv_do(1, 2, 200, 64, seed=9))
    o, lse = fa.fwd(q, k, v, causal=True)
    bad = lse.clone()
    bad[0, 1, 57] = float("inf")
    fa.bwd(q, k, v, o, dO, bad, causal=True)
    with pytest.raises(fa.FAError) as e:
        fa.check_device_errors(dev)
    assert e.value.status == -8  # FA_ERR_DEVICE_ASSERT
    fa.check_device_errors(dev)  # cleared
    dq, dk, dv = fa.bwd(q, k, v, o, dO, lse, causal=True)
    fa.check_device_errors(dev)
    dq_r, _, _, _, _ = oracle.bwd(q.cpu(), k.cpu(), v.cpu(), dO.cpu(), causal=True)
    assert np.abs(dq.double().cpu().numpy() - dq_r).max() <= 2e-2
