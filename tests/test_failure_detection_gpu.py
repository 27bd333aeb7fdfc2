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
