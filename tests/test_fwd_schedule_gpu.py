"""The persistent forward's causal schedule on the GPU: every Q tile of every
head must be computed exactly once with its own head's K and V, whether its
tile pair was dealt alone or merged with the complementary pair of the same
head.  One row of every 128-row Q tile of every head (at a different offset
in each tile) is checked against the fp64 oracle, on shapes where the
schedule merges pairs (an even number of tile pairs >= 8 and more heads than
the single-pair tail) and on shapes where it does not."""
import numpy as np
import pytest
import torch

import oracle
from tiled_attention_20_b200 import inputs
from tests.parity import assert_close, np64

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _rows_per_tile(N, salt):
    """One row in each 128-row Q tile, at an offset that varies by tile."""
    return np.array([min(N - 1, t * 128 + (37 * t + salt) % 128) for t in range((N + 127) // 128)],
                    dtype=np.int32)


def _check_all_tiles(o, lse, q, k, v, scale, tol_o, ctx):
    B, H, N, _ = q.shape
    og, lg = np64(o), np64(lse)
    for b in range(B):
        for h in range(H):
            rows = _rows_per_tile(N, b * H + h)
            ro, rl = oracle.fwd_rows(q[b, h], k[b, h], v[b, h], rows, scale, causal=True)
            assert_close("o", og[b, h, rows], ro, tol=tol_o, ctx=f"{ctx} b={b} h={h}")
            assert_close("lse", lg[b, h, rows], rl, ctx=f"{ctx} b={b} h={h}")


# (B, H, N, d): 80 heads of 8 tile pairs, 64 heads of 16 pairs and 16 heads
# of 26 pairs merge some of their heads' pairs (single-pair tails of 64, 32
# and 13 heads); 9 pairs (odd) do not.
@pytest.mark.parametrize("B,H,N,d", [(1, 80, 2048, 64), (2, 32, 4096, 128), (1, 16, 6656, 64),
                                     (2, 20, 2300, 64)],
                         ids=lambda x: str(x))
def test_every_tile_computed_bf16(B, H, N, d):
    import tiled_attention_20_b200.fa as fa
    q, k, v, _ = inputs.qkv_do(B, H, N, d, seed=21)
    o, lse = fa.fwd(q.to(DEV), k.to(DEV), v.to(DEV), causal=True)
    fa.check_device_errors()
    _check_all_tiles(o, lse, q, k, v, d ** -0.5, None, f"N={N} d={d}")


def test_every_tile_computed_fp8():
    """The E4M3 forward shares the schedule (merged at 64 heads x 16 pairs);
    a tile computed against the wrong head or not at all is off by O(1),
    far above the FP8 rounding error."""
    import tiled_attention_20_b200.fa as fa
    B, H, N, d = 2, 32, 4096, 128
    q8, k8, v8, fq, fk, fv = inputs.fp8_qkv(B, H, N, d, seed=21)
    o, lse = fa.fwd_fp8(q8.to(DEV), k8.to(DEV), v8.to(DEV), fq.to(DEV), fk.to(DEV), fv.to(DEV),
                        causal=True)
    fa.check_device_errors()
    deq = lambda x, f: x.to(torch.float64) * f.to(torch.float64)[:, :, None, None]
    _check_all_tiles(o, lse, deq(q8, fq), deq(k8, fk), deq(v8, fv), d ** -0.5, 1e-1, "fp8")
