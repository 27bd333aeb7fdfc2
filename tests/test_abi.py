"""The C ABI without a GPU: the library loads, exports every symbol the header
declares, and rejects bad arguments before touching the device."""
import os
import re

import pytest

import tiled_attention_20_b200.build as fa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    fa_build.build()
    import tiled_attention_20_b200.fa as fa
    return fa.load()


def _declared():
    text = open(os.path.join(ROOT, "include", "fa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z_0-9]+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    names = _declared()
    assert {"fa_fwd", "fa_bwd", "fa_bwd_workspace_size", "fa_strerror",
            "fa_check_device_errors"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_strerror_covers_all_codes(lib):
    import tiled_attention_20_b200.fa as fa
    for code in fa.STATUS_NAMES:
        assert fa.strerror(code) != "unknown status"
    assert fa.strerror(12345) == "unknown status"


def test_workspace_size(lib):
    import tiled_attention_20_b200.fa as fa
    ws = fa.workspace_size(2, 32, 4096, 128)
    rows = 2 * 32 * 4096
    assert ws >= rows * 128 * 4 + rows * 4 and ws % 256 == 0
    assert fa.workspace_size(0, 1, 1, 64) == 0
    assert fa.workspace_size(1, 1, 1, 96) == 0


P = 0x10000  # a fake, 16-byte aligned "device pointer": validation fails before any use


@pytest.mark.parametrize("args,code", [
    ((0, P, P, P, P, 1, 1, 1, 64, 0.1, 0), -1),        # NULL q
    ((P, P, P, P, P, 0, 1, 1, 64, 0.1, 0), -2),        # B = 0
    ((P, P, P, P, P, 1, 1, 0, 64, 0.1, 0), -2),        # N = 0
    ((P, P, P, P, P, 1, 1, 16, 96, 0.1, 0), -3),       # d = 96
    ((P, P, P, P, P, 1024, 1024, 1024, 64, 0.1, 0), -2),  # too large
    ((P + 2, P, P, P, P, 1, 1, 16, 64, 0.1, 0), -4),   # misaligned q
    ((P, P, P, P, P, 1, 1, 16, 64, -1.0, 0), -10),     # negative scale
    ((P, P, P, P, P, 1, 1, 16, 64, float("nan"), 0), -10),
])
def test_fwd_validation(lib, args, code):
    assert lib.fa_fwd(*args, None) == code


def test_bwd_validation(lib):
    base = [P] * 9 + [1, 1, 16, 64, 0.1, 0, P, 1 << 20, 0, None]
    assert lib.fa_bwd(*base[:15], 0, 1 << 20, 0, None) == -1          # NULL workspace
    bad = list(base); bad[17] = 2
    assert lib.fa_bwd(*bad) == -10                                     # grad_dtype
    bad = list(base); bad[16] = 16
    assert lib.fa_bwd(*bad) == -5                                      # workspace too small
    bad = list(base); bad[12] = 32
    assert lib.fa_bwd(*bad) == -3
    bad = list(base); bad[6] = P + 8
    assert lib.fa_bwd(*bad) == -4


def test_no_device_means_launch_error_not_crash(lib):
    """Valid arguments on a machine without a GPU: an error status, no crash."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    code = lib.fa_fwd(P, P, P, P, P, 1, 1, 16, 64, 0.125, 0, None)
    assert code in (-6, -9)


# fa_decode(q, k, v, o, lse, lens, B, H, Nq, Nk, ld_kv, d, scale, causal, num_splits,
#           workspace, workspace_bytes, stream): shape and pointer checks come
# before any device access.
@pytest.mark.parametrize("args,code", [
    ((0, P, P, P, P, None, 1, 1, 1, 64, 64, 64, 0.1, 0, 0, None, 0, None), -1),   # NULL q
    ((P, P, P, P, P, None, 1, 1, 0, 64, 64, 64, 0.1, 0, 0, None, 0, None), -2),   # Nq = 0
    ((P, P, P, P, P, None, 1, 1, 9, 64, 64, 64, 0.1, 0, 0, None, 0, None), -2),   # Nq = 9
    ((P, P, P, P, P, None, 1, 1, 1, 0, 64, 64, 0.1, 0, 0, None, 0, None), -2),    # Nk = 0
    ((P, P, P, P, P, None, 1, 1, 1, 65, 64, 64, 0.1, 0, 0, None, 0, None), -2),   # ld < Nk
    ((P, P, P, P, P, None, 300, 300, 1, 64, 64, 64, 0.1, 0, 0, None, 0, None), -2),  # B*H
    ((P, P, P, P, P, None, 1, 1, 1, 64, 64, 96, 0.1, 0, 0, None, 0, None), -3),   # d = 96
    ((P, P + 8, P, P, P, None, 1, 1, 1, 64, 64, 64, 0.1, 0, 0, None, 0, None), -4),  # misaligned k
    ((P, P, P, P, P, P + 2, 1, 1, 1, 64, 64, 64, 0.1, 0, 0, None, 0, None), -4),  # misaligned lens
    ((P, P, P, P, P, None, 1, 1, 1, 64, 64, 64, -1.0, 0, 0, None, 0, None), -10),  # scale < 0
    ((P, P, P, P, P, None, 1, 1, 1, 64, 64, 64, 0.1, 0, -1, None, 0, None), -10),  # splits < 0
])
def test_decode_validation(lib, args, code):
    assert lib.fa_decode(*args) == code


def test_decode_plan(lib):
    """The split covers every key with whole 64-key tiles, respects the
    chunk limit (16 KB of scores: 4096 / padded Nq keys), honours a forced
    split count, and fills but does not overflow one wave when that is best."""
    import tiled_attention_20_b200.fa as fa
    for BH, Nq, Nk, d in [(256, 1, 8192, 128), (32, 1, 8192, 128), (8, 4, 32768, 128),
                          (2048, 1, 1024, 64), (1, 8, 100, 128), (64, 1, 131072, 128),
                          (1, 1, 1, 64)]:
        sp, ck = fa.decode_plan(BH, Nq, Nk, d)
        nqp = 1 if Nq <= 1 else 2 if Nq <= 2 else 4 if Nq <= 4 else 8
        assert ck % 64 == 0 and 64 <= ck <= 4096 // nqp
        assert (sp - 1) * ck < Nk <= sp * ck
    # 32 heads of an 8192-key cache on 148 SMs x 2 CTAs: one full wave.
    sp, ck = fa.decode_plan(32, 1, 8192, 128)
    assert 148 * 2 * 0.9 <= 32 * sp <= 148 * 2
    # Forced counts round to whole tiles; a count above the tile count clamps.
    assert fa.decode_plan(4, 1, 3000, 128, num_splits=7) == (7, 448)
    assert fa.decode_plan(4, 1, 100, 128, num_splits=50) == (2, 64)
    assert fa.decode_plan(4, 8, 100000, 128, num_splits=1) == (196, 512)
    with pytest.raises(fa.FAError):
        fa.decode_plan(4, 9, 100, 128)


# fa_fwd_fp8(q, k, v, dq, dk, dv, o, lse, B, H, N, d, scale, causal, stream)
@pytest.mark.parametrize("args,code", [
    ((P, P, P, 0, P, P, P, P, 1, 1, 16, 128, 0.1, 0, None), -1),      # NULL descale_q
    ((P, P, P, P, P, P, P, P, 1, 1, 16, 64, 0.1, 0, None), -3),       # d = 64 (FP8 is d = 128)
    ((P, P, P, P, P, P, P, P, 0, 1, 16, 128, 0.1, 0, None), -2),      # B = 0
    ((P, P, P + 4, P, P, P, P, P, 1, 1, 16, 128, 0.1, 0, None), -4),  # misaligned v
    ((P, P, P, P + 1, P, P, P, P, 1, 1, 16, 128, 0.1, 0, None), -4),  # misaligned descale
    ((P, P, P, P, P, P, P, P, 1, 1, 16, 128, float("nan"), 0, None), -10),  # scale NaN
])
def test_fwd_fp8_validation(lib, args, code):
    assert lib.fa_fwd_fp8(*args) == code


def test_gemm_tiles(lib):
    """Tile width 256 once a 256-wide tiling still covers every SM, else 128;
    the lecture's 1792 -> 1793 example in 256 x 128 tiles is 98 -> 120 tiles."""
    import tiled_attention_20_b200.fa as fa
    assert fa.gemm_tiles(1792, 1792, 108) == (128, 7, 14)    # 98 tiles
    assert fa.gemm_tiles(1793, 1793, 108) == (128, 8, 15)    # 120 tiles
    assert fa.gemm_tiles(8192, 8192, 148) == (256, 32, 32)   # 1024 >= 148
    assert fa.gemm_tiles(2048, 2048, 148) == (128, 8, 16)    # 64 wide tiles < 148
    assert fa.gemm_tiles(3328, 3328, 148) == (256, 13, 13)   # 169 >= 148
    with pytest.raises(fa.FAError):
        fa.gemm_tiles(0, 5, 148)


def test_fwd_schedule_values(lib):
    """Causal B=2 H=32 N=4096: 16 tile pairs per head; the single-pair tail
    needs R * 16 >= 2 * 148, R = 8 << s, so s = 2 and R = 32: 32 heads of 8
    merged items and 32 heads of 16 single pairs.  B=8 H=16 N=8192: 32 pairs,
    R = 16 (16 * 32 = 512 >= 296), 112 merged heads.  No merging for
    non-causal problems, an odd pair count, fewer than 8 pairs, or heads not
    outnumbering the tail."""
    import tiled_attention_20_b200.fa as fa
    assert fa.fwd_schedule(2, 32, 4096, True) == (32 * 8 + 32 * 16, 32, 2)
    assert fa.fwd_schedule(8, 16, 8192, True) == (112 * 16 + 16 * 32, 112, 0)
    assert fa.fwd_schedule(2, 32, 4096, False) == (64 * 16, 0, 0)
    assert fa.fwd_schedule(2, 20, 2300, True) == (40 * 9, 0, 0)      # 9 pairs: odd
    assert fa.fwd_schedule(16, 16, 1024, True) == (256 * 4, 0, 0)    # 4 pairs
    assert fa.fwd_schedule(1, 16, 16384, True) == (16 * 64, 0, 0)    # 16 heads <= R = 32
    assert fa.fwd_schedule(1, 16, 6656, True) == (3 * 13 + 13 * 26, 3, 0)
    with pytest.raises(fa.FAError):
        fa.fwd_schedule(0, 1, 256, True)
    with pytest.raises(fa.FAError):
        fa.fwd_schedule(1, 1, 256, True, sms=0)


def test_fwd_schedule_rule(lib):
    """The defining properties of the schedule over many shapes and SM
    counts: merging only for causal problems with an even pair count P >= 8;
    the single-pair tail is R = (P/2) << s heads with s the smallest shift
    giving R * P >= 2 * sms; the item count adds up."""
    import tiled_attention_20_b200.fa as fa
    for sms in (1, 7, 108, 132, 148):
        for BH in (1, 3, 8, 16, 33, 64, 100, 128, 257):
            for N in (1, 256, 1792, 1793, 2048, 2300, 4000, 4096, 6656, 8192, 16384):
                P = (N + 255) // 256
                for causal in (False, True):
                    items, h1, s = fa.fwd_schedule(1, BH, N, causal, sms)
                    eligible = causal and P >= 8 and P % 2 == 0
                    if not eligible:
                        assert (items, h1, s) == (BH * P, 0, 0)
                        continue
                    half = P // 2
                    s_min = 0
                    while (half << s_min) * P < 2 * sms:
                        s_min += 1
                    assert s == (s_min if h1 else 0)
                    R = half << s_min
                    assert h1 == (BH - R if BH > R else 0)
                    assert items == h1 * half + (BH - h1) * P
                    if h1:
                        assert (half << s) * P >= 2 * sms
                        assert s == 0 or (half << (s - 1)) * P < 2 * sms


def test_selftest_limit_validation(lib):
    assert lib.fa_selftest_wait_timeout(0, None) == -10
    assert lib.fa_selftest_wait_timeout(2001, None) == -10
