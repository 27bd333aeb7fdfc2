"""Pins for the oracle's decode-shaped attention (``oracle.decode``): each check
ties it to something other than its own code (a closed form, the already
pinned square forward, an independent library routine, or an invariant), so
that a wrong cache length, a mask shifted by one, a stride mix-up between the
query and cache lengths, or a dropped normalisation fails one of them.
"""
import math

import numpy as np
import pytest
import torch

import oracle


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def test_single_key_returns_its_value():
    # One visible key: softmax of one score is 1, so O = V_0 and lse = s_0.
    B, H, Nq, L, d = 2, 3, 1, 5, 16
    q, k, v = _rand((B, H, Nq, d), 1), _rand((B, H, L, d), 2), _rand((B, H, L, d), 3)
    o, lse = oracle.decode(q, k, v, scale=0.3, lens=[1, 1])
    np.testing.assert_allclose(o[:, :, 0], v[:, :, 0], rtol=0, atol=1e-15)
    s0 = 0.3 * np.einsum("bhd,bhd->bh", q[:, :, 0], k[:, :, 0])
    np.testing.assert_allclose(lse[:, :, 0], s0, rtol=0, atol=1e-13)


def test_identical_keys_average_the_values():
    # Equal scores: every visible key gets weight 1/len, lse = s + ln(len).
    B, H, Nq, L, d = 2, 2, 3, 40, 8
    q = _rand((B, H, Nq, d), 4)
    k = np.broadcast_to(_rand((B, H, 1, d), 5), (B, H, L, d)).copy()
    v = _rand((B, H, L, d), 6)
    lens = [17, 40]
    o, lse = oracle.decode(q, k, v, scale=0.5, lens=lens)
    for b, n in enumerate(lens):
        np.testing.assert_allclose(o[b], np.broadcast_to(v[b, :, :n].mean(axis=1)[:, None], o[b].shape),
                                   rtol=0, atol=1e-13)
        s = 0.5 * np.einsum("hqd,hd->hq", q[b], k[b, :, 0])
        np.testing.assert_allclose(lse[b], s + math.log(n), rtol=0, atol=1e-12)


def test_two_keys_closed_form():
    # Two keys: O = sigma(s0 - s1) V_0 + sigma(s1 - s0) V_1.
    d = 4
    q = np.array([1.0, -2.0, 0.5, 3.0]).reshape(1, 1, 1, d)
    k = np.array([[0.2, 0.1, -1.0, 0.4], [-0.3, 0.5, 0.0, 1.1]]).reshape(1, 1, 2, d)
    v = np.array([[1.0, 2.0, 3.0, 4.0], [-4.0, 0.0, 2.0, 8.0]]).reshape(1, 1, 2, d)
    o, lse = oracle.decode(q, k, v, scale=1.0)
    s0, s1 = float(q[0, 0, 0] @ k[0, 0, 0]), float(q[0, 0, 0] @ k[0, 0, 1])
    w0 = 1.0 / (1.0 + math.exp(s1 - s0))
    np.testing.assert_allclose(o[0, 0, 0], w0 * v[0, 0, 0] + (1 - w0) * v[0, 0, 1], rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse[0, 0, 0], math.log(math.exp(s0) + math.exp(s1)), rtol=1e-14)


@pytest.mark.parametrize("causal", [False, True])
def test_square_case_is_the_forward(causal):
    # Nq = L with every row valid: decode is the (pinned) square forward.
    B, H, N, d = 1, 2, 70, 16
    q, k, v = _rand((B, H, N, d), 7), _rand((B, H, N, d), 8), _rand((B, H, N, d), 9)
    o, lse = oracle.decode(q, k, v, scale=0.25, causal=causal)
    o_f, lse_f = oracle.fwd(q, k, v, 0.25, causal)
    np.testing.assert_allclose(o, o_f, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse, lse_f, rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_rows_past_the_length_are_never_read(causal):
    # NaN in every cache row at or past lens[b]: results equal those on the
    # truncated cache, so nothing beyond the valid length is touched.
    B, H, Nq, L, d = 2, 2, 4, 64, 8
    q, k, v = _rand((B, H, Nq, d), 10), _rand((B, H, L, d), 11), _rand((B, H, L, d), 12)
    lens = [23, 50]
    kn, vn = k.copy(), v.copy()
    for b, n in enumerate(lens):
        kn[b, :, n:] = np.nan
        vn[b, :, n:] = np.nan
    o, lse = oracle.decode(q, kn, vn, scale=0.4, causal=causal, lens=lens)
    for b, n in enumerate(lens):
        o_t, lse_t = oracle.decode(q[b:b + 1], k[b:b + 1, :, :n], v[b:b + 1, :, :n], scale=0.4,
                                   causal=causal)
        np.testing.assert_array_equal(o[b:b + 1], o_t)
        np.testing.assert_array_equal(lse[b:b + 1], lse_t)


def test_causal_mask_ends_at_the_newest_key():
    # Query i of Nq under the causal mask equals a single non-causal query
    # against the first lens - Nq + i + 1 rows of the cache.
    B, H, Nq, L, d = 1, 3, 5, 30, 8
    q, k, v = _rand((B, H, Nq, d), 13), _rand((B, H, L, d), 14), _rand((B, H, L, d), 15)
    n = 21
    o, lse = oracle.decode(q, k, v, scale=0.6, causal=True, lens=[n])
    for i in range(Nq):
        vis = n - Nq + i + 1
        o1, lse1 = oracle.decode(q[:, :, i:i + 1], k[:, :, :vis], v[:, :, :vis], scale=0.6)
        np.testing.assert_array_equal(o[:, :, i:i + 1], o1)
        np.testing.assert_array_equal(lse[:, :, i:i + 1], lse1)


def test_rows_with_no_visible_key():
    # Causal with more queries than cache rows: the first Nq - len queries see
    # nothing (O = 0, lse = -inf); the rest see 1, 2, ... keys.
    B, H, Nq, L, d = 1, 1, 6, 6, 4
    q, k, v = _rand((B, H, Nq, d), 16), _rand((B, H, L, d), 17), _rand((B, H, L, d), 18)
    o, lse = oracle.decode(q, k, v, scale=1.0, causal=True, lens=[3])
    assert np.all(o[0, 0, :3] == 0.0) and np.all(np.isneginf(lse[0, 0, :3]))
    np.testing.assert_allclose(o[0, 0, 3], v[0, 0, 0], rtol=0, atol=1e-15)
    o0, lse0 = oracle.decode(q, k, v, scale=1.0, causal=False, lens=[0])
    assert np.all(o0 == 0.0) and np.all(np.isneginf(lse0))


def test_permuting_visible_cache_rows():
    # Without a mask the result does not depend on the order of the valid rows.
    B, H, Nq, L, d = 1, 2, 3, 48, 8
    q, k, v = _rand((B, H, Nq, d), 19), _rand((B, H, L, d), 20, 2.0), _rand((B, H, L, d), 21)
    n = 37
    perm = np.random.default_rng(22).permutation(n)
    kp, vp = k.copy(), v.copy()
    kp[:, :, :n], vp[:, :, :n] = k[:, :, perm], v[:, :, perm]
    o, lse = oracle.decode(q, k, v, lens=[n])
    o_p, lse_p = oracle.decode(q, kp, vp, lens=[n])
    np.testing.assert_allclose(o_p, o, rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse_p, lse, rtol=0, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_against_torch_sdpa_fp64(causal):
    # An independent library routine: torch's fp64 attention with an explicit
    # boolean mask built from the lengths and the bottom-right diagonal.
    B, H, Nq, L, d = 3, 2, 4, 33, 16
    q, k, v = _rand((B, H, Nq, d), 23), _rand((B, H, L, d), 24), _rand((B, H, L, d), 25)
    lens = [33, 12, 7]
    o, _ = oracle.decode(q, k, v, scale=0.2, causal=causal, lens=lens)
    j = np.arange(L)[None, :]
    i = np.arange(Nq)[:, None]
    for b, n in enumerate(lens):
        mask = (j < n) & ((j <= n - Nq + i) if causal else True)
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q[b]), torch.from_numpy(k[b]), torch.from_numpy(v[b]),
            attn_mask=torch.from_numpy(np.broadcast_to(mask, (Nq, L)).copy()), scale=0.2)
        np.testing.assert_allclose(o[b], ref.numpy(), rtol=0, atol=1e-12)
