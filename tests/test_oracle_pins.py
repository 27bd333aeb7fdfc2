"""Pins for the fp64 oracle: each check ties it to something other than itself
(a closed form, an invariant of the mathematics, a second formulation the
pages give, an independent library routine, or finite differences), so that a
dropped term, a wrong sign or index, or a transposed operand fails one of them.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from tiled_attention_20_b200 import inputs


def _rand(shape, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    return rng.standard_normal(shape) * scale


# --- the online recurrence (first page §8.3) equals the three-pass definition ---

@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("tile", [1, 7, 64, 128])
def test_online_softmax_equals_three_pass(causal, tile):
    N, d = 300, 32
    q, k, v = _rand((N, d), 1), _rand((N, d), 2, 2.0), _rand((N, d), 3)
    scale = 1 / math.sqrt(d)
    o_ref, lse_ref = oracle.fwd(q[None, None], k[None, None], v[None, None], scale, causal)
    o_on, lse_on = oracle.online_fwd(q, k, v, scale, causal, tile)
    np.testing.assert_allclose(o_on, o_ref[0, 0], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse_on, lse_ref[0, 0], rtol=1e-12, atol=1e-12)


# --- softmax rows: non-negative, sum to one, zero above the diagonal when causal ---

@pytest.mark.parametrize("causal", [False, True])
def test_probability_rows(causal):
    N, d = 97, 16
    q, k = _rand((N, d), 4, 3.0), _rand((N, d), 5, 3.0)
    P = oracle.probs(q, k, 0.25, causal)
    assert (P >= 0).all()
    np.testing.assert_allclose(P.sum(axis=1), 1.0, rtol=0, atol=1e-14)
    if causal:
        assert np.all(np.triu(P, 1) == 0.0)
        assert np.all(np.diag(P) > 0)
    # P matches its definition entry by entry (a direct exp-normalise).
    s = 0.25 * q @ k.T
    if causal:
        s = np.where(np.tril(np.ones((N, N), bool)), s, -np.inf)
    e = np.exp(s - s.max(axis=1, keepdims=True))
    np.testing.assert_allclose(P, e / e.sum(axis=1, keepdims=True), rtol=1e-12, atol=1e-15)


# --- causal row 0 sees only key 0: O_0 = V_0 and lse_0 = scale q_0.k_0 exactly ---

def test_causal_row0_exact():
    B, H, N, d = 2, 3, 40, 64
    q, k, v = _rand((B, H, N, d), 6), _rand((B, H, N, d), 7), _rand((B, H, N, d), 8)
    scale = 0.125
    o, lse = oracle.fwd(q, k, v, scale, causal=True)
    assert np.array_equal(o[:, :, 0], v[:, :, 0])
    s00 = scale * np.einsum("bhc,bhc->bh", q[:, :, 0], k[:, :, 0])
    np.testing.assert_allclose(lse[:, :, 0], s00, rtol=1e-15, atol=1e-15)


# --- uniform scores (Q = 0): O is the mean of the visible V rows, lse = ln(count) ---

@pytest.mark.parametrize("causal", [False, True])
def test_uniform_scores(causal):
    B, H, N, d = 1, 2, 33, 8
    q = np.zeros((B, H, N, d))
    k, v = _rand((B, H, N, d), 9), _rand((B, H, N, d), 10)
    o, lse = oracle.fwd(q, k, v, 0.3, causal)
    for i in range(N):
        cnt = i + 1 if causal else N
        np.testing.assert_allclose(o[:, :, i], v[:, :, :cnt].mean(axis=2), rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(lse[:, :, i], math.log(cnt), rtol=0, atol=1e-13)


# --- key-shift invariance: adding c to every K row leaves O unchanged and shifts
#     lse_i by scale q_i.c; its derivative says sum_j dK_j = 0 per head ---

@pytest.mark.parametrize("causal", [False, True])
def test_key_shift_invariance(causal):
    B, H, N, d = 1, 2, 50, 16
    q, k, v = _rand((B, H, N, d), 11), _rand((B, H, N, d), 12), _rand((B, H, N, d), 13)
    c = _rand((d,), 14)
    scale = 0.2
    o1, lse1 = oracle.fwd(q, k, v, scale, causal)
    o2, lse2 = oracle.fwd(q, k + c, v, scale, causal)
    np.testing.assert_allclose(o2, o1, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(lse2 - lse1, scale * q @ c, rtol=1e-11, atol=1e-11)


@pytest.mark.parametrize("causal", [False, True])
def test_gradient_sum_rules(causal):
    B, H, N, d = 2, 2, 45, 16
    q, k, v, dO = (_rand((B, H, N, d), s) for s in (15, 16, 17, 18))
    dq, dk, dv, D, gap = oracle.bwd(q, k, v, dO, 0.25, causal)
    # sum_j dK_j = 0: key-shift invariance
    np.testing.assert_allclose(dk.sum(axis=2), 0.0, atol=1e-12)
    # sum_j dV_j = sum_i dO_i: rows of P sum to one
    np.testing.assert_allclose(dv.sum(axis=2), dO.sum(axis=2), rtol=1e-12, atol=1e-12)
    # D computed as sum_j P dP agrees with rowsum(dO * O)
    assert gap < 1e-12
    o, _ = oracle.fwd(q, k, v, 0.25, causal)
    np.testing.assert_allclose(D, (dO * o).sum(axis=3), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_dS_rows_sum_to_zero(causal):
    """With every key row equal to the same vector c, dQ_i = scale c sum_j dS_ij,
    which is zero because the rows of dS sum to zero."""
    B, H, N, d = 1, 1, 30, 8
    q, v, dO = _rand((B, H, N, d), 19), _rand((B, H, N, d), 20), _rand((B, H, N, d), 21)
    k = np.broadcast_to(_rand((d,), 22), (B, H, N, d)).copy()
    dq, _, _, _, _ = oracle.bwd(q, k, v, dO, 0.5, causal)
    np.testing.assert_allclose(dq, 0.0, atol=1e-13)


# --- closed form, d = 1, N = 2 ---

def test_closed_form_two_keys():
    q = np.array([[0.7], [-1.1]])
    k = np.array([[0.4], [2.0]])
    v = np.array([[3.0], [-5.0]])
    scale = 0.9
    o, lse = oracle.fwd(q[None, None], k[None, None], v[None, None], scale, causal=False)
    for i in range(2):
        a, b = scale * q[i, 0] * k[0, 0], scale * q[i, 0] * k[1, 0]
        want = (math.exp(a) * v[0, 0] + math.exp(b) * v[1, 0]) / (math.exp(a) + math.exp(b))
        assert abs(o[0, 0, i, 0] - want) < 1e-15
        assert abs(lse[0, 0, i] - math.log(math.exp(a) + math.exp(b))) < 1e-15
    oc, _ = oracle.fwd(q[None, None], k[None, None], v[None, None], scale, causal=True)
    assert oc[0, 0, 0, 0] == v[0, 0]
    a, b = scale * q[1, 0] * k[0, 0], scale * q[1, 0] * k[1, 0]
    want1 = (math.exp(a) * v[0, 0] + math.exp(b) * v[1, 0]) / (math.exp(a) + math.exp(b))
    assert abs(oc[0, 0, 1, 0] - want1) < 1e-15


# --- central finite differences of L = sum(O * dO) against the analytic gradient ---

@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 2, 3, 5, 8])
@pytest.mark.parametrize("d", [1, 4])
def test_finite_differences(causal, N, d):
    q, k, v, dO = (_rand((N, d), 100 + s + 10 * N + d) for s in range(4))
    scale = 0.7
    dq, dk, dv, _, _ = oracle.bwd(q[None, None], k[None, None], v[None, None], dO[None, None],
                                  scale, causal)
    h = 1e-6
    for name, x, g in (("q", q, dq[0, 0]), ("k", k, dk[0, 0]), ("v", v, dv[0, 0])):
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = {"q": q, "k": k, "v": v}
            args_m = {"q": q, "k": k, "v": v}
            args_p[name], args_m[name] = xp, xm
            Lp = oracle.loss(args_p["q"], args_p["k"], args_p["v"], dO, scale, causal)
            Lm = oracle.loss(args_m["q"], args_m["k"], args_m["v"], dO, scale, causal)
            fd[idx] = (Lp - Lm) / (2 * h)
        np.testing.assert_allclose(g, fd, rtol=1e-7, atol=1e-8, err_msg=name)


# --- an independent library routine: torch's fp64 CPU attention and autograd ---

@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,d", [(1, 64), (129, 64), (200, 128)])
def test_against_torch_sdpa_fp64(causal, N, d):
    B, H = 2, 2
    q, k, v, dO = (torch.from_numpy(_rand((B, H, N, d), 200 + s)) for s in range(4))
    scale = 1 / math.sqrt(d)
    qt, kt, vt = (t.clone().requires_grad_(True) for t in (q, k, v))
    ot = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=causal,
                                                          scale=scale)
    ot.backward(dO)
    o, lse = oracle.fwd(q.numpy(), k.numpy(), v.numpy(), scale, causal)
    np.testing.assert_allclose(o, ot.detach().numpy(), rtol=1e-10, atol=1e-12)
    dq, dk, dv, _, _ = oracle.bwd(q.numpy(), k.numpy(), v.numpy(), dO.numpy(), scale, causal)
    np.testing.assert_allclose(dq, qt.grad.numpy(), rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(dk, kt.grad.numpy(), rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(dv, vt.grad.numpy(), rtol=1e-9, atol=1e-11)
    s = scale * torch.einsum("bhid,bhjd->bhij", q, k)
    if causal:
        s = s.masked_fill(~torch.ones(N, N, dtype=torch.bool).tril(), float("-inf"))
    np.testing.assert_allclose(lse, torch.logsumexp(s, dim=-1).numpy(), rtol=1e-12, atol=1e-12)


def test_selected_rows_match_full_forward():
    B, H, N, d = 1, 1, 77, 32
    q, k, v = (_rand((B, H, N, d), 300 + s) for s in range(3))
    for causal in (False, True):
        o, lse = oracle.fwd(q, k, v, 0.3, causal)
        rows = np.array([0, 5, 76, 33])
        orow, lrow = oracle.fwd_rows(q[0, 0], k[0, 0], v[0, 0], rows, 0.3, causal)
        np.testing.assert_array_equal(orow, o[0, 0, rows])
        np.testing.assert_array_equal(lrow, lse[0, 0, rows])


def test_large_logits_stay_finite():
    """Scores of several hundred (the long-context distribution) must not
    overflow: the row maximum is subtracted before exponentiating."""
    q, k, v, _ = inputs.qkv_do(1, 1, 300, 64, seed=3, dist="long_context")
    o, lse = oracle.fwd(q, k, v, 1 / 8.0, causal=True)
    assert np.isfinite(o).all() and np.isfinite(lse).all()
    o_on, lse_on = oracle.online_fwd(q[0, 0], k[0, 0], v[0, 0], 1 / 8.0, True, 128)
    np.testing.assert_allclose(o_on, o[0, 0], rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(lse_on, lse[0, 0], rtol=1e-12, atol=1e-12)
