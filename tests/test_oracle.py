"""Pins for the fp64 oracle: closed forms, invariants, special cases, brute force.

Each check is chosen so that a plausible mistake in the oracle (a dropped term,
a wrong sign or index, a transposed operand, a missing scale, the normalisation
slip of the pages' blockwise listing) fails at least one of them.  None of them
calls the CUDA path.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import (attention_bwd, attention_bwd_gqa, attention_bwd_sampled, attention_fwd, attention_fwd_blockwise,
                    attention_fwd_decode, attention_fwd_gqa, attention_fwd_rows, bwd_operand_rounding_bound,
                    softmax_merge)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _rand(shape, seed, mult=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * mult


def _bhnd(x):
    x = np.asarray(x, dtype=np.float64)
    return x[None, None]


# --- worked closed forms (tests/golden) ------------------------------------

@pytest.mark.parametrize("causal", [False, True])
def test_golden_forward(causal):
    g = json.load(open(os.path.join(GOLDEN, "closed_form_fwd.json")))
    o, lse = attention_fwd(_bhnd(g["q"]), _bhnd(g["k"]), _bhnd(g["v"]),
                           g["scale"], causal)
    exp = g["causal" if causal else "noncausal"]
    np.testing.assert_allclose(o[0, 0], exp["o"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse[0, 0], exp["lse"], rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_golden_backward(causal):
    g = json.load(open(os.path.join(GOLDEN, "closed_form_bwd.json")))
    dq, dk, dv = attention_bwd(_bhnd(g["q"]), _bhnd(g["k"]), _bhnd(g["v"]),
                               _bhnd(g["do"]), g["scale"], causal)
    exp = g["causal" if causal else "noncausal"]
    np.testing.assert_allclose(dq[0, 0], exp["dq"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(dk[0, 0], exp["dk"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(dv[0, 0], exp["dv"], rtol=0, atol=1e-12)


def test_two_key_sigmoid_closed_form_random():
    """With two keys softmax is a sigmoid; O, lse and all gradients in closed form."""
    rng = np.random.default_rng(5)
    N, d, scale = 2, 3, 0.7
    q, k, v, do = (rng.standard_normal((N, d)) for _ in range(4))
    o, lse = attention_fwd(_bhnd(q), _bhnd(k), _bhnd(v), scale, False)
    dq, dk, dv = attention_bwd(_bhnd(q), _bhnd(k), _bhnd(v), _bhnd(do), scale, False)
    s = scale * np.array([[q[i] @ k[j] for j in range(N)] for i in range(N)])
    p1 = 1.0 / (1.0 + np.exp(-(s[:, 1] - s[:, 0])))
    o_cf = v[0][None, :] + p1[:, None] * (v[1] - v[0])[None, :]
    lse_cf = s[:, 0] + np.log1p(np.exp(s[:, 1] - s[:, 0]))
    g = (do @ (v[1] - v[0])) * p1 * (1 - p1)
    dq_cf = scale * g[:, None] * (k[1] - k[0])[None, :]
    dk1 = scale * (g[:, None] * q).sum(0)
    dv0 = ((1 - p1)[:, None] * do).sum(0)
    dv1 = (p1[:, None] * do).sum(0)
    np.testing.assert_allclose(o[0, 0], o_cf, atol=1e-12)
    np.testing.assert_allclose(lse[0, 0], lse_cf, atol=1e-12)
    np.testing.assert_allclose(dq[0, 0], dq_cf, atol=1e-12)
    np.testing.assert_allclose(dk[0, 0], np.stack([-dk1, dk1]), atol=1e-12)
    np.testing.assert_allclose(dv[0, 0], np.stack([dv0, dv1]), atol=1e-12)


# --- invariants and special cases ------------------------------------------

@pytest.mark.parametrize("causal", [False, True])
def test_probability_rows_sum_to_one(causal):
    """With V = identity (d = N) the output rows ARE the rows of P."""
    N = 37
    q, k = _rand((1, 2, N, N), 1), _rand((1, 2, N, N), 2)
    v = np.broadcast_to(np.eye(N), (1, 2, N, N))
    p, _ = attention_fwd(q, k, v, 0.3, causal)
    np.testing.assert_allclose(p.sum(-1), 1.0, rtol=0, atol=1e-12)
    assert (p >= 0).all()
    if causal:
        upper = np.triu(np.ones((N, N), bool), k=1)
        assert (p[..., upper] == 0).all()
        np.testing.assert_allclose(p[..., 0, 0], 1.0, atol=0)


def test_single_key_gives_v_and_dot_lse():
    q, k, v = _rand((2, 3, 1, 8), 3), _rand((2, 3, 1, 8), 4), _rand((2, 3, 1, 8), 5)
    for causal in (False, True):
        o, lse = attention_fwd(q, k, v, 0.25, causal)
        np.testing.assert_allclose(o, v, rtol=0, atol=1e-15)
        np.testing.assert_allclose(lse, 0.25 * (q * k).sum(-1), atol=1e-14)


def test_causal_row_zero():
    q, k, v = _rand((2, 2, 50, 16), 6), _rand((2, 2, 50, 16), 7), _rand((2, 2, 50, 16), 8)
    o, lse = attention_fwd(q, k, v, 0.25, True)
    np.testing.assert_allclose(o[:, :, 0], v[:, :, 0], atol=1e-15)
    np.testing.assert_allclose(lse[:, :, 0], 0.25 * (q[:, :, 0] * k[:, :, 0]).sum(-1), atol=1e-14)


@pytest.mark.parametrize("causal", [False, True])
def test_constant_v_gives_constant_o(causal):
    q, k = _rand((1, 3, 70, 16), 9, 3.0), _rand((1, 3, 70, 16), 10, 3.0)
    row = _rand((16,), 11)
    v = np.broadcast_to(row, (1, 3, 70, 16)).copy()
    o, _ = attention_fwd(q, k, v, 0.25, causal)
    np.testing.assert_allclose(o, v, rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_zero_q_uniform_weights(causal):
    N = 33
    q = np.zeros((1, 2, N, 8))
    k, v = _rand((1, 2, N, 8), 12), _rand((1, 2, N, 8), 13)
    o, lse = attention_fwd(q, k, v, 0.35, causal)
    if causal:
        cnt = np.arange(1, N + 1)
        exp_o = np.cumsum(v, axis=2) / cnt[None, None, :, None]
        exp_lse = np.broadcast_to(np.log(cnt), (1, 2, N))
    else:
        exp_o = np.broadcast_to(v.mean(axis=2, keepdims=True), v.shape)
        exp_lse = np.full((1, 2, N), math.log(N))
    np.testing.assert_allclose(o, exp_o, atol=1e-12)
    np.testing.assert_allclose(lse, exp_lse, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_key_shift_invariance(causal):
    q, k, v = _rand((1, 2, 40, 8), 14), _rand((1, 2, 40, 8), 15), _rand((1, 2, 40, 8), 16)
    u = _rand((8,), 17)
    o1, l1 = attention_fwd(q, k, v, 0.4, causal)
    o2, l2 = attention_fwd(q, k + u, v, 0.4, causal)
    np.testing.assert_allclose(o2, o1, atol=1e-10)
    np.testing.assert_allclose(l2, l1 + 0.4 * (q @ u), atol=1e-10)


def test_joint_key_value_permutation_invariance():
    q, k, v = _rand((2, 2, 45, 8), 18), _rand((2, 2, 45, 8), 19), _rand((2, 2, 45, 8), 20)
    perm = np.random.default_rng(21).permutation(45)
    o1, l1 = attention_fwd(q, k, v, 0.3, False)
    o2, l2 = attention_fwd(q, k[:, :, perm], v[:, :, perm], 0.3, False)
    np.testing.assert_allclose(o2, o1, atol=1e-12)
    np.testing.assert_allclose(l2, l1, atol=1e-12)


def test_scale_is_applied_to_scores():
    """Multiplying K by c is the same as multiplying the scale by c."""
    q, k, v = _rand((1, 1, 20, 8), 22), _rand((1, 1, 20, 8), 23), _rand((1, 1, 20, 8), 24)
    o1, l1 = attention_fwd(q, 3.0 * k, v, 0.2, True)
    o2, l2 = attention_fwd(q, k, v, 0.6, True)
    np.testing.assert_allclose(o1, o2, atol=1e-12)
    np.testing.assert_allclose(l1, l2, atol=1e-12)


def test_row_panels_match_whole_rows():
    q, k, v = _rand((1, 2, 300, 16), 25), _rand((1, 2, 300, 16), 26), _rand((1, 2, 300, 16), 27)
    for causal in (False, True):
        o1, l1 = attention_fwd(q, k, v, 0.25, causal, panel_rows=4096)
        o2, l2 = attention_fwd(q, k, v, 0.25, causal, panel_rows=7)
        np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-14)
        np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-14)


def test_sampled_rows_match_full():
    q, k, v = _rand((1, 1, 257, 16), 28), _rand((1, 1, 257, 16), 29), _rand((1, 1, 257, 16), 30)
    rows = np.array([0, 5, 128, 256])
    for causal in (False, True):
        o, l = attention_fwd(q, k, v, 0.25, causal)
        o_r, l_r = attention_fwd_rows(q[0, 0, rows], k[0, 0], v[0, 0], rows, 0.25, causal)
        np.testing.assert_allclose(o_r, o[0, 0, rows], atol=1e-14)
        np.testing.assert_allclose(l_r, l[0, 0, rows], atol=1e-14)


# --- an independent library routine ----------------------------------------

@pytest.mark.parametrize("causal", [False, True])
def test_matches_torch_sdpa_fp64(causal):
    """torch's own scaled-dot-product attention (CPU, float64) and its autograd."""
    B, H, N, d, scale = 2, 3, 67, 16, 0.21
    q, k, v, do = (_rand((B, H, N, d), 31 + i) for i in range(4))
    o, lse = attention_fwd(q, k, v, scale, causal)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    to = torch.nn.functional.scaled_dot_product_attention(
        tq, tk, tv, is_causal=causal, scale=scale)
    np.testing.assert_allclose(o, to.detach().numpy(), atol=1e-12)
    s = scale * (tq @ tk.transpose(-1, -2))
    if causal:
        s = s.masked_fill(torch.ones(N, N, dtype=torch.bool).triu(1), float("-inf"))
    np.testing.assert_allclose(lse, torch.logsumexp(s, -1).detach().numpy(), atol=1e-12)
    to.backward(torch.tensor(do))
    dq, dk, dv = attention_bwd(q, k, v, do, scale, causal)
    np.testing.assert_allclose(dq, tq.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dk, tk.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dv, tv.grad.numpy(), atol=1e-11)


# --- brute force: finite differences ---------------------------------------

@pytest.mark.parametrize("causal", [False, True])
def test_gradients_by_central_differences(causal):
    N, d, scale, h = 6, 3, 0.8, 1e-6
    q, k, v, do = (_rand((1, 1, N, d), 40 + i) for i in range(4))
    dq, dk, dv = attention_bwd(q, k, v, do, scale, causal)

    def loss(qq, kk, vv):
        o, _ = attention_fwd(qq, kk, vv, scale, causal)
        return float((o * do).sum())

    for which, grad in ((0, dq), (1, dk), (2, dv)):
        fd = np.zeros_like(grad)
        for idx in np.ndindex(grad.shape):
            args = [q.copy(), k.copy(), v.copy()]
            args[which][idx] += h
            lp = loss(*args)
            args[which][idx] -= 2 * h
            lm = loss(*args)
            fd[idx] = (lp - lm) / (2 * h)
        rel = np.abs(fd - grad).max() / max(np.abs(grad).max(), 1e-30)
        assert rel < 1e-6, (which, rel)


def test_delta_identity():
    """sum_j P_ij dP_ij == sum_c dO_ic O_ic (the D term of the backward)."""
    N, d = 30, 8
    q, k, v, do = (_rand((1, 1, N, d), 50 + i) for i in range(4))
    p, _ = attention_fwd(q, k, np.broadcast_to(np.eye(N), (1, 1, N, N)), 0.3, True)
    o, _ = attention_fwd(q, k, v, 0.3, True)
    dp = do[0, 0] @ v[0, 0].T
    np.testing.assert_allclose((p[0, 0] * dp).sum(1), (do * o)[0, 0].sum(1), atol=1e-10)


def test_gradient_sums():
    """Softmax rows are shift invariant: sum_j dS_ij = 0, so sum over keys of dK = 0
    for a single query row's contribution only; globally dV column sums equal dO sums."""
    q, k, v, do = (_rand((1, 2, 25, 8), 60 + i) for i in range(4))
    for causal in (False, True):
        dq, dk, dv = attention_bwd(q, k, v, do, 0.3, causal)
        np.testing.assert_allclose(dv.sum(2), do.sum(2), atol=1e-12)
        np.testing.assert_allclose(dk.sum(2), 0.0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_sampled_gradients_match_the_whole_gradients(causal):
    """attention_bwd_sampled equals attention_bwd on the selected rows and keys (panels smaller
    than N, so the forward it relies on runs in several panels)."""
    N, d, scale = 300, 16, 0.25
    q, k, v, do = (_rand((1, 1, N, d), 70 + i, 2.0 if i == 1 else 1.0) for i in range(4))
    dq, dk, dv = attention_bwd(q, k, v, do, scale, causal)
    rows, keys = np.array([0, 1, 77, 150, 299]), np.array([0, 5, 150, 298, 299])
    sq, sk, sv = attention_bwd_sampled(q[0, 0], k[0, 0], v[0, 0], do[0, 0], rows, keys, scale, causal, panel_rows=64)
    np.testing.assert_allclose(sq, dq[0, 0, rows], rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(sk, dk[0, 0, keys], rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(sv, dv[0, 0, keys], rtol=1e-11, atol=1e-13)


def test_sampled_gradients_by_central_differences():
    """Independent of attention_bwd: the sampled entries against central differences of the loss."""
    N, d, scale, h = 7, 3, 0.7, 1e-6
    q, k, v, do = (_rand((N, d), 74 + i) for i in range(4))
    rows, keys = np.array([0, 4, 6]), np.array([1, 6])
    sq, sk, sv = attention_bwd_sampled(q, k, v, do, rows, keys, scale, True)

    def loss(qq, kk, vv):
        o, _ = attention_fwd(qq[None, None], kk[None, None], vv[None, None], scale, True)
        return float((o[0, 0] * do).sum())

    for which, idx_rows, got in ((0, rows, sq), (1, keys, sk), (2, keys, sv)):
        for a, r in enumerate(idx_rows):
            for c in range(d):
                args = [q.copy(), k.copy(), v.copy()]
                args[which][r, c] += h
                lp = loss(*args)
                args[which][r, c] -= 2 * h
                fd = (lp - loss(*args)) / (2 * h)
                assert abs(fd - got[a, c]) <= 1e-6 * max(1.0, abs(fd)), (which, r, c, fd, got[a, c])


# --- the operand-rounding bound used as a tolerance term -------------------

def _grads_with_rounded_operands(q, k, v, do, scale, causal, group):
    """Brute force in torch float64: P and dS rounded to bfloat16 before the three
    products, everything else exact; a shared key/value head sums its uses."""
    q, k, v, do = (torch.from_numpy(np.ascontiguousarray(x)) for x in (q, k, v, do))
    B, H, N, _ = q.shape
    dq, dk, dv = torch.zeros_like(q), torch.zeros_like(k), torch.zeros_like(v)
    bf = lambda x: x.to(torch.bfloat16).to(torch.float64)  # noqa: E731
    mask = torch.triu(torch.ones(N, N, dtype=torch.bool), 1)
    for b in range(B):
        for h in range(H):
            g = h // group
            s = scale * q[b, h] @ k[b, g].T
            if causal:
                s = s.masked_fill(mask, float("-inf"))
            p = torch.softmax(s, dim=1)
            dp = do[b, h] @ v[b, g].T
            ds = p * (dp - (p * dp).sum(1, keepdim=True))
            dv[b, g] += bf(p).T @ do[b, h]
            dq[b, h] = scale * bf(ds) @ k[b, g]
            dk[b, g] += scale * bf(ds).T @ q[b, h]
    return dq.numpy(), dk.numpy(), dv.numpy()


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("H,H_kv", [(2, 2), (4, 2)])
def test_operand_rounding_bound_holds_by_brute_force(causal, H, H_kv):
    """Rounding P and dS to bfloat16 moves every gradient entry by no more than the bound
    (u = 2^-8), and the bound is tight enough to mean something: for each of dQ, dK, dV the
    largest move reaches 40 % of it (a bound missing the scale factor would not)."""
    B, N, d, scale = 1, 40, 8, 0.35
    q, do = _rand((B, H, N, d), 91), _rand((B, H, N, d), 92)
    k, v = _rand((B, H_kv, N, d), 93, 4.0), _rand((B, H_kv, N, d), 94)
    exact = attention_bwd_gqa(q, k, v, do, scale, causal)
    rounded = _grads_with_rounded_operands(q, k, v, do, scale, causal, H // H_kv)
    bounds = bwd_operand_rounding_bound(q, k, v, do, scale, causal)
    for e, r, bnd in zip(exact, rounded, bounds):
        move = np.abs(r - e)
        assert (move <= bnd + 1e-12).all(), float((move - bnd).max())
        worst = float((move / np.maximum(bnd, 1e-300)).max())
        assert worst > 0.4, worst


def test_operand_rounding_bound_scales_with_u_and_vanishes_for_exact_operands():
    q, k, v, do = (_rand((1, 1, 20, 4), 95 + i) for i in range(4))
    b1 = bwd_operand_rounding_bound(q, k, v, do, 0.5, True)
    b2 = bwd_operand_rounding_bound(q, k, v, do, 0.5, True, unit_roundoff=2.0 ** -9)
    for x, y in zip(b1, b2):
        np.testing.assert_allclose(x, 2 * y, rtol=1e-14)
        assert (x >= 0).all()
    assert all((x == 0).all() for x in bwd_operand_rounding_bound(q, k, v, do, 0.5, True, unit_roundoff=0.0))


# --- grouped-query attention ---------------------------------------------

@pytest.mark.parametrize("causal", [False, True])
def test_gqa_matches_torch_sdpa_enable_gqa(causal):
    """torch's scaled-dot-product attention with enable_gqa (CPU, float64), forward and autograd:
    an independent implementation of contiguous query-head sets sharing a key/value head."""
    B, H, H_kv, N, d, scale = 2, 6, 2, 41, 8, 0.3
    q, do = _rand((B, H, N, d), 81), _rand((B, H, N, d), 82)
    k, v = _rand((B, H_kv, N, d), 83), _rand((B, H_kv, N, d), 84)
    o, lse = attention_fwd_gqa(q, k, v, scale, causal)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    to = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=scale,
                                                          enable_gqa=True)
    np.testing.assert_allclose(o, to.detach().numpy(), atol=1e-12)
    to.backward(torch.tensor(do))
    dq, dk, dv = attention_bwd_gqa(q, k, v, do, scale, causal)
    np.testing.assert_allclose(dq, tq.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dk, tk.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dv, tv.grad.numpy(), atol=1e-11)
    # lse of query head h equals the plain forward's lse against key/value head h // 3
    _, lse1 = attention_fwd(q[:, 4:5], k[:, 1:2], v[:, 1:2], scale, causal)
    np.testing.assert_allclose(lse[:, 4], lse1[:, 0], atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_gqa_gradients_by_central_differences(causal):
    """Brute force on a tiny case: the shared key/value heads' gradients sum over their sets."""
    H, H_kv, N, d, scale, h = 4, 2, 5, 3, 0.7, 1e-6
    q, do = _rand((1, H, N, d), 91), _rand((1, H, N, d), 92)
    k, v = _rand((1, H_kv, N, d), 93), _rand((1, H_kv, N, d), 94)
    grads = attention_bwd_gqa(q, k, v, do, scale, causal)

    def loss(qq, kk, vv):
        o, _ = attention_fwd_gqa(qq, kk, vv, scale, causal)
        return float((o * do).sum())

    for which, grad in enumerate(grads):
        fd = np.zeros_like(grad)
        for idx in np.ndindex(grad.shape):
            args = [q.copy(), k.copy(), v.copy()]
            args[which][idx] += h
            lp = loss(*args)
            args[which][idx] -= 2 * h
            lm = loss(*args)
            fd[idx] = (lp - lm) / (2 * h)
        rel = np.abs(fd - grad).max() / max(np.abs(grad).max(), 1e-30)
        assert rel < 1e-6, (which, rel)


def test_gqa_special_cases():
    """H_kv = H is plain multi-head attention; identical query heads over one shared
    key/value head (multi-query) give identical outputs and H times one head's dK, dV."""
    q, k, v, do = (_rand((2, 3, 19, 8), 100 + i) for i in range(4))
    for causal in (False, True):
        o, lse = attention_fwd_gqa(q, k, v, 0.4, causal)
        o1, lse1 = attention_fwd(q, k, v, 0.4, causal)
        np.testing.assert_allclose(o, o1, atol=1e-14)
        np.testing.assert_allclose(lse, lse1, atol=1e-14)
        for a, b in zip(attention_bwd_gqa(q, k, v, do, 0.4, causal), attention_bwd(q, k, v, do, 0.4, causal)):
            np.testing.assert_allclose(a, b, atol=1e-14)
    q1, do1 = _rand((1, 1, 23, 8), 110), _rand((1, 1, 23, 8), 111)
    k1, v1 = _rand((1, 1, 23, 8), 112), _rand((1, 1, 23, 8), 113)
    H = 4
    qh, doh = np.repeat(q1, H, axis=1), np.repeat(do1, H, axis=1)
    o, _ = attention_fwd_gqa(qh, k1, v1, 0.5, True)
    for hh in range(H):
        np.testing.assert_allclose(o[:, hh], o[:, 0], atol=1e-15)
    _, dk, dv = attention_bwd_gqa(qh, k1, v1, doh, 0.5, True)
    _, dk1, dv1 = attention_bwd(q1, k1, v1, do1, 0.5, True)
    np.testing.assert_allclose(dk, H * dk1, atol=1e-12)
    np.testing.assert_allclose(dv, H * dv1, atol=1e-12)


def test_gqa_rejects_uneven_sets():
    with pytest.raises(ValueError):
        attention_fwd_gqa(_rand((1, 3, 4, 2), 1), _rand((1, 2, 4, 2), 2), _rand((1, 2, 4, 2), 3), 1.0, False)


# --- decoding: fewer queries than keys, bottom-right causal alignment ------

@pytest.mark.parametrize("causal", [False, True])
def test_decode_matches_torch_sdpa_with_explicit_mask(causal):
    """torch SDPA (float64) with an explicit bottom-right boolean mask and enable_gqa."""
    B, H, H_kv, Nq, Nk, d, scale = 2, 4, 2, 5, 37, 8, 0.35
    q = _rand((B, H, Nq, d), 121)
    k, v = _rand((B, H_kv, Nk, d), 122), _rand((B, H_kv, Nk, d), 123)
    o, lse = attention_fwd_decode(q, k, v, scale, causal)
    mask = None
    if causal:
        mask = torch.ones(Nq, Nk, dtype=torch.bool).tril(Nk - Nq)     # query i sees j <= Nk - Nq + i
    to = torch.nn.functional.scaled_dot_product_attention(torch.tensor(q), torch.tensor(k), torch.tensor(v),
                                                          attn_mask=mask, scale=scale, enable_gqa=True)
    np.testing.assert_allclose(o, to.numpy(), atol=1e-12)
    s = scale * torch.tensor(q) @ torch.tensor(k).repeat_interleave(H // H_kv, 1).transpose(-1, -2)
    if causal:
        s = s.masked_fill(~mask, float("-inf"))
    np.testing.assert_allclose(lse, torch.logsumexp(s, -1).numpy(), atol=1e-12)


def test_decode_special_cases():
    """N_q == N_k is the square (top-left == bottom-right) case; one query, or the last
    query of any causal decode, sees every key."""
    q, k, v = (_rand((1, 4, 23, 8), 130 + i) for i in range(3))
    for causal in (False, True):
        o, lse = attention_fwd_decode(q, k[:, :2], v[:, :2], 0.3, causal)
        o1, lse1 = attention_fwd_gqa(q, k[:, :2], v[:, :2], 0.3, causal)
        np.testing.assert_allclose(o, o1, atol=1e-14)
        np.testing.assert_allclose(lse, lse1, atol=1e-14)
    q4 = _rand((1, 4, 6, 8), 140)
    oc, lc = attention_fwd_decode(q4, k, v, 0.3, True)
    on, ln = attention_fwd_decode(q4, k, v, 0.3, False)
    np.testing.assert_allclose(oc[:, :, -1], on[:, :, -1], atol=1e-14)
    np.testing.assert_allclose(lc[:, :, -1], ln[:, :, -1], atol=1e-14)
    assert not np.allclose(oc[:, :, 0], on[:, :, 0])
    o1c, _ = attention_fwd_decode(q4[:, :, :1], k, v, 0.3, True)
    o1n, _ = attention_fwd_decode(q4[:, :, :1], k, v, 0.3, False)
    np.testing.assert_allclose(o1c, o1n, atol=1e-14)


def test_decode_split_keys_merge_to_the_whole():
    """Partial results over disjoint key ranges, merged with softmax_merge, give the
    whole decode result (the split-KV structure, in the oracle's own terms)."""
    q = _rand((1, 2, 3, 8), 150)
    k, v = _rand((1, 1, 50, 8), 151, 2.0), _rand((1, 1, 50, 8), 152)
    o, lse = attention_fwd_decode(q, k, v, 0.4, False)
    parts = [(0, 17), (17, 40), (40, 50)]
    m_acc, l_acc, o_acc = None, None, None
    for a, b in parts:
        op, lp = attention_fwd_decode(q, k[:, :, a:b], v[:, :, a:b], 0.4, False)
        m_p, l_p = lp.reshape(-1), np.ones(lp.size)          # lse as the max with l = 1
        o_p = op.reshape(-1, 8)
        if m_acc is None:
            m_acc, l_acc, o_acc = m_p, l_p, o_p
        else:
            m_acc, l_acc, o_acc = softmax_merge(m_acc, l_acc, o_acc, m_p, l_p, o_p)
    np.testing.assert_allclose(o_acc, o.reshape(-1, 8), atol=1e-13)
    np.testing.assert_allclose(m_acc + np.log(l_acc), lse.reshape(-1), atol=1e-13)


# --- the softmax merge and the blockwise algorithm -------------------------

@pytest.mark.parametrize("causal", [False, True])
def test_blockwise_matches_two_pass(causal):
    q, k, v = _rand((1, 2, 131, 16), 70, 2.0), _rand((1, 2, 131, 16), 71, 2.0), _rand((1, 2, 131, 16), 72)
    o_ref, l_ref = attention_fwd(q, k, v, 0.25, causal)
    for bq, bk in ((1, 1), (7, 13), (64, 64), (131, 17), (200, 200)):
        o, l = attention_fwd_blockwise(q, k, v, 0.25, causal, bq, bk)
        np.testing.assert_allclose(o, o_ref, atol=1e-12)
        np.testing.assert_allclose(l, l_ref, atol=1e-12)


def test_merge_over_random_splits_matches_two_pass():
    rng = np.random.default_rng(80)
    N, d, scale = 90, 8, 0.5
    q, k, v = rng.standard_normal((N, d)) * 2, rng.standard_normal((N, d)) * 2, rng.standard_normal((N, d))
    rows = np.arange(N)
    o_ref, lse_ref = attention_fwd_rows(q, k, v, rows, scale, False)
    for trial in range(5):
        cuts = np.sort(rng.choice(np.arange(1, N), size=trial + 1, replace=False))
        parts = np.split(rng.permutation(N), cuts)
        m = np.full(N, -np.inf)
        l = np.zeros(N)
        o = np.zeros((N, d))
        for idx in parts:
            s = scale * q @ k[idx].T
            m_x = s.max(1)
            o_x, lse_x = attention_fwd_rows(q, k[idx], v[idx], rows, scale, False)
            l_x = np.exp(lse_x - m_x)
            m, l, o = softmax_merge(m, l, o, m_x, l_x, o_x)
        np.testing.assert_allclose(o, o_ref, atol=1e-12)
        np.testing.assert_allclose(m + np.log(l), lse_ref, atol=1e-12)


def test_merge_with_empty_side():
    o_x = np.ones((3, 2))
    m, l, o = softmax_merge(np.full(3, -np.inf), np.zeros(3), np.zeros((3, 2)),
                            np.zeros(3), np.ones(3), o_x)
    np.testing.assert_array_equal(o, o_x)
    np.testing.assert_array_equal(l, 1.0)


def _blockwise_divide_every_step(q, k, v, scale, block):
    """Planted mistake: divide the running output by the new running sum at
    every key block while rescaling the old (already divided) output by the
    max correction alone -- the normalisation slip of the pages' simplified
    blockwise listing.  Test helper only."""
    N, d = q.shape
    M = np.full(N, -np.inf)
    L = np.zeros(N)
    O = np.zeros((N, d))
    for j0 in range(0, N, block):
        s = scale * q @ k[j0:j0 + block].T
        m_new = np.maximum(M, s.max(1))
        p = np.exp(s - m_new[:, None])
        alpha = np.where(np.isneginf(M), 0.0, np.exp(M - m_new))
        L_new = alpha * L + p.sum(1)
        O = (alpha[:, None] * O + p @ v[j0:j0 + block]) / L_new[:, None]
        L, M = L_new, m_new
    return O


def test_constant_v_catches_the_listing_normalisation_slip():
    rng = np.random.default_rng(90)
    N, d = 64, 4
    q, k = rng.standard_normal((N, d)), rng.standard_normal((N, d))
    v = np.broadcast_to(rng.standard_normal(d), (N, d)).copy()
    bad = _blockwise_divide_every_step(q, k, v, 0.5, 16)
    assert np.abs(bad - v).max() > 1e-3          # the slip is visible
    good, _ = attention_fwd_blockwise(q[None, None], k[None, None], v[None, None], 0.5, False, 64, 16)
    np.testing.assert_allclose(good[0, 0], v, atol=1e-12)
    # with a single key block the slip is harmless, which is why it needs >= 2 blocks
    one = _blockwise_divide_every_step(q, k, v, 0.5, N)
    np.testing.assert_allclose(one, v, atol=1e-12)
