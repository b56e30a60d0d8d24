"""Pins for the oracle's general-length and variable-length functions.

Any number of queries against any number of keys (bottom-right causal
alignment, rows that see no key give O = 0 and lse = -inf), and packed
variable-length batches.  Checked against torch's scaled-dot-product attention
in float64 with an explicit mask (an independent implementation), closed
forms, invariants and finite differences.  None of them calls the CUDA path.
"""
import numpy as np
import pytest
import torch

from oracle import (attention_bwd_general, attention_bwd_varlen, attention_fwd_general, attention_fwd_gqa,
                    attention_fwd_varlen)

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _rand(shape, seed, mult=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * mult


def _mask(nq, nk):
    """Bottom-right causal mask: query i sees key j <= nk - nq + i."""
    return torch.ones(nq, nk, dtype=torch.bool).tril(nk - nq)


def _torch_ref(q, k, v, scale, causal):
    """torch SDPA (float64) per (b, h) head with an explicit mask; NaN rows (no key) are left NaN.
    q [B,H,Nq,d], k/v [B,H_kv,Nk,d].  Returns (O, lse) as numpy."""
    tq, tk, tv = torch.tensor(q), torch.tensor(k), torch.tensor(v)
    nq, nk = q.shape[2], k.shape[2]
    mask = _mask(nq, nk) if causal else torch.ones(nq, nk, dtype=torch.bool)
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask, scale=scale, enable_gqa=True)
    s = scale * tq @ tk.repeat_interleave(q.shape[1] // k.shape[1], 1).transpose(-1, -2)
    s = s.masked_fill(~mask, float("-inf"))
    return o.numpy(), torch.logsumexp(s, -1).numpy(), mask.any(1).numpy()


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("nq,nk", [(5, 37), (37, 20), (16, 16), (1, 9)])
def test_general_matches_torch_sdpa(causal, nq, nk):
    B, H, H_kv, d, scale = 2, 4, 2, 8, 0.35
    q = _rand((B, H, nq, d), 300 + nq)
    k, v = _rand((B, H_kv, nk, d), 301 + nk), _rand((B, H_kv, nk, d), 302 + nk)
    o, lse = attention_fwd_general(q, k, v, scale, causal)
    to, tl, seen = _torch_ref(q, k, v, scale, causal)
    np.testing.assert_allclose(o[:, :, seen], to[:, :, seen], atol=1e-12)
    np.testing.assert_allclose(lse, tl, atol=1e-12)       # -inf where no key is seen
    assert np.all(o[:, :, ~seen] == 0.0)


def test_general_empty_rows_and_first_seen_row():
    """10 queries, 4 keys, causal: queries 0-5 see nothing (O = 0, lse = -inf); query 6
    sees key 0 alone (O = v_0, lse = scale q_6 . k_0); with no keys every row is empty."""
    q, k, v = _rand((1, 1, 10, 5), 310), _rand((1, 1, 4, 5), 311), _rand((1, 1, 4, 5), 312)
    o, lse = attention_fwd_general(q, k, v, 0.6, True)
    assert np.all(o[0, 0, :6] == 0.0) and np.all(np.isneginf(lse[0, 0, :6]))
    np.testing.assert_allclose(o[0, 0, 6], v[0, 0, 0], atol=1e-15)
    np.testing.assert_allclose(lse[0, 0, 6], 0.6 * q[0, 0, 6] @ k[0, 0, 0], atol=1e-14)
    for causal in (False, True):
        o0, l0 = attention_fwd_general(q, k[:, :, :0], v[:, :, :0], 0.6, causal)
        assert np.all(o0 == 0.0) and np.all(np.isneginf(l0))


def test_general_square_is_the_top_left_case():
    q, k, v = (_rand((2, 4, 19, 8), 320 + i) for i in range(3))
    for causal in (False, True):
        o, lse = attention_fwd_general(q, k[:, :2], v[:, :2], 0.3, causal)
        o1, lse1 = attention_fwd_gqa(q, k[:, :2], v[:, :2], 0.3, causal)
        np.testing.assert_allclose(o, o1, atol=1e-14)
        np.testing.assert_allclose(lse, lse1, atol=1e-14)


@pytest.mark.parametrize("nq,nk", [(4, 7), (8, 16)])
def test_general_gradients_match_torch_autograd(nq, nk):
    """Every query sees a key (nq <= nk), so torch's autograd of SDPA is defined everywhere."""
    B, H, H_kv, d, scale = 1, 4, 2, 6, 0.45
    q, do = _rand((B, H, nq, d), 330), _rand((B, H, nq, d), 331)
    k, v = _rand((B, H_kv, nk, d), 332), _rand((B, H_kv, nk, d), 333)
    for causal in (False, True):
        tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
        mask = _mask(nq, nk) if causal else None
        to = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask, scale=scale,
                                                              enable_gqa=True)
        to.backward(torch.tensor(do))
        dq, dk, dv = attention_bwd_general(q, k, v, do, scale, causal)
        np.testing.assert_allclose(dq, tq.grad.numpy(), atol=1e-11)
        np.testing.assert_allclose(dk, tk.grad.numpy(), atol=1e-11)
        np.testing.assert_allclose(dv, tv.grad.numpy(), atol=1e-11)


def _central_differences(loss, arrays, h=1e-6):
    out = []
    for which, a in enumerate(arrays):
        fd = np.zeros_like(a)
        for idx in np.ndindex(a.shape):
            args = [x.copy() for x in arrays]
            args[which][idx] += h
            lp = loss(*args)
            args[which][idx] -= 2 * h
            lm = loss(*args)
            fd[idx] = (lp - lm) / (2 * h)
        out.append(fd)
    return out


@pytest.mark.parametrize("nq,nk", [(6, 3), (3, 5)])
def test_general_gradients_by_central_differences(nq, nk):
    """Brute force, causal, including queries that see no key (their gradient is zero)."""
    H, H_kv, d, scale = 2, 1, 3, 0.7
    q, do = _rand((1, H, nq, d), 340), _rand((1, H, nq, d), 341)
    k, v = _rand((1, H_kv, nk, d), 342), _rand((1, H_kv, nk, d), 343)
    grads = attention_bwd_general(q, k, v, do, scale, True)

    def loss(qq, kk, vv):
        o, _ = attention_fwd_general(qq, kk, vv, scale, True)
        return float((o * do).sum())

    for which, (fd, grad) in enumerate(zip(_central_differences(loss, [q, k, v]), grads)):
        rel = np.abs(fd - grad).max() / max(np.abs(grad).max(), 1e-30)
        assert rel < 1e-6, (which, rel)
    if nq > nk:
        assert np.all(grads[0][:, :, :nq - nk] == 0.0)


def _pack(seqs):
    """list of [n_b, H, d] arrays -> (packed [sum n_b, H, d], offsets [B + 1])."""
    cu = np.concatenate([[0], np.cumsum([s.shape[0] for s in seqs])]).astype(np.int64)
    return np.concatenate(seqs, axis=0), cu


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_matches_torch_per_sequence(causal):
    """Each sequence of a packed batch against torch SDPA on that sequence alone."""
    H, H_kv, d, scale = 4, 2, 8, 0.3
    lens = [(7, 7), (0, 5), (12, 30), (9, 4), (3, 0), (1, 1), (20, 13)]
    qs = [_rand((a, H, d), 350 + i) for i, (a, _) in enumerate(lens)]
    ks = [_rand((b, H_kv, d), 360 + i) for i, (_, b) in enumerate(lens)]
    vs = [_rand((b, H_kv, d), 370 + i) for i, (_, b) in enumerate(lens)]
    q, cu_q = _pack(qs)
    k, cu_k = _pack(ks)
    v, _ = _pack(vs)
    o, lse = attention_fwd_varlen(q, k, v, cu_q, cu_k, scale, causal)
    assert o.shape == (q.shape[0], H, d) and lse.shape == (H, q.shape[0])
    for b, (nq, nk) in enumerate(lens):
        rows = slice(cu_q[b], cu_q[b + 1])
        if nq == 0:
            continue
        if nk == 0:
            assert np.all(o[rows] == 0.0) and np.all(np.isneginf(lse[:, rows]))
            continue
        to, tl, seen = _torch_ref(qs[b].transpose(1, 0, 2)[None], ks[b].transpose(1, 0, 2)[None],
                                  vs[b].transpose(1, 0, 2)[None], scale, causal)
        ob = o[rows].transpose(1, 0, 2)
        np.testing.assert_allclose(ob[:, seen], to[0][:, seen], atol=1e-12)
        assert np.all(ob[:, ~seen] == 0.0)
        np.testing.assert_allclose(lse[:, rows], tl[0], atol=1e-12)


def test_varlen_sequences_are_independent():
    """Changing one sequence's queries, keys and values changes no other sequence's result."""
    H, d = 2, 4
    lens_q, lens_k = [5, 8, 3], [6, 8, 9]
    q, cu_q = _pack([_rand((n, H, d), 380 + i) for i, n in enumerate(lens_q)])
    k, cu_k = _pack([_rand((n, H, d), 390 + i) for i, n in enumerate(lens_k)])
    v, _ = _pack([_rand((n, H, d), 400 + i) for i, n in enumerate(lens_k)])
    o, lse = attention_fwd_varlen(q, k, v, cu_q, cu_k, 0.5, True)
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    q2[cu_q[1]:cu_q[2]] += 3.0
    k2[cu_k[1]:cu_k[2]] *= -2.0
    v2[cu_k[1]:cu_k[2]] += 1.0
    o2, lse2 = attention_fwd_varlen(q2, k2, v2, cu_q, cu_k, 0.5, True)
    for b in (0, 2):
        rows = slice(cu_q[b], cu_q[b + 1])
        assert np.array_equal(o[rows], o2[rows]) and np.array_equal(lse[:, rows], lse2[:, rows])
    rows = slice(cu_q[1], cu_q[2])
    assert not np.allclose(o[rows], o2[rows])


def test_varlen_equal_lengths_is_the_batched_case():
    """B sequences of one length, packed, equal the [B, H, N, d] general forward."""
    B, H, H_kv, nq, nk, d = 3, 4, 2, 6, 11, 5
    q, k, v = _rand((B, H, nq, d), 410), _rand((B, H_kv, nk, d), 411), _rand((B, H_kv, nk, d), 412)
    o, lse = attention_fwd_general(q, k, v, 0.4, True)
    pq = q.transpose(0, 2, 1, 3).reshape(B * nq, H, d)
    pk = k.transpose(0, 2, 1, 3).reshape(B * nk, H_kv, d)
    pv = v.transpose(0, 2, 1, 3).reshape(B * nk, H_kv, d)
    ov, lv = attention_fwd_varlen(pq, pk, pv, np.arange(B + 1) * nq, np.arange(B + 1) * nk, 0.4, True)
    np.testing.assert_allclose(ov.reshape(B, nq, H, d).transpose(0, 2, 1, 3), o, atol=1e-14)
    np.testing.assert_allclose(lv.reshape(H, B, nq).transpose(1, 0, 2), lse, atol=1e-14)


def test_varlen_gradients_by_central_differences():
    """Brute force over a packed batch with an empty-query, an empty-key and an N_q > N_k sequence."""
    H, H_kv, d, scale = 2, 1, 2, 0.9
    lens = [(3, 4), (0, 2), (2, 0), (4, 2)]
    q, cu_q = _pack([_rand((a, H, d), 420 + i) for i, (a, _) in enumerate(lens)])
    k, cu_k = _pack([_rand((b, H_kv, d), 430 + i) for i, (_, b) in enumerate(lens)])
    v, _ = _pack([_rand((b, H_kv, d), 440 + i) for i, (_, b) in enumerate(lens)])
    do = _rand(q.shape, 450)
    for causal in (False, True):
        grads = attention_bwd_varlen(q, k, v, do, cu_q, cu_k, scale, causal)

        def loss(qq, kk, vv):
            o, _ = attention_fwd_varlen(qq, kk, vv, cu_q, cu_k, scale, causal)
            return float((o * do).sum())

        for which, (fd, grad) in enumerate(zip(_central_differences(loss, [q, k, v]), grads)):
            rel = np.abs(fd - grad).max() / max(np.abs(grad).max(), 1e-30)
            assert rel < 1e-6, (causal, which, rel)


def test_varlen_rejects_bad_offsets():
    q, k = np.zeros((5, 1, 2)), np.zeros((4, 1, 2))
    for cu_q, cu_k in (([0, 3, 5], [0, 4]), ([1, 5], [0, 4]), ([0, 6], [0, 4]), ([0, 4, 3, 5], [0, 1, 2, 4])):
        with pytest.raises(ValueError):
            attention_fwd_varlen(q, k, k, cu_q, cu_k, 1.0, False)


@pytest.mark.parametrize("causal", [False, True])
def test_head_dim_256_matches_torch_sdpa(causal):
    """Head dimension 256 (the width the d = 256 kernel is checked at) against torch SDPA in float64."""
    B, H, N, d = 1, 2, 40, 256
    q, k, v = (_rand((B, H, N, d), 460 + i) for i in range(3))
    o, lse = attention_fwd_general(q, k, v, d ** -0.5, causal)
    to, tl, seen = _torch_ref(q, k, v, d ** -0.5, causal)
    assert seen.all()
    np.testing.assert_allclose(o, to, atol=1e-12)
    np.testing.assert_allclose(lse, tl, atol=1e-12)
