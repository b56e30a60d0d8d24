"""Head dim 256 forward and backward on the GPU against the fp64 oracle.

The nearauto.com FlashAttention-2 digest lists head dimensions up to 256; the
result is the same attention as at d = 64 / 128 (oracle attention_fwd,
attention_fwd_gqa, attention_fwd_general, attention_fwd_varlen) with the same
tolerances.  Covers ragged lengths around the 128-row tile and 64-key block,
grouped heads, N_q != N_k (with rows that see no key), packed sequences,
strided tensors and run-to-run determinism.
"""
import numpy as np
import pytest

from exact_io_aware_100_b200 import inputs
from helpers import assert_close, assert_lse, to_device, to_f64
from oracle import (attention_bwd_general, attention_bwd_gqa, attention_bwd_varlen, attention_fwd_general,
                    attention_fwd_gqa, attention_fwd_varlen)

pytestmark = pytest.mark.gpu
D = 256


def _tensor(seed, name, shape, mult=1.0):
    host = inputs.make_tensor(seed, name, shape, mult)
    return to_device(host, "bf16"), inputs.to_f64(host, "bf16")


def _check_lse(got, ref, tol=1e-3):
    got = np.asarray(got, np.float64)
    empty = np.isneginf(ref)
    assert np.array_equal(np.isneginf(got), empty), "lse: -inf rows differ"
    if (~empty).any():
        assert_lse(got[~empty], ref[~empty], tol)


@pytest.mark.parametrize("B,H,H_kv,N,causal", [
    (1, 2, 2, 1, True),
    (1, 2, 2, 63, False),
    (1, 2, 2, 127, True),
    (2, 2, 2, 129, True),
    (1, 3, 3, 300, False),
    (2, 4, 2, 513, True),       # grouped heads
    (1, 4, 1, 1000, True),      # multi-query
    (1, 2, 2, 2048, True),
])
def test_forward_d256(B, H, H_kv, N, causal):
    import torch
    import exact_io_aware_100_b200 as fa
    seed = 4100 + N + H_kv
    q, fq = _tensor(seed, "q", (B, H, N, D))
    k, fk = _tensor(seed, "k", (B, H_kv, N, D), 1.5)
    v, fv = _tensor(seed, "v", (B, H_kv, N, D))
    o, lse = fa.forward(q, k, v, causal)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == fa.FA_OK
    ro, rl = attention_fwd_gqa(fq, fk, fv, 1.0 / np.sqrt(D), causal)
    assert_close("O", to_f64(o), ro)
    assert_lse(to_f64(lse), rl)
    o2, lse2 = fa.forward(q, k, v, causal)
    assert torch.equal(o, o2) and torch.equal(lse, lse2)        # bitwise run to run


@pytest.mark.parametrize("Nq,Nk,causal", [(200, 700, True), (700, 200, True), (333, 130, False), (1, 1000, True)])
def test_forward_d256_any_lengths(Nq, Nk, causal):
    import torch
    import exact_io_aware_100_b200 as fa
    B, H, H_kv = 2, 4, 2
    seed = 4200 + Nq + Nk
    q, fq = _tensor(seed, "q", (B, H, Nq, D))
    k, fk = _tensor(seed, "k", (B, H_kv, Nk, D))
    v, fv = _tensor(seed, "v", (B, H_kv, Nk, D))
    o, lse = fa.forward(q, k, v, causal)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == fa.FA_OK
    ro, rl = attention_fwd_general(fq, fk, fv, 1.0 / np.sqrt(D), causal)
    assert_close("O", to_f64(o), ro)
    _check_lse(to_f64(lse), rl)
    assert np.all(to_f64(o)[np.isneginf(rl)] == 0.0)


@pytest.mark.parametrize("causal", [True, False])
def test_forward_d256_varlen(causal):
    import torch
    import exact_io_aware_100_b200 as fa
    lens = [(300, 300), (0, 50), (77, 0), (129, 700), (500, 130), (1, 1), (64, 64), (1000, 1000)]
    H, H_kv = 4, 2
    tq, tk = sum(a for a, _ in lens), sum(b for _, b in lens)
    q, fq = _tensor(4300, "q", (tq, H, D))
    k, fk = _tensor(4300, "k", (tk, H_kv, D))
    v, fv = _tensor(4300, "v", (tk, H_kv, D))
    cu_q = np.concatenate([[0], np.cumsum([a for a, _ in lens])]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum([b for _, b in lens])]).astype(np.int32)
    o, lse = fa.forward_varlen(q, k, v, torch.from_numpy(cu_q).cuda(), torch.from_numpy(cu_k).cuda(),
                               max(a for a, _ in lens), max(b for _, b in lens), causal)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == fa.FA_OK
    ro, rl = attention_fwd_varlen(fq, fk, fv, cu_q, cu_k, 1.0 / np.sqrt(D), causal)
    assert_close("O", to_f64(o), ro)
    _check_lse(to_f64(lse), rl)


def test_forward_d256_strided_is_the_dense_result():
    import torch
    import exact_io_aware_100_b200 as fa
    B, H, N = 2, 4, 400
    q, _ = _tensor(4400, "q", (B, H, N, D))
    k, _ = _tensor(4400, "k", (B, H, N, D))
    v, _ = _tensor(4400, "v", (B, H, N, D))
    o_ref, lse_ref = fa.forward(q, k, v, True)
    qs, ks, vs = (t.transpose(1, 2).contiguous().transpose(1, 2) for t in (q, k, v))
    o_s, lse_s = fa.forward(qs, ks, vs, True)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == fa.FA_OK
    assert torch.equal(o_s.contiguous(), o_ref) and torch.equal(lse_s, lse_ref)


# ---------------------------------------------------------------- backward
def _bwd_case(B, H, H_kv, Nq, Nk, seed, k_mult=1.0):
    q, fq = _tensor(seed, "q", (B, H, Nq, D))
    k, fk = _tensor(seed, "k", (B, H_kv, Nk, D), k_mult)
    v, fv = _tensor(seed, "v", (B, H_kv, Nk, D))
    do, fdo = _tensor(seed, "do", (B, H, Nq, D))
    return (q, k, v, do), (fq, fk, fv, fdo)


def _check_grads(got, ref, grouped):
    for name, g, r in zip(("dQ", "dK", "dV"), got, ref):
        # a shared head's dK, dV sum its set's gradients: max-abs scales with their magnitude
        assert_close(name, to_f64(g), r, scale_max_abs=grouped and name != "dQ")


@pytest.mark.parametrize("B,H,H_kv,N,causal", [
    (1, 2, 2, 1, True),
    (1, 2, 2, 63, False),
    (1, 2, 2, 64, True),
    (2, 2, 2, 65, True),
    (1, 3, 3, 127, False),
    (1, 2, 2, 129, True),
    (2, 2, 2, 300, True),
    (1, 2, 2, 513, False),
    (1, 4, 2, 640, True),       # grouped heads
    (2, 3, 1, 200, False),      # multi-query
    (1, 2, 2, 1000, True),
])
def test_backward_d256(B, H, H_kv, N, causal):
    import torch
    import exact_io_aware_100_b200 as fa
    dev, f = _bwd_case(B, H, H_kv, N, N, 4500 + N + H_kv)
    q, k, v, do = dev
    o, lse = fa.forward(q, k, v, causal)
    grads = fa.backward(q, k, v, o, lse, do, causal)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == fa.FA_OK
    ref = attention_bwd_gqa(*f, 1.0 / np.sqrt(D), causal)
    _check_grads(grads, ref, H_kv != H)


def test_backward_d256_sharp_rows():
    """Keys x4: sharp softmax rows; gradients reach |x| ~ 16, where a bf16 ulp is 0.0625."""
    import torch
    import exact_io_aware_100_b200 as fa
    dev, f = _bwd_case(1, 2, 2, 400, 400, 4550, k_mult=4.0)
    q, k, v, do = dev
    o, lse = fa.forward(q, k, v, True)
    grads = fa.backward(q, k, v, o, lse, do, True)
    torch.cuda.synchronize()
    ref = attention_bwd_gqa(*f, 1.0 / np.sqrt(D), True)
    for name, g, r in zip(("dQ", "dK", "dV"), grads, ref):
        assert_close(name, to_f64(g), r, scale_max_abs=True)


@pytest.mark.parametrize("Nq,Nk,causal", [(200, 700, True), (700, 200, True), (333, 130, False), (64, 1000, True)])
def test_backward_d256_any_lengths(Nq, Nk, causal):
    import torch
    import exact_io_aware_100_b200 as fa
    dev, f = _bwd_case(2, 4, 2, Nq, Nk, 4600 + Nq + Nk)
    q, k, v, do = dev
    o, lse = fa.forward(q, k, v, causal)
    grads = fa.backward(q, k, v, o, lse, do, causal)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == fa.FA_OK
    ref = attention_bwd_general(*f, 1.0 / np.sqrt(D), causal)
    _check_grads(grads, ref, True)


@pytest.mark.parametrize("causal", [True, False])
def test_backward_d256_varlen(causal):
    import torch
    import exact_io_aware_100_b200 as fa
    lens = [(300, 300), (0, 50), (77, 0), (129, 700), (500, 130), (1, 1), (64, 64), (1000, 1000)]
    H, H_kv = 4, 2
    tq, tk = sum(a for a, _ in lens), sum(b for _, b in lens)
    q, fq = _tensor(4700, "q", (tq, H, D))
    k, fk = _tensor(4700, "k", (tk, H_kv, D))
    v, fv = _tensor(4700, "v", (tk, H_kv, D))
    do, fdo = _tensor(4700, "do", (tq, H, D))
    cu_q = np.concatenate([[0], np.cumsum([a for a, _ in lens])]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum([b for _, b in lens])]).astype(np.int32)
    cq, ck = torch.from_numpy(cu_q).cuda(), torch.from_numpy(cu_k).cuda()
    mq, mk = max(a for a, _ in lens), max(b for _, b in lens)
    o, lse = fa.forward_varlen(q, k, v, cq, ck, mq, mk, causal)
    grads = fa.backward_varlen(q, k, v, o, lse, do, cq, ck, mq, mk, causal)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == fa.FA_OK
    ref = attention_bwd_varlen(fq, fk, fv, fdo, cu_q, cu_k, 1.0 / np.sqrt(D), causal)
    _check_grads(grads, ref, True)


def test_backward_d256_strided_is_the_dense_result():
    import torch
    import exact_io_aware_100_b200 as fa
    dev, _ = _bwd_case(2, 4, 4, 300, 300, 4800)
    q, k, v, do = dev
    o, lse = fa.forward(q, k, v, True)
    ref = fa.backward(q, k, v, o, lse, do, True)
    qs, ks, vs, os_, dos = (t.transpose(1, 2).contiguous().transpose(1, 2) for t in (q, k, v, o, do))
    got = fa.backward(qs, ks, vs, os_, lse, dos, True)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == fa.FA_OK
    for g, r in zip(got, ref):       # dQ goes through fp32 atomics: equal within rounding, not bitwise
        assert_close("strided", to_f64(g.contiguous()), to_f64(r))
