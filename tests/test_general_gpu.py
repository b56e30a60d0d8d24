"""General lengths and layouts on the GPU against the fp64 oracle.

Any query and key lengths (bottom-right causal alignment, queries that see no
key give O = 0 and lse = -inf), packed variable-length batches, and strided
tensors ([B, N, H, d] memory, views of wider tensors).  The oracle is
attention_fwd_general / attention_bwd_general / attention_fwd_varlen /
attention_bwd_varlen; same tolerances as the square path.  A strided call
computes exactly what the dense call computes, so those outputs are compared
bit for bit (dQ, summed with atomic adds in no fixed order, within tolerance).
"""
import numpy as np
import pytest

from exact_io_aware_100_b200 import inputs
from helpers import assert_close, to_device, to_f64
from oracle import attention_bwd_general, attention_bwd_varlen, attention_fwd_general, attention_fwd_varlen

pytestmark = pytest.mark.gpu


def _tensor(seed, name, shape):
    host = inputs.make_tensor(seed, name, shape)
    return to_device(host, "bf16"), inputs.to_f64(host, "bf16")


def _check_lse(got, ref, tol=1e-3):
    got = np.asarray(got, np.float64)
    empty = np.isneginf(ref)
    assert np.array_equal(np.isneginf(got), empty), "lse: -inf rows differ"
    if (~empty).any():
        ma = float(np.abs(got[~empty] - ref[~empty]).max())
        assert np.isfinite(got[~empty]).all() and ma <= tol, f"lse: max_abs={ma:.3e}"


def _status_ok():
    import torch
    import exact_io_aware_100_b200 as fa
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == fa.FA_OK


@pytest.mark.parametrize("B,H,H_kv,Nq,Nk,d,causal", [
    (2, 4, 2, 200, 700, 128, True),
    (2, 4, 2, 200, 700, 128, False),
    (1, 4, 4, 700, 200, 128, True),     # queries 0-499 see no key
    (1, 2, 1, 1, 300, 128, True),
    (2, 4, 2, 130, 1000, 64, True),
    (1, 4, 2, 513, 129, 64, True),
    (1, 2, 2, 300, 257, 128, False),
])
def test_forward_any_lengths(B, H, H_kv, Nq, Nk, d, causal):
    import exact_io_aware_100_b200 as fa
    seed = 3100 + Nq + Nk
    q, fq = _tensor(seed, "q", (B, H, Nq, d))
    k, fk = _tensor(seed, "k", (B, H_kv, Nk, d))
    v, fv = _tensor(seed, "v", (B, H_kv, Nk, d))
    o, lse = fa.forward(q, k, v, causal)
    _status_ok()
    ro, rl = attention_fwd_general(fq, fk, fv, 1.0 / np.sqrt(d), causal)
    assert_close("O", to_f64(o), ro)
    _check_lse(to_f64(lse), rl)
    assert np.all(to_f64(o)[np.isneginf(rl)] == 0.0)


@pytest.mark.parametrize("N,d,causal,H_kv", [(300, 128, True, 4), (517, 64, False, 2), (1030, 128, True, 1)])
def test_forward_strided_is_the_dense_result(N, d, causal, H_kv):
    """[B, N, H, d] memory (passed as transpose(1, 2) views) and views of wider rows give
    bitwise the dense [B, H, N, d] result."""
    import torch
    import exact_io_aware_100_b200 as fa
    B, H = 2, 4
    q, _ = _tensor(3200 + N, "q", (B, H, N, d))
    k, _ = _tensor(3200 + N, "k", (B, H_kv, N, d))
    v, _ = _tensor(3200 + N, "v", (B, H_kv, N, d))
    o_ref, lse_ref = fa.forward(q, k, v, causal)
    qs, ks, vs = (t.transpose(1, 2).contiguous().transpose(1, 2) for t in (q, k, v))   # [B, N, H, d] memory
    assert not qs.is_contiguous()
    o_s, lse_s = fa.forward(qs, ks, vs, causal)
    assert o_s.stride() == qs.stride()
    # rows padded to 2d + 64 columns: q lives in columns 64 .. 64 + d of a wider tensor
    wide = torch.zeros((B, H, N, 2 * d + 64), dtype=q.dtype, device=q.device)
    wide[..., 64:64 + d] = q
    o_w, lse_w = fa.forward(wide[..., 64:64 + d], k, v, causal)
    _status_ok()
    for o_x, lse_x in ((o_s, lse_s), (o_w, lse_w)):
        assert torch.equal(o_x.contiguous(), o_ref) and torch.equal(lse_x, lse_ref)


def _packed_case(lens, H, H_kv, d, seed):
    import torch
    tq, tk = sum(a for a, _ in lens), sum(b for _, b in lens)
    q, fq = _tensor(seed, "q", (max(tq, 1), H, d))
    k, fk = _tensor(seed, "k", (max(tk, 1), H_kv, d))
    v, fv = _tensor(seed, "v", (max(tk, 1), H_kv, d))
    q, fq, k, fk, v, fv = q[:tq], fq[:tq], k[:tk], fk[:tk], v[:tk], fv[:tk]
    cu_q = np.concatenate([[0], np.cumsum([a for a, _ in lens])]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum([b for _, b in lens])]).astype(np.int32)
    dev = lambda x: torch.from_numpy(x).cuda()
    return (q, k, v, dev(cu_q), dev(cu_k)), (fq, fk, fv, cu_q, cu_k)


LENS = [(300, 300), (0, 50), (77, 0), (129, 700), (500, 130), (1, 1), (256, 256), (1000, 1000), (3, 513)]


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("H,H_kv,d", [(4, 4, 128), (4, 2, 64)])
def test_forward_varlen(causal, H, H_kv, d):
    import exact_io_aware_100_b200 as fa
    (q, k, v, cu_q, cu_k), (fq, fk, fv, hq, hk) = _packed_case(LENS, H, H_kv, d, 3300 + d)
    mq, mk = max(a for a, _ in LENS), max(b for _, b in LENS)
    o, lse = fa.forward_varlen(q, k, v, cu_q, cu_k, mq, mk, causal)
    _status_ok()
    ro, rl = attention_fwd_varlen(fq, fk, fv, hq, hk, 1.0 / np.sqrt(d), causal)
    assert_close("O", to_f64(o), ro)
    _check_lse(to_f64(lse), rl)
    assert np.all(to_f64(o).transpose(1, 0, 2)[np.isneginf(rl)] == 0.0)


@pytest.mark.parametrize("B,H,H_kv,Nq,Nk,d,causal", [
    (1, 4, 2, 200, 700, 128, True),
    (1, 4, 4, 700, 200, 128, True),     # empty query rows
    (2, 2, 2, 300, 170, 128, False),
    (1, 4, 2, 130, 600, 64, True),
    (1, 2, 1, 513, 129, 64, True),
])
def test_backward_any_lengths(B, H, H_kv, Nq, Nk, d, causal):
    import exact_io_aware_100_b200 as fa
    seed = 3400 + Nq + Nk
    q, fq = _tensor(seed, "q", (B, H, Nq, d))
    k, fk = _tensor(seed, "k", (B, H_kv, Nk, d))
    v, fv = _tensor(seed, "v", (B, H_kv, Nk, d))
    do, fdo = _tensor(seed, "do", (B, H, Nq, d))
    o, lse = fa.forward(q, k, v, causal)
    dq, dk, dv = fa.backward(q, k, v, o, lse, do, causal)
    _status_ok()
    rq, rk, rv = attention_bwd_general(fq, fk, fv, fdo, 1.0 / np.sqrt(d), causal)
    assert_close("dQ", to_f64(dq), rq)
    assert_close("dK", to_f64(dk), rk, scale_max_abs=H_kv < H)
    assert_close("dV", to_f64(dv), rv, scale_max_abs=H_kv < H)


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("H,H_kv,d", [(4, 4, 128), (4, 2, 64)])
def test_backward_varlen(causal, H, H_kv, d):
    import exact_io_aware_100_b200 as fa
    (q, k, v, cu_q, cu_k), (fq, fk, fv, hq, hk) = _packed_case(LENS, H, H_kv, d, 3500 + d)
    do, fdo = _tensor(3500 + d, "do", (q.shape[0], H, d))
    mq, mk = max(a for a, _ in LENS), max(b for _, b in LENS)
    o, lse = fa.forward_varlen(q, k, v, cu_q, cu_k, mq, mk, causal)
    dq, dk, dv = fa.backward_varlen(q, k, v, o, lse, do, cu_q, cu_k, mq, mk, causal)
    _status_ok()
    rq, rk, rv = attention_bwd_varlen(fq, fk, fv, fdo, hq, hk, 1.0 / np.sqrt(d), causal)
    assert_close("dQ", to_f64(dq), rq)
    assert_close("dK", to_f64(dk), rk, scale_max_abs=H_kv < H)
    assert_close("dV", to_f64(dv), rv, scale_max_abs=H_kv < H)


@pytest.mark.parametrize("N,d,causal", [(300, 128, True), (520, 64, False)])
def test_backward_strided_is_the_dense_result(N, d, causal):
    """[B, N, H, d] memory: dK, dV bitwise equal to the dense call; dQ within tolerance of it."""
    import exact_io_aware_100_b200 as fa
    B, H = 2, 4
    t = {n: _tensor(3600 + N, n, (B, H, N, d))[0] for n in ("q", "k", "v", "do")}
    o, lse = fa.forward(t["q"], t["k"], t["v"], causal)
    ref = fa.backward(t["q"], t["k"], t["v"], o, lse, t["do"], causal)
    s = {n: x.transpose(1, 2).contiguous().transpose(1, 2) for n, x in t.items()}
    os_ = o.transpose(1, 2).contiguous().transpose(1, 2)
    got = fa.backward(s["q"], s["k"], s["v"], os_, lse, s["do"], causal)
    _status_ok()
    assert got[0].stride() == s["q"].stride()
    import torch
    assert torch.equal(got[1].contiguous(), ref[1]) and torch.equal(got[2].contiguous(), ref[2])
    assert_close("dQ", to_f64(got[0].contiguous()), to_f64(ref[0]), max_abs=1e-2, rel_l2=1e-3)


def test_inconsistent_offsets_are_reported_not_followed():
    """Offsets past the packed tensors, or a sequence longer than the stated maximum, are
    skipped on the device and reported as FA_ERR_INVALID; the other sequences are computed."""
    import torch
    import exact_io_aware_100_b200 as fa
    H, d = 2, 128
    (q, k, v, cu_q, cu_k), (fq, fk, fv, hq, hk) = _packed_case([(100, 100), (50, 60)], H, H, d, 3700)
    o, lse = fa.forward_varlen(q, k, v, cu_q, cu_k, 100, 100, True)
    _status_ok()
    # sequence 1 ends past the packed tensor; then sequence 0 is longer than the stated maximum
    for bad_q, mq, good, bad in (([0, 100, 400], 100, slice(0, 100), slice(100, 150)),
                                 ([0, 100, 150], 60, slice(100, 150), slice(0, 100))):
        o2 = torch.full_like(o, 7.0)
        lse2 = torch.empty_like(lse)
        L = fa.layout_packed(q, k, v, o2, torch.tensor(bad_q, dtype=torch.int32, device="cuda"), cu_k, mq, 100)
        fa.fa_fwd_general(q, k, v, o2, lse2, L, True)
        torch.cuda.synchronize()
        assert fa.fa_get_device_status() == fa.FA_ERR_INVALID
        assert torch.equal(o2[good], o[good])              # the consistent sequence is still computed
        assert torch.all(o2[bad] == 7.0)                   # the inconsistent one is not written
