"""Parity at the full sizes the benchmark times, on sampled heads, rows and sequences.

Each workload runs through the C ABI exactly as bench.py launches it (same
entry point, same sizes, same seeded inputs), so every scheduling group of the
persistent tile orders is exercised; the fp64 oracle then checks whole heads
(backward), sampled query rows (forward) or whole sequences (packed batches)
taken from different scheduling groups.  Tolerances are the ones every parity
test uses: max-abs 2e-2 and relative L2 5e-3 on O, dQ, dK, dV; 1e-3 on lse.

Definitions: the unite.ai page's ``standard_attention`` listing (forward) and
the deepfa.ir page, section "Technique 2: recomputation" (the backward is the
exact gradient of that forward); grouped heads and head dim 256 from the
nearauto.com FlashAttention-2 digest, section on head dimensions up to 256 and
multi-query attention.
"""
import numpy as np
import pytest

from exact_io_aware_100_b200 import inputs
from oracle import (attention_bwd, attention_bwd_gqa, attention_bwd_sampled, attention_bwd_varlen,
                    attention_fwd_rows, attention_fwd_varlen, bwd_operand_rounding_bound)
from tests.helpers import assert_close, assert_close_bwd, assert_lse, to_device, to_f64

pytestmark = pytest.mark.gpu


def _bf16(host):
    return {n: to_device(x, "bf16") for n, x in host.items()}


def _status_ok():
    import torch
    import exact_io_aware_100_b200 as fa
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == fa.FA_OK


def _sampled_rows(w, host, o, lse, heads, rows_per_head=256):
    """O and lse of sampled query rows of the given (b * H + h) heads against all keys."""
    o64, lse64 = to_f64(o), to_f64(lse)
    group = w.H // w.kv_heads
    got_o, ref_o, got_l, ref_l = [], [], [], []
    for bh in heads:
        b, h = divmod(bh, w.H)
        g = h // group
        rows = inputs.sample_rows(w.seed + 31 * bh, w.N, rows_per_head)
        q = inputs.to_f64(host["q"][b, h, rows], "bf16")
        k = inputs.to_f64(host["k"][b, g], "bf16")
        v = inputs.to_f64(host["v"][b, g], "bf16")
        ro, rl = attention_fwd_rows(q, k, v, rows, w.scale, w.causal)
        got_o.append(o64[b, h, rows]); ref_o.append(ro)
        got_l.append(lse64[b, h, rows]); ref_l.append(rl)
    assert_close("O(sampled rows)", np.concatenate(got_o), np.concatenate(ref_o))
    assert_lse(np.concatenate(got_l), np.concatenate(ref_l))
    assert np.isfinite(o64).all() and np.isfinite(lse64).all()


def test_prefill_backward_full_size_sampled_heads():
    """The benchmark's default step (B=2 H=32 N=8192 d=128, K x2, causal): forward, then the
    backward's three phases; whole heads from four different backward scheduling groups."""
    import exact_io_aware_100_b200 as fa
    w = inputs.WORKLOADS["prefill"]
    host = inputs.make_inputs(w, names=("q", "k", "v", "do"))
    t = _bf16(host)
    o, lse = fa.forward(t["q"], t["k"], t["v"], w.causal)
    dq, dk, dv = fa.backward(t["q"], t["k"], t["v"], o, lse, t["do"], w.causal)
    _status_ok()
    g, r, bnd = ({"dq": [], "dk": [], "dv": []} for _ in range(3))
    for bh in (0, 21, 42, 63):
        b, h = divmod(bh, w.H)
        f = {n: inputs.to_f64(host[n][b:b + 1, h:h + 1], "bf16") for n in ("q", "k", "v", "do")}
        ref = attention_bwd(f["q"], f["k"], f["v"], f["do"], w.scale, w.causal)
        bound = bwd_operand_rounding_bound(f["q"], f["k"], f["v"], f["do"], w.scale, w.causal)
        for name, got, rr, bb in zip(("dq", "dk", "dv"), (dq, dk, dv), ref, bound):
            g[name].append(to_f64(got[b, h]))
            r[name].append(rr[0, 0])
            bnd[name].append(bb[0, 0])
    # keys x2: dQ reaches |x| ~ 7 here; checked with the output and operand rounding terms
    for name in ("dq", "dk", "dv"):
        assert_close_bwd(name, np.concatenate(g[name]), np.concatenate(r[name]), np.concatenate(bnd[name]))
    for x in (dq, dk, dv):
        assert np.isfinite(to_f64(x)).all()


def test_prefill_noncausal_full_size():
    """The prefill shape without the causal mask (B=2 H=32 N=8192 d=128, K x2), as the benchmark's
    configuration table times it: the forward on sampled rows of heads from different tile groups,
    the backward on two whole heads."""
    import exact_io_aware_100_b200 as fa
    w = inputs.WORKLOADS["prefill_noncausal"]
    host = inputs.make_inputs(w, names=("q", "k", "v", "do"))
    t = _bf16(host)
    o, lse = fa.forward(t["q"], t["k"], t["v"], w.causal)
    dq, dk, dv = fa.backward(t["q"], t["k"], t["v"], o, lse, t["do"], w.causal)
    _status_ok()
    _sampled_rows(w, host, o, lse, (0, 21, 42, 63), rows_per_head=128)
    for bh in (5, 50):
        b, h = divmod(bh, w.H)
        f = {n: inputs.to_f64(host[n][b:b + 1, h:h + 1], "bf16") for n in ("q", "k", "v", "do")}
        ref = attention_bwd(f["q"], f["k"], f["v"], f["do"], w.scale, w.causal)
        bound = bwd_operand_rounding_bound(f["q"], f["k"], f["v"], f["do"], w.scale, w.causal)
        for name, got, rr, bb in zip(("dq", "dk", "dv"), (dq, dk, dv), ref, bound):
            assert_close_bwd(name, to_f64(got[b, h]), rr[0, 0], bb[0, 0])


def test_prefill_gqa_full_size():
    """32 query heads over 8 key/value heads at the prefill sizes: forward rows from both causal
    tile groups, and the backward of whole key/value heads (each the sum over its four query
    heads) from the first and last backward scheduling groups."""
    import exact_io_aware_100_b200 as fa
    w = inputs.WORKLOADS["prefill_gqa"]
    host = {}
    for n in ("q", "k", "v", "do"):
        heads = w.kv_heads if n in ("k", "v") else w.H
        host[n] = inputs.make_tensor(w.seed, n, (w.B, heads, w.N, w.d), w.k_scale if n == "k" else 1.0)
    t = _bf16(host)
    o, lse = fa.forward(t["q"], t["k"], t["v"], w.causal)
    dq, dk, dv = fa.backward(t["q"], t["k"], t["v"], o, lse, t["do"], w.causal)
    _status_ok()
    _sampled_rows(w, host, o, lse, heads=[0, 17, 47, 48, 63])
    group = w.H // w.kv_heads
    g, r, bnd = ({"dq": [], "dk": [], "dv": []} for _ in range(3))
    for bg in (0, 15):                      # b * H_kv + kv head
        b, kv = divmod(bg, w.kv_heads)
        hs = slice(kv * group, (kv + 1) * group)
        f = {n: inputs.to_f64(host[n][b:b + 1, hs if n in ("q", "do") else slice(kv, kv + 1)], "bf16")
             for n in ("q", "k", "v", "do")}
        rq, rk, rv = attention_bwd_gqa(f["q"], f["k"], f["v"], f["do"], w.scale, w.causal)
        bq, bk, bv = bwd_operand_rounding_bound(f["q"], f["k"], f["v"], f["do"], w.scale, w.causal)
        g["dq"].append(to_f64(dq[b, hs])); r["dq"].append(rq[0]); bnd["dq"].append(bq[0])
        g["dk"].append(to_f64(dk[b, kv])); r["dk"].append(rk[0, 0]); bnd["dk"].append(bk[0, 0])
        g["dv"].append(to_f64(dv[b, kv])); r["dv"].append(rv[0, 0]); bnd["dv"].append(bv[0, 0])
    # keys x2, and a shared head's dK, dV sum four heads' gradients: outputs of several units,
    # checked with the output and operand rounding terms
    for name in ("dq", "dk", "dv"):
        assert_close_bwd(name, np.concatenate(g[name]), np.concatenate(r[name]), np.concatenate(bnd[name]))


def test_prefill_d256_full_size():
    """Head dim 256 at B=2 H=16 N=8192, causal: forward rows from five different causal tile
    groups, and the backward of whole heads from three different backward scheduling groups."""
    import exact_io_aware_100_b200 as fa
    w = inputs.WORKLOADS["prefill_d256"]
    host = inputs.make_inputs(w, names=("q", "k", "v", "do"))
    t = _bf16(host)
    o, lse = fa.forward(t["q"], t["k"], t["v"], w.causal)
    dq, dk, dv = fa.backward(t["q"], t["k"], t["v"], o, lse, t["do"], w.causal)
    _status_ok()
    _sampled_rows(w, host, o, lse, heads=[0, 7, 14, 20, 31])
    g, r = {"dq": [], "dk": [], "dv": []}, {"dq": [], "dk": [], "dv": []}
    for bh in (0, 13, 31):
        b, h = divmod(bh, w.H)
        f = {n: inputs.to_f64(host[n][b:b + 1, h:h + 1], "bf16") for n in ("q", "k", "v", "do")}
        ref = attention_bwd(f["q"], f["k"], f["v"], f["do"], w.scale, w.causal)
        for name, got, rr in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
            g[name].append(to_f64(got[b, h]))
            r[name].append(rr[0, 0])
    for name in ("dq", "dk", "dv"):
        assert_close(name, np.concatenate(g[name]), np.concatenate(r[name]))


def test_varlen_full_size_sampled_sequences():
    """The packed batch the benchmark times (16 sequences of lengths N/8..N, 32 heads, causal):
    forward and backward of whole (sequence, head) pairs, the longest sequence and shorter ones."""
    import torch
    import exact_io_aware_100_b200 as fa
    w = inputs.WORKLOADS["varlen"]
    lens = w.seq_lengths()
    total = sum(lens)
    host = {n: inputs.make_tensor(w.seed, n, (total, w.H, w.d)) for n in ("q", "k", "v", "do")}
    t = _bf16(host)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    cu_d = torch.from_numpy(cu).cuda()
    n_max = max(lens)
    o, lse = fa.forward_varlen(t["q"], t["k"], t["v"], cu_d, cu_d, n_max, n_max, w.causal)
    dq, dk, dv = fa.backward_varlen(t["q"], t["k"], t["v"], o, lse, t["do"], cu_d, cu_d, n_max, n_max, w.causal)
    _status_ok()
    o64, lse64 = to_f64(o), to_f64(lse)
    shortest = int(np.argmin(lens))
    picks = [(0, 0), (len(lens) // 2, 17), (shortest, 31)]
    got, ref = {n: [] for n in ("o", "lse", "dq", "dk", "dv")}, {n: [] for n in ("o", "lse", "dq", "dk", "dv")}
    for s, h in picks:
        rows = slice(cu[s], cu[s + 1])
        one = np.array([0, lens[s]])
        f = {n: inputs.to_f64(host[n][rows, h:h + 1], "bf16") for n in ("q", "k", "v", "do")}
        ro, rl = attention_fwd_varlen(f["q"], f["k"], f["v"], one, one, w.scale, w.causal)
        rq, rk, rv = attention_bwd_varlen(f["q"], f["k"], f["v"], f["do"], one, one, w.scale, w.causal)
        got["o"].append(o64[rows, h]); ref["o"].append(ro[:, 0])
        got["lse"].append(lse64[h, rows]); ref["lse"].append(rl[0])
        for name, x, rr in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
            got[name].append(to_f64(x[rows, h])); ref[name].append(rr[:, 0])
    assert_close("O", np.concatenate(got["o"]), np.concatenate(ref["o"]))
    assert_lse(np.concatenate(got["lse"]), np.concatenate(ref["lse"]))
    for name in ("dq", "dk", "dv"):
        assert_close(name, np.concatenate(got[name]), np.concatenate(ref[name]))
    assert np.isfinite(o64).all() and np.isfinite(lse64).all()


def test_long_context_backward_sampled():
    """B=1 H=16 N=65536 d=128, causal (the long-context configuration; the benchmark times its
    forward and backward): dQ on 128 sampled query rows and dK, dV on 128 sampled keys of one
    head, each against the oracle's complete row or column (the oracle's forward runs the whole
    head in panels for lse and O)."""
    import exact_io_aware_100_b200 as fa
    w = inputs.WORKLOADS["long_context"]
    host = inputs.make_inputs(w, names=("q", "k", "v", "do"))
    t = _bf16(host)
    o, lse = fa.forward(t["q"], t["k"], t["v"], w.causal)
    dq, dk, dv = fa.backward(t["q"], t["k"], t["v"], o, lse, t["do"], w.causal)
    _status_ok()
    h = 11
    rows = inputs.sample_rows(w.seed + 5, w.N, 128)
    keys = inputs.sample_rows(w.seed + 6, w.N, 128)
    f = {n: inputs.to_f64(host[n][0, h], "bf16") for n in ("q", "k", "v", "do")}
    rq, rk, rv = attention_bwd_sampled(f["q"], f["k"], f["v"], f["do"], rows, keys, w.scale, w.causal)
    assert_close("dq(sampled rows)", to_f64(dq[0, h, rows]), rq)
    assert_close("dk(sampled keys)", to_f64(dk[0, h, keys]), rk)
    assert_close("dv(sampled keys)", to_f64(dv[0, h, keys]), rv)
    for x in (dq, dk, dv):
        assert np.isfinite(to_f64(x)).all()
