"""Grouped-query and multi-query attention on the GPU against the fp64 oracle.

Query heads in contiguous sets share one key/value head (the nearauto.com
FlashAttention-2 digest, section on multi-query and grouped-query attention);
the oracle is attention_fwd_gqa / attention_bwd_gqa.  Same tolerances as the
multi-head path.
"""
import numpy as np
import pytest

from exact_io_aware_100_b200 import inputs
from helpers import assert_close, assert_lse, to_device, to_f64
from oracle import attention_bwd_gqa, attention_fwd_gqa

pytestmark = pytest.mark.gpu


def _case(B, H, H_kv, N, d, seed, names):
    host, f64 = {}, {}
    for n in names:
        heads = H_kv if n in ("k", "v") else H
        host[n] = inputs.make_tensor(seed, n, (B, heads, N, d))
        f64[n] = inputs.to_f64(host[n], "bf16")
    return host, f64


@pytest.mark.parametrize("B,H,H_kv,N,d,causal", [
    (2, 8, 2, 300, 128, True),
    (2, 8, 2, 300, 128, False),
    (1, 6, 1, 257, 128, True),      # multi-query
    (1, 6, 6, 129, 128, True),      # H_kv == H: plain multi-head through the grouped entry point
    (2, 4, 2, 520, 64, True),
    (1, 8, 1, 333, 64, False),
])
def test_gqa_forward_matches_oracle(B, H, H_kv, N, d, causal):
    import torch
    import exact_io_aware_100_b200 as fa
    host, f64 = _case(B, H, H_kv, N, d, 2100 + H + N, ("q", "k", "v"))
    q, k, v = (to_device(host[n], "bf16") for n in ("q", "k", "v"))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    fa.fa_fwd_gqa(q, k, v, o, lse, causal)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == fa.FA_OK
    ro, rl = attention_fwd_gqa(f64["q"], f64["k"], f64["v"], 1.0 / np.sqrt(d), causal)
    assert_close("O", to_f64(o), ro)
    assert_lse(to_f64(lse), rl)


@pytest.mark.parametrize("B,H,H_kv,N,causal,d", [
    (1, 4, 2, 300, True, 128),
    (1, 4, 2, 257, False, 128),
    (2, 3, 1, 200, True, 128),      # multi-query
    (1, 8, 2, 640, True, 128),
    (1, 4, 2, 300, True, 64),
    (2, 6, 1, 200, False, 64),
])
def test_gqa_backward_matches_oracle(B, H, H_kv, N, causal, d):
    import torch
    import exact_io_aware_100_b200 as fa
    host, f64 = _case(B, H, H_kv, N, d, 2200 + H + N, ("q", "k", "v", "do"))
    q, k, v, do = (to_device(host[n], "bf16") for n in ("q", "k", "v", "do"))
    o, lse = fa.forward(q, k, v, causal)
    dq, dk, dv = fa.backward(q, k, v, o, lse, do, causal)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == fa.FA_OK
    assert dk.shape == k.shape and dv.shape == v.shape
    rq, rk, rv = attention_bwd_gqa(f64["q"], f64["k"], f64["v"], f64["do"], 1.0 / np.sqrt(d), causal)
    assert_close("dQ", to_f64(dq), rq)
    # dK, dV of a shared head sum its set's gradients (fp32, one bf16 rounding at the
    # end), so their magnitude -- and a bf16 ulp of it -- grows with the set: the
    # max-abs bound scales with max(1, max|ref|), the rel-L2 bound does not change
    assert_close("dK", to_f64(dk), rk, scale_max_abs=True)
    assert_close("dV", to_f64(dv), rv, scale_max_abs=True)


def test_gqa_matches_repeated_heads_bitwise():
    """The forward of a grouped case equals, bit for bit, the multi-head forward
    with each key/value head repeated for its set (same kernel arithmetic)."""
    import torch
    import exact_io_aware_100_b200 as fa
    B, H, H_kv, N, d = 1, 8, 2, 384, 128
    host, _ = _case(B, H, H_kv, N, d, 2300, ("q", "k", "v"))
    q, k, v = (to_device(host[n], "bf16") for n in ("q", "k", "v"))
    o, lse = fa.forward(q, k, v, True)
    g = H // H_kv
    o2, lse2 = fa.forward(q, k.repeat_interleave(g, dim=1).contiguous(), v.repeat_interleave(g, dim=1).contiguous(),
                          True)
    torch.cuda.synchronize()
    assert torch.equal(o, o2) and torch.equal(lse, lse2)
