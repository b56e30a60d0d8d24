"""Backward parity: dQ, dK, dV from the CUDA path against the fp64 oracle."""
import numpy as np
import pytest

from exact_io_aware_100_b200 import inputs
from oracle import attention_bwd
from tests.helpers import assert_close, make_case, to_device, to_f64

pytestmark = pytest.mark.gpu


def run_bwd(host, causal, scale=None):
    import torch
    import exact_io_aware_100_b200 as fa
    q, k, v, do = (to_device(host[n], "bf16") for n in ("q", "k", "v", "do"))
    o, lse = fa.forward(q, k, v, causal, scale)
    dq, dk, dv = fa.backward(q, k, v, o, lse, do, causal, scale)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == fa.FA_OK
    return dq, dk, dv


def check_heads(host, dq, dk, dv, heads, H, causal, scale, scale_max_abs=False):
    g = {"dq": [], "dk": [], "dv": []}
    r = {"dq": [], "dk": [], "dv": []}
    for bh in heads:
        b, h = divmod(bh, H)
        f = {n: inputs.to_f64(host[n][b:b + 1, h:h + 1], "bf16") for n in ("q", "k", "v", "do")}
        rq, rk, rv = attention_bwd(f["q"], f["k"], f["v"], f["do"], scale, causal)
        g["dq"].append(to_f64(dq[b, h])); r["dq"].append(rq[0, 0])
        g["dk"].append(to_f64(dk[b, h])); r["dk"].append(rk[0, 0])
        g["dv"].append(to_f64(dv[b, h])); r["dv"].append(rv[0, 0])
    for n in ("dq", "dk", "dv"):
        assert_close(n, np.concatenate(g[n]), np.concatenate(r[n]), scale_max_abs=scale_max_abs)


def test_backward_workload_sampled_heads():
    w = inputs.WORKLOADS["backward"]
    host = inputs.make_inputs(w, names=("q", "k", "v", "do"))
    dq, dk, dv = run_bwd(host, w.causal)
    heads = [0, 9, 18, 27, 36, 45, 54, 63]
    check_heads(host, dq, dk, dv, heads, w.H, w.causal, w.scale)
    for t in (dq, dk, dv):
        assert np.isfinite(to_f64(t)).all()


@pytest.mark.parametrize("N", [1, 63, 64, 100, 128, 129, 257, 500])
@pytest.mark.parametrize("causal", [False, True])
def test_backward_ragged(N, causal):
    B, H, d = 2, 2, 128
    host, _ = make_case(B, H, N, d, 9000 + N, names=("q", "k", "v", "do"))
    dq, dk, dv = run_bwd(host, causal)
    check_heads(host, dq, dk, dv, range(B * H), H, causal, 1.0 / np.sqrt(d))


@pytest.mark.parametrize("N", [1, 100, 129, 300, 640])
@pytest.mark.parametrize("causal", [False, True])
def test_backward_head_dim_64(N, causal):
    B, H, d = 2, 3, 64
    host, _ = make_case(B, H, N, d, 9300 + N, names=("q", "k", "v", "do"))
    dq, dk, dv = run_bwd(host, causal)
    check_heads(host, dq, dk, dv, range(B * H), H, causal, 1.0 / np.sqrt(d))


@pytest.mark.parametrize("name", ["multi_head", "multi_head_causal"])
def test_backward_multi_head_workload_sampled_heads(name):
    """The multi-head configuration (B=4 H=16 N=2048, d = 64, causal and not) on sampled heads,
    with the workload's own seeded inputs."""
    w = inputs.WORKLOADS[name]
    host = inputs.make_inputs(w, names=("q", "k", "v", "do"))
    dq, dk, dv = run_bwd(host, w.causal)
    check_heads(host, dq, dk, dv, [0, 21, 42, 63], w.H, w.causal, w.scale)


def test_backward_many_heads_and_sharp_rows():
    B, H, N, d = 3, 7, 320, 128
    host, _ = make_case(B, H, N, d, 9100, k_scale=4.0, names=("q", "k", "v", "do"))
    dq, dk, dv = run_bwd(host, True)
    # keys x4: gradients reach |x| ~ 16, where one bf16 ulp is 0.0625
    check_heads(host, dq, dk, dv, range(B * H), H, True, 1.0 / np.sqrt(d), scale_max_abs=True)


def test_backward_single_key_closed_form():
    """N = 1: O = V, so dV = dO and dQ = dK = 0 (up to fp32 rounding of dP - D)."""
    host, _ = make_case(1, 3, 1, 128, 9200, names=("q", "k", "v", "do"))
    dq, dk, dv = run_bwd(host, True)
    assert np.abs(to_f64(dq)).max() < 1e-3 and np.abs(to_f64(dk)).max() < 1e-3
    assert_close("dv", to_f64(dv), inputs.to_f64(host["do"], "bf16"))
