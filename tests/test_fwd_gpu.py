"""Forward parity: the CUDA path (through the C ABI) against the fp64 oracle."""
import numpy as np
import pytest

from exact_io_aware_100_b200 import inputs
from oracle import attention_fwd, attention_fwd_rows
from tests.helpers import assert_close, assert_lse, errors, make_case, to_device, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    import torch
    import exact_io_aware_100_b200 as fa
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    fa.load_library()


def run_fwd(host, dtype, causal, scale=None):
    import torch
    import exact_io_aware_100_b200 as fa
    q, k, v = (to_device(host[n], dtype) for n in ("q", "k", "v"))
    o, lse = fa.forward(q, k, v, causal, scale)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == fa.FA_OK
    return o, lse


def full_check(B, H, N, d, causal, seed, k_scale=1.0, dtype="bf16", scale_max_abs=False):
    host, f = make_case(B, H, N, d, seed, k_scale, dtype)
    if dtype == "f32":   # the library rounds fp32 inputs to bf16; the oracle sees the same values
        f = {n: inputs.to_f64(inputs.f32_to_bf16_bits(host[n]), "bf16") for n in host}
    o, lse = run_fwd(host, dtype, causal)
    o_ref, lse_ref = attention_fwd(f["q"], f["k"], f["v"], 1.0 / np.sqrt(d), causal)
    assert_close("O", to_f64(o), o_ref, scale_max_abs=scale_max_abs)
    assert_lse(to_f64(lse), lse_ref)
    return host, o, lse


# ---------------------------------------------------------------- the workloads
def test_single_head_fp32_inputs():
    w = inputs.WORKLOADS["single_head"]
    host, o, lse = full_check(w.B, w.H, w.N, w.d, w.causal, w.seed, dtype="f32")
    # against the unrounded fp32 inputs the bf16 rounding of q, k, v shows up
    f32 = {n: host[n].astype(np.float64) for n in host}
    o_ref, _ = attention_fwd(f32["q"], f32["k"], f32["v"], w.scale, w.causal)
    ma, rl = errors(to_f64(o), o_ref)
    assert ma < 3e-2 and rl < 1e-2, (ma, rl)


@pytest.mark.parametrize("B,H,N,d,causal", [
    (1, 1, 1, 64, True), (2, 3, 17, 64, False), (1, 2, 100, 128, True), (2, 2, 128, 128, False),
    (1, 1, 128, 64, True), (1, 2, 129, 64, True), (1, 1, 300, 128, False),
])
def test_fp32_inputs_short_and_long(B, H, N, d, causal):
    """fa_fwd_ex(FA_F32) on short and ragged lengths: cast to bf16, then the tensor-core kernel."""
    full_check(B, H, N, d, causal, 8800 + N + d, dtype="f32")


@pytest.mark.parametrize("name", ["multi_head", "multi_head_causal"])
def test_multi_head(name):
    w = inputs.WORKLOADS[name]
    full_check(w.B, w.H, w.N, w.d, w.causal, w.seed)


def sampled_check(w, heads, rows_per_head):
    host = inputs.make_inputs(w)
    o, lse = run_fwd(host, "bf16", w.causal)
    o64, lse64 = to_f64(o), to_f64(lse)
    got_o, ref_o, got_l, ref_l = [], [], [], []
    for hh, bh in enumerate(heads):
        b, h = divmod(bh, w.H)
        rows = inputs.sample_rows(w.seed + 17 * bh, w.N, rows_per_head)
        q = inputs.to_f64(host["q"][b, h, rows], "bf16")
        k = inputs.to_f64(host["k"][b, h], "bf16")
        v = inputs.to_f64(host["v"][b, h], "bf16")
        ro, rl = attention_fwd_rows(q, k, v, rows, w.scale, w.causal)
        got_o.append(o64[b, h, rows]); ref_o.append(ro)
        got_l.append(lse64[b, h, rows]); ref_l.append(rl)
        if w.causal:   # causal row 0 sees key 0 only: O_0 = V_0 (rounded once to bf16)
            np.testing.assert_allclose(o64[b, h, 0], v[0], atol=1e-6)
    assert_close("O(sampled)", np.concatenate(got_o), np.concatenate(ref_o))
    assert_lse(np.concatenate(got_l), np.concatenate(ref_l))
    assert np.isfinite(o64).all() and np.isfinite(lse64).all()


def test_prefill_causal_sampled():
    w = inputs.WORKLOADS["prefill"]
    sampled_check(w, heads=[0, 13, 31, 32, 50, 63], rows_per_head=256)


def test_long_context_sampled():
    w = inputs.WORKLOADS["long_context"]
    sampled_check(w, heads=list(range(w.B * w.H)), rows_per_head=256)


# ---------------------------------------------------------------- edge cases
@pytest.mark.parametrize("N", [1, 2, 127, 128, 129, 255, 256, 257, 383, 640, 1000])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_ragged_lengths(N, d, causal):
    full_check(2, 3, N, d, causal, seed=7000 + N + d)


@pytest.mark.parametrize("BH", [(1, 1), (1, 200), (37, 5)])
def test_batch_head_counts_around_sm_count(BH):
    B, H = BH
    full_check(B, H, 384, 64, True, seed=8000 + B * H)


def test_sharp_softmax_rows():
    # large scores: several rescales per row and near one-hot rows
    full_check(1, 4, 700, 128, True, seed=8100, k_scale=6.0, scale_max_abs=True)
    full_check(1, 4, 700, 64, False, seed=8101, k_scale=6.0, scale_max_abs=True)


def test_constant_v_gives_constant_o():
    import torch
    import exact_io_aware_100_b200 as fa
    host, _ = make_case(1, 2, 1000, 128, 8200, k_scale=3.0)
    row = host["v"][0, 0, 0].copy()
    host["v"][:] = row
    q, k, v = (to_device(host[n], "bf16") for n in ("q", "k", "v"))
    o, _ = fa.forward(q, k, v, True)
    vf = inputs.to_f64(row, "bf16")
    np.testing.assert_allclose(to_f64(o)[0, 0], np.broadcast_to(vf, (1000, 128)), atol=2e-2)


def test_deterministic_and_no_out_of_bounds_writes():
    import torch
    import exact_io_aware_100_b200 as fa
    B, H, N, d = 2, 2, 333, 128
    host, _ = make_case(B, H, N, d, 8300)
    q, k, v = (to_device(host[n], "bf16") for n in ("q", "k", "v"))
    guard = 4096
    o_buf = torch.full((B * H * N * d + 2 * guard,), 7.0, dtype=torch.bfloat16, device="cuda")
    l_buf = torch.full((B * H * N + 2 * guard,), 7.0, dtype=torch.float32, device="cuda")
    o = o_buf[guard:guard + B * H * N * d].view(B, H, N, d)
    lse = l_buf[guard:guard + B * H * N].view(B, H, N)
    outs = []
    for _ in range(2):
        fa.fa_fwd(q, k, v, o, lse, True)
        torch.cuda.synchronize()
        outs.append((o.clone(), lse.clone()))
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])
    assert (o_buf[:guard] == 7).all() and (o_buf[-guard:] == 7).all()
    assert (l_buf[:guard] == 7).all() and (l_buf[-guard:] == 7).all()


def test_custom_scale():
    import exact_io_aware_100_b200 as fa
    host, f = make_case(1, 2, 300, 64, 8400)
    q, k, v = (to_device(host[n], "bf16") for n in ("q", "k", "v"))
    o, lse = fa.forward(q, k, v, True, scale=0.05)
    o_ref, l_ref = attention_fwd(f["q"], f["k"], f["v"], 0.05, True)
    assert_close("O", to_f64(o), o_ref)
    assert_lse(to_f64(lse), l_ref)


def test_timeout_path_reports_status_and_context_survives():
    import torch
    import exact_io_aware_100_b200 as fa
    fa.fa_selftest_wait_timeout(20_000_000)          # 20 ms bounded wait nobody completes
    assert fa.fa_get_device_status() == fa.FA_ERR_TIMEOUT
    assert fa.fa_get_device_status() == fa.FA_OK      # read-and-clear
    full_check(1, 1, 200, 64, True, seed=8500)       # the context still works
