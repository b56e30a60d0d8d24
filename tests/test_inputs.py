"""The seeded input generator: determinism and bfloat16 rounding."""
import numpy as np
import torch

from exact_io_aware_100_b200 import inputs


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32),
                        np.array([1.0, -2.5, 1e-30, 3.0e38, 0.0, -0.0], np.float32),
                        # exact ties: mantissa ends in 0x8000
                        (np.arange(64, dtype=np.uint32) << 16 | 0x8000).view(np.float32)])
    ours = inputs.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)
    back = inputs.bf16_bits_to_f32(ours)
    np.testing.assert_array_equal(back, torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_seeded_and_distinct():
    a = inputs.make_tensor(7, "q", (4, 5))
    b = inputs.make_tensor(7, "q", (4, 5))
    c = inputs.make_tensor(7, "k", (4, 5))
    np.testing.assert_array_equal(a, b)
    assert not np.array_equal(a, c)


def test_workload_shapes_and_k_scale():
    w = inputs.WORKLOADS["prefill"]
    assert (w.B, w.H, w.N, w.d, w.causal, w.k_scale) == (2, 32, 8192, 128, True, 2.0)
    small = inputs.Workload("t", 1, 1, 64, 8, True, "bf16", 2.0, 5)
    x = inputs.make_inputs(small)
    k = inputs.to_f64(x["k"], "bf16")
    k_raw = inputs.to_f64(inputs.make_tensor(5, "k", (1, 1, 64, 8)), "bf16")
    np.testing.assert_array_equal(k, 2.0 * k_raw)   # x2 is exact in bf16
    assert inputs.WORKLOADS["single_head"].dtype == "f32"


def test_flops_convention():
    w = inputs.WORKLOADS["multi_head"]
    assert w.fwd_flops() == 4 * 4 * 16 * 2048 * 2048 * 64
    assert inputs.WORKLOADS["multi_head_causal"].fwd_flops() == w.fwd_flops() / 2


def test_sample_rows():
    r = inputs.sample_rows(3, 65536, 256)
    assert r[0] == 0 and r[-1] == 65535 and len(r) <= 256 and len(set(r)) == len(r)
    assert (np.diff(r) > 0).all()


def test_varlen_lengths_and_flops():
    w = inputs.WORKLOADS["varlen"]
    lens = w.seq_lengths()
    assert len(lens) == w.B and lens[0] == w.N and all(w.N // 8 <= n <= w.N for n in lens)
    assert lens == w.seq_lengths() and len(set(lens)) > w.B // 2
    assert w.fwd_flops() == sum(4 * w.H * n * n * w.d for n in lens) / 2
    assert inputs.WORKLOADS["prefill"].seq_lengths() == [8192, 8192]
