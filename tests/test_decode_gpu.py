"""Decode (few queries against a key/value cache, split keys merged) on the GPU
against the fp64 oracle's attention_fwd_decode.  Same tolerances as the forward."""
import numpy as np
import pytest

from exact_io_aware_100_b200 import inputs
from helpers import assert_close, assert_lse, to_device, to_f64
from oracle import attention_fwd_decode

pytestmark = pytest.mark.gpu


def _case(B, H, H_kv, Lq, Nk, seed, k_scale=1.0):
    d = 128
    host = {"q": inputs.make_tensor(seed, "q", (B, H, Lq, d)),
            "k": inputs.make_tensor(seed, "k", (B, H_kv, Nk, d), k_scale),
            "v": inputs.make_tensor(seed, "v", (B, H_kv, Nk, d))}
    f64 = {n: inputs.to_f64(x, "bf16") for n, x in host.items()}
    return host, f64


@pytest.mark.parametrize("B,H,H_kv,Lq,Nk,causal", [
    (2, 8, 2, 1, 1000, True),       # one token, grouped heads
    (1, 4, 4, 1, 4096, False),      # plain multi-head
    (2, 8, 1, 2, 777, True),        # multi-query, two tokens, ragged cache
    (1, 4, 1, 4, 63, True),         # cache shorter than one tile
    (1, 2, 2, 16, 2049, True),      # 16 tokens per head (causal bottom-right inside the last tile)
    (3, 6, 3, 8, 5000, False),
    (1, 16, 2, 2, 65536, True),     # long cache: many splits
    (4, 8, 4, 1, 8192, False),      # two rows per key/value head (warp-tiled kernel)
    (1, 4, 1, 1, 100, True),        # four rows, cache shorter than one split's first tiles
    (2, 4, 2, 2, 333, True),        # two query heads x two positions (causal inside the last tile)
    (1, 3, 1, 1, 17, True),         # three rows, one partial tile
    (2, 2, 2, 1, 1, True),          # a single cached key
])
def test_decode_matches_oracle(B, H, H_kv, Lq, Nk, causal):
    import torch
    import exact_io_aware_100_b200 as fa
    host, f64 = _case(B, H, H_kv, Lq, Nk, 3100 + Lq + Nk % 97)
    q, k, v = (to_device(host[n], "bf16") for n in ("q", "k", "v"))
    o, lse = fa.decode(q, k, v, causal)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == fa.FA_OK
    ro, rl = attention_fwd_decode(f64["q"], f64["k"], f64["v"], 1.0 / np.sqrt(128), causal)
    assert_close("O", to_f64(o), ro)
    assert_lse(to_f64(lse), rl)


def test_decode_sharp_scores():
    """K scaled by 4: sharp softmax rows, the split partials differ by many e-folds."""
    import torch
    import exact_io_aware_100_b200 as fa
    host, f64 = _case(1, 8, 2, 1, 3000, 3200, k_scale=4.0)
    q, k, v = (to_device(host[n], "bf16") for n in ("q", "k", "v"))
    o, lse = fa.decode(q, k, v, True)
    torch.cuda.synchronize()
    ro, rl = attention_fwd_decode(f64["q"], f64["k"], f64["v"], 1.0 / np.sqrt(128), True)
    assert_close("O", to_f64(o), ro)
    assert_lse(to_f64(lse), rl)


def test_decode_of_the_whole_sequence_matches_the_forward():
    """Lq == Nk is ordinary causal attention: decode equals the forward kernel's result
    within the forward tolerance."""
    import torch
    import exact_io_aware_100_b200 as fa
    host, _ = _case(1, 4, 4, 16, 16, 3300)
    q, k, v = (to_device(host[n], "bf16") for n in ("q", "k", "v"))
    o1, l1 = fa.decode(q, k, v, True)
    o2, l2 = fa.forward(q, k, v, True)
    torch.cuda.synchronize()
    assert_close("O", to_f64(o1), to_f64(o2))
    assert_lse(to_f64(l1), to_f64(l2).astype(np.float64))


@pytest.mark.parametrize("B,H,H_kv,Lq,Nk,d,causal", [
    (2, 32, 1, 1, 1000, 128, True),     # 32 query rows per key/value head: beyond the split-key kernel
    (1, 8, 2, 4, 700, 64, True),        # head dim 64
    (1, 4, 4, 3, 500, 256, False),      # head dim 256
    (1, 4, 2, 9, 300, 256, True),
])
def test_decode_other_shapes_match_oracle(B, H, H_kv, Lq, Nk, d, causal):
    """Shapes the split-key kernel does not take run the general forward; same result."""
    import torch
    import exact_io_aware_100_b200 as fa
    seed = 3300 + Lq + d
    host = {"q": inputs.make_tensor(seed, "q", (B, H, Lq, d)),
            "k": inputs.make_tensor(seed, "k", (B, H_kv, Nk, d)),
            "v": inputs.make_tensor(seed, "v", (B, H_kv, Nk, d))}
    f64 = {n: inputs.to_f64(x, "bf16") for n, x in host.items()}
    q, k, v = (to_device(host[n], "bf16") for n in ("q", "k", "v"))
    o, lse = fa.decode(q, k, v, causal)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == fa.FA_OK
    ro, rl = attention_fwd_decode(f64["q"], f64["k"], f64["v"], 1.0 / np.sqrt(d), causal)
    assert_close("O", to_f64(o), ro)
    assert_lse(to_f64(lse), rl)


def test_decode_workload_full_size():
    """The benchmarked decode workload: 16 sequences, 32 query heads over 8 key/value heads, one
    new token against 8192 cached keys, every query head checked."""
    import torch
    import exact_io_aware_100_b200 as fa
    w = inputs.WORKLOADS["decode"]
    shapes = {"q": (w.B, w.H, w.lq, w.d), "k": (w.B, w.kv_heads, w.N, w.d), "v": (w.B, w.kv_heads, w.N, w.d)}
    host = {n: inputs.make_tensor(w.seed, n, shp) for n, shp in shapes.items()}
    q, k, v = (to_device(host[n], "bf16") for n in ("q", "k", "v"))
    o, lse = fa.decode(q, k, v, w.causal)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == fa.FA_OK
    f64 = {n: inputs.to_f64(x, "bf16") for n, x in host.items()}
    ro, rl = attention_fwd_decode(f64["q"], f64["k"], f64["v"], w.scale, w.causal)
    assert_close("O", to_f64(o), ro)
    assert_lse(to_f64(lse), rl)
