"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the oracle.

This module holds no attention arithmetic: it draws i.i.d. standard normals
from numpy's PCG64 generator and rounds them to bfloat16 (round to nearest,
ties to even).  Both sides of every parity check are fed the same bytes.

Workloads (the pages measure on no dataset; these shapes follow the attention
benchmarks the FlashAttention-2 digest on nearauto.com describes: head dim 64
or 128, causal and non-causal, long sequences):

  ``single_head``  B=1  H=1  N=128    d=64   fp32 inputs, non-causal
  ``multi_head``   B=4  H=16 N=2048   d=64   bf16, non-causal and causal
  ``prefill``      B=2  H=32 N=8192   d=128  bf16, K scaled by 2, causal
  ``prefill_noncausal``  the same, non-causal
  ``long_context`` B=1  H=16 N=65536  d=128  bf16, causal
  ``backward``     B=4  H=16 N=4096   d=128  bf16 Q,K,V,dO, causal

Seeds: each workload has a base seed; tensor ids 0..3 select Q, K, V, dO.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

TENSOR_IDS = {"q": 0, "k": 1, "v": 2, "do": 3}


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    causal: bool
    dtype: str          # "f32" or "bf16": element type handed to the library
    k_scale: float      # K is multiplied by this before rounding
    seed: int
    backward: bool = False
    h_kv: int = 0       # key/value heads (0: as many as query heads)
    lq: int = 0         # decoding: this many query positions against N cached keys (0: N queries)
    varlen: bool = False  # packed batch of B sequences of seq_lengths() rows (N the longest)

    @property
    def kv_heads(self) -> int:
        return self.h_kv or self.H

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def seq_lengths(self) -> list:
        """Rows of each sequence: N for fixed-length workloads; for a packed batch,
        seeded lengths uniform in [N / 8, N] (ragged, not tile multiples), the first
        one N itself."""
        if not self.varlen:
            return [self.N] * self.B
        rng = np.random.default_rng([int(self.seed), 7])
        lens = rng.integers(self.N // 8, self.N + 1, size=self.B)
        lens[0] = self.N
        return [int(x) for x in lens]

    def fwd_flops(self) -> float:
        if self.varlen:
            f = sum(4.0 * self.H * n * n * self.d for n in self.seq_lengths())
            return f / 2 if self.causal else f
        if self.lq:
            # query i of the last lq positions sees N - lq + i + 1 keys when causal, all N otherwise
            keys = (self.lq * (self.N - self.lq) + self.lq * (self.lq + 1) // 2) if self.causal else self.lq * self.N
            return 4.0 * self.B * self.H * keys * self.d
        f = 4.0 * self.B * self.H * self.N * self.N * self.d
        return f / 2 if self.causal else f


WORKLOADS = {
    "single_head": Workload("single_head", 1, 1, 128, 64, False, "f32", 1.0, 1001),
    "multi_head": Workload("multi_head", 4, 16, 2048, 64, False, "bf16", 1.0, 1002),
    "multi_head_causal": Workload("multi_head_causal", 4, 16, 2048, 64, True, "bf16", 1.0, 1002),
    "prefill": Workload("prefill", 2, 32, 8192, 128, True, "bf16", 2.0, 1003),
    "prefill_noncausal": Workload("prefill_noncausal", 2, 32, 8192, 128, False, "bf16", 2.0, 1010),
    "long_context": Workload("long_context", 1, 16, 65536, 128, True, "bf16", 1.0, 1004),
    "backward": Workload("backward", 4, 16, 4096, 128, True, "bf16", 1.0, 1005, True),
    # grouped-query attention on the prefill shape: 32 query heads over 8 key/value heads
    "prefill_gqa": Workload("prefill_gqa", 2, 32, 8192, 128, True, "bf16", 2.0, 1006, False, 8),
    # decoding one token per sequence against an 8192-key cache, 32 query heads over 8 key/value heads
    "decode": Workload("decode", 16, 32, 8192, 128, True, "bf16", 1.0, 1007, False, 8, 1),
    # head dim 256: 16 heads of 8192 rows, causal
    "prefill_d256": Workload("prefill_d256", 2, 16, 8192, 256, True, "bf16", 1.0, 1009),
    # a packed batch of 16 sequences of mixed lengths (up to 8192), causal
    "varlen": Workload("varlen", 16, 32, 8192, 128, True, "bf16", 1.0, 1008, varlen=True),
}


def normal_f32(seed: int, tensor_id: int, shape) -> np.ndarray:
    """i.i.d. N(0,1) float32 of ``shape`` from PCG64 seeded by (seed, tensor_id)."""
    rng = np.random.default_rng([int(seed), int(tensor_id)])
    return rng.standard_normal(size=tuple(shape), dtype=np.float32)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest, ties to even); returns uint16 bits.

    Inputs here are finite normals, so NaN handling is not needed.
    """
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns (uint16) to float32."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def make_tensor(seed: int, name: str, shape, mult: float = 1.0,
                dtype: str = "bf16") -> np.ndarray:
    """One seeded input tensor.

    ``dtype="bf16"`` returns uint16 bfloat16 bits; ``dtype="f32"`` returns the
    float32 values themselves.
    """
    x = normal_f32(seed, TENSOR_IDS[name], shape)
    if mult != 1.0:
        x = x * np.float32(mult)
    if dtype == "f32":
        return x
    return f32_to_bf16_bits(x)


def make_inputs(w: Workload, names=("q", "k", "v")) -> dict:
    """All inputs of a workload, as the library consumes them.

    bf16 workloads give uint16 bit arrays [B,H,N,d]; the fp32 workload gives
    float32 arrays.
    """
    shape = (w.B, w.H, w.N, w.d)
    out = {}
    for n in names:
        mult = w.k_scale if n == "k" else 1.0
        out[n] = make_tensor(w.seed, n, shape, mult, w.dtype)
    return out


def to_f64(x: np.ndarray, dtype: str) -> np.ndarray:
    """The exact float64 values of an input array produced by ``make_tensor``."""
    if dtype == "bf16":
        return bf16_bits_to_f32(x).astype(np.float64)
    return np.asarray(x, dtype=np.float64)


def sample_rows(seed: int, N: int, count: int) -> np.ndarray:
    """Sorted distinct query rows to check on long sequences (always row 0 and N-1)."""
    rng = np.random.default_rng([int(seed), 99])
    count = min(count, N)
    rows = set(rng.choice(N, size=max(0, count - 2), replace=False).tolist())
    rows.update({0, N - 1})
    return np.array(sorted(rows), dtype=np.int64)
