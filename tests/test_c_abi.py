"""A plain C caller of the library (tests/c_abi_example.c): it compiles and links
against include/fa.h and libfa.so with a C compiler alone, and (GPU) its forward
and backward, driven only through the C ABI, match the fp64 oracle on seeded
inputs (definition: the unite.ai page's standard_attention listing; the backward
is its exact gradient, the deepfa.ir page, section "Technique 2: recomputation")."""
import os
import subprocess

import numpy as np
import pytest

from exact_io_aware_100_b200 import inputs
from oracle import attention_bwd, attention_fwd, bwd_operand_rounding_bound
from tests.helpers import assert_close, assert_close_bwd, assert_lse

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


def _compile(tmp_path):
    from exact_io_aware_100_b200 import build
    lib = build.build()
    exe = str(tmp_path / "c_abi_example")
    libdir = os.path.dirname(lib)
    cmd = ["gcc", "-std=c11", "-O2", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
           "-I", os.path.join(CUDA, "include"), os.path.join(ROOT, "tests", "c_abi_example.c"), "-o", exe,
           "-L", libdir, "-lfa", "-L", os.path.join(CUDA, "lib64"), "-lcudart", "-lm",
           "-Wl,-rpath," + libdir, "-Wl,-rpath," + os.path.join(CUDA, "lib64")]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    return exe


def test_c_caller_compiles_and_links(tmp_path):
    assert os.path.exists(_compile(tmp_path))


@pytest.mark.gpu
@pytest.mark.parametrize("B,H,N,d,causal", [(1, 2, 300, 128, 1), (2, 1, 257, 64, 0)])
def test_c_caller_matches_the_oracle(tmp_path, B, H, N, d, causal):
    exe = _compile(tmp_path)
    seed = 7100 + N + d
    shape = (B, H, N, d)
    bits = {nm: inputs.make_tensor(seed, nm, shape) for nm in ("q", "k", "v", "do")}
    fin, fout = tmp_path / "in.bin", tmp_path / "out.bin"
    with open(fin, "wb") as f:
        for nm in ("q", "k", "v", "do"):
            f.write(np.ascontiguousarray(bits[nm]).tobytes())
    r = subprocess.run([exe, str(fin), str(fout), str(B), str(H), str(N), str(d), str(causal)],
                       capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout + r.stderr
    n = B * H * N * d
    raw = np.fromfile(fout, dtype=np.uint8)
    out16 = raw[: 8 * n].view(np.uint16)
    o, dq, dk, dv = (inputs.to_f64(out16[i * n:(i + 1) * n].reshape(shape), "bf16") for i in range(4))
    lse = raw[8 * n:].view(np.float32).astype(np.float64).reshape(B, H, N)
    f64 = {nm: inputs.to_f64(bits[nm], "bf16") for nm in bits}
    scale = 1.0 / np.sqrt(d)
    ro, rl = attention_fwd(f64["q"], f64["k"], f64["v"], scale, bool(causal))
    assert_close("O", o, ro)
    assert_lse(lse, rl)
    ref = attention_bwd(f64["q"], f64["k"], f64["v"], f64["do"], scale, bool(causal))
    bound = bwd_operand_rounding_bound(f64["q"], f64["k"], f64["v"], f64["do"], scale, bool(causal))
    for name, got, rr, bb in zip(("dq", "dk", "dv"), (dq, dk, dv), ref, bound):
        assert_close_bwd(name, got, rr, bb)
