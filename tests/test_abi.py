"""The C ABI library: builds, loads without a GPU, exports what include/fa.h
declares, and rejects bad arguments before touching the device."""
import os
import re
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa.h")


@pytest.fixture(scope="module")
def lib():
    from exact_io_aware_100_b200 import build, load_library
    build.build()
    return load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("fa_fwd", "fa_bwd", "fa_fwd_ex", "fa_bwd_workspace_size", "fa_get_device_status",
              "fa_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", lib._name], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (fa_\w+)", out))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing


def test_binding_names_match_header():
    import exact_io_aware_100_b200 as fa
    assert sorted(fa.EXPORTS) == declared_functions()


def test_status_strings(lib):
    import exact_io_aware_100_b200 as fa
    assert fa.status_string(0) == "FA_OK"
    assert fa.status_string(6) == "FA_ERR_TIMEOUT"
    assert fa.version().count(".") == 2


def test_argument_validation_without_device(lib):
    P16 = 16  # a fake but aligned "pointer"; validation fails before any use
    f = lib.fa_fwd
    assert f(None, None, None, None, None, 1, 1, 128, 64, 0.125, 0, None) == 3     # null
    assert f(P16, P16, P16, P16, P16 + 4, 1, 1, 128, 64, 0.125, 0, None) == 3      # misaligned
    assert f(P16, P16, P16, P16, P16, 1, 1, 128, 96, 0.125, 0, None) == 2          # d
    assert f(P16, P16, P16, P16, P16, 1, 1, 0, 64, 0.125, 0, None) == 1            # N
    assert f(P16, P16, P16, P16, P16, 0, 1, 8, 64, 0.125, 0, None) == 1            # B
    assert f(P16, P16, P16, P16, P16, 1, 1, 8, 64, float("nan"), 0, None) == 1     # scale
    assert f(P16, P16, P16, P16, P16, 1, 1, 1 << 25, 64, 0.1, 0, None) == 1        # N too large
    assert f(P16, P16, P16, P16, P16, 64, 64, 1 << 20, 64, 0.1, 0, None) == 1      # > 2^31 elems
    g = lib.fa_fwd_ex   # fp32 needs a workspace
    assert g(P16, P16, P16, P16, P16, 1, 1, 128, 64, 0.125, 0, 1, None, 0, None) == 4
    assert g(P16, P16, P16, P16, P16, 1, 1, 128, 64, 0.125, 0, 7, None, 0, None) == 2
    b = lib.fa_bwd
    args = [P16] * 9
    assert b(*args, 1, 1, 128, 96, 0.125, 1, P16, 1 << 30, None) == 2              # bwd d=96
    assert b(*args, 1, 1, 128, 320, 0.125, 1, P16, 1 << 30, None) == 2             # bwd d=320
    assert b(*args, 1, 1, 128, 256, 0.125, 1, 16, 1 << 30, None) == 4              # bwd d=256 passes to the workspace check
    assert b(*args, 1, 1, 128, 128, 0.0, 1, P16, 1 << 30, None) == 1               # scale must be positive
    assert b(*args, 1, 1, 128, 128, -0.125, 1, P16, 1 << 30, None) == 1
    assert f(P16, P16, P16, P16, P16, 1, 1, 8, 64, 0.0, 0, None) == 1              # fwd scale 0
    assert f(P16, P16, P16, P16, P16, 1, 1, 8, 64, -1.0, 1, None) == 1             # fwd negative scale
    assert g(P16, P16, P16, P16, P16, 1, 1, 128, 256, 0.125, 0, 1, P16, 1 << 30, None) == 2   # fp32 at d=256
    assert b(*args, 1, 1, 128, 128, 0.125, 1, None, 0, None) == 4                  # no workspace
    need = lib.fa_bwd_workspace_size(1, 1, 128, 128)
    assert b(*args, 1, 1, 128, 128, 0.125, 1, 256, need - 1, None) == 4           # too small
    assert b(*args, 1, 1, 128, 128, 0.125, 1, 16, need, None) == 4                 # not 256-aligned


def test_grouped_query_validation_without_device(lib):
    P16 = 16
    f, b = lib.fa_fwd_gqa, lib.fa_bwd_gqa
    assert f(P16, P16, P16, P16, P16, 1, 6, 4, 128, 64, 0.125, 0, None) == 1     # 6 heads over 4 sets
    assert f(P16, P16, P16, P16, P16, 1, 6, 0, 128, 64, 0.125, 0, None) == 1     # no key/value head
    assert f(P16, P16, P16, P16, P16 + 4, 1, 6, 2, 128, 64, 0.125, 0, None) == 3  # misaligned
    args = [P16] * 9
    assert b(*args, 1, 6, 4, 128, 128, 0.125, 1, P16, 1 << 30, None) == 1         # uneven sets
    assert b(*args, 1, 6, 3, 128, 96, 0.125, 1, P16, 1 << 30, None) == 2          # d = 96
    assert b(*args, 1, 6, 3, 128, 128, 0.125, 1, None, 0, None) == 4              # no workspace


def test_decode_validation_without_device(lib):
    P16 = 16
    f = lib.fa_decode
    ok = (P16, P16, P16, P16, P16)
    assert f(*ok, 2, 8, 2, 1, 1000, 128, 0.088, 1, None, 0, None) == 4             # no workspace
    assert f(*ok, 2, 8, 2, 1, 1000, 96, 0.125, 1, P16, 1 << 30, None) == 2        # d = 96
    assert f(*ok, 2, 8, 3, 1, 1000, 128, 0.088, 1, P16, 1 << 30, None) == 1       # uneven sets
    assert f(*ok, 2, 8, 2, 9, 8, 128, 0.088, 1, P16, 1 << 30, None) == 1          # more queries than keys
    assert f(*ok, 2, 8, 2, 0, 8, 128, 0.088, 1, P16, 1 << 30, None) == 1          # no query
    assert f(P16, P16, P16, P16, P16 + 4, 2, 8, 2, 1, 1000, 128, 0.088, 1, P16, 1 << 30, None) == 3
    assert lib.fa_decode_workspace_size(2, 8, 2, 1, 1000, 128) > 0
    assert lib.fa_decode_workspace_size(2, 8, 3, 1, 1000, 128) == 0


def test_layout_struct_matches_the_header(tmp_path):
    """ctypes' fa_layout has the size and field offsets the C compiler gives include/fa.h's."""
    import ctypes
    import exact_io_aware_100_b200 as fa
    src = tmp_path / "layout.c"
    src.write_text(
        '#include <stdio.h>\n#include <stddef.h>\n#include "fa.h"\n'
        'int main(void) { printf("%zu %zu %zu %zu %zu %zu\\n", sizeof(fa_layout), offsetof(fa_layout, cu_seqlens_q),'
        ' offsetof(fa_layout, total_q), offsetof(fa_layout, q), offsetof(fa_layout, dv), sizeof(fa_strides));'
        ' return 0; }\n')
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), "-o", str(exe), str(src)], check=True)
    got = [int(x) for x in subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()]
    L = fa.FaLayout
    assert got == [ctypes.sizeof(L), L.cu_seqlens_q.offset, L.total_q.offset, L.q.offset, L.dv.offset,
                   ctypes.sizeof(fa.FaStrides)]


def _dense_layout(fa, B, H, H_kv, Nq, Nk, d):
    L = fa.FaLayout(B=B, H=H, H_kv=H_kv, d=d, Nq=Nq, Nk=Nk, cu_seqlens_q=None, cu_seqlens_k=None,
                    total_q=0, total_k=0)
    for n in ("q", "o", "dout", "dq"):
        setattr(L, n, fa.FaStrides(H * Nq * d, Nq * d, d))
    for n in ("k", "v", "dk", "dv"):
        setattr(L, n, fa.FaStrides(H_kv * Nk * d, Nk * d, d))
    return L


def test_general_validation_without_device(lib):
    import ctypes
    import exact_io_aware_100_b200 as fa
    P16 = 16
    f, b = lib.fa_fwd_general, lib.fa_bwd_general
    ref = ctypes.byref
    assert f(P16, P16, P16, P16, P16, None, 0.1, 1, None) == 1                       # no layout
    L = _dense_layout(fa, 2, 4, 2, 100, 300, 128)
    assert f(P16, P16, P16, P16, P16 + 4, ref(L), 0.1, 1, None) == 3                 # misaligned lse
    assert f(P16, P16, P16, P16, P16, ref(L), float("inf"), 1, None) == 1           # scale
    bad = _dense_layout(fa, 2, 4, 2, 100, 300, 128)
    bad.q = fa.FaStrides(4 * 100 * 128, 100 * 128, 132)                             # row stride not 16 B
    assert f(P16, P16, P16, P16, P16, ref(bad), 0.1, 1, None) == 3
    bad = _dense_layout(fa, 2, 4, 3, 100, 300, 128)                                   # uneven sets
    assert f(P16, P16, P16, P16, P16, ref(bad), 0.1, 1, None) == 1
    bad = _dense_layout(fa, 2, 4, 2, 100, 300, 96)                                    # d
    assert f(P16, P16, P16, P16, P16, ref(bad), 0.1, 1, None) == 2
    bad = _dense_layout(fa, 2, 4, 2, -1, 300, 128)                                    # negative length
    assert f(P16, P16, P16, P16, P16, ref(bad), 0.1, 1, None) == 1
    bad = _dense_layout(fa, 2, 4, 2, 100, 300, 128)
    bad.cu_seqlens_q = 256                                                             # offsets for q only
    assert f(P16, P16, P16, P16, P16, ref(bad), 0.1, 1, None) == 1
    bad.cu_seqlens_k = 258                                                             # misaligned offsets
    bad.total_q, bad.total_k = 100, 300
    assert f(P16, P16, P16, P16, P16, ref(bad), 0.1, 1, None) == 3
    args = [P16] * 9
    assert b(*args, ref(L), 0.1, 1, None, 0, None) == 4                               # no workspace
    need = lib.fa_bwd_general_workspace_size(ref(L))
    assert b(*args, ref(L), 0.1, 1, 256, need - 1, None) == 4


def test_general_workspace_sizes(lib):
    import ctypes
    import exact_io_aware_100_b200 as fa
    L = _dense_layout(fa, 2, 4, 2, 100, 300, 128)
    # fp32 dQ accumulator for B*H*Nq rows, then lse * log2(e) and D for rows padded to 128 per head
    acc = 2 * 4 * 100 * 128 * 4
    vec = (2 * 4 * 128 * 4 + 255) // 256 * 256
    assert lib.fa_bwd_general_workspace_size(ctypes.byref(L)) == (acc + 255) // 256 * 256 + 2 * vec
    # packed: H * total_q accumulator rows; the vectors are padded to the longest sequence
    L.cu_seqlens_q, L.cu_seqlens_k, L.total_q, L.total_k, L.Nq = 256, 512, 1000, 3000, 700
    acc = 4 * 1000 * 128 * 4
    vec = (2 * 4 * 768 * 4 + 255) // 256 * 256
    assert lib.fa_bwd_general_workspace_size(ctypes.byref(L)) == (acc + 255) // 256 * 256 + 2 * vec
    assert lib.fa_bwd_general_workspace_size(None) == 0
    assert lib.fa_bwd_workspace_size(4, 16, 4096, 128) == lib.fa_bwd_general_workspace_size(
        ctypes.byref(_dense_layout(fa, 4, 16, 16, 4096, 4096, 128)))


def test_workspace_sizes(lib):
    assert lib.fa_fwd_workspace_size(1, 1, 128, 64, 0) == 0
    assert lib.fa_fwd_workspace_size(1, 1, 128, 64, 1) == 3 * 128 * 64 * 2
    # dQ accumulator (fp32) + lse and D for rows padded to a multiple of 128
    assert lib.fa_bwd_workspace_size(4, 16, 4096, 128) == 4 * 16 * 4096 * 128 * 4 + 2 * 4 * 16 * 4096 * 4
    assert lib.fa_bwd_workspace_size(1, 1, 100, 128) == 100 * 128 * 4 + 2 * 512


def test_product_path_does_not_import_the_oracle():
    code = ("import sys, exact_io_aware_100_b200 as fa; fa.load_library(); "
            "assert not any(m == 'oracle' or m.startswith('oracle.') for m in sys.modules), 'oracle imported'")
    subprocess.run([sys.executable, "-c", code], check=True, cwd=ROOT)


def test_binding_refuses_host_tensors(lib):
    """Host (CPU) tensors never reach the library: it takes device pointers only."""
    import torch
    import exact_io_aware_100_b200 as fa
    q = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        fa.forward(q, q, q, True)
    with pytest.raises(ValueError):
        fa.forward(q.transpose(1, 2).contiguous().transpose(1, 2), q, q, True)
    cu = torch.tensor([0, 128], dtype=torch.int32)
    with pytest.raises(ValueError):
        fa.forward_varlen(q[0].transpose(0, 1), q[0].transpose(0, 1), q[0].transpose(0, 1), cu, cu, 128, 128, True)
