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
    assert f(*ok, 2, 8, 2, 1, 1000, 64, 0.125, 1, P16, 1 << 30, None) == 2        # d = 64
    assert f(*ok, 2, 32, 1, 1, 1000, 128, 0.088, 1, P16, 1 << 30, None) == 2      # 32 rows in one set
    assert f(*ok, 2, 8, 3, 1, 1000, 128, 0.088, 1, P16, 1 << 30, None) == 1       # uneven sets
    assert f(*ok, 2, 8, 2, 9, 8, 128, 0.088, 1, P16, 1 << 30, None) == 1          # more queries than keys
    assert f(*ok, 2, 8, 2, 0, 8, 128, 0.088, 1, P16, 1 << 30, None) == 1          # no query
    assert f(P16, P16, P16, P16, P16 + 4, 2, 8, 2, 1, 1000, 128, 0.088, 1, P16, 1 << 30, None) == 3
    assert lib.fa_decode_workspace_size(2, 8, 2, 1, 1000, 128) > 0
    assert lib.fa_decode_workspace_size(2, 8, 3, 1, 1000, 128) == 0


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
