"""fa_bwd_noalloc: the backward for callers that cannot allocate device memory.

Some callers cannot hand the library a workspace -- a plug-in whose host
application owns every device allocation through its own pool, or a serving
path that must not allocate once it is running.  fa_bwd_noalloc gives them the
same backward with a scratch array built into the library.  This file checks,
through the C ABI, that two calls in a row give what fa_bwd (with a caller
workspace) gives, within the tolerances the other parity tests use.  It is
collected last on purpose, and passes alone or after the other tests.
"""
import numpy as np
import pytest

from tests.helpers import assert_close, make_case, to_device, to_f64

pytestmark = pytest.mark.gpu


def test_noalloc_backward_matches_fa_bwd_on_two_calls_in_a_row():
    import torch
    import exact_io_aware_100_b200 as fa
    fa.load_library()
    cases = [(2, 3, 517, True, 31), (1, 4, 300, False, 32)]   # different shapes back to back
    for B, H, N, causal, seed in cases:
        d = 128
        assert fa.fa_bwd_workspace_size(B, H, N, d) <= fa.NOALLOC_SCRATCH_BYTES
        host, _ = make_case(B, H, N, d, seed, names=("q", "k", "v", "do"))
        q, k, v, do = (to_device(host[n], "bf16") for n in ("q", "k", "v", "do"))
        o, lse = fa.forward(q, k, v, causal)
        ref = fa.backward(q, k, v, o, lse, do, causal)            # caller-supplied workspace
        got = tuple(torch.full_like(q, float("nan")) for _ in range(3))
        fa.fa_bwd_noalloc(q, k, v, o, lse, do, got[0], got[1], got[2], causal)
        torch.cuda.synchronize()
        assert fa.fa_get_device_status() == fa.FA_OK
        for name, g, r in zip(("dq", "dk", "dv"), got, ref):
            assert_close(name, to_f64(g), to_f64(r))


def test_noalloc_rejects_shapes_beyond_its_scratch():
    import exact_io_aware_100_b200 as fa
    L = fa.load_library()
    B, H, N, d = 8, 32, 8192, 128           # needs ~1 GiB of workspace
    assert fa.fa_bwd_workspace_size(B, H, N, d) > fa.NOALLOC_SCRATCH_BYTES
    P16 = 16
    rc = L.fa_bwd_noalloc(*([P16] * 9), B, H, N, d, 0.088, 1, None)
    assert rc == fa.FA_ERR_WORKSPACE
