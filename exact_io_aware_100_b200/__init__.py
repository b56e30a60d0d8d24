"""Python binding of libfa.so (exact IO-aware attention for B200, sm_100a).

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI declared in ``include/fa.h``.  PyTorch provides device
memory and streams.  There is no CPU fallback: if ``libfa.so`` is missing the
calls raise.

Low-level names mirror the C ABI (``fa_fwd``, ``fa_fwd_ex``, ``fa_bwd``, ...)
and take torch tensors for the pointer arguments.  ``forward`` / ``backward``
allocate the outputs (and workspace) with torch and call them.
"""
from __future__ import annotations

import ctypes
import math
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfa.so")

FA_OK, FA_ERR_INVALID, FA_ERR_UNSUPPORTED, FA_ERR_ALIGN, FA_ERR_WORKSPACE, FA_ERR_CUDA, FA_ERR_TIMEOUT = range(7)
FA_BF16, FA_F32 = 0, 1

EXPORTS = (
    "fa_fwd", "fa_fwd_ex", "fa_fwd_workspace_size", "fa_bwd", "fa_bwd_workspace_size",
    "fa_bwd_prepare", "fa_bwd_main", "fa_bwd_finish", "fa_bwd_noalloc", "fa_fwd_gqa", "fa_bwd_gqa",
    "fa_decode", "fa_decode_workspace_size", "fa_fwd_general", "fa_bwd_general", "fa_bwd_general_workspace_size",
    "fa_get_device_status", "fa_selftest_wait_timeout", "fa_status_string", "fa_version",
)


class FaStrides(ctypes.Structure):
    """fa_strides: element strides of one [batch][head][row][d] operand."""
    _fields_ = [("batch", ctypes.c_int64), ("head", ctypes.c_int64), ("row", ctypes.c_int64)]


class FaLayout(ctypes.Structure):
    """fa_layout: sizes, packed-sequence offsets and operand strides (include/fa.h)."""
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("H_kv", ctypes.c_int), ("d", ctypes.c_int),
                ("Nq", ctypes.c_int), ("Nk", ctypes.c_int),
                ("cu_seqlens_q", ctypes.c_void_p), ("cu_seqlens_k", ctypes.c_void_p),
                ("total_q", ctypes.c_int), ("total_k", ctypes.c_int)] + \
               [(n, FaStrides) for n in ("q", "k", "v", "o", "dout", "dq", "dk", "dv")]


class FaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where} failed: {status_string(code)} ({code})")


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libfa.so and declare the C signatures (no GPU needed)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is not built; run `python -m exact_io_aware_100_b200.build`")
    L = ctypes.CDLL(path)
    P, I, F, Z, U64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t, ctypes.c_uint64
    L.fa_fwd.argtypes = [P, P, P, P, P, I, I, I, I, F, I, P]
    L.fa_fwd_ex.argtypes = [P, P, P, P, P, I, I, I, I, F, I, I, P, Z, P]
    L.fa_fwd_workspace_size.argtypes = [I, I, I, I, I]
    L.fa_fwd_workspace_size.restype = Z
    L.fa_bwd.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, F, I, P, Z, P]
    L.fa_bwd_prepare.argtypes = [P, P, P, I, I, I, I, P, Z, P]
    L.fa_bwd_main.argtypes = [P, P, P, P, P, P, I, I, I, I, F, I, P, Z, P]
    L.fa_bwd_finish.argtypes = [P, I, I, I, I, F, P, Z, P]
    L.fa_bwd_noalloc.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, F, I, P]
    L.fa_fwd_gqa.argtypes = [P, P, P, P, P, I, I, I, I, I, F, I, P]
    L.fa_bwd_gqa.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, I, F, I, P, Z, P]
    L.fa_decode.argtypes = [P, P, P, P, P, I, I, I, I, I, I, F, I, P, Z, P]
    L.fa_decode_workspace_size.argtypes = [I, I, I, I, I, I]
    L.fa_decode_workspace_size.restype = Z
    L.fa_bwd_workspace_size.argtypes = [I, I, I, I]
    L.fa_bwd_workspace_size.restype = Z
    LP = ctypes.POINTER(FaLayout)
    L.fa_fwd_general.argtypes = [P, P, P, P, P, LP, F, I, P]
    L.fa_bwd_general.argtypes = [P, P, P, P, P, P, P, P, P, LP, F, I, P, Z, P]
    L.fa_bwd_general_workspace_size.argtypes = [LP]
    L.fa_bwd_general_workspace_size.restype = Z
    L.fa_get_device_status.argtypes = [P]
    L.fa_selftest_wait_timeout.argtypes = [U64, P]
    L.fa_status_string.argtypes = [I]
    L.fa_status_string.restype = ctypes.c_char_p
    L.fa_version.restype = ctypes.c_char_p
    for name in ("fa_fwd", "fa_fwd_ex", "fa_bwd", "fa_bwd_prepare", "fa_bwd_main", "fa_bwd_finish", "fa_bwd_noalloc",
                 "fa_fwd_gqa", "fa_bwd_gqa", "fa_decode", "fa_fwd_general", "fa_bwd_general",
                 "fa_get_device_status", "fa_selftest_wait_timeout"):
        getattr(L, name).restype = I
    _lib = L
    return L


def status_string(code: int) -> str:
    return load_library().fa_status_string(int(code)).decode()


def version() -> str:
    return load_library().fa_version().decode()


def _check(code: int, where: str) -> None:
    if code != FA_OK:
        raise FaError(code, where)


def _ptr(t) -> int | None:
    """Device address of a CUDA tensor (None stays None).  Host tensors are refused here: the library
    takes device pointers only and would otherwise launch kernels on host addresses."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor: the library reads and writes device memory only")
    return t.data_ptr()


def _stream(stream) -> int:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _bhnd(t):
    if t.dim() != 4 or not t.is_contiguous():
        raise ValueError("expected a contiguous [B, H, N, d] tensor")
    return t.shape


# ----------------------------------------------------------------- C ABI mirrors
def fa_fwd(q, k, v, o, lse, causal: bool, scale: float | None = None, stream=None) -> None:
    B, H, N, d = _bhnd(q)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    _check(load_library().fa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d, scale,
                                 int(bool(causal)), _stream(stream)), "fa_fwd")


def fa_fwd_ex(q, k, v, o, lse, causal: bool, dtype: int, workspace, scale: float | None = None,
              stream=None) -> None:
    B, H, N, d = _bhnd(q)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load_library().fa_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d, scale,
                                    int(bool(causal)), int(dtype), _ptr(workspace), ws_bytes,
                                    _stream(stream)), "fa_fwd_ex")


def fa_fwd_workspace_size(B: int, H: int, N: int, d: int, dtype: int) -> int:
    return int(load_library().fa_fwd_workspace_size(B, H, N, d, dtype))


def fa_bwd(q, k, v, o, lse, dout, dq, dk, dv, causal: bool, workspace, scale: float | None = None,
           stream=None) -> None:
    B, H, N, d = _bhnd(q)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load_library().fa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), _ptr(dq),
                                 _ptr(dk), _ptr(dv), B, H, N, d, scale, int(bool(causal)),
                                 _ptr(workspace), ws_bytes, _stream(stream)), "fa_bwd")


def _ws_bytes(workspace) -> int:
    return 0 if workspace is None else workspace.numel() * workspace.element_size()


def fa_bwd_prepare(o, lse, dout, workspace, stream=None) -> None:
    B, H, N, d = _bhnd(o)
    _check(load_library().fa_bwd_prepare(_ptr(o), _ptr(lse), _ptr(dout), B, H, N, d, _ptr(workspace),
                                         _ws_bytes(workspace), _stream(stream)), "fa_bwd_prepare")


def fa_bwd_main(q, k, v, dout, dk, dv, causal: bool, workspace, scale: float | None = None, stream=None) -> None:
    B, H, N, d = _bhnd(q)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    _check(load_library().fa_bwd_main(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(dk), _ptr(dv), B, H, N, d,
                                      scale, int(bool(causal)), _ptr(workspace), _ws_bytes(workspace),
                                      _stream(stream)), "fa_bwd_main")


def fa_bwd_finish(dq, workspace, scale: float | None = None, stream=None) -> None:
    B, H, N, d = _bhnd(dq)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    _check(load_library().fa_bwd_finish(_ptr(dq), B, H, N, d, scale, _ptr(workspace), _ws_bytes(workspace),
                                        _stream(stream)), "fa_bwd_finish")


NOALLOC_SCRATCH_BYTES = 64 << 20   # FA_NOALLOC_SCRATCH_BYTES in include/fa.h


def fa_bwd_noalloc(q, k, v, o, lse, dout, dq, dk, dv, causal: bool, scale: float | None = None,
                   stream=None) -> None:
    """fa_bwd using the library's built-in scratch array instead of a workspace.

    For callers that cannot allocate device memory themselves (for example a
    plug-in whose host application owns all device allocations, or a serving
    path that must not allocate after start-up).  Shapes needing more than
    NOALLOC_SCRATCH_BYTES of workspace are rejected; the first call on a device
    looks up the array's address; calls that overlap on the GPU race.
    """
    B, H, N, d = _bhnd(q)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    _check(load_library().fa_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), _ptr(dq),
                                         _ptr(dk), _ptr(dv), B, H, N, d, scale, int(bool(causal)),
                                         _stream(stream)), "fa_bwd_noalloc")


def fa_fwd_gqa(q, k, v, o, lse, causal: bool, scale: float | None = None, stream=None) -> None:
    """Grouped-query forward: q, o [B,H,N,d]; k, v [B,H_kv,N,d] (H a multiple of H_kv)."""
    B, H, N, d = _bhnd(q)
    H_kv = _bhnd(k)[1]
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    _check(load_library().fa_fwd_gqa(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, H_kv, N, d, scale,
                                     int(bool(causal)), _stream(stream)), "fa_fwd_gqa")


def fa_bwd_gqa(q, k, v, o, lse, dout, dq, dk, dv, causal: bool, workspace, scale: float | None = None,
               stream=None) -> None:
    """Grouped-query backward: dk, dv [B,H_kv,N,d] are sums over each key/value head's query set."""
    B, H, N, d = _bhnd(q)
    H_kv = _bhnd(k)[1]
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    _check(load_library().fa_bwd_gqa(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), _ptr(dq),
                                     _ptr(dk), _ptr(dv), B, H, H_kv, N, d, scale, int(bool(causal)),
                                     _ptr(workspace), _ws_bytes(workspace), _stream(stream)), "fa_bwd_gqa")


def fa_decode_workspace_size(B: int, H: int, H_kv: int, Lq: int, Nk: int, d: int) -> int:
    return int(load_library().fa_decode_workspace_size(B, H, H_kv, Lq, Nk, d))


def fa_decode(q, k, v, o, lse, causal: bool, workspace, scale: float | None = None, stream=None) -> None:
    """Decode: q, o [B,H,Lq,d] (the last Lq positions); k, v [B,H_kv,Nk,d]; lse [B,H,Lq]."""
    B, H, Lq, d = _bhnd(q)
    _, H_kv, Nk, _ = _bhnd(k)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    _check(load_library().fa_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, H_kv, Lq, Nk, d, scale,
                                    int(bool(causal)), _ptr(workspace), _ws_bytes(workspace), _stream(stream)),
           "fa_decode")


def decode(q, k, v, causal: bool, scale: float | None = None, stream=None, workspace=None):
    """O, lse of the last Lq query positions q [B,H,Lq,d] against a cache k, v [B,H_kv,Nk,d] (bf16)."""
    import torch
    B, H, Lq, d = _bhnd(q)
    _, H_kv, Nk, _ = _bhnd(k)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Lq), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = _workspace(fa_decode_workspace_size(B, H, H_kv, Lq, Nk, d), q.device)
    fa_decode(q, k, v, o, lse, causal, workspace, scale, stream)
    return o, lse


def fa_bwd_workspace_size(B: int, H: int, N: int, d: int) -> int:
    return int(load_library().fa_bwd_workspace_size(B, H, N, d))


# ----------------------------------------------------------------- general layouts
def _strides_4d(t) -> FaStrides:
    """Strides of a tensor viewed as [B, heads, rows, d] (d contiguous), any other strides."""
    if t is None:
        return FaStrides(0, 0, 0)
    if t.dim() != 4 or (t.shape[3] > 1 and t.stride(3) != 1):
        raise ValueError("expected a [B, heads, rows, d] tensor with contiguous d")
    return FaStrides(t.stride(0), t.stride(1), t.stride(2))


def _strides_packed(t) -> FaStrides:
    """Strides of a packed [rows, heads, d] tensor (d contiguous)."""
    if t is None:
        return FaStrides(0, 0, 0)
    if t.dim() != 3 or (t.shape[2] > 1 and t.stride(2) != 1):
        raise ValueError("expected a packed [rows, heads, d] tensor with contiguous d")
    return FaStrides(0, t.stride(1), t.stride(0))


def layout_4d(q, k, v, o, dout=None, dq=None, dk=None, dv=None) -> FaLayout:
    """fa_layout for fixed lengths: q, o, dout, dq [B, H, Nq, d] and k, v, dk, dv [B, H_kv, Nk, d],
    as tensors of any strides (a [B, N, H, d] tensor is passed as its transpose(1, 2))."""
    B, H, Nq, d = q.shape
    Nk, H_kv = k.shape[2], k.shape[1]
    L = FaLayout(B=B, H=H, H_kv=H_kv, d=d, Nq=Nq, Nk=Nk, cu_seqlens_q=None, cu_seqlens_k=None, total_q=0,
                 total_k=0)
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dout", dout), ("dq", dq), ("dk", dk), ("dv", dv)):
        setattr(L, name, _strides_4d(t))
    return L


def layout_packed(q, k, v, o, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int, max_seqlen_k: int,
                  dout=None, dq=None, dk=None, dv=None) -> FaLayout:
    """fa_layout for packed sequences: q, o [total_q, H, d]; k, v [total_k, H_kv, d]; cu_seqlens_*
    int32 device tensors of B + 1 row offsets; max_seqlen_* at least every sequence's length."""
    total_q, H, d = q.shape
    total_k, H_kv = k.shape[0], k.shape[1]
    for cu in (cu_seqlens_q, cu_seqlens_k):
        import torch
        if cu.dtype != torch.int32 or cu.dim() != 1 or not cu.is_contiguous():
            raise ValueError("sequence offsets must be a contiguous 1-D int32 tensor")
    if cu_seqlens_q.numel() != cu_seqlens_k.numel() or cu_seqlens_q.numel() < 2:
        raise ValueError("query and key offsets must both hold B + 1 entries")
    L = FaLayout(B=cu_seqlens_q.numel() - 1, H=H, H_kv=H_kv, d=d, Nq=int(max_seqlen_q), Nk=int(max_seqlen_k),
                 cu_seqlens_q=_ptr(cu_seqlens_q), cu_seqlens_k=_ptr(cu_seqlens_k),
                 total_q=total_q, total_k=total_k)
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dout", dout), ("dq", dq), ("dk", dk), ("dv", dv)):
        setattr(L, name, _strides_packed(t))
    return L


def fa_fwd_general(q, k, v, o, lse, layout: FaLayout, causal: bool, scale: float | None = None,
                   stream=None) -> None:
    scale = 1.0 / math.sqrt(layout.d) if scale is None else float(scale)
    _check(load_library().fa_fwd_general(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), ctypes.byref(layout),
                                         scale, int(bool(causal)), _stream(stream)), "fa_fwd_general")


def fa_bwd_general(q, k, v, o, lse, dout, dq, dk, dv, layout: FaLayout, causal: bool, workspace,
                   scale: float | None = None, stream=None) -> None:
    scale = 1.0 / math.sqrt(layout.d) if scale is None else float(scale)
    _check(load_library().fa_bwd_general(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), _ptr(dq),
                                         _ptr(dk), _ptr(dv), ctypes.byref(layout), scale, int(bool(causal)),
                                         _ptr(workspace), _ws_bytes(workspace), _stream(stream)), "fa_bwd_general")


def fa_bwd_general_workspace_size(layout: FaLayout) -> int:
    return int(load_library().fa_bwd_general_workspace_size(ctypes.byref(layout)))


def fa_get_device_status(stream=None) -> int:
    return int(load_library().fa_get_device_status(_stream(stream)))


def fa_selftest_wait_timeout(timeout_ns: int, stream=None) -> None:
    _check(load_library().fa_selftest_wait_timeout(int(timeout_ns), _stream(stream)),
           "fa_selftest_wait_timeout")


# ----------------------------------------------------------------- conveniences
def _workspace(nbytes: int, device):
    import torch
    if nbytes == 0:
        return None
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def _is_dense(*ts) -> bool:
    return all(t.dim() == 4 and t.is_contiguous() for t in ts)


def forward(q, k, v, causal: bool, scale: float | None = None, stream=None):
    """O, lse for q [B,H,Nq,d] and k, v [B,H_kv,Nk,d] (bf16; float32 via the bf16 tensor-core path when
    the tensors are dense, H_kv == H and Nq == Nk).  H_kv < H is grouped-query attention (contiguous sets
    of H / H_kv query heads); Nq != Nk aligns the causal mask bottom-right.  The tensors may have any
    strides with d contiguous (e.g. a [B, N, H, d] tensor passed as its transpose(1, 2)); O comes back
    with q's strides."""
    import torch
    if q.dtype == torch.bfloat16 and (not _is_dense(q, k, v) or q.shape[2] != k.shape[2]):
        o = torch.empty_like(q)    # q's strides when q is dense in some order, else contiguous
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
        fa_fwd_general(q, k, v, o, lse, layout_4d(q, k, v, o), causal, scale, stream)
        return o, lse
    if q.shape[2] != k.shape[2]:
        raise ValueError("query and key lengths differ: bf16 inputs only")
    B, H, N, d = _bhnd(q)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    if _bhnd(k)[1] != H:          # fewer key/value heads: grouped-query attention
        fa_fwd_gqa(q, k, v, o, lse, causal, scale, stream)
    elif q.dtype == torch.bfloat16:
        fa_fwd(q, k, v, o, lse, causal, scale, stream)
    elif q.dtype == torch.float32:
        ws = _workspace(fa_fwd_workspace_size(B, H, N, d, FA_F32), q.device)
        fa_fwd_ex(q, k, v, o, lse, causal, FA_F32, ws, scale, stream)
    else:
        raise ValueError(f"unsupported dtype {q.dtype}")
    return o, lse


def _like(t):
    import torch
    return torch.empty_like(t)     # t's strides when t is dense in some order, else contiguous


def backward(q, k, v, o, lse, dout, causal: bool, scale: float | None = None, stream=None, workspace=None):
    """dQ, dK, dV (bf16) from the forward's O and lse; dK, dV have k's head count (grouped-query
    attention sums each shared head's gradient over its set).  Any strides and Nq != Nk as in
    ``forward``; the gradients come back with the strides of q, k, v."""
    import torch
    if not _is_dense(q, k, v, o, dout) or q.shape[2] != k.shape[2]:
        dq, dk, dv = _like(q), _like(k), _like(v)
        L = layout_4d(q, k, v, o, dout, dq, dk, dv)
        if workspace is None:
            workspace = _workspace(fa_bwd_general_workspace_size(L), q.device)
        fa_bwd_general(q, k, v, o, lse, dout, dq, dk, dv, L, causal, workspace, scale, stream)
        return dq, dk, dv
    B, H, N, d = _bhnd(q)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    if workspace is None:
        workspace = _workspace(fa_bwd_workspace_size(B, H, N, d), q.device)
    if _bhnd(k)[1] != H:
        fa_bwd_gqa(q, k, v, o, lse, dout, dq, dk, dv, causal, workspace, scale, stream)
    else:
        fa_bwd(q, k, v, o, lse, dout, dq, dk, dv, causal, workspace, scale, stream)
    return dq, dk, dv


def forward_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int, max_seqlen_k: int, causal: bool,
                   scale: float | None = None, stream=None):
    """Packed variable-length batch (bf16): q [total_q, H, d], k, v [total_k, H_kv, d]; sequence b is rows
    cu_seqlens_q[b]:cu_seqlens_q[b+1] (int32 device offsets).  Returns O [total_q, H, d] and
    lse [H, total_q]; bottom-right causal alignment per sequence."""
    import torch
    o = _like(q)
    lse = torch.empty((q.shape[1], q.shape[0]), dtype=torch.float32, device=q.device)
    L = layout_packed(q, k, v, o, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k)
    fa_fwd_general(q, k, v, o, lse, L, causal, scale, stream)
    return o, lse


def backward_varlen(q, k, v, o, lse, dout, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int, max_seqlen_k: int,
                    causal: bool, scale: float | None = None, stream=None, workspace=None):
    """dQ, dK, dV of ``forward_varlen`` (packed like q, k, v)."""
    dq, dk, dv = _like(q), _like(k), _like(v)
    L = layout_packed(q, k, v, o, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, dout, dq, dk, dv)
    if workspace is None:
        workspace = _workspace(fa_bwd_general_workspace_size(L), q.device)
    fa_bwd_general(q, k, v, o, lse, dout, dq, dk, dv, L, causal, workspace, scale, stream)
    return dq, dk, dv
