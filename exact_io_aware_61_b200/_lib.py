"""ctypes binding of ``libfa_b200.so`` (the C ABI in ``include/fa.h``).

Argument marshalling only: every step of the attention computation runs in
the CUDA kernels behind ``fa_fwd`` / ``fa_bwd``. PyTorch supplies device
memory and the current stream. There is no CPU or library fallback: if the
shared library is missing or cannot be loaded, every call raises.
"""

from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfa_b200.so")

FA_OK, FA_ERR_INVALID, FA_ERR_UNSUPPORTED, FA_ERR_CUDA, FA_ERR_TIMEOUT, FA_ERR_WORKSPACE = range(6)
FA_BF16, FA_F32 = 0, 1

EXPORTED = (
    "fa_fwd",
    "fa_fwd_varlen",
    "fa_fwd_partial",
    "fa_merge_partials",
    "fa_bwd",
    "fa_bwd_prep",
    "fa_bwd_main",
    "fa_bwd_dq",
    "fa_bwd_noalloc",
    "fa_bwd_workspace_size",
    "fa_bwd_varlen",
    "fa_bwd_varlen_workspace_size",
    "fa_bwd_partial",
    "fa_f32_to_bf16",
    "fa_fwd_kvcache",
    "fa_fwd_kvcache_workspace_size",
    "fa_status_string",
    "fa_last_device_status",
    "fa_set_wait_timeout_ns",
    "fa_selftest_wait_timeout",
)

_lock = threading.Lock()
_handle = None


class FAError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the library once and declare every exported signature."""
    global _handle
    with _lock:
        if _handle is not None:
            return _handle
        if not os.path.exists(path):
            raise RuntimeError(
                f"CUDA library {path} is missing: build it with "
                "`python -m exact_io_aware_61_b200.build` (no CPU fallback exists)")
        lib = ctypes.CDLL(path)
        vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        lib.fa_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, vp]
        lib.fa_fwd.restype = i
        lib.fa_fwd_varlen.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, f, i, i, vp]
        lib.fa_fwd_varlen.restype = i
        lib.fa_fwd_partial.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, i, vp]
        lib.fa_fwd_partial.restype = i
        lib.fa_merge_partials.argtypes = [vp, vp, i, ctypes.c_longlong, vp, vp, i, i, vp]
        lib.fa_merge_partials.restype = i
        lib.fa_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, i, i, i, i, i, f, i, i, vp]
        lib.fa_bwd.restype = i
        lib.fa_bwd_prep.argtypes = [vp, vp, vp, vp, sz, i, i, i, i, i, i, vp]
        lib.fa_bwd_prep.restype = i
        lib.fa_bwd_main.argtypes = [vp, vp, vp, vp, vp, vp, vp, sz, i, i, i, i, i, f, i, i, vp]
        lib.fa_bwd_main.restype = i
        lib.fa_bwd_dq.argtypes = [vp, vp, sz, i, i, i, i, i, i, vp]
        lib.fa_bwd_dq.restype = i
        lib.fa_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, vp]
        lib.fa_bwd_noalloc.restype = i
        lib.fa_bwd_varlen.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, f, i,
                                      vp, sz, i, vp]
        lib.fa_bwd_varlen.restype = i
        lib.fa_bwd_partial.argtypes = [vp, vp, vp, vp, vp, vp, vp, sz, i, i, i, i, i, f, i, i, i, vp]
        lib.fa_bwd_partial.restype = i
        lib.fa_f32_to_bf16.argtypes = [vp, vp, sz, vp]
        lib.fa_f32_to_bf16.restype = i
        lib.fa_bwd_varlen_workspace_size.argtypes = [i, i, i, i, i, i]
        lib.fa_bwd_varlen_workspace_size.restype = sz
        lib.fa_bwd_workspace_size.argtypes = [i, i, i, i, i]
        lib.fa_bwd_workspace_size.restype = sz
        lib.fa_fwd_kvcache.argtypes = [vp, vp, vp, vp, vp, vp, sz, i, i, i, i, i, i, f, i, i, vp]
        lib.fa_fwd_kvcache.restype = i
        lib.fa_fwd_kvcache_workspace_size.argtypes = [i, i, i, i, i, i]
        lib.fa_fwd_kvcache_workspace_size.restype = sz
        lib.fa_status_string.argtypes = [i]
        lib.fa_status_string.restype = ctypes.c_char_p
        lib.fa_last_device_status.argtypes = [vp]
        lib.fa_last_device_status.restype = i
        lib.fa_set_wait_timeout_ns.argtypes = [ctypes.c_longlong]
        lib.fa_set_wait_timeout_ns.restype = None
        lib.fa_selftest_wait_timeout.argtypes = [ctypes.c_longlong, vp]
        lib.fa_selftest_wait_timeout.restype = i
        _handle = lib
        return lib


def status_string(status: int) -> str:
    return load().fa_status_string(int(status)).decode()


def _stream_ptr(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return FA_BF16
    if t.dtype == torch.float32:
        return FA_F32
    raise TypeError(f"unsupported dtype {t.dtype}: bf16 or float32 tensors expected")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _check_tensor(name, t, device):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous (dense BHND layout)")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")


def fa_fwd(q, k, v, o, lse, causal: bool, scale: float, stream=None) -> None:
    """Call ``fa_fwd`` on existing tensors: q [B,Hq,N,d], k/v [B,Hkv,N,d], o like q, lse [B,Hq,N] f32."""
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("lse", lse)):
        _check_tensor(name, t, q.device)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    rc = load().fa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, N, d, float(scale),
                       int(bool(causal)), _dtype_code(q), ctypes.c_void_p(_stream_ptr(stream)))
    if rc != FA_OK:
        raise FAError(rc, "fa_fwd")


def fa_fwd_varlen(q, k, v, o, lse, cu_q, cu_k, max_seqlen_q: int, causal: bool, scale: float, stream=None) -> None:
    """Call ``fa_fwd_varlen``: q [total_q, Hq, d], k/v [total_k, Hkv, d], o like q, lse [total_q, Hq] f32;
    cu_q, cu_k int32 CUDA tensors of batch + 1 offsets."""
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("lse", lse), ("cu_q", cu_q), ("cu_k", cu_k)):
        _check_tensor(name, t, q.device)
    if cu_q.dtype != torch.int32 or cu_k.dtype != torch.int32:
        raise TypeError("cu_q and cu_k must be int32")
    total_q, Hq, d = q.shape
    total_k, Hkv = k.shape[0], k.shape[1]
    rc = load().fa_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(cu_q), _ptr(cu_k),
                              cu_q.numel() - 1, int(max_seqlen_q), total_q, total_k, Hq, Hkv, d, float(scale),
                              int(bool(causal)), _dtype_code(q), ctypes.c_void_p(_stream_ptr(stream)))
    if rc != FA_OK:
        raise FAError(rc, "fa_fwd_varlen")


def fa_fwd_partial(q, k, v, o, lse, causal: bool, scale: float, diag_offset: int, stream=None) -> None:
    """Call ``fa_fwd_partial``: ``fa_fwd`` with query row i seeing key row j iff j <= i + diag_offset (causal)."""
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("lse", lse)):
        _check_tensor(name, t, q.device)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    rc = load().fa_fwd_partial(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, N, d, float(scale),
                               int(bool(causal)), int(diag_offset), _dtype_code(q), ctypes.c_void_p(_stream_ptr(stream)))
    if rc != FA_OK:
        raise FAError(rc, "fa_fwd_partial")


def fa_merge_partials(o_parts, lse_parts, o, lse, stream=None) -> None:
    """Call ``fa_merge_partials``: o_parts [P, ..., d] and lse_parts [P, ...] into o [..., d] and lse [...]."""
    for name, t in (("o_parts", o_parts), ("lse_parts", lse_parts), ("o", o), ("lse", lse)):
        _check_tensor(name, t, o_parts.device)
    n_parts, d = o_parts.shape[0], o_parts.shape[-1]
    rows = o.numel() // d
    if o_parts.numel() != n_parts * rows * d or lse_parts.numel() != n_parts * rows or lse.numel() != rows:
        raise ValueError("o_parts, lse_parts, o and lse disagree on the number of rows")
    if lse_parts.dtype != torch.float32 or lse.dtype != torch.float32:
        raise TypeError("LSE tensors must be float32")
    rc = load().fa_merge_partials(_ptr(o_parts), _ptr(lse_parts), n_parts, rows, _ptr(o), _ptr(lse), d,
                                  _dtype_code(o_parts), ctypes.c_void_p(_stream_ptr(stream)))
    if rc != FA_OK:
        raise FAError(rc, "fa_merge_partials")


def forward_varlen(q, k, v, cu_q, cu_k, max_seqlen_q: int, causal: bool = False, scale: float | None = None,
                   stream=None):
    """Allocate O [total_q, Hq, d] and LSE [total_q, Hq] with torch and run ``fa_fwd_varlen``."""
    if scale is None:
        scale = q.shape[-1] ** -0.5
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:-1], dtype=torch.float32, device=q.device)
    fa_fwd_varlen(q, k, v, o, lse, cu_q, cu_k, max_seqlen_q, causal, scale, stream)
    return o, lse


def forward_bnhd(q, k, v, causal: bool = False, scale: float | None = None, stream=None):
    """Forward over strided [B, N, H, d] tensors (a packed batch of B sequences of N tokens).

    Returns ``(o [B, N, Hq, d], lse [B, N, Hq])``; runs ``fa_fwd_varlen`` with offsets 0, N, ..., B*N.
    """
    B, N, Hq, d = q.shape
    offs = torch.arange(0, (B + 1) * N, N, dtype=torch.int32, device=q.device)
    o, lse = forward_varlen(q.reshape(B * N, Hq, d), k.reshape(B * N, k.shape[2], d), v.reshape(B * N, v.shape[2], d),
                            offs, offs, N, causal, scale, stream)
    return o.view(B, N, Hq, d), lse.view(B, N, Hq)


def fa_bwd_varlen_workspace_size(batch: int, total_q: int, total_k: int, Hq: int, Hkv: int, d: int) -> int:
    return int(load().fa_bwd_varlen_workspace_size(batch, total_q, total_k, Hq, Hkv, d))


def fa_bwd_varlen(q, k, v, o, lse, do, dq, dk, dv, cu_q, cu_k, max_seqlen_q: int, max_seqlen_k: int, workspace,
                  causal: bool, scale: float, stream=None) -> None:
    """Call ``fa_bwd_varlen``: packed layouts as ``fa_fwd_varlen`` (q, o, do, dq [total_q, Hq, d]; k, v, dk, dv
    [total_k, Hkv, d]; lse [total_q, Hq] f32), int32 offsets cu_q, cu_k, a uint8 workspace."""
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("lse", lse), ("do", do), ("dq", dq), ("dk", dk),
                    ("dv", dv), ("cu_q", cu_q), ("cu_k", cu_k)):
        _check_tensor(name, t, q.device)
    if cu_q.dtype != torch.int32 or cu_k.dtype != torch.int32:
        raise TypeError("cu_q and cu_k must be int32")
    total_q, Hq, d = q.shape
    total_k, Hkv = k.shape[0], k.shape[1]
    ws_ptr, ws_bytes = _ws(workspace)
    rc = load().fa_bwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), _ptr(dq), _ptr(dk), _ptr(dv),
                              _ptr(cu_q), _ptr(cu_k), cu_q.numel() - 1, int(max_seqlen_q), int(max_seqlen_k), total_q,
                              total_k, Hq, Hkv, d, float(scale), int(bool(causal)), ws_ptr, ws_bytes,
                              _dtype_code(q), ctypes.c_void_p(_stream_ptr(stream)))
    if rc != FA_OK:
        raise FAError(rc, "fa_bwd_varlen")


def backward_varlen(q, k, v, o, lse, do, cu_q, cu_k, max_seqlen_q: int, max_seqlen_k: int, causal: bool = False,
                    scale: float | None = None, stream=None):
    """Allocate dQ, dK, dV and the workspace with torch and run ``fa_bwd_varlen``."""
    if scale is None:
        scale = q.shape[-1] ** -0.5
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    nbytes = fa_bwd_varlen_workspace_size(cu_q.numel() - 1, q.shape[0], k.shape[0], q.shape[1], k.shape[1],
                                          q.shape[2])
    ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=q.device)
    fa_bwd_varlen(q, k, v, o, lse, do, dq, dk, dv, cu_q, cu_k, max_seqlen_q, max_seqlen_k, ws, causal, scale, stream)
    return dq, dk, dv


def backward_bnhd(q, k, v, o, lse, do, causal: bool = False, scale: float | None = None, stream=None):
    """Backward over strided [B, N, H, d] tensors (``o``, ``lse`` as ``forward_bnhd`` returns them).

    Returns ``(dq, dk, dv)`` in the same [B, N, H, d] layouts; runs ``fa_bwd_varlen`` with offsets 0, N, ..., B*N.
    """
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    offs = torch.arange(0, (B + 1) * N, N, dtype=torch.int32, device=q.device)
    dq, dk, dv = backward_varlen(q.reshape(B * N, Hq, d), k.reshape(B * N, Hkv, d), v.reshape(B * N, Hkv, d),
                                 o.reshape(B * N, Hq, d), lse.reshape(B * N, Hq), do.reshape(B * N, Hq, d), offs, offs,
                                 N, N, causal, scale, stream)
    return dq.view(B, N, Hq, d), dk.view(B, N, Hkv, d), dv.view(B, N, Hkv, d)


def fa_bwd_partial(q, k, v, do, dk_acc, dv_acc, workspace, causal: bool, scale: float, diag_offset: int,
                   stream=None) -> None:
    """Call ``fa_bwd_partial``: add one key block's dK, dV into the f32 ``dk_acc``, ``dv_acc`` and its dQ into
    the workspace accumulator (after ``fa_bwd_prep``)."""
    for name, t in (("q", q), ("k", k), ("v", v), ("do", do), ("dk_acc", dk_acc), ("dv_acc", dv_acc)):
        _check_tensor(name, t, q.device)
    if dk_acc.dtype != torch.float32 or dv_acc.dtype != torch.float32:
        raise TypeError("dk_acc and dv_acc must be float32")
    B, Hq, N, d = q.shape
    ws_ptr, ws_bytes = _ws(workspace)
    rc = load().fa_bwd_partial(_ptr(q), _ptr(k), _ptr(v), _ptr(do), _ptr(dk_acc), _ptr(dv_acc), ws_ptr, ws_bytes, B,
                               Hq, k.shape[1], N, d, float(scale), int(bool(causal)), int(diag_offset),
                               _dtype_code(q), ctypes.c_void_p(_stream_ptr(stream)))
    if rc != FA_OK:
        raise FAError(rc, "fa_bwd_partial")


def fa_f32_to_bf16(src, dst, stream=None) -> None:
    """Call ``fa_f32_to_bf16``: dst (bf16) = src (f32), same number of elements."""
    for name, t in (("src", src), ("dst", dst)):
        _check_tensor(name, t, src.device)
    if src.dtype != torch.float32 or dst.dtype != torch.bfloat16 or src.numel() != dst.numel():
        raise TypeError("src must be float32 and dst bfloat16 with as many elements")
    rc = load().fa_f32_to_bf16(_ptr(src), _ptr(dst), src.numel(), ctypes.c_void_p(_stream_ptr(stream)))
    if rc != FA_OK:
        raise FAError(rc, "fa_f32_to_bf16")


def fa_bwd_workspace_size(B: int, Hq: int, Hkv: int, N: int, d: int) -> int:
    return int(load().fa_bwd_workspace_size(B, Hq, Hkv, N, d))


def fa_bwd(q, k, v, o, lse, do, dq, dk, dv, workspace, causal: bool, scale: float, stream=None) -> None:
    """Call ``fa_bwd`` on existing tensors; ``workspace`` is a uint8 CUDA tensor."""
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("lse", lse), ("do", do), ("dq", dq),
                    ("dk", dk), ("dv", dv)):
        _check_tensor(name, t, q.device)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    ws_ptr = None if workspace is None else ctypes.c_void_p(workspace.data_ptr())
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = load().fa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), _ptr(dq), _ptr(dk), _ptr(dv),
                       ws_ptr, ws_bytes, B, Hq, Hkv, N, d, float(scale), int(bool(causal)), _dtype_code(q),
                       ctypes.c_void_p(_stream_ptr(stream)))
    if rc != FA_OK:
        raise FAError(rc, "fa_bwd")


def _ws(workspace):
    if workspace is None:
        return None, 0
    return ctypes.c_void_p(workspace.data_ptr()), workspace.numel() * workspace.element_size()


def fa_bwd_prep(o, lse, do, workspace, Hkv: int, stream=None) -> None:
    """Stage 1 of ``fa_bwd``: D, padded log2 LSE and a zeroed dQ accumulator in ``workspace``."""
    B, Hq, N, d = o.shape
    ws, nbytes = _ws(workspace)
    rc = load().fa_bwd_prep(_ptr(o), _ptr(lse), _ptr(do), ws, nbytes, B, Hq, Hkv, N, d, _dtype_code(o),
                            ctypes.c_void_p(_stream_ptr(stream)))
    if rc != FA_OK:
        raise FAError(rc, "fa_bwd_prep")


def fa_bwd_main(q, k, v, do, dk, dv, workspace, causal: bool, scale: float, stream=None) -> None:
    """Stage 2 of ``fa_bwd``: the recompute kernel (dK, dV, and dQ into the accumulator)."""
    B, Hq, N, d = q.shape
    ws, nbytes = _ws(workspace)
    rc = load().fa_bwd_main(_ptr(q), _ptr(k), _ptr(v), _ptr(do), _ptr(dk), _ptr(dv), ws, nbytes, B, Hq,
                            k.shape[1], N, d, float(scale), int(bool(causal)), _dtype_code(q),
                            ctypes.c_void_p(_stream_ptr(stream)))
    if rc != FA_OK:
        raise FAError(rc, "fa_bwd_main")


def fa_bwd_dq(dq, workspace, Hkv: int, stream=None) -> None:
    """Stage 3 of ``fa_bwd``: f32 accumulator -> bf16 ``dq``."""
    B, Hq, N, d = dq.shape
    ws, nbytes = _ws(workspace)
    rc = load().fa_bwd_dq(_ptr(dq), ws, nbytes, B, Hq, Hkv, N, d, _dtype_code(dq),
                          ctypes.c_void_p(_stream_ptr(stream)))
    if rc != FA_OK:
        raise FAError(rc, "fa_bwd_dq")


NOALLOC_SCRATCH_BYTES = 16 * 1024 * 1024  # FA_NOALLOC_SCRATCH_BYTES in include/fa.h


def fa_bwd_noalloc(q, k, v, o, lse, do, dq, dk, dv, causal: bool, scale: float, stream=None) -> None:
    """Call ``fa_bwd_noalloc``: the backward with the library's built-in scratch.

    For callers that cannot allocate device memory (a locked or pre-planned
    allocator, plain C callers without one). Problems needing more than
    ``NOALLOC_SCRATCH_BYTES`` of scratch raise ``FAError`` (FA_ERR_WORKSPACE).
    Calls share one scratch array per GPU: do not let two of them overlap on
    the device.
    """
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("lse", lse), ("do", do), ("dq", dq),
                    ("dk", dk), ("dv", dv)):
        _check_tensor(name, t, q.device)
    B, Hq, N, d = q.shape
    rc = load().fa_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), _ptr(dq), _ptr(dk),
                               _ptr(dv), B, Hq, k.shape[1], N, d, float(scale), int(bool(causal)),
                               _dtype_code(q), ctypes.c_void_p(_stream_ptr(stream)))
    if rc != FA_OK:
        raise FAError(rc, "fa_bwd_noalloc")


def fa_fwd_kvcache_workspace_size(B: int, Hq: int, Hkv: int, Nq: int, Nk: int, d: int) -> int:
    return int(load().fa_fwd_kvcache_workspace_size(B, Hq, Hkv, Nq, Nk, d))


def fa_fwd_kvcache(q, k, v, o, lse, workspace, causal: bool, scale: float, stream=None) -> None:
    """Call ``fa_fwd_kvcache``: q [B,Hq,Nq,d] against k/v [B,Hkv,Nk,d] (Nk >= Nq); o like q, lse [B,Hq,Nq]."""
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("lse", lse)):
        _check_tensor(name, t, q.device)
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    ws, nbytes = _ws(workspace)
    rc = load().fa_fwd_kvcache(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), ws, nbytes, B, Hq, Hkv, Nq, Nk, d,
                               float(scale), int(bool(causal)), _dtype_code(q), ctypes.c_void_p(_stream_ptr(stream)))
    if rc != FA_OK:
        raise FAError(rc, "fa_fwd_kvcache")


def forward_kvcache(q, k, v, causal: bool = False, scale: float | None = None, stream=None):
    """Allocate O, LSE and the workspace with torch and run ``fa_fwd_kvcache``. Returns ``(o, lse)``."""
    if scale is None:
        scale = q.shape[-1] ** -0.5
    B, Hq, Nq, d = q.shape
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:-1], dtype=torch.float32, device=q.device)
    nbytes = fa_fwd_kvcache_workspace_size(B, Hq, k.shape[1], Nq, k.shape[2], d)
    ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=q.device)
    fa_fwd_kvcache(q, k, v, o, lse, ws, causal, scale, stream)
    return o, lse


def forward(q, k, v, causal: bool = False, scale: float | None = None, stream=None):
    """Allocate O and LSE with torch and run ``fa_fwd``. Returns ``(o, lse)``."""
    if scale is None:
        scale = q.shape[-1] ** -0.5
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:-1], dtype=torch.float32, device=q.device)
    fa_fwd(q, k, v, o, lse, causal, scale, stream)
    return o, lse


def backward(q, k, v, o, lse, do, causal: bool = False, scale: float | None = None, stream=None):
    """Allocate dQ, dK, dV and the workspace with torch and run ``fa_bwd``."""
    if scale is None:
        scale = q.shape[-1] ** -0.5
    B, Hq, N, d = q.shape
    dq = torch.empty_like(q)
    dk = torch.empty_like(k)
    dv = torch.empty_like(v)
    ws = torch.empty(max(fa_bwd_workspace_size(B, Hq, k.shape[1], N, d), 16), dtype=torch.uint8, device=q.device)
    fa_bwd(q, k, v, o, lse, do, dq, dk, dv, ws, causal, scale, stream)
    return dq, dk, dv


def fa_last_device_status(stream=None) -> int:
    return int(load().fa_last_device_status(ctypes.c_void_p(_stream_ptr(stream))))


def fa_set_wait_timeout_ns(ns: int) -> None:
    load().fa_set_wait_timeout_ns(int(ns))


def fa_selftest_wait_timeout(ns: int, stream=None) -> int:
    return int(load().fa_selftest_wait_timeout(int(ns), ctypes.c_void_p(_stream_ptr(stream))))
