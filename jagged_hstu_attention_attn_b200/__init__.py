"""Jagged HSTU pointwise attention for NVIDIA B200 (sm_100a).

Thin Python binding of ``libhstu.so`` (C ABI in ``include/hstu.h``).  The
functions have the C names and only marshal arguments: torch supplies device
memory and the current CUDA stream, every step of the computation runs in the
library's CUDA kernels.  There is no CPU fallback: if the library is missing
or no GPU is present the calls raise.

    O = Mask(SiLU(scale (Q K^T + Bias))) V
    Bias[i, j] = w_pos[min(i - j, P - 1)] + w_ts[min(bitlen(max(t_i - t_j, 0)), NB - 1)]

("Scaling Generative Recommendations with Context Parallelism on
Hierarchical Sequential Transducers", §2.1-§2.3; "Actions Speak Louder than
Words", §3.1 and App. F.3.)
"""
from __future__ import annotations

import ctypes
import math
import os
import threading
from typing import Optional, Tuple

__all__ = [
    "HstuError", "lib", "lib_path", "hstu_status_str", "hstu_version", "hstu_kernel_launches",
    "hstu_last_cuda_error", "hstu_jagged_attn_fwd", "hstu_jagged_attn_fwd_targets",
    "hstu_jagged_attn_bwd", "hstu_jagged_attn_bwd_workspace_bytes",
    "hstu_cp_reorder", "hstu_cp_restore", "hstu_cp_paired_attn_fwd", "hstu_bucket_indices",
    "hstu_jagged_attn_bwd_noalloc", "NOALLOC_MAX_ELEMS", "EXPORTED_SYMBOLS",
    "hstu_selftest_wait_timeout", "hstu_jagged_attn_fwd_candidates", "hstu_norm_gate_fwd",
    "hstu_norm_gate_bwd", "hstu_sl_select", "hstu_gather_rows", "hstu_gather_rows_multi",
    "sl_target_length",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
lib_path = os.path.join(_PKG, "libhstu.so")
_lock = threading.Lock()
_lib = None

EXPORTED_SYMBOLS = (
    "hstu_status_str", "hstu_version", "hstu_kernel_launches", "hstu_jagged_attn_fwd",
    "hstu_jagged_attn_bwd_workspace_bytes", "hstu_jagged_attn_bwd", "hstu_cp_reorder",
    "hstu_cp_restore", "hstu_cp_paired_attn_fwd", "hstu_bucket_indices",
    "hstu_jagged_attn_bwd_noalloc", "hstu_last_cuda_error", "hstu_jagged_attn_fwd_targets",
    "hstu_selftest_wait_timeout", "hstu_jagged_attn_fwd_candidates", "hstu_norm_gate_fwd",
    "hstu_norm_gate_bwd", "hstu_sl_select", "hstu_gather_rows", "hstu_gather_rows_multi",
)

_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
_int = ctypes.c_int
_f32 = ctypes.c_float


class HstuError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = int(code)
        msg = f"{where}: {hstu_status_str(code)} ({code})"
        if self.code == -8:   # HSTU_ERR_CUDA: name the CUDA error behind it
            msg += f": {hstu_last_cuda_error()}"
        super().__init__(msg)


def lib() -> ctypes.CDLL:
    """The loaded libhstu.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(lib_path):
            raise ImportError(
                f"{lib_path} is missing: build it with "
                "`python -m jagged_hstu_attention_attn_b200.build`")
        L = ctypes.CDLL(lib_path)
        L.hstu_status_str.restype = ctypes.c_char_p
        L.hstu_status_str.argtypes = [_int]
        L.hstu_version.restype = _int
        L.hstu_last_cuda_error.restype = ctypes.c_char_p
        L.hstu_last_cuda_error.argtypes = []
        L.hstu_kernel_launches.restype = _i64
        L.hstu_jagged_attn_fwd.restype = _int
        L.hstu_jagged_attn_fwd.argtypes = [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _vp, _i64,
                                           _vp, _i64, _int, _int, _int, _f32, _int, _vp, _vp, _vp]
        L.hstu_jagged_attn_fwd_targets.restype = _int
        L.hstu_jagged_attn_fwd_targets.argtypes = [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp,
                                                   _vp, _i64, _vp, _i64, _int, _int, _int, _f32,
                                                   _int, _vp, _vp, _vp]
        L.hstu_jagged_attn_fwd_candidates.restype = _int
        L.hstu_jagged_attn_fwd_candidates.argtypes = [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64,
                                                      _i64, _vp, _vp, _i64, _vp, _i64, _int, _int,
                                                      _int, _f32, _int, _vp, _vp, _vp]
        L.hstu_cp_paired_attn_fwd.restype = _int
        L.hstu_cp_paired_attn_fwd.argtypes = [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _int, _vp,
                                              _vp, _i64, _vp, _i64, _int, _int, _int, _f32, _int,
                                              _vp, _vp, _vp]
        L.hstu_jagged_attn_bwd_workspace_bytes.restype = _i64
        L.hstu_jagged_attn_bwd_workspace_bytes.argtypes = [_i64, _int, _int]
        L.hstu_jagged_attn_bwd.restype = _int
        L.hstu_jagged_attn_bwd.argtypes = [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _vp, _i64,
                                           _vp, _i64, _int, _int, _int, _f32, _vp, _vp, _vp, _vp,
                                           _vp, _vp, _vp, _i64, _vp, _vp]
        L.hstu_cp_reorder.restype = _int
        L.hstu_cp_reorder.argtypes = [_vp, _vp, _i64, _vp, _i64, _i64, _int, _vp, _vp, _vp, _vp]
        L.hstu_cp_restore.restype = _int
        L.hstu_cp_restore.argtypes = [_vp, _vp, _i64, _vp, _i64, _i64, _int, _vp, _vp]
        L.hstu_jagged_attn_bwd_noalloc.restype = _int
        L.hstu_jagged_attn_bwd_noalloc.argtypes = [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp,
                                                   _vp, _i64, _vp, _i64, _int, _int, _int, _f32,
                                                   _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]
        L.hstu_bucket_indices.restype = _int
        L.hstu_bucket_indices.argtypes = [_vp, _vp, _i64, _i64, _vp, _vp]
        L.hstu_selftest_wait_timeout.restype = _int
        L.hstu_selftest_wait_timeout.argtypes = [_i64, _vp, _vp, _vp]
        L.hstu_norm_gate_fwd.restype = _int
        L.hstu_norm_gate_fwd.argtypes = [_vp, _vp, _vp, _i64, _i64, _f32, _vp]
        L.hstu_norm_gate_bwd.restype = _int
        L.hstu_norm_gate_bwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _f32, _vp]
        L.hstu_sl_select.restype = _int
        L.hstu_sl_select.argtypes = [_vp, _i64, _i64, _vp, _vp, _i64, _vp, _vp, _vp, _vp]
        L.hstu_gather_rows.restype = _int
        L.hstu_gather_rows.argtypes = [_vp, _i64, _vp, _i64, _vp, _vp, _i64, _vp]
        L.hstu_gather_rows_multi.restype = _int
        L.hstu_gather_rows_multi.argtypes = [_int, _vp, _vp, _vp, _i64, _vp, _vp, _i64, _vp]
        _lib = L
        return L


def hstu_status_str(code: int) -> str:
    return lib().hstu_status_str(int(code)).decode()


def hstu_last_cuda_error() -> str:
    """The CUDA error behind the last HSTU_ERR_CUDA on this host thread."""
    return lib().hstu_last_cuda_error().decode()


def hstu_version() -> int:
    return int(lib().hstu_version())


def hstu_kernel_launches() -> int:
    """Kernels libhstu has launched in this process so far."""
    return int(lib().hstu_kernel_launches())


# ---------------------------------------------------------------------------
# marshalling helpers (torch is only the allocator and the stream source)
# ---------------------------------------------------------------------------

def _torch():
    import torch
    return torch


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _need(t, name, dtype=None, ndim=None):
    torch = _torch()
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (libhstu has no CPU path)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims")


def _check(code: int, where: str):
    if code != 0:
        raise HstuError(code, where)


def _attn_inputs(q, k, v, seq_offsets, timestamps, w_pos, w_ts):
    torch = _torch()
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, torch.bfloat16, 3)
    _need(seq_offsets, "seq_offsets", torch.int64, 1)
    _need(timestamps, "timestamps", torch.int64, 1)
    _need(w_pos, "w_pos", torch.float32, 1)
    _need(w_ts, "w_ts", torch.float32, 1)
    T, H, d = q.shape
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must have the same [T, H, d] shape")
    if timestamps.shape[0] != T:
        raise ValueError("timestamps must have T entries")
    return T, H, d, seq_offsets.shape[0] - 1


def hstu_jagged_attn_fwd(q, k, v, seq_offsets, timestamps, w_pos, w_ts, *, scale=None,
                         max_seq_len: int = 0, out_fp32: bool = False, out=None,
                         dev_status=None, stream=None):
    """out [T, H, d] = HSTU attention over the jagged batch (bf16, or fp32 if out_fp32)."""
    torch = _torch()
    T, H, d, B = _attn_inputs(q, k, v, seq_offsets, timestamps, w_pos, w_ts)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((T, H, d), dtype=torch.float32 if out_fp32 else torch.bfloat16,
                          device=q.device)
    _need(out, "out", torch.float32 if out_fp32 else torch.bfloat16, 3)
    code = lib().hstu_jagged_attn_fwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(seq_offsets), B, T, int(max_seq_len), _ptr(timestamps),
        _ptr(w_pos), w_pos.shape[0], _ptr(w_ts), w_ts.shape[0], H, d, d, float(scale),
        1 if out_fp32 else 0, _ptr(out), _ptr(dev_status), _stream(stream))
    _check(code, "hstu_jagged_attn_fwd")
    return out


def hstu_jagged_attn_fwd_targets(q, k, v, seq_offsets, num_targets, timestamps, w_pos, w_ts, *,
                                 scale=None, max_seq_len: int = 0, out_fp32: bool = False,
                                 out=None, dev_status=None, stream=None):
    """Target-aware forward: the last num_targets[b] rows of sequence b are
    candidates that attend the history and themselves only (int64 [B] on the
    device)."""
    torch = _torch()
    T, H, d, B = _attn_inputs(q, k, v, seq_offsets, timestamps, w_pos, w_ts)
    _need(num_targets, "num_targets", torch.int64, 1)
    if num_targets.shape[0] != B:
        raise ValueError("num_targets must hold one count per sequence")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((T, H, d), dtype=torch.float32 if out_fp32 else torch.bfloat16,
                          device=q.device)
    _need(out, "out", torch.float32 if out_fp32 else torch.bfloat16, 3)
    code = lib().hstu_jagged_attn_fwd_targets(
        _ptr(q), _ptr(k), _ptr(v), _ptr(seq_offsets), _ptr(num_targets), B, T,
        int(max_seq_len), _ptr(timestamps), _ptr(w_pos), w_pos.shape[0], _ptr(w_ts),
        w_ts.shape[0], H, d, d, float(scale), 1 if out_fp32 else 0, _ptr(out), _ptr(dev_status),
        _stream(stream))
    _check(code, "hstu_jagged_attn_fwd_targets")
    return out


def hstu_jagged_attn_fwd_candidates(q, k, v, seq_offsets, num_targets, timestamps, w_pos, w_ts,
                                    *, scale=None, max_seq_len: int = 0, max_targets: int = 0,
                                    out_fp32: bool = False, out=None, dev_status=None,
                                    stream=None):
    """Candidates-only target-aware forward: computes and writes only the last
    num_targets[b] rows of every sequence (history rows of out untouched)."""
    torch = _torch()
    T, H, d, B = _attn_inputs(q, k, v, seq_offsets, timestamps, w_pos, w_ts)
    _need(num_targets, "num_targets", torch.int64, 1)
    if num_targets.shape[0] != B:
        raise ValueError("num_targets must hold one count per sequence")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.zeros((T, H, d), dtype=torch.float32 if out_fp32 else torch.bfloat16,
                          device=q.device)
    _need(out, "out", torch.float32 if out_fp32 else torch.bfloat16, 3)
    code = lib().hstu_jagged_attn_fwd_candidates(
        _ptr(q), _ptr(k), _ptr(v), _ptr(seq_offsets), _ptr(num_targets), B, T,
        int(max_seq_len), int(max_targets), _ptr(timestamps), _ptr(w_pos), w_pos.shape[0],
        _ptr(w_ts), w_ts.shape[0], H, d, d, float(scale), 1 if out_fp32 else 0, _ptr(out),
        _ptr(dev_status), _stream(stream))
    _check(code, "hstu_jagged_attn_fwd_candidates")
    return out


def hstu_jagged_attn_bwd_workspace_bytes(T: int, num_heads: int, d: int) -> int:
    n = int(lib().hstu_jagged_attn_bwd_workspace_bytes(int(T), int(num_heads), int(d)))
    if n < 0:
        raise HstuError(n, "hstu_jagged_attn_bwd_workspace_bytes")
    return n


def hstu_jagged_attn_bwd(q, k, v, seq_offsets, timestamps, w_pos, w_ts, dout, *, scale=None,
                         max_seq_len: int = 0, dq=None, dk=None, dv=None, dw_pos=None,
                         dw_ts=None, workspace=None, dev_status=None, stream=None):
    """(dq, dk, dv, dw_pos, dw_ts) for the loss sum(out * dout)."""
    torch = _torch()
    T, H, d, B = _attn_inputs(q, k, v, seq_offsets, timestamps, w_pos, w_ts)
    _need(dout, "dout", torch.bfloat16, 3)
    dev = q.device
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    dw_pos = torch.empty_like(w_pos) if dw_pos is None else dw_pos
    dw_ts = torch.empty_like(w_ts) if dw_ts is None else dw_ts
    nbytes = hstu_jagged_attn_bwd_workspace_bytes(T, H, d)
    if workspace is None:
        workspace = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=dev)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    code = lib().hstu_jagged_attn_bwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(seq_offsets), B, T, int(max_seq_len), _ptr(timestamps),
        _ptr(w_pos), w_pos.shape[0], _ptr(w_ts), w_ts.shape[0], H, d, d, float(scale),
        _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dw_pos), _ptr(dw_ts), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(dev_status), _stream(stream))
    _check(code, "hstu_jagged_attn_bwd")
    return dq, dk, dv, dw_pos, dw_ts


# T * num_heads * d limit of hstu_jagged_attn_bwd_noalloc (HSTU_BWD_NOALLOC_MAX_ELEMS)
NOALLOC_MAX_ELEMS = 4 * 1024 * 1024


def hstu_jagged_attn_bwd_noalloc(q, k, v, seq_offsets, timestamps, w_pos, w_ts, dout, *, dq,
                                 dk, dv, dw_pos, dw_ts, scale=None, max_seq_len: int = 0,
                                 dev_status=None, stream=None):
    """Backward that allocates nothing inside the library: it uses the library's
    static scratch array instead of a workspace.  For callers that cannot
    allocate device memory; every output buffer must be passed in.  Calls on a
    device share the scratch, so overlapping calls race (see include/hstu.h)."""
    torch = _torch()
    T, H, d, B = _attn_inputs(q, k, v, seq_offsets, timestamps, w_pos, w_ts)
    _need(dout, "dout", torch.bfloat16, 3)
    for t, n in ((dq, "dq"), (dk, "dk"), (dv, "dv")):
        _need(t, n, torch.bfloat16, 3)
    _need(dw_pos, "dw_pos", torch.float32, 1)
    _need(dw_ts, "dw_ts", torch.float32, 1)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    code = lib().hstu_jagged_attn_bwd_noalloc(
        _ptr(q), _ptr(k), _ptr(v), _ptr(seq_offsets), B, T, int(max_seq_len), _ptr(timestamps),
        _ptr(w_pos), w_pos.shape[0], _ptr(w_ts), w_ts.shape[0], H, d, d, float(scale),
        _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dw_pos), _ptr(dw_ts), _ptr(dev_status),
        _stream(stream))
    _check(code, "hstu_jagged_attn_bwd_noalloc")
    return dq, dk, dv, dw_pos, dw_ts


def _row_bytes(t) -> int:
    T = t.shape[0]
    return (t.numel() // max(T, 1)) * t.element_size() if T else \
        int(t.element_size() * max(1, int(_prod(t.shape[1:]))))


def _prod(xs):
    r = 1
    for x in xs:
        r *= int(x)
    return r


def hstu_cp_reorder(src, seq_offsets, C: int, *, dst=None, dst_offsets=None, global_pos=None,
                    want_maps: bool = True, dev_status=None, stream=None):
    """Paired layout of ``src`` (rows along dim 0): returns (dst, dst_offsets, global_pos)."""
    torch = _torch()
    _need(src, "src")
    _need(seq_offsets, "seq_offsets", torch.int64, 1)
    B = seq_offsets.shape[0] - 1
    T = src.shape[0]
    dst = torch.empty_like(src) if dst is None else dst
    if want_maps:
        if dst_offsets is None:
            dst_offsets = torch.empty(C * B + 1, dtype=torch.int64, device=src.device)
        if global_pos is None:
            global_pos = torch.empty(T, dtype=torch.int32, device=src.device)
    code = lib().hstu_cp_reorder(_ptr(src), _ptr(dst), _row_bytes(src), _ptr(seq_offsets), B, T,
                                 int(C), _ptr(dst_offsets), _ptr(global_pos), _ptr(dev_status),
                                 _stream(stream))
    _check(code, "hstu_cp_reorder")
    return dst, dst_offsets, global_pos


def hstu_cp_restore(src, seq_offsets, C: int, *, dst=None, dev_status=None, stream=None):
    """Inverse of hstu_cp_reorder."""
    torch = _torch()
    _need(src, "src")
    _need(seq_offsets, "seq_offsets", torch.int64, 1)
    B = seq_offsets.shape[0] - 1
    T = src.shape[0]
    dst = torch.empty_like(src) if dst is None else dst
    code = lib().hstu_cp_restore(_ptr(src), _ptr(dst), _row_bytes(src), _ptr(seq_offsets), B, T,
                                 int(C), _ptr(dev_status), _stream(stream))
    _check(code, "hstu_cp_restore")
    return dst


def hstu_cp_paired_attn_fwd(pq, pk, pv, seq_offsets, ptimestamps, C: int, w_pos, w_ts, *,
                            scale=None, max_seq_len: int = 0, out_fp32: bool = False, out=None,
                            dev_status=None, stream=None):
    """Attention on paired buffers (hstu_cp_reorder outputs); out is in the paired layout."""
    torch = _torch()
    T, H, d, B = _attn_inputs(pq, pk, pv, seq_offsets, ptimestamps, w_pos, w_ts)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((T, H, d), dtype=torch.float32 if out_fp32 else torch.bfloat16,
                          device=pq.device)
    code = lib().hstu_cp_paired_attn_fwd(
        _ptr(pq), _ptr(pk), _ptr(pv), _ptr(seq_offsets), B, T, int(max_seq_len), int(C),
        _ptr(ptimestamps), _ptr(w_pos), w_pos.shape[0], _ptr(w_ts), w_ts.shape[0], H, d, d,
        float(scale), 1 if out_fp32 else 0, _ptr(out), _ptr(dev_status), _stream(stream))
    _check(code, "hstu_cp_paired_attn_fwd")
    return out


def hstu_bucket_indices(t_q, t_k, NB: int, *, out=None, stream=None):
    """int32 buckets of t_q - t_k exactly as the attention kernels compute them."""
    torch = _torch()
    _need(t_q, "t_q", torch.int64, 1)
    _need(t_k, "t_k", torch.int64, 1)
    n = t_q.shape[0]
    out = torch.empty(n, dtype=torch.int32, device=t_q.device) if out is None else out
    code = lib().hstu_bucket_indices(_ptr(t_q), _ptr(t_k), n, int(NB), _ptr(out),
                                     _stream(stream))
    _check(code, "hstu_bucket_indices")
    return out


def hstu_selftest_wait_timeout(limit_ns: int, *, dev_status, result, stream=None):
    """Run the bounded-wait self-test: one warp waits on an mbarrier nothing
    arrives on; afterwards dev_status holds HSTU_ERR_TIMEOUT and result 0."""
    torch = _torch()
    _need(dev_status, "dev_status", torch.int32, 1)
    _need(result, "result", torch.int32, 1)
    code = lib().hstu_selftest_wait_timeout(int(limit_ns), _ptr(dev_status), _ptr(result),
                                            _stream(stream))
    _check(code, "hstu_selftest_wait_timeout")


def _rows2d(t, name):
    """[T, N] view of a contiguous bf16 tensor whose trailing dims are the
    token's features ([T, H, d] or [T, N])."""
    torch = _torch()
    _need(t, name, torch.bfloat16)
    if t.dim() < 2:
        raise ValueError(f"{name} must have a token dim and feature dims")
    n = 1
    for s_ in t.shape[1:]:
        n *= int(s_)
    return t.reshape(t.shape[0], n)


def hstu_norm_gate_fwd(o, u, *, eps: float = 1e-5, out=None, stream=None):
    """y = LayerNorm(o) * u per token over all its H*d features (no affine),
    the HSTU layer's Norm(A(X)V(X)) ⊙ U(X); o, u bf16 of the same shape."""
    torch = _torch()
    o2, u2 = _rows2d(o, "o"), _rows2d(u, "u")
    if o2.shape != u2.shape:
        raise ValueError("o and u must have the same shape")
    out = torch.empty_like(o) if out is None else out
    y2 = _rows2d(out, "out")
    if y2.shape != o2.shape:
        raise ValueError("out must have the shape of o")
    code = lib().hstu_norm_gate_fwd(_ptr(o2), _ptr(u2), _ptr(y2), o2.shape[0], o2.shape[1],
                                    float(eps), _stream(stream))
    _check(code, "hstu_norm_gate_fwd")
    return out


def hstu_norm_gate_bwd(o, u, dy, *, eps: float = 1e-5, d_o=None, d_u=None, stream=None):
    """(d_o, d_u): the exact gradients of hstu_norm_gate_fwd for the output
    gradient dy (bf16, same shape as o and u)."""
    torch = _torch()
    o2, u2, dy2 = _rows2d(o, "o"), _rows2d(u, "u"), _rows2d(dy, "dy")
    if not (o2.shape == u2.shape == dy2.shape):
        raise ValueError("o, u and dy must have the same shape")
    d_o = torch.empty_like(o) if d_o is None else d_o
    d_u = torch.empty_like(u) if d_u is None else d_u
    do2, du2 = _rows2d(d_o, "d_o"), _rows2d(d_u, "d_u")
    if do2.shape != o2.shape or du2.shape != o2.shape:
        raise ValueError("d_o and d_u must have the shape of o")
    code = lib().hstu_norm_gate_bwd(_ptr(o2), _ptr(u2), _ptr(dy2), _ptr(do2), _ptr(du2),
                                    o2.shape[0], o2.shape[1], float(eps), _stream(stream))
    _check(code, "hstu_norm_gate_bwd")
    return d_o, d_u


def sl_target_length(N: int, alpha: float) -> int:
    """Stochastic Length target length floor(N^(alpha / 2)), between 1 and N."""
    if N < 1 or not alpha > 0:
        raise ValueError("N >= 1 and alpha > 0 required")
    v = math.pow(float(N), alpha / 2.0)
    L = int(math.floor(v))
    if L + 1 <= N and abs(v - (L + 1)) < 1e-9 * v:  # a power landing just below an integer
        L += 1
    return max(1, min(L, N))


def hstu_sl_select(seq_offsets, u_tok, u_seq, L: int, *, dst_offsets=None, src_rows=None,
                   dev_status=None, stream=None):
    """Stochastic Length selection: (dst_offsets [B + 1], src_rows [T]) with the
    input row of every selected row in src_rows[:dst_offsets[B]] (device values;
    nothing is read back).  u_tok: uint32 [T] and u_seq: uint32 [B] random draws
    (torch.int32 tensors holding the uint32 bits)."""
    torch = _torch()
    _need(seq_offsets, "seq_offsets", torch.int64, 1)
    _need(u_tok, "u_tok", None, 1)
    _need(u_seq, "u_seq", None, 1)
    if u_tok.element_size() != 4 or u_seq.element_size() != 4:
        raise TypeError("u_tok and u_seq must hold 32-bit draws")
    B = seq_offsets.shape[0] - 1
    T = u_tok.shape[0]
    if u_seq.shape[0] != B:
        raise ValueError("u_seq must have one draw per sequence")
    dev = seq_offsets.device
    if dst_offsets is None:
        dst_offsets = torch.empty(B + 1, dtype=torch.int64, device=dev)
    if src_rows is None:
        src_rows = torch.empty(max(T, 1), dtype=torch.int32, device=dev)
    code = lib().hstu_sl_select(_ptr(seq_offsets), B, T, _ptr(u_tok), _ptr(u_seq), int(L),
                                _ptr(dst_offsets), _ptr(src_rows), _ptr(dev_status),
                                _stream(stream))
    _check(code, "hstu_sl_select")
    return dst_offsets, src_rows


def hstu_gather_rows(src, src_rows, n_rows, *, max_rows=None, out=None, stream=None):
    """out[r] = src[src_rows[r]] for r < n_rows (a device int64 scalar tensor,
    e.g. dst_offsets[B:]); out has max_rows rows (default: src's)."""
    torch = _torch()
    _need(src, "src")
    _need(src_rows, "src_rows", torch.int32, 1)
    _need(n_rows, "n_rows", torch.int64)
    if max_rows is None:
        max_rows = src.shape[0]
    if out is None:
        out = torch.empty((max_rows,) + tuple(src.shape[1:]), dtype=src.dtype, device=src.device)
    if out.shape[0] < max_rows or src_rows.shape[0] < max_rows:
        raise ValueError("out and src_rows must hold max_rows rows")
    code = lib().hstu_gather_rows(_ptr(src), src.shape[0], _ptr(out), _row_bytes(src),
                                  _ptr(src_rows), _ptr(n_rows), int(max_rows), _stream(stream))
    _check(code, "hstu_gather_rows")
    return out


def hstu_gather_rows_multi(srcs, src_rows, n_rows, *, max_rows=None, outs=None, stream=None):
    """hstu_gather_rows for up to 8 tensors with the same rows, in one launch."""
    torch = _torch()
    srcs = list(srcs)
    if not 1 <= len(srcs) <= 8:
        raise ValueError("1 to 8 tensors")
    T = srcs[0].shape[0]
    for i, t in enumerate(srcs):
        _need(t, f"srcs[{i}]")
        if t.shape[0] != T:
            raise ValueError("every src must have the same number of rows")
    _need(src_rows, "src_rows", torch.int32, 1)
    _need(n_rows, "n_rows", torch.int64)
    if max_rows is None:
        max_rows = T
    if outs is None:
        outs = [torch.empty((max_rows,) + tuple(t.shape[1:]), dtype=t.dtype, device=t.device)
                for t in srcs]
    if src_rows.shape[0] < max_rows or any(o.shape[0] < max_rows for o in outs):
        raise ValueError("outs and src_rows must hold max_rows rows")
    n = len(srcs)
    sp = (ctypes.c_void_p * n)(*[t.data_ptr() for t in srcs])
    dp = (ctypes.c_void_p * n)(*[o.data_ptr() for o in outs])
    rb = (ctypes.c_int64 * n)(*[_row_bytes(t) for t in srcs])
    code = lib().hstu_gather_rows_multi(n, ctypes.cast(sp, ctypes.c_void_p),
                                        ctypes.cast(dp, ctypes.c_void_p),
                                        ctypes.cast(rb, ctypes.c_void_p), T, _ptr(src_rows),
                                        _ptr(n_rows), int(max_rows), _stream(stream))
    _check(code, "hstu_gather_rows_multi")
    return outs

