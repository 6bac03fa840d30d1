"""fp64 CPU oracle for jagged HSTU attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its
``cpu_baseline`` leg and ``--impl reference`` arm) may import this package.
The product path (``jagged_hstu_attention_attn_b200``) never imports it and
shares no code with it.

The arithmetic lives in ``hstu_oracle.c`` (plain C, double precision); this
module compiles it with gcc on first use and marshals numpy arrays.

Functions and the passages they follow:

* :func:`fwd`, :func:`fwd_rows` -- the HSTUAttention equation of "Scaling
  Generative Recommendations with Context Parallelism on Hierarchical
  Sequential Transducers" §2.1, with the timestamp bias of the same section
  and the relative attention bias of "Actions Speak Louder than Words"
  App. F.3.
* :func:`bwd`, :func:`bwd_rows` -- the exact derivative of :func:`fwd`.
* :func:`bucket`, :func:`bucket_of`, :func:`bucket_of_many` -- the bucket reading
  min(bitlen(max(dt, 0)), NB - 1) of the CP paper's "grouping" step (§2.1).
* :func:`cp_reorder`, :func:`cp_restore`, :func:`cp_rank_pairs`,
  :func:`paired_fwd` -- the load-balanced 2C mini-chunk pairing of the CP
  paper §2.3 (figure "Load Balanced CP with 2*CP_size Mini-chunks").
* :func:`fwd_targets`, :func:`fwd_targets_rows` -- the target-aware forward
  of M-FALCON ("Actions Speak Louder than Words", App. H): the last
  num_targets[b] rows of sequence b are candidates that do not attend to one
  another, and one pass must give what separate forward passes, one per
  candidate over the user history followed by that candidate, give.  The
  oracle is that statement written out: history rows are the causal rows of
  :func:`fwd`; each candidate is the last row of :func:`fwd_rows` over its own
  pass [history, candidate].

* :func:`norm_gate_fwd`, :func:`norm_gate_bwd` -- the HSTU layer's
  ``Norm(A(X)V(X)) ⊙ U(X)`` ("Actions Speak Louder than Words" §3), in numpy
  float64 in ``norm_gate.py`` (the reading of ``Norm`` is stated there).

* ``oracle.stochastic_length`` -- Stochastic Length subsequence selection
  ("Actions Speak Louder than Words" §3.2, §4.2), in numpy in
  ``stochastic_length.py`` (the reading of the selection rule is stated there).

All of them are pinned in ``tests/test_oracle.py``,
``tests/test_oracle_norm_gate.py`` and ``tests/test_oracle_stochastic_length.py``;
none is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional, Tuple

import numpy as np

from .norm_gate import DEFAULT_EPS as NORM_EPS, norm_gate_bwd, norm_gate_fwd  # noqa: F401
from . import stochastic_length  # noqa: F401

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hstu_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

_i64p = ctypes.POINTER(ctypes.c_int64)
_i32p = ctypes.POINTER(ctypes.c_int32)
_f64p = ctypes.POINTER(ctypes.c_double)
_u8p = ctypes.POINTER(ctypes.c_uint8)


def build(force: bool = False) -> str:
    """Compile hstu_oracle.c into oracle/liboracle.so (gcc, -O2, OpenMP)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        lib.oracle_bucket.restype = ctypes.c_int64
        lib.oracle_bucket.argtypes = [ctypes.c_int64, ctypes.c_int64]
        lib.oracle_bucket_of.restype = ctypes.c_int64
        lib.oracle_bucket_of.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64]
        lib.oracle_bucket_of_many.restype = None
        lib.oracle_bucket_of_many.argtypes = [_i64p, _i64p, ctypes.c_int64, ctypes.c_int64, _i64p]
        lib.oracle_set_threads.argtypes = [ctypes.c_int]
        lib.oracle_get_threads.restype = ctypes.c_int
        common = [_f64p, _f64p, _f64p, _i64p, ctypes.c_int64, _i64p, _f64p, ctypes.c_int64,
                  _f64p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_double]
        lib.oracle_fwd.argtypes = common + [_f64p]
        lib.oracle_fwd_rows.argtypes = common + [_i64p, _i64p, ctypes.c_int64, _f64p]
        lib.oracle_bwd.argtypes = common + [_f64p, _f64p, _f64p, _f64p, _f64p, _f64p]
        lib.oracle_bwd_rows.argtypes = common + [_f64p, _i64p, _i64p, ctypes.c_int64, _f64p,
                                                 _f64p, _f64p]
        lib.oracle_cp_reorder.restype = ctypes.c_int
        lib.oracle_cp_reorder.argtypes = [_u8p, _u8p, ctypes.c_int64, _i64p, ctypes.c_int64,
                                          ctypes.c_int64, _i64p, _i32p]
        lib.oracle_cp_restore.restype = ctypes.c_int
        lib.oracle_cp_restore.argtypes = [_u8p, _u8p, ctypes.c_int64, _i64p, ctypes.c_int64,
                                          ctypes.c_int64]
        lib.oracle_cp_rank_pairs.restype = ctypes.c_int
        lib.oracle_cp_rank_pairs.argtypes = [_i64p, ctypes.c_int64, ctypes.c_int64, _i64p]
        lib.oracle_paired_fwd.restype = ctypes.c_int
        lib.oracle_paired_fwd.argtypes = [_f64p, _f64p, _f64p, _i64p, _i64p, ctypes.c_int64,
                                          ctypes.c_int64, _f64p, ctypes.c_int64, _f64p,
                                          ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                          ctypes.c_double, _f64p]
        _lib = lib
        return lib


def _p(a: np.ndarray, ptype):
    return a.ctypes.data_as(ptype)


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


def _i64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.int64)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact bf16 -> double widening (bf16 bits given as uint16)."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def set_threads(n: int) -> None:
    _load().oracle_set_threads(int(n))


def get_threads() -> int:
    return int(_load().oracle_get_threads())


def bucket(dt: int, NB: int) -> int:
    return int(_load().oracle_bucket(int(dt), int(NB)))


def bucket_of(t_q: int, t_k: int, NB: int) -> int:
    return int(_load().oracle_bucket_of(int(t_q), int(t_k), int(NB)))


def bucket_of_many(t_q, t_k, NB: int) -> np.ndarray:
    """bucket_of for arrays of (t_q, t_k) pairs (same function, one C loop)."""
    t_q, t_k = _i64(t_q), _i64(t_k)
    assert t_q.shape == t_k.shape
    out = np.empty(t_q.shape[0], np.int64)
    _load().oracle_bucket_of_many(_p(t_q, _i64p), _p(t_k, _i64p), t_q.shape[0], int(NB),
                                  _p(out, _i64p))
    return out


def _common(q, k, v, offsets, ts, w_pos, w_ts, H, d, scale):
    q, k, v = _f64(q), _f64(k), _f64(v)
    offsets, ts = _i64(offsets), _i64(ts)
    w_pos, w_ts = _f64(w_pos), _f64(w_ts)
    B = offsets.shape[0] - 1
    keep = (q, k, v, offsets, ts, w_pos, w_ts)
    args = [_p(q, _f64p), _p(k, _f64p), _p(v, _f64p), _p(offsets, _i64p), B, _p(ts, _i64p),
            _p(w_pos, _f64p), w_pos.shape[0], _p(w_ts, _f64p), w_ts.shape[0], int(H), int(d),
            float(scale)]
    return keep, args


def fwd(q, k, v, offsets, ts, w_pos, w_ts, H, d, scale) -> np.ndarray:
    """O [T, H, d] in float64; q/k/v given as float arrays [T, H, d]."""
    T = int(np.asarray(offsets)[-1])
    out = np.zeros((T, H, d), np.float64)
    keep, args = _common(q, k, v, offsets, ts, w_pos, w_ts, H, d, scale)
    _load().oracle_fwd(*args, _p(out, _f64p))
    return out


def fwd_rows(q, k, v, offsets, ts, w_pos, w_ts, H, d, scale, tok, head) -> np.ndarray:
    tok, head = _i64(tok), _i64(head)
    out = np.zeros((tok.shape[0], d), np.float64)
    keep, args = _common(q, k, v, offsets, ts, w_pos, w_ts, H, d, scale)
    _load().oracle_fwd_rows(*args, _p(tok, _i64p), _p(head, _i64p), tok.shape[0],
                            _p(out, _f64p))
    return out


def bwd(q, k, v, offsets, ts, w_pos, w_ts, H, d, scale, dout):
    """(dq, dk, dv, dw_pos, dw_ts) in float64."""
    T = int(np.asarray(offsets)[-1])
    dout = _f64(dout)
    dq = np.zeros((T, H, d)); dk = np.zeros((T, H, d)); dv = np.zeros((T, H, d))
    dw_pos = np.zeros(np.asarray(w_pos).shape[0]); dw_ts = np.zeros(np.asarray(w_ts).shape[0])
    keep, args = _common(q, k, v, offsets, ts, w_pos, w_ts, H, d, scale)
    _load().oracle_bwd(*args, _p(dout, _f64p), _p(dq, _f64p), _p(dk, _f64p), _p(dv, _f64p),
                       _p(dw_pos, _f64p), _p(dw_ts, _f64p))
    return dq, dk, dv, dw_pos, dw_ts


def bwd_rows(q, k, v, offsets, ts, w_pos, w_ts, H, d, scale, dout, tok, head):
    """(dq_rows, dk_rows, dv_rows) [n, d] for the listed (token, head) rows."""
    tok, head = _i64(tok), _i64(head)
    n = tok.shape[0]
    dout = _f64(dout)
    dq = np.zeros((n, d)); dk = np.zeros((n, d)); dv = np.zeros((n, d))
    keep, args = _common(q, k, v, offsets, ts, w_pos, w_ts, H, d, scale)
    _load().oracle_bwd_rows(*args, _p(dout, _f64p), _p(tok, _i64p), _p(head, _i64p), n,
                            _p(dq, _f64p), _p(dk, _f64p), _p(dv, _f64p))
    return dq, dk, dv


def _targets_split(offsets, num_targets):
    offsets = _i64(offsets)
    nt = _i64(num_targets)
    L = offsets[1:] - offsets[:-1]
    if nt.shape[0] != L.shape[0] or np.any(nt < 0) or np.any(nt > L):
        raise ValueError("num_targets must hold one value in [0, L_b] per sequence")
    return offsets, L - nt


def fwd_targets_rows(q, k, v, offsets, ts, w_pos, w_ts, H, d, scale, num_targets, tok,
                     head) -> np.ndarray:
    """Rows [n, d] of the target-aware forward for the listed (token, head) pairs.

    A history row (position < L_h = L_b - num_targets[b]) attends causally
    and only to history keys, so it is the plain causal row.  A candidate row
    is the last row of a separate pass over the sequence made of the history
    rows of its sequence followed by the candidate row alone (M-FALCON,
    "Actions Speak Louder than Words", App. H): it sits at position L_h,
    attends every history key j at relative position L_h - j and itself at
    relative position 0, with its own timestamp."""
    q, k, v, ts = _f64(q), _f64(k), _f64(v), _i64(ts)
    offsets, lh = _targets_split(offsets, num_targets)
    tok, head = _i64(tok), _i64(head)
    out = np.zeros((tok.shape[0], d), np.float64)
    seq = np.searchsorted(offsets, tok, side="right") - 1
    is_hist = (tok - offsets[seq]) < lh[seq]
    if np.any(is_hist):
        out[is_hist] = fwd_rows(q, k, v, offsets, ts, w_pos, w_ts, H, d, scale, tok[is_hist],
                                head[is_hist])
    for n in np.nonzero(~is_hist)[0]:
        b, h, t = int(seq[n]), int(head[n]), int(tok[n])
        rows = np.concatenate([np.arange(offsets[b], offsets[b] + lh[b]), [t]])
        one = lambda a: np.ascontiguousarray(a[rows][:, h:h + 1, :])
        pass_off = np.array([0, rows.shape[0]], np.int64)
        out[n] = fwd_rows(one(q), one(k), one(v), pass_off, ts[rows], w_pos, w_ts, 1, d, scale,
                          [rows.shape[0] - 1], [0])[0]
    return out


def fwd_targets(q, k, v, offsets, ts, w_pos, w_ts, H, d, scale, num_targets) -> np.ndarray:
    """O [T, H, d] in float64 of the target-aware forward (see fwd_targets_rows)."""
    offsets, lh = _targets_split(offsets, num_targets)
    out = fwd(q, k, v, offsets, ts, w_pos, w_ts, H, d, scale)  # history rows are causal rows
    cand = np.concatenate([np.arange(offsets[b] + lh[b], offsets[b + 1])
                           for b in range(offsets.shape[0] - 1)] + [np.zeros(0, np.int64)])
    if cand.shape[0]:
        tok = np.repeat(cand, H)
        head = np.tile(np.arange(H), cand.shape[0])
        out[tok, head] = fwd_targets_rows(q, k, v, offsets, ts, w_pos, w_ts, H, d, scale,
                                          num_targets, tok, head)
    return out


class OracleError(RuntimeError):
    def __init__(self, code: int):
        super().__init__(f"oracle returned status {code}")
        self.code = code


def cp_reorder(src: np.ndarray, offsets, C: int) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Paired layout of ``src`` (rows along axis 0). Returns (dst, dst_offsets, global_pos)."""
    src = np.ascontiguousarray(src)
    offsets = _i64(offsets)
    B = offsets.shape[0] - 1
    T = src.shape[0]
    row_bytes = src.nbytes // T if T else src.itemsize * int(np.prod(src.shape[1:]))
    dst = np.empty_like(src)
    dst_offsets = np.zeros(C * B + 1, np.int64)
    gpos = np.zeros(T, np.int32)
    st = _load().oracle_cp_reorder(src.view(np.uint8).ctypes.data_as(_u8p),
                                   dst.view(np.uint8).ctypes.data_as(_u8p), row_bytes,
                                   _p(offsets, _i64p), B, int(C), _p(dst_offsets, _i64p),
                                   _p(gpos, _i32p))
    if st != 0:
        raise OracleError(st)
    return dst, dst_offsets, gpos


def cp_restore(src: np.ndarray, offsets, C: int) -> np.ndarray:
    src = np.ascontiguousarray(src)
    offsets = _i64(offsets)
    B = offsets.shape[0] - 1
    T = src.shape[0]
    row_bytes = src.nbytes // T if T else src.itemsize * int(np.prod(src.shape[1:]))
    dst = np.empty_like(src)
    st = _load().oracle_cp_restore(src.view(np.uint8).ctypes.data_as(_u8p),
                                   dst.view(np.uint8).ctypes.data_as(_u8p), row_bytes,
                                   _p(offsets, _i64p), B, int(C))
    if st != 0:
        raise OracleError(st)
    return dst


def cp_rank_pairs(offsets, C: int) -> np.ndarray:
    offsets = _i64(offsets)
    counts = np.zeros(C, np.int64)
    st = _load().oracle_cp_rank_pairs(_p(offsets, _i64p), offsets.shape[0] - 1, int(C),
                                      _p(counts, _i64p))
    if st != 0:
        raise OracleError(st)
    return counts


def paired_fwd(pq, pk, pv, pts, offsets, C, w_pos, w_ts, H, d, scale) -> np.ndarray:
    pq, pk, pv = _f64(pq), _f64(pk), _f64(pv)
    pts, offsets = _i64(pts), _i64(offsets)
    w_pos, w_ts = _f64(w_pos), _f64(w_ts)
    T = int(offsets[-1])
    out = np.zeros((T, H, d), np.float64)
    st = _load().oracle_paired_fwd(_p(pq, _f64p), _p(pk, _f64p), _p(pv, _f64p), _p(pts, _i64p),
                                   _p(offsets, _i64p), offsets.shape[0] - 1, int(C),
                                   _p(w_pos, _f64p), w_pos.shape[0], _p(w_ts, _f64p),
                                   w_ts.shape[0], int(H), int(d), float(scale),
                                   _p(out, _f64p))
    if st != 0:
        raise OracleError(st)
    return out


# ---------------------------------------------------------------------------
# convenience on a workloads.JaggedBatch
# ---------------------------------------------------------------------------

def batch_inputs(batch):
    """(q, k, v, dout) of a JaggedBatch widened exactly to float64."""
    dout = None if batch.dout is None else bf16_to_f64(batch.dout)
    return bf16_to_f64(batch.q), bf16_to_f64(batch.k), bf16_to_f64(batch.v), dout


def batch_fwd(batch) -> np.ndarray:
    q, k, v, _ = batch_inputs(batch)
    return fwd(q, k, v, batch.offsets, batch.timestamps, batch.w_pos, batch.w_ts,
               batch.num_heads, batch.d, batch.scale)


def batch_bwd(batch):
    q, k, v, dout = batch_inputs(batch)
    return bwd(q, k, v, batch.offsets, batch.timestamps, batch.w_pos, batch.w_ts,
               batch.num_heads, batch.d, batch.scale, dout)
