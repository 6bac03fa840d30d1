"""Oracle of Stochastic Length subsequence selection -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` may import this
module; the product path never does.

"Actions Speak Louder than Words" (§3.2 and §4.2) says that Stochastic Length
raises sparsity by selecting subsequences of long user histories, with a
parameter α (smaller α for longer sequences), and that at α = 1.6 length-4096
sequences become length 776 "most of the time" (4096^0.8 = 776.05).  The
pages give neither the selection rule nor the probability.  Reading taken:

* target length ``L = floor(N^(α/2))`` for maximum length ``N``;
* a sequence of length ``n <= L`` is kept whole; a longer one is replaced, with
  probability ``1 - (L / n)^2``, by ``L`` of its tokens chosen uniformly at
  random (its order kept), and kept whole otherwise, so that its expected
  quadratic attention cost is at most ``2 L^2`` (at n = N = 4096, α = 1.6 the
  probability is 0.964: "most of the time");
* the random draws are inputs: one uint32 ``u_seq[b]`` per sequence (the
  decision: subsample iff ``u_seq[b] / 2^32 < 1 - (L / n)^2``, evaluated in
  float64 as written) and one uint32 ``u_tok[t]`` per token (the ``L`` tokens
  with the smallest ``(u_tok, position)`` are kept).

Plain Python/numpy, one sequence at a time.
"""
from __future__ import annotations

import math

import numpy as np


def target_length(N: int, alpha: float) -> int:
    """L = floor(N^(alpha / 2)), at least 1."""
    if N < 1 or not (alpha > 0):
        raise ValueError("N >= 1 and alpha > 0 required")
    v = math.pow(float(N), alpha / 2.0)
    L = int(math.floor(v))
    # a power that should be an integer may land just below it
    if L + 1 <= N and abs(v - (L + 1)) < 1e-9 * v:
        L += 1
    return max(1, min(L, N))


def subsample_decision(n: int, L: int, u: int) -> bool:
    """True when a sequence of length n is cut to L tokens: n > L and
    u / 2^32 < 1 - (L / n)^2 (float64, in this order)."""
    if n <= L:
        return False
    frac = float(L) / float(n)
    thresh = 1.0 - frac * frac
    return float(u) / 4294967296.0 < thresh


def select(offsets, u_tok, u_seq, L: int):
    """(dst_offsets [B + 1], src_rows [T_out]): the rows each output sequence
    takes from the input, in order."""
    offsets = np.asarray(offsets, dtype=np.int64)
    u_tok = np.asarray(u_tok, dtype=np.uint32)
    u_seq = np.asarray(u_seq, dtype=np.uint32)
    B = offsets.shape[0] - 1
    dst = [0]
    rows = []
    for b in range(B):
        o0, o1 = int(offsets[b]), int(offsets[b + 1])
        n = o1 - o0
        if subsample_decision(n, L, int(u_seq[b])):
            # the L smallest (u, position) pairs, then back in position order
            keys = sorted(range(n), key=lambda i: (int(u_tok[o0 + i]), i))[:L]
            keep = sorted(keys)
        else:
            keep = list(range(n))
        rows.extend(o0 + i for i in keep)
        dst.append(dst[-1] + len(keep))
    return np.array(dst, dtype=np.int64), np.array(rows, dtype=np.int64)


def gather(src: np.ndarray, src_rows) -> np.ndarray:
    """Rows of src (any row shape) in the order src_rows gives."""
    return np.asarray(src)[np.asarray(src_rows, dtype=np.int64)]
