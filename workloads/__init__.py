"""Seeded synthetic jagged HSTU attention workloads.

This module only draws random inputs. It holds none of the attention
arithmetic, so both the fp64 oracle (``oracle/``) and the CUDA path
(``jagged_hstu_attention_attn_b200``) can take their inputs from it without
sharing any of the method's code.

The workloads follow the shapes the two source pages work with:

* jagged (offset-indexed) user-action sequences, "values + offsets"
  (Scaling Generative Recommendations with Context Parallelism on HSTU,
  §2.2 Jagged Tensors);
* per-token int64 timestamps and a learnable ``ts_weights`` table drawn
  from a normal distribution (same page, §2.1);
* a relative-position table (Actions Speak Louder than Words, App. F.3,
  "HSTU variants with and without relative attention bias").

Draw order per workload (one ``numpy.random.default_rng(seed)``):
lengths, timestamps, q, k, v, w_pos, w_ts, dO.  Floating point inputs are
drawn in fp32 and rounded to bf16 with round-to-nearest-even; the bf16 bits
are kept as ``uint16`` so every consumer reads the very same values.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, Optional

import numpy as np

TS_EPOCH = 1_700_000_000  # plausible unix-epoch start for every sequence


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 -> bf16 (round to nearest, ties to even); returns uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    # u + 0x7FFF + lsb cannot overflow uint32 for finite inputs below 2^128
    rounding = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return ((u + rounding) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bits to fp32."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclass
class JaggedBatch:
    """One jagged batch: every array is host (numpy) memory."""

    name: str
    lengths: np.ndarray          # int64 [B]
    offsets: np.ndarray          # int64 [B+1], offsets[0] = 0, offsets[B] = T
    timestamps: np.ndarray       # int64 [T]
    q: np.ndarray                # uint16 bf16 bits [T, H, d]
    k: np.ndarray                # uint16 bf16 bits [T, H, d]
    v: np.ndarray                # uint16 bf16 bits [T, H, d]
    w_pos: np.ndarray            # float32 [P]
    w_ts: np.ndarray             # float32 [NB]
    dout: Optional[np.ndarray]   # uint16 bf16 bits [T, H, d] or None
    num_heads: int
    d: int
    scale: float
    meta: Dict[str, object] = field(default_factory=dict)

    @property
    def B(self) -> int:
        return int(self.lengths.shape[0])

    @property
    def T(self) -> int:
        return int(self.offsets[-1])

    @property
    def P(self) -> int:
        return int(self.w_pos.shape[0])

    @property
    def NB(self) -> int:
        return int(self.w_ts.shape[0])

    def causal_pairs(self) -> int:
        """sum_b L_b (L_b + 1) / 2 (one head)."""
        L = self.lengths.astype(np.int64)
        return int(np.sum(L * (L + 1) // 2))

    def subset(self, seq_ids) -> "JaggedBatch":
        """The same batch restricted to the listed sequences (in that order)."""
        seq_ids = [int(s) for s in seq_ids]
        rows = np.concatenate([np.arange(self.offsets[s], self.offsets[s + 1]) for s in seq_ids]) \
            if seq_ids else np.zeros(0, np.int64)
        lengths = self.lengths[seq_ids].astype(np.int64)
        offsets = np.zeros(len(seq_ids) + 1, np.int64)
        offsets[1:] = np.cumsum(lengths)
        pick = lambda a: None if a is None else np.ascontiguousarray(a[rows])
        return JaggedBatch(self.name + "[subset]", lengths, offsets, pick(self.timestamps),
                           pick(self.q), pick(self.k), pick(self.v), self.w_pos.copy(),
                           self.w_ts.copy(), pick(self.dout), self.num_heads, self.d,
                           self.scale, dict(self.meta, subset=seq_ids))


    def head_subset(self, heads) -> "JaggedBatch":
        """The same batch restricted to the listed heads (in that order); the
        timestamps and bias tables are shared by all heads and stay as they are."""
        heads = [int(h) for h in heads]
        pick = lambda a: None if a is None else np.ascontiguousarray(a[:, heads, :])
        return JaggedBatch(self.name + "[heads]", self.lengths.copy(), self.offsets.copy(),
                           self.timestamps.copy(), pick(self.q), pick(self.k), pick(self.v),
                           self.w_pos.copy(), self.w_ts.copy(), pick(self.dout), len(heads),
                           self.d, self.scale, dict(self.meta, heads=heads))


def _timestamps(rng: np.random.Generator, lengths: np.ndarray, gap: str, mean: float,
                sigma: float = 0.0) -> np.ndarray:
    parts = []
    for L in lengths:
        L = int(L)
        if gap == "exp":
            g = rng.exponential(mean, size=max(L - 1, 0))
        elif gap == "lognormal":
            g = rng.lognormal(mean, sigma, size=max(L - 1, 0))
        else:
            raise ValueError(gap)
        g = np.rint(g).astype(np.int64)
        t = np.empty(L, np.int64)
        if L:
            t[0] = TS_EPOCH
            t[1:] = TS_EPOCH + np.cumsum(g)
        parts.append(t)
    return np.concatenate(parts) if parts else np.zeros(0, np.int64)


def _normal_bf16(rng: np.random.Generator, shape, std: float) -> np.ndarray:
    """N(0, std^2) drawn in fp32, rounded to bf16 bits."""
    x = rng.standard_normal(shape, dtype=np.float32)
    x *= np.float32(std)
    return f32_to_bf16_bits(x)


def make_batch(name: str, lengths: np.ndarray, rng: np.random.Generator, *, H: int, d: int,
               gap: str, gap_mean: float, gap_sigma: float = 0.0, P: int, NB: int = 128,
               qkv_std: float = 0.5, w_std: float = 0.02, with_dout: bool = True,
               scale: Optional[float] = None, meta=None) -> JaggedBatch:
    lengths = np.asarray(lengths, dtype=np.int64)
    offsets = np.zeros(len(lengths) + 1, np.int64)
    offsets[1:] = np.cumsum(lengths)
    T = int(offsets[-1])
    ts = _timestamps(rng, lengths, gap, gap_mean, gap_sigma)
    q = _normal_bf16(rng, (T, H, d), qkv_std)
    k = _normal_bf16(rng, (T, H, d), qkv_std)
    v = _normal_bf16(rng, (T, H, d), qkv_std)
    w_pos = (rng.standard_normal(P, dtype=np.float32) * np.float32(w_std)).astype(np.float32)
    w_ts = (rng.standard_normal(NB, dtype=np.float32) * np.float32(w_std)).astype(np.float32)
    dout = _normal_bf16(rng, (T, H, d), qkv_std) if with_dout else None
    if scale is None:
        scale = 1.0 / float(np.sqrt(d))
    return JaggedBatch(name, lengths, offsets, ts, q, k, v, w_pos, w_ts, dout, H, d,
                       float(scale), dict(meta or {}))


# ---------------------------------------------------------------------------
# The five workload recipes.  Sizes and distributions are the ones quoted for
# the jagged HSTU attention workloads.
# ---------------------------------------------------------------------------

def tiny(seed: int = 0, with_dout: bool = True) -> JaggedBatch:
    """B=4, L ~ U{16..128}, H=2, d=32, Exp(3600 s) gaps, P=256, NB=128."""
    rng = np.random.default_rng(seed)
    lengths = rng.integers(16, 128, size=4, endpoint=True)
    return make_batch("tiny", lengths, rng, H=2, d=32, gap="exp", gap_mean=3600.0, P=256,
                      with_dout=with_dout)


def zipf(seed: int = 1, with_dout: bool = True, B: int = 32) -> JaggedBatch:
    """B=32, L = clip(Zipf(1.2), 256, 3072), H=4, d=128, Exp(600 s) gaps, P=3072."""
    rng = np.random.default_rng(seed)
    lengths = np.clip(rng.zipf(1.2, size=B), 256, 3072)
    return make_batch("zipf", lengths, rng, H=4, d=128, gap="exp", gap_mean=600.0, P=3072,
                      with_dout=with_dout)


def fixed8192(seed: int = 2, with_dout: bool = True, B: int = 16) -> JaggedBatch:
    """B=16 sequences of length 8192 (as jagged offsets), H=8, d=64, Exp(60 s), P=3072."""
    rng = np.random.default_rng(seed)
    lengths = np.full(B, 8192, np.int64)
    return make_batch("fixed8192", lengths, rng, H=8, d=64, gap="exp", gap_mean=60.0, P=3072,
                      with_dout=with_dout)


def long_hist(seed: int = 3, with_dout: bool = True, B: int = 8) -> JaggedBatch:
    """B=8, L ~ U{4096..16384}, H=4, d=128, LogNormal(6, 2) s gaps, P=3072."""
    rng = np.random.default_rng(seed)
    lengths = rng.integers(4096, 16384, size=B, endpoint=True)
    return make_batch("long", lengths, rng, H=4, d=128, gap="lognormal", gap_mean=6.0,
                      gap_sigma=2.0, P=3072, with_dout=with_dout)


def paired(C: int, seed: int = 4, with_dout: bool = False, B: int = 64) -> JaggedBatch:
    """B=64, L ~ U{1024..16384} rounded up to a multiple of 2C, H=4, d=128, Exp(600 s)."""
    if C < 1:
        raise ValueError("C must be >= 1")
    rng = np.random.default_rng(seed)
    lengths = rng.integers(1024, 16384, size=B, endpoint=True)
    lengths = ((lengths + 2 * C - 1) // (2 * C)) * (2 * C)
    return make_batch(f"paired_C{C}", lengths, rng, H=4, d=128, gap="exp", gap_mean=600.0,
                      P=3072, with_dout=with_dout, meta={"C": C})


WORKLOADS = {
    "tiny": tiny,
    "zipf": zipf,
    "fixed8192": fixed8192,
    "long": long_hist,
}


def with_candidates(batch: JaggedBatch, num_targets: np.ndarray) -> JaggedBatch:
    """Mark the last num_targets[b] rows of each sequence as ranking candidates
    (M-FALCON, Actions Speak Louder than Words, App. H): they are scored at one
    request time, so each takes the timestamp the draw gave its sequence's
    first candidate row.  The counts go to meta["num_targets"]."""
    nt = np.asarray(num_targets, np.int64)
    assert nt.shape[0] == batch.B and np.all(nt >= 0) and np.all(nt <= batch.lengths)
    ts = batch.timestamps.copy()
    for b in range(batch.B):
        s, e = int(batch.offsets[b]), int(batch.offsets[b + 1])
        if nt[b] > 0:
            ts[e - nt[b]:e] = ts[e - nt[b]]
    batch.timestamps = ts
    batch.meta["num_targets"] = nt
    return batch


def mfalcon(seed: int = 6, with_dout: bool = False, B: int = 16, b_m: int = 1024) -> JaggedBatch:
    """B=16 users, history L_h ~ U{1024..3072}, a microbatch of b_m = 1024
    candidates per user after it, H=4, d=128, Exp(600 s) gaps, P=3072."""
    rng = np.random.default_rng(seed)
    hist = rng.integers(1024, 3072, size=B, endpoint=True)
    batch = make_batch("mfalcon", hist + b_m, rng, H=4, d=128, gap="exp", gap_mean=600.0,
                       P=3072, with_dout=with_dout)
    return with_candidates(batch, np.full(B, b_m, np.int64))


def random_small(seed: int, B: int, Lmin: int, Lmax: int, H: int, d: int, P: int = 64,
                 NB: int = 128, gap_mean: float = 100.0, with_dout: bool = True,
                 pad_to: int = 1) -> JaggedBatch:
    """Small random jagged batch for parity and edge cases (lengths may be 0)."""
    rng = np.random.default_rng(seed)
    lengths = rng.integers(Lmin, Lmax, size=B, endpoint=True)
    if pad_to > 1:
        lengths = ((lengths + pad_to - 1) // pad_to) * pad_to
    return make_batch(f"small{seed}", lengths, rng, H=H, d=d, gap="exp", gap_mean=gap_mean, P=P,
                      NB=NB, with_dout=with_dout)


@dataclass
class NormGateInputs:
    """Inputs of the post-attention norm gate, bf16 bits as uint16 [T, N]."""
    o: np.ndarray    # attention output of each token (all heads together)
    u: np.ndarray    # the gate U(X) from the pointwise projection
    dy: np.ndarray   # output gradient

    @property
    def T(self) -> int:
        return int(self.o.shape[0])

    @property
    def N(self) -> int:
        return int(self.o.shape[1])


def norm_gate_inputs(T: int, N: int, seed: int = 7) -> NormGateInputs:
    """Seeded [T, N] rows for the norm gate.  Draw order: per-row offset
    ~ N(0, 2), per-row spread ~ U(0.25, 8), o = offset + spread * N(0, 1),
    u ~ N(0, 1), dy ~ N(0, 1).  The offsets and spreads make rows whose mean
    is far from zero relative to their spread, as attention outputs summed
    over thousands of keys are."""
    rng = np.random.default_rng(seed)
    off = rng.normal(0.0, 2.0, size=(T, 1)).astype(np.float32)
    spread = rng.uniform(0.25, 8.0, size=(T, 1)).astype(np.float32)
    o = off + spread * rng.standard_normal((T, N), dtype=np.float32)
    u = rng.standard_normal((T, N), dtype=np.float32)
    dy = rng.standard_normal((T, N), dtype=np.float32)
    return NormGateInputs(f32_to_bf16_bits(o), f32_to_bf16_bits(u), f32_to_bf16_bits(dy))



def sl_draws(T: int, B: int, seed: int = 9, tie_range: int = 0):
    """Stochastic Length random draws: (u_tok uint32 [T], u_seq uint32 [B]).
    With tie_range > 0 the token draws come from [0, tie_range), so equal keys
    are common (the selection then orders them by position)."""
    rng = np.random.default_rng(seed)
    hi = tie_range if tie_range > 0 else (1 << 32)
    u_tok = rng.integers(0, hi, size=T, dtype=np.uint64).astype(np.uint32)
    u_seq = rng.integers(0, 1 << 32, size=B, dtype=np.uint64).astype(np.uint32)
    return u_tok, u_seq
