"""Bit-exact check of the bias indices the attention kernels themselves use,
read back through the public forward entry points.

With q = k = 0 every pre-activation is x_ij = scale * (w_pos[rel_ij] +
w_ts[bucket_ij]) (the HSTUAttention equation of "Scaling Generative
Recommendations with Context Parallelism on Hierarchical Sequential
Transducers", §2.1).  One of the two tables is set to zero and the other to
an injective, non-negative table (entry r = r / 8), so x_ij names one table
entry.  V is one-hot per key: head h carries one block of d keys, key
j = kb_h + c in feature column c, so O[i, h, c] = SiLU(x_ij) of that single
pair.  SiLU is increasing on x >= 0, so the nearest entry of SiLU(table)
recovers the index the kernel used for every pair j <= i, and it must equal
the oracle's integer bucket function (timestamp buckets) or min(i - j, P - 1)
(relative positions) exactly.  Masked pairs must give exactly 0.

The timestamp designs drive every epilogue mode: a single bucket per tile,
32-bit relative timestamps, the 64-bit path (differences beyond 2^30, up to
2^62, non-monotone rows), and differences at 2^k - 1, 2^k and 2^k + 1 for
every k.  The relative-position cases cover the clamp at P - 1, the
shared-memory table and the per-tile window used when P is larger than that
table, the target-aware (M-FALCON) candidate rows and the paired layout."""
import numpy as np
import pytest

import oracle
import workloads
from hstu_util import to_device, to_f64

pytestmark = pytest.mark.gpu

BF16_ONE = 0x3F80


def _silu(x):
    return x / (1.0 + np.exp(-x))


def _timestamps(kind, L, rng):
    if kind == "exp":
        return np.cumsum(np.concatenate([[0], rng.exponential(3000.0, L - 1)])).astype(np.int64) \
            + workloads.TS_EPOCH
    if kind == "powers":
        # t_i - t_0 runs through 2^k - 1, 2^k, 2^k + 1 for k = 1..61, then small steps
        s = sorted({0} | {2 ** k + e for k in range(1, 62) for e in (-1, 0, 1)})
        t = list(s[:L])
        while len(t) < L:
            t.append(t[-1] + int(rng.integers(0, 5)))
        return np.array(t, np.int64)
    if kind == "wild":
        t = rng.integers(-(2 ** 62), 2 ** 62, L).astype(np.int64)
        t[:10] = [0, 2 ** 62, -(2 ** 62), 5, 5, 4, 3, 2 ** 40, -1, 0]
        return t
    if kind == "const":
        return np.full(L, 1_700_000_000, np.int64)
    if kind == "jump":
        # small monotone steps with one jump of 2^31 in the middle
        g = rng.integers(0, 3, L).astype(np.int64)
        g[0] = 0
        g[L // 2] = 2 ** 31
        return np.cumsum(g) + 12345
    raise ValueError(kind)


def _probe_batch(lengths, ts, d, key_blocks, w_pos, w_ts, name="probe"):
    """q = k = 0, V one-hot: head h carries keys key_blocks[h] .. + d - 1 of
    every sequence in its feature columns 0 .. d - 1."""
    lengths = np.asarray(lengths, np.int64)
    offsets = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    T, H = int(offsets[-1]), len(key_blocks)
    z = np.zeros((T, H, d), np.uint16)
    v = np.zeros((T, H, d), np.uint16)
    for b in range(len(lengths)):
        o, L = int(offsets[b]), int(lengths[b])
        for h, kb in enumerate(key_blocks):
            for c in range(d):
                if kb + c < L:
                    v[o + kb + c, h, c] = BF16_ONE
    return workloads.JaggedBatch(name, lengths, offsets, np.asarray(ts, np.int64), z, z.copy(),
                                 v, np.asarray(w_pos, np.float32), np.asarray(w_ts, np.float32),
                                 None, H, d, 1.0)


def _decode(batch, out, table, allowed, expected):
    """For every sequence b, head h and key column c: the pairs j <= i that
    `allowed` keeps must decode to expected(b, i, j) through SiLU(table);
    the others must be exactly 0."""
    out = np.asarray(out, np.float64)
    tv = _silu(np.asarray(table, np.float64))
    assert np.all(np.diff(tv) > 0)
    mids = 0.5 * (tv[1:] + tv[:-1])
    checked = 0
    for b in range(batch.B):
        o, L = int(batch.offsets[b]), int(batch.lengths[b])
        if L == 0:
            continue
        i = np.arange(L)[:, None]
        for h, kb in enumerate(batch.meta["key_blocks"]):
            j = kb + np.arange(batch.d)[None, :]
            blk = out[o:o + L, h, :]
            inseq = np.broadcast_to(j < L, blk.shape)
            keep = allowed(b, i, j) & inseq
            assert np.all(blk[~keep & inseq] == 0.0), f"seq {b} head {h}: masked pair not 0"
            ii, cc = np.nonzero(keep)
            if ii.size == 0:
                continue
            got = blk[ii, cc]
            idx = np.searchsorted(mids, got)
            assert np.all(np.abs(got - tv[idx]) <= 1e-3 * np.maximum(1.0, tv[idx])), \
                f"seq {b} head {h}: an output is not a table value"
            want = expected(b, ii, kb + cc)
            bad = np.nonzero(idx != want)[0]
            assert bad.size == 0, (
                f"seq {b} head {h}: pair (i={ii[bad[0]]}, j={kb + cc[bad[0]]}) index "
                f"{idx[bad[0]]} != {want[bad[0]]} ({bad.size} mismatches)")
            checked += ii.size
    return checked


def _fwd(batch, *, targets=None, paired_C=None):
    import torch
    import jagged_hstu_attention_attn_b200 as hstu
    d = to_device(batch)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    ml = int(batch.lengths.max())
    if targets is not None:
        nt = torch.from_numpy(np.asarray(targets, np.int64)).cuda()
        out = hstu.hstu_jagged_attn_fwd_targets(d["q"], d["k"], d["v"], d["offsets"], nt,
                                                d["ts"], d["w_pos"], d["w_ts"], scale=1.0,
                                                max_seq_len=ml, out_fp32=True, dev_status=st)
    elif paired_C is not None:
        C, off = paired_C, d["offsets"]
        pq, _, _ = hstu.hstu_cp_reorder(d["q"], off, C, want_maps=False, dev_status=st)
        pk, _, _ = hstu.hstu_cp_reorder(d["k"], off, C, want_maps=False, dev_status=st)
        pv, _, _ = hstu.hstu_cp_reorder(d["v"], off, C, want_maps=False, dev_status=st)
        pts, _, _ = hstu.hstu_cp_reorder(d["ts"], off, C, want_maps=False, dev_status=st)
        pout = hstu.hstu_cp_paired_attn_fwd(pq, pk, pv, off, pts, C, d["w_pos"], d["w_ts"],
                                            scale=1.0, max_seq_len=ml, out_fp32=True,
                                            dev_status=st)
        out = hstu.hstu_cp_restore(pout, off, C, dev_status=st)
    else:
        out = hstu.hstu_jagged_attn_fwd(d["q"], d["k"], d["v"], d["offsets"], d["ts"],
                                        d["w_pos"], d["w_ts"], scale=1.0, max_seq_len=ml,
                                        out_fp32=True, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return to_f64(out)


def _causal(b, i, j):
    return j <= i


def _bucket_expect(batch):
    ts, off, NB = batch.timestamps, batch.offsets, batch.NB

    def expected(b, i, j):
        o = int(off[b])
        return np.array([oracle.bucket_of(int(ts[o + a]), int(ts[o + c]), NB)
                         for a, c in zip(i, j)], np.int64)
    return expected


def _blocks(d, L):
    """Key blocks of d keys covering 0 .. L - 1."""
    return list(range(0, L, d))


# ------------------------------------------------------------------ timestamp buckets

KINDS = ["exp", "powers", "wild", "const", "jump"]


@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("NB", [128, 20])
def test_timestamp_buckets_bit_exact(d, NB):
    rng = np.random.default_rng(100 + d + NB)
    Lmax = 512   # H = Lmax / d heads
    lengths = [Lmax, 182 + 60, 300, 257, Lmax - 3, 129, 1]
    kinds = ["exp", "powers", "wild", "const", "jump", "exp", "exp"]
    ts = np.concatenate([_timestamps(k, L, rng) for k, L in zip(kinds, lengths)])
    w_ts = np.arange(NB, dtype=np.float32) / 8
    batch = _probe_batch(lengths, ts, d, _blocks(d, Lmax), np.zeros(8, np.float32), w_ts)
    batch.meta["key_blocks"] = _blocks(d, Lmax)
    out = _fwd(batch)
    n = _decode(batch, out, w_ts, _causal, _bucket_expect(batch))
    assert n == batch.causal_pairs()


def test_timestamp_buckets_bit_exact_candidates():
    """Target-aware forward: candidates attend the history and themselves
    (bucket 0); history rows are causal."""
    rng = np.random.default_rng(7)
    d, Lmax = 128, 512
    lengths = [512, 300, 260]
    nt = [200, 300, 7]
    kinds = ["exp", "wild", "powers"]
    ts = np.concatenate([_timestamps(k, L, rng) for k, L in zip(kinds, lengths)])
    w_ts = np.arange(128, dtype=np.float32) / 8
    batch = _probe_batch(lengths, ts, d, _blocks(d, Lmax), np.zeros(8, np.float32), w_ts)
    batch.meta["key_blocks"] = _blocks(d, Lmax)
    lh = np.asarray(lengths) - np.asarray(nt)

    def allowed(b, i, j):
        return (j <= i) & ((i < lh[b]) | (j < lh[b]) | (j == i))

    out = _fwd(batch, targets=nt)
    _decode(batch, out, w_ts, allowed, _bucket_expect(batch))


@pytest.mark.parametrize("C", [2, 4])
def test_timestamp_buckets_bit_exact_paired(C):
    rng = np.random.default_rng(20 + C)
    d, Lmax = 128, 512
    lengths = [512, 248, 296, 2 * C]
    kinds = ["exp", "powers", "wild", "exp"]
    ts = np.concatenate([_timestamps(k, L, rng) for k, L in zip(kinds, lengths)])
    w_ts = np.arange(128, dtype=np.float32) / 8
    batch = _probe_batch(lengths, ts, d, _blocks(d, Lmax), np.zeros(8, np.float32), w_ts)
    batch.meta["key_blocks"] = _blocks(d, Lmax)
    out = _fwd(batch, paired_C=C)
    _decode(batch, out, w_ts, _causal, _bucket_expect(batch))


# ------------------------------------------------------------------ relative positions

def _rel_expect(P, lh=None):
    def expected(b, i, j):
        pos = i if lh is None else np.minimum(i, lh[b])
        return np.minimum(pos - j, P - 1)
    return expected


@pytest.mark.parametrize("d,P", [(128, 200), (128, 3072), (64, 300), (32, 100)])
def test_relative_positions_bit_exact(d, P):
    """Shared-memory w_pos table; P below the sequence lengths exercises the
    clamp at P - 1 and the rows whose whole tile is clamped."""
    rng = np.random.default_rng(P + d)
    Lmax = 512
    lengths = [Lmax, 130, 1, Lmax - 1]
    ts = np.concatenate([_timestamps("exp", L, rng) for L in lengths])
    w_pos = np.arange(P, dtype=np.float32) / 8
    batch = _probe_batch(lengths, ts, d, _blocks(d, Lmax), w_pos, np.zeros(128, np.float32))
    batch.meta["key_blocks"] = _blocks(d, Lmax)
    out = _fwd(batch)
    n = _decode(batch, out, w_pos, _causal, _rel_expect(P))
    assert n == batch.causal_pairs()


@pytest.mark.parametrize("d,P,blocks", [
    (128, 5000, [0, 128, 2560, 5120]),             # per-tile windows (P > 3328 at d = 128)
    (64, 4100, [0, 64, 128, 2560, 4096, 5184]),    # per-tile windows (P > 4096 at d = 64)
])
def test_relative_positions_window_path_bit_exact(d, P, blocks):
    """P larger than the shared-memory table: the kernel builds a window of
    w_pos per key tile.  Sequences of 5300 rows reach relative positions past
    P - 1; the heads carry key blocks near the start, the middle and the end."""
    rng = np.random.default_rng(P)
    lengths = [5300, 4300]
    ts = np.concatenate([_timestamps("exp", L, rng) for L in lengths])
    w_pos = np.arange(P, dtype=np.float32) / 8
    batch = _probe_batch(lengths, ts, d, blocks, w_pos, np.zeros(128, np.float32))
    batch.meta["key_blocks"] = blocks
    out = _fwd(batch)
    _decode(batch, out, w_pos, _causal, _rel_expect(P))


@pytest.mark.parametrize("C", [2, 8])
def test_relative_positions_window_path_paired(C):
    d, P = 128, 5000
    rng = np.random.default_rng(50 + C)
    lengths = [5296, 4304]
    blocks = [0, 2560, 3968, 5120]
    ts = np.concatenate([_timestamps("exp", L, rng) for L in lengths])
    w_pos = np.arange(P, dtype=np.float32) / 8
    batch = _probe_batch(lengths, ts, d, blocks, w_pos, np.zeros(128, np.float32))
    batch.meta["key_blocks"] = blocks
    out = _fwd(batch, paired_C=C)
    _decode(batch, out, w_pos, _causal, _rel_expect(P))


@pytest.mark.parametrize("P", [200, 3072])
def test_relative_positions_bit_exact_candidates(P):
    """Candidate rows sit at position L_h: history key j at min(L_h - j,
    P - 1), the candidate itself at 0."""
    rng = np.random.default_rng(P + 1)
    d, Lmax = 128, 512
    lengths = [512, 400, 300]
    nt = [100, 400, 1]
    ts = np.concatenate([_timestamps("exp", L, rng) for L in lengths])
    w_pos = np.arange(P, dtype=np.float32) / 8
    batch = _probe_batch(lengths, ts, d, _blocks(d, Lmax), w_pos, np.zeros(128, np.float32))
    batch.meta["key_blocks"] = _blocks(d, Lmax)
    lh = np.asarray(lengths) - np.asarray(nt)

    def allowed(b, i, j):
        return (j <= i) & ((i < lh[b]) | (j < lh[b]) | (j == i))

    def expected(b, i, j):
        cand = i >= lh[b]
        rel = np.where(cand, np.where(j == i, 0, lh[b] - j), i - j)
        return np.minimum(rel, P - 1)

    out = _fwd(batch, targets=nt)
    _decode(batch, out, w_pos, allowed, expected)


# ------------------------------------------------------------------ backward bias gradients

def _count_batch(lengths, ts, d, H, P, NB):
    """q = k = 0 and bias tables 0, so every pre-activation is 0; v and dO
    are e_0, so every causal pair has dO_i . v_j = 1.  The backward's G for a
    pair is then dP * 2 SiLU'(0) = 1 exactly, and with scale = 1 the bias
    gradients are exact pair counts: dw[k] = H * (1/2) * #pairs with index k."""
    lengths = np.asarray(lengths, np.int64)
    offsets = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    T = int(offsets[-1])
    z = np.zeros((T, H, d), np.uint16)
    e0 = np.zeros((T, H, d), np.uint16)
    e0[:, :, 0] = BF16_ONE
    return workloads.JaggedBatch("counts", lengths, offsets, np.asarray(ts, np.int64), z,
                                 z.copy(), e0, np.zeros(P, np.float32),
                                 np.zeros(NB, np.float32), e0.copy(), H, d, 1.0)


def _expected_counts(batch):
    P, NB = batch.P, batch.NB
    cpos = np.zeros(P, np.int64)
    cts = np.zeros(NB, np.int64)
    for b in range(batch.B):
        o, L = int(batch.offsets[b]), int(batch.lengths[b])
        if L == 0:
            continue
        i, j = np.tril_indices(L)
        cpos += np.bincount(np.minimum(i - j, P - 1), minlength=P)
        bk = oracle.bucket_of_many(batch.timestamps[o + i], batch.timestamps[o + j], NB)
        cts += np.bincount(bk, minlength=NB)
    return 0.5 * batch.num_heads * cpos, 0.5 * batch.num_heads * cts


@pytest.mark.parametrize("d,P,NB", [(64, 1000, 128), (128, 700, 128), (32, 300, 20),
                                    (64, 5000, 128)])
def test_backward_bias_gradients_are_exact_pair_counts(d, P, NB):
    """dw_pos and dw_ts of the backward equal (1/2) H times the number of
    causal pairs of each clamped relative position and each timestamp bucket,
    exactly: every bucket and clamp path of the backward epilogue (one or
    two buckets per row segment, per-pair buckets, 64-bit differences,
    blocks across the clamp at P - 1, masked diagonal steps)."""
    import torch
    import jagged_hstu_attention_attn_b200 as hstu
    rng = np.random.default_rng(200 + d + P)
    lengths = [3000, 700, 600, 300, 257, 129, 1]
    kinds = ["exp", "exp", "powers", "wild", "jump", "const", "exp"]
    ts = np.concatenate([_timestamps(k, L, rng) for k, L in zip(kinds, lengths)])
    if P == 5000:   # window path of the forward's sibling: lengths beyond P - 1
        lengths = [5300, 700]
        ts = np.concatenate([_timestamps("exp", L, rng) for L in lengths])
    batch = _count_batch(lengths, ts, d, 2, P, NB)
    dv = to_device(batch)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    dq, dk, dvv, dwp, dwt = hstu.hstu_jagged_attn_bwd(
        dv["q"], dv["k"], dv["v"], dv["offsets"], dv["ts"], dv["w_pos"], dv["w_ts"], dv["dout"],
        scale=1.0, max_seq_len=int(max(lengths)), dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    want_pos, want_ts = _expected_counts(batch)
    got_pos, got_ts = to_f64(dwp), to_f64(dwt)
    bad = np.nonzero(got_pos != want_pos)[0]
    assert bad.size == 0, f"dw_pos[{bad[:5]}] = {got_pos[bad[:5]]}, want {want_pos[bad[:5]]}"
    bad = np.nonzero(got_ts != want_ts)[0]
    assert bad.size == 0, f"dw_ts[{bad[:5]}] = {got_ts[bad[:5]]}, want {want_ts[bad[:5]]}"
    # p = SiLU(0) = 0 and dS is zero away from e_0: dV, dQ, dK vanish
    for t in (dq, dk, dvv):
        assert float(t.abs().max()) == 0.0
