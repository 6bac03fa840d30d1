"""Pins for the fp64 oracle (CPU only).

Every oracle function is checked against something other than itself:
hand-worked examples (tests/golden), dense numpy / torch-autograd evaluation
of special cases, closed forms, central finite differences and the
load-balancing invariants of the mini-chunk pairing.
"""
import math
import random

import numpy as np
import pytest
import torch

import oracle
import workloads
from conftest import read_fixture


# ---------------------------------------------------------------------------
# helpers: independent routes (dense library evaluation), not the oracle loops
# ---------------------------------------------------------------------------

def dense_bias(ts, w_pos, w_ts):
    """Bias matrix of one sequence via numpy broadcasting and frexp."""
    L = ts.shape[0]
    i = np.arange(L)[:, None]
    j = np.arange(L)[None, :]
    rel = np.clip(i - j, 0, w_pos.shape[0] - 1)
    delta = (ts[:, None] - ts[None, :]).astype(np.float64)
    # frexp: x = m 2^e with m in [0.5, 1): e = bit length for positive ints < 2^53
    bl = np.where(delta > 0, np.frexp(np.where(delta > 0, delta, 1.0))[1], 0)
    bucket = np.minimum(bl, w_ts.shape[0] - 1)
    return w_pos[rel] + w_ts[bucket]


def dense_fwd(q, k, v, offsets, ts, w_pos, w_ts, H, d, scale):
    out = np.zeros_like(q)
    for b in range(len(offsets) - 1):
        s, e = offsets[b], offsets[b + 1]
        if e == s:
            continue
        bias = dense_bias(ts[s:e], w_pos, w_ts)
        for h in range(H):
            S = q[s:e, h, :] @ k[s:e, h, :].T
            X = scale * (S + bias)
            Pm = np.tril(X / (1.0 + np.exp(-X)))
            out[s:e, h, :] = Pm @ v[s:e, h, :]
    return out


def torch_autograd(q, k, v, offsets, ts, w_pos, w_ts, H, d, scale, dout):
    """Gradients through torch autograd of a dense formulation (float64)."""
    qt = torch.tensor(q, requires_grad=True)
    kt = torch.tensor(k, requires_grad=True)
    vt = torch.tensor(v, requires_grad=True)
    wp = torch.tensor(np.asarray(w_pos, np.float64), requires_grad=True)
    wt = torch.tensor(np.asarray(w_ts, np.float64), requires_grad=True)
    loss = 0.0
    P, NB = wp.shape[0], wt.shape[0]
    for b in range(len(offsets) - 1):
        s, e = int(offsets[b]), int(offsets[b + 1])
        L = e - s
        if L == 0:
            continue
        ii = torch.arange(L)[:, None]
        jj = torch.arange(L)[None, :]
        rel = (ii - jj).clamp(0, P - 1)
        tsb = [int(x) for x in ts[s:e]]
        bucket = torch.tensor([[min((max(a - c, 0)).bit_length(), NB - 1) for c in tsb]
                               for a in tsb], dtype=torch.long)
        bias = wp[rel] + wt[bucket]
        S = torch.einsum("ihc,jhc->hij", qt[s:e], kt[s:e])
        X = scale * (S + bias[None])
        Pm = torch.nn.functional.silu(X) * torch.tril(torch.ones(L, L, dtype=torch.float64))
        O = torch.einsum("hij,jhc->ihc", Pm, vt[s:e])
        loss = loss + (O * torch.tensor(dout[s:e])).sum()
    loss.backward()
    g = lambda t: t.grad.numpy() if t.grad is not None else np.zeros(t.shape)
    return g(qt), g(kt), g(vt), g(wp), g(wt)


def rand_case(seed, lengths, H, d, P, NB, gap=100.0, std=0.5):
    rng = np.random.default_rng(seed)
    lengths = np.asarray(lengths, np.int64)
    offsets = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    T = int(offsets[-1])
    ts = np.concatenate([1000 + np.cumsum(np.rint(rng.exponential(gap, L)).astype(np.int64))
                         for L in lengths]) if T else np.zeros(0, np.int64)
    q = rng.normal(0, std, (T, H, d))
    k = rng.normal(0, std, (T, H, d))
    v = rng.normal(0, std, (T, H, d))
    w_pos = rng.normal(0, 0.3, P)
    w_ts = rng.normal(0, 0.3, NB)
    dout = rng.normal(0, std, (T, H, d))
    return q, k, v, offsets, ts.astype(np.int64), w_pos, w_ts, dout


# ---------------------------------------------------------------------------
# bucket
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("dt,expect", [(0, 0), (1, 1), (2, 2), (3, 2), (4, 3), (7, 3), (8, 4),
                                       (3600, 12), (86400, 17), (-1, 0), (-86400, 0),
                                       (2**31 - 1, 31), (2**31, 32), (2**62, 63)])
def test_bucket_hand_values(dt, expect):
    assert oracle.bucket(dt, 128) == expect


def test_bucket_matches_int_bit_length():
    rnd = random.Random(7)
    vals = [0, 1, 2, 3, -1, -(2**63), 2**63 - 1]
    for kexp in range(64):
        vals += [2**kexp - 1, 2**kexp, 2**kexp + 1]
    vals += [rnd.randrange(-(2**63), 2**63) for _ in range(2000)]
    for NB in (1, 2, 4, 17, 64, 65, 128):
        for dt in vals:
            dt = max(min(dt, 2**63 - 1), -(2**63))
            assert oracle.bucket(dt, NB) == min(max(dt, 0).bit_length(), NB - 1)


def test_bucket_of_many_matches_python_bit_length():
    rnd = random.Random(11)
    tq = [rnd.randrange(-(2**63), 2**63) for _ in range(3000)] + [0, 5, 2**62, -(2**63)]
    tk = [rnd.randrange(-(2**63), 2**63) for _ in range(3000)] + [0, 4, -(2**62), 2**63 - 1]
    for NB in (1, 20, 65, 128):
        got = oracle.bucket_of_many(np.array(tq, np.int64), np.array(tk, np.int64), NB)
        want = [min(max(a - b, 0).bit_length(), NB - 1) for a, b in zip(tq, tk)]
        assert got.tolist() == want


def test_bucket_of_exact_difference():
    # differences that do not fit in int64 are still exact
    big, small = 2**63 - 1, -(2**63)
    assert oracle.bucket_of(big, small, 128) == (big - small).bit_length() == 64
    assert oracle.bucket_of(2**62, -(2**62), 128) == 64
    assert oracle.bucket_of(small, big, 128) == 0
    rnd = random.Random(3)
    for _ in range(2000):
        a = rnd.randrange(-(2**63), 2**63)
        b = rnd.randrange(-(2**63), 2**63)
        assert oracle.bucket_of(a, b, 128) == min(max(a - b, 0).bit_length(), 127)


# ---------------------------------------------------------------------------
# hand-worked 3-token example
# ---------------------------------------------------------------------------

def _hand3():
    fx = read_fixture("hand3.txt")
    f = lambda key: np.array([float(x) for x in fx[key][0]])
    q, k, v, ts = f("q"), f("k"), f("v"), f("ts").astype(np.int64)
    w_pos, w_ts, dout = f("w_pos"), f("w_ts"), f("dout")
    pairs = [[float(x) for x in row] for row in fx["pair"]]
    return q, k, v, ts, w_pos, w_ts, dout, pairs


def _silu(x):
    return x / (1.0 + math.exp(-x))


def _dsilu(x):
    s = 1.0 / (1.0 + math.exp(-x))
    return s * (1.0 + x * (1.0 - s))


def test_hand3_buckets_and_bias():
    q, k, v, ts, w_pos, w_ts, dout, pairs = _hand3()
    for (i, j, qk, rel, wp, dt, bl, bk, wt, x) in pairs:
        i, j = int(i), int(j)
        assert q[i] * k[j] == qk
        assert ts[i] - ts[j] == dt
        assert oracle.bucket(int(dt), len(w_ts)) == int(bk)
        assert oracle.bucket_of(int(ts[i]), int(ts[j]), len(w_ts)) == int(bk)
        assert min(i - j, len(w_pos) - 1) == rel and w_pos[int(rel)] == wp
        assert w_ts[int(bk)] == wt
        assert abs((qk + wp + wt) - x) < 1e-12


def test_hand3_forward_and_backward():
    q, k, v, ts, w_pos, w_ts, dout, pairs = _hand3()
    x = {(int(r[0]), int(r[1])): r[9] for r in pairs}
    bk = {(int(r[0]), int(r[1])): int(r[7]) for r in pairs}
    rel = {(int(r[0]), int(r[1])): int(r[3]) for r in pairs}
    # the worked example, written out pair by pair
    O = [sum(_silu(x[i, j]) * v[j] for j in range(i + 1)) for i in range(3)]
    g = {(i, j): dout[i] * v[j] * _dsilu(x[i, j]) for (i, j) in x}
    dQ = [sum(g[i, j] * k[j] for j in range(i + 1)) for i in range(3)]
    dK = [sum(g[i, j] * q[i] for i in range(j, 3)) for j in range(3)]
    dV = [sum(_silu(x[i, j]) * dout[i] for i in range(j, 3)) for j in range(3)]
    dwp = [sum(g[p] for p in g if rel[p] == r) for r in range(3)]
    dwt = [sum(g[p] for p in g if bk[p] == r) for r in range(4)]
    # sanity on the worked numbers themselves (a few digits, derived by hand)
    assert abs(O[0] - 0.8252861162) < 1e-9 and abs(O[1] - 6.2717652896) < 1e-9
    assert abs(O[2] - 3.0235387146) < 1e-9
    offsets = np.array([0, 3])
    sh = lambda a: np.asarray(a, np.float64).reshape(3, 1, 1)
    out = oracle.fwd(sh(q), sh(k), sh(v), offsets, ts, w_pos, w_ts, 1, 1, 1.0)
    np.testing.assert_allclose(out.ravel(), O, rtol=0, atol=1e-12)
    dq, dk, dv, dw_pos, dw_ts = oracle.bwd(sh(q), sh(k), sh(v), offsets, ts, w_pos, w_ts, 1, 1,
                                           1.0, sh(dout))
    np.testing.assert_allclose(dq.ravel(), dQ, rtol=0, atol=1e-12)
    np.testing.assert_allclose(dk.ravel(), dK, rtol=0, atol=1e-12)
    np.testing.assert_allclose(dv.ravel(), dV, rtol=0, atol=1e-12)
    np.testing.assert_allclose(dw_pos, dwp, rtol=0, atol=1e-12)
    np.testing.assert_allclose(dw_ts, dwt, rtol=0, atol=1e-12)
    assert dw_ts[2] == 0.0


# ---------------------------------------------------------------------------
# dense library evaluation of the same formula (independent route)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("seed,lengths,H,d,P,NB", [
    (0, [37], 1, 8, 64, 128),
    (1, [5, 0, 17, 1, 40], 2, 4, 8, 6),      # P and NB clamps, empty and 1-token sequences
    (2, [64, 33], 3, 16, 16, 128),
])
def test_fwd_matches_dense_numpy(seed, lengths, H, d, P, NB):
    q, k, v, off, ts, wp, wt, _ = rand_case(seed, lengths, H, d, P, NB)
    scale = 1.0 / math.sqrt(d)
    got = oracle.fwd(q, k, v, off, ts, wp, wt, H, d, scale)
    ref = dense_fwd(q, k, v, off, ts, wp, wt, H, d, scale)
    np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("seed,lengths,H,d,P,NB", [
    (3, [9, 0, 14], 2, 4, 5, 6),
    (4, [31], 1, 8, 64, 128),
])
def test_bwd_matches_torch_autograd(seed, lengths, H, d, P, NB):
    q, k, v, off, ts, wp, wt, dout = rand_case(seed, lengths, H, d, P, NB)
    scale = 0.7
    got = oracle.bwd(q, k, v, off, ts, wp, wt, H, d, scale, dout)
    ref = torch_autograd(q, k, v, off, ts, wp, wt, H, d, scale, dout)
    for a, b in zip(got, ref):
        np.testing.assert_allclose(a, b, rtol=1e-10, atol=1e-11)


def test_bwd_central_finite_differences():
    q, k, v, off, ts, wp, wt, dout = rand_case(5, [3, 5], 2, 3, 4, 5, gap=3.0)
    H, d, scale = 2, 3, 0.9
    loss = lambda q_, k_, v_, wp_, wt_: float(np.sum(
        oracle.fwd(q_, k_, v_, off, ts, wp_, wt_, H, d, scale) * dout))
    grads = oracle.bwd(q, k, v, off, ts, wp, wt, H, d, scale, dout)
    args = [q, k, v, wp, wt]
    h = 1e-6
    for which in range(5):
        base = args[which]
        fd = np.zeros_like(base)
        it = np.nditer(base, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            plus = [a.copy() for a in args]
            minus = [a.copy() for a in args]
            plus[which][idx] += h
            minus[which][idx] -= h
            fd[idx] = (loss(*plus) - loss(*minus)) / (2 * h)
        np.testing.assert_allclose(grads[which], fd, rtol=1e-6, atol=1e-8)


# ---------------------------------------------------------------------------
# closed forms
# ---------------------------------------------------------------------------

def test_single_token_sequences_closed_form():
    q, k, v, off, ts, wp, wt, _ = rand_case(6, [1, 1, 1], 2, 5, 7, 9)
    scale = 0.3
    out = oracle.fwd(q, k, v, off, ts, wp, wt, 2, 5, scale)
    for t in range(3):
        for h in range(2):
            x = scale * (float(q[t, h] @ k[t, h]) + wp[0] + wt[0])
            np.testing.assert_allclose(out[t, h], _silu(x) * v[t, h], rtol=1e-14, atol=1e-15)


def test_zero_queries_reduce_to_bias_weighted_cumsum():
    q, k, v, off, ts, wp, wt, _ = rand_case(7, [12], 1, 3, 5, 6, gap=4.0)
    q[:] = 0.0
    scale = 1.3
    out = oracle.fwd(q, k, v, off, ts, wp, wt, 1, 3, scale)
    for i in range(12):
        acc = np.zeros(3)
        for j in range(i + 1):
            bk = min(max(int(ts[i] - ts[j]), 0).bit_length(), 5)
            acc += _silu(scale * (wp[min(i - j, 4)] + wt[bk])) * v[j, 0]
        np.testing.assert_allclose(out[i, 0], acc, rtol=1e-13, atol=1e-14)


def test_one_hot_values_isolate_one_column_of_P():
    q, k, v, off, ts, wp, wt, _ = rand_case(8, [10], 1, 4, 16, 16)
    L = 10
    v = np.zeros((L, 1, 4))
    col = 6
    v[col, 0, 2] = 1.0
    scale = 0.5
    out = oracle.fwd(q, k, v, off, ts, wp, wt, 1, 4, scale)
    bias = dense_bias(ts, wp, wt)
    for i in range(L):
        expect = 0.0 if i < col else _silu(scale * (float(q[i, 0] @ k[col, 0]) + bias[i, col]))
        assert abs(out[i, 0, 2] - expect) < 1e-14
        assert np.all(out[i, 0, [0, 1, 3]] == 0.0)


def test_row_samplers_equal_full_evaluation():
    q, k, v, off, ts, wp, wt, dout = rand_case(9, [20, 0, 7, 33], 2, 6, 10, 12)
    H, d, scale = 2, 6, 0.4
    full = oracle.fwd(q, k, v, off, ts, wp, wt, H, d, scale)
    dq, dk, dv, _, _ = oracle.bwd(q, k, v, off, ts, wp, wt, H, d, scale, dout)
    tok = np.array([0, 5, 19, 20, 26, 27, 59])
    head = np.array([0, 1, 1, 0, 1, 0, 1])
    rows = oracle.fwd_rows(q, k, v, off, ts, wp, wt, H, d, scale, tok, head)
    np.testing.assert_array_equal(rows, full[tok, head])
    rq, rk, rv = oracle.bwd_rows(q, k, v, off, ts, wp, wt, H, d, scale, dout, tok, head)
    np.testing.assert_array_equal(rq, dq[tok, head])
    np.testing.assert_allclose(rk, dk[tok, head], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(rv, dv[tok, head], rtol=1e-13, atol=1e-14)


def test_bias_gradient_invariants():
    q, k, v, off, ts, wp, wt, dout = rand_case(10, [40, 25], 2, 4, 8, 128, gap=50.0)
    dq, dk, dv, dwp, dwt = oracle.bwd(q, k, v, off, ts, wp, wt, 2, 4, 0.5, dout)
    # both tables receive scale * g of every pair exactly once
    assert abs(dwp.sum() - dwt.sum()) < 1e-10 * max(1.0, abs(dwp.sum()))
    # buckets above 64 cannot be reached by int64 differences; neither can any
    # bucket above the largest difference in the batch
    maxdt = max(int(ts[e - 1] - ts[s]) for s, e in zip(off[:-1], off[1:]) if e > s)
    assert np.all(dwt[maxdt.bit_length() + 1:] == 0.0)


# ---------------------------------------------------------------------------
# mini-chunk pairing
# ---------------------------------------------------------------------------

def test_cp_reorder_hand_fixture():
    fx = read_fixture("cp_pairing_small.txt")
    ints = lambda key: np.array([int(x) for x in fx[key][0]], np.int64)
    lengths, C = ints("lengths"), int(fx["C"][0][0])
    offsets = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    src = np.arange(int(offsets[-1]), dtype=np.int64)
    dst, dst_off, gpos = oracle.cp_reorder(src, offsets, C)
    np.testing.assert_array_equal(dst, ints("src_row"))
    np.testing.assert_array_equal(dst_off, ints("dst_offsets"))
    np.testing.assert_array_equal(gpos, ints("global_pos"))
    np.testing.assert_array_equal(oracle.cp_rank_pairs(offsets, C), ints("rank_pairs"))
    np.testing.assert_array_equal(oracle.cp_restore(dst, offsets, C), src)


def test_cp_c1_is_identity():
    offsets = np.array([0, 6, 6, 10], np.int64)
    src = np.arange(10 * 3, dtype=np.float32).reshape(10, 3)
    dst, dst_off, gpos = oracle.cp_reorder(src, offsets, 1)
    np.testing.assert_array_equal(dst, src)
    np.testing.assert_array_equal(dst_off, offsets)
    np.testing.assert_array_equal(gpos, [0, 1, 2, 3, 4, 5, 0, 1, 2, 3])


@pytest.mark.parametrize("C", [1, 2, 4, 8])
def test_cp_roundtrip_and_permutation(C):
    rng = np.random.default_rng(C)
    lengths = rng.integers(0, 12, 9) * 2 * C
    offsets = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    T = int(offsets[-1])
    for row in [(2, 3), (5,), (1,)]:
        src = rng.integers(0, 2**15, size=(T,) + row).astype(np.uint16)
        dst, dst_off, gpos = oracle.cp_reorder(src, offsets, C)
        np.testing.assert_array_equal(oracle.cp_restore(dst, offsets, C), src)
    ids = np.arange(T, dtype=np.int64)
    dst, dst_off, gpos = oracle.cp_reorder(ids, offsets, C)
    assert sorted(dst.tolist()) == list(range(T))
    # every paired row sits in the sequence segment it came from
    B = len(lengths)
    for r in range(C):
        for b in range(B):
            s, e = dst_off[r * B + b], dst_off[r * B + b + 1]
            assert e - s == lengths[b] // C
            assert np.all((dst[s:e] >= offsets[b]) & (dst[s:e] < offsets[b + 1]))
            np.testing.assert_array_equal(dst[s:e] - offsets[b], gpos[s:e])


def test_cp_not_divisible_is_rejected():
    with pytest.raises(oracle.OracleError) as e:
        oracle.cp_reorder(np.arange(10, dtype=np.int64), np.array([0, 4, 10]), 2)
    assert e.value.code == -6


@pytest.mark.parametrize("C", [1, 2, 4, 8])
def test_cp_rank_pair_counts_balanced(C):
    rng = np.random.default_rng(10 + C)
    lengths = rng.integers(1, 40, 11) * 2 * C
    offsets = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    counts = oracle.cp_rank_pairs(offsets, C)
    m = lengths // (2 * C)
    per_rank = int(np.sum(m * m * (2 * C - 1) + m * (m + 1)))
    assert np.all(counts == per_rank)
    assert counts.sum() == int(np.sum(lengths * (lengths + 1) // 2))


@pytest.mark.parametrize("C", [1, 2, 4, 8])
def test_paired_equals_unsharded_bit_for_bit(C):
    rng = np.random.default_rng(20 + C)
    lengths = rng.integers(1, 6, 4) * 2 * C
    q, k, v, off, ts, wp, wt, _ = rand_case(30 + C, lengths, 2, 4, 13, 20, gap=30.0)
    H, d, scale = 2, 4, 0.5
    full = oracle.fwd(q, k, v, off, ts, wp, wt, H, d, scale)
    pq, _, _ = oracle.cp_reorder(q, off, C)
    pk, _, _ = oracle.cp_reorder(k, off, C)
    pv, _, _ = oracle.cp_reorder(v, off, C)
    pts, _, _ = oracle.cp_reorder(ts, off, C)
    pout = oracle.paired_fwd(pq, pk, pv, pts, off, C, wp, wt, H, d, scale)
    np.testing.assert_array_equal(oracle.cp_restore(pout, off, C), full)


def test_workload_generators_are_seeded_and_shaped():
    a = workloads.tiny(0)
    b = workloads.tiny(0)
    np.testing.assert_array_equal(a.q, b.q)
    np.testing.assert_array_equal(a.timestamps, b.timestamps)
    assert a.q.shape == (a.T, 2, 32) and a.P == 256 and a.NB == 128
    assert np.all(np.diff(a.offsets) >= 16) and np.all(np.diff(a.offsets) <= 128)
    for s, e in zip(a.offsets[:-1], a.offsets[1:]):
        assert np.all(np.diff(a.timestamps[s:e]) >= 0)
    p = workloads.paired(4, B=4)
    assert np.all(p.lengths % 8 == 0)
    # bf16 rounding is round-to-nearest-even
    x = np.array([1.0, 1.00390625, 1.01171875, -2.5], np.float32)
    np.testing.assert_array_equal(workloads.bf16_bits_to_f32(workloads.f32_to_bf16_bits(x)),
                                  np.array([1.0, 1.0, 1.015625, -2.5], np.float32))


# ---------------------------------------------------------------------------
# target-aware forward (M-FALCON, "Actions Speak Louder than Words", App. H)
# ---------------------------------------------------------------------------

def dense_fwd_targets(q, k, v, offsets, ts, w_pos, w_ts, H, d, scale, num_targets):
    """Independent route: the mask formulation on dense matrices.  Candidate
    rows take position L_h (where a separate pass puts them), attend history
    keys and themselves; history rows are causal."""
    out = np.zeros_like(q)
    P, NB = w_pos.shape[0], w_ts.shape[0]
    for b in range(len(offsets) - 1):
        s, e = offsets[b], offsets[b + 1]
        L = e - s
        if L == 0:
            continue
        lh = L - num_targets[b]
        i = np.arange(L)[:, None]
        j = np.arange(L)[None, :]
        pos = np.minimum(i, lh)
        rel = np.clip(pos - j, 0, P - 1)
        delta = (ts[s:e][:, None] - ts[s:e][None, :]).astype(np.float64)
        bl = np.where(delta > 0, np.frexp(np.where(delta > 0, delta, 1.0))[1], 0)
        bias = w_pos[rel] + w_ts[np.minimum(bl, NB - 1)]
        mask = (j <= i) & ((i < lh) | (j < lh) | (j == i))
        for h in range(H):
            X = scale * (q[s:e, h, :] @ k[s:e, h, :].T + bias)
            out[s:e, h, :] = (np.where(mask, X / (1.0 + np.exp(-X)), 0.0)) @ v[s:e, h, :]
    return out


@pytest.mark.parametrize("seed,lengths,targets,H,d,P,NB", [
    (20, [9, 0, 14, 1], [3, 0, 14, 1], 2, 4, 5, 6),   # all-candidate and 1-token sequences
    (21, [40, 23], [7, 1], 1, 8, 64, 128),
    (22, [33, 17, 5], [0, 16, 2], 3, 4, 3, 4),         # P and NB clamps
])
def test_fwd_targets_matches_dense_mask(seed, lengths, targets, H, d, P, NB):
    q, k, v, off, ts, wp, wt, _ = rand_case(seed, lengths, H, d, P, NB)
    got = oracle.fwd_targets(q, k, v, off, ts, wp, wt, H, d, 0.6, targets)
    ref = dense_fwd_targets(q, k, v, off, ts, wp, wt, H, d, 0.6, np.asarray(targets))
    np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-12)


def test_fwd_targets_one_candidate_is_causal():
    q, k, v, off, ts, wp, wt, _ = rand_case(23, [12, 0, 30, 1], 2, 8, 16, 32)
    got = oracle.fwd_targets(q, k, v, off, ts, wp, wt, 2, 8, 0.4, [1, 0, 1, 1])
    assert np.array_equal(got, oracle.fwd(q, k, v, off, ts, wp, wt, 2, 8, 0.4))


def test_fwd_targets_all_candidates_closed_form():
    """No history: each row attends only itself at relative position 0 and
    timestamp difference 0: O_i = SiLU(scale (q_i.k_i + w_pos[0] + w_ts[0])) v_i."""
    q, k, v, off, ts, wp, wt, _ = rand_case(24, [6, 11], 2, 4, 8, 8)
    got = oracle.fwd_targets(q, k, v, off, ts, wp, wt, 2, 4, 0.9, [6, 11])
    x = 0.9 * (np.einsum("thc,thc->th", q, k) + wp[0] + wt[0])
    np.testing.assert_allclose(got, (x / (1.0 + np.exp(-x)))[:, :, None] * v, rtol=1e-12,
                               atol=1e-13)


def test_fwd_targets_candidates_are_independent_and_permutable():
    q, k, v, off, ts, wp, wt, _ = rand_case(25, [20, 15], 2, 4, 16, 16)
    nt = [6, 4]
    base = oracle.fwd_targets(q, k, v, off, ts, wp, wt, 2, 4, 0.5, nt)
    # changing candidate 19 of sequence 0 changes its own row only
    q2, k2, v2, ts2 = q.copy(), k.copy(), v.copy(), ts.copy()
    q2[19] += 1.0; k2[19] -= 0.5; v2[19] *= 3.0; ts2[19] += 10 ** 6
    alt = oracle.fwd_targets(q2, k2, v2, off, ts2, wp, wt, 2, 4, 0.5, nt)
    changed = np.nonzero(np.any(alt != base, axis=(1, 2)))[0]
    assert changed.tolist() == [19]
    # reversing the candidates of sequence 1 reverses their outputs
    perm = np.arange(35)
    perm[31:35] = perm[31:35][::-1]
    rev = oracle.fwd_targets(q[perm], k[perm], v[perm], off, ts[perm], wp, wt, 2, 4, 0.5, nt)
    assert np.array_equal(rev, base[perm])


def test_fwd_targets_rejects_bad_counts():
    q, k, v, off, ts, wp, wt, _ = rand_case(26, [4, 3], 1, 4, 8, 8)
    with pytest.raises(ValueError):
        oracle.fwd_targets(q, k, v, off, ts, wp, wt, 1, 4, 0.5, [5, 0])
    with pytest.raises(ValueError):
        oracle.fwd_targets(q, k, v, off, ts, wp, wt, 1, 4, 0.5, [-1, 0])


def test_mfalcon_workload_shape_and_request_time():
    a = workloads.mfalcon(B=4, b_m=64)
    b = workloads.mfalcon(B=4, b_m=64)
    np.testing.assert_array_equal(a.q, b.q)
    nt = a.meta["num_targets"]
    assert nt.tolist() == [64] * 4 and a.num_heads == 4 and a.d == 128 and a.P == 3072
    lh = a.lengths - nt
    assert np.all(lh >= 1024) and np.all(lh <= 3072)
    rng = np.random.default_rng(6)
    rng.integers(1024, 3072, size=4, endpoint=True)  # the history lengths come first
    plain = workloads.make_batch("mfalcon", a.lengths, rng, H=4, d=128, gap="exp",
                                 gap_mean=600.0, P=3072, with_dout=False)
    for i, (s, e) in enumerate(zip(a.offsets[:-1], a.offsets[1:])):
        h = s + lh[i]
        # one request time for every candidate; the history is the plain draw
        assert np.all(a.timestamps[h:e] == a.timestamps[h])
        np.testing.assert_array_equal(a.timestamps[s:h], plain.timestamps[s:h])
        assert a.timestamps[h] >= a.timestamps[h - 1]
