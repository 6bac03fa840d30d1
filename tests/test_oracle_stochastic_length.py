"""Pins of the Stochastic Length selection oracle against the page's worked
number (α = 1.6 turns length-4096 sequences into length 776), a hand-worked
selection, and properties that define the selection independently of how the
oracle computes it."""
import numpy as np
import pytest

from oracle import stochastic_length as sl


def test_target_length_page_example():
    # "Actions Speak Louder than Words" §4.2: at α = 1.6, length 4096 -> 776
    assert sl.target_length(4096, 1.6) == 776
    assert sl.target_length(8192, 2.0) == 8192    # α = 2 keeps everything
    assert sl.target_length(16, 1.0) == 4         # 16^0.5, an exact power
    assert sl.target_length(1000, 0.0001) == 1


def test_hand_worked_selection():
    # one sequence of 5 tokens, L = 2, decision draw 0 (subsample, as 0 < 1 - 0.16):
    # keys (u, position) = (50,0) (10,1) (40,2) (10,3) (30,4); the two smallest
    # are (10,1) and (10,3): rows 1 and 3, in order
    dst, rows = sl.select([0, 5], [50, 10, 40, 10, 30], [0], 2)
    assert dst.tolist() == [0, 2]
    assert rows.tolist() == [1, 3]


def test_short_and_undrawn_sequences_stay_whole():
    offsets = [0, 3, 3, 10]     # lengths 3, 0, 7
    u_tok = np.arange(10, dtype=np.uint32)[::-1]
    # L = 7: no sequence is longer, nothing changes
    dst, rows = sl.select(offsets, u_tok, [0, 0, 0], 7)
    assert dst.tolist() == [0, 3, 3, 10] and rows.tolist() == list(range(10))
    # L = 6, length 7: threshold 1 - 36/49 = 0.265; a draw of 2^31 (0.5) keeps it whole
    dst, rows = sl.select(offsets, u_tok, [0, 0, 1 << 31], 6)
    assert dst.tolist() == [0, 3, 3, 10]
    # a draw of 0 cuts it to 6 tokens: the largest key (position 3, u = 6) goes
    dst, rows = sl.select(offsets, u_tok, [0, 0, 0], 6)
    assert dst.tolist() == [0, 3, 3, 9]
    assert rows.tolist() == [0, 1, 2, 4, 5, 6, 7, 8, 9]


def test_decision_boundary_in_float64():
    # n = 4, L = 2: threshold exactly 0.75 = 3221225472 / 2^32
    assert sl.subsample_decision(4, 2, 3221225471)
    assert not sl.subsample_decision(4, 2, 3221225472)
    assert not sl.subsample_decision(2, 2, 0)


@pytest.mark.parametrize("seed", [0, 1, 2, 3])
def test_selection_properties(seed):
    rng = np.random.default_rng(seed)
    lengths = rng.integers(0, 300, size=12)
    offsets = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    T = int(offsets[-1])
    u_tok = rng.integers(0, 64, size=T, dtype=np.uint32)   # many equal keys
    u_seq = rng.integers(0, 1 << 32, size=12, dtype=np.uint32)
    L = 40
    dst, rows = sl.select(offsets, u_tok, u_seq, L)
    for b in range(12):
        o0, o1 = int(offsets[b]), int(offsets[b + 1])
        n = o1 - o0
        got = rows[dst[b]:dst[b + 1]]
        cut = sl.subsample_decision(n, L, int(u_seq[b]))
        if not cut:
            assert got.tolist() == list(range(o0, o1))
            continue
        # exactly L rows of the sequence, strictly increasing
        assert got.shape[0] == L
        assert np.all(np.diff(got) > 0) and got.min() >= o0 and got.max() < o1
        # every kept token precedes every dropped one in (u, position) order
        kept = set(got.tolist())
        kmax = max((int(u_tok[r]), r) for r in kept)
        dropped = [(int(u_tok[r]), r) for r in range(o0, o1) if r not in kept]
        assert all(kmax < d for d in dropped)


def test_subsample_rate_matches_reading():
    # at n = 4096, L = 776 the reading cuts with probability 1 - (776/4096)^2 = 0.9641
    rng = np.random.default_rng(7)
    draws = rng.integers(0, 1 << 32, size=20000, dtype=np.uint64)
    rate = np.mean([sl.subsample_decision(4096, 776, int(u)) for u in draws])
    p = 1 - (776 / 4096) ** 2
    assert abs(rate - p) < 4 * np.sqrt(p * (1 - p) / draws.shape[0])


def test_gather_rows():
    src = np.arange(24, dtype=np.int64).reshape(6, 4)
    assert sl.gather(src, [5, 0, 2]).tolist() == [[20, 21, 22, 23], [0, 1, 2, 3], [8, 9, 10, 11]]
