"""GPU parity of Stochastic Length selection and the row gather against the
oracle ("Actions Speak Louder than Words" §3.2, §4.2), bit for bit."""
import numpy as np
import pytest

import workloads
from oracle import stochastic_length as sl

pytestmark = pytest.mark.gpu


def _dev_u32(a):
    import torch
    return torch.from_numpy(np.asarray(a, np.uint32).view(np.int32).copy()).cuda()


def _select(offsets, u_tok, u_seq, L, status=None):
    import torch
    import jagged_hstu_attention_attn_b200 as hstu
    off = torch.from_numpy(np.asarray(offsets, np.int64).copy()).cuda()
    dst, rows = hstu.hstu_sl_select(off, _dev_u32(u_tok), _dev_u32(u_seq), L, dev_status=status)
    torch.cuda.synchronize()
    return dst.cpu().numpy(), rows.cpu().numpy().astype(np.int64)


def _check(offsets, u_tok, u_seq, L):
    dst, rows = _select(offsets, u_tok, u_seq, L)
    ref_dst, ref_rows = sl.select(offsets, u_tok, u_seq, L)
    assert np.array_equal(dst, ref_dst)
    assert np.array_equal(rows[:ref_dst[-1]], ref_rows)
    return ref_dst


CASES = [
    # seed, B, Lmin, Lmax, L, tie_range
    (1, 12, 0, 300, 40, 0),
    (2, 9, 0, 300, 40, 64),          # many equal keys
    (3, 5, 100, 101, 100, 0),        # lengths L and L + 1
    (4, 7, 1, 5000, 777, 1000),
    (5, 3, 0, 2, 1, 2),              # L = 1, tiny sequences
]


@pytest.mark.parametrize("case", CASES)
def test_selection_matches_oracle(case):
    seed, B, lo, hi, L, tie = case
    rng = np.random.default_rng(seed)
    lengths = rng.integers(lo, hi, size=B, endpoint=True)
    offsets = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    u_tok, u_seq = workloads.sl_draws(int(offsets[-1]), B, seed, tie)
    # force some sequences through both branches
    u_seq[::3] = 0
    u_seq[1::3] = np.uint32(0xFFFFFFFF)
    _check(offsets, u_tok, u_seq, L)


def test_full_size_fixed8192_alpha_1_6():
    """16 sequences of 8192 (the headline workload's batch), alpha = 1.6:
    L = floor(8192^0.8) = 1351."""
    import jagged_hstu_attention_attn_b200 as hstu
    L = hstu.sl_target_length(8192, 1.6)
    assert L == sl.target_length(8192, 1.6) == 1351
    offsets = np.arange(17, dtype=np.int64) * 8192
    u_tok, u_seq = workloads.sl_draws(int(offsets[-1]), 16, 11)
    dst = _check(offsets, u_tok, u_seq, L)
    assert dst[-1] < offsets[-1]


def test_gather_matches_numpy():
    import torch
    import jagged_hstu_attention_attn_b200 as hstu
    batch = workloads.random_small(8, 6, 0, 700, 2, 64, P=64)
    u_tok, u_seq = workloads.sl_draws(batch.T, batch.B, 8)
    u_seq[:] = 0
    L = 200
    off = torch.from_numpy(batch.offsets.copy()).cuda()
    dst, rows = hstu.hstu_sl_select(off, _dev_u32(u_tok), _dev_u32(u_seq), L)
    n = dst[-1:]
    q = torch.from_numpy(batch.q.view(np.int16).copy()).cuda()
    ts = torch.from_numpy(batch.timestamps.copy()).cuda()
    gq = hstu.hstu_gather_rows(q, rows, n)
    gts = hstu.hstu_gather_rows(ts, rows, n)
    torch.cuda.synchronize()
    ref_dst, ref_rows = sl.select(batch.offsets, u_tok, u_seq, L)
    m = int(ref_dst[-1])
    assert np.array_equal(gq.cpu().numpy()[:m], sl.gather(batch.q.view(np.int16), ref_rows))
    assert np.array_equal(gts.cpu().numpy()[:m], sl.gather(batch.timestamps, ref_rows))


def test_bad_offsets_select_nothing_and_report():
    import torch
    import jagged_hstu_attention_attn_b200 as hstu
    offsets = np.array([0, 50, 40, 100], np.int64)   # decreasing in the middle
    u_tok, u_seq = workloads.sl_draws(100, 3, 3)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    dst, rows = _select(offsets, u_tok, u_seq, 10, status=st)
    assert int(st.item()) == -5   # HSTU_ERR_OFFSETS
    # the bad sequence (offsets 50 -> 40) contributes no rows
    assert dst[2] - dst[1] == 0


def test_launch_counts_and_empty_batch():
    import torch
    import jagged_hstu_attention_attn_b200 as hstu
    n0 = hstu.hstu_kernel_launches()
    off = torch.zeros(1, dtype=torch.int64, device="cuda")
    dst, rows = hstu.hstu_sl_select(off, _dev_u32([]), _dev_u32([]), 5)
    torch.cuda.synchronize()
    assert dst.cpu().tolist() == [0]
    assert hstu.hstu_kernel_launches() == n0 + 1   # the offsets pass only


def test_gather_rows_multi_one_launch():
    """q (1 KB rows), timestamps (8-byte rows) and an odd 6-byte row tensor in
    one launch, bit for bit."""
    import torch
    import jagged_hstu_attention_attn_b200 as hstu
    batch = workloads.random_small(9, 5, 0, 600, 4, 128, P=64)
    u_tok, u_seq = workloads.sl_draws(batch.T, batch.B, 9)
    u_seq[::2] = 0
    off = torch.from_numpy(batch.offsets.copy()).cuda()
    dst, rows = hstu.hstu_sl_select(off, _dev_u32(u_tok), _dev_u32(u_seq), 150)
    q = torch.from_numpy(batch.q.view(np.int16).copy()).cuda()
    ts = torch.from_numpy(batch.timestamps.copy()).cuda()
    odd_np = np.random.default_rng(9).integers(0, 255, size=(batch.T, 6), dtype=np.uint8)
    odd = torch.from_numpy(odd_np).cuda()
    n0 = hstu.hstu_kernel_launches()
    gq, gts, godd = hstu.hstu_gather_rows_multi([q, ts, odd], rows, dst[-1:])
    torch.cuda.synchronize()
    assert hstu.hstu_kernel_launches() == n0 + 1
    ref_dst, ref_rows = sl.select(batch.offsets, u_tok, u_seq, 150)
    m = int(ref_dst[-1])
    assert np.array_equal(gq.cpu().numpy()[:m], sl.gather(batch.q.view(np.int16), ref_rows))
    assert np.array_equal(gts.cpu().numpy()[:m], sl.gather(batch.timestamps, ref_rows))
    assert np.array_equal(godd.cpu().numpy()[:m], sl.gather(odd_np, ref_rows))
