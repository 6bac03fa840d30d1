"""GPU parity: mini-chunk pairing reorder / restore and the bucket function
are bit-exact against the oracle."""
import numpy as np
import pytest

import oracle
import workloads

pytestmark = pytest.mark.gpu


def _torch():
    import torch
    import jagged_hstu_attention_attn_b200 as hstu
    return torch, hstu


@pytest.mark.parametrize("C", [1, 2, 4, 8])
@pytest.mark.parametrize("row", [(4, 128), (2, 32), (1,), (3,)])
def test_reorder_restore_bit_exact(C, row):
    torch, hstu = _torch()
    rng = np.random.default_rng(100 + C + len(row))
    lengths = rng.integers(0, 40, 13) * 2 * C
    lengths[3] = 0
    offsets = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    T = int(offsets[-1])
    dtype = np.int16 if len(row) > 1 else np.int64 if row == (1,) else np.uint8
    src = rng.integers(-30000, 30000, size=(T,) + row).astype(dtype)
    ref, ref_off, ref_pos = oracle.cp_reorder(src, offsets, C)
    tsrc = torch.from_numpy(src).cuda()
    toff = torch.from_numpy(offsets).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    dst, dst_off, gpos = hstu.hstu_cp_reorder(tsrc, toff, C, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    np.testing.assert_array_equal(dst.cpu().numpy(), ref)
    np.testing.assert_array_equal(dst_off.cpu().numpy(), ref_off)
    np.testing.assert_array_equal(gpos.cpu().numpy(), ref_pos)
    back = hstu.hstu_cp_restore(dst, toff, C, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    np.testing.assert_array_equal(back.cpu().numpy(), src)


def test_reorder_full_size_paired_workload():
    torch, hstu = _torch()
    for C in (2, 4, 8):
        batch = workloads.paired(C, B=16)
        toff = torch.from_numpy(batch.offsets).cuda()
        q = torch.from_numpy(batch.q.view(np.int16)).cuda()
        ts = torch.from_numpy(batch.timestamps).cuda()
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        pq, poff, gpos = hstu.hstu_cp_reorder(q, toff, C, dev_status=status)
        pts, _, _ = hstu.hstu_cp_reorder(ts, toff, C, dev_status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        ref_q, ref_off, ref_pos = oracle.cp_reorder(batch.q.view(np.int16), batch.offsets, C)
        ref_ts, _, _ = oracle.cp_reorder(batch.timestamps, batch.offsets, C)
        np.testing.assert_array_equal(pq.cpu().numpy(), ref_q)
        np.testing.assert_array_equal(pts.cpu().numpy(), ref_ts)
        np.testing.assert_array_equal(poff.cpu().numpy(), ref_off)
        np.testing.assert_array_equal(gpos.cpu().numpy(), ref_pos)
        back = hstu.hstu_cp_restore(pq, toff, C)
        assert torch.equal(back, q)


def test_reorder_reports_not_divisible():
    torch, hstu = _torch()
    offsets = torch.tensor([0, 8, 14], dtype=torch.int64, device="cuda")  # 6 % 4 != 0
    src = torch.arange(14, dtype=torch.int64, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    dst = torch.full_like(src, -1)
    hstu.hstu_cp_reorder(src, offsets, 2, dst=dst, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == -6
    # the divisible sequence was still paired correctly
    np.testing.assert_array_equal(dst.cpu().numpy()[[0, 1, 2, 3]], [0, 1, 6, 7])


def test_reorder_reports_bad_offsets():
    torch, hstu = _torch()
    offsets = torch.tensor([0, 8, 4], dtype=torch.int64, device="cuda")
    src = torch.arange(8, dtype=torch.int64, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    hstu.hstu_cp_reorder(src, offsets, 2, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == -5


def test_bucket_indices_bit_exact():
    torch, hstu = _torch()
    rng = np.random.default_rng(5)
    tq = [0, 1, 5, 2**62, 2**63 - 1, -(2**63), 3600, 86400, -5, 7, 1 << 40]
    tk = [0, 0, 1, -(2**62), -(2**63), 2**63 - 1, 0, 0, 0, 8, 3]
    edge = [(2**k, 0) for k in range(63)] + [(2**k - 1, 0) for k in range(1, 64)]
    tq += [a for a, _ in edge]
    tk += [b for _, b in edge]
    n = 100000
    tq += list(rng.integers(-(2**62), 2**62, n))
    tk += list(rng.integers(-(2**62), 2**62, n))
    base = 1_700_000_000
    tq += list(base + rng.integers(0, 10**7, n))
    tk += list(base + rng.integers(0, 10**7, n))
    tq = np.array(tq, np.int64)
    tk = np.array(tk, np.int64)
    for NB in (128, 65, 64, 17, 2, 1):
        got = hstu.hstu_bucket_indices(torch.from_numpy(tq).cuda(), torch.from_numpy(tk).cuda(),
                                       NB).cpu().numpy()
        ref = np.array([oracle.bucket_of(int(a), int(b), NB) for a, b in zip(tq[:3000], tk[:3000])])
        np.testing.assert_array_equal(got[:3000], ref)
        # the rest against Python's exact integers
        exp = np.array([min(max(int(a) - int(b), 0).bit_length(), NB - 1)
                        for a, b in zip(tq[3000:], tk[3000:])])
        np.testing.assert_array_equal(got[3000:], exp)
