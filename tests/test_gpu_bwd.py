"""GPU parity of the tcgen05 backward kernel against the fp64 oracle:
dq, dk, dv element by element on small cases, sampled rows at full size, and
the bias gradients dw_pos / dw_ts against the oracle (small cases and
sequence subsets) and against invariants that hold at any size."""
import numpy as np
import pytest

import oracle
import workloads
from hstu_util import assert_close_grad, sample_rows, to_device, to_f64

pytestmark = pytest.mark.gpu


def _run_bwd(batch, max_seq_len=None, status=None):
    import torch
    import jagged_hstu_attention_attn_b200 as hstu
    d = to_device(batch)
    if max_seq_len is None:
        max_seq_len = int(batch.lengths.max()) if batch.B else 0
    res = hstu.hstu_jagged_attn_bwd(d["q"], d["k"], d["v"], d["offsets"], d["ts"], d["w_pos"],
                                    d["w_ts"], d["dout"], scale=batch.scale,
                                    max_seq_len=max_seq_len, dev_status=status)
    torch.cuda.synchronize()
    return res


def _status():
    import torch
    return torch.zeros(1, dtype=torch.int32, device="cuda")


def _check_all(batch, res, name):
    dq, dk, dv, dwp, dwt = res
    rq, rk, rv, rwp, rwt = oracle.batch_bwd(batch)
    assert_close_grad(to_f64(dq), rq, name=f"{name} dq")
    assert_close_grad(to_f64(dk), rk, name=f"{name} dk")
    assert_close_grad(to_f64(dv), rv, name=f"{name} dv")
    assert_close_grad(to_f64(dwp), rwp, bf16_out=False, name=f"{name} dw_pos")
    assert_close_grad(to_f64(dwt), rwt, bf16_out=False, name=f"{name} dw_ts")
    # buckets the oracle never selects get exactly zero
    assert np.all(to_f64(dwt)[rwt == 0.0] == 0.0)


def test_tiny_workload_full():
    batch = workloads.tiny(0)
    st = _status()
    res = _run_bwd(batch, status=st)
    assert int(st.item()) == 0
    _check_all(batch, res, "tiny")


CASES = [
    # seed, B, Lmin, Lmax, H, d, P, NB, gap
    (1, 5, 0, 300, 2, 32, 40, 128, 500.0),
    (2, 3, 129, 520, 3, 64, 600, 20, 50.0),
    (3, 4, 1, 400, 2, 128, 3072, 128, 3000.0),
    (4, 2, 255, 257, 1, 64, 8, 128, 1.0),
    (5, 2, 600, 700, 2, 128, 5000, 128, 20.0),   # P above the shared-memory window
]


@pytest.mark.parametrize("case", CASES)
def test_small_random_full(case):
    seed, B, lo, hi, H, d, P, NB, gap = case
    batch = workloads.random_small(seed, B, lo, hi, H, d, P=P, NB=NB, gap_mean=gap)
    st = _status()
    res = _run_bwd(batch, status=st)
    assert int(st.item()) == 0
    _check_all(batch, res, f"case{seed}")


def test_non_monotone_timestamps():
    batch = workloads.random_small(7, 3, 100, 300, 2, 64, P=300, NB=128, gap_mean=100.0)
    rng = np.random.default_rng(7)
    batch.timestamps = rng.integers(-(2**40), 2**40, batch.T).astype(np.int64)
    st = _status()
    res = _run_bwd(batch, status=st)
    assert int(st.item()) == 0
    _check_all(batch, res, "non-monotone")


@pytest.mark.parametrize("name", ["zipf", "fixed8192", "long"])
def test_full_size_sampled_rows_and_invariants(name):
    import torch
    batch = workloads.WORKLOADS[name]()
    st = _status()
    dq, dk, dv, dwp, dwt = _run_bwd(batch, status=st)
    assert int(st.item()) == 0
    tok, head = sample_rows(batch, 96, seed=2)
    q, k, v, dout = oracle.batch_inputs(batch)
    rq, rk, rv = oracle.bwd_rows(q, k, v, batch.offsets, batch.timestamps, batch.w_pos,
                                 batch.w_ts, batch.num_heads, batch.d, batch.scale, dout, tok, head)
    it, ih = torch.from_numpy(tok).cuda(), torch.from_numpy(head).cuda()
    assert_close_grad(to_f64(dq[it, ih]), rq, name=f"{name} dq")
    assert_close_grad(to_f64(dk[it, ih]), rk, name=f"{name} dk")
    assert_close_grad(to_f64(dv[it, ih]), rv, name=f"{name} dv")
    wp, wt = to_f64(dwp), to_f64(dwt)
    # every pair adds scale*g to exactly one entry of each table
    tot = np.abs(wp).sum() + np.abs(wt).sum()
    assert abs(wp.sum() - wt.sum()) <= 1e-3 * tot
    # buckets above the largest time difference of any sequence are never selected
    maxdt = max(int(batch.timestamps[e - 1] - batch.timestamps[s])
                for s, e in zip(batch.offsets[:-1], batch.offsets[1:]) if e > s)
    assert np.all(wt[maxdt.bit_length() + 1:] == 0.0)
    for t in (dq, dk, dv):
        assert bool(torch.isfinite(t).all())


def test_zipf_subset_bias_gradients_full():
    batch = workloads.zipf()
    order = np.argsort(batch.lengths)
    sub = batch.subset([int(order[0]), int(order[-1]), int(order[len(order) // 2])])
    st = _status()
    res = _run_bwd(sub, status=st)
    assert int(st.item()) == 0
    _check_all(sub, res, "zipf-subset")


def test_bwd_reports_bad_offsets():
    import torch
    import jagged_hstu_attention_attn_b200 as hstu
    batch = workloads.random_small(11, 3, 50, 60, 1, 32, P=64)
    d = to_device(batch)
    off = d["offsets"].clone()
    off[2] = off[1] - 5
    st = _status()
    hstu.hstu_jagged_attn_bwd(d["q"], d["k"], d["v"], off, d["ts"], d["w_pos"], d["w_ts"],
                              d["dout"], max_seq_len=200, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == -5
