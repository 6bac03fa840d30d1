"""GPU parity of the tcgen05 forward kernel against the fp64 oracle.

Small cases are compared element by element over the whole output; the
full-size workloads run in the launch configuration bench.py uses and are
compared on sampled rows (first / last rows of sequences, tile boundaries,
random rows) that the oracle evaluates one by one."""
import math

import numpy as np
import pytest

import oracle
import workloads
from hstu_util import assert_close, sample_rows, to_device, to_f64

pytestmark = pytest.mark.gpu


def _run_fwd(batch, out_fp32=True, max_seq_len=None, status=None):
    import torch
    import jagged_hstu_attention_attn_b200 as hstu
    d = to_device(batch)
    if max_seq_len is None:
        max_seq_len = int(batch.lengths.max()) if batch.B else 0
    out = hstu.hstu_jagged_attn_fwd(d["q"], d["k"], d["v"], d["offsets"], d["ts"], d["w_pos"],
                                    d["w_ts"], scale=batch.scale, max_seq_len=max_seq_len,
                                    out_fp32=out_fp32, dev_status=status)
    torch.cuda.synchronize()
    return out


def _status():
    import torch
    return torch.zeros(1, dtype=torch.int32, device="cuda")


@pytest.mark.parametrize("out_fp32", [True, False])
def test_tiny_workload_full_output(out_fp32):
    batch = workloads.tiny(0)
    st = _status()
    out = to_f64(_run_fwd(batch, out_fp32, status=st))
    assert int(st.item()) == 0
    ref = oracle.batch_fwd(batch)
    assert_close(out, ref, bf16_out=not out_fp32, name="tiny")


CASES = [
    # seed, B, Lmin, Lmax, H, d, P, NB, gap
    (1, 5, 0, 300, 2, 32, 40, 128, 500.0),      # empty sequences, ragged tails, P clamp
    (2, 3, 129, 520, 3, 64, 600, 20, 50.0),     # NB clamp
    (3, 4, 1, 400, 2, 128, 3072, 128, 3000.0),
    (4, 2, 255, 257, 1, 64, 8, 128, 1.0),       # tile boundary lengths, small P
    # P above the shared-memory table (3328 at d = 128, 4096 at d <= 64): the
    # kernel builds a w_pos window per key tile; lengths reach past P - 1
    (5, 3, 3000, 5400, 2, 128, 5000, 128, 30.0),
    (6, 3, 3000, 5400, 2, 64, 4100, 128, 30.0),
    (12, 2, 4000, 4600, 2, 32, 4097, 128, 30.0),
]


@pytest.mark.parametrize("case", CASES)
def test_small_random_full_output(case):
    seed, B, lo, hi, H, d, P, NB, gap = case
    batch = workloads.random_small(seed, B, lo, hi, H, d, P=P, NB=NB, gap_mean=gap)
    st = _status()
    out = to_f64(_run_fwd(batch, True, status=st))
    assert int(st.item()) == 0
    ref = oracle.batch_fwd(batch)
    assert_close(out, ref, name=f"case{seed}")


def test_non_monotone_and_extreme_timestamps():
    """Buckets along a row are not monotone: the per-pair bucket path."""
    batch = workloads.random_small(7, 3, 100, 300, 2, 64, P=300, NB=128, gap_mean=100.0)
    rng = np.random.default_rng(7)
    batch.timestamps = rng.integers(-(2**62), 2**62, batch.T).astype(np.int64)
    batch.timestamps[:10] = [0, 2**62, -(2**62), 5, 5, 4, 3, 2**40, -1, 0]
    st = _status()
    out = to_f64(_run_fwd(batch, True, status=st))
    assert int(st.item()) == 0
    assert_close(out, oracle.batch_fwd(batch), name="non-monotone")


def test_scale_and_bias_magnitudes():
    batch = workloads.random_small(8, 2, 200, 260, 2, 32, P=64, NB=128, gap_mean=10.0)
    batch.w_pos = (np.arange(64, dtype=np.float32) - 32) / 16
    batch.w_ts = np.linspace(-1, 1, 128).astype(np.float32)
    batch.scale = 0.3
    out = to_f64(_run_fwd(batch, True))
    assert_close(out, oracle.batch_fwd(batch), name="bias")


def test_deterministic_bitwise():
    import torch
    batch = workloads.random_small(9, 4, 100, 700, 2, 128, P=3072)
    a = _run_fwd(batch, False)
    b = _run_fwd(batch, False)
    assert torch.equal(a, b)


def test_max_seq_len_too_small_is_reported():
    batch = workloads.random_small(10, 2, 300, 300, 1, 64, P=64)
    st = _status()
    _run_fwd(batch, True, max_seq_len=100, status=st)
    assert int(st.item()) == -2


def test_bad_offsets_are_reported_without_fault():
    import torch
    import jagged_hstu_attention_attn_b200 as hstu
    batch = workloads.random_small(11, 3, 50, 60, 1, 32, P=64)
    d = to_device(batch)
    off = d["offsets"].clone()
    off[2] = off[1] - 5   # decreasing
    st = _status()
    hstu.hstu_jagged_attn_fwd(d["q"], d["k"], d["v"], off, d["ts"], d["w_pos"], d["w_ts"],
                              max_seq_len=200, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == -5


@pytest.mark.parametrize("name", ["zipf", "fixed8192", "long"])
def test_full_size_sampled_rows(name):
    batch = workloads.WORKLOADS[name](with_dout=False)
    st = _status()
    out = _run_fwd(batch, True, status=st)
    assert int(st.item()) == 0
    tok, head = sample_rows(batch, 192, seed=1)
    q, k, v, _ = oracle.batch_inputs(batch)
    ref = oracle.fwd_rows(q, k, v, batch.offsets, batch.timestamps, batch.w_pos, batch.w_ts,
                          batch.num_heads, batch.d, batch.scale, tok, head)
    import torch
    got = to_f64(out[torch.from_numpy(tok).cuda(), torch.from_numpy(head).cuda()])
    assert_close(got, ref, name=name)
    # the whole output is finite and rows of every sequence were written
    assert bool(torch.isfinite(out).all())
