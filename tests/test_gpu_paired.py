"""GPU parity of attention on the load-balanced paired layout: reorder ->
paired attention -> restore reproduces the unsharded result (oracle and GPU),
including rows at mini-chunk boundaries."""
import numpy as np
import pytest

import oracle
import workloads
from hstu_util import assert_close, to_device, to_f64

pytestmark = pytest.mark.gpu


def _paired_pipeline(batch, C, out_fp32=True, status=None):
    import torch
    import jagged_hstu_attention_attn_b200 as hstu
    d = to_device(batch)
    off = d["offsets"]
    pq, _, _ = hstu.hstu_cp_reorder(d["q"], off, C, want_maps=False, dev_status=status)
    pk, _, _ = hstu.hstu_cp_reorder(d["k"], off, C, want_maps=False, dev_status=status)
    pv, _, _ = hstu.hstu_cp_reorder(d["v"], off, C, want_maps=False, dev_status=status)
    pts, _, _ = hstu.hstu_cp_reorder(d["ts"], off, C, want_maps=False, dev_status=status)
    pout = hstu.hstu_cp_paired_attn_fwd(pq, pk, pv, off, pts, C, d["w_pos"], d["w_ts"],
                                        scale=batch.scale, max_seq_len=int(batch.lengths.max()),
                                        out_fp32=out_fp32, dev_status=status)
    out = hstu.hstu_cp_restore(pout, off, C, dev_status=status)
    unsharded = hstu.hstu_jagged_attn_fwd(d["q"], d["k"], d["v"], off, d["ts"], d["w_pos"],
                                          d["w_ts"], scale=batch.scale,
                                          max_seq_len=int(batch.lengths.max()), out_fp32=out_fp32,
                                          dev_status=status)
    torch.cuda.synchronize()
    return out, unsharded


@pytest.mark.parametrize("C", [1, 2, 4, 8])
@pytest.mark.parametrize("d", [32, 128])
def test_paired_small_equals_unsharded(C, d):
    import torch
    batch = workloads.random_small(40 + C, 5, 1, 700 // (2 * C), 2, d, P=200, pad_to=2 * C)
    batch.lengths = np.diff(batch.offsets)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, uns = _paired_pipeline(batch, C, status=st)
    assert int(st.item()) == 0
    ref = oracle.batch_fwd(batch)
    assert_close(to_f64(out), ref, name=f"paired C={C}")
    assert_close(to_f64(uns), ref, name="unsharded")
    # paired and unsharded GPU results agree to rounding
    np.testing.assert_allclose(to_f64(out), to_f64(uns), rtol=0, atol=1e-3)


@pytest.mark.parametrize("C,d,P", [(2, 128, 5000), (8, 128, 5000), (4, 64, 4100)])
def test_paired_window_path_full_output(C, d, P):
    """P above the kernel's shared-memory w_pos table: per-tile windows on the
    paired layout, where a query tile's key tiles come from two mini-chunks."""
    import torch
    batch = workloads.random_small(70 + C, 3, 3000, 5400, 2, d, P=P, gap_mean=30.0,
                                   pad_to=2 * C)
    batch.lengths = np.diff(batch.offsets)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, uns = _paired_pipeline(batch, C, status=st)
    assert int(st.item()) == 0
    ref = oracle.batch_fwd(batch)
    assert_close(to_f64(out), ref, name=f"paired window C={C}")
    assert_close(to_f64(uns), ref, name="unsharded window")


@pytest.mark.parametrize("C", [2, 4, 8])
def test_paired_full_size_sampled(C):
    import torch
    batch = workloads.paired(C)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, uns = _paired_pipeline(batch, C, status=st)
    assert int(st.item()) == 0
    rng = np.random.default_rng(C)
    toks = []
    for b in rng.choice(batch.B, 6, replace=False):
        s, e = int(batch.offsets[b]), int(batch.offsets[b + 1])
        m = (e - s) // (2 * C)
        for c in range(2 * C):     # rows on both sides of every mini-chunk boundary
            for u in (0, 1, m - 1):
                toks.append(s + c * m + u)
    toks = np.array(sorted(set(toks)), np.int64)
    heads = rng.integers(0, batch.num_heads, toks.shape[0]).astype(np.int64)
    q, k, v, _ = oracle.batch_inputs(batch)
    ref = oracle.fwd_rows(q, k, v, batch.offsets, batch.timestamps, batch.w_pos, batch.w_ts,
                          batch.num_heads, batch.d, batch.scale, toks, heads)
    it, ih = torch.from_numpy(toks).cuda(), torch.from_numpy(heads).cuda()
    assert_close(to_f64(out[it, ih]), ref, name=f"paired full C={C}")
    assert_close(to_f64(uns[it, ih]), ref, name="unsharded full")


def test_paired_rejects_non_divisible_lengths():
    import torch
    import jagged_hstu_attention_attn_b200 as hstu
    batch = workloads.make_batch("nondiv", [12, 13, 8], np.random.default_rng(50), H=1, d=32,
                                 gap="exp", gap_mean=10.0, P=64)
    d = to_device(batch)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    hstu.hstu_cp_paired_attn_fwd(d["q"], d["k"], d["v"], d["offsets"], d["ts"], 2, d["w_pos"],
                                 d["w_ts"], max_seq_len=16, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == -6
