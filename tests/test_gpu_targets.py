"""GPU parity of the target-aware forward (M-FALCON, "Actions Speak Louder
than Words", App. H) against the fp64 oracle, which builds one separate
pass over [history, candidate] per candidate.

Small cases are compared element by element over the whole output (ragged
histories, candidate blocks that span several key tiles so the tiles between
the history and a candidate block are skipped, histories of length 0 and
sequences made only of history); the full-size ranking workload runs in the
launch configuration bench.py uses and is compared on sampled rows."""
import numpy as np
import pytest

import oracle
import workloads
from hstu_util import assert_close, to_device, to_f64

pytestmark = pytest.mark.gpu


def _run(batch, nt, out_fp32=True, status=None, max_seq_len=None):
    import torch
    import jagged_hstu_attention_attn_b200 as hstu
    d = to_device(batch)
    ntd = torch.from_numpy(np.asarray(nt, np.int64)).cuda()
    if max_seq_len is None:
        max_seq_len = int(batch.lengths.max()) if batch.B else 0
    out = hstu.hstu_jagged_attn_fwd_targets(d["q"], d["k"], d["v"], d["offsets"], ntd, d["ts"],
                                            d["w_pos"], d["w_ts"], scale=batch.scale,
                                            max_seq_len=max_seq_len, out_fp32=out_fp32,
                                            dev_status=status)
    torch.cuda.synchronize()
    return out


def _status():
    import torch
    return torch.zeros(1, dtype=torch.int32, device="cuda")


def _oracle(batch, nt):
    q, k, v, _ = oracle.batch_inputs(batch)
    return oracle.fwd_targets(q, k, v, batch.offsets, batch.timestamps, batch.w_pos,
                              batch.w_ts, batch.num_heads, batch.d, batch.scale, nt)


CASES = [
    # seed, lengths, num_targets, H, d, P
    (30, [700, 300, 129], [400, 0, 1], 2, 64, 3072),     # skipped tiles, history only, one
    (31, [260, 513, 90], [260, 13, 45], 1, 128, 600),    # no history at all; ragged
    (32, [1000, 385], [617, 257], 2, 32, 64),            # small P: clamped history biases
    (33, [128, 256, 257], [128, 128, 129], 1, 64, 3072),  # tile-aligned history ends
]


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("out_fp32", [True, False])
def test_small_targets_full_output(case, out_fp32):
    seed, lengths, nt, H, d, P = case
    rng = np.random.default_rng(seed)
    batch = workloads.make_batch("targets", np.asarray(lengths), rng, H=H, d=d, gap="exp",
                                 gap_mean=300.0, P=P, with_dout=False)
    batch = workloads.with_candidates(batch, nt)
    st = _status()
    out = to_f64(_run(batch, nt, out_fp32, status=st))
    assert int(st.item()) == 0
    assert_close(out, _oracle(batch, nt), bf16_out=not out_fp32, name=f"targets{seed}")


def test_zero_targets_is_plain_forward_and_one_target_is_causal():
    import torch
    import jagged_hstu_attention_attn_b200 as hstu
    batch = workloads.random_small(34, 4, 1, 600, 2, 64, P=3072)
    d = to_device(batch)
    ref = hstu.hstu_jagged_attn_fwd(d["q"], d["k"], d["v"], d["offsets"], d["ts"], d["w_pos"],
                                    d["w_ts"], scale=batch.scale,
                                    max_seq_len=int(batch.lengths.max()), out_fp32=True)
    zero = _run(batch, np.zeros(batch.B, np.int64))
    assert torch.equal(zero, ref)
    one = _run(batch, np.minimum(batch.lengths, 1))
    assert torch.equal(one, ref)


def test_bad_counts_and_large_P_are_rejected():
    import torch
    import jagged_hstu_attention_attn_b200 as hstu
    batch = workloads.random_small(35, 2, 50, 60, 1, 64, P=64)
    st = _status()
    _run(batch, [int(batch.lengths[0]) + 1, 0], status=st)
    assert int(st.item()) == -2  # HSTU_ERR_SHAPE
    big = workloads.random_small(36, 2, 50, 60, 1, 128, P=4000)
    with pytest.raises(hstu.HstuError) as e:
        _run(big, [3, 3])
    assert e.value.code == -4    # HSTU_ERR_UNSUPPORTED


def test_mfalcon_workload_sampled_rows():
    """The ranking workload bench.py times (bf16 out), on sampled rows: the
    first and last history rows, the first and last candidates, candidates at
    tile boundaries, random candidates."""
    batch = workloads.mfalcon(with_dout=False)
    nt = batch.meta["num_targets"]
    out = to_f64(_run(batch, nt, out_fp32=False))
    rng = np.random.default_rng(0)
    rows = []
    for b in range(batch.B):
        s, e = int(batch.offsets[b]), int(batch.offsets[b + 1])
        lh = s + (e - s) - int(nt[b])
        rows += [s, lh - 1, lh, e - 1]
        tb = [r for r in range(lh, e) if (r - s) % 128 in (0, 127)]
        rows += tb[:2]
        rows += rng.integers(lh, e, size=2).tolist()
    rows = np.unique(np.asarray(rows, np.int64))
    H = batch.num_heads
    tok = np.repeat(rows, H)
    head = np.tile(np.arange(H), rows.shape[0])
    q, k, v, _ = oracle.batch_inputs(batch)
    ref = oracle.fwd_targets_rows(q, k, v, batch.offsets, batch.timestamps, batch.w_pos,
                                  batch.w_ts, H, batch.d, batch.scale, nt, tok, head)
    assert_close(out[tok, head], ref, bf16_out=True, name="mfalcon")


# ------------------------------------------------------------------ candidates only

def _run_cand(batch, nt, max_targets=0, out_fp32=True, status=None):
    import torch
    import jagged_hstu_attention_attn_b200 as hstu
    d = to_device(batch)
    ntd = torch.from_numpy(np.asarray(nt, np.int64)).cuda()
    T, H = batch.T, batch.num_heads
    out = torch.full((T, H, batch.d), float("nan"), device="cuda",
                     dtype=torch.float32 if out_fp32 else torch.bfloat16)
    hstu.hstu_jagged_attn_fwd_candidates(d["q"], d["k"], d["v"], d["offsets"], ntd, d["ts"],
                                         d["w_pos"], d["w_ts"], scale=batch.scale,
                                         max_seq_len=int(batch.lengths.max()),
                                         max_targets=max_targets, out_fp32=out_fp32, out=out,
                                         dev_status=status)
    torch.cuda.synchronize()
    return out


def _cand_rows(batch, nt):
    rows, hist = [], []
    for b in range(batch.B):
        s, e = int(batch.offsets[b]), int(batch.offsets[b + 1])
        lh = e - int(nt[b])
        rows += list(range(lh, e))
        hist += list(range(s, lh))
    return np.asarray(rows, np.int64), np.asarray(hist, np.int64)


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("hint", ["exact", "unknown"])
def test_candidates_only_rows(case, hint):
    """Candidate rows equal the target-aware oracle; history rows are not
    written (they keep the NaN the output was filled with)."""
    seed, lengths, nt, H, d, P = case
    rng = np.random.default_rng(seed)
    batch = workloads.make_batch("targets", np.asarray(lengths), rng, H=H, d=d, gap="exp",
                                 gap_mean=300.0, P=P, with_dout=False)
    batch = workloads.with_candidates(batch, nt)
    st = _status()
    out = to_f64(_run_cand(batch, nt, max_targets=max(nt) if hint == "exact" else 0, status=st))
    assert int(st.item()) == 0
    rows, hist = _cand_rows(batch, nt)
    ref = _oracle(batch, nt)
    assert_close(out[rows], ref[rows], name=f"candidates{seed}")
    assert np.all(np.isnan(out[hist]))


def test_candidates_only_mfalcon_sampled():
    """The ranking workload: every user's microbatch of 1024 candidates over
    its cached history, sampled candidate rows against the oracle."""
    batch = workloads.mfalcon(with_dout=False)
    nt = batch.meta["num_targets"]
    out = to_f64(_run_cand(batch, nt, max_targets=int(nt.max()), out_fp32=False))
    rows, hist = _cand_rows(batch, nt)
    assert np.all(np.isnan(out[hist]))
    rng = np.random.default_rng(1)
    pick = np.unique(np.concatenate([rng.choice(rows, 48, replace=False),
                                     rows[:2], rows[-2:]]))
    H = batch.num_heads
    tok = np.repeat(pick, H)
    head = np.tile(np.arange(H), pick.shape[0])
    q, k, v, _ = oracle.batch_inputs(batch)
    ref = oracle.fwd_targets_rows(q, k, v, batch.offsets, batch.timestamps, batch.w_pos,
                                  batch.w_ts, H, batch.d, batch.scale, nt, tok, head)
    assert_close(out[tok, head], ref, bf16_out=True, name="mfalcon candidates")
