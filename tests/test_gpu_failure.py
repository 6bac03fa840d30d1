"""Failure detection without a GPU fault: a bounded wait that runs out ends
with HSTU_ERR_TIMEOUT in the device status word, and the context stays usable.

The wait is provoked in the allowed way only: one warp waits, with a short
limit, on an mbarrier that nothing arrives on (no copy or tensor-core work in
flight).  The attention kernels use the same bounded wait for every
pipeline stage."""
import pytest

import oracle
import workloads
from hstu_util import assert_close, to_device, to_f64

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    import torch
    import jagged_hstu_attention_attn_b200 as hstu
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    res = torch.full((1,), 7, dtype=torch.int32, device="cuda")
    hstu.hstu_selftest_wait_timeout(20_000_000, dev_status=st, result=res)   # 20 ms
    torch.cuda.synchronize()
    assert int(st.item()) == -7   # HSTU_ERR_TIMEOUT
    assert int(res.item()) == 0   # the wait gave up
    # the context is still usable: a forward afterwards runs and is correct
    batch = workloads.tiny(0)
    d = to_device(batch)
    st2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = hstu.hstu_jagged_attn_fwd(d["q"], d["k"], d["v"], d["offsets"], d["ts"], d["w_pos"],
                                    d["w_ts"], scale=batch.scale,
                                    max_seq_len=int(batch.lengths.max()), out_fp32=True,
                                    dev_status=st2)
    torch.cuda.synchronize()
    assert int(st2.item()) == 0
    assert_close(to_f64(out), oracle.batch_fwd(batch), name="after timeout")
