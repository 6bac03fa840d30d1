"""hstu_jagged_attn_bwd_noalloc: the backward for callers that cannot
allocate device memory (inside another runtime's plugin callback, or a
process whose device-memory plan is fixed up front).  It uses the library's
own static scratch array instead of a caller workspace.

Checked here through the C ABI: two calls in a row give the same gradients as
the regular hstu_jagged_attn_bwd (within the gradient tolerance of the other
tests), and a problem larger than the scratch array is refused without a
launch.  This file is collected last so a failure here never hides another
test; it also passes on its own in a fresh process (where its first call is
the one that looks up the scratch array's address)."""
import ctypes

import numpy as np
import pytest

import workloads
from hstu_util import assert_close_grad, to_device, to_f64

pytestmark = pytest.mark.gpu


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _call_noalloc(lib, batch, d, outs, stream):
    dq, dk, dv, dwp, dwt = outs
    return lib.hstu_jagged_attn_bwd_noalloc(
        _ptr(d["q"]), _ptr(d["k"]), _ptr(d["v"]), _ptr(d["offsets"]), batch.B, batch.T,
        int(batch.lengths.max()), _ptr(d["ts"]), _ptr(d["w_pos"]), batch.P, _ptr(d["w_ts"]),
        batch.NB, batch.num_heads, batch.d, batch.d, ctypes.c_float(batch.scale),
        _ptr(d["dout"]), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dwp), _ptr(dwt), None,
        ctypes.c_void_p(stream))


def test_noalloc_matches_workspace_backward_twice():
    import torch
    import jagged_hstu_attention_attn_b200 as hstu
    lib = hstu.lib()
    batch = workloads.random_small(61, 3, 100, 700, 2, 128, P=3072)
    assert batch.T * batch.num_heads * batch.d <= hstu.NOALLOC_MAX_ELEMS
    d = to_device(batch)
    ref = hstu.hstu_jagged_attn_bwd(d["q"], d["k"], d["v"], d["offsets"], d["ts"], d["w_pos"],
                                    d["w_ts"], d["dout"], scale=batch.scale,
                                    max_seq_len=int(batch.lengths.max()))
    torch.cuda.synchronize()
    ref = [to_f64(t) for t in ref]
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        outs = [torch.full_like(d["q"], float("nan")), torch.full_like(d["k"], float("nan")),
                torch.full_like(d["v"], float("nan")), torch.full_like(d["w_pos"], float("nan")),
                torch.full_like(d["w_ts"], float("nan"))]
        code = _call_noalloc(lib, batch, d, outs, stream)
        assert code == 0, hstu.hstu_status_str(code)
        torch.cuda.synchronize()
        for name, got, r in zip(("dq", "dk", "dv", "dw_pos", "dw_ts"), outs, ref):
            assert_close_grad(to_f64(got), r, bf16_out=name in ("dq", "dk", "dv"),
                              name=f"call {call} {name}")


def test_noalloc_rejects_problems_above_the_scratch_size():
    import torch
    import jagged_hstu_attention_attn_b200 as hstu
    lib = hstu.lib()
    H, dd = 4, 128
    T = hstu.NOALLOC_MAX_ELEMS // (H * dd) + 1   # one token too many
    q = torch.zeros((T, H, dd), dtype=torch.bfloat16, device="cuda")
    off = torch.tensor([0, T], dtype=torch.int64, device="cuda")
    ts = torch.zeros(T, dtype=torch.int64, device="cuda")
    wp = torch.zeros(8, device="cuda")
    wt = torch.zeros(8, device="cuda")
    before = hstu.hstu_kernel_launches()
    code = lib.hstu_jagged_attn_bwd_noalloc(
        _ptr(q), _ptr(q), _ptr(q), _ptr(off), 1, T, T, _ptr(ts), _ptr(wp), 8, _ptr(wt), 8, H, dd,
        dd, ctypes.c_float(0.1), _ptr(q), _ptr(q), _ptr(q), _ptr(q), _ptr(wp), _ptr(wt), None,
        None)
    assert code == -9   # HSTU_ERR_WORKSPACE: larger than the static scratch
    assert hstu.hstu_kernel_launches() == before
