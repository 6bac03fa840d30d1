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


def _nan_outputs(d):
    import torch
    return [torch.full_like(d["q"], float("nan")), torch.full_like(d["k"], float("nan")),
            torch.full_like(d["v"], float("nan")), torch.full_like(d["w_pos"], float("nan")),
            torch.full_like(d["w_ts"], float("nan"))]


def _check_against_workspace_backward(batch, calls=2):
    import torch
    import jagged_hstu_attention_attn_b200 as hstu
    lib = hstu.lib()
    assert batch.T * batch.num_heads * batch.d <= hstu.NOALLOC_MAX_ELEMS
    d = to_device(batch)
    ref = hstu.hstu_jagged_attn_bwd(d["q"], d["k"], d["v"], d["offsets"], d["ts"], d["w_pos"],
                                    d["w_ts"], d["dout"], scale=batch.scale,
                                    max_seq_len=int(batch.lengths.max()))
    torch.cuda.synchronize()
    ref = [to_f64(t) for t in ref]
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(calls):
        outs = _nan_outputs(d)
        code = _call_noalloc(lib, batch, d, outs, stream)
        assert code == 0, hstu.hstu_status_str(code)
        torch.cuda.synchronize()
        for name, got, r in zip(("dq", "dk", "dv", "dw_pos", "dw_ts"), outs, ref):
            assert_close_grad(to_f64(got), r, bf16_out=name in ("dq", "dk", "dv"),
                              name=f"call {call} {name}")


@pytest.mark.parametrize("d", [32, 64, 128])
def test_noalloc_matches_workspace_backward_twice(d):
    P = 3072 if d == 128 else 600
    batch = workloads.random_small(61 + d, 3, 100, 700, 2, d, P=P)
    _check_against_workspace_backward(batch)


def test_noalloc_at_exactly_the_scratch_size():
    """T * H * d equal to the scratch capacity: the workspace the backward
    needs (rounded up to 256 bytes) still fits, so the call must succeed."""
    import jagged_hstu_attention_attn_b200 as hstu
    H, dd = 2, 64
    T = hstu.NOALLOC_MAX_ELEMS // (H * dd)
    assert T * H * dd == hstu.NOALLOC_MAX_ELEMS
    lengths = np.array([T // 8] * 8, np.int64)
    assert int(lengths.sum()) == T
    rng = np.random.default_rng(65)
    batch = workloads.make_batch("noalloc_full", lengths, rng, H=H, d=dd, gap="exp",
                                 gap_mean=600.0, P=3072, NB=128, with_dout=True)
    _check_against_workspace_backward(batch, calls=1)


def test_noalloc_empty_problem_zeroes_bias_gradients():
    """T = 0: nothing to differentiate; the bias gradients are still
    overwritten with zeros and no attention kernel runs."""
    import torch
    import jagged_hstu_attention_attn_b200 as hstu
    lib = hstu.lib()
    q = torch.zeros((1, 2, 64), dtype=torch.bfloat16, device="cuda")
    off = torch.zeros(3, dtype=torch.int64, device="cuda")
    ts = torch.zeros(1, dtype=torch.int64, device="cuda")
    wp = torch.zeros(16, device="cuda")
    wt = torch.zeros(8, device="cuda")
    dwp = torch.full((16,), float("nan"), device="cuda")
    dwt = torch.full((8,), float("nan"), device="cuda")
    before = hstu.hstu_kernel_launches()
    code = lib.hstu_jagged_attn_bwd_noalloc(
        _ptr(q), _ptr(q), _ptr(q), _ptr(off), 2, 0, 0, _ptr(ts), _ptr(wp), 16, _ptr(wt), 8, 2, 64,
        64, ctypes.c_float(0.125), _ptr(q), _ptr(q), _ptr(q), _ptr(q), _ptr(dwp), _ptr(dwt), None,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert code == 0, hstu.hstu_status_str(code)
    torch.cuda.synchronize()
    assert hstu.hstu_kernel_launches() == before
    assert bool((dwp == 0).all()) and bool((dwt == 0).all())


def test_noalloc_rejects_unsupported_head_size_before_any_work():
    import torch
    import jagged_hstu_attention_attn_b200 as hstu
    lib = hstu.lib()
    q = torch.zeros((64, 1, 48), dtype=torch.bfloat16, device="cuda")
    off = torch.tensor([0, 64], dtype=torch.int64, device="cuda")
    ts = torch.zeros(64, dtype=torch.int64, device="cuda")
    wp = torch.zeros(8, device="cuda")
    wt = torch.zeros(8, device="cuda")
    before = hstu.hstu_kernel_launches()
    code = lib.hstu_jagged_attn_bwd_noalloc(
        _ptr(q), _ptr(q), _ptr(q), _ptr(off), 1, 64, 64, _ptr(ts), _ptr(wp), 8, _ptr(wt), 8, 1, 48,
        48, ctypes.c_float(0.1), _ptr(q), _ptr(q), _ptr(q), _ptr(q), _ptr(wp), _ptr(wt), None,
        None)
    assert code == -4   # HSTU_ERR_UNSUPPORTED
    assert hstu.hstu_kernel_launches() == before


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
