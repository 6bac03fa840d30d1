"""GPU parity of the post-attention norm gate (Y = LayerNorm(O) ⊙ U over each
token's H·d features, "Actions Speak Louder than Words" §3) and its backward
against the fp64 oracle, element by element, through the C ABI."""
import numpy as np
import pytest

import oracle
import workloads
from hstu_util import assert_close, half_ulp_bf16, to_f64

pytestmark = pytest.mark.gpu

EPS = 1e-5


def _dev(bits):
    import torch
    return torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).cuda()


def _tight(got, ref, name):
    """The kernel computes in fp32 from the same bf16 inputs and rounds once to
    bf16: beyond that rounding, only fp32 arithmetic error remains."""
    err = np.abs(got - ref)
    bound = half_ulp_bf16(ref) + 2e-4 * np.maximum(1.0, np.abs(ref))
    worst = int(np.argmax(err - bound))
    assert np.all(err <= bound), (
        f"{name}: {err.ravel()[worst]:.4g} > {bound.ravel()[worst]:.4g} at {worst} "
        f"(ref {ref.ravel()[worst]:.6g}, got {got.ravel()[worst]:.6g})")


CASES = [
    # T, N, seed: N = H·d from 8 (one vector per row, most lanes idle) to 2048
    # (eight vectors per lane); T not a multiple of the 8 rows per block
    (1, 8, 1),
    (37, 8, 2),
    (100, 64, 3),
    (257, 256, 4),
    (1000, 512, 5),
    (333, 264, 6),
    (50, 1024, 7),
    (19, 1032, 8),
    (20, 2048, 9),
]


@pytest.mark.parametrize("T,N,seed", CASES)
def test_forward_matches_oracle(T, N, seed):
    import jagged_hstu_attention_attn_b200 as hstu
    x = workloads.norm_gate_inputs(T, N, seed)
    y = hstu.hstu_norm_gate_fwd(_dev(x.o), _dev(x.u), eps=EPS)
    got = to_f64(y)
    ref, _, _ = oracle.norm_gate_fwd(oracle.bf16_to_f64(x.o), oracle.bf16_to_f64(x.u), EPS)
    assert_close(got, ref, bf16_out=True, name=f"y T={T} N={N}")
    _tight(got, ref, f"y T={T} N={N}")


@pytest.mark.parametrize("T,N,seed", CASES)
def test_backward_matches_oracle(T, N, seed):
    import jagged_hstu_attention_attn_b200 as hstu
    x = workloads.norm_gate_inputs(T, N, seed)
    d_o, d_u = hstu.hstu_norm_gate_bwd(_dev(x.o), _dev(x.u), _dev(x.dy), eps=EPS)
    ref_o, ref_u = oracle.norm_gate_bwd(oracle.bf16_to_f64(x.o), oracle.bf16_to_f64(x.u),
                                        oracle.bf16_to_f64(x.dy), EPS)
    got_o, got_u = to_f64(d_o), to_f64(d_u)
    assert_close(got_o, ref_o, bf16_out=True, name=f"dO T={T} N={N}")
    assert_close(got_u, ref_u, bf16_out=True, name=f"dU T={T} N={N}")
    _tight(got_u, ref_u, f"dU T={T} N={N}")
    # dO = rstd (g - mean g - x̂ mean(g x̂)) subtracts row means: its fp32 error
    # scales with rstd |g|, not with |dO|
    scale = np.sqrt(np.mean(ref_o ** 2, axis=1, keepdims=True))
    err = np.abs(got_o - ref_o)
    assert np.all(err <= half_ulp_bf16(ref_o) + 1e-3 * np.maximum(1.0, scale)), \
        f"dO T={T} N={N}: max err {err.max():.4g}"


def test_full_size_fixed8192_rows():
    """The fixed-8192 workload's output shape: T = 16 x 8192 tokens, N = 8 heads
    x 64; every row compared."""
    import jagged_hstu_attention_attn_b200 as hstu
    T, N = 16 * 8192, 8 * 64
    x = workloads.norm_gate_inputs(T, N, 11)
    o, u, dy = _dev(x.o), _dev(x.u), _dev(x.dy)
    y = to_f64(hstu.hstu_norm_gate_fwd(o, u, eps=EPS))
    d_o, d_u = hstu.hstu_norm_gate_bwd(o, u, dy, eps=EPS)
    fo, fu, fdy = (oracle.bf16_to_f64(a) for a in (x.o, x.u, x.dy))
    ref, _, _ = oracle.norm_gate_fwd(fo, fu, EPS)
    assert_close(y, ref, bf16_out=True, name="y fixed8192")
    _tight(y, ref, "y fixed8192")
    ref_o, ref_u = oracle.norm_gate_bwd(fo, fu, fdy, EPS)
    assert_close(to_f64(d_o), ref_o, bf16_out=True, name="dO fixed8192")
    assert_close(to_f64(d_u), ref_u, bf16_out=True, name="dU fixed8192")


def test_three_dim_rows_and_eps():
    """[T, H, d] tensors are normalised over H·d per token; a large eps is
    honoured."""
    import jagged_hstu_attention_attn_b200 as hstu
    T, H, d = 70, 4, 32
    x = workloads.norm_gate_inputs(T, H * d, 12)
    o = _dev(x.o).view(T, H, d)
    u = _dev(x.u).view(T, H, d)
    y = hstu.hstu_norm_gate_fwd(o, u, eps=0.5)
    assert tuple(y.shape) == (T, H, d)
    ref, _, _ = oracle.norm_gate_fwd(oracle.bf16_to_f64(x.o), oracle.bf16_to_f64(x.u), 0.5)
    _tight(to_f64(y).reshape(T, H * d), ref, "y eps=0.5")


def test_constant_rows():
    """Rows with zero spread: x̂ = 0, so y = 0 and dU = 0 exactly, and
    dO = (g - mean g) / sqrt(eps)."""
    import torch
    import jagged_hstu_attention_attn_b200 as hstu
    T, N = 9, 512
    x = workloads.norm_gate_inputs(T, N, 13)
    o = torch.full((T, N), 3.0, dtype=torch.bfloat16, device="cuda")
    u, dy = _dev(x.u), _dev(x.dy)
    y = hstu.hstu_norm_gate_fwd(o, u, eps=1e-2)
    assert torch.count_nonzero(y).item() == 0
    d_o, d_u = hstu.hstu_norm_gate_bwd(o, u, dy, eps=1e-2)
    assert torch.count_nonzero(d_u).item() == 0
    ref_o, _ = oracle.norm_gate_bwd(np.full((T, N), 3.0), oracle.bf16_to_f64(x.u),
                                    oracle.bf16_to_f64(x.dy), 1e-2)
    _tight(to_f64(d_o), ref_o, "dO constant rows")


def test_empty_batch_launches_nothing():
    import torch
    import jagged_hstu_attention_attn_b200 as hstu
    o = torch.empty((0, 512), dtype=torch.bfloat16, device="cuda")
    n0 = hstu.hstu_kernel_launches()
    y = hstu.hstu_norm_gate_fwd(o, o.clone())
    d_o, d_u = hstu.hstu_norm_gate_bwd(o, o.clone(), o.clone())
    assert y.shape == (0, 512) and d_o.shape == (0, 512) and d_u.shape == (0, 512)
    assert hstu.hstu_kernel_launches() == n0


def test_one_launch_per_call_and_refusals():
    import torch
    import jagged_hstu_attention_attn_b200 as hstu
    x = workloads.norm_gate_inputs(64, 512, 14)
    o, u = _dev(x.o), _dev(x.u)
    n0 = hstu.hstu_kernel_launches()
    hstu.hstu_norm_gate_fwd(o, u)
    hstu.hstu_norm_gate_bwd(o, u, u.clone())
    torch.cuda.synchronize()
    assert hstu.hstu_kernel_launches() == n0 + 2
    with pytest.raises(hstu.HstuError):
        hstu.hstu_norm_gate_fwd(o, u, out=o)        # output overlapping an input
    big = torch.zeros((4, 4096), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(hstu.HstuError):
        hstu.hstu_norm_gate_fwd(big, big.clone())   # N above 2048
    with pytest.raises(hstu.HstuError):
        hstu.hstu_norm_gate_fwd(o, u, eps=0.0)
