"""Pins of the fp64 norm-gate oracle (Y = LayerNorm(O) ⊙ U, "Actions Speak
Louder than Words" §3) against values fixed independently of its code: a
hand-worked 3-value row, torch's own layer_norm and autograd in float64 (the
special case of a library routine), central finite differences, and the
invariants of a normalisation."""
import math

import numpy as np
import pytest
import torch

import oracle


def _rand(shape, seed, scale=1.0, shift=0.0):
    rng = np.random.default_rng(seed)
    return rng.standard_normal(shape) * scale + shift


def test_hand_worked_row():
    # o = [1, 2, 3]: mean 2, biased variance 2/3, so with eps = 0
    # x̂ = [-√(3/2), 0, √(3/2)]; gated by u = [2, 3, 4]: y = [-2√(3/2), 0, 4√(3/2)].
    y, mean, rstd = oracle.norm_gate_fwd([[1.0, 2.0, 3.0]], [[2.0, 3.0, 4.0]], 0.0)
    r = math.sqrt(1.5)
    assert np.allclose(y[0], [-2 * r, 0.0, 4 * r], rtol=0, atol=1e-15)
    assert mean[0] == 2.0
    assert abs(rstd[0] - r) < 1e-15
    # dy = [1, 0, 0] at eps = 0: dU = x̂ ⊙ dy = [-√1.5, 0, 0]; g = dy ⊙ u = [2, 0, 0],
    # mean(g) = 2/3, mean(g x̂) = -2√1.5 / 3, so
    # dO = √1.5 (g - 2/3 - x̂ (-2√1.5/3)) = √1.5 ([4/3, -2/3, -2/3] + x̂ √1.5 · 2/3)
    #    = √1.5 [4/3 - 1, -2/3, -2/3 + 1] = √1.5 [1/3, -2/3, 1/3].
    do, du = oracle.norm_gate_bwd([[1.0, 2.0, 3.0]], [[2.0, 3.0, 4.0]], [[1.0, 0.0, 0.0]], 0.0)
    assert np.allclose(du[0], [-r, 0.0, 0.0], rtol=0, atol=1e-15)
    assert np.allclose(do[0], [r / 3, -2 * r / 3, r / 3], rtol=0, atol=1e-14)


@pytest.mark.parametrize("T,N,eps", [(5, 8, 1e-5), (3, 512, 1e-5), (4, 96, 1e-2), (2, 1, 1e-5)])
def test_forward_matches_torch_layer_norm(T, N, eps):
    o = _rand((T, N), 1 + N, scale=3.0, shift=0.7)
    u = _rand((T, N), 2 + N)
    y, mean, rstd = oracle.norm_gate_fwd(o, u, eps)
    ref = torch.nn.functional.layer_norm(torch.from_numpy(o), (N,), eps=eps) * torch.from_numpy(u)
    assert np.allclose(y, ref.numpy(), rtol=1e-12, atol=1e-12)
    assert np.allclose(mean, o.mean(axis=1), rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("T,N,eps", [(5, 8, 1e-5), (3, 512, 1e-5), (4, 96, 1e-2)])
def test_backward_matches_torch_autograd(T, N, eps):
    o = _rand((T, N), 3 + N, scale=2.0, shift=-1.0)
    u = _rand((T, N), 4 + N)
    dy = _rand((T, N), 5 + N)
    to = torch.from_numpy(o).requires_grad_(True)
    tu = torch.from_numpy(u).requires_grad_(True)
    y = torch.nn.functional.layer_norm(to, (N,), eps=eps) * tu
    y.backward(torch.from_numpy(dy))
    do, du = oracle.norm_gate_bwd(o, u, dy, eps)
    assert np.allclose(do, to.grad.numpy(), rtol=1e-11, atol=1e-11)
    assert np.allclose(du, tu.grad.numpy(), rtol=1e-11, atol=1e-11)


def test_backward_central_finite_differences():
    T, N, eps = 2, 7, 1e-3
    o = _rand((T, N), 11, scale=1.5)
    u = _rand((T, N), 12)
    dy = _rand((T, N), 13)
    do, du = oracle.norm_gate_bwd(o, u, dy, eps)

    def loss(oo, uu):
        return float((oracle.norm_gate_fwd(oo, uu, eps)[0] * dy).sum())

    h = 1e-6
    for t in range(T):
        for j in range(N):
            e = np.zeros_like(o)
            e[t, j] = h
            fd_o = (loss(o + e, u) - loss(o - e, u)) / (2 * h)
            fd_u = (loss(o, u + e) - loss(o, u - e)) / (2 * h)
            assert abs(fd_o - do[t, j]) < 1e-7 * max(1.0, abs(do[t, j]))
            assert abs(fd_u - du[t, j]) < 1e-7 * max(1.0, abs(du[t, j]))


def test_normalised_rows_have_zero_mean_and_known_variance():
    T, N, eps = 6, 64, 1e-5
    o = _rand((T, N), 21, scale=0.3, shift=5.0)
    y, _, _ = oracle.norm_gate_fwd(o, np.ones((T, N)), eps)
    var = o.var(axis=1)
    assert np.allclose(y.mean(axis=1), 0.0, atol=1e-13)
    assert np.allclose((y * y).mean(axis=1), var / (var + eps), rtol=1e-12)


def test_shift_and_scale_invariance_at_zero_eps():
    T, N = 3, 40
    o = _rand((T, N), 31)
    u = _rand((T, N), 32)
    y0, _, _ = oracle.norm_gate_fwd(o, u, 0.0)
    y1, _, _ = oracle.norm_gate_fwd(o * 7.5 + 3.25, u, 0.0)
    assert np.allclose(y0, y1, rtol=1e-12, atol=1e-12)
    # the gate enters linearly
    y2, _, _ = oracle.norm_gate_fwd(o, 2.0 * u, 0.0)
    assert np.allclose(y2, 2.0 * y0, rtol=1e-14, atol=1e-14)


def test_constant_row_closed_form():
    # a constant row has x̂ = 0, so y = 0 and dU = 0, and dO = (g - mean(g)) / √eps
    N, eps = 8, 1e-4
    o = np.full((1, N), 3.0)
    u = _rand((1, N), 41)
    dy = _rand((1, N), 42)
    y, _, rstd = oracle.norm_gate_fwd(o, u, eps)
    assert np.all(y == 0.0)
    assert abs(rstd[0] - 1 / math.sqrt(eps)) < 1e-9
    do, du = oracle.norm_gate_bwd(o, u, dy, eps)
    g = dy * u
    assert np.all(du == 0.0)
    assert np.allclose(do, (g - g.mean()) / math.sqrt(eps), rtol=1e-12)


def test_gradient_of_o_sums_to_zero_per_row():
    # the normalised row does not change when a constant is added to o
    T, N = 4, 33
    do, _ = oracle.norm_gate_bwd(_rand((T, N), 51), _rand((T, N), 52), _rand((T, N), 53))
    assert np.allclose(do.sum(axis=1), 0.0, atol=1e-11)


def test_shape_mismatch_is_rejected():
    with pytest.raises(ValueError):
        oracle.norm_gate_fwd(np.zeros((2, 4)), np.zeros((2, 5)))
    with pytest.raises(ValueError):
        oracle.norm_gate_bwd(np.zeros((2, 4)), np.zeros((2, 4)), np.zeros((3, 4)))
