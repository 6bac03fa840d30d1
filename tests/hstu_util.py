"""Shared helpers for the GPU parity tests: device upload of a JaggedBatch,
the tolerance checks, and sampling of rows for full-size comparisons."""
import math

import numpy as np

import oracle
import workloads

# tolerance for attention outputs (bf16 in, fp32 accumulate)
MAX_ABS = 2e-2
REL_L2 = 1e-2


def to_device(batch, device="cuda"):
    import torch
    d = {}
    as_bf16 = lambda bits: torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16)
    d["q"] = as_bf16(batch.q).to(device)
    d["k"] = as_bf16(batch.k).to(device)
    d["v"] = as_bf16(batch.v).to(device)
    d["dout"] = None if batch.dout is None else as_bf16(batch.dout).to(device)
    d["offsets"] = torch.from_numpy(batch.offsets.copy()).to(device)
    d["ts"] = torch.from_numpy(batch.timestamps.copy()).to(device)
    d["w_pos"] = torch.from_numpy(batch.w_pos.copy()).to(device)
    d["w_ts"] = torch.from_numpy(batch.w_ts.copy()).to(device)
    return d


def to_f64(t) -> np.ndarray:
    import torch
    return t.detach().to(torch.float64).cpu().numpy()


def half_ulp_bf16(x: np.ndarray) -> np.ndarray:
    """Half a bf16 unit in the last place at |x| (7 stored mantissa bits)."""
    ax = np.maximum(np.abs(x), np.finfo(np.float32).tiny)
    e = np.floor(np.log2(ax))
    return 0.5 * np.exp2(e - 7)


def rel_l2(got, ref) -> float:
    den = float(np.linalg.norm(ref.ravel()))
    return float(np.linalg.norm((got - ref).ravel())) / max(den, 1e-30)


def assert_close(got, ref, *, bf16_out=False, name="", scale_abs=1.0):
    """max-abs <= MAX_ABS (+ half a bf16 ulp of the reference when the output
    itself is bf16) and rel-L2 <= REL_L2."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    err = np.abs(got - ref)
    bound = MAX_ABS * scale_abs + (half_ulp_bf16(ref) if bf16_out else 0.0)
    worst = np.argmax(err - bound) if err.size else 0
    assert np.all(err <= bound), (
        f"{name}: max-abs violation {err.ravel()[worst]:.4g} > {np.ravel(bound)[worst] if np.ndim(bound) else bound:.4g}"
        f" at flat index {worst} (ref {ref.ravel()[worst]:.5g}, got {got.ravel()[worst]:.5g})")
    r = rel_l2(got, ref)
    assert r <= REL_L2, f"{name}: rel-L2 {r:.3g} > {REL_L2}"
    return float(err.max()) if err.size else 0.0, r


def sample_rows(batch, n, seed=0, include_edges=True):
    """(token, head) pairs: random rows plus the first / last rows of sequences
    and rows at tile boundaries (multiples of 128 and their neighbours)."""
    rng = np.random.default_rng(seed)
    toks = list(rng.integers(0, batch.T, n)) if batch.T else []
    if include_edges:
        for b in range(batch.B):
            s, e = int(batch.offsets[b]), int(batch.offsets[b + 1])
            if e <= s:
                continue
            for p in (0, 1, 127, 128, 129, e - s - 1, e - s - 2):
                if 0 <= p < e - s:
                    toks.append(s + p)
            if len(toks) > 4 * n:
                break
    toks = np.array(sorted(set(int(t) for t in toks)), np.int64)
    heads = rng.integers(0, batch.num_heads, toks.shape[0]).astype(np.int64)
    return toks, heads


def assert_close_grad(got, ref, *, bf16_out=True, name=""):
    """Gradient tolerance: rel-L2 <= REL_L2 and, element by element,
    |err| <= MAX_ABS * max(1, rms(ref)) (+ half a bf16 ulp of ref when the
    output is bf16).  The backward feeds bf16 P^T / dS^T to the tensor cores,
    whose rounding error grows with the length of the sums like the result
    itself, so the absolute bound scales with the reference's magnitude."""
    ref = np.asarray(ref, np.float64)
    rms = float(np.sqrt(np.mean(ref ** 2))) if ref.size else 0.0
    return assert_close(got, ref, bf16_out=bf16_out, name=name, scale_abs=max(1.0, rms))
