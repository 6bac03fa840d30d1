"""The C ABI library loads and exports every entry point include/hstu.h
declares; host-side argument checks return their status codes (CPU only:
none of these calls reaches a CUDA API)."""
import ctypes
import os
import re
import subprocess

import pytest

import jagged_hstu_attention_attn_b200 as hstu
from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "hstu.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(hstu_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from jagged_hstu_attention_attn_b200 import build
    build.build()
    return hstu.lib()


def test_header_declares_the_planned_entry_points():
    names = declared_functions()
    for n in ("hstu_jagged_attn_fwd", "hstu_jagged_attn_bwd", "hstu_cp_reorder",
              "hstu_cp_restore", "hstu_cp_paired_attn_fwd", "hstu_status_str",
              "hstu_jagged_attn_fwd_targets", "hstu_norm_gate_fwd", "hstu_norm_gate_bwd"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", hstu.lib_path], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT\s+(hstu_[a-z0-9_]+)\b", out))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, f"declared but not exported: {missing}"
    for n in declared_functions():
        assert hasattr(lib, n)
    assert set(hstu.EXPORTED_SYMBOLS) <= exported


def test_status_strings_and_version(lib):
    assert hstu.hstu_status_str(0) == "HSTU_OK"
    for code in range(-1, -10, -1):
        s = hstu.hstu_status_str(code)
        assert s.startswith("HSTU_ERR_")
    assert "unknown" in hstu.hstu_status_str(-99)
    assert hstu.hstu_version() >= 100


def test_workspace_size(lib):
    assert hstu.hstu_jagged_attn_bwd_workspace_bytes(1000, 4, 128) == 1000 * 4 * 128 * 4
    assert hstu.hstu_jagged_attn_bwd_workspace_bytes(3, 1, 32) == 512  # rounded to 256
    with pytest.raises(hstu.HstuError):
        hstu.hstu_jagged_attn_bwd_workspace_bytes(10, 2, 48)


def _fwd_raw(lib, **kw):
    a = dict(q=1 << 12, k=1 << 12, v=1 << 12, off=1 << 12, B=2, T=10, maxlen=0, ts=1 << 12,
             wp=1 << 12, P=4, wt=1 << 12, NB=8, H=2, dqk=64, dv=64, scale=0.125, f32=0,
             out=1 << 12, st=None, stream=None)
    a.update(kw)
    return lib.hstu_jagged_attn_fwd(a["q"], a["k"], a["v"], a["off"], a["B"], a["T"], a["maxlen"],
                                    a["ts"], a["wp"], a["P"], a["wt"], a["NB"], a["H"], a["dqk"],
                                    a["dv"], a["scale"], a["f32"], a["out"], a["st"], a["stream"])


def test_fwd_host_checks(lib):
    # these are rejected before any CUDA call, so they run without a GPU
    assert _fwd_raw(lib, dqk=48, dv=48) == -4
    assert _fwd_raw(lib, dqk=64, dv=128) == -4
    assert _fwd_raw(lib, H=0) == -2
    assert _fwd_raw(lib, B=-1) == -2
    assert _fwd_raw(lib, P=0) == -2
    assert _fwd_raw(lib, NB=0) == -2
    assert _fwd_raw(lib, T=1 << 31) == -2
    assert _fwd_raw(lib, off=None) == -1
    assert _fwd_raw(lib, q=None) == -1
    assert _fwd_raw(lib, q=(1 << 12) + 8) == -3   # q must be 16-byte aligned
    assert _fwd_raw(lib, ts=(1 << 12) + 4) == -3
    assert _fwd_raw(lib, out=None) == -1
    assert _fwd_raw(lib, T=0) == 0                # empty batch: nothing to launch
    assert _fwd_raw(lib, B=0) == 0


def _fwd_targets_raw(lib, **kw):
    a = dict(q=1 << 12, k=1 << 12, v=1 << 12, off=1 << 12, nt=1 << 12, B=2, T=10, maxlen=0,
             ts=1 << 12, wp=1 << 12, P=4, wt=1 << 12, NB=8, H=2, dqk=64, dv=64, scale=0.125,
             f32=0, out=1 << 12, st=None, stream=None)
    a.update(kw)
    return lib.hstu_jagged_attn_fwd_targets(a["q"], a["k"], a["v"], a["off"], a["nt"], a["B"],
                                            a["T"], a["maxlen"], a["ts"], a["wp"], a["P"],
                                            a["wt"], a["NB"], a["H"], a["dqk"], a["dv"],
                                            a["scale"], a["f32"], a["out"], a["st"], a["stream"])


def test_fwd_targets_host_checks(lib):
    # rejected before any CUDA call, so they run without a GPU
    assert _fwd_targets_raw(lib, nt=None) == -1
    assert _fwd_targets_raw(lib, nt=(1 << 12) + 4) == -3     # int64 counts, 8-byte aligned
    assert _fwd_targets_raw(lib, out=None) == -1
    assert _fwd_targets_raw(lib, dqk=48, dv=48) == -4
    assert _fwd_targets_raw(lib, P=3329, dqk=128, dv=128) == -4  # beyond the smem w_pos table
    assert _fwd_targets_raw(lib, P=4097, dqk=64, dv=64) == -4
    assert _fwd_targets_raw(lib, q=None) == -1
    assert _fwd_targets_raw(lib, T=0) == 0
    assert _fwd_targets_raw(lib, B=0) == 0


def test_cp_host_checks(lib):
    f = lib.hstu_cp_reorder
    assert f(1 << 12, 1 << 13, 1024, 1 << 14, 4, 100, 0, None, None, None, None) == -2  # C < 1
    assert f(1 << 12, 1 << 13, 0, 1 << 14, 4, 100, 2, None, None, None, None) == -2   # row_bytes
    assert f(1 << 12, 1 << 13, 8, None, 4, 100, 2, None, None, None, None) == -1
    assert f(None, 1 << 13, 8, 1 << 14, 4, 100, 2, None, None, None, None) == -1
    assert f(1 << 12, 1 << 13, 8, (1 << 14) + 4, 4, 100, 2, None, None, None, None) == -3
    assert f(1 << 12, 1 << 13, 8, 1 << 14, 0, 0, 2, None, None, None, None) == 0
    g = lib.hstu_cp_restore
    assert g(1 << 12, 1 << 13, 8, 1 << 14, 4, 100, 0, None, None) == -2
    assert g(1 << 12, None, 8, 1 << 14, 4, 100, 2, None, None) == -1


def test_bwd_host_checks(lib):
    f = lib.hstu_jagged_attn_bwd
    base = [1 << 12] * 4 + [2, 10, 0, 1 << 12, 1 << 12, 4, 1 << 12, 8, 2, 64, 64, 0.125]
    tail = [1 << 12] * 6 + [1 << 12, 1 << 20, None, None]
    args = base + tail
    bad_d = list(args)
    bad_d[13] = bad_d[14] = 96
    assert f(*bad_d) == -4
    no_dw = list(args)
    no_dw[21] = None   # dw_pos
    assert f(*no_dw) == -1


def test_product_path_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "jagged_hstu_attention_attn_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, fn)).read()
                assert "import oracle" not in text and "from oracle" not in text, fn
                assert "hstu_oracle" not in text and "liboracle" not in text, fn
    for fn in os.listdir(os.path.join(ROOT, "oracle")):
        if fn.endswith((".py", ".c")):
            text = open(os.path.join(ROOT, "oracle", fn)).read()
            assert not re.search(r"^\s*(import|from)\s+jagged_hstu_attention_attn_b200", text,
                                 flags=re.M), fn
            assert "libhstu.so" not in text and "CDLL(hstu" not in text, fn


def test_no_call_to_the_cuda_path_without_gpu():
    import torch
    if torch.cuda.is_available():
        pytest.skip("GPU present")
    x = torch.zeros(4, 1, 32, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        hstu.hstu_jagged_attn_fwd(x, x, x, torch.tensor([0, 4]), torch.zeros(4, dtype=torch.int64),
                                  torch.zeros(4), torch.zeros(8))
    with pytest.raises(ValueError):
        hstu.hstu_jagged_attn_fwd_targets(x, x, x, torch.tensor([0, 4]), torch.tensor([2]),
                                          torch.zeros(4, dtype=torch.int64), torch.zeros(4),
                                          torch.zeros(8))


def test_selftest_wait_timeout_host_checks(lib):
    # limit outside 1 us .. 1 s, or a missing status word: refused before any launch
    assert lib.hstu_selftest_wait_timeout(10, 1 << 12, 1 << 12, None) == -2
    assert lib.hstu_selftest_wait_timeout(2_000_000_000, 1 << 12, 1 << 12, None) == -2
    assert lib.hstu_selftest_wait_timeout(1_000_000, None, 1 << 12, None) == -1
    assert lib.hstu_selftest_wait_timeout(1_000_000, 1 << 12, None, None) == -1
    assert lib.hstu_selftest_wait_timeout(1_000_000, (1 << 12) + 2, 1 << 12, None) == -3


def test_norm_gate_host_checks(lib):
    import ctypes
    f32 = ctypes.c_float
    A = 1 << 12  # a 16-byte-aligned fake address: every case below is refused before a launch
    fwd, bwd = lib.hstu_norm_gate_fwd, lib.hstu_norm_gate_bwd
    # T = 0 launches nothing, whatever the pointers
    assert fwd(None, None, None, 0, 512, f32(1e-5), None) == 0
    assert bwd(None, None, None, None, None, 0, 512, f32(1e-5), None) == 0
    # N not a positive multiple of 8, negative T, eps <= 0 or not finite
    for T, N, eps in ((4, 12, 1e-5), (4, 0, 1e-5), (-1, 512, 1e-5), (4, 512, 0.0),
                      (4, 512, -1.0), (4, 512, float("inf")), (4, 512, float("nan"))):
        assert fwd(A, A * 2, A * 3, T, N, f32(eps), None) == -2, (T, N, eps)
        assert bwd(A, A * 2, A * 3, A * 4, A * 5, T, N, f32(eps), None) == -2, (T, N, eps)
    # N above 2048
    assert fwd(A, A * 2, A * 3, 4, 4096, f32(1e-5), None) == -4
    # missing and misaligned pointers
    assert fwd(None, A * 2, A * 3, 4, 512, f32(1e-5), None) == -1
    assert bwd(A, A * 2, A * 3, A * 4, None, 4, 512, f32(1e-5), None) == -1
    assert fwd(A + 8, A * 2, A * 3, 4, 512, f32(1e-5), None) == -3
    assert bwd(A, A * 2, A * 3, A * 4 + 2, A * 5, 4, 512, f32(1e-5), None) == -3
    # outputs overlapping inputs (rows of 1 KB: y at o + 1 KB overlaps o's second row)
    B = 1 << 20
    assert fwd(B, 2 * B, B + 1024, 4, 512, f32(1e-5), None) == -2
    assert fwd(B, 2 * B, 2 * B, 4, 512, f32(1e-5), None) == -2
    assert bwd(B, 2 * B, 3 * B, 4 * B, 4 * B + 1024, 4, 512, f32(1e-5), None) == -2
    assert bwd(B, 2 * B, 3 * B, 3 * B, 5 * B, 4, 512, f32(1e-5), None) == -2



def test_stochastic_length_host_checks(lib):
    A = 1 << 12  # aligned fake addresses; every case below is refused before a launch
    sel, gat = lib.hstu_sl_select, lib.hstu_gather_rows
    # L < 1, negative sizes, T at 2^31
    assert sel(A, 2, 10, A, A, 0, A, A, None, None) == -2
    assert sel(A, -1, 10, A, A, 5, A, A, None, None) == -2
    assert sel(A, 2, 1 << 31, A, A, 5, A, A, None, None) == -2
    # missing pointers
    assert sel(None, 2, 10, A, A, 5, A, A, None, None) == -1
    assert sel(A, 2, 10, None, A, 5, A, A, None, None) == -1
    assert sel(A, 2, 10, A, None, 5, A, A, None, None) == -1
    assert sel(A, 2, 10, A, A, 5, None, A, None, None) == -1
    # misaligned
    assert sel(A + 4, 2, 10, A, A, 5, A, A, None, None) == -3
    assert sel(A, 2, 10, A + 2, A, 5, A, A, None, None) == -3
    # gather: bad sizes, missing pointers, misaligned count, overlap
    assert gat(A, 10, 2 * A, 0, A, A, 10, None) == -2
    assert gat(A, -1, 2 * A, 8, A, A, 10, None) == -2
    assert gat(A, 10, 2 * A, 8, A, A, 0, None) == 0        # nothing to do
    assert gat(None, 10, 2 * A, 8, A, A, 10, None) == -1
    assert gat(A, 10, 2 * A, 8, A, A + 4, 10, None) == -3
    B = 1 << 20
    assert gat(B, 10, B + 40, 8, A, A, 10, None) == -2   # dst inside src


def test_gather_rows_multi_host_checks(lib):
    import ctypes
    A = 1 << 12
    arr = lambda *v: ctypes.cast((ctypes.c_void_p * len(v))(*v), ctypes.c_void_p)
    rb = lambda *v: ctypes.cast((ctypes.c_int64 * len(v))(*v), ctypes.c_void_p)
    f = lib.hstu_gather_rows_multi
    assert f(0, arr(A), arr(2 * A), rb(8), 10, A, A, 10, None) == -2      # count < 1
    assert f(9, arr(A), arr(2 * A), rb(8), 10, A, A, 10, None) == -2      # count > 8
    assert f(1, None, arr(2 * A), rb(8), 10, A, A, 10, None) == -1
    assert f(1, arr(A), arr(2 * A), rb(0), 10, A, A, 10, None) == -2      # row_bytes < 1
    assert f(1, arr(None), arr(2 * A), rb(8), 10, A, A, 10, None) == -1
    assert f(1, arr(A), arr(2 * A), rb(8), 10, A + 2, A, 10, None) == -3  # src_rows misaligned
    B = 1 << 20
    assert f(2, arr(B, 2 * B), arr(3 * B, 2 * B + 8), rb(8, 8), 10, A, A, 10, None) == -2
    assert f(1, arr(A), arr(2 * A), rb(8), 10, A, A, 0, None) == 0        # nothing to do
