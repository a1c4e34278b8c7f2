"""The prefill softmax's FMA-pipe exponential (pkv::tc::poly_exp2 in csrc/tcgen05_common.cuh).

CPU: its coefficients are re-derived here (minimax relative error of a cubic for 2^f on
[-1/2, 1/2] with p(0) = 1, a linear program over a dense grid) and must equal the
source's; a float32 emulation of the whole function (range reduction, Horner steps with
single-rounding fused multiply-adds, exponent add) is checked over [-126, 8] against
2^x in float64: relative error at most 1.05e-4, exact at integers, +0 at -127 and below.
GPU: the device function itself against CUDA's exp2f (torch.exp2) on the same grid.
"""
import ctypes
import os
import re
import shutil
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "paged_kv_cache_423_b200", "csrc")
REL_BOUND = 1.05e-4


def source_coefficients():
    with open(os.path.join(CSRC, "tcgen05_common.cuh")) as f:
        src = f.read()
    return [np.float32(float(re.search(rf"constexpr float kExp2C{k} = ([0-9.e+-]+)f;", src).group(1)))
            for k in (1, 2, 3)]


def minimax_fit():
    from scipy.optimize import linprog
    f = np.linspace(-0.5, 0.5, 20001)
    y = 2.0 ** f
    A = np.stack([f, f ** 2, f ** 3], 1) / y[:, None]
    r = 1 - 1 / y                       # p(f)/2^f - 1 = A c - r
    A_ub = np.vstack([np.hstack([A, -np.ones((len(f), 1))]), np.hstack([-A, -np.ones((len(f), 1))])])
    b_ub = np.concatenate([r, -r])
    res = linprog([0, 0, 0, 1], A_ub=A_ub, b_ub=b_ub, bounds=[(None, None)] * 3 + [(0, None)], method="highs")
    assert res.success
    return res.x[:3], res.x[3]


def emulate(x, c1, c2, c3):
    """poly_exp2 step by step in float32 (a fused multiply-add rounds once: the float32
    product is exact in float64)."""
    def fma(a, b, c):
        return (a.astype(np.float64) * b.astype(np.float64) + np.float64(c)).astype(np.float32)

    x = np.maximum(np.asarray(x, np.float32), np.float32(-127.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    f = (x - (t - magic).astype(np.float32)).astype(np.float32)
    p = fma(f, np.full_like(f, c3), c2)
    p = fma(p, f, c1)
    p = fma(p, f, 1.0)
    bits = (p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << np.uint64(23))) \
        & np.uint64(0xFFFFFFFF)
    return bits.astype(np.uint32).view(np.float32)


def grid():
    rng = np.random.default_rng(5)
    return np.concatenate([np.linspace(-126, 8, 400001), rng.uniform(-126, 8, 100000),
                           np.arange(-126, 9)]).astype(np.float32)


def test_coefficients_are_the_minimax_fit():
    c, err = minimax_fit()
    assert err < 1.02e-4
    got = source_coefficients()
    assert np.allclose(np.asarray(got, np.float64), c, rtol=0, atol=2e-7), (got, c)


def test_emulation_error_bound():
    c1, c2, c3 = source_coefficients()
    x = grid()
    y = emulate(x, c1, c2, c3).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y / ref - 1)
    assert rel.max() <= REL_BOUND, rel.max()
    ints = np.arange(-126, 9).astype(np.float32)
    assert np.array_equal(emulate(ints, c1, c2, c3).astype(np.float64), np.exp2(ints.astype(np.float64)))
    low = np.array([-127.0, -130.0, -1e30, -np.inf], np.float32)
    out = emulate(low, c1, c2, c3)
    assert np.all(out == 0) and not np.any(np.signbit(out))


def test_emulation_catches_a_wrong_coefficient():
    """The bound is tight enough that a slip in one coefficient (a truncated digit) fails it."""
    c1, c2, c3 = source_coefficients()
    x = grid()
    ref = np.exp2(x.astype(np.float64))
    for bad in ((np.float32(0.6931472), c2, c3), (c1, np.float32(0.2402265), c3), (c1, c2, np.float32(0.0555))):
        rel = np.abs(emulate(x, *bad).astype(np.float64) / ref - 1)
        assert rel.max() > REL_BOUND


@pytest.mark.gpu
def test_device_function_against_cuda_exp2(tmp_path):
    import torch
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    lib_path = tmp_path / "poly_exp2_probe.so"
    subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-I",
                    os.path.join(ROOT, "include"), "-I", CSRC, "-Xcompiler", "-fPIC", "-shared",
                    os.path.join(ROOT, "tests", "native", "poly_exp2_probe.cu"), "-o", str(lib_path)], check=True)
    lib = ctypes.CDLL(str(lib_path))
    lib.poly_exp2_probe.restype = ctypes.c_int
    lib.poly_exp2_probe.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p]
    x = torch.from_numpy(np.concatenate([grid(), np.array([-127, -200, -np.inf], np.float32)])).cuda()
    y = torch.empty_like(x)
    rc = lib.poly_exp2_probe(x.data_ptr(), y.data_ptr(), x.numel(), torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    ref = torch.exp2(x.double())
    n = x.numel() - 3
    rel = (y[:n].double() / ref[:n] - 1).abs()
    assert rel.max().item() <= REL_BOUND
    # and against CUDA's own single-precision exp2f, which is within a few ulp of 2^x
    rel_f = (y[:n].double() / torch.exp2(x[:n]).double() - 1).abs()
    assert rel_f.max().item() <= REL_BOUND + 2.0 ** -21
    # the device agrees with the float32 emulation (to one unit in the last place: the
    # emulation's fused multiply-add rounds through float64 first)
    c1, c2, c3 = source_coefficients()
    ulps = np.abs(y[:n].cpu().numpy().view(np.int32).astype(np.int64)
                  - emulate(x[:n].cpu().numpy(), c1, c2, c3).view(np.int32).astype(np.int64))
    assert ulps.max() <= 1
    assert torch.all(y[n:] == 0)
