"""CPU pins of the test-side binary32 fma emulation (tests/fp32_fma.py)
against glibc's fmaf, which is correctly rounded, and of the bf16 rounding
against torch's bfloat16 cast."""
import ctypes
import ctypes.util

import numpy as np
import torch

import fp32_fma


def _libm_fmaf():
    lib = ctypes.CDLL(ctypes.util.find_library("m") or "libm.so.6")
    f = lib.fmaf
    f.restype = ctypes.c_float
    f.argtypes = [ctypes.c_float, ctypes.c_float, ctypes.c_float]
    return f


def test_fmaf_matches_libm_on_random_and_hard_cases():
    f = _libm_fmaf()
    rng = np.random.default_rng(0)
    n = 40000
    a = rng.standard_normal(n).astype(np.float32)
    # bf16-valued multiplicands, as combine's Y rows are
    b = fp32_fma.bf16_bits_to_f32(fp32_fma.bf16_bits_rne(rng.standard_normal(n).astype(np.float32)))
    c = (rng.standard_normal(n) * 10.0 ** rng.integers(-8, 8, n)).astype(np.float32)
    # hard cases: c cancels a*b almost exactly, and sums that land on or near
    # binary32 midpoints
    m = n // 4
    c[:m] = (-(a[:m].astype(np.float64) * b[:m])).astype(np.float32)
    half = np.spacing(np.abs(c[m:2 * m])).astype(np.float64) / 2
    a[m:2 * m] = np.float32(1.0)
    b[m:2 * m] = (half * rng.choice([-1.0, 1.0], m)).astype(np.float32)
    got = fp32_fma.fmaf(a, b, c)
    want = np.array([f(float(x), float(y), float(z)) for x, y, z in zip(a, b, c)], np.float32)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))


def test_fmaf_differs_from_two_roundings_somewhere():
    """The emulation is a single rounding: on cases built to sit just past a
    binary32 midpoint it differs from round(round(a*b) + c)."""
    rng = np.random.default_rng(1)
    n = 20000
    a = (1.0 + rng.integers(1, 2 ** 12, n) * 2.0 ** -12).astype(np.float32)
    b = (1.0 + rng.integers(1, 2 ** 12, n) * 2.0 ** -12).astype(np.float32)
    c = rng.standard_normal(n).astype(np.float32)
    two = (a * b).astype(np.float32) + c
    one = fp32_fma.fmaf(a, b, c)
    assert (one != two).any()


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(2)
    x = (rng.standard_normal(100000) * 10.0 ** rng.integers(-20, 20, 100000)).astype(np.float32)
    # exact bf16 midpoints in both tie directions
    mid = (np.arange(1000, dtype=np.uint32) << np.uint32(16)) | np.uint32(0x8000)
    x = np.concatenate([x, (mid + np.uint32(0x3F800000)).view(np.float32)])
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(fp32_fma.bf16_bits_rne(x), want)
