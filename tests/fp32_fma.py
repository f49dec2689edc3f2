"""Exact IEEE binary32 fused multiply-add, vectorised in numpy (test helper).

numpy has no fma.  For binary32 operands a and b the product a*b has at most
48 significant bits, so it is exact in binary64.  The sum p + c is then
formed in binary64 and its rounding error recovered exactly with Knuth's
TwoSum.  Rounding that sum to binary64 "to odd" (keep it if its last bit is
odd or the error is zero, else step one ulp towards the error) and then
rounding the result to binary32 to nearest even gives the correctly rounded
binary32 fma: rounding to odd at p >= q + 2 bits followed by rounding to
nearest at q bits equals one rounding to nearest at q bits (Boldo and
Melquiond, "Emulation of FMA and correctly rounded sums: proved algorithms
using rounding to odd", IEEE Trans. Computers 57(4), 2008).  Here p = 53 and
q = 24.

bf16 rounding to nearest even from binary32 bits is the usual carry trick on
the upper 16 bits.  Both are pinned on the CPU against libm's fmaf and
torch's bfloat16 cast by tests/test_fp32_fma.py.
"""
from __future__ import annotations

import numpy as np


def fmaf(a, b, c) -> np.ndarray:
    """Correctly rounded binary32 a*b + c for finite binary32 arrays."""
    a64 = np.asarray(a, np.float32).astype(np.float64)
    b64 = np.asarray(b, np.float32).astype(np.float64)
    c64 = np.asarray(c, np.float32).astype(np.float64)
    p = a64 * b64                      # exact
    s = p + c64
    bb = s - p
    err = (p - (s - bb)) + (c64 - bb)  # s + err == p + c exactly
    bits = s.view(np.uint64)
    even = (bits & np.uint64(1)) == 0
    step = (err != 0) & even
    towards = np.where(err > 0, np.inf, -np.inf)
    s_odd = np.where(step, np.nextafter(s, towards), s)
    return s_odd.astype(np.float32)


def bf16_bits_rne(f32: np.ndarray) -> np.ndarray:
    """binary32 -> bfloat16 bits, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(f32, np.float32).view(np.uint32).astype(np.uint64)
    u = u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))
    return (u >> np.uint64(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)
