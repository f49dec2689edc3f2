"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each pin takes an ``oracle.Oracle`` and raises AssertionError when the oracle
disagrees with brute force, a closed form, an invariant, a hand-worked example
(tests/golden/hand_example.json) or a library routine.  ``test_oracle_pins``
runs them on the committed oracle; ``test_oracle_mutants`` runs them on
deliberately broken copies of it and expects at least one to fail each time.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_example.json")


def _rng(seed=0):
    return np.random.default_rng(seed)


def _tie_free_logits(n, e, seed=0):
    # distinct values per row: a random permutation of a spread grid plus noise
    r = _rng(seed)
    base = np.stack([r.permutation(e) for _ in range(n)]).astype(np.float64)
    return (base * 0.37 + r.uniform(-0.1, 0.1, (n, e))).astype(np.float32)


# ------------------------------------------------------------------ router
def _bf16_of(a: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16) \
        .view(torch.int16).numpy().view(np.uint16)


def _bf16_f64(b: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(torch.bfloat16) \
        .double().numpy()


def pin_router_logits_exact_integers(o):
    """Small integer-valued bf16 operands make every product and partial sum
    exact: the logits equal numpy's integer matmul (library) bit for bit,
    on shapes where E != D so that a transposed operand cannot pass."""
    r = _rng(11)
    for (n, d, e) in [(5, 96, 8), (17, 256, 64), (3, 1024, 256)]:
        xi = r.integers(-8, 9, (n, d))
        wi = r.integers(-8, 9, (e, d))
        got = o.router_logits(_bf16_of(xi), _bf16_of(wi))
        assert np.array_equal(got, (xi @ wi.T).astype(np.float32)), (n, d, e)


def pin_router_logits_matmul(o):
    """Gaussian operands at the router's sizes: the logits are numpy's float64
    matmul (library) of the decoded bf16 operands rounded to fp32 -- equal
    except where the two double sums straddle an fp32 rounding point, and
    never more than one fp32 ulp apart."""
    r = _rng(12)
    for (n, d, e) in [(32, 7168, 64), (16, 4096, 128)]:
        xb = _bf16_of(r.standard_normal((n, d)))
        wb = _bf16_of(r.standard_normal((e, d)) * 0.02)
        got = o.router_logits(xb, wb).astype(np.float64)
        ref64 = _bf16_f64(xb) @ _bf16_f64(wb).T
        ref = ref64.astype(np.float32).astype(np.float64)
        ulp = np.spacing(np.abs(ref).astype(np.float32)).astype(np.float64)
        assert np.all(np.abs(got - ref) <= ulp), (n, d, e)
        assert np.mean(got == ref) > 0.99, (n, d, e)


# ------------------------------------------------------------------ route
def pin_route_bruteforce(o):
    """Top-k = first k of the full sort of (-logit, id): brute force, with ties."""
    r = _rng(1)
    for (n, e, k) in [(37, 8, 2), (20, 16, 5), (9, 6, 6), (12, 32, 1)]:
        # coarse grid -> many exact ties
        logits = r.integers(-3, 4, size=(n, e)).astype(np.float32) * 0.5
        idx, _ = o.route(logits, k)
        for t in range(n):
            ref = sorted(range(e), key=lambda ex: (-float(logits[t, ex]), ex))[:k]
            assert list(idx[t]) == ref, (n, e, k, t, list(idx[t]), ref)


def pin_route_torch_topk(o):
    """On tie-free rows the selection equals torch.topk (a library routine)."""
    for (n, e, k) in [(64, 8, 2), (50, 256, 8), (40, 128, 4)]:
        logits = _tie_free_logits(n, e, seed=n + e)
        idx, _ = o.route(logits, k)
        ref = torch.topk(torch.from_numpy(logits), k, dim=1, sorted=True).indices.numpy()
        assert np.array_equal(idx, ref)


def pin_route_special_cases(o):
    """All-equal logits pick experts 0..k-1 with weight 1/k; k=1 gives weight 1;
    k=E returns every expert in descending logit order."""
    logits = np.full((3, 8), 0.25, np.float32)
    idx, w = o.route(logits, 3)
    assert np.array_equal(idx, np.tile(np.arange(3), (3, 1)))
    assert np.all(w == np.float32(1.0 / 3.0))
    logits = _tie_free_logits(10, 16, seed=5)
    idx, w = o.route(logits, 1)
    assert np.array_equal(idx[:, 0], logits.argmax(1)) and np.all(w == 1.0)
    idx, w = o.route(logits, 16)
    assert np.array_equal(idx, np.argsort(-logits, axis=1, kind="stable"))


def pin_route_weights_closed_form(o):
    """k=2: w0 = 1/(1+exp(L1-L0)) (the logistic form); general k: softmax of
    the selected logits via scipy; weights sum to 1 and do not increase in j."""
    from scipy.special import softmax
    logits = _tie_free_logits(40, 8, seed=7) * 3.0
    idx, w = o.route(logits, 2)
    for t in range(40):
        l0, l1 = float(logits[t, idx[t, 0]]), float(logits[t, idx[t, 1]])
        ref0 = 1.0 / (1.0 + math.exp(l1 - l0))
        assert abs(float(w[t, 0]) - ref0) <= 2 ** -24 * ref0 * 2
        assert abs(float(w[t, 1]) - (1.0 - ref0)) <= 2 ** -24 * 2
    logits = _tie_free_logits(30, 64, seed=8) * 2.0
    idx, w = o.route(logits, 6)
    sel = np.take_along_axis(logits.astype(np.float64), idx.astype(np.int64), axis=1)
    ref = softmax(sel, axis=1)
    assert np.allclose(w, ref, rtol=2 ** -22, atol=0)
    assert np.allclose(w.astype(np.float64).sum(1), 1.0, atol=1e-6)
    assert np.all(np.diff(w, axis=1) <= 0)


# ------------------------------------------------------------------ layout
def pin_counts_bincount(o):
    """counts = numpy bincount of the flattened picks; they sum to N*k."""
    logits = _tie_free_logits(100, 16, seed=9)
    idx, _ = o.route(logits, 4)
    c = o.counts(idx, 16)
    assert np.array_equal(c, np.bincount(idx.ravel(), minlength=16))
    assert c.sum() == 100 * 4


def pin_offsets(o):
    """R=1: exclusive prefix sum (numpy cumsum).  R>1: each rank's experts
    start at the fixed base r*N*min(k,E/R) and are packed inside it."""
    r = _rng(3)
    for (n, e, k, ranks) in [(50, 16, 4, 1), (50, 16, 4, 4), (33, 8, 4, 4), (7, 12, 3, 3)]:
        idx = np.stack([r.permutation(e)[:k] for _ in range(n)]).astype(np.int32)
        c = o.counts(idx, e)
        off = o.offsets(n, e, k, ranks, c)
        per = e // ranks
        c_r = n * min(k, per)
        assert o.region_rows(n, e, k, ranks) == c_r
        assert off[e] == ranks * c_r
        for rank in range(ranks):
            lo = rank * per
            seg = off[lo:lo + per]
            ref = rank * c_r + np.concatenate([[0], np.cumsum(c[lo:lo + per])[:-1]])
            assert np.array_equal(seg, ref)
            assert seg[-1] + c[lo + per - 1] <= (rank + 1) * c_r
    # worst case: every token sends min(k, E/R) rows to rank 0 -> exactly fills it
    n, e, k, ranks = 5, 8, 4, 4
    idx = np.tile(np.array([0, 1, 2, 3], np.int32), (n, 1))
    c = o.counts(idx, e)
    off = o.offsets(n, e, k, ranks, c)
    assert off[1] + c[1] == o.region_rows(n, e, k, ranks) == off[2]


def pin_slots_stable_sort(o):
    """R=1: slot order is the stable argsort of the flattened picks (the sorted
    gather path); any R: brute-force count of earlier tokens per expert, the
    map is a bijection onto the filled slots and src_of inverts slot_of."""
    r = _rng(4)
    for (n, e, k, ranks) in [(60, 8, 2, 1), (60, 8, 2, 2), (45, 16, 4, 4), (10, 4, 4, 2)]:
        idx = np.stack([r.permutation(e)[:k] for _ in range(n)]).astype(np.int32)
        c = o.counts(idx, e)
        off = o.offsets(n, e, k, ranks, c)
        slot_of, src_of = o.slots(idx, off, e)
        if ranks == 1:
            order = np.argsort(idx.ravel(), kind="stable")
            assert np.array_equal(src_of[: n * k], order)
        for t in range(n):
            for j in range(k):
                ex = idx[t, j]
                earlier = sum(1 for t2 in range(t) if ex in idx[t2])
                assert slot_of[t, j] == off[ex] + earlier
        flat = slot_of.ravel()
        assert len(np.unique(flat)) == n * k
        assert np.array_equal(src_of[flat], np.arange(n * k))
        filled = np.zeros(src_of.size, bool)
        filled[flat] = True
        assert np.all(src_of[~filled] == -1)


def pin_dispatch_repeat_interleave(o):
    """recv gathered at slot_of equals x.repeat_interleave(k) (the unsorted
    path); every source row appears exactly k times; unfilled rows are zero."""
    r = _rng(5)
    n, e, k, ranks, d = 40, 8, 3, 2, 24
    idx = np.stack([r.permutation(e)[:k] for _ in range(n)]).astype(np.int32)
    x = r.standard_normal((n, d)).astype(np.float32)
    c = o.counts(idx, e)
    off = o.offsets(n, e, k, ranks, c)
    slot_of, src_of = o.slots(idx, off, e)
    recv = o.scatter_rows(x, slot_of, int(off[e]))
    ref = torch.from_numpy(x).repeat_interleave(k, dim=0).numpy()
    assert np.array_equal(recv[slot_of.ravel()], ref)
    filled = src_of >= 0
    assert np.all(recv[~filled] == 0)
    # bytes too: a bf16 and an fp8 payload travel unchanged
    xb = r.integers(0, 2 ** 16, size=(n, d), dtype=np.uint16)
    rb = o.scatter_rows(xb, slot_of, int(off[e]))
    assert np.array_equal(rb[slot_of.ravel()], np.repeat(xb, k, axis=0))


# ------------------------------------------------------------------ numbers
def pin_e4m3_decode(o):
    """All 256 e4m3 codes decode as torch.float8_e4m3fn does (library)."""
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([o.e4m3_to_float(c) for c in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def pin_bf16_rounding(o):
    """Round-to-nearest-even to bf16: hand cases (ties, subnormals, overflow)
    and agreement with torch's float32 -> bfloat16 cast on random floats."""
    assert o.bf16_from_float(1.0) == 0x3F80
    assert o.bf16_from_float(1.0 + 2 ** -8) == 0x3F80          # tie -> even
    assert o.bf16_from_float(1.0 + 3 * 2 ** -8) == 0x3F82      # tie -> even (up)
    assert o.bf16_from_float(1.0 + 2 ** -8 + 2 ** -30) == 0x3F81
    assert o.bf16_from_float(-2.0) == 0xC000
    assert o.bf16_from_float(2 ** -133) == 0x0001              # smallest subnormal
    assert o.bf16_from_float(2 ** -134) == 0x0000              # tie -> even (zero)
    assert o.bf16_from_float(1.5 * 2 ** -133) == 0x0002        # tie -> even (up)
    assert o.bf16_from_float(3.0e38) == 0x7F62
    assert o.bf16_from_float(3.4e38) == 0x7F80                 # overflow -> inf
    assert o.bf16_from_float(float("inf")) == 0x7F80
    r = _rng(6)
    f = np.concatenate([r.standard_normal(4000) * 10.0 ** r.integers(-30, 30, 4000),
                        r.standard_normal(1000)]).astype(np.float32)
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    got = np.array([o.bf16_from_float(float(v)) for v in f], np.uint16)
    assert np.array_equal(got, ref)
    # decode is exact widening
    bits = r.integers(0, 0x7F80, 500).astype(np.uint16)
    ref = torch.from_numpy(bits.astype(np.int16)).view(torch.bfloat16).double().numpy()
    got = np.array([o.bf16_to_float(int(b)) for b in bits])
    assert np.array_equal(got, ref)


def pin_dequant(o):
    """Identity expert on FP8 rows: with power-of-two scales code*scale is exact,
    so it equals torch's e4m3 -> float -> bf16 cast bit for bit; with general
    scales it is within half a bf16 ulp of the exact double product."""
    r = _rng(7)
    t, d, blk = 6, 256, 128
    q = r.integers(0, 256, size=(t, d), dtype=np.uint8)
    q[(q & 0x7F) == 0x7F] = 0x11           # no NaN codes
    scale = (2.0 ** r.integers(-8, 8, size=(t, d // blk))).astype(np.float32)
    rows = np.arange(t, dtype=np.int32)
    y = o.dequant_rows(rows, q, scale, blk)
    qf = torch.from_numpy(q).view(torch.float8_e4m3fn).float()
    ref = (qf * torch.from_numpy(np.repeat(scale, blk, axis=1))).to(torch.bfloat16)
    assert np.array_equal(y, ref.view(torch.int16).numpy().astype(np.uint16))
    scale = r.uniform(0.001, 3.0, size=(t, d // blk)).astype(np.float32)
    y = o.dequant_rows(rows, q, scale, blk)
    exact = (qf.double() * torch.from_numpy(np.repeat(scale, blk, axis=1)).double()).numpy()
    yv = o.to_float(y, "bf16")
    ulp = np.where(exact != 0, 2.0 ** (np.floor(np.log2(np.abs(exact) + 1e-300)) - 7), 0)
    assert np.all(np.abs(yv - exact) <= 0.5 * ulp + 1e-300)
    # rows not listed stay untouched (zero)
    y2 = o.dequant_rows(np.array([1], np.int32), q, scale, blk)
    assert np.all(y2[0] == 0) and np.array_equal(y2[1], y[1])


def _bf16_bits(a: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16) \
        .view(torch.int16).numpy().astype(np.uint16)


def _bf16_val(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def pin_swiglu_dense(o):
    """One expert holding every row reduces to a dense SwiGLU MLP, computed
    here with numpy float64 matmuls (library); zero weights give zero output;
    the expert id selects the weights."""
    r = _rng(8)
    rows_n, d, inter, e = 9, 64, 48, 3
    x = _bf16_bits(r.standard_normal((rows_n, d)))
    wgu = _bf16_bits(r.standard_normal((e, 2 * inter, d)) * 0.1)
    wd = _bf16_bits(r.standard_normal((e, d, inter)) * 0.1)
    rows = np.arange(rows_n, dtype=np.int32)
    for ex in range(e):
        y, h = o.swiglu_rows(rows, np.full(rows_n, ex, np.int32), x, wgu, wd, want_h=True)
        xv = _bf16_val(x)
        g = xv @ _bf16_val(wgu[ex, :inter]).T
        u = xv @ _bf16_val(wgu[ex, inter:]).T
        h_ref = g / (1.0 + np.exp(-g)) * u
        hv = _bf16_val(h)
        assert np.all(np.abs(hv - h_ref) <= np.abs(h_ref) * 2 ** -8 + 1e-30)
        y_ref = hv @ _bf16_val(wd[ex]).T
        yv = _bf16_val(y)
        assert np.all(np.abs(yv - y_ref) <= np.abs(y_ref) * 2 ** -8 + 1e-30)
    # mixed experts per row pick the right weights
    re = (np.arange(rows_n) % e).astype(np.int32)
    ymix = o.swiglu_rows(rows, re, x, wgu, wd)
    for i in range(rows_n):
        yi = o.swiglu_rows(np.array([i], np.int32), np.array([re[i]], np.int32), x, wgu, wd)
        assert np.array_equal(ymix[i], yi[i])
    yz = o.swiglu_rows(rows, re, x, np.zeros_like(wgu), wd)
    assert np.all(_bf16_val(yz) == 0)


# ------------------------------------------------------------------ FP8 experts
def _e4m3_val(q: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(q)).view(torch.float8_e4m3fn).double().numpy()


def _fp8_codes(r, shape):
    q = r.integers(0, 256, size=shape, dtype=np.uint8)
    q[(q & 0x7F) == 0x7F] = 0x3C            # no NaN codes
    return q


def _distinct_pow2(r, shape, lo):
    """Scales that are distinct powers of two, so that any mix-up of two
    blocks' scales changes a result."""
    count = int(np.prod(shape))
    return (2.0 ** (lo - r.permutation(count))).reshape(shape).astype(np.float32)


def pin_e4m3_encode(o):
    """fp32 -> e4m3, nearest with ties to even and saturation at +-448: hand
    cases (ties, subnormals, signed zero, overflow) and torch's
    float8_e4m3fn cast (library) on random values inside the finite range."""
    cases = [(1.0, 0x38), (1.0625, 0x38), (1.1875, 0x3A), (-1.75, 0xBE), (448.0, 0x7E),
             (464.0, 0x7E), (500.0, 0x7E), (1e30, 0x7E), (-500.0, 0xFE), (2.0 ** -9, 0x01),
             (2.0 ** -10, 0x00), (3 * 2.0 ** -10, 0x02), (0.0, 0x00), (-0.0, 0x80),
             (2.0 ** -6, 0x08), (0.875 * 2.0 ** -6, 0x07)]
    for v, code in cases:
        assert o.e4m3_from_float(v) == code, (v, hex(o.e4m3_from_float(v)), hex(code))
    r = _rng(10)
    f = np.concatenate([r.uniform(-448, 448, 3000),
                        r.choice([-1, 1], 3000) * 2.0 ** r.uniform(-12, 8.8, 3000)])
    f = f.astype(np.float32)
    ref = torch.from_numpy(f).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([o.e4m3_from_float(float(v)) for v in f], np.uint8)
    assert np.array_equal(got, ref)


def pin_quant_rows(o):
    """H quantisation: the scale is the fp32 quotient amax / 448 (numpy
    float32 division, IEEE), the codes are torch's e4m3 cast of the fp32
    quotients h / scale; an all-zero block gets scale 1 and zero codes; rows
    not listed stay untouched."""
    r = _rng(11)
    t, w, blk = 5, 384, 128
    h = _bf16_bits(r.standard_normal((t, w)) * 10.0 ** r.integers(-3, 3, (t, 1)))
    h[2, 128:256] = 0
    h[3, :128] = _bf16_bits(np.linspace(-448, 448, 128))     # amax 448: scale 1
    rows = np.arange(t, dtype=np.int32)
    q, sc = o.quant_rows(rows, h, blk)
    hv = _bf16_val(h).astype(np.float32)                       # exact: bf16 is a subset
    amax = np.abs(hv).reshape(t, w // blk, blk).max(axis=2)
    sc_ref = np.where(amax > 0, amax / np.float32(448), np.float32(1)).astype(np.float32)
    assert np.array_equal(sc, sc_ref)
    assert sc[2, 1] == 1.0 and np.all(q[2, 128:256] == 0) and sc[3, 0] == 1.0
    quo = (hv.reshape(t, w // blk, blk) / sc_ref[:, :, None]).astype(np.float32).reshape(t, w)
    ref = torch.from_numpy(np.clip(quo, -448, 448)).to(torch.float8_e4m3fn).view(torch.uint8)
    assert np.array_equal(q, ref.numpy())
    q1, sc1 = o.quant_rows(np.array([4], np.int32), h, blk)
    assert np.all(q1[:4] == 0) and np.all(sc1[:4] == 0) and np.array_equal(q1[4], q[4])


def pin_fp8_gate_up_dense(o):
    """FP8 GEMM1 + SwiGLU against numpy float64 matmuls (library) of operands
    dequantised here, the weight scale grid expanded with np.kron: g and u
    agree to double rounding, h = bf16(silu(g) u) to half a bf16 ulp.  The
    scales are distinct powers of two, so a wrong block index, a dropped
    scale or the gate's scale on the up rows fails."""
    r = _rng(12)
    rows_n, d, inter, e, blk = 5, 256, 256, 2, 128
    xq = _fp8_codes(r, (rows_n, d))
    xs = _distinct_pow2(r, (rows_n, d // blk), -2)
    wq = _fp8_codes(r, (e, 2 * inter, d))
    ws = _distinct_pow2(r, (e, 2 * inter // blk, d // blk), -4)
    rows = np.arange(rows_n, dtype=np.int32)
    xv = _e4m3_val(xq) * np.repeat(xs.astype(np.float64), blk, axis=1)
    for ex in range(e):
        h, g, u = o.fp8_gate_up_rows(rows, np.full(rows_n, ex, np.int32), xq, xs, wq, ws, blk,
                                     want_gu=True)
        wv = _e4m3_val(wq[ex]) * np.kron(ws[ex].astype(np.float64), np.ones((blk, blk)))
        g_ref, u_ref = xv @ wv[:inter].T, xv @ wv[inter:].T
        g_abs, u_abs = np.abs(xv) @ np.abs(wv[:inter]).T, np.abs(xv) @ np.abs(wv[inter:]).T
        assert np.all(np.abs(g - g_ref) <= 1e-12 * g_abs)
        assert np.all(np.abs(u - u_ref) <= 1e-12 * u_abs)
        with np.errstate(over="ignore"):
            h_ref = g / (1.0 + np.exp(-g)) * u
        # half a bf16 ulp: 2^-8 relative, or half the subnormal quantum 2^-133
        assert np.all(np.abs(_bf16_val(h) - h_ref) <= np.abs(h_ref) * 2 ** -8 + 2.0 ** -134)


def pin_fp8_down_dense(o):
    """FP8 GEMM2 against a numpy float64 matmul (library) of operands
    dequantised here (row scales by np.repeat, weight tiles by np.kron), with
    distinct power-of-two scales; y within half a bf16 ulp; the expert id
    selects the weights."""
    r = _rng(13)
    rows_n, d, inter, e, blk = 6, 256, 384, 3, 128
    hq = _fp8_codes(r, (rows_n, inter))
    hs = _distinct_pow2(r, (rows_n, inter // blk), 0)
    wq = _fp8_codes(r, (e, d, inter))
    ws = _distinct_pow2(r, (e, d // blk, inter // blk), -6)
    rows = np.arange(rows_n, dtype=np.int32)
    re = (np.arange(rows_n) % e).astype(np.int32)
    y = o.fp8_down_rows(rows, re, hq, hs, wq, ws, blk)
    hv = _e4m3_val(hq) * np.repeat(hs.astype(np.float64), blk, axis=1)
    for i in range(rows_n):
        wv = _e4m3_val(wq[re[i]]) * np.kron(ws[re[i]].astype(np.float64), np.ones((blk, blk)))
        y_ref = wv @ hv[i]
        assert np.all(np.abs(_bf16_val(y[i]) - y_ref) <= np.abs(y_ref) * 2 ** -8 + 2.0 ** -134)


def pin_fp8_gate_up_equals_bf16_with_unit_scales(o):
    """With every scale 1 the FP8 gate/up step is the (separately pinned) bf16
    SwiGLU step on the decoded values, bit for bit: every e4m3 value is a bf16
    value, and both sum the same products in the same order."""
    r = _rng(14)
    rows_n, d, inter, blk = 4, 256, 128, 128
    xq = _fp8_codes(r, (rows_n, d))
    wq = _fp8_codes(r, (1, 2 * inter, d))
    rows = np.arange(rows_n, dtype=np.int32)
    ex = np.zeros(rows_n, np.int32)
    h8 = o.fp8_gate_up_rows(rows, ex, xq, np.ones((rows_n, d // blk), np.float32), wq,
                            np.ones((1, 2 * inter // blk, d // blk), np.float32), blk)
    as_bf16 = lambda q: _bf16_bits(_e4m3_val(q))  # noqa: E731  (exact)
    _, h16 = o.swiglu_rows(rows, ex, as_bf16(xq), as_bf16(wq), np.zeros((1, d, inter), np.uint16),
                           want_h=True)
    assert np.array_equal(h8, h16)


def pin_run_path_fp8_layer(o):
    """The composed FP8 expert path keeps its invariants: H codes times their
    scale reproduce H to within half an e4m3 step of the block, every block
    scale is its amax / 448, Y equals the down projection of the quantised H,
    and rows outside the filled slots stay zero."""
    import workloads
    cfg = workloads.CONFIGS["layer_fp8"].replace(n=24, hidden=256, inter=256, n_experts=4,
                                                 top_k=2, n_ranks=2)
    inp = {kk: workloads.as_numpy_bits(v) for kk, v in workloads.make_inputs(cfg).items()}
    res = o.run_path(cfg, inp)
    fs = np.sort(res["slot_of"].reshape(-1))
    hv = _bf16_val(res["h"][fs])
    dq = _e4m3_val(res["hq"][fs]) * np.repeat(res["h_scale"][fs].astype(np.float64), 128, axis=1)
    amax = np.abs(hv).reshape(len(fs), -1, 128).max(axis=2)
    sc = res["h_scale"][fs].astype(np.float64)
    assert np.allclose(sc, np.where(amax > 0, amax / 448.0, 1.0), rtol=2 ** -23, atol=0)
    # an e4m3 step is at most 2^-3 of the value (normal) or 2^-9 of the block scale (subnormal)
    step = np.maximum(np.abs(hv) * 2.0 ** -3, np.repeat(sc, 128, axis=1) * 2.0 ** -9)
    assert np.all(np.abs(dq - hv) <= 0.5 * step + 1e-300)
    expert = res["topk_idx"].reshape(-1)[res["src_of"][fs]]
    y = o.fp8_down_rows(fs, expert, res["hq"], res["h_scale"], inp["w_down"], inp["w_down_scale"])
    assert np.array_equal(y[fs], res["y"][fs])
    unfilled = np.setdiff1d(np.arange(res["y"].shape[0]), fs)
    assert np.all(res["y"][unfilled] == 0) and np.all(res["hq"][unfilled] == 0)


# ------------------------------------------------------------------ combine
def pin_combine_identity_roundtrip(o):
    """combine(dispatch(x)) with identity experts and renormalised weights is
    x * sum(w) = x: within 1e-6 in fp32 and bit-exact after bf16 rounding."""
    r = _rng(9)
    n, e, k, ranks, d = 70, 16, 4, 4, 32
    logits = r.standard_normal((n, e)).astype(np.float32)
    idx, w = o.route(logits, k)
    c = o.counts(idx, e)
    off = o.offsets(n, e, k, ranks, c)
    slot_of, _ = o.slots(idx, off, e)
    x = r.standard_normal((n, d)).astype(np.float32)
    recv = o.scatter_rows(x, slot_of, int(off[e]))
    out = o.combine(recv, "f32", w, slot_of, "f32")
    assert np.allclose(out, x, rtol=1e-6, atol=0)
    xb = _bf16_bits(x)
    recvb = o.scatter_rows(xb, slot_of, int(off[e]))
    outb = o.combine(recvb, "bf16", w, slot_of, "bf16")
    assert np.array_equal(outb, xb)


def pin_combine_einsum(o):
    """Weighted sum equals numpy's einsum over the gathered rows (float64,
    then one rounding to fp32), element for element."""
    r = _rng(10)
    n, k, d, total = 25, 3, 40, 90
    y = r.standard_normal((total, d)).astype(np.float32)
    slot_of = np.stack([r.choice(total, k, replace=False) for _ in range(n)]).astype(np.int32)
    w = r.uniform(0, 1, (n, k)).astype(np.float32)
    out = o.combine(y, "f32", w, slot_of, "f32")
    ref = np.einsum("tj,tjd->td", w.astype(np.float64), y.astype(np.float64)[slot_of])
    assert np.array_equal(out, ref.astype(np.float32))
    ab = o.combine_abs(y, "f32", w, slot_of)
    assert np.allclose(ab, np.einsum("tj,tjd->td", w.astype(np.float64),
                                     np.abs(y.astype(np.float64))[slot_of]), rtol=1e-15)


def pin_hand_example(o):
    """The hand-worked example in tests/golden/hand_example.json."""
    with open(GOLDEN) as f:
        g = json.load(f)
    logits = np.array(g["logits"], np.float32)
    k, e = g["top_k"], g["n_experts"]
    idx, w = o.route(logits, k)
    assert idx.tolist() == g["topk_idx"]
    assert np.allclose(w, np.array(g["topk_w"]), rtol=0, atol=1e-7)
    c = o.counts(idx, e)
    assert c.tolist() == g["counts"]
    x = np.array(g["x"], np.float32)
    for lay in g["layouts"]:
        off = o.offsets(g["n"], e, k, lay["n_ranks"], c)
        assert off.tolist() == lay["expert_off"]
        assert o.region_rows(g["n"], e, k, lay["n_ranks"]) == lay["region_rows"]
        slot_of, src_of = o.slots(idx, off, e)
        assert slot_of.tolist() == lay["slot_of"]
        assert src_of.tolist() == lay["src_of"]
        total = int(off[e])
        ys = np.stack([np.arange(total), -np.arange(total)], 1).astype(np.float32)
        out = o.combine(ys, "f32", w, slot_of, "f32")
        assert np.allclose(out, np.array(lay["combine_with_y_slot"]), rtol=1e-6, atol=1e-6)
        recv = o.scatter_rows(x, slot_of, total)
        assert np.allclose(o.combine(recv, "f32", w, slot_of, "f32"), x, rtol=1e-6)


def pin_run_path_tiny(o):
    """The composed path on the tiny workload keeps every invariant: counts sum
    to N*k, the slot map is a bijection, recv holds k copies of each row, and
    combine(dispatch(x)) returns x."""
    import workloads
    cfg = workloads.CONFIGS["tiny"]
    inp = {kk: workloads.as_numpy_bits(v) for kk, v in workloads.make_inputs(cfg).items()}
    res = o.run_path(cfg, inp)
    assert res["counts"].sum() == cfg.n * cfg.top_k
    flat = res["slot_of"].ravel()
    assert len(np.unique(flat)) == flat.size
    assert np.array_equal(res["recv"][flat], np.repeat(inp["x"], cfg.top_k, axis=0))
    assert np.allclose(res["out"], inp["x"], rtol=1e-6, atol=0)


ALL_PINS = [v for kname, v in sorted(globals().items()) if kname.startswith("pin_")]
