"""moe_combine's arithmetic contract, bit for bit.

The boundary promises out[t, c] = sum_j w[t, j] * Y[slot_of[t, j], c]
accumulated in binary32 with one fused multiply-add per j in increasing j,
starting from +0, then rounded to nearest even into the output type (the
fixed-order fp32 accumulation of the weighted sum that "MLX expert
parallelism all_to_all PR 3158", Facts, names combine_weighted_sum).  The
oracle sums in binary64, so its tolerance cannot tell a different order or a
multiply-then-add from that contract.  Here the same Y, weights and slots go
to the GPU and to a CPU evaluation of exactly that sequence of binary32 fmas
(tests/fp32_fma.py, pinned against libm's fmaf on the CPU); the outputs must
agree in every bit.

The inputs are built so that a different order or a separate rounding of
each product changes results: weights of both signs spread over 2^-6..2^6,
and Y rows whose magnitudes differ by up to 2^12 between choices, so that
partial sums carry rounding errors that depend on the order.
"""
import zlib

import numpy as np
import pytest
import torch

import fp32_fma
import workloads


def _inputs(n, k, T, D, y_dtype, seed):
    """Slots, weights, the Y rows the slots point at ([n, k, D] values) and
    the whole Y buffer [T, D] as a tensor (rows nobody reads stay zero)."""
    g = np.random.default_rng(seed)
    # distinct slots of [0, T) for the n*k choices (any layout is legal input)
    slot_of = g.choice(T, n * k, replace=False).astype(np.int32).reshape(n, k)
    w = (g.choice([-1.0, 1.0], (n, k)) * 2.0 ** g.uniform(-6, 6, (n, k))).astype(np.float32)
    row_scale = 2.0 ** g.integers(-6, 7, (n, k, 1))
    y32 = (g.standard_normal((n, k, D), dtype=np.float32) * row_scale).astype(np.float32)
    if y_dtype == "bf16":
        y_bits = fp32_fma.bf16_bits_rne(y32)
        y_vals = fp32_fma.bf16_bits_to_f32(y_bits)
        rows = torch.from_numpy(y_bits.view(np.int16).reshape(n * k, D)).view(torch.bfloat16)
    else:
        y_vals = y32
        rows = torch.from_numpy(y32.reshape(n * k, D))
    y_t = torch.zeros(T, D, dtype=rows.dtype)
    y_t[torch.from_numpy(slot_of.reshape(-1).astype(np.int64))] = rows
    return slot_of, w, y_vals, y_t


def _expected(w, y_vals, out_dtype):
    n, k, d = y_vals.shape
    acc = np.zeros((n, d), np.float32)
    for j in range(k):
        acc = fp32_fma.fmaf(w[:, j:j + 1], y_vals[:, j], acc)
    if out_dtype == "bf16":
        return fp32_fma.bf16_bits_rne(acc)
    return acc.view(np.uint32)


CASES = [
    # prefill: bf16 Y, bf16 out, D = 7168, k = 8
    ("prefill_bf16", workloads.CONFIGS["prefill"], 384, "bf16", "bf16"),
    # the same width with fp32 Y and fp32 out (no final rounding)
    ("prefill_f32", workloads.CONFIGS["prefill"].replace(x_dtype="f32", y_dtype="f32",
                                                         out_dtype="f32", scale_block=0),
     256, "f32", "f32"),
    # bf16 Y with fp32 out: the accumulator itself is compared
    ("bf16_to_f32", workloads.CONFIGS["decode"].replace(out_dtype="f32"), 128, "bf16", "f32"),
    # k = 32: the kernel loads the expert rows in groups of eight; the order
    # must still run over all 32 choices in increasing j
    ("k32", workloads.CONFIGS["skewed"].replace(top_k=32, n_ranks=1), 200, "bf16", "bf16"),
]


@pytest.mark.gpu
@pytest.mark.parametrize("name,cfg,n,y_dtype,out_dtype", CASES, ids=[c[0] for c in CASES])
def test_combine_is_fma_in_increasing_j(name, cfg, n, y_dtype, out_dtype):
    import combine_moe_route_11_b200 as mr
    assert cfg.y_dtype == y_dtype and cfg.out_dtype == out_dtype
    dev = torch.device("cuda", 0)
    plan = mr.Plan.from_config(cfg, n_max=n)
    T = plan.recv_rows(n)
    slot_of, w, y_vals, y_t = _inputs(n, cfg.top_k, T, cfg.hidden, y_dtype,
                                      seed=zlib.crc32(name.encode()))
    ws = plan.new_workspace(dev)
    out_t = torch.bfloat16 if out_dtype == "bf16" else torch.float32
    out = torch.empty(n, cfg.hidden, dtype=out_t, device=dev)
    mr.moe_combine(plan, y_t.to(dev), torch.from_numpy(w).to(dev),
                   torch.from_numpy(slot_of).to(dev), out, ws)
    assert mr.moe_get_status(plan, ws) == 0
    got = out.cpu()
    got_bits = (got.view(torch.int16).numpy().view(np.uint16) if out_dtype == "bf16"
                else got.numpy().view(np.uint32))
    want = _expected(w, y_vals, out_dtype)
    diff = got_bits != want
    assert not diff.any(), f"{int(diff.sum())} of {diff.size} outputs differ from the fma sequence"


def test_expected_values_are_order_sensitive():
    """The inputs above can tell orders apart: summing the same products in
    decreasing j changes some outputs (checked on the CPU)."""
    _, w, y_vals, _ = _inputs(64, 8, 4096, 512, "bf16", seed=3)
    fwd = _expected(w, y_vals, "f32")
    acc = np.zeros((64, 512), np.float32)
    for j in reversed(range(8)):
        acc = fp32_fma.fmaf(w[:, j:j + 1], y_vals[:, j], acc)
    assert (acc.view(np.uint32) != fwd).any()
