"""Shared helpers of the GPU parity tests: run the CUDA path through the
C-ABI binding, fetch results as raw numpy bits, and compare with the oracle.

Tolerances (written here once, used by every parity test):
  * integers, indices and dispatched bytes: bit-exact;
  * gate weights (fp32): |g - r| <= 8 ulp(r) -- the GPU evaluates k fp32
    exponentials (error <= 2 ulp each) and one division against the oracle's
    double evaluation rounded once;
  * FP8 identity expert: bit-exact (both sides round the exact product once);
  * combine: |g - r| <= rtol * sum_j |w_j * Y_j| with rtol = 1e-5 for fp32
    output and 2e-2 for bf16 output (fp32 accumulation in fixed j order on
    the GPU against a double sum rounded once in the oracle).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import workloads

RTOL_COMBINE = {"f32": 1e-5, "bf16": 2e-2}


def to_bits(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float8_e4m3fn:
        return t.view(torch.uint8).numpy()
    return t.numpy()


def numpy_inputs(inp: dict) -> dict:
    return {k: workloads.as_numpy_bits(v) for k, v in inp.items()}


def run_gpu(cfg, inp: dict, plan=None, n_max=None, want=("all",), fused=False,
            ws=None) -> dict:
    """route -> dispatch -> (dequant) -> combine on cuda:0 via the C-ABI;
    with fused=True route + dispatch go through moe_route_dispatch."""
    import combine_moe_route_11_b200 as mr
    n = inp["logits"].shape[0]
    dev = torch.device("cuda", 0)
    plan = plan or mr.Plan.from_config(cfg, n_max=n_max or max(n, 1))
    ws = plan.new_workspace(dev) if ws is None else ws
    b = plan.new_buffers(n, dev)
    logits = inp["logits"].to(dev)
    x = inp["x"].to(dev)
    xs = inp["x_scale"].to(dev) if inp.get("x_scale") is not None else None
    if fused:
        mr.moe_route_dispatch(plan, logits, x, xs, b["topk_idx"], b["topk_w"], b["counts"],
                              b["expert_off"], b["recv"], b["recv_scale"], b["slot_of"],
                              b["src_of"], ws)
    else:
        mr.moe_route_topk(plan, logits, b["topk_idx"], b["topk_w"], b["counts"],
                          b["expert_off"], ws)
        mr.moe_dispatch(plan, x, xs, b["topk_idx"], b["recv"], b["recv_scale"], b["slot_of"],
                        b["src_of"], ws)
    if cfg.x_dtype == "fp8_e4m3":
        mr.moe_expert_dequant(plan, n, b["recv"], b["recv_scale"], b["slot_of"], b["y"], ws)
        y = b["y"]
    else:
        y = b["recv"]
    mr.moe_combine(plan, y, b["topk_w"], b["slot_of"], b["out"], ws)
    status = mr.moe_get_status(plan, ws)
    torch.cuda.synchronize()
    res = {"status": status, "plan": plan, "ws": ws, "dev": b}
    for key in ("topk_idx", "topk_w", "counts", "expert_off", "slot_of", "src_of", "out"):
        res[key] = to_bits(b[key])
    if "all" in want:
        res["recv"] = to_bits(b["recv"])
        if b.get("recv_scale") is not None:
            res["recv_scale"] = to_bits(b["recv_scale"])
        if "y" in b:
            res["y"] = to_bits(b["y"])
    return res


def assert_weights_close(g: np.ndarray, r: np.ndarray, ulps: int = 8):
    g = g.astype(np.float64)
    r = r.astype(np.float64)
    ulp = np.spacing(np.abs(r).astype(np.float32)).astype(np.float64)
    bad = np.abs(g - r) > ulps * ulp
    assert not bad.any(), f"{bad.sum()} weights off by more than {ulps} ulp; max |d| = " \
                          f"{np.abs(g - r).max()}"


def assert_combine_close(g_bits: np.ndarray, r_bits: np.ndarray, r_abs: np.ndarray,
                         dtype: str):
    g = oracle.to_float(g_bits, dtype)
    r = oracle.to_float(r_bits, dtype)
    rtol = RTOL_COMBINE[dtype]
    err = np.abs(g - r)
    bound = rtol * r_abs + 1e-30
    bad = err > bound
    assert not bad.any(), (f"{bad.sum()} of {bad.size} combine outputs outside rtol {rtol}; "
                           f"worst ratio {np.max(err / bound)}")


def filled_slots(slot_of: np.ndarray) -> np.ndarray:
    return np.sort(slot_of.reshape(-1))


def compare_path(cfg, inp_np: dict, ref: dict, got: dict, check_rows: bool = True):
    """Element-by-element comparison of every stage against the oracle."""
    assert got["status"] == 0, f"device status {got['status']}"
    assert np.array_equal(got["topk_idx"], ref["topk_idx"]), "topk_idx differs"
    assert_weights_close(got["topk_w"], ref["topk_w"])
    assert np.array_equal(got["counts"], ref["counts"]), "counts differ"
    assert np.array_equal(got["expert_off"].astype(np.int64), ref["expert_off"]), "expert_off"
    assert np.array_equal(got["slot_of"], ref["slot_of"]), "slot_of differs"
    fs = filled_slots(ref["slot_of"])
    assert np.array_equal(got["src_of"][fs], ref["src_of"][fs]), "src_of differs"
    if check_rows:
        assert np.array_equal(got["recv"][fs], ref["recv"][fs]), "dispatched rows differ"
        if "recv_scale" in ref:
            assert np.array_equal(got["recv_scale"][fs], ref["recv_scale"][fs]), "scales differ"
        if cfg.x_dtype == "fp8_e4m3":
            assert np.array_equal(got["y"][fs], ref["y"][fs]), "identity-expert rows differ"
    assert_combine_close(got["out"], ref["out"], ref["out_abs"], cfg.out_dtype)


RTOL_GEMM = 2e-2


def assert_gemm_rows_close(g_bits: np.ndarray, r_bits: np.ndarray, what: str):
    """bf16 expert outputs (H or Y rows): |g - r| <= 2e-2 * max(|r|, rms of
    the reference row).  The GPU sums bf16 products in fp32 on the tensor
    cores and rounds once to bf16; the oracle sums in double and rounds once;
    the row-RMS term keeps the bound well posed where an output cancels to ~0."""
    g = oracle.to_float(g_bits, "bf16")
    r = oracle.to_float(r_bits, "bf16")
    rms = np.sqrt(np.mean(r * r, axis=1, keepdims=True)) + 1e-30
    bound = RTOL_GEMM * np.maximum(np.abs(r), rms)
    bad = np.abs(g - r) > bound
    assert not bad.any(), (f"{what}: {bad.sum()} of {bad.size} elements outside tolerance; "
                           f"worst ratio {np.max(np.abs(g - r) / bound):.3g}")
    # and nearly all elements agree within one bf16 ulp; the rest are outputs
    # that cancel to a small magnitude, where the fp32 (GPU) and double
    # (oracle) sums of thousands of terms round to different neighbours
    same = np.abs(g - r) <= np.abs(r) * 2.0 ** -7 + 1e-30
    assert same.mean() > 0.95, f"{what}: only {same.mean():.4f} within one bf16 ulp"


def assert_layer_out_close(g_bits: np.ndarray, ref: dict):
    """Layer output with SwiGLU experts: the combine bound plus the expert
    output's own bound carried through the weights,
        |g - r| <= 2e-2 * sum_j |w_j * Y_j|  +  sum_j |w_j| * 2e-2 * rms(Y_j row),
    since out = sum_j w_j Y_j and each Y_j carries the GEMM tolerance above."""
    y = oracle.to_float(ref["y"], "bf16")
    rms = np.sqrt(np.mean(y * y, axis=1))
    w = np.abs(ref["topk_w"].astype(np.float64))
    carried = (w * rms[ref["slot_of"]]).sum(axis=1, keepdims=True)
    g = oracle.to_float(g_bits, "bf16")
    r = oracle.to_float(ref["out"], "bf16")
    bound = RTOL_COMBINE["bf16"] * ref["out_abs"] + RTOL_GEMM * carried + 1e-30
    bad = np.abs(g - r) > bound
    assert not bad.any(), (f"{bad.sum()} of {bad.size} layer outputs outside tolerance; "
                           f"worst ratio {np.max(np.abs(g - r) / bound):.3g}")
