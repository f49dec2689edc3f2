"""FP8 block-scaled SwiGLU experts (moe_expert_swiglu_fp8, moe_layer_fp8)
against the CPU oracle, step by step on every filled slot:

  H        bf16, within the bound below of the oracle's fp64 H of the same rows;
  Hq, Hs   bit for bit the oracle's quantisation of the GPU's own H (both
           sides take every rounding decision on the same fp32 quotients);
  Y        bf16, within the bound below of the oracle's down projection of
           the GPU's own Hq and Hs;
  out      the combine of the GPU's Y within the combine tolerance.

Bound.  The GPU sums each 128-column block of e4m3 code products on the
tensor cores in fp32 (the products themselves are exact) and folds the
block sums, times the block's row and tile scales, into an fp32 accumulator.
With at most 128 additions inside a block and 56 blocks (D = 7168), each
rounding to nearest in fp32, the textbook bound on the pre-rounding error is
(128 + 56 + 2) * 2^-24 * sum|x_d w_d| < EPS * sum|x_d w_d| with EPS = 2^-16.
Rounding both sides to bf16 adds at most one bf16 ulp (2^-7 relative).  For
H = silu(g) u the g and u errors carry through |silu'| <= 1.1 and |silu(g)|.
(Measured on a B200 at the full layer shape: the largest error beyond the
bf16 ulp was 2^-25.8 of the absolute sum.)

Inputs.  The scales of the synthetic inputs are spread over 2^-4 .. 2^4 per
row block and per weight tile (the codes stay the same), so that a scale
read from the wrong block or tile moves a result far outside the bound.
"""
import numpy as np
import pytest
import torch

import oracle
import parity
import workloads

pytestmark = pytest.mark.gpu

LAYER8 = workloads.CONFIGS["layer_fp8"]
EPS = 2.0 ** -16
BF16_ULP = 2.0 ** -7
TINY = 2.0 ** -133


def _spread_scales(inp, seed):
    g = torch.Generator().manual_seed(seed)
    for key in ("x_scale", "w_gate_up_scale", "w_down_scale"):
        s = inp[key]
        inp[key] = (s * torch.pow(2.0, torch.randint(-4, 5, s.shape, generator=g).float())).contiguous()
    return inp


def _dec(codes: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).double().numpy()


def _rows_deq(codes, scale):
    return _dec(codes) * np.repeat(scale.astype(np.float64), 128, axis=1)


def _tiles_deq(codes, scale):
    return _dec(codes) * np.kron(scale.astype(np.float64), np.ones((128, 128)))


def run_fp8_gpu(cfg, inp, n, fused=False):
    import combine_moe_route_11_b200 as mr
    dev = torch.device("cuda", 0)
    plan = mr.Plan.from_config(cfg, n_max=n)
    ws = plan.new_workspace(dev)
    b = plan.new_buffers(n, dev)
    w = {k: inp[k].to(dev) for k in ("w_gate_up", "w_gate_up_scale", "w_down", "w_down_scale")}
    logits, x, xs = inp["logits"].to(dev), inp["x"].to(dev), inp["x_scale"].to(dev)
    if fused:
        mr.moe_route_dispatch(plan, logits, x, xs, b["topk_idx"], b["topk_w"], b["counts"],
                              b["expert_off"], b["recv"], b["recv_scale"], b["slot_of"],
                              b["src_of"], ws)
    else:
        mr.moe_route_topk(plan, logits, b["topk_idx"], b["topk_w"], b["counts"], b["expert_off"],
                          ws)
        mr.moe_dispatch(plan, x, xs, b["topk_idx"], b["recv"], b["recv_scale"], b["slot_of"],
                        b["src_of"], ws)
    mr.moe_expert_swiglu_fp8(plan, n, b["recv"], b["recv_scale"], b["counts"], b["expert_off"],
                             b["slot_of"], w["w_gate_up"], w["w_gate_up_scale"], w["w_down"],
                             w["w_down_scale"], b["h"], b["hq"], b["h_scale"], b["y"], ws)
    mr.moe_combine(plan, b["y"], b["topk_w"], b["slot_of"], b["out"], ws)
    assert mr.moe_get_status(plan, ws) == 0
    torch.cuda.synchronize()
    return plan, ws, {k: (v.cpu() if v is not None else None) for k, v in b.items()}


def check_rows(inp_np, b, slots, expert, x_rows=None, x_scale_rows=None):
    """H, Hq/Hs and Y of the listed slots against the oracle (module doc).
    x_rows / x_scale_rows: the source rows of the slots (default: the GPU's
    recv rows, which the dispatch parity tests pin to the oracle's)."""
    slots = np.asarray(slots, np.int64)
    expert = np.asarray(expert, np.int32)
    rows = np.arange(len(slots), dtype=np.int32)
    if x_rows is None:
        x_rows = workloads.as_numpy_bits(b["recv"])[slots]
        x_scale_rows = b["recv_scale"].numpy()[slots]
    wgu, sgu = inp_np["w_gate_up"], inp_np["w_gate_up_scale"]
    wd, sd = inp_np["w_down"], inp_np["w_down_scale"]
    inter = wd.shape[2]

    h_ref, g, u = oracle.fp8_gate_up_rows(rows, expert, x_rows, x_scale_rows, wgu, sgu,
                                          want_gu=True)
    xabs = np.abs(_rows_deq(x_rows, x_scale_rows))
    g_abs = np.zeros_like(g)
    u_abs = np.zeros_like(u)
    for e in np.unique(expert):
        sel = expert == e
        wabs = np.abs(_tiles_deq(wgu[e], sgu[e]))
        g_abs[sel] = xabs[sel] @ wabs[:inter].T
        u_abs[sel] = xabs[sel] @ wabs[inter:].T
    with np.errstate(over="ignore"):
        silu = g / (1.0 + np.exp(-g))
    h_gpu_bits = parity.to_bits(b["h"])[slots]
    hg = oracle.to_float(h_gpu_bits, "bf16")
    hr = oracle.to_float(h_ref, "bf16")
    bound = BF16_ULP * np.abs(hr) + 1.1 * EPS * g_abs * np.abs(u) + EPS * u_abs * np.abs(silu) + TINY
    bad = np.abs(hg - hr) > bound
    assert not bad.any(), (f"H: {bad.sum()} of {bad.size} outside the bound; worst ratio "
                           f"{np.max(np.abs(hg - hr) / bound):.3g}")

    hq_ref, hs_ref = oracle.quant_rows(rows, h_gpu_bits, 128)
    hq_gpu = b["hq"].numpy()[slots]
    hs_gpu = b["h_scale"].numpy()[slots]
    assert np.array_equal(hs_gpu, hs_ref), "H scales differ from the oracle's"
    assert np.array_equal(hq_gpu, hq_ref), (f"H codes: {(hq_gpu != hq_ref).sum()} differ from "
                                            f"the oracle's")

    y_ref = oracle.fp8_down_rows(rows, expert, hq_gpu, hs_gpu, wd, sd)
    habs = np.abs(_rows_deq(hq_gpu, hs_gpu))
    y_abs = np.zeros((len(slots), wd.shape[1]))
    for e in np.unique(expert):
        sel = expert == e
        y_abs[sel] = habs[sel] @ np.abs(_tiles_deq(wd[e], sd[e])).T
    yg = oracle.to_float(parity.to_bits(b["y"])[slots], "bf16")
    yr = oracle.to_float(y_ref, "bf16")
    bound = BF16_ULP * np.abs(yr) + EPS * y_abs + TINY
    bad = np.abs(yg - yr) > bound
    assert not bad.any(), (f"Y: {bad.sum()} of {bad.size} outside the bound; worst ratio "
                           f"{np.max(np.abs(yg - yr) / bound):.3g}")


def check_all(cfg, inp, n, fused=False):
    inp_np = parity.numpy_inputs(inp)
    ref = oracle.run_path(cfg, inp_np, with_recv=False)
    _, _, b = run_fp8_gpu(cfg, inp, n, fused=fused)
    for key in ("topk_idx", "counts", "expert_off", "slot_of"):
        assert np.array_equal(parity.to_bits(b[key]).astype(np.int64),
                              np.asarray(ref[key]).astype(np.int64)), key
    fs = np.sort(ref["slot_of"].reshape(-1))
    expert = ref["topk_idx"].reshape(-1)[ref["src_of"][fs]]
    # the receive buffer holds each slot's source row and scales, bit for bit
    tok = ref["src_of"][fs] // cfg.top_k
    assert np.array_equal(workloads.as_numpy_bits(b["recv"])[fs], inp_np["x"][tok])
    assert np.array_equal(b["recv_scale"].numpy()[fs], inp_np["x_scale"][tok])
    check_rows(inp_np, b, fs, expert)
    # combine of the GPU's own Y
    y_bits = parity.to_bits(b["y"])
    out_ref = oracle.combine(y_bits, "bf16", ref["topk_w"], ref["slot_of"], "bf16")
    out_abs = oracle.combine_abs(y_bits, "bf16", ref["topk_w"], ref["slot_of"])
    parity.assert_combine_close(parity.to_bits(b["out"]), out_ref, out_abs, "bf16")
    return b


SMALL = [
    ("E8_k2", LAYER8.replace(hidden=256, inter=128, n_experts=8, top_k=2, n_ranks=2), 200),
    ("zipf_multi_mtile", LAYER8.replace(hidden=256, inter=256, n_experts=16, top_k=2, n_ranks=4,
                                        logits="zipf1.2"), 1000),
    ("k1_R1", LAYER8.replace(hidden=512, inter=384, n_experts=4, top_k=1, n_ranks=1), 130),
]


@pytest.mark.parametrize("name,cfg,n", SMALL, ids=[c[0] for c in SMALL])
def test_fp8_swiglu_small_matches_oracle(name, cfg, n):
    inp = _spread_scales(workloads.make_inputs(cfg, seed=21, n=n), seed=22)
    check_all(cfg, inp, n)


def test_fp8_swiglu_after_one_launch_route_dispatch():
    cfg = SMALL[0][1]
    inp = _spread_scales(workloads.make_inputs(cfg, seed=23, n=150), seed=24)
    check_all(cfg, inp, 150, fused=True)


def test_fp8_swiglu_tile_shapes_from_designed_counts():
    """Expert segments of 1, 16, 17, 96, 97, 128, 261 and 0 rows (k = 1):
    partial last tiles of many sizes, a full tile, a full tile followed by a
    partial one, and an empty expert."""
    counts = [1, 16, 17, 96, 97, 128, 261, 0]
    cfg = LAYER8.replace(hidden=512, inter=256, n_experts=8, top_k=1, n_ranks=2)
    n = sum(counts)
    inp = _spread_scales(workloads.make_inputs(cfg, seed=25, n=n), seed=26)
    g = torch.Generator().manual_seed(27)
    assign = torch.repeat_interleave(torch.arange(8), torch.tensor(counts))
    assign = assign[torch.randperm(n, generator=g)]
    logits = 0.1 * torch.randn(n, 8, generator=g)
    logits[torch.arange(n), assign] = 10.0
    inp["logits"] = logits
    b = check_all(cfg, inp, n)
    assert list(b["counts"].numpy()) == counts


def test_fp8_swiglu_layer_config():
    """The FP8 layer workload exactly as configured and benchmarked: N = 1024,
    D = 7168, E = 64, k = 8, R = 8, I = 2048, route and dispatch in one
    launch.  Integer results against the oracle on the whole batch; H, Hq/Hs
    and Y (check_rows) on the first, middle and last row of every segment and
    both sides of every 128-row tile boundary, from each slot's source row;
    the whole output against the oracle's combine of the GPU's Y."""
    from test_gpu_swiglu import segment_sample
    cfg = LAYER8
    n = cfg.n
    inp = _spread_scales(workloads.make_inputs(cfg, seed=42, n=n), seed=43)
    inp_np = parity.numpy_inputs(inp)
    ref = oracle.run_path(cfg, inp_np, with_recv=False)
    _, _, b = run_fp8_gpu(cfg, inp, n, fused=True)
    for key in ("topk_idx", "counts", "expert_off", "slot_of"):
        assert np.array_equal(parity.to_bits(b[key]).astype(np.int64),
                              np.asarray(ref[key]).astype(np.int64)), key
    off, cnt = ref["expert_off"], ref["counts"]
    assert int(cnt.max()) > 128 and int(cnt[cnt > 0].min()) < 128
    slots = segment_sample(off, cnt, cfg.n_experts)
    tok = ref["src_of"][slots] // cfg.top_k
    expert = np.searchsorted(off[:cfg.n_experts], slots, side="right") - 1
    check_rows(inp_np, b, slots, expert, x_rows=inp_np["x"][tok],
               x_scale_rows=inp_np["x_scale"][tok])
    y_bits = parity.to_bits(b["y"])
    out_ref = oracle.combine(y_bits, "bf16", ref["topk_w"], ref["slot_of"], "bf16")
    out_abs = oracle.combine_abs(y_bits, "bf16", ref["topk_w"], ref["slot_of"])
    parity.assert_combine_close(parity.to_bits(b["out"]), out_ref, out_abs, "bf16")


@pytest.mark.parametrize("n,k", [(300, 4), (1000, 8)])
def test_fp8_swiglu_layer_shape_sampled_rows(n, k):
    """Full D = 7168 and I = 2048 (E = 16 experts to bound the weight bytes):
    the first, middle and last row of every expert segment and the rows on
    each side of every 128-row tile boundary, each checked against the oracle
    from its source token's row."""
    cfg = LAYER8.replace(n_experts=16, top_k=k, n_ranks=4)
    inp = _spread_scales(workloads.make_inputs(cfg, seed=28, n=n), seed=29)
    _, _, b = run_fp8_gpu(cfg, inp, n)
    off = b["expert_off"].numpy()
    cnt = b["counts"].numpy()
    src = b["src_of"].numpy()
    slots = []
    for e in range(cfg.n_experts):
        if cnt[e]:
            slots += [off[e], off[e] + cnt[e] - 1, off[e] + cnt[e] // 2]
            for edge in range(128, int(cnt[e]), 128):
                slots += [off[e] + edge - 1, off[e] + edge]
    slots = np.unique(np.array(slots, np.int64))
    tok = src[slots] // cfg.top_k
    expert = np.searchsorted(off[:cfg.n_experts], slots, side="right") - 1
    inp_np = parity.numpy_inputs(inp)
    check_rows(inp_np, b, slots, expert, x_rows=inp_np["x"][tok],
               x_scale_rows=inp_np["x_scale"][tok])


def test_layer_fp8_entry_point_equals_the_steps():
    """moe_layer_fp8 launches the same kernels as the step-by-step calls, so
    its output and intermediates are the same bytes; moe_layer refuses a plan
    with FP8 experts."""
    import combine_moe_route_11_b200 as mr
    cfg, n = SMALL[1][1], 700
    inp = _spread_scales(workloads.make_inputs(cfg, seed=30, n=n), seed=31)
    _, _, b = run_fp8_gpu(cfg, inp, n, fused=True)
    dev = torch.device("cuda", 0)
    plan = mr.Plan.from_config(cfg, n_max=n)
    ws = plan.new_workspace(dev, layer=True)
    out = torch.empty(n, cfg.hidden, dtype=torch.bfloat16, device=dev)
    w = {k: inp[k].to(dev) for k in ("w_gate_up", "w_gate_up_scale", "w_down", "w_down_scale")}
    mr.moe_layer_fp8(plan, inp["logits"].to(dev), inp["x"].to(dev), inp["x_scale"].to(dev),
                     w["w_gate_up"], w["w_gate_up_scale"], w["w_down"], w["w_down_scale"], out, ws)
    assert mr.moe_get_status(plan, ws) == 0
    assert torch.equal(out.cpu(), b["out"])
    T = plan.recv_rows(n)
    fs = np.sort(b["slot_of"].numpy().reshape(-1))
    hq = mr.moe_layer_buffer(plan, ws, "hq", torch.uint8, (T, cfg.inter)).cpu().numpy()
    hs = mr.moe_layer_buffer(plan, ws, "h_scale", torch.float32, (T, cfg.inter // 128)).cpu()
    assert np.array_equal(hq[fs], b["hq"].numpy()[fs])
    assert np.array_equal(hs.numpy()[fs], b["h_scale"].numpy()[fs])
    with pytest.raises(mr.MoeError):
        mr.moe_layer(plan, inp["logits"].to(dev), inp["x"].to(dev), inp["x_scale"].to(dev),
                     None, None, out, ws)
