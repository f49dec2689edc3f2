"""Grouped SwiGLU expert GEMMs (tcgen05) against the CPU oracle.

The GPU reads the dispatched rank-major buffer in place; the oracle computes
each expert row from its own source row.  H and Y are compared row by row on
the filled slots (tolerance in tests/parity.py), and the layer output through
combine with the combine tolerance.
"""
import numpy as np
import pytest
import torch

import oracle
import parity
import workloads

pytestmark = pytest.mark.gpu

LAYER = workloads.CONFIGS["layer"]


def run_layer_gpu(cfg, inp, n, fused=False):
    """route + dispatch (two calls, or moe_route_dispatch with fused=True) ->
    grouped SwiGLU GEMMs -> combine on cuda:0."""
    import combine_moe_route_11_b200 as mr
    dev = torch.device("cuda", 0)
    plan = mr.Plan.from_config(cfg, n_max=n)
    ws = plan.new_workspace(dev)
    b = plan.new_buffers(n, dev)
    wgu, wd = inp["w_gate_up"].to(dev), inp["w_down"].to(dev)
    logits, x = inp["logits"].to(dev), inp["x"].to(dev)
    if fused:
        mr.moe_route_dispatch(plan, logits, x, None, b["topk_idx"], b["topk_w"], b["counts"],
                              b["expert_off"], b["recv"], None, b["slot_of"], b["src_of"], ws)
    else:
        mr.moe_route_topk(plan, logits, b["topk_idx"], b["topk_w"], b["counts"],
                          b["expert_off"], ws)
        mr.moe_dispatch(plan, x, None, b["topk_idx"], b["recv"], None, b["slot_of"],
                        b["src_of"], ws)
    mr.moe_expert_swiglu(plan, n, b["recv"], b["counts"], b["expert_off"], wgu, wd, b["h"],
                         b["y"], ws)
    mr.moe_combine(plan, b["y"], b["topk_w"], b["slot_of"], b["out"], ws)
    assert mr.moe_get_status(plan, ws) == 0
    torch.cuda.synchronize()
    return plan, ws, b


SMALL = [
    ("E8_k2", LAYER.replace(hidden=256, inter=128, n_experts=8, top_k=2, n_ranks=2), 200),
    ("zipf_multi_mtile", LAYER.replace(hidden=256, inter=256, n_experts=16, top_k=2, n_ranks=4,
                                       logits="zipf1.2"), 1000),
    ("k1_R1", LAYER.replace(hidden=512, inter=384, n_experts=4, top_k=1, n_ranks=1), 130),
]


@pytest.mark.parametrize("name,cfg,n", SMALL, ids=[c[0] for c in SMALL])
def test_swiglu_small_matches_oracle(name, cfg, n):
    inp = workloads.make_inputs(cfg, seed=5, n=n)
    inp_np = parity.numpy_inputs(inp)
    ref = oracle.run_path(cfg, inp_np)
    _, _, b = run_layer_gpu(cfg, inp, n)
    got_slot = parity.to_bits(b["slot_of"])
    assert np.array_equal(got_slot, ref["slot_of"])
    fs = np.sort(ref["slot_of"].reshape(-1))
    # H: recompute the oracle's H on the filled rows
    expert_of_slot = ref["topk_idx"].reshape(-1)[ref["src_of"][fs]]
    _, h_ref = oracle.swiglu_rows(fs, expert_of_slot, ref["recv"], inp_np["w_gate_up"],
                                  inp_np["w_down"], want_h=True)
    parity.assert_gemm_rows_close(parity.to_bits(b["h"])[fs], h_ref[fs], "H")
    parity.assert_gemm_rows_close(parity.to_bits(b["y"])[fs], ref["y"][fs], "Y")
    parity.assert_layer_out_close(parity.to_bits(b["out"]), ref)


def segment_sample(off, cnt, n_experts):
    """Slots of the first, middle and last row of every expert segment and of
    the rows on each side of every 128-row tile boundary inside it."""
    slots = []
    for e in range(n_experts):
        if cnt[e]:
            slots += [off[e], off[e] + cnt[e] - 1, off[e] + cnt[e] // 2]
            for edge in range(128, int(cnt[e]), 128):
                slots += [off[e] + edge - 1, off[e] + edge]
    return np.unique(np.array(slots, np.int64))


def test_swiglu_layer_config():
    """The layer workload exactly as configured and benchmarked: N = 1024,
    D = 7168, E = 64, k = 8, R = 8, I = 2048, route and dispatch in one launch
    (moe_route_dispatch, as moe_layer and the bench call it).  About 128 rows
    per expert, so segments end just below, at or just above a 128-row tile.
    Integer results are compared with the oracle on the whole batch; Y on the
    sampled rows of every segment (segment_sample) from each slot's source
    row; the whole output against the oracle's combine of the GPU's Y."""
    cfg = LAYER
    n = cfg.n
    inp = workloads.make_inputs(cfg, seed=41, n=n)
    inp_np = parity.numpy_inputs(inp)
    ref = oracle.run_path(cfg, inp_np, with_recv=False)
    _, _, b = run_layer_gpu(cfg, inp, n, fused=True)
    for key in ("topk_idx", "counts", "expert_off", "slot_of"):
        assert np.array_equal(parity.to_bits(b[key]).astype(np.int64),
                              np.asarray(ref[key]).astype(np.int64)), key
    parity.assert_weights_close(parity.to_bits(b["topk_w"]), ref["topk_w"])
    off, cnt = ref["expert_off"], ref["counts"]
    assert int(cnt.max()) > 128 and int(cnt[cnt > 0].min()) < 128
    slots = segment_sample(off, cnt, cfg.n_experts)
    tok = ref["src_of"][slots] // cfg.top_k
    expert = np.searchsorted(off[:cfg.n_experts], slots, side="right") - 1
    rows = np.arange(len(slots), dtype=np.int32)
    y_ref = oracle.swiglu_rows(rows, expert.astype(np.int32), inp_np["x"][tok],
                               inp_np["w_gate_up"], inp_np["w_down"])
    y_bits = parity.to_bits(b["y"])
    parity.assert_gemm_rows_close(y_bits[slots], y_ref, "Y")
    out_ref = oracle.combine(y_bits, "bf16", ref["topk_w"], ref["slot_of"], "bf16")
    out_abs = oracle.combine_abs(y_bits, "bf16", ref["topk_w"], ref["slot_of"])
    parity.assert_combine_close(parity.to_bits(b["out"]), out_ref, out_abs, "bf16")


@pytest.mark.parametrize("n,k", [(300, 4), (1000, 8)])
def test_swiglu_layer_shape_sampled_rows(n, k):
    """Full D = 7168 and I = 2048 (E = 16 experts to bound the weight bytes):
    every output row of the GPU is checked on a sample of filled slots,
    including the first and last row of every expert segment and the rows
    on each side of every 128-row tile boundary.  At n=300, k=4 every expert
    is one short tile (operand roles swapped); at n=1000, k=8 experts span
    several full tiles and a last one."""
    cfg = LAYER.replace(n_experts=16, top_k=k, n_ranks=4)
    inp = workloads.make_inputs(cfg, seed=7, n=n)
    _, _, b = run_layer_gpu(cfg, inp, n)
    off = b["expert_off"].cpu().numpy()
    cnt = b["counts"].cpu().numpy()
    src = b["src_of"].cpu().numpy()
    slots = segment_sample(off, cnt, cfg.n_experts)
    tok = src[slots] // cfg.top_k
    expert = np.searchsorted(off[:cfg.n_experts], slots, side="right") - 1
    x_rows = workloads.as_numpy_bits(inp["x"])[tok]
    rows = np.arange(len(slots), dtype=np.int32)
    y_ref = oracle.swiglu_rows(rows, expert.astype(np.int32), x_rows,
                               workloads.as_numpy_bits(inp["w_gate_up"]),
                               workloads.as_numpy_bits(inp["w_down"]))
    parity.assert_gemm_rows_close(parity.to_bits(b["y"])[slots], y_ref, "Y")


def test_layer_entry_point_with_swiglu():
    import combine_moe_route_11_b200 as mr
    cfg, n = SMALL[0][1], 150
    inp = workloads.make_inputs(cfg, seed=9, n=n)
    ref = oracle.run_path(cfg, parity.numpy_inputs(inp))
    dev = torch.device("cuda", 0)
    plan = mr.Plan.from_config(cfg, n_max=n)
    ws = plan.new_workspace(dev, layer=True)
    out = torch.empty(n, cfg.hidden, dtype=torch.bfloat16, device=dev)
    mr.moe_layer(plan, inp["logits"].to(dev), inp["x"].to(dev), None, inp["w_gate_up"].to(dev),
                 inp["w_down"].to(dev), out, ws)
    assert mr.moe_get_status(plan, ws) == 0
    parity.assert_layer_out_close(parity.to_bits(out), ref)


def test_swiglu_tile_shapes_from_designed_counts():
    """Expert segments of 1, 16, 17, 96, 97, 128, 261 and 0 rows (k = 1, each
    token sent to a chosen expert): last m-tiles of every size class -- swapped
    roles with N = 16, 32 and 96, the first normal size (97), a full tile, a
    full tile followed by a swapped tail, and an empty expert."""
    counts = [1, 16, 17, 96, 97, 128, 261, 0]
    cfg = LAYER.replace(hidden=512, inter=256, n_experts=8, top_k=1, n_ranks=2)
    n = sum(counts)
    inp = workloads.make_inputs(cfg, seed=13, n=n)
    g = torch.Generator().manual_seed(14)
    assign = torch.repeat_interleave(torch.arange(8), torch.tensor(counts))
    assign = assign[torch.randperm(n, generator=g)]
    logits = 0.1 * torch.randn(n, 8, generator=g)
    logits[torch.arange(n), assign] = 10.0
    inp["logits"] = logits
    inp_np = parity.numpy_inputs(inp)
    ref = oracle.run_path(cfg, inp_np)
    assert list(ref["counts"]) == counts
    _, _, b = run_layer_gpu(cfg, inp, n)
    assert np.array_equal(parity.to_bits(b["slot_of"]), ref["slot_of"])
    fs = np.sort(ref["slot_of"].reshape(-1))
    expert_of_slot = ref["topk_idx"].reshape(-1)[ref["src_of"][fs]]
    _, h_ref = oracle.swiglu_rows(fs, expert_of_slot, ref["recv"], inp_np["w_gate_up"],
                                  inp_np["w_down"], want_h=True)
    parity.assert_gemm_rows_close(parity.to_bits(b["h"])[fs], h_ref[fs], "H")
    parity.assert_gemm_rows_close(parity.to_bits(b["y"])[fs], ref["y"][fs], "Y")
    parity.assert_layer_out_close(parity.to_bits(b["out"]), ref)
