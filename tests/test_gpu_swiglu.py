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


def run_layer_gpu(cfg, inp, n):
    import combine_moe_route_11_b200 as mr
    dev = torch.device("cuda", 0)
    plan = mr.Plan.from_config(cfg, n_max=n)
    ws = plan.new_workspace(dev)
    b = plan.new_buffers(n, dev)
    wgu, wd = inp["w_gate_up"].to(dev), inp["w_down"].to(dev)
    mr.moe_route_topk(plan, inp["logits"].to(dev), b["topk_idx"], b["topk_w"], b["counts"],
                      b["expert_off"], ws)
    mr.moe_dispatch(plan, inp["x"].to(dev), None, b["topk_idx"], b["recv"], None, b["slot_of"],
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
    slots = []
    for e in range(cfg.n_experts):
        if cnt[e]:
            slots += [off[e], off[e] + cnt[e] - 1, off[e] + cnt[e] // 2]
            for edge in range(128, int(cnt[e]), 128):
                slots += [off[e] + edge - 1, off[e] + edge]
    slots = np.unique(np.array(slots, np.int64))
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
