"""moe_route_dispatch (one cooperative launch for n <= 1024 tokens, each block
routing and scattering its own tokens around one grid barrier) against the CPU
oracle and against the two-call path, through the C ABI.

The fused call must give exactly what moe_route_topk followed by moe_dispatch
gives: every integer result and every dispatched byte bit-exact, gate weights
within the same 8-ulp bound.  It shares the workspace's barrier generation and
expert-total halves with the route kernel, so calls of both kinds are also
interleaved on one workspace.
"""
import numpy as np
import pytest
import torch

import oracle
import parity
import workloads

pytestmark = pytest.mark.gpu

C = workloads.CONFIGS
TINY = C["tiny"]

# (name, config, n) -- every case runs the full oracle
CASES = [
    ("tiny", TINY, 64),
    ("tiny_n1", TINY, 1),
    ("tiny_n61", TINY, 61),
    ("decode", C["decode"], 128),
    ("decode_n33", C["decode"], 33),
    ("prefill_fp8_ragged", C["prefill"], 300),
    ("skewed_ragged", C["skewed"], 1000),
    ("k1", TINY.replace(top_k=1), 100),
    ("k_eq_E", TINY.replace(top_k=8, n_ranks=4), 70),
    ("one_rank", TINY.replace(n_ranks=1), 90),
    ("E6_scalar", TINY.replace(n_experts=6, top_k=3, n_ranks=3, hidden=64), 200),
    ("E33_ragged_lanes", TINY.replace(n_experts=33, top_k=5, n_ranks=1, hidden=96), 150),
    ("E512", TINY.replace(n_experts=512, top_k=8, n_ranks=8, hidden=128, x_dtype="bf16",
                          y_dtype="bf16", out_dtype="bf16"), 130),
    ("k16", TINY.replace(n_experts=32, top_k=16, n_ranks=2, hidden=64), 100),
    ("k32_max", TINY.replace(n_experts=64, top_k=32, n_ranks=2, hidden=64), 90),
    ("E512_n128", TINY.replace(n_experts=512, top_k=8, n_ranks=8, hidden=128, x_dtype="bf16",
                               y_dtype="bf16", out_dtype="bf16"), 128),
    # more tokens than resident blocks: blocks own several tokens
    ("owned_many_777", C["decode"].replace(hidden=512), 777),
    ("decode_n257", C["decode"].replace(hidden=512), 257),
    # 32 route blocks: the largest batch the single launch takes
    ("max_blocks_1024", TINY.replace(n_experts=64, top_k=6, n_ranks=4, hidden=32,
                                     x_dtype="bf16", y_dtype="bf16", out_dtype="f32"), 1024),
    # one token more: the call runs the two kernels
    ("two_kernels_1025", TINY.replace(n_experts=64, top_k=6, n_ranks=4, hidden=32,
                                      x_dtype="bf16", y_dtype="bf16", out_dtype="f32"), 1025),
    ("fp8_small_D", C["prefill"].replace(hidden=256, n_experts=16, top_k=4, n_ranks=4), 129),
]


@pytest.mark.parametrize("name,cfg,n", CASES, ids=[c[0] for c in CASES])
def test_fused_matches_oracle(name, cfg, n):
    inp = workloads.make_inputs(cfg, seed=17, n=n)
    inp_np = parity.numpy_inputs(inp)
    ref = oracle.run_path(cfg, inp_np)
    got = parity.run_gpu(cfg, inp, fused=True)
    parity.compare_path(cfg, inp_np, ref, got)


@pytest.mark.parametrize("name,n", [("decode", 128), ("prefill", 512), ("skewed", 1024)])
def test_fused_equals_two_calls(name, n):
    """Bit-exact agreement with moe_route_topk + moe_dispatch at workload
    shapes, every output including the weights."""
    cfg = C[name]
    inp = workloads.make_inputs(cfg, seed=5, n=n)
    a = parity.run_gpu(cfg, inp, fused=True)
    b = parity.run_gpu(cfg, inp, fused=False)
    assert a["status"] == 0 and b["status"] == 0
    for key in ("topk_idx", "topk_w", "counts", "expert_off", "slot_of", "out"):
        assert np.array_equal(a[key], b[key]), key
    filled = np.sort(b["slot_of"].reshape(-1))
    for key in ("src_of", "recv", "recv_scale", "y"):
        if key in b:
            assert np.array_equal(a[key][filled], b[key][filled]), key


def test_fused_and_route_interleave_on_one_workspace():
    """The two launch kinds alternate on one workspace.  Both keep tables in
    two halves chosen by the barrier generation (the route kernel's expert
    totals, the fused kernel's token masks), and each must leave the halves
    the next call of either kind uses at zero."""
    import combine_moe_route_11_b200 as mr
    cfg = TINY.replace(n_experts=16, top_k=4, n_ranks=4, hidden=64)
    plan = mr.Plan.from_config(cfg, n_max=420)
    ws = plan.new_workspace(torch.device("cuda", 0))
    order = [False, True, False, True, False, False, True, True, False, True]
    for i, fused in enumerate(order):
        n = 37 + 41 * i
        inp = workloads.make_inputs(cfg, seed=100 + i, n=n)
        inp_np = parity.numpy_inputs(inp)
        ref = oracle.run_path(cfg, inp_np)
        got = parity.run_gpu(cfg, inp, plan=plan, fused=fused, ws=ws)
        parity.compare_path(cfg, inp_np, ref, got)


def test_fused_zero_tokens():
    import combine_moe_route_11_b200 as mr
    plan = mr.Plan.from_config(TINY, n_max=64)
    dev = torch.device("cuda", 0)
    ws = plan.new_workspace(dev)
    b = plan.new_buffers(0, dev)
    b["counts"].fill_(-7)
    b["expert_off"].fill_(-7)
    mr.moe_route_dispatch(plan, torch.empty(0, 8, device=dev), torch.empty(0, 256, device=dev),
                          None, b["topk_idx"], b["topk_w"], b["counts"], b["expert_off"],
                          b["recv"], None, b["slot_of"], b["src_of"], ws)
    assert mr.moe_get_status(plan, ws) == 0
    assert int(b["counts"].abs().sum()) == 0
    assert int(b["expert_off"].abs().sum()) == 0


def test_fused_leaves_unfilled_rows_untouched():
    """Rows of a region past its filled count are never written by the one-
    launch path either, and the filled rows are exactly the expert segments."""
    import combine_moe_route_11_b200 as mr
    cfg = C["prefill"]
    n = 300
    inp = workloads.make_inputs(cfg, seed=8, n=n)
    plan = mr.Plan.from_config(cfg, n_max=n)
    dev = torch.device("cuda", 0)
    ws = plan.new_workspace(dev)
    b = plan.new_buffers(n, dev)
    b["recv"].fill_(0xAB)
    b["recv_scale"].fill_(-3.0)
    mr.moe_route_dispatch(plan, inp["logits"].cuda(), inp["x"].cuda(), inp["x_scale"].cuda(),
                          b["topk_idx"], b["topk_w"], b["counts"], b["expert_off"], b["recv"],
                          b["recv_scale"], b["slot_of"], b["src_of"], ws)
    assert mr.moe_get_status(plan, ws) == 0
    filled = torch.zeros(b["recv"].shape[0], dtype=torch.bool, device=dev)
    filled[b["slot_of"].view(-1).long()] = True
    assert bool((b["recv"][~filled] == 0xAB).all())
    assert bool((b["recv_scale"][~filled] == -3.0).all())
    off = b["expert_off"].cpu().numpy()
    cnt = b["counts"].cpu().numpy()
    want = np.zeros(b["recv"].shape[0], bool)
    for e in range(cfg.n_experts):
        want[off[e]:off[e] + cnt[e]] = True
    assert np.array_equal(filled.cpu().numpy(), want)


def test_fused_flags_nonfinite_logit_rows():
    """A row with fewer than k finite logits sets MOE_ERR_NONFINITE in the
    one-launch path too; every pick stays a valid expert and every (t, j)
    still gets a slot, so the dispatched layout stays consistent."""
    import combine_moe_route_11_b200 as mr
    cfg = TINY
    n = 64
    inp = workloads.make_inputs(cfg, seed=1, n=n)
    inp["logits"][7, :] = float("nan")
    inp["logits"][8, 1:] = float("-inf")
    plan = mr.Plan.from_config(cfg, n_max=n)
    dev = torch.device("cuda", 0)
    ws = plan.new_workspace(dev)
    b = plan.new_buffers(n, dev)
    mr.moe_route_dispatch(plan, inp["logits"].cuda(), inp["x"].cuda(), None, b["topk_idx"],
                          b["topk_w"], b["counts"], b["expert_off"], b["recv"], None,
                          b["slot_of"], b["src_of"], ws)
    assert mr.moe_get_status(plan, ws) == -7  # MOE_ERR_NONFINITE
    idx = b["topk_idx"].cpu().numpy()
    assert ((idx >= 0) & (idx < cfg.n_experts)).all()
    assert int(b["counts"].sum()) == n * cfg.top_k
    slots = np.sort(b["slot_of"].cpu().numpy().reshape(-1))
    assert len(np.unique(slots)) == n * cfg.top_k and slots.min() >= 0


def test_captured_graph_replays_match_oracle():
    """moe_route_dispatch + moe_combine captured once in a CUDA graph and
    replayed with new inputs copied into the captured buffers: every replay
    matches the oracle (the double-buffered tables alternate between
    replays), and eager calls on the same workspace still do afterwards."""
    import combine_moe_route_11_b200 as mr
    cfg = C["decode"].replace(hidden=1024)
    n = 96
    dev = torch.device("cuda", 0)
    plan = mr.Plan.from_config(cfg, n_max=n)
    ws = plan.new_workspace(dev)
    b = plan.new_buffers(n, dev)
    first = workloads.make_inputs(cfg, seed=40, n=n)
    logits = first["logits"].to(dev)
    x = first["x"].to(dev)
    stream = torch.cuda.Stream(dev)
    with torch.cuda.stream(stream):
        # warm the library's per-device set-up outside the capture
        mr.moe_route_dispatch(plan, logits, x, None, b["topk_idx"], b["topk_w"], b["counts"],
                              b["expert_off"], b["recv"], None, b["slot_of"], b["src_of"], ws)
        mr.moe_combine(plan, b["recv"], b["topk_w"], b["slot_of"], b["out"], ws)
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        mr.moe_route_dispatch(plan, logits, x, None, b["topk_idx"], b["topk_w"], b["counts"],
                              b["expert_off"], b["recv"], None, b["slot_of"], b["src_of"], ws,
                              stream)
        mr.moe_combine(plan, b["recv"], b["topk_w"], b["slot_of"], b["out"], ws, stream)
    for seed in (41, 42, 43):
        inp = workloads.make_inputs(cfg, seed=seed, n=n)
        logits.copy_(inp["logits"])
        x.copy_(inp["x"])
        g.replay()
        torch.cuda.synchronize()
        assert mr.moe_get_status(plan, ws) == 0
        inp_np = parity.numpy_inputs(inp)
        ref = oracle.run_path(cfg, inp_np)
        assert np.array_equal(parity.to_bits(b["slot_of"]), ref["slot_of"]), seed
        assert np.array_equal(parity.to_bits(b["counts"]), ref["counts"]), seed
        parity.assert_combine_close(parity.to_bits(b["out"]), ref["out"], ref["out_abs"],
                                    cfg.out_dtype)
    del g
    inp = workloads.make_inputs(cfg, seed=44, n=n)
    got = parity.run_gpu(cfg, inp, plan=plan, fused=True, ws=ws)
    parity.compare_path(cfg, parity.numpy_inputs(inp), oracle.run_path(cfg,
                        parity.numpy_inputs(inp)), got)
