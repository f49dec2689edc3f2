"""CUDA path against the CPU oracle, element by element, through the C-ABI.

Small cases run the whole oracle; the full-size workloads compare every
integer result at full size, check the dispatched rows by a property that
holds at any size (recv[slot_of[t, j]] == x[t], untouched unfilled rows) and
compare combine on sampled tokens, whose outputs the oracle computes from
their own rows alone.
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
SMALL_CASES = [
    ("tiny", TINY, 64),
    ("tiny_n1", TINY, 1),
    ("tiny_n61", TINY, 61),
    ("tiny_n65", TINY, 65),
    ("decode", C["decode"], 128),
    ("prefill_ragged", C["prefill"], 300),
    ("skewed_ragged", C["skewed"], 1000),
    ("k1", TINY.replace(top_k=1), 100),
    ("k_eq_E", TINY.replace(top_k=8, n_ranks=4), 70),
    ("one_rank", TINY.replace(n_ranks=1), 90),
    ("rank_per_expert", TINY.replace(n_ranks=8, top_k=3), 90),
    ("E6_scalar_scan", TINY.replace(n_experts=6, top_k=3, n_ranks=3, hidden=64), 200),
    ("E33_ragged_lanes", TINY.replace(n_experts=33, top_k=5, n_ranks=1, hidden=96), 150),
    ("E512", TINY.replace(n_experts=512, top_k=8, n_ranks=8, hidden=128, x_dtype="bf16",
                          y_dtype="bf16", out_dtype="bf16"), 130),
    ("many_blocks", TINY.replace(n_experts=64, top_k=6, n_ranks=4, hidden=32, x_dtype="bf16",
                                 y_dtype="bf16", out_dtype="f32"), 5000),
    # four to five route blocks per CTA of the route kernel, the last one ragged
    ("blocks_per_cta", TINY.replace(n_experts=128, top_k=4, n_ranks=4, hidden=32,
                                    x_dtype="bf16", y_dtype="bf16", out_dtype="f32"), 20011),
    ("bf16_to_f32", C["decode"].replace(hidden=512, out_dtype="f32"), 77),
    ("fp8_small_D", C["prefill"].replace(hidden=256, n_experts=16, top_k=4, n_ranks=4), 129),
    ("k16", TINY.replace(n_experts=32, top_k=16, n_ranks=2, hidden=64), 100),
    # the largest top-k: one pick per lane of the routing warp
    ("k32_max", TINY.replace(n_experts=64, top_k=32, n_ranks=2, hidden=64), 90),
]


@pytest.mark.parametrize("name,cfg,n", SMALL_CASES, ids=[c[0] for c in SMALL_CASES])
def test_path_matches_oracle(name, cfg, n):
    inp = workloads.make_inputs(cfg, seed=11, n=n)
    inp_np = parity.numpy_inputs(inp)
    ref = oracle.run_path(cfg, inp_np)
    got = parity.run_gpu(cfg, inp)
    parity.compare_path(cfg, inp_np, ref, got)


def test_ties_break_to_lower_expert():
    cfg = TINY.replace(n_experts=16, top_k=4, n_ranks=4)
    inp = workloads.make_inputs(cfg, seed=3, n=200)
    g = torch.Generator().manual_seed(5)
    inp["logits"] = torch.randint(-2, 3, (200, 16), generator=g).float() * 0.5
    inp_np = parity.numpy_inputs(inp)
    ref = oracle.run_path(cfg, inp_np)
    got = parity.run_gpu(cfg, inp)
    parity.compare_path(cfg, inp_np, ref, got)


def test_zero_tokens():
    import combine_moe_route_11_b200 as mr
    plan = mr.Plan.from_config(TINY, n_max=64)
    dev = torch.device("cuda", 0)
    ws = plan.new_workspace(dev)
    b = plan.new_buffers(0, dev)
    b["counts"].fill_(-7)
    b["expert_off"].fill_(-7)
    mr.moe_route_topk(plan, torch.empty(0, 8, device=dev), b["topk_idx"], b["topk_w"],
                      b["counts"], b["expert_off"], ws)
    x = torch.empty(0, 256, device=dev)
    mr.moe_dispatch(plan, x, None, b["topk_idx"], b["recv"], None, b["slot_of"], b["src_of"], ws)
    mr.moe_combine(plan, b["recv"], b["topk_w"], b["slot_of"], b["out"], ws)
    assert mr.moe_get_status(plan, ws) == 0
    assert b["counts"].cpu().tolist() == [0] * 8
    assert b["expert_off"].cpu().tolist() == [0] * 9


def test_repeat_calls_vary_n_and_are_deterministic():
    """One plan and one workspace serve calls of different n; identical inputs
    give identical bytes."""
    cfg = C["decode"]
    import combine_moe_route_11_b200 as mr
    plan = mr.Plan.from_config(cfg, n_max=256)
    for n in (256, 3, 128, 64, 65):
        inp = workloads.make_inputs(cfg, seed=n, n=n)
        inp_np = parity.numpy_inputs(inp)
        ref = oracle.run_path(cfg, inp_np)
        a = parity.run_gpu(cfg, inp, plan=plan)
        b = parity.run_gpu(cfg, inp, plan=plan)
        parity.compare_path(cfg, inp_np, ref, a)
        for key in ("topk_idx", "topk_w", "slot_of", "out"):
            assert np.array_equal(a[key], b[key])


@pytest.mark.parametrize("name", ["prefill", "skewed", "decode"])
def test_full_size(name):
    cfg = C[name]
    inp = workloads.make_inputs(cfg, seed=0)
    inp_np = parity.numpy_inputs(inp)
    ref = oracle.run_path(cfg, inp_np, with_recv=False)
    got = parity.run_gpu(cfg, inp, want=())
    assert got["status"] == 0
    assert np.array_equal(got["topk_idx"], ref["topk_idx"])
    parity.assert_weights_close(got["topk_w"], ref["topk_w"])
    assert np.array_equal(got["counts"], ref["counts"])
    assert np.array_equal(got["expert_off"].astype(np.int64), ref["expert_off"])
    assert np.array_equal(got["slot_of"], ref["slot_of"])
    fs = parity.filled_slots(ref["slot_of"])
    assert np.array_equal(got["src_of"][fs], ref["src_of"][fs])
    # property at any size: every (t, j) slot holds a byte copy of x[t]
    dev = got["dev"]
    x = inp["x"].cuda()
    idx = dev["slot_of"].view(-1).long()
    k = cfg.top_k
    for lo in range(0, idx.numel(), 8192):
        sl = idx[lo:lo + 8192]
        src = torch.arange(lo, lo + sl.numel(), device=x.device) // k
        assert torch.equal(dev["recv"][sl], x[src])
        if cfg.scale_block:
            assert torch.equal(dev["recv_scale"][sl], inp["x_scale"].cuda()[src])
    # combine on sampled tokens: the oracle runs the whole path on them alone
    g = np.random.default_rng(1)
    sample = np.sort(g.choice(cfg.n, size=min(cfg.n, 96), replace=False))
    sub = {kk: (v[sample] if v is not None and kk in ("logits", "x", "x_scale") else v)
           for kk, v in inp_np.items()}
    sref = oracle.run_path(cfg, sub)
    parity.assert_combine_close(got["out"][sample], sref["out"], sref["out_abs"], cfg.out_dtype)


def test_unfilled_rows_are_never_written():
    cfg = C["prefill"]
    import combine_moe_route_11_b200 as mr
    n = 1024
    inp = workloads.make_inputs(cfg, seed=2, n=n)
    plan = mr.Plan.from_config(cfg, n_max=n)
    dev = torch.device("cuda", 0)
    ws = plan.new_workspace(dev)
    b = plan.new_buffers(n, dev)
    b["recv"].fill_(0xAB)
    b["recv_scale"].fill_(-3.0)
    mr.moe_route_topk(plan, inp["logits"].cuda(), b["topk_idx"], b["topk_w"], b["counts"],
                      b["expert_off"], ws)
    mr.moe_dispatch(plan, inp["x"].cuda(), inp["x_scale"].cuda(), b["topk_idx"], b["recv"],
                    b["recv_scale"], b["slot_of"], b["src_of"], ws)
    assert mr.moe_get_status(plan, ws) == 0
    filled = torch.zeros(b["recv"].shape[0], dtype=torch.bool, device=dev)
    filled[b["slot_of"].view(-1).long()] = True
    assert bool((b["recv"][~filled] == 0xAB).all())
    assert bool((b["recv_scale"][~filled] == -3.0).all())
    # filled rows of a region are exactly [expert_off[e], expert_off[e] + counts[e])
    off = b["expert_off"].cpu().numpy()
    cnt = b["counts"].cpu().numpy()
    want = np.zeros(b["recv"].shape[0], bool)
    for e in range(cfg.n_experts):
        want[off[e]:off[e] + cnt[e]] = True
    assert np.array_equal(filled.cpu().numpy(), want)


def test_layer_identity_matches_oracle():
    import combine_moe_route_11_b200 as mr
    # up to 1024 tokens moe_layer routes and dispatches in one launch, above in two
    for cfg, n in ((TINY, 64), (C["prefill"], 300), (C["decode"], 128),
                   (C["skewed"].replace(hidden=512), 1500)):
        inp = workloads.make_inputs(cfg, seed=4, n=n)
        inp_np = parity.numpy_inputs(inp)
        ref = oracle.run_path(cfg, inp_np)
        plan = mr.Plan.from_config(cfg, n_max=n)
        dev = torch.device("cuda", 0)
        ws = plan.new_workspace(dev, layer=True)
        out = torch.empty(n, cfg.hidden, dtype=plan.new_buffers(1, dev)["out"].dtype, device=dev)
        xs = inp["x_scale"].cuda() if inp["x_scale"] is not None else None
        mr.moe_layer(plan, inp["logits"].cuda(), inp["x"].cuda(), xs, None, None, out, ws)
        assert mr.moe_get_status(plan, ws) == 0
        parity.assert_combine_close(parity.to_bits(out), ref["out"], ref["out_abs"],
                                    cfg.out_dtype)
        so = mr.moe_layer_buffer(plan, ws, "slot_of", torch.int32, (n, cfg.top_k))
        assert np.array_equal(parity.to_bits(so), ref["slot_of"])


def test_device_detects_bad_indices():
    """Caller-supplied out-of-range ids and slots are flagged, skipped, and
    never dereferenced."""
    import combine_moe_route_11_b200 as mr
    cfg = TINY
    n = 64
    inp = workloads.make_inputs(cfg, seed=1, n=n)
    plan = mr.Plan.from_config(cfg, n_max=n)
    dev = torch.device("cuda", 0)
    ws = plan.new_workspace(dev)
    b = plan.new_buffers(n, dev)
    mr.moe_route_topk(plan, inp["logits"].cuda(), b["topk_idx"], b["topk_w"], b["counts"],
                      b["expert_off"], ws)
    assert mr.moe_get_status(plan, ws) == 0
    bad_idx = b["topk_idx"].clone()
    bad_idx[5, 1] = cfg.n_experts + 3
    bad_idx[9, 0] = -1
    mr.moe_dispatch(plan, inp["x"].cuda(), None, bad_idx, b["recv"], None, b["slot_of"],
                    b["src_of"], ws)
    assert mr.moe_get_status(plan, ws) == mr_status("MOE_ERR_DEVICE_INDEX")
    assert mr.moe_get_status(plan, ws) == 0          # read clears
    bad_slot = b["slot_of"].clone()
    bad_slot[3, 0] = plan.recv_rows(n)
    bad_slot[4, 1] = -5
    mr.moe_combine(plan, b["recv"], b["topk_w"], bad_slot, b["out"], ws)
    assert mr.moe_get_status(plan, ws) == mr_status("MOE_ERR_DEVICE_INDEX")
    logits = inp["logits"].clone()
    logits[7, :] = float("nan")
    logits[8, 1:] = float("-inf")
    mr.moe_route_topk(plan, logits.cuda(), b["topk_idx"], b["topk_w"], b["counts"],
                      b["expert_off"], ws)
    assert mr.moe_get_status(plan, ws) == mr_status("MOE_ERR_NONFINITE")
    idx = b["topk_idx"].cpu().numpy()
    assert ((idx >= 0) & (idx < cfg.n_experts)).all()
    assert int(b["counts"].sum()) == n * cfg.top_k


def mr_status(name):
    return {"MOE_ERR_DEVICE_INDEX": -5, "MOE_ERR_NONFINITE": -7}[name]
