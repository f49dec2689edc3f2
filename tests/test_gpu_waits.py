"""Bounded device-side waits, and CUDA-graph replays of the kernels that keep
state in the workspace's control block (route kernel, grouped GEMMs).

The route kernel's scanners and the one-launch route + dispatch kernel's
grid barrier wait on words in the workspace's control block.  Here the
failure is made on the host: the arrival counter is set to a value from
which the last arrival is never reached, so nothing ever bumps the
generation the waiting blocks poll.  Each wait gives up after its bound
(2^31 SM cycles, about a second), the kernel records MOE_ERR_TIMEOUT in the
status word and returns without writing through the workspace's tables,
and the context stays usable: moe_workspace_init clears the control words
and the next call matches the oracle.

The route kernel's expert totals alternate between two halves by a call
generation kept in the workspace.  A CUDA graph replays the same launches
with the generation advancing on the device, so the replays below check
that every replay still routes and dispatches exactly.
"""
import time

import numpy as np
import pytest
import torch

import oracle
import parity
import workloads

pytestmark = pytest.mark.gpu

MOE_ERR_TIMEOUT = -6
C = workloads.CONFIGS
# control block words (uint32): arrive, status, gen, ticket, rgen
ARRIVE, STATUS, GEN, TICKET, RGEN = 0, 1, 2, 3, 4


def _ctrl(ws):
    return ws[:256].view(torch.int32)


def test_route_scanner_wait_times_out_then_recovers():
    import combine_moe_route_11_b200 as mr
    cfg = C["decode"]
    n = 100  # 4 route blocks, 4 CTAs, all of them scanners
    inp = workloads.make_inputs(cfg, seed=71, n=n)
    dev = torch.device("cuda", 0)
    plan = mr.Plan.from_config(cfg, n_max=n)
    ws = plan.new_workspace(dev)
    b = plan.new_buffers(n, dev)
    logits = inp["logits"].to(dev)
    _ctrl(ws)[TICKET] = 1000  # arrivals 1000..1003: none is the last of 4
    torch.cuda.synchronize()
    t0 = time.time()
    mr.moe_route_topk(plan, logits, b["topk_idx"], b["topk_w"], b["counts"], b["expert_off"], ws)
    assert mr.moe_get_status(plan, ws) == MOE_ERR_TIMEOUT
    assert time.time() - t0 < 30.0
    mr.moe_workspace_init(plan, ws)
    torch.cuda.synchronize()
    assert int(_ctrl(ws)[:8].abs().sum()) == 0
    inp_np = parity.numpy_inputs(inp)
    ref = oracle.run_path(cfg, inp_np)
    got = parity.run_gpu(cfg, inp, plan=plan, ws=ws)
    assert got["status"] == 0
    parity.compare_path(cfg, inp_np, ref, got)


def test_fused_grid_barrier_times_out_then_recovers():
    import combine_moe_route_11_b200 as mr
    cfg = C["decode"]
    n = 64
    inp = workloads.make_inputs(cfg, seed=72, n=n)
    dev = torch.device("cuda", 0)
    plan = mr.Plan.from_config(cfg, n_max=n)
    ws = plan.new_workspace(dev)
    b = plan.new_buffers(n, dev)
    _ctrl(ws)[ARRIVE] = 1000  # the barrier's count never reaches the grid size
    torch.cuda.synchronize()
    t0 = time.time()
    mr.moe_route_dispatch(plan, inp["logits"].to(dev), inp["x"].to(dev), None, b["topk_idx"],
                          b["topk_w"], b["counts"], b["expert_off"], b["recv"], None,
                          b["slot_of"], b["src_of"], ws)
    assert mr.moe_get_status(plan, ws) == MOE_ERR_TIMEOUT
    assert time.time() - t0 < 30.0
    mr.moe_workspace_init(plan, ws)
    inp_np = parity.numpy_inputs(inp)
    ref = oracle.run_path(cfg, inp_np)
    got = parity.run_gpu(cfg, inp, plan=plan, ws=ws, fused=True)
    assert got["status"] == 0
    parity.compare_path(cfg, inp_np, ref, got)


@pytest.mark.parametrize("name,n", [("prefill", 300), ("skewed", 6000)])
def test_route_and_dispatch_replayed_in_a_cuda_graph(name, n):
    """moe_route_topk + moe_dispatch captured once and replayed with new
    logits and rows copied into the captured inputs: every replay matches
    the oracle (the totals' halves and the generation advance on the device
    between replays; 6000 tokens give several route blocks per CTA)."""
    import combine_moe_route_11_b200 as mr
    cfg = C[name]
    dev = torch.device("cuda", 0)
    plan = mr.Plan.from_config(cfg, n_max=n)
    ws = plan.new_workspace(dev)
    b = plan.new_buffers(n, dev)
    first = workloads.make_inputs(cfg, seed=80, n=n)
    logits = first["logits"].to(dev)
    x = first["x"].to(dev)
    xs = first["x_scale"].to(dev) if first.get("x_scale") is not None else None
    stream = torch.cuda.Stream(dev)
    stream.wait_stream(torch.cuda.current_stream(dev))
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        # one eager call first, so that the first-call work (attributes, maps) is done
        mr.moe_route_topk(plan, logits, b["topk_idx"], b["topk_w"], b["counts"],
                          b["expert_off"], ws, stream)
        mr.moe_dispatch(plan, x, xs, b["topk_idx"], b["recv"], b["recv_scale"], b["slot_of"],
                        b["src_of"], ws, stream)
        stream.synchronize()
        with torch.cuda.graph(graph, stream=stream):
            mr.moe_route_topk(plan, logits, b["topk_idx"], b["topk_w"], b["counts"],
                              b["expert_off"], ws, stream)
            mr.moe_dispatch(plan, x, xs, b["topk_idx"], b["recv"], b["recv_scale"],
                            b["slot_of"], b["src_of"], ws, stream)
    torch.cuda.current_stream(dev).wait_stream(stream)
    for rep, seed in enumerate((81, 82, 83)):
        inp = workloads.make_inputs(cfg, seed=seed, n=n)
        logits.copy_(inp["logits"].to(dev))
        x.copy_(inp["x"].to(dev))
        if xs is not None:
            xs.copy_(inp["x_scale"].to(dev))
        torch.cuda.synchronize()
        graph.replay()
        torch.cuda.synchronize()
        assert mr.moe_get_status(plan, ws) == 0
        ref = oracle.run_path(cfg, parity.numpy_inputs(inp))
        for key in ("topk_idx", "counts", "expert_off", "slot_of"):
            got = parity.to_bits(b[key]).astype(np.int64)
            assert np.array_equal(got, np.asarray(ref[key]).astype(np.int64)), (rep, key)
        parity.assert_weights_close(parity.to_bits(b["topk_w"]), ref["topk_w"])
        slot_of = parity.to_bits(b["slot_of"]).reshape(-1)
        recv = parity.to_bits(b["recv"])
        x_bits = parity.to_bits(inp["x"])
        tok = np.arange(slot_of.size) // cfg.top_k
        assert np.array_equal(recv[slot_of], x_bits[tok]), rep
    del graph


@pytest.mark.parametrize("fp8", [False, True], ids=["bf16_experts", "fp8_experts"])
def test_layer_replayed_in_a_cuda_graph_equals_eager(fp8):
    """The whole layer (route kernel, dispatch, grouped GEMMs with tiles taken
    from the workspace counter, combine) captured once and replayed with
    other inputs gives, on every replay, the bytes of an eager call on the
    same inputs: the tile counter is reset by each launch's last CTA, and
    which CTA computes a tile does not change its result.  1300 tokens take
    the two-launch route + dispatch path; Zipf routing gives experts several
    m-tiles."""
    import combine_moe_route_11_b200 as mr
    base = C["layer_fp8" if fp8 else "layer"]
    cfg = base.replace(hidden=256, inter=256, n_experts=16, top_k=2, n_ranks=4, logits="zipf1.2")
    n = 1300
    dev = torch.device("cuda", 0)
    plan = mr.Plan.from_config(cfg, n_max=n)
    first = workloads.make_inputs(cfg, seed=90, n=n)
    w = {k: first[k].to(dev) for k in ("w_gate_up", "w_gate_up_scale", "w_down", "w_down_scale")
         if first.get(k) is not None}
    logits = first["logits"].to(dev)
    x = first["x"].to(dev)
    xs = first["x_scale"].to(dev) if first.get("x_scale") is not None else None
    out = torch.empty(n, cfg.hidden, dtype=torch.bfloat16, device=dev)
    ws = plan.new_workspace(dev, layer=True)

    def layer(stream=None):
        if fp8:
            mr.moe_layer_fp8(plan, logits, x, xs, w["w_gate_up"], w["w_gate_up_scale"],
                             w["w_down"], w["w_down_scale"], out, ws, stream)
        else:
            mr.moe_layer(plan, logits, x, xs, w["w_gate_up"], w["w_down"], out, ws, stream)

    def load(inp):
        logits.copy_(inp["logits"].to(dev))
        x.copy_(inp["x"].to(dev))
        if xs is not None:
            xs.copy_(inp["x_scale"].to(dev))

    inputs = [workloads.make_inputs(cfg, seed=s, n=n) for s in (91, 92)]
    eager = []
    for inp in inputs:
        load(inp)
        layer()
        assert mr.moe_get_status(plan, ws) == 0
        eager.append(out.clone())
    stream = torch.cuda.Stream(dev)
    stream.wait_stream(torch.cuda.current_stream(dev))
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(graph, stream=stream):
            layer(stream)
    torch.cuda.current_stream(dev).wait_stream(stream)
    for i in (0, 1, 0):
        load(inputs[i])
        torch.cuda.synchronize()
        graph.replay()
        torch.cuda.synchronize()
        assert mr.moe_get_status(plan, ws) == 0
        assert torch.equal(out, eager[i]), f"replay of input {i} differs from the eager call"
    del graph
