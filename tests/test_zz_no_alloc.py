"""moe_route_topk_noalloc against moe_route_topk, through the C ABI.

The allocation-free routing call serves callers that cannot allocate device
memory for a workspace (a plugin whose host framework owns every device
allocation, or code that must not allocate once running).  Its scratch is a
fixed array inside the library, so these tests check that it returns exactly
what the workspace-based call returns, on two calls in a row (the second call
finds the first call's leftovers in the shared array), and that a call too
large for the array is refused before anything runs.
"""
import ctypes

import numpy as np
import pytest
import torch

import parity
import workloads

pytestmark = pytest.mark.gpu

MOE_ERR_WORKSPACE = -4
MOE_ERR_NONFINITE = -7


def _lib():
    import combine_moe_route_11_b200 as mr
    lib = mr._lib
    P, i32 = ctypes.c_void_p, ctypes.c_int32
    lib.moe_route_topk_noalloc.restype = ctypes.c_int
    lib.moe_route_topk_noalloc.argtypes = [P, i32, P, P, P, P, P, P]
    lib.moe_route_topk_noalloc_bytes.restype = ctypes.c_size_t
    lib.moe_route_topk_noalloc_bytes.argtypes = [P, i32]
    lib.moe_route_topk_noalloc_status.restype = ctypes.c_int
    lib.moe_route_topk_noalloc_status.argtypes = [P]
    return mr, lib


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _route_noalloc(lib, plan, logits, out, stream):
    return lib.moe_route_topk_noalloc(plan.handle, logits.shape[0], _ptr(logits),
                                      _ptr(out["topk_idx"]), _ptr(out["topk_w"]),
                                      _ptr(out["counts"]), _ptr(out["expert_off"]),
                                      ctypes.c_void_p(stream.cuda_stream))


@pytest.mark.parametrize("name,n", [("prefill", 4096), ("skewed", 3000), ("skewed", 6001),
                                    ("tiny", 61)])
def test_noalloc_matches_workspace_route_twice(name, n):
    mr, lib = _lib()
    cfg = workloads.CONFIGS[name]
    dev = torch.device("cuda", 0)
    plan = mr.Plan.from_config(cfg, n_max=n)
    assert lib.moe_route_topk_noalloc_bytes(plan.handle, n) <= (1 << 20)
    stream = torch.cuda.current_stream(dev)
    ws = plan.new_workspace(dev)
    for call, seed in enumerate((21, 22)):
        logits = workloads.make_inputs(cfg, seed=seed, n=n)["logits"].to(dev)
        ref = plan.new_buffers(n, dev)
        mr.moe_route_topk(plan, logits, ref["topk_idx"], ref["topk_w"], ref["counts"],
                          ref["expert_off"], ws)
        got = plan.new_buffers(n, dev)
        for key in ("topk_idx", "counts", "expert_off"):
            got[key].fill_(-1)
        assert _route_noalloc(lib, plan, logits, got, stream) == 0, f"call {call}"
        torch.cuda.synchronize()
        for key in ("topk_idx", "counts", "expert_off"):
            assert torch.equal(got[key], ref[key]), f"{key} differs on call {call}"
        parity.assert_weights_close(parity.to_bits(got["topk_w"]), parity.to_bits(ref["topk_w"]))
    assert mr.moe_get_status(plan, ws) == 0


def test_noalloc_refuses_calls_beyond_its_scratch():
    mr, lib = _lib()
    # E=512 experts over 16384 tokens: two 512 x 512 int32 tables, over 1 MiB
    cfg = workloads.CONFIGS["tiny"].replace(n_experts=512, top_k=8, n_ranks=8, hidden=128)
    n = 16384
    plan = mr.Plan.from_config(cfg, n_max=n)
    assert lib.moe_route_topk_noalloc_bytes(plan.handle, n) > (1 << 20)
    assert lib.moe_route_topk_noalloc_bytes(plan.handle, 1024) <= (1 << 20)
    dev = torch.device("cuda", 0)
    logits = torch.zeros(n, cfg.n_experts, device=dev)
    out = {"topk_idx": torch.empty(n, 8, dtype=torch.int32, device=dev),
           "topk_w": torch.empty(n, 8, dtype=torch.float32, device=dev),
           "counts": torch.full((512,), -9, dtype=torch.int32, device=dev),
           "expert_off": torch.empty(513, dtype=torch.int32, device=dev)}
    rc = _route_noalloc(lib, plan, logits, out, torch.cuda.current_stream(dev))
    assert rc == MOE_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert bool((out["counts"] == -9).all())  # nothing ran


def test_noalloc_zero_tokens_then_a_batch():
    """n = 0 returns MOE_OK with zero counts and offsets (as moe_route_topk
    does), and a following call with tokens still matches the workspace call."""
    mr, lib = _lib()
    cfg = workloads.CONFIGS["decode"]
    n = 128
    dev = torch.device("cuda", 0)
    plan = mr.Plan.from_config(cfg, n_max=n)
    stream = torch.cuda.current_stream(dev)
    ws = plan.new_workspace(dev)
    empty = torch.empty(0, cfg.n_experts, device=dev)
    ref0, got0 = plan.new_buffers(1, dev), plan.new_buffers(1, dev)
    got0["counts"].fill_(-1)
    got0["expert_off"].fill_(-1)
    mr.moe_route_topk(plan, empty, ref0["topk_idx"][:0], ref0["topk_w"][:0], ref0["counts"],
                      ref0["expert_off"], ws)
    assert _route_noalloc(lib, plan, empty, got0, stream) == 0
    torch.cuda.synchronize()
    assert lib.moe_route_topk_noalloc_status(ctypes.c_void_p(stream.cuda_stream)) == 0
    assert bool((got0["counts"] == 0).all())
    assert torch.equal(got0["expert_off"], ref0["expert_off"])
    logits = workloads.make_inputs(cfg, seed=23, n=n)["logits"].to(dev)
    ref, got = plan.new_buffers(n, dev), plan.new_buffers(n, dev)
    mr.moe_route_topk(plan, logits, ref["topk_idx"], ref["topk_w"], ref["counts"],
                      ref["expert_off"], ws)
    assert _route_noalloc(lib, plan, logits, got, stream) == 0
    torch.cuda.synchronize()
    for key in ("topk_idx", "counts", "expert_off"):
        assert torch.equal(got[key], ref[key]), key
    assert mr.moe_get_status(plan, ws) == 0


def test_noalloc_status_reports_the_last_call():
    """A logit row with fewer than k finite values is a device-detected error
    of the allocation-free call too: moe_route_topk_noalloc_status reports it,
    and the next clean call starts again from MOE_OK."""
    mr, lib = _lib()
    cfg = workloads.CONFIGS["tiny"]
    n = 64
    dev = torch.device("cuda", 0)
    plan = mr.Plan.from_config(cfg, n_max=n)
    stream = torch.cuda.current_stream(dev)
    sp = ctypes.c_void_p(stream.cuda_stream)
    logits = workloads.make_inputs(cfg, seed=24, n=n)["logits"]
    bad = logits.clone()
    bad[5, :] = float("nan")
    out = plan.new_buffers(n, dev)
    assert _route_noalloc(lib, plan, bad.to(dev), out, stream) == 0
    assert lib.moe_route_topk_noalloc_status(sp) == MOE_ERR_NONFINITE
    assert _route_noalloc(lib, plan, logits.to(dev), out, stream) == 0
    assert lib.moe_route_topk_noalloc_status(sp) == 0
