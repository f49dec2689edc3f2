"""Router GEMM with the top-k fused (moe_router_topk) against the CPU oracle.

The GPU sums bf16 products in fp32 on the tensor cores, split over the CTAs
of a cluster and added in a fixed order; the oracle sums in double and
rounds once.  So:
  * logits: |g - r| <= 2^-14 * sum_d |x_d w_d| (a generous multiple of the
    fp32 accumulation bound of D / 16 + 16 roundings of 2^-24 each; a
    missing k-block, a wrong row or a transposed operand is off by O(1));
  * the selection is checked exactly on the GPU's own logits: topk_idx,
    counts and expert_off bit for bit against the oracle's route of the
    logits the GPU returned (near-ties between the fp32 and the double sums
    cannot flip it), weights within 8 fp32 ulp of the oracle's softmax;
  * the positions left for moe_dispatch give the oracle's slots.
"""
import numpy as np
import pytest
import torch

import oracle
import parity
import workloads

pytestmark = pytest.mark.gpu

C = workloads.CONFIGS


def _inputs(cfg, n, seed, w_std=0.02):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(n, cfg.hidden, generator=g).to(torch.bfloat16)
    w = (torch.randn(cfg.n_experts, cfg.hidden, generator=g) * w_std).to(torch.bfloat16)
    return x, w


def _bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _abs_dot(x_bits, w_bits):
    xa = np.abs(torch.from_numpy(x_bits.view(np.int16)).view(torch.bfloat16).double().numpy())
    wa = np.abs(torch.from_numpy(w_bits.view(np.int16)).view(torch.bfloat16).double().numpy())
    return xa @ wa.T


def run_router(cfg, x, w, want_logits=True, dispatch=False):
    import combine_moe_route_11_b200 as mr
    n = x.shape[0]
    dev = torch.device("cuda", 0)
    plan = mr.Plan.from_config(cfg.replace(x_dtype="bf16", y_dtype="bf16", out_dtype="bf16",
                                           scale_block=0), n_max=max(n, 1))
    ws = plan.new_workspace(dev)
    b = plan.new_buffers(n, dev)
    logits = torch.empty(n, cfg.n_experts, device=dev) if want_logits else None
    xd = x.to(dev)
    mr.moe_router_topk(plan, xd, w.to(dev), logits, b["topk_idx"], b["topk_w"], b["counts"],
                       b["expert_off"], ws)
    if dispatch:
        mr.moe_dispatch(plan, xd, None, b["topk_idx"], b["recv"], None, b["slot_of"],
                        b["src_of"], ws)
    assert mr.moe_get_status(plan, ws) == 0
    torch.cuda.synchronize()
    out = {k: v.cpu() for k, v in b.items() if v is not None}
    if logits is not None:
        out["logits"] = logits.cpu()
    return out


def check(cfg, n, seed, rows=None):
    x, w = _inputs(cfg, n, seed)
    got = run_router(cfg, x, w, dispatch=True)
    xb, wb = _bits(x), _bits(w)
    sel = np.arange(n) if rows is None else np.asarray(rows)
    ref = oracle.router_logits(xb[sel], wb)
    g = got["logits"].numpy()
    bound = 2.0 ** -14 * _abs_dot(xb[sel], wb) + 1e-30
    err = np.abs(g[sel].astype(np.float64) - ref.astype(np.float64))
    assert (err <= bound).all(), f"logits: worst ratio {np.max(err / bound):.3g}"
    # the selection on the GPU's own logits, exactly
    idx, wt = oracle.route(g, cfg.top_k)
    assert np.array_equal(got["topk_idx"].numpy(), idx)
    parity.assert_weights_close(got["topk_w"].numpy(), wt)
    cnt = oracle.counts(idx, cfg.n_experts)
    off = oracle.offsets(n, cfg.n_experts, cfg.top_k, cfg.n_ranks, cnt)
    assert np.array_equal(got["counts"].numpy(), cnt)
    assert np.array_equal(got["expert_off"].numpy().astype(np.int64), off)
    slot_of, _ = oracle.slots(idx, off, cfg.n_experts)
    assert np.array_equal(got["slot_of"].numpy(), slot_of)
    return got


CASES = [
    # decode shape: one 128-token tile split over a cluster of 8
    ("decode", C["decode"], 128, None),
    # the layer's router: E = 64 (scalar lane layout), two k per expert block
    ("layer", C["layer"], 1024, None),
    # ragged last tile, E = 128, D = 4096
    ("skewed_ragged", C["skewed"], 300, None),
    # E = 8 padded to an MMA of 16 columns, D = 256 (4 k-blocks)
    ("tiny_e8", C["tiny"].replace(x_dtype="bf16", y_dtype="bf16", out_dtype="bf16"), 200, None),
    # E = 48: neither a multiple of 32 nor of 128
    ("e48_k5", C["decode"].replace(n_experts=48, top_k=5, n_ranks=4, hidden=1024), 257, None),
    # 18 tiles, the last one ragged, over clusters of 4
    ("many_tiles_ragged", C["skewed"], 2300, None),
    # 188 route blocks: the count kernel's CTAs take more than one each
    ("route_blocks_per_cta", C["skewed"], 6001, np.arange(0, 6001, 7)),
    # k = 1 and k = E
    ("k1", C["decode"].replace(top_k=1, n_ranks=1), 130, None),
    ("k_eq_e", C["decode"].replace(n_experts=16, top_k=16, n_ranks=2, hidden=512), 70, None),
]


@pytest.mark.parametrize("name,cfg,n,rows", CASES, ids=[c[0] for c in CASES])
def test_router_matches_oracle(name, cfg, n, rows):
    check(cfg, n, seed=len(name) * 7 + n, rows=rows)


def test_router_prefill_shape_sampled_rows():
    """N = 4096, D = 7168, E = 256, k = 8, R = 8 (the prefill routing shape
    with bf16 hidden rows): logits of 300 sampled rows against the oracle,
    the selection and the layout of every token exactly."""
    cfg = C["prefill"]
    rows = np.random.default_rng(5).choice(4096, 300, replace=False)
    check(cfg, 4096, seed=99, rows=np.sort(rows))


def test_router_without_logits_output_selects_the_same():
    cfg = C["decode"]
    x, w = _inputs(cfg, 128, seed=3)
    a = run_router(cfg, x, w, want_logits=True)
    b = run_router(cfg, x, w, want_logits=False)
    for key in ("topk_idx", "topk_w", "counts", "expert_off"):
        assert torch.equal(a[key], b[key]), key


@pytest.mark.parametrize("n", [1024, 4096])
def test_router_is_deterministic(n):
    """The split-K partial sums are added in cluster-rank order: two calls
    give the same logits bit for bit (clusters of 8 and of 4)."""
    cfg = C["prefill"]
    x, w = _inputs(cfg, n, seed=4)
    a = run_router(cfg, x, w)
    b = run_router(cfg, x, w)
    assert torch.equal(a["logits"], b["logits"])
    assert torch.equal(a["topk_idx"], b["topk_idx"])


def test_router_zero_tokens():
    import combine_moe_route_11_b200 as mr
    cfg = C["decode"]
    dev = torch.device("cuda", 0)
    plan = mr.Plan.from_config(cfg, n_max=8)
    ws = plan.new_workspace(dev)
    b = plan.new_buffers(1, dev)
    b["counts"].fill_(-1)
    mr.moe_router_topk(plan, torch.empty(0, cfg.hidden, dtype=torch.bfloat16, device=dev),
                       torch.zeros(cfg.n_experts, cfg.hidden, dtype=torch.bfloat16, device=dev),
                       None, b["topk_idx"][:0], b["topk_w"][:0], b["counts"], b["expert_off"], ws)
    assert mr.moe_get_status(plan, ws) == 0
    assert int(b["counts"].abs().sum()) == 0
    assert int(b["expert_off"].abs().sum()) == 0
