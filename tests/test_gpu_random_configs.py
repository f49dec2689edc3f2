"""Randomised configurations, each checked against the oracle on both GPU
paths (moe_route_topk + moe_dispatch, and moe_route_dispatch) and the two
paths against each other bit for bit.

The configurations are drawn from a fixed seed, so the set is the same on
every run: expert counts 2..96 (with and without the float4 logit path), any
rank count dividing E, top-k up to min(E, 32), batches 0..700 (ragged route
blocks, and both sides of the one-launch limit at small sizes), row widths of
several 16-byte multiples, and every supported dtype combination, FP8 with
its per-128-column scales.
"""
import random

import numpy as np
import pytest

import oracle
import parity
import workloads

pytestmark = pytest.mark.gpu


def _random_configs(count=48, seed=2027):
    rng = random.Random(seed)
    base = workloads.CONFIGS["tiny"]
    out = []
    while len(out) < count:
        E = rng.choice([2, 3, 8, 12, 16, 33, 64, 96, 128])
        R = rng.choice([r for r in range(1, E + 1) if E % r == 0 and r <= 16])
        k = rng.randint(1, min(E, 32))
        kind = rng.choice(["f32", "bf16", "bf16_f32", "fp8"])
        if kind == "fp8":
            D = rng.choice([128, 256, 512])
            cfg = base.replace(x_dtype="fp8_e4m3", y_dtype="bf16", out_dtype="bf16",
                               scale_block=128)
        elif kind == "f32":
            D = rng.choice([4, 12, 64, 200])
            cfg = base.replace(x_dtype="f32", y_dtype="f32", out_dtype="f32")
        elif kind == "bf16":
            D = rng.choice([8, 24, 128, 520])
            cfg = base.replace(x_dtype="bf16", y_dtype="bf16", out_dtype="bf16")
        else:
            D = rng.choice([8, 64, 264])
            cfg = base.replace(x_dtype="bf16", y_dtype="bf16", out_dtype="f32")
        n = rng.choice([0, 1, 31, 32, 33, rng.randint(2, 300), rng.randint(300, 700)])
        logits = rng.choice(["normal", "zipf1.2"])
        cfg = cfg.replace(name=f"rand{len(out)}", n=max(n, 1), hidden=D, n_experts=E,
                          top_k=k, n_ranks=R, logits=logits)
        out.append((cfg, n))
    return out


CASES = _random_configs()


@pytest.mark.parametrize("cfg,n", CASES, ids=[f"{c.name}-E{c.n_experts}-k{c.top_k}-R{c.n_ranks}"
                                               f"-D{c.hidden}-{c.x_dtype}-n{n}"
                                               for c, n in CASES])
def test_random_config_both_paths(cfg, n):
    if n == 0:
        pytest.skip("n = 0 is covered by the zero-token tests")
    inp = workloads.make_inputs(cfg, seed=n + cfg.hidden, n=n)
    inp_np = parity.numpy_inputs(inp)
    ref = oracle.run_path(cfg, inp_np)
    two = parity.run_gpu(cfg, inp, fused=False)
    one = parity.run_gpu(cfg, inp, fused=True)
    parity.compare_path(cfg, inp_np, ref, two)
    parity.compare_path(cfg, inp_np, ref, one)
    for key in ("topk_idx", "topk_w", "counts", "expert_off", "slot_of", "out"):
        assert np.array_equal(one[key], two[key]), key
