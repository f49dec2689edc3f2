"""Host-side logic of bench.py without a GPU: max-over-ranks timing and the
whole-job aggregate across two gloo ranks, the algorithmic byte counts, and
the buffer-set rotation that keeps steps out of L2."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch
    import bench
    w, r, _ = bench.init_dist()
    dev = torch.device("cpu")
    bench.barrier(dev)
    # rank r "took" 10 + 5r ms per step; the job is as slow as its slowest rank
    t = bench.reduce_max(10.0 + 5.0 * r, dev)
    value = bench.job_throughput(w, 4096, t)
    bench.barrier(dev)
    import torch.distributed as dist
    dist.destroy_process_group()
    q.put((r, w, t, value))


def test_two_gloo_ranks_report_the_slowest_rank():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    for r, w, t, value in got:
        assert w == world
        assert t == 15.0  # max over ranks
        assert value == pytest.approx(2 * 4096 / 0.015)


def test_algorithmic_bytes_and_rotation():
    sys.path.insert(0, ROOT)
    import bench
    import workloads
    b = bench.algorithmic_bytes(workloads.CONFIGS["prefill"], 4096)
    assert b["step"] == 805961728
    assert b["combine"] == 4096 * 8 * 7168 * 2 + 4096 * 8 * 8 + 4096 * 7168 * 2
    # a prefill step streams > 4x L2 on its own; a decode step needs rotation
    assert bench.buffer_sets(workloads.CONFIGS["prefill"], 4096) == 1
    nd = bench.buffer_sets(workloads.CONFIGS["decode"], 128)
    step = bench.algorithmic_bytes(workloads.CONFIGS["decode"], 128)["step"]
    assert (nd - 1) * step >= 4 * bench.L2_BYTES


def test_fused_batch_limit_agrees_with_the_library():
    """bench.py describes the step without importing the library (the
    reference arm runs without it); its copy of the one-launch limit must be
    the binding's, which the header documents (32 route blocks of 32)."""
    sys.path.insert(0, ROOT)
    import bench
    import combine_moe_route_11_b200 as mr
    assert bench.FUSED_MAX_TOKENS == mr.FUSED_MAX_TOKENS == 32 * 32
    with open(os.path.join(ROOT, "include", "moeroute.h")) as f:
        assert "n <= 1024 tokens" in f.read()


def test_clock_sampler_window_and_short_region_fallback():
    """Samples inside the timed region decide the clock record; a region
    shorter than the sampling period reports the nearest samples and says so.
    Reasons seen in any sample of the window are reported."""
    sys.path.insert(0, ROOT)
    import bench
    s = bench.ClockSampler.__new__(bench.ClockSampler)
    s.running, s.proc, s.thread, s.source = False, None, None, "test"
    s.samples = [(1.00, 1965.0, 1965.0, set()), (1.01, 1410.0, 1965.0, {"sw_power_cap"}),
                 (1.02, 1400.0, 1965.0, {"sw_power_cap"}), (1.05, 1965.0, 1965.0, set())]

    class _Proc:  # stands in for the nvidia-smi child that stop() ends
        def terminate(self):
            pass

        def wait(self, timeout=None):
            return 0

    s.proc = _Proc()
    rec = s.stop(1.005, 1.025)
    assert rec["samples"] == 2 and rec["sm_mhz"] == 1405.0
    assert rec["reasons"] == ["sw_power_cap"] and rec["window"] == "during the timed region"
    s.proc = _Proc()
    rec = s.stop(1.031, 1.032)  # between samples: the two nearest
    assert rec["samples"] == 2 and rec["window"].startswith("nearest")


def test_percentiles_nearest_rank():
    sys.path.insert(0, ROOT)
    import bench
    p = bench.percentiles([5.0, 1.0, 4.0, 2.0, 3.0, 10.0, 6.0, 7.0, 8.0, 9.0, 0.0])
    assert (p["n"], p["min"], p["max"], p["p50"]) == (11, 0.0, 10.0, 5.0)
    assert (p["p10"], p["p90"]) == (1.0, 9.0)
    assert bench.percentiles([]) == {}


def test_path_dtype_names_what_the_path_moves():
    sys.path.insert(0, ROOT)
    import bench
    import workloads
    d = bench.path_dtype(workloads.CONFIGS["prefill"])
    assert d.startswith("fp8_e4m3 + fp32 scale per 128 cols rows") and "fp32 accumulate" in d
    assert "bf16 Y / bf16 out" in d
    assert bench.path_dtype(workloads.CONFIGS["tiny"]).startswith("fp32 rows")


def test_oracle_on_host_cores_splits_the_batch():
    """OracleCores runs the unchanged oracle in worker processes, one slice
    of the batch each: two workers on the tiny workload start, answer every
    step with a positive wall time, and cover all tokens; host_cpu names the
    cores and the CPU model the numbers come from."""
    sys.path.insert(0, ROOT)
    import bench
    import workloads
    import oracle
    oracle.build()
    cfg = workloads.CONFIGS["tiny"]
    pool = bench.OracleCores(cfg, bench.oracle_inputs(cfg, 64), workers=2)
    try:
        assert pool.workers == 2 and pool.tokens == 64
        walls = [pool.step() for _ in range(2)]
    finally:
        pool.close()
    assert all(w > 0 for w in walls)
    host = bench.host_cpu()
    assert host["cores_available"] >= 1 and host["nproc"] >= 1
    assert "cpu_model" in host


def test_reference_line_reports_measured_steps(capsys):
    """The reference arm's ms_per_step is the measured time of the steps it
    ran on its sample (tokens_per_step), so steps x ms_per_step is time that
    was spent; value = sampled tokens / step time."""
    sys.path.insert(0, ROOT)
    import json
    import bench
    import oracle
    oracle.build()
    bench.main(["--impl", "reference", "--workload", "tiny", "--steps", "3", "--warmup", "3"])
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["steps"] == 3
    assert line["tokens_per_step"] <= 64
    assert line["value"] == pytest.approx(line["tokens_per_step"] / (line["ms_per_step"] * 1e-3))
    assert line["cpu_baseline"]["cores"] >= 1 and "cpu_model" in line["cpu_baseline"]
    assert line["step_ms"]["n"] == 3


def test_traffic_record_hash_ignores_comments_only():
    """A traffic record stays tied to the code it was captured on: comment
    edits keep the hash, a code edit changes it."""
    import bench
    a = b"// header\nint f(int x) {  /* twice */\n  return 2 * x;  // done\n}\n"
    b = b"int f(int x) {\n\n  return 2 * x;\n}   \n// trailing note\n"
    c = b"int f(int x) {\n  return 3 * x;\n}\n"
    assert bench._strip_comments(a) == bench._strip_comments(b)
    assert bench._strip_comments(a) != bench._strip_comments(c)
