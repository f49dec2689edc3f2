"""One host core's share of a timed oracle run -- TEST INFRASTRUCTURE ONLY.

bench.py's CPU-baseline and reference legs start one of these per host core
(``python -m oracle.timing_worker <inputs.npz> <config.json>``).  The worker
loads its slice of the batch, then for every line "go" on standard input
runs the oracle's whole path (route, counts, offsets, slots, dispatch,
expert, combine) on that slice -- the unchanged single-threaded C oracle --
and prints the seconds it took; "quit" ends it.  It imports numpy and the
oracle only, so a worker starts quickly and holds little memory besides its
slice.
"""
from __future__ import annotations

import json
import os
import sys
import time
import types

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import oracle  # noqa: E402


def main(argv) -> int:
    data = np.load(argv[1])
    inp = {k: data[k] for k in data.files}
    for k in ("x_scale", "w_gate_up", "w_down", "w_gate_up_scale", "w_down_scale"):
        inp.setdefault(k, None)
    with open(argv[2]) as f:
        cfg = types.SimpleNamespace(**json.load(f))
    orc = oracle.default()
    print("ready", flush=True)
    for line in sys.stdin:
        cmd = line.strip()
        if cmd == "quit":
            break
        if cmd != "go":
            continue
        t0 = time.perf_counter()
        orc.run_path(cfg, inp)
        print(f"{time.perf_counter() - t0:.9f}", flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main(sys.argv))
