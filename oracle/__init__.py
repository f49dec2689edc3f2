"""CPU oracle for MoE token dispatch / combine -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It wraps ``moe_oracle.c`` (plain C,
fp64 arithmetic) through ctypes and composes its steps into the whole path.
It shares no code with the CUDA library and never calls it.

Every function takes and returns numpy arrays.  bf16 values travel as their
raw uint16 bits and FP8 e4m3 values as raw uint8 codes.

Parity pins: each step is pinned by the ``-m "not gpu"`` tests in
``tests/test_oracle_pins.py`` (brute force, closed forms, invariants and
library-routine equivalences); no step is left unpinned.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")

DT = {"f32": 0, "bf16": 1, "fp8_e4m3": 2}
DT_NP = {"f32": np.float32, "bf16": np.uint16, "fp8_e4m3": np.uint8}
ELEM_BYTES = {"f32": 4, "bf16": 2, "fp8_e4m3": 1}


def build(force: bool = False) -> str:
    """Compile moe_oracle.c with gcc (no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-std=c11", "-O2", "-fno-fast-math", "-ffp-contract=off",
               "-fPIC", "-shared", "-o", _LIB, _SRC, "-lm"]
        subprocess.check_call(cmd)
    return _LIB


def _sigs():
    P = ctypes.c_void_p
    i64, i32, ci = ctypes.c_int64, ctypes.c_int32, ctypes.c_int
    return {
        "oracle_route": (ci, [i64, i32, i32, P, P, P]),
        "oracle_router_logits": (ci, [i64, i32, i32, P, P, P]),
        "oracle_counts": (ci, [i64, i32, i32, P, P]),
        "oracle_region_rows": (i64, [i64, i32, i32, i32]),
        "oracle_offsets": (ci, [i64, i32, i32, i32, P, P]),
        "oracle_slots": (ci, [i64, i32, i32, P, P, i64, P, P]),
        "oracle_scatter_rows": (ci, [i64, i32, i64, P, P, i64, P]),
        "oracle_dequant_rows": (ci, [i64, P, i32, i32, P, P, P]),
        "oracle_swiglu_rows": (ci, [i64, P, P, i32, i32, P, P, P, P, P]),
        "oracle_combine": (ci, [i64, i32, i32, ci, P, P, P, i64, ci, P]),
        "oracle_combine_abs": (ci, [i64, i32, i32, ci, P, P, P, i64, P]),
        "oracle_bf16_to_double": (ctypes.c_double, [ctypes.c_uint16]),
        "oracle_bf16_from_double": (ctypes.c_uint16, [ctypes.c_double]),
        "oracle_e4m3_to_double": (ctypes.c_double, [ctypes.c_uint8]),
        "oracle_e4m3_from_float": (ctypes.c_uint8, [ctypes.c_float]),
        "oracle_quant_rows": (ci, [i64, P, i32, i32, P, P, P]),
        "oracle_fp8_gate_up_rows": (ci, [i64, P, P, i32, i32, i32, P, P, P, P, P, P, P]),
        "oracle_fp8_down_rows": (ci, [i64, P, P, i32, i32, i32, P, P, P, P, P]),
    }


def _p(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle {what} failed with code {rc}")


class Oracle:
    """One loaded copy of the compiled oracle (the default one, or a test's
    deliberately mutated copy)."""

    def __init__(self, lib_path: str):
        lib = ctypes.CDLL(lib_path)
        for name, (res, args) in _sigs().items():
            f = getattr(lib, name)
            f.restype, f.argtypes = res, args
        self.lib = lib

    # -------------------------------------------------------------- numbers
    def bf16_to_float(self, bits: int) -> float:
        return self.lib.oracle_bf16_to_double(int(bits))

    def bf16_from_float(self, v: float) -> int:
        return int(self.lib.oracle_bf16_from_double(float(v)))

    def e4m3_to_float(self, code: int) -> float:
        return self.lib.oracle_e4m3_to_double(int(code))

    # -------------------------------------------------------------- steps
    def route(self, logits: np.ndarray, top_k: int):
        """Top-k experts (ties to the lower id) and softmax-over-the-k weights."""
        logits = np.ascontiguousarray(logits, dtype=np.float32)
        n, e = logits.shape
        idx = np.empty((n, top_k), np.int32)
        w = np.empty((n, top_k), np.float32)
        _check(self.lib.oracle_route(n, e, top_k, _p(logits), _p(idx), _p(w)), "route")
        return idx, w

    def router_logits(self, x: np.ndarray, w_router: np.ndarray) -> np.ndarray:
        """logits[t, e] = x[t] . w_router[e] over bf16 bits, summed in double,
        rounded to fp32 ([n, D] and [E, D] uint16 -> [n, E] float32)."""
        x = np.ascontiguousarray(x, np.uint16)
        w = np.ascontiguousarray(w_router, np.uint16)
        n, d = x.shape
        e, d2 = w.shape
        assert d == d2, "x and the router weights disagree on D"
        out = np.empty((n, e), np.float32)
        _check(self.lib.oracle_router_logits(n, d, e, _p(x), _p(w), _p(out)), "router_logits")
        return out

    def counts(self, topk_idx: np.ndarray, n_experts: int) -> np.ndarray:
        topk_idx = np.ascontiguousarray(topk_idx, dtype=np.int32)
        n, k = topk_idx.shape
        c = np.empty(n_experts, np.int32)
        _check(self.lib.oracle_counts(n, n_experts, k, _p(topk_idx), _p(c)), "counts")
        return c

    def region_rows(self, n: int, n_experts: int, top_k: int, n_ranks: int) -> int:
        return int(self.lib.oracle_region_rows(n, n_experts, top_k, n_ranks))

    def offsets(self, n: int, n_experts: int, top_k: int, n_ranks: int,
                cnt: np.ndarray) -> np.ndarray:
        cnt = np.ascontiguousarray(cnt, dtype=np.int32)
        off = np.empty(n_experts + 1, np.int64)
        _check(self.lib.oracle_offsets(n, n_experts, top_k, n_ranks, _p(cnt), _p(off)),
               "offsets")
        return off

    def slots(self, topk_idx: np.ndarray, expert_off: np.ndarray, n_experts: int):
        topk_idx = np.ascontiguousarray(topk_idx, dtype=np.int32)
        expert_off = np.ascontiguousarray(expert_off, dtype=np.int64)
        n, k = topk_idx.shape
        total = int(expert_off[n_experts])
        slot_of = np.empty((n, k), np.int32)
        src_of = np.empty(total, np.int32)
        _check(self.lib.oracle_slots(n, n_experts, k, _p(topk_idx), _p(expert_off), total,
                                     _p(slot_of), _p(src_of)), "slots")
        return slot_of, src_of

    def scatter_rows(self, rows: np.ndarray, slot_of: np.ndarray,
                     total_slots: int) -> np.ndarray:
        """recv[slot_of[t, j]] = rows[t] as opaque bytes; unfilled slots stay zero."""
        rows = np.ascontiguousarray(rows)
        n = rows.shape[0]
        raw = rows.view(np.uint8).reshape(n, -1)
        row_bytes = raw.shape[1]
        k = slot_of.shape[1]
        slot_of = np.ascontiguousarray(slot_of, dtype=np.int32)
        recv = np.zeros((total_slots, row_bytes), np.uint8)
        _check(self.lib.oracle_scatter_rows(n, k, row_bytes, _p(raw), _p(slot_of),
                                            total_slots, _p(recv)), "scatter")
        return recv.view(rows.dtype).reshape((total_slots,) + rows.shape[1:])

    def dequant_rows(self, rows: np.ndarray, q: np.ndarray, scale: np.ndarray,
                     block: int) -> np.ndarray:
        """Identity expert on FP8 rows: bf16(code * block scale), listed rows only."""
        rows = np.ascontiguousarray(rows, dtype=np.int32)
        q = np.ascontiguousarray(q, dtype=np.uint8)
        scale = np.ascontiguousarray(scale, dtype=np.float32)
        total, hidden = q.shape
        y = np.zeros((total, hidden), np.uint16)
        _check(self.lib.oracle_dequant_rows(rows.size, _p(rows), hidden, block, _p(q),
                                            _p(scale), _p(y)), "dequant")
        return y

    def swiglu_rows(self, rows: np.ndarray, row_expert: np.ndarray, x: np.ndarray,
                    w_gate_up: np.ndarray, w_down: np.ndarray, want_h: bool = False):
        """SwiGLU expert on the listed rows of X (bf16 bits). Returns Y (and H)."""
        rows = np.ascontiguousarray(rows, dtype=np.int32)
        row_expert = np.ascontiguousarray(row_expert, dtype=np.int32)
        x = np.ascontiguousarray(x, dtype=np.uint16)
        w_gate_up = np.ascontiguousarray(w_gate_up, dtype=np.uint16)
        w_down = np.ascontiguousarray(w_down, dtype=np.uint16)
        total, hidden = x.shape
        inter = w_down.shape[2]
        assert w_gate_up.shape[1:] == (2 * inter, hidden) and w_down.shape[1] == hidden
        y = np.zeros((total, hidden), np.uint16)
        h = np.zeros((total, inter), np.uint16) if want_h else None
        _check(self.lib.oracle_swiglu_rows(rows.size, _p(rows), _p(row_expert), hidden, inter,
                                           _p(x), _p(w_gate_up), _p(w_down), _p(h), _p(y)),
               "swiglu")
        return (y, h) if want_h else y

    def e4m3_from_float(self, v: float) -> int:
        """Nearest finite e4m3 code, ties to even, saturating at +-448."""
        return int(self.lib.oracle_e4m3_from_float(float(v)))

    def quant_rows(self, rows: np.ndarray, h: np.ndarray, block: int):
        """FP8 codes and per-block fp32 scales of the listed bf16 rows."""
        rows = np.ascontiguousarray(rows, dtype=np.int32)
        h = np.ascontiguousarray(h, dtype=np.uint16)
        total, width = h.shape
        q = np.zeros((total, width), np.uint8)
        scale = np.zeros((total, width // block), np.float32)
        _check(self.lib.oracle_quant_rows(rows.size, _p(rows), width, block, _p(h), _p(q),
                                          _p(scale)), "quant")
        return q, scale

    def fp8_gate_up_rows(self, rows: np.ndarray, row_expert: np.ndarray, xq: np.ndarray,
                         xs: np.ndarray, w_gate_up: np.ndarray, w_gate_up_scale: np.ndarray,
                         block: int = 128, want_gu: bool = False):
        """FP8 GEMM1 + SwiGLU on the listed rows: H bf16 bits (and g, u in double)."""
        rows = np.ascontiguousarray(rows, dtype=np.int32)
        row_expert = np.ascontiguousarray(row_expert, dtype=np.int32)
        xq = np.ascontiguousarray(xq, dtype=np.uint8)
        xs = np.ascontiguousarray(xs, dtype=np.float32)
        w_gate_up = np.ascontiguousarray(w_gate_up, dtype=np.uint8)
        w_gate_up_scale = np.ascontiguousarray(w_gate_up_scale, dtype=np.float32)
        total, hidden = xq.shape
        inter = w_gate_up.shape[1] // 2
        assert w_gate_up.shape[2] == hidden and xs.shape == (total, hidden // block)
        assert w_gate_up_scale.shape == (w_gate_up.shape[0], 2 * inter // block, hidden // block)
        h = np.zeros((total, inter), np.uint16)
        g = np.zeros((total, inter)) if want_gu else None
        u = np.zeros((total, inter)) if want_gu else None
        _check(self.lib.oracle_fp8_gate_up_rows(rows.size, _p(rows), _p(row_expert), hidden,
                                                inter, block, _p(xq), _p(xs), _p(w_gate_up),
                                                _p(w_gate_up_scale), _p(h), _p(g), _p(u)),
               "fp8_gate_up")
        return (h, g, u) if want_gu else h

    def fp8_down_rows(self, rows: np.ndarray, row_expert: np.ndarray, hq: np.ndarray,
                      hs: np.ndarray, w_down: np.ndarray, w_down_scale: np.ndarray,
                      block: int = 128) -> np.ndarray:
        """FP8 GEMM2 on the listed rows: Y bf16 bits."""
        rows = np.ascontiguousarray(rows, dtype=np.int32)
        row_expert = np.ascontiguousarray(row_expert, dtype=np.int32)
        hq = np.ascontiguousarray(hq, dtype=np.uint8)
        hs = np.ascontiguousarray(hs, dtype=np.float32)
        w_down = np.ascontiguousarray(w_down, dtype=np.uint8)
        w_down_scale = np.ascontiguousarray(w_down_scale, dtype=np.float32)
        total, inter = hq.shape
        hidden = w_down.shape[1]
        assert w_down.shape[2] == inter and hs.shape == (total, inter // block)
        assert w_down_scale.shape == (w_down.shape[0], hidden // block, inter // block)
        y = np.zeros((total, hidden), np.uint16)
        _check(self.lib.oracle_fp8_down_rows(rows.size, _p(rows), _p(row_expert), hidden, inter,
                                             block, _p(hq), _p(hs), _p(w_down),
                                             _p(w_down_scale), _p(y)), "fp8_down")
        return y

    def combine(self, y: np.ndarray, y_dtype: str, topk_w: np.ndarray, slot_of: np.ndarray,
                out_dtype: str) -> np.ndarray:
        y = np.ascontiguousarray(y, dtype=DT_NP[y_dtype])
        topk_w = np.ascontiguousarray(topk_w, dtype=np.float32)
        slot_of = np.ascontiguousarray(slot_of, dtype=np.int32)
        total, hidden = y.shape
        n, k = slot_of.shape
        out = np.empty((n, hidden), DT_NP[out_dtype])
        _check(self.lib.oracle_combine(n, k, hidden, DT[y_dtype], _p(y), _p(topk_w),
                                       _p(slot_of), total, DT[out_dtype], _p(out)), "combine")
        return out

    def combine_abs(self, y: np.ndarray, y_dtype: str, topk_w: np.ndarray,
                    slot_of: np.ndarray) -> np.ndarray:
        """sum_j |w[t,j] * Y[slot,c]| per output element (the tolerance scale)."""
        y = np.ascontiguousarray(y, dtype=DT_NP[y_dtype])
        topk_w = np.ascontiguousarray(topk_w, dtype=np.float32)
        slot_of = np.ascontiguousarray(slot_of, dtype=np.int32)
        total, hidden = y.shape
        n, k = slot_of.shape
        out = np.empty((n, hidden), np.float64)
        _check(self.lib.oracle_combine_abs(n, k, hidden, DT[y_dtype], _p(y), _p(topk_w),
                                           _p(slot_of), total, _p(out)), "combine_abs")
        return out

    def to_float(self, a: np.ndarray, dtype: str) -> np.ndarray:
        """Widen raw bits of an array to float64 with the oracle's own decoders."""
        if dtype == "f32":
            return a.astype(np.float64)
        if dtype == "bf16":
            return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        lut = np.array([self.e4m3_to_float(c) for c in range(256)], np.float64)
        return lut[a]

    # -------------------------------------------------------------- the path
    def run_path(self, cfg, inp: dict, with_recv: bool = True) -> dict:
        """route -> counts -> offsets -> slots -> dispatch -> expert -> combine.

        ``cfg`` is a workloads.Config (or anything with the same fields) and
        ``inp`` holds numpy arrays (bf16 as uint16 bits, FP8 as uint8 codes).
        Returns every intermediate the CUDA path exposes.
        """
        logits = np.ascontiguousarray(inp["logits"], np.float32)
        n = logits.shape[0]
        E, k, R = cfg.n_experts, cfg.top_k, cfg.n_ranks
        idx, w = self.route(logits, k)
        cnt = self.counts(idx, E)
        off = self.offsets(n, E, k, R, cnt)
        slot_of, src_of = self.slots(idx, off, E)
        total = int(off[E])
        res = {"topk_idx": idx, "topk_w": w, "counts": cnt, "expert_off": off,
               "slot_of": slot_of, "src_of": src_of, "total_slots": total,
               "region_rows": self.region_rows(n, E, k, R)}
        if not with_recv:
            return res
        x = inp["x"]
        filled = slot_of.reshape(-1)
        recv = self.scatter_rows(x, slot_of, total)
        res["recv"] = recv
        if inp.get("x_scale") is not None:
            res["recv_scale"] = self.scatter_rows(inp["x_scale"], slot_of, total)
        if cfg.inter > 0 and cfg.x_dtype == "fp8_e4m3":
            blk = cfg.scale_block
            h = self.fp8_gate_up_rows(filled, idx.reshape(-1), recv, res["recv_scale"],
                                      inp["w_gate_up"], inp["w_gate_up_scale"], blk)
            hq, hs = self.quant_rows(filled, h, blk)
            y = self.fp8_down_rows(filled, idx.reshape(-1), hq, hs, inp["w_down"],
                                   inp["w_down_scale"], blk)
            res["h"], res["hq"], res["h_scale"] = h, hq, hs
            y_dtype = "bf16"
        elif cfg.inter > 0:
            y = self.swiglu_rows(filled, idx.reshape(-1), recv, inp["w_gate_up"], inp["w_down"])
            y_dtype = "bf16"
        elif cfg.x_dtype == "fp8_e4m3":
            y = self.dequant_rows(filled, recv, res["recv_scale"], cfg.scale_block)
            y_dtype = "bf16"
        else:
            y, y_dtype = recv, cfg.x_dtype
        res["y"], res["y_dtype"] = y, y_dtype
        res["out"] = self.combine(y, y_dtype, w, slot_of, cfg.out_dtype)
        res["out_abs"] = self.combine_abs(y, y_dtype, w, slot_of)
        return res


_default: Oracle | None = None


def default() -> Oracle:
    """The oracle built from moe_oracle.c as committed."""
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default


def build_variant(src_text: str, out_path: str) -> str:
    """Compile a modified copy of the oracle source (used by mutation tests)."""
    src = out_path + ".c"
    with open(src, "w") as f:
        f.write(src_text)
    subprocess.check_call(["gcc", "-std=c11", "-O2", "-fno-fast-math", "-ffp-contract=off",
                           "-fPIC", "-shared", "-o", out_path, src, "-lm"])
    return out_path


def source_text() -> str:
    with open(_SRC) as f:
        return f.read()


def __getattr__(name):
    # module-level shortcuts: oracle.route(...) == oracle.default().route(...)
    if name.startswith("_"):
        raise AttributeError(name)
    return getattr(default(), name)


