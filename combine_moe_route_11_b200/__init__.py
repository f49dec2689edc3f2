"""Python binding of libmoeroute (MoE token dispatch / combine on B200).

Argument marshalling only: every step of the path runs in the CUDA kernels
of ``libmoeroute.so``; PyTorch supplies device memory and streams.  The
functions carry the names of the C entry points in ``include/moeroute.h``
and take torch tensors; ``n`` comes from the leading dimension of the token
arrays.  Importing this package fails loudly when the library is not built.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "MoeError", "Plan", "LIB_PATH", "moe_route_topk", "moe_router_topk", "moe_dispatch",
    "moe_route_dispatch",
    "moe_expert_dequant", "moe_expert_swiglu", "moe_expert_swiglu_fp8", "moe_combine",
    "moe_layer", "moe_layer_fp8", "moe_layer_buffer",
    "moe_get_status", "moe_workspace_init", "moe_strerror", "DTYPE_CODES", "ELEM_BYTES",
    "FUSED_MAX_TOKENS",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoeroute.so")
if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python combine_moe_route_11_b200/build.py` "
        "(nvcc, sm_100a). There is no fallback implementation.")
_lib = ctypes.CDLL(LIB_PATH)

DTYPE_CODES = {"f32": 0, "bf16": 1, "fp8_e4m3": 2}
# Largest batch that moe_route_dispatch runs as one launch (32 route blocks
# of 32 tokens); larger batches run the route and dispatch kernels.
FUSED_MAX_TOKENS = 1024
ELEM_BYTES = {"f32": 4, "bf16": 2, "fp8_e4m3": 1}
_TORCH = {"f32": (torch.float32,), "bf16": (torch.bfloat16,),
          "fp8_e4m3": (torch.uint8, torch.float8_e4m3fn)}


class _Desc(ctypes.Structure):
    _fields_ = [(name, ctypes.c_int32) for name in (
        "n_max", "hidden", "n_experts", "top_k", "n_ranks", "x_dtype", "y_dtype", "out_dtype",
        "scale_block", "inter")]


_P = ctypes.c_void_p
_i32 = ctypes.c_int32
_SIGS = {
    "moe_plan_create": (ctypes.c_int, [ctypes.POINTER(_Desc), ctypes.POINTER(_P)]),
    "moe_plan_destroy": (None, [_P]),
    "moe_workspace_bytes": (ctypes.c_size_t, [_P]),
    "moe_layer_workspace_bytes": (ctypes.c_size_t, [_P]),
    "moe_region_rows": (ctypes.c_int64, [_P, _i32]),
    "moe_recv_rows": (ctypes.c_int64, [_P, _i32]),
    "moe_route_topk": (ctypes.c_int, [_P, _i32, _P, _P, _P, _P, _P, _P, _P]),
    "moe_router_topk": (ctypes.c_int, [_P, _i32, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_dispatch": (ctypes.c_int, [_P, _i32, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_route_dispatch": (ctypes.c_int, [_P, _i32] + [_P] * 13),
    "moe_expert_dequant": (ctypes.c_int, [_P, _i32, _P, _P, _P, _P, _P, _P]),
    "moe_expert_swiglu": (ctypes.c_int, [_P, _i32, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_expert_swiglu_fp8": (ctypes.c_int, [_P, _i32] + [_P] * 15),
    "moe_combine": (ctypes.c_int, [_P, _i32, _P, _P, _P, _P, _P, _P]),
    "moe_layer": (ctypes.c_int, [_P, _i32, _P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_layer_fp8": (ctypes.c_int, [_P, _i32] + [_P] * 10),
    "moe_layer_buffer": (_P, [_P, _P, ctypes.c_char_p]),
    "moe_get_status": (ctypes.c_int, [_P, _P, _P]),
    "moe_workspace_init": (ctypes.c_int, [_P, _P, _P]),
    "moe_strerror": (ctypes.c_char_p, [ctypes.c_int]),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.restype, _f.argtypes = _res, _args


class MoeError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {moe_strerror(code)} ({code})")
        self.code = code


def moe_strerror(code: int) -> str:
    return _lib.moe_strerror(int(code)).decode()


def _check(code: int, what: str):
    if code != 0:
        raise MoeError(code, what)


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _ws(plan: "Plan", ws: torch.Tensor, layer: bool = False):
    """The workspace pointer, after checking the tensor is large enough (the
    C entry points take no size for it)."""
    need = plan.layer_workspace_bytes if layer else plan.workspace_bytes
    if ws.dtype != torch.uint8 or ws.dim() != 1 or ws.numel() < need:
        raise ValueError(f"ws: need a 1-D uint8 tensor of at least {need} bytes, got "
                         f"{ws.dtype} {tuple(ws.shape)}")
    return _ptr(ws)


def _expect(t: torch.Tensor, dtypes, shape, name: str):
    if t is None:
        raise ValueError(f"{name}: required")
    if t.dtype not in dtypes:
        raise TypeError(f"{name}: dtype {t.dtype}, expected one of {dtypes}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")


def _expect_rows(t: torch.Tensor, dtypes, rows: int, width: int, name: str):
    """A [>= rows, width] buffer indexed by slot: the kernels reach any row
    below T, so a shorter tensor would be written or read out of bounds."""
    if t is None:
        raise ValueError(f"{name}: required")
    if t.dtype not in dtypes:
        raise TypeError(f"{name}: dtype {t.dtype}, expected one of {dtypes}")
    if t.dim() != 2 or t.shape[0] < rows or t.shape[1] != width:
        raise ValueError(f"{name}: shape {tuple(t.shape)}, need at least ({rows}, {width})")


def _expect_scales(plan: "Plan", t, rows: int, name: str, exact: bool = False):
    """fp32 per-block scales of FP8 rows; ignored (may be None) without them."""
    if not plan.scale_cols:
        return
    if exact:
        _expect(t, (torch.float32,), (rows, plan.scale_cols), name)
    else:
        _expect_rows(t, (torch.float32,), rows, plan.scale_cols, name)


class Plan:
    """A validated MoE configuration (wraps moe_plan_create)."""

    def __init__(self, n_max: int, hidden: int, n_experts: int, top_k: int, n_ranks: int,
                 x_dtype: str = "bf16", y_dtype: str = "bf16", out_dtype: str = "bf16",
                 scale_block: int = 0, inter: int = 0):
        self.n_max, self.hidden, self.n_experts = n_max, hidden, n_experts
        self.top_k, self.n_ranks, self.inter = top_k, n_ranks, inter
        self.x_dtype, self.y_dtype, self.out_dtype = x_dtype, y_dtype, out_dtype
        self.scale_block = scale_block
        self.scale_cols = hidden // scale_block if scale_block else 0
        d = _Desc(n_max, hidden, n_experts, top_k, n_ranks, DTYPE_CODES[x_dtype],
                  DTYPE_CODES[y_dtype], DTYPE_CODES[out_dtype], scale_block, inter)
        h = _P()
        _check(_lib.moe_plan_create(ctypes.byref(d), ctypes.byref(h)), "moe_plan_create")
        self._h = h
        # constant for the plan's lifetime: asked once, not on every call
        self._ws_bytes = int(_lib.moe_workspace_bytes(h))
        self._layer_ws_bytes = int(_lib.moe_layer_workspace_bytes(h))
        self._recv_rows = {}

    @classmethod
    def from_config(cls, cfg, n_max: int | None = None) -> "Plan":
        return cls(n_max or cfg.n, cfg.hidden, cfg.n_experts, cfg.top_k, cfg.n_ranks,
                   cfg.x_dtype, cfg.y_dtype, cfg.out_dtype, cfg.scale_block, cfg.inter)

    @property
    def handle(self):
        return self._h

    def close(self):
        if getattr(self, "_h", None) is not None and self._h.value:
            _lib.moe_plan_destroy(self._h)
            self._h = _P()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @property
    def workspace_bytes(self) -> int:
        return self._ws_bytes

    @property
    def layer_workspace_bytes(self) -> int:
        return self._layer_ws_bytes

    def region_rows(self, n: int) -> int:
        return int(_lib.moe_region_rows(self._h, n))

    def recv_rows(self, n: int) -> int:
        rows = self._recv_rows.get(n)
        if rows is None:
            rows = self._recv_rows[n] = int(_lib.moe_recv_rows(self._h, n))
        return rows

    def new_workspace(self, device="cuda", layer: bool = False) -> torch.Tensor:
        nbytes = self.layer_workspace_bytes if layer else self.workspace_bytes
        return torch.zeros(nbytes, dtype=torch.uint8, device=device)

    def new_buffers(self, n: int, device="cuda") -> dict:
        """Output tensors of route/dispatch/combine for a call with n tokens."""
        T, k, E, D = self.recv_rows(n), self.top_k, self.n_experts, self.hidden
        xt = _TORCH[self.x_dtype][0]
        b = {
            "topk_idx": torch.empty(n, k, dtype=torch.int32, device=device),
            "topk_w": torch.empty(n, k, dtype=torch.float32, device=device),
            "counts": torch.empty(E, dtype=torch.int32, device=device),
            "expert_off": torch.empty(E + 1, dtype=torch.int32, device=device),
            "slot_of": torch.empty(n, k, dtype=torch.int32, device=device),
            "src_of": torch.empty(T, dtype=torch.int32, device=device),
            "recv": torch.empty(T, D, dtype=xt, device=device),
            "recv_scale": (torch.empty(T, self.scale_cols, dtype=torch.float32, device=device)
                           if self.scale_cols else None),
            "out": torch.empty(n, D, dtype=_TORCH[self.out_dtype][0], device=device),
        }
        if self.x_dtype == "fp8_e4m3" or self.inter > 0:
            b["y"] = torch.empty(T, D, dtype=_TORCH[self.y_dtype][0], device=device)
        if self.inter > 0:
            b["h"] = torch.empty(T, self.inter, dtype=torch.bfloat16, device=device)
        if self.fp8_experts:
            b["hq"] = torch.empty(T, self.inter, dtype=torch.uint8, device=device)
            b["h_scale"] = torch.empty(T, self.inter // 128, dtype=torch.float32, device=device)
        return b

    @property
    def fp8_experts(self) -> bool:
        """SwiGLU experts on FP8 rows run in FP8 (moe_expert_swiglu_fp8)."""
        return self.inter > 0 and self.x_dtype == "fp8_e4m3"


def moe_route_topk(plan: Plan, logits, topk_idx, topk_w, counts, expert_off, ws, stream=None):
    n = logits.shape[0]
    _expect(logits, (torch.float32,), (n, plan.n_experts), "logits")
    _expect(topk_idx, (torch.int32,), (n, plan.top_k), "topk_idx")
    _expect(topk_w, (torch.float32,), (n, plan.top_k), "topk_w")
    _expect(counts, (torch.int32,), (plan.n_experts,), "counts")
    _expect(expert_off, (torch.int32,), (plan.n_experts + 1,), "expert_off")
    _check(_lib.moe_route_topk(plan.handle, n, _ptr(logits), _ptr(topk_idx), _ptr(topk_w),
                               _ptr(counts), _ptr(expert_off), _ws(plan, ws), _stream(stream)),
           "moe_route_topk")


def moe_router_topk(plan: Plan, x, w_router, logits, topk_idx, topk_w, counts, expert_off, ws,
                    stream=None):
    """Router GEMM (logits = x w_router^T) with top-k and softmax fused, then
    counts and offsets; x is the bf16 [n, D] hidden rows, logits may be None."""
    n = x.shape[0]
    _expect(x, (torch.bfloat16,), (n, plan.hidden), "x")
    _expect(w_router, (torch.bfloat16,), (plan.n_experts, plan.hidden), "w_router")
    if logits is not None:
        _expect(logits, (torch.float32,), (n, plan.n_experts), "logits")
    _expect(topk_idx, (torch.int32,), (n, plan.top_k), "topk_idx")
    _expect(topk_w, (torch.float32,), (n, plan.top_k), "topk_w")
    _expect(counts, (torch.int32,), (plan.n_experts,), "counts")
    _expect(expert_off, (torch.int32,), (plan.n_experts + 1,), "expert_off")
    _check(_lib.moe_router_topk(plan.handle, n, _ptr(x), _ptr(w_router), _ptr(logits),
                                _ptr(topk_idx), _ptr(topk_w), _ptr(counts), _ptr(expert_off),
                                _ws(plan, ws), _stream(stream)), "moe_router_topk")


def _check_dispatch_outputs(plan: Plan, T: int, x_scale, n: int, recv, recv_scale, slot_of,
                            src_of):
    _expect_rows(recv, _TORCH[plan.x_dtype], T, plan.hidden, "recv")
    _expect(slot_of, (torch.int32,), (n, plan.top_k), "slot_of")
    if src_of is None or src_of.dtype != torch.int32 or src_of.dim() != 1 or src_of.shape[0] < T:
        raise ValueError(f"src_of: need a 1-D int32 tensor of at least {T} entries")
    _expect_scales(plan, x_scale, n, "x_scale", exact=True)
    _expect_scales(plan, recv_scale, T, "recv_scale")


def moe_dispatch(plan: Plan, x, x_scale, topk_idx, recv, recv_scale, slot_of, src_of, ws,
                 stream=None):
    n = x.shape[0]
    T = plan.recv_rows(n)
    _expect(x, _TORCH[plan.x_dtype], (n, plan.hidden), "x")
    _expect(topk_idx, (torch.int32,), (n, plan.top_k), "topk_idx")
    _check_dispatch_outputs(plan, T, x_scale, n, recv, recv_scale, slot_of, src_of)
    _check(_lib.moe_dispatch(plan.handle, n, _ptr(x), _ptr(x_scale), _ptr(topk_idx), _ptr(recv),
                             _ptr(recv_scale), _ptr(slot_of), _ptr(src_of), _ws(plan, ws),
                             _stream(stream)), "moe_dispatch")


def moe_route_dispatch(plan: Plan, logits, x, x_scale, topk_idx, topk_w, counts, expert_off,
                       recv, recv_scale, slot_of, src_of, ws, stream=None):
    """moe_route_topk followed by moe_dispatch; one launch for n <= 1024."""
    n = logits.shape[0]
    T = plan.recv_rows(n)
    _expect(logits, (torch.float32,), (n, plan.n_experts), "logits")
    _expect(x, _TORCH[plan.x_dtype], (n, plan.hidden), "x")
    _expect(topk_idx, (torch.int32,), (n, plan.top_k), "topk_idx")
    _expect(topk_w, (torch.float32,), (n, plan.top_k), "topk_w")
    _expect(counts, (torch.int32,), (plan.n_experts,), "counts")
    _expect(expert_off, (torch.int32,), (plan.n_experts + 1,), "expert_off")
    _check_dispatch_outputs(plan, T, x_scale, n, recv, recv_scale, slot_of, src_of)
    _check(_lib.moe_route_dispatch(plan.handle, n, _ptr(logits), _ptr(x), _ptr(x_scale),
                                   _ptr(topk_idx), _ptr(topk_w), _ptr(counts), _ptr(expert_off),
                                   _ptr(recv), _ptr(recv_scale), _ptr(slot_of), _ptr(src_of),
                                   _ws(plan, ws), _stream(stream)), "moe_route_dispatch")


def moe_expert_dequant(plan: Plan, n: int, recv, recv_scale, slot_of, y, ws, stream=None):
    T = plan.recv_rows(n)
    _expect(slot_of, (torch.int32,), (n, plan.top_k), "slot_of")
    _expect_rows(recv, _TORCH["fp8_e4m3"], T, plan.hidden, "recv")
    if recv_scale is not None:
        _expect_scales(plan, recv_scale, T, "recv_scale")
    _expect_rows(y, (torch.bfloat16,), T, plan.hidden, "y")
    _check(_lib.moe_expert_dequant(plan.handle, n, _ptr(recv), _ptr(recv_scale), _ptr(slot_of),
                                   _ptr(y), _ws(plan, ws), _stream(stream)), "moe_expert_dequant")


def moe_expert_swiglu(plan: Plan, n: int, recv, counts, expert_off, w_gate_up, w_down, h, y, ws,
                      stream=None):
    E, D, I = plan.n_experts, plan.hidden, plan.inter
    T = plan.recv_rows(n)
    _expect(w_gate_up, (torch.bfloat16,), (E, 2 * I, D), "w_gate_up")
    _expect(w_down, (torch.bfloat16,), (E, D, I), "w_down")
    _expect_rows(recv, (torch.bfloat16,), T, D, "recv")
    _expect(counts, (torch.int32,), (E,), "counts")
    _expect(expert_off, (torch.int32,), (E + 1,), "expert_off")
    _expect_rows(h, (torch.bfloat16,), T, I, "h")
    _expect_rows(y, (torch.bfloat16,), T, D, "y")
    _check(_lib.moe_expert_swiglu(plan.handle, n, _ptr(recv), _ptr(counts), _ptr(expert_off),
                                  _ptr(w_gate_up), _ptr(w_down), _ptr(h), _ptr(y), _ws(plan, ws),
                                  _stream(stream)), "moe_expert_swiglu")


def _expect_fp8_weights(plan: Plan, w_gate_up, w_gate_up_scale, w_down, w_down_scale):
    E, D, I = plan.n_experts, plan.hidden, plan.inter
    _expect(w_gate_up, _TORCH["fp8_e4m3"], (E, 2 * I, D), "w_gate_up")
    _expect(w_gate_up_scale, (torch.float32,), (E, 2 * I // 128, D // 128), "w_gate_up_scale")
    _expect(w_down, _TORCH["fp8_e4m3"], (E, D, I), "w_down")
    _expect(w_down_scale, (torch.float32,), (E, D // 128, I // 128), "w_down_scale")


def moe_expert_swiglu_fp8(plan: Plan, n: int, recv, recv_scale, counts, expert_off, slot_of,
                          w_gate_up, w_gate_up_scale, w_down, w_down_scale, h, hq, h_scale, y,
                          ws, stream=None):
    """FP8 SwiGLU experts on the FP8 receive buffer: GEMM1 -> H (bf16) ->
    per-128-column e4m3 Hq and scales -> GEMM2 -> Y (bf16)."""
    E, D, I = plan.n_experts, plan.hidden, plan.inter
    T = plan.recv_rows(n)
    _expect_fp8_weights(plan, w_gate_up, w_gate_up_scale, w_down, w_down_scale)
    _expect_rows(recv, _TORCH["fp8_e4m3"], T, D, "recv")
    _expect_rows(recv_scale, (torch.float32,), T, D // 128, "recv_scale")
    _expect(counts, (torch.int32,), (E,), "counts")
    _expect(expert_off, (torch.int32,), (E + 1,), "expert_off")
    _expect(slot_of, (torch.int32,), (n, plan.top_k), "slot_of")
    _expect_rows(h, (torch.bfloat16,), T, I, "h")
    _expect_rows(hq, _TORCH["fp8_e4m3"], T, I, "hq")
    _expect_rows(h_scale, (torch.float32,), T, I // 128, "h_scale")
    _expect_rows(y, (torch.bfloat16,), T, D, "y")
    _check(_lib.moe_expert_swiglu_fp8(plan.handle, n, _ptr(recv), _ptr(recv_scale), _ptr(counts),
                                      _ptr(expert_off), _ptr(slot_of), _ptr(w_gate_up),
                                      _ptr(w_gate_up_scale), _ptr(w_down), _ptr(w_down_scale),
                                      _ptr(h), _ptr(hq), _ptr(h_scale), _ptr(y), _ws(plan, ws),
                                      _stream(stream)), "moe_expert_swiglu_fp8")


def moe_combine(plan: Plan, y, topk_w, slot_of, out, ws, stream=None):
    n = out.shape[0]
    _expect(out, _TORCH[plan.out_dtype], (n, plan.hidden), "out")
    _expect(topk_w, (torch.float32,), (n, plan.top_k), "topk_w")
    _expect(slot_of, (torch.int32,), (n, plan.top_k), "slot_of")
    _expect_rows(y, _TORCH[plan.y_dtype], plan.recv_rows(n), plan.hidden, "y")
    _check(_lib.moe_combine(plan.handle, n, _ptr(y), _ptr(topk_w), _ptr(slot_of), _ptr(out),
                            _ws(plan, ws), _stream(stream)), "moe_combine")


def moe_layer(plan: Plan, logits, x, x_scale, w_gate_up, w_down, out, ws, stream=None):
    n = x.shape[0]
    _expect(logits, (torch.float32,), (n, plan.n_experts), "logits")
    _expect(x, _TORCH[plan.x_dtype], (n, plan.hidden), "x")
    _expect(out, _TORCH[plan.out_dtype], (n, plan.hidden), "out")
    _expect_scales(plan, x_scale, n, "x_scale", exact=True)
    if plan.inter > 0 and not plan.fp8_experts:
        E, D, I = plan.n_experts, plan.hidden, plan.inter
        _expect(w_gate_up, (torch.bfloat16,), (E, 2 * I, D), "w_gate_up")
        _expect(w_down, (torch.bfloat16,), (E, D, I), "w_down")
    _check(_lib.moe_layer(plan.handle, n, _ptr(logits), _ptr(x), _ptr(x_scale), _ptr(w_gate_up),
                          _ptr(w_down), _ptr(out), _ws(plan, ws, layer=True), _stream(stream)),
           "moe_layer")


def moe_layer_fp8(plan: Plan, logits, x, x_scale, w_gate_up, w_gate_up_scale, w_down,
                  w_down_scale, out, ws, stream=None):
    """moe_layer for plans with FP8 experts (FP8 rows and inter > 0)."""
    n = x.shape[0]
    _expect(logits, (torch.float32,), (n, plan.n_experts), "logits")
    _expect(x, _TORCH[plan.x_dtype], (n, plan.hidden), "x")
    _expect(out, _TORCH[plan.out_dtype], (n, plan.hidden), "out")
    _expect_scales(plan, x_scale, n, "x_scale", exact=True)
    if plan.fp8_experts:
        _expect_fp8_weights(plan, w_gate_up, w_gate_up_scale, w_down, w_down_scale)
    _check(_lib.moe_layer_fp8(plan.handle, n, _ptr(logits), _ptr(x), _ptr(x_scale),
                              _ptr(w_gate_up), _ptr(w_gate_up_scale), _ptr(w_down),
                              _ptr(w_down_scale), _ptr(out), _ws(plan, ws, layer=True),
                              _stream(stream)), "moe_layer_fp8")


def moe_layer_buffer(plan: Plan, ws, name: str, dtype, shape) -> torch.Tensor:
    """A view of one intermediate that moe_layer keeps in its workspace."""
    addr = _lib.moe_layer_buffer(plan.handle, _ws(plan, ws, layer=True), name.encode())
    if not addr:
        raise KeyError(name)
    off = addr - ws.data_ptr()
    count = 1
    for s in shape:
        count *= s
    nbytes = count * torch.empty((), dtype=dtype).element_size()
    if off < 0 or off + nbytes > ws.numel():
        raise ValueError(f"{name}: {nbytes} bytes at offset {off} exceed the workspace")
    return ws[off:off + nbytes].view(dtype).view(*shape)


def moe_get_status(plan: Plan, ws, stream=None) -> int:
    """Read and clear the device status word (synchronises the stream)."""
    return int(_lib.moe_get_status(plan.handle, _ws(plan, ws), _stream(stream)))


def moe_workspace_init(plan: Plan, ws, stream=None):
    _check(_lib.moe_workspace_init(plan.handle, _ws(plan, ws), _stream(stream)),
           "moe_workspace_init")
