"""The C-ABI library without a GPU: it loads, exports every symbol that
include/moeroute.h declares, and its host-side validation behaves as the
header states.  No call here reaches a CUDA launch."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moeroute.h")


def build_library():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_moeroute_build", os.path.join(ROOT, "combine_moe_route_11_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.build()


@pytest.fixture(scope="module")
def mr():
    build_library()
    import combine_moe_route_11_b200 as m
    return m


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_0-9]+)\s*\(", src)))


def test_header_declares_the_path():
    names = declared_functions()
    for must in ["moe_route_topk", "moe_dispatch", "moe_combine", "moe_layer",
                 "moe_expert_swiglu", "moe_expert_dequant", "moe_plan_create",
                 "moe_get_status", "moe_strerror"]:
        assert must in names


def test_library_exports_every_declared_symbol(mr):
    lib = ctypes.CDLL(mr.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def _plan_code(mr, **kw):
    base = dict(n_max=64, hidden=256, n_experts=8, top_k=2, n_ranks=2, x_dtype=0, y_dtype=0,
                out_dtype=0, scale_block=0, inter=0)
    base.update(kw)
    d = mr._Desc(*[base[f] for f, _ in mr._Desc._fields_])
    h = ctypes.c_void_p()
    rc = mr._lib.moe_plan_create(ctypes.byref(d), ctypes.byref(h))
    if rc == 0:
        mr._lib.moe_plan_destroy(h)
    return rc


@pytest.mark.parametrize("kw,code", [
    ({}, 0),
    ({"n_max": 0}, -1),
    ({"top_k": 9}, -1),                       # k > E
    ({"n_ranks": 3}, -1),                     # E % R != 0
    ({"hidden": 250}, -1),                    # fp32 row of 1000 bytes, not 16-byte whole
    ({"x_dtype": 1, "y_dtype": 1, "out_dtype": 1, "hidden": 8}, 0),
    ({"x_dtype": 2, "hidden": 16, "scale_block": 16, "y_dtype": 1, "out_dtype": 1}, 0),
    ({"x_dtype": 2, "hidden": 256, "scale_block": 12, "y_dtype": 1, "out_dtype": 1}, -1),
    ({"scale_block": 128}, -1),               # scales only with FP8 rows
    ({"n_experts": 1024, "top_k": 2, "n_ranks": 1}, -2),
    ({"top_k": 33, "n_experts": 64}, -2),
    ({"y_dtype": 2}, -2),
    ({"inter": 128}, -2),                     # SwiGLU needs bf16 rows
    ({"inter": 128, "x_dtype": 1, "y_dtype": 1, "out_dtype": 1}, 0),
    ({"inter": 100, "x_dtype": 1, "y_dtype": 1, "out_dtype": 1}, -2),
    # FP8 experts: FP8 rows with 128-column scales and bf16 Y
    ({"inter": 128, "x_dtype": 2, "scale_block": 128, "y_dtype": 1, "out_dtype": 1}, 0),
    ({"inter": 128, "x_dtype": 2, "scale_block": 64, "y_dtype": 1, "out_dtype": 1}, -2),
    ({"inter": 128, "x_dtype": 2, "scale_block": 128, "y_dtype": 0, "out_dtype": 1}, -2),
    ({"n_max": 1 << 27, "n_experts": 256, "top_k": 8, "n_ranks": 8}, -2),  # T >= 2^31
])
def test_plan_validation(mr, kw, code):
    assert _plan_code(mr, **kw) == code


def test_capacity_and_workspace(mr):
    import oracle
    for (n_max, e, k, r) in [(64, 8, 2, 2), (4096, 256, 8, 8), (100, 8, 4, 4), (77, 12, 3, 3)]:
        p = mr.Plan(n_max, 256, e, k, r, "f32", "f32", "f32")
        for n in (0, 1, n_max // 2, n_max):
            assert p.region_rows(n) == oracle.region_rows(n, e, k, r)
            assert p.recv_rows(n) == r * oracle.region_rows(n, e, k, r)
        assert p.region_rows(n_max + 1) == -1
        assert p.workspace_bytes > 0 and p.workspace_bytes % 256 == 0
        assert p.layer_workspace_bytes > p.workspace_bytes
        p.close()


def test_host_argument_errors_return_before_any_launch(mr):
    p = mr.Plan(64, 256, 8, 2, 2, "f32", "f32", "f32")
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: every call below fails validation
    lib = mr._lib
    assert lib.moe_route_topk(p.handle, 65, fake, fake, fake, fake, fake, fake, None) == -1
    assert lib.moe_route_topk(p.handle, -1, fake, fake, fake, fake, fake, fake, None) == -1
    assert lib.moe_route_topk(p.handle, 4, fake, fake, fake, fake, fake,
                              ctypes.c_void_p((1 << 20) + 16), None) == -4  # ws misaligned
    assert lib.moe_route_topk(p.handle, 4, fake, fake, fake, None, fake, fake, None) == -1
    assert lib.moe_dispatch(p.handle, 4, ctypes.c_void_p((1 << 20) + 8), None, fake, fake, None,
                            fake, fake, fake, None) == -1          # x not 16-byte aligned
    assert lib.moe_dispatch(p.handle, 0, None, None, None, None, None, None, None, fake,
                            None) == 0                               # n = 0 is a no-op
    # moe_route_dispatch validates both halves before it launches anything
    rd = lib.moe_route_dispatch
    assert rd(p.handle, 65, fake, fake, None, fake, fake, fake, fake, fake, None, fake, fake,
              fake, None) == -1                                      # n > n_max
    assert rd(p.handle, 4, fake, fake, None, fake, fake, fake, fake, fake, None, fake, fake,
              ctypes.c_void_p((1 << 20) + 16), None) == -4          # ws misaligned
    assert rd(p.handle, 4, fake, fake, None, fake, fake, None, fake, fake, None, fake, fake,
              fake, None) == -1                                      # no counts
    assert rd(p.handle, 4, fake, ctypes.c_void_p((1 << 20) + 8), None, fake, fake, fake, fake,
              fake, None, fake, fake, fake, None) == -1              # x not 16-byte aligned
    assert rd(p.handle, 4, fake, fake, None, fake, fake, fake, fake, None, None, fake, fake,
              fake, None) == -1                                      # no recv
    assert lib.moe_combine(p.handle, 65, fake, fake, fake, fake, fake, None) == -1
    assert lib.moe_expert_dequant(p.handle, 4, fake, fake, fake, fake, fake, None) == -2
    assert lib.moe_expert_swiglu(p.handle, 4, fake, fake, fake, fake, fake, fake, fake, fake,
                                 None) == -2
    assert lib.moe_layer_buffer(p.handle, fake, b"nope") is None
    assert lib.moe_layer_buffer(p.handle, fake, b"recv") is not None
    assert lib.moe_get_status(None, fake, None) == -1
    for code in range(-7, 1):
        assert mr.moe_strerror(code) not in ("", "unknown status")
    p.close()


def test_layer_rejects_bad_arguments_before_its_first_stage(mr):
    """moe_layer checks every argument that a later stage would reject before
    it enqueues route and dispatch.  Without a GPU any launch fails with
    MOE_ERR_CUDA (-3), so the host-side codes below show that no stage ran."""
    fake = ctypes.c_void_p(1 << 20)
    odd = ctypes.c_void_p((1 << 20) + 8)
    lib = mr._lib
    # FP8 rows with identity experts dequantise to bf16: an fp32 Y is unsupported
    p = mr.Plan(64, 256, 8, 2, 2, "fp8_e4m3", "f32", "f32", scale_block=128)
    assert lib.moe_layer(p.handle, 4, fake, fake, fake, None, None, fake, fake, None) == -2
    p.close()
    p = mr.Plan(64, 256, 8, 2, 2, "fp8_e4m3", "bf16", "bf16", scale_block=128)
    assert lib.moe_layer(p.handle, 4, fake, fake, None, None, None, fake, fake, None) == -1
    assert lib.moe_layer(p.handle, 4, fake, fake, fake, None, None, None, fake, None) == -1
    assert lib.moe_layer(p.handle, 4, fake, fake, fake, None, None, odd, fake, None) == -1
    assert lib.moe_layer(p.handle, 4, odd, fake, fake, None, None, fake, fake, None) == -1
    p.close()
    p = mr.Plan(64, 256, 8, 2, 2, "bf16", "bf16", "bf16", inter=128)
    assert lib.moe_layer(p.handle, 4, fake, fake, None, None, fake, fake, fake, None) == -1
    assert lib.moe_layer(p.handle, 4, fake, fake, None, fake, odd, fake, fake, None) == -1
    p.close()


def test_fp8_expert_entry_points_validate_on_the_host(mr):
    fake = ctypes.c_void_p(1 << 20)
    odd = ctypes.c_void_p((1 << 20) + 8)
    lib = mr._lib
    sw8 = lib.moe_expert_swiglu_fp8
    p = mr.Plan(64, 256, 8, 2, 2, "fp8_e4m3", "bf16", "bf16", scale_block=128, inter=128)
    args = [fake] * 13 + [fake, None]          # recv .. y, ws, stream
    assert sw8(p.handle, 4, *args) != -2       # the plan is accepted (the launch then fails)
    bad = list(args); bad[1] = None            # no recv_scale
    assert sw8(p.handle, 4, *bad) == -1
    bad = list(args); bad[10] = odd            # hq misaligned
    assert sw8(p.handle, 4, *bad) == -1
    assert sw8(p.handle, 65, *args) == -1      # n > n_max
    assert sw8(p.handle, 0, *args) == 0        # n = 0 is a no-op
    # the bf16 expert call and moe_layer refuse FP8 experts; moe_layer_fp8 needs the scales
    assert lib.moe_expert_swiglu(p.handle, 4, *([fake] * 8), None) == -2
    assert lib.moe_layer(p.handle, 4, fake, fake, fake, fake, fake, fake, fake, None) == -2
    assert lib.moe_layer_fp8(p.handle, 4, fake, fake, fake, fake, None, fake, fake, fake, fake,
                             None) == -1
    assert lib.moe_layer_buffer(p.handle, fake, b"hq") is not None
    assert lib.moe_layer_buffer(p.handle, fake, b"h_scale") is not None
    p.close()
    p = mr.Plan(64, 256, 8, 2, 2, "bf16", "bf16", "bf16", inter=128)
    assert sw8(p.handle, 4, *args) == -2       # bf16 experts
    assert lib.moe_layer_fp8(p.handle, 4, *([fake] * 9), None) == -2
    p.close()


def test_binding_checks_the_workspace_size(mr):
    """The C entry points take no workspace size, so the binding checks it."""
    import torch
    p = mr.Plan(64, 256, 8, 2, 2, "f32", "f32", "f32")
    small = torch.zeros(p.workspace_bytes - 256, dtype=torch.uint8)
    with pytest.raises(ValueError):
        mr.moe_get_status(p, small)
    with pytest.raises(ValueError):
        mr.moe_workspace_init(p, torch.zeros(p.workspace_bytes // 4, dtype=torch.int32))
    with pytest.raises(ValueError):
        mr._ws(p, torch.zeros(p.workspace_bytes, dtype=torch.uint8), layer=True)
    p.close()


def test_binding_checks_slot_indexed_buffers(mr):
    """Buffers indexed by slot must hold T rows of the plan's width and dtype:
    the binding rejects shorter or mistyped tensors before any pointer reaches
    the library.  The tensors here are on the CPU, so a call that passes every
    check stops at the binding's CUDA-tensor check instead."""
    import torch
    n = 16
    p = mr.Plan(64, 256, 8, 2, 2, "bf16", "bf16", "bf16")
    T = p.recv_rows(n)
    ws = torch.zeros(p.workspace_bytes, dtype=torch.uint8)
    w = torch.zeros(n, 2)
    so = torch.zeros(n, 2, dtype=torch.int32)
    out = torch.zeros(n, 256, dtype=torch.bfloat16)
    bf = lambda r, c=256: torch.zeros(r, c, dtype=torch.bfloat16)  # noqa: E731
    with pytest.raises(ValueError, match="need at least"):
        mr.moe_combine(p, bf(T - 1), w, so, out, ws)
    with pytest.raises(TypeError, match="y: dtype"):
        mr.moe_combine(p, torch.zeros(T, 256), w, so, out, ws)
    with pytest.raises(ValueError, match="CUDA tensor"):
        mr.moe_combine(p, bf(T), w, so, out, ws)
    x = bf(n)
    idx = torch.zeros(n, 2, dtype=torch.int32)
    src = torch.zeros(T, dtype=torch.int32)
    with pytest.raises(ValueError, match="recv: shape"):
        mr.moe_dispatch(p, x, None, idx, bf(T, 128), None, so, src, ws)
    with pytest.raises(TypeError, match="recv: dtype"):
        mr.moe_dispatch(p, x, None, idx, torch.zeros(T, 256, dtype=torch.uint8), None, so, src, ws)
    with pytest.raises(ValueError, match="src_of"):
        mr.moe_dispatch(p, x, None, idx, bf(T), None, so, src[:-1], ws)
    with pytest.raises(ValueError, match="CUDA tensor"):
        mr.moe_dispatch(p, x, None, idx, bf(T), None, so, src, ws)
    p.close()

    p = mr.Plan(64, 256, 8, 2, 2, "fp8_e4m3", "bf16", "bf16", scale_block=128)
    T = p.recv_rows(n)
    ws = torch.zeros(p.layer_workspace_bytes, dtype=torch.uint8)
    q = lambda r: torch.zeros(r, 256, dtype=torch.uint8)  # noqa: E731
    xs = torch.ones(n, 2)
    with pytest.raises(ValueError, match="recv_scale"):
        mr.moe_dispatch(p, q(n), xs, idx, q(T), torch.ones(T - 1, 2), so, src, ws)
    with pytest.raises(ValueError, match="x_scale: required"):
        mr.moe_dispatch(p, q(n), None, idx, q(T), torch.ones(T, 2), so, src, ws)
    with pytest.raises(TypeError, match="y: dtype"):
        mr.moe_expert_dequant(p, n, q(T), torch.ones(T, 2), so, torch.zeros(T, 256), ws)
    with pytest.raises(ValueError, match="y: shape"):
        mr.moe_expert_dequant(p, n, q(T), torch.ones(T, 2), so, bf(T // 2), ws)
    with pytest.raises(ValueError, match="x_scale: required"):
        mr.moe_layer(p, torch.zeros(n, 8), q(n), None, None, None, out, ws)
    p.close()

    p = mr.Plan(64, 256, 8, 2, 2, "bf16", "bf16", "bf16", inter=128)
    T = p.recv_rows(n)
    ws = torch.zeros(p.workspace_bytes, dtype=torch.uint8)
    counts = torch.zeros(8, dtype=torch.int32)
    off = torch.zeros(9, dtype=torch.int32)
    wgu = torch.zeros(8, 256, 256, dtype=torch.bfloat16)
    wd = torch.zeros(8, 256, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="h: shape"):
        mr.moe_expert_swiglu(p, n, bf(T), counts, off, wgu, wd, bf(T, 64), bf(T), ws)
    with pytest.raises(ValueError, match="w_down: shape"):
        mr.moe_expert_swiglu(p, n, bf(T), counts, off, wgu, wd[:, :, :64], bf(T, 128), bf(T), ws)
    with pytest.raises(ValueError, match="CUDA tensor"):
        mr.moe_expert_swiglu(p, n, bf(T), counts, off, wgu, wd, bf(T, 128), bf(T), ws)
    with pytest.raises(ValueError, match="w_gate_up: required"):
        mr.moe_layer(p, torch.zeros(n, 8), bf(n), None, None, wd, out,
                     torch.zeros(p.layer_workspace_bytes, dtype=torch.uint8))
    p.close()


def test_binding_checks_fp8_expert_buffers(mr):
    """moe_expert_swiglu_fp8 / moe_layer_fp8 reject mistyped or short weights,
    scales and intermediates before any pointer reaches the library."""
    import torch
    n, E, D, I = 16, 8, 256, 128
    p = mr.Plan(64, D, E, 2, 2, "fp8_e4m3", "bf16", "bf16", scale_block=128, inter=I)
    assert p.fp8_experts
    T = p.recv_rows(n)
    ws = torch.zeros(p.workspace_bytes, dtype=torch.uint8)
    u8 = lambda *s: torch.zeros(*s, dtype=torch.uint8)  # noqa: E731
    f32 = lambda *s: torch.zeros(*s, dtype=torch.float32)  # noqa: E731
    bf = lambda *s: torch.zeros(*s, dtype=torch.bfloat16)  # noqa: E731
    i32 = lambda *s: torch.zeros(*s, dtype=torch.int32)  # noqa: E731
    args = dict(recv=u8(T, D), recv_scale=f32(T, D // 128), counts=i32(E), expert_off=i32(E + 1),
                slot_of=i32(n, 2), w_gate_up=u8(E, 2 * I, D), w_gate_up_scale=f32(E, 2 * I // 128, D // 128),
                w_down=u8(E, D, I), w_down_scale=f32(E, D // 128, I // 128), h=bf(T, I), hq=u8(T, I),
                h_scale=f32(T, I // 128), y=bf(T, D))

    def call(**over):
        a = dict(args, **over)
        mr.moe_expert_swiglu_fp8(p, n, a["recv"], a["recv_scale"], a["counts"], a["expert_off"],
                                 a["slot_of"], a["w_gate_up"], a["w_gate_up_scale"], a["w_down"],
                                 a["w_down_scale"], a["h"], a["hq"], a["h_scale"], a["y"], ws)

    with pytest.raises(ValueError, match="CUDA tensor"):
        call()                                               # every check passes
    with pytest.raises(TypeError, match="w_gate_up: dtype"):
        call(w_gate_up=bf(E, 2 * I, D))
    with pytest.raises(ValueError, match="w_down_scale: shape"):
        call(w_down_scale=f32(E, D // 128, I // 64))
    with pytest.raises(ValueError, match="hq: shape"):
        call(hq=u8(T - 1, I))
    with pytest.raises(ValueError, match="h_scale: shape"):
        call(h_scale=f32(T, I // 64))
    with pytest.raises(ValueError, match="recv_scale: shape"):
        call(recv_scale=f32(T, 1))
    with pytest.raises(ValueError, match="w_gate_up_scale: required"):
        call(w_gate_up_scale=None)
    lws = torch.zeros(p.layer_workspace_bytes, dtype=torch.uint8)
    with pytest.raises(ValueError, match="w_down: shape"):
        mr.moe_layer_fp8(p, f32(n, E), u8(n, D), f32(n, D // 128), args["w_gate_up"],
                         args["w_gate_up_scale"], u8(E, D, I // 2), args["w_down_scale"],
                         bf(n, D), lws)
    buf = p.new_buffers(0, device="cpu")
    assert set(("hq", "h_scale", "h", "y")) <= set(buf)
    p.close()
