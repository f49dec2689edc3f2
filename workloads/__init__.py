"""Seeded synthetic workloads for MoE token dispatch / combine.

This module only draws and lays out inputs; it holds none of the method's
arithmetic (no routing, no counting, no scatter, no combine).  Both the CPU
oracle (``oracle/``) and the CUDA path are fed from here, so the two sides see
byte-identical inputs.

Workload shapes follow the configurations quoted for the method: a tiny parity
case, a decode-shaped batch, a prefill-shaped batch with FP8 activations and
per-128-column scales, a Zipf-skewed batch, and a full MoE layer with SwiGLU
experts.  The draws are made with ``torch.Generator('cpu').manual_seed(seed)``
in the order logits, x, expert weights.

FP8 inputs: each 128-column block of a row gets ``scale = amax / 448`` (1 when
the block is all zero), the block is divided by its scale, clamped to the
e4m3 finite range and rounded to nearest-even by torch's float8_e4m3fn cast.
With FP8 rows the SwiGLU expert weights are FP8 as well, quantised the same
way per 128x128 tile.  That is input preparation: the method receives the FP8
codes and the scales.
"""
from __future__ import annotations

import dataclasses
import torch

__all__ = ["Config", "CONFIGS", "make_inputs", "as_numpy_bits", "DTYPE_BYTES",
           "quantise_fp8_tiles"]

# Element size in bytes of each activation encoding the library accepts.
DTYPE_BYTES = {"f32": 4, "bf16": 2, "fp8_e4m3": 1}
FP8_E4M3_MAX = 448.0


@dataclasses.dataclass(frozen=True)
class Config:
    name: str
    n: int                 # tokens N
    hidden: int            # D
    n_experts: int         # E
    top_k: int             # k
    n_ranks: int           # R virtual ranks (E % R == 0)
    x_dtype: str = "bf16"  # "f32" | "bf16" | "fp8_e4m3"
    y_dtype: str = "bf16"  # expert-output dtype read by combine
    out_dtype: str = "bf16"
    scale_block: int = 0   # 128 with FP8 activations, else 0
    inter: int = 0         # SwiGLU intermediate size; 0 = identity experts
    logits: str = "normal"  # "normal" | "zipf1.2"
    w_std: float = 0.02

    def replace(self, **kw) -> "Config":
        return dataclasses.replace(self, **kw)

    @property
    def scale_cols(self) -> int:
        return self.hidden // self.scale_block if self.scale_block else 0


CONFIGS = {
    # N=64, D=256, fp32, E=8, k=2, R=2, identity experts.
    "tiny": Config("tiny", 64, 256, 8, 2, 2, "f32", "f32", "f32"),
    # N=128, D=7168, bf16, E=256, k=8, R=8.
    "decode": Config("decode", 128, 7168, 256, 8, 8),
    # N=4096, D=7168, FP8 e4m3 + per-128-column fp32 scales, bf16 combine.
    "prefill": Config("prefill", 4096, 7168, 256, 8, 8, "fp8_e4m3", "bf16", "bf16",
                      scale_block=128),
    # N=16384, D=4096, bf16, E=128, k=4, R=4, Zipf(1.2)-skewed popularity.
    "skewed": Config("skewed", 16384, 4096, 128, 4, 4, logits="zipf1.2"),
    # N=1024, D=7168, bf16, E=64, k=8, SwiGLU experts with I=2048.
    "layer": Config("layer", 1024, 7168, 64, 8, 8, inter=2048),
    # The same layer with FP8 rows (per-128-column scales, as dispatched at
    # prefill) and FP8 expert weights (one scale per 128x128 tile).
    "layer_fp8": Config("layer_fp8", 1024, 7168, 64, 8, 8, "fp8_e4m3", "bf16", "bf16",
                        scale_block=128, inter=2048),
}


def _zipf_log_popularity(n_experts: int, s: float = 1.2) -> torch.Tensor:
    """log p_e with p_e proportional to (e+1)^-s, normalised to sum to 1."""
    e = torch.arange(1, n_experts + 1, dtype=torch.float64)
    p = e.pow(-s)
    p = p / p.sum()
    return p.log().to(torch.float32)


def _quantise_fp8_blocks(xf: torch.Tensor, block: int):
    """Per-(row, 128-column block) amax scaling to e4m3 codes (input prep)."""
    n, d = xf.shape
    xb = xf.view(n, d // block, block)
    amax = xb.abs().amax(dim=2)
    scale = torch.where(amax > 0, amax / FP8_E4M3_MAX, torch.ones_like(amax))
    q = (xb / scale.unsqueeze(2)).clamp(-FP8_E4M3_MAX, FP8_E4M3_MAX)
    q = q.to(torch.float8_e4m3fn).view(n, d).view(torch.uint8)
    return q.contiguous(), scale.to(torch.float32).contiguous()


def quantise_fp8_tiles(wf: torch.Tensor, block: int):
    """Per-(block x block tile) amax scaling of a weight matrix to e4m3 codes."""
    r, c = wf.shape
    wb = wf.view(r // block, block, c // block, block)
    amax = wb.abs().amax(dim=(1, 3))
    scale = torch.where(amax > 0, amax / FP8_E4M3_MAX, torch.ones_like(amax))
    q = (wb / scale[:, None, :, None]).clamp(-FP8_E4M3_MAX, FP8_E4M3_MAX)
    q = q.to(torch.float8_e4m3fn).view(r, c).view(torch.uint8)
    return q.contiguous(), scale.to(torch.float32).contiguous()


def make_inputs(cfg: Config, seed: int = 0, n: int | None = None,
                with_weights: bool | None = None) -> dict:
    """Draw one batch of inputs on the CPU.

    Returns a dict of CPU torch tensors:
      logits  [N, E] float32
      x       [N, D] float32 | bfloat16 | uint8 (e4m3 codes)
      x_scale [N, D/128] float32 or None
      w_gate_up [E, 2I, D] bfloat16 (gate rows first, then up rows) or None
      w_down    [E, D, I]  bfloat16 or None
    With FP8 rows the weights are e4m3 codes (uint8) instead, with
      w_gate_up_scale [E, 2I/128, D/128] and w_down_scale [E, D/128, I/128]
    float32, one scale per 128x128 tile.
    """
    n = cfg.n if n is None else n
    g = torch.Generator("cpu").manual_seed(seed)
    logits = torch.randn(n, cfg.n_experts, generator=g, dtype=torch.float32)
    if cfg.logits == "zipf1.2":
        logits = logits + _zipf_log_popularity(cfg.n_experts, 1.2)
    elif cfg.logits != "normal":
        raise ValueError(cfg.logits)
    xf = torch.randn(n, cfg.hidden, generator=g, dtype=torch.float32)
    x_scale = None
    if cfg.x_dtype == "f32":
        x = xf
    elif cfg.x_dtype == "bf16":
        x = xf.to(torch.bfloat16)
    elif cfg.x_dtype == "fp8_e4m3":
        x, x_scale = _quantise_fp8_blocks(xf, cfg.scale_block)
    else:
        raise ValueError(cfg.x_dtype)
    out = {"logits": logits.contiguous(), "x": x.contiguous(), "x_scale": x_scale,
           "w_gate_up": None, "w_down": None, "w_gate_up_scale": None, "w_down_scale": None}
    if with_weights is None:
        with_weights = cfg.inter > 0
    if with_weights and cfg.x_dtype == "fp8_e4m3":
        e, d, i, b = cfg.n_experts, cfg.hidden, cfg.inter, cfg.scale_block
        wgu = torch.empty(e, 2 * i, d, dtype=torch.uint8)
        wd = torch.empty(e, d, i, dtype=torch.uint8)
        sgu = torch.empty(e, 2 * i // b, d // b, dtype=torch.float32)
        sd = torch.empty(e, d // b, i // b, dtype=torch.float32)
        for ex in range(e):
            wgu[ex], sgu[ex] = quantise_fp8_tiles(torch.randn(2 * i, d, generator=g) * cfg.w_std, b)
        for ex in range(e):
            wd[ex], sd[ex] = quantise_fp8_tiles(torch.randn(d, i, generator=g) * cfg.w_std, b)
        out.update(w_gate_up=wgu, w_down=wd, w_gate_up_scale=sgu, w_down_scale=sd)
    elif with_weights:
        e, d, i = cfg.n_experts, cfg.hidden, cfg.inter
        wgu = torch.empty(e, 2 * i, d, dtype=torch.bfloat16)
        wd = torch.empty(e, d, i, dtype=torch.bfloat16)
        # Draw expert by expert so the fp32 staging stays small.
        for ex in range(e):
            wgu[ex] = (torch.randn(2 * i, d, generator=g) * cfg.w_std).to(torch.bfloat16)
        for ex in range(e):
            wd[ex] = (torch.randn(d, i, generator=g) * cfg.w_std).to(torch.bfloat16)
        out["w_gate_up"], out["w_down"] = wgu, wd
    return out


def as_numpy_bits(t: torch.Tensor | None):
    """Raw element bits as numpy (bf16 -> uint16, fp8 -> uint8, f32 stays f32)."""
    if t is None:
        return None
    if t.dtype == torch.bfloat16:
        return t.contiguous().view(torch.uint16).numpy()
    return t.contiguous().numpy()
