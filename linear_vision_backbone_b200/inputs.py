"""Seeded synthetic inputs for the Key-only GLA token mixer.

This module only draws random tensors and rounds them to their storage dtype.
It holds none of the operator's arithmetic: both the CUDA path and the fp64
oracle consume exactly the tensors produced here.  Random draws use a torch CPU
``Generator`` seeded as stated per workload; draws are fp32 and are rounded
(round-to-nearest-even) to the storage dtype afterwards.

Workloads are shaped like the GTR pages' own: image token grids at stride-16
patches (a 640x640 image gives a 40x40 grid, T = 1600; about 2048x2048 gives a
128x128 grid, T = 16384), width-384 activations, six heads of 64 dims, a
rank-16 gate projection with temperature 16 (GTR article, 方法详解 §1 and §4).
No image, dataset or trained weight is involved: activations are N(0, 1) and
projection weights are N(0, 1/fan_in), so q, k, v and the output-gate logits
come out roughly N(0, 1).

Recipes
-------
``proj``   : draw order x, W_q, W_k, W_v, W_g, W_down, W_up.  x ~ N(0,1) of
             width d_model; W_* ~ N(0, 1/fan_in); q, k, v, z = round(x_r @ W)
             with x_r = round(x); bias = 0.  The gate g is NOT produced here:
             it is the output of the gate projection under test.
``direct`` : draw order q, k, v, g, z.  q, k ~ N(0,1)*qk_std, v ~ N(0,1)*v_std,
             z ~ N(0,1), and the log-gate is drawn from the distribution
             logsigmoid(N(g_mu, 1)) / 16 per key dim (fp32).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional, Tuple

import torch

DTYPES = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    gh: int
    gw: int
    dk: int
    dv: int
    dtype: str
    dirs: Tuple[str, ...]
    seed: int
    recipe: str                  # "proj" or "direct"
    chunk: int = 64
    d_model: int = 384
    rank: int = 16
    tau: float = 16.0
    qk_std: float = 1.0
    v_std: float = 1.0
    g_mu: float = 0.0

    @property
    def T(self) -> int:
        return self.gh * self.gw

    @property
    def token_heads(self) -> int:
        return self.B * self.T * self.H

    def with_grid(self, gh: int, gw: Optional[int] = None, name: Optional[str] = None) -> "Workload":
        gw = gh if gw is None else gw
        return dataclasses.replace(self, gh=gh, gw=gw, name=name or f"{self.name}-{gh}x{gw}")


# The five workloads.  "640" and "640b8" share seed 1 (the batched case is
# generated "as the 640x640 case, from seed 1").
WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", B=1, H=1, gh=8, gw=8, dk=16, dv=16, dtype="f32", dirs=("LR",),
                     seed=0, recipe="direct", chunk=16, qk_std=1.0 / 4.0, v_std=1.0 / 4.0, g_mu=0.0),
    "640": Workload("640", B=1, H=6, gh=40, gw=40, dk=64, dv=64, dtype="f16",
                    dirs=("LR", "RL", "TB", "BT"), seed=1, recipe="proj"),
    "640b8": Workload("640b8", B=8, H=6, gh=40, gw=40, dk=64, dv=64, dtype="bf16",
                      dirs=("ROTATE",), seed=1, recipe="proj"),
    "16k": Workload("16k", B=1, H=6, gh=128, gw=128, dk=64, dv=64, dtype="f16",
                    dirs=("TB", "BT"), seed=2, recipe="proj"),
    "sweep": Workload("sweep", B=1, H=4, gh=16, gw=16, dk=128, dv=128, dtype="bf16", dirs=("LR",),
                      seed=3, recipe="direct", qk_std=1.0 / math.sqrt(128.0), v_std=1.0, g_mu=2.0),
}
SWEEP_GRIDS = (16, 32, 64, 128, 256)


def _randn(gen: torch.Generator, *shape) -> torch.Tensor:
    return torch.randn(*shape, generator=gen, dtype=torch.float32)


def make_inputs(wl: Workload) -> Dict[str, torch.Tensor]:
    """Draw the inputs of one workload (CPU tensors).

    Returns q, k, v, z (storage dtype, [B, T, H, d]), w (rms weight, fp32 [dv],
    all ones) and either
      * x [B, T, d_model] (storage dtype), w_down [d_model, rank], w_up
        [rank, H*dk], bias [H*dk] (fp32) for the ``proj`` recipe, or
      * g [B, T, H, dk] (fp32) for the ``direct`` recipe.
    """
    dt = DTYPES[wl.dtype]
    gen = torch.Generator(device="cpu")
    gen.manual_seed(wl.seed)
    B, T, H, dk, dv = wl.B, wl.T, wl.H, wl.dk, wl.dv
    out: Dict[str, torch.Tensor] = {}
    if wl.recipe == "proj":
        dm = wl.d_model
        x = _randn(gen, B, T, dm)
        wq = _randn(gen, dm, H * dk) / math.sqrt(dm)
        wk = _randn(gen, dm, H * dk) / math.sqrt(dm)
        wv = _randn(gen, dm, H * dv) / math.sqrt(dm)
        wg = _randn(gen, dm, H * dv) / math.sqrt(dm)
        wd = _randn(gen, dm, wl.rank) / math.sqrt(dm)
        wu = _randn(gen, wl.rank, H * dk) / math.sqrt(wl.rank)
        xr = x.to(dt)
        xf = xr.float()
        out["x"] = xr.contiguous()
        out["q"] = (xf @ wq).to(dt).reshape(B, T, H, dk).contiguous()
        out["k"] = (xf @ wk).to(dt).reshape(B, T, H, dk).contiguous()
        out["v"] = (xf @ wv).to(dt).reshape(B, T, H, dv).contiguous()
        out["z"] = (xf @ wg).to(dt).reshape(B, T, H, dv).contiguous()
        out["w_down"] = wd.contiguous()
        out["w_up"] = wu.contiguous()
        out["bias"] = torch.zeros(H * dk, dtype=torch.float32)
    elif wl.recipe == "direct":
        q = _randn(gen, B, T, H, dk) * wl.qk_std
        k = _randn(gen, B, T, H, dk) * wl.qk_std
        v = _randn(gen, B, T, H, dv) * wl.v_std
        u = _randn(gen, B, T, H, dk) + wl.g_mu
        z = _randn(gen, B, T, H, dv)
        out["q"] = q.to(dt).contiguous()
        out["k"] = k.to(dt).contiguous()
        out["v"] = v.to(dt).contiguous()
        out["z"] = z.to(dt).contiguous()
        # the log-gate distribution of the direct recipe: logsigmoid(N(g_mu,1))/16
        out["g"] = (torch.nn.functional.logsigmoid(u) / 16.0).contiguous()
    else:
        raise ValueError(f"unknown recipe {wl.recipe!r}")
    out["w"] = torch.ones(dv, dtype=torch.float32)
    return out


def make_custom(B: int, H: int, gh: int, gw: int, dk: int, dv: int, dtype: str, seed: int,
                qk_std: float = 1.0, v_std: float = 1.0, g_mu: float = 0.0,
                g_scale: float = 1.0 / 16.0, w_random: bool = False) -> Dict[str, torch.Tensor]:
    """``direct``-recipe inputs of any shape, for edge-case tests.

    The log-gate is logsigmoid(N(g_mu, 1)) * g_scale; a large g_scale or a very
    negative g_mu makes strong decays.  With ``w_random`` the RMSNorm weight is
    drawn from N(1, 0.25) instead of ones (draw order q, k, v, g, z, w).
    """
    dt = DTYPES[dtype]
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    T = gh * gw
    q = _randn(gen, B, T, H, dk) * qk_std
    k = _randn(gen, B, T, H, dk) * qk_std
    v = _randn(gen, B, T, H, dv) * v_std
    u = _randn(gen, B, T, H, dk) + g_mu
    z = _randn(gen, B, T, H, dv)
    w = (1.0 + 0.25 * _randn(gen, dv)) if w_random else torch.ones(dv)
    return {
        "q": q.to(dt).contiguous(), "k": k.to(dt).contiguous(), "v": v.to(dt).contiguous(),
        "z": z.to(dt).contiguous(),
        "g": (torch.nn.functional.logsigmoid(u) * g_scale).contiguous(),
        "w": w.float().contiguous(),
    }


def make_stack(nblocks: int, B: int, gh: int, gw: int, *, d_model: int = 384, H: int = 6, dk: int = 64,
               dv: int = 64, hidden: int = 1024, rank: int = 16, dtype: str = "f16", seed: int = 0,
               random_norms: bool = False, bias_std: float = 0.0):
    """Random-init input and weights of a stack of GTR blocks (the block's
    shapes: the token mixer's projections, the rank-``rank`` gate, the
    S-SwiGLU expansion to 2 * ``hidden`` channels, its 3x3 depthwise taps and
    its projection back to ``d_model``).

    Draw order: x [B, gh*gw, d_model] ~ N(0, 1) (fp32, the residual stream),
    then per block norm_mixer, w_in, w_down, w_up, gate_bias, gla_norm, w_o,
    norm_ffn, w_e, conv_w, conv_b, w_p.  Projection weights ~ N(0, 1/fan_in),
    rounded to ``dtype`` (w_down and w_up stay fp32, as the gate takes them);
    taps ~ N(0, 1)/3 and conv_b ~ N(0, 1)*0.1 (fp32); normalisation weights are
    ones, or N(1, 0.1^2) with ``random_norms``; gate_bias ~ N(0, 1)*bias_std
    (None when bias_std is 0).  Returns (x, [block dict, ...]).
    """
    dt = DTYPES[dtype]
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    T = gh * gw
    x = _randn(gen, B, T, d_model).contiguous()

    def norm(n):
        w = 1.0 + 0.1 * _randn(gen, n)
        return (w if random_norms else torch.ones(n)).float().contiguous()

    def proj(fan_in, n):
        return (_randn(gen, fan_in, n) / math.sqrt(fan_in)).to(dt).contiguous()

    blocks = []
    for _ in range(nblocks):
        p = {"norm_mixer": norm(d_model),
             "w_in": proj(d_model, 2 * H * dk + 2 * H * dv),
             "w_down": (_randn(gen, d_model, rank) / math.sqrt(d_model)).float().contiguous(),
             "w_up": (_randn(gen, rank, H * dk) / math.sqrt(rank)).float().contiguous()}
        b = _randn(gen, H * dk) * bias_std
        p["gate_bias"] = b.float().contiguous() if bias_std else None
        p["gla_norm"] = norm(dv)
        p["w_o"] = proj(H * dv, d_model)
        p["norm_ffn"] = norm(d_model)
        p["w_e"] = proj(d_model, 2 * hidden)
        p["conv_w"] = (_randn(gen, 3, 3, hidden) / 3.0).float().contiguous()
        p["conv_b"] = (_randn(gen, hidden) * 0.1).float().contiguous()
        p["w_p"] = proj(hidden, d_model)
        blocks.append(p)
    return x, blocks
