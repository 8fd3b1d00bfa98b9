"""Seeded synthetic inputs for the Grok-1 MoE layer.

This module draws random tensors and nothing else: it holds none of the layer's
arithmetic, so both the CPU oracle (``oracle/``) and the CUDA path take their
inputs from here without sharing any computation.

Shapes and distributions (the five workloads the layer is measured and tested on):

* router weight ``router_w``  fp32 ``[d, E]``      ~ N(0, 1/d)
* expert weights ``wl, wv``   int8 ``[E, d, F]``   ~ uniform integers in {-127..127}
* expert weight  ``w1``       int8 ``[E, F, d]``   ~ uniform integers in {-127..127}
* scales ``sl, sv``           bf16 ``[E, F]``      = bf16(N(0,1) / (127*sqrt(d)))
* scale  ``s1``               bf16 ``[E, d]``      = bf16(N(0,1) / (127*sqrt(d)))
* tokens ``x``                bf16 ``[T, d]``      ~ N(0, 1)

One ``torch.Generator`` per workload, seeded, draws in the fixed order
router_w, wl, sl, wv, sv, w1, s1, x (then the stacked workload's per-block
tensors).  Tensors may be drawn on the GPU (fast, for the 4.8 GB layers) or on
the CPU; a parity test copies the very same tensors to both sides, so the
device only changes which random stream is used, never the comparison.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Dict, List, Optional

import torch

# Grok-1 MoE shape: emb 6144, 8 experts, 2 selected, ffn 32768.
GROK_D = 6144
GROK_F = 32768
GROK_E = 8
GROK_K = 2


@dataclass(frozen=True)
class Workload:
    """One named synthetic workload (sizes, seed and routing bias)."""

    name: str
    T: int
    d: int
    F: int
    E: int = GROK_E
    k: int = GROK_K
    seed: int = 0
    bias: Optional[List[float]] = None   # additive router-logit bias, fp32 [E]
    blocks: int = 0                      # >0: stacked pre/post-RMSNorm residual blocks
    eps: float = 1e-5                    # RMSNorm epsilon of the stacked workload
    note: str = ""


WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", T=64, d=256, F=512,
                     note="T=64, d=256, ffn=512; weights L2-resident; parity only"),
    "decode": Workload("decode", T=8, d=GROK_D, F=GROK_F,
                       note="T=8 tokens, one decode step at Grok-1 shape; HBM-bound"),
    "prefill": Workload("prefill", T=8192, d=GROK_D, F=GROK_F,
                        note="T=8192 tokens, one full 8192 context; tensor-bound"),
    "skewed": Workload("skewed", T=4096, d=GROK_D, F=GROK_F,
                       bias=[3.0, 1.5, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0],
                       note="T=4096, router logits biased +3 on expert 0 and +1.5 on expert 1"),
    "stacked": Workload("stacked", T=32, d=GROK_D, F=GROK_F, blocks=4,
                        note="4 stacked MoE blocks with pre/post RMSNorm and residual, T=32"),
}


def generator(seed: int, device: str | torch.device = "cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _int8_uniform(shape, g, device):
    # integers uniform on {-127, ..., 127}; -128 never occurs
    return torch.randint(-127, 128, shape, generator=g, device=device, dtype=torch.int8)


def _scale(shape, d, g, device):
    s = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    return (s / (127.0 * math.sqrt(d))).to(torch.bfloat16)


def draw_layer(d: int, F: int, E: int, g: torch.Generator, device) -> Dict[str, torch.Tensor]:
    """Draw one MoE layer's parameters in the fixed order router_w, wl, sl, wv, sv, w1, s1."""
    router_w = torch.randn((d, E), generator=g, device=device, dtype=torch.float32) / math.sqrt(d)
    wl = _int8_uniform((E, d, F), g, device)
    sl = _scale((E, F), d, g, device)
    wv = _int8_uniform((E, d, F), g, device)
    sv = _scale((E, F), d, g, device)
    w1 = _int8_uniform((E, F, d), g, device)
    s1 = _scale((E, d), d, g, device)
    return dict(router_w=router_w, wl=wl, sl=sl, wv=wv, sv=sv, w1=w1, s1=s1)


def block_scales(layer: Dict[str, torch.Tensor], kb: int, g: torch.Generator) -> Dict[str, torch.Tensor]:
    """The layer with per-block scales instead of per-output-channel ones: every block of kb
    input rows of every matrix gets its own scale row ([E, in/kb, out]), drawn like the
    per-channel scales.  Weights and router are shared with ``layer``."""
    E, d, F = layer["wl"].shape
    dev = layer["wl"].device
    out = dict(layer)
    out["sl"] = _scale((E, d // kb, F), d, g, dev)
    out["sv"] = _scale((E, d // kb, F), d, g, dev)
    out["s1"] = _scale((E, F // kb, d), d, g, dev)
    return out


def draw_tokens(T: int, d: int, g: torch.Generator, device) -> torch.Tensor:
    return torch.randn((T, d), generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)


@dataclass
class Inputs:
    workload: Workload
    layers: List[Dict[str, torch.Tensor]]
    x: torch.Tensor                      # bf16 [T, d]: layer input, or the residual stream h (stacked)
    bias: Optional[torch.Tensor] = None  # fp32 [E] or None
    gammas: List[Dict[str, torch.Tensor]] = field(default_factory=list)  # stacked: pre/post RMSNorm gains


def make_inputs(w: Workload | str, device="cpu", T: Optional[int] = None,
                seed: Optional[int] = None) -> Inputs:
    """Draw every tensor of a workload with its seeded generator.

    ``T`` overrides the token count (the parameters are drawn first, so the layer
    weights do not depend on T); ``seed`` overrides the workload's seed.
    """
    if isinstance(w, str):
        w = WORKLOADS[w]
    T = w.T if T is None else int(T)
    g = generator(w.seed if seed is None else seed, device)
    nblk = max(1, w.blocks)
    layers = [draw_layer(w.d, w.F, w.E, g, device) for _ in range(nblk)]
    x = draw_tokens(T, w.d, g, device)
    gammas = []
    if w.blocks:
        for _ in range(w.blocks):
            # unit RMSNorm gains: the workload has no trained weights
            gammas.append(dict(pre=torch.ones(w.d, dtype=torch.bfloat16, device=device),
                               post=torch.ones(w.d, dtype=torch.bfloat16, device=device)))
    bias = None
    if w.bias is not None:
        bias = torch.tensor(w.bias, dtype=torch.float32, device=device)
    return Inputs(workload=w, layers=layers, x=x, bias=bias, gammas=gammas)


def token_sample(T: int, n: int, seed: int = 1234, must_include: Optional[List[int]] = None) -> List[int]:
    """A seeded, sorted subset of ``n`` token indices out of ``T`` (plus required ones)."""
    g = generator(seed, "cpu")
    n = min(n, T)
    pick = torch.randperm(T, generator=g)[:n].tolist()
    s = set(int(i) for i in pick)
    for t in must_include or []:
        if 0 <= t < T:
            s.add(int(t))
    return sorted(s)
