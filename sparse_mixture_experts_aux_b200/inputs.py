"""Seeded synthetic inputs for the routed MoE FFN layer.

This module is the one piece shared by the CUDA path's callers (tests, bench)
and the oracle's callers: it only draws random tensors of the right shapes and
distributions. It holds none of the layer's arithmetic (no routing, no
softmax, no expert evaluation).

Recipe (the same for every workload):
  * x      ~ N(0, 1)           [T, d]         sampled in fp32, RNE-cast to the
                                              workload dtype (bf16 or fp32)
  * W_r    ~ N(0, 1/d)         [E, d]   fp32  (the router stays fp32)
  * W_g,W_u~ N(0, 1/d)         [E, d_e, d]    nn.Linear weight layout
  * W_d    ~ N(0, 1/d_e)       [E, d, d_e]
  * shared ~ same, width d_s, packed [gate (d_s x d) | up (d_s x d) | down (d x d_s)]
  * skewed router bias b_e = -1.2 * ln(e + 1) for the Zipf-skewed workload
  * selection-only bias (routing variants) ~ U(-0.05, 0.05) per expert, fp32, from
    its own seed: a stand-in for a learned balancing bias
"N(0, 1/fan_in)" is read as variance 1/fan_in.

FP8 expert weights drawn directly as data (make_fp8_weights): E4M3 codes
uniform over the 254 finite codes (a random sign, a magnitude field uniform in
0..0x7E), and one fp32 scale per output row ~ U(0.5, 1.5) / (100 sqrt(fan_in)),
so that the weights' RMS is near 1/sqrt(fan_in) (the RMS of a uniform finite
code is about 104).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and options of one layer call."""
    name: str
    T: int
    d: int
    E: int
    d_e: int
    k: int
    dtype: str = "bf16"          # "bf16" or "f32": dtype of x, expert weights and y
    d_s: int = 0                 # shared expert width (0 = none)
    capacity_factor: float = 0.0  # <= 0: no capacity limit
    zipf_bias: bool = False      # add b_e = -1.2 ln(e+1) to the router logits
    seed: int = 0
    gate_mode: int = 0           # 0 renormalised softmax, 1 raw softmax, 2 sigmoid
    selection_bias: bool = False  # draw a selection-only per-expert bias
    n_group: int = 0             # group-limited selection (0/1 = none)
    topk_group: int = 0

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads the layer is measured and checked on.
TINY_F32 = Workload("tiny-fp32 T=64 d=512 E=8 d_e=1024 k=2", 64, 512, 8, 1024, 2, "f32", seed=0)
MIXTRAL = Workload("mixtral-8x7b-layer T=4096 d=4096 E=8 d_e=14336 k=2", 4096, 4096, 8, 14336, 2, seed=1)
DEEPSEEK_V3 = Workload("deepseek-v3-layer T=8192 d=7168 E=256 d_e=2048 k=8 +shared 2048",
                       8192, 7168, 256, 2048, 8, d_s=2048, seed=2)
SWITCH_ZIPF = Workload("switch-top1-cf1.25-zipf T=16384 d=2048 E=64 d_e=8192 k=1",
                       16384, 2048, 64, 8192, 1, capacity_factor=1.25, zipf_bias=True, seed=3)
MIXTRAL_DECODE = Workload("mixtral-decode T=32 d=4096 E=8 d_e=14336 k=2", 32, 4096, 8, 14336, 2, seed=4)

ALL_WORKLOADS = (TINY_F32, MIXTRAL, DEEPSEEK_V3, SWITCH_ZIPF, MIXTRAL_DECODE)

# A smaller case with the Mixtral expert shape and the full layer's load of
# 1024 routed rows per expert (so the same kernel choices: 1-CTA gate/up, CTA
# pairs for down), about 0.8 GB on the device, for hardware-counter captures.
MIXTRAL_PROFILE = Workload("mixtral-shape-profile T=1024 d=4096 E=2 d_e=14336 k=2",
                           1024, 4096, 2, 14336, 2, seed=1)
# The decode shape with 2 experts (about 0.7 GB of bf16 weights), likewise.
DECODE_PROFILE = Workload("decode-shape-profile T=32 d=4096 E=2 d_e=14336 k=2",
                          32, 4096, 2, 14336, 2, seed=4)
# The Mixtral-shaped layer's routing, permute and combine work (T, d, E and k
# as in the full layer; those kernels do not depend on d_e) with narrow
# experts, so the whole case holds about 0.2 GB, for hardware-counter captures.
ROUTING_PROFILE = Workload("routing-kernels-profile T=4096 d=4096 E=8 d_e=256 k=2",
                           4096, 4096, 8, 256, 2, seed=1)
# The DeepSeek-V3 expert shape (d = 7168, d_e = 2048, k = 8, the shared expert)
# with 32 experts and 1024 tokens: the full layer's load of 256 routed rows per
# expert, so the same kernel choices, with about 3 GB on the device.
DSV3_PROFILE = Workload("dsv3-shape-profile T=1024 d=7168 E=32 d_e=2048 k=8 +shared 2048",
                        1024, 7168, 32, 2048, 8, d_s=2048, seed=2)
# The DeepSeek-V3-shaped router (T, d, E and k of that layer) with narrow
# experts, about 1 GB on the device.
DSV3_ROUTING_PROFILE = Workload("dsv3-routing-profile T=8192 d=7168 E=256 d_e=64 k=8",
                                8192, 7168, 256, 64, 8, seed=2)


def zipf_router_bias(E: int) -> torch.Tensor:
    """Per-expert logit offset log(1/rank^1.2) with rank = e + 1 (fp32)."""
    return torch.tensor([-1.2 * math.log(e + 1.0) for e in range(E)], dtype=torch.float32)


def _normal(shape, std: float, gen: torch.Generator, device) -> torch.Tensor:
    return torch.randn(*shape, generator=gen, device=device, dtype=torch.float32).mul_(std)


def make_inputs(w: Workload, device: str = "cpu", x_seed_offset: int = 0) -> dict:
    """Draw every input of one layer call for workload `w` on `device`.

    Returns a dict with x, W_r, W_g, W_u, W_d, W_shared (or None), router_bias
    (or None). Values are sampled in fp32 then cast (RNE) to the workload dtype.
    """
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed)
    dt = w.torch_dtype
    T, d, E, de = w.T, w.d, w.E, w.d_e
    W_r = _normal((E, d), 1.0 / math.sqrt(d), gen, device)
    W_g = _normal((E, de, d), 1.0 / math.sqrt(d), gen, device).to(dt)
    W_u = _normal((E, de, d), 1.0 / math.sqrt(d), gen, device).to(dt)
    W_d = _normal((E, d, de), 1.0 / math.sqrt(de), gen, device).to(dt)
    W_shared = None
    if w.d_s > 0:
        ds = w.d_s
        sg = _normal((ds, d), 1.0 / math.sqrt(d), gen, device)
        su = _normal((ds, d), 1.0 / math.sqrt(d), gen, device)
        sd = _normal((d, ds), 1.0 / math.sqrt(ds), gen, device)
        W_shared = torch.cat([sg.reshape(-1), su.reshape(-1), sd.reshape(-1)]).to(dt)
    x = make_x(w, device, x_seed_offset)
    bias = zipf_router_bias(E).to(device) if w.zipf_bias else None
    sel = None
    if w.selection_bias:
        gs = torch.Generator(device="cpu")
        gs.manual_seed(20_000 + w.seed)
        sel = (torch.rand(E, generator=gs, dtype=torch.float32) * 0.1 - 0.05).to(device)
    return dict(x=x, W_r=W_r, W_g=W_g, W_u=W_u, W_d=W_d, W_shared=W_shared, router_bias=bias,
                selection_bias=sel)


def make_x(w: Workload, device: str = "cpu", seed_offset: int = 0, T: Optional[int] = None) -> torch.Tensor:
    """Token activations x ~ N(0,1) [T, d] in the workload dtype, from their own seed."""
    gen = torch.Generator(device=device)
    gen.manual_seed(10_000 + 7919 * w.seed + seed_offset)
    T = w.T if T is None else T
    return _normal((T, w.d), 1.0, gen, device).to(w.torch_dtype)


def split_shared(W_shared: torch.Tensor, d: int, d_s: int):
    """View the packed shared-expert buffer as (gate [d_s,d], up [d_s,d], down [d,d_s])."""
    n = d_s * d
    return (W_shared[:n].view(d_s, d), W_shared[n:2 * n].view(d_s, d), W_shared[2 * n:3 * n].view(d, d_s))


def make_fp8_weights(w: Workload, device: str = "cpu") -> dict:
    """Random E4M3 expert weights for workload `w`: uint8 codes W_g, W_u [E, d_e, d],
    W_d [E, d, d_e] and weight_scales fp32 [E*d_e | E*d_e | E*d] (that order)."""
    gen = torch.Generator(device=device)
    gen.manual_seed(30_000 + w.seed)
    E, d, de = w.E, w.d, w.d_e

    def codes(shape):
        mag = torch.randint(0, 0x7F, shape, generator=gen, device=device, dtype=torch.int32)
        sign = torch.randint(0, 2, shape, generator=gen, device=device, dtype=torch.int32) << 7
        return (mag | sign).to(torch.uint8)

    def scales(n, fan_in):
        u = torch.rand(n, generator=gen, device=device, dtype=torch.float32) + 0.5
        return u / (100.0 * math.sqrt(fan_in))

    W_g, W_u, W_d = codes((E, de, d)), codes((E, de, d)), codes((E, d, de))
    sc = torch.cat([scales(E * de, d), scales(E * de, d), scales(E * d, de)])
    return dict(W_g=W_g, W_u=W_u, W_d=W_d, weight_scales=sc)
