"""Seeded synthetic inputs for the MoE layer with zero-computation experts.

This module only draws tensors; it holds none of the layer's arithmetic. Both
the CPU oracle (through the tests and the bench's CPU leg) and the CUDA library
are fed from the tensors made here, so the two sides always see identical
inputs.

Shapes follow the LongCat-2.0 model card (archdb), section "Mixture of
experts": routed experts plus identity zero-experts scored together by one
router classifier, top-k per token, and an expert FFN width. The workloads are
scaled-down versions of that layer (see ``CONFIGS``).

Recipe (every tensor has its own ``torch.Generator`` seeded from
``(seed, tensor tag, expert)``, so any expert can be drawn alone):

* ``x``      [T, d]      ~ N(0, 1), cast to the activation dtype.
* ``w_router`` [E, d]    ~ N(0, 1/d), fp32 (E = n_routed + n_zero; routed ids
  first, zero-expert ids last).
* ``bias``   [E]         ~ U(-0.1, 0.1), fp32, plus the routing skew below.
* ``w_gate``, ``w_up`` [N, F, d] and ``w_down`` [N, d, F] ~ N(0, 1/d), cast to
  the activation dtype (row-major, the contraction dimension innermost).

Routing skew added to ``bias`` (selection-only input; the layer itself never
changes it):

* ``uniform``    : nothing added.
* ``zipf``       : routed expert e gets ``3.0 * r_e ** -1.1`` where r_e in 1..N is
  a seeded permutation rank; zero experts get 0. This reproduces the load
  imbalance the Ascend deployment article describes (section on dynamic
  expert load balancing).
* ``zero_share`` : every zero expert gets the same offset beta, tuned per seed
  on the oracle's router so that about 30 % of routing slots land on zero
  experts (stored in ``zero_share_beta.json`` by ``tune_zero_share.py``).
"""
from __future__ import annotations

import json
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, replace
from typing import Dict, Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
BETA_FILE = os.path.join(_HERE, "zero_share_beta.json")


@dataclass(frozen=True)
class MoEShape:
    name: str
    T: int
    d: int
    n_routed: int
    n_zero: int
    top_k: int
    ffn: int
    act_dtype: str = "bf16"  # "f32" or "bf16"
    routed_scale: float = 1.0
    routing: str = "uniform"  # "uniform" | "zipf" | "zero_share"

    @property
    def E(self) -> int:
        return self.n_routed + self.n_zero

    def with_T(self, T: int) -> "MoEShape":
        return replace(self, T=T, name=f"{self.name}_T{T}")


CONFIGS: Dict[str, MoEShape] = {
    # tiny fp32 layer: 8 routed (SwiGLU, F=512) + 2 zero experts, top-2
    "tiny_fp32": MoEShape("tiny_fp32", T=128, d=256, n_routed=8, n_zero=2,
                          top_k=2, ffn=512, act_dtype="f32"),
    # bf16 decode layer: weight-streaming bound
    "decode": MoEShape("decode", T=64, d=4096, n_routed=128, n_zero=32,
                       top_k=8, ffn=1024),
    # bf16 prefill layer with Zipf-skewed expert load
    "prefill": MoEShape("prefill", T=16384, d=4096, n_routed=128, n_zero=32,
                        top_k=8, ffn=1024, routing="zipf"),
    # bf16 large-expert-count layer, ~30 % of slots on zero experts
    "large_e": MoEShape("large_e", T=8192, d=6144, n_routed=256, n_zero=64,
                        top_k=12, ffn=2048, routing="zero_share"),
    # small cases of the same kernels for profiler captures (weights ~0.8 GB,
    # still larger than L2)
    "profile_decode": MoEShape("profile_decode", T=64, d=4096, n_routed=32,
                               n_zero=8, top_k=8, ffn=1024),
    "profile_prefill": MoEShape("profile_prefill", T=4096, d=4096, n_routed=32,
                                n_zero=8, top_k=8, ffn=1024, routing="zipf"),
    # the decode layer's router (T=64, 160 experts) with narrow experts, so
    # that a profiler capture holds ~0.4 GB of weights
    "profile_router": MoEShape("profile_router", T=64, d=4096, n_routed=128,
                               n_zero=32, top_k=8, ffn=128),
    # the large-expert layer's density (~270 rows per expert), 32 experts
    "profile_large_e": MoEShape("profile_large_e", T=1024, d=6144, n_routed=32,
                                n_zero=8, top_k=12, ffn=2048),
    # the same density above 1024 tokens, where the expert GEMMs run on CTA
    # pairs: 64 routed + 28 zero experts (~70 % routed slots, ~270 rows per
    # expert), 4.8 GB of weights
    "profile_large_e_pairs": MoEShape("profile_large_e_pairs", T=2048, d=6144,
                                      n_routed=64, n_zero=28, top_k=12, ffn=2048),
}

SWEEP_T = (1, 8, 64, 512, 4096, 32768)


def sweep_config(T: int, routing: str = "uniform") -> MoEShape:
    """Sweep layer: d=6144, 256 routed (F=2048) + 64 zero experts, top-12."""
    if routing not in ("uniform", "zipf"):
        raise ValueError(routing)
    return MoEShape(f"sweep_{routing}_T{T}", T=T, d=6144, n_routed=256,
                    n_zero=64, top_k=12, ffn=2048, routing=routing)


def get_config(name: str) -> MoEShape:
    if name in CONFIGS:
        return CONFIGS[name]
    if name.startswith("sweep_"):
        _, routing, t = name.split("_")
        return sweep_config(int(t[1:]), routing)
    raise KeyError(name)


_TAGS = {"x": 1, "w_router": 2, "bias": 3, "w_gate": 4, "w_up": 5,
         "w_down": 6, "zipf": 7}


def _gen(seed: int, tag: str, sub: int = 0) -> torch.Generator:
    s = (int(seed) * 1_000_003 + _TAGS[tag] * 100_003 + int(sub)) % (2 ** 62)
    return torch.Generator().manual_seed(s)


def torch_dtype(act_dtype: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[act_dtype]


@dataclass
class Inputs:
    shape: MoEShape
    seed: int
    x: torch.Tensor
    w_router: torch.Tensor
    bias: torch.Tensor
    w_gate: Optional[torch.Tensor]
    w_up: Optional[torch.Tensor]
    w_down: Optional[torch.Tensor]

    def to(self, device) -> "Inputs":
        mv = lambda t: None if t is None else t.to(device)
        return Inputs(self.shape, self.seed, mv(self.x), mv(self.w_router),
                      mv(self.bias), mv(self.w_gate), mv(self.w_up),
                      mv(self.w_down))


def zipf_offsets(shape: MoEShape, seed: int) -> torch.Tensor:
    """Per-expert selection offset 3.0 * rank**-1.1 over a seeded rank order."""
    g = _gen(seed, "zipf")
    rank = torch.randperm(shape.n_routed, generator=g).to(torch.float64) + 1.0
    off = torch.zeros(shape.E, dtype=torch.float64)
    off[: shape.n_routed] = 3.0 * rank.pow(-1.1)
    return off.to(torch.float32)


def load_betas() -> dict:
    if not os.path.exists(BETA_FILE):
        return {}
    with open(BETA_FILE) as f:
        return json.load(f)


def beta_key(shape: MoEShape, seed: int) -> str:
    return (f"T{shape.T}_d{shape.d}_N{shape.n_routed}_Z{shape.n_zero}"
            f"_k{shape.top_k}_seed{seed}")


def base_bias(shape: MoEShape, seed: int) -> torch.Tensor:
    g = _gen(seed, "bias")
    return (torch.rand(shape.E, generator=g, dtype=torch.float32) * 0.2 - 0.1)


def make_tokens(shape: MoEShape, seed: int) -> torch.Tensor:
    """x [T, d] alone: the token batch of `seed` (the same tensor make_inputs
    draws for that seed)."""
    dt = torch_dtype(shape.act_dtype)
    return torch.randn(shape.T, shape.d, generator=_gen(seed, "x")).to(dt).contiguous()


def make_router_inputs(shape: MoEShape, seed: int, beta: Optional[float] = None):
    """x, w_router and bias only (no expert weights)."""
    x = make_tokens(shape, seed)
    w_r = torch.randn(shape.E, shape.d, generator=_gen(seed, "w_router")) * (
        1.0 / shape.d ** 0.5)
    b = base_bias(shape, seed)
    if shape.routing == "zipf":
        b = b + zipf_offsets(shape, seed)
    elif shape.routing == "zero_share":
        if beta is None:
            betas = load_betas()
            key = beta_key(shape, seed)
            if key not in betas:
                raise KeyError(
                    f"no tuned zero-expert offset for {key}; run "
                    f"python -m moe_synth.tune_zero_share")
            beta = float(betas[key]["beta"])
        b = b.clone()
        b[shape.n_routed:] += float(beta)
    return x.contiguous(), w_r.contiguous(), b.contiguous()


def make_expert(shape: MoEShape, seed: int, e: int):
    """Weights of routed expert e: (w_gate[e] [F,d], w_up[e] [F,d], w_down[e] [d,F])."""
    dt = torch_dtype(shape.act_dtype)
    std = 1.0 / shape.d ** 0.5
    wg = (torch.randn(shape.ffn, shape.d, generator=_gen(seed, "w_gate", e)) * std).to(dt)
    wu = (torch.randn(shape.ffn, shape.d, generator=_gen(seed, "w_up", e)) * std).to(dt)
    wd = (torch.randn(shape.d, shape.ffn, generator=_gen(seed, "w_down", e)) * std).to(dt)
    return wg, wu, wd


_expert_cache: dict = {}


def make_experts(shape: MoEShape, seed: int):
    """All routed experts' weights. They depend only on (seed, N, F, d, dtype),
    so layers that differ only in T or routing share them; the last set drawn
    is kept (read-only use)."""
    key = (seed, shape.n_routed, shape.ffn, shape.d, shape.act_dtype)
    if key in _expert_cache:
        return _expert_cache[key]
    _expert_cache.clear()
    dt = torch_dtype(shape.act_dtype)
    N, F, d = shape.n_routed, shape.ffn, shape.d
    wg = torch.empty(N, F, d, dtype=dt)
    wu = torch.empty(N, F, d, dtype=dt)
    wd = torch.empty(N, d, F, dtype=dt)

    def draw(e):
        wg[e], wu[e], wd[e] = make_expert(shape, seed, e)

    # every expert has its own generator, so drawing them on several threads
    # gives the same tensors as drawing them in order
    with ThreadPoolExecutor(max(1, min(16, os.cpu_count() or 1))) as ex:
        list(ex.map(draw, range(N)))
    _expert_cache[key] = (wg, wu, wd)
    return wg, wu, wd


def make_inputs(shape: MoEShape, seed: int = 0, with_experts: bool = True,
                beta: Optional[float] = None) -> Inputs:
    x, w_r, b = make_router_inputs(shape, seed, beta)
    wg = wu = wd = None
    if with_experts:
        wg, wu, wd = make_experts(shape, seed)
    return Inputs(shape, seed, x, w_r, b, wg, wu, wd)
