"""Seeded synthetic inputs for the VideoMLA latent-KV hot path.

This module is shared by the tests, the benchmark and the smoke check. It draws
random tensors and describes workload shapes; it holds none of the method's
arithmetic (no projection, normalisation, rotation or attention), so both the
CUDA path and the fp64 oracle can consume its output without sharing any code.

Shapes follow the Wan2.1-T2V-1.3B backbone described in "VideoMLA: Low-Rank
Latent KV Cache for Minute-Scale Autoregressive Video Diffusion" (arXiv
2605.30351): App. C.1 and D.1 (30 x 52 = 1560 tokens per latent frame, 12 heads,
d = 1536, 3-latent-frame chunks) and App. D.2 / Table 4 (d_c = 192,
d_rope = 32, d_nope = 96, 3D-RoPE pairs (6, 5, 5)).

Distributions:
  * activations x, q_nope, q_rope ~ N(0, 1), rounded to bf16 (RNE);
  * weights ~ N(0, 1/fan_in): fan_in = d_model for W_dkv and W_kr, fan_in = d_c
    for the up-projections W_uk and W_uv;
  * gamma (RMSNorm gain) = 1, or 1 + 0.1 N(0, 1) for tests that must see it;
  * "peaky" workloads scale a Bernoulli(p) subset of tokens of x by a factor.
All draws use a CPU ``torch.Generator`` seeded with
``1000 * config + 10 * layer + step``.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import torch


@dataclasses.dataclass(frozen=True)
class Dims:
    """Layer geometry. ``pairs`` is the 3D-RoPE complex-pair split over (t, h, w)."""

    d_model: int = 1536
    n_heads: int = 12
    d_c: int = 192
    d_rope: int = 32
    d_nope: int = 96
    d_v: int = 128
    grid_h: int = 30
    grid_w: int = 52
    pairs: tuple = (6, 5, 5)
    rope_base: float = 10000.0
    rms_eps: float = 1e-6
    d_q: int = 768          # query latent width (App. D.2)

    @property
    def tokens_per_frame(self) -> int:
        return self.grid_h * self.grid_w

    @property
    def cache_width(self) -> int:
        return self.d_c + self.d_rope


@dataclasses.dataclass(frozen=True)
class Workload:
    """One benchmark / parity configuration.

    ``slots``: ring capacity in frames.  ``prefill``: frames written before the
    measured step.  ``chunk``: frames written and queried per step.  ``steps``:
    consecutive steps (rolling workloads).  ``layers``: independent layers.
    """

    name: str
    index: int
    dims: Dims
    batch: int
    slots: int
    prefill: int
    chunk: int
    steps: int = 1
    layers: int = 1
    peaky_fraction: float = 0.0
    peaky_scale: float = 1.0

    @property
    def n_query(self) -> int:
        return self.chunk * self.dims.tokens_per_frame

    @property
    def n_keys_full(self) -> int:
        return self.slots * self.dims.tokens_per_frame


WAN = Dims()
TINY = dataclasses.replace(WAN, grid_h=6, grid_w=8)

# The five workloads: tiny single layer, the Wan-1.3B-shaped layer (the headline
# measurement), a 40-step rolling ring, a 63-frame long window with peaky
# tokens, and a 30-layer sweep over (d_c, d_rope).
WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", 0, TINY, batch=1, slots=3, prefill=2, chunk=1),
    "wan_layer": Workload("wan_layer", 1, WAN, batch=1, slots=21, prefill=18, chunk=3),
    "rolling": Workload("rolling", 2, WAN, batch=1, slots=21, prefill=0, chunk=1, steps=40),
    "long": Workload("long", 3, WAN, batch=2, slots=63, prefill=60, chunk=3,
                     peaky_fraction=0.01, peaky_scale=8.0),
}

# (d_c, d_rope) points of the rank / RoPE allocation sweep; d_nope = 128 - d_rope.
SWEEP_POINTS = ((96, 32), (192, 16), (192, 32), (192, 64), (384, 32))
# 3D-RoPE pair split for each d_rope of the sweep: (6, 5, 5) is printed for
# d_rope = 32; the other two follow the same split rule.
SWEEP_PAIRS = {16: (4, 2, 2), 32: (6, 5, 5), 64: (12, 10, 10)}


def sweep_dims(d_c: int, d_rope: int) -> Dims:
    return dataclasses.replace(WAN, d_c=d_c, d_rope=d_rope, d_nope=128 - d_rope,
                               pairs=SWEEP_PAIRS[d_rope])


def sweep_workload(d_c: int, d_rope: int, layers: int = 30) -> Workload:
    return Workload(f"sweep_c{d_c}_r{d_rope}", 4, sweep_dims(d_c, d_rope), batch=1,
                    slots=21, prefill=18, chunk=3, layers=layers)


def seed_for(config: int, layer: int = 0, step: int = 0) -> int:
    return 1000 * config + 10 * layer + step


def _normal(gen: torch.Generator, shape, std: float = 1.0) -> torch.Tensor:
    t = torch.randn(*shape, generator=gen, dtype=torch.float32)
    if std != 1.0:
        t = t * std
    return t.to(torch.bfloat16)


def projection_weights(dims: Dims, seed: int, random_gamma: bool = False) -> Dict[str, torch.Tensor]:
    """Random-init query-path and output weights of one layer (CPU tensors):
    W_dq [d_q, d_model], W_uq [H*d_nope, d_q], W_qr [H*d_rope, d_q],
    W_O [d_model, H*d_v] in bf16 (N(0, 1/fan_in)); gamma_q [d_q] in fp32."""
    g = torch.Generator().manual_seed(seed)
    d, H = dims.d_model, dims.n_heads
    w = {
        "W_dq": _normal(g, (dims.d_q, d), d ** -0.5),
        "W_uq": _normal(g, (H * dims.d_nope, dims.d_q), dims.d_q ** -0.5),
        "W_qr": _normal(g, (H * dims.d_rope, dims.d_q), dims.d_q ** -0.5),
        "W_O": _normal(g, (d, H * dims.d_v), (H * dims.d_v) ** -0.5),
    }
    if random_gamma:
        w["gamma_q"] = 1.0 + 0.1 * torch.randn(dims.d_q, generator=g, dtype=torch.float32)
    else:
        w["gamma_q"] = torch.ones(dims.d_q, dtype=torch.float32)
    return w


def layer_weights(dims: Dims, seed: int, random_gamma: bool = False) -> Dict[str, torch.Tensor]:
    """Random-init weights of one VideoMLA attention layer (CPU tensors).

    W_dkv [d_c, d_model], W_kr [d_rope, d_model], W_uk [H*d_nope, d_c],
    W_uv [H*d_v, d_c] in bf16; gamma [d_c] in fp32.
    """
    g = torch.Generator().manual_seed(seed)
    d, H = dims.d_model, dims.n_heads
    w = {
        "W_dkv": _normal(g, (dims.d_c, d), d ** -0.5),
        "W_kr": _normal(g, (dims.d_rope, d), d ** -0.5),
        "W_uk": _normal(g, (H * dims.d_nope, dims.d_c), dims.d_c ** -0.5),
        "W_uv": _normal(g, (H * dims.d_v, dims.d_c), dims.d_c ** -0.5),
    }
    if random_gamma:
        w["gamma"] = 1.0 + 0.1 * torch.randn(dims.d_c, generator=g, dtype=torch.float32)
    else:
        w["gamma"] = torch.ones(dims.d_c, dtype=torch.float32)
    return w


def tokens(dims: Dims, batch: int, n_tok: int, seed: int,
           peaky_fraction: float = 0.0, peaky_scale: float = 1.0) -> torch.Tensor:
    """Token activations x [B, n_tok, d_model] bf16; optional peaky subset."""
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(batch, n_tok, dims.d_model, generator=g, dtype=torch.float32)
    if peaky_fraction > 0.0:
        mask = torch.rand(batch, n_tok, 1, generator=g) < peaky_fraction
        x = torch.where(mask, x * peaky_scale, x)
    return x.to(torch.bfloat16)


def queries(dims: Dims, batch: int, n_query: int, seed: int) -> Dict[str, torch.Tensor]:
    """Per-head queries: q_nope [B, Nq, H, d_nope] and unrotated q_rope
    [B, Nq, H, d_rope], both bf16."""
    g = torch.Generator().manual_seed(seed)
    H = dims.n_heads
    return {
        "q_nope": _normal(g, (batch, n_query, H, dims.d_nope)),
        "q_rope": _normal(g, (batch, n_query, H, dims.d_rope)),
    }


def latent_cache(dims: Dims, batch: int, slots: int, seed: int,
                 rope_scale: float = 1.0) -> torch.Tensor:
    """A directly drawn bf16 cache [B, slots*T_f, d_c + d_rope] with N(0, 1)
    entries (rope columns times ``rope_scale``), for attention-only cases."""
    g = torch.Generator().manual_seed(seed)
    c = torch.randn(batch, slots * dims.tokens_per_frame, dims.cache_width, generator=g)
    if rope_scale != 1.0:
        c[..., dims.d_c:] *= rope_scale
    return c.to(torch.bfloat16)


def rolling_window(step: int, slots: int) -> Dict[str, int]:
    """Ring bookkeeping of a frame-by-frame rollout starting from an empty ring:
    step s writes frame s into slot s mod slots and then attends over the
    min(s + 1, slots) newest frames.  Pure index bookkeeping."""
    n_valid = min(step + 1, slots)
    oldest = 0 if step + 1 <= slots else (step + 1) % slots
    return {"write_slot": step % slots, "oldest": oldest, "n_valid": n_valid}


def to_numpy64(t: torch.Tensor):
    """Exact decode of a (bf16 / fp32) CPU tensor to a float64 numpy array."""
    return t.detach().to("cpu", torch.float64).numpy()


def optional(t: Optional[torch.Tensor]):
    return None if t is None else to_numpy64(t)
