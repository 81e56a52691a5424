"""Batch scaling of a fixed memory budget: latent cache vs dense per-head KV.

"VideoMLA: Low-Rank Latent KV Cache for Minute-Scale Autoregressive Video
Diffusion" (arXiv 2605.30351), Sec. 4.3 and Fig. 7: under one B200's memory,
dense MHA runs out of memory at batch 28, the per-request memory slope falls
from 6.26 GB for MHA to 0.57-1.43 GB for the latent cache at
d_c in {64, 128, 192, 256, 512}, and d_c = 192 gives 8.0x the batch.

Model: memory(B) = fixed + B * slope, slope = per-request cache bytes (closed
form: layers x window frames x tokens per frame x cached scalars per token x
2 bytes) + a per-request non-cache term (activations of one request).  The
pages print the slopes but not their split, so the non-cache terms are fitted
to the printed slopes (one for the dense layout, one for the latent layout):
that part of the model is not closed form.  The largest batch is
floor((budget - fixed) / slope).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Iterable

GB = 1e9


@dataclasses.dataclass(frozen=True)
class Geometry:
    layers: int = 30              # Wan2.1-1.3B transformer blocks (App. C.1)
    frames: int = 21              # latent frames of a 5 s clip held in the cache (App. C.1)
    tokens_per_frame: int = 1560  # 30 x 52 latent grid (App. D.1)
    n_heads: int = 12
    d_head: int = 128
    d_rope: int = 32
    bytes_per_scalar: int = 2     # bf16


def latent_cache_gb(d_c: int, g: Geometry = Geometry()) -> float:
    """Per-request latent cache: (d_c + d_rope) scalars per token and layer."""
    return g.layers * g.frames * g.tokens_per_frame * (d_c + g.d_rope) * g.bytes_per_scalar / GB


def dense_cache_gb(g: Geometry = Geometry()) -> float:
    """Per-request dense cache: 2 n_h d_h scalars (per-head K and V) per token and layer."""
    return g.layers * g.frames * g.tokens_per_frame * 2 * g.n_heads * g.d_head * g.bytes_per_scalar / GB


# Slopes printed in Sec. 4.3 (GB per request).
PRINTED_DENSE_SLOPE = 6.26
PRINTED_LATENT_SLOPES = {64: 0.57, 512: 1.43}   # the two ends of the printed 0.57-1.43 range


def fitted_non_cache_gb(g: Geometry = Geometry()) -> Dict[str, float]:
    """Per-request non-cache memory fitted to the printed slopes: the dense
    term from the MHA slope, the latent term as the mean over the printed ends
    of the latent range."""
    dense = PRINTED_DENSE_SLOPE - dense_cache_gb(g)
    latent = sum(s - latent_cache_gb(dc, g) for dc, s in PRINTED_LATENT_SLOPES.items()) / len(PRINTED_LATENT_SLOPES)
    return {"dense": dense, "latent": latent}


def max_batch(free_gb: float, slope_gb: float) -> int:
    """Largest batch whose per-request memory fits ``free_gb`` (budget - fixed)."""
    return int(math.floor(free_gb / slope_gb))


def free_budget_from_dense_oom(oom_batch: int = 28, g: Geometry = Geometry()) -> float:
    """Budget left after the fixed memory, read from the printed dense OOM point:
    batch oom_batch - 1 fits, oom_batch does not; the midpoint of that interval."""
    slope = dense_cache_gb(g) + fitted_non_cache_gb(g)["dense"]
    return (oom_batch - 0.5) * slope


def batch_scaling(d_cs: Iterable[int] = (64, 128, 192, 256, 512), g: Geometry = Geometry()) -> Dict:
    """Slopes, largest batches and batch headroom against dense MHA for each d_c."""
    nc = fitted_non_cache_gb(g)
    free = free_budget_from_dense_oom(g=g)
    dense_slope = dense_cache_gb(g) + nc["dense"]
    dense_b = max_batch(free, dense_slope)
    rows = {}
    for dc in d_cs:
        s = latent_cache_gb(dc, g) + nc["latent"]
        b = max_batch(free, s)
        rows[dc] = {"cache_gb": latent_cache_gb(dc, g), "slope_gb": s, "max_batch": b, "headroom": b / dense_b,
                    "slope_reduction": 1.0 - s / dense_slope}
    return {"free_gb": free, "dense": {"cache_gb": dense_cache_gb(g), "slope_gb": dense_slope, "max_batch": dense_b},
            "latent": rows, "non_cache_gb": nc}
