"""Shared helpers of the parity tests: seeded inputs -> oracle references, and
the tolerance checks.  Expected values come only from ``oracle/``."""
from __future__ import annotations

import math

import numpy as np
import torch

from mla_latent_kv_write_b200 import inputs as I
from oracle import videomla_oracle as O

# Attention: output RMS relative error <= 5e-3 and max abs <= 1e-2 max|ref| + 1e-3.
ATTN_RMS_REL = 5e-3
ATTN_MAX_REL, ATTN_MAX_ABS = 1e-2, 1e-3
# lse of the scaled scores (natural log): its error is a weighted mean of score
# errors, which grow with the score magnitude, hence abs + rel.
LSE_ABS, LSE_REL = 5e-3, 1e-3
# cache_write latent: norm-wise relative error <= 2e-3; elementwise within one
# bf16 ulp of the oracle (bf16 RNE output of an fp32 sum may round either way).
CACHE_NORM_REL = 2e-3


def f64(t: torch.Tensor) -> np.ndarray:
    return I.to_numpy64(t)


def oracle_cache(dims: I.Dims, x: torch.Tensor, w: dict, slots: int, first_slot: int,
                 base: np.ndarray | None = None, normalize: bool = True, chunk_frames: int = 6) -> np.ndarray:
    """fp64 cache after writing the tokens ``x`` (CPU bf16) into ``base``
    (fp64, or zeros).  Written frame-chunk by frame-chunk to bound memory."""
    B, n_tok, _ = x.shape
    T_f = dims.tokens_per_frame
    cache = np.zeros((B, slots * T_f, dims.cache_width)) if base is None else base
    W_dkv, W_kr = f64(w["W_dkv"]), f64(w["W_kr"])
    gamma = f64(w["gamma"])
    for f0 in range(0, n_tok // T_f, chunk_frames):
        f1 = min(f0 + chunk_frames, n_tok // T_f)
        O.cache_write(f64(x[:, f0 * T_f:f1 * T_f]), W_dkv, W_kr, gamma, dims.rms_eps, cache,
                      slots, (first_slot + f0) % slots, T_f, normalize=normalize)
    return cache


def to_bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(a).to(torch.bfloat16)


def oracle_attention(dims: I.Dims, q: dict, w: dict, cache_bf16: torch.Tensor, slots: int, oldest: int,
                     n_valid: int, rows=None, sink_bf16: torch.Tensor = None):
    """The oracle's absorbed form; pinned sink frames (``sink_bf16`` [B, n_sink T_f, W])
    go before the ring rows, the layout the oracle's window functions read."""
    cache = f64(cache_bf16)
    n_sink = 0
    if sink_bf16 is not None:
        n_sink = sink_bf16.shape[1] // dims.tokens_per_frame
        cache = np.concatenate([f64(sink_bf16), cache], axis=1)
    return O.attention_absorbed(f64(q["q_nope"]), f64(q["q_rope"]), f64(w["W_uk"]), f64(w["W_uv"]),
                                cache, slots, oldest, n_valid, dims.grid_h, dims.grid_w, dims.d_c,
                                dims.rope_base, dims.pairs, query_rows=rows, n_sink=n_sink)


def check_attention(got: np.ndarray, ref: np.ndarray, what: str = ""):
    err = got - ref
    rms_rel = np.linalg.norm(err) / np.linalg.norm(ref)
    max_abs = np.max(np.abs(err))
    bound = ATTN_MAX_REL * np.max(np.abs(ref)) + ATTN_MAX_ABS
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    assert rms_rel <= ATTN_RMS_REL, f"{what}: rms rel err {rms_rel:.3e}"
    assert max_abs <= bound, f"{what}: max abs err {max_abs:.3e} > {bound:.3e}"
    return rms_rel, max_abs


def check_lse(got: np.ndarray, ref: np.ndarray, what: str = ""):
    e = np.abs(got - ref)
    assert np.all(e <= LSE_ABS + LSE_REL * np.abs(ref)), f"{what}: lse err {np.max(e):.3e}"
    return float(np.max(e))


def check_cache(got: np.ndarray, ref: np.ndarray, d_c: int, what: str = ""):
    """got: decoded bf16 rows, ref: fp64 oracle rows (same shape)."""
    for name, sl in (("latent", slice(0, d_c)), ("rope key", slice(d_c, None))):
        g, r = got[..., sl], ref[..., sl]
        rel = np.linalg.norm(g - r) / np.linalg.norm(r)
        assert rel <= CACHE_NORM_REL, f"{what} {name}: norm rel err {rel:.3e}"
        # one bf16 ulp of the oracle value (2^-7 of its power of two), plus an
        # absolute slack of 1e-5 rms for results that cancel to ~0: the fp32
        # accumulation over d_model = 1536 products leaves ~1e-6 rms absolute error
        ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(r), 1e-30))) - 7)
        ratio = np.abs(g - r) / (ulp + 1e-5 * np.sqrt(np.mean(r * r)))
        k = np.unravel_index(np.argmax(ratio), ratio.shape)
        info = (f"{what} {name}: norm rel {rel:.2e}, worst {ratio[k]:.2f} ulp at {k}: got {g[k]:.6g} "
                f"ref {r[k]:.6g}; {np.mean(ratio > 1):.2e} of elements beyond 1 ulp")
        print(info)
        assert ratio[k] <= 1.0001, info


def sample_rows(n: int, k: int, seed: int) -> np.ndarray:
    """k query rows of n: the first and last tile edges plus seeded random rows."""
    rng = np.random.default_rng(seed)
    edge = [0, 1, 127, 128, n - 1, n - 2]
    rows = set(r for r in edge if 0 <= r < n)
    rows |= set(rng.choice(n, size=min(k, n), replace=False).tolist())
    return np.array(sorted(rows))


def rms(a):
    return math.sqrt(float(np.mean(np.square(a))))
