"""fp64 CPU oracle for the VideoMLA latent-KV hot path.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's
CPU-baseline leg may import this module.  It shares no code with the CUDA path
(no kernels, headers, helpers, tables or constants) and never imports it.

Everything here follows "VideoMLA: Low-Rank Latent KV Cache for Minute-Scale
Autoregressive Video Diffusion" (arXiv 2605.30351), cited below as [VideoMLA]
with the section / equation / table of the paper.  The method reaches exactly
(up to rounding order) results that have plain definitions, so each function is
that definition written out in float64 with numpy; matrix products are the only
library primitive used.  Where the paper is silent, the reading taken is stated
in the docstring.

Parity status: every function below is pinned by tests under ``tests/`` that do
not re-type its formula (printed counts, closed forms, invariants, special cases
and a brute-force formulation with explicit rotation matrices).
"""
from __future__ import annotations

import math
from typing import Optional, Tuple

import numpy as np

# ---------------------------------------------------------------------------
# Cache-size accounting  ([VideoMLA] §3.1, App. C.1, App. E Eq. 13-14, Table 5a)
# ---------------------------------------------------------------------------


def latent_scalars_per_token(d_c: int, d_rope: int) -> int:
    """Scalars cached per token per layer: the latent c^KV plus the shared
    unrotated RoPE key k^R ([VideoMLA] §3.1 and App. E Eq. 13)."""
    return d_c + d_rope


def dense_scalars_per_token(n_heads: int, d_head: int) -> int:
    """Dense per-head K and V cache per token per layer: 2 n_h d_h
    ([VideoMLA] App. C.1 and App. E Eq. 14)."""
    return 2 * n_heads * d_head


def cache_scalars(layers: int, frames: int, tokens_per_frame: int, per_token: int) -> int:
    """Total cached scalars over a window of ``frames`` latent frames
    ([VideoMLA] App. C.1)."""
    return layers * frames * tokens_per_frame * per_token


def cache_bytes(scalars: int, bytes_per_scalar: int = 2) -> int:
    """Bytes of a bf16/fp16 cache ([VideoMLA] App. C.1)."""
    return scalars * bytes_per_scalar


# ---------------------------------------------------------------------------
# Decoupled 3D-RoPE  ([VideoMLA] §3.2 Eq. 5-6, App. D.3, App. E Eq. 12)
# ---------------------------------------------------------------------------


def rope_pair_split(d_rope: int) -> Tuple[int, int, int]:
    """Complex pairs given to the (t, h, w) axes.

    [VideoMLA] App. D.3 / Table 4 print (6, 5, 5) for d_rope = 32.  Reading for
    other widths: the h and w axes get floor(n/3) pairs each and t takes the
    rest (n = d_rope / 2), which reproduces (6, 5, 5).
    """
    if d_rope % 2:
        raise ValueError("d_rope must be even")
    n = d_rope // 2
    n_hw = n // 3
    return (n - 2 * n_hw, n_hw, n_hw)


def rope_frequencies(d_rope: int, d_head: int, base: float = 10000.0,
                     split: Optional[Tuple[int, int, int]] = None):
    """Per-pair angular frequency and axis of the decoupled 3D-RoPE.

    [VideoMLA] §3.2 and App. D.3 split the RoPE pairs over (t, h, w) "as in Wan",
    using the highest-frequency bands of each axis group.  Reading: an axis that
    would own D_a dims of a full d_head-dim head (same split rule applied to
    d_head / 2 pairs) has the frequency ladder base^(-2k / D_a), k = 0, 1, ...;
    the decoupled key keeps its first n_a (highest) frequencies.  Pairs are laid
    out t first, then h, then w.

    Returns (omega[n], axis[n]) with axis 0 = t, 1 = h, 2 = w.
    """
    n_t, n_h, n_w = split if split is not None else rope_pair_split(d_rope)
    if 2 * (n_t + n_h + n_w) != d_rope:
        raise ValueError("pair split does not cover d_rope")
    full = rope_pair_split(d_head)
    omegas, axes = [], []
    for a, (n_a, N_a) in enumerate(zip((n_t, n_h, n_w), full)):
        D_a = 2 * N_a
        for k in range(n_a):
            omegas.append(base ** (-2.0 * k / D_a))
            axes.append(a)
    return np.asarray(omegas, dtype=np.float64), np.asarray(axes, dtype=np.int64)


def rope_angles(pos: np.ndarray, omega: np.ndarray, axis: np.ndarray) -> np.ndarray:
    """Angle of every pair: theta_p = pos[axis(p)] * omega_p.

    ``pos`` is [..., 3] integer (t, h, w); result is [..., n_pairs]."""
    pos = np.asarray(pos, dtype=np.float64)
    return pos[..., axis] * omega


def rope_rotate(v: np.ndarray, theta: np.ndarray) -> np.ndarray:
    """Rotate adjacent pairs (2p, 2p+1) of ``v`` by ``theta[..., p]``:
    (x, y) -> (x cos - y sin, x sin + y cos)  (complex multiplication by
    exp(i theta)).  Reading: interleaved pair layout, same for q and k."""
    x = v[..., 0::2]
    y = v[..., 1::2]
    c, s = np.cos(theta), np.sin(theta)
    rx = x * c - y * s
    ry = x * s + y * c
    return np.stack([rx, ry], axis=-1).reshape(rx.shape[:-1] + (2 * rx.shape[-1],))


# ---------------------------------------------------------------------------
# Ring-buffer window and RoPE re-indexing  ([VideoMLA] App. D.4, D.5)
# ---------------------------------------------------------------------------


def token_grid_position(p: np.ndarray, grid_w: int) -> Tuple[np.ndarray, np.ndarray]:
    """Row-major (h, w) of token p inside a latent frame (reading: tokens of a
    frame are stored row-major over the patch grid)."""
    p = np.asarray(p, dtype=np.int64)
    return p // grid_w, p % grid_w


def window_keys(slots: int, oldest: int, n_valid: int, grid_h: int, grid_w: int, n_sink: int = 0):
    """Valid cache rows of the window in logical order, with their positions.

    The ring holds ``slots`` frames of T_f = grid_h * grid_w tokens; logical frame
    j (0 = oldest valid) lives in slot (oldest + j) mod slots.  [VideoMLA] App.
    D.5 gives the keys local temporal coordinates inside the current window:
    reading t = j.  Returns (rows[N], pos[N, 3]) with N = n_valid * T_f.

    With ``n_sink`` pinned sink frames ([VideoMLA] App. D.4: one sink latent frame
    plus a FIFO of the last frames) the cache rows are those of the sink frames,
    rows [0, n_sink T_f), followed by the ring, rows n_sink T_f + (slot T_f + p).
    The re-indexing of App. D.5 is read as: sink frame s at t = s, ring frame j at
    t = n_sink + j, so the sink sits at local t = 0 before the FIFO frames.
    """
    if not (1 <= n_valid <= slots and 0 <= oldest < slots and n_sink >= 0):
        raise ValueError("bad window")
    T_f = grid_h * grid_w
    j = np.repeat(np.arange(n_valid), T_f)
    p = np.tile(np.arange(T_f), n_valid)
    slot = (oldest + j) % slots
    rows = n_sink * T_f + slot * T_f + p
    t = n_sink + j
    if n_sink:
        s_frame = np.repeat(np.arange(n_sink), T_f)
        s_tok = np.tile(np.arange(T_f), n_sink)
        rows = np.concatenate([s_frame * T_f + s_tok, rows])
        t = np.concatenate([s_frame, t])
        p = np.concatenate([s_tok, p])
    h, w = token_grid_position(p, grid_w)
    return rows, np.stack([t, h, w], axis=-1)


def window_queries(n_valid: int, n_query: int, grid_h: int, grid_w: int, n_sink: int = 0) -> np.ndarray:
    """Positions of the query chunk: the newest ``n_query`` tokens of the window
    in logical order, in the same local frame as the keys ([VideoMLA] App. D.5:
    the current chunk is rotated in the same local coordinate system).  Sink
    frames come first in that frame (see ``window_keys``)."""
    T_f = grid_h * grid_w
    if not (1 <= n_query <= (n_sink + n_valid) * T_f):
        raise ValueError("bad query count")
    L = (n_sink + n_valid) * T_f - n_query + np.arange(n_query)
    h, w = token_grid_position(L % T_f, grid_w)
    return np.stack([L // T_f, h, w], axis=-1)


# ---------------------------------------------------------------------------
# cache_write  ([VideoMLA] §3.1 Eq. 1, §3.2 Eq. 5, App. D.2, App. D.4)
# ---------------------------------------------------------------------------


def rms_norm(v: np.ndarray, gamma: Optional[np.ndarray], eps: float) -> np.ndarray:
    """RMSNorm over the last axis: gamma * v / sqrt(mean(v^2) + eps)."""
    r = v / np.sqrt(np.mean(v * v, axis=-1, keepdims=True) + eps)
    return r if gamma is None else r * gamma


def cache_write(x: np.ndarray, W_dkv: np.ndarray, W_kr: np.ndarray,
                gamma: Optional[np.ndarray], eps: float, cache: np.ndarray,
                slots: int, first_slot: int, tokens_per_frame: int,
                normalize: bool = True) -> np.ndarray:
    """Project new tokens into the latent ring cache (in place; returns cache).

    c = W_dkv x  (Eq. 1) followed by RMSNorm ([VideoMLA] App. D.2: c^KV is
    RMS-normalised before the up-projections; reading: the normalised latent is
    what is cached), and the shared RoPE key k^R = W_kr x (Eq. 5), stored
    unrotated (§3.2).  Token t of the chunk goes to slot (first_slot + t // T_f)
    mod slots, row t mod T_f of that slot: the FIFO ring of App. D.4.

    x [B, n_tok, d], W_dkv [d_c, d], W_kr [d_rope, d], cache [B, slots*T_f,
    d_c + d_rope] float64.  ``normalize=False`` (gamma ignored) caches the raw
    down-projection.
    """
    B, n_tok, _ = x.shape
    d_c = W_dkv.shape[0]
    if n_tok % tokens_per_frame:
        raise ValueError("n_tok must be a whole number of frames")
    c = x @ W_dkv.T
    if normalize:
        c = rms_norm(c, gamma, eps)
    kr = x @ W_kr.T
    t = np.arange(n_tok)
    rows = ((first_slot + t // tokens_per_frame) % slots) * tokens_per_frame + t % tokens_per_frame
    cache[:, rows, :d_c] = c
    cache[:, rows, d_c:] = kr
    return cache


# ---------------------------------------------------------------------------
# Attention over the window
# ---------------------------------------------------------------------------


def _softmax_rows(s: np.ndarray):
    m = s.max(axis=-1, keepdims=True)
    e = np.exp(s - m)
    l = e.sum(axis=-1, keepdims=True)
    return e / l, (m + np.log(l))[..., 0]


def _prepare(q_nope, q_rope, W_uk, W_uv, cache, slots, oldest, n_valid,
             grid_h, grid_w, d_c, rope_base, pair_split, query_rows, n_sink):
    B, Nq, H, d_nope = q_nope.shape
    d_rope = q_rope.shape[-1]
    d_v = W_uv.shape[0] // H
    rows, kpos = window_keys(slots, oldest, n_valid, grid_h, grid_w, n_sink)
    qpos = window_queries(n_valid, Nq, grid_h, grid_w, n_sink)
    sel = np.arange(Nq) if query_rows is None else np.asarray(query_rows)
    omega, axis = rope_frequencies(d_rope, d_nope + d_rope, rope_base, pair_split)
    C = cache[:, rows, :d_c]                       # [B, N, d_c]
    k_rope = rope_rotate(cache[:, rows, d_c:], rope_angles(kpos, omega, axis))
    q_rot = rope_rotate(q_rope[:, sel], rope_angles(qpos[sel], omega, axis)[None, :, None, :])
    return B, H, d_nope, d_rope, d_v, sel, C, k_rope, q_rot


def attention_explicit(q_nope, q_rope, W_uk, W_uv, cache, slots, oldest, n_valid,
                       grid_h, grid_w, d_c, rope_base=10000.0, pair_split=None,
                       query_rows=None, return_probs=False, n_sink=0):
    """Training-time form ([VideoMLA] §3.3, Eq. 2, 6, 7; App. D.3-D.4).

    Per head h the keys and values are reconstructed from the cached latent:
    k^nope_{j,h} = W_uk,h c_j and v_{j,h} = W_uv,h c_j (Eq. 2; W_uk,h / W_uv,h
    are the h-th row blocks of W_uk [H d_nope, d_c] and W_uv [H d_v, d_c]); the
    shared key k^R_j and the query q^R_{i,h} are rotated by their window-local
    (t, h, w) positions (Eq. 5-6, App. D.5); the score is
    (q^nope . k^nope + q^rope . k^rope) / sqrt(d_nope + d_rope) (Eq. 7); a
    softmax over the whole active window (no mask inside the window) weights the
    values.  Returns out [B, nq, H, d_v] and lse [B, nq, H] (natural log of the
    softmax denominator of the scaled scores), optionally the probabilities.

    Query rows are independent, so ``query_rows`` picks a subset of them; rows
    are processed in blocks only to bound memory, with identical arithmetic.
    ``cache`` holds ``n_sink`` sink frames before the ring (see ``window_keys``).
    """
    B, H, d_nope, d_rope, d_v, sel, C, k_rope, q_rot = _prepare(
        q_nope, q_rope, W_uk, W_uv, cache, slots, oldest, n_valid, grid_h, grid_w,
        d_c, rope_base, pair_split, query_rows, n_sink)
    scale = 1.0 / math.sqrt(d_nope + d_rope)
    out = np.empty((B, len(sel), H, d_v))
    lse = np.empty((B, len(sel), H))
    probs = np.empty((B, H, len(sel), C.shape[1])) if return_probs else None
    for b in range(B):
        for h in range(H):
            K_nope = C[b] @ W_uk[h * d_nope:(h + 1) * d_nope].T      # [N, d_nope]
            V = C[b] @ W_uv[h * d_v:(h + 1) * d_v].T                  # [N, d_v]
            K = np.concatenate([K_nope, k_rope[b]], axis=-1)          # [N, 128]
            for i0 in range(0, len(sel), 1024):
                blk = slice(i0, i0 + 1024)
                Q = np.concatenate([q_nope[b, sel[blk], h], q_rot[b, blk, h]], axis=-1)
                P, l = _softmax_rows((Q @ K.T) * scale)
                out[b, blk, h] = P @ V
                lse[b, blk, h] = l
                if return_probs:
                    probs[b, h, blk] = P
    return (out, lse, probs) if return_probs else (out, lse)


def attention_absorbed(q_nope, q_rope, W_uk, W_uv, cache, slots, oldest, n_valid,
                       grid_h, grid_w, d_c, rope_base=10000.0, pair_split=None,
                       query_rows=None, n_sink=0):
    """Inference-time reparametrisation ([VideoMLA] App. E, Eq. 8-12).

    The key up-projection is absorbed into the query, q_abs = W_uk,h^T q^nope
    (Eq. 8-9 with the query-side up-projection already applied), so the content
    score is q_abs . c_j; the value up-projection is applied after the weighted
    sum over latents, o_h = W_uv,h (sum_j p_j c_j) (Eq. 10, without the output
    projection W_O); the RoPE term q^rope . k^rope is kept separate (Eq. 12).
    Same arguments and results as ``attention_explicit``.
    """
    B, H, d_nope, d_rope, d_v, sel, C, k_rope, q_rot = _prepare(
        q_nope, q_rope, W_uk, W_uv, cache, slots, oldest, n_valid, grid_h, grid_w,
        d_c, rope_base, pair_split, query_rows, n_sink)
    scale = 1.0 / math.sqrt(d_nope + d_rope)
    out = np.empty((B, len(sel), H, d_v))
    lse = np.empty((B, len(sel), H))
    for b in range(B):
        for h in range(H):
            W_uk_h = W_uk[h * d_nope:(h + 1) * d_nope]               # [d_nope, d_c]
            W_uv_h = W_uv[h * d_v:(h + 1) * d_v]                     # [d_v, d_c]
            for i0 in range(0, len(sel), 1024):
                blk = slice(i0, i0 + 1024)
                q_abs = q_nope[b, sel[blk], h] @ W_uk_h               # [nq, d_c]
                s = (q_abs @ C[b].T + q_rot[b, blk, h] @ k_rope[b].T) * scale
                P, l = _softmax_rows(s)
                out[b, blk, h] = (P @ C[b]) @ W_uv_h.T
                lse[b, blk, h] = l
    return out, lse


def composite_kv_operator(W_uk: np.ndarray, W_uv: np.ndarray, W_dkv: np.ndarray) -> np.ndarray:
    """M = [W_uk W_dkv ; W_uv W_dkv] ([VideoMLA] §5): the dense-equivalent
    key/value operator, of rank at most d_c by construction."""
    return np.concatenate([W_uk @ W_dkv, W_uv @ W_dkv], axis=0)


# ---------------------------------------------------------------------------
# query path and output projection  ([VideoMLA] §3.1 Eq. 3-4, §3.2 Eq. 6,
# App. D.2, App. E Eq. 10-11)
# ---------------------------------------------------------------------------


def query_projection(x: np.ndarray, W_dq: np.ndarray, gamma_q: Optional[np.ndarray], eps: float,
                     W_uq: np.ndarray, W_qr: np.ndarray, n_heads: int):
    """Per-head queries of new tokens x [..., d]: the query latent
    c^Q = W_dq x (Eq. 3, W_dq [d_q, d]), RMS-normalised before the
    up-projections (App. D.2), then q^nope_h = W_uq,h c^Q (Eq. 4,
    W_uq [H d_nope, d_q]) and the unrotated q^R_h = W_qr,h c^Q (Eq. 6 before
    RoPE3D, W_qr [H d_rope, d_q]); head h owns row block h of each matrix.
    Returns (q_nope [..., H, d_nope], q_rope [..., H, d_rope])."""
    c_q = rms_norm(x @ W_dq.T, gamma_q, eps)
    q_nope = c_q @ W_uq.T
    q_rope = c_q @ W_qr.T
    lead = x.shape[:-1]
    return (q_nope.reshape(*lead, n_heads, W_uq.shape[0] // n_heads),
            q_rope.reshape(*lead, n_heads, W_qr.shape[0] // n_heads))


def output_projection(o: np.ndarray, W_O: np.ndarray) -> np.ndarray:
    """Layer output y = sum_h W_O,h o_h for per-head outputs o [..., H, d_v]:
    W_O [d, H d_v] with column block h applied to head h (the output
    projection whose per-head slices Eq. 10-11 fold into B_h = W_O,h W_uv,h).
    Returns y [..., d]."""
    lead = o.shape[:-2]
    return o.reshape(*lead, -1) @ W_O.T
