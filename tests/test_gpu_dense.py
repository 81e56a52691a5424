"""GPU parity of the dense multi-head attention baseline (VideoMLA App. C.1).

The dense cache holds, for every key and head, k_h = [W_uk,h c | RoPE3D(k^R)] and
v_h = W_uv,h c.  Built here from a latent ring window with the oracle's own
window, RoPE and projection pieces (fp64, then rounded to bf16 as a dense bf16
cache would be), the dense kernel must reproduce the oracle's explicit form
(Sec. 3.3) on the latent cache: the same attention, up to the bf16 rounding of
the reconstructed keys and values.  Same tolerance as the latent kernel.
"""
import dataclasses

import numpy as np
import pytest
import torch

from mla_latent_kv_write_b200 import inputs as I
from mla_latent_kv_write_b200 import videomla as V
from oracle import videomla_oracle as O
from tests.common import check_attention, f64, sample_rows, to_bf16

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _dense_kv(dims, w, cache, slots, oldest, n_valid):
    """Per-head keys and values of the window in logical order, [B, N, H, 128]."""
    rows, kpos = O.window_keys(slots, oldest, n_valid, dims.grid_h, dims.grid_w)
    omega, axis = O.rope_frequencies(dims.d_rope, dims.d_nope + dims.d_rope, dims.rope_base, dims.pairs)
    c = f64(cache)[:, rows]
    C, kr = c[..., :dims.d_c], O.rope_rotate(c[..., dims.d_c:], O.rope_angles(kpos, omega, axis))
    H = dims.n_heads
    W_uk = f64(w["W_uk"]).reshape(H, dims.d_nope, dims.d_c)
    W_uv = f64(w["W_uv"]).reshape(H, dims.d_v, dims.d_c)
    k_nope = np.einsum("bnc,hdc->bnhd", C, W_uk)
    k = np.concatenate([k_nope, np.broadcast_to(kr[:, :, None, :], k_nope.shape[:3] + (dims.d_rope,))], axis=-1)
    v = np.einsum("bnc,hdc->bnhd", C, W_uv)
    return to_bf16(np.ascontiguousarray(k)), to_bf16(np.ascontiguousarray(v))


def _case(dims, B, slots, oldest, n_valid, Nq, seed, rows=None):
    w = I.layer_weights(dims, seed)
    q = I.queries(dims, B, Nq, seed + 1)
    cache = I.latent_cache(dims, B, slots, seed + 2)
    k, v = _dense_kv(dims, w, cache, slots, oldest, n_valid)
    out = V.dense_attention(q["q_nope"].to(DEV), q["q_rope"].to(DEV), k.to(DEV), v.to(DEV), dims)
    torch.cuda.synchronize()
    assert V.device_status(reset=True) == V.OK
    ref, _ = O.attention_explicit(f64(q["q_nope"]), f64(q["q_rope"]), f64(w["W_uk"]), f64(w["W_uv"]), f64(cache),
                                  slots, oldest, n_valid, dims.grid_h, dims.grid_w, dims.d_c, dims.rope_base,
                                  dims.pairs, query_rows=rows)
    got = f64(out.cpu())
    if rows is not None:
        got = got[:, rows]
    rms_rel, max_abs = check_attention(got, ref, f"dense {dims.d_nope}/{dims.d_rope} B={B} Nq={Nq}")
    print(f"\ndense {dims.d_nope}/{dims.d_rope} B={B} n_valid={n_valid} Nq={Nq}: rms rel {rms_rel:.2e} "
          f"max abs {max_abs:.2e}")


@pytest.mark.parametrize("d_c,d_rope", [(192, 32), (192, 16), (192, 64)])
def test_dense_attention_tiny_wrapped_window(d_c, d_rope):
    # 6 x 8 grid, ring of 5 slots wrapped (oldest 3), 4 valid frames = 192 keys
    # (a full and a ragged key tile), 100 queries (a ragged query tile), batch 2
    dims = dataclasses.replace(I.sweep_dims(d_c, d_rope), grid_h=6, grid_w=8)
    _case(dims, B=2, slots=5, oldest=3, n_valid=4, Nq=100, seed=5100 + d_rope)


def test_dense_attention_wan_layer_sampled_rows():
    # the Wan-1.3B layer: 4680 queries over the 21-frame window (32760 keys)
    rows = sample_rows(4680, 48, seed=51)
    _case(I.WAN, B=1, slots=21, oldest=0, n_valid=21, Nq=4680, seed=5200, rows=rows)
