"""GPU parity of the rank / RoPE allocation sweep at its own shape.

The sweep workload of [VideoMLA] App. F (Table 5(a) ranks, Table 5(b) RoPE
widths) runs a stack of independent layers, each a 3-frame chunk (4680 query
tokens on the 30 x 52 grid) against a 21-frame window (32,760 keys), for every
(d_c, d_rope) point.  Each case here is one layer of that stack at full size,
with the layer's own seed (1000 * 4 + 10 * layer):

* the 21-frame window's tokens go through the oracle's cache write; its bf16
  rounding is the cache both sides attend over, so attention parity excludes
  the cache's rounding;
* the GPU cache write of the newest 3-frame chunk (slots 18-20) is checked on
  every written row against the oracle, and untouched rows must stay bit-exact;
* the GPU attention of the 4680 queries runs in the launch configuration the
  benchmark times (the default workspace and split choice) and is compared on
  sampled query rows (all heads, all keys: each sampled row is exact).
"""
import numpy as np
import pytest
import torch

from mla_latent_kv_write_b200 import inputs as I
from mla_latent_kv_write_b200 import videomla as V
from tests.common import check_attention, check_cache, check_lse, f64, oracle_attention, oracle_cache, \
    sample_rows, to_bf16

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("layer", [0, 1])
@pytest.mark.parametrize("d_c,d_rope", I.SWEEP_POINTS)
def test_sweep_layer_full_shape(d_c, d_rope, layer):
    wl = I.sweep_workload(d_c, d_rope)
    dims = wl.dims
    T_f = dims.tokens_per_frame
    seed = I.seed_for(wl.index, layer)
    w = I.layer_weights(dims, seed, random_gamma=True)
    x = I.tokens(dims, wl.batch, wl.slots * T_f, seed + 1)
    q = I.queries(dims, wl.batch, wl.n_query, seed + 2)

    # oracle cache of the whole window: the prefill rows and the chunk's rows
    ref_cache = oracle_cache(dims, x, w, wl.slots, 0)
    cache_bf16 = to_bf16(ref_cache)

    # GPU cache write of the chunk into slots 18-20 of a cache holding the
    # oracle's prefill rows, and sentinel rows where the chunk goes
    chunk = slice(wl.prefill * T_f, wl.slots * T_f)
    start = cache_bf16.clone()
    start[:, chunk] = I.latent_cache(dims, wl.batch, wl.chunk, seed + 3)
    cache = start.to(DEV)
    wd = {k: t.to(DEV) for k, t in w.items()}
    V.cache_write(x[:, chunk].contiguous().to(DEV), wd["W_dkv"], wd["W_kr"], wd["gamma"], cache, dims,
                  wl.slots, wl.prefill)
    torch.cuda.synchronize()
    assert V.device_status(reset=True) == V.OK
    got_cache = f64(cache.cpu())
    check_cache(got_cache[:, chunk], ref_cache[:, chunk], d_c, f"sweep ({d_c},{d_rope}) layer {layer} chunk")
    assert np.array_equal(got_cache[:, :chunk.start], f64(start)[:, :chunk.start]), "prefill rows were modified"
    del got_cache, ref_cache

    # attention of the chunk's queries over the window (the oracle's bf16 cache)
    qd = {k: t.to(DEV) for k, t in q.items()}
    out, lse = V.attention(qd["q_nope"], qd["q_rope"], wd["W_uk"], wd["W_uv"], cache_bf16.to(DEV), dims,
                           wl.slots, 0, wl.slots, want_lse=True)
    torch.cuda.synchronize()
    assert V.device_status(reset=True) == V.OK
    rows = sample_rows(wl.n_query, 40, seed=700 + 10 * layer + d_rope)
    ref_out, ref_lse = oracle_attention(dims, q, w, cache_bf16, wl.slots, 0, wl.slots, rows)
    got_out, got_lse = f64(out.cpu())[:, rows], f64(lse.cpu())[:, rows]
    what = f"sweep ({d_c},{d_rope}) layer {layer} attention"
    rms_rel, max_abs = check_attention(got_out, ref_out, what)
    lse_err = check_lse(got_lse, ref_lse, what + " lse")
    print(f"\n{what}: rms rel {rms_rel:.2e} max abs {max_abs:.2e} lse {lse_err:.2e} ({len(rows)} rows)")
