"""GPU parity of the sm_100a kernels against the fp64 oracle, through the C ABI.

Sizes: the tiny 6 x 8 grid (several key tiles, ragged tails, two-run ring
windows, ragged query counts, batch 2) checked element by element, and the
Wan-1.3B-shaped workloads at full size checked on sampled query rows (rows are
independent, so each sampled row is exact) with every head and every key.
"""
import dataclasses

import numpy as np
import pytest
import torch

from mla_latent_kv_write_b200 import inputs as I
from mla_latent_kv_write_b200 import videomla as V
from oracle import videomla_oracle as O
from tests.common import (check_attention, check_cache, check_lse, f64, oracle_attention, oracle_cache,
                          sample_rows, to_bf16)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _dev(d):
    return {k: v.to(DEV) for k, v in d.items()}


def _attention_case(dims, B, slots, oldest, n_valid, Nq, seed, rows=None, rope_scale=1.0, n_sink=0,
                    tiling=V.TILING_AUTO):
    w = I.layer_weights(dims, seed)
    q = I.queries(dims, B, Nq, seed + 1)
    cache = I.latent_cache(dims, B, slots, seed + 2, rope_scale=rope_scale)
    sink = I.latent_cache(dims, B, n_sink, seed + 3, rope_scale=rope_scale) if n_sink else None
    wd, qd = _dev(w), _dev(q)
    with V.attention_tiling(tiling):
        out, lse = V.attention(qd["q_nope"], qd["q_rope"], wd["W_uk"], wd["W_uv"], cache.to(DEV), dims,
                               slots, oldest, n_valid, want_lse=True, sink=None if sink is None else sink.to(DEV))
    torch.cuda.synchronize()
    assert V.device_status(reset=True) == V.OK
    ref_out, ref_lse = oracle_attention(dims, q, w, cache, slots, oldest, n_valid, rows, sink_bf16=sink)
    got_out, got_lse = f64(out.cpu()), f64(lse.cpu())
    if rows is not None:
        got_out, got_lse = got_out[:, rows], got_lse[:, rows]
    what = (f"attention {dims.d_c}/{dims.d_rope} B={B} slots={slots} oldest={oldest} n_valid={n_valid} Nq={Nq}"
            f"{f' sink={n_sink}' if n_sink else ''}")
    err = got_out - ref_out
    print(f"\n{what}: rms rel {np.linalg.norm(err) / np.linalg.norm(ref_out):.2e} "
          f"max abs {np.max(np.abs(err)):.2e} lse {np.max(np.abs(got_lse - ref_lse)):.2e}")
    check_attention(got_out, ref_out, what)
    check_lse(got_lse, ref_lse, "lse")


# ---------------------------------------------------------------------------
# attention
# ---------------------------------------------------------------------------

def test_attention_tiny_config():
    # 6 x 8 grid, 1 query frame vs a 3-frame window (144 keys: one full and one ragged tile)
    _attention_case(I.TINY, B=1, slots=3, oldest=0, n_valid=3, Nq=48, seed=11)


@pytest.mark.parametrize("slots,oldest,n_valid,Nq,B", [
    (7, 4, 5, 100, 2),    # ring wraps: two runs of rows, ragged tiles in both, ragged query tile
    (7, 0, 7, 336, 1),    # full window, 3 query tiles with a ragged one
    (5, 2, 1, 48, 1),     # a single valid frame
    (6, 5, 6, 129, 2),    # full window starting at the last slot, 2 query tiles (second has 1 row)
    (3, 1, 2, 96, 1),     # window not yet full, contiguous run that does not start at slot 0
])
def test_attention_ragged_windows(slots, oldest, n_valid, Nq, B):
    _attention_case(I.TINY, B=B, slots=slots, oldest=oldest, n_valid=n_valid, Nq=Nq, seed=13 + slots + oldest)


def test_attention_wan_layer_sampled_rows():
    # 4680 queries x 32760 keys, 12 heads, every output computed on the GPU
    dims = I.WAN
    rows = sample_rows(4680, 96, seed=5)
    _attention_case(dims, B=1, slots=21, oldest=0, n_valid=21, Nq=4680, seed=1001, rows=rows)


def test_attention_wan_wrapped_window_sampled_rows():
    dims = I.WAN
    rows = sample_rows(1560, 48, seed=6)
    _attention_case(dims, B=1, slots=21, oldest=13, n_valid=21, Nq=1560, seed=1002, rows=rows)


@pytest.mark.parametrize("d_c,d_rope", [(96, 32), (192, 16), (192, 64), (384, 32)])
def test_attention_sweep_points(d_c, d_rope):
    dims = dataclasses.replace(I.sweep_dims(d_c, d_rope), grid_h=6, grid_w=8)
    seed = 4000 + d_rope + (0 if d_c == 192 else d_c)
    _attention_case(dims, B=2, slots=5, oldest=3, n_valid=4, Nq=150, seed=seed)


@pytest.mark.parametrize("slots,oldest,n_valid,Nq,B", [
    (6, 4, 6, 144, 2),    # sink + full wrapping FIFO: three runs of key rows, ragged tiles
    (6, 0, 2, 96, 1),     # sink + FIFO not yet full
    (4, 3, 3, 192, 1),    # queries reach back into the sink frame
])
def test_attention_sink_window(slots, oldest, n_valid, Nq, B):
    _attention_case(I.TINY, B=B, slots=slots, oldest=oldest, n_valid=n_valid, Nq=Nq, seed=21 + slots + oldest,
                    n_sink=1)


def test_attention_sink_window_q_in_shared_memory():
    dims = dataclasses.replace(I.sweep_dims(384, 32), grid_h=6, grid_w=8)
    _attention_case(dims, B=2, slots=4, oldest=1, n_valid=4, Nq=96, seed=4500, n_sink=1)


def test_attention_wan_sink_plus_six_frames_sampled_rows():
    """The pages' inference cache: one sink latent frame plus a FIFO of six
    (10,920 keys), the 3-frame chunk as queries, a wrapped FIFO."""
    rows = sample_rows(4680, 64, seed=7)
    _attention_case(I.WAN, B=1, slots=6, oldest=2, n_valid=6, Nq=4680, seed=1003, rows=rows, n_sink=1)


def test_attention_peaky_scores():
    # rope keys scaled x8 make scores peaky (std ~ 4): online-softmax rescaling is exercised
    _attention_case(I.TINY, B=1, slots=7, oldest=2, n_valid=7, Nq=200, seed=17, rope_scale=8.0)


def test_attention_long_window_peaky_tokens():
    """Minute-scale workload: batch 2, 63-frame ring (98280 keys), 4680 queries;
    1% of the tokens of x scaled x8 before the (oracle) cache write, so their
    unnormalised rope keys make scores peaky.  Sampled rows, all heads / keys."""
    wl = I.WORKLOADS["long"]
    dims = wl.dims
    T_f = dims.tokens_per_frame
    seed = I.seed_for(wl.index)
    w = I.layer_weights(dims, seed)
    x = I.tokens(dims, wl.batch, wl.slots * T_f, seed + 3, wl.peaky_fraction, wl.peaky_scale)
    cache = to_bf16(oracle_cache(dims, x, w, wl.slots, 0))
    del x
    q = I.queries(dims, wl.batch, wl.n_query, seed + 5)
    wd, qd = _dev(w), _dev(q)
    out = V.attention(qd["q_nope"], qd["q_rope"], wd["W_uk"], wd["W_uv"], cache.to(DEV), dims, wl.slots, 0, wl.slots)
    torch.cuda.synchronize()
    assert V.device_status(reset=True) == V.OK
    rows = sample_rows(wl.n_query, 24, seed=7)
    ref, _ = oracle_attention(dims, q, w, cache, wl.slots, 0, wl.slots, rows)
    rms_rel, max_abs = check_attention(f64(out.cpu())[:, rows], ref, "long window")
    print(f"\nlong window: rms rel {rms_rel:.2e} max abs {max_abs:.2e}")


# ---------------------------------------------------------------------------
# cache_write
# ---------------------------------------------------------------------------

def _cache_write_case(dims, B, frames, slots, first_slot, seed, raw=False):
    w = I.layer_weights(dims, seed, random_gamma=True)
    x = I.tokens(dims, B, frames * dims.tokens_per_frame, seed + 1)
    sentinel = I.latent_cache(dims, B, slots, seed + 2)
    cache = sentinel.clone().to(DEV)
    wd = _dev(w)
    V.cache_write(x.to(DEV), wd["W_dkv"], wd["W_kr"], wd["gamma"], cache, dims, slots, first_slot, raw_latent=raw)
    torch.cuda.synchronize()
    assert V.device_status(reset=True) == V.OK
    ref = oracle_cache(dims, x, w, slots, first_slot, base=f64(sentinel), normalize=not raw)
    got = f64(cache.cpu())
    T_f = dims.tokens_per_frame
    written = np.zeros(slots, dtype=bool)
    for f in range(frames):
        written[(first_slot + f) % slots] = True
    for s in range(slots):
        sl = slice(s * T_f, (s + 1) * T_f)
        if written[s]:
            check_cache(got[:, sl], ref[:, sl], dims.d_c, f"slot {s}")
        else:
            assert np.array_equal(got[:, sl], f64(sentinel)[:, sl]), f"slot {s} was modified"


def test_cache_write_tiny_wraps_ring():
    _cache_write_case(I.TINY, B=2, frames=2, slots=3, first_slot=2, seed=21)


def test_cache_write_wan_chunk():
    # 3 frames = 4680 tokens: 36 full token tiles and a ragged one, into slots 18-20
    _cache_write_case(I.WAN, B=1, frames=3, slots=21, first_slot=18, seed=22)


def test_cache_write_raw_latent():
    _cache_write_case(I.TINY, B=1, frames=3, slots=4, first_slot=1, seed=23, raw=True)


def test_cache_write_one_frame_chunk():
    """One Wan frame (13 token tiles, the last ragged) into the last slot of the
    ring: the cluster kernel with its widest K split, written twice in a row."""
    dims, B, slots, first = I.WAN, 1, 21, 20
    T_f = dims.tokens_per_frame
    w = I.layer_weights(dims, 25, random_gamma=True)
    x = I.tokens(dims, B, T_f, 26)
    sentinel = I.latent_cache(dims, B, slots, 27)
    cache = sentinel.clone().to(DEV)
    wd = _dev(w)
    for _ in range(2):
        V.cache_write(x.to(DEV), wd["W_dkv"], wd["W_kr"], wd["gamma"], cache, dims, slots, first)
    torch.cuda.synchronize()
    assert V.device_status(reset=True) == V.OK
    ref = oracle_cache(dims, x, w, slots, first, base=f64(sentinel))
    got = f64(cache.cpu())
    sl = slice(first * T_f, (first + 1) * T_f)
    check_cache(got[:, sl], ref[:, sl], dims.d_c, "one frame")
    assert np.array_equal(got[:, :sl.start], f64(sentinel)[:, :sl.start])


def test_cache_write_persistent_rounds():
    """Batch 2 x 12 frames = 294 token tiles: the stream kernel, each CTA of the
    persistent grid taking two tiles, the second one's MMAs running into the other
    tensor-memory accumulator while the first one's rows are normalised and stored."""
    dims, B, frames, slots, first = I.WAN, 2, 12, 21, 15
    _cache_write_case(dims, B=B, frames=frames, slots=slots, first_slot=first, seed=28)


@pytest.mark.parametrize("d_c,d_rope", I.SWEEP_POINTS)
def test_cache_write_stream_kernel_sweep_points(d_c, d_rope):
    """Every (d_c, d_rope) point through the stream kernel: batch 2 x 5 Wan frames
    (122 tiles), ring wrapping; d_c = 384 has one tensor-memory accumulator."""
    dims = I.sweep_dims(d_c, d_rope)
    _cache_write_case(dims, B=2, frames=5, slots=7, first_slot=4, seed=29 + d_c + d_rope)


@pytest.mark.parametrize("d_c,d_rope", I.SWEEP_POINTS)
def test_cache_write_sweep_points(d_c, d_rope):
    dims = dataclasses.replace(I.sweep_dims(d_c, d_rope), grid_h=6, grid_w=8)
    _cache_write_case(dims, B=1, frames=3, slots=5, first_slot=4, seed=24 + d_c + d_rope)


# ---------------------------------------------------------------------------
# the whole path: rolling ring of 40 frame steps
# ---------------------------------------------------------------------------

def test_rolling_chain_40_steps():
    """Frame-by-frame rollout on a 21-slot ring of 30 x 52 frames: each step writes
    one frame (GPU cache_write) then attends 1560 queries over the window (GPU
    attention); the oracle runs the same chain with its own fp64 cache rounded
    to bf16.  Outputs are compared on sampled rows at every step."""
    wl = I.WORKLOADS["rolling"]
    dims = wl.dims
    T_f = dims.tokens_per_frame
    w = I.layer_weights(dims, I.seed_for(wl.index))
    wd = _dev(w)
    cache = torch.zeros(1, wl.slots * T_f, dims.cache_width, dtype=torch.bfloat16, device=DEV)
    ref_cache = np.zeros((1, wl.slots * T_f, dims.cache_width))
    for step in range(wl.steps):
        rw = I.rolling_window(step, wl.slots)
        x = I.tokens(dims, 1, T_f, I.seed_for(wl.index, 0, 100 + step))
        q = I.queries(dims, 1, T_f, I.seed_for(wl.index, 0, 200 + step))
        V.cache_write(x.to(DEV), wd["W_dkv"], wd["W_kr"], wd["gamma"], cache, dims, wl.slots, rw["write_slot"])
        qd = _dev(q)
        out = V.attention(qd["q_nope"], qd["q_rope"], wd["W_uk"], wd["W_uv"], cache, dims, wl.slots,
                          rw["oldest"], rw["n_valid"])
        oracle_cache(dims, x, w, wl.slots, rw["write_slot"], base=ref_cache)
        rows = sample_rows(T_f, 12, seed=step)
        ref_out, _ = oracle_attention(dims, q, w, to_bf16(ref_cache), wl.slots, rw["oldest"], rw["n_valid"], rows)
        check_attention(f64(out.cpu())[:, rows], ref_out, f"step {step}")
    assert V.device_status(reset=True) == V.OK


# ---------------------------------------------------------------------------
# query path, output projection and the whole layer ([VideoMLA] Eq. 3-4, 6,
# App. D.2, Eq. 10-11)
# ---------------------------------------------------------------------------

# Tolerances, from the bf16 roundings on each path.  Round-to-nearest to bf16
# (8 significant bits) leaves a relative error uniform in +-ulp/2 with ulp/|v|
# between 2^-8 and 2^-7, i.e. an RMS relative error of 2^-7 / sqrt(24) = 1.6e-3
# per rounding of values spread over a binade; independent roundings add in
# quadrature.  The fp32 accumulations add nothing visible at this scale.
#   q_nope, q_rope: two roundings (the normalised query latent, then q itself):
#     sqrt(2) * 1.6e-3 = 2.3e-3; bound 4e-3.
#   y = W_O o: one rounding of y (o is an exact bf16 input): 1.6e-3; bound 3e-3.
#   whole layer: q (2.3e-3), the cached latent (1.6e-3), the attention output
#     (its own bound, 5e-3) and y (1.6e-3) in quadrature: 5.9e-3; bound 8e-3.
BF16_RMS_REL = 2.0 ** -7 / 24 ** 0.5
Q_NORM_REL, Y_NORM_REL = 4e-3, 3e-3
LAYER_NORM_REL = 8e-3
assert Q_NORM_REL > 2 ** 0.5 * BF16_RMS_REL and Y_NORM_REL > BF16_RMS_REL
assert LAYER_NORM_REL > (2 * BF16_RMS_REL ** 2 + BF16_RMS_REL ** 2 + 5e-3 ** 2 + BF16_RMS_REL ** 2) ** 0.5


def _norm_rel(got, ref):
    return float(np.linalg.norm(got - ref) / np.linalg.norm(ref))


@pytest.mark.parametrize("dims,n_tok,B,rows,unit_gain", [
    (I.TINY, 144, 2, None, False),
    (I.TINY, 144, 1, None, True),     # gamma_q = NULL: the GEMM epilogue applies no column gain
    (I.WAN, 4680, 1, "sample", False),
])
def test_query_projection(dims, n_tok, B, rows, unit_gain):
    pw = I.projection_weights(dims, 610, random_gamma=not unit_gain)
    x = I.tokens(dims, B, n_tok, 611)
    d = _dev(pw)
    qn, qr = V.query_projection(x.to(DEV), d["W_dq"], None if unit_gain else d["gamma_q"], d["W_uq"], d["W_qr"],
                                dims)
    torch.cuda.synchronize()
    assert V.device_status(reset=True) == V.OK
    sel = np.arange(n_tok) if rows is None else sample_rows(n_tok, 64, seed=612)
    xs = f64(x)[:, sel]
    ref_n, ref_r = O.query_projection(xs, f64(pw["W_dq"]), f64(pw["gamma_q"]), dims.rms_eps, f64(pw["W_uq"]),
                                      f64(pw["W_qr"]), dims.n_heads)
    got_n, got_r = f64(qn.cpu())[:, sel], f64(qr.cpu())[:, sel]
    en, er = _norm_rel(got_n, ref_n), _norm_rel(got_r, ref_r)
    print(f"\nquery projection n_tok={n_tok} B={B}: q_nope rel {en:.2e} q_rope rel {er:.2e}")
    assert en <= Q_NORM_REL and er <= Q_NORM_REL


@pytest.mark.parametrize("n_tok", [144, 4680])
def test_query_projection_deterministic(n_tok):
    """Each row's sum of squares is stored per column tile and added in tile
    order, so repeated calls give bitwise-equal queries (both column-tile widths:
    288 rows take 128-wide tiles, 4680 rows 256-wide ones)."""
    dims = I.TINY if n_tok == 144 else I.WAN
    B = 2 if n_tok == 144 else 1
    pw = I.projection_weights(dims, 615, random_gamma=True)
    x = I.tokens(dims, B, n_tok, 616).to(DEV)
    d = _dev(pw)
    runs = [V.query_projection(x, d["W_dq"], d["gamma_q"], d["W_uq"], d["W_qr"], dims) for _ in range(3)]
    torch.cuda.synchronize()
    assert V.device_status(reset=True) == V.OK
    for qn, qr in runs[1:]:
        assert torch.equal(qn, runs[0][0]) and torch.equal(qr, runs[0][1])


def test_output_projection():
    dims = I.WAN
    pw = I.projection_weights(dims, 620)
    g = torch.Generator().manual_seed(621)
    o = torch.randn(1, 4680, dims.n_heads, dims.d_v, generator=g).to(torch.bfloat16)
    y = V.output_projection(o.to(DEV), pw["W_O"].to(DEV), dims)
    torch.cuda.synchronize()
    sel = sample_rows(4680, 64, seed=622)
    ref = O.output_projection(f64(o)[:, sel], f64(pw["W_O"]))
    e = _norm_rel(f64(y.cpu())[:, sel], ref)
    print(f"\noutput projection: rel {e:.2e}")
    assert e <= Y_NORM_REL


def test_layer_chain_tiny():
    """One attention layer step: new chunk x -> cache write and query path ->
    latent attention over the window -> output projection, against the
    oracle's fp64 chain on the same bf16 inputs."""
    dims, B, slots, first, n_new = I.TINY, 2, 5, 3, 2
    T_f = dims.tokens_per_frame
    w = I.layer_weights(dims, 630, random_gamma=True)
    pw = I.projection_weights(dims, 631, random_gamma=True)
    cache0 = I.latent_cache(dims, B, slots, 632)
    x = I.tokens(dims, B, n_new * T_f, 633)
    wd, pd = _dev(w), _dev(pw)
    cache = cache0.to(DEV).clone()
    xd = x.to(DEV)
    V.cache_write(xd, wd["W_dkv"], wd["W_kr"], wd["gamma"], cache, dims, slots, first)
    qn, qr = V.query_projection(xd, pd["W_dq"], pd["gamma_q"], pd["W_uq"], pd["W_qr"], dims)
    oldest = (first + n_new) % slots   # window full after the write: oldest = slot after the newest frame
    o = V.attention(qn, qr, wd["W_uk"], wd["W_uv"], cache, dims, slots, oldest, slots)
    y = V.output_projection(o, pd["W_O"], dims)
    torch.cuda.synchronize()
    assert V.device_status(reset=True) == V.OK
    ref_cache = oracle_cache(dims, x, w, slots, first, base=f64(cache0).copy())
    ref_qn, ref_qr = O.query_projection(f64(x), f64(pw["W_dq"]), f64(pw["gamma_q"]), dims.rms_eps,
                                        f64(pw["W_uq"]), f64(pw["W_qr"]), dims.n_heads)
    ref_o, _ = O.attention_absorbed(ref_qn, ref_qr, f64(w["W_uk"]), f64(w["W_uv"]), ref_cache, slots, oldest, slots,
                                    dims.grid_h, dims.grid_w, dims.d_c, dims.rope_base, dims.pairs)
    ref_y = O.output_projection(ref_o, f64(pw["W_O"]))
    e = _norm_rel(f64(y.cpu()), ref_y)
    print(f"\nlayer chain tiny: y rel {e:.2e}")
    assert e <= LAYER_NORM_REL


# ---------------------------------------------------------------------------
# split-KV: 1560 queries x 12 heads = 156 units do not fill 148 SMs in whole
# waves, so the key tiles of each unit are shared by several CTAs
# ---------------------------------------------------------------------------

# (per-head tiles forced: left to itself the library runs these shapes on
# head-packed tiles, tested below)

def test_attention_split_kv_sink_window_sampled_rows():
    rows = sample_rows(1560, 48, seed=8)
    _attention_case(I.WAN, B=1, slots=6, oldest=4, n_valid=6, Nq=1560, seed=1004, rows=rows, n_sink=1,
                    tiling=V.TILING_PER_HEAD)


def test_attention_split_kv_matches_unsplit_call():
    """The same call with a workspace too small for any split partials (one CTA
    per unit) and with the default one (split): both against the oracle."""
    dims, slots, oldest, Nq = I.WAN, 21, 7, 1560
    assert V.workspace_size(dims, slots, oldest, slots, 1, n_query=Nq) > V.workspace_size(dims, slots, oldest, slots, 1)
    w = I.layer_weights(dims, 1005)
    q = I.queries(dims, 1, Nq, 1006)
    cache = I.latent_cache(dims, 1, slots, 1007)
    wd, qd, cd = _dev(w), _dev(q), cache.to(DEV)
    small = torch.empty(V.workspace_size(dims, slots, oldest, slots, 1), dtype=torch.uint8, device=DEV)
    with V.attention_tiling(V.TILING_PER_HEAD):
        o1, l1 = V.attention(qd["q_nope"], qd["q_rope"], wd["W_uk"], wd["W_uv"], cd, dims, slots, oldest, slots,
                             want_lse=True, workspace=small)
        o2, l2 = V.attention(qd["q_nope"], qd["q_rope"], wd["W_uk"], wd["W_uv"], cd, dims, slots, oldest, slots,
                             want_lse=True)
    torch.cuda.synchronize()
    assert V.device_status(reset=True) == V.OK
    rows = sample_rows(Nq, 32, seed=9)
    ref_out, ref_lse = oracle_attention(dims, q, w, cache, slots, oldest, slots, rows)
    for o, l, what in ((o1, l1, "unsplit"), (o2, l2, "split")):
        got, got_l = f64(o.cpu())[:, rows], f64(l.cpu())[:, rows]
        check_attention(got, ref_out, f"split-KV {what}")
        check_lse(got_l, ref_lse, f"split-KV {what} lse")
    d = np.max(np.abs(f64(o1.cpu()) - f64(o2.cpu())))
    print(f"\nsplit vs unsplit: max abs diff {d:.2e}")


def test_attention_split_kv_batch_two_sampled_rows():
    """1560 queries x 12 heads x batch 2 = 312 units: split over 4 CTAs, so the
    grid's z index carries both the batch element and the split."""
    rows = sample_rows(1560, 24, seed=10)
    _attention_case(I.WAN, B=2, slots=21, oldest=20, n_valid=21, Nq=1560, seed=1008, rows=rows,
                    tiling=V.TILING_PER_HEAD)


def test_attention_split_kv_q_in_shared_memory():
    """d_c = 384 (Q in shared memory, 64-key tiles, two N = 192 MMA halves) with
    1560 queries: split-KV merge over the wide latent."""
    dims = I.sweep_dims(384, 32)
    rows = sample_rows(1560, 24, seed=11)
    _attention_case(dims, B=1, slots=21, oldest=3, n_valid=21, Nq=1560, seed=1009, rows=rows)


# ---------------------------------------------------------------------------
# head-packed tiles: a CTA takes 128 consecutive rows of the head-major (head,
# query) order, so a tile may end with the first queries of the next head
# ("mixed"): its q_abs comes from two accumulated MMAs over zero-padded q_nope
# boxes, its output from a second W_uv MMA into other tensor-memory columns
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("slots,oldest,n_valid,Nq,B,n_sink", [
    (7, 4, 5, 200, 2, 0),   # 19 tiles per batch element, 11 of them mixed; wrapped ring, ragged key tiles
    (7, 0, 7, 130, 1, 0),   # each head's last 2 queries start a tile; 13 tiles
    (5, 2, 3, 144, 2, 0),   # 144 keys, two key tiles: the W_uv load is the first to reuse a q_nope / W_uk stage
    (6, 4, 6, 144, 1, 1),   # sink frame + wrapping FIFO: three runs of key rows
    (7, 3, 7, 336, 1, 0),   # 32 tiles, the last one ragged (the last head's rows end inside it)
])
def test_attention_head_packed_tiles(slots, oldest, n_valid, Nq, B, n_sink):
    _attention_case(I.TINY, B=B, slots=slots, oldest=oldest, n_valid=n_valid, Nq=Nq, seed=6100 + Nq + slots,
                    n_sink=n_sink, tiling=V.TILING_HEAD_PACKED)


@pytest.mark.parametrize("d_c,d_rope", [(96, 32), (192, 16), (192, 64)])
def test_attention_head_packed_sweep_points(d_c, d_rope):
    # d_c = 96: the second head's output sits in the P / Q columns (O is narrower
    # than d_v); (192, 64): 3 ring stages
    dims = dataclasses.replace(I.sweep_dims(d_c, d_rope), grid_h=6, grid_w=8)
    _attention_case(dims, B=2, slots=5, oldest=3, n_valid=4, Nq=150, seed=6300 + d_c + d_rope,
                    tiling=V.TILING_HEAD_PACKED)


def test_attention_rolling_shape_head_packed_sampled_rows():
    """The rolling step's attention: 1560 queries x 12 heads over the full
    21-frame ring, which the library runs on 147 head-packed CTAs (one wave)."""
    rows = sample_rows(1560, 48, seed=12)
    _attention_case(I.WAN, B=1, slots=21, oldest=5, n_valid=21, Nq=1560, seed=6400, rows=rows)


@pytest.mark.parametrize("dims,slots,oldest,n_valid,Nq,B", [
    (I.TINY, 7, 4, 5, 200, 2),
    (I.WAN, 21, 0, 21, 1560, 1),
])
def test_attention_head_packed_equals_per_head(dims, slots, oldest, n_valid, Nq, B):
    """A row's arithmetic does not depend on the tile that holds it: head-packed
    and unsplit per-head tiles give the same bits (the per-head call gets a
    workspace with no room for split-KV partials)."""
    w = _dev(I.layer_weights(dims, 6500))
    q = _dev(I.queries(dims, B, Nq, 6501))
    cache = I.latent_cache(dims, B, slots, 6502).to(DEV)
    small = torch.empty(V.workspace_size(dims, slots, oldest, n_valid, B), dtype=torch.uint8, device=DEV)
    outs = []
    for mode in (V.TILING_PER_HEAD, V.TILING_HEAD_PACKED):
        with V.attention_tiling(mode):
            outs.append(V.attention(q["q_nope"], q["q_rope"], w["W_uk"], w["W_uv"], cache, dims, slots, oldest,
                                    n_valid, want_lse=True, workspace=small))
    torch.cuda.synchronize()
    assert V.device_status(reset=True) == V.OK
    (o1, l1), (o2, l2) = outs
    assert torch.equal(o1, o2)
    assert torch.equal(l1, l2)


# ---------------------------------------------------------------------------
# d_c = 96: two softmax groups on alternate key tiles, each with its own S
# buffer, O accumulator and running (max, sum), merged at the end
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("slots,oldest,n_valid,Nq,B,n_sink,rope_scale", [
    (5, 2, 1, 48, 1, 0, 1.0),    # one key tile: the second group has no tile at all
    (5, 1, 2, 96, 2, 0, 1.0),    # 96 keys, still one (ragged) tile
    (5, 3, 3, 144, 1, 0, 1.0),   # two tiles, the second ragged: one per group
    (7, 4, 5, 200, 2, 0, 1.0),   # wrapped ring, two runs with ragged tiles, 3 tiles (odd count)
    (7, 2, 7, 200, 1, 0, 8.0),   # peaky scores: the stale-max rescale of each group's O
    (6, 4, 6, 144, 2, 1, 1.0),   # sink frame + wrapping FIFO: three runs of key rows
])
def test_attention_two_group_narrow_latent(slots, oldest, n_valid, Nq, B, n_sink, rope_scale):
    dims = dataclasses.replace(I.sweep_dims(96, 32), grid_h=6, grid_w=8)
    _attention_case(dims, B=B, slots=slots, oldest=oldest, n_valid=n_valid, Nq=Nq, seed=6600 + 7 * slots + Nq,
                    rope_scale=rope_scale, n_sink=n_sink, tiling=V.TILING_PER_HEAD)


def test_attention_two_group_narrow_latent_wan_window_sampled_rows():
    """d_c = 96 at the Wan shape (256 key tiles: 128 per group), sampled rows."""
    dims = I.sweep_dims(96, 32)
    rows = sample_rows(4680, 48, seed=13)
    _attention_case(dims, B=1, slots=21, oldest=9, n_valid=21, Nq=4680, seed=6700, rows=rows)
