"""The attention entry point that needs no caller workspace.

Some callers cannot hand the library a scratch buffer: their device memory is
owned by a pool or arena they do not expose, or they run where a cudaMalloc is
not allowed.  ``videomla_attention_static_workspace`` serves them with a scratch
array compiled into the library.  This test calls it through the C ABI four
times in a row, on different windows (one split-KV, one on head-packed query
tiles), and checks each
result against the regular ``videomla_attention`` (caller workspace) on the same
inputs, with the tolerance the other attention tests use.  It also checks that
a window too large for the built-in array is refused before anything is
launched.
"""
import ctypes

import numpy as np
import pytest
import torch

from mla_latent_kv_write_b200 import inputs as I
from mla_latent_kv_write_b200 import videomla as V
from tests.common import check_attention, check_lse

pytestmark = pytest.mark.gpu
STATIC_BYTES = 16 << 20  # VIDEOMLA_STATIC_WORKSPACE_BYTES


def _entry():
    lib = V.load_library()
    f = lib.videomla_attention_static_workspace
    vp, ci = ctypes.c_void_p, ctypes.c_int
    f.argtypes = [ctypes.POINTER(V.CDims), vp, vp, vp, vp, vp, ctypes.POINTER(V.CWindow), ci, ci, vp, vp, vp]
    f.restype = ci
    return f


def _case(dims, B, slots, oldest, n_valid, Nq, seed):
    w = {k: t.cuda() for k, t in I.layer_weights(dims, seed).items()}
    q = {k: t.cuda() for k, t in I.queries(dims, B, Nq, seed + 1).items()}
    cache = I.latent_cache(dims, B, slots, seed + 2).cuda()
    return w, q, cache


def _static_call(f, dims, w, q, cache, slots, oldest, n_valid):
    B, Nq = q["q_nope"].shape[:2]
    out = torch.empty(B, Nq, dims.n_heads, dims.d_v, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B, Nq, dims.n_heads, dtype=torch.float32, device="cuda")
    cd, win = V.c_dims(dims), V.CWindow(slots, oldest, n_valid)
    rc = f(ctypes.byref(cd), q["q_nope"].data_ptr(), q["q_rope"].data_ptr(), w["W_uk"].data_ptr(),
           w["W_uv"].data_ptr(), cache.data_ptr(), ctypes.byref(win), B, Nq, out.data_ptr(), lse.data_ptr(),
           torch.cuda.current_stream().cuda_stream)
    assert rc == V.OK, V.strerror(rc)
    return out, lse


def test_static_workspace_matches_regular_entry_point_in_a_row():
    f = _entry()
    cases = [
        # Wan-1.3B layer window (2 MiB of scratch, unsplit), then one query tile
        # against the same 21-frame window, which splits its key tiles 4 ways
        # with the partials and counters in the array behind the RoPE keys, on
        # top of what the first call left there; then a wrapped tiny window with
        # ragged tiles and batch 2: no call may see another's rows; last the
        # 1560-query frame step, which runs on 147 head-packed CTAs
        (I.WAN, 1, 21, 0, 21, 4680, 31, False),
        (I.WAN, 1, 21, 5, 21, 128, 33, True),
        (I.TINY, 2, 7, 4, 5, 100, 32, None),
        (I.WAN, 1, 21, 9, 21, 1560, 34, None),
    ]
    for dims, B, slots, oldest, n_valid, Nq, seed, splits in cases:
        rope = V.workspace_size(dims, slots, oldest, n_valid, B)
        preferred = V.workspace_size(dims, slots, oldest, n_valid, B, n_query=Nq)
        if splits is not None:
            # the split path runs iff its partials fit in the array beside the RoPE keys
            assert (rope < preferred <= STATIC_BYTES) == splits
        w, q, cache = _case(dims, B, slots, oldest, n_valid, Nq, seed)
        got, got_lse = _static_call(f, dims, w, q, cache, slots, oldest, n_valid)
        ref, ref_lse = V.attention(q["q_nope"], q["q_rope"], w["W_uk"], w["W_uv"], cache, dims, slots, oldest,
                                   n_valid, want_lse=True)
        torch.cuda.synchronize()
        assert V.device_status(reset=True) == V.OK
        g, r = I.to_numpy64(got.cpu()), I.to_numpy64(ref.cpu())
        check_attention(g, r, f"static workspace vs caller workspace, slots={slots} B={B}")
        check_lse(I.to_numpy64(got_lse.cpu()), I.to_numpy64(ref_lse.cpu()), "static workspace lse")


def test_static_workspace_rejects_windows_beyond_its_size():
    f = _entry()
    dims = I.WAN
    slots = 63
    B = STATIC_BYTES // (slots * dims.tokens_per_frame * dims.d_rope * 2) + 1   # one batch element too many
    assert V.workspace_size(dims, slots, 0, slots, B) > STATIC_BYTES
    cd, win = V.c_dims(dims), V.CWindow(slots, 0, slots)
    P = 0x10000  # never dereferenced: the size check comes first
    rc = f(ctypes.byref(cd), P, P, P, P, P, ctypes.byref(win), B, 16, P, None, None)
    assert rc == V.EINVAL
