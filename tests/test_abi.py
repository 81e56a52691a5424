"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point that include/videomla.h declares, names its error codes, and
rejects invalid arguments before touching the device."""
import ctypes
import os
import re

import pytest

from mla_latent_kv_write_b200 import build as vbuild
from mla_latent_kv_write_b200 import inputs as I
from mla_latent_kv_write_b200 import videomla as V

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(videomla_\w+)\s*\(", text))
    return names


@pytest.fixture(scope="module")
def lib():
    vbuild.build()
    return V.load_library()


def test_library_exports_every_declared_symbol(lib):
    declared = declared_symbols()
    assert declared, "no declarations found"
    assert declared == set(V.EXPORTED)
    for name in declared:
        assert hasattr(lib, name), name


def test_strerror_and_version(lib):
    assert lib.videomla_version() >= 100
    for code in (V.OK, V.EINVAL, V.EUNSUPPORTED, V.ECUDA, V.ETIMEOUT, V.ENODEVICE):
        assert lib.videomla_strerror(code)
    assert b"unknown" in lib.videomla_strerror(12345)


def test_attention_tiling_knob(lib):
    # header constants and the binding's names agree; unknown modes change nothing
    hdr = open(os.path.join(ROOT, "include", "videomla.h")).read()
    for name, val in (("AUTO", V.TILING_AUTO), ("PER_HEAD", V.TILING_PER_HEAD), ("HEAD_PACKED", V.TILING_HEAD_PACKED)):
        assert re.search(rf"#define VIDEOMLA_TILING_{name} {val}\b", hdr), name
    assert lib.videomla_set_attention_tiling(V.TILING_PER_HEAD) == V.TILING_AUTO
    assert lib.videomla_set_attention_tiling(3) == V.EINVAL
    assert lib.videomla_set_attention_tiling(-1) == V.EINVAL
    assert lib.videomla_set_attention_tiling(V.TILING_HEAD_PACKED) == V.TILING_PER_HEAD
    with V.attention_tiling(V.TILING_PER_HEAD):
        assert lib.videomla_set_attention_tiling(V.TILING_PER_HEAD) == V.TILING_PER_HEAD
    assert lib.videomla_set_attention_tiling(V.TILING_AUTO) == V.TILING_HEAD_PACKED
    with pytest.raises(V.VideoMLAError):
        V.set_attention_tiling(7)


def _dims(**kw):
    return V.c_dims(I.Dims(**kw) if kw else I.WAN)


P = ctypes.c_void_p(0x10000)  # a fake, 16-byte aligned device address: never dereferenced


def test_cache_write_rejects_bad_arguments(lib):
    d = _dims()
    f = lib.videomla_cache_write
    T_f = 1560
    ok_args = [ctypes.byref(d), P, 1, 3 * T_f, P, P, None, P, 21, 18, 0, None]
    def call(**over):
        a = list(ok_args)
        for i, v in over.items():
            a[int(i[1:])] = v
        return f(*a)
    assert call(a1=None) == V.EINVAL                      # x null
    assert call(a4=None) == V.EINVAL                      # W_dkv null
    assert call(a7=None) == V.EINVAL                      # cache null
    assert call(a3=T_f + 1) == V.EINVAL                   # not a whole number of frames
    assert call(a3=22 * T_f) == V.EINVAL                  # more frames than slots
    assert call(a9=21) == V.EINVAL                        # first_slot out of range
    assert call(a9=-1) == V.EINVAL
    assert call(a2=0) == V.EINVAL                         # batch
    assert call(a10=8) == V.EINVAL                        # unknown flag
    assert call(a1=ctypes.c_void_p(0x10008)) == V.EINVAL  # misaligned
    assert f(None, *ok_args[1:]) == V.EINVAL              # dims null
    bad = _dims(); bad.pairs_t = 7                         # pairs do not cover d_rope
    assert f(ctypes.byref(bad), *ok_args[1:]) == V.EINVAL
    odd = _dims(); odd.d_model = 1000                      # d_model not a multiple of 64
    assert f(ctypes.byref(odd), *ok_args[1:]) == V.EUNSUPPORTED


def test_attention_rejects_bad_arguments(lib):
    d = _dims()
    f = lib.videomla_attention
    win = V.CWindow(21, 0, 21)
    ws = lib.videomla_attention_workspace_size(ctypes.byref(d), ctypes.byref(win), 1)
    assert ws == 21 * 1560 * 32 * 2
    ok_args = [ctypes.byref(d), P, P, P, P, P, ctypes.byref(win), 1, 4680, P, None, P, ws, None]
    def call(**over):
        a = list(ok_args)
        for i, v in over.items():
            a[int(i[1:])] = v
        return f(*a)
    for i in (1, 2, 3, 4, 5, 9):
        assert call(**{f"a{i}": None}) == V.EINVAL
    assert call(a6=None) == V.EINVAL
    for w in ((0, 0, 1), (21, 21, 1), (21, -1, 1), (21, 0, 0), (21, 0, 22)):
        bad = V.CWindow(*w)
        assert call(a6=ctypes.byref(bad)) == V.EINVAL
    assert call(a8=21 * 1560 + 1) == V.EINVAL             # more queries than window tokens
    assert call(a8=0) == V.EINVAL
    assert call(a10=ctypes.c_void_p(0x10002)) == V.EINVAL  # misaligned lse
    assert call(a11=None) == V.EINVAL                     # no workspace
    assert call(a12=ws - 1) == V.EINVAL                   # workspace too small
    assert call(a11=ctypes.c_void_p(0x10008)) == V.EINVAL  # misaligned workspace


def test_valid_call_without_device_reports_no_device(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    d = _dims()
    win = V.CWindow(21, 0, 21)
    rc = lib.videomla_attention(ctypes.byref(d), P, P, P, P, P, ctypes.byref(win), 1, 4680, P, None, P,
                                1 << 30, None)
    assert rc == V.ENODEVICE
    rc = lib.videomla_cache_write(ctypes.byref(d), P, 1, 4680, P, P, None, P, 21, 18, 0, None)
    assert rc == V.ENODEVICE


def test_dense_attention_rejects_bad_arguments(lib):
    d = _dims()
    f = lib.videomla_dense_attention
    T_f = 1560
    ok_args = [ctypes.byref(d), P, P, P, P, 1, 4680, 21 * T_f, P, None]
    def call(**over):
        a = list(ok_args)
        for i, v in over.items():
            a[int(i[1:])] = v
        return f(*a)
    for i in (1, 2, 3, 4, 8):
        assert call(**{f"a{i}": None}) == V.EINVAL
    assert call(a7=21 * T_f + 1) == V.EINVAL              # not a whole number of frames
    assert call(a6=21 * T_f + 1) == V.EINVAL              # more queries than keys
    assert call(a6=0) == V.EINVAL
    assert call(a3=ctypes.c_void_p(0x10008)) == V.EINVAL   # misaligned
    wide = _dims(); wide.d_v = 192                          # the baseline keeps 128-wide heads
    assert f(ctypes.byref(wide), *ok_args[1:]) == V.EUNSUPPORTED


def test_unsupported_geometry_is_reported(lib):
    import torch
    if not torch.cuda.is_available():
        pytest.skip("the geometry check follows the device check")
    d = _dims(); d.d_c = 160
    win = V.CWindow(21, 0, 21)
    P2 = ctypes.c_void_p(0x10000)
    assert lib.videomla_attention(ctypes.byref(d), P2, P2, P2, P2, P2, ctypes.byref(win), 1, 16, P2, None,
                                  P2, 1 << 30, None) == V.EUNSUPPORTED


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    monkeypatch.setenv("VIDEOMLA_LIBRARY", str(tmp_path / "missing.so"))
    monkeypatch.setattr(V, "_LIB", None)
    with pytest.raises(V.VideoMLAError):
        V.load_library()


def test_attention_sink_rejects_bad_arguments(lib):
    d = _dims()
    win = V.CWindow(6, 0, 6)
    P = ctypes.c_void_p(0x10000)
    T_f = d.grid_h * d.grid_w
    ws = lib.videomla_attention_sink_workspace_size(ctypes.byref(d), ctypes.byref(win), 1, 1)
    assert ws == (6 + 1) * T_f * d.d_rope * 2
    assert lib.videomla_attention_workspace_size(ctypes.byref(d), ctypes.byref(win), 1) == 6 * T_f * d.d_rope * 2

    def call(sink=P, n_sink=1, nq=T_f, ws_bytes=ws):
        return lib.videomla_attention_sink(ctypes.byref(d), P, P, P, P, P, ctypes.byref(win), sink, n_sink, 1, nq, P,
                                           None, P, ws_bytes, None)
    assert call(n_sink=-1) == V.EINVAL
    assert call(n_sink=9) == V.EINVAL                              # above VIDEOMLA_MAX_SINK_FRAMES
    assert call(sink=None) == V.EINVAL                             # sink cache missing
    assert call(sink=ctypes.c_void_p(0x10008)) == V.EINVAL         # misaligned sink cache
    assert call(nq=7 * T_f + 1) == V.EINVAL                        # more queries than sink + window tokens
    assert call(ws_bytes=ws - 1) == V.EINVAL                       # workspace without the sink rows


def test_split_workspace_follows_the_wave_count(lib):
    """Split-KV only when the (query tile, head, batch) units leave the last wave of
    a 148-SM grid mostly empty: the Wan chunk (37 query tiles x 12 heads = 444 units,
    three full waves) is not split; one query frame (13 x 12 = 156 units, 148 + 8)
    is, and its workspace adds fp32 partial O tiles and per-row (max, sum) of every
    split plus one arrival counter per unit.  Without a device the library assumes
    148 SMs, the B200's count."""
    d = _dims()
    T_f = d.grid_h * d.grid_w
    win = V.CWindow(21, 0, 21)
    rope = lib.videomla_attention_workspace_size(ctypes.byref(d), ctypes.byref(win), 1)
    assert rope == 21 * T_f * d.d_rope * 2
    full = lib.videomla_attention_workspace_size_split(ctypes.byref(d), ctypes.byref(win), 0, 1, 3 * T_f)
    assert full == rope
    one = lib.videomla_attention_workspace_size_split(ctypes.byref(d), ctypes.byref(win), 0, 1, T_f)
    units = 13 * 12
    per_split = units * (128 * d.d_c * 4 + 128 * 2 * 4)
    extra = one - (rope + 255) // 256 * 256
    counters = (units * 4 + 255) // 256 * 256
    assert (extra - counters) % per_split == 0
    assert 2 <= (extra - counters) // per_split <= 4
    # a bad window sizes nothing
    assert lib.videomla_attention_workspace_size_split(ctypes.byref(d), ctypes.byref(V.CWindow(21, 0, 22)), 0, 1,
                                                       T_f) == 0


C_CALLER = r"""
#include <stdio.h>
#include <string.h>
#include "videomla.h"

int main(void) {
    videomla_dims d;
    videomla_window w;
    memset(&d, 0, sizeof d);
    d.d_model = 1536; d.n_heads = 12; d.d_c = 192; d.d_rope = 32; d.d_nope = 96; d.d_v = 128;
    d.grid_h = 30; d.grid_w = 52; d.pairs_t = 6; d.pairs_h = 5; d.pairs_w = 5;
    d.rope_base = 10000.0f; d.rms_eps = 1e-6f;
    w.slots = 21; w.oldest_slot = 0; w.n_valid = 21;
    int prev = videomla_set_attention_tiling(VIDEOMLA_TILING_HEAD_PACKED);
    int back = videomla_set_attention_tiling(prev);
    int bad = videomla_set_attention_tiling(99);
    printf("%d|%s|%zu|%d|%d|%d\n", videomla_version(), videomla_strerror(VIDEOMLA_EINVAL),
           videomla_attention_workspace_size(&d, &w, 1), prev, back, bad);
    return 0;
}
"""


def test_plain_c_caller_links_and_calls_host_entry_points(lib):
    """The header is C (no C++ in the declarations) and the library exports
    unmangled names: a C99 program includes it, links the library and calls
    the entry points that need no device."""
    import shutil
    import subprocess
    cc = shutil.which("gcc")
    if cc is None:
        pytest.skip("no C compiler")
    out = os.path.join(ROOT, "_build", "abi_c")
    os.makedirs(out, exist_ok=True)
    src = os.path.join(out, "caller.c")
    with open(src, "w") as f:
        f.write(C_CALLER)
    exe = os.path.join(out, "caller")
    pkg = os.path.dirname(vbuild.LIB)
    subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"), src,
                    "-L", pkg, "-lvideomla", "-Wl,-rpath," + pkg, "-o", exe], check=True)
    r = subprocess.run([exe], check=True, capture_output=True, text=True)
    version, err, ws, prev, back, bad = r.stdout.strip().split("|")
    assert int(version) == lib.videomla_version()
    assert err == lib.videomla_strerror(V.EINVAL).decode()
    assert int(ws) == 21 * 1560 * 32 * 2
    # a fresh process starts in automatic tiling; setting returns the previous mode
    assert (int(prev), int(back), int(bad)) == (V.TILING_AUTO, V.TILING_HEAD_PACKED, V.EINVAL)
