"""ctypes binding of ``libvideomla.so`` (C ABI: ``include/videomla.h``).

Argument marshalling only: tensors are checked for dtype, device, shape and
contiguity, and their device pointers are passed with the current CUDA stream.
Every step of the computation runs in the library's sm_100a kernels.  If the
library is missing or cannot be loaded the calls raise: there is no fallback.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import threading
from typing import Optional

import torch

from .inputs import Dims

_PKG = os.path.dirname(os.path.abspath(__file__))
_LOCK = threading.RLock()
_LIB: Optional[ctypes.CDLL] = None

OK, EINVAL, EUNSUPPORTED, ECUDA, ETIMEOUT, ENODEVICE = 0, -1, -2, -3, -4, -5
CACHE_RAW_LATENT = 1

# every symbol the header declares
EXPORTED = (
    "videomla_cache_write",
    "videomla_attention",
    "videomla_attention_workspace_size",
    "videomla_attention_static_workspace",
    "videomla_attention_sink",
    "videomla_attention_sink_workspace_size",
    "videomla_attention_workspace_size_split",
    "videomla_dense_attention",
    "videomla_query_projection",
    "videomla_query_projection_workspace_size",
    "videomla_output_projection",
    "videomla_strerror",
    "videomla_device_status",
    "videomla_set_wait_timeout_ns",
    "videomla_set_attention_tiling",
    "videomla_selftest_wait_timeout",
    "videomla_version",
)


class VideoMLAError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {strerror(code)} ({code})")


class CDims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("d_model", "n_heads", "d_c", "d_rope", "d_nope", "d_v",
                                            "grid_h", "grid_w", "pairs_t", "pairs_h", "pairs_w")] + [
        ("rope_base", ctypes.c_float), ("rms_eps", ctypes.c_float)]


class CWindow(ctypes.Structure):
    _fields_ = [("slots", ctypes.c_int), ("oldest_slot", ctypes.c_int), ("n_valid", ctypes.c_int)]


def library_path() -> str:
    return os.environ.get("VIDEOMLA_LIBRARY", os.path.join(_PKG, "libvideomla.so"))


def load_library() -> ctypes.CDLL:
    global _LIB
    with _LOCK:
        if _LIB is not None:
            return _LIB
        path = library_path()
        if not os.path.exists(path):
            raise VideoMLAError(ECUDA, f"{path} is missing; build it with "
                                       "`python -m mla_latent_kv_write_b200.build`")
        lib = ctypes.CDLL(path)
        vp, ci, cu = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint
        lib.videomla_cache_write.argtypes = [ctypes.POINTER(CDims), vp, ci, ci, vp, vp, vp, vp, ci, ci, cu, vp]
        lib.videomla_cache_write.restype = ci
        lib.videomla_attention.argtypes = [ctypes.POINTER(CDims), vp, vp, vp, vp, vp, ctypes.POINTER(CWindow),
                                           ci, ci, vp, vp, vp, ctypes.c_size_t, vp]
        lib.videomla_attention.restype = ci
        lib.videomla_attention_workspace_size.argtypes = [ctypes.POINTER(CDims), ctypes.POINTER(CWindow), ci]
        lib.videomla_attention_workspace_size.restype = ctypes.c_size_t
        lib.videomla_attention_sink.argtypes = [ctypes.POINTER(CDims), vp, vp, vp, vp, vp, ctypes.POINTER(CWindow),
                                                vp, ci, ci, ci, vp, vp, vp, ctypes.c_size_t, vp]
        lib.videomla_attention_sink.restype = ci
        lib.videomla_attention_sink_workspace_size.argtypes = [ctypes.POINTER(CDims), ctypes.POINTER(CWindow), ci, ci]
        lib.videomla_attention_sink_workspace_size.restype = ctypes.c_size_t
        lib.videomla_attention_workspace_size_split.argtypes = [ctypes.POINTER(CDims), ctypes.POINTER(CWindow), ci, ci,
                                                                ci]
        lib.videomla_attention_workspace_size_split.restype = ctypes.c_size_t
        lib.videomla_query_projection_workspace_size.argtypes = [ctypes.POINTER(CDims), ci, ci, ci]
        lib.videomla_query_projection_workspace_size.restype = ctypes.c_size_t
        lib.videomla_query_projection.argtypes = [ctypes.POINTER(CDims), ci, vp, ci, ci, vp, vp, vp, vp, vp, vp, vp,
                                                  ctypes.c_size_t, vp]
        lib.videomla_query_projection.restype = ci
        lib.videomla_dense_attention.argtypes = [ctypes.POINTER(CDims), vp, vp, vp, vp, ci, ci, ci, vp, vp]
        lib.videomla_dense_attention.restype = ci
        lib.videomla_output_projection.argtypes = [ctypes.POINTER(CDims), vp, ci, ci, vp, vp, vp]
        lib.videomla_output_projection.restype = ci
        lib.videomla_strerror.argtypes = [ci]
        lib.videomla_strerror.restype = ctypes.c_char_p
        lib.videomla_device_status.argtypes = [ci]
        lib.videomla_device_status.restype = ci
        lib.videomla_set_wait_timeout_ns.argtypes = [ctypes.c_uint64]
        lib.videomla_set_wait_timeout_ns.restype = ctypes.c_uint64
        lib.videomla_set_attention_tiling.argtypes = [ci]
        lib.videomla_set_attention_tiling.restype = ci
        lib.videomla_selftest_wait_timeout.argtypes = [ctypes.c_uint64, vp]
        lib.videomla_selftest_wait_timeout.restype = ci
        lib.videomla_version.argtypes = []
        lib.videomla_version.restype = ci
        _LIB = lib
        return lib


_NAMES = {OK: "ok", EINVAL: "invalid argument", EUNSUPPORTED: "unsupported geometry",
          ECUDA: "CUDA error", ETIMEOUT: "device-side wait timed out", ENODEVICE: "no sm_100 device"}


def strerror(code: int) -> str:
    """Name of a status code (host-side table; the library's
    ``videomla_strerror`` gives the same names)."""
    return _NAMES.get(code, f"unknown error {code}")


def c_dims(d: Dims) -> CDims:
    return CDims(d.d_model, d.n_heads, d.d_c, d.d_rope, d.d_nope, d.d_v, d.grid_h, d.grid_w,
                 d.pairs[0], d.pairs[1], d.pairs[2], d.rope_base, d.rms_eps)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _check(t: torch.Tensor, name: str, dtype: torch.dtype, shape=None, device=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def cache_write(x: torch.Tensor, W_dkv: torch.Tensor, W_kr: torch.Tensor, gamma: Optional[torch.Tensor],
                cache: torch.Tensor, dims: Dims, slots: int, first_slot: int, raw_latent: bool = False,
                stream=None) -> torch.Tensor:
    """Write the latent cache rows of the tokens ``x`` [B, n_tok, d_model] into
    ``cache`` [B, slots*T_f, d_c + d_rope] (in place; returns ``cache``)."""
    lib = load_library()
    B, n_tok = x.shape[0], x.shape[1]
    dev = x.device
    _check(x, "x", torch.bfloat16, (B, n_tok, dims.d_model))
    _check(W_dkv, "W_dkv", torch.bfloat16, (dims.d_c, dims.d_model), dev)
    _check(W_kr, "W_kr", torch.bfloat16, (dims.d_rope, dims.d_model), dev)
    if gamma is not None:
        _check(gamma, "gamma", torch.float32, (dims.d_c,), dev)
    _check(cache, "cache", torch.bfloat16, (B, slots * dims.tokens_per_frame, dims.cache_width), dev)
    cd = c_dims(dims)
    rc = lib.videomla_cache_write(ctypes.byref(cd), _ptr(x), B, n_tok, _ptr(W_dkv), _ptr(W_kr), _ptr(gamma),
                                  _ptr(cache), slots, first_slot, CACHE_RAW_LATENT if raw_latent else 0,
                                  _stream(stream))
    if rc != OK:
        raise VideoMLAError(rc, "videomla_cache_write")
    return cache


def workspace_size(dims: Dims, slots: int, oldest: int, n_valid: int, batch: int, n_sink: int = 0,
                   n_query: Optional[int] = None) -> int:
    """Bytes of the attention workspace: the window's rotated RoPE keys, plus the
    split-KV partials of the preferred split when ``n_query`` is given."""
    cd, win = c_dims(dims), CWindow(slots, oldest, n_valid)
    lib = load_library()
    if n_query is None:
        return int(lib.videomla_attention_sink_workspace_size(ctypes.byref(cd), ctypes.byref(win), n_sink, batch))
    return int(lib.videomla_attention_workspace_size_split(ctypes.byref(cd), ctypes.byref(win), n_sink, batch,
                                                           n_query))


def attention(q_nope: torch.Tensor, q_rope: torch.Tensor, W_uk: torch.Tensor, W_uv: torch.Tensor,
              cache: torch.Tensor, dims: Dims, slots: int, oldest: int, n_valid: int,
              out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
              want_lse: bool = False, workspace: Optional[torch.Tensor] = None, stream=None,
              sink: Optional[torch.Tensor] = None):
    """Latent attention of the queries over the window; returns ``out``
    [B, Nq, H, d_v] (and ``lse`` [B, Nq, H] if requested or given).

    ``sink`` [B, n_sink T_f, d_c + d_rope] holds pinned sink frames that join
    the window before the ring frames (``videomla_attention_sink``).
    ``workspace`` is a device byte buffer of at least ``workspace_size(...)``
    bytes; if omitted, one is taken from torch's stream-ordered caching
    allocator for this call."""
    lib = load_library()
    B, Nq, H = q_nope.shape[0], q_nope.shape[1], dims.n_heads
    dev = q_nope.device
    _check(q_nope, "q_nope", torch.bfloat16, (B, Nq, H, dims.d_nope))
    _check(q_rope, "q_rope", torch.bfloat16, (B, Nq, H, dims.d_rope), dev)
    _check(W_uk, "W_uk", torch.bfloat16, (H * dims.d_nope, dims.d_c), dev)
    _check(W_uv, "W_uv", torch.bfloat16, (H * dims.d_v, dims.d_c), dev)
    _check(cache, "cache", torch.bfloat16, (B, slots * dims.tokens_per_frame, dims.cache_width), dev)
    if out is None:
        out = torch.empty(B, Nq, H, dims.d_v, dtype=torch.bfloat16, device=dev)
    _check(out, "out", torch.bfloat16, (B, Nq, H, dims.d_v), dev)
    if lse is None and want_lse:
        lse = torch.empty(B, Nq, H, dtype=torch.float32, device=dev)
    if lse is not None:
        _check(lse, "lse", torch.float32, (B, Nq, H), dev)
    T_f = dims.tokens_per_frame
    n_sink = 0
    if sink is not None:
        if sink.dim() != 3 or sink.shape[1] % T_f != 0:
            raise ValueError("sink must be [B, n_sink * T_f, d_c + d_rope]")
        n_sink = sink.shape[1] // T_f
        _check(sink, "sink", torch.bfloat16, (B, n_sink * T_f, dims.cache_width), dev)
    cd = c_dims(dims)
    win = CWindow(slots, oldest, n_valid)
    need = int(lib.videomla_attention_sink_workspace_size(ctypes.byref(cd), ctypes.byref(win), n_sink, B))
    if workspace is None:  # room for the split-KV partials too
        need = int(lib.videomla_attention_workspace_size_split(ctypes.byref(cd), ctypes.byref(win), n_sink, B, Nq))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    elif workspace.device != dev or workspace.numel() * workspace.element_size() < need:
        raise ValueError(f"workspace must be a {need}-byte buffer on {dev}")
    if sink is None:
        rc = lib.videomla_attention(ctypes.byref(cd), _ptr(q_nope), _ptr(q_rope), _ptr(W_uk), _ptr(W_uv),
                                    _ptr(cache), ctypes.byref(win), B, Nq, _ptr(out), _ptr(lse), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _stream(stream))
    else:
        rc = lib.videomla_attention_sink(ctypes.byref(cd), _ptr(q_nope), _ptr(q_rope), _ptr(W_uk), _ptr(W_uv),
                                         _ptr(cache), ctypes.byref(win), _ptr(sink), n_sink, B, Nq, _ptr(out),
                                         _ptr(lse), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                         _stream(stream))
    if rc != OK:
        raise VideoMLAError(rc, "videomla_attention_sink" if sink is not None else "videomla_attention")
    return (out, lse) if lse is not None else out


def query_projection(x: torch.Tensor, W_dq: torch.Tensor, gamma_q: Optional[torch.Tensor], W_uq: torch.Tensor,
                     W_qr: torch.Tensor, dims: Dims, q_nope: Optional[torch.Tensor] = None,
                     q_rope: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None, stream=None):
    """Per-head queries (q_nope [B, n, H, d_nope], unrotated q_rope [B, n, H, d_rope])
    of the tokens x [B, n, d_model]: query latent, RMSNorm, up-projections."""
    lib = load_library()
    B, n = x.shape[0], x.shape[1]
    H, dq, dev = dims.n_heads, dims.d_q, x.device
    _check(x, "x", torch.bfloat16, (B, n, dims.d_model))
    _check(W_dq, "W_dq", torch.bfloat16, (dq, dims.d_model), dev)
    _check(W_uq, "W_uq", torch.bfloat16, (H * dims.d_nope, dq), dev)
    _check(W_qr, "W_qr", torch.bfloat16, (H * dims.d_rope, dq), dev)
    if gamma_q is not None:
        _check(gamma_q, "gamma_q", torch.float32, (dq,), dev)
    if q_nope is None:
        q_nope = torch.empty(B, n, H, dims.d_nope, dtype=torch.bfloat16, device=dev)
    if q_rope is None:
        q_rope = torch.empty(B, n, H, dims.d_rope, dtype=torch.bfloat16, device=dev)
    _check(q_nope, "q_nope", torch.bfloat16, (B, n, H, dims.d_nope), dev)
    _check(q_rope, "q_rope", torch.bfloat16, (B, n, H, dims.d_rope), dev)
    cd = c_dims(dims)
    need = int(lib.videomla_query_projection_workspace_size(ctypes.byref(cd), dq, B, n))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    elif workspace.device != dev or workspace.numel() * workspace.element_size() < need:
        raise ValueError(f"workspace must be a {need}-byte buffer on {dev}")
    rc = lib.videomla_query_projection(ctypes.byref(cd), dq, _ptr(x), B, n, _ptr(W_dq), _ptr(gamma_q), _ptr(W_uq),
                                       _ptr(W_qr), _ptr(q_nope), _ptr(q_rope), _ptr(workspace),
                                       workspace.numel() * workspace.element_size(), _stream(stream))
    if rc != OK:
        raise VideoMLAError(rc, "videomla_query_projection")
    return q_nope, q_rope


def output_projection(o: torch.Tensor, W_O: torch.Tensor, dims: Dims, y: Optional[torch.Tensor] = None, stream=None):
    """Layer output y [B, n, d_model] = W_O [o_1 .. o_H] of per-head outputs o [B, n, H, d_v]."""
    lib = load_library()
    B, n, H, dev = o.shape[0], o.shape[1], dims.n_heads, o.device
    _check(o, "o", torch.bfloat16, (B, n, H, dims.d_v))
    _check(W_O, "W_O", torch.bfloat16, (dims.d_model, H * dims.d_v), dev)
    if y is None:
        y = torch.empty(B, n, dims.d_model, dtype=torch.bfloat16, device=dev)
    _check(y, "y", torch.bfloat16, (B, n, dims.d_model), dev)
    cd = c_dims(dims)
    rc = lib.videomla_output_projection(ctypes.byref(cd), _ptr(o), B, n, _ptr(W_O), _ptr(y), _stream(stream))
    if rc != OK:
        raise VideoMLAError(rc, "videomla_output_projection")
    return y


def dense_attention(q_nope: torch.Tensor, q_rope: torch.Tensor, k: torch.Tensor, v: torch.Tensor, dims: Dims,
                    out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Dense multi-head attention baseline over per-head keys ``k`` and values
    ``v`` [B, n_keys, H, 128] of a window in logical order (RoPE part of k already
    rotated); queries are its newest n_query tokens (q_rope unrotated)."""
    lib = load_library()
    B, Nq, H = q_nope.shape[0], q_nope.shape[1], dims.n_heads
    Nk = k.shape[1]
    dev = q_nope.device
    _check(q_nope, "q_nope", torch.bfloat16, (B, Nq, H, dims.d_nope))
    _check(q_rope, "q_rope", torch.bfloat16, (B, Nq, H, dims.d_rope), dev)
    _check(k, "k", torch.bfloat16, (B, Nk, H, 128), dev)
    _check(v, "v", torch.bfloat16, (B, Nk, H, 128), dev)
    if out is None:
        out = torch.empty(B, Nq, H, 128, dtype=torch.bfloat16, device=dev)
    _check(out, "out", torch.bfloat16, (B, Nq, H, 128), dev)
    cd = c_dims(dims)
    rc = lib.videomla_dense_attention(ctypes.byref(cd), _ptr(q_nope), _ptr(q_rope), _ptr(k), _ptr(v), B, Nq, Nk,
                                      _ptr(out), _stream(stream))
    if rc != OK:
        raise VideoMLAError(rc, "videomla_dense_attention")
    return out


def device_status(reset: bool = False) -> int:
    return load_library().videomla_device_status(1 if reset else 0)


def set_wait_timeout_ns(ns: int) -> int:
    return load_library().videomla_set_wait_timeout_ns(ns)


TILING_AUTO, TILING_PER_HEAD, TILING_HEAD_PACKED = 0, 1, 2


def set_attention_tiling(mode: int) -> int:
    """Query-row tiling of the attention calls (process-wide); returns the previous mode."""
    rc = load_library().videomla_set_attention_tiling(mode)
    if rc < 0:
        raise VideoMLAError(rc, "videomla_set_attention_tiling")
    return rc


@contextlib.contextmanager
def attention_tiling(mode: int):
    """Run the enclosed calls with one tiling mode, then restore the previous one."""
    prev = set_attention_tiling(mode)
    try:
        yield
    finally:
        set_attention_tiling(prev)
