"""B200-native VideoMLA latent-KV cache write and latent attention.

The compute path is the C-ABI library ``libvideomla.so`` (hand-written CUDA for
sm_100a); :mod:`.videomla` is its thin ctypes binding.  The library is loaded on
first use and the binding raises if it is missing: there is no CPU fallback.
"""
from .videomla import (  # noqa: F401
    VideoMLAError,
    attention,
    cache_write,
    library_path,
    load_library,
    strerror,
)
