"""Failure detection on the GPU without faulting it: a bounded device wait that
runs out must end its kernel normally, record VIDEOMLA_ETIMEOUT in the device
status word, and leave the context usable (a normal call afterwards is exact)."""
import time

import numpy as np
import pytest
import torch

from mla_latent_kv_write_b200 import inputs as I
from mla_latent_kv_write_b200 import videomla as V
from tests.common import check_attention, f64, oracle_attention

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    lib = V.load_library()
    assert V.device_status(reset=True) == V.OK
    t0 = time.time()
    assert lib.videomla_selftest_wait_timeout(50_000_000, None) == V.OK   # 50 ms
    torch.cuda.synchronize()
    elapsed = time.time() - t0
    assert 0.04 <= elapsed < 5.0, elapsed
    assert V.device_status(reset=False) == V.ETIMEOUT
    assert V.device_status(reset=True) == V.ETIMEOUT
    assert V.device_status(reset=False) == V.OK

    # the context is intact: a regular attention call still matches the oracle
    dims = I.TINY
    w = I.layer_weights(dims, 51)
    q = I.queries(dims, 1, 48, 52)
    cache = I.latent_cache(dims, 1, 3, 53)
    out = V.attention(q["q_nope"].cuda(), q["q_rope"].cuda(), w["W_uk"].cuda(), w["W_uv"].cuda(), cache.cuda(),
                      dims, 3, 0, 3)
    torch.cuda.synchronize()
    assert V.device_status(reset=True) == V.OK
    ref, _ = oracle_attention(dims, q, w, cache, 3, 0, 3)
    check_attention(f64(out.cpu()), ref, "after a timed-out wait")


def test_selftest_rejects_bad_timeouts():
    lib = V.load_library()
    assert lib.videomla_selftest_wait_timeout(0, None) == V.EINVAL
    assert lib.videomla_selftest_wait_timeout(20_000_000_000, None) == V.EINVAL
