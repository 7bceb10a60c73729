"""Failure reporting on the GPU without faulting it: a device wait that runs out of time.

The library's kernels bound every wait; when one runs out, the kernel records
MLA_ERR_DEVICE_TIMEOUT in the cache's status word and returns.  The self-test entry point runs
that same wait against a barrier phase nothing completes (a flag that nothing sets), so the
timeout path is exercised for real, and the GPU context must stay usable afterwards.
"""
import time

import pytest
import torch

import mla_synth
from mla_latent_kv_window_b200 import binding as B
from tests.harness import Pair
from tests.test_gpu_parity import full_check, small

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_the_context_survives():
    w = small(window=2, q=1, seed=40)
    p = Pair(w)
    p.append(p.hidden(2, 750))
    assert B.mla_cache_sync(p.gpu.handle) == B.MLA_OK
    t0 = time.time()
    gave_up = B.mla_cache_selftest_timeout(p.gpu.handle)
    waited = time.time() - t0
    assert gave_up, "the device wait did not report giving up"
    assert 1.5 < waited < 60.0, f"the bounded wait took {waited:.2f} s (limit 2 s)"
    assert B.mla_cache_sync(p.gpu.handle) == B.MLA_ERR_DEVICE_TIMEOUT
    assert B.mla_cache_sync(p.gpu.handle) == B.MLA_ERR_DEVICE_TIMEOUT   # reading clears nothing
    p.gpu.close()
    # The context is intact: a fresh cache on the same device computes correct results.
    q = Pair(w)
    q.append(q.hidden(2, 751))
    full_check(q, q.hidden(1, 752), "fresh cache after a device timeout")
    torch.cuda.synchronize()
