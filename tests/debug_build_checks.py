"""Checks that run only on the bounds-checked build, libmla_debug.so (MLA_DEBUG).

Not collected on its own (the file name does not start with test_): tests/test_gpu_debug_build.py
runs it in a child process with MLA_LIBRARY pointing at the debug build, so that the binding
loads that library instead of libmla.so.
"""
import os

import pytest
import torch

import mla_synth
from tests.harness import Pair

pytestmark = pytest.mark.gpu


def test_the_debug_library_is_loaded():
    from mla_latent_kv_window_b200 import binding
    assert os.path.basename(binding.LIB_PATH) == "libmla_debug.so"


def _tiny_pair(seed=90):
    w = mla_synth.Workload("dbg", frame_h=4, frame_w=6, window_frames=2, fill_frames=2,
                           query_frames=1, seed=seed)
    p = Pair(w)
    p.append(p.hidden(2, seed * 16 + 1), oracle=False)
    p.gpu.attention(p.hidden(1, seed * 16 + 2).cuda())
    torch.cuda.synchronize()
    return p


def test_guard_bands_are_clean_and_a_write_into_one_is_reported():
    # A byte written into the guard band right after the c_kv plane (an in-bounds write of the
    # allocation, made from the host) must turn the next sync into MLA_ERR_BOUNDS.
    import mla_latent_kv_window_b200 as M
    from cuda.bindings import runtime as cudart
    p = _tiny_pair()
    assert M.mla_cache_sync(p.gpu.handle) == 0
    dbg = M.mla_cache_debug_buffers(p.gpu.handle)
    plane_bytes = p.gpu.cfg.batch * dbg.rows_per_stream * 192 * 2
    err, = cudart.cudaMemset(dbg.ckv + plane_bytes + 100, 0, 1)
    assert int(err) == 0
    assert M.mla_cache_sync(p.gpu.handle) == M.MLA_ERR_BOUNDS
    assert "c_kv plane" in M.load_library().mla_last_error().decode()
    p.gpu.close()


def test_device_bounds_check_catches_an_out_of_range_row():
    import mla_latent_kv_window_b200 as M
    p = _tiny_pair(91)
    assert M.mla_cache_selftest_bounds(p.gpu.handle) is True
    assert M.mla_cache_sync(p.gpu.handle) == M.MLA_ERR_BOUNDS
    p.gpu.close()
    # the context is still usable: a fresh cache computes and syncs clean
    q = _tiny_pair(92)
    assert M.mla_cache_sync(q.gpu.handle) == 0
    q.gpu.close()
