"""The commit's row moves (mla_commit_plan, the host logic mla_cache_commit launches), bit-exact
against a simulation of the planes, without a GPU.

The simulation holds one label per plane row.  An attention call writes its chunk's tokens at
the chunk tail (the rows right after the valid sink region and window); a commit applies the
planned moves in order; an append writes each surviving frame at the rows mla_ring_slot names.
After every step, every frame that should be cached - the first sink_frames frames ever
appended, then the newest W of the others, stated directly - must sit at the rows mla_ring_slot
names for it.
"""
import random

import pytest

import mla_synth
from mla_latent_kv_window_b200 import binding as B


def _cfg(window, sink, frame_w, max_chunk):
    return B.make_config(dict(mla_synth.DIMS_WAN13B), 1, frame_w, window, max_chunk, sink_frames=sink)


def _expected_frames(appended, window, sink):
    n_sink = min(appended, sink)
    return list(range(n_sink)) + list(range(max(n_sink, appended - window), appended))


@pytest.mark.parametrize("window,sink,frame_w,max_chunk", [
    (1, 0, 3, 1), (2, 0, 3, 3), (3, 0, 2, 2), (2, 1, 3, 3), (3, 2, 5, 4), (4, 1, 130, 2), (2, 3, 2, 5)])
def test_commit_plan_against_plane_simulation(window, sink, frame_w, max_chunk):
    cfg = _cfg(window, sink, frame_w, max_chunk)
    F = frame_w
    sink_rows = 0 if sink == 0 else -(-sink * F // 128) * 128
    rows = sink_rows + (window + max_chunk) * F
    plane = [None] * rows
    appended = 0
    rng = random.Random(window * 100 + sink * 10 + frame_w)
    for _ in range(40):
        n = rng.randint(1, max_chunk)
        n_sink = min(appended, sink)
        n_win = min(appended - n_sink, window)
        base = sink_rows + n_win * F
        if rng.random() < 0.7:
            # attention call writes the chunk tail, then the chunk is committed
            for i in range(n):
                for k in range(F):
                    plane[base + i * F + k] = (appended + i, k)
            for src, dst, cnt in B.mla_commit_plan(cfg, appended, n):
                assert cnt == F
                assert 0 <= src and src + cnt <= rows and 0 <= dst and dst + cnt <= rows
                plane[dst:dst + cnt] = plane[src:src + cnt]
        else:
            # an append writes each frame at its slot, in frame order (later frames win)
            for i in range(n):
                for k in range(F):
                    plane[B.mla_ring_slot(cfg, appended + i, k)] = (appended + i, k)
        appended += n
        for f in _expected_frames(appended, window, sink):
            for k in range(F):
                assert plane[B.mla_ring_slot(cfg, f, k)] == (f, k), (appended, f, k)


def test_commit_plan_rejects_bad_arguments():
    cfg = _cfg(2, 0, 3, 2)
    for frames_appended, n in ((0, 0), (0, 3), (-1, 1)):
        with pytest.raises(B.MLAError):
            B.mla_commit_plan(cfg, frames_appended, n)
