"""GPU: mla_cache_commit (append the last attention call's chunk from the latents that call
computed) against the oracle appending the same hidden states ([VideoMLA] App. D.4: denoise a
chunk against the window, then append its latents).  Covers the full ring (latents copied from
the chunk tail), a filling ring (frames already in place, frames that wrap), sink frames filled
by a chunk (rows moved inside the planes), a chunk longer than the window, and batched streams.
"""
import pytest

import mla_synth
from tests.harness import Pair
from tests.test_gpu_parity import check_ring, full_check

pytestmark = pytest.mark.gpu


def small(window, fill, q, batch=1, seed=0, sink=0, scale=False):
    return mla_synth.Workload("small", frame_h=4, frame_w=6, window_frames=window, fill_frames=fill,
                              query_frames=q, batch=batch, seed=seed, sink_frames=sink, stream_scale=scale)


@pytest.mark.parametrize("window,fill,chunks,sink,batch", [
    (2, 2, [1, 1, 1], 0, 1),       # ring full: every frame copied from the tail
    (3, 1, [2, 2, 2], 0, 1),       # in place, then wrapping frames copied
    (2, 0, [2, 2, 1], 1, 1),       # the first chunk fills the sink and the ring's first slot
    (2, 1, [3, 3], 0, 1),          # a chunk longer than the window: its first frame is evicted
    (2, 2, [1, 2, 1], 0, 2),       # batched streams with their own scales
])
def test_commit_equals_append(window, fill, chunks, sink, batch):
    w = small(window, fill, max(chunks), batch=batch, seed=60 + window + fill + sink, sink=sink,
              scale=batch > 1)
    p = Pair(w, max_chunk_frames=max(chunks))
    seed = 7000
    if fill:
        p.append(p.hidden(fill, seed))
        seed += 1
    for i, n in enumerate(chunks):
        x = p.hidden(n, seed)
        seed += 1
        full_check(p, x, f"chunk {i} ({n} frames)")
        p.gpu.commit(n)
        for b, o in enumerate(p.oracles):
            o.append(x[b])
        check_ring(p, f"after committing chunk {i}")
    full_check(p, p.hidden(1, seed), "after the commits")
    p.gpu.close()


def test_commit_refuses_without_a_matching_chunk():
    import mla_latent_kv_window_b200 as M
    w = small(2, 2, 2, seed=70)
    p = Pair(w, max_chunk_frames=2)
    p.append(p.hidden(2, 7100))
    with pytest.raises(M.MLAError) as e:
        p.gpu.commit(1)                          # no attention call yet
    assert e.value.status == M.MLA_ERR_STATE
    p.gpu.attention(p.hidden(2, 7101).cuda())
    with pytest.raises(M.MLAError):
        p.gpu.commit(1)                          # the chunk had 2 frames
    p.gpu.append(p.hidden(1, 7102).cuda())
    with pytest.raises(M.MLAError):
        p.gpu.commit(2)                          # an append came in between
    p.gpu.attention(p.hidden(1, 7103).cuda())
    p.gpu.commit(1)
    with pytest.raises(M.MLAError):
        p.gpu.commit(1)                          # already committed
    assert p.gpu.state() == (4, 2)
    p.gpu.sync()
    p.gpu.close()


@pytest.mark.parametrize("sink", [0, 1])
def test_cache_slot_names_the_configs_rows(sink):
    # mla_cache_slot reads the configuration the cache holds; it must name the rows that
    # mla_ring_slot names for that configuration, sink region included.
    import mla_latent_kv_window_b200 as M
    w = small(3, 2, 1, seed=72 + sink, sink=sink)
    p = Pair(w)
    for f in (0, 1, 2, 3, 7, 10**6 + 1):
        for k in (0, w.F - 1):
            assert M.mla_cache_slot(p.gpu.handle, f, k) == M.mla_ring_slot(p.gpu.cfg, f, k)
    with pytest.raises(M.MLAError):
        M.mla_cache_slot(p.gpu.handle, -1, 0)
    p.gpu.close()
