"""The allocation-free attention entry point against the regular one, through the C ABI.

mla_window_attention_noalloc exists for callers that may not allocate device memory while they
run (memory owned by a pooled or budgeted allocator, or latency-critical loops that cannot take
the device synchronisation of a cudaMalloc/cudaFree).  Its per-call scratch sits in a fixed
32 MiB array inside the library.  These tests check that two calls in a row give the regular
entry point's output within the parity tolerance, and that a call too large for the fixed array
is refused cleanly.  This file is collected last on purpose.
"""
import pytest
import torch

import mla_synth
from tests.harness import assert_close

pytestmark = pytest.mark.gpu


def _cache(w: mla_synth.Workload, max_chunk: int):
    import mla_latent_kv_window_b200 as M
    dims = dict(w.dims)
    wts = {k: v.cuda() for k, v in mla_synth.make_weights(dims, mla_synth.weight_seed(w, 0)).items()}
    cfg = M.make_config(dims, w.frame_h, w.frame_w, w.window_frames, max_chunk, batch=w.batch,
                        sink_frames=w.sink_frames)
    h = M.mla_cache_create(cfg, wts)
    fill = mla_synth.make_hidden(w.batch, w.fill_frames * w.F, dims["hidden"], mla_synth.fill_seed(w, 0)).cuda()
    M.mla_cache_append(h, fill, w.fill_frames)
    return M, h, dims


@pytest.mark.parametrize("name", ["tiny", "wan_w21_q1", "paper_tiny", "sink_tiny"])
def test_noalloc_matches_regular_entry_point_twice(name):
    w = mla_synth.WORKLOADS[name]
    M, h, dims = _cache(w, w.query_frames)
    try:
        for call in range(2):
            x = mla_synth.make_hidden(w.batch, w.query_frames * w.F, dims["hidden"],
                                      mla_synth.chunk_seed(w, 0, call)).cuda()
            ref = torch.empty_like(x)
            got = torch.full_like(x, float("nan"))
            M.mla_window_attention(h, x, w.query_frames, ref)
            M.mla_window_attention_noalloc(h, x, w.query_frames, got)
            torch.cuda.synchronize()
            assert M.mla_cache_sync(h) == 0
            assert torch.isfinite(got.float()).all()
            for b in range(w.batch):
                assert_close(got[b].cpu(), ref[b].float().cpu().double().numpy(), f"{name} call {call} stream {b}")
    finally:
        M.mla_cache_destroy(h)


def test_noalloc_refuses_calls_larger_than_its_scratch():
    # 4 streams x 3 frames x 1560 tokens x 12 heads x 832 B = 187 MB > 32 MiB.
    w = mla_synth.WORKLOADS["wan_b4_w21_q3"]
    M, h, dims = _cache(w, 3)
    try:
        x = mla_synth.make_hidden(w.batch, 3 * w.F, dims["hidden"], 5).cuda()
        out = torch.empty_like(x)
        before = M.mla_cache_state(h)
        with pytest.raises(M.MLAError) as e:
            M.mla_window_attention_noalloc(h, x, 3, out)
        assert e.value.status == 1 and "scratch" in str(e.value)
        assert M.mla_cache_state(h) == before
    finally:
        M.mla_cache_destroy(h)
