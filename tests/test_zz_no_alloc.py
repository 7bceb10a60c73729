"""The allocation-free attention entry point, through the C ABI.

mla_window_attention_noalloc exists for callers that may not allocate device memory while they
run (memory owned by a pooled or budgeted allocator, or latency-critical loops that cannot take
the device synchronisation of a cudaMalloc/cudaFree).  Its per-call scratch sits in a fixed
32 MiB array inside the library.  These tests check, on two calls in a row, that it gives the
regular entry point's output and the fp64 oracle's within the parity tolerance, that the second
call changes neither the device's free memory nor torch's allocated bytes, and that a call too
large for the fixed array is refused cleanly.  This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

import mla_synth
from tests.harness import Pair, assert_close

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["tiny", "wan_w21_q1", "paper_tiny", "sink_tiny"])
def test_noalloc_matches_regular_entry_point_and_oracle_twice(name):
    import mla_latent_kv_window_b200 as M
    w = mla_synth.WORKLOADS[name]
    # Two caches from the same seeds: one only ever sees the allocation-free call, so the chunk
    # latents it attends to are the ones its own projection wrote.
    p_na, p_reg = Pair(w), Pair(w)
    fill = p_na.hidden(w.fill_frames, mla_synth.fill_seed(w, 0))
    p_na.append(fill)
    p_reg.append(fill, oracle=False)
    nq = w.query_frames * w.F
    xs = [p_na.hidden(w.query_frames, mla_synth.chunk_seed(w, 0, call)) for call in range(2)]
    xs_dev = [x.cuda() for x in xs]
    got = [torch.full_like(x, float("nan")) for x in xs_dev]
    ref = [torch.empty_like(x) for x in xs_dev]
    # Oracle rows: every query token of the small cases, a seeded sample at the Wan size.
    rows = None if nq <= 64 else np.sort(np.random.default_rng(7).choice(nq, 64, replace=False))
    try:
        for call in range(2):
            torch.cuda.synchronize()
            free0, alloc0 = torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated()
            M.mla_window_attention_noalloc(p_na.gpu.handle, xs_dev[call], w.query_frames, got[call])
            torch.cuda.synchronize()
            if call == 1:
                # The first call has looked up the scratch address; from then on nothing allocates.
                assert torch.cuda.mem_get_info()[0] == free0, "the no-alloc call changed free device memory"
                assert torch.cuda.memory_allocated() == alloc0
            M.mla_window_attention(p_reg.gpu.handle, xs_dev[call], w.query_frames, ref[call])
            torch.cuda.synchronize()
            assert M.mla_cache_sync(p_na.gpu.handle) == 0 and M.mla_cache_sync(p_reg.gpu.handle) == 0
            g = got[call].cpu()
            assert torch.isfinite(g.float()).all()
            for b, orc in enumerate(p_na.oracles):
                assert_close(g[b], ref[call][b].float().cpu().double().numpy(),
                             f"{name} call {call} stream {b}: no-alloc vs regular")
                want = orc.attention(xs[call][b], rows=rows)
                mine = g[b] if rows is None else g[b][torch.from_numpy(rows)]
                assert_close(mine, want, f"{name} call {call} stream {b}: no-alloc vs oracle")
    finally:
        p_na.gpu.close()
        p_reg.gpu.close()


def test_noalloc_refuses_calls_larger_than_its_scratch():
    # 4 streams x 3 frames x 1560 tokens x 12 heads x 832 B = 187 MB > 32 MiB.
    import mla_latent_kv_window_b200 as M
    w = mla_synth.WORKLOADS["wan_b4_w21_q3"]
    p = Pair(w, max_chunk_frames=3)
    try:
        p.append(p.hidden(2, mla_synth.fill_seed(w, 0)), oracle=False)
        x = p.hidden(3, 5).cuda()
        out = torch.empty_like(x)
        before = M.mla_cache_state(p.gpu.handle)
        with pytest.raises(M.MLAError) as e:
            M.mla_window_attention_noalloc(p.gpu.handle, x, 3, out)
        assert e.value.status == 1 and "scratch" in str(e.value)
        assert M.mla_cache_state(p.gpu.handle) == before
    finally:
        p.gpu.close()
