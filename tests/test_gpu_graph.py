"""GPU: the attention call captured in a CUDA graph and replayed (the serving pattern: static
input buffers, one graph per denoising step, no host work per replay).

A graph holds the launches as they were made at capture time, including the cache state they saw
(the number of valid frames, the chunk's temporal index): it stays valid while that state does,
i.e. for the denoising steps of one chunk, which run against the same window ([VideoMLA] App.
D.4).  The chunk is then appended (committed) outside the graph.
"""
import pytest
import torch

import mla_synth
from tests.harness import Pair, assert_close
from tests.test_gpu_parity import check_ring

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["tiny", "sink_tiny", "wan_w21_q1"])
def test_attention_graph_replays_match_the_oracle(name):
    w = mla_synth.WORKLOADS[name]
    p = Pair(w)
    p.append(p.hidden(w.fill_frames, mla_synth.fill_seed(w, 0)))
    nq = w.query_frames * w.F
    xs = [p.hidden(w.query_frames, mla_synth.chunk_seed(w, 0, s)) for s in range(3)]
    x_static = xs[0].cuda()
    out_static = torch.empty_like(x_static)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):                     # warm-up outside the capture
        p.gpu.attention(x_static, out_static)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        p.gpu.attention(x_static, out_static)
    rows = None if nq <= 64 else torch.arange(0, nq, 13)
    for step, x in enumerate(xs):                     # denoising steps: new inputs, same window
        x_static.copy_(x.cuda())
        g.replay()
        torch.cuda.synchronize()
        got = out_static.cpu()
        for b, orc in enumerate(p.oracles):
            ref = orc.attention(x[b], rows=None if rows is None else rows.numpy())
            mine = got[b] if rows is None else got[b][rows]
            assert_close(mine, ref, f"{name}: graph replay {step}, stream {b}")
    p.check_status()
    # the last step's chunk joins the window, outside the graph
    p.gpu.commit(w.query_frames)
    for b, orc in enumerate(p.oracles):
        orc.append(xs[-1][b])
    check_ring(p, f"{name}: after committing the replayed chunk")
    del g
    p.gpu.close()
