"""GPU: B independent streams sharded over ranks (the multi-GPU layout of
mla_latent_kv_window_b200.replicas, [VideoMLA] §4.3's batch scaling), run here on one GPU as one
cache per shard.  Each shard's streams must match the oracle stream by stream, and the full-batch
cache, which shows that the batched layout couples no streams (no collective is needed).
"""
import numpy as np
import pytest
import torch

import mla_synth
from mla_latent_kv_window_b200 import LatentWindowCache, replicas
from oracle import OracleLayer
from tests.harness import assert_close, dims_of

pytestmark = pytest.mark.gpu


def _run(w, streams, rows=None):
    """One cache over `streams` of workload w: fill, one chunk; returns outputs [len(streams), n, d]."""
    dims = dict(w.dims)
    wts = mla_synth.make_weights(dims, mla_synth.weight_seed(w, 0))
    scales = mla_synth.stream_scales(w.batch, w.seed)
    fill = mla_synth.make_hidden(w.batch, w.fill_frames * w.F, dims["hidden"], mla_synth.fill_seed(w, 0), scales)
    x = mla_synth.make_hidden(w.batch, w.query_frames * w.F, dims["hidden"], mla_synth.chunk_seed(w, 0, 0), scales)
    c = LatentWindowCache(dims, {k: v.cuda() for k, v in wts.items()}, w.frame_h, w.frame_w,
                          w.window_frames, w.query_frames, batch=len(streams))
    c.append(fill[streams].cuda())
    out = c.attention(x[streams].cuda())
    torch.cuda.synchronize()
    c.sync()
    c.close()
    return out.cpu(), wts, fill, x


@pytest.mark.parametrize("name,rows", [("small_b4", None), ("wan_b4_w21_q3", 64)])
def test_two_shards_match_oracle_and_full_batch(name, rows):
    if name == "small_b4":
        w = mla_synth.Workload("small_b4", frame_h=5, frame_w=6, window_frames=2, fill_frames=3,
                               query_frames=1, batch=4, seed=80, stream_scale=True)
    else:
        w = mla_synth.WORKLOADS[name]
    full, wts, fill, x = _run(w, list(range(w.batch)))
    nq = x.shape[1]
    sel = None if rows is None else np.sort(np.random.default_rng(9).choice(nq, rows, replace=False))
    for rank in range(2):
        mine = list(replicas.shard(w.batch, rank, 2))
        got, _, _, _ = _run(w, mine)
        for i, b in enumerate(mine):
            orc = OracleLayer(dims_of(w), wts)
            orc.append(fill[b])
            ref = orc.attention(x[b], rows=sel)
            mine_rows = got[i] if sel is None else got[i][torch.from_numpy(sel)]
            assert_close(mine_rows, ref, f"{name}: shard {rank}, stream {b} vs oracle")
            # Both runs are within the bar of the oracle, so (triangle inequality) within twice
            # the bar of each other; they differ only in rounding order (each CTA starts its key
            # walk at a tile that depends on its stream index).
            assert_close(got[i], full[b].float().double().numpy(), f"{name}: shard {rank}, stream {b} vs full batch",
                         rel_tol=2e-2, max_tol=6e-2)
