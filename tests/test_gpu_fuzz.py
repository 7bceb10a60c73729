"""GPU: seeded random shapes and call sequences against the fp64 oracle (every element).

Each case draws a small model (4 or 12 heads of 128, hidden 512 or 1536), a frame grid (1 to 40
tokens, ragged against the 128-key tiles), a window of 1 to 4 frames, 0 to 2 sink frames, 1 to 3
streams with their own scales, chunks of 1 to 3 frames, and a sequence of appends, attention calls
and commits; after every attention call every output element is compared with the oracle, and
after every append or commit every cached frame's rows.
"""
import random

import pytest
import torch

import mla_synth
from tests.harness import Pair
from tests.test_gpu_parity import check_ring, full_check

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("case", range(12))
def test_random_shapes_and_sequences(case):
    rng = random.Random(1000 + case)
    heads = rng.choice([4, 12])
    dims = dict(mla_synth.DIMS_WAN13B, hidden=128 * heads, n_heads=heads)
    fh, fw = rng.randint(1, 5), rng.randint(1, 8)
    max_chunk = rng.randint(1, 3)
    w = mla_synth.Workload(f"fuzz{case}", frame_h=fh, frame_w=fw, window_frames=rng.randint(1, 4),
                           fill_frames=0, query_frames=max_chunk, batch=rng.randint(1, 3),
                           seed=7000 + case, stream_scale=True, sink_frames=rng.choice([0, 0, 1, 2]),
                           dims=tuple(sorted(dims.items())))
    p = Pair(w, max_chunk_frames=max_chunk)
    seed = 90000 + 100 * case
    for _ in range(8):
        op = rng.random()
        n = rng.randint(1, max_chunk)
        x = p.hidden(n, seed)
        seed += 1
        if op < 0.35:
            p.append(x)
            check_ring(p, f"fuzz {case}: after append of {n}")
        else:
            full_check(p, x, f"fuzz {case}: {n}-frame chunk", intermediates=op < 0.5)
            if op > 0.7:
                p.gpu.commit(n)
                for b, o in enumerate(p.oracles):
                    o.append(x[b])
                check_ring(p, f"fuzz {case}: after commit of {n}")
    p.gpu.close()


@pytest.mark.parametrize("heads", [3, 5])
def test_odd_head_counts(heads):
    # Odd head counts: the query launch's column blocks (n_h heads + two latent blocks) and
    # the output projection's 3 n_h k-blocks come out odd; every element against the oracle.
    dims = dict(mla_synth.DIMS_WAN13B, hidden=128 * heads, n_heads=heads)
    w = mla_synth.Workload(f"odd{heads}", frame_h=3, frame_w=7, window_frames=2, fill_frames=0,
                           query_frames=2, batch=2, seed=7100 + heads, stream_scale=True,
                           dims=tuple(sorted(dims.items())))
    p = Pair(w, max_chunk_frames=2)
    p.append(p.hidden(3, 91000 + heads))
    check_ring(p, f"{heads} heads: after append")
    full_check(p, p.hidden(2, 91100 + heads), f"{heads} heads: 2-frame chunk")
    full_check(p, p.hidden(1, 91200 + heads), f"{heads} heads: 1-frame chunk")
    p.gpu.close()


@pytest.mark.parametrize("d_nope", [96, 64])
def test_full_rank_query_other_head_splits(d_nope):
    # A full-rank query whose content part is not 128 wide keeps the absorbed query weight
    # W_UK[h]^T W_Q[h] as a bf16 pair (the GEMM whose A column wraps), not the two-step query
    # kernel; every element against the oracle, with stream scales and a ragged frame.
    dims = dict(mla_synth.DIMS_WAN13B, d_nope=d_nope)
    w = mla_synth.Workload(f"split{d_nope}", frame_h=3, frame_w=5, window_frames=2, fill_frames=0,
                           query_frames=2, batch=2, seed=7200 + d_nope, stream_scale=True,
                           dims=tuple(sorted(dims.items())))
    p = Pair(w, max_chunk_frames=2)
    p.append(p.hidden(3, 92000 + d_nope))
    check_ring(p, f"d_nope {d_nope}: after append")
    full_check(p, p.hidden(2, 92100 + d_nope), f"d_nope {d_nope}: 2-frame chunk")
    full_check(p, p.hidden(1, 92200 + d_nope), f"d_nope {d_nope}: 1-frame chunk")
    p.gpu.close()


def test_multi_tile_query_kernel_and_multi_wave_attention_every_element():
    # 3 streams x a 2-frame chunk of 20 x 32 tokens: the query launch has 3 x 5 row tiles x 14
    # column blocks = 210 tiles, so 62 of its 148 CTAs run two tiles (the accumulator reuse and
    # phase bookkeeping across tiles), and the attention grid has 3 x 120 CTAs (more than two
    # waves).  Every element of Qp and of the output against the oracle.
    w = mla_synth.Workload("multitile", frame_h=20, frame_w=32, window_frames=2, fill_frames=0,
                           query_frames=2, batch=3, seed=7300, stream_scale=True)
    p = Pair(w, max_chunk_frames=2)
    p.append(p.hidden(3, 93000))
    check_ring(p, "multi-tile: after append")
    x = p.hidden(2, 93100)
    full_check(p, x, "multi-tile: 2-frame chunk")
    p.gpu.commit(2)
    for b, o in enumerate(p.oracles):
        o.append(x[b])
    check_ring(p, "multi-tile: after commit")
    full_check(p, p.hidden(1, 93200), "multi-tile: 1-frame chunk after the commit")
    p.gpu.close()
