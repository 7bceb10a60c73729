"""GPU parity: the CUDA path through the C ABI against the fp64 oracle, on identical seeded inputs.

Bar (bf16 inputs, fp32 accumulation): relative L2 error <= 1e-2 and max-abs error <= 3e-2 x RMS of
the oracle output, for the layer output and the intermediates (ring contents, absorbed queries,
latent-space attention output); ring slot placement exact.  Small cases compare every element;
the full-size workloads compare seeded samples of query rows, which the oracle computes exactly
(the 21- and 63-frame one-frame workloads: every element).
"""
import math

import numpy as np
import pytest
import torch

import mla_synth
from oracle import ring_slot, rope3d
from tests.harness import Pair, assert_close, dims_of, errors

pytestmark = pytest.mark.gpu

LOG2E = 1.0 / math.log(2.0)


def small(frame_h=4, frame_w=6, window=2, fill=2, q=1, batch=1, seed=0, scale=False):
    return mla_synth.Workload("small", frame_h=frame_h, frame_w=frame_w, window_frames=window,
                              fill_frames=fill, query_frames=q, batch=batch, seed=seed, stream_scale=scale)


def check_ring(pair: Pair, what: str):
    """Every valid frame f sits at slots (f mod W) F + k with the oracle's c_kv and k_rope (with
    a sink: at the rows mla_ring_slot names, which the host tests pin against a FIFO simulation)."""
    W, F = pair.w.window_frames, pair.F
    for b, orc in enumerate(pair.oracles):
        ckv, kr, n_valid = pair.gpu.read_ring(b)
        contents = orc.cache_contents()
        assert n_valid == len(contents) * F
        for f, c, r in contents:
            s0 = pair.gpu_slot(f, 0)
            if not pair.w.sink_frames:
                assert s0 == ring_slot(f, 0, W, F)
            assert_close(ckv[s0:s0 + F], c, f"{what}: c_kv of frame {f} (stream {b})")
            assert_close(kr[s0:s0 + F], r, f"{what}: k_rope of frame {f} (stream {b})")


def oracle_qp(pair: Pair, x_chunk, b: int):
    """Absorbed, rotated, pre-scaled queries in the GPU's row order (q, h), at absolute positions."""
    orc = pair.oracles[b]
    d = pair.dims
    ctx = orc.keys_and_queries(x_chunk, positions="absolute")
    rows = []
    xq = orc.query_input(ctx["x"])
    for h in range(d["n_heads"]):
        dn, dr = d["d_nope"], d["d_rope"]
        q_nope = xq @ orc.W["w_q"][h * dn:(h + 1) * dn].T
        q_abs = q_nope @ orc.W["w_uk"][h * dn:(h + 1) * dn]
        q_rope = rope3d(xq @ orc.W["w_qr"][h * dr:(h + 1) * dr].T, ctx["t_q"], ctx["h_q"], ctx["w_q"],
                        d["rope_t"], d["rope_h"], d["rope_w"], d["rope_base"])
        rows.append(np.concatenate([q_abs, q_rope], axis=1) * orc.scale * LOG2E)
    return np.stack(rows, axis=1).reshape(-1, 224)


def _slot(self, f, k):
    from mla_latent_kv_window_b200 import mla_ring_slot
    return mla_ring_slot(self.gpu.cfg, f, k)


Pair.gpu_slot = _slot


def full_check(pair: Pair, x_chunk, what: str, intermediates: bool = True):
    out = pair.attention(x_chunk)
    nq = x_chunk.shape[1]
    for b, orc in enumerate(pair.oracles):
        ref, parts = orc.attention(x_chunk[b], return_parts=True)
        assert_close(out[b], ref, f"{what}: out (stream {b})")
        if intermediates:
            nh = pair.dims["n_heads"]
            qp = pair.gpu.copy_buffer(0, (pair.w.batch, pair.gpu.cfg.max_chunk_frames * pair.F * nh, 224))
            assert_close(qp[b, :nq * nh], oracle_qp(pair, x_chunk[b], b), f"{what}: Qp (stream {b})")
            ol = pair.gpu.copy_buffer(1, (pair.w.batch, pair.gpu.cfg.max_chunk_frames * pair.F * nh, 192))
            # o_lat, the fp16 latent-space attention output, meets the same bar as the layer
            # output (worst observed max-abs/RMS 6.5e-3); the observed errors are printed
            # (pytest -s).
            rel_o, mx_o = assert_close(ol[b, :nq * nh], parts["Pc"].reshape(-1, 192),
                                       f"{what}: o_lat (stream {b})")
            print(f"o_lat parity [{what}, stream {b}]: rel L2 {rel_o:.3e}, max-abs/RMS {mx_o:.3e}")
    pair.check_status()
    return out


# ---------------------------------------------------------------------------- small, every element
def test_tiny_layer_full():
    w = mla_synth.WORKLOADS["tiny"]
    p = Pair(w)
    p.append(p.hidden(w.fill_frames, mla_synth.fill_seed(w, 0)))
    check_ring(p, "tiny")
    full_check(p, p.hidden(w.query_frames, mla_synth.chunk_seed(w, 0, 0)), "tiny")


def test_ring_wrap_and_bulk_append():
    w = small(window=3, q=2, seed=11)
    p = Pair(w, max_chunk_frames=2)
    seed = 500
    for n in (2, 2, 5, 1):          # wraps twice; the 5-frame append is larger than the window
        p.append(p.hidden(n, seed))
        seed += 1
        check_ring(p, f"after append of {n}")
    assert p.gpu.state() == (10, 3)
    full_check(p, p.hidden(2, seed), "wrapped window, 2-frame chunk")


def test_empty_window_attends_to_chunk_only():
    w = small(window=3, q=1, seed=12)
    p = Pair(w)
    assert p.gpu.state() == (0, 0)
    full_check(p, p.hidden(1, 900), "empty window")


def test_partial_window():
    w = small(window=3, q=2, seed=13)
    p = Pair(w, max_chunk_frames=2)
    p.append(p.hidden(1, 901))
    full_check(p, p.hidden(2, 902), "one of three frames valid")
    p.append(p.hidden(1, 903))
    full_check(p, p.hidden(1, 904), "two of three frames valid")


def test_multi_tile_ragged():
    # F = 200: 1000 keys = 7 full 128-key tiles + 104; R = 400 tokens x 12 heads = 37.5 row tiles.
    w = small(frame_h=10, frame_w=20, window=3, fill=4, q=2, seed=14)
    p = Pair(w, max_chunk_frames=2)
    p.append(p.hidden(4, 905))
    check_ring(p, "ragged")
    full_check(p, p.hidden(2, 906), "ragged multi-tile")


def test_batched_streams_with_scales():
    w = small(frame_h=6, frame_w=7, window=2, fill=3, q=1, batch=3, seed=15, scale=True)
    p = Pair(w)
    p.append(p.hidden(3, 907))
    check_ring(p, "batched")
    full_check(p, p.hidden(1, 908), "batched streams")


def test_repeated_calls_same_cache():
    # Several denoising steps over one window, then the chunk is appended (the rollout pattern).
    w = small(window=2, q=1, seed=16)
    p = Pair(w)
    p.append(p.hidden(2, 909))
    for s in range(3):
        full_check(p, p.hidden(1, 910 + s), f"step {s}", intermediates=False)
    x = p.hidden(1, 913)
    full_check(p, x, "last step", intermediates=False)
    p.append(x)
    check_ring(p, "after chunk append")
    full_check(p, p.hidden(1, 914), "next chunk")


def test_invalid_calls_change_nothing():
    from mla_latent_kv_window_b200 import MLAError
    w = small(window=2, q=1, seed=17)
    p = Pair(w)
    p.append(p.hidden(2, 915))
    with pytest.raises(MLAError):
        p.gpu.attention(p.hidden(2, 916).cuda())          # 2 frames > max_chunk_frames = 1
    with pytest.raises(ValueError):
        p.gpu.attention(p.hidden(1, 917).cuda().float())  # wrong dtype, rejected in marshalling
    assert p.gpu.state() == (2, 2)
    full_check(p, p.hidden(1, 918), "after rejected calls", intermediates=False)


# ---------------------------------------------------------------------------- full-size, sampled rows
def sampled_check(pair: Pair, x_chunk, what: str, n_rows: int, seed: int):
    out = pair.attention(x_chunk)
    nq = x_chunk.shape[1]
    rng = np.random.default_rng(seed)
    worst = (0.0, 0.0)
    for b, orc in enumerate(pair.oracles):
        rows = np.sort(rng.choice(nq, size=min(n_rows, nq), replace=False))
        ref = orc.attention(x_chunk[b], rows=rows)
        rel, mx = assert_close(out[b][rows], ref, f"{what}: out rows (stream {b})")
        worst = (max(worst[0], rel), max(worst[1], mx))
        assert torch.isfinite(out[b].float()).all()
    pair.check_status()
    return worst


def test_wan_w21_q1_full_size():
    # The benchmarked workload, every element: all 21 ring frames (32,760 rows of c_kv and
    # k_rope), the absorbed queries and the layer output for all 1,560 query tokens.  (o_lat is
    # compared element by element on the small workloads; here the oracle's per-head softmax
    # matrices would take 5 GB.)
    w = mla_synth.WORKLOADS["wan_w21_q1"]
    p = Pair(w)
    p.append(p.hidden(w.fill_frames, mla_synth.fill_seed(w, 0)))
    check_ring(p, "21-frame fill")
    x = p.hidden(1, mla_synth.chunk_seed(w, 0, 0))
    out = p.attention(x)
    nh = p.dims["n_heads"]
    qp = p.gpu.copy_buffer(0, (1, w.F * nh, 224))
    assert_close(qp[0], oracle_qp(p, x[0], 0), "21-frame window: Qp, every row")
    assert_close(out[0], p.oracles[0].attention(x[0]), "21-frame window: out, every element")
    assert torch.isfinite(out.float()).all()
    p.check_status()


def test_wan_b4_w21_q3_full_size():
    w = mla_synth.WORKLOADS["wan_b4_w21_q3"]
    p = Pair(w)
    p.append(p.hidden(w.fill_frames, mla_synth.fill_seed(w, 0)))
    sampled_check(p, p.hidden(3, mla_synth.chunk_seed(w, 0, 0)), "B=4 streams", 256, 3)


def test_wan_w63_q1_full_size():
    # The 63-frame window (98,280 cached tokens + the chunk), every output element.
    w = mla_synth.WORKLOADS["wan_w63_q1"]
    p = Pair(w)
    p.append(p.hidden(w.fill_frames, mla_synth.fill_seed(w, 0)))
    x = p.hidden(1, mla_synth.chunk_seed(w, 0, 0))
    out = p.attention(x)
    assert_close(out[0], p.oracles[0].attention(x[0]), "63-frame window: out, every element")
    assert torch.isfinite(out.float()).all()
    p.check_status()


def test_wan_30_layers_4_steps_wrapped():
    # 30 independent layers; each: append 24 frames (the ring wraps once, frames 3..23 stay), four
    # denoising steps with a fresh 3-frame chunk over the same window, then the step-4 chunk is
    # appended (even layers: mla_cache_append of its hidden states; odd layers: mla_cache_commit
    # of the latents the last step computed).  The oracle checks 256 sampled rows at 8
    # layer-steps spread over layers and steps; every layer's output must be finite and its
    # status word clean.
    w = mla_synth.WORKLOADS["wan_30l_w21_q3_wrap"]
    checked = {0: (0, 3), 7: (1,), 13: (2,), 19: (1, 2), 29: (0, 3)}
    for layer in range(w.layers):
        p = Pair(w, layer=layer)
        oracle_on = layer in checked
        p.append(p.hidden(w.fill_frames, mla_synth.fill_seed(w, layer)), oracle=oracle_on)
        assert p.gpu.state() == (24, 21)
        x = None
        for step in range(w.steps):
            x = p.hidden(w.query_frames, mla_synth.chunk_seed(w, layer, step))
            if oracle_on and step in checked[layer]:
                sampled_check(p, x, f"layer {layer} step {step}", 256, 100 * layer + step)
            else:
                out = p.attention(x)
                assert torch.isfinite(out.float()).all()
        if layer % 2:
            p.gpu.commit(w.query_frames)
            if oracle_on:
                p.oracles[0].append(x[0])
        else:
            p.append(x, oracle=oracle_on)
        assert p.gpu.state() == (27, 21)
        if oracle_on:
            ckv, kr, _ = p.gpu.read_ring(0)
            f, c, r = p.oracles[0].cache_contents()[-1]
            assert f == 26
            s0 = ring_slot(f, 0, w.window_frames, w.F)
            assert_close(ckv[s0:s0 + w.F], c, "appended chunk c_kv")
            assert_close(kr[s0:s0 + w.F], r, "appended chunk k_rope")
        p.check_status()
        p.gpu.close()


# ---------------------------------------------------------------------------- next rows
def test_paper_dims_tiny():
    # [VideoMLA] §4.1 defaults: 96/32 key split (scale 1/sqrt(128)), low-rank query d_q = 768,
    # RoPE (6,5,5) pairs; every element against the oracle's low-rank path.
    w = mla_synth.WORKLOADS["paper_tiny"]
    p = Pair(w)
    p.append(p.hidden(w.fill_frames, mla_synth.fill_seed(w, 0)))
    check_ring(p, "paper dims")
    full_check(p, p.hidden(w.query_frames, mla_synth.chunk_seed(w, 0, 0)), "paper dims")


def test_paper_dims_w21_full_size():
    w = mla_synth.WORKLOADS["paper_w21_q1"]
    p = Pair(w)
    p.append(p.hidden(w.fill_frames, mla_synth.fill_seed(w, 0)))
    sampled_check(p, p.hidden(1, mla_synth.chunk_seed(w, 0, 0)), "paper dims, 21-frame window", 64, 5)


def test_sink_tiny_through_wraps():
    # 1 sink frame + a 2-frame window: appends of 1, 1, 3 and 1 frames (the window slides and
    # wraps while frame 0 stays); every element checked after each stage, including a chunk that
    # sees the sink, the window and itself at App. D.5 window-local positions.
    w = mla_synth.WORKLOADS["sink_tiny"]
    p = Pair(w, max_chunk_frames=2)
    seed = 700
    for n in (1, 1, 3, 1):
        p.append(p.hidden(n, seed))
        seed += 1
        check_ring(p, f"sink: after append of {n}")
        full_check(p, p.hidden(2, seed), f"sink: chunk after append of {n}")
        seed += 1
    assert p.gpu.state() == (6, 3)


def test_sink_ragged_tiles():
    # F = 200 (sink region padded from 200 to 256 rows), window of 3, 2-frame chunks.
    w = mla_synth.Workload("sink_ragged", frame_h=10, frame_w=20, window_frames=3, fill_frames=6,
                           query_frames=2, seed=19, sink_frames=1)
    p = Pair(w, max_chunk_frames=2)
    p.append(p.hidden(6, 720))
    check_ring(p, "sink ragged")
    full_check(p, p.hidden(2, 721), "sink ragged")


def test_sink_w6_q3_full_size():
    # The long-rollout configuration: 1 sink frame + 6 recent frames (10,920 cached keys) and a
    # 3-frame chunk, after 10 appended frames (the window has wrapped).
    w = mla_synth.WORKLOADS["sink_w6_q3"]
    p = Pair(w)
    p.append(p.hidden(w.fill_frames, mla_synth.fill_seed(w, 0)))
    assert p.gpu.state() == (10, 7)
    ckv, kr, n = p.gpu.read_ring(0)
    contents = p.oracles[0].cache_contents()
    assert [f for f, _, _ in contents] == [0, 4, 5, 6, 7, 8, 9]
    for f, c, r in (contents[0], contents[1], contents[-1]):
        s0 = p.gpu_slot(f, 0)
        assert_close(ckv[s0:s0 + w.F], c, f"c_kv frame {f}")
        assert_close(kr[s0:s0 + w.F], r, f"k_rope frame {f}")
    sampled_check(p, p.hidden(3, mla_synth.chunk_seed(w, 0, 0)), "sink + 6-frame window", 64, 6)


def test_sink_batched_scaled_streams():
    # Two streams, each with its own sink frame, window and hidden-state scale in [0.5, 2]
    # (sharper softmax for the larger one): every element after the window has slid.
    w = mla_synth.Workload("sink_b2", frame_h=4, frame_w=6, window_frames=2, fill_frames=5,
                           query_frames=2, batch=2, seed=21, sink_frames=1, stream_scale=True)
    p = Pair(w, max_chunk_frames=2)
    p.append(p.hidden(2, 730))
    full_check(p, p.hidden(2, 731), "sink, 2 scaled streams, window filling")
    p.append(p.hidden(3, 732))
    check_ring(p, "sink, 2 scaled streams")
    full_check(p, p.hidden(2, 733), "sink, 2 scaled streams, slid window")


def test_sink_w6_q3_two_streams_sampled():
    # The long-rollout configuration with B = 2 scaled streams: sampled rows of each stream.
    base = mla_synth.WORKLOADS["sink_w6_q3"]
    w = mla_synth.Workload("sink_w6_q3_b2", frame_h=base.frame_h, frame_w=base.frame_w,
                           window_frames=base.window_frames, fill_frames=base.fill_frames,
                           query_frames=base.query_frames, batch=2, seed=6100, sink_frames=1,
                           stream_scale=True)
    p = Pair(w)
    p.append(p.hidden(w.fill_frames, mla_synth.fill_seed(w, 0)))
    assert p.gpu.state() == (10, 7)
    sampled_check(p, p.hidden(3, mla_synth.chunk_seed(w, 0, 0)), "sink + 6-frame window, B = 2", 64, 7)


# ---------------------------------------------------------------------------- reconstruct-then-dense
def reconstruct_check(pair: Pair, x_chunk, what: str, rows=None):
    out = pair.gpu.attention_reconstruct(x_chunk.cuda())
    torch.cuda.synchronize()
    out = out.cpu()
    for b, orc in enumerate(pair.oracles):
        if rows is None:
            assert_close(out[b], orc.attention(x_chunk[b]), f"{what}: out (stream {b})")
        else:
            assert_close(out[b][rows], orc.attention(x_chunk[b], rows=rows), f"{what}: out rows (stream {b})")
    pair.check_status()
    return out


def test_reconstruct_dense_paper_tiny():
    # The training-time form ([VideoMLA] §3.3): per-head K/V materialised from the latent, dense
    # attention, W_O.  Every element against the oracle, and against the absorbed path.
    w = mla_synth.WORKLOADS["paper_tiny"]
    p = Pair(w)
    p.append(p.hidden(w.fill_frames, mla_synth.fill_seed(w, 0)))
    x = p.hidden(w.query_frames, mla_synth.chunk_seed(w, 0, 0))
    dense = reconstruct_check(p, x, "reconstruct (paper tiny)")
    absorbed = p.attention(x)
    assert_close(dense, absorbed.float().numpy(), "reconstruct vs absorbed")


def test_reconstruct_dense_ragged_batched():
    # F = 200 tokens: 600 + 400 keys (ragged 128-key tiles), 400 query rows, 2 streams.
    w = mla_synth.Workload("paper_ragged", frame_h=10, frame_w=20, window_frames=3, fill_frames=4,
                           query_frames=2, batch=2, seed=29,
                           dims=tuple(sorted(mla_synth.DIMS_PAPER.items())))
    p = Pair(w, max_chunk_frames=2)
    p.append(p.hidden(4, 730))
    reconstruct_check(p, p.hidden(2, 731), "reconstruct (ragged, batched)")


def test_reconstruct_dense_paper_w21_full_size():
    w = mla_synth.WORKLOADS["paper_w21_q1"]
    p = Pair(w)
    p.append(p.hidden(w.fill_frames, mla_synth.fill_seed(w, 0)))
    rows = np.sort(np.random.default_rng(7).choice(w.F, size=48, replace=False))
    reconstruct_check(p, p.hidden(1, mla_synth.chunk_seed(w, 0, 0)), "reconstruct (21-frame window)", rows)


def test_reconstruct_dense_unsupported_configs():
    from mla_latent_kv_window_b200 import MLAError
    for w in (small(window=2, q=1, seed=30),                       # d_nope + d_rope = 160
              mla_synth.WORKLOADS["sink_tiny"]):                    # sink frames
        p = Pair(w, max_chunk_frames=1)
        p.append(p.hidden(2, 740))
        with pytest.raises(MLAError, match="UNSUPPORTED"):
            p.gpu.attention_reconstruct(p.hidden(1, 741).cuda())
        p.check_status()


# ---------------------------------------------------------------------------- degenerate and other shapes
def test_single_token_frames_single_key():
    # F = 1 (a 1 x 1 frame grid) and an empty window: one query attends to exactly one key, its own
    # latent, so the output is the value projection of that latent (the oracle's single-key case).
    w = mla_synth.Workload("one_token", frame_h=1, frame_w=1, window_frames=1, fill_frames=0,
                           query_frames=1, seed=31)
    p = Pair(w)
    full_check(p, p.hidden(1, 760), "one key")
    p.append(p.hidden(1, 761))
    check_ring(p, "one-token frame")
    full_check(p, p.hidden(1, 762), "two keys")


def test_narrower_model_four_heads():
    # hidden 512 = 4 heads x 128: other column-block counts in the projections (4 + 1 blocks of
    # 224, 512 / 192 output blocks with a ragged last one) and 4-head query rows.
    dims = dict(mla_synth.DIMS_WAN13B, hidden=512, n_heads=4)
    w = mla_synth.Workload("narrow_model", frame_h=6, frame_w=10, window_frames=3, fill_frames=4,
                           query_frames=2, seed=32, dims=tuple(sorted(dims.items())))
    p = Pair(w, max_chunk_frames=2)
    p.append(p.hidden(4, 763))
    check_ring(p, "4 heads")
    full_check(p, p.hidden(2, 764), "4 heads")


def test_two_sink_frames_partly_filled_then_sliding():
    # sink_frames = 2 with F = 200: the sink region is 400 rows padded to 512 (4 key tiles).
    # After one append only one sink frame exists, so two whole key tiles are padding (every key
    # masked; CTAs that start their key walk there must not produce NaN); then the sink fills, the
    # window (W = 2) fills and slides, and the query's temporal bands turn for the sink keys.
    w = mla_synth.Workload("two_sinks", frame_h=10, frame_w=20, window_frames=2, fill_frames=1,
                           query_frames=1, seed=33, sink_frames=2)
    p = Pair(w)
    seed = 770
    for n in (1, 2, 2):
        p.append(p.hidden(n, seed))
        seed += 1
        check_ring(p, f"two sinks: after append of {n}")
        full_check(p, p.hidden(1, seed), f"two sinks: chunk after append of {n}")
        seed += 1
    assert p.gpu.state() == (5, 4)
