"""Pins of the fp64 oracle against what the VideoMLA paper page and the mathematics fix.

None of these tests compares the oracle with itself: each checks it against a
number printed on the pages (tests/golden/accounting.json), a closed form, an
invariant, a special case that reduces to a library routine, or the independent
scalar brute force in tests/brute_mla.py.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import mla_synth
from oracle import (OracleLayer, cache_scalars, dense_mha, dense_scalars_per_token,
                    latent_scalars_per_token, ring_slot, rope3d, rope_bands, valid_frames)
from tests import brute_mla

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _dims(**over):
    d = dict(mla_synth.DIMS_WAN13B)
    d.update(over)
    return d


def _tiny_dims(**over):
    d = dict(hidden=10, n_heads=2, d_head=3, d_nope=4, d_latent=3, d_rope=6,
             rope_t=2, rope_h=2, rope_w=2, rope_base=10000.0,
             frame_h=2, frame_w=2, window_frames=2)
    d.update(over)
    return d


def _layer(dims, seed=0, **scale):
    w = mla_synth.make_weights(dims, seed)
    return OracleLayer(dims, w, **scale), w


# ---------------------------------------------------------------------------- accounting (closed form)
def test_accounting_matches_printed_numbers():
    g = json.load(open(os.path.join(GOLDEN, "accounting.json")))
    d = g["dims"]
    dense = dense_scalars_per_token(d["n_heads"], d["d_head"])
    lat = latent_scalars_per_token(d["d_latent"], d["d_rope"])
    assert dense == g["dense_scalars_per_token"]["value"]
    assert lat == g["latent_scalars_per_token"]["value"]
    assert round(100 * (1 - lat / dense), 1) == g["reduction_percent"]["value"]
    assert round(dense / lat, 1) == g["reduction_factor"]["value"]
    total = cache_scalars(d["layers"], d["window_frames"], d["tokens_per_frame"], dense)
    assert total == 3_019_161_600
    assert round(total / 1e9, 2) == g["dense_cache_scalars_billions"]["value"]
    assert round(total * 2 / 1e9, 1) == g["dense_cache_gb_bf16"]["value"]
    assert d["frame_h"] * d["frame_w"] == d["tokens_per_frame"]
    assert d["window_frames"] * d["tokens_per_frame"] == d["clip_tokens"]
    scd_layers, all_layers = g["scd_caching_layers"]["value"], g["scd_caching_layers"]["of"]
    assert round(100 * (1 - scd_layers / all_layers), 1) == g["scd_reduction_percent"]["value"]
    scd = cache_scalars(scd_layers, d["window_frames"], d["tokens_per_frame"], dense)
    ours = cache_scalars(all_layers, d["window_frames"], d["tokens_per_frame"], lat)
    assert round(scd / ours, 1) == g["vs_scd_factor"]["value"]
    assert d["tokens_per_frame"] == g["sink_slots"]["value"]
    assert 6 * d["tokens_per_frame"] == g["local_window_slots"]["value"]


def test_long_window_equals_dense_frames():
    # 63 latent frames of 224-scalar tokens hold as much as ~4.6 dense-KV frames of 3072 scalars.
    lat = latent_scalars_per_token(192, 32)
    dense = dense_scalars_per_token(12, 128)
    assert round(63 * 1560 * lat / (1560 * dense), 2) == 4.59


# ---------------------------------------------------------------------------- RoPE
def test_rope_first_band_closed_form():
    # Pair 0 of each axis turns at frequency 1: a unit vector at position p rotates by p radians,
    # counter-clockwise, and only that axis's channels move.
    split = (8, 12, 12)
    for axis, first_ch in ((0, 0), (1, 8), (2, 20)):
        v = np.zeros(32)
        v[first_ch] = 1.0
        pos = [0, 0, 0]
        pos[axis] = 3
        out = rope3d(v, *pos, *split, 10000.0)
        exp = np.zeros(32)
        exp[first_ch] = math.cos(3.0)
        exp[first_ch + 1] = math.sin(3.0)
        np.testing.assert_allclose(out, exp, atol=1e-15)


def test_rope_band_frequencies():
    axes, freqs = rope_bands(8, 12, 12, 10000.0)
    assert list(axes) == [0] * 4 + [1] * 6 + [2] * 6
    np.testing.assert_allclose(freqs[:4], [10000.0 ** (-2 * i / 8) for i in range(4)], rtol=1e-15)
    np.testing.assert_allclose(freqs[4:10], [10000.0 ** (-2 * i / 12) for i in range(6)], rtol=1e-15)
    assert freqs[0] == freqs[4] == freqs[10] == 1.0       # highest band first on every axis
    assert np.all(np.diff(freqs[4:10]) < 0)


def test_rope_identity_at_origin_and_norm():
    rng = np.random.default_rng(1)
    v = rng.standard_normal((50, 32))
    np.testing.assert_array_equal(rope3d(v, 0, 0, 0, 8, 12, 12, 1e4), v)
    t, h, w = rng.integers(0, 900, 50), rng.integers(0, 30, 50), rng.integers(0, 52, 50)
    out = rope3d(v, t, h, w, 8, 12, 12, 1e4)
    np.testing.assert_allclose(np.linalg.norm(out, axis=1), np.linalg.norm(v, axis=1), rtol=1e-13)


@pytest.mark.parametrize("split", [(8, 12, 12), (12, 10, 10), (2, 2, 2)])
def test_rope_relative_shift_invariance(split):
    rng = np.random.default_rng(2)
    d = sum(split)
    q, k = rng.standard_normal((40, d)), rng.standard_normal((40, d))
    pq = rng.integers(0, 60, (3, 40))
    pk = rng.integers(0, 60, (3, 40))
    base = np.einsum("nd,nd->n", rope3d(q, *pq, *split, 1e4), rope3d(k, *pk, *split, 1e4))
    for delta in ([5, 0, 0], [0, 7, 0], [0, 0, 11], [123, 4, 9]):
        dd = np.array(delta)[:, None]
        s = np.einsum("nd,nd->n", rope3d(q, *(pq + dd), *split, 1e4), rope3d(k, *(pk + dd), *split, 1e4))
        np.testing.assert_allclose(s, base, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------------------- attention structure
def _tiny_run(dims=None, seed=3, window=2, fill=3, q_frames=1):
    dims = dims or _tiny_dims(window_frames=window)
    layer, w = _layer(dims, seed)
    F = dims["frame_h"] * dims["frame_w"]
    x_fill = mla_synth.make_hidden(1, fill * F, dims["hidden"], seed + 100)[0]
    x_q = mla_synth.make_hidden(1, q_frames * F, dims["hidden"], seed + 200)[0]
    if fill:
        layer.append(x_fill)
    return layer, w, x_fill, x_q


def test_absorbed_equals_unabsorbed_scores():
    layer, w, _, x_q = _tiny_run(_dims(frame_h=3, frame_w=4, window_frames=3), fill=4)
    out, parts = layer.attention(x_q, return_parts=True)
    ctx = parts["ctx"]
    for h in range(layer.d["n_heads"]):
        Q, K, _ = layer.head_qkv(ctx, h)
        s_unabs = (Q @ K.T) * layer.scale
        s_abs = layer.absorbed_scores(x_q, h)
        np.testing.assert_allclose(s_abs, s_unabs, rtol=1e-12, atol=1e-12 * np.abs(s_unabs).max())


def test_softmax_rows_sum_to_one():
    layer, _, _, x_q = _tiny_run(_dims(frame_h=3, frame_w=4, window_frames=2), fill=3)
    _, parts = layer.attention(x_q, return_parts=True)
    P = parts["P"]
    assert np.all(P >= 0)
    np.testing.assert_allclose(P.sum(axis=-1), 1.0, atol=1e-12)


def test_single_key_returns_value_projection():
    # Empty window and a one-token chunk: the only key is the token itself, softmax is exactly 1,
    # so out = concat_h(c W_UV[h]^T) W_O^T.
    dims = _dims(frame_h=1, frame_w=1, window_frames=1)
    layer, w = _layer(dims, 5)
    x = mla_synth.make_hidden(1, 1, dims["hidden"], 9)[0]
    out = layer.attention(x)
    xf = x.double().numpy()
    c = xf @ w["w_dkv"].double().numpy().T
    v = c @ w["w_uv"].double().numpy().T          # all heads at once: [n_h * d_head]
    np.testing.assert_allclose(out, v @ w["w_o"].double().numpy().T, rtol=1e-12, atol=1e-12)


def test_zero_query_attends_uniformly():
    dims = _dims(frame_h=2, frame_w=3, window_frames=2)
    w = mla_synth.make_weights(dims, 6)
    w["w_q"] = torch.zeros_like(w["w_q"])
    w["w_qr"] = torch.zeros_like(w["w_qr"])
    layer = OracleLayer(dims, w)
    xf = mla_synth.make_hidden(1, 12, dims["hidden"], 10)[0]
    xq = mla_synth.make_hidden(1, 6, dims["hidden"], 11)[0]
    layer.append(xf)
    out = layer.attention(xq)
    allx = np.concatenate([xf.double().numpy(), xq.double().numpy()])
    vmean = (allx @ w["w_dkv"].double().numpy().T @ w["w_uv"].double().numpy().T).mean(axis=0)
    exp = np.broadcast_to(vmean @ w["w_o"].double().numpy().T, out.shape)
    np.testing.assert_allclose(out, exp, rtol=1e-11, atol=1e-12)


def test_reduces_to_textbook_mha_via_sdpa():
    # d_rope = 0 and W_UK = W_UV = identity (d_c = n_h d_h): per-head keys and values are slices of
    # the latent, and the layer is textbook MHA; compare with torch's SDPA in float64.
    nh, dh, F = 3, 4, 6
    dims = dict(hidden=12, n_heads=nh, d_head=dh, d_nope=dh, d_latent=nh * dh, d_rope=0,
                rope_t=0, rope_h=0, rope_w=0, rope_base=1e4, frame_h=2, frame_w=3, window_frames=2)
    w = mla_synth.make_weights(dims, 7)
    eye = torch.eye(nh * dh, dtype=torch.bfloat16)
    w["w_uk"], w["w_uv"] = eye.clone(), eye.clone()
    w["w_qr"] = torch.zeros(0, 12, dtype=torch.bfloat16)
    w["w_kr"] = torch.zeros(0, 12, dtype=torch.bfloat16)
    layer = OracleLayer(dims, w)
    xf = mla_synth.make_hidden(1, 3 * F, 12, 12)[0]
    xq = mla_synth.make_hidden(1, F, 12, 13)[0]
    layer.append(xf)
    out = layer.attention(xq)
    X = torch.cat([xf[F:], xq]).double()                         # window keeps the last 2 frames
    kv = (X @ w["w_dkv"].double().T).view(-1, nh, dh).transpose(0, 1)        # [nh, N, dh]
    q = (xq.double() @ w["w_q"].double().T).view(-1, nh, dh).transpose(0, 1)
    o = torch.nn.functional.scaled_dot_product_attention(q, kv, kv)          # scale 1/sqrt(dh)
    ref = o.transpose(0, 1).reshape(F, nh * dh) @ w["w_o"].double().T
    np.testing.assert_allclose(out, ref.numpy(), rtol=1e-11, atol=1e-12)


def test_dense_mha_matches_sdpa():
    g = torch.Generator().manual_seed(4)
    q = torch.randn(7, 3, 5, generator=g, dtype=torch.float64)
    k = torch.randn(11, 3, 5, generator=g, dtype=torch.float64)
    v = torch.randn(11, 3, 4, generator=g, dtype=torch.float64)
    ref = torch.nn.functional.scaled_dot_product_attention(q.transpose(0, 1), k.transpose(0, 1), v.transpose(0, 1))
    np.testing.assert_allclose(dense_mha(q, k, v, 1 / math.sqrt(5)), ref.transpose(0, 1).numpy(), rtol=1e-12)


def test_brute_force_tiny():
    dims = _tiny_dims()
    layer, w, x_fill, x_q = _tiny_run(dims, seed=21, window=2, fill=3, q_frames=2)
    out = layer.attention(x_q)
    F = 4
    Wl = {k: v.double().tolist() for k, v in w.items()}
    frames = [x_fill[i * F:(i + 1) * F].double().tolist() for i in range(3)][-2:]
    chunk = [x_q[i * F:(i + 1) * F].double().tolist() for i in range(2)]
    ref = np.array(brute_mla.attention(dims, Wl, frames, chunk))
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)


def test_brute_force_paper_rope_split():
    # The paper's own (6,5,5)-pair split ([VideoMLA] §4.1) through the same brute force.
    dims = _tiny_dims(d_rope=12, rope_t=4, rope_h=4, rope_w=4, d_nope=2)
    layer, w, x_fill, x_q = _tiny_run(dims, seed=22, window=2, fill=1, q_frames=1)
    out = layer.attention(x_q)
    Wl = {k: v.double().tolist() for k, v in w.items()}
    ref = np.array(brute_mla.attention(dims, Wl, [x_fill.double().tolist()], [x_q.double().tolist()]))
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)


def test_local_positions_equal_absolute_without_sink():
    # App. D.5 re-indexing shifts every temporal coordinate by one offset; RoPE scores depend on
    # differences only, so absolute positions give the same output when there is no sink.
    layer, _, _, x_q = _tiny_run(_dims(frame_h=2, frame_w=3, window_frames=3), fill=7, q_frames=2)
    a = layer.attention(x_q, positions="local")
    b = layer.attention(x_q, positions="absolute")
    np.testing.assert_allclose(a, b, rtol=1e-10, atol=1e-12)


def test_key_order_is_irrelevant():
    # Softmax attention is invariant under a permutation of the keys (the GPU walks ring slots in
    # physical order): permute the assembled keys and recompute one head.
    layer, _, _, x_q = _tiny_run(_dims(frame_h=2, frame_w=3, window_frames=3), fill=5)
    ctx = layer.keys_and_queries(x_q)
    Q, K, V = layer.head_qkv(ctx, 1)
    perm = np.random.default_rng(0).permutation(K.shape[0])

    def att(K, V):
        S = Q @ K.T * layer.scale
        E = np.exp(S - S.max(1, keepdims=True))
        return (E / E.sum(1, keepdims=True)) @ V
    np.testing.assert_allclose(att(K[perm], V[perm]), att(K, V), rtol=1e-12, atol=1e-14)


def test_rows_subset_is_exact():
    layer, _, _, x_q = _tiny_run(_dims(frame_h=3, frame_w=4, window_frames=2), fill=2)
    full = layer.attention(x_q)
    rows = np.array([0, 5, 11])
    np.testing.assert_allclose(layer.attention(x_q, rows=rows), full[rows], rtol=1e-13)


def test_window_keeps_newest_frames():
    dims = _tiny_dims(window_frames=3)
    layer, _ = _layer(dims, 1)
    x = mla_synth.make_hidden(1, 7 * 4, dims["hidden"], 2)[0]
    layer.append(x[:8])
    layer.append(x[8:])
    assert layer.frames_appended == 7
    assert [f for f, _, _ in layer.frames] == [4, 5, 6]
    c, _ = layer.latent(x[16:20])
    np.testing.assert_array_equal(layer.frames[0][1], c)


# ---------------------------------------------------------------------------- ring slot mapping
def test_ring_slot_matches_fifo_simulation():
    # A FIFO of W frame buffers: a new frame takes a fresh buffer until all W are used, then the
    # buffer of the frame it evicts.  The closed form (f mod W) F + k must name the same slot.
    from collections import deque
    F, W = 5, 4
    fifo, owner, fresh, appended = deque(), {}, 0, 0
    for n in [1, 2, 1, 3, 9, 2, 4, 1, 1, 5]:
        for _ in range(n):
            if len(fifo) == W:
                buf = owner.pop(fifo.popleft())
            else:
                buf, fresh = fresh, fresh + 1
            owner[appended] = buf
            fifo.append(appended)
            appended += 1
        assert valid_frames(appended, W) == len(fifo)
        for f in fifo:
            for k in (0, 3, F - 1):
                assert ring_slot(f, k, W, F) == owner[f] * F + k
    assert appended == 29


# ---------------------------------------------------------------------------- next rows: low-rank query, sink
def test_brute_force_low_rank_query():
    # [VideoMLA] §4.1's low-rank query (x -> c_q = W_DQ x -> W_Q c_q, W_QR c_q) with the paper's
    # 96/32-style split and (6,5,5)-style pairs, shrunk: the oracle against the scalar loops.
    dims = _tiny_dims(d_q=5, d_nope=3, d_rope=12, rope_t=4, rope_h=4, rope_w=4)
    layer, w, x_fill, x_q = _tiny_run(dims, seed=23, window=2, fill=3, q_frames=1)
    assert "w_dq" in w and tuple(w["w_q"].shape) == (2 * 3, 5)
    out = layer.attention(x_q)
    F = 4
    Wl = {k: v.double().tolist() for k, v in w.items()}
    frames = [x_fill[i * F:(i + 1) * F].double().tolist() for i in range(3)][-2:]
    ref = np.array(brute_mla.attention(dims, Wl, frames, [x_q.double().tolist()]))
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)


def test_low_rank_query_equals_composed_full_rank():
    # A low-rank query is a full-rank one with W_Q = W_UQ W_DQ and W_QR = W_QR' W_DQ (matrix
    # associativity): the two code paths of the oracle must agree in fp64.
    dims = _dims(frame_h=2, frame_w=3, window_frames=2, hidden=64, n_heads=2, d_head=16, d_nope=12,
                 d_q=24)
    lr, w, x_fill, x_q = _tiny_run(dims, seed=24, window=2, fill=3, q_frames=1)
    wf = {k: v.double() for k, v in w.items() if k != "w_dq"}
    wf["w_q"] = w["w_q"].double() @ w["w_dq"].double()
    wf["w_qr"] = w["w_qr"].double() @ w["w_dq"].double()
    fr_dims = dict(dims)
    fr_dims.pop("d_q")
    fr = OracleLayer(fr_dims, wf)
    fr.append(x_fill)
    np.testing.assert_allclose(lr.attention(x_q), fr.attention(x_q), rtol=1e-11, atol=1e-13)


def test_sink_and_window_bookkeeping():
    # App. D.4/D.5: the first sink_frames frames stay for good; the window keeps the newest W of
    # the others.  Frame lists after each append, against a direct statement of that rule.
    dims = _tiny_dims(window_frames=2, sink_frames=1)
    layer, _ = _layer(dims, 3)
    x = mla_synth.make_hidden(1, 9 * 4, dims["hidden"], 4)[0]
    seen = 0
    for n in (1, 1, 2, 4, 1):
        layer.append(x[seen * 4:(seen + n) * 4])
        seen += n
        assert [f for f, _, _ in layer.sink] == [0]
        assert [f for f, _, _ in layer.frames] == list(range(max(1, seen - 2), seen))
        assert [f for f, _, _ in layer.active_frames()] == [0] + list(range(max(1, seen - 2), seen))


def test_brute_force_sink():
    # One sink frame + a 2-frame window after 5 appended frames: the brute force gets the logical
    # key frames [0, 3, 4] written out by hand, numbered 0, 1, 2 (App. D.5), then the chunk.
    dims = _tiny_dims(window_frames=2, sink_frames=1)
    layer, w, x_fill, x_q = _tiny_run(dims, seed=25, window=2, fill=5, q_frames=2)
    out = layer.attention(x_q)
    F = 4
    Wl = {k: v.double().tolist() for k, v in w.items()}
    fr = [x_fill[i * F:(i + 1) * F].double().tolist() for i in range(5)]
    chunk = [x_q[i * F:(i + 1) * F].double().tolist() for i in range(2)]
    ref = np.array(brute_mla.attention(dims, Wl, [fr[0], fr[3], fr[4]], chunk))
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)


def test_sink_changes_the_absolute_reading():
    # With a sink and a slid window, absolute frame indices no longer differ from the local ones
    # by one shared offset, so the two readings give different outputs (the GPU must rotate the
    # query separately for the sink keys).
    dims = _tiny_dims(window_frames=2, sink_frames=1)
    layer, _, _, x_q = _tiny_run(dims, seed=26, window=2, fill=6, q_frames=1)
    a = layer.attention(x_q, positions="local")
    b = layer.attention(x_q, positions="absolute")
    assert np.max(np.abs(a - b)) > 1e-6


def test_sink_segment_rotation_equals_local():
    # The GPU keeps keys rotated at their absolute frame index and rotates the query at its
    # absolute index for window and chunk keys, but at its window-local index for sink keys
    # (RoPE(a) . RoPE(b) depends on a - b only).  Those scores equal the App. D.5 local ones.
    dims = _tiny_dims(window_frames=2, sink_frames=1)
    layer, _, _, x_q = _tiny_run(dims, seed=27, window=2, fill=6, q_frames=2)
    loc = layer.keys_and_queries(x_q, "local")
    ab = layer.keys_and_queries(x_q, "absolute")
    d = dims
    rope = lambda v, t, h, w: rope3d(v, t, h, w, d["rope_t"], d["rope_h"], d["rope_w"], d["rope_base"])
    n_sink_keys = layer.n_sink * 4
    for hd in range(d["n_heads"]):
        xq = layer.query_input(loc["x"])
        qr = xq @ layer.W["w_qr"][hd * d["d_rope"]:(hd + 1) * d["d_rope"]].T
        k_abs = rope(ab["r"], ab["t_key"], ab["h_key"], ab["w_key"])
        q_abs = rope(qr, ab["t_q"], ab["h_q"], ab["w_q"])
        q_loc = rope(qr, loc["t_q"], loc["h_q"], loc["w_q"])
        s_gpu = q_abs @ k_abs.T
        s_gpu[:, :n_sink_keys] = q_loc @ k_abs[:n_sink_keys].T
        k_loc = rope(loc["r"], loc["t_key"], loc["h_key"], loc["w_key"])
        np.testing.assert_allclose(s_gpu, q_loc @ k_loc.T, rtol=1e-10, atol=1e-12)



# ---------------------------------------------------------------------------- ring contents (rotate at append)
def _brute_ring_contents(dims, W, x_all, n_appended):
    """What a ring rotating at append time holds, written out with the scalar loops of
    tests/brute_mla.py: which frames survive is stated directly (the first sink_frames frames,
    then the newest window_frames of the rest), and each token's positional key is turned at its
    frame's ABSOLUTE index t = f and grid position (k // frame_w, k % frame_w)."""
    S, Wn = dims.get("sink_frames", 0), dims["window_frames"]
    F, fw = dims["frame_h"] * dims["frame_w"], dims["frame_w"]
    split = (dims["rope_t"], dims["rope_h"], dims["rope_w"])
    n_sink = min(n_appended, S)
    kept = list(range(n_sink)) + list(range(max(n_sink, n_appended - Wn), n_appended))
    out = []
    for f in kept:
        cs, rs = [], []
        for k in range(F):
            x = x_all[f * F + k]
            cs.append(brute_mla.matvec(W["w_dkv"], x))
            rs.append(brute_mla.rotate(brute_mla.matvec(W["w_kr"], x), f, k // fw, k % fw, split,
                                       dims["rope_base"]))
        out.append((f, cs, rs))
    return out


@pytest.mark.parametrize("sink", [0, 1, 2])
def test_cache_contents_brute_force_absolute_index(sink):
    # The GPU ring is checked against OracleLayer.cache_contents, so it is pinned here on its
    # own: after appends that slide the window (and wrap a 3-frame ring twice), every kept frame's
    # c_kv and k_rope (turned at the absolute frame index, App. D.5 read as "rotate at append")
    # must equal the scalar-loop statement above.  A non-square frame grid (2 x 3) and
    # unequal per-axis widths make an h/w swap or a wrong axis visible.
    dims = _tiny_dims(window_frames=3, frame_h=2, frame_w=3, sink_frames=sink, d_rope=8,
                      rope_t=2, rope_h=4, rope_w=2)
    layer, w = _layer(dims, 31 + sink)
    F = 6
    x = mla_synth.make_hidden(1, 12 * F, dims["hidden"], 40 + sink)[0]
    Wl = {k: v.double().tolist() for k, v in w.items()}
    xl = x.double().tolist()
    seen = 0
    for n in (2, 1, 5, 1, 3):
        layer.append(x[seen * F:(seen + n) * F])
        seen += n
        got = layer.cache_contents()
        ref = _brute_ring_contents(dims, Wl, xl, seen)
        assert [f for f, _, _ in got] == [f for f, _, _ in ref]
        for (f, c, r), (_, c_ref, r_ref) in zip(got, ref):
            np.testing.assert_allclose(c, np.array(c_ref), rtol=1e-13, atol=1e-13)
            np.testing.assert_allclose(r, np.array(r_ref), rtol=1e-13, atol=1e-13)
    assert seen == 12 and layer.frames_appended == 12


def test_head_subsets_add_up_to_the_full_output():
    # The output projection is linear in the per-head outputs, so attention restricted to a
    # subset of heads (used to time bounded samples) must give that subset's share of the output:
    # disjoint subsets covering every head add up to the full output.
    layer, _, _, x_q = _tiny_run(_dims(frame_h=2, frame_w=3, window_frames=2, hidden=256, n_heads=4,
                                       d_head=64, d_nope=64), fill=3)
    full = layer.attention(x_q)
    parts = layer.attention(x_q, heads=[0, 2]) + layer.attention(x_q, heads=[1]) + layer.attention(x_q, heads=[3])
    np.testing.assert_allclose(parts, full, rtol=1e-12, atol=1e-12)
