"""GPU: the fp16 range of the internal planes, and temporal positions far from the origin.

The cache planes and absorbed queries are fp16 (16-bit like the paper's bf16/fp16 cache,
[VideoMLA] §1).  A projected value beyond +-65504 is clamped and reported once by
mla_cache_sync as MLA_ERR_RANGE; values inside the range never set it.  Keys are rotated at
their absolute frame index, which after a minute-scale rollout ([VideoMLA] §4.2) or a long
stream is far from the window-local positions of App. D.5 that the oracle uses: parity there
checks the fp32 angle reduction of the rotation.
"""
import numpy as np
import pytest
import torch

import mla_synth
from oracle import rope3d
from tests.harness import Pair, assert_close, errors
from tests.test_gpu_parity import check_ring, full_check

pytestmark = pytest.mark.gpu


def small(frame_h=4, frame_w=6, window=2, fill=2, q=1, batch=1, seed=0, **kw):
    return mla_synth.Workload("small", frame_h=frame_h, frame_w=frame_w, window_frames=window,
                              fill_frames=fill, query_frames=q, batch=batch, seed=seed, **kw)


def test_outlier_tokens_set_the_range_flag_once():
    import mla_latent_kv_window_b200 as M
    w = small(window=2, seed=40)
    p = Pair(w)
    x = p.hidden(2, 4000).float()
    x[0, 5] *= 2.0e5            # one token whose latents are far beyond +-65504
    p.append(x.to(torch.bfloat16), oracle=False)
    torch.cuda.synchronize()
    assert M.mla_cache_sync(p.gpu.handle) == M.MLA_ERR_RANGE
    assert M.mla_cache_sync(p.gpu.handle) == 0          # reported once, then cleared
    # The clamped frame still gives finite outputs, and in-range work afterwards is clean.
    out = p.gpu.attention(p.hidden(1, 4001).cuda())
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all()
    assert M.mla_cache_sync(p.gpu.handle) == 0
    p.gpu.close()


def test_query_outlier_sets_the_range_flag():
    import mla_latent_kv_window_b200 as M
    w = small(window=2, seed=41)
    p = Pair(w)
    p.append(p.hidden(2, 4010), oracle=False)
    xq = p.hidden(1, 4011).float()
    xq[0, 3] *= 3.0e6           # absorbed query (and chunk latent) of one token out of range
    p.gpu.attention(xq.to(torch.bfloat16).cuda())
    torch.cuda.synchronize()
    assert M.mla_cache_sync(p.gpu.handle) == M.MLA_ERR_RANGE
    p.gpu.close()


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16).double().numpy()


def _f16(a):
    return np.asarray(a).astype(np.float16).astype(np.float64)


def _rounding_model(dims, W, x_fill, xq, wq="two_step"):
    """The absorbed path in float64 with a 16-bit rounding exactly where the library stores 16-bit
    values.  The query's latent part W_UK[h]^T W_Q[h] x is formed in one of four ways:
    wq="two_step" (the library's form for a full-rank query with d_nope = 128): q = W_Q[h] x in
    fp32, carried as an fp16 pair hi + lo into the product with W_UK[h] (fp16); "pair": the
    absorbed weight as a bf16 pair hi + lo (the library's form for other head splits);
    "single": the absorbed weight rounded to one bf16; "exact": float64.  Then the absorbed
    queries and the cache planes (fp16), P and o_lat (fp16), W_OV (fp16) and the output (bf16).
    Keys and queries are rotated at absolute frame indices.  A model of where precision is lost
    at large input scales."""
    nh, dn, dr, dv = dims["n_heads"], dims["d_nope"], dims["d_rope"], dims["d_head"]
    F, fw = dims["frame_h"] * dims["frame_w"], dims["frame_w"]
    rope = lambda v, t, h, w: rope3d(v, t, h, w, dims["rope_t"], dims["rope_h"], dims["rope_w"], dims["rope_base"])
    Wd = {k: v.double().numpy() for k, v in W.items()}
    x_all = np.concatenate([x_fill.double().numpy(), xq.double().numpy()])
    n_f = x_all.shape[0] // F
    t = np.repeat(np.arange(n_f, dtype=np.float64), F)
    hh = np.tile(np.arange(F) // fw, n_f)
    ww = np.tile(np.arange(F) % fw, n_f)
    c = _f16(x_all @ Wd["w_dkv"].T)
    kr = _f16(rope(x_all @ Wd["w_kr"].T, t, hh, ww))
    keys = np.concatenate([c, kr], axis=1)
    nq = xq.shape[0]
    xqd = x_all[-nq:]
    scale = 1.0 / np.sqrt(dn + dr) / np.log(2.0)
    out = np.zeros((nq, dims["hidden"]))
    for h in range(nh):
        w_uk = Wd["w_uk"][h * dn:(h + 1) * dn]
        if wq == "two_step":
            q = xqd @ Wd["w_q"][h * dn:(h + 1) * dn].T
            q_hi = _f16(q)
            q_nope = (q_hi + _f16(q - q_hi)) @ _f16(w_uk)
        else:
            wq_abs = w_uk.T @ Wd["w_q"][h * dn:(h + 1) * dn]
            if wq == "single":
                wq_abs = _bf16(wq_abs)
            elif wq == "pair":
                hi = _bf16(wq_abs)
                wq_abs = hi + _bf16(wq_abs - hi)
            q_nope = xqd @ wq_abs.T
        q_r = rope(xqd @ Wd["w_qr"][h * dr:(h + 1) * dr].T, t[-nq:], hh[-nq:], ww[-nq:])
        qp = _f16(np.concatenate([q_nope, q_r], axis=1) * scale)
        sc = qp @ keys.T
        P = np.exp2(sc - sc.max(axis=1, keepdims=True))
        o_lat = _f16((_f16(P) @ c) / P.sum(axis=1, keepdims=True))
        w_ov = _f16(Wd["w_o"][:, h * dv:(h + 1) * dv] @ Wd["w_uv"][h * dv:(h + 1) * dv])
        out += o_lat @ w_ov.T
    return _bf16(out)


@pytest.mark.parametrize("scale", [8.0, 32.0, 128.0])
def test_large_hidden_scales_stay_in_range_and_in_parity(scale):
    # N(0,1) x scale hidden states: the latents reach about 6 x scale, far below 65504, so the
    # range flag must stay clear.  Scores grow with scale^2; a softmax that sharp turns every
    # perturbation of the scores into an output error, and the absorbed query weight rounded to
    # a single bf16 (8 significant bits) would miss the bar at scales 8 and 32 (the rounding
    # model prints by how much).  The library never rounds that product: it multiplies W_Q and
    # then W_UK with q carried as an fp16 pair, so the GPU must meet the bar against the oracle
    # at every scale, and match its own rounding model.
    import mla_latent_kv_window_b200 as M
    w = small(window=2, fill=2, q=1, seed=42)
    p = Pair(w)
    x = (p.hidden(2, 4020).float() * scale).to(torch.bfloat16)
    p.append(x)
    xq = (p.hidden(1, 4021).float() * scale).to(torch.bfloat16)
    out = p.attention(xq)
    assert M.mla_cache_sync(p.gpu.handle) == 0
    assert torch.isfinite(out.float()).all()
    ref = p.oracles[0].attention(xq[0])
    model = _rounding_model(p.dims, p.weights, x[0], xq[0])
    rel, mx = errors(out[0], ref)
    rel_s, mx_s = errors(torch.from_numpy(_rounding_model(p.dims, p.weights, x[0], xq[0], wq="single")), ref)
    print(f"hidden scale {scale}: vs exact oracle: GPU rel L2 {rel:.3e} max-abs/RMS {mx:.3e}; "
          f"with a single-bf16 absorbed query weight (model) {rel_s:.3e} / {mx_s:.3e}")
    assert_close(out[0], ref, f"scale {scale}: GPU vs oracle")
    assert_close(out[0], model, f"scale {scale}: GPU vs the rounding model of its path")
    p.gpu.close()


def _long_stream(sink: int, n_total: int, seed: int):
    # One-token-wide frames of a 4-head, 512-wide model so that a bulk append of ~10^5 frames
    # needs only ~0.4 GB of hidden states; the GPU computes only the frames that survive.
    dims = dict(mla_synth.DIMS_WAN13B, hidden=512, n_heads=4)
    w = mla_synth.Workload("long", frame_h=1, frame_w=2, window_frames=3, fill_frames=0,
                           query_frames=1, seed=seed, sink_frames=sink, dims=tuple(sorted(dims.items())))
    p = Pair(w)
    x = p.hidden(n_total, seed * 16 + 1)
    p.gpu.append(x.cuda())
    for i in range(0, n_total, 10000):         # the oracle keeps every frame's index exactly
        for b, o in enumerate(p.oracles):
            o.append(x[b, i * w.F:min(n_total, i + 10000) * w.F])
    return p, w


@pytest.mark.parametrize("sink", [0, 1])
def test_temporal_index_near_1e5(sink):
    n_total = 100_003
    p, w = _long_stream(sink, n_total, 43 + sink)
    assert p.gpu.state() == (n_total, 3 + sink)
    check_ring(p, f"after {n_total} frames")        # keys rotated at t ~ 1e5 vs fp64
    for s in range(2):
        full_check(p, p.hidden(1, 4030 + s), f"t ~ 1e5, sink {sink}, call {s}")
        p.append(p.hidden(1, 4040 + s))
    check_ring(p, "after two more appends")
    p.gpu.close()
