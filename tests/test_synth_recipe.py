"""The seeded input recipe shared by the oracle and the GPU tests: deterministic bits per seed,
the stated distributions (hidden states N(0,1), weights N(0, 1/fan_in), stream scales uniform in
[0.5, 2]), the weight shapes of the workloads' dims, and seeds that do not collide between the
weights, the window fill and the query chunks of a workload."""
import math

import torch

import mla_synth


def test_bits_are_deterministic_per_seed():
    a = mla_synth.make_hidden(2, 100, 64, 17)
    b = mla_synth.make_hidden(2, 100, 64, 17)
    c = mla_synth.make_hidden(2, 100, 64, 18)
    assert a.dtype == torch.bfloat16 and torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert not torch.equal(a, c)


def test_stated_distributions():
    x = mla_synth.make_hidden(1, 4096, 256, 3).float()
    assert abs(x.mean().item()) < 0.01 and abs(x.std().item() - 1.0) < 0.01
    dims = dict(mla_synth.DIMS_WAN13B)
    w = mla_synth.make_weights(dims, 5)
    for name, t in w.items():
        assert t.dtype == torch.bfloat16
        fan_in = t.shape[1]
        assert abs(t.float().std().item() * math.sqrt(fan_in) - 1.0) < 0.02, name
    s = mla_synth.stream_scales(1000, 11)
    assert min(s) >= 0.5 and max(s) <= 2.0 and abs(sum(s) / len(s) - 1.25) < 0.05


def test_weight_shapes_follow_the_dims():
    d = dict(mla_synth.DIMS_WAN13B)
    w = mla_synth.make_weights(d, 0)
    nh, dn, dv, dc, dr, hid = d["n_heads"], d["d_nope"], d["d_head"], d["d_latent"], d["d_rope"], d["hidden"]
    assert w["w_q"].shape == (nh * dn, hid) and w["w_qr"].shape == (nh * dr, hid)
    assert w["w_dkv"].shape == (dc, hid) and w["w_kr"].shape == (dr, hid)
    assert w["w_uk"].shape == (nh * dn, dc) and w["w_uv"].shape == (nh * dv, dc)
    assert w["w_o"].shape == (hid, nh * dv) and "w_dq" not in w
    p = dict(mla_synth.WORKLOADS["paper_tiny"].dims)
    wp = mla_synth.make_weights(p, 0)
    assert wp["w_dq"].shape == (p["d_q"], p["hidden"]) and wp["w_q"].shape == (p["n_heads"] * 96, p["d_q"])


def test_seeds_do_not_collide_within_a_workload():
    for w in mla_synth.WORKLOADS.values():
        weight_streams = {mla_synth.weight_seed(w, l) * 16 + i for l in range(w.layers) for i in range(8)}
        fills = {mla_synth.fill_seed(w, l) for l in range(w.layers)}
        chunks = {mla_synth.chunk_seed(w, l, s, c) for l in range(w.layers) for s in range(w.steps)
                  for c in range(2)}
        assert not (weight_streams & fills) and not (weight_streams & chunks) and not (fills & chunks), w.name
