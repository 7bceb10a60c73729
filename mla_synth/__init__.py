"""Seeded synthetic inputs for the VideoMLA latent-window attention path.

This module only draws random numbers and names workload shapes.  It holds
none of the method's arithmetic: both the CUDA path and the fp64 oracle take
their inputs from here, so they see identical bf16 bits.

Shapes follow the VideoMLA paper (Wan2.1-T2V-1.3B backbone, App. D.1 "Backbone
and Tokenization"): hidden 1536, 12 heads x 128, 30 x 52 = 1560 tokens per
latent frame, 3-frame chunks.  Distributions: hidden states ~ N(0, 1) (times an
optional per-stream scale), every weight ~ N(0, 1/fan_in), all rounded to bf16.
Weights use the nn.Linear convention [out_features, in_features] with
head-major output channels (channel c = head * dim + j).
"""
from __future__ import annotations

import dataclasses

import torch

# Workload shapes.  Pure data: sizes and seeds, no arithmetic of the method.
DIMS_WAN13B = dict(
    hidden=1536, n_heads=12, d_head=128, d_nope=128, d_latent=192, d_rope=32,
    rope_t=8, rope_h=12, rope_w=12, rope_base=10000.0,
)
# The paper's default attention dims ([VideoMLA] §4.1): content key 96 + positional key 32
# (= the backbone's 128 per head), a low-rank query of width d_q = 768, RoPE (6, 5, 5) pairs.
DIMS_PAPER = dict(
    hidden=1536, n_heads=12, d_head=128, d_nope=96, d_latent=192, d_rope=32,
    rope_t=12, rope_h=10, rope_w=10, rope_base=10000.0, d_q=768,
)


@dataclasses.dataclass(frozen=True)
class Workload:
    """One benchmark/parity workload: dims, frame grid, window and call pattern."""
    name: str
    frame_h: int
    frame_w: int
    window_frames: int
    fill_frames: int          # frames appended before the first attention call
    query_frames: int         # frames in each query chunk
    batch: int = 1
    layers: int = 1
    steps: int = 1            # denoising steps per chunk (same cache)
    seed: int = 0
    stream_scale: bool = False  # per-stream random scale in [0.5, 2]
    dims: tuple = tuple(sorted(DIMS_WAN13B.items()))
    sink_frames: int = 0        # first frames kept for good besides the window (App. D.4/D.5)

    @property
    def F(self) -> int:
        return self.frame_h * self.frame_w

    def dim(self, key):
        return dict(self.dims)[key]


# The five workloads.  "tiny" is the small case the oracle finishes in well under a second.
WORKLOADS = {
    "tiny": Workload("tiny", frame_h=4, frame_w=6, window_frames=2, fill_frames=2,
                     query_frames=1, seed=0),
    "wan_w21_q1": Workload("wan_w21_q1", frame_h=30, frame_w=52, window_frames=21,
                           fill_frames=21, query_frames=1, seed=1000),
    "wan_30l_w21_q3_wrap": Workload("wan_30l_w21_q3_wrap", frame_h=30, frame_w=52,
                                    window_frames=21, fill_frames=24, query_frames=3,
                                    layers=30, steps=4, seed=2000),
    "wan_b4_w21_q3": Workload("wan_b4_w21_q3", frame_h=30, frame_w=52, window_frames=21,
                              fill_frames=21, query_frames=3, batch=4, seed=3000,
                              stream_scale=True),
    "wan_w63_q1": Workload("wan_w63_q1", frame_h=30, frame_w=52, window_frames=63,
                           fill_frames=63, query_frames=1, seed=4000),
    # Next rows: the paper-default dims, and a sink frame plus a short window.
    "paper_tiny": Workload("paper_tiny", frame_h=4, frame_w=6, window_frames=2, fill_frames=3,
                           query_frames=1, seed=5, dims=tuple(sorted(DIMS_PAPER.items()))),
    "paper_w21_q1": Workload("paper_w21_q1", frame_h=30, frame_w=52, window_frames=21,
                             fill_frames=21, query_frames=1, seed=5000,
                             dims=tuple(sorted(DIMS_PAPER.items()))),
    "sink_tiny": Workload("sink_tiny", frame_h=4, frame_w=6, window_frames=2, fill_frames=5,
                          query_frames=2, seed=6, sink_frames=1),
    "sink_w6_q3": Workload("sink_w6_q3", frame_h=30, frame_w=52, window_frames=6,
                           fill_frames=10, query_frames=3, seed=6000, sink_frames=1),
}


def gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def normal_bf16(shape, std: float, seed: int) -> torch.Tensor:
    """N(0, std^2) drawn in fp32 on the CPU from `seed`, rounded to bf16."""
    t = torch.randn(*shape, generator=gen(seed), dtype=torch.float32)
    return (t * std).to(torch.bfloat16)


def make_weights(dims: dict, seed: int) -> dict:
    """The projection weights of one layer, bf16, N(0, 1/fan_in).

    With a low-rank query (dims["d_q"] > 0) the query projections read the d_q-wide query
    latent, w_q is [n_h d_nope, d_q], w_qr [n_h d_rope, d_q], and w_dq [d_q, hidden] is added.
    """
    d = dims["hidden"]
    nh = dims["n_heads"]
    dn = dims["d_nope"]
    dv = dims["d_head"]
    dc = dims["d_latent"]
    dr = dims["d_rope"]
    dq = dims.get("d_q", 0)
    q_in = dq if dq else d
    shapes = {
        "w_q": (nh * dn, q_in),
        "w_qr": (nh * dr, q_in),
        "w_dkv": (dc, d),
        "w_kr": (dr, d),
        "w_uk": (nh * dn, dc),
        "w_uv": (nh * dv, dc),
        "w_o": (d, nh * dv),
    }
    if dq:
        shapes["w_dq"] = (dq, d)
    out = {}
    for i, (name, shp) in enumerate(shapes.items()):
        out[name] = normal_bf16(shp, 1.0 / float(shp[1]) ** 0.5, seed * 16 + i)
    return out


def make_hidden(batch: int, n_tokens: int, hidden: int, seed: int,
                stream_scales=None) -> torch.Tensor:
    """Hidden states [batch, n_tokens, hidden] bf16, N(0,1) times an optional per-stream scale."""
    t = torch.randn(batch, n_tokens, hidden, generator=gen(seed), dtype=torch.float32)
    if stream_scales is not None:
        t = t * torch.tensor(stream_scales, dtype=torch.float32).view(-1, 1, 1)
    return t.to(torch.bfloat16)


def stream_scales(batch: int, seed: int):
    """One scale per stream, uniform in [0.5, 2], drawn from `seed`."""
    u = torch.rand(batch, generator=gen(seed * 7 + 3), dtype=torch.float64)
    return [float(0.5 + 1.5 * v) for v in u]


def layer_seed(w: Workload, layer: int, step: int = 0) -> int:
    """Seed for layer `layer`, denoising step `step` of a workload."""
    return w.seed + 10 * layer + step


def weight_seed(w: Workload, layer: int) -> int:
    return layer_seed(w, layer, 0)


def fill_seed(w: Workload, layer: int) -> int:
    """Seed of the hidden states that fill a layer's window (disjoint from weight seeds mod 16)."""
    return layer_seed(w, layer, 0) * 16 + 8


def chunk_seed(w: Workload, layer: int, step: int, chunk: int = 0) -> int:
    """Seed of the query chunk's hidden states for (layer, denoising step, chunk index)."""
    return (layer_seed(w, layer, step) + 100000 * chunk) * 16 + 9
