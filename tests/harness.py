"""Shared helpers of the GPU parity tests: run one seeded workload through the C ABI and the
fp64 oracle on identical bf16 inputs, and compare with the stated tolerance.

Tolerance (bf16 inputs and weights; fp16 cache, queries, P and o_lat; fp32 accumulation) against
the fp64 oracle: relative L2 error <= 1e-2 and max-abs error <= 3e-2 x RMS(oracle output).
"""
from __future__ import annotations

import math

import numpy as np
import torch

import mla_synth
from oracle import OracleLayer

REL_L2 = 1e-2
MAX_ABS_RMS = 3e-2


def errors(gpu, ref) -> tuple[float, float]:
    g = np.asarray(gpu.float().cpu().numpy() if hasattr(gpu, "float") else gpu, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    assert np.all(np.isfinite(g)), "non-finite GPU output"
    rel = float(np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-300))
    rms = float(np.sqrt(np.mean(r * r)))
    mx = float(np.max(np.abs(g - r)) / max(rms, 1e-300))
    return rel, mx


def assert_close(gpu, ref, what: str, rel_tol: float = REL_L2, max_tol: float = MAX_ABS_RMS):
    rel, mx = errors(gpu, ref)
    assert rel <= rel_tol and mx <= max_tol, f"{what}: rel L2 {rel:.3e} (tol {rel_tol}), max-abs/RMS {mx:.3e} (tol {max_tol})"
    return rel, mx


def dims_of(w: mla_synth.Workload) -> dict:
    d = dict(w.dims)
    d.update(frame_h=w.frame_h, frame_w=w.frame_w, window_frames=w.window_frames,
             sink_frames=w.sink_frames)
    return d


class Pair:
    """One layer on the GPU (LatentWindowCache) and in the oracle (one OracleLayer per stream)."""

    def __init__(self, w: mla_synth.Workload, layer: int = 0, max_chunk_frames: int | None = None,
                 weights: dict | None = None):
        from mla_latent_kv_window_b200 import LatentWindowCache
        self.w = w
        self.dims = dims_of(w)
        self.F = w.F
        self.weights = weights if weights is not None else mla_synth.make_weights(dict(w.dims), mla_synth.weight_seed(w, layer))
        dev_w = {k: v.cuda() for k, v in self.weights.items()}
        self.gpu = LatentWindowCache(dict(w.dims), dev_w, w.frame_h, w.frame_w, w.window_frames,
                                     max_chunk_frames or w.query_frames, batch=w.batch,
                                     sink_frames=w.sink_frames)
        self.oracles = [OracleLayer(self.dims, self.weights) for _ in range(w.batch)]
        self.scales = mla_synth.stream_scales(w.batch, w.seed) if w.stream_scale else None

    def hidden(self, n_frames: int, seed: int) -> torch.Tensor:
        return mla_synth.make_hidden(self.w.batch, n_frames * self.F, self.dims["hidden"], seed, self.scales)

    def append(self, x: torch.Tensor, oracle: bool = True) -> None:
        self.gpu.append(x.cuda())
        if oracle:
            for b, o in enumerate(self.oracles):
                o.append(x[b])

    def attention(self, x: torch.Tensor) -> torch.Tensor:
        out = self.gpu.attention(x.cuda())
        torch.cuda.synchronize()
        return out.cpu()

    def check_status(self):
        self.gpu.sync()
