"""fp64 CPU oracle of VideoMLA latent-window attention.  TEST INFRASTRUCTURE ONLY.

Only the tests, the smoke check and the benchmark's CPU-baseline leg may import
this module.  The CUDA library never calls it, and it shares no code with the
CUDA path: it is a plain, slow, obviously correct restatement of what the
method computes, written so that a reader can check it against the paper by eye.

Source: "VideoMLA: Low-Rank Latent KV Cache for Minute-Scale Autoregressive
Video Diffusion" (paper text page), cited below as [VideoMLA] with its section.

What it computes (the unabsorbed plain definition, in float64, from bf16 inputs):

* Cache construction ([VideoMLA] §3.1, §3.2): every appended token stores a
  head-shared content latent c = x W_DKV^T (d_c) and a head-shared positional
  state r = x W_KR^T (d_rope).  Following [VideoMLA] App. D.5, r is stored
  *before* RoPE and rotated when the window is assembled.
* Sliding window ([VideoMLA] §1, App. D.4): a FIFO of the last W latent frames,
  optionally after `sink_frames` sink frames: the first frames of the video,
  kept for good (App. D.4/D.5 "sink + local window").
* Attention ([VideoMLA] §3.3): per head, keys and values are reconstructed
  from the latent, k_h = [c W_UK[h]^T || RoPE3D(r)], v_h = c W_UV[h]^T, the
  query is q_h = [x W_Q[h]^T || RoPE3D(x W_QR[h]^T)] (with a low-rank query,
  [VideoMLA] §4.1 d_q = 768, x is first projected to c_q = x W_DQ^T and W_Q, W_QR
  read c_q), and textbook softmax attention runs over the sink and window frames
  plus the chunk's own frames (the query
  chunk is the newest, so chunk-causal masking ([VideoMLA] App. D.4) masks
  nothing).  out = concat_h(o_h) W_O^T.
* Positions ([VideoMLA] App. D.5): the active frames (sink frames, then the
  window frames, oldest first) and the query chunk get window-local temporal
  coordinates 0, 1, ... and are rotated at use.
* 3D RoPE ([VideoMLA] §3.2, §4.1, App. C.1): the d_rope channels split into
  temporal / height / width groups of adjacent pairs; axis a with d_a channels
  rotates pair i by angle pos_a * base^(-2 i / d_a) (i = 0 is the highest
  frequency band).

Readings taken where the page is silent or its equations were lost (Eqs. 1, 2,
5 and App. D.2/D.3 did not survive): no biases or norms inside the block;
softmax scale 1/sqrt(d_nope + d_rope); pairs are adjacent channels (2i, 2i+1);
channel order [t pairs | h pairs | w pairs]; token k of a frame sits at
(h, w) = (k // frame_w, k % frame_w).

Pins (tests/test_oracle_pins.py): every function here is pinned against closed
forms, invariants, special cases that reduce to a library routine, or a
scalar brute-force implementation.  No function is "parity unpinned".
"""
from __future__ import annotations

import math

import numpy as np


# ----------------------------------------------------------------------------- accounting
def latent_scalars_per_token(d_latent: int, d_rope: int) -> int:
    """Cached scalars per token per layer: d_c + d_h^rope ([VideoMLA] §3.1)."""
    return d_latent + d_rope


def dense_scalars_per_token(n_heads: int, d_head: int) -> int:
    """Dense per-head KV scalars per token per layer: 2 n_h d_h ([VideoMLA] §1)."""
    return 2 * n_heads * d_head


def cache_scalars(layers: int, frames: int, tokens_per_frame: int, per_token: int) -> int:
    """Total cached scalars of a window: layers x frames x tokens/frame x per-token ([VideoMLA] §1)."""
    return layers * frames * tokens_per_frame * per_token


# ----------------------------------------------------------------------------- 3D RoPE
def rope_bands(rope_t: int, rope_h: int, rope_w: int, base: float):
    """Per rotation pair: (axis index 0/1/2 for t/h/w, angular frequency).

    Axis a owns d_a channels = d_a/2 adjacent pairs; pair i of that axis turns at
    base^(-2 i / d_a), so i = 0 is the highest-frequency band ([VideoMLA] §3.2,
    §4.1 "using the highest-frequency bands").
    """
    axes, freqs = [], []
    for a, d_a in enumerate((rope_t, rope_h, rope_w)):
        if d_a % 2:
            raise ValueError("each RoPE axis needs an even channel count")
        for i in range(d_a // 2):
            axes.append(a)
            freqs.append(float(base) ** (-2.0 * i / d_a))
    return np.array(axes, dtype=np.int64), np.array(freqs, dtype=np.float64)


def rope3d(v: np.ndarray, t, h, w, rope_t: int, rope_h: int, rope_w: int, base: float) -> np.ndarray:
    """Rotate the last axis of v (d_rope = rope_t + rope_h + rope_w channels) at positions (t, h, w).

    t, h, w broadcast against v.shape[:-1].  Pair p = (v[2p], v[2p+1]) is treated as the
    complex number v[2p] + i v[2p+1] and multiplied by exp(i * pos_axis(p) * freq(p)).
    """
    v = np.asarray(v, dtype=np.float64)
    d_r = rope_t + rope_h + rope_w
    if v.shape[-1] != d_r:
        raise ValueError("rope3d: last axis must have rope_t + rope_h + rope_w channels")
    if d_r == 0:
        return v.copy()
    axes, freqs = rope_bands(rope_t, rope_h, rope_w, base)
    lead = v.shape[:-1]
    pos = np.stack([np.broadcast_to(np.asarray(p, dtype=np.float64), lead) for p in (t, h, w)], axis=-1)
    ang = pos[..., axes] * freqs                     # [..., d_r/2]
    cs, sn = np.cos(ang), np.sin(ang)
    re, im = v[..., 0::2], v[..., 1::2]
    out = np.empty_like(v)
    out[..., 0::2] = re * cs - im * sn
    out[..., 1::2] = re * sn + im * cs
    return out


def token_hw(k, frame_w: int):
    """(h, w) grid position of token k inside a latent frame, row-major ([VideoMLA] App. C.1, S = F H W)."""
    k = np.asarray(k)
    return k // frame_w, k % frame_w


# ----------------------------------------------------------------------------- ring bookkeeping
def ring_slot(frame: int, token: int, window_frames: int, tokens_per_frame: int) -> int:
    """Physical slot of (absolute frame, token) in a frame-granular ring of W frames."""
    return (frame % window_frames) * tokens_per_frame + token


def valid_frames(frames_appended: int, window_frames: int) -> int:
    return min(frames_appended, window_frames)


# ----------------------------------------------------------------------------- model pieces
def _f64(a) -> np.ndarray:
    """Widen a torch/numpy array (bf16, fp32, ...) to float64 numpy."""
    if hasattr(a, "detach"):
        a = a.detach().to("cpu")
        import torch  # local: only for dtype widening of torch inputs
        a = a.to(torch.float64).numpy()
    return np.asarray(a, dtype=np.float64)


class OracleLayer:
    """One VideoMLA self-attention layer with its sliding-window latent cache, in float64.

    dims: hidden, n_heads, d_head, d_nope, d_latent, d_rope, rope_t, rope_h, rope_w,
    rope_base, plus frame_h, frame_w, window_frames and optionally sink_frames.  weights:
    w_q [n_h d_nope, d], w_qr [n_h d_rope, d], w_dkv [d_c, d], w_kr [d_rope, d],
    w_uk [n_h d_nope, d_c], w_uv [n_h d_head, d_c], w_o [d, n_h d_head] (nn.Linear [out, in]
    layout); with a low-rank query also w_dq [d_q, d], and then w_q, w_qr read d_q columns.
    """

    def __init__(self, dims: dict, weights: dict, softmax_scale: float | None = None):
        self.d = dict(dims)
        self.W = {k: _f64(v) for k, v in weights.items()}
        self.F = self.d["frame_h"] * self.d["frame_w"]
        dn, dr = self.d["d_nope"], self.d["d_rope"]
        self.scale = softmax_scale if softmax_scale else 1.0 / math.sqrt(dn + dr)
        # Sink frames (the first sink_frames frames appended, kept for good) and the FIFO of the
        # other cached frames, oldest first; each entry is (absolute frame index, c [F,d_c], r [F,d_r]).
        self.n_sink = int(self.d.get("sink_frames", 0))
        self.sink: list[tuple[int, np.ndarray, np.ndarray]] = []
        self.frames: list[tuple[int, np.ndarray, np.ndarray]] = []
        self.frames_appended = 0

    # -- §3.1 / §3.2: what one token caches (r is kept unrotated, App. D.5)
    def latent(self, x: np.ndarray):
        x = _f64(x)
        c = x @ self.W["w_dkv"].T
        r = x @ self.W["w_kr"].T
        return c, r

    def append(self, x) -> None:
        """Append n whole latent frames of hidden states x [n F, d]: the first sink_frames frames
        ever appended become the sink, the others go through the FIFO of the newest W frames."""
        x = _f64(x)
        if x.shape[0] % self.F:
            raise ValueError("append takes whole latent frames")
        c, r = self.latent(x)
        for i in range(x.shape[0] // self.F):
            sl = slice(i * self.F, (i + 1) * self.F)
            entry = (self.frames_appended, c[sl], r[sl])
            self.frames_appended += 1
            if len(self.sink) < self.n_sink:
                self.sink.append(entry)
                continue
            self.frames.append(entry)
            if len(self.frames) > self.d["window_frames"]:
                self.frames.pop(0)

    def active_frames(self):
        """The cached frames attention sees, in logical order: sink frames, then the window."""
        return self.sink + self.frames

    def query_input(self, x: np.ndarray) -> np.ndarray:
        """What the query projections read: x itself, or with a low-rank query the query latent
        c_q = x W_DQ^T ([VideoMLA] §4.1: d_q = 768; no norm on c_q, as elsewhere in the block)."""
        return x @ self.W["w_dq"].T if "w_dq" in self.W else x

    def _rope(self, v, t, h, w):
        d = self.d
        return rope3d(v, t, h, w, d["rope_t"], d["rope_h"], d["rope_w"], d["rope_base"])

    def cache_contents(self):
        """What a ring that rotates at append time would hold: per valid frame (sink frames first,
        then the window oldest first) the absolute frame index, c [F, d_c] and r rotated at the
        frame's ABSOLUTE index [F, d_r]."""
        hh, ww = token_hw(np.arange(self.F), self.d["frame_w"])
        out = []
        for f, c, r in self.active_frames():
            out.append((f, c.copy(), self._rope(r, f, hh, ww)))
        return out

    def keys_and_queries(self, x_chunk, positions: str = "local"):
        """Assemble the attention context: latent keys (window frames oldest first, then the chunk)
        with their positions, and the chunk's query inputs with theirs.

        positions="local" is the App. D.5 re-indexing (window-local temporal coordinates: sink
        frames, window frames and the chunk numbered 0, 1, ... in that order); "absolute" uses
        absolute frame indices (equal results for a window without a sink).
        """
        x = _f64(x_chunk)
        if x.shape[0] % self.F or x.shape[0] == 0:
            raise ValueError("a query chunk is one or more whole latent frames")
        nq_frames = x.shape[0] // self.F
        c_new, r_new = self.latent(x)
        active = self.active_frames()
        frame_ids = [f for f, _, _ in active] + [self.frames_appended + i for i in range(nq_frames)]
        c_all = np.concatenate([c for _, c, _ in active] + [c_new], axis=0)
        r_all = np.concatenate([r for _, _, r in active] + [r_new], axis=0)
        if positions == "local":
            t_of_frame = np.arange(len(frame_ids), dtype=np.float64)
        elif positions == "absolute":
            t_of_frame = np.array(frame_ids, dtype=np.float64)
        else:
            raise ValueError(positions)
        hh, ww = token_hw(np.arange(self.F), self.d["frame_w"])
        t_key = np.repeat(t_of_frame, self.F)
        h_key = np.tile(hh, len(frame_ids))
        w_key = np.tile(ww, len(frame_ids))
        t_q = t_key[-x.shape[0]:]
        h_q = h_key[-x.shape[0]:]
        w_q = w_key[-x.shape[0]:]
        return dict(x=x, c=c_all, r=r_all, t_key=t_key, h_key=h_key, w_key=w_key,
                    t_q=t_q, h_q=h_q, w_q=w_q)

    def head_qkv(self, ctx: dict, h: int, rows=None):
        """Materialise head h's Q [n_q, d_nope + d_r], K [N, d_nope + d_r], V [N, d_head] (no absorption)."""
        d = self.d
        dn, dv, dr = d["d_nope"], d["d_head"], d["d_rope"]
        x = ctx["x"] if rows is None else ctx["x"][rows]
        tq, hq, wq = (ctx["t_q"], ctx["h_q"], ctx["w_q"]) if rows is None else \
            (ctx["t_q"][rows], ctx["h_q"][rows], ctx["w_q"][rows])
        w_uk = self.W["w_uk"][h * dn:(h + 1) * dn]          # [d_nope, d_c]
        w_uv = self.W["w_uv"][h * dv:(h + 1) * dv]          # [d_head, d_c]
        k_nope = ctx["c"] @ w_uk.T                          # Eq. 2 (up-projection), keys
        v = ctx["c"] @ w_uv.T                               # Eq. 2 (up-projection), values
        k_rope = self._rope(ctx["r"], ctx["t_key"], ctx["h_key"], ctx["w_key"])   # shared by heads
        xq = self.query_input(x)
        q_nope = xq @ self.W["w_q"][h * dn:(h + 1) * dn].T
        q_rope = self._rope(xq @ self.W["w_qr"][h * dr:(h + 1) * dr].T, tq, hq, wq)
        K = np.concatenate([k_nope, k_rope], axis=1)
        Q = np.concatenate([q_nope, q_rope], axis=1)
        return Q, K, v

    def attention(self, x_chunk, rows=None, positions: str = "local", return_parts: bool = False,
                  heads=None):
        """Output [n_q, d] for the query chunk x_chunk [n_q, d] (or for the query rows `rows` only).

        With return_parts, also returns per head the softmax matrix P [n_h, n_q, N], the
        latent-space output P c [n_q, n_h, d_c] and the head outputs O [n_q, n_h, d_head].
        `heads` restricts the work to a subset of heads (the other heads contribute zero to the
        output); it exists only to time bounded samples and is never used for parity.
        """
        d = self.d
        ctx = self.keys_and_queries(x_chunk, positions)
        nh, dv = d["n_heads"], d["d_head"]
        nq = ctx["x"].shape[0] if rows is None else len(np.atleast_1d(rows))
        O = np.zeros((nq, nh, dv))
        Pc = np.zeros((nq, nh, d["d_latent"]))
        Ps = []
        for h in (range(nh) if heads is None else heads):
            Q, K, V = self.head_qkv(ctx, h, rows)
            S = (Q @ K.T) * self.scale                       # [n_q, N]
            S = S - S.max(axis=1, keepdims=True)
            E = np.exp(S)
            P = E / E.sum(axis=1, keepdims=True)
            O[:, h, :] = P @ V
            if return_parts:
                Pc[:, h, :] = P @ ctx["c"]
                Ps.append(P)
        out = O.reshape(nq, nh * dv) @ self.W["w_o"].T
        if return_parts:
            return out, dict(P=np.stack(Ps), Pc=Pc, O=O, ctx=ctx)
        return out

    def absorbed_scores(self, x_chunk, h: int, positions: str = "local"):
        """Scores of head h computed the absorbed way: (W_UK[h]^T q_nope) . c + q_rope . k_rope.

        Used only to pin the unabsorbed path (they must agree up to rounding order)."""
        d = self.d
        dn, dr = d["d_nope"], d["d_rope"]
        ctx = self.keys_and_queries(x_chunk, positions)
        w_uk = self.W["w_uk"][h * dn:(h + 1) * dn]
        xq = self.query_input(ctx["x"])
        q_nope = xq @ self.W["w_q"][h * dn:(h + 1) * dn].T
        q_abs = q_nope @ w_uk                                   # [n_q, d_c]
        q_rope = self._rope(xq @ self.W["w_qr"][h * dr:(h + 1) * dr].T, ctx["t_q"], ctx["h_q"], ctx["w_q"])
        k_rope = self._rope(ctx["r"], ctx["t_key"], ctx["h_key"], ctx["w_key"])
        return (q_abs @ ctx["c"].T + q_rope @ k_rope.T) * self.scale


def dense_mha(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float) -> np.ndarray:
    """Textbook multi-head attention over dense per-head K/V, the layout baseline
    ([VideoMLA] §1: 12 heads x 128 keys and values per token).  q [n_q, n_h, d],
    k [N, n_h, d], v [N, n_h, d_v] -> [n_q, n_h, d_v]."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    out = np.zeros((q.shape[0], q.shape[1], v.shape[2]))
    for h in range(q.shape[1]):
        S = (q[:, h, :] @ k[:, h, :].T) * scale
        S = S - S.max(axis=1, keepdims=True)
        E = np.exp(S)
        out[:, h, :] = (E / E.sum(axis=1, keepdims=True)) @ v[:, h, :]
    return out
