"""Scalar-loop brute force of one VideoMLA attention call, for pinning the oracle on tiny shapes.

Written independently of oracle/: plain Python lists, the math module and explicit
loops, no array helpers.  It follows the same reading of the VideoMLA paper page
(§3.1-§3.3 cache construction and reconstruction, App. D.5 window-local RoPE):
every step is spelled out so that a dropped term, a wrong sign or index, or a
transposed operand in the oracle shows up as a mismatch.
"""
import math


def matvec(W, x):
    """y[o] = sum_i W[o][i] x[i]   (W in [out][in] layout)."""
    return [sum(W[o][i] * x[i] for i in range(len(x))) for o in range(len(W))]


def rotate(vec, t, h, w, split, base):
    """Rotate vec (len = sum(split)) pair by pair; pair j of axis a turns by pos_a * base**(-2j/d_a)."""
    out = list(vec)
    ch = 0
    for pos, d_a in zip((t, h, w), split):
        for j in range(d_a // 2):
            ang = pos * base ** (-2.0 * j / d_a)
            a, b = vec[ch], vec[ch + 1]
            out[ch] = a * math.cos(ang) - b * math.sin(ang)
            out[ch + 1] = a * math.sin(ang) + b * math.cos(ang)
            ch += 2
    return out


def attention(dims, W, window_x, chunk_x):
    """window_x: list of cached frames in logical order (sink frames, then the window oldest
    first) of token hidden vectors; chunk_x: the query frames.  Frames get window-local temporal
    coordinates 0, 1, ... in that order.  With W["w_dq"] the query projections read the low-rank
    query latent W_DQ x instead of x.

    Returns out[q][d] for every token of the chunk.
    """
    nh, dn, dv, dr = dims["n_heads"], dims["d_nope"], dims["d_head"], dims["d_rope"]
    fw = dims["frame_w"]
    split = (dims["rope_t"], dims["rope_h"], dims["rope_w"])
    base = dims["rope_base"]
    scale = 1.0 / math.sqrt(dn + dr)

    frames = list(window_x) + list(chunk_x)
    keys = []  # (c, rotated r, index) per key
    for lt, frame in enumerate(frames):          # window-local temporal coordinate
        for k, x in enumerate(frame):
            c = matvec(W["w_dkv"], x)
            r = matvec(W["w_kr"], x)
            keys.append((c, rotate(r, lt, k // fw, k % fw, split, base)))

    out = []
    q_t0 = len(window_x)
    for qf, frame in enumerate(chunk_x):
        for k, x in enumerate(frame):
            head_out = []
            for hd in range(nh):
                Wq = W["w_q"][hd * dn:(hd + 1) * dn]
                Wqr = W["w_qr"][hd * dr:(hd + 1) * dr]
                Wuk = W["w_uk"][hd * dn:(hd + 1) * dn]
                Wuv = W["w_uv"][hd * dv:(hd + 1) * dv]
                xq = matvec(W["w_dq"], x) if "w_dq" in W else x
                q = matvec(Wq, xq) + rotate(matvec(Wqr, xq), q_t0 + qf, k // fw, k % fw, split, base)
                scores = []
                vals = []
                for c, kr in keys:
                    kvec = matvec(Wuk, c) + kr
                    scores.append(scale * sum(q[i] * kvec[i] for i in range(len(q))))
                    vals.append(matvec(Wuv, c))
                m = max(scores)
                e = [math.exp(s - m) for s in scores]
                z = sum(e)
                o = [sum(e[j] / z * vals[j][i] for j in range(len(keys))) for i in range(dv)]
                head_out.extend(o)
            out.append(matvec(W["w_o"], head_out))
    return out
