"""Host side of the C ABI, without a GPU: the library loads, exports every symbol that
include/mla.h declares, validates configurations, maps ring slots exactly like the oracle's
definition, and reproduces the cache accounting printed on the VideoMLA paper page."""
import ctypes
import json
import os
import re

import pytest

import mla_synth
from mla_latent_kv_window_b200 import binding as B
from oracle import cache_scalars, dense_scalars_per_token, ring_slot

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def cfg(**over):
    d = dict(mla_synth.DIMS_WAN13B)
    kw = dict(frame_h=30, frame_w=52, window_frames=21, max_chunk_frames=3, batch=1, sink_frames=0)
    kw.update({k: over.pop(k) for k in list(over) if k in kw})
    d.update(over)
    return B.make_config(d, **kw)


def test_library_exports_every_declared_symbol():
    lib = B.load_library()
    header = open(os.path.join(ROOT, "include", "mla.h")).read()
    declared = set(re.findall(r"^\s*(?:const\s+)?[\w\s\*]*?\b(mla_\w+)\s*\(", header, re.M))
    assert {"mla_cache_create", "mla_cache_append", "mla_window_attention", "mla_cache_destroy"} <= declared
    for name in sorted(declared):
        assert hasattr(lib, name), f"{name} declared in include/mla.h but not exported"
    assert set(B.EXPORTED) == declared


def test_binding_signatures_match_header():
    """Every declared function's parameter list (count and C type, pointers as one class) and
    return type agree with the argtypes/restype the ctypes binding installs."""
    lib = B.load_library()
    header = open(os.path.join(ROOT, "include", "mla.h")).read()
    header = re.sub(r"/\*.*?\*/", "", header, flags=re.S)
    decls = re.findall(r"^\s*((?:const\s+)?\w+\s*\**)\s*(mla_\w+)\s*\(([^)]*)\)\s*;", header, re.M | re.S)
    assert len(decls) == len(B.EXPORTED)
    scalar = {"int32_t": ctypes.c_int32, "int64_t": ctypes.c_int64, "float": ctypes.c_float,
              "double": ctypes.c_double, "size_t": ctypes.c_size_t, "mla_status": ctypes.c_int32,
              "mla_buffer": ctypes.c_int32}   # enums are int-sized

    def kind(ctype):
        if ctype in (ctypes.c_void_p, ctypes.c_char_p) or (
                isinstance(ctype, type) and issubclass(ctype, ctypes._Pointer)):
            return "ptr"
        return ctype

    for ret, name, params in decls:
        fn = getattr(lib, name)
        params = " ".join(params.split())
        plist = [] if params in ("", "void") else [q.strip() for q in params.split(",")]
        assert len(plist) == len(fn.argtypes), f"{name}: {len(plist)} parameters, binding {len(fn.argtypes)}"
        for q, at in zip(plist, fn.argtypes):
            want = "ptr" if "*" in q else scalar[q.split()[0]]
            assert kind(at) == want, f"{name}: parameter '{q}' bound as {at}"
        ret = ret.replace(" ", "")
        want_ret = None if ret == "void" else ("ptr" if "*" in ret else scalar[ret])
        assert (fn.restype if want_ret is None else kind(fn.restype)) == want_ret, f"{name}: return {ret}"


def test_config_check():
    assert B.mla_config_check(cfg()) == B.MLA_OK
    bad = [
        dict(rope_t=7, rope_h=13),                 # odd axis widths
        dict(rope_t=10),                           # widths do not sum to d_rope
        dict(window_frames=0), dict(max_chunk_frames=0), dict(batch=0), dict(frame_h=0),
        dict(hidden=0), dict(n_heads=-1), dict(rope_base=-1.0),
    ]
    for over in bad:
        assert B.mla_config_check(cfg(**over)) == B.MLA_ERR_INVALID_ARGUMENT, over
    assert B.mla_config_check(cfg(d_latent=128)) == B.MLA_ERR_UNSUPPORTED
    assert b"d_latent" in B.load_library().mla_last_error()
    assert B.mla_config_check(cfg(hidden=1600)) == B.MLA_ERR_UNSUPPORTED
    # the paper's default (6,5,5)-pair split, 96/32 split and d_q = 768 are valid, and a sink
    assert B.mla_config_check(cfg(rope_t=12, rope_h=10, rope_w=10)) == B.MLA_OK
    assert B.mla_config_check(cfg(d_nope=96, d_q=768)) == B.MLA_OK
    assert B.mla_config_check(cfg(sink_frames=1, window_frames=6)) == B.MLA_OK
    for over in (dict(d_q=-1), dict(sink_frames=-1)):
        assert B.mla_config_check(cfg(**over)) == B.MLA_ERR_INVALID_ARGUMENT, over


def test_ring_slot_matches_oracle_exactly():
    for W, fh, fw in ((21, 30, 52), (2, 4, 6), (63, 30, 52), (1, 1, 1), (5, 3, 7)):
        c = cfg(window_frames=W, frame_h=fh, frame_w=fw)
        F = fh * fw
        for f in list(range(0, 3 * W + 2)) + [10**6 + 7, 2**40 + 3]:
            for k in sorted({0, min(1, F - 1), F // 2, F - 1}):
                assert B.mla_ring_slot(c, f, k) == ring_slot(f, k, W, F)
    with pytest.raises(B.MLAError):
        B.mla_ring_slot(cfg(), -1, 0)
    with pytest.raises(B.MLAError):
        B.mla_ring_slot(cfg(), 0, 1560)


def test_cache_named_slot_and_bytes():
    # The boundary's cache-named forms: mla_cache_bytes is the ring footprint; mla_cache_slot
    # reads the configuration of a cache, so without a GPU only its argument checks run.
    for over in ({}, dict(batch=4), dict(sink_frames=1), dict(window_frames=63)):
        assert B.mla_cache_bytes(cfg(**over)) == B.mla_ring_bytes(cfg(**over))
    assert B.mla_cache_bytes(cfg(d_latent=0)) == 0
    lib = B.load_library()
    out = ctypes.c_int64(-5)
    assert lib.mla_cache_slot(None, 0, 0, ctypes.byref(out)) == B.MLA_ERR_INVALID_ARGUMENT
    assert out.value == -5


def test_ring_slot_with_sink_matches_fifo_simulation():
    # Sink frames keep their own buffer for good (rows f*F of a sink region rounded up to whole
    # 128-row key tiles); the other frames cycle through W window buffers like a FIFO.  The
    # closed form of mla_ring_slot must name the same row as this simulation.
    from collections import deque
    for S, W, fh, fw in ((1, 6, 30, 52), (1, 2, 4, 6), (2, 3, 3, 5), (3, 1, 1, 1)):
        F = fh * fw
        sink_rows = -(-S * F // 128) * 128
        c = cfg(window_frames=W, frame_h=fh, frame_w=fw, sink_frames=S)
        fifo, owner, fresh = deque(), {}, 0
        for f in range(S + 3 * W + 2):
            if f < S:
                owner[f] = ("sink", f)
            else:
                if len(fifo) == W:
                    buf = owner.pop(fifo.popleft())[1]
                else:
                    buf, fresh = fresh, fresh + 1
                owner[f] = ("win", buf)
                fifo.append(f)
            for g, (kind, buf) in owner.items():
                row0 = buf * F if kind == "sink" else sink_rows + buf * F
                for k in sorted({0, F // 2, F - 1}):
                    assert B.mla_ring_slot(c, g, k) == row0 + k, (S, W, g, k)
        assert B.mla_ring_bytes(c) == (S + W) * F * 224 * 2


def test_ring_bytes_reproduce_printed_accounting():
    g = json.load(open(os.path.join(ROOT, "tests", "golden", "accounting.json")))
    d = g["dims"]
    per_layer = B.mla_ring_bytes(cfg())
    assert per_layer == 21 * 1560 * 224 * 2
    dense_bytes = cache_scalars(d["layers"], d["window_frames"], d["tokens_per_frame"],
                                dense_scalars_per_token(d["n_heads"], d["d_head"])) * 2
    assert round(dense_bytes / 1e9, 1) == g["dense_cache_gb_bf16"]["value"]
    assert round(dense_bytes / (d["layers"] * per_layer), 1) == g["reduction_factor"]["value"]
    assert B.mla_ring_bytes(cfg(batch=4)) == 4 * per_layer
    assert B.mla_cache_device_bytes(cfg()) > per_layer
    assert B.mla_cache_device_bytes(cfg(d_latent=128)) == 0
    # The paper's 96 + 32 split enables the reconstruct-then-dense call, whose per-head weights
    # (W_Qd and W_O: 1536 x 1536 bf16 each, W_UV: 1536 x 192 and W_UK: 1152 x 192 fp16) come on top.
    # Its query weights are the absorbed bf16 pairs (13 x 224 rows of 2 x 1536 bf16), while the
    # full-rank d_nope = 128 query keeps the caller's rows (12 x 160 rows, padded to 2016, then
    # 224 latent rows, of 1536 bf16) and W_UK (1536 x 192 fp16).
    wan = B.mla_cache_device_bytes(cfg(d_nope=128))
    paper = B.mla_cache_device_bytes(cfg(d_nope=96))
    pair = 13 * 224 * 2 * 1536 * 2
    two_step = (2016 + 224) * 1536 * 2 + 1536 * 192 * 2
    assert paper - wan == 2 * 1536 * 1536 * 2 + 1536 * 192 * 2 + 1152 * 192 * 2 + pair - two_step
    # A sink frame adds its padded region (1560 -> 1664 rows) to the planes.
    assert B.mla_cache_device_bytes(cfg(sink_frames=1)) - B.mla_cache_device_bytes(cfg()) == 1664 * 224 * 2


def test_calls_validate_before_any_device_work():
    lib = B.load_library()
    c = cfg()
    out = ctypes.c_void_p(1234)
    assert lib.mla_cache_create(ctypes.byref(c), None, None, ctypes.byref(out)) == B.MLA_ERR_INVALID_ARGUMENT
    assert out.value is None
    bad = cfg(window_frames=0)
    w = B.mla_weights()
    assert lib.mla_cache_create(ctypes.byref(bad), ctypes.byref(w), None, ctypes.byref(out)) == B.MLA_ERR_INVALID_ARGUMENT
    assert lib.mla_cache_append(None, None, 1, None) == B.MLA_ERR_INVALID_ARGUMENT
    assert lib.mla_window_attention(None, None, 1, None, None) == B.MLA_ERR_INVALID_ARGUMENT
    assert lib.mla_cache_sync(None, None) == B.MLA_ERR_INVALID_ARGUMENT
    assert lib.mla_cache_commit(None, 1, None) == B.MLA_ERR_INVALID_ARGUMENT
    lib.mla_cache_destroy(None)  # NULL-safe
    assert lib.mla_status_string(5) == b"MLA_ERR_DEVICE_TIMEOUT"
    assert lib.mla_status_string(B.MLA_ERR_RANGE) == b"MLA_ERR_RANGE"


def test_binding_checks_tensor_extents_before_calling():
    """The C calls take a pointer and a frame count; the binding checks that the tensors really
    are [batch, n * F, hidden] (and out the same) so that no call can read or write past them."""
    import torch
    c = B.LatentWindowCache.__new__(B.LatentWindowCache)   # no device: only the shape logic
    c.cfg, c.F, c.handle = cfg(batch=2), 30 * 52, None
    F, H = c.F, c.cfg.hidden
    assert c._frames(torch.empty(2, 3 * F, H), "x") == 3
    for bad in [(2, 3 * F + 1, H), (1, F, H), (2, F, H + 1), (2, 0, H), (3 * F, H)]:
        with pytest.raises(ValueError):
            c._frames(torch.empty(bad), "x")
    x = torch.empty(2, F, H)
    assert c._out_for(x, torch.empty(2, F, H)).shape == x.shape
    with pytest.raises(ValueError):
        c._out_for(x, torch.empty(2, F - 1, H))
    q, kv = torch.empty(1, 5, 2, 128, dtype=torch.bfloat16), torch.empty(1, 7, 2, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        B.mla_dense_attention(q, kv, torch.empty(1, 6, 2, 128, dtype=torch.bfloat16), q.clone())
    with pytest.raises(ValueError):
        B.mla_dense_attention(q, kv, kv, torch.empty(1, 4, 2, 128, dtype=torch.bfloat16))


def test_dense_split_plan_covers_every_key_once():
    """The key ranges the dense kernel launches: whole 128-key tiles, the last range non-empty,
    together exactly [0, n_kv); one range without a workspace; never more than 8, and the grid's
    z extent (batch x ranges) within 65,535.  At the 21-frame, one-frame Wan shape (156 items on
    148 SMs) the plan splits; with 444 items (three frames: three full waves) it does not."""
    import random
    big = 1 << 40
    rng = random.Random(5)
    shapes = [(1, 1560, 34320, 12), (1, 4680, 37440, 12), (2, 200, 1000, 3), (1, 5, 130, 2),
              (1, 128, 128, 1), (3, 300, 77, 4), (1, 130, 1281, 2), (1, 40, 1, 2), (65535, 1, 5000, 1)]
    shapes += [(rng.randint(1, 4), rng.randint(1, 5000), rng.randint(1, 120000), rng.randint(1, 16))
               for _ in range(200)]
    for batch, nq, nkv, nh in shapes:
        for sms in (1, 7, 148):
            assert B.mla_dense_split_plan(batch, nq, nkv, nh, sms, 0) == (1, nkv)
            prev = 1
            for ws in (1 << 20, 1 << 26, big):
                s, per = B.mla_dense_split_plan(batch, nq, nkv, nh, sms, ws)
                assert 1 <= s <= 8 and batch * s <= 65535
                if s == 1:
                    assert per == nkv
                else:
                    assert per % 128 == 0 and (s - 1) * per < nkv <= s * per
                assert s >= prev or ws == (1 << 20)
                prev = s
    assert B.mla_dense_split_plan(1, 1560, 34320, 12, 148, big)[0] > 1
    assert B.mla_dense_split_plan(1, 4680, 37440, 12, 148, big)[0] == 1
    with pytest.raises(B.MLAError):
        B.mla_dense_split_plan(0, 1, 1, 1, 148, big)
