"""ctypes binding of libmla.so: the C ABI of include/mla.h, same names, argument marshalling only.

Every step of the attention path runs in the library's CUDA kernels; this module only turns
torch tensors into device pointers and streams into cudaStream_t handles.  There is no fallback:
if the shared library is missing or the device is not an sm_100 GPU, calls raise.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
# MLA_LIBRARY selects another build of the same library (the MLA_DEBUG build, libmla_debug.so).
LIB_PATH = os.environ.get("MLA_LIBRARY") or os.path.join(HERE, "libmla.so")

# mla_status values
MLA_OK = 0
MLA_ERR_INVALID_ARGUMENT = 1
MLA_ERR_UNSUPPORTED = 2
MLA_ERR_OUT_OF_MEMORY = 3
MLA_ERR_CUDA = 4
MLA_ERR_DEVICE_TIMEOUT = 5
MLA_ERR_STATE = 6
MLA_ERR_RANGE = 7
MLA_ERR_BOUNDS = 8

MLA_KERNEL_APPEND, MLA_KERNEL_QPROJ, MLA_KERNEL_ATTENTION, MLA_KERNEL_OPROJ = range(4)
KERNEL_NAMES = ("append", "qproj", "attention", "oproj")

EXPORTED = (
    "mla_config_check", "mla_ring_slot", "mla_ring_bytes", "mla_cache_slot", "mla_cache_bytes",
    "mla_cache_device_bytes",
    "mla_cache_create", "mla_cache_append", "mla_cache_commit", "mla_commit_plan", "mla_window_attention",
    "mla_window_attention_noalloc",
    "mla_window_attention_reconstruct", "mla_cache_selftest_timeout", "mla_cache_selftest_bounds",
    "mla_cache_destroy", "mla_dense_split_plan", "mla_dense_workspace_bytes", "mla_dense_attention",
    "mla_dense_sync",
    "mla_cache_state", "mla_cache_sync", "mla_cache_read", "mla_cache_debug_buffers", "mla_cache_copy_buffer",
    "mla_cache_profile_enable", "mla_cache_profile_read", "mla_status_string", "mla_last_error",
)


class MLAError(RuntimeError):
    def __init__(self, status: int, where: str, message: str):
        super().__init__(f"{where}: {_status_name(status)}: {message}")
        self.status = status


class mla_config(ctypes.Structure):
    _fields_ = [
        ("hidden", ctypes.c_int32), ("n_heads", ctypes.c_int32), ("d_head", ctypes.c_int32),
        ("d_nope", ctypes.c_int32), ("d_latent", ctypes.c_int32), ("d_rope", ctypes.c_int32),
        ("rope_t", ctypes.c_int32), ("rope_h", ctypes.c_int32), ("rope_w", ctypes.c_int32),
        ("rope_base", ctypes.c_double),
        ("frame_h", ctypes.c_int32), ("frame_w", ctypes.c_int32),
        ("window_frames", ctypes.c_int32), ("max_chunk_frames", ctypes.c_int32),
        ("batch", ctypes.c_int32), ("softmax_scale", ctypes.c_float),
        ("d_q", ctypes.c_int32), ("sink_frames", ctypes.c_int32),
    ]


class mla_weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("w_q", "w_qr", "w_dkv", "w_kr", "w_uk", "w_uv", "w_o", "w_dq")]


class mla_debug_buffers(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("ckv", "krope", "qp", "o_lat", "w_qcat", "w_ov")] + \
        [("rows_per_stream", ctypes.c_int64)]


class mla_row_move(ctypes.Structure):
    _fields_ = [("src_row", ctypes.c_int64), ("dst_row", ctypes.c_int64), ("rows", ctypes.c_int64)]


class mla_profile(ctypes.Structure):
    _fields_ = [("ms", ctypes.c_double * 4), ("launches", ctypes.c_int64 * 4)]


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libmla.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"libmla.so not built at {path}: run mla_latent_kv_window_b200/build.py")
    lib = ctypes.CDLL(path)
    P, I32, I64, VP = ctypes.POINTER, ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p
    sig = {
        "mla_config_check": (I32, [P(mla_config)]),
        "mla_ring_slot": (I32, [P(mla_config), I64, I32, P(I64)]),
        "mla_ring_bytes": (ctypes.c_size_t, [P(mla_config)]),
        "mla_cache_slot": (I32, [VP, I64, I32, P(I64)]),
        "mla_cache_bytes": (ctypes.c_size_t, [P(mla_config)]),
        "mla_cache_device_bytes": (ctypes.c_size_t, [P(mla_config)]),
        "mla_cache_create": (I32, [P(mla_config), P(mla_weights), VP, P(VP)]),
        "mla_cache_append": (I32, [VP, VP, I32, VP]),
        "mla_cache_commit": (I32, [VP, I32, VP]),
        "mla_commit_plan": (I32, [P(mla_config), I64, I32, P(mla_row_move), I32, P(I32)]),
        "mla_window_attention": (I32, [VP, VP, I32, VP, VP]),
        "mla_window_attention_noalloc": (I32, [VP, VP, I32, VP, VP]),
        "mla_window_attention_reconstruct": (I32, [VP, VP, I32, VP, VP]),
        "mla_cache_selftest_timeout": (I32, [VP, VP, P(I32)]),
        "mla_cache_selftest_bounds": (I32, [VP, VP, P(I32)]),
        "mla_dense_split_plan": (I32, [I32, I32, I32, I32, I32, ctypes.c_size_t, P(I32), P(I32)]),
        "mla_dense_workspace_bytes": (ctypes.c_size_t, [I32, I32, I32, I32]),
        "mla_dense_attention": (I32, [VP, VP, VP, VP, I32, I32, I32, I32, I32, ctypes.c_float, VP,
                                      ctypes.c_size_t, VP]),
        "mla_dense_sync": (I32, [VP]),
        "mla_cache_destroy": (None, [VP]),
        "mla_cache_state": (I32, [VP, P(I64), P(I32)]),
        "mla_cache_sync": (I32, [VP, VP]),
        "mla_cache_read": (I32, [VP, I32, VP, VP, P(I64)]),
        "mla_cache_debug_buffers": (I32, [VP, P(mla_debug_buffers)]),
        "mla_cache_copy_buffer": (I32, [VP, I32, VP, ctypes.c_size_t, P(ctypes.c_size_t)]),
        "mla_cache_profile_enable": (I32, [VP, I32]),
        "mla_cache_profile_read": (I32, [VP, P(mla_profile)]),
        "mla_status_string": (ctypes.c_char_p, [I32]),
        "mla_last_error": (ctypes.c_char_p, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype, fn.argtypes = res, args
    _lib = lib
    return lib


def _status_name(s: int) -> str:
    try:
        return load_library().mla_status_string(s).decode()
    except Exception:  # pragma: no cover - only when the library itself is missing
        return str(s)


def _check(status: int, where: str) -> None:
    if status != MLA_OK:
        raise MLAError(status, where, load_library().mla_last_error().decode())


def make_config(dims: dict, frame_h: int, frame_w: int, window_frames: int, max_chunk_frames: int,
                batch: int = 1, softmax_scale: float = 0.0, sink_frames: int = 0) -> mla_config:
    return mla_config(
        hidden=dims["hidden"], n_heads=dims["n_heads"], d_head=dims["d_head"], d_nope=dims["d_nope"],
        d_latent=dims["d_latent"], d_rope=dims["d_rope"], rope_t=dims["rope_t"], rope_h=dims["rope_h"],
        rope_w=dims["rope_w"], rope_base=float(dims["rope_base"]), frame_h=frame_h, frame_w=frame_w,
        window_frames=window_frames, max_chunk_frames=max_chunk_frames, batch=batch,
        softmax_scale=softmax_scale, d_q=int(dims.get("d_q", 0)), sink_frames=sink_frames)


# ---------------------------------------------------------------------------- C names, torch args
def _stream_handle(stream) -> int:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


def _dev_ptr(t, name: str) -> int:
    import torch
    if not (t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous()):
        raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor")
    return int(t.data_ptr())


def mla_config_check(cfg: mla_config) -> int:
    return load_library().mla_config_check(ctypes.byref(cfg))


def mla_ring_slot(cfg: mla_config, frame: int, token: int) -> int:
    out = ctypes.c_int64()
    _check(load_library().mla_ring_slot(ctypes.byref(cfg), frame, token, ctypes.byref(out)), "mla_ring_slot")
    return out.value


def mla_ring_bytes(cfg: mla_config) -> int:
    return int(load_library().mla_ring_bytes(ctypes.byref(cfg)))


def mla_cache_slot(handle, frame: int, token: int) -> int:
    """mla_ring_slot for the configuration the cache was created with."""
    out = ctypes.c_int64()
    _check(load_library().mla_cache_slot(handle, frame, token, ctypes.byref(out)), "mla_cache_slot")
    return out.value


def mla_cache_bytes(cfg: mla_config) -> int:
    return int(load_library().mla_cache_bytes(ctypes.byref(cfg)))


def mla_cache_device_bytes(cfg: mla_config) -> int:
    return int(load_library().mla_cache_device_bytes(ctypes.byref(cfg)))


def mla_cache_create(cfg: mla_config, weights: dict, stream=None) -> int:
    w = mla_weights(**{k: _dev_ptr(weights[k], k) for k in ("w_q", "w_qr", "w_dkv", "w_kr", "w_uk", "w_uv", "w_o")})
    if cfg.d_q > 0:
        w.w_dq = _dev_ptr(weights["w_dq"], "w_dq")
    h = ctypes.c_void_p()
    _check(load_library().mla_cache_create(ctypes.byref(cfg), ctypes.byref(w), _stream_handle(stream),
                                           ctypes.byref(h)), "mla_cache_create")
    return h.value


def mla_cache_append(cache: int, x, n_frames: int, stream=None) -> None:
    _check(load_library().mla_cache_append(cache, _dev_ptr(x, "x"), n_frames, _stream_handle(stream)),
           "mla_cache_append")


def mla_cache_commit(cache: int, n_frames: int, stream=None) -> None:
    _check(load_library().mla_cache_commit(cache, n_frames, _stream_handle(stream)), "mla_cache_commit")


def mla_commit_plan(cfg: mla_config, frames_appended: int, n_frames: int) -> list:
    """Host-only: the (src_row, dst_row, rows) moves mla_cache_commit makes, in order."""
    buf = (mla_row_move * max(n_frames, 1))()
    n = ctypes.c_int32()
    _check(load_library().mla_commit_plan(ctypes.byref(cfg), frames_appended, n_frames, buf,
                                          max(n_frames, 1), ctypes.byref(n)), "mla_commit_plan")
    return [(buf[i].src_row, buf[i].dst_row, buf[i].rows) for i in range(n.value)]


def mla_window_attention(cache: int, x_chunk, n_frames: int, out, stream=None) -> None:
    _check(load_library().mla_window_attention(cache, _dev_ptr(x_chunk, "x_chunk"), n_frames,
                                               _dev_ptr(out, "out"), _stream_handle(stream)),
           "mla_window_attention")


def mla_window_attention_noalloc(cache: int, x_chunk, n_frames: int, out, stream=None) -> None:
    """mla_window_attention with its per-call scratch in the library's fixed 32 MiB device array
    (no device allocation in the call); see include/mla.h for the size limit and sharing rules."""
    _check(load_library().mla_window_attention_noalloc(cache, _dev_ptr(x_chunk, "x_chunk"), n_frames,
                                                       _dev_ptr(out, "out"), _stream_handle(stream)),
           "mla_window_attention_noalloc")


def mla_window_attention_reconstruct(cache: int, x_chunk, n_frames: int, out, stream=None) -> None:
    """mla_window_attention computed as reconstruct-then-dense (per-head K/V materialised)."""
    _check(load_library().mla_window_attention_reconstruct(cache, _dev_ptr(x_chunk, "x_chunk"), n_frames,
                                                           _dev_ptr(out, "out"), _stream_handle(stream)),
           "mla_window_attention_reconstruct")


def mla_cache_selftest_timeout(cache: int, stream=None) -> bool:
    """Run the bounded-wait self-test (about 2 s); True when the device wait gave up."""
    flag = ctypes.c_int32()
    _check(load_library().mla_cache_selftest_timeout(cache, _stream_handle(stream), ctypes.byref(flag)),
           "mla_cache_selftest_timeout")
    return flag.value == 1


def mla_cache_selftest_bounds(cache: int, stream=None) -> bool:
    """Run the debug build's bounds-check self-test; True when the kernel's check caught the
    out-of-range row (raises MLAError with MLA_ERR_UNSUPPORTED on the normal build)."""
    flag = ctypes.c_int32()
    _check(load_library().mla_cache_selftest_bounds(cache, _stream_handle(stream), ctypes.byref(flag)),
           "mla_cache_selftest_bounds")
    return flag.value == 1


def mla_dense_split_plan(batch: int, n_q: int, n_kv: int, n_heads: int, num_sms: int,
                         workspace_bytes: int) -> tuple[int, int]:
    """(key ranges per item, keys per range) that mla_dense_attention would launch (host only)."""
    sp, kv = ctypes.c_int32(), ctypes.c_int32()
    _check(load_library().mla_dense_split_plan(batch, n_q, n_kv, n_heads, num_sms, workspace_bytes,
                                               ctypes.byref(sp), ctypes.byref(kv)), "mla_dense_split_plan")
    return sp.value, kv.value


def mla_dense_workspace_bytes(batch: int, n_q: int, n_kv: int, n_heads: int) -> int:
    return int(load_library().mla_dense_workspace_bytes(batch, n_q, n_kv, n_heads))


def mla_dense_attention(q, k, v, out, softmax_scale: float = 0.0, stream=None, workspace=None) -> None:
    """Dense per-head attention baseline: q [B, n_q, H, 128], k/v [B, n_kv, H, 128], out like q (bf16).
    workspace: None runs one pass per item; otherwise a uint8 device tensor (see
    mla_dense_workspace_bytes) that holds the split-key partials."""
    B, nq, H, D = q.shape
    if k.dim() != 4 or k.shape[0] != B or k.shape[2:] != q.shape[2:] or v.shape != k.shape:
        raise ValueError(f"k and v must be [{B}, n_kv, {H}, {D}] like each other; got {tuple(k.shape)}, "
                         f"{tuple(v.shape)}")
    if out.shape != q.shape:
        raise ValueError(f"out must have the shape of q {tuple(q.shape)}; got {tuple(out.shape)}")
    ws, ws_bytes = None, 0
    if workspace is not None and workspace.numel() > 0:
        if not (workspace.is_cuda and workspace.is_contiguous()):
            raise ValueError("workspace must be a contiguous CUDA tensor")
        ws, ws_bytes = int(workspace.data_ptr()), workspace.numel() * workspace.element_size()
    _check(load_library().mla_dense_attention(_dev_ptr(q, "q"), _dev_ptr(k, "k"), _dev_ptr(v, "v"),
                                              _dev_ptr(out, "out"), B, nq, k.shape[1], H, D,
                                              float(softmax_scale), ws, ws_bytes, _stream_handle(stream)),
           "mla_dense_attention")


def mla_dense_sync(stream=None) -> int:
    return load_library().mla_dense_sync(_stream_handle(stream))


def mla_cache_destroy(cache: int) -> None:
    load_library().mla_cache_destroy(cache)


def mla_cache_state(cache: int):
    fa, vf = ctypes.c_int64(), ctypes.c_int32()
    _check(load_library().mla_cache_state(cache, ctypes.byref(fa), ctypes.byref(vf)), "mla_cache_state")
    return fa.value, vf.value


def mla_cache_sync(cache: int, stream=None) -> int:
    return load_library().mla_cache_sync(cache, _stream_handle(stream))


def mla_cache_read(cache: int, b: int, ckv_host=None, krope_host=None) -> int:
    n = ctypes.c_int64()
    _check(load_library().mla_cache_read(cache, b, None if ckv_host is None else ckv_host.data_ptr(),
                                         None if krope_host is None else krope_host.data_ptr(),
                                         ctypes.byref(n)), "mla_cache_read")
    return n.value


def mla_cache_debug_buffers(cache: int) -> mla_debug_buffers:
    d = mla_debug_buffers()
    _check(load_library().mla_cache_debug_buffers(cache, ctypes.byref(d)), "mla_cache_debug_buffers")
    return d


MLA_BUFFER_QP, MLA_BUFFER_O_LAT, MLA_BUFFER_W_QCAT, MLA_BUFFER_W_OV = range(4)


def mla_cache_copy_buffer(cache: int, which: int, host_out) -> int:
    """Copy the start of an internal buffer into the CPU tensor host_out; returns the buffer size."""
    size = ctypes.c_size_t()
    _check(load_library().mla_cache_copy_buffer(cache, which, host_out.data_ptr(),
                                                host_out.numel() * host_out.element_size(),
                                                ctypes.byref(size)), "mla_cache_copy_buffer")
    return size.value


def mla_cache_profile_enable(cache: int, enable: bool) -> None:
    _check(load_library().mla_cache_profile_enable(cache, int(bool(enable))), "mla_cache_profile_enable")


def mla_cache_profile_read(cache: int) -> dict:
    p = mla_profile()
    _check(load_library().mla_cache_profile_read(cache, ctypes.byref(p)), "mla_cache_profile_read")
    return {KERNEL_NAMES[k]: (p.ms[k], p.launches[k]) for k in range(4)}


# ---------------------------------------------------------------------------- convenience object
class LatentWindowCache:
    """One layer's latent window on the current CUDA device (owns the C handle)."""

    def __init__(self, dims: dict, weights: dict, frame_h: int, frame_w: int, window_frames: int,
                 max_chunk_frames: int, batch: int = 1, softmax_scale: float = 0.0, stream=None,
                 sink_frames: int = 0):
        self.cfg = make_config(dims, frame_h, frame_w, window_frames, max_chunk_frames, batch, softmax_scale,
                               sink_frames)
        self.F = frame_h * frame_w
        self.handle = mla_cache_create(self.cfg, weights, stream)

    def _frames(self, x, name: str) -> int:
        """Whole frames in x, which must be [batch, n * F, hidden] (the C calls take only a pointer
        and a frame count, so the tensor's extent is checked here)."""
        shape = tuple(x.shape)
        if (len(shape) != 3 or shape[0] != self.cfg.batch or shape[2] != self.cfg.hidden or
                shape[1] < self.F or shape[1] % self.F):
            raise ValueError(f"{name} must be [{self.cfg.batch}, n * {self.F}, {self.cfg.hidden}] with "
                             f"n >= 1; got {shape}")
        return shape[1] // self.F

    def _out_for(self, x_chunk, out):
        import torch
        if out is None:
            return torch.empty_like(x_chunk)
        if out.shape != x_chunk.shape:
            raise ValueError(f"out must have the shape of x_chunk {tuple(x_chunk.shape)}; got {tuple(out.shape)}")
        return out

    def append(self, x, stream=None) -> None:
        mla_cache_append(self.handle, x, self._frames(x, "x"), stream)

    def commit(self, n_frames: int, stream=None) -> None:
        mla_cache_commit(self.handle, n_frames, stream)

    def attention(self, x_chunk, out=None, stream=None):
        n = self._frames(x_chunk, "x_chunk")
        out = self._out_for(x_chunk, out)
        mla_window_attention(self.handle, x_chunk, n, out, stream)
        return out

    def attention_reconstruct(self, x_chunk, out=None, stream=None):
        n = self._frames(x_chunk, "x_chunk")
        out = self._out_for(x_chunk, out)
        mla_window_attention_reconstruct(self.handle, x_chunk, n, out, stream)
        return out

    def state(self):
        return mla_cache_state(self.handle)

    def sink_rows(self) -> int:
        """Rows of the sink region: sink_frames * F rounded up to a multiple of 128."""
        return (self.cfg.sink_frames * self.F + 127) // 128 * 128

    def sync(self, stream=None) -> None:
        _check(mla_cache_sync(self.handle, stream), "mla_cache_sync")

    def read_ring(self, b: int = 0):
        """(ckv [rows, 192], krope [rows, 32]) fp16 of stream b in physical row order (rows =
        sink rows + W*F, see mla_ring_slot), and the valid row count."""
        import torch
        rows = self.sink_rows() + self.cfg.window_frames * self.F
        ckv = torch.empty(rows, self.cfg.d_latent, dtype=torch.float16)
        kr = torch.empty(rows, self.cfg.d_rope, dtype=torch.float16)
        n = mla_cache_read(self.handle, b, ckv, kr)
        return ckv, kr, n

    def copy_buffer(self, which: int, shape):
        """Host copy (tensor of `shape`) of an internal buffer: MLA_BUFFER_QP, _O_LAT, _W_OV (fp16)
        or MLA_BUFFER_W_QCAT (bf16)."""
        import torch
        out = torch.empty(shape, dtype=torch.bfloat16 if which == MLA_BUFFER_W_QCAT else torch.float16)
        mla_cache_copy_buffer(self.handle, which, out)
        return out

    def close(self) -> None:
        if getattr(self, "handle", None):
            mla_cache_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
