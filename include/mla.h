/*
 * mla.h - C ABI of the VideoMLA latent-window attention library (libmla.so, sm_100a).
 *
 * Source of the method: "VideoMLA: Low-Rank Latent KV Cache for Minute-Scale
 * Autoregressive Video Diffusion" (paper text page), cited as [VideoMLA] with its section.
 *
 * The library keeps, per attention layer, a sliding window of the last W latent frames.
 * Each cached token stores one head-shared content latent c_kv (d_latent scalars) and one
 * head-shared decoupled 3D-RoPE key k_rope (d_rope scalars): 192 + 32 = 224 scalars instead
 * of 2 x 12 x 128 = 3072 for a dense per-head K/V cache ([VideoMLA] §1, §3.1, §3.2).
 * The current chunk's queries attend to the window plus the chunk itself through
 * W_UK-absorbed scores q_c . c_kv + q_rope . k_rope, an online softmax, P . c_kv, and the
 * W_UV / W_O up-projections folded into one output projection.
 *
 * Precision: the caller's hidden states, weights and outputs are bf16.  The cached latent
 * (c_kv, k_rope), the absorbed queries, the softmax weights P, the latent-space output and the
 * folded output weight are 16-bit fp16 internally (the paper sizes the cache as bf16/fp16; fp16
 * keeps three more mantissa bits for the same 448 bytes per token), saturating at +-65504; every
 * product accumulates in fp32.
 *
 * Conventions shared by every call:
 *  - Tensors are bf16, row-major, 16-byte aligned device pointers unless stated otherwise.
 *  - Weights follow the nn.Linear layout [out_features, in_features] with head-major output
 *    channels (channel c = head * dim + j).
 *  - Hidden states are [batch, n_frames * F, hidden], F = frame_h * frame_w tokens per latent
 *    frame, tokens of a frame in row-major (h, w) order ([VideoMLA] App. C.1, S = F H W).
 *  - Positions are implicit: the i-th frame ever appended has temporal index t = i; a query
 *    chunk gets the indices the next append will use.  Token k of a frame sits at
 *    (h, w) = (k / frame_w, k % frame_w).  Angles are formed in fp32 from t, exact for
 *    t < 2^24: an append or attention call that would reach frame index 2^24 returns
 *    MLA_ERR_UNSUPPORTED (2^24 latent frames are days of video).
 *  - Calls are stream-ordered and asynchronous: append and attention make no host sync.
 *    `stream` is a cudaStream_t (NULL = legacy default stream).
 *  - Errors: arguments are validated on the host before anything is launched; a failed check
 *    returns MLA_ERR_INVALID_ARGUMENT / MLA_ERR_UNSUPPORTED / MLA_ERR_STATE and changes no
 *    state.  Kernels never trap: a device-side wait that runs out of time sets the cache's
 *    status word, which mla_cache_sync() returns as MLA_ERR_DEVICE_TIMEOUT.
 *  - Range: the cache planes (c_kv, k_rope), the absorbed queries, P and o_lat are fp16
 *    internally (16-bit like the paper's bf16/fp16 cache, [VideoMLA] §1; fp16 keeps three more
 *    mantissa bits, bf16 more exponent range).  A projected value whose magnitude exceeds
 *    65504 (the fp16 maximum) is clamped to +-65504; the kernel records it and computes on,
 *    and the next mla_cache_sync() returns MLA_ERR_RANGE once.  P is bounded by 256 and o_lat
 *    by the largest cached |c_kv|, so only the projections can clamp.  Hidden states and
 *    weights stay bf16, out is bf16.
 *  - Debug build (libmla_debug.so, the same sources compiled with MLA_DEBUG): every plain
 *    global access whose index a kernel computes is bounds-checked first (a violation skips the
 *    access and records MLA_ERR_BOUNDS in the status word), the tensor maps over the library's
 *    own buffers are checked against the buffers' extents on the host, and every device buffer
 *    of a cache carries a 4 KiB guard band that mla_cache_sync checks (MLA_ERR_BOUNDS when a
 *    kernel wrote into one).  A stand-in for a memory checker; same results, slower.
 *  - Threading: a cache may be used by one host thread and one stream at a time.
 */
#ifndef MLA_LATENT_WINDOW_H
#define MLA_LATENT_WINDOW_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct mla_cache mla_cache; /* opaque */

typedef enum {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARGUMENT = 1, /* bad shape, pointer, alignment or size          */
  MLA_ERR_UNSUPPORTED = 2,      /* valid for the method, not built into the kernels */
  MLA_ERR_OUT_OF_MEMORY = 3,    /* cudaMalloc failed                                 */
  MLA_ERR_CUDA = 4,             /* a CUDA runtime call failed                        */
  MLA_ERR_DEVICE_TIMEOUT = 5,   /* a kernel's bounded wait ran out (status word)    */
  MLA_ERR_STATE = 6,            /* call not valid in the cache's current state      */
  MLA_ERR_RANGE = 7,            /* a value exceeded the fp16 range and was clamped   */
  MLA_ERR_BOUNDS = 8            /* debug build: an index or a guard band out of range */
} mla_status;

/* The problem statement of one attention layer ([VideoMLA] §3, §4.1, App. D.1).
 * Built kernels: d_latent == 192 and d_rope == 32; hidden a multiple of 128. */
typedef struct {
  int32_t hidden;           /* model width d (1536 for Wan-1.3B)                         */
  int32_t n_heads;          /* n_h (12)                                                  */
  int32_t d_head;           /* value width per head, W_O input per head (128)            */
  int32_t d_nope;           /* content-key width per head (128 here; 96 in §4.1 default) */
  int32_t d_latent;         /* d_c, shared content latent (192)                          */
  int32_t d_rope;           /* d_h^rope, shared positional key (32)                      */
  int32_t rope_t, rope_h, rope_w; /* channels per axis; each even, sum == d_rope        */
  double rope_base;         /* RoPE base (10000); pair i of axis a turns at base^(-2i/d_a) */
  int32_t frame_h, frame_w; /* latent-frame token grid (30 x 52 -> F = 1560)             */
  int32_t window_frames;    /* W: cached latent frames kept in the ring (21)             */
  int32_t max_chunk_frames; /* largest query chunk, in frames (3)                        */
  int32_t batch;            /* B independent streams sharing the weights                 */
  float softmax_scale;      /* 0 -> 1 / sqrt(d_nope + d_rope)                            */
  int32_t d_q;              /* low-rank query width ([VideoMLA] §4.1 default: 768); 0 -> the
                               query projections read x directly (full-rank W_Q)           */
  int32_t sink_frames;      /* first frames of the video kept for good besides the window
                               ([VideoMLA] App. D.4/D.5 "sink + local window"); 0 -> none   */
} mla_config;

/* Device bf16 weights, nn.Linear layout [out, in]:
 *  w_q  [n_heads*d_nope, q_in]      w_qr [n_heads*d_rope, q_in]
 *  w_dkv[d_latent, hidden]          w_kr [d_rope, hidden]
 *  w_uk [n_heads*d_nope, d_latent]  w_uv [n_heads*d_head, d_latent]
 *  w_o  [hidden, n_heads*d_head]    w_dq [d_q, hidden] (only with d_q > 0, else ignored)
 * q_in = hidden for a full-rank query (d_q == 0); with d_q > 0 the query projections read the
 * low-rank query latent c_q = x W_DQ^T and q_in = d_q.
 * Read only during mla_cache_create; the caller keeps ownership. */
typedef struct {
  const void *w_q, *w_qr, *w_dkv, *w_kr, *w_uk, *w_uv, *w_o;
  const void* w_dq;
} mla_weights;

/* Validate a configuration on the host (no GPU needed).  MLA_OK, MLA_ERR_INVALID_ARGUMENT
 * for values the method does not allow, MLA_ERR_UNSUPPORTED for values the kernels lack. */
mla_status mla_config_check(const mla_config* cfg);

/* Physical row of (absolute frame index, token in frame) in a stream's latent planes
 * ([VideoMLA] §1, App. D.4: fixed-size sliding window of W latent frames, oldest evicted):
 *   no sink:                      (frame mod W) * F + token
 *   frame < sink_frames:          frame * F + token               (sink frames, kept for good)
 *   otherwise:                    sink_rows + ((frame - sink_frames) mod W) * F + token
 * with sink_rows = sink_frames * F rounded up to a multiple of 128 (the sink region ends on a
 * key-tile boundary; its padding rows are never attended).
 * Host only.  MLA_ERR_INVALID_ARGUMENT for frame < 0 or token outside [0, F). */
mla_status mla_ring_slot(const mla_config* cfg, int64_t frame, int32_t token, int64_t* slot);

/* Bytes of the latent window itself: batch * (sink_frames + W) * F * (d_latent + d_rope) * 2
 * (16-bit cache). */
size_t mla_ring_bytes(const mla_config* cfg);

/* The same two host-only functions under the names of a cache: mla_cache_slot is mla_ring_slot
 * for the configuration c was created with (MLA_ERR_INVALID_ARGUMENT for a NULL c or slot, and
 * as mla_ring_slot otherwise); mla_cache_bytes is mla_ring_bytes (the ring footprint; 0 for a
 * NULL or invalid config). */
mla_status mla_cache_slot(const mla_cache* c, int64_t frame, int32_t token, int64_t* slot);
size_t mla_cache_bytes(const mla_config* cfg);

/* Bytes of device memory mla_cache_create allocates for this configuration (ring with its
 * chunk tail, absorbed weights, per-call scratch, status word, RoPE tables, and the per-head
 * weights of mla_window_attention_reconstruct when the configuration allows that call).
 * 0 for an invalid config. */
size_t mla_cache_device_bytes(const mla_config* cfg);

/* Create a cache on the current device.  Owns the projection weights in the form the kernels
 * multiply, the RoPE tables and a zeroed ring ([VideoMLA] §3.3 reconstructs per-head K/V from
 * the latent through W_UK/W_UV; folding them into the query and output projections is the
 * standard MLA absorption):
 *   queries, full-rank W_Q with d_nope = 128: the caller's W_Q, W_QR, W_DKV, W_KR (bf16) and
 *             W_UK (fp16); a query projection forms q = W_Q[h] x and then W_UK[h]^T q, so the
 *             product W_UK[h]^T W_Q[h] is never rounded;
 *   queries, other head splits or a low-rank query: W_Qabs[h] = W_UK[h]^T W_Q[h] (with a
 *             low-rank query W_UK[h]^T W_Q[h] W_DQ, and W_QR W_DQ for the RoPE part) composed
 *             in fp32 and kept as a bf16 pair hi + lo;
 *   outputs:  W_OV[h] = W_O[:, h] W_UV[h] (d_latent per head -> hidden), fp16.
 * Synchronises `stream` once before returning, so the caller may free the
 * weights afterwards.  *out receives the handle (NULL on failure).  MLA_ERR_RANGE (and no
 * cache) when an fp16 weight - W_OV, W_UK, or the dense form's W_UK / W_UV - exceeds +-65504. */
mla_status mla_cache_create(const mla_config* cfg, const mla_weights* w, void* stream,
                            mla_cache** out);

/* Append n_frames >= 1 whole latent frames x [batch, n_frames*F, hidden] to every stream's
 * window: c_kv = x W_DKV^T and k_rope = RoPE3D(x W_KR^T) at the frames' own (t, h, w), written
 * to the rows mla_ring_slot names ([VideoMLA] §3.1, §3.2): the first sink_frames frames ever
 * appended to the sink, the others to ring slots.  Frames that would be evicted within the
 * call (more than W non-sink frames) are not computed. */
mla_status mla_cache_append(mla_cache* c, const void* x, int32_t n_frames, void* stream);

/* Latent-window attention for one query chunk x_chunk [batch, n_frames*F, hidden],
 * 1 <= n_frames <= max_chunk_frames, writing out [batch, n_frames*F, hidden].
 * The chunk attends to the sink frames, the valid window frames and all of its own tokens
 * (chunk-causal, [VideoMLA] App. D.4).  Positions follow the window-local re-indexing of
 * App. D.5 (sink, window, chunk numbered 0, 1, ...): keys are stored rotated at their absolute
 * frame index, which differs from the local one by a single offset for window and chunk
 * frames; for the sink keys the query's temporal RoPE bands are turned back by that offset.
 * The chunk's latents go to a scratch tail, not into the ring: call mla_cache_append with the
 * final hidden states, or mla_cache_commit when those are this call's x_chunk, to make them
 * part of the window.  With an empty window (nothing appended yet) the chunk attends to itself
 * alone. */
mla_status mla_window_attention(mla_cache* c, const void* x_chunk, int32_t n_frames, void* out,
                                void* stream);

/* Append the chunk of the last attention call on this cache to the window, using the latents
 * that call already computed: the same result as mla_cache_append(c, x_chunk, n_frames) with
 * that call's x_chunk, without reading x_chunk again or recomputing c_kv and k_rope.  This is
 * the rollout's last step of a chunk ([VideoMLA] App. D.4: denoise the chunk against the
 * window, then append its latents) when the hidden states appended are the ones the last
 * denoising step attended with.  The latents move from the chunk tail to the rows
 * mla_ring_slot names (frames already in place are not copied; one small copy kernel per frame
 * that moves).
 *  - n_frames must equal the last attention call's n_frames (mla_window_attention, _noalloc or
 *    _reconstruct), and no append or commit may have happened since; otherwise MLA_ERR_STATE
 *    and nothing changes.
 *  - Stream-ordered like mla_cache_append. */
mla_status mla_cache_commit(mla_cache* c, int32_t n_frames, void* stream);

/* One frame's move inside a stream's latent planes: rows [src_row, src_row + rows) go to
 * [dst_row, dst_row + rows) (both plane rows, per stream). */
typedef struct {
  int64_t src_row, dst_row, rows;
} mla_row_move;

/* Host-only view of the moves mla_cache_commit launches for a chunk of n_frames frames attended
 * when frames_appended frames had been appended: the chunk's latents sit at the chunk tail (the
 * rows right after the valid sink region and window) and each surviving frame goes to the rows
 * mla_ring_slot names for its frame index; frames already in place are not listed, and frames
 * the chunk itself evicts (more than W new window frames) are skipped.  The moves must be applied
 * in the listed order: a destination may be the source of an earlier move, never of a later one.
 * *n_moves receives the count; at most max_moves are written (MLA_ERR_INVALID_ARGUMENT if more
 * are needed, or for an invalid config, n_frames outside [1, max_chunk_frames], or
 * frames_appended < 0).  No GPU needed. */
mla_status mla_commit_plan(const mla_config* cfg, int64_t frames_appended, int32_t n_frames,
                           mla_row_move* moves, int32_t max_moves, int32_t* n_moves);

/* Same computation and result as mla_window_attention, for callers that must not allocate
 * device memory while they run: code whose device memory belongs to a pooled or budgeted
 * allocator it may not bypass, and latency-critical loops that cannot afford the implicit
 * device synchronisation a cudaMalloc/cudaFree can cause.  The paper has no counterpart; this
 * is a property of the library, not of the method.
 *
 * The per-call scratch - absorbed queries and the latent-space attention output, 832 bytes per
 * (stream, query token, head) - lives in one fixed 32 MiB array inside the library on every GPU
 * that loads it (held until the process exits), not in the cache.  This call allocates nothing:
 * no cudaMalloc, no cudaFree, no allocating library routine.  The cache itself still has to be
 * created once, beforehand, with mla_cache_create.
 *  - Limit: batch * n_frames * F * n_heads * 832 bytes (plus 256 for alignment) must fit in
 *    32 MiB, else MLA_ERR_INVALID_ARGUMENT with the required size in mla_last_error().
 *  - The first call on a device looks up the array's device address (once per device, with
 *    the cache's device current) and keeps it for the life of the process; make that first
 *    call before any stream capture.  A device reset (cudaDeviceReset, or anything else that
 *    destroys the device's primary context) invalidates that address together with every
 *    cache on the device: do not call this entry point again in a process that has reset the
 *    device while the library was loaded.
 *  - Every call on a device shares the one array and leaves the last call's contents in it.
 *    Nothing in it has to start at zero (each call writes every row it reads back), but calls
 *    whose kernels overlap on the GPU (other streams, other caches) race on it: serialise them.
 *  - Arguments, layouts, stream ordering and errors otherwise as mla_window_attention. */
mla_status mla_window_attention_noalloc(mla_cache* c, const void* x_chunk, int32_t n_frames,
                                        void* out, void* stream);

/* The same attention call computed the training-time way ([VideoMLA] §3.3): per-head keys
 * K_h = [c W_UK[h]^T | k_rope] and values V_h = c W_UV[h]^T are materialised for every key of
 * the window and the chunk, the per-head queries [q_nope | RoPE3D(q_rope)] are projected, dense
 * per-head softmax attention runs over them, and out = concat_h(o_h) W_O^T.  Same arguments and
 * the same result (up to rounding) as mla_window_attention; it exists to measure where
 * reconstruct-then-dense beats the absorbed kernel (per (query, head, key) it needs 512 flop
 * instead of 832, plus the reconstruction of every key for every call).
 *  - Needs d_nope + d_rope == 128, d_head == 128 (the paper's default dims), d_nope a multiple
 *    of 32, and sink_frames == 0; otherwise MLA_ERR_UNSUPPORTED.
 *  - The first call allocates the dense per-call buffers (per-head K and V of the largest
 *    window: 2 x batch x (W + max_chunk_frames) x F x n_heads x 256 bytes, the per-head
 *    queries and outputs of one chunk, and the fp32 split-key partials of the dense attention,
 *    up to 8 x batch x max_chunk_frames x F x n_heads x 520 bytes); they live until
 *    mla_cache_destroy. */
mla_status mla_window_attention_reconstruct(mla_cache* c, const void* x_chunk, int32_t n_frames,
                                            void* out, void* stream);

/* Bytes of device workspace with which mla_dense_attention splits the keys of each
 * (128-query tile, head, stream) item into ranges on the current device: 0 when one pass is
 * best for this shape (enough items to fill the GPU evenly, or too few keys to split). */
size_t mla_dense_workspace_bytes(int32_t batch, int32_t n_q, int32_t n_kv, int32_t n_heads);

/* Host-only view of the key split mla_dense_attention launches on a GPU with num_sms SMs and a
 * workspace of workspace_bytes bytes: *splits key ranges per (128-query tile, head, stream)
 * item, each of *kv_per_split keys (a multiple of 128 when *splits > 1; the last range holds
 * the rest and is never empty; *splits == 1 and *kv_per_split == n_kv without a workspace).
 * No GPU needed.  MLA_ERR_INVALID_ARGUMENT for a NULL output or a size below 1. */
mla_status mla_dense_split_plan(int32_t batch, int32_t n_q, int32_t n_kv, int32_t n_heads,
                                int32_t num_sms, size_t workspace_bytes, int32_t* splits,
                                int32_t* kv_per_split);

/* Dense per-head attention, the layout VideoMLA replaces ([VideoMLA] §1: every cached token
 * keeps 12 x 128 keys and 12 x 128 values, 3,072 scalars): the measurement baseline of the
 * latent-window kernel.  Stateless; no device memory is allocated.
 *   q   [batch][n_q][n_heads][d_head]  bf16      k, v [batch][n_kv][n_heads][d_head]  bf16
 *   out [batch][n_q][n_heads][d_head]  bf16      out = softmax(scale q k^T) v per head
 * softmax_scale 0 -> 1/sqrt(d_head).  Built for d_head == 128 (MLA_ERR_UNSUPPORTED otherwise).
 * Every query attends to all n_kv keys (no mask).
 * workspace: NULL (or workspace_bytes 0) runs one pass per item.  Otherwise a caller-owned,
 * 256-byte aligned device buffer of workspace_bytes bytes, in use until the call's work on
 * `stream` completes; with mla_dense_workspace_bytes(...) bytes or more the keys are split
 * into ranges whose fp32 partials a second kernel merges (fewer ranges if it is smaller).
 * Device waits are bounded; a timeout is reported by mla_dense_sync (one status word per
 * device, shared by all dense calls, whose address the first call on a device looks up and
 * keeps: a device reset invalidates it, as it invalidates every cache). */
mla_status mla_dense_attention(const void* q, const void* k, const void* v, void* out,
                               int32_t batch, int32_t n_q, int32_t n_kv, int32_t n_heads,
                               int32_t d_head, float softmax_scale, void* workspace,
                               size_t workspace_bytes, void* stream);

/* Synchronise `stream` and return the dense kernels' device status word (MLA_OK or
 * MLA_ERR_DEVICE_TIMEOUT). */
mla_status mla_dense_sync(void* stream);

/* Diagnostic self-test of the library's bounded device waits: launches one thread that waits on
 * a barrier phase nothing will complete, using the same wait as every kernel of the library.
 * The wait gives up after its limit (2 s), records MLA_ERR_DEVICE_TIMEOUT in the cache's status
 * word and the kernel returns, so the GPU context stays usable.  Synchronises `stream`;
 * *gave_up receives 1 when the wait ran out.  Afterwards mla_cache_sync reports the timeout,
 * and the status word stays set (kernels launched later on this cache stop waiting at once):
 * use a fresh cache for further work.  Not part of the method; exists to test failure
 * reporting without faulting a GPU. */
mla_status mla_cache_selftest_timeout(mla_cache* c, void* stream, int32_t* gave_up);

/* Diagnostic self-test of the debug build's bounds checks: launches the chunk-commit copy kernel
 * with a row range that runs one row past the end of the cache's planes; the kernel's bounds
 * check catches the out-of-range row before any access to it (the in-range row is copied onto
 * itself), records MLA_ERR_BOUNDS and the kernel returns.  Synchronises `stream`; *caught
 * receives 1 when the status word then holds MLA_ERR_BOUNDS.  The status word stays set: use a
 * fresh cache afterwards.  MLA_ERR_UNSUPPORTED (and nothing launched) in the normal build,
 * which has no bounds checks.  Not part of the method. */
mla_status mla_cache_selftest_bounds(mla_cache* c, void* stream, int32_t* caught);

/* Free everything the cache owns (synchronises the device first).  NULL-safe. */
void mla_cache_destroy(mla_cache* c);

/* Frames appended so far and cached frames attention currently sees: valid sink frames plus
 * valid window frames (min(appended, sink_frames) + min(max(appended - sink_frames, 0), W)). */
mla_status mla_cache_state(const mla_cache* c, int64_t* frames_appended, int32_t* valid_frames);

/* Synchronise `stream` and return the device status: MLA_OK, or the fatal error a kernel
 * recorded (MLA_ERR_DEVICE_TIMEOUT, or MLA_ERR_BOUNDS in the debug build; it stays set), else
 * MLA_ERR_BOUNDS when (debug build) a guard band after one of the cache's buffers or after the
 * allocation-free scratch was overwritten, else MLA_ERR_RANGE when a projected value was clamped
 * to the fp16 range since the previous sync (reported once, then cleared). */
mla_status mla_cache_sync(mla_cache* c, void* stream);

/* Copy stream b's cached planes to host memory, in physical row order (the rows mla_ring_slot
 * names): ckv_host receives sink_rows + W*F rows of d_latent fp16, krope_host as many rows of
 * d_rope fp16 (either may be NULL); *n_valid_rows = valid_frames * F (mla_cache_state).
 * Synchronous; diagnostic, not on the hot path. */
mla_status mla_cache_read(const mla_cache* c, int32_t b, void* ckv_host, void* krope_host,
                          int64_t* n_valid_rows);

/* Device pointers of the cache's internal planes, for diagnostics and tests. */
typedef struct {
  void* ckv;          /* fp16 [batch][rows_per_stream][d_latent];
                         rows = sink_rows + (W + max_chunk)*F                              */
  void* krope;        /* fp16 [batch][rows_per_stream][d_rope]                               */
  void* qp;           /* fp16 [batch][max_chunk*F*n_heads][d_latent + d_rope]: absorbed,
                         rotated queries of the last attention call, times scale * log2(e)   */
  void* o_lat;        /* fp16 [batch][max_chunk*F][n_heads*d_latent]: normalised P . c_kv     */
  void* w_qcat;       /* bf16 query and latent projection weights.  Full-rank W_Q with
                         d_nope = 128: [L + d_latent + d_rope][hidden], per head W_Q[h] (128
                         rows) and W_QR[h] (d_rope rows), zero rows up to L = n_heads * 160
                         rounded up to a multiple of 224, then W_DKV and W_KR.  Otherwise
                         [(n_heads+1)*(d_latent+d_rope)][2*hidden]: per head W_Qabs|W_QR,
                         then W_DKV|W_KR, each row [hi | lo]                                 */
  void* w_ov;         /* fp16 [hidden][n_heads*d_latent]                                     */
  int64_t rows_per_stream;
} mla_debug_buffers;
mla_status mla_cache_debug_buffers(const mla_cache* c, mla_debug_buffers* out);

/* Synchronous copy of the first min(bytes, size) bytes of an internal buffer to host memory;
 * *size receives the buffer's full size in bytes (may be NULL).  Diagnostic only. */
typedef enum {
  MLA_BUFFER_QP = 0,     /* Qp of the last attention call (fp16)   */
  MLA_BUFFER_O_LAT = 1,  /* o_lat of the last attention call (fp16) */
  MLA_BUFFER_W_QCAT = 2, /* query + latent weights, bf16 (layout: w_qcat above)             */
  MLA_BUFFER_W_OV = 3    /* absorbed output weights (fp16)          */
} mla_buffer;
mla_status mla_cache_copy_buffer(const mla_cache* c, mla_buffer which, void* host_dst, size_t bytes,
                                 size_t* size);

/* Per-kernel device time.  With enable != 0 every later call records CUDA events around each
 * kernel on its stream; mla_cache_profile_read synchronises those events, returns the sums
 * since the last read and clears them. */
typedef enum {
  MLA_KERNEL_APPEND = 0,     /* fused down-projection + RoPE + ring write              */
  MLA_KERNEL_QPROJ = 1,      /* query projection (absorbed W_UK) + RoPE + chunk latents */
  MLA_KERNEL_ATTENTION = 2,  /* latent-window attention (scores, softmax, P . c_kv)    */
  MLA_KERNEL_OPROJ = 3,      /* absorbed output projection                             */
  MLA_KERNEL_COUNT = 4
} mla_kernel;
typedef struct {
  double ms[MLA_KERNEL_COUNT];
  int64_t launches[MLA_KERNEL_COUNT];
} mla_profile;
mla_status mla_cache_profile_enable(mla_cache* c, int32_t enable);
mla_status mla_cache_profile_read(mla_cache* c, mla_profile* out);

/* Human-readable name of a status, and the last error message recorded on this thread. */
const char* mla_status_string(mla_status s);
const char* mla_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* MLA_LATENT_WINDOW_H */
