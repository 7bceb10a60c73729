// mla_api.cu - the C ABI of libmla.so (declared in include/mla.h): host-side validation,
// cache state, absorbed-weight derivation, tensor maps and kernel launches.
//
// Path of one attention call (VideoMLA paper page, §3.1-§3.3, App. D.4):
//   1. query_proj_kernel     (full-rank W_Q, d_nope = 128) x_chunk x [W_Q|W_QR per head ;
//                            W_DKV|W_KR]^T, then W_UK[h]^T q for each head in the same launch;
//      or tc_gemm<kEpiLatent> (other head splits, low-rank query) x_chunk x [W_Qabs|W_QR per
//                            head ; W_DKV|W_KR]^T with W_Qabs as a bf16 pair (tile shape per
//                            launch from TileShape)
//        heads  -> Qp[(q,h)] = [W_UK[h]^T q_nope | RoPE3D(q_rope)] * scale * log2 e
//        latent -> chunk tail rows (c_kv, RoPE3D k_rope)
//   2. window_attn_kernel     o_lat[(q,h)] = softmax(Qp . [c_kv|k_rope]^T) c_kv
//   3. tc_gemm<192, kEpiStore>  out = o_lat x W_OV^T,  W_OV[h] = W_O[:, h] W_UV[h]
// An append is step 1's latent block alone, written to the rows mla_ring_slot names (sink frames
// first, then ring slots): one launch per contiguous run of rows (two when the frames wrap
// around the end of the ring).  mla_window_attention_reconstruct is the training-time form of
// the same call (per-head K/V materialised, dense attention), kept for comparison.
// Every kernel of the path is launched with programmatic stream serialization, so its
// prologue overlaps the tail of the kernel before it.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <algorithm>
#include <mutex>
#include <string>
#include <utility>
#include <vector>

#include "../../include/mla.h"
#include "gemm_tc.cuh"
#include "query_proj.cuh"
#include "window_attn.cuh"
#include "dense_attn.cuh"

namespace {

using mla::EpiArgs;
using mla::RopeBands;

constexpr int kLatent = 192;
constexpr int kRope = 32;
constexpr int kQK = kLatent + kRope;  // 224

// Pipeline depths of the launched kernel variants (A = activations, B = weights); each GEMM
// CTA runs alone on its SM.  The weight ring is deep too: its L2 latency sets the k-block rate
// when only a few CTAs run.
constexpr int kProjAStages = 4;     // 128 x 224 tiles: shared ring, 4 x (16 + 28) KB
constexpr int kProjBStages = 0;     // (B_STAGES = 0: B shares A's ring)
constexpr int kProjWideAStages = 4; // 256 x 224 tiles (the HBM-bound fill): 4 x 32 KB of
constexpr int kProjWideBStages = 2; //   activations in flight, weights in their own ring
constexpr int kProjNarrowAStages = 8;   // 128 x 32 latent blocks: shared ring, 8 x (16 + 4) KB
constexpr int kProjNarrowBStages = 0;
constexpr int kProjMidAStages = 3;      // 256 x 160 tiles: shared ring, 3 x (32 + 20) KB
constexpr int kProjMidBStages = 0;
constexpr int kOutBN = 192;             // output projection column block (also the dense form's GEMMs)
constexpr int kOutAStages = 4;          // shared ring, 4 x (16 + 24) KB
constexpr int kOutBStages = 0;

// Tile shapes of the projection GEMMs with the steady-state time of one 64-wide k-block in
// microseconds, measured on B200 for one CTA per SM.  A 128-row tile's k-block time barely
// depends on BN (the per-k-block latency of loads, waits and commits dominates); a 256-row
// tile moves twice the activations per k-block.  A launch picks the shape with the smallest
// (waves of tiles) x (k-blocks) x (k-block time).
struct TileShape {
  int bn, m_sub;
  double kb_us;
};
constexpr TileShape kShapeQ224{224, 1, 0.333}, kShapeQ160W{160, 2, 0.468},
    kShapeQ224W{224, 2, 0.597}, kShapeL32{32, 1, 0.318};
// Temporal positions are formed in fp32 from the integer frame index (exact below 2^24).
constexpr int64_t kMaxFrames = int64_t(1) << 24;

// Guard bands of the MLA_DEBUG build: every device buffer of a cache is allocated kGuardBytes
// longer and the tail is filled with kGuardByte; mla_cache_sync checks that no kernel wrote
// into it.  Zero in the normal build.
#ifdef MLA_DEBUG
constexpr size_t kGuardBytes = 4096;
#else
constexpr size_t kGuardBytes = 0;
#endif
constexpr unsigned char kGuardByte = 0xA5;
constexpr int kAttnStages = 4;      // 4 key tiles in flight (Q and P live in tensor memory)

thread_local std::string g_last_error;

mla_status fail(mla_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

#define MLA_CUDA(call)                                                                \
  do {                                                                                \
    cudaError_t e_ = (call);                                                          \
    if (e_ != cudaSuccess)                                                            \
      return fail(e_ == cudaErrorMemoryAllocation ? MLA_ERR_OUT_OF_MEMORY : MLA_ERR_CUDA, \
                  "%s failed: %s", #call, cudaGetErrorString(e_));                    \
  } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Rows of the sink region of a stream's planes: sink_frames * F rounded up to whole 128-key
// tiles, so that no key tile mixes sink keys (attended with their own query rotation) and
// window keys.
int64_t sink_rows_of(const mla_config& c) {
  const int64_t n = (int64_t)c.sink_frames * c.frame_h * c.frame_w;
  return (n + 127) / 128 * 128;
}

// ------------------------------------------------------------------------------ tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 3-D 16-bit map (bf16, or fp16 when f16): (inner, rows, batch) with byte strides; box
// (box_inner, box_rows, 1).
mla_status make_map(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows,
                    uint64_t batch, uint64_t row_bytes, uint64_t batch_bytes, uint32_t box_inner,
                    uint32_t box_rows, CUtensorMapSwizzle swz, bool f16 = false) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(MLA_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  cuuint64_t dims[3] = {inner, rows, batch};
  cuuint64_t strides[2] = {row_bytes, batch_bytes};
  cuuint32_t box[3] = {box_inner, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                   const_cast<void*>(base), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(MLA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d): inner=%llu rows=%llu batch=%llu",
                (int)r, (unsigned long long)inner, (unsigned long long)rows,
                (unsigned long long)batch);
  return MLA_OK;
}

// Output map of a GEMM epilogue: 32 x 32 boxes with the 64-byte swizzle of its staging.
mla_status make_out_map(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows,
                        uint64_t batch, uint64_t row_bytes, uint64_t batch_bytes, bool f16) {
  return make_map(map, base, inner, rows, batch, row_bytes, batch_bytes, 32, 32,
                  CU_TENSOR_MAP_SWIZZLE_64B, f16);
}

// Launch with programmatic stream serialization (the kernel waits for its predecessor with
// griddepcontrol.wait before touching global memory).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// ------------------------------------------------------------------------------ kernels
// Create-time derivation of the absorbed weights for the low-rank query and head splits other
// than d_nope = 128 (fp32 accumulation), stored as bf16 pairs:
// row r of Wqcat is [hi | lo] (2 * hidden columns), hi = bf16(w), lo = bf16(w - hi).  Rows,
// per head h: [h*224, h*224+192) = W_UK[h]^T W_Q[h], [h*224+192, h*224+224) = W_QR[h];
// then [n_h*224, n_h*224+192) = W_DKV and [n_h*224+192, (n_h+1)*224) = W_KR.  The absorbed
// product carried in one bf16 (8 significant bits) would perturb every score by about 2^-10
// relative, which sharp softmaxes (large hidden states) turn into visible output errors.
// With a low-rank query the head rows come precomposed in fp32: qabs_f32 [n_heads*192][hidden]
// (W_UK[h]^T W_Q[h] W_DQ) and qr_f32 [n_heads*32][hidden] (W_QR W_DQ); w_q, w_qr, w_uk unused.
__global__ void build_wqcat_kernel(const __nv_bfloat16* __restrict__ w_q,
                                   const __nv_bfloat16* __restrict__ w_qr,
                                   const __nv_bfloat16* __restrict__ w_dkv,
                                   const __nv_bfloat16* __restrict__ w_kr,
                                   const __nv_bfloat16* __restrict__ w_uk,
                                   const float* __restrict__ qabs_f32,
                                   const float* __restrict__ qr_f32,
                                   __nv_bfloat16* __restrict__ wqcat, int hidden, int n_heads,
                                   int d_nope) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  const int rowq = blockIdx.y;  // 0 .. (n_heads+1)*224 - 1
  if (k >= hidden) return;
  const int h = rowq / kQK;
  const int c = rowq % kQK;
  float acc = 0.f;
  if (h < n_heads && qabs_f32) {
    acc = c < kLatent ? qabs_f32[(size_t)(h * kLatent + c) * hidden + k]
                      : qr_f32[(size_t)(h * kRope + c - kLatent) * hidden + k];
  } else if (h < n_heads) {
    if (c < kLatent) {
      for (int j = 0; j < d_nope; ++j) {
        const int r = h * d_nope + j;
        acc += __bfloat162float(w_uk[(size_t)r * kLatent + c]) *
               __bfloat162float(w_q[(size_t)r * hidden + k]);
      }
    } else {
      acc = __bfloat162float(w_qr[(size_t)(h * kRope + c - kLatent) * hidden + k]);
    }
  } else {
    acc = c < kLatent ? __bfloat162float(w_dkv[(size_t)c * hidden + k])
                      : __bfloat162float(w_kr[(size_t)(c - kLatent) * hidden + k]);
  }
  // hi + lo: the weight to about 16 significant bits in two bf16 halves of the row (the lo half
  // is zero where the weight is the caller's own bf16 value).
  const __nv_bfloat16 hi = __float2bfloat16_rn(acc);
  wqcat[(size_t)rowq * 2 * hidden + k] = hi;
  wqcat[(size_t)rowq * 2 * hidden + hidden + k] = __float2bfloat16_rn(acc - __bfloat162float(hi));
}

// W_OV[o][h*192 + c] = sum_j W_O[o][h*d_head + j] * W_UV[h*d_head + j][c], stored fp16 (it
// multiplies the fp16 o_lat).
// Create-time fp32 product for composing low-rank weights: per batch index z,
//   C[z][m][n] = sum_k A(z, m, k) B(z, k, n),  A(z,m,k) = A[z*a_sz + m*a_sm + k*a_sk] (TA),
//   B(z,k,n) = B[z*b_sz + k*b_sk + n] (TB), C row-major [M][N] per z at C + z*c_sz.
template <typename TA, typename TB>
__global__ void compose_kernel(const TA* __restrict__ A, int64_t a_sz, int64_t a_sm, int64_t a_sk,
                               const TB* __restrict__ B, int64_t b_sz, int64_t b_sk,
                               float* __restrict__ C, int64_t c_sz, int M, int N, int K) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  const int m = blockIdx.y;
  const int z = blockIdx.z;
  if (n >= N || m >= M) return;
  const TA* a = A + z * a_sz + (int64_t)m * a_sm;
  const TB* b = B + z * b_sz + n;
  float acc = 0.f;
  for (int k = 0; k < K; ++k) acc += (float)a[(int64_t)k * a_sk] * (float)b[(int64_t)k * b_sk];
  C[z * c_sz + (int64_t)m * N + n] = acc;
}
// fp32 -> fp16, clamped to +-65504; a clamp sets *range (the status block's range word).
__device__ __forceinline__ __half to_f16_checked(float v, int* range) {
  if (!(fabsf(v) <= mla::kF16Max)) {
    atomicOr(range, 1);
    v = fminf(fmaxf(v, -mla::kF16Max), mla::kF16Max);
  }
  return __float2half_rn(v);
}
__global__ void build_wov_kernel(const __nv_bfloat16* __restrict__ w_o,
                                 const __nv_bfloat16* __restrict__ w_uv,
                                 __half* __restrict__ wov, int hidden, int n_heads,
                                 int d_head, int* range) {
  const int col = blockIdx.x * blockDim.x + threadIdx.x;  // h*192 + c
  const int o = blockIdx.y;
  if (col >= n_heads * kLatent) return;
  const int h = col / kLatent;
  const int c = col % kLatent;
  const int in_o = n_heads * d_head;
  float acc = 0.f;
  for (int j = 0; j < d_head; ++j) {
    const int r = h * d_head + j;
    acc += __bfloat162float(w_o[(size_t)o * in_o + r]) *
           __bfloat162float(w_uv[(size_t)r * kLatent + c]);
  }
  wov[(size_t)o * (n_heads * kLatent) + col] = to_f16_checked(acc, range);
}

template <typename K>
mla_status set_smem(K kernel, int bytes) {
  MLA_CUDA(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
  return MLA_OK;
}

// Per-head query weight of the dense form: rows h*128 + j = W_Q[h*d_nope + j] (j < d_nope),
// W_QR[h*32 + j - d_nope] (j >= d_nope); with a low-rank query the fp32 compositions with W_DQ.
__global__ void build_wqd_kernel(const __nv_bfloat16* __restrict__ w_q,
                                 const __nv_bfloat16* __restrict__ w_qr,
                                 const float* __restrict__ qeff_f32, const float* __restrict__ qreff_f32,
                                 __nv_bfloat16* __restrict__ wqd, int hidden, int n_heads, int d_nope) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  const int row = blockIdx.y;  // h*128 + j
  if (k >= hidden) return;
  const int h = row / 128, j = row % 128;
  float v;
  if (j < d_nope) {
    const size_t r = (size_t)(h * d_nope + j) * hidden + k;
    v = qeff_f32 ? qeff_f32[r] : __bfloat162float(w_q[r]);
  } else {
    const size_t r = (size_t)(h * kRope + j - d_nope) * hidden + k;
    v = qreff_f32 ? qreff_f32[r] : __bfloat162float(w_qr[r]);
  }
  wqd[(size_t)row * hidden + k] = __float2bfloat16_rn(v);
}
// Two-step query weights, wq2 [latent_row0 + 224][hidden], a copy of the caller's bf16 values:
// per head h, rows h*160 + j hold W_Q[h*128 + j] (j < 128) and W_QR[h*32 + j - 128] (the next 32
// rows); rows [n_h*160, latent_row0) are zero; then W_DKV (192 rows) and W_KR (32 rows).
// latent_row0 is n_h*160 rounded up to a multiple of 224, the period by which the latent-only
// projection (tc_gemm_kernel) tells the c_kv and k_rope columns of its block apart.
__global__ void build_wq2_kernel(const __nv_bfloat16* __restrict__ w_q,
                                 const __nv_bfloat16* __restrict__ w_qr,
                                 const __nv_bfloat16* __restrict__ w_dkv,
                                 const __nv_bfloat16* __restrict__ w_kr,
                                 __nv_bfloat16* __restrict__ wq2, int hidden, int n_heads,
                                 int latent_row0) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  const int row = blockIdx.y;
  if (k >= hidden) return;
  const int per = mla::kQpBN;
  const __nv_bfloat16* src = nullptr;
  if (row < n_heads * per) {
    const int h = row / per, j = row % per;
    src = j < mla::kQpNope ? w_q + (size_t)(h * mla::kQpNope + j) * hidden
                           : w_qr + (size_t)(h * kRope + j - mla::kQpNope) * hidden;
  } else if (row >= latent_row0) {
    const int j = row - latent_row0;
    src = j < kLatent ? w_dkv + (size_t)j * hidden : w_kr + (size_t)(j - kLatent) * hidden;
  }
  wq2[(size_t)row * hidden + k] = src ? src[k] : __float2bfloat16_rn(0.f);
}
__global__ void bf16_to_f16_kernel(const __nv_bfloat16* __restrict__ in, __half* __restrict__ out,
                                   int64_t n, int* range) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) out[i] = to_f16_checked(__bfloat162float(in[i]), range);
}
// k_rope of every key into the RoPE channels [d_nope, 128) of every head of the dense K:
// kd[z][n][h][d_nope + r] = krope[z][n][r].
__global__ void krope_broadcast_kernel(const __half* __restrict__ krope, int64_t krope_stream_rows,
                                       __nv_bfloat16* __restrict__ kd, int n_keys, int n_heads,
                                       int d_nope, int64_t kd_rows_cap, int* status) {
  const int n = blockIdx.x;
  const int z = blockIdx.y;
  // kd rows are compact per call ([z][n]); the buffer holds kd_rows_cap of them.
  if (!mla::in_bounds(n < krope_stream_rows && ((int64_t)z * n_keys + n) < kd_rows_cap, status)) return;
  const __half* src = krope + ((int64_t)z * krope_stream_rows + n) * kRope;
  __nv_bfloat16* dst = kd + ((int64_t)z * n_keys + n) * n_heads * 128 + d_nope;
  for (int i = threadIdx.x; i < n_heads * kRope; i += blockDim.x) {
    const int h = i / kRope, r = i % kRope;
    dst[h * 128 + r] = __float2bfloat16_rn(__half2float(src[r]));
  }
}

// Move `rows` rows of both latent planes of every stream from src_row to dst_row (16-byte
// pieces: 24 per c_kv row, 4 per k_rope row).  The two ranges never overlap (mla_cache_commit).
__global__ void move_rows_kernel(__half* __restrict__ ckv, __half* __restrict__ krope,
                                 int64_t rows_per_stream, int64_t src_row, int64_t dst_row,
                                 int64_t rows, int* status) {
  constexpr int kPieces = kLatent / 8 + kRope / 8;   // 16-byte pieces per row of both planes
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int z = blockIdx.y;
  mla::grid_dependency_wait();
  if (i >= rows * kPieces) return;
  const int64_t r = i / kPieces;
  const int u = (int)(i - r * kPieces);
  if (!mla::in_bounds(src_row + r < rows_per_stream && dst_row + r < rows_per_stream && src_row >= 0 &&
                      dst_row >= 0, status))
    return;
  if (u < kLatent / 8) {
    const uint4* s = reinterpret_cast<const uint4*>(ckv + (z * rows_per_stream + src_row + r) * kLatent);
    uint4* d = reinterpret_cast<uint4*>(ckv + (z * rows_per_stream + dst_row + r) * kLatent);
    d[u] = s[u];
  } else {
    const uint4* s = reinterpret_cast<const uint4*>(krope + (z * rows_per_stream + src_row + r) * kRope);
    uint4* d = reinterpret_cast<uint4*>(krope + (z * rows_per_stream + dst_row + r) * kRope);
    d[u - kLatent / 8] = s[u - kLatent / 8];
  }
}

// Self-test of the bounded device wait: one thread waits on an mbarrier phase that nothing
// completes; mbar_wait gives up after its limit and records MLA_ERR_DEVICE_TIMEOUT.
__global__ void selftest_wait_kernel(int* status, int* gave_up) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mla::mbar_init(&bar, 1);
    mla::fence_mbar_init();
    const bool ok = mla::mbar_wait(&bar, 0, status);
    *gave_up = ok ? 0 : 1;
  }
}

mla_status check_launch(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(MLA_ERR_CUDA, "%s launch failed: %s", what, cudaGetErrorString(e));
  return MLA_OK;
}

// Persistent GEMM launch: one CTA per SM at most, each walking its share of the tiles.
template <int BN, int SA, int SB, int EPI, bool F16, int M_SUB = 1>
mla_status launch_gemm(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& mo0,
                       const CUtensorMap& mo1, const CUtensorMap& mo2, int M, int K, int b_row0,
                       mla::GemmTiles tiles, const EpiArgs& ep, int* status, int num_sms,
                       cudaStream_t st, const char* what, int a_kwrap = 0) {
  const int n = tiles.count();
  if (n <= 0) return MLA_OK;
  const int grid = n < num_sms ? n : num_sms;
  const cudaError_t e = launch_pdl(mla::tc_gemm_kernel<BN, SA, SB, EPI, F16, M_SUB>, dim3(grid),
                                   dim3(mla::kGemmThreads),
                                   mla::GemmSmem<BN, SA, SB, M_SUB>::kBytes, st, ma, mb, mo0, mo1,
                                   mo2, M, K, a_kwrap, b_row0, tiles, ep, status);
  if (e != cudaSuccess) return fail(MLA_ERR_CUDA, "%s launch failed: %s", what, cudaGetErrorString(e));
  return check_launch(what);
}

}  // namespace

// ------------------------------------------------------------------------------ the cache
struct mla_cache {
  mla_config cfg;
  int F = 0;
  int64_t rows_per_stream = 0;     // sink_rows + (W + max_chunk) * F
  int64_t sink_rows = 0;           // sink region: sink_frames * F rounded up to 128 rows
  int64_t max_q_tokens = 0;        // max_chunk * F
  int64_t frames_appended = 0;
  // Chunk of the last attention call whose latents sit in the chunk tail (mla_cache_commit):
  // its frame count (0: none) and the frames_appended it was computed at.
  int32_t pending_frames = 0;
  int64_t pending_at = -1;
  float softmax_scale = 0.f;
  RopeBands rope{};
  int device = 0;
  int num_sms = 148;

  __half* ckv = nullptr;           // fp16 latent planes (ring + chunk tail)
  __half* krope = nullptr;
  __half* qp = nullptr;            // fp16 absorbed queries
  __half* o_lat = nullptr;         // fp16 P . c_kv
  // Query and latent projection weights (bf16: they multiply the caller's bf16 hidden states).
  // Full-rank query with d_nope = 128 (two_step): the caller's rows [W_Q[h]; W_QR[h]] per head,
  // then W_DKV and W_KR, hidden columns each; query_proj_kernel multiplies them and then
  // W_UK[h] (wuk16).  Otherwise the absorbed bf16 pairs [hi | lo] of 2 * hidden columns.
  __nv_bfloat16* wqcat = nullptr;
  bool two_step = false;
  int64_t wq_rows = 0;             // rows of wqcat
  int64_t wq_cols = 0;             // columns of a wqcat row (hidden or 2 * hidden)
  int32_t latent_row0 = 0;         // first W_DKV row of wqcat (a multiple of 224)
  __half* wuk16 = nullptr;         // two_step: W_UK [n_h*128][192] fp16 (multiplies the fp16 q pair)
  CUtensorMap map_wuk16{};
  __half* wov = nullptr;           // fp16: multiplies o_lat
  float2* rope_hw = nullptr;       // RoPE (cos, sin) of the h and w bands, [16][frame_h + frame_w]

  // Reconstruct-then-dense form (mla_window_attention_reconstruct), when d_nope + d_rope == 128,
  // d_head == 128 and there is no sink: per-head weights, built at creation, and per-call
  // buffers allocated on first use.
  bool dense_ok = false;
  __nv_bfloat16* wqd = nullptr;    // [n_h*128][hidden]: per head [W_Q (d_nope) | W_QR (32)]
  __half* wukh = nullptr;          // [n_h*d_nope][192] W_UK (fp16: multiplies the fp16 cache)
  __half* wuvh = nullptr;          // [n_h*128][192] W_UV
  __nv_bfloat16* wo = nullptr;     // [hidden][n_h*128] W_O
  CUtensorMap map_wqd{}, map_wukh{}, map_wuvh{}, map_wo{};
  __nv_bfloat16* qd = nullptr;     // [B][n_q][n_h][128]   per call, compact
  __nv_bfloat16* kd = nullptr;     // [B][n_keys][n_h][128] per call, compact
  __nv_bfloat16* vd = nullptr;     // [B][n_keys][n_h][128]
  __nv_bfloat16* od = nullptr;     // [B][n_q][n_h][128]
  void* dws = nullptr;             // split-key partials of the dense attention
  size_t dws_bytes = 0;
  int* status = nullptr;

  CUtensorMap map_wqcat{};         // B operand of the projections: box 64 x 224
  CUtensorMap map_wqcat160{};      // the same weights in 160-row boxes
  CUtensorMap map_wqcat32{};       // ... and in 32-row boxes (32-column latent blocks)
  CUtensorMap map_wov{};           // B operand of the output projection: box 64 x 192

  struct Guard {
    const unsigned char* p;   // first guard byte (the buffer's end)
    const char* name;
  };
  std::vector<Guard> guards;   // MLA_DEBUG build only

  bool profiling = false;
  struct Rec {
    int kind;
    cudaEvent_t a, b;
  };
  std::vector<Rec> pending;
  std::vector<cudaEvent_t> pool;
  double prof_ms[MLA_KERNEL_COUNT] = {0, 0, 0, 0};
  int64_t prof_n[MLA_KERNEL_COUNT] = {0, 0, 0, 0};
};

namespace {

// The last attention call's chunk latents are in the chunk tail (see mla_cache_commit).
void set_pending(mla_cache* c, int32_t n_frames) {
  c->pending_frames = n_frames;
  c->pending_at = c->frames_appended;
}

// Valid sink frames (vs) and valid window frames (vw) of a cache: the first sink_frames frames
// ever appended are the sink, the newest W of the others the window.
void valid_counts_of(const mla_config& cfg, int64_t A, int64_t& vs, int64_t& vw) {
  const int64_t S = cfg.sink_frames, W = cfg.window_frames;
  vs = A < S ? A : S;
  vw = A - vs < W ? A - vs : W;
}
void valid_counts(const mla_cache* c, int64_t& vs, int64_t& vw) {
  valid_counts_of(c->cfg, c->frames_appended, vs, vw);
}

// cudaMalloc of a cache buffer; the MLA_DEBUG build adds a guard band after it (filled on
// `st`) and records it for mla_cache_sync.
template <typename T>
cudaError_t alloc_buffer(mla_cache* c, T** p, size_t bytes, const char* name, cudaStream_t st) {
  void* v = nullptr;
  cudaError_t e = cudaMalloc(&v, bytes + kGuardBytes);
  if (e != cudaSuccess) return e;
  *p = static_cast<T*>(v);
  if (kGuardBytes) {
    unsigned char* g = static_cast<unsigned char*>(v) + bytes;
    c->guards.push_back({g, name});
    e = cudaMemsetAsync(g, kGuardByte, kGuardBytes, st);
  }
  return e;
}

// Host-side extent check of a tensor map over a buffer the library owns (MLA_DEBUG build):
// the last byte the map can reach must lie inside [buf, buf + buf_bytes).
mla_status check_extent(const void* base, uint64_t inner_bytes, uint64_t rows, uint64_t row_stride,
                        uint64_t batch, uint64_t batch_stride, const void* buf, size_t buf_bytes,
                        const char* what) {
#ifdef MLA_DEBUG
  const uintptr_t b0 = reinterpret_cast<uintptr_t>(buf), a = reinterpret_cast<uintptr_t>(base);
  if (rows == 0 || batch == 0) return MLA_OK;
  const uintptr_t last = a + (batch - 1) * batch_stride + (rows - 1) * row_stride + inner_bytes;
  if (a < b0 || last > b0 + buf_bytes)
    return fail(MLA_ERR_BOUNDS, "%s: tensor map reaches %zu bytes past its buffer", what,
                (size_t)(last > b0 + buf_bytes ? last - (b0 + buf_bytes) : 0));
#else
  (void)base; (void)inner_bytes; (void)rows; (void)row_stride; (void)batch; (void)batch_stride;
  (void)buf; (void)buf_bytes; (void)what;
#endif
  return MLA_OK;
}

cudaEvent_t take_event(mla_cache* c) {
  if (!c->pool.empty()) {
    cudaEvent_t e = c->pool.back();
    c->pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

struct ProfScope {
  mla_cache* c;
  int kind;
  cudaStream_t s;
  cudaEvent_t a = nullptr;
  ProfScope(mla_cache* c_, int k, cudaStream_t s_, bool enabled = true) : c(c_), kind(k), s(s_) {
    if (enabled && c->profiling && (a = take_event(c)) != nullptr) cudaEventRecord(a, s);
  }
  ~ProfScope() {
    if (!a) return;
    cudaEvent_t b = take_event(c);
    if (!b) {
      c->pool.push_back(a);
      return;
    }
    cudaEventRecord(b, s);
    c->pending.push_back({kind, a, b});
  }
};

// Band frequencies base^(-2i/d_a), computed in double and carried as float hi + lo.
RopeBands make_bands(const mla_config& cfg) {
  RopeBands rb{};
  int p = 0;
  const int dims[3] = {cfg.rope_t, cfg.rope_h, cfg.rope_w};
  for (int a = 0; a < 3; ++a)
    for (int i = 0; i < dims[a] / 2; ++i, ++p) {
      const double f = std::pow(cfg.rope_base, -2.0 * i / dims[a]);
      rb.axis[p] = a;
      rb.freq_hi[p] = (float)f;
      rb.freq_lo[p] = (float)(f - (double)rb.freq_hi[p]);
    }
  return rb;
}

// (cos, sin) of the h and w RoPE bands for every h in [0, frame_h) and w in [0, frame_w),
// evaluated in double and rounded once, pair-major: [16][frame_h] for h, then [16][frame_w]
// for w (pairs of the other axes hold (1, 0)).
std::vector<float2> make_rope_hw(const mla_config& cfg) {
  const size_t H = cfg.frame_h, Wd = cfg.frame_w;
  std::vector<float2> tab(16 * (H + Wd), make_float2(1.f, 0.f));
  int p = 0;
  const int dims[3] = {cfg.rope_t, cfg.rope_h, cfg.rope_w};
  for (int a = 0; a < 3; ++a)
    for (int i = 0; i < dims[a] / 2; ++i, ++p) {
      const double f = std::pow(cfg.rope_base, -2.0 * i / dims[a]);
      if (a == 1)
        for (size_t h = 0; h < H; ++h)
          tab[p * H + h] = make_float2((float)std::cos(h * f), (float)std::sin(h * f));
      if (a == 2)
        for (size_t w = 0; w < Wd; ++w)
          tab[16 * H + p * Wd + w] = make_float2((float)std::cos(w * f), (float)std::sin(w * f));
    }
  return tab;
}

// Launch the latent (and, with queries, the query) projection over `rows` rows of x per
// stream: query_proj_kernel for a full-rank query with d_nope = 128, else the absorbed-pair
// GEMM.  The latent rows land at cache rows [dst_row0, dst_row0 + rows) of every stream; query
// rows go to qp ([batch][qp_tokens][n_heads * 224]).  The GEMM's tile shape is the TileShape
// candidate with the least estimated time: with queries 128 x 224, 256 x 160 or 256 x 224
// tiles; latent only 128 x 32 (seven column blocks, so that a one-frame append spreads over
// 91 SMs instead of 13), 128 x 224 or 256 x 224.
mla_status launch_latent_gemm(mla_cache* c, const void* x, int64_t rows, int64_t x_batch_rows,
                              bool with_queries, int64_t t0, int64_t dst_row0, cudaStream_t st,
                              __half* qp = nullptr, int64_t qp_tokens = 0) {
  const mla_config& cfg = c->cfg;
  // Full-rank query with d_nope = 128: query_proj_kernel (256-row tiles, the caller's weights
  // and W_UK in two chained products).
  const bool two_step = with_queries && c->two_step;
  const int n_cols = with_queries ? (cfg.n_heads + 1) * kQK : kQK;   // columns of this launch
  // With absorbed queries the weights' lo halves are multiplied too (K = 2 x hidden, A wraps);
  // the latent-only launch reads the first hidden columns, which hold W_DKV and W_KR exactly.
  const int K = with_queries && !two_step ? 2 * cfg.hidden : cfg.hidden;
  const int a_kwrap = with_queries && !two_step ? cfg.hidden : 0;
  const int num_kb = K / 64;
  // Pick the tile shape with the least estimated time (waves x k-blocks x k-block time).
  auto tiles_of = [&](const TileShape& t) {
    return mla::GemmTiles{(int32_t)((rows + 128 * t.m_sub - 1) / (128 * t.m_sub)),
                          (n_cols + t.bn - 1) / t.bn, cfg.batch};
  };
  auto cost = [&](const TileShape& t) {
    const int64_t n = tiles_of(t).count();
    return (double)((n + c->num_sms - 1) / c->num_sms) * num_kb * t.kb_us;
  };
  const TileShape cands_q[3] = {kShapeQ224, kShapeQ160W, kShapeQ224W};
  const TileShape cands_l[3] = {kShapeL32, kShapeQ224, kShapeQ224W};
  const TileShape* cands = with_queries ? cands_q : cands_l;
  TileShape shape = cands[0];
  for (int i = 1; i < 3; ++i)
    if (cost(cands[i]) < cost(shape)) shape = cands[i];
  const mla::GemmTiles tiles = tiles_of(shape);

  CUtensorMap map_x, map_ckv, map_krope, map_qp;
  mla_status s = make_map(&map_x, x, cfg.hidden, rows, cfg.batch, (uint64_t)cfg.hidden * 2,
                          (uint64_t)x_batch_rows * cfg.hidden * 2, 64,
                          two_step ? 256 : 128 * shape.m_sub, CU_TENSOR_MAP_SWIZZLE_128B);
  if (s != MLA_OK) return s;
  const uint64_t plane_rows = (uint64_t)c->rows_per_stream;
  if ((s = make_out_map(&map_ckv, c->ckv + dst_row0 * kLatent, kLatent, rows, cfg.batch,
                        kLatent * 2, plane_rows * kLatent * 2, true)) != MLA_OK)
    return s;
  if ((s = make_out_map(&map_krope, c->krope + dst_row0 * kRope, kRope, rows, cfg.batch,
                        kRope * 2, plane_rows * kRope * 2, true)) != MLA_OK)
    return s;
  if (with_queries) {
    const uint64_t qcols = (uint64_t)cfg.n_heads * kQK;
    if (!qp) {
      qp = c->qp;
      qp_tokens = c->max_q_tokens;
    }
    if ((s = make_out_map(&map_qp, qp, qcols, rows, cfg.batch, qcols * 2,
                          (uint64_t)qp_tokens * qcols * 2, true)) != MLA_OK)
      return s;
  } else {
    map_qp = map_ckv;   // no query columns in this launch
  }
  {
    // MLA_DEBUG build: the output maps stay inside the cache planes and the Qp buffer.
    const size_t plane_bytes = (size_t)cfg.batch * c->rows_per_stream * kLatent * 2;
    if ((s = check_extent(c->ckv + dst_row0 * kLatent, kLatent * 2, rows, kLatent * 2, cfg.batch,
                          plane_rows * kLatent * 2, c->ckv, plane_bytes, "c_kv output")) != MLA_OK ||
        (s = check_extent(c->krope + dst_row0 * kRope, kRope * 2, rows, kRope * 2, cfg.batch,
                          plane_rows * kRope * 2, c->krope, plane_bytes / kLatent * kRope,
                          "k_rope output")) != MLA_OK)
      return s;
    if (with_queries) {
      const uint64_t qcols = (uint64_t)cfg.n_heads * kQK;
      const size_t qp_bytes = (size_t)cfg.batch * (qp == c->qp ? c->max_q_tokens : qp_tokens) * qcols * 2;
      if ((s = check_extent(qp, qcols * 2, rows, qcols * 2, cfg.batch, (uint64_t)qp_tokens * qcols * 2,
                            qp, qp_bytes, "Qp output")) != MLA_OK)
        return s;
    }
  }
  EpiArgs ep{};
  // Output columns are B rows: the latent block starts at the absorbed heads' end (queries) or
  // at the weights' latent rows (latent only).
  ep.latent_col0 = with_queries ? cfg.n_heads * kQK : c->latent_row0;
  ep.n_cols = ep.latent_col0 + kQK;
  ep.t0 = t0;
  ep.tokens_per_frame = c->F;
  ep.frame_w = cfg.frame_w;
  ep.q_scale = c->softmax_scale * 1.4426950408889634f;
  ep.rope = c->rope;
  ep.rope_hw = c->rope_hw;
  ep.frame_h = cfg.frame_h;
  const char* what = "latent projection";
  if (two_step) {
    const mla::GemmTiles qt{(int32_t)((rows + 255) / 256), cfg.n_heads + 2, cfg.batch};
    const int n = qt.count();
    if (n <= 0) return MLA_OK;
    const cudaError_t e = launch_pdl(mla::query_proj_kernel, dim3(n < c->num_sms ? n : c->num_sms),
                                     dim3(mla::kQpThreads), mla::QpSmem::kBytes, st, map_x,
                                     c->map_wqcat160, c->map_wuk16, map_qp, map_ckv, map_krope,
                                     (int)rows, cfg.hidden, cfg.n_heads, c->latent_row0, qt, ep,
                                     c->status);
    if (e != cudaSuccess) return fail(MLA_ERR_CUDA, "query projection launch failed: %s", cudaGetErrorString(e));
    return check_launch("query projection");
  }
  const int b_row0 = with_queries ? 0 : c->latent_row0;
  if (shape.bn == 32)
    return launch_gemm<32, kProjNarrowAStages, kProjNarrowBStages, mla::kEpiLatent, false, 1>(
        map_x, c->map_wqcat32, map_qp, map_ckv, map_krope, (int)rows, K, b_row0, tiles,
        ep, c->status, c->num_sms, st, what, a_kwrap);
  if (shape.bn == 160)
    return launch_gemm<160, kProjMidAStages, kProjMidBStages, mla::kEpiLatent, false, 2>(
        map_x, c->map_wqcat160, map_qp, map_ckv, map_krope, (int)rows, K, b_row0, tiles,
        ep, c->status, c->num_sms, st, what, a_kwrap);
  if (shape.m_sub == 2)
    return launch_gemm<kQK, kProjWideAStages, kProjWideBStages, mla::kEpiLatent, false, 2>(
        map_x, c->map_wqcat, map_qp, map_ckv, map_krope, (int)rows, K, b_row0, tiles,
        ep, c->status, c->num_sms, st, what, a_kwrap);
  return launch_gemm<kQK, kProjAStages, kProjBStages, mla::kEpiLatent, false, 1>(
      map_x, c->map_wqcat, map_qp, map_ckv, map_krope, (int)rows, K, b_row0, tiles, ep,
      c->status, c->num_sms, st, what, a_kwrap);
}

// Output projection out[z][m][:] = o_lat[z][m][:] W_OV^T over nq tokens per stream.
mla_status launch_out_proj(mla_cache* c, const __half* o_lat, int64_t o_lat_tokens, int64_t nq,
                           void* out, cudaStream_t st, const char* what) {
  const mla_config& cfg = c->cfg;
  CUtensorMap ma, mo;
  mla_status s;
  const uint64_t kin = (uint64_t)cfg.n_heads * kLatent;
  if ((s = make_map(&ma, o_lat, kin, nq, cfg.batch, kin * 2, (uint64_t)o_lat_tokens * kin * 2,
                    64, 128, CU_TENSOR_MAP_SWIZZLE_128B, true)) != MLA_OK)
    return s;
  if ((s = check_extent(o_lat, kin * 2, nq, kin * 2, cfg.batch, (uint64_t)o_lat_tokens * kin * 2, o_lat,
                        (size_t)cfg.batch * o_lat_tokens * kin * 2, "o_lat input")) != MLA_OK)
    return s;
  if ((s = make_out_map(&mo, out, cfg.hidden, nq, cfg.batch, (uint64_t)cfg.hidden * 2,
                        (uint64_t)nq * cfg.hidden * 2, false)) != MLA_OK)
    return s;
  EpiArgs ep{};
  ep.n_cols = cfg.hidden;
  const mla::GemmTiles tiles{(int32_t)((nq + 127) / 128), (cfg.hidden + kOutBN - 1) / kOutBN,
                             cfg.batch};
  return launch_gemm<kOutBN, kOutAStages, kOutBStages, mla::kEpiStore, true>(
      ma, c->map_wov, mo, mo, mo, (int)nq, (int)kin, 0, tiles, ep, c->status, c->num_sms, st,
      what);
}

// Window attention of R query rows per stream over keys [0, n_keys) of every stream's ring.
mla_status launch_attention(mla_cache* c, const __half* qp, int64_t qp_batch_stride, int64_t R,
                            int64_t n_keys, __half* o_lat, int64_t o_lat_batch_stride,
                            cudaStream_t st, bool profile) {
  const mla_config& cfg = c->cfg;
  CUtensorMap mkc, mkr;
  mla_status s;
  if ((s = make_map(&mkc, c->ckv, kLatent, n_keys, cfg.batch, kLatent * 2,
                    (uint64_t)c->rows_per_stream * kLatent * 2, 64, 128,
                    CU_TENSOR_MAP_SWIZZLE_128B, true)) != MLA_OK)
    return s;
  if ((s = make_map(&mkr, c->krope, kRope, n_keys, cfg.batch, kRope * 2,
                    (uint64_t)c->rows_per_stream * kRope * 2, 32, 128,
                    CU_TENSOR_MAP_SWIZZLE_64B, true)) != MLA_OK)
    return s;
  {
    // MLA_DEBUG build: the key maps stay inside the cache planes.
    const size_t rows_all = (size_t)cfg.batch * c->rows_per_stream;
    if ((s = check_extent(c->ckv, kLatent * 2, n_keys, kLatent * 2, cfg.batch,
                          (uint64_t)c->rows_per_stream * kLatent * 2, c->ckv, rows_all * kLatent * 2,
                          "c_kv keys")) != MLA_OK ||
        (s = check_extent(c->krope, kRope * 2, n_keys, kRope * 2, cfg.batch,
                          (uint64_t)c->rows_per_stream * kRope * 2, c->krope, rows_all * kRope * 2,
                          "k_rope keys")) != MLA_OK)
      return s;
  }
  mla::AttnArgs a{};
  a.qp = qp;
  a.qp_batch_stride = qp_batch_stride;
  a.rows = (int32_t)R;
  a.n_keys = (int32_t)n_keys;
  a.o_lat = o_lat;
  a.o_lat_batch_stride = o_lat_batch_stride;
  // Capacity of the row buffers (debug bounds checks): both hold the same rows per stream.
  a.qp_rows_cap = qp_batch_stride / kQK < o_lat_batch_stride / kLatent ? qp_batch_stride / kQK
                                                                         : o_lat_batch_stride / kLatent;
  a.batch = cfg.batch;
  // Sink keys (rows [0, sink_rows), valid below vs * F) are stored rotated at their absolute
  // frame index, which is also their window-local one; the queries (rotated at absolute t) must
  // meet them at their local t = absolute t + delta, delta = (vs + vw) - frames_appended: turn
  // the temporal RoPE bands by delta (computed in double, rounded once).
  int64_t vs, vw;
  valid_counts(c, vs, vw);
  a.sink_tiles = (int32_t)(c->sink_rows / 128);
  a.sink_keys = (int32_t)(vs * c->F);
  {
    const double delta = (double)(vs + vw) - (double)c->frames_appended;
    for (int p = 0; p < 16; ++p) a.sink_rot[p] = make_float2(1.f, 0.f);
    for (int i = 0; i < cfg.rope_t / 2; ++i) {
      const double ang = delta * std::pow(cfg.rope_base, -2.0 * i / cfg.rope_t);
      a.sink_rot[i] = make_float2((float)std::cos(ang), (float)std::sin(ang));
    }
  }
  using Sm = mla::AttnSmem<kAttnStages>;
  dim3 grid((unsigned)((R + 127) / 128), (unsigned)cfg.batch);
  ProfScope p(c, MLA_KERNEL_ATTENTION, st, profile);
  const cudaError_t e = launch_pdl(mla::window_attn_kernel<kAttnStages>, grid,
                                   dim3(mla::kAttnThreads), Sm::kBytes, st, mkc, mkr, a, c->status);
  if (e != cudaSuccess)
    return fail(MLA_ERR_CUDA, "window attention launch failed: %s", cudaGetErrorString(e));
  return check_launch("window attention");
}

}  // namespace

// ------------------------------------------------------------------------------ no-alloc variant
// Scratch of mla_window_attention_noalloc: the absorbed queries (Qp) and the latent-space
// attention output (o_lat) of one call, in a fixed per-device array instead of cache-owned
// buffers.  Every GPU that loads this library holds these 32 MiB until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;
// Per-device tables of looked-up device addresses (the no-alloc scratch, the dense status word).
constexpr int kMaxDevices = 64;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes + kGuardBytes];

namespace {

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  In host code the array's name
// is only a host-side stand-in, so the address is looked up once per device (with that device
// current) and cached.
mla_status noalloc_scratch(void** out) {
  int dev = 0;
  MLA_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return fail(MLA_ERR_UNSUPPORTED, "device index %d too large", dev);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr)
      return fail(MLA_ERR_CUDA, "cudaGetSymbolAddress of the no-alloc scratch failed: %s",
                  cudaGetErrorString(e));
    if (kGuardBytes) {
      // MLA_DEBUG build: the guard band after the scratch (no allocation: the array holds it).
      const cudaError_t e2 =
          cudaMemset(static_cast<unsigned char*>(p) + kNoAllocScratchBytes, kGuardByte, kGuardBytes);
      if (e2 != cudaSuccess)
        return fail(MLA_ERR_CUDA, "guard band of the no-alloc scratch: %s", cudaGetErrorString(e2));
    }
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return MLA_OK;
}

// Guard band of the current device's no-alloc scratch, if that scratch has been set up.
const unsigned char* noalloc_guard() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  return g_noalloc_ptr[dev] ? static_cast<const unsigned char*>(g_noalloc_ptr[dev]) + kNoAllocScratchBytes
                            : nullptr;
}

size_t align256(size_t n) { return (n + 255) & ~size_t(255); }

}  // namespace

// ------------------------------------------------------------------------------ dense baseline
// Status word of the stateless dense-attention entry point, one per device.
static __device__ int g_dense_status;

namespace {

constexpr int kDenseStages = 3;
std::mutex g_dense_mu;
int* g_dense_status_ptr[kMaxDevices] = {};

mla_status dense_status_word(int** out) {
  int dev = 0;
  MLA_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return fail(MLA_ERR_UNSUPPORTED, "device index %d too large", dev);
  std::lock_guard<std::mutex> lock(g_dense_mu);
  if (!g_dense_status_ptr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_dense_status);
    if (e != cudaSuccess || p == nullptr)
      return fail(MLA_ERR_CUDA, "cudaGetSymbolAddress of the dense status word failed: %s",
                  cudaGetErrorString(e));
    const cudaError_t e2 =
        cudaFuncSetAttribute(mla::dense_attn_kernel<kDenseStages>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             mla::DenseSmem<kDenseStages>::kBytes);
    if (e2 != cudaSuccess)
      return fail(MLA_ERR_CUDA, "cudaFuncSetAttribute failed: %s", cudaGetErrorString(e2));
    g_dense_status_ptr[dev] = static_cast<int*>(p);
  }
  *out = g_dense_status_ptr[dev];
  return MLA_OK;
}

constexpr int kDenseMaxSplits = 8;

// Bytes of the split-key partials for `splits` ranges: fp32 O rows, then (max, sum) pairs.
size_t dense_ws_bytes(int splits, int batch, int n_q, int n_heads) {
  if (splits <= 1) return 0;
  const size_t rows = (size_t)batch * n_q * n_heads;
  return align256((size_t)splits * rows * 128 * 4) + (size_t)splits * rows * 8;
}

// Key ranges per (query tile, head, stream) item.  Cost model in units of one 128-key tile step
// of a full wave: the waves the CTAs take, each as long as its range plus about two tiles of
// fixed cost (the Q tile, pipeline fill, epilogue); every split adds fp32 partial traffic of
// about 0.018 tile steps per item (128 rows x 128 channels x 4 bytes, written and read once).
int dense_splits(int batch, int n_q, int n_kv, int n_heads, int num_sms) {
  const int64_t items = (int64_t)((n_q + 127) / 128) * n_heads * batch;
  const int nt = (n_kv + 127) / 128;
  int best = 1;
  double best_cost = 0.0;
  for (int s = 1; s <= kDenseMaxSplits && s <= nt; ++s) {
    const int per = (nt + s - 1) / s;              // tiles per range
    if ((int64_t)(s - 1) * per >= nt) break;       // the last range would be empty
    const double waves = (double)((items * s + num_sms - 1) / num_sms);
    const double cost = waves * (per + 2.0) + (s > 1 ? 0.018 * (double)items * (s + 1) : 0.0);
    if (s == 1 || cost < best_cost) {
      best = s;
      best_cost = cost;
    }
  }
  return best;
}

// Key ranges actually launched: dense_splits, lowered until the workspace holds the partials,
// the grid's z extent (batch x splits) fits and the last range is not empty.  Ranges are whole
// 128-key tiles; one range (no workspace) covers all n_kv keys.
void dense_plan(int batch, int n_q, int n_kv, int n_heads, int num_sms, size_t ws_bytes,
                int* splits_out, int* kv_per_split_out) {
  const int nt = (n_kv + 127) / 128;
  int splits = ws_bytes ? dense_splits(batch, n_q, n_kv, n_heads, num_sms) : 1;
  while (splits > 1 && (dense_ws_bytes(splits, batch, n_q, n_heads) > ws_bytes ||
                        (int64_t)batch * splits > 65535 ||
                        (splits - 1) * ((nt + splits - 1) / splits) >= nt))
    --splits;
  *splits_out = splits;
  *kv_per_split_out = splits > 1 ? (nt + splits - 1) / splits * 128 : n_kv;
}

// Dense per-head attention over compact q [B][n_q][H][128], k, v [B][n_kv][H][128] (bf16).
// With a workspace of dense_ws_bytes(s, ...) bytes the keys are split into s ranges (the count
// dense_splits chooses, or fewer when the workspace holds fewer) and merged by a second kernel.
mla_status launch_dense(const void* q, const void* k, const void* v, void* out, int batch,
                        int n_q, int n_kv, int n_heads, float scale, int* status, void* ws,
                        size_t ws_bytes, int num_sms, cudaStream_t st) {
  const uint64_t row = (uint64_t)n_heads * 128;
  CUtensorMap mq, mk, mv;
  mla_status s;
  if ((s = make_map(&mq, q, row, n_q, batch, row * 2, row * n_q * 2, 64, 128,
                    CU_TENSOR_MAP_SWIZZLE_128B)) != MLA_OK)
    return s;
  if ((s = make_map(&mk, k, row, n_kv, batch, row * 2, row * n_kv * 2, 64, 128,
                    CU_TENSOR_MAP_SWIZZLE_128B)) != MLA_OK)
    return s;
  if ((s = make_map(&mv, v, row, n_kv, batch, row * 2, row * n_kv * 2, 64, 128,
                    CU_TENSOR_MAP_SWIZZLE_128B)) != MLA_OK)
    return s;
  mla::DenseArgs a{};
  a.n_q = n_q;
  a.n_kv = n_kv;
  a.n_heads = n_heads;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.out = static_cast<__nv_bfloat16*>(out);
  int splits = 1, kv_per_split = n_kv;
  dense_plan(batch, n_q, n_kv, n_heads, num_sms, ws ? ws_bytes : 0, &splits, &kv_per_split);
  a.splits = splits;
  a.kv_per_split = kv_per_split;
  a.batch = batch;
  a.part_rows = (int64_t)splits * batch * n_q * n_heads;
#ifdef MLA_DEBUG
  if (splits > 1 && dense_ws_bytes(splits, batch, n_q, n_heads) > ws_bytes)
    return fail(MLA_ERR_BOUNDS, "dense split partials need more than the %zu-byte workspace", ws_bytes);
#endif
  if (splits > 1) {
    const size_t rows = (size_t)batch * n_q * n_heads;
    a.o_part = static_cast<float*>(ws);
    a.ml_part = reinterpret_cast<float2*>(static_cast<uint8_t*>(ws) +
                                          align256((size_t)splits * rows * 128 * 4));
  }
  dim3 grid((unsigned)((n_q + 127) / 128), (unsigned)n_heads, (unsigned)(batch * splits));
  mla::dense_attn_kernel<kDenseStages>
      <<<grid, mla::kDenseThreads, mla::DenseSmem<kDenseStages>::kBytes, st>>>(mq, mk, mv, a, status);
  mla_status s2 = check_launch("dense attention");
  if (s2 != MLA_OK || splits == 1) return s2;
  const int64_t rows = (int64_t)batch * n_q * n_heads;
  mla::dense_combine_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(
      a.o_part, a.ml_part, splits, batch, n_q, n_heads, static_cast<__nv_bfloat16*>(out), a.part_rows, status);
  return check_launch("dense split combine");
}

}  // namespace

extern "C" {

const char* mla_status_string(mla_status s) {
  switch (s) {
    case MLA_OK: return "MLA_OK";
    case MLA_ERR_INVALID_ARGUMENT: return "MLA_ERR_INVALID_ARGUMENT";
    case MLA_ERR_UNSUPPORTED: return "MLA_ERR_UNSUPPORTED";
    case MLA_ERR_OUT_OF_MEMORY: return "MLA_ERR_OUT_OF_MEMORY";
    case MLA_ERR_CUDA: return "MLA_ERR_CUDA";
    case MLA_ERR_DEVICE_TIMEOUT: return "MLA_ERR_DEVICE_TIMEOUT";
    case MLA_ERR_STATE: return "MLA_ERR_STATE";
    case MLA_ERR_RANGE: return "MLA_ERR_RANGE";
    case MLA_ERR_BOUNDS: return "MLA_ERR_BOUNDS";
  }
  return "MLA_ERR_UNKNOWN";
}

const char* mla_last_error(void) { return g_last_error.c_str(); }

mla_status mla_config_check(const mla_config* cfg) {
  if (!cfg) return fail(MLA_ERR_INVALID_ARGUMENT, "config is NULL");
  const mla_config& c = *cfg;
  if (c.hidden <= 0 || c.n_heads <= 0 || c.d_head <= 0 || c.d_nope <= 0 || c.d_latent <= 0 ||
      c.d_rope < 0)
    return fail(MLA_ERR_INVALID_ARGUMENT, "dimensions must be positive");
  if (c.rope_t < 0 || c.rope_h < 0 || c.rope_w < 0 || (c.rope_t | c.rope_h | c.rope_w) & 1)
    return fail(MLA_ERR_INVALID_ARGUMENT, "RoPE axis widths must be even and non-negative");
  if (c.rope_t + c.rope_h + c.rope_w != c.d_rope)
    return fail(MLA_ERR_INVALID_ARGUMENT, "rope_t + rope_h + rope_w must equal d_rope");
  if (!(c.rope_base > 0.0) || !std::isfinite(c.rope_base))
    return fail(MLA_ERR_INVALID_ARGUMENT, "rope_base must be positive and finite");
  if (c.frame_h <= 0 || c.frame_w <= 0 || c.window_frames <= 0 || c.max_chunk_frames <= 0 ||
      c.batch <= 0)
    return fail(MLA_ERR_INVALID_ARGUMENT, "frame grid, window, chunk and batch must be >= 1");
  if (!(c.softmax_scale >= 0.f) || !std::isfinite(c.softmax_scale))
    return fail(MLA_ERR_INVALID_ARGUMENT, "softmax_scale must be finite and >= 0");
  if (c.d_q < 0 || c.sink_frames < 0)
    return fail(MLA_ERR_INVALID_ARGUMENT, "d_q and sink_frames must be >= 0");
  if (c.sink_frames > (1 << 20))
    return fail(MLA_ERR_INVALID_ARGUMENT, "sink_frames too large");
  const int64_t F = (int64_t)c.frame_h * c.frame_w;
  const int64_t rows = sink_rows_of(c) + (int64_t)(c.window_frames + (int64_t)c.max_chunk_frames) * F;
  if (rows > (int64_t)1 << 30 || (int64_t)c.max_chunk_frames * F * c.n_heads > (int64_t)1 << 30)
    return fail(MLA_ERR_INVALID_ARGUMENT, "window or chunk too large (row index overflow)");
  if ((int64_t)c.batch * rows * kQK > ((int64_t)1 << 40))
    return fail(MLA_ERR_INVALID_ARGUMENT, "cache too large");
  if (c.d_latent != kLatent || c.d_rope != kRope)
    return fail(MLA_ERR_UNSUPPORTED, "kernels are built for d_latent = 192 and d_rope = 32");
  if (c.hidden % 128 != 0)
    return fail(MLA_ERR_UNSUPPORTED, "hidden must be a multiple of 128");
  if (c.batch > 65535 || (c.n_heads + 1) > 65535)
    return fail(MLA_ERR_UNSUPPORTED, "batch and heads must fit a grid dimension");
  return MLA_OK;
}

mla_status mla_ring_slot(const mla_config* cfg, int64_t frame, int32_t token, int64_t* slot) {
  if (!cfg || !slot) return fail(MLA_ERR_INVALID_ARGUMENT, "NULL argument");
  if (cfg->window_frames <= 0 || cfg->frame_h <= 0 || cfg->frame_w <= 0)
    return fail(MLA_ERR_INVALID_ARGUMENT, "window and frame grid must be >= 1");
  const int64_t F = (int64_t)cfg->frame_h * cfg->frame_w;
  if (frame < 0 || token < 0 || token >= F)
    return fail(MLA_ERR_INVALID_ARGUMENT, "frame must be >= 0 and token in [0, F)");
  if (cfg->sink_frames < 0) return fail(MLA_ERR_INVALID_ARGUMENT, "sink_frames must be >= 0");
  if (frame < cfg->sink_frames)
    *slot = frame * F + token;
  else
    *slot = sink_rows_of(*cfg) + ((frame - cfg->sink_frames) % cfg->window_frames) * F + token;
  return MLA_OK;
}

mla_status mla_cache_slot(const mla_cache* c, int64_t frame, int32_t token, int64_t* slot) {
  if (!c) return fail(MLA_ERR_INVALID_ARGUMENT, "NULL cache");
  return mla_ring_slot(&c->cfg, frame, token, slot);
}

mla_status mla_commit_plan(const mla_config* cfg, int64_t frames_appended, int32_t n_frames,
                           mla_row_move* moves, int32_t max_moves, int32_t* n_moves) {
  if (!cfg || !n_moves || (max_moves > 0 && !moves))
    return fail(MLA_ERR_INVALID_ARGUMENT, "NULL argument");
  mla_status s = mla_config_check(cfg);
  if (s != MLA_OK) return s;
  const mla_config& k = *cfg;
  if (n_frames < 1 || n_frames > k.max_chunk_frames || frames_appended < 0)
    return fail(MLA_ERR_INVALID_ARGUMENT, "n_frames must be in [1, max_chunk_frames] and frames_appended >= 0");
  const int64_t S = k.sink_frames, W = k.window_frames, F = (int64_t)k.frame_h * k.frame_w;
  const int64_t A = frames_appended, sink_rows = sink_rows_of(k);
  int64_t vs, vw;
  valid_counts_of(k, A, vs, vw);
  const int64_t base_row = sink_rows + vw * F;      // where the attention call put the chunk
  // Chunk frames that become sink frames, then the others, of which only the last W survive.
  const int64_t to_sink = A < S ? (S - A < n_frames ? S - A : n_frames) : 0;
  const int64_t n_window = n_frames - to_sink;
  const int64_t skip = n_window > W ? n_window - W : 0;
  int32_t n = 0;
  for (int64_t i = 0; i < n_frames; ++i) {
    if (i >= to_sink && i - to_sink < skip) continue;            // evicted within the chunk
    const int64_t t = A + i;
    const int64_t dst = t < S ? t * F : sink_rows + ((t - S) % W) * F;
    const int64_t src = base_row + i * F;
    if (dst == src) continue;                                    // already in place
    if (n >= max_moves) return fail(MLA_ERR_INVALID_ARGUMENT, "more than max_moves moves");
    moves[n++] = mla_row_move{src, dst, F};
  }
  *n_moves = n;
  return MLA_OK;
}

size_t mla_ring_bytes(const mla_config* cfg) {
  if (!cfg || cfg->batch <= 0 || cfg->window_frames <= 0 || cfg->frame_h <= 0 ||
      cfg->frame_w <= 0 || cfg->d_latent <= 0 || cfg->d_rope < 0 || cfg->sink_frames < 0)
    return 0;
  return (size_t)cfg->batch * (size_t)(cfg->sink_frames + cfg->window_frames) * cfg->frame_h *
         cfg->frame_w * (size_t)(cfg->d_latent + cfg->d_rope) * 2;
}

size_t mla_cache_bytes(const mla_config* cfg) { return mla_ring_bytes(cfg); }

size_t mla_cache_device_bytes(const mla_config* cfg) {
  if (mla_config_check(cfg) != MLA_OK) return 0;
  const mla_config& c = *cfg;
  const size_t F = (size_t)c.frame_h * c.frame_w;
  const size_t rows = (size_t)sink_rows_of(c) + (size_t)(c.window_frames + c.max_chunk_frames) * F;
  const size_t q = (size_t)c.max_chunk_frames * F;
  size_t b = 0;
  b += (size_t)c.batch * rows * kQK * 2;                   // ckv + krope (ring + chunk tail)
  b += (size_t)c.batch * q * c.n_heads * kQK * 2;          // Qp
  b += (size_t)c.batch * q * c.n_heads * kLatent * 2;      // o_lat
  if (c.d_q == 0 && c.d_nope == mla::kQpNope)              // the caller's query and latent
    b += ((size_t)(c.n_heads * mla::kQpBN + kQK - 1) / kQK * kQK + kQK) * c.hidden * 2 +
         (size_t)c.n_heads * mla::kQpNope * kLatent * 2;      // weights (bf16), W_UK (fp16)
  else
    b += (size_t)(c.n_heads + 1) * kQK * c.hidden * 4;     // Wqcat (bf16 hi + lo)
  b += (size_t)c.hidden * c.n_heads * kLatent * 2;         // W_OV
  b += 256;                                                // status word
  b += (size_t)(c.frame_h + c.frame_w) * 16 * 8;           // RoPE h / w tables
  if (c.d_nope + c.d_rope == 128 && c.d_head == 128 && c.d_nope % 32 == 0 && c.sink_frames == 0)
    b += (size_t)c.n_heads * 128 * ((size_t)c.hidden * 2 * 2 + kLatent * 2) +   // W_Qd, W_O; W_UV
         (size_t)c.n_heads * c.d_nope * kLatent * 2;                           // W_UK
  return b;
}

void mla_cache_destroy(mla_cache* c) {
  if (!c) return;
  cudaDeviceSynchronize();
  for (auto& r : c->pending) {
    cudaEventDestroy(r.a);
    cudaEventDestroy(r.b);
  }
  for (auto e : c->pool) cudaEventDestroy(e);
  cudaFree(c->ckv);
  cudaFree(c->krope);
  cudaFree(c->qp);
  cudaFree(c->o_lat);
  cudaFree(c->wqcat);
  cudaFree(c->wuk16);
  cudaFree(c->wov);
  cudaFree(c->rope_hw);
  cudaFree(c->wqd);
  cudaFree(c->wukh);
  cudaFree(c->wuvh);
  cudaFree(c->wo);
  cudaFree(c->qd);
  cudaFree(c->kd);
  cudaFree(c->vd);
  cudaFree(c->od);
  cudaFree(c->dws);
  cudaFree(c->status);
  delete c;
}

mla_status mla_cache_create(const mla_config* cfg, const mla_weights* w, void* stream,
                            mla_cache** out) {
  if (!out) return fail(MLA_ERR_INVALID_ARGUMENT, "out is NULL");
  *out = nullptr;
  mla_status s = mla_config_check(cfg);
  if (s != MLA_OK) return s;
  if (!w || !w->w_q || !w->w_qr || !w->w_dkv || !w->w_kr || !w->w_uk || !w->w_uv || !w->w_o)
    return fail(MLA_ERR_INVALID_ARGUMENT, "a weight pointer is NULL");
  if (cfg->d_q > 0 && !w->w_dq)
    return fail(MLA_ERR_INVALID_ARGUMENT, "d_q > 0 needs w_dq");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);

  mla_cache* c = new mla_cache();
  c->cfg = *cfg;
  c->F = cfg->frame_h * cfg->frame_w;
  c->sink_rows = sink_rows_of(*cfg);
  c->rows_per_stream = c->sink_rows + (int64_t)(cfg->window_frames + cfg->max_chunk_frames) * c->F;
  c->max_q_tokens = (int64_t)cfg->max_chunk_frames * c->F;
  c->softmax_scale = cfg->softmax_scale > 0.f
                         ? cfg->softmax_scale
                         : (float)(1.0 / std::sqrt((double)(cfg->d_nope + cfg->d_rope)));
  c->rope = make_bands(*cfg);
  cudaGetDevice(&c->device);
  if (cudaDeviceGetAttribute(&c->num_sms, cudaDevAttrMultiProcessorCount, c->device) != cudaSuccess ||
      c->num_sms <= 0)
    c->num_sms = 148;

  auto cleanup = [&](mla_status r) {
    mla_cache_destroy(c);
    return r;
  };
#define MLA_TRY(call)                                                                \
  do {                                                                               \
    cudaError_t e_ = (call);                                                         \
    if (e_ != cudaSuccess)                                                           \
      return cleanup(fail(e_ == cudaErrorMemoryAllocation ? MLA_ERR_OUT_OF_MEMORY : MLA_ERR_CUDA, \
                          "%s failed: %s", #call, cudaGetErrorString(e_)));          \
  } while (0)

  const mla_config& k = *cfg;
  const size_t ring_rows = (size_t)k.batch * c->rows_per_stream;
  const size_t q_rows = (size_t)k.batch * c->max_q_tokens;
  MLA_TRY(alloc_buffer(c, &c->ckv, ring_rows * kLatent * 2, "c_kv plane", st));
  MLA_TRY(alloc_buffer(c, &c->krope, ring_rows * kRope * 2, "k_rope plane", st));
  MLA_TRY(alloc_buffer(c, &c->qp, q_rows * k.n_heads * kQK * 2, "Qp", st));
  MLA_TRY(alloc_buffer(c, &c->o_lat, q_rows * k.n_heads * kLatent * 2, "o_lat", st));
  c->two_step = k.d_q == 0 && k.d_nope == mla::kQpNope;
  c->latent_row0 = c->two_step ? (k.n_heads * mla::kQpBN + kQK - 1) / kQK * kQK : k.n_heads * kQK;
  c->wq_rows = (int64_t)c->latent_row0 + kQK;
  c->wq_cols = c->two_step ? k.hidden : 2 * (int64_t)k.hidden;
  MLA_TRY(alloc_buffer(c, &c->wqcat, (size_t)c->wq_rows * c->wq_cols * 2, "W_qcat", st));
  if (c->two_step)
    MLA_TRY(alloc_buffer(c, &c->wuk16, (size_t)k.n_heads * mla::kQpNope * kLatent * 2, "W_UK fp16", st));
  MLA_TRY(alloc_buffer(c, &c->wov, (size_t)k.hidden * k.n_heads * kLatent * 2, "W_OV", st));
  MLA_TRY(alloc_buffer(c, &c->status, 256, "status block", st));
  const std::vector<float2> rope_hw = make_rope_hw(k);
  MLA_TRY(alloc_buffer(c, &c->rope_hw, rope_hw.size() * sizeof(float2), "RoPE table", st));
  MLA_TRY(cudaMemcpyAsync(c->rope_hw, rope_hw.data(), rope_hw.size() * sizeof(float2),
                          cudaMemcpyHostToDevice, st));
  MLA_TRY(cudaMemsetAsync(c->ckv, 0, ring_rows * kLatent * 2, st));
  MLA_TRY(cudaMemsetAsync(c->krope, 0, ring_rows * kRope * 2, st));
  MLA_TRY(cudaMemsetAsync(c->qp, 0, q_rows * k.n_heads * kQK * 2, st));
  MLA_TRY(cudaMemsetAsync(c->o_lat, 0, q_rows * k.n_heads * kLatent * 2, st));
  MLA_TRY(cudaMemsetAsync(c->status, 0, 256, st));

  // fp32 temporaries of the low-rank query composition, freed on every exit (after the
  // stream synchronisation below on success).
  struct DevTmp {
    float* p = nullptr;
    ~DevTmp() {
      if (p) cudaFree(p);
    }
  } t_f32, qabs_f32, qr_f32;
  {
    const __nv_bfloat16* w_q = (const __nv_bfloat16*)w->w_q;
    const __nv_bfloat16* w_qr = (const __nv_bfloat16*)w->w_qr;
    const __nv_bfloat16* w_uk = (const __nv_bfloat16*)w->w_uk;
    if (k.d_q > 0) {
      // Low-rank query ([VideoMLA] §4.1): the query projections read c_q = x W_DQ^T, so
      // W_Qabs[h] = (W_UK[h]^T W_Q[h]) W_DQ and W_QR,eff = W_QR W_DQ, composed in fp32.
      const __nv_bfloat16* w_dq = (const __nv_bfloat16*)w->w_dq;
      const int dn = k.d_nope, dq = k.d_q, nh = k.n_heads;
      MLA_TRY(cudaMalloc(&t_f32.p, (size_t)nh * kLatent * dq * 4));
      MLA_TRY(cudaMalloc(&qabs_f32.p, (size_t)nh * kLatent * k.hidden * 4));
      MLA_TRY(cudaMalloc(&qr_f32.p, (size_t)nh * kRope * k.hidden * 4));
      // T[h][c][j] = sum_n W_UK[h*dn + n][c] W_Q[h*dn + n][j]
      compose_kernel<__nv_bfloat16, __nv_bfloat16><<<dim3((dq + 255) / 256, kLatent, nh), 256, 0, st>>>(
          w_uk, (int64_t)dn * kLatent, 1, kLatent, w_q, (int64_t)dn * dq, dq, t_f32.p,
          (int64_t)kLatent * dq, kLatent, dq, dn);
      MLA_TRY(cudaGetLastError());
      // W_Qabs[h*192 + c][i] = sum_j T[h][c][j] W_DQ[j][i]
      compose_kernel<float, __nv_bfloat16><<<dim3((k.hidden + 255) / 256, nh * kLatent, 1), 256, 0, st>>>(
          t_f32.p, 0, dq, 1, w_dq, 0, k.hidden, qabs_f32.p, 0, nh * kLatent, k.hidden, dq);
      MLA_TRY(cudaGetLastError());
      // W_QR,eff[r][i] = sum_j W_QR[r][j] W_DQ[j][i]
      compose_kernel<__nv_bfloat16, __nv_bfloat16><<<dim3((k.hidden + 255) / 256, nh * kRope, 1), 256, 0, st>>>(
          w_qr, 0, dq, 1, w_dq, 0, k.hidden, qr_f32.p, 0, nh * kRope, k.hidden, dq);
      MLA_TRY(cudaGetLastError());
    }
    dim3 g((k.hidden + 255) / 256, (unsigned)c->wq_rows);
    if (c->two_step) {
      build_wq2_kernel<<<g, 256, 0, st>>>(w_q, w_qr, (const __nv_bfloat16*)w->w_dkv,
                                          (const __nv_bfloat16*)w->w_kr, c->wqcat, k.hidden,
                                          k.n_heads, c->latent_row0);
      const int64_t n_uk = (int64_t)k.n_heads * mla::kQpNope * kLatent;
      bf16_to_f16_kernel<<<(unsigned)((n_uk + 255) / 256), 256, 0, st>>>(
          w_uk, c->wuk16, n_uk, c->status + mla::kStatusRangeWord);
    } else {
      build_wqcat_kernel<<<g, 256, 0, st>>>(w_q, w_qr, (const __nv_bfloat16*)w->w_dkv,
                                            (const __nv_bfloat16*)w->w_kr, w_uk, qabs_f32.p,
                                            qr_f32.p, c->wqcat, k.hidden, k.n_heads, k.d_nope);
    }
    MLA_TRY(cudaGetLastError());
    dim3 g2((k.n_heads * kLatent + 255) / 256, k.hidden);
    build_wov_kernel<<<g2, 256, 0, st>>>((const __nv_bfloat16*)w->w_o,
                                         (const __nv_bfloat16*)w->w_uv, c->wov, k.hidden,
                                         k.n_heads, k.d_head, c->status + mla::kStatusRangeWord);
    MLA_TRY(cudaGetLastError());
  }
  // Weights of the reconstruct-then-dense form (training-time layout, [VideoMLA] §3.3).
  c->dense_ok = k.d_nope + k.d_rope == 128 && k.d_head == 128 && k.d_nope % 32 == 0 &&
                k.sink_frames == 0;
  DevTmp qeff_f32;
  if (c->dense_ok) {
    const int nh = k.n_heads, dn = k.d_nope;
    MLA_TRY(alloc_buffer(c, &c->wqd, (size_t)nh * 128 * k.hidden * 2, "dense W_Q", st));
    MLA_TRY(alloc_buffer(c, &c->wukh, (size_t)nh * dn * kLatent * 2, "dense W_UK", st));
    MLA_TRY(alloc_buffer(c, &c->wuvh, (size_t)nh * 128 * kLatent * 2, "dense W_UV", st));
    MLA_TRY(alloc_buffer(c, &c->wo, (size_t)k.hidden * nh * 128 * 2, "dense W_O", st));
    if (k.d_q > 0) {
      // W_Q W_DQ in fp32 (W_QR W_DQ is qr_f32 above).
      MLA_TRY(cudaMalloc(&qeff_f32.p, (size_t)nh * dn * k.hidden * 4));
      compose_kernel<__nv_bfloat16, __nv_bfloat16><<<dim3((k.hidden + 255) / 256, nh * dn, 1), 256, 0, st>>>(
          (const __nv_bfloat16*)w->w_q, 0, k.d_q, 1, (const __nv_bfloat16*)w->w_dq, 0, k.hidden,
          qeff_f32.p, 0, nh * dn, k.hidden, k.d_q);
      MLA_TRY(cudaGetLastError());
    }
    build_wqd_kernel<<<dim3((k.hidden + 255) / 256, nh * 128), 256, 0, st>>>(
        (const __nv_bfloat16*)w->w_q, (const __nv_bfloat16*)w->w_qr, qeff_f32.p, qr_f32.p, c->wqd,
        k.hidden, nh, dn);
    MLA_TRY(cudaGetLastError());
    const int64_t n_uk = (int64_t)nh * dn * kLatent, n_uv = (int64_t)nh * 128 * kLatent;
    bf16_to_f16_kernel<<<(unsigned)((n_uk + 255) / 256), 256, 0, st>>>(
        (const __nv_bfloat16*)w->w_uk, c->wukh, n_uk, c->status + mla::kStatusRangeWord);
    bf16_to_f16_kernel<<<(unsigned)((n_uv + 255) / 256), 256, 0, st>>>(
        (const __nv_bfloat16*)w->w_uv, c->wuvh, n_uv, c->status + mla::kStatusRangeWord);
    MLA_TRY(cudaGetLastError());
    MLA_TRY(cudaMemcpyAsync(c->wo, w->w_o, (size_t)k.hidden * nh * 128 * 2,
                            cudaMemcpyDeviceToDevice, st));
    const uint64_t qd_cols = (uint64_t)nh * 128;
    if ((s = make_map(&c->map_wqd, c->wqd, k.hidden, qd_cols, 1, (uint64_t)k.hidden * 2,
                      qd_cols * k.hidden * 2, 64, kOutBN, CU_TENSOR_MAP_SWIZZLE_128B)) != MLA_OK ||
        (s = make_map(&c->map_wukh, c->wukh, kLatent, (uint64_t)nh * dn, 1, kLatent * 2,
                      (uint64_t)nh * dn * kLatent * 2, 64, kOutBN, CU_TENSOR_MAP_SWIZZLE_128B,
                      true)) != MLA_OK ||
        (s = make_map(&c->map_wuvh, c->wuvh, kLatent, qd_cols, 1, kLatent * 2,
                      qd_cols * kLatent * 2, 64, kOutBN, CU_TENSOR_MAP_SWIZZLE_128B, true)) != MLA_OK ||
        (s = make_map(&c->map_wo, c->wo, qd_cols, k.hidden, 1, qd_cols * 2,
                      qd_cols * k.hidden * 2, 64, kOutBN, CU_TENSOR_MAP_SWIZZLE_128B)) != MLA_OK)
      return cleanup(s);
  }
  {
    const uint64_t wr = (uint64_t)c->wq_rows, wc = (uint64_t)c->wq_cols;
    if ((s = make_map(&c->map_wqcat, c->wqcat, wc, wr, 1, wc * 2, wr * wc * 2, 64, kQK,
                      CU_TENSOR_MAP_SWIZZLE_128B)) != MLA_OK ||
        (s = make_map(&c->map_wqcat160, c->wqcat, wc, wr, 1, wc * 2, wr * wc * 2, 64, 160,
                      CU_TENSOR_MAP_SWIZZLE_128B)) != MLA_OK ||
        (s = make_map(&c->map_wqcat32, c->wqcat, wc, wr, 1, wc * 2, wr * wc * 2, 64, 32,
                      CU_TENSOR_MAP_SWIZZLE_128B)) != MLA_OK)
      return cleanup(s);
    if (c->two_step) {
      const uint64_t ur = (uint64_t)k.n_heads * mla::kQpNope;
      if ((s = make_map(&c->map_wuk16, c->wuk16, kLatent, ur, 1, kLatent * 2, ur * kLatent * 2, 64,
                        mla::kQpNope, CU_TENSOR_MAP_SWIZZLE_128B, true)) != MLA_OK)
        return cleanup(s);
    }
  }
  s = make_map(&c->map_wov, c->wov, (uint64_t)k.n_heads * kLatent, k.hidden, 1,
               (uint64_t)k.n_heads * kLatent * 2, (uint64_t)k.hidden * k.n_heads * kLatent * 2,
               64, kOutBN, CU_TENSOR_MAP_SWIZZLE_128B, true);
  if (s != MLA_OK) return cleanup(s);

  static std::once_flag attr_once;
  static mla_status attr_status = MLA_OK;
  std::call_once(attr_once, [] {
    mla_status r = set_smem(mla::tc_gemm_kernel<kQK, kProjAStages, kProjBStages, mla::kEpiLatent, false, 1>,
                            mla::GemmSmem<kQK, kProjAStages, kProjBStages, 1>::kBytes);
    if (r == MLA_OK)
      r = set_smem(mla::tc_gemm_kernel<kQK, kProjWideAStages, kProjWideBStages, mla::kEpiLatent, false, 2>,
                   mla::GemmSmem<kQK, kProjWideAStages, kProjWideBStages, 2>::kBytes);
    if (r == MLA_OK)
      r = set_smem(mla::tc_gemm_kernel<160, kProjMidAStages, kProjMidBStages, mla::kEpiLatent, false, 2>,
                   mla::GemmSmem<160, kProjMidAStages, kProjMidBStages, 2>::kBytes);
    if (r == MLA_OK)
      r = set_smem(mla::tc_gemm_kernel<32, kProjNarrowAStages, kProjNarrowBStages, mla::kEpiLatent, false, 1>,
                   mla::GemmSmem<32, kProjNarrowAStages, kProjNarrowBStages, 1>::kBytes);
    if (r == MLA_OK)
      r = set_smem(mla::tc_gemm_kernel<kOutBN, kOutAStages, kOutBStages, mla::kEpiStore, true, 1>,
                   mla::GemmSmem<kOutBN, kOutAStages, kOutBStages>::kBytes);
    if (r == MLA_OK)
      r = set_smem(mla::tc_gemm_kernel<kOutBN, kOutAStages, kOutBStages, mla::kEpiDense, false, 1>,
                   mla::GemmSmem<kOutBN, kOutAStages, kOutBStages>::kBytes);
    if (r == MLA_OK)
      r = set_smem(mla::tc_gemm_kernel<kOutBN, kOutAStages, kOutBStages, mla::kEpiDense, true, 1>,
                   mla::GemmSmem<kOutBN, kOutAStages, kOutBStages>::kBytes);
    if (r == MLA_OK)
      r = set_smem(mla::tc_gemm_kernel<kOutBN, kOutAStages, kOutBStages, mla::kEpiStore, false, 1>,
                   mla::GemmSmem<kOutBN, kOutAStages, kOutBStages>::kBytes);
    if (r == MLA_OK)
      r = set_smem(mla::dense_attn_kernel<kDenseStages>, mla::DenseSmem<kDenseStages>::kBytes);
    if (r == MLA_OK)
      r = set_smem(mla::query_proj_kernel, mla::QpSmem::kBytes);
    if (r == MLA_OK)
      r = set_smem(mla::window_attn_kernel<kAttnStages>,
                   mla::AttnSmem<kAttnStages>::kBytes);
    attr_status = r;
  });
  if (attr_status != MLA_OK) return cleanup(attr_status);

  MLA_TRY(cudaStreamSynchronize(st));
  {
    // The fp16 weights (W_OV, and the dense form's W_UK, W_UV) must fit the fp16 range.
    int range = 0;
    MLA_TRY(cudaMemcpy(&range, c->status + mla::kStatusRangeWord, sizeof(int), cudaMemcpyDeviceToHost));
    if (range != 0)
      return cleanup(fail(MLA_ERR_RANGE, "an fp16 weight (W_OV = W_O W_UV per head, or W_UK / W_UV) "
                                         "exceeds the fp16 range +-65504"));
  }
#undef MLA_TRY
  *out = c;
  return MLA_OK;
}

mla_status mla_cache_append(mla_cache* c, const void* x, int32_t n_frames, void* stream) {
  if (!c || !x) return fail(MLA_ERR_INVALID_ARGUMENT, "NULL argument");
  if (n_frames < 1) return fail(MLA_ERR_INVALID_ARGUMENT, "n_frames must be >= 1");
  if (!aligned16(x)) return fail(MLA_ERR_INVALID_ARGUMENT, "x must be 16-byte aligned");
  if ((int64_t)n_frames * c->F > ((int64_t)1 << 30))
    return fail(MLA_ERR_INVALID_ARGUMENT, "too many frames in one append");
  if (c->frames_appended + n_frames > kMaxFrames)
    return fail(MLA_ERR_UNSUPPORTED, "temporal index would pass 2^24 frames (RoPE angles are formed "
                                     "in fp32 from the frame index, exact below 2^24)");
  const mla_config& cfg = c->cfg;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t S = cfg.sink_frames, W = cfg.window_frames;
  const int64_t x_batch_rows = (int64_t)n_frames * c->F;
  const int64_t frame_elems = c->F * (int64_t)cfg.hidden;
  const __nv_bfloat16* xp = static_cast<const __nv_bfloat16*>(x);
  int64_t t = c->frames_appended;   // absolute index of the next frame
  int64_t left = n_frames;
  mla_status s = MLA_OK;
  {
    ProfScope p(c, MLA_KERNEL_APPEND, st);
    // 1. Frames that are still sink frames go to rows t * F of the sink region.
    if (t < S) {
      const int64_t nf = left < S - t ? left : S - t;
      s = launch_latent_gemm(c, xp, nf * c->F, x_batch_rows, false, t, t * c->F, st);
      xp += nf * frame_elems;
      t += nf;
      left -= nf;
    }
    // 2. Of the rest, only the last W frames survive in the ring.
    if (left > W) {
      xp += (left - W) * frame_elems;
      t += left - W;
      left = W;
    }
    // 3. Window frames go to ring slots ((t - S) mod W): one launch per run of consecutive slots.
    while (left > 0 && s == MLA_OK) {
      const int64_t slot = (t - S) % W;
      const int64_t nf = left < W - slot ? left : W - slot;
      s = launch_latent_gemm(c, xp, nf * c->F, x_batch_rows, false, t,
                             c->sink_rows + slot * c->F, st);
      xp += nf * frame_elems;
      t += nf;
      left -= nf;
    }
  }
  if (s != MLA_OK) return s;
  c->frames_appended += n_frames;
  c->pending_frames = 0;
  return MLA_OK;
}

mla_status mla_cache_commit(mla_cache* c, int32_t n_frames, void* stream) {
  if (!c) return fail(MLA_ERR_INVALID_ARGUMENT, "NULL cache");
  if (c->pending_frames == 0 || c->pending_at != c->frames_appended)
    return fail(MLA_ERR_STATE, "no attention chunk to commit (no attention call since the last "
                               "append or commit)");
  if (n_frames != c->pending_frames)
    return fail(MLA_ERR_STATE, "n_frames %d differs from the last attention call's %d", n_frames,
                c->pending_frames);
  const mla_config& cfg = c->cfg;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  std::vector<mla_row_move> moves((size_t)n_frames);
  int32_t n_moves = 0;
  mla_status s = mla_commit_plan(&cfg, c->frames_appended, n_frames, moves.data(), n_frames, &n_moves);
  if (s != MLA_OK) return s;
  {
    ProfScope p(c, MLA_KERNEL_APPEND, st);
    // In the plan's order (a destination can be the source of an earlier move only), one launch
    // per frame, stream-ordered.
    for (int32_t i = 0; i < n_moves; ++i) {
      const int64_t work = moves[i].rows * (kLatent / 8 + kRope / 8);
      dim3 grid((unsigned)((work + 255) / 256), (unsigned)cfg.batch);
      const cudaError_t e = launch_pdl(move_rows_kernel, grid, dim3(256), 0, st, c->ckv, c->krope,
                                       (int64_t)c->rows_per_stream, moves[i].src_row,
                                       moves[i].dst_row, moves[i].rows, c->status);
      if (e != cudaSuccess)
        return fail(MLA_ERR_CUDA, "commit copy launch failed: %s", cudaGetErrorString(e));
      if ((s = check_launch("commit copy")) != MLA_OK) return s;
    }
  }
  c->frames_appended += n_frames;
  c->pending_frames = 0;
  return MLA_OK;
}

mla_status mla_window_attention(mla_cache* c, const void* x_chunk, int32_t n_frames, void* out,
                                void* stream) {
  if (!c || !x_chunk || !out) return fail(MLA_ERR_INVALID_ARGUMENT, "NULL argument");
  const mla_config& cfg = c->cfg;
  if (n_frames < 1 || n_frames > cfg.max_chunk_frames)
    return fail(MLA_ERR_INVALID_ARGUMENT, "n_frames must be in [1, max_chunk_frames=%d]",
                cfg.max_chunk_frames);
  if (!aligned16(x_chunk) || !aligned16(out))
    return fail(MLA_ERR_INVALID_ARGUMENT, "x_chunk and out must be 16-byte aligned");
  if (c->frames_appended + n_frames > kMaxFrames)
    return fail(MLA_ERR_UNSUPPORTED, "temporal index of the chunk would pass 2^24 frames");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t nq = (int64_t)n_frames * c->F;
  int64_t vs, vw;
  valid_counts(c, vs, vw);
  const int64_t base_row = c->sink_rows + vw * c->F;   // chunk latents go right after the window
  const int64_t n_keys = base_row + nq;
  mla_status s;

  // 1. absorbed queries + chunk latents (one GEMM over [heads | latent] column blocks)
  {
    ProfScope p(c, MLA_KERNEL_QPROJ, st);
    s = launch_latent_gemm(c, x_chunk, nq, nq, true, c->frames_appended, base_row, st);
  }
  if (s != MLA_OK) return s;

  // 2. window attention over [0, n_keys) of every stream
  {
    const int64_t R = nq * cfg.n_heads;
    const uint64_t qp_rows = (uint64_t)c->max_q_tokens * cfg.n_heads;
    if ((s = launch_attention(c, c->qp, (int64_t)qp_rows * kQK, R, n_keys, c->o_lat,
                              (int64_t)c->max_q_tokens * cfg.n_heads * kLatent, st, true)) != MLA_OK)
      return s;
  }

  // 3. output projection out = o_lat W_OV^T
  {
    ProfScope p(c, MLA_KERNEL_OPROJ, st);
    s = launch_out_proj(c, c->o_lat, c->max_q_tokens, nq, out, st, "output projection");
  }
  if (s == MLA_OK) set_pending(c, n_frames);
  return s;
}

mla_status mla_window_attention_noalloc(mla_cache* c, const void* x_chunk, int32_t n_frames,
                                        void* out, void* stream) {
  if (!c || !x_chunk || !out) return fail(MLA_ERR_INVALID_ARGUMENT, "NULL argument");
  const mla_config& cfg = c->cfg;
  if (n_frames < 1 || n_frames > cfg.max_chunk_frames)
    return fail(MLA_ERR_INVALID_ARGUMENT, "n_frames must be in [1, max_chunk_frames=%d]",
                cfg.max_chunk_frames);
  if (!aligned16(x_chunk) || !aligned16(out))
    return fail(MLA_ERR_INVALID_ARGUMENT, "x_chunk and out must be 16-byte aligned");
  if (c->frames_appended + n_frames > kMaxFrames)
    return fail(MLA_ERR_UNSUPPORTED, "temporal index of the chunk would pass 2^24 frames");
  const int64_t nq = (int64_t)n_frames * c->F;
  const int64_t R = nq * cfg.n_heads;                    // Qp / o_lat rows per stream
  const size_t qp_bytes = align256((size_t)cfg.batch * R * kQK * 2);
  const size_t ol_bytes = (size_t)cfg.batch * R * kLatent * 2;
  if (qp_bytes + ol_bytes > kNoAllocScratchBytes)
    return fail(MLA_ERR_INVALID_ARGUMENT,
                "no-alloc scratch too small: this call needs %zu bytes (batch * tokens * heads * "
                "832 B), the fixed scratch holds %zu; use mla_window_attention instead",
                qp_bytes + ol_bytes, kNoAllocScratchBytes);
  int dev = 0;
  MLA_CUDA(cudaGetDevice(&dev));
  if (dev != c->device)
    return fail(MLA_ERR_STATE, "the cache lives on device %d but device %d is current",
                c->device, dev);
  void* scratch = nullptr;
  mla_status s = noalloc_scratch(&scratch);
  if (s != MLA_OK) return s;
  __half* qp = static_cast<__half*>(scratch);
  __half* o_lat = reinterpret_cast<__half*>(static_cast<unsigned char*>(scratch) + qp_bytes);

  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int64_t vs, vw;
  valid_counts(c, vs, vw);
  const int64_t base_row = c->sink_rows + vw * c->F;
  const int64_t n_keys = base_row + nq;

  // 1. absorbed queries (into the scratch) + chunk latents (into the cache's chunk tail)
  if ((s = launch_latent_gemm(c, x_chunk, nq, nq, true, c->frames_appended, base_row, st, qp,
                              nq)) != MLA_OK)
    return s;
  // 2. window attention, o_lat into the scratch
  if ((s = launch_attention(c, qp, R * kQK, R, n_keys, o_lat, R * kLatent, st, false)) != MLA_OK)
    return s;
  // 3. output projection from the scratch o_lat
  s = launch_out_proj(c, o_lat, nq, nq, out, st, "no-alloc output projection");
  if (s == MLA_OK) set_pending(c, n_frames);
  return s;
}

mla_status mla_window_attention_reconstruct(mla_cache* c, const void* x_chunk, int32_t n_frames,
                                            void* out, void* stream) {
  if (!c || !x_chunk || !out) return fail(MLA_ERR_INVALID_ARGUMENT, "NULL argument");
  const mla_config& cfg = c->cfg;
  if (!c->dense_ok)
    return fail(MLA_ERR_UNSUPPORTED,
                "the dense form needs d_nope + d_rope == 128, d_head == 128, d_nope a multiple "
                "of 32 and no sink frames");
  if (n_frames < 1 || n_frames > cfg.max_chunk_frames)
    return fail(MLA_ERR_INVALID_ARGUMENT, "n_frames must be in [1, max_chunk_frames=%d]",
                cfg.max_chunk_frames);
  if (!aligned16(x_chunk) || !aligned16(out))
    return fail(MLA_ERR_INVALID_ARGUMENT, "x_chunk and out must be 16-byte aligned");
  if (c->frames_appended + n_frames > kMaxFrames)
    return fail(MLA_ERR_UNSUPPORTED, "temporal index of the chunk would pass 2^24 frames");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int nh = cfg.n_heads, dn = cfg.d_nope;
  const uint64_t hd = (uint64_t)nh * 128;                 // dense row: n_h heads x 128
  if (!c->qd) {
    // Per-call dense buffers, allocated once: the per-head K and V of the largest window are the
    // dense cache the latent layout avoids (B x rows x n_h x 128 x 2 bytes each).  All four or
    // none: a failed allocation leaves the cache as it was.
    void* p[5] = {nullptr, nullptr, nullptr, nullptr, nullptr};
    const char* names[5] = {"dense Q", "dense O", "dense K", "dense V", "dense split partials"};
    const size_t n_guards = c->guards.size();
    const size_t bytes[5] = {(size_t)cfg.batch * c->max_q_tokens * hd * 2,
                             (size_t)cfg.batch * c->max_q_tokens * hd * 2,
                             (size_t)cfg.batch * c->rows_per_stream * hd * 2,
                             (size_t)cfg.batch * c->rows_per_stream * hd * 2,
                             dense_ws_bytes(kDenseMaxSplits, cfg.batch, (int)c->max_q_tokens, nh)};
    for (int i = 0; i < 5; ++i) {
      if (bytes[i] == 0) continue;
      const cudaError_t e = alloc_buffer(c, &p[i], bytes[i], names[i], st);
      if (e != cudaSuccess) {
        for (int k = 0; k <= i; ++k) cudaFree(p[k]);
        c->guards.resize(n_guards);
        return fail(e == cudaErrorMemoryAllocation ? MLA_ERR_OUT_OF_MEMORY : MLA_ERR_CUDA,
                    "dense-form buffers: cudaMalloc of %zu bytes failed: %s", bytes[i],
                    cudaGetErrorString(e));
      }
    }
    c->qd = static_cast<__nv_bfloat16*>(p[0]);
    c->od = static_cast<__nv_bfloat16*>(p[1]);
    c->kd = static_cast<__nv_bfloat16*>(p[2]);
    c->vd = static_cast<__nv_bfloat16*>(p[3]);
    c->dws = p[4];
    c->dws_bytes = bytes[4];
  }
  const int64_t nq = (int64_t)n_frames * c->F;
  int64_t vs, vw;
  valid_counts(c, vs, vw);
  const int64_t base_row = c->sink_rows + vw * c->F;
  const int64_t n_keys = base_row + nq;
  mla_status s;

  // 1. the chunk's latents into the chunk tail (as the absorbed path does)
  if ((s = launch_latent_gemm(c, x_chunk, nq, nq, false, c->frames_appended, base_row, st)) != MLA_OK)
    return s;
  // 2. per-head queries [q_nope | RoPE3D(q_rope)] at the chunk's absolute positions
  {
    CUtensorMap ma, mo;
    if ((s = make_map(&ma, x_chunk, cfg.hidden, nq, cfg.batch, (uint64_t)cfg.hidden * 2,
                      (uint64_t)nq * cfg.hidden * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B)) != MLA_OK ||
        (s = make_out_map(&mo, c->qd, hd, nq, cfg.batch, hd * 2, hd * nq * 2, false)) != MLA_OK)
      return s;
    EpiArgs ep{};
    ep.n_cols = (int)hd;
    ep.rope_period = 128;
    ep.t0 = c->frames_appended;
    ep.tokens_per_frame = c->F;
    ep.frame_w = cfg.frame_w;
    ep.rope = c->rope;
    ep.rope_hw = c->rope_hw;
    ep.frame_h = cfg.frame_h;
    const mla::GemmTiles tiles{(int32_t)((nq + 127) / 128), (int32_t)((hd + kOutBN - 1) / kOutBN), cfg.batch};
    if ((s = launch_gemm<kOutBN, kOutAStages, kOutBStages, mla::kEpiDense, false>(
             ma, c->map_wqd, mo, mo, mo, (int)nq, cfg.hidden, 0, tiles, ep, c->status, c->num_sms,
             st, "dense query projection")) != MLA_OK)
      return s;
  }
  // 3. per-head keys and values of every key from the latent: K_h = [c W_UK[h]^T | k_rope],
  //    V_h = c W_UV[h]^T ([VideoMLA] §3.3)
  {
    CUtensorMap ma, mk, mv;
    if ((s = make_map(&ma, c->ckv, kLatent, n_keys, cfg.batch, kLatent * 2,
                      (uint64_t)c->rows_per_stream * kLatent * 2, 64, 128,
                      CU_TENSOR_MAP_SWIZZLE_128B, true)) != MLA_OK ||
        (s = make_out_map(&mk, c->kd, hd, n_keys, cfg.batch, hd * 2, hd * n_keys * 2, false)) != MLA_OK ||
        (s = make_out_map(&mv, c->vd, hd, n_keys, cfg.batch, hd * 2, hd * n_keys * 2, false)) != MLA_OK)
      return s;
    const int32_t m_tiles = (int32_t)((n_keys + 127) / 128);
    EpiArgs ek{};
    ek.n_cols = nh * dn;
    ek.head_in = dn;
    ek.head_out = 128;
    if ((s = launch_gemm<kOutBN, kOutAStages, kOutBStages, mla::kEpiDense, true>(
             ma, c->map_wukh, mk, mk, mk, (int)n_keys, kLatent, 0,
             mla::GemmTiles{m_tiles, (nh * dn + kOutBN - 1) / kOutBN, cfg.batch}, ek, c->status,
             c->num_sms, st, "key reconstruction")) != MLA_OK)
      return s;
    krope_broadcast_kernel<<<dim3((unsigned)n_keys, (unsigned)cfg.batch), 128, 0, st>>>(
        c->krope, c->rows_per_stream, c->kd, (int)n_keys, nh, dn,
        (int64_t)cfg.batch * c->rows_per_stream, c->status);
    if ((s = check_launch("k_rope broadcast")) != MLA_OK) return s;
    EpiArgs ev{};
    ev.n_cols = (int)hd;
    if ((s = launch_gemm<kOutBN, kOutAStages, kOutBStages, mla::kEpiDense, true>(
             ma, c->map_wuvh, mv, mv, mv, (int)n_keys, kLatent, 0,
             mla::GemmTiles{m_tiles, (int32_t)((hd + kOutBN - 1) / kOutBN), cfg.batch}, ev,
             c->status, c->num_sms, st, "value reconstruction")) != MLA_OK)
      return s;
  }
  // 4. dense per-head attention
  if ((s = launch_dense(c->qd, c->kd, c->vd, c->od, cfg.batch, (int)nq, (int)n_keys, nh,
                        c->softmax_scale, c->status, c->dws, c->dws_bytes, c->num_sms, st)) != MLA_OK)
    return s;
  // 5. out = concat_h(o_h) W_O^T
  {
    CUtensorMap ma, mo;
    if ((s = make_map(&ma, c->od, hd, nq, cfg.batch, hd * 2, hd * nq * 2, 64, 128,
                      CU_TENSOR_MAP_SWIZZLE_128B)) != MLA_OK ||
        (s = make_out_map(&mo, out, cfg.hidden, nq, cfg.batch, (uint64_t)cfg.hidden * 2,
                          (uint64_t)nq * cfg.hidden * 2, false)) != MLA_OK)
      return s;
    EpiArgs ep{};
    ep.n_cols = cfg.hidden;
    const mla::GemmTiles tiles{(int32_t)((nq + 127) / 128), (cfg.hidden + kOutBN - 1) / kOutBN, cfg.batch};
    s = launch_gemm<kOutBN, kOutAStages, kOutBStages, mla::kEpiStore, false>(
        ma, c->map_wo, mo, mo, mo, (int)nq, (int)hd, 0, tiles, ep, c->status, c->num_sms, st,
        "dense output projection");
    if (s == MLA_OK) set_pending(c, n_frames);
    return s;
  }
}

mla_status mla_cache_selftest_timeout(mla_cache* c, void* stream, int32_t* gave_up) {
  if (!c || !gave_up) return fail(MLA_ERR_INVALID_ARGUMENT, "NULL argument");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int* flag = c->status + 1;   // second word of the 256-byte status block
  MLA_CUDA(cudaMemsetAsync(flag, 0, sizeof(int), st));
  selftest_wait_kernel<<<1, 32, 0, st>>>(c->status, flag);
  mla_status s = check_launch("self-test wait");
  if (s != MLA_OK) return s;
  MLA_CUDA(cudaStreamSynchronize(st));
  int h = 0;
  MLA_CUDA(cudaMemcpy(&h, flag, sizeof(int), cudaMemcpyDeviceToHost));
  *gave_up = h;
  return MLA_OK;
}

mla_status mla_cache_selftest_bounds(mla_cache* c, void* stream, int32_t* caught) {
  if (!c || !caught) return fail(MLA_ERR_INVALID_ARGUMENT, "NULL argument");
#ifndef MLA_DEBUG
  return fail(MLA_ERR_UNSUPPORTED, "bounds checks exist only in the MLA_DEBUG build (libmla_debug.so)");
#else
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // Rows [last, last + 2) of every stream onto themselves: row `last` is the last row of the
  // planes (copied onto itself, a no-op), row last + 1 is past them and must be caught.
  const int64_t last = c->rows_per_stream - 1;
  const int64_t work = 2 * (kLatent / 8 + kRope / 8);
  move_rows_kernel<<<dim3((unsigned)((work + 255) / 256), (unsigned)c->cfg.batch), 256, 0, st>>>(
      c->ckv, c->krope, (int64_t)c->rows_per_stream, last, last, 2, c->status);
  mla_status s = check_launch("bounds self-test");
  if (s != MLA_OK) return s;
  MLA_CUDA(cudaStreamSynchronize(st));
  int word = 0;
  MLA_CUDA(cudaMemcpy(&word, c->status, sizeof(int), cudaMemcpyDeviceToHost));
  *caught = word == MLA_ERR_BOUNDS ? 1 : 0;
  return MLA_OK;
#endif
}

mla_status mla_dense_split_plan(int32_t batch, int32_t n_q, int32_t n_kv, int32_t n_heads,
                                int32_t num_sms, size_t workspace_bytes, int32_t* splits,
                                int32_t* kv_per_split) {
  if (!splits || !kv_per_split) return fail(MLA_ERR_INVALID_ARGUMENT, "NULL argument");
  if (batch < 1 || n_q < 1 || n_kv < 1 || n_heads < 1 || num_sms < 1)
    return fail(MLA_ERR_INVALID_ARGUMENT, "batch, n_q, n_kv, n_heads and num_sms must be >= 1");
  int s = 1, kvps = n_kv;
  dense_plan(batch, n_q, n_kv, n_heads, num_sms, workspace_bytes, &s, &kvps);
  *splits = s;
  *kv_per_split = kvps;
  return MLA_OK;
}

size_t mla_dense_workspace_bytes(int32_t batch, int32_t n_q, int32_t n_kv, int32_t n_heads) {
  if (batch < 1 || n_q < 1 || n_kv < 1 || n_heads < 1) return 0;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1)
    return 0;
  return dense_ws_bytes(dense_splits(batch, n_q, n_kv, n_heads, sms), batch, n_q, n_heads);
}

mla_status mla_dense_attention(const void* q, const void* k, const void* v, void* out,
                               int32_t batch, int32_t n_q, int32_t n_kv, int32_t n_heads,
                               int32_t d_head, float softmax_scale, void* workspace,
                               size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !out) return fail(MLA_ERR_INVALID_ARGUMENT, "NULL argument");
  if (batch < 1 || n_q < 1 || n_kv < 1 || n_heads < 1)
    return fail(MLA_ERR_INVALID_ARGUMENT, "batch, n_q, n_kv and n_heads must be >= 1");
  if (d_head != 128) return fail(MLA_ERR_UNSUPPORTED, "the dense kernel is built for d_head = 128");
  if (!(softmax_scale >= 0.f) || !std::isfinite(softmax_scale))
    return fail(MLA_ERR_INVALID_ARGUMENT, "softmax_scale must be finite and >= 0");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return fail(MLA_ERR_INVALID_ARGUMENT, "q, k, v and out must be 16-byte aligned");
  if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return fail(MLA_ERR_INVALID_ARGUMENT, "workspace must be 256-byte aligned");
  if (batch > 65535 || n_heads > 65535 || (int64_t)n_q * n_heads * 128 > ((int64_t)1 << 40))
    return fail(MLA_ERR_UNSUPPORTED, "problem too large for one launch");
  int* status = nullptr;
  mla_status s = dense_status_word(&status);
  if (s != MLA_OK) return s;
  const float scale = softmax_scale > 0.f ? softmax_scale : (float)(1.0 / std::sqrt(128.0));
  int dev = 0, sms = 0;
  MLA_CUDA(cudaGetDevice(&dev));
  MLA_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  return launch_dense(q, k, v, out, batch, n_q, n_kv, n_heads, scale, status,
                      workspace_bytes ? workspace : nullptr, workspace_bytes, sms,
                      reinterpret_cast<cudaStream_t>(stream));
}

mla_status mla_dense_sync(void* stream) {
  int* status = nullptr;
  mla_status s = dense_status_word(&status);
  if (s != MLA_OK) return s;
  MLA_CUDA(cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)));
  int word = 0;
  MLA_CUDA(cudaMemcpy(&word, status, sizeof(int), cudaMemcpyDeviceToHost));
  if (word != 0) return fail((mla_status)word, "the dense kernel recorded device status %d", word);
  return MLA_OK;
}

mla_status mla_cache_state(const mla_cache* c, int64_t* frames_appended, int32_t* valid) {
  if (!c) return fail(MLA_ERR_INVALID_ARGUMENT, "NULL cache");
  if (frames_appended) *frames_appended = c->frames_appended;
  if (valid) {
    int64_t vs, vw;
    valid_counts(c, vs, vw);
    *valid = (int32_t)(vs + vw);
  }
  return MLA_OK;
}

mla_status mla_cache_sync(mla_cache* c, void* stream) {
  if (!c) return fail(MLA_ERR_INVALID_ARGUMENT, "NULL cache");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  MLA_CUDA(cudaStreamSynchronize(st));
  int words[mla::kStatusRangeWord + 1] = {0};
  MLA_CUDA(cudaMemcpy(words, c->status, sizeof(words), cudaMemcpyDeviceToHost));
  if (words[0] != 0) return fail((mla_status)words[0], "a kernel recorded device status %d", words[0]);
  if (kGuardBytes) {
    // MLA_DEBUG build: no kernel may have written past the end of a buffer.
    std::vector<unsigned char> h(kGuardBytes);
    auto intact = [&](const unsigned char* g) {
      return cudaMemcpy(h.data(), g, kGuardBytes, cudaMemcpyDeviceToHost) == cudaSuccess &&
             std::all_of(h.begin(), h.end(), [](unsigned char b) { return b == kGuardByte; });
    };
    for (const auto& g : c->guards)
      if (!intact(g.p)) return fail(MLA_ERR_BOUNDS, "guard band after the %s was overwritten", g.name);
    if (const unsigned char* g = noalloc_guard())
      if (!intact(g)) return fail(MLA_ERR_BOUNDS, "guard band after the no-alloc scratch was overwritten");
  }
  if (words[mla::kStatusRangeWord] != 0) {
    // Reported once: clear the word so that the next sync covers the calls made after this one.
    MLA_CUDA(cudaMemsetAsync(c->status + mla::kStatusRangeWord, 0, sizeof(int), st));
    MLA_CUDA(cudaStreamSynchronize(st));
    return fail(MLA_ERR_RANGE, "a projected value exceeded the fp16 range and was clamped to "
                               "+-65504 (cache planes or absorbed queries) since the last sync");
  }
  return MLA_OK;
}

mla_status mla_cache_read(const mla_cache* c, int32_t b, void* ckv_host, void* krope_host,
                          int64_t* n_valid_rows) {
  if (!c) return fail(MLA_ERR_INVALID_ARGUMENT, "NULL cache");
  if (b < 0 || b >= c->cfg.batch) return fail(MLA_ERR_INVALID_ARGUMENT, "stream index out of range");
  const int64_t ring = c->sink_rows + (int64_t)c->cfg.window_frames * c->F;
  if (ckv_host)
    MLA_CUDA(cudaMemcpy(ckv_host, c->ckv + (int64_t)b * c->rows_per_stream * kLatent,
                        ring * kLatent * 2, cudaMemcpyDeviceToHost));
  if (krope_host)
    MLA_CUDA(cudaMemcpy(krope_host, c->krope + (int64_t)b * c->rows_per_stream * kRope,
                        ring * kRope * 2, cudaMemcpyDeviceToHost));
  if (n_valid_rows) {
    int64_t vs, vw;
    valid_counts(c, vs, vw);
    *n_valid_rows = (vs + vw) * c->F;
  }
  return MLA_OK;
}

mla_status mla_cache_debug_buffers(const mla_cache* c, mla_debug_buffers* out) {
  if (!c || !out) return fail(MLA_ERR_INVALID_ARGUMENT, "NULL argument");
  out->ckv = c->ckv;
  out->krope = c->krope;
  out->qp = c->qp;
  out->o_lat = c->o_lat;
  out->w_qcat = c->wqcat;
  out->w_ov = c->wov;
  out->rows_per_stream = c->rows_per_stream;
  return MLA_OK;
}

mla_status mla_cache_copy_buffer(const mla_cache* c, mla_buffer which, void* host_dst,
                                 size_t bytes, size_t* size) {
  if (!c) return fail(MLA_ERR_INVALID_ARGUMENT, "NULL cache");
  const mla_config& k = c->cfg;
  const size_t q_rows = (size_t)k.batch * c->max_q_tokens * k.n_heads;
  const void* src = nullptr;
  size_t total = 0;
  switch (which) {
    case MLA_BUFFER_QP: src = c->qp; total = q_rows * kQK * 2; break;
    case MLA_BUFFER_O_LAT: src = c->o_lat; total = q_rows * kLatent * 2; break;
    case MLA_BUFFER_W_QCAT: src = c->wqcat; total = (size_t)c->wq_rows * c->wq_cols * 2; break;
    case MLA_BUFFER_W_OV: src = c->wov; total = (size_t)k.hidden * k.n_heads * kLatent * 2; break;
    default: return fail(MLA_ERR_INVALID_ARGUMENT, "unknown buffer %d", (int)which);
  }
  if (size) *size = total;
  if (host_dst && bytes)
    MLA_CUDA(cudaMemcpy(host_dst, src, bytes < total ? bytes : total, cudaMemcpyDeviceToHost));
  return MLA_OK;
}

mla_status mla_cache_profile_enable(mla_cache* c, int32_t enable) {
  if (!c) return fail(MLA_ERR_INVALID_ARGUMENT, "NULL cache");
  c->profiling = enable != 0;
  return MLA_OK;
}

mla_status mla_cache_profile_read(mla_cache* c, mla_profile* out) {
  if (!c || !out) return fail(MLA_ERR_INVALID_ARGUMENT, "NULL argument");
  for (auto& r : c->pending) {
    MLA_CUDA(cudaEventSynchronize(r.b));
    float ms = 0.f;
    MLA_CUDA(cudaEventElapsedTime(&ms, r.a, r.b));
    c->prof_ms[r.kind] += ms;
    c->prof_n[r.kind] += 1;
    c->pool.push_back(r.a);
    c->pool.push_back(r.b);
  }
  c->pending.clear();
  for (int k = 0; k < MLA_KERNEL_COUNT; ++k) {
    out->ms[k] = c->prof_ms[k];
    out->launches[k] = c->prof_n[k];
    c->prof_ms[k] = 0;
    c->prof_n[k] = 0;
  }
  return MLA_OK;
}

}  // extern "C"
