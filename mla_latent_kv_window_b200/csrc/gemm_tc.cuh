// gemm_tc.cuh - tcgen05 GEMM for the projections of the latent-window attention path.
//
//   D[m, n] = sum_k A[z][m, k] * B[n, k]    (A: [batch][M][K], B: [N][K], K-major, both bf16 or
//                                            both fp16, fp32 accumulation)
//
// One CTA computes a 128 x BN tile with fp32 accumulation in tensor memory:
//   warp 0      TMA producer of A k-blocks (64 wide) into an A_STAGES-deep ring
//   warp 6      TMA producer of B k-blocks into a B_STAGES-deep ring
//   warp 1      TMEM allocator + single-thread tcgen05.mma issuer (M=128, N=BN, K=16 steps)
//   warps 2..5  epilogue: tcgen05.ld of the accumulator (one row per thread), fused row
//               transform, staged through shared memory for coalesced 16-byte row stores.
// A (hidden states, streamed once from HBM) and B (weights, shared by every CTA and
// L2-resident) have separate rings so that A can run far ahead of the short-latency B loads;
// each CTA starts its k-loop at a rotated block so the CTAs do not all hit the same weight
// block at once.
//
// Epilogues (kEpi):
//   kEpiStore   bf16 store of the tile into out[z][m][n]                (output projection)
//   kEpiLatent  columns 0..191 -> c_kv, 192..223 -> RoPE3D -> k_rope, written as fp16 to ring
//               slots (t mod W)*F + k, or to the chunk tail; for blockIdx.y below latent_y the
//               tile is one head's absorbed query [W_UK^T q_nope | RoPE3D(q_rope)] * scale ->
//               Qp (fp16).  The latent path is 16-bit like the paper's cache; fp16 keeps three
//               more mantissa bits than bf16 for the same bytes.
//
// The latent epilogue is the fused "append" of the VideoMLA paper page: c_kv = x W_DKV^T and
// the decoupled positional key k_R = RoPE3D(x W_KR^T) (§3.1, §3.2), one head-shared copy per
// token, stored in a fixed window of W latent frames (§1, App. D.4).
#pragma once

#include "ptx.cuh"

namespace mla {

constexpr int kEpiStore = 0;
constexpr int kEpiLatent = 1;
constexpr int kGemmThreads = 224;

// Rotary bands of the d_rope = 32 positional channels: pair p rotates by pos[axis[p]] * freq[p].
struct RopeBands {
  double freq[16];
  int axis[16];  // 0 = t, 1 = h, 2 = w
};

struct EpiArgs {
  // kEpiStore
  __nv_bfloat16* out;
  int64_t out_batch_stride;  // elements
  int32_t ld_out;            // elements per output row
  // kEpiLatent
  __half* ckv;               // [batch][rows_per_stream][192] fp16
  __half* krope;             // [batch][rows_per_stream][32]  fp16
  int64_t rows_per_stream;
  __half* qp;                // [batch][qp_rows_per_stream][224] fp16
  int64_t qp_rows_per_stream;
  int32_t latent_y;          // blockIdx.y >= latent_y -> latent tile, else query head blockIdx.y
  int32_t n_heads;
  int32_t ring_mode;         // 1: slot (t mod W)*F + k; 0: chunk tail row base_row + m
  int64_t t0;                // temporal index of row 0's frame
  int32_t window_frames;
  int32_t tokens_per_frame;
  int32_t frame_w;
  int64_t base_row;
  float q_scale;             // softmax_scale * log2(e)
  RopeBands rope;
};

template <int BN, int A_STAGES, int B_STAGES>
struct GemmSmem {
  static constexpr int kABytes = 128 * 64 * 2;
  static constexpr int kBBytes = BN * 64 * 2;
  static constexpr int kBOffset = A_STAGES * kABytes;
  static constexpr int kBarOffset = kBOffset + B_STAGES * kBBytes;
  static constexpr int kBytes = kBarOffset + 512 + 1024;  // barriers + alignment slack
  static_assert(kABytes % 1024 == 0 && kBBytes % 1024 == 0, "stage atoms must stay 1 KB aligned");
  static_assert(kBarOffset >= 128 * (BN * 2 + 16), "staging must fit in the rings");
  static_assert(kBytes <= 232448, "GEMM tile does not fit in shared memory");
};

__device__ __forceinline__ void rope_rotate32(float* v, int64_t t, int h, int w,
                                              const RopeBands& rb) {
#pragma unroll
  for (int p = 0; p < 16; ++p) {
    const int ax = rb.axis[p];
    const double pos = ax == 0 ? (double)t : (ax == 1 ? (double)h : (double)w);
    double ang = pos * rb.freq[p];
    ang -= 6.283185307179586 * rint(ang * 0.15915494309189535);  // reduce to [-pi, pi]
    float s, c;
    __sincosf((float)ang, &s, &c);
    const float a = v[2 * p], b = v[2 * p + 1];
    v[2 * p] = a * c - b * s;
    v[2 * p + 1] = a * s + b * c;
  }
}

template <int BN, int A_STAGES, int B_STAGES, int kEpi, bool kF16In>
__global__ void __launch_bounds__(kGemmThreads, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap map_a,
                   const __grid_constant__ CUtensorMap map_b, int32_t M, int32_t K,
                   int32_t b_row0, EpiArgs ep, int* status) {
  using L = GemmSmem<BN, A_STAGES, B_STAGES>;
  static_assert(kEpi != kEpiLatent || BN == 224, "the latent epilogue owns 192 + 32 columns");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* a_full = reinterpret_cast<uint64_t*>(smem + L::kBarOffset);
  uint64_t* a_empty = a_full + A_STAGES;
  uint64_t* b_full = a_empty + A_STAGES;
  uint64_t* b_empty = b_full + B_STAGES;
  uint64_t* acc_full = b_empty + B_STAGES;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(acc_full + 1);

  const uint32_t warp = warp_id();
  const uint32_t lane = lane_id();
  const int m0 = blockIdx.x * 128;
  const int y = blockIdx.y;
  const int z = blockIdx.z;
  const int num_kb = K / 64;
  const int kb_rot = (int)((blockIdx.x * 7u + blockIdx.y * 3u + blockIdx.z) % (unsigned)num_kb);
  constexpr uint32_t kTmemCols = BN <= 128 ? 128 : 256;

  if (threadIdx.x == 0) {
    for (int s = 0; s < A_STAGES; ++s) {
      mbar_init(&a_full[s], 1);
      mbar_init(&a_empty[s], 1);
    }
    for (int s = 0; s < B_STAGES; ++s) {
      mbar_init(&b_full[s], 1);
      mbar_init(&b_empty[s], 1);
    }
    mbar_init(acc_full, 1);
    fence_mbar_init();
    tma_prefetch(&map_a);
    tma_prefetch(&map_b);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0 || warp == 6) {
    // ------------------------------------------------------------------ TMA producers
    if (lane == 0) {
      const bool is_a = warp == 0;
      const int stages = is_a ? A_STAGES : B_STAGES;
      uint64_t* full = is_a ? a_full : b_full;
      uint64_t* empty = is_a ? a_empty : b_empty;
      const uint32_t bytes = is_a ? L::kABytes : L::kBBytes;
      const uint64_t policy = is_a ? l2_policy_evict_first() : l2_policy_evict_last();
      int issued = 0;
      for (int kb = 0; kb < num_kb; ++kb) {
        const int s = kb % stages;
        if (!mbar_wait(&empty[s], ((uint32_t)(kb / stages) & 1u) ^ 1u, status)) break;
        const int kx = ((kb + kb_rot) % num_kb) * 64;
        mbar_arrive_expect_tx(&full[s], bytes);
        if (is_a)
          tma_load_3d_hint(smem + s * L::kABytes, &map_a, &full[s], kx, m0, z, policy);
        else
          tma_load_3d_hint(smem + L::kBOffset + s * L::kBBytes, &map_b, &full[s], kx,
                           b_row0 + y * BN, 0, policy);
        issued = kb + 1;
      }
      // Drain: never leave the CTA with a copy still landing in its shared memory.
      for (int kb = issued > stages ? issued - stages : 0; kb < issued; ++kb)
        mbar_wait(&full[kb % stages], (uint32_t)(kb / stages) & 1u, status);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f32acc(128, BN, false, kF16In);
      for (int kb = 0; kb < num_kb; ++kb) {
        const int sa = kb % A_STAGES;
        const int sb = kb % B_STAGES;
        if (!mbar_wait(&a_full[sa], (uint32_t)(kb / A_STAGES) & 1u, status)) break;
        if (!mbar_wait(&b_full[sb], (uint32_t)(kb / B_STAGES) & 1u, status)) break;
        tc_fence_after();
        const uint32_t a_addr = smem_u32(smem + sa * L::kABytes);
        const uint32_t b_addr = smem_u32(smem + L::kBOffset + sb * L::kBBytes);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint64_t da = smem_desc(a_addr + k * 32, 16, 1024, kSwizzle128B);
          const uint64_t db = smem_desc(b_addr + k * 32, 16, 1024, kSwizzle128B);
          umma_ss(tmem, da, db, idesc, (kb | k) != 0 ? 1u : 0u);
        }
        tc_commit(&a_empty[sa]);
        tc_commit(&b_empty[sb]);
      }
      tc_commit(acc_full);
    }
  } else {
    // ------------------------------------------------------------------ epilogue warps
    const uint32_t sub = warp & 3u;            // TMEM lane quarter this warp may access
    const int row = sub * 32 + lane;           // tile row owned by this thread
    const int m = m0 + row;
    const bool ok = mbar_wait(acc_full, 0, status);
    tc_fence_after();
    constexpr int kStageStride = BN * 2 + 16;  // bytes per staged row (bank-conflict padding)
    uint8_t* stage_row = smem + row * kStageStride;
    const uint32_t tbase = tmem + ((sub * 32u) << 16);

    // Row geometry for the latent / query epilogue.
    bool latent = false;
    int64_t t = 0;
    int hh = 0, ww = 0;
    if constexpr (kEpi == kEpiLatent) {
      latent = y >= ep.latent_y;
      const int F = ep.tokens_per_frame;
      t = ep.t0 + m / F;
      const int k = m % F;
      hh = k / ep.frame_w;
      ww = k % ep.frame_w;
    }
    if (ok) {
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tbase + c * 32, r);
        tmem_ld_wait();
        float v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
        if constexpr (kEpi == kEpiLatent) {
          if (c == 6) rope_rotate32(v, t, hh, ww, ep.rope);   // columns 192..223
          if (!latent) {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] *= ep.q_scale;
          }
        }
        uint4* dst = reinterpret_cast<uint4*>(stage_row + c * 64);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if constexpr (kEpi == kEpiLatent) {
            dst[q] = make_uint4(pack_f16x2(v[8 * q + 0], v[8 * q + 1]),
                                pack_f16x2(v[8 * q + 2], v[8 * q + 3]),
                                pack_f16x2(v[8 * q + 4], v[8 * q + 5]),
                                pack_f16x2(v[8 * q + 6], v[8 * q + 7]));
          } else {
            dst[q] = make_uint4(pack_bf16x2(v[8 * q + 0], v[8 * q + 1]),
                                pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
                                pack_bf16x2(v[8 * q + 4], v[8 * q + 5]),
                                pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
          }
        }
      }
    }
    tc_fence_before();
    __syncwarp();
    // Coalesced copy-out: the warp walks its own 32 rows, one 16-byte chunk per lane.
    if (ok) {
      constexpr int kChunks = BN / 8;  // 16-byte chunks per row
      for (int rr = 0; rr < 32; ++rr) {
        const int trow = sub * 32 + rr;
        const int gm = m0 + trow;
        if (gm >= M) break;
        const uint4* src = reinterpret_cast<const uint4*>(smem + trow * kStageStride);
        if constexpr (kEpi == kEpiStore) {
          __nv_bfloat16* o = ep.out + z * ep.out_batch_stride + (int64_t)gm * ep.ld_out + y * BN;
          for (int q = lane; q < kChunks; q += 32) reinterpret_cast<uint4*>(o)[q] = src[q];
        } else {
          if (latent) {
            int64_t dst_row;
            if (ep.ring_mode) {
              const int F = ep.tokens_per_frame;
              const int64_t f = ep.t0 + gm / F;
              dst_row = (f % ep.window_frames) * F + gm % F;
            } else {
              dst_row = ep.base_row + gm;
            }
            dst_row += z * ep.rows_per_stream;
            if (lane < 24) {
              reinterpret_cast<uint4*>(ep.ckv + dst_row * 192)[lane] = src[lane];
            } else if (lane < 28) {
              reinterpret_cast<uint4*>(ep.krope + dst_row * 32)[lane - 24] = src[lane];
            }
          } else {
            const int64_t qrow = z * ep.qp_rows_per_stream + (int64_t)gm * ep.n_heads + y;
            if (lane < 28) reinterpret_cast<uint4*>(ep.qp + qrow * 224)[lane] = src[lane];
          }
        }
      }
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace mla
