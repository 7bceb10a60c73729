// query_proj.cuh - the query projection of an attention call as two chained tcgen05 products,
// with the chunk's own latents in the same launch (full-rank query, d_nope = 128).
//
// For head h and query token m (VideoMLA paper page, §3.3 with W_UK absorbed into the query):
//   q[m]      = W_Q[h] x[m]                        (128 channels, fp32 accumulation)
//   Qp[m, h]  = [W_UK[h]^T q[m] | RoPE3D(W_QR[h] x[m])] * scale * log2 e
// The absorbed weight W_UK[h]^T W_Q[h] is never formed: its single bf16 rounding perturbs
// every score by about 2^-10 relative, which a sharp softmax turns into visible output errors.
// Here both products multiply the caller's weights as given, and q enters the second product
// as an fp16 pair hi + lo (hi = fp16(q), lo = fp16(q - hi); about 22 significant bits), so q
// is carried essentially exactly.  The two products also cost less than the absorbed one:
// 1536 x (128 + 32) then 2 x 128 x 192 (the pair) multiply-adds per (token, head), against
// 1536 x 224 for one absorbed weight and twice that for it as a bf16 pair.
//
// Tiles: 256 rows (two M=128 halves sharing every weight k-block) x one column block of 160 B
// rows.  B = [W_Q[0]; W_QR[0]; ...; W_Q[n_h-1]; W_QR[n_h-1]; zero rows; W_DKV; W_KR] (bf16,
// K-major, W_DKV from row latent_row0): block y < n_h is head y (rows 160 y..); blocks n_h and
// n_h + 1 (rows latent_row0 + 160 (y - n_h)..) are the chunk's latents c_kv = x W_DKV^T and
// k_rope = RoPE3D(x W_KR^T) (the second block is 64 rows of weights and 96 rows past the end
// of B, which the tensor map reads as zeros).  Roles (352 threads):
//   warp 0      TMA producer: per tile, K/64 k-blocks of [x rows | B rows] into a 3-deep ring
//               of 52 KB stages; for a head tile one more stage holding W_UK[h] (fp16,
//               [128 q channels][192 latent channels], three 64-column 128B-swizzled boxes).
//   warp 1      TMEM allocator + single-thread MMA issuer.  First product: acc1 of half s at
//               TMEM columns [320 s, 320 s + 160).  Second product (head tiles): for each half,
//               once the epilogue has put q's hi/lo pair into TMEM columns [192, 320), 16
//               MMAs (M=128, N=192, K=16; A from TMEM, W_UK[h] read MN-major) into acc2 at
//               [320 s, 320 s + 192) - over acc1 of the same half, which has been read by then.
//   warps 3-10  epilogue; the warps 3-6 take half 0, 7-10 half 1 (one row per thread).  Head
//               tile: load acc1's RoPE chunk, convert q to the hi/lo pair into TMEM (half 1
//               first waits for the half-0 product, which frees the pair's columns), release
//               the second product, rotate and scale the RoPE chunk, then scale acc2 into Qp.
//               Latent tiles: c_kv and the rotated k_rope into the cache planes.  Every 32 x 32
//               output box is packed to fp16 in shared memory and written by one TMA store.
//   warp 2      idle.
// TMEM of a tile is reused by the next one only after the epilogue has released all of it;
// the ring keeps streaming the next tile's k-blocks meanwhile.
// A value beyond the fp16 range (a query channel, Qp, c_kv or k_rope) is clamped to +-65504
// and sets the status block's range word.
#pragma once

#include "gemm_tc.cuh"

namespace mla {

constexpr int kQpThreads = 352;
constexpr int kQpStages = 3;
constexpr int kQpBN = 160;          // B rows per column block: W_Q[h] (128) + W_QR[h] (32)
constexpr int kQpNope = 128;        // q channels per head (d_nope)

struct QpSmem {
  static constexpr int kABytes = 256 * 64 * 2;              // 32 KB: 256 rows x 64 bf16
  static constexpr int kBBytes = kQpBN * 64 * 2;            // 20 KB
  static constexpr int kStageBytes = kABytes + kBBytes;     // 52 KB
  static constexpr int kUkAtom = 128 * 64 * 2;              // 16 KB: 128 q rows x 64 fp16
  static constexpr int kStagingOffset = kQpStages * kStageBytes;
  static constexpr int kBarOffset = kStagingOffset + 8 * 2 * 2048;
  static constexpr int kBytes = kBarOffset + 256 + 1024;
  static_assert(3 * kUkAtom <= kStageBytes, "W_UK[h] must fit in one ring stage");
  static_assert(kStageBytes % 1024 == 0, "stages must stay 1 KB aligned");
  static_assert(kBytes <= 232448, "query projection does not fit in shared memory");
};

// TMEM columns: acc1 / acc2 of half s at 320 s; the q pair (hi [192, 256), lo [256, 320)).
constexpr uint32_t kQpAcc1 = 320;
constexpr uint32_t kQpPair = 192;

// Pack 32 fp32 values to fp16 into a 32 x 32 staging box (64-byte swizzle of the output maps)
// and store it with one TMA store at (col, row0, z).  Box `issued % 2` is reused only after
// the store issued from it two boxes earlier has read it.
__device__ __forceinline__ void qp_store_box(const float* v, uint8_t* stage, int& issued,
                                             const CUtensorMap* map, int col, int row0, int z,
                                             bool live, uint32_t lane) {
  if (lane == 0) bulk_wait_read_1();
  __syncwarp();
  uint8_t* box_base = stage + (issued & 1) * 2048;
  uint4* box = reinterpret_cast<uint4*>(box_base + lane * 64);
  const uint32_t swz = (lane >> 1) & 3u;
#pragma unroll
  for (int u = 0; u < 4; ++u)
    box[u ^ swz] = make_uint4(pack_f16x2(v[8 * u + 0], v[8 * u + 1]), pack_f16x2(v[8 * u + 2], v[8 * u + 3]),
                              pack_f16x2(v[8 * u + 4], v[8 * u + 5]), pack_f16x2(v[8 * u + 6], v[8 * u + 7]));
  fence_proxy_async_smem();
  __syncwarp();
  if (live) {
    if (lane == 0) {
      tma_store_3d(map, box_base, col, row0, z);
      bulk_commit();
    }
    ++issued;
  }
}

// Whole-warp wait on a phase that follows shortly (a chained step of this tile): every lane
// polls, so the warp resumes without a sleep back-off.  Bounded like mbar_wait; the warp
// agrees on the result.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, int* status) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, status));
}

__global__ void __launch_bounds__(kQpThreads, 1)
    query_proj_kernel(const __grid_constant__ CUtensorMap map_x,
                      const __grid_constant__ CUtensorMap map_w,
                      const __grid_constant__ CUtensorMap map_uk,
                      const __grid_constant__ CUtensorMap map_qp,
                      const __grid_constant__ CUtensorMap map_ckv,
                      const __grid_constant__ CUtensorMap map_krope, int32_t M, int32_t K,
                      int32_t n_heads, int32_t latent_row0, GemmTiles tiles, EpiArgs ep,
                      int* status) {
  using L = QpSmem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOffset);
  uint64_t* empty = full + kQpStages;
  uint64_t* acc1_full = empty + kQpStages;
  uint64_t* pair_full = acc1_full + 1;     // [2]: the half's q pair is in TMEM
  uint64_t* acc2_full = pair_full + 2;     // [2]: the half's second product has completed
  uint64_t* acc_empty = acc2_full + 2;     // the epilogue has released the tile's TMEM
  uint64_t* mma_quiesce = acc_empty + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mma_quiesce + 1);

  const uint32_t warp = warp_id();
  const uint32_t lane = lane_id();
  const int num_kb = K / 64;
  const int n_tiles = tiles.count();
  const int my_tiles = n_tiles > (int)blockIdx.x
                           ? (n_tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;

  if (threadIdx.x == 0) {
    grid_launch_dependents();
    for (int s = 0; s < kQpStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc1_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&pair_full[s], 128);
      mbar_init(&acc2_full[s], 1);
    }
    mbar_init(acc_empty, kEpiWarps * 32);
    mbar_init(mma_quiesce, 1);
    fence_mbar_init();
    tma_prefetch(&map_x);
    tma_prefetch(&map_w);
    tma_prefetch(&map_uk);
    tma_prefetch(&map_qp);
    tma_prefetch(&map_ckv);
    tma_prefetch(&map_krope);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncwarp();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  grid_dependency_wait();   // the previous kernel's outputs are visible from here on

  // Tile t -> (256-row tile, column block, batch); consecutive tiles share the column block.
  auto tile_coords = [&](int t, int& m0, int& y, int& z) {
    const int per_batch = tiles.m_tiles * tiles.n_blocks;
    z = t / per_batch;
    const int r = t - z * per_batch;
    y = r / tiles.m_tiles;
    m0 = (r - y * tiles.m_tiles) * 256;
  };

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t pa = l2_policy_evict_first(), pb = l2_policy_evict_last();
      int g = 0;
      bool ok = true;
      for (int i = 0; i < my_tiles && ok; ++i) {
        int m0, y, z;
        tile_coords(blockIdx.x + i * gridDim.x, m0, y, z);
        const int rot = (int)((blockIdx.x + i * gridDim.x) * 7u % (unsigned)num_kb);
        for (int kb = 0; kb < num_kb; ++kb, ++g) {
          const int s = g % kQpStages;
          if (!mbar_wait(&empty[s], ((uint32_t)(g / kQpStages) & 1u) ^ 1u, status)) { ok = false; break; }
          const int kx = ((kb + rot) % num_kb) * 64;
          uint8_t* stage = smem + s * L::kStageBytes;
          mbar_arrive_expect_tx(&full[s], L::kStageBytes);
          tma_load_3d_hint(stage, &map_x, &full[s], kx, m0, z, pa);
          const int b_row = y < n_heads ? y * kQpBN : latent_row0 + (y - n_heads) * kQpBN;
          tma_load_3d_hint(stage + L::kABytes, &map_w, &full[s], kx, b_row, 0, pb);
        }
        if (ok && y < n_heads) {
          // W_UK[h]: rows = the head's 128 q channels, columns = 192 latent channels.
          const int s = g % kQpStages;
          if (!mbar_wait(&empty[s], ((uint32_t)(g / kQpStages) & 1u) ^ 1u, status)) { ok = false; break; }
          uint8_t* stage = smem + s * L::kStageBytes;
          mbar_arrive_expect_tx(&full[s], 3 * L::kUkAtom);
          for (int a = 0; a < 3; ++a)
            tma_load_3d_hint(stage + a * L::kUkAtom, &map_uk, &full[s], a * 64, y * kQpNope, 0, pb);
          ++g;
        }
      }
      for (int q = g > kQpStages ? g - kQpStages : 0; q < g; ++q)
        mbar_wait_quiesce(&full[q % kQpStages], (uint32_t)(q / kQpStages) & 1u, status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc1 = idesc_f32acc(128, kQpBN, false, false);   // bf16, B K-major
      constexpr uint32_t idesc2 = idesc_f32acc(128, 192, true, true);       // fp16, B MN-major
      int g = 0, nq = 0;
      bool ok = true;
      for (int i = 0; i < my_tiles && ok; ++i) {
        int m0, y, z;
        tile_coords(blockIdx.x + i * gridDim.x, m0, y, z);
        if (!mbar_wait(acc_empty, ((uint32_t)i & 1u) ^ 1u, status)) break;
        tc_fence_after();
        for (int kb = 0; kb < num_kb; ++kb, ++g) {
          const int s = g % kQpStages;
          if (!mbar_wait(&full[s], (uint32_t)(g / kQpStages) & 1u, status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + s * L::kStageBytes);
          const uint32_t b_addr = a_addr + L::kABytes;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint64_t db = smem_desc(b_addr + k * 32, 16, 1024, kSwizzle128B);
#pragma unroll
            for (int sub = 0; sub < 2; ++sub) {
              const uint64_t da = smem_desc(a_addr + sub * 16384 + k * 32, 16, 1024, kSwizzle128B);
              umma_ss(tmem + sub * kQpAcc1, da, db, idesc1, (kb | k) != 0 ? 1u : 0u);
            }
          }
          tc_commit(&empty[s]);
        }
        if (!ok) break;
        tc_commit(acc1_full);
        if (y < n_heads) {
          const int s = g % kQpStages;
          if (!mbar_wait(&full[s], (uint32_t)(g / kQpStages) & 1u, status)) break;
          const uint32_t uk = smem_u32(smem + s * L::kStageBytes);
          for (int h = 0; h < 2 && ok; ++h) {
            if (!mbar_wait(&pair_full[h], (uint32_t)nq & 1u, status)) { ok = false; break; }
            tc_fence_after();
#pragma unroll
            for (int part = 0; part < 2; ++part) {      // hi, then lo
#pragma unroll
              for (int kk = 0; kk < 8; ++kk) {
                // 16 q channels per step = two 8-row core groups of 1 KB; the three 64-column
                // atoms of W_UK[h] are 16 KB apart (leading byte offset).
                const uint64_t db = smem_desc(uk + kk * 2048, L::kUkAtom, 1024, kSwizzle128B);
                umma_ts(tmem + h * kQpAcc1, tmem + kQpPair + part * 64 + kk * 8, db, idesc2,
                        (part | kk) != 0 ? 1u : 0u);
              }
            }
            tc_commit(&acc2_full[h]);
          }
          tc_commit(&empty[s]);
          ++g;
          ++nq;
        }
      }
      tc_commit(mma_quiesce);
      mbar_wait_quiesce(mma_quiesce, 0, status);
    }
  } else if (warp >= 3) {
    // ------------------------------------------------------------------ epilogue warps
    const uint32_t sub_q = warp & 3u;              // TMEM lane quarter
    const int half = (int)(warp - 3) >> 2;         // 128-row half of the tile
    const uint32_t lane_off = (sub_q * 32u) << 16;
    uint8_t* stage = smem + L::kStagingOffset + (warp - 3) * 2 * 2048;
    int issued = 0;
    int nq = 0;
    float2 rf[16];
    float amax = 0.f;
    for (int i = 0; i < my_tiles; ++i) {
      int m0t, y, z;
      tile_coords(blockIdx.x + i * gridDim.x, m0t, y, z);
      const int row0 = m0t + half * 128 + (int)sub_q * 32;   // first row of this warp's boxes
      const int m = row0 + (int)lane;
      const bool live = row0 < M;
      const bool head = y < n_heads;
      // The RoPE factors of this row (the head's q_rope chunk, or k_rope in block n_h + 1),
      // formed while the tile's MMAs run.
      if (head || y == n_heads + 1) {
        const int F = ep.tokens_per_frame;
        const int fi = m / F;
        const int k = m - fi * F;
        const int hh = k / ep.frame_w;
        rope_factors(rf, ep.t0 + fi, ep.rope_hw + hh, ep.frame_h,
                     ep.rope_hw + 16 * ep.frame_h + (k - hh * ep.frame_w), ep.frame_w, ep.rope);
      }
      if (!mbar_wait_warp_sleepy(acc1_full, (uint32_t)i & 1u, status)) break;
      tc_fence_after();
      const uint32_t acc = tmem + half * kQpAcc1 + lane_off;
      float v[32];
      uint32_t r[32];
      if (head) {
        // acc1 columns [128, 160): q_rope.  Read before the second product overwrites them.
        tmem_ld32(acc + 128, r);
        tmem_ld_wait();
        tmem_regs_ready(r);
        float vr[32];
#pragma unroll
        for (int q = 0; q < 32; ++q) vr[q] = __uint_as_float(r[q]);
        rope_apply(vr, rf);
#pragma unroll
        for (int q = 0; q < 32; ++q) {
          vr[q] *= ep.q_scale;
          amax = fmaxf(amax, fabsf(vr[q]));
        }
        if (half == 1) {
          // Store the RoPE chunk now; the pair's columns are free once the half-0 product is done.
          qp_store_box(vr, stage, issued, &map_qp, y * 224 + 192, row0, z, live, lane);
          if (!warp_wait(&acc2_full[0], (uint32_t)nq & 1u, status)) break;
          tc_fence_after();
        }
        // q channels -> fp16 pair (hi, lo) in TMEM columns [192, 256) and [256, 320).
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          tmem_ld32(acc + c * 32, r);
          tmem_ld_wait();
          tmem_regs_ready(r);
          uint32_t hi[16], lo[16];
#pragma unroll
          for (int p = 0; p < 16; ++p) {
            const float a = __uint_as_float(r[2 * p]), b = __uint_as_float(r[2 * p + 1]);
            amax = fmaxf(amax, fmaxf(fabsf(a), fabsf(b)));
            hi[p] = pack_f16x2(a, b);
            const float2 h = __half22float2(*reinterpret_cast<const __half2*>(&hi[p]));
            lo[p] = pack_f16x2(a - h.x, b - h.y);
          }
          tmem_st16(tmem + lane_off + kQpPair + c * 16, hi);
          tmem_st16(tmem + lane_off + kQpPair + 64 + c * 16, lo);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&pair_full[half]);
        if (half == 0) qp_store_box(vr, stage, issued, &map_qp, y * 224 + 192, row0, z, live, lane);
        // Qp latent part: acc2 = W_UK[h]^T q, scaled.
        if (!warp_wait(&acc2_full[half], (uint32_t)nq & 1u, status)) break;
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < 6; ++c) {
          tmem_ld32(acc + c * 32, r);
          tmem_ld_wait();
          tmem_regs_ready(r);
#pragma unroll
          for (int q = 0; q < 32; ++q) {
            v[q] = __uint_as_float(r[q]) * ep.q_scale;
            amax = fmaxf(amax, fabsf(v[q]));
          }
          qp_store_box(v, stage, issued, &map_qp, y * 224 + c * 32, row0, z, live, lane);
        }
        ++nq;
      } else {
        // Chunk latents: block n_h holds c_kv channels [0, 160); block n_h + 1 holds c_kv
        // [160, 192) and k_rope (its last three chunks are the zero rows past the weights).
        const int n_chunks = y == n_heads ? 5 : 2;
#pragma unroll 1
        for (int c = 0; c < n_chunks; ++c) {
          tmem_ld32(acc + c * 32, r);
          tmem_ld_wait();
          tmem_regs_ready(r);
#pragma unroll
          for (int q = 0; q < 32; ++q) v[q] = __uint_as_float(r[q]);
          const bool is_rope = y == n_heads + 1 && c == 1;
          if (is_rope) rope_apply(v, rf);
#pragma unroll
          for (int q = 0; q < 32; ++q) amax = fmaxf(amax, fabsf(v[q]));
          if (is_rope)
            qp_store_box(v, stage, issued, &map_krope, 0, row0, z, live, lane);
          else
            qp_store_box(v, stage, issued, &map_ckv, (y - n_heads) * 160 + c * 32, row0, z, live, lane);
        }
      }
      tc_fence_before();
      mbar_arrive(acc_empty);
    }
    // Rows past the launch's extent hold zeros (the loads zero-fill), so every value counts.
    if (__any_sync(0xffffffffu, !(amax <= kF16Max)) && lane == 0)
      atomicOr(status + kStatusRangeWord, 1);
    if (lane == 0) bulk_wait_all();
  }

  __syncwarp();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace mla
