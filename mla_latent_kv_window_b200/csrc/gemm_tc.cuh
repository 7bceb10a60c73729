// gemm_tc.cuh - tcgen05 GEMM for the projections of the latent-window attention path.
//
//   D[m, n] = sum_k A[z][m, k] * B[n, k]    (A: [batch][M][K], B: [N][K], K-major, both bf16 or
//                                            both fp16, fp32 accumulation)
// With a_kwrap > 0, A has only a_kwrap columns and column k of the product reads A's column
// k mod a_kwrap: D = A B_0^T + A B_1^T for B = [B_0 | B_1], the form of a weight carried as a
// bf16 pair hi + lo (two bf16 products per element, one fp32 accumulator).
//
// Persistent: one CTA per SM walks the tiles t = blockIdx.x, blockIdx.x + gridDim.x, ... of a
// (row tile, column block, batch) grid.  Each 128 x BN tile accumulates in fp32 tensor memory:
//   warp 0      TMA producer of A k-blocks (64 wide) into an A_STAGES-deep ring
//   warp 2      TMA producer of B k-blocks into a B_STAGES-deep ring
//   warp 1      TMEM allocator + single-thread tcgen05.mma issuer (M=128, N=BN, K=16 steps)
//   warps 3..10 epilogue, two warps per TMEM lane quarter: each thread converts one row of
//               the tile (256-row tiles: one 128-row sub-tile per warp of the pair; 128-row
//               tiles: half of the 32-column chunks each).  Per chunk: tcgen05.ld of the
//               accumulator (the next chunk is loaded while the current one is converted),
//               fused column transform, 16-bit pack into one of the warp's two 32 x 32 staging
//               boxes, then one TMA tensor store issued by lane 0 right away, so the TMA engine
//               writes a box while the warp converts the next chunk.  The boxes use the 64-byte
//               swizzle of the output tensor maps, which also makes the row-per-thread writes
//               bank-conflict free; rows past the end of the launch are clipped by the maps'
//               extents.
// The rings run continuously across tile boundaries.  With M_SUB = 1 the accumulator is
// double-buffered in TMEM (2 x 256 columns), so the epilogue of tile i overlaps the MMAs of
// tile i+1.  With M_SUB = 2 a tile is 256 rows: two M=128 accumulators (TMEM columns [0,256)
// and [256,512)) share every weight k-block, halving the weight bytes per row - the right
// trade when there are more tiles than SMs and the per-SM load path is the limit; the loads
// of tile i+1 still stream during the epilogue of tile i.
// A (activations, streamed once from HBM) and B (weights, shared by every CTA and L2-resident)
// have separate rings so that A can run ahead of the short-latency B loads; each tile starts
// its k-loop at a rotated block so concurrent CTAs do not all hit the same weight block.
// Launched with programmatic stream serialization, the prologue (barrier init, TMEM
// allocation, tensor-map prefetch) overlaps the previous kernel's tail; every global access
// comes after grid_dependency_wait().

// Output columns.  Column block y of a launch covers global columns col = b_row0 + y*BN + [0,BN),
// the same index that selects the rows of B.  Each 32-column chunk goes to one output map:
//   kEpiStore   map_o0 (bf16 out[z][m][col])                            (output projection)
//   kEpiLatent  col < latent_col0: one head's absorbed query
//               [W_UK^T q_nope | RoPE3D(q_rope)] * scale -> map_o0 = Qp[z][m][col] (fp16);
//               latent_col0 + [0,192) -> map_o1 = c_kv, latent_col0 + [192,224) -> RoPE3D ->
//               map_o2 = k_rope (fp16), at rows dst_row0 + m of the cache planes (the host
//               encodes the maps at the destination rows, so each launch writes one
//               contiguous row range per stream).  The latent path is 16-bit like the paper's
//               cache; fp16 keeps three more mantissa bits than bf16 for the same bytes.  A
//               value beyond the fp16 range is clamped to +-65504 and sets the status block's
//               range word (not fatal; mla_cache_sync reports it).
//   RoPE applies to the chunks with col mod 224 == 192 (every 224-column block is 192 + 32).
//   kEpiDense   bf16 to map_o0 at column (col / head_in) * head_out + col % head_in (identity
//               when head_in == 0), with RoPE on the chunks where col mod rope_period ==
//               rope_period - 32 (none when rope_period == 0): the per-head Q, K and V of the
//               reconstruct-then-dense form (head-interleaved [n_h][128] rows).
//
// The latent epilogue is the fused "append" of the VideoMLA paper page: c_kv = x W_DKV^T and
// the decoupled positional key k_R = RoPE3D(x W_KR^T) (§3.1, §3.2), one head-shared copy per
// token, stored in a fixed window of W latent frames (§1, App. D.4).
#pragma once

#include "ptx.cuh"

namespace mla {

constexpr int kEpiStore = 0;
constexpr int kEpiLatent = 1;
constexpr int kEpiDense = 2;
constexpr int kGemmThreads = 352;
constexpr int kEpiWarps = 8;       // two per TMEM lane quarter, each owning half of every row

// Rotary bands of the d_rope = 32 positional channels: pair p rotates by pos[axis[p]] * freq[p].
// Each frequency is carried as an unevaluated float sum hi + lo (|lo| <= ulp(hi) / 2), so that
// pos * freq is formed to about 2^-45 relative in fp32 arithmetic.
struct RopeBands {
  float freq_hi[16];
  float freq_lo[16];
  int axis[16];  // 0 = t, 1 = h, 2 = w
};

struct EpiArgs {
  int32_t n_cols;            // global columns < n_cols are stored; the rest of a block is padding
  int32_t latent_col0;       // kEpiLatent: first column of the latent block (a multiple of 224)
  int64_t t0;                // kEpiLatent: temporal index of row 0's frame
  int32_t tokens_per_frame;
  int32_t frame_w;
  float q_scale;             // softmax_scale * log2(e), applied to the query columns
  RopeBands rope;
  const float2* rope_hw;     // (cos, sin) tables: [16][frame_h] for h, then [16][frame_w] for w
  int32_t frame_h;
  int32_t head_in, head_out; // kEpiDense: output column remap (0: identity)
  int32_t rope_period;       // kEpiDense: RoPE on chunks with col % rope_period == rope_period - 32
};

template <int BN, int A_STAGES, int B_STAGES, int M_SUB = 1>
struct GemmSmem {
  static constexpr int kABytes = M_SUB * 128 * 64 * 2;
  static constexpr int kBBytes = BN * 64 * 2;
  static constexpr int kBOffset = A_STAGES * kABytes;
  static constexpr int kBSlots = B_STAGES ? B_STAGES : A_STAGES;   // B_STAGES == 0: shared ring
  static constexpr int kStagingOffset = kBOffset + kBSlots * kBBytes;   // 8 warps x 2 boxes of 2 KB
  static constexpr int kBarOffset = kStagingOffset + 8 * 2 * 2048;
  static constexpr int kBytes = kBarOffset + 512 + 1024;    // barriers + alignment slack
  static_assert(kABytes % 1024 == 0 && kBBytes % 1024 == 0, "stage atoms must stay 1 KB aligned");
  static_assert(BN % 32 == 0 && BN >= 32 && BN <= 256, "column blocks are whole 32-column chunks");
  static_assert(kBytes <= 232448, "GEMM tile does not fit in shared memory");
};

// Tile grid of one GEMM launch: row tiles (of 128 * M_SUB rows) x column blocks of BN x batch.
struct GemmTiles {
  int32_t m_tiles, n_blocks, batch;
  __host__ __device__ int32_t count() const { return m_tiles * n_blocks * batch; }
};

// RoPE factors of one token: f[p] = (cos, sin) of pos[axis[p]] * freq[p] for the 16 pairs.
// The h and w factors come from pair-major tables (computed in double on the host and rounded
// once): pair p of position h at tab_h[p * h_stride], of position w at tab_w[p * w_stride], so
// the 32 rows of a warp (consecutive tokens) read consecutive entries.  The t factors are formed here: the angle is p + e
// with p = fl(t * hi), e = (t * hi - p) + t * lo (exact product error by FMA), reduced to
// [-pi, pi] by Cody-Waite reduction with 2 pi split into two floats (accurate for integer t
// below 2^24), and evaluated with the hardware sine/cosine.  The table loads cost an L2 round
// trip (about a microsecond under a full HBM stream), so the epilogue calls this well before
// it needs the factors: the loads are issued here in program order, each register is written
// by exactly one of load or compute, and nothing waits for a load until rope_apply.
__device__ __forceinline__ void rope_factors(float2* f, int64_t t, const float2* tab_h,
                                             int h_stride, const float2* tab_w, int w_stride,
                                             const RopeBands& rb) {
  constexpr float kInv2Pi = 0.15915494309189535f;
  constexpr float kTwoPiHi = 6.28318548202514648f;       // fl(2 pi)
  constexpr float kTwoPiLo = -1.7484556000744e-07f;      // 2 pi - fl(2 pi)
#pragma unroll
  for (int p = 0; p < 16; ++p)
    if (rb.axis[p] != 0)
      f[p] = ld_nc_f2(rb.axis[p] == 2 ? tab_w + p * w_stride : tab_h + p * h_stride);
  const float tf = (float)t;
#pragma unroll
  for (int p = 0; p < 16; ++p) {
    if (rb.axis[p] == 0) {
      const float hi = rb.freq_hi[p];
      const float prod = tf * hi;
      const float err = fmaf(tf, hi, -prod) + tf * rb.freq_lo[p];
      const float k = rintf(prod * kInv2Pi);
      float r = fmaf(-k, kTwoPiHi, prod);
      r = fmaf(-k, kTwoPiLo, r) + err;
      __sincosf(r, &f[p].y, &f[p].x);
      pin_f2(f[p]);
    }
  }
}

// Row of a 128-row sub-tile held by TMEM lane quarter q, lane l (32x32b access shape).
__device__ __forceinline__ int row_in_sub(uint32_t q, uint32_t l) { return (int)(q * 32u + l); }

// Rotate the 16 (re, im) pairs of v by the factors f.
__device__ __forceinline__ void rope_apply(float* v, const float2* f) {
#pragma unroll
  for (int p = 0; p < 16; ++p) {
    const float a = v[2 * p], b = v[2 * p + 1];
    v[2 * p] = a * f[p].x - b * f[p].y;
    v[2 * p + 1] = a * f[p].y + b * f[p].x;
  }
}

template <int BN, int A_STAGES, int B_STAGES, int kEpi, bool kF16In, int M_SUB>
__global__ void __launch_bounds__(kGemmThreads, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap map_a,
                   const __grid_constant__ CUtensorMap map_b,
                   const __grid_constant__ CUtensorMap map_o0,
                   const __grid_constant__ CUtensorMap map_o1,
                   const __grid_constant__ CUtensorMap map_o2, int32_t M, int32_t K,
                   int32_t a_kwrap, int32_t b_row0, GemmTiles tiles, EpiArgs ep, int* status) {
  using L = GemmSmem<BN, A_STAGES, B_STAGES, M_SUB>;
  // B_STAGES == 0: one ring for A and B (one producer, one full/empty barrier pair per stage,
  // one wait and one commit per k-block); otherwise separate rings with their own producers.
  constexpr bool kShared = B_STAGES == 0;
  static_assert(M_SUB == 1 || M_SUB == 2, "tiles are 128 or 256 rows");
  constexpr int kAccBufs = M_SUB == 1 ? 2 : 1;   // accumulator buffers in 512 TMEM columns
  constexpr int kTileRows = 128 * M_SUB;
  static_assert(BN <= 256, "one accumulator buffer holds at most 256 columns");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* a_full = reinterpret_cast<uint64_t*>(smem + L::kBarOffset);
  uint64_t* a_empty = a_full + A_STAGES;
  uint64_t* b_full = a_empty + A_STAGES;
  uint64_t* b_empty = b_full + B_STAGES;
  uint64_t* acc_full = b_empty + B_STAGES;     // [2]
  uint64_t* acc_empty = acc_full + 2;          // [2]
  uint64_t* mma_quiesce = acc_empty + 2;       // all of this CTA's MMAs have completed
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mma_quiesce + 1);

  const uint32_t warp = warp_id();
  const uint32_t lane = lane_id();
  const int num_kb = K / 64;
  const int n_tiles = tiles.count();
  const int my_tiles = n_tiles > (int)blockIdx.x
                           ? (n_tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;

  if (threadIdx.x == 0) {
    grid_launch_dependents();
    for (int s = 0; s < A_STAGES; ++s) {
      mbar_init(&a_full[s], 1);
      mbar_init(&a_empty[s], 1);
    }
    for (int s = 0; s < B_STAGES; ++s) {
      mbar_init(&b_full[s], 1);
      mbar_init(&b_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&acc_full[s], 1);
      mbar_init(&acc_empty[s], kEpiWarps * 32);
    }
    mbar_init(mma_quiesce, 1);
    fence_mbar_init();
    tma_prefetch(&map_a);
    tma_prefetch(&map_b);
    tma_prefetch(&map_o0);
    if (kEpi == kEpiLatent) {
      tma_prefetch(&map_o1);
      tma_prefetch(&map_o2);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncwarp();      // reconverge single-lane branches: bar.sync must be warp-uniform
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  grid_dependency_wait();   // the previous kernel's outputs are visible from here on

  // Tile t -> (row tile, column block, batch); consecutive tiles share the column block.
  auto tile_coords = [&](int t, int& m0, int& y, int& z) {
    const int per_batch = tiles.m_tiles * tiles.n_blocks;
    z = t / per_batch;
    const int r = t - z * per_batch;
    y = r / tiles.m_tiles;
    m0 = (r - y * tiles.m_tiles) * kTileRows;
  };

  if (kShared && warp == 0) {
    // ------------------------------------------------------------------ TMA producer (shared ring)
    if (lane == 0) {
      const uint64_t pa = l2_policy_evict_first(), pb = l2_policy_evict_last();
      int g = 0;
      bool ok = true;
      for (int i = 0; i < my_tiles && ok; ++i) {
        int m0, y, z;
        tile_coords(blockIdx.x + i * gridDim.x, m0, y, z);
        const int rot = (int)((blockIdx.x + i * gridDim.x) * 7u % (unsigned)num_kb);
        for (int kb = 0; kb < num_kb; ++kb, ++g) {
          const int s = g % A_STAGES;
          if (!mbar_wait(&a_empty[s], ((uint32_t)(g / A_STAGES) & 1u) ^ 1u, status)) { ok = false; break; }
          const int kx = ((kb + rot) % num_kb) * 64;
          const int kxa = a_kwrap > 0 && kx >= a_kwrap ? kx - a_kwrap : kx;
          mbar_arrive_expect_tx(&a_full[s], L::kABytes + L::kBBytes);
          tma_load_3d_hint(smem + s * L::kABytes, &map_a, &a_full[s], kxa, m0, z, pa);
          tma_load_3d_hint(smem + L::kBOffset + s * L::kBBytes, &map_b, &a_full[s], kx,
                           b_row0 + y * BN, 0, pb);
        }
      }
      // Drain: never leave the CTA with a copy still landing in its shared memory (also when
      // the loop above stopped on an error).
      for (int q = g > A_STAGES ? g - A_STAGES : 0; q < g; ++q)
        mbar_wait_quiesce(&a_full[q % A_STAGES], (uint32_t)(q / A_STAGES) & 1u, status);
    }
  } else if (kShared && warp == 2) {
    // idle with a shared ring
  } else if (warp == 0 || warp == 2) {
    // ------------------------------------------------------------------ TMA producers
    if constexpr (!kShared) if (lane == 0) {
      const bool is_a = warp == 0;
      const int stages = is_a ? A_STAGES : B_STAGES;
      uint64_t* full = is_a ? a_full : b_full;
      uint64_t* empty = is_a ? a_empty : b_empty;
      const uint32_t bytes = is_a ? L::kABytes : L::kBBytes;
      const uint64_t policy = is_a ? l2_policy_evict_first() : l2_policy_evict_last();
      int g = 0;  // k-blocks issued so far (continuous across tiles)
      bool ok = true;
      for (int i = 0; i < my_tiles && ok; ++i) {
        int m0, y, z;
        tile_coords(blockIdx.x + i * gridDim.x, m0, y, z);
        const int rot = (int)((blockIdx.x + i * gridDim.x) * 7u % (unsigned)num_kb);
        for (int kb = 0; kb < num_kb; ++kb, ++g) {
          const int s = g % stages;
          if (!mbar_wait(&empty[s], ((uint32_t)(g / stages) & 1u) ^ 1u, status)) { ok = false; break; }
          const int kx = ((kb + rot) % num_kb) * 64;
          mbar_arrive_expect_tx(&full[s], bytes);
          if (is_a)
            tma_load_3d_hint(smem + s * L::kABytes, &map_a, &full[s],
                             a_kwrap > 0 && kx >= a_kwrap ? kx - a_kwrap : kx, m0, z, policy);
          else
            tma_load_3d_hint(smem + L::kBOffset + s * L::kBBytes, &map_b, &full[s], kx,
                             b_row0 + y * BN, 0, policy);
        }
      }
      // Drain: never leave the CTA with a copy still landing in its shared memory (also when
      // the loop above stopped on an error).
      for (int q = g > stages ? g - stages : 0; q < g; ++q)
        mbar_wait_quiesce(&full[q % stages], (uint32_t)(q / stages) & 1u, status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f32acc(128, BN, false, kF16In);
      int g = 0;
      bool ok = true;
      for (int i = 0; i < my_tiles && ok; ++i) {
        const int buf = i % kAccBufs;
        if (!mbar_wait(&acc_empty[buf], ((uint32_t)(i / kAccBufs) & 1u) ^ 1u, status)) break;
        tc_fence_after();
        const uint32_t acc = tmem + buf * 256;
        for (int kb = 0; kb < num_kb; ++kb, ++g) {
          const int sa = g % A_STAGES;
          const int sb = kShared ? sa : g % L::kBSlots;
          if (!mbar_wait(&a_full[sa], (uint32_t)(g / A_STAGES) & 1u, status) ||
              (!kShared && !mbar_wait(&b_full[sb], (uint32_t)(g / L::kBSlots) & 1u, status))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + sa * L::kABytes);
          const uint32_t b_addr = smem_u32(smem + L::kBOffset + sb * L::kBBytes);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint64_t db = smem_desc(b_addr + k * 32, 16, 1024, kSwizzle128B);
#pragma unroll
            for (int sub = 0; sub < M_SUB; ++sub) {   // rows 128*sub.. of the A box
              const uint64_t da = smem_desc(a_addr + sub * 16384 + k * 32, 16, 1024, kSwizzle128B);
              umma_ss(acc + sub * 256, da, db, idesc, (kb | k) != 0 ? 1u : 0u);
            }
          }
          tc_commit(&a_empty[sa]);
          if (!kShared) tc_commit(&b_empty[sb]);
        }
        tc_commit(&acc_full[buf]);
      }
      // Every MMA issued above has finished reading shared memory and writing TMEM before the
      // CTA may free either (also when the loop stopped on an error).
      tc_commit(mma_quiesce);
      mbar_wait_quiesce(mma_quiesce, 0, status);
    }
  } else {
    // ------------------------------------------------------------------ epilogue warps
    // Each thread converts one row of the tile: with 256-row tiles the two warps of a TMEM lane
    // quarter take one 128-row sub-tile each; with 128-row tiles they split the columns.
    const uint32_t sub_q = warp & 3u;          // TMEM lane quarter = rows 32*sub_q.. of a sub-tile
    const int pair = (int)(warp - 3) >> 2;     // which warp of the quarter's pair
    constexpr int kChunks = BN / 32;
    constexpr int kSplit = (kChunks + 1) / 2;
    constexpr int kMaxChunks = M_SUB == 2 ? kChunks : kSplit;   // chunks per warp and tile
    const int my_sub = M_SUB == 2 ? pair : 0;
    const int c_lo = M_SUB == 2 ? 0 : (pair ? kSplit : 0);
    const int c_hi = M_SUB == 2 ? kChunks : (pair ? kChunks : kSplit);
    // Two 2 KB staging boxes per warp (32 rows x 64 B); 16-byte unit u of row r sits at slot
    // u ^ ((r >> 1) & 3), the 64-byte swizzle of the output maps.  A box is rewritten only after
    // the tensor store issued from it two chunks earlier has read it.
    uint8_t* stage = smem + L::kStagingOffset + (warp - 3) * 2 * 2048;
    const uint32_t swz = (lane >> 1) & 3u;
    int issued = 0;                            // tensor stores issued by this warp (lane 0)
    float2 rf[16];                             // RoPE factors of this thread's row
    float amax = 0.f;                          // largest |value| this thread packed to fp16
    for (int i = 0; i < my_tiles; ++i) {
      const int buf = i % kAccBufs;
      int m0t, y, z;
      tile_coords(blockIdx.x + i * gridDim.x, m0t, y, z);
      const int col_base = b_row0 + y * BN;
      const int m = m0t + my_sub * 128 + row_in_sub(sub_q, lane);
      const int row0 = m0t + my_sub * 128 + (int)sub_q * 32;
      // The RoPE chunk of this warp's columns (at most one: one per 224 columns); its factors
      // are formed now, while the tile's MMAs still run.
      int rc = -1;
      if constexpr (kEpi == kEpiLatent || kEpi == kEpiDense) {
        const int rp = kEpi == kEpiLatent ? 224 : ep.rope_period;
        if (rp > 0)
          for (int c = c_lo; c < c_hi; ++c)
            if ((col_base + c * 32) % rp == rp - 32) rc = c;
        if (rc >= 0) {
          const int F = ep.tokens_per_frame;
          const int fi = m / F;                // frame within this launch
          const int k = m - fi * F;
          const int hh = k / ep.frame_w;
          rope_factors(rf, ep.t0 + fi, ep.rope_hw + hh, ep.frame_h,
                       ep.rope_hw + 16 * ep.frame_h + (k - hh * ep.frame_w), ep.frame_w, ep.rope);
        }
      }
      if (!mbar_wait_warp_sleepy(&acc_full[buf], (uint32_t)(i / kAccBufs) & 1u, status)) break;
      tc_fence_after();
      const uint32_t tbase = tmem + (buf + my_sub) * 256 + ((sub_q * 32u) << 16);
      // Chunk order: the RoPE chunk first, then the rest in order.
      auto chunk_at = [&](int cc) {
        if (rc < 0) return c_lo + cc;
        if (cc == 0) return rc;
        const int e = c_lo + cc - 1;
        return e >= rc ? e + 1 : e;
      };
      uint32_t r[2][32];
      if (c_lo < c_hi) tmem_ld32(tbase + chunk_at(0) * 32, r[0]);   // (BN = 32: one warp owns nothing)
#pragma unroll
      for (int cc = 0; cc < kMaxChunks; ++cc) {
        if (c_lo + cc >= c_hi) break;
        const int c = chunk_at(cc);
        uint32_t* cur = r[cc & 1];
        tmem_ld_wait();
        tmem_regs_ready(cur);
        if (c_lo + cc + 1 < c_hi) tmem_ld32(tbase + chunk_at(cc + 1) * 32, r[(cc + 1) & 1]);
        float v[32];
#pragma unroll
        for (int q = 0; q < 32; ++q) v[q] = __uint_as_float(cur[q]);
        const int col = col_base + c * 32;
        if constexpr (kEpi == kEpiDense) {
          if (c == rc) rope_apply(v, rf);
        }
        if constexpr (kEpi == kEpiLatent) {
          if (c == rc) rope_apply(v, rf);
          if (col < ep.latent_col0) {
#pragma unroll
            for (int q = 0; q < 32; ++q) v[q] *= ep.q_scale;
          }
#pragma unroll
          for (int q = 0; q < 32; ++q) amax = fmaxf(amax, fabsf(v[q]));
        }
        // Box issued % 2 is free once at most one later store is still reading.
        if (lane == 0) bulk_wait_read_1();
        __syncwarp();
        uint8_t* box_base = stage + (issued & 1) * 2048;
        uint4* box = reinterpret_cast<uint4*>(box_base + lane * 64);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          uint4 w;
          if constexpr (kEpi == kEpiLatent)
            w = make_uint4(pack_f16x2(v[8 * u + 0], v[8 * u + 1]), pack_f16x2(v[8 * u + 2], v[8 * u + 3]),
                           pack_f16x2(v[8 * u + 4], v[8 * u + 5]), pack_f16x2(v[8 * u + 6], v[8 * u + 7]));
          else
            w = make_uint4(pack_bf16x2(v[8 * u + 0], v[8 * u + 1]), pack_bf16x2(v[8 * u + 2], v[8 * u + 3]),
                           pack_bf16x2(v[8 * u + 4], v[8 * u + 5]), pack_bf16x2(v[8 * u + 6], v[8 * u + 7]));
          box[u ^ swz] = w;
        }
        fence_proxy_async_smem();   // staging writes -> visible to the TMA engine
        __syncwarp();
        if (col < ep.n_cols && row0 < M) {
          if (lane == 0) {
            if constexpr (kEpi == kEpiLatent) {
              const int j = col - ep.latent_col0;
              if (j < 0)
                tma_store_3d(&map_o0, box_base, col, row0, z);
              else if (j < 192)
                tma_store_3d(&map_o1, box_base, j, row0, z);
              else
                tma_store_3d(&map_o2, box_base, j - 192, row0, z);
            } else if constexpr (kEpi == kEpiDense) {
              const int x = ep.head_in ? (col / ep.head_in) * ep.head_out + col % ep.head_in : col;
              tma_store_3d(&map_o0, box_base, x, row0, z);
            } else {
              tma_store_3d(&map_o0, box_base, col, row0, z);
            }
            bulk_commit();
          }
          ++issued;
        }
      }
      // This thread has read all its accumulator columns of the tile.
      tc_fence_before();
      mbar_arrive(&acc_empty[buf]);
    }
    // fp16 packing saturates at +-65504 (cvt.satfinite): record that it happened.  Rows and
    // columns past the launch's extent hold zeros (the loads zero-fill), so every value counts.
    if constexpr (kEpi == kEpiLatent) {
      if (__any_sync(0xffffffffu, !(amax <= kF16Max)) && lane == 0)
        atomicOr(status + kStatusRangeWord, 1);
    }
    if (lane == 0) bulk_wait_all();
  }

  __syncwarp();      // reconverge single-lane roles before the CTA-wide barrier
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace mla
