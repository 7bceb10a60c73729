// window_attn.cuh - latent-window attention on tcgen05 (sm_100a).
//
// Rows r = (query token, head) of the absorbed, rotated, pre-scaled queries Qp[r] (224 =
// 192 latent + 32 RoPE channels) attend to every key j of the window plus the chunk.  Qp, the
// latent cache, P and o_lat are fp16 (16-bit like the paper's bf16/fp16 cache; fp16 keeps three
// more mantissa bits); every MMA accumulates in fp32:
//
//   s_j = Qp[r] . [c_kv_j | k_rope_j]          (log2-domain scores: Qp carries scale*log2 e)
//   o_lat[r] = sum_j 2^(s_j - m) c_kv_j / sum_j 2^(s_j - m)
//
// This is the W_UK-absorbed form of the VideoMLA paper page's §3.3 attention: per-head keys
// k_h = [c W_UK[h]^T | k_R] and values v_h = c W_UV[h]^T are never built; all heads read the
// same head-shared latent tile, which makes the contraction an MQA-shaped dense GEMM.
//
// One CTA owns 128 rows.  Shared-memory bandwidth is the scarce resource here (the MMAs, the
// TMA writes and the softmax all share it), so both MMAs take their A operand from tensor
// memory and shared memory only holds the streamed key tiles:
//   warp 0      TMA producer: 128-key tiles of c_kv (3 x 64-column 128B-swizzled boxes) and
//               k_rope (one 32-column 64B-swizzled box) into a KV_STAGES-deep ring, starting at
//               a CTA-dependent tile.  Keys past n_keys are zero-filled by the tensor map.
//   warp 1      TMEM allocator + issuer of S_j = Q K_j^T  (M=128 N=128 K=224, 14 k-steps; Q
//               from TMEM, K_j K-major).  S_{j+1} is issued as soon as the softmax has copied
//               S_j to registers, so it runs while the softmax works on tile j.
//   warp 6      issuer of O += P_j C_j  (M=128 N=192 K=128, 8 k-steps; P_j from TMEM, C_j is the
//               SAME smem tile as K_j, read MN-major).  Two issuing threads keep the tensor
//               pipe fed: neither stream waits behind the other's barrier checks.
//   warps 2..5  first load this CTA's Qp rows into TMEM (one row per thread), then softmax:
//               one row per thread, running max with lazy rescaling (O is rescaled in TMEM
//               only when the max grows by > 2^8), ex2, P_j as fp16 into TMEM; finally O / l ->
//               fp16 o_lat, staged in shared memory and written by one bulk copy per row.
//
// TMEM columns: S [0,128), P [128,192), Q [192,304), O [304,496), QS [496,512).
//
// Sink keys ([VideoMLA] App. D.4/D.5 "sink + local window"): the first sink_tiles key tiles
// hold the sink frames (rows past sink_keys are padding and are masked).  Their k_rope was
// rotated at the sink frame's absolute index, which is also its window-local one, while Qp
// was rotated at the query's absolute index; so for sink tiles the two RoPE k-steps of S take
// QS, the query's RoPE part turned by the temporal offset between the two (sink_rot).
// Launched with programmatic stream serialization: barrier init, TMEM allocation and the
// tensor-map prefetch overlap the projection kernel's tail; griddepcontrol.wait precedes the first
// global access.
#pragma once

#include "ptx.cuh"

namespace mla {

constexpr int kAttnThreads = 224;
constexpr int kTileKeys = 128;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: lazy O rescale when max grows > 2^8

template <int KV_STAGES>
struct AttnSmem {
  static constexpr int kAtomC = 128 * 128;           // 128 keys x 64 fp16 (SW128)
  static constexpr int kAtomR = 128 * 64;            // 128 keys x 32 fp16 (SW64)
  static constexpr int kTileBytes = 3 * kAtomC + kAtomR;   // 57344: one key tile
  static constexpr int kKV = 0;
  static constexpr int kBar = kKV + KV_STAGES * kTileBytes;
  static constexpr int kBytes = kBar + 256 + 1024;
  static constexpr int kStageStride = 400;           // o_lat staging row: 384 B + 16 padding
  static_assert(kBytes <= 232448, "attention tile does not fit in shared memory");
  static_assert(128 * kStageStride <= kTileBytes, "o_lat staging must fit in one KV stage");
};

// TMEM column map (512 allocated).
constexpr uint32_t kTmemS = 0;
constexpr uint32_t kTmemP = 128;
constexpr uint32_t kTmemQ = 192;
constexpr uint32_t kTmemO = 304;
constexpr uint32_t kTmemQS = 496;   // RoPE part of Q turned for the sink keys (2 k-steps)

struct AttnArgs {
  const __half* qp;            // [batch][qp_rows][224] fp16
  int64_t qp_batch_stride;     // elements
  int32_t rows;                // R = n_q * n_heads valid rows per stream
  int32_t n_keys;              // keys per stream (window + chunk)
  __half* o_lat;               // fp16
  int64_t o_lat_batch_stride;  // elements
  int32_t sink_tiles;          // leading key tiles that hold sink frames (0: no sink)
  int32_t sink_keys;           // valid sink keys; keys [sink_keys, 128 * sink_tiles) are padding
  float2 sink_rot[16];         // (cos, sin) turning each RoPE pair of Q for the sink keys
  int64_t qp_rows_cap;         // rows each stream's Qp and o_lat buffers hold (bounds checks)
  int32_t batch;               // streams the buffers hold (bounds checks)
};

template <int KV_STAGES>
__global__ void __launch_bounds__(kAttnThreads, 1)
    window_attn_kernel(const __grid_constant__ CUtensorMap map_kc,
                       const __grid_constant__ CUtensorMap map_kr, AttnArgs args, int* status) {
  using L = AttnSmem<KV_STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* q_ready = bars;
  uint64_t* kv_full = bars + 1;                  // [KV_STAGES]
  uint64_t* kv_empty = kv_full + KV_STAGES;      // [KV_STAGES]
  uint64_t* s_full = kv_empty + KV_STAGES;
  uint64_t* s_free = s_full + 1;
  uint64_t* p_full = s_free + 1;
  uint64_t* pv_done = p_full + 1;
  uint64_t* quiesce_s = pv_done + 1;             // all S MMAs of this CTA have completed
  uint64_t* quiesce_pv = quiesce_s + 1;          // all PV MMAs of this CTA have completed
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(quiesce_pv + 1);

  const uint32_t warp = warp_id();
  const uint32_t lane = lane_id();
  const int m0 = blockIdx.x * 128;
  const int z = blockIdx.y;
  const int n_keys = args.n_keys;
  const int nt = (n_keys + kTileKeys - 1) / kTileKeys;
  // Every CTA walks all key tiles, each from its own starting tile: CTAs that stream the same
  // tiles in lockstep pile onto the same L2 lines (softmax does not depend on key order).
  const int rot = (int)(((unsigned)blockIdx.x * 37u + (unsigned)blockIdx.y * 11u) % (unsigned)nt);

  if (threadIdx.x == 0) {
    grid_launch_dependents();
    mbar_init(q_ready, 128);
    for (int s = 0; s < KV_STAGES; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, 128);
    mbar_init(p_full, 128);
    mbar_init(pv_done, 1);
    mbar_init(quiesce_s, 1);
    mbar_init(quiesce_pv, 1);
    fence_mbar_init();
    tma_prefetch(&map_kc);
    tma_prefetch(&map_kr);
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
  grid_dependency_wait();   // the projection's Qp and chunk latents are visible from here on

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t keep = l2_policy_evict_last();    // keys are re-read by every row tile
      int issued = 0;
      for (int j = 0; j < nt; ++j) {
        const int st = j % KV_STAGES;
        const uint32_t round = j / KV_STAGES;
        if (!mbar_wait(&kv_empty[st], (round & 1u) ^ 1u, status)) break;
        uint8_t* kv = smem + L::kKV + st * L::kTileBytes;
        mbar_arrive_expect_tx(&kv_full[st], L::kTileBytes);
        const int key0 = ((j + rot) % nt) * kTileKeys;
        for (int a = 0; a < 3; ++a)
          tma_load_3d_hint(kv + a * L::kAtomC, &map_kc, &kv_full[st], a * 64, key0, z, keep);
        tma_load_3d_hint(kv + 3 * L::kAtomC, &map_kr, &kv_full[st], 0, key0, z, keep);
        issued = j + 1;
      }
      // Drain: never leave the CTA with a copy still landing in its shared memory (also when
      // the loop above stopped on an error).
      for (int j = issued > KV_STAGES ? issued - KV_STAGES : 0; j < issued; ++j)
        mbar_wait_quiesce(&kv_full[j % KV_STAGES], (uint32_t)(j / KV_STAGES) & 1u, status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ S issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_f32acc(128, kTileKeys, false, true);
      bool ok = mbar_wait(q_ready, 0, status);
      for (int j = 0; ok && j < nt; ++j) {
        const int st = j % KV_STAGES;
        if (!mbar_wait(&kv_full[st], (uint32_t)(j / KV_STAGES) & 1u, status)) break;
        // S is single-buffered: the softmax must have copied S_{j-1} to registers.
        if (j >= 1 && !mbar_wait(s_free, (uint32_t)(j - 1) & 1u, status)) break;
        tc_fence_after();
        const uint32_t kv_base = smem_u32(smem + L::kKV + st * L::kTileBytes);
        const bool sink_tile = (j + rot) % nt < args.sink_tiles;
#pragma unroll
        for (int kk = 0; kk < 14; ++kk) {
          // A = Q from TMEM: 16 fp16 of K per step = 8 packed columns.
          uint64_t db;
          uint32_t qa = tmem + kTmemQ + kk * 8;
          if (kk < 12) {
            db = smem_desc(kv_base + (kk >> 2) * L::kAtomC + (kk & 3) * 32, 16, 1024,
                           kSwizzle128B);
          } else {
            db = smem_desc(kv_base + 3 * L::kAtomC + (kk - 12) * 32, 16, 512, kSwizzle64B);
            if (sink_tile) qa = tmem + kTmemQS + (kk - 12) * 8;
          }
          umma_ts(tmem + kTmemS, qa, db, idesc_s, kk > 0 ? 1u : 0u);
        }
        tc_commit(s_full);
      }
      // The CTA frees shared and tensor memory only after every issued MMA has completed.
      tc_commit(quiesce_s);
      mbar_wait_quiesce(quiesce_s, 0, status);
    }
  } else if (warp == 6) {
    // ------------------------------------------------------------------ PV issuer
    // A second issuing thread, so that the S and PV streams each wait only for their own
    // inputs and the tensor pipe always has queued work.  tcgen05.commit tracks the MMAs of
    // the committing thread; a key stage is released after PV_j, which (through P_j) follows
    // S_j on the same stage.
    if (lane == 0) {
      constexpr uint32_t idesc_o = idesc_f32acc(128, 192, true, true);
      for (int j = 0; j < nt; ++j) {
        const int st = j % KV_STAGES;
        if (!mbar_wait(p_full, (uint32_t)j & 1u, status)) break;
        tc_fence_after();
        const uint32_t c_base = smem_u32(smem + L::kKV + st * L::kTileBytes);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          // C_j read MN-major: 16 keys per step = two 8-row core groups of 1 KB; the three
          // 64-column atoms are 16 KB apart (leading byte offset).
          const uint64_t db = smem_desc(c_base + kk * 2048, L::kAtomC, 1024, kSwizzle128B);
          umma_ts(tmem + kTmemO, tmem + kTmemP + kk * 8, db, idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(pv_done);
        tc_commit(&kv_empty[st]);
      }
      tc_commit(quiesce_pv);
      mbar_wait_quiesce(quiesce_pv, 0, status);
    }
  } else {
    // ------------------------------------------------------------------ softmax warps
    const uint32_t quarter = warp & 3u;          // TMEM lane quarter (rows 32q .. 32q+31)
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = (quarter * 32u) << 16;

    // Q rows -> TMEM (A operand of S): row r's 224 fp16 = 112 packed columns at lane r.
    {
      const int gr = m0 + row;
      const uint4* src = reinterpret_cast<const uint4*>(args.qp + z * args.qp_batch_stride +
                                                        (int64_t)gr * 224);
      const bool in = gr < args.rows && in_bounds(gr < args.qp_rows_cap && z < args.batch, status);
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {                // columns [32c, 32c + 32) of 112
        uint32_t q[32];
        const int n16 = c < 3 ? 8 : 4;             // 16-byte pieces in this chunk (last: 16 cols)
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint4 v = (in && i < n16) ? src[c * 8 + i] : make_uint4(0u, 0u, 0u, 0u);
          q[4 * i + 0] = v.x;
          q[4 * i + 1] = v.y;
          q[4 * i + 2] = v.z;
          q[4 * i + 3] = v.w;
        }
        if (c < 3) {
          tmem_st32(tmem + kTmemQ + lane_off + c * 32, q);
        } else {
          tmem_st16(tmem + kTmemQ + lane_off + 96, q);      // columns [96, 112)
          if (args.sink_tiles > 0) {
            // QS: pair p of the RoPE part (packed column p) turned by sink_rot[p].
#pragma unroll
            for (int p = 0; p < 16; ++p) {
              const float2 v = __half22float2(*reinterpret_cast<const __half2*>(&q[p]));
              const float2 r = args.sink_rot[p];
              q[p] = pack_f16x2(v.x * r.x - v.y * r.y, v.x * r.y + v.y * r.x);
            }
            tmem_st16(tmem + kTmemQS + lane_off, q);
          }
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(q_ready);
    }

    float m_used = -INFINITY;
    float l_sum = 0.f;
    bool ok = true;
    for (int j = 0; j < nt; ++j) {
      if (!mbar_wait(s_full, (uint32_t)j & 1u, status)) { ok = false; break; }
      tc_fence_after();
      float s[kTileKeys];
#pragma unroll
      for (int c = 0; c < 4; ++c)
        tmem_ld32(tmem + kTmemS + lane_off + c * 32, reinterpret_cast<uint32_t*>(s) + c * 32);
      tmem_ld_wait();
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_regs_ready(reinterpret_cast<uint32_t*>(s) + c * 32);
      tc_fence_before();
      mbar_arrive(s_free);

      // Keys of this tile that exist: below n_keys, and for a sink tile below sink_keys.
      const int tile = (j + rot) % nt;
      const int valid = (tile < args.sink_tiles ? args.sink_keys : n_keys) - tile * kTileKeys;
      if (valid < kTileKeys) {
#pragma unroll
        for (int i = 0; i < kTileKeys; ++i)
          if (i >= valid) s[i] = -INFINITY;
      }
      // Row max with 8 independent partial maxima.
      float pm[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) pm[k] = s[k];
#pragma unroll
      for (int i = 8; i < kTileKeys; ++i) pm[i & 7] = fmaxf(pm[i & 7], s[i]);
      const float mx = fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])),
                             fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7])));
      float alpha = 1.f;
      bool rescale = false;
      if (j == 0) {
        m_used = fmaxf(mx, -1e30f);   // finite even if the first tile is all padding
      } else if (mx > m_used + kRescaleThreshold) {
        alpha = ex2_approx(m_used - mx);
        m_used = mx;
        rescale = true;
        l_sum *= alpha;
      }
      // Exponentials of the keys in pairs: the subtraction of the running max and the row-sum
      // additions run as packed fp32 pairs (4 partial sums of pairs).
      const uint64_t m2 = f32x2_pack(m_used, m_used);
      uint64_t ps[4] = {0ull, 0ull, 0ull, 0ull};
      uint32_t pk[kTileKeys / 2];
#pragma unroll
      for (int i = 0; i < kTileKeys / 2; ++i) {
        float d0, d1;
        f32x2_unpack(f32x2_sub(f32x2_pack(s[2 * i], s[2 * i + 1]), m2), d0, d1);
        const float p0 = ex2_approx(d0);
        const float p1 = ex2_approx(d1);
        pk[i] = pack_f16x2(p0, p1);
        ps[i & 3] = f32x2_add(ps[i & 3], f32x2_pack(p0, p1));
      }
      {
        float a0, a1, b0, b1;
        f32x2_unpack(f32x2_add(ps[0], ps[1]), a0, a1);
        f32x2_unpack(f32x2_add(ps[2], ps[3]), b0, b1);
        l_sum += (a0 + a1) + (b0 + b1);
      }

      // P buffer and O become free once PV_{j-1} has completed.
      if (j >= 1 && !mbar_wait(pv_done, (uint32_t)(j - 1) & 1u, status)) { ok = false; break; }
      tc_fence_after();
      if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
        for (int c = 0; c < 6; ++c) {
          uint32_t o[32];
          tmem_ld32(tmem + kTmemO + lane_off + c * 32, o);
          tmem_ld_wait();
          tmem_regs_ready(o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(tmem + kTmemO + lane_off + c * 32, o);
        }
        tmem_st_wait();
      }
      tmem_st32(tmem + kTmemP + lane_off, pk);
      tmem_st32(tmem + kTmemP + lane_off + 32, pk + 32);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(p_full);
    }

    // ---------------------------------------------------------------- epilogue: O / l
    if (ok && mbar_wait(pv_done, (uint32_t)(nt - 1) & 1u, status)) {
      tc_fence_after();
      const float inv_l = 1.f / l_sum;
      // Stage the row in the (now idle) first KV stage, then one bulk copy of 384 bytes.
      uint8_t* st_row = smem + L::kKV + row * L::kStageStride;
#pragma unroll 1
      for (int c = 0; c < 6; ++c) {
        uint32_t o[32];
        tmem_ld32(tmem + kTmemO + lane_off + c * 32, o);
        tmem_ld_wait();
        tmem_regs_ready(o);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          reinterpret_cast<uint4*>(st_row + c * 64)[q] = make_uint4(
              pack_f16x2(__uint_as_float(o[8 * q + 0]) * inv_l, __uint_as_float(o[8 * q + 1]) * inv_l),
              pack_f16x2(__uint_as_float(o[8 * q + 2]) * inv_l, __uint_as_float(o[8 * q + 3]) * inv_l),
              pack_f16x2(__uint_as_float(o[8 * q + 4]) * inv_l, __uint_as_float(o[8 * q + 5]) * inv_l),
              pack_f16x2(__uint_as_float(o[8 * q + 6]) * inv_l, __uint_as_float(o[8 * q + 7]) * inv_l));
        }
      }
      const int gr = m0 + row;
      if (gr < args.rows && in_bounds(gr < args.qp_rows_cap && z < args.batch, status)) {
        fence_proxy_async_smem();
        bulk_store(args.o_lat + z * args.o_lat_batch_stride + (int64_t)gr * 192, st_row, 384);
        bulk_commit();
        bulk_wait_all();
      }
    }
    tc_fence_before();
  }

  __syncwarp();      // reconverge single-lane roles before the CTA-wide barrier
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace mla
