// dense_attn.cuh - dense per-head attention (12 x 128 keys and values per token), the layout the
// VideoMLA paper page replaces (§1: 2 x 12 x 128 = 3,072 cached scalars per token).  Built as
// the measurement baseline next to the latent-window kernel, on the same sm_100a machinery.
//
//   out[q, h] = sum_j softmax_j(scale * Q[q, h] . K[j, h]) V[j, h]
//
// One CTA owns 128 query rows of one head.  Warp roles (192 threads):
//   warp 0      TMA producer: the Q tile once (2 x 64-column SW128 boxes), then per 128-key tile
//               K (2 boxes) and V (2 boxes) of this head into a KV_STAGES-deep ring.
//   warp 1      TMEM allocator + single-thread MMA issuer:
//                 S_j = Q K_j^T   M=128 N=128 K=128 (8 k-steps, both K-major)
//                 O  += P_j V_j   M=128 N=128 K=128 (8 k-steps, V read MN-major, P from TMEM)
//   warps 2..5  softmax (one row per thread, base 2, lazy O rescale), then O / l -> bf16 out.
// TMEM columns: S0 [0,128), S1 [128,256), O [256,384), P [384,448).
//
// Split keys: when there are too few (query tile, head, stream) items to fill the GPU evenly
// (1,560 queries x 12 heads = 156 items on 148 SMs would take two full waves), blockIdx.z also
// selects one of `splits` key ranges; each CTA then writes its unnormalised O, running max and
// sum in fp32, and dense_combine_kernel merges the ranges: out = sum_s 2^(m_s - M) O_s /
// sum_s 2^(m_s - M) l_s.
#pragma once

#include "ptx.cuh"

namespace mla {

constexpr int kDenseThreads = 192;
constexpr float kDenseRescaleLog2 = 8.0f;  // lazy O rescale when the max grows by > 2^8

// a * b + c on packed fp32 pairs (one sm_100 instruction for both).
__device__ __forceinline__ uint64_t dense_fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}

template <int KV_STAGES>
struct DenseSmem {
  static constexpr int kAtom = 128 * 128;                 // 128 rows x 64 bf16 (SW128)
  static constexpr int kQ = 0;                            // 2 atoms
  static constexpr int kKV = 2 * kAtom;
  static constexpr int kStage = 4 * kAtom;                // K (2 atoms) + V (2 atoms)
  static constexpr int kBar = kKV + KV_STAGES * kStage;
  static constexpr int kBytes = kBar + 256 + 1024;
  static_assert(kBytes <= 232448, "dense attention tile does not fit in shared memory");
};

struct DenseArgs {
  int32_t n_q;         // query tokens per stream
  int32_t n_kv;        // keys per stream
  int32_t n_heads;
  float scale_log2;    // softmax_scale * log2(e)
  __nv_bfloat16* out;  // [B][n_q][n_heads][128]
  int32_t splits;      // key ranges per (query tile, head, stream); 1 -> out directly
  int32_t kv_per_split;  // keys per range (a multiple of 128)
  float* o_part;       // splits > 1: [splits][B][n_q][n_heads][128] unnormalised O
  float2* ml_part;     // splits > 1: [splits][B][n_q][n_heads] (max in log2 units, sum)
  int64_t part_rows;   // rows the partials hold (splits x B x n_q x n_heads; bounds checks)
  int32_t batch;       // streams (bounds checks)
};

template <int KV_STAGES>
__global__ void __launch_bounds__(kDenseThreads, 1)
    dense_attn_kernel(const __grid_constant__ CUtensorMap map_q,
                      const __grid_constant__ CUtensorMap map_k,
                      const __grid_constant__ CUtensorMap map_v, DenseArgs args, int* status) {
  using L = DenseSmem<KV_STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = kv_full + KV_STAGES;
  uint64_t* s_full = kv_empty + KV_STAGES;
  uint64_t* s_free = s_full + 2;
  uint64_t* p_full = s_free + 2;
  uint64_t* pv_done = p_full + 1;
  uint64_t* quiesce = pv_done + 1;               // all MMAs of this CTA have completed
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(quiesce + 1);

  const uint32_t warp = warp_id();
  const uint32_t lane = lane_id();
  const int m0 = blockIdx.x * 128;
  const int h = blockIdx.y;
  const int z = (int)blockIdx.z / args.splits;
  const int sp = (int)blockIdx.z - z * args.splits;   // key range of this CTA
  const int kv0 = sp * args.kv_per_split;
  const int kv_end = args.n_kv < kv0 + args.kv_per_split ? args.n_kv : kv0 + args.kv_per_split;
  const int n_kv = kv_end - kv0;                      // keys of this CTA (>= 1)
  const int nt = (n_kv + 127) / 128;
  const int col0 = h * 128;  // this head's columns in the [tokens][n_heads * 128] views

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < KV_STAGES; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&s_free[s], 128);
    }
    mbar_init(p_full, 128);
    mbar_init(pv_done, 1);
    mbar_init(quiesce, 1);
    fence_mbar_init();
    tma_prefetch(&map_q);
    tma_prefetch(&map_k);
    tma_prefetch(&map_v);
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
  const uint32_t tmem_o = tmem + 256;
  const uint32_t tmem_p = tmem + 384;

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t keep = l2_policy_evict_last();   // K/V are re-read by every row tile of h
      const uint64_t once = l2_policy_evict_first();
      mbar_arrive_expect_tx(q_full, 2 * L::kAtom);
      for (int a = 0; a < 2; ++a)
        tma_load_3d_hint(smem + L::kQ + a * L::kAtom, &map_q, q_full, col0 + a * 64, m0, z, once);
      int issued = 0;
      for (int j = 0; j < nt; ++j) {
        const int st = j % KV_STAGES;
        if (!mbar_wait(&kv_empty[st], ((uint32_t)(j / KV_STAGES) & 1u) ^ 1u, status)) break;
        uint8_t* kv = smem + L::kKV + st * L::kStage;
        mbar_arrive_expect_tx(&kv_full[st], L::kStage);
        for (int a = 0; a < 2; ++a) {
          tma_load_3d_hint(kv + a * L::kAtom, &map_k, &kv_full[st], col0 + a * 64, kv0 + j * 128, z,
                           keep);
          tma_load_3d_hint(kv + (2 + a) * L::kAtom, &map_v, &kv_full[st], col0 + a * 64, kv0 + j * 128, z,
                           keep);
        }
        issued = j + 1;
      }
      // Drain: no copy may still land in shared memory when the CTA exits (also after an error).
      for (int j = issued > KV_STAGES ? issued - KV_STAGES : 0; j < issued; ++j)
        mbar_wait_quiesce(&kv_full[j % KV_STAGES], (uint32_t)(j / KV_STAGES) & 1u, status);
      mbar_wait_quiesce(q_full, 0, status);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_f32acc(128, 128, false, false);
      constexpr uint32_t idesc_o = idesc_f32acc(128, 128, true, false);
      const uint32_t q_base = smem_u32(smem + L::kQ);
      bool ok = mbar_wait(q_full, 0, status);
      for (int j = 0; ok && j <= nt; ++j) {
        if (j < nt) {
          const int st = j % KV_STAGES;
          const int sb = j & 1;
          if (!mbar_wait(&kv_full[st], (uint32_t)(j / KV_STAGES) & 1u, status)) break;
          if (j >= 2 && !mbar_wait(&s_free[sb], (uint32_t)((j >> 1) - 1) & 1u, status)) break;
          tc_fence_after();
          const uint32_t k_base = smem_u32(smem + L::kKV + st * L::kStage);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * L::kAtom + (kk & 3) * 32;
            umma_ss(tmem + sb * 128, smem_desc(q_base + off, 16, 1024, kSwizzle128B),
                    smem_desc(k_base + off, 16, 1024, kSwizzle128B), idesc_s, kk > 0 ? 1u : 0u);
          }
          tc_commit(&s_full[sb]);
        }
        if (j >= 1) {
          const int jj = j - 1;
          const int st = jj % KV_STAGES;
          if (!mbar_wait(p_full, (uint32_t)jj & 1u, status)) break;
          tc_fence_after();
          const uint32_t v_base = smem_u32(smem + L::kKV + st * L::kStage + 2 * L::kAtom);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t db = smem_desc(v_base + kk * 2048, L::kAtom, 1024, kSwizzle128B);
            umma_ts(tmem_o, tmem_p + kk * 8, db, idesc_o, (jj > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(pv_done);
          tc_commit(&kv_empty[st]);
        }
      }
      // The CTA frees shared and tensor memory only after every issued MMA has completed.
      tc_commit(quiesce);
      mbar_wait_quiesce(quiesce, 0, status);
    }
  } else {
    const uint32_t sub = warp & 3u;
    const int row = sub * 32 + lane;
    const uint32_t lane_off = (sub * 32u) << 16;
    const float c = args.scale_log2;
    float m_used = -INFINITY;   // running max of the raw scores
    float l_sum = 0.f;
    bool ok = true;
    for (int j = 0; j < nt; ++j) {
      const int sb = j & 1;
      if (!mbar_wait(&s_full[sb], (uint32_t)(j >> 1) & 1u, status)) { ok = false; break; }
      tc_fence_after();
      float s[128];
#pragma unroll
      for (int q = 0; q < 4; ++q)
        tmem_ld32(tmem + lane_off + sb * 128 + q * 32, reinterpret_cast<uint32_t*>(s) + q * 32);
      tmem_ld_wait();
#pragma unroll
      for (int q = 0; q < 4; ++q) tmem_regs_ready(reinterpret_cast<uint32_t*>(s) + q * 32);
      tc_fence_before();
      mbar_arrive(&s_free[sb]);
      const int valid = n_kv - j * 128;
      if (valid < 128) {
#pragma unroll
        for (int i = 0; i < 128; ++i)
          if (i >= valid) s[i] = -INFINITY;
      }
      float pm[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) pm[k] = s[k];
#pragma unroll
      for (int i = 8; i < 128; ++i) pm[i & 7] = fmaxf(pm[i & 7], s[i]);
      const float mx = fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])),
                             fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7])));
      float alpha = 1.f;
      bool rescale = false;
      if (j == 0) {
        m_used = mx;
      } else if ((mx - m_used) * c > kDenseRescaleLog2) {
        alpha = ex2_approx((m_used - mx) * c);
        m_used = mx;
        rescale = true;
        l_sum *= alpha;
      }
      // Scaled, shifted scores and the row sums as packed fp32 pairs (4 partial sums of pairs).
      const float mc = m_used * c;
      const uint64_t c2 = f32x2_pack(c, c), nmc2 = f32x2_pack(-mc, -mc);
      uint64_t ps[4] = {0ull, 0ull, 0ull, 0ull};
      uint32_t pk[64];
#pragma unroll
      for (int i = 0; i < 64; ++i) {
        float d0, d1;
        f32x2_unpack(dense_fma2(f32x2_pack(s[2 * i], s[2 * i + 1]), c2, nmc2), d0, d1);
        const float p0 = ex2_approx(d0);
        const float p1 = ex2_approx(d1);
        pk[i] = pack_bf16x2(p0, p1);
        ps[i & 3] = f32x2_add(ps[i & 3], f32x2_pack(p0, p1));
      }
      {
        float a0, a1, b0, b1;
        f32x2_unpack(f32x2_add(ps[0], ps[1]), a0, a1);
        f32x2_unpack(f32x2_add(ps[2], ps[3]), b0, b1);
        l_sum += (a0 + a1) + (b0 + b1);
      }
      if (j >= 1 && !mbar_wait(pv_done, (uint32_t)(j - 1) & 1u, status)) { ok = false; break; }
      tc_fence_after();
      if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
        for (int q = 0; q < 4; ++q) {
          uint32_t o[32];
          tmem_ld32(tmem_o + lane_off + q * 32, o);
          tmem_ld_wait();
          tmem_regs_ready(o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(tmem_o + lane_off + q * 32, o);
        }
        tmem_st_wait();
      }
      tmem_st32(tmem_p + lane_off, pk);
      tmem_st32(tmem_p + lane_off + 32, pk + 32);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    if (ok && args.splits > 1 && mbar_wait(pv_done, (uint32_t)(nt - 1) & 1u, status)) {
      // Partial of one key range: unnormalised O, the max in log2 units and the sum, in fp32.
      tc_fence_after();
      const int q = m0 + row;
      const int64_t prow = (((int64_t)sp * (gridDim.z / args.splits) + z) * args.n_q + q) * args.n_heads + h;
#pragma unroll 1
      for (int cq = 0; cq < 4; ++cq) {
        uint32_t o[32];
        tmem_ld32(tmem_o + lane_off + cq * 32, o);
        tmem_ld_wait();
        tmem_regs_ready(o);
        if (q < args.n_q && in_bounds(prow < args.part_rows, status)) {
          float4* dst = reinterpret_cast<float4*>(args.o_part + prow * 128 + cq * 32);
#pragma unroll
          for (int v4 = 0; v4 < 8; ++v4)
            dst[v4] = make_float4(__uint_as_float(o[4 * v4]), __uint_as_float(o[4 * v4 + 1]),
                                  __uint_as_float(o[4 * v4 + 2]), __uint_as_float(o[4 * v4 + 3]));
        }
      }
      if (q < args.n_q && in_bounds(prow < args.part_rows, status))
        args.ml_part[prow] = make_float2(m_used * c, l_sum);
    } else if (ok && mbar_wait(pv_done, (uint32_t)(nt - 1) & 1u, status)) {
      tc_fence_after();
      const float inv_l = 1.f / l_sum;
      constexpr int kStride = 272;  // 256 bytes of bf16 + 16 padding
      uint8_t* st_row = smem + L::kKV + row * kStride;
#pragma unroll 1
      for (int q = 0; q < 4; ++q) {
        uint32_t o[32];
        tmem_ld32(tmem_o + lane_off + q * 32, o);
        tmem_ld_wait();
        tmem_regs_ready(o);
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          reinterpret_cast<uint4*>(st_row + q * 64)[v] = make_uint4(
              pack_bf16x2(__uint_as_float(o[8 * v + 0]) * inv_l, __uint_as_float(o[8 * v + 1]) * inv_l),
              pack_bf16x2(__uint_as_float(o[8 * v + 2]) * inv_l, __uint_as_float(o[8 * v + 3]) * inv_l),
              pack_bf16x2(__uint_as_float(o[8 * v + 4]) * inv_l, __uint_as_float(o[8 * v + 5]) * inv_l),
              pack_bf16x2(__uint_as_float(o[8 * v + 6]) * inv_l, __uint_as_float(o[8 * v + 7]) * inv_l));
        }
      }
      __syncwarp();
      for (int rr = 0; rr < 32; rr += 2) {   // two rows per pass, 16 lanes x 16 bytes each
        const int trow = sub * 32 + rr + (lane >> 4);
        const int q = m0 + trow;
        if (q < args.n_q && in_bounds(z < args.batch && h < args.n_heads, status)) {
          __nv_bfloat16* o = args.out + (((int64_t)z * args.n_q + q) * args.n_heads + h) * 128;
          reinterpret_cast<uint4*>(o)[lane & 15] =
              reinterpret_cast<const uint4*>(smem + L::kKV + trow * kStride)[lane & 15];
        }
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

// Merge of the key ranges of the split dense attention: one warp per (stream, query, head),
// four of the 128 channels per lane.
__global__ void dense_combine_kernel(const float* __restrict__ o_part,
                                     const float2* __restrict__ ml_part, int splits, int batch,
                                     int n_q, int n_heads, __nv_bfloat16* __restrict__ out,
                                     int64_t part_rows, int* status) {
  const int64_t rows = (int64_t)batch * n_q * n_heads;
  const int64_t r = (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  if (!in_bounds((int64_t)(splits - 1) * rows + r < part_rows, status)) return;
  float mmax = -INFINITY;
  for (int s = 0; s < splits; ++s) mmax = fmaxf(mmax, ml_part[(int64_t)s * rows + r].x);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float lsum = 0.f;
  for (int s = 0; s < splits; ++s) {
    const float2 ml = ml_part[(int64_t)s * rows + r];
    const float wgt = ex2_approx(ml.x - mmax);
    lsum += wgt * ml.y;
    const float4 o = reinterpret_cast<const float4*>(o_part + ((int64_t)s * rows + r) * 128)[lane];
    acc.x += wgt * o.x;
    acc.y += wgt * o.y;
    acc.z += wgt * o.z;
    acc.w += wgt * o.w;
  }
  const float inv = 1.f / lsum;
  uint2 packed = make_uint2(pack_bf16x2(acc.x * inv, acc.y * inv), pack_bf16x2(acc.z * inv, acc.w * inv));
  reinterpret_cast<uint2*>(out + r * 128)[lane] = packed;
}

}  // namespace mla
