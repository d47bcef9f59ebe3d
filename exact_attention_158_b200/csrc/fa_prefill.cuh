// fa_prefill.cuh -- exact attention forward on sm_100a: TMA-staged tiles, tcgen05 tensor-core
// MMAs with TMEM accumulators, warp-specialised online softmax, persistent tile scheduler.
//
// Method: "Flash Attention" (velog.io/@myungum), section 2 and its pseudocode -- split Q, K, V
// into blocks that fit on chip, compute S_ij = Q_i K_j^T, keep the running row max m and row sum
// l, rescale the partial output when m grows, and write only O (and the row statistics) back.
// The loop order is the one "FlashAttention-2 GPU work partitioning" (section 3) describes: each
// query tile is owned by one group of threads that streams every key/value block past it, so O,
// m and l never leave the chip between blocks, and work is parallel over batch, head and query
// tile.  Normalisation by l is deferred to the end (fewer non-matmul operations, section 3 (1)).
//
// B200 mapping (one CTA per SM, 384 threads, persistent over work tiles):
//   warps 0-3   softmax for query tile 0 of the current pair (one TMEM lane = one query row)
//   warps 4-7   softmax for query tile 1 of the pair
//   warp  8     TMA producer: Q pair once per work tile, then K_j / V_j into an smem ring
//   warp  9     MMA issuer (one thread) + TMEM owner
//   warps 10-11 idle
// TMEM (512 columns): S0 [0,128)  S1 [128,256)  O0 [256,256+d)  O1 [256+d, 256+2d).
// P_i (bf16, two per 32-bit column) overwrites the first 64 columns of S_i and feeds the second
// MMA straight from TMEM: O_i += P_i V_j.
// The two tiles ping-pong: while softmax i works on S_i, the tensor core runs the other tile's
// S = Q K^T and O += P V.
#pragma once
#include "sm100_ptx.cuh"

namespace fa {

constexpr int kBM = 128;  // query rows per tile
constexpr int kBN = 128;  // keys per key/value block
constexpr int kPrefillThreads = 384;
constexpr float kRescaleLog2 = 8.0f;  // lazy rescale: tolerate a stale max up to 2^8 below
constexpr float kLn2 = 0.6931471805599453f;

template <int HD>
struct PrefillCfg {
  static_assert(HD == 64 || HD == 128, "head dim");
  static constexpr int kChunks = HD / 64;          // 64-element (128-byte) swizzle chunks per row
  static constexpr int kChunkBytes = 128 * 128;    // 128 rows x 128 bytes
  static constexpr int kTileBytes = 128 * HD * 2;  // one 128 x HD bf16 tile
  static constexpr int kStages = HD == 128 ? 4 : 8;
  static constexpr int kTmemCols = 512;
  static constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO0 = 256, kColO1 = 256 + HD;
  static constexpr int kNumBars = 1 + 1 + 2 * kStages + 2 + 2 + 2 + 1;
  static constexpr size_t kSmemBytes =
      1024 /* alignment slack */ + (2 + kStages) * kTileBytes + kNumBars * 8 + 16;
  static constexpr uint32_t kIdescQK = idesc_bf16_f32(kBM, kBN, 0, 0);  // Q, K both K-major
  static constexpr uint32_t kIdescPV = idesc_bf16_f32(kBM, HD, 0, 1);   // P (TMEM), V MN-major
};

struct PrefillParams {
  void *o;
  float *lse;
  int o_f32;
  int BH, N, causal;
  float scale_log2;  // scale * log2(e)
  int num_pairs;     // ceil(N / 256)
  int num_super;     // work units handed out round-robin to the persistent CTAs
};

// A work unit ("super tile") is one or two query-tile pairs of one (b, h).  Causal units pair the
// query pair p with the pair num_pairs-1-p, whose key-block counts add up to a constant, so every
// unit costs the same; non-causal units are single pairs.  Units are numbered head-major so CTAs
// running at the same time share the same heads' K/V in L2.
struct WorkUnit {
  int bh;
  int pairs[2];
  int count;
};

__device__ __forceinline__ WorkUnit decode_unit(const PrefillParams &p, int u) {
  WorkUnit w;
  if (p.causal) {
    const int half = (p.num_pairs + 1) / 2;
    w.bh = u / half;
    const int s = u % half;
    const int partner = p.num_pairs - 1 - s;
    w.pairs[0] = partner;  // the heavier pair first
    w.pairs[1] = s;
    w.count = (partner == s) ? 1 : 2;
  } else {
    w.bh = u / p.num_pairs;
    w.pairs[0] = u % p.num_pairs;
    w.pairs[1] = -1;
    w.count = 1;
  }
  return w;
}

// Key blocks visited by query tile i (0/1) of pair `pr`: 0 if the tile starts past N.
__device__ __forceinline__ int tile_blocks(const PrefillParams &p, int pr, int i) {
  const int q0 = pr * 2 * kBM + i * kBM;
  if (q0 >= p.N) return 0;
  const int nkb = (p.N + kBN - 1) / kBN;
  return p.causal ? (q0 / kBN + 1) : nkb;
}

template <int HD>
__device__ __forceinline__ void issue_qk(uint32_t d_tmem, uint32_t q_smem, uint32_t k_smem) {
  using C = PrefillCfg<HD>;
#pragma unroll
  for (int kk = 0; kk < HD / 16; ++kk) {
    const uint32_t off = (kk / 4) * C::kChunkBytes + (kk % 4) * 32;
    const uint64_t a = smem_desc_sw128(q_smem + off, 16, 1024);
    const uint64_t b = smem_desc_sw128(k_smem + off, 16, 1024);
    umma_ss(d_tmem, a, b, C::kIdescQK, kk > 0 ? 1u : 0u);
  }
}

template <int HD>
__device__ __forceinline__ void issue_pv(uint32_t o_tmem, uint32_t p_tmem, uint32_t v_smem,
                                         bool accumulate) {
  using C = PrefillCfg<HD>;
#pragma unroll
  for (int kk = 0; kk < kBN / 16; ++kk) {
    // 16 keys per MMA: 8 TMEM columns of packed P; 16 rows x 128 B of V (two 8-row atoms).
    // V is MN-major: LBO = distance between 64-element chunks of d, SBO = between 8-key groups.
    const uint64_t b = smem_desc_sw128(v_smem + kk * 16 * 128, C::kChunkBytes, 1024);
    umma_ts(o_tmem, p_tmem + kk * 8, b, C::kIdescPV, (accumulate || kk > 0) ? 1u : 0u);
  }
}

template <int HD>
__global__ void __launch_bounds__(kPrefillThreads, 1)
    fa_prefill_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const PrefillParams p) {
  using C = PrefillCfg<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *sQ = smem;                        // 2 tiles
  uint8_t *sKV = smem + 2 * C::kTileBytes;   // kStages tiles
  uint64_t *bars = reinterpret_cast<uint64_t *>(sKV + C::kStages * C::kTileBytes);
  uint64_t *q_full = bars;
  uint64_t *q_empty = bars + 1;
  uint64_t *kv_full = bars + 2;
  uint64_t *kv_empty = kv_full + C::kStages;
  uint64_t *s_full = kv_empty + C::kStages;  // [2]
  uint64_t *p_ready = s_full + 2;            // [2]
  uint64_t *o_done = p_ready + 2;            // [2]
  uint64_t *drain = o_done + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_ready[i], kBM);
      mbar_init(&o_done[i], 1);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int nkb = (p.N + kBN - 1) / kBN;

  if (warp == 8) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t kv_it = 0, q_ph = 0;
      bool q_issued = false;
      uint32_t last_ph[C::kStages];
      bool issued[C::kStages];
      for (int s = 0; s < C::kStages; ++s) issued[s] = false;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < p.num_super; u += gridDim.x) {
        const WorkUnit w = decode_unit(p, u);
        for (int t = 0; ok && t < w.count; ++t) {
          const int pr = w.pairs[t];
          const int n0 = tile_blocks(p, pr, 0), n1 = tile_blocks(p, pr, 1);
          const int nmax = n0 > n1 ? n0 : n1;
          if (!mbar_wait(q_empty, q_ph ^ 1, abort_flag)) { ok = false; break; }
          q_ph ^= 1;
          mbar_arrive_expect_tx(q_full, (n0 > 0 ? C::kTileBytes : 0) + (n1 > 0 ? C::kTileBytes : 0));
          q_issued = true;
          for (int i = 0; i < 2; ++i) {
            if ((i == 0 ? n0 : n1) == 0) continue;
            for (int ch = 0; ch < C::kChunks; ++ch)
              tma_load_3d(sQ + i * C::kTileBytes + ch * C::kChunkBytes, &tm_q, q_full, ch * 64,
                          pr * 2 * kBM + i * kBM, w.bh);
          }
          for (int j = 0; ok && j < nmax; ++j) {
            for (int kv = 0; kv < 2; ++kv) {
              const uint32_t st = kv_it % C::kStages, ph = (kv_it / C::kStages) & 1;
              if (!mbar_wait(&kv_empty[st], ph ^ 1, abort_flag)) { ok = false; break; }
              mbar_arrive_expect_tx(&kv_full[st], C::kTileBytes);
              for (int ch = 0; ch < C::kChunks; ++ch)
                tma_load_3d(sKV + st * C::kTileBytes + ch * C::kChunkBytes, kv ? &tm_v : &tm_k,
                            &kv_full[st], ch * 64, j * kBN, w.bh);
              issued[st] = true;
              last_ph[st] = ph;
              ++kv_it;
            }
          }
        }
      }
      if (!ok) {
        // abandoned: let every copy already in flight land before the CTA's smem goes away
        volatile int never = 0;
        for (int s = 0; s < C::kStages; ++s)
          if (issued[s]) mbar_wait(&kv_full[s], last_ph[s], &never);
        if (q_issued) mbar_wait(q_full, q_ph ^ 1, &never);
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t kv_it = 0, q_ph = 0, p_ph[2] = {0, 0};
      const uint32_t sQ0 = smem_u32(sQ), sQ1 = smem_u32(sQ + C::kTileBytes);
      const uint32_t sKV0 = smem_u32(sKV);
      bool ok = true;
      for (int u = blockIdx.x; ok && u < p.num_super; u += gridDim.x) {
        const WorkUnit w = decode_unit(p, u);
        for (int t = 0; ok && t < w.count; ++t) {
          const int pr = w.pairs[t];
          const int n[2] = {tile_blocks(p, pr, 0), tile_blocks(p, pr, 1)};
          const int nmax = n[0] > n[1] ? n[0] : n[1];
          if (!mbar_wait(q_full, q_ph, abort_flag)) { ok = false; break; }
          q_ph ^= 1;
          // S_i = Q_i K_0^T
          {
            const uint32_t st = kv_it % C::kStages, ph = (kv_it / C::kStages) & 1;
            if (!mbar_wait(&kv_full[st], ph, abort_flag)) { ok = false; break; }
            tc_fence_after();
            const uint32_t ks = sKV0 + st * C::kTileBytes;
            if (n[0] > 0) { issue_qk<HD>(tmem + C::kColS0, sQ0, ks); umma_commit(&s_full[0]); }
            if (n[1] > 0) { issue_qk<HD>(tmem + C::kColS1, sQ1, ks); umma_commit(&s_full[1]); }
            umma_commit(&kv_empty[st]);
            if (nmax == 1) umma_commit(q_empty);  // no further Q K^T in this work tile
            ++kv_it;
          }
          for (int j = 0; ok && j < nmax; ++j) {
            const uint32_t vst = kv_it % C::kStages, vph = (kv_it / C::kStages) & 1;
            if (!mbar_wait(&kv_full[vst], vph, abort_flag)) { ok = false; break; }
            ++kv_it;
            const uint32_t kst = kv_it % C::kStages, kph = (kv_it / C::kStages) & 1;
            const bool has_next = j + 1 < nmax;
            bool k_ready = false;
            for (int i = 0; ok && i < 2; ++i) {
              if (j >= n[i]) continue;
              if (!mbar_wait(&p_ready[i], p_ph[i], abort_flag)) { ok = false; break; }
              p_ph[i] ^= 1;
              tc_fence_after();
              const uint32_t colS = i ? C::kColS1 : C::kColS0;
              const uint32_t colO = i ? C::kColO1 : C::kColO0;
              issue_pv<HD>(tmem + colO, tmem + colS, sKV0 + vst * C::kTileBytes, j > 0);
              if (j == n[i] - 1) umma_commit(&o_done[i]);
              if (j + 1 < n[i]) {
                if (!k_ready) {
                  if (!mbar_wait(&kv_full[kst], kph, abort_flag)) { ok = false; break; }
                  tc_fence_after();
                  k_ready = true;
                }
                issue_qk<HD>(tmem + colS, i ? sQ1 : sQ0, sKV0 + kst * C::kTileBytes);
                umma_commit(&s_full[i]);
              }
            }
            if (!ok) break;
            umma_commit(&kv_empty[vst]);
            if (has_next) {
              umma_commit(&kv_empty[kst]);
              ++kv_it;
              if (j + 2 == nmax) umma_commit(q_empty);  // that was the last Q K^T of the tile
            }
          }
        }
      }
      // every MMA issued by this thread completes before TMEM is released
      umma_commit(drain);
      volatile int never = 0;
      mbar_wait(drain, 0, &never);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------------ softmax / epilogue
    const int wg = warp / 4;                       // which tile of the pair
    const int row = threadIdx.x % 128;             // TMEM lane == query row within the tile
    const uint32_t lane_off = static_cast<uint32_t>((warp % 4) * 32) << 16;
    const uint32_t tS = tmem + lane_off + (wg ? C::kColS1 : C::kColS0);
    const uint32_t tO = tmem + lane_off + (wg ? C::kColO1 : C::kColO0);
    const float sl2 = p.scale_log2;
    uint32_t s_ph = 0, o_ph = 0;
    bool ok = true;
    for (int u = blockIdx.x; ok && u < p.num_super; u += gridDim.x) {
      const WorkUnit w = decode_unit(p, u);
      for (int t = 0; ok && t < w.count; ++t) {
        const int pr = w.pairs[t];
        const int n = tile_blocks(p, pr, wg);
        if (n == 0) continue;
        const int qrow = pr * 2 * kBM + wg * kBM + row;
        float m_ref = -INFINITY, l = 0.f;
        for (int j = 0; j < n; ++j) {
          // the decision to go on must be warp-uniform: tcgen05.ld/st below are warp-collective
          if (!__all_sync(0xffffffffu, mbar_wait(&s_full[wg], s_ph, abort_flag))) { ok = false; break; }
          s_ph ^= 1;
          tc_fence_after();
          float s[kBN];
          tmem_ld32(tS + 0, reinterpret_cast<uint32_t *>(s));
          tmem_ld32(tS + 32, reinterpret_cast<uint32_t *>(s) + 32);
          tmem_ld32(tS + 64, reinterpret_cast<uint32_t *>(s) + 64);
          tmem_ld32(tS + 96, reinterpret_cast<uint32_t *>(s) + 96);
          tmem_wait_ld();
          const bool edge = (p.causal && j == n - 1) || (j == nkb - 1 && (p.N % kBN) != 0);
          if (edge) {
            int lim = (p.causal ? min(qrow + 1, p.N) : p.N) - j * kBN;  // visible keys in block
#pragma unroll
            for (int c = 0; c < kBN; ++c)
              if (c >= lim) s[c] = -INFINITY;
          }
          float mx0 = s[0], mx1 = s[1], mx2 = s[2], mx3 = s[3];
#pragma unroll
          for (int c = 4; c < kBN; c += 4) {
            mx0 = fmaxf(mx0, s[c]);
            mx1 = fmaxf(mx1, s[c + 1]);
            mx2 = fmaxf(mx2, s[c + 2]);
            mx3 = fmaxf(mx3, s[c + 3]);
          }
          const float m_blk = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * sl2;
          // lazy rescale: move the reference max only when the block max exceeds it by > 2^8
          const bool need = m_blk > m_ref + kRescaleLog2;
          const float alpha = need ? ex2(m_ref - m_blk) : 1.f;  // 2^-inf = 0 on the first block
          if (need) {
            m_ref = m_blk;
            l *= alpha;
          }
          const float mneg = (m_ref == -INFINITY) ? 0.f : -m_ref;
          float rs0 = 0.f, rs1 = 0.f;
          uint32_t pk[kBN / 2];
#pragma unroll
          for (int c = 0; c < kBN / 2; ++c) {
            const float p0 = ex2(fmaf(s[2 * c], sl2, mneg));
            const float p1 = ex2(fmaf(s[2 * c + 1], sl2, mneg));
            rs0 += p0;
            rs1 += p1;
            pk[c] = pack_bf16x2(p0, p1);
          }
          tmem_st32(tS + 0, pk);
          tmem_st32(tS + 32, pk + 32);
          l += rs0 + rs1;
          if (j > 0 && __any_sync(0xffffffffu, need)) {
            // O_i holds the sum through block j-1 (S_ij's commit covers that MMA): rescale it in
            // place before P_ij V_j is accumulated on top.  Rows that keep their max use alpha 1.
#pragma unroll
            for (int cc = 0; cc < HD; cc += 32) {
              uint32_t o[32];
              tmem_ld32(tO + cc, o);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
              tmem_st32(tO + cc, o);
            }
          }
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(&p_ready[wg]);
        }
        if (!ok) break;
        // epilogue: O_i / l and LSE once the last P V of this tile has completed
        if (!__all_sync(0xffffffffu, mbar_wait(&o_done[wg], o_ph, abort_flag))) { ok = false; break; }
        o_ph ^= 1;
        tc_fence_after();
        const float inv = 1.f / l;
        const bool live = qrow < p.N;
        const size_t grow = static_cast<size_t>(w.bh) * p.N + qrow;
#pragma unroll
        for (int cc = 0; cc < HD; cc += 32) {
          uint32_t o[32];
          tmem_ld32(tO + cc, o);
          tmem_wait_ld();
          if (live) {
            if (p.o_f32) {
              float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(p.o) + grow * HD + cc);
#pragma unroll
              for (int e = 0; e < 8; ++e)
                dst[e] = make_float4(__uint_as_float(o[4 * e]) * inv, __uint_as_float(o[4 * e + 1]) * inv,
                                     __uint_as_float(o[4 * e + 2]) * inv, __uint_as_float(o[4 * e + 3]) * inv);
            } else {
              uint4 *dst = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(p.o) + grow * HD + cc);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                uint4 v;
                v.x = pack_bf16x2(__uint_as_float(o[8 * e + 0]) * inv, __uint_as_float(o[8 * e + 1]) * inv);
                v.y = pack_bf16x2(__uint_as_float(o[8 * e + 2]) * inv, __uint_as_float(o[8 * e + 3]) * inv);
                v.z = pack_bf16x2(__uint_as_float(o[8 * e + 4]) * inv, __uint_as_float(o[8 * e + 5]) * inv);
                v.w = pack_bf16x2(__uint_as_float(o[8 * e + 6]) * inv, __uint_as_float(o[8 * e + 7]) * inv);
                dst[e] = v;
              }
            }
          }
        }
        if (live && p.lse) p.lse[grow] = (m_ref + lg2(l)) * kLn2;
      }
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace fa
