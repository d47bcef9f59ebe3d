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
#ifndef FA_POLY_EVERY
#define FA_POLY_EVERY 0
#endif
#ifndef FA_OPTIMISTIC_EXP
#define FA_OPTIMISTIC_EXP 0
#endif
#ifndef FA_KV_STAGES_D128
#define FA_KV_STAGES_D128 4
#endif
// every FA_POLY_EVERY-th pair of P's exponentials on the FMA pipe, the rest on MUFU (0: all MUFU)
constexpr int kPolyEvery = FA_POLY_EVERY;

template <int HD>
struct PrefillCfg {
  static_assert(HD == 64 || HD == 128, "head dim");
  static constexpr int kChunks = HD / 64;          // 64-element (128-byte) swizzle chunks per row
  static constexpr int kChunkBytes = 128 * 128;    // 128 rows x 128 bytes
  static constexpr int kTileBytes = 128 * HD * 2;  // one 128 x HD bf16 tile
  static constexpr int kStages = HD == 128 ? FA_KV_STAGES_D128 : 8;
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
  int num_units;     // BH * num_pairs query-tile pairs, scheduled over the persistent CTAs
};

// Work units are query-tile pairs (two 128-row tiles of one (b, h) that share every K/V block).
// Non-causal units all cost the same; they are numbered head-major (unit = bh * pairs + pair) so
// the CTAs running at the same time share a few heads' K/V in L2, and handed out round-robin.
// Causal units cost in proportion to their key-block count (4p + 3 blocks for pair p), so they are
// numbered from the most expensive pair level down (unit = level * BH + bh, pair = pairs-1-level)
// and dealt to the CTAs in snake order (round r gives CTA c the unit r*G + c for even r and
// r*G + G-1-c for odd r), a static form of longest-processing-time-first scheduling.
struct WorkUnit {
  int bh;
  int pair;
};

// The unit CTA blockIdx.x processes in its round r, or -1 once it has none left.
__device__ __forceinline__ int unit_for_round(const PrefillParams &p, int r) {
  const int G = gridDim.x, c = blockIdx.x;
  const int u = r * G + ((p.causal && (r & 1)) ? G - 1 - c : c);
  return u < p.num_units ? u : -1;
}

__device__ __forceinline__ WorkUnit decode_unit(const PrefillParams &p, int u) {
  WorkUnit w;
  if (p.causal) {
    w.bh = u % p.BH;
    w.pair = p.num_pairs - 1 - u / p.BH;
  } else {
    w.bh = u / p.num_pairs;
    w.pair = u % p.num_pairs;
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

#ifndef FA_PACKED_F32X2
#define FA_PACKED_F32X2 1
#endif
#ifndef FA_P_CHUNKS
#define FA_P_CHUNKS 0
#endif

// One row of a score block -> P: p = 2^(s * scale*log2e - m_ref) for the 128 scores of this
// thread's row (MUFU ex2, or the FMA-pipe polynomial for every kPolyEvery-th pair).  P is written
// to TMEM as bf16 pairs (2 per 32-bit column), in 16-column chunks as each is ready
// (FA_P_CHUNKS) or in two 32-column stores at the end.  Returns the sum of the fp32 p (for the LSE)
// and the sum of the bf16-rounded p that P V actually uses (the normaliser of O, so that O is an
// exact convex combination of V rows even when one key dominates).  kTrackMax also returns the
// row's maximum score.
template <bool kTrackMax>
__device__ __forceinline__ void exp_row(float (&s)[kBN], float sl2, float mneg, uint32_t tP,
                                        float &sum_exact, float &sum_rounded, float &smax) {
  float mx0 = -INFINITY, mx1 = -INFINITY;
#if FA_PACKED_F32X2
  const uint64_t c2 = f2_pack(sl2, sl2), m2 = f2_pack(mneg, mneg);
  uint64_t le2 = 0, lr2 = 0;
#else
  float le0 = 0.f, le1 = 0.f, lr0 = 0.f, lr1 = 0.f;
#endif
#if !FA_P_CHUNKS
  uint32_t pall[kBN / 2];
#endif
#pragma unroll
  for (int g = 0; g < kBN / 32; ++g) {
#if FA_P_CHUNKS
    uint32_t pk[16];
#else
    uint32_t *pk = pall + g * 16;
#endif
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      const int e = g * 32 + 2 * c;
      if (kTrackMax) {
        if (c & 1) mx1 = fmax3(mx1, s[e], s[e + 1]);
        else mx0 = fmax3(mx0, s[e], s[e + 1]);
      }
      const bool poly = kPolyEvery > 0 && (g * 16 + c) % (kPolyEvery > 0 ? kPolyEvery : 1) == kPolyEvery - 1;
      float p0, p1;
#if FA_PACKED_F32X2
      const uint64_t x2 = f2_fma(f2_pack(s[e], s[e + 1]), c2, m2);
      uint64_t p2;
      if (poly) {
        p2 = exp2_poly_x2(x2);
      } else {
        float x0, x1;
        f2_unpack(x2, x0, x1);
        p2 = f2_pack(ex2(x0), ex2(x1));
      }
      le2 = f2_add(le2, p2);
      f2_unpack(p2, p0, p1);
      pk[c] = pack_bf16x2(p0, p1);
      lr2 = f2_add(lr2, f2_pack(__uint_as_float(pk[c] << 16), __uint_as_float(pk[c] & 0xffff0000u)));
#else
      const float x0 = fmaf(s[e], sl2, mneg), x1 = fmaf(s[e + 1], sl2, mneg);
      if (poly) {
        f2_unpack(exp2_poly_x2(f2_pack(x0, x1)), p0, p1);
      } else {
        p0 = ex2(x0);
        p1 = ex2(x1);
      }
      le0 += p0;
      le1 += p1;
      pk[c] = pack_bf16x2(p0, p1);
      lr0 += __uint_as_float(pk[c] << 16);
      lr1 += __uint_as_float(pk[c] & 0xffff0000u);
#endif
    }
#if FA_P_CHUNKS
    tmem_st16(tP + g * 16, pk);
#endif
  }
#if !FA_P_CHUNKS
  tmem_st32(tP, pall);
  tmem_st32(tP + 32, pall + 32);
#endif
#if FA_PACKED_F32X2
  float a, b;
  f2_unpack(le2, a, b);
  sum_exact = a + b;
  f2_unpack(lr2, a, b);
  sum_rounded = a + b;
#else
  sum_exact = le0 + le1;
  sum_rounded = lr0 + lr1;
#endif
  smax = fmaxf(mx0, mx1);
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
      mbar_init(&p_ready[i], kBM / 32);
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
  if (warp >= 8) {
  if (warp == 8) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t kv_it = 0, q_ph = 0;
      bool q_issued = false;
      uint32_t last_ph[C::kStages];
      bool issued[C::kStages];
      for (int s = 0; s < C::kStages; ++s) issued[s] = false;
      bool ok = true;
      for (int r = 0; ok; ++r) {
        const int u = unit_for_round(p, r);
        if (u < 0) break;
        const WorkUnit w = decode_unit(p, u);
        {
          const int pr = w.pair;
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
      for (int r = 0; ok; ++r) {
        const int u = unit_for_round(p, r);
        if (u < 0) break;
        const WorkUnit w = decode_unit(p, u);
        {
          const int pr = w.pair;
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
  }
  } else {
    // ------------------------------------------------------------------ softmax / epilogue
    const int wg = warp / 4;                       // which tile of the pair
    const int row = threadIdx.x % 128;             // TMEM lane == query row within the tile
    const uint32_t lane_off = static_cast<uint32_t>((warp % 4) * 32) << 16;
    const uint32_t tS = tmem + lane_off + (wg ? C::kColS1 : C::kColS0);
    const uint32_t tO = tmem + lane_off + (wg ? C::kColO1 : C::kColO0);
    const float sl2 = p.scale_log2;
    uint32_t s_ph = 0, o_ph = 0;
    bool ok = true;
    for (int r = 0; ok; ++r) {
      const int u = unit_for_round(p, r);
      if (u < 0) break;
      const WorkUnit w = decode_unit(p, u);
      {
        const int pr = w.pair;
        const int n = tile_blocks(p, pr, wg);
        if (n == 0) continue;
        const int qrow = pr * 2 * kBM + wg * kBM + row;
        float m_ref = -INFINITY, l = 0.f, lr = 0.f;
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
          // Lazy rescale: the reference max m_ref (log2 units) moves only when a block's max
          // exceeds it by more than 2^8.  After the first block the exponentials are computed
          // optimistically against the current m_ref while the block max is found in the same
          // pass; only if some row of the warp moved its reference (rare) is the pass redone.
          bool need;
          float alpha, le, lrb, smax;
          if (j == 0 || !FA_OPTIMISTIC_EXP) {
            float mx0 = fmax3(s[0], s[1], s[2]), mx1 = fmax3(s[3], s[4], s[5]);
            float mx2 = fmax3(s[6], s[7], s[8]), mx3 = fmax3(s[9], s[10], s[11]);
#pragma unroll
            for (int c = 12; c < kBN - 8; c += 8) {
              mx0 = fmax3(mx0, s[c], s[c + 1]);
              mx1 = fmax3(mx1, s[c + 2], s[c + 3]);
              mx2 = fmax3(mx2, s[c + 4], s[c + 5]);
              mx3 = fmax3(mx3, s[c + 6], s[c + 7]);
            }
            mx0 = fmax3(mx0, s[kBN - 4], s[kBN - 3]);
            mx1 = fmax3(mx1, s[kBN - 2], s[kBN - 1]);
            const float m_blk = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * sl2;
            need = m_blk > m_ref + kRescaleLog2;  // always true on the first block (m_ref = -inf)
            alpha = 1.f;
            if (need) {
              alpha = ex2(m_ref - m_blk);  // 2^-inf = 0 on the first block
              m_ref = m_blk;
            }
            exp_row<false>(s, sl2, (m_ref == -INFINITY) ? 0.f : -m_ref, tS, le, lrb, smax);
          } else {
            exp_row<true>(s, sl2, -m_ref, tS, le, lrb, smax);
            const float m_blk = smax * sl2;
            need = m_blk > m_ref + kRescaleLog2;
            alpha = 1.f;
            if (__any_sync(0xffffffffu, need)) {
              if (need) {
                alpha = ex2(m_ref - m_blk);
                m_ref = m_blk;
              }
              exp_row<false>(s, sl2, -m_ref, tS, le, lrb, smax);
            }
          }
          l = l * alpha + le;
          lr = lr * alpha + lrb;
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
          __syncwarp();
          if ((threadIdx.x & 31) == 0) mbar_arrive(&p_ready[wg]);  // one arrival per warp
        }
        if (!ok) break;
        // epilogue: O_i / l and LSE once the last P V of this tile has completed
        if (!__all_sync(0xffffffffu, mbar_wait(&o_done[wg], o_ph, abort_flag))) { ok = false; break; }
        o_ph ^= 1;
        tc_fence_after();
        const float inv = 1.f / lr;
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
    tmem_dealloc(*tmem_slot, C::kTmemCols);  // the address exactly as the allocation wrote it
  }
}

}  // namespace fa
