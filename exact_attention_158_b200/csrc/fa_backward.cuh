// fa_backward.cuh -- exact attention backward on sm_100a: dQ, dK, dV from Q, K, V, O, dO and the
// forward's log-sum-exp, with the probabilities recomputed tile by tile and never stored.
//
// Method: the gradient of sum(dO * O) through O = softmax(scale Q K^T) V, blockwise.  The pages
// give the backward in prose: gradients from the stored intermediate results, processed block by
// block ("Paged vs Flash attention", training), and the attention matrix recomputed instead of
// kept ("LLM study notes", FlashAttention; "Flash Attention" (myungum), section 1).  What is kept
// from the forward is the row statistic LSE; P is recomputed as exp(scale S - LSE).  With
// D_i = sum_c dO[i,c] O[i,c] (= sum_j P_ij dP_ij):
//     dV_j = sum_i P_ij dO_i      dP_ij = dO_i . V_j      dS_ij = P_ij (dP_ij - D_i)
//     dK_j = scale sum_i dS_ij Q_i                         dQ_i = scale sum_j dS_ij K_j
//
// Work partition: one CTA per (b, h, key block j of 128 keys).  K_j and V_j stay in shared memory;
// the CTA streams every query block i that sees them (i >= j when causal) and keeps dK_j and dV_j
// in TMEM for the whole loop.  dQ_i gets one 128 x d partial per (i, j) pair, added into an fp32
// accumulator in global memory.
//
// The scores are computed transposed, S^T = K_j Q_i^T (TMEM lane = key), so each compute thread
// owns one key row: P^T and dS^T are written by rows into one 128 x 128 bf16 tile X in the
// 128-byte-swizzled layout the tensor core reads.  X is the K-major A operand of dV += P^T dO and
// dK += dS^T Q, and, read through an MN-major descriptor, the A operand of dQ = dS K.
//
//   warps 0-3  compute: S^T -> P^T (X), dP^T -> dS^T (X), and the final dK, dV write
//   warps 4-7  dQ: TMEM -> fp32 red.add into the accumulator
//   warp  8    TMA producer: K_j, V_j once; Q_i (+ its LSE and D rows), dO_i per query block
//   warp  9    MMA issuer (one thread) + TMEM owner
// TMEM (512 columns): S^T [0,128)  dP^T [128,256)  dV [256,256+d)  dK [256+d,256+2d)  and dQ at
// [256+2d, 256+3d) when d = 64; at d = 128 the columns are full and dQ_i takes dP^T's columns,
// which are free once dS^T_i has been formed.
#pragma once
#include "fa_prefill.cuh"

namespace fa {

constexpr int kBwdThreads = 320;
constexpr size_t kMaxDynSmem = 232448;  // 227 KB per CTA on sm_100

template <int HD>
struct BwdCfg {
  static_assert(HD == 64 || HD == 128, "head dim");
  static constexpr int kChunks = HD / 64;
  static constexpr int kChunkBytes = 128 * 128;
  static constexpr int kTileBytes = 128 * HD * 2;
  static constexpr int kXBytes = 128 * 128 * 2;
  static constexpr int kStages = 2;                // Q and dO rings
  static constexpr int kVecFloats = 2 * kBM;       // LSE (log2 units) and D of one query block
  static constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 256 + HD;
  static constexpr bool kDqOnDp = HD == 128;
  static constexpr uint32_t kColDQ = kDqOnDp ? kColDP : 256 + 2 * HD;
  static constexpr int kTmemCols = 512;
  static constexpr int kNumBars = 1 + 4 * kStages + 10;
  static constexpr size_t kBodyBytes = 2 * kTileBytes + 2 * kStages * kTileBytes + kXBytes +
                                       kStages * kVecFloats * 4 + kNumBars * 8 + 16;
  // up to 1 KB of slack to align the tiles to the 1024-byte swizzle atom
  static constexpr size_t kSmemBytes =
      kBodyBytes + 1024 <= kMaxDynSmem ? kBodyBytes + 1024 : kMaxDynSmem;
  static_assert(kBodyBytes <= kMaxDynSmem, "shared memory budget");
  static_assert(kColDQ + (kDqOnDp ? 0 : HD) <= kTmemCols, "TMEM budget");
  static constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128, 0, 0);  // K/V and Q/dO K-major
  static constexpr uint32_t kIdescKV = idesc_bf16_f32(128, HD, 0, 1);  // X K-major, Q/dO MN-major
  static constexpr uint32_t kIdescQ = idesc_bf16_f32(128, HD, 1, 1);   // X MN-major, K MN-major
};

struct BwdParams {
  const float *lse2;  // [BH, Np]  LSE * log2(e) per query row; +inf on padding rows
  const float *dvec;  // [BH, Np]  D = rowsum(dO * O); 0 on padding rows
  float *dq_acc;      // [BH, Np, d] fp32, zero before the launch
  void *dk, *dv;      // [BH, N, d]
  int g_f32;          // dK / dV as fp32 (1) or bf16 (0)
  int BH, N, Np, nkb, causal;
  float scale_log2, scale;
};

// D (TMEM, 128 x N) (+)= A (X: 128 x 128 bf16, K-major over the 128 k) * B, with B the 128 k-rows
// of a [128][N] tile read MN-major (N = HD in 64-element chunks).
template <int HD>
__device__ __forceinline__ void issue_x_kmajor(uint32_t d_tmem, uint32_t x_smem, uint32_t b_smem,
                                               uint32_t idesc, bool accumulate) {
#pragma unroll
  for (int kk = 0; kk < 128 / 16; ++kk) {
    const uint64_t a = smem_desc_sw128(x_smem + (kk / 4) * 16384 + (kk % 4) * 32, 16, 1024);
    const uint64_t b = smem_desc_sw128(b_smem + kk * 16 * 128, 16384, 1024);
    umma_ss(d_tmem, a, b, idesc, (accumulate || kk > 0) ? 1u : 0u);
  }
}

// dQ (TMEM, 128 queries x HD) = dS K: A = X read MN-major (m = query = X's column, k = key = X's
// row), B = K_j read MN-major (n = d, k = key).
template <int HD>
__device__ __forceinline__ void issue_dq(uint32_t d_tmem, uint32_t x_smem, uint32_t k_smem) {
  using C = BwdCfg<HD>;
#pragma unroll
  for (int kk = 0; kk < 128 / 16; ++kk) {
    const uint64_t a = smem_desc_sw128(x_smem + kk * 16 * 128, 16384, 1024);
    const uint64_t b = smem_desc_sw128(k_smem + kk * 16 * 128, 16384, 1024);
    umma_ss(d_tmem, a, b, C::kIdescQ, kk > 0 ? 1u : 0u);
  }
}

// One TMEM row of HD fp32 values (this thread's lane) times `mul`, to global row `grow`.
template <int HD>
__device__ __forceinline__ void store_grad_row(uint32_t taddr, float mul, void *dst_base, int f32,
                                               size_t grow, bool live) {
#pragma unroll
  for (int cc = 0; cc < HD; cc += 32) {
    uint32_t v[32];
    tmem_ld32(taddr + cc, v);
    tmem_wait_ld();
    if (!live) continue;
    if (f32) {
      float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(dst_base) + grow * HD + cc);
#pragma unroll
      for (int e = 0; e < 8; ++e)
        dst[e] = make_float4(__uint_as_float(v[4 * e]) * mul, __uint_as_float(v[4 * e + 1]) * mul,
                             __uint_as_float(v[4 * e + 2]) * mul, __uint_as_float(v[4 * e + 3]) * mul);
    } else {
      uint4 *dst = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(dst_base) + grow * HD + cc);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        uint4 w;
        w.x = pack_bf16x2(__uint_as_float(v[8 * e + 0]) * mul, __uint_as_float(v[8 * e + 1]) * mul);
        w.y = pack_bf16x2(__uint_as_float(v[8 * e + 2]) * mul, __uint_as_float(v[8 * e + 3]) * mul);
        w.z = pack_bf16x2(__uint_as_float(v[8 * e + 4]) * mul, __uint_as_float(v[8 * e + 5]) * mul);
        w.w = pack_bf16x2(__uint_as_float(v[8 * e + 6]) * mul, __uint_as_float(v[8 * e + 7]) * mul);
        dst[e] = w;
      }
    }
  }
}

template <int HD>
__global__ void __launch_bounds__(kBwdThreads, 1)
    fa_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                  const BwdParams p) {
  using C = BwdCfg<HD>;
  extern __shared__ uint8_t smem_raw[];
  const uintptr_t raw = reinterpret_cast<uintptr_t>(smem_raw);
  const uintptr_t base = (raw + 1023) & ~static_cast<uintptr_t>(1023);
  if (base - raw + C::kBodyBytes > C::kSmemBytes) {  // the same for every thread of the CTA
    if (threadIdx.x == 0) atomicExch(&g_device_status, 4 /* FA_ERR_LAUNCH */);
    return;
  }
  uint8_t *sK = reinterpret_cast<uint8_t *>(base);
  uint8_t *sV = sK + C::kTileBytes;
  uint8_t *sQ = sV + C::kTileBytes;                 // kStages tiles
  uint8_t *sDO = sQ + C::kStages * C::kTileBytes;   // kStages tiles
  uint8_t *sX = sDO + C::kStages * C::kTileBytes;   // P^T, then dS^T
  float *sVec = reinterpret_cast<float *>(sX + C::kXBytes);  // [kStages][LSE2 128 | D 128]
  uint64_t *bars = reinterpret_cast<uint64_t *>(sVec + C::kStages * C::kVecFloats);
  uint64_t *kv_full = bars;                    // K_j, V_j landed
  uint64_t *q_full = bars + 1;                 // [kStages] Q_i + its LSE2 / D rows landed
  uint64_t *q_empty = q_full + C::kStages;     // [kStages] dK_i done (last reader of Q_i)
  uint64_t *do_full = q_empty + C::kStages;    // [kStages] dO_i landed
  uint64_t *do_empty = do_full + C::kStages;   // [kStages] dV_i done (last reader of dO_i)
  uint64_t *s_full = do_empty + C::kStages;    // S^T_i computed
  uint64_t *s_free = s_full + 1;               // S^T_i copied out (4 warp arrivals)
  uint64_t *dp_full = s_free + 1;              // dP^T_i computed
  uint64_t *p_full = dp_full + 1;              // P^T_i written to X (4 warp arrivals)
  uint64_t *dv_done = p_full + 1;              // dV += P^T_i dO_i done: X may take dS^T_i
  uint64_t *ds_full = dv_done + 1;             // dS^T_i written to X (4 warp arrivals)
  uint64_t *x_free = ds_full + 1;              // dK_i and dQ_i done: X may take P^T_i+1
  uint64_t *dq_full = x_free + 1;              // dQ_i computed
  uint64_t *dq_free = dq_full + 1;             // dQ_i read out (4 warp arrivals)
  uint64_t *drain = dq_free + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int jb = blockIdx.x % p.nkb;  // key block
  const int bh = blockIdx.x / p.nkb;
  const int i_lo = p.causal ? jb : 0;  // first query block that sees key block jb
  const int n = p.Np / kBM - i_lo;     // query blocks visited (>= 1)

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 1);
      mbar_init(&do_full[s], 1);
      mbar_init(&do_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, 4);
    mbar_init(dp_full, 1);
    mbar_init(p_full, 4);
    mbar_init(dv_done, 1);
    mbar_init(ds_full, 4);
    mbar_init(x_free, 1);
    mbar_init(dq_full, 1);
    mbar_init(dq_free, 4);
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
    tma_prefetch_desc(&tm_do);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 8) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      bool ok = true;
      int q_loads = 0, do_loads = 0;
      mbar_arrive_expect_tx(kv_full, 2 * C::kTileBytes);
      for (int ch = 0; ch < C::kChunks; ++ch) {
        tma_load_3d(sK + ch * C::kChunkBytes, &tm_k, kv_full, ch * 64, jb * kBN, bh);
        tma_load_3d(sV + ch * C::kChunkBytes, &tm_v, kv_full, ch * 64, jb * kBN, bh);
      }
      const size_t vec_row = static_cast<size_t>(bh) * p.Np;
      for (int t = 0; t < n; ++t) {
        const int i = i_lo + t, st = t % C::kStages;
        const uint32_t ph = (t / C::kStages) & 1;
        if (!mbar_wait(&q_empty[st], ph ^ 1, abort_flag)) { ok = false; break; }
        mbar_arrive_expect_tx(&q_full[st], C::kTileBytes + C::kVecFloats * 4);
        for (int ch = 0; ch < C::kChunks; ++ch)
          tma_load_3d(sQ + st * C::kTileBytes + ch * C::kChunkBytes, &tm_q, &q_full[st], ch * 64,
                      i * kBM, bh);
        float *vec = sVec + st * C::kVecFloats;
        bulk_load_1d(vec, p.lse2 + vec_row + i * kBM, kBM * 4, &q_full[st]);
        bulk_load_1d(vec + kBM, p.dvec + vec_row + i * kBM, kBM * 4, &q_full[st]);
        ++q_loads;
        if (!mbar_wait(&do_empty[st], ph ^ 1, abort_flag)) { ok = false; break; }
        mbar_arrive_expect_tx(&do_full[st], C::kTileBytes);
        for (int ch = 0; ch < C::kChunks; ++ch)
          tma_load_3d(sDO + st * C::kTileBytes + ch * C::kChunkBytes, &tm_do, &do_full[st],
                      ch * 64, i * kBM, bh);
        ++do_loads;
      }
      if (!ok) {
        // abandoned: every copy already issued lands before the CTA's shared memory goes away
        volatile int never = 0;
        mbar_wait(kv_full, 0, &never);
        for (int t = q_loads - C::kStages; t < q_loads; ++t)
          if (t >= 0) mbar_wait(&q_full[t % C::kStages], (t / C::kStages) & 1, &never);
        for (int t = do_loads - C::kStages; t < do_loads; ++t)
          if (t >= 0) mbar_wait(&do_full[t % C::kStages], (t / C::kStages) & 1, &never);
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------------ MMA issuer
    // Per query block t: S^T_t+1 as soon as the compute warps have copied S^T_t out, then
    // dV += P^T_t dO_t, dK += dS^T_t Q_t, dQ_t = dS_t K, then dP^T_t+1.
    if (lane == 0) {
      const uint32_t sK0 = smem_u32(sK), sV0 = smem_u32(sV), sQ0 = smem_u32(sQ);
      const uint32_t sDO0 = smem_u32(sDO), sX0 = smem_u32(sX);
      auto issue_s = [&](int t) -> bool {  // S^T_t = K_j Q_t^T
        const int st = t % C::kStages;
        if (!mbar_wait(&q_full[st], (t / C::kStages) & 1, abort_flag)) return false;
        if (t > 0 && !mbar_wait(s_free, (t - 1) & 1, abort_flag)) return false;
        tc_fence_after();
        issue_qk<HD>(tmem + C::kColS, sK0, sQ0 + st * C::kTileBytes);
        umma_commit(s_full);
        return true;
      };
      auto issue_dp = [&](int t) -> bool {  // dP^T_t = V_j dO_t^T
        const int st = t % C::kStages;
        if (!mbar_wait(&do_full[st], (t / C::kStages) & 1, abort_flag)) return false;
        // at d = 128 these columns held dQ_t-1: it must have been read out
        if (C::kDqOnDp && t > 0 && !mbar_wait(dq_free, (t - 1) & 1, abort_flag)) return false;
        tc_fence_after();
        issue_qk<HD>(tmem + C::kColDP, sV0, sDO0 + st * C::kTileBytes);
        umma_commit(dp_full);
        return true;
      };
      bool ok = mbar_wait(kv_full, 0, abort_flag) && issue_s(0) && issue_dp(0);
      for (int t = 0; ok && t < n; ++t) {
        const int st = t % C::kStages;
        if (t + 1 < n && !issue_s(t + 1)) { ok = false; break; }
        if (!mbar_wait(p_full, t & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        issue_x_kmajor<HD>(tmem + C::kColDV, sX0, sDO0 + st * C::kTileBytes, C::kIdescKV, t > 0);
        umma_commit(dv_done);
        umma_commit(&do_empty[st]);
        if (!mbar_wait(ds_full, t & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        issue_x_kmajor<HD>(tmem + C::kColDK, sX0, sQ0 + st * C::kTileBytes, C::kIdescKV, t > 0);
        umma_commit(&q_empty[st]);
        if (!C::kDqOnDp && t > 0 && !mbar_wait(dq_free, (t - 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        issue_dq<HD>(tmem + C::kColDQ, sX0, sK0);
        umma_commit(dq_full);
        umma_commit(x_free);
        if (t + 1 < n && !issue_dp(t + 1)) { ok = false; break; }
      }
      // every MMA issued by this thread completes before TMEM is released
      umma_commit(drain);
      volatile int never = 0;
      mbar_wait(drain, 0, &never);
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------------ compute: P^T, dS^T
    const int r = threadIdx.x;  // key row within the block == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t tS = tmem + lane_off + C::kColS, tDP = tmem + lane_off + C::kColDP;
    const float sl2 = p.scale_log2;
    const bool key_live = jb * kBN + r < p.N;  // keys past N (zero-filled rows) get P = 0
    bool ok = true;
    for (int t = 0; t < n; ++t) {
      const int i = i_lo + t, st = t % C::kStages;
      const float *vlse = sVec + st * C::kVecFloats, *vd = vlse + kBM;
      if (!__all_sync(0xffffffffu, mbar_wait(s_full, t & 1, abort_flag))) { ok = false; break; }
      // S^T_t was computed from this stage, so it has landed; waiting makes its LSE2 / D rows
      // visible to these threads
      if (!__all_sync(0xffffffffu, mbar_wait(&q_full[st], (t / C::kStages) & 1, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      float s[kBN];
      tmem_ld32(tS + 0, reinterpret_cast<uint32_t *>(s));
      tmem_ld32(tS + 32, reinterpret_cast<uint32_t *>(s) + 32);
      tmem_ld32(tS + 64, reinterpret_cast<uint32_t *>(s) + 64);
      tmem_ld32(tS + 96, reinterpret_cast<uint32_t *>(s) + 96);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_free);
      // P^T row: p_c = 2^(s_c scale log2(e) - LSE2_c); on the diagonal block (causal) key r is
      // visible to query c only if r <= c
      const bool diag = p.causal && i == jb;
      uint32_t pk[kBN / 2];
#pragma unroll
      for (int c = 0; c < kBN; c += 2) {
        float p0 = ex2(fmaf(s[c], sl2, -vlse[c]));
        float p1 = ex2(fmaf(s[c + 1], sl2, -vlse[c + 1]));
        if (!key_live || (diag && c < r)) p0 = 0.f;
        if (!key_live || (diag && c + 1 < r)) p1 = 0.f;
        pk[c / 2] = pack_bf16x2(p0, p1);
      }
      if (t > 0 && !__all_sync(0xffffffffu, mbar_wait(x_free, (t - 1) & 1, abort_flag))) {
        ok = false;
        break;
      }
      store_p_row(sX, r, pk);
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
      // dS^T row: ds_c = p_c (dP_c - D_c), with the bf16 p the tensor core used for dV
      if (!__all_sync(0xffffffffu, mbar_wait(dp_full, t & 1, abort_flag))) { ok = false; break; }
      tc_fence_after();
      uint32_t dk[kBN / 2];
#pragma unroll
      for (int cc = 0; cc < kBN; cc += 32) {
        uint32_t dp[32];
        tmem_ld32(tDP + cc, dp);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const uint32_t pp = pk[(cc + e) / 2];
          const float p0 = __uint_as_float(pp << 16), p1 = __uint_as_float(pp & 0xffff0000u);
          const float d0 = p0 * (__uint_as_float(dp[e]) - vd[cc + e]);
          const float d1 = p1 * (__uint_as_float(dp[e + 1]) - vd[cc + e + 1]);
          dk[(cc + e) / 2] = pack_bf16x2(d0, d1);
        }
      }
      tc_fence_before();
      if (!__all_sync(0xffffffffu, mbar_wait(dv_done, t & 1, abort_flag))) { ok = false; break; }
      store_p_row(sX, r, dk);
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(ds_full);
    }
    // epilogue: dV_j and dK_j (times scale) once every MMA of the loop has completed
    if (ok && __all_sync(0xffffffffu, mbar_wait(x_free, (n - 1) & 1, abort_flag))) {
      tc_fence_after();
      const size_t grow = static_cast<size_t>(bh) * p.N + jb * kBN + r;
      store_grad_row<HD>(tmem + lane_off + C::kColDV, 1.f, p.dv, p.g_f32, grow, key_live);
      store_grad_row<HD>(tmem + lane_off + C::kColDK, p.scale, p.dk, p.g_f32, grow, key_live);
    }
  } else {
    // ------------------------------------------------------------------ dQ read-out
    const int qr = threadIdx.x - 128;  // query row within the block == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp % 4) * 32) << 16;
    const uint32_t tQ = tmem + lane_off + C::kColDQ;
    for (int t = 0; t < n; ++t) {
      const int row = (i_lo + t) * kBM + qr;
      if (!__all_sync(0xffffffffu, mbar_wait(dq_full, t & 1, abort_flag))) break;
      tc_fence_after();
      float *dst = p.dq_acc + (static_cast<size_t>(bh) * p.Np + row) * HD;
#pragma unroll
      for (int cc = 0; cc < HD; cc += 32) {
        uint32_t v[32];
        tmem_ld32(tQ + cc, v);
        tmem_wait_ld();
        if (row < p.N) {
#pragma unroll
          for (int e = 0; e < 8; ++e)
            atomicAdd(reinterpret_cast<float4 *>(dst + cc + 4 * e),
                      make_float4(__uint_as_float(v[4 * e]), __uint_as_float(v[4 * e + 1]),
                                  __uint_as_float(v[4 * e + 2]), __uint_as_float(v[4 * e + 3])));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(dq_free);
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(*tmem_slot, C::kTmemCols);
  }
}

// D_i = sum_c dO[i,c] O[i,c] and LSE2_i = LSE_i log2(e) for every row of the padded [BH, Np]
// layout (padding rows: D = 0, LSE2 = +inf so that their P is 0), and the dQ accumulator row
// cleared.  HD / 8 threads per row, 8 elements each; O is bf16 or (kOF32) fp32.
template <int HD, bool kOF32>
__global__ void __launch_bounds__(256) fa_bwd_prep_kernel(const void *__restrict__ o,
                                                          const uint16_t *__restrict__ dout,
                                                          const float *__restrict__ lse, float *lse2,
                                                          float *dvec, float *dq_acc, int BH, int N,
                                                          int Np) {
  constexpr int kT = HD / 8;
  const long long gt = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long row = gt / kT;
  const int part = static_cast<int>(gt % kT);
  const bool in_range = row < static_cast<long long>(BH) * Np;
  const int bh = in_range ? static_cast<int>(row / Np) : 0;
  const int nrow = in_range ? static_cast<int>(row % Np) : 0;
  const bool live = in_range && nrow < N;
  float acc = 0.f;
  if (live) {
    const size_t off = (static_cast<size_t>(bh) * N + nrow) * HD + part * 8;
    const uint4 b = *reinterpret_cast<const uint4 *>(dout + off);
    const uint32_t bv[4] = {b.x, b.y, b.z, b.w};
    float ov[8];
    if constexpr (kOF32) {
      const float4 a0 = reinterpret_cast<const float4 *>(static_cast<const float *>(o) + off)[0];
      const float4 a1 = reinterpret_cast<const float4 *>(static_cast<const float *>(o) + off)[1];
      ov[0] = a0.x; ov[1] = a0.y; ov[2] = a0.z; ov[3] = a0.w;
      ov[4] = a1.x; ov[5] = a1.y; ov[6] = a1.z; ov[7] = a1.w;
    } else {
      const uint4 a = *reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(o) + off);
      const uint32_t av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        ov[2 * e] = __uint_as_float(av[e] << 16);
        ov[2 * e + 1] = __uint_as_float(av[e] & 0xffff0000u);
      }
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      acc = fmaf(ov[2 * e], __uint_as_float(bv[e] << 16), acc);
      acc = fmaf(ov[2 * e + 1], __uint_as_float(bv[e] & 0xffff0000u), acc);
    }
  }
#pragma unroll
  for (int off = kT / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (!in_range) return;
  if (part == 0) {
    dvec[row] = live ? acc : 0.f;
    lse2[row] = live ? lse[static_cast<size_t>(bh) * N + nrow] * 1.4426950408889634f : INFINITY;
  }
  float4 *z = reinterpret_cast<float4 *>(dq_acc + row * HD + part * 8);
  z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
  z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// dQ = scale * accumulator, rows < N, to bf16 or fp32.  8 elements per thread.
template <int HD>
__global__ void __launch_bounds__(256) fa_bwd_dq_kernel(const float *__restrict__ dq_acc, void *dq,
                                                        int f32, float scale, int BH, int N, int Np) {
  constexpr int kT = HD / 8;
  const long long gt = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long row = gt / kT;  // over BH * N
  if (row >= static_cast<long long>(BH) * N) return;
  const int part = static_cast<int>(gt % kT);
  const long long bh = row / N, nrow = row % N;
  const float4 *src = reinterpret_cast<const float4 *>(dq_acc + (bh * Np + nrow) * HD + part * 8);
  const float4 a = src[0], b = src[1];
  const size_t off = static_cast<size_t>(row) * HD + part * 8;
  if (f32) {
    float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(dq) + off);
    dst[0] = make_float4(a.x * scale, a.y * scale, a.z * scale, a.w * scale);
    dst[1] = make_float4(b.x * scale, b.y * scale, b.z * scale, b.w * scale);
  } else {
    uint4 w;
    w.x = pack_bf16x2(a.x * scale, a.y * scale);
    w.y = pack_bf16x2(a.z * scale, a.w * scale);
    w.z = pack_bf16x2(b.x * scale, b.y * scale);
    w.w = pack_bf16x2(b.z * scale, b.w * scale);
    *reinterpret_cast<uint4 *>(static_cast<uint16_t *>(dq) + off) = w;
  }
}

}  // namespace fa
