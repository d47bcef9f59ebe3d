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
// Work partition: a (b, h, key block j of 128 keys) sub-unit keeps K_j and V_j in shared memory,
// streams every query block i that sees them (i >= j when causal) and keeps dK_j and dV_j in TMEM
// for the whole loop.  dQ_i gets one 128 x d partial per (i, j) pair, added into an fp32
// accumulator in global memory.  The kernel is persistent (at most one CTA per SM): each CTA
// walks its sub-units in turn, so the next K_j, V_j and query blocks load, and the next block's
// S^T and dP^T run on the tensor core, while the compute warps write the previous dK_j, dV_j.
//
// The scores are computed transposed, S^T = K_j Q_i^T (TMEM lane = key), so each compute thread
// owns one key row: P^T and dS^T are written by rows into one 128 x 128 bf16 tile X in the
// 128-byte-swizzled layout the tensor core reads.  X is the K-major A operand of dV += P^T dO and
// dK += dS^T Q, and, read through MN-major descriptors, an operand of the dQ product.  At d = 128
// that product is dQ^T = K_j^T dS^T (TMEM lane = feature), so the read-out adds 32 consecutive
// floats of one dQ row per warp instruction; at d = 64 it is dQ = dS K_j (lane = query).
//
//   warps 0-3, 4-7  compute, one key row per thread, query columns [0,64) and [64,128): P^T and
//                   dS^T, and each sub-unit's dK, dV write
//   warps 8-11      dQ read-out: TMEM -> a shared-memory staging box -> a bulk tensor reduction
//                   (fp32 add) into the accumulator, one box of 32 features per warp at a time
//   warp  12        TMA producer: K_j, V_j per sub-unit; Q_i (+ its LSE and D rows), dO_i per
//                   query block
//   warp  13        MMA issuer (one thread) + TMEM owner
// TMEM (512 columns): S^T [0,128)  dP^T [128,256)  dV [256,256+d)  dK [256+d,256+2d); dQ at
// [256+2d, 256+3d) when d = 64, and in S^T's columns when d = 128 (they are full otherwise).
// MMA order per query block t: dV_t, S^T_t+1, dK_t, dQ_t, dP^T_t+1 -- so that the tensor core has
// the next block's products queued while the compute warps turn S^T into P^T and dP^T into dS^T.
#pragma once
#include "fa_prefill.cuh"

namespace fa {

constexpr int kBwdThreads = 448;
constexpr size_t kMaxDynSmem = 232448;  // 227 KB per CTA on sm_100

template <int HD>
struct BwdCfg {
  static_assert(HD == 64 || HD == 128, "head dim");
  static constexpr int kChunks = HD / 64;
  static constexpr int kChunkBytes = 128 * 128;
  static constexpr int kTileBytes = 128 * HD * 2;
  static constexpr int kXBytes = 128 * 128 * 2;
  static constexpr int kStages = 2;                // Q ring
  static constexpr int kDoStages = HD == 128 ? 1 : 2;  // dO ring (one stage frees room at d = 128)
  // dQ staging: one 8 KB slot per read-out warp, boxes of 32 features x 32 rows (4 KB), fp32,
  // 128-byte swizzle.  d = 128: the slot's two halves take the warp's boxes in turn (one is
  // written while the other is read by its reduction; 32-row boxes measured faster than 64, 16 or
  // 8); d = 64: the warp's two boxes of its 32 query rows.
  static constexpr int kBoxRows = 32;
  static constexpr int kStageSlotBytes = 8192;
  static constexpr int kVecFloats = 2 * kBM;       // LSE (log2 units) and D of one query block
  static constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 256 + HD;
  static constexpr bool kDqT = HD == 128;          // dQ^T in S^T's columns (lane = feature)
  static constexpr uint32_t kColDQ = kDqT ? kColS : 256 + 2 * HD;
  static constexpr int kTmemCols = 512;
  static constexpr int kNumBars = 2 + 2 * kStages + 2 * kDoStages + 9;
  static constexpr size_t kBodyBytes = 2 * kTileBytes + (kStages + kDoStages) * kTileBytes +
                                       kXBytes + 4 * kStageSlotBytes + kStages * kVecFloats * 4 +
                                       kNumBars * 8 + 16;
  // up to 1 KB of slack to align the tiles to the 1024-byte swizzle atom
  static constexpr size_t kSmemBytes =
      kBodyBytes + 1024 <= kMaxDynSmem ? kBodyBytes + 1024 : kMaxDynSmem;
  static_assert(kBodyBytes <= kMaxDynSmem, "shared memory budget");
  static_assert(kColDQ + (kDqT ? 0 : HD) <= kTmemCols, "TMEM budget");
  static constexpr uint32_t kIdescKV = idesc_bf16_f32(128, HD, 0, 1);  // X K-major, Q/dO MN-major
  // dQ^T (d = 128): A = K^T MN-major (m = feature), B = dS^T MN-major (n = query);
  // dQ (d = 64): A = dS MN-major (m = query), B = K MN-major (n = feature)
  static constexpr uint32_t kIdescQ = kDqT ? idesc_bf16_f32(HD, 128, 1, 1)
                                           : idesc_bf16_f32(128, HD, 1, 1);
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

// The dQ product over the 128 keys of the block, both operands MN-major with the key as K:
// d = 128: dQ^T = K^T dS^T (A from the K tile, B from X); d = 64: dQ = dS K (A from X, B from K).
template <int HD>
__device__ __forceinline__ void issue_dq(uint32_t d_tmem, uint32_t x_smem, uint32_t k_smem) {
  using C = BwdCfg<HD>;
  const uint32_t a_base = C::kDqT ? k_smem : x_smem, b_base = C::kDqT ? x_smem : k_smem;
#pragma unroll
  for (int kk = 0; kk < 128 / 16; ++kk) {
    const uint64_t a = smem_desc_sw128(a_base + kk * 16 * 128, 16384, 1024);
    const uint64_t b = smem_desc_sw128(b_base + kk * 16 * 128, 16384, 1024);
    umma_ss(d_tmem, a, b, C::kIdescQ, kk > 0 ? 1u : 0u);
  }
}

// Half a row of X (this thread's key row r, query columns [64 h, 64 h + 64) = swizzle chunk h):
// 32 packed bf16 pairs, the 16-byte unit u stored at unit u ^ (r % 8).
__device__ __forceinline__ void store_x_half(uint8_t *x_tile, int r, int h, const uint32_t (&pk)[32]) {
  uint8_t *rowp = x_tile + h * 16384 + r * 128;
#pragma unroll
  for (int u = 0; u < 8; ++u)
    *reinterpret_cast<uint4 *>(rowp + ((u ^ (r & 7)) * 16)) =
        make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
}

// Columns [c0, c0 + 32 * NCH) of this thread's TMEM row, times `mul`, to global row `grow`.
template <int HD, int NCH>
__device__ __forceinline__ void store_grad_cols(uint32_t taddr, int c0, float mul, void *dst_base,
                                                int f32, size_t grow, bool live) {
#pragma unroll
  for (int ch = 0; ch < NCH; ++ch) {
    const int cc = c0 + 32 * ch;
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

// Add dQ_i's partial (TMEM) into the accumulator through this read-out warp's staging slot.
// Warp w (0..3) reads TMEM lanes 32 w .. 32 w + 31 and owns the boxes those lanes fill:
//   d = 128 (dQ^T, lane = feature f = 32 w + lane): two boxes of 64 query rows x 32 features; each
//           query column of TMEM becomes one 128-byte row of the box (one 4-byte store per lane).
//   d = 64  (dQ, lane = query 32 w + lane): two boxes of the warp's 32 query rows x 32 features;
//           each thread stores its row (8 x 16 bytes).
// Stores use the 128-byte swizzle of the tensor map (16-byte unit u of row r at u ^ (r % 8)).
// The dQ columns are released (dq_free) as soon as TMEM has been read; the slot is reused once the
// bulk reduction has finished reading it.
template <int HD>
__device__ __forceinline__ void read_out_dq(uint32_t tq, int w, int lane, uint8_t *slot,
                                            const CUtensorMap *tm_dq, int row0, uint64_t *dq_free) {
  using C = BwdCfg<HD>;
  if constexpr (C::kDqT) {
    // boxes of kBoxRows query rows, cycling through the slot's kBufs buffers: a box is written
    // while the kBufs - 1 before it are still being read by their reductions
    constexpr int kRows = C::kBoxRows, kBufs = C::kStageSlotBytes / (kRows * 128);
#pragma unroll 1
    for (int q0 = 0; q0 < kBM; q0 += 32) {
      uint32_t v[32];
      tmem_ld32(tq + q0, v);
      tmem_wait_ld();
      if (q0 + 32 == kBM) {  // TMEM fully read: the columns may take the next block's S^T
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(dq_free);
      }
#pragma unroll
      for (int b0 = 0; b0 < 32; b0 += kRows) {
        const int bi = (q0 + b0) / kRows;
        if (lane == 0) bulk_wait_group_read<kBufs - 1>();  // this buffer's last box has left it
        __syncwarp();
        uint8_t *box = slot + (bi % kBufs) * (kRows * 128);
        const int unit = lane / 4, sub = (lane % 4) * 4;
#pragma unroll
        for (int q = 0; q < kRows; ++q)
          *reinterpret_cast<float *>(box + q * 128 + ((unit ^ (q & 7)) * 16) + sub) =
              __uint_as_float(v[b0 + q]);
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_reduce_add_2d(tm_dq, box, 32 * w, row0 + q0 + b0);
          bulk_commit_group();
        }
      }
    }
  } else {
    uint32_t v[2][32];
    tmem_ld32(tq, v[0]);
    tmem_ld32(tq + 32, v[1]);
    tmem_wait_ld();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(dq_free);
    if (lane == 0) bulk_wait_group_read<0>();
    __syncwarp();
#pragma unroll
    for (int fg = 0; fg < 2; ++fg) {
      uint8_t *rowp = slot + fg * 4096 + lane * 128;
#pragma unroll
      for (int u = 0; u < 8; ++u)
        *reinterpret_cast<uint4 *>(rowp + ((u ^ (lane & 7)) * 16)) =
            make_uint4(v[fg][4 * u], v[fg][4 * u + 1], v[fg][4 * u + 2], v[fg][4 * u + 3]);
    }
    fence_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_reduce_add_2d(tm_dq, slot, 0, row0 + 32 * w);
      tma_reduce_add_2d(tm_dq, slot + 4096, 32, row0 + 32 * w);
      bulk_commit_group();
    }
  }
}

template <int HD>
__global__ void __launch_bounds__(kBwdThreads, 1)
    fa_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                  const __grid_constant__ CUtensorMap tm_dq,
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
  uint8_t *sDO = sQ + C::kStages * C::kTileBytes;   // kDoStages tiles
  uint8_t *sX = sDO + C::kDoStages * C::kTileBytes; // P^T, then dS^T
  uint8_t *sStage = sX + C::kXBytes;                // 4 dQ staging slots
  float *sVec = reinterpret_cast<float *>(sStage + 4 * C::kStageSlotBytes);  // [kStages][LSE2 | D]
  uint64_t *bars = reinterpret_cast<uint64_t *>(sVec + C::kStages * C::kVecFloats);
  uint64_t *kv_full = bars;                    // K_j, V_j landed
  uint64_t *q_full = bars + 1;                 // [kStages] Q_i + its LSE2 / D rows landed
  uint64_t *q_empty = q_full + C::kStages;     // [kStages] dK_i done (last reader of Q_i)
  uint64_t *do_full = q_empty + C::kStages;    // [kDoStages] dO_i landed
  uint64_t *do_empty = do_full + C::kDoStages; // [kDoStages] dV_i done (last reader of dO_i)
  uint64_t *s_full = do_empty + C::kDoStages;  // S^T_i computed
  uint64_t *s_free = s_full + 1;               // S^T_i copied out (8 warp arrivals)
  uint64_t *dp_full = s_free + 1;              // dP^T_i computed
  uint64_t *p_full = dp_full + 1;              // P^T_i written to X (8 warp arrivals)
  uint64_t *dv_done = p_full + 1;              // dV += P^T_i dO_i done: X may take dS^T_i
  uint64_t *ds_full = dv_done + 1;             // dS^T_i written to X (8 warp arrivals)
  uint64_t *dq_full = ds_full + 1;             // dK_i and dQ_i done: dQ_i readable, X free
  uint64_t *dq_free = dq_full + 1;             // dQ_i read out (4 warp arrivals)
  uint64_t *drain = dq_free + 1;
  uint64_t *kv_empty = drain + 1;              // every product that reads K_j, V_j has completed
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(kv_empty + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  // Persistent schedule.  The CTA takes pairs of key blocks (jb, nkb - 1 - jb) of one head, pair
  // pu = blockIdx.x + m * gridDim.x (head-major), and processes the two as consecutive sub-units,
  // the smaller jb first.  With the causal mask key block jb sees nkb - jb query blocks, so every
  // pair costs the same nkb + 1 blocks and the round-robin deal is balanced; the CTAs running at
  // the same time cover few heads, whose Q, dO and dQ rows stay in L2.
  // sub_unit(k, bh, jb): 1 with (bh, jb) set, 0 once the CTA has no more, -1 for the empty second
  // half of the middle pair (odd nkb).  Every role walks the same sequence.
  const int npairs = (p.nkb + 1) / 2;
  const int total_pairs = p.BH * npairs;
  auto sub_unit = [&](int k, int &bh, int &jb) -> int {
    const int pu = static_cast<int>(blockIdx.x) + (k / 2) * static_cast<int>(gridDim.x);
    if (pu >= total_pairs) return 0;
    bh = pu / npairs;
    const int pp = pu % npairs;
    jb = (k & 1) ? p.nkb - 1 - pp : pp;
    return ((k & 1) && jb == pp) ? -1 : 1;
  };
  // Query blocks of key block jb (>= 1) and their visit order: step t takes query block
  // i_lo + (t + rot) mod n.  Without the mask rot = jb staggers the key blocks of one head, so the
  // CTAs adding into that head's dQ do not reduce into the same rows at the same moment (with it,
  // i_lo = jb already staggers them).
  struct Span {
    int i_lo, n, rot;
  };
  auto span_of = [&](int jb) -> Span {
    const int i_lo = p.causal ? jb : 0;
    const int n = p.Np / kBM - i_lo;
    return {i_lo, n, p.causal ? 0 : jb % n};
  };
  // Barrier phases run over the CTA's whole sequence of query blocks: block t of a sub-unit whose
  // first block is the CTA's T-th has the global index T + t.

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    mbar_init(kv_empty, 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 1);
    }
    for (int s = 0; s < C::kDoStages; ++s) {
      mbar_init(&do_full[s], 1);
      mbar_init(&do_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, 8);
    mbar_init(dp_full, 1);
    mbar_init(p_full, 8);
    mbar_init(dv_done, 1);
    mbar_init(ds_full, 8);
    mbar_init(dq_full, 1);
    mbar_init(dq_free, 4);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 13) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  if (warp == 12 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_do);
    tma_prefetch_desc(&tm_dq);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 12) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      bool ok = true;
      int q_loads = 0, do_loads = 0, kv_loads = 0;  // loads issued so far (= their global index)
      for (int k = 0; ok; ++k) {
        int bh, jb;
        const int su = sub_unit(k, bh, jb);
        if (su == 0) break;
        if (su < 0) continue;
        const Span sp = span_of(jb);
        // K_j, V_j once every product of the previous sub-unit that read its K and V has completed.
        // After the first sub-unit the query block t = 0 goes first: its Q and dO stages free up
        // before the previous sub-unit's last dQ product releases K and V.
        auto load_kv = [&]() -> bool {
          if (kv_loads > 0 && !mbar_wait(kv_empty, (kv_loads - 1) & 1, abort_flag)) return false;
          mbar_arrive_expect_tx(kv_full, 2 * C::kTileBytes);
          for (int ch = 0; ch < C::kChunks; ++ch) {
            tma_load_3d(sK + ch * C::kChunkBytes, &tm_k, kv_full, ch * 64, jb * kBN, bh);
            tma_load_3d(sV + ch * C::kChunkBytes, &tm_v, kv_full, ch * 64, jb * kBN, bh);
          }
          ++kv_loads;
          return true;
        };
        bool kv_issued = false;
        if (kv_loads == 0) {
          if (!load_kv()) { ok = false; break; }
          kv_issued = true;
        }
        const size_t vec_row = static_cast<size_t>(bh) * p.Np;
        for (int t = 0; t < sp.n; ++t) {
          const int i = sp.i_lo + (t + sp.rot) % sp.n;
          const int g = q_loads, st = g % C::kStages;
          const uint32_t ph = (g / C::kStages) & 1;
          if (!mbar_wait(&q_empty[st], ph ^ 1, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(&q_full[st], C::kTileBytes + C::kVecFloats * 4);
          for (int ch = 0; ch < C::kChunks; ++ch)
            tma_load_3d(sQ + st * C::kTileBytes + ch * C::kChunkBytes, &tm_q, &q_full[st], ch * 64,
                        i * kBM, bh);
          float *vec = sVec + st * C::kVecFloats;
          bulk_load_1d(vec, p.lse2 + vec_row + i * kBM, kBM * 4, &q_full[st]);
          bulk_load_1d(vec + kBM, p.dvec + vec_row + i * kBM, kBM * 4, &q_full[st]);
          ++q_loads;
          const int sd = g % C::kDoStages;
          if (!mbar_wait(&do_empty[sd], ((g / C::kDoStages) & 1) ^ 1, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(&do_full[sd], C::kTileBytes);
          for (int ch = 0; ch < C::kChunks; ++ch)
            tma_load_3d(sDO + sd * C::kTileBytes + ch * C::kChunkBytes, &tm_do, &do_full[sd],
                        ch * 64, i * kBM, bh);
          ++do_loads;
          if (!kv_issued) {
            if (!load_kv()) { ok = false; break; }
            kv_issued = true;
          }
        }
      }
      if (!ok) {
        // abandoned: every copy already issued lands before the CTA's shared memory goes away
        // (a K/V load is issued only after the previous one was consumed, so the last alone can
        // be in flight)
        volatile int never = 0;
        if (kv_loads > 0) mbar_wait(kv_full, (kv_loads - 1) & 1, &never);
        for (int t = q_loads - C::kStages; t < q_loads; ++t)
          if (t >= 0) mbar_wait(&q_full[t % C::kStages], (t / C::kStages) & 1, &never);
        for (int t = do_loads - C::kDoStages; t < do_loads; ++t)
          if (t >= 0) mbar_wait(&do_full[t % C::kDoStages], (t / C::kDoStages) & 1, &never);
      }
    }
  } else if (warp == 13) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t sK0 = smem_u32(sK), sV0 = smem_u32(sV), sQ0 = smem_u32(sQ);
      const uint32_t sDO0 = smem_u32(sDO), sX0 = smem_u32(sX);
      // S^T_g = K_j Q_g^T into S^T's columns.  At d = 128 those columns also take the dQ^T
      // partials.  Within a sub-unit S^T_g is issued before dQ^T_g-1 (which waits for S^T_g to be
      // copied out), so S^T_g waits for dQ^T_g-2 to be read out; the first block of a sub-unit
      // comes after the previous sub-unit's last dQ^T, g - 1, and waits for that one.
      auto issue_s = [&](int g, bool first) -> bool {
        const int st = g % C::kStages;
        if (!mbar_wait(&q_full[st], (g / C::kStages) & 1, abort_flag)) return false;
        if (g > 0 && !mbar_wait(s_free, (g - 1) & 1, abort_flag)) return false;
        const int dq_prev = first ? g - 1 : g - 2;
        if (C::kDqT && dq_prev >= 0 && !mbar_wait(dq_free, dq_prev & 1, abort_flag)) return false;
        tc_fence_after();
        issue_qk<HD>(tmem + C::kColS, sK0, sQ0 + st * C::kTileBytes);
        umma_commit(s_full);
        return true;
      };
      auto issue_dp = [&](int g) -> bool {  // dP^T_g = V_j dO_g^T (dS^T_g-1 already formed)
        const int sd = g % C::kDoStages;
        if (!mbar_wait(&do_full[sd], (g / C::kDoStages) & 1, abort_flag)) return false;
        tc_fence_after();
        issue_qk<HD>(tmem + C::kColDP, sV0, sDO0 + sd * C::kTileBytes);
        umma_commit(dp_full);
        return true;
      };
      bool ok = true;
      int T = 0, kv_used = 0;
      for (int k = 0; ok; ++k) {
        int bh, jb;
        const int su = sub_unit(k, bh, jb);
        if (su == 0) break;
        if (su < 0) continue;
        const int n = span_of(jb).n;
        ok = mbar_wait(kv_full, kv_used & 1, abort_flag) && issue_s(T, true) && issue_dp(T);
        ++kv_used;
        for (int t = 0; ok && t < n; ++t) {
          const int g = T + t, st = g % C::kStages, sd = g % C::kDoStages;
          if (!mbar_wait(p_full, g & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          issue_x_kmajor<HD>(tmem + C::kColDV, sX0, sDO0 + sd * C::kTileBytes, C::kIdescKV, t > 0);
          umma_commit(dv_done);
          umma_commit(&do_empty[sd]);
          if (t + 1 < n && !issue_s(g + 1, false)) { ok = false; break; }
          if (!mbar_wait(ds_full, g & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          issue_x_kmajor<HD>(tmem + C::kColDK, sX0, sQ0 + st * C::kTileBytes, C::kIdescKV, t > 0);
          umma_commit(&q_empty[st]);
          // dQ_g-1 must have been read out of the dQ columns
          if (g > 0 && !mbar_wait(dq_free, (g - 1) & 1, abort_flag)) { ok = false; break; }
          if constexpr (C::kDqT) {
            // dQ^T_g goes where S^T_g+1 sits: wait until the compute warps have copied it out
            const int last_s = t + 1 < n ? g + 1 : g;
            if (!mbar_wait(s_free, last_s & 1, abort_flag)) { ok = false; break; }
          }
          tc_fence_after();
          issue_dq<HD>(tmem + C::kColDQ, sX0, sK0);
          umma_commit(dq_full);
          if (t + 1 < n && !issue_dp(g + 1)) { ok = false; break; }
        }
        if (!ok) break;
        umma_commit(kv_empty);  // K_j and V_j are free once every product of the sub-unit has completed
        T += n;
      }
      // every MMA issued by this thread completes before TMEM is released
      umma_commit(drain);
      volatile int never = 0;
      mbar_wait(drain, 0, &never);
    }
  } else if (warp >= 8) {
    // ------------------------------------------------------------------ dQ read-out
    const int w4 = warp % 4;
    const uint32_t tQ = tmem + (static_cast<uint32_t>(w4 * 32) << 16) + C::kColDQ;
    uint8_t *slot = sStage + w4 * C::kStageSlotBytes;
    bool ok = true;
    int T = 0;
    for (int k = 0; ok; ++k) {
      int bh, jb;
      const int su = sub_unit(k, bh, jb);
      if (su == 0) break;
      if (su < 0) continue;
      const Span sp = span_of(jb);
      const int row_head = bh * p.Np;  // the head's first row in the accumulator's [BH * Np, d] view
      for (int t = 0; t < sp.n; ++t) {
        const int i = sp.i_lo + (t + sp.rot) % sp.n;
        if (!__all_sync(0xffffffffu, mbar_wait(dq_full, (T + t) & 1, abort_flag))) { ok = false; break; }
        tc_fence_after();
        read_out_dq<HD>(tQ, w4, lane, slot, &tm_dq, row_head + i * kBM, dq_free);
      }
      T += sp.n;
    }
    if (lane == 0) bulk_wait_group_all();  // every reduction has landed before the CTA retires
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ compute: P^T, dS^T
    const int h = warp / 4;                   // query columns [64 h, 64 h + 64)
    const int w4 = warp % 4;
    const int r = threadIdx.x % 128;          // key row within the block == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(w4 * 32) << 16;
    const uint32_t tS = tmem + lane_off + C::kColS + 64 * h;
    const uint32_t tDP = tmem + lane_off + C::kColDP + 64 * h;
    const uint64_t sl2x2 = f2_pack(p.scale_log2, p.scale_log2);
    bool ok = true;
    int T = 0;
    for (int k = 0; ok; ++k) {
      int bh, jb;
      const int su = sub_unit(k, bh, jb);
      if (su == 0) break;
      if (su < 0) continue;
      const Span sp = span_of(jb);
      const int n = sp.n;
      const bool key_live = jb * kBN + r < p.N;  // keys past N (zero-filled rows) get P = 0
      const bool ragged_keys = (jb + 1) * kBN > p.N;
      for (int t = 0; t < n; ++t) {
        const int g = T + t;
        const int i = sp.i_lo + (t + sp.rot) % n, st = g % C::kStages;
        const float *vlse = sVec + st * C::kVecFloats + 64 * h, *vd = vlse + kBM;
        if (!__all_sync(0xffffffffu, mbar_wait(s_full, g & 1, abort_flag))) { ok = false; break; }
        // S^T_g was computed from this stage, so it has landed; waiting makes its LSE2 / D rows
        // visible to these threads
        if (!__all_sync(0xffffffffu, mbar_wait(&q_full[st], (g / C::kStages) & 1, abort_flag))) {
          ok = false;
          break;
        }
        tc_fence_after();
        float s[64];
        tmem_ld32(tS, reinterpret_cast<uint32_t *>(s));
        tmem_ld32(tS + 32, reinterpret_cast<uint32_t *>(s) + 32);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_free);
        // P^T: p = 2^(s scale log2(e) - LSE2_q); on the diagonal block (causal) key r is visible
        // to query q only if r <= q, and keys past N are dropped
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 64; c += 4) {
          const float4 l4 = *reinterpret_cast<const float4 *>(vlse + c);
          const uint64_t x01 = f2_fma(f2_pack(s[c], s[c + 1]), sl2x2, f2_pack(-l4.x, -l4.y));
          const uint64_t x23 = f2_fma(f2_pack(s[c + 2], s[c + 3]), sl2x2, f2_pack(-l4.z, -l4.w));
          float x0, x1, x2, x3;
          f2_unpack(x01, x0, x1);
          f2_unpack(x23, x2, x3);
          s[c] = ex2(x0);
          s[c + 1] = ex2(x1);
          s[c + 2] = ex2(x2);
          s[c + 3] = ex2(x3);
        }
        if ((p.causal && i == jb) || ragged_keys) {
          const int qmin = r - 64 * h;  // visible iff local column >= qmin (diagonal block)
          const bool diag = p.causal && i == jb;
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (!key_live || (diag && c < qmin)) s[c] = 0.f;
        }
#pragma unroll
        for (int c = 0; c < 32; ++c) pk[c] = pack_bf16x2(s[2 * c], s[2 * c + 1]);
        // X still feeds the previous block's dQ product (the previous sub-unit's last one was
        // waited for before its gradients were written)
        if (t > 0) {
          if (!__all_sync(0xffffffffu, mbar_wait(dq_full, (g - 1) & 1, abort_flag))) { ok = false; break; }
          tc_fence_after();
        }
        store_x_half(sX, r, h, pk);
        fence_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full);
        // dS^T: ds = p (dP - D_q), with the bf16 p the tensor core used for dV
        if (!__all_sync(0xffffffffu, mbar_wait(dp_full, g & 1, abort_flag))) { ok = false; break; }
        tc_fence_after();
        uint32_t dk[32];
#pragma unroll
        for (int cc = 0; cc < 64; cc += 32) {
          uint32_t dp[32];
          tmem_ld32(tDP + cc, dp);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            const float4 d4 = *reinterpret_cast<const float4 *>(vd + cc + e);
            const uint32_t pa = pk[(cc + e) / 2], pb = pk[(cc + e) / 2 + 1];
            const uint64_t g01 = f2_mul(f2_pack(__uint_as_float(pa << 16), __uint_as_float(pa & 0xffff0000u)),
                                        f2_sub(f2_pack(__uint_as_float(dp[e]), __uint_as_float(dp[e + 1])),
                                               f2_pack(d4.x, d4.y)));
            const uint64_t g23 = f2_mul(f2_pack(__uint_as_float(pb << 16), __uint_as_float(pb & 0xffff0000u)),
                                        f2_sub(f2_pack(__uint_as_float(dp[e + 2]), __uint_as_float(dp[e + 3])),
                                               f2_pack(d4.z, d4.w)));
            float a0, a1, a2, a3;
            f2_unpack(g01, a0, a1);
            f2_unpack(g23, a2, a3);
            dk[(cc + e) / 2] = pack_bf16x2(a0, a1);
            dk[(cc + e) / 2 + 1] = pack_bf16x2(a2, a3);
          }
        }
        tc_fence_before();
        if (!__all_sync(0xffffffffu, mbar_wait(dv_done, g & 1, abort_flag))) { ok = false; break; }
        store_x_half(sX, r, h, dk);
        fence_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(ds_full);
      }
      if (!ok) break;
      // dV_j and dK_j (times scale) once every product of the sub-unit has completed.  The next
      // sub-unit's first dV and dK products overwrite these columns; the issuer starts them only
      // after this warp's next P^T / dS^T signals, i.e. after these reads.
      if (!__all_sync(0xffffffffu, mbar_wait(dq_full, (T + n - 1) & 1, abort_flag))) { ok = false; break; }
      tc_fence_after();
      const size_t grow = static_cast<size_t>(bh) * p.N + jb * kBN + r;
      store_grad_cols<HD, HD / 64>(tmem + lane_off + C::kColDV, h * (HD / 2), 1.f, p.dv, p.g_f32,
                                   grow, key_live);
      store_grad_cols<HD, HD / 64>(tmem + lane_off + C::kColDK, h * (HD / 2), p.scale, p.dk,
                                   p.g_f32, grow, key_live);
      tc_fence_before();
      T += n;
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 13) {
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
