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
// B200 mapping (one CTA per SM, 384 threads, persistent over work units):
//   warps 0-3   softmax for query tile 0 of the current pair (one TMEM lane = one query row)
//   warps 4-7   softmax for query tile 1 of the pair; warp w and warp w + 4 share an SM
//               sub-partition and take turns on its exponential unit
//   warp  8     TMA producer: the Q pair once per unit, then K_0, and K_{j+1}, V_j per block
//   warp  9     Q K^T issuer (one thread) + TMEM owner
//   warp  10    P V issuer (one thread); in the paged mode it first ranks the sequences
//   warp  11    idle
// TMEM (512 columns): S0 [0,128)  S1 [128,256)  O0 [256,256+d)  O1 [256+d, 256+2d).
// P_i (bf16) is written by the softmax threads into a shared-memory tile in the layout the tensor
// core reads, so S_i's TMEM columns are free as soon as the softmax has copied S_i,j into
// registers: the Q K^T issuer then computes S_i,j+1 while the softmax is still turning S_i,j into
// P_i,j, and the P V issuer adds O_i += P_i,j V_j when P_i,j is ready.  Each softmax warpgroup
// thus runs back to back, and the two tiles keep the tensor core fed in turn.
// Epilogue: O_i / l_i per row.  In the square and paged modes with bf16 O each warp stages its
// 32 rows in the tile's P buffer (free once the last P V has completed) and writes them with TMA
// tensor stores, so the warp starts the next unit while the stores drain; otherwise every thread
// stores its own row.
#pragma once
#include <type_traits>

#include "sm100_ptx.cuh"

namespace fa {

// Tile store shared -> global through a 3-D tensor map (rows past the map's extent are not
// written); completion is tracked by this thread's bulk groups.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap *map, const void *src, int c0, int c1,
                                             int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

constexpr int kBM = 128;  // query rows per tile
constexpr int kBN = 128;  // keys per key/value block
constexpr int kPrefillThreads = 384;
constexpr float kRescaleLog2 = 8.0f;  // lazy rescale: tolerate a stale max up to 2^8 below
constexpr float kLn2 = 0.6931471805599453f;
// every kPolyEvery-th pair of P's exponentials is evaluated on the FMA pipe, the rest on MUFU
// (0: all MUFU).  Measured on the B200: at d = 128 every share tried (1/8 .. 1/2) was slower; at
// d = 64 a quarter was 14-20% slower once the normaliser sums the rounded values exactly (which
// the polynomial share needs for parity on rows dominated by one key).  So MUFU only.
#ifndef FA_POLY_EVERY
#define FA_POLY_EVERY 0
#endif
template <int HD>
constexpr int kPolyEvery = FA_POLY_EVERY;
#ifndef FA_EXP_TURNS
#define FA_EXP_TURNS 1
#endif

template <int HD>
struct PrefillCfg {
  static_assert(HD == 64 || HD == 128, "head dim");
  static constexpr int kChunks = HD / 64;          // 64-element (128-byte) swizzle chunks per row
  static constexpr int kChunkBytes = 128 * 128;    // 128 rows x 128 bytes
  static constexpr int kTileBytes = 128 * HD * 2;  // one 128 x HD bf16 tile
  // P is staged in shared memory at both head dims.  At d = 64 it would also fit in TMEM beside S
  // and O (S 2x128 + O 2x64 + P 2x64 columns = 512), and P V could read it from there, but the
  // asynchronous tcgen05.st of P keeps its 64 registers allocated longer and the instance spilled;
  // staged in shared memory it does not, and measured 4-6% faster.  kPInTmem keeps both paths.
  static constexpr bool kPInTmem = false;
  // Exponential turns: softmax warp w (tile 0) and warp w + 4 (tile 1) run on the same SM
  // sub-partition and share its special-function unit, which evaluates a row block's 128
  // exponentials per thread about as fast as the tensor core does the block's MMAs.  Left to
  // themselves the two warps fall into step and slow each other's exponentials; taking turns (one
  // warp's exponentials while the other loads scores, finds its maximum and stores P) keeps the
  // unit busy without contention.
  static constexpr bool kExpTurns = FA_EXP_TURNS != 0;
  static constexpr int kPBytes = kPInTmem ? 0 : 128 * kBN * 2;  // one 128 x 128 bf16 P tile
  // bf16 O staging for the tensor-store epilogue: the P tile where there is one (both head dims
  // as built), else a buffer of its own per query tile (128 rows x d bf16)
  static constexpr int kOStageBytes = kPInTmem ? 128 * HD * 2 : 0;
  // K/V ring depth: K_{j+1} is loaded one block ahead of V_j, so three stages give every load
  // about one block of slack.
  static constexpr int kStages = HD == 128 ? 3 : 8;
  static constexpr int kTmemCols = 512;
  static constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO0 = 256, kColO1 = 256 + HD;
  static constexpr uint32_t kColP0 = 256 + 2 * HD, kColP1 = kColP0 + kBN / 2;  // TMEM P (d = 64)
  static constexpr int kNumBars = 2 + 3 * kStages + 4 * 2 + 2 + 8;
  static constexpr int kSchedBytes = 2 * 128 * 4;  // paged mode: sequence lengths and their order
  static constexpr size_t kSmemBytes = 1024 /* alignment slack */ + 2 * kTileBytes +
                                       kStages * kTileBytes + 2 * kPBytes + 2 * kOStageBytes +
                                       kNumBars * 8 + 16 + kSchedBytes;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
  static constexpr uint32_t kIdescQK = idesc_bf16_f32(kBM, kBN, 0, 0);  // Q, K both K-major
  static constexpr uint32_t kIdescPV = idesc_bf16_f32(kBM, HD, 0, 1);   // P K-major, V MN-major
  static_assert(!kPInTmem || kColP1 + kBN / 2 <= kTmemCols, "TMEM budget");
};

struct PrefillParams {
  void *o;
  float *lse;
  int o_f32;
  int BH, N, causal;  // N: query rows per (b, h) processed; also the key count in the square mode
  float scale_log2;   // scale * log2(e)
  int num_pairs;      // ceil(N / 256)
  int num_units;      // BH * num_pairs query-tile pairs, scheduled over the persistent CTAs
  // paged mode (chunked prefill over a paged KV cache): the N queries of (s, h) are the last N of
  // the sequence's L = seq_lens[s] cached tokens, whose 16-token blocks are listed in block_table
  const int32_t *seq_lens;
  const int32_t *block_table;
  int max_blocks, num_blocks, H;
  // tree verification (paged mode, causal = 0): the N queries are the nodes of a draft-token tree,
  // the last N cached tokens in topological order; bit u of tree_mask[s * N + t] set when node t
  // sees node u (N <= 64).  Null otherwise.
  const uint64_t *tree_mask;
  // key-range mode: the processed queries are rows q_row0 .. q_row0 + N - 1 of Q / O / LSE tensors
  // with q_rows rows per (b, h); the keys are the Nk rows of K / V; query row r sits at key
  // position q_off + r (>= 0).  The other modes use q_row0 = 0 and q_rows = N.
  int q_row0, q_rows, Nk, q_off;
  // square mode, d = 128, bf16 O: 1 when the O tensor map was encoded, so the epilogue stages O in
  // the tile's (by then unused) P buffer and writes it with tensor stores
  int o_tma;
};

// Kernel modes: square prefill (keys = queries), paged cache (keys gathered through the block
// table, queries the last N of each sequence), key range (contiguous keys of one range of the
// sequence, queries a suffix of the query rows).
constexpr int kModeSquare = 0, kModePaged = 1, kModeRange = 2;

// Key count of unit (b, h) and the position of its first query among the keys.
struct KvSpan {
  int L;      // keys
  int q_off;  // query row r sits at key position q_off + r
};

template <int kMode>
__device__ __forceinline__ KvSpan kv_span(const PrefillParams &p, int bh) {
  if constexpr (kMode == kModeRange) {
    return {p.Nk, p.q_off};
  } else if constexpr (kMode == kModePaged) {
    int L = p.seq_lens[bh / p.H];
    const int hi = p.max_blocks * 16;
    L = L < p.N ? p.N : (L > hi ? hi : L);  // out-of-contract lengths are clamped, not trusted
    return {L, L - p.N};
  } else {
    return {p.N, 0};
  }
}

// Work units are query-tile pairs (two 128-row tiles of one (b, h) that share every K/V block).
// Non-causal units all cost the same; they are numbered head-major (unit = bh * pairs + pair) so
// the CTAs running at the same time share a few heads' K/V in L2, and handed out round-robin.
// Causal units cost in proportion to their key-block count (4p + 3 blocks for pair p), so they are
// numbered from the most expensive pair level down (unit = level * BH + bh, pair = pairs-1-level)
// and dealt to the CTAs in snake order (round r gives CTA c the unit r*G + c for even r and
// r*G + G-1-c for odd r), a static form of longest-processing-time-first scheduling.
//
// That order keeps every head's K and V in play at once, more than L2 holds at N >= 2k, so causal
// launches re-read K/V from DRAM.  At d = 128, up to kMaxSchedUnits units, the host instead passes
// a UnitTable:
// list scheduling (each unit to the CTA that frees up first, under the cost above) over the units
// taken in groups of heads whose K and V fill a fraction of L2, longest first within a group.  It
// balances the CTAs as well as the snake and keeps about one group of heads in flight.
struct WorkUnit {
  int bh;
  int pair;
};

// Paged units cost in proportion to their sequence's cached length, which only the device
// knows.  With at most kMaxSortedSeqs sequences each CTA ranks them itself at start-up (longest
// first, ties by index; the same order in every CTA) and numbers the units sequence by sequence in
// that order, dealt in snake order like the causal levels; with more sequences, or in the
// key-range mode, units are numbered head-major and dealt round-robin.
constexpr int kMaxSortedSeqs = 128;

constexpr int kMaxSchedUnits = 2048;
constexpr int kMaxSchedCtas = 160;

// Causal square launches: CTA c runs the units unit[start[c]] .. unit[start[c+1] - 1] in that
// order (unit numbers as in the level-major numbering above).  count = 0: no table.
struct UnitTable {
  int count;
  uint16_t start[kMaxSchedCtas + 1];
  uint16_t unit[kMaxSchedUnits];
};

// Only the d = 128 square instance takes a table.  The paged and key-range modes order their units
// otherwise; at d = 64 the kernel is bound by its exponentials, so DRAM re-reads cost it nothing,
// while the table lookup made that instance spill (2-5% slower, non-causal launches included).
struct NoUnitTable {};
template <int HD, int kMode> struct UnitTableOf { using type = NoUnitTable; };
template <> struct UnitTableOf<128, kModeSquare> { using type = UnitTable; };

// The unit CTA blockIdx.x processes in its round r, or -1 once it has none left.
template <bool kGeneral, class Table>
__device__ __forceinline__ int unit_for_round(const PrefillParams &p, const Table &tab, int r,
                                              const int *seq_order = nullptr) {
  const int G = gridDim.x, c = blockIdx.x;
  if constexpr (!std::is_same_v<Table, NoUnitTable>) {
    if (tab.count > 0) {
      const int i = tab.start[c] + r;
      return i < tab.start[c + 1] ? tab.unit[i] : -1;
    }
  }
  const bool snake = kGeneral ? seq_order != nullptr : p.causal;
  const int u = r * G + ((snake && (r & 1)) ? G - 1 - c : c);
  return u < p.num_units ? u : -1;
}

template <bool kGeneral = false>
__device__ __forceinline__ WorkUnit decode_unit(const PrefillParams &p, int u,
                                                const int *seq_order = nullptr) {
  WorkUnit w;
  if (!kGeneral && p.causal) {
    w.bh = u % p.BH;
    w.pair = p.num_pairs - 1 - u / p.BH;
  } else if (kGeneral && seq_order != nullptr) {
    const int per_seq = p.H * p.num_pairs;
    const int rem = u % per_seq;
    w.bh = seq_order[u / per_seq] * p.H + rem / p.num_pairs;
    w.pair = rem % p.num_pairs;
  } else {
    w.bh = u / p.num_pairs;
    w.pair = u % p.num_pairs;
  }
  return w;
}

// Key blocks visited by query tile i (0/1) of pair `pr`: 0 if the tile starts past the last query;
// causal tiles stop at the block holding the key of their last row.
__device__ __forceinline__ int tile_blocks(const PrefillParams &p, const KvSpan &kv, int pr, int i) {
  const int q0 = pr * 2 * kBM + i * kBM;
  if (q0 >= p.N) return 0;
  if (!p.causal) return (kv.L + kBN - 1) / kBN;
  // (the key-range mode may have more queries than keys: clamp to the last key)
  const int last_key = min(kv.q_off + min(q0 + kBM, p.N) - 1, kv.L - 1);
  return last_key / kBN + 1;
}

// The tensor core takes a new MMA only about as fast as it completes one, so the issuing thread
// runs in step with it: every instruction between two MMAs is tensor-core idle time.  The
// descriptors of a group are therefore formed once, and each MMA adds a constant to them: for an
// address below 2^18 (all of shared memory), desc(addr + off) = desc(addr) + off / 16 exactly.

// S (TMEM) = Q (smem, K-major) K^T (smem, K-major), K = HD in steps of 16.
// K tile layouts: [64-column chunk][128 keys][128 B] (8-key atoms 1 KB apart, chunks kChunkBytes
// apart), or with kPageKV (paged mode, d = 128: one 4 KB load per 16-token page)
// [page][8-key group][chunk][8 keys][128 B]: 8-key atoms 2 KB apart, chunk 1 at +1 KB.
template <int HD, bool kPageKV = false>
__device__ __forceinline__ void issue_qk(uint32_t d_tmem, uint32_t q_smem, uint32_t k_smem) {
  using C = PrefillCfg<HD>;
  constexpr uint32_t kKChunk = kPageKV ? 1024 : C::kChunkBytes;
  const uint64_t qd = smem_desc_sw128(q_smem, 16, 1024);
  const uint64_t kd = smem_desc_sw128(k_smem, 16, kPageKV ? 2048 : 1024);
#pragma unroll
  for (int kk = 0; kk < HD / 16; ++kk) {
    const uint64_t qoff = static_cast<uint64_t>(((kk / 4) * C::kChunkBytes + (kk % 4) * 32) >> 4);
    const uint64_t koff = static_cast<uint64_t>(((kk / 4) * kKChunk + (kk % 4) * 32) >> 4);
    umma_ss(d_tmem, qd + qoff, kd + koff, C::kIdescQK, kk > 0 ? 1u : 0u);
  }
}

// O (TMEM) (+)= P (smem, K-major over the 128 keys) V (smem, MN-major), K = 128 keys in steps of
// 16.  V's descriptor: LBO = distance between 64-element chunks of d, SBO = between 8-key groups.
// p_addr is a shared-memory address, or with kPInTmem a TMEM address (2 bf16 per column, 8
// columns per 16 keys).
// V tile layouts: [64-column chunk][128 keys][128 B] (chunks kChunkBytes apart), or with kPageKV
// (paged mode, d = 128: one 4 KB load per 16-token page) [page][64-column half][16 keys][128 B],
// a page per 16-key step and its halves 2 KB apart.
template <int HD, bool kPageKV = false>
__device__ __forceinline__ void issue_pv(uint32_t o_tmem, uint32_t p_addr, uint32_t v_smem,
                                         bool accumulate) {
  using C = PrefillCfg<HD>;
  constexpr uint32_t kStepBytes = kPageKV ? 4096 : 16 * 128;  // V bytes per 16-key step
  const uint64_t vd = smem_desc_sw128(v_smem, kPageKV ? 2048 : C::kChunkBytes, 1024);
  const uint64_t pd = C::kPInTmem ? 0 : smem_desc_sw128(p_addr, 16, 1024);
#pragma unroll
  for (int kk = 0; kk < kBN / 16; ++kk) {
    const uint64_t b = vd + static_cast<uint64_t>((kk * kStepBytes) >> 4);
    if constexpr (C::kPInTmem) {
      umma_ts(o_tmem, p_addr + kk * 8, b, C::kIdescPV, (accumulate || kk > 0) ? 1u : 0u);
    } else {
      const uint64_t off = static_cast<uint64_t>(((kk / 4) * C::kChunkBytes + (kk % 4) * 32) >> 4);
      umma_ss(o_tmem, pd + off, b, C::kIdescPV, (accumulate || kk > 0) ? 1u : 0u);
    }
  }
}

// One row of a score block -> P: p = 2^(s * scale*log2e - m_ref) for the 128 scores of this
// thread's row (MUFU ex2, or the FMA-pipe polynomial for every kPolyEvery-th pair), packed to
// bf16 pairs in pk.  Returns the sum of the fp32 p.
// With kPoly > 0 it also returns in `rounded` the exact sum of the bf16 values in pk (the P that
// P V uses): the polynomial and MUFU round differently, so the single-element correction the
// MUFU-only path uses (below) would not match the element actually stored.
template <int kPoly>
__device__ __forceinline__ float exp_row(float (&s)[kBN], float sl2, float mneg,
                                         uint32_t (&pk)[kBN / 2], float &rounded) {
  const uint64_t c2 = f2_pack(sl2, sl2), m2 = f2_pack(mneg, mneg);
  uint64_t le2 = 0, lr2 = 0;
#pragma unroll
  for (int c = 0; c < kBN / 2; ++c) {
    const uint64_t x2 = f2_fma(f2_pack(s[2 * c], s[2 * c + 1]), c2, m2);
    uint64_t p2;
    if (kPoly > 0 && c % (kPoly > 0 ? kPoly : 1) == kPoly - 1) {
      p2 = exp2_poly_x2(x2);
    } else {
      float x0, x1;
      f2_unpack(x2, x0, x1);
      p2 = f2_pack(ex2(x0), ex2(x1));
    }
    le2 = f2_add(le2, p2);
    float p0, p1;
    f2_unpack(p2, p0, p1);
    pk[c] = pack_bf16x2(p0, p1);
    if constexpr (kPoly > 0)
      lr2 = f2_add(lr2, f2_pack(__uint_as_float(pk[c] << 16), __uint_as_float(pk[c] & 0xffff0000u)));
  }
  float a, b;
  if constexpr (kPoly > 0) {
    f2_unpack(lr2, a, b);
    rounded = a + b;
  }
  f2_unpack(le2, a, b);
  return a + b;
}

// Write this thread's row of P (128 bf16 = 256 bytes) into the 128-byte-swizzled K-major tile the
// MMA reads: keys 0..63 in chunk 0, 64..127 in chunk 1; the 16-byte unit u of row r goes to
// unit u ^ (r % 8) of that row.
__device__ __forceinline__ void store_p_row(uint8_t *p_tile, int row, const uint32_t (&pk)[kBN / 2]) {
#pragma unroll
  for (int ch = 0; ch < 2; ++ch) {
    uint8_t *rowp = p_tile + ch * 16384 + row * 128;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int q = ch * 32 + u * 4;
      *reinterpret_cast<uint4 *>(rowp + ((u ^ (row & 7)) * 16)) =
          make_uint4(pk[q], pk[q + 1], pk[q + 2], pk[q + 3]);
    }
  }
}

// kMode: kModeSquare, kModePaged (tm_k / tm_v map the pools [num_blocks, H, 16, d]; a 128-key
// tile is gathered as eight 16-row pages through the block table, one TMA box per page: 4-D maps
// at d = 64, 5-D maps at d = 128 whose box reorders the page into the operand layout) or
// kModeRange.
template <int HD, int kMode>
__global__ void __launch_bounds__(kPrefillThreads, 1)
    fa_prefill_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v,
                      const __grid_constant__ CUtensorMap tm_o, const PrefillParams p,
                      const __grid_constant__ typename UnitTableOf<HD, kMode>::type tab) {
  using C = PrefillCfg<HD>;
  constexpr bool kPaged = kMode == kModePaged;
  constexpr bool kGeneral = kMode != kModeSquare;  // key count and query offset per unit
  constexpr bool kPageKV = kPaged && HD == 128;     // K and V pages arrive as whole 4 KB boxes
  // bf16 O through a shared-memory staging tile and tensor stores (square and paged modes: the
  // processed rows of (b, h) are rows 0 .. N-1 of its O slice)
  constexpr bool kTmaO = kMode != kModeRange;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *sQ = smem;                                   // 2 tiles
  uint8_t *sKV = sQ + 2 * C::kTileBytes;                // kStages tiles
  uint8_t *sP = sKV + C::kStages * C::kTileBytes;       // 2 P tiles
  uint8_t *sO = sP + 2 * C::kPBytes;                     // 2 O staging tiles (d = 64)
  uint64_t *bars = reinterpret_cast<uint64_t *>(sO + 2 * C::kOStageBytes);
  uint64_t *q_full = bars;
  uint64_t *q_empty = bars + 1;
  // kv_full[st]: a K tile has landed in stage st; kv_full[kStages + st]: a V tile has.  Each
  // has one waiter (the Q K^T issuer for K, the P V issuer for V) that sees all of its phases
  // in order, so a parity wait is exact: the next load of the same kind into the stage can only
  // start after that waiter has consumed and released the current one.
  uint64_t *kv_full = bars + 2;
  uint64_t *kv_empty = kv_full + 2 * C::kStages;
  uint64_t *s_full = kv_empty + C::kStages;  // [2] S_i computed (MMA commit)
  uint64_t *s_free = s_full + 2;             // [2] S_i copied out by the softmax (4 warp arrivals)
  uint64_t *p_full = s_free + 2;             // [2] P_i written to smem (4 warp arrivals)
  uint64_t *pv_done = p_full + 2;            // [2] O_i += P_i V finished (MMA commit)
  uint64_t *drain = pv_done + 2;             // [2] every MMA of issuer 0 / 1 has completed
  uint64_t *turn = drain + 2;                // [8] exponential turns: [k] warp k, [4 + k] warp 4 + k
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(turn + 8);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  int *s_lens = const_cast<int *>(reinterpret_cast<volatile int *>(abort_flag + 1));  // [128]
  int *s_order = s_lens + kMaxSortedSeqs;                                              // [128]

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  // paged mode with few sequences: longest-first order of the sequences (computed below)
  const int n_seqs = kPaged ? p.BH / p.H : 0;
  const int *seq_order = (kPaged && n_seqs <= kMaxSortedSeqs) ? s_order : nullptr;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_full[C::kStages + s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], kBM / 32);
      mbar_init(&p_full[i], kBM / 32);
      mbar_init(&pv_done[i], 1);
    }
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    for (int k = 0; k < 8; ++k) mbar_init(&turn[k], 1);
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
    if (kTmaO && p.o_tma) tma_prefetch_desc(&tm_o);
  }
  if (seq_order != nullptr && warp == 10) {
    // rank the sequences by cached length (clamped as the units will see it), longest first
    for (int sq = lane; sq < n_seqs; sq += 32) s_lens[sq] = kv_span<kMode>(p, sq * p.H).L;
    __syncwarp();
    for (int sq = lane; sq < n_seqs; sq += 32) {
      const int L = s_lens[sq];
      int rank = 0;
      for (int o = 0; o < n_seqs; ++o) {
        const int Lo = s_lens[o];
        rank += (Lo > L || (Lo == L && o < sq)) ? 1 : 0;
      }
      s_order[rank] = sq;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 8) {
    // ------------------------------------------------------------------ TMA producer
    // Load order per unit: Q pair, K_0, then for each block j: K_{j+1} (if any), V_j -- the
    // order in which the MMA warp consumes them.
    if (lane == 0) {
      uint32_t kv_it = 0, q_ph = 0;
      bool q_issued = false;
      uint32_t loads[2 * C::kStages];  // loads issued on each landing barrier (its phase count)
      for (int b = 0; b < 2 * C::kStages; ++b) loads[b] = 0;
      bool ok = true;
      int kv_len = 0;  // key count of the current unit (paged mode)
      auto load_kv = [&](const CUtensorMap *map, int row, int bh, bool is_v) -> bool {
        const uint32_t st = kv_it % C::kStages, ph = (kv_it / C::kStages) & 1;
        if (!mbar_wait(&kv_empty[st], ph ^ 1, abort_flag)) return false;
        uint64_t *full = &kv_full[(is_v ? C::kStages : 0) + st];
        mbar_arrive_expect_tx(full, C::kTileBytes);
        if constexpr (kPaged) {
          // keys row .. row+127 of sequence s live in eight 16-token pages; pages past the
          // sequence's end (masked by the softmax) read as zeros through an out-of-range block
          const int sq = bh / p.H, h = bh % p.H;
          const int npages = (kv_len + 15) / 16;
          int blk[kBN / 16];
#pragma unroll
          for (int r = 0; r < kBN / 16; ++r) {
            const int page = row / 16 + r;
            int b = page < npages ? p.block_table[static_cast<size_t>(sq) * p.max_blocks + page]
                                  : p.num_blocks;
            if (page < npages && (b < 0 || b >= p.num_blocks)) {
              atomicExch(&g_device_status, 1 /* FA_ERR_INVALID_ARG: bad block-table entry */);
              b = p.num_blocks;
            }
            blk[r] = b;
          }
          if (kPageKV) {
            // d = 128: one 4 KB box per page (the layouts issue_qk and issue_pv read with
            // kPageKV): a TMA box costs about as much fixed time as 10 KB of data, so eight boxes
            // per tile instead of sixteen.  K's map indexes pages of one head as block * H + head
            // (an out-of-range block stays out of range), V's as (head, block).
#pragma unroll
            for (int r = 0; r < kBN / 16; ++r) {
              if (is_v)
                tma_load_5d(sKV + st * C::kTileBytes + r * 4096, map, full, 0, 0, 0, h, blk[r]);
              else
                tma_load_5d(sKV + st * C::kTileBytes + r * 4096, map, full, 0, 0, 0, 0,
                            blk[r] * p.H + h);
            }
          } else {
#pragma unroll
            for (int r = 0; r < kBN / 16; ++r)
              for (int ch = 0; ch < C::kChunks; ++ch)
                tma_load_4d(sKV + st * C::kTileBytes + ch * C::kChunkBytes + r * 16 * 128, map,
                            full, ch * 64, 0, h, blk[r]);
          }
        } else {
          for (int ch = 0; ch < C::kChunks; ++ch)
            tma_load_3d(sKV + st * C::kTileBytes + ch * C::kChunkBytes, map, full, ch * 64, row,
                        bh);
        }
        ++loads[(is_v ? C::kStages : 0) + st];
        ++kv_it;
        return true;
      };
      for (int r = 0; ok; ++r) {
        const int u = unit_for_round<kGeneral>(p, tab, r, seq_order);
        if (u < 0) break;
        const WorkUnit w = decode_unit<kGeneral>(p, u, seq_order);
        const int pr = w.pair;
        const KvSpan kv = kv_span<kMode>(p, w.bh);
        kv_len = kv.L;
        if (kPaged && p.seq_lens[w.bh / p.H] != kv.L)
          atomicExch(&g_device_status, 1 /* FA_ERR_INVALID_ARG: length outside [Lq, 16*max_blocks] */);
        const int n0 = tile_blocks(p, kv, pr, 0), n1 = tile_blocks(p, kv, pr, 1);
        const int nmax = n0 > n1 ? n0 : n1;
        if (!mbar_wait(q_empty, q_ph ^ 1, abort_flag)) { ok = false; break; }
        q_ph ^= 1;
        mbar_arrive_expect_tx(q_full, (n0 > 0 ? C::kTileBytes : 0) + (n1 > 0 ? C::kTileBytes : 0));
        q_issued = true;
        for (int i = 0; i < 2; ++i) {
          if ((i == 0 ? n0 : n1) == 0) continue;
          for (int ch = 0; ch < C::kChunks; ++ch)
            tma_load_3d(sQ + i * C::kTileBytes + ch * C::kChunkBytes, &tm_q, q_full, ch * 64,
                        (kGeneral ? p.q_row0 : 0) + pr * 2 * kBM + i * kBM, w.bh);
        }
        if (!load_kv(&tm_k, 0, w.bh, false)) { ok = false; break; }
        for (int j = 0; ok && j < nmax; ++j) {
          if (j + 1 < nmax && !load_kv(&tm_k, (j + 1) * kBN, w.bh, false)) { ok = false; break; }
          if (!load_kv(&tm_v, j * kBN, w.bh, true)) { ok = false; break; }
        }
      }
      if (!ok) {
        // abandoned: let every copy already in flight land before the CTA's smem goes away
        volatile int never = 0;
        for (int b = 0; b < 2 * C::kStages; ++b)
          if (loads[b] > 0) mbar_wait(&kv_full[b], (loads[b] - 1) & 1, &never);
        if (q_issued) mbar_wait(q_full, q_ph ^ 1, &never);
      }
    }
  } else if (warp == 9 || warp == 10) {
    // ------------------------------------------------------------------ MMA issuers (two)
    // Warp 9 issues S_i,j = Q_i K_j^T, warp 10 issues O_i += P_i,j V_j, each in block order and
    // each committing its own barriers; K_j's stage is released by the first, V_j's by the second.
    // Per unit the loads arrive in the order K_0, then K_{j+1}, V_j for j = 0, 1, ...: load index
    // of K_j is 2j-1 (K_0: 0), of V_j 2j+2 (2j+1 for the last block).
    if (lane == 0) {
      const bool scores = warp == 9;
      uint32_t kv_base = 0, q_ph = 0;
      uint32_t s_cnt[2] = {0, 0};  // S_i computed so far (s_free phases follow it)
      uint32_t p_cnt[2] = {0, 0};  // P_i consumed so far (p_full phases follow it)
      uint32_t full_ph = 0;        // bit st: phase parity of this issuer's landing barrier of stage st
      const uint32_t sQ0 = smem_u32(sQ), sQ1 = smem_u32(sQ + C::kTileBytes);
      const uint32_t sKV0 = smem_u32(sKV), sP0 = smem_u32(sP);
      uint64_t *my_full = kv_full + (scores ? 0 : C::kStages);
      auto wait_load = [&](uint32_t st) -> bool {
        if (!mbar_wait(&my_full[st], (full_ph >> st) & 1u, abort_flag)) return false;
        full_ph ^= 1u << st;
        return true;
      };
      bool ok = true;
      for (int r = 0; ok; ++r) {
        const int u = unit_for_round<kGeneral>(p, tab, r, seq_order);
        if (u < 0) break;
        const WorkUnit w = decode_unit<kGeneral>(p, u, seq_order);
        const KvSpan kv = kv_span<kMode>(p, w.bh);
        const int n[2] = {tile_blocks(p, kv, w.pair, 0), tile_blocks(p, kv, w.pair, 1)};
        const int nmax = n[0] > n[1] ? n[0] : n[1];
        if (scores) {
          if (!mbar_wait(q_full, q_ph, abort_flag)) { ok = false; break; }
          q_ph ^= 1;
          for (int j = 0; ok && j < nmax; ++j) {
            const uint32_t ld = kv_base + (j == 0 ? 0u : static_cast<uint32_t>(2 * j - 1));
            const uint32_t st = ld % C::kStages;
            if (!wait_load(st)) { ok = false; break; }
            for (int i = 0; i < 2; ++i) {
              if (j >= n[i]) continue;
              if (s_cnt[i] > 0 && !mbar_wait(&s_free[i], (s_cnt[i] - 1) & 1, abort_flag)) {
                ok = false;
                break;
              }
              tc_fence_after();
              issue_qk<HD, kPageKV>(tmem + (i ? C::kColS1 : C::kColS0), i ? sQ1 : sQ0,
                                    sKV0 + st * C::kTileBytes);
              umma_commit(&s_full[i]);
              ++s_cnt[i];
            }
            if (!ok) break;
            umma_commit(&kv_empty[st]);  // K_j is free once both S_i,j have been computed
          }
          if (!ok) break;
          umma_commit(q_empty);  // every Q K^T of the unit is issued
        } else {
          for (int j = 0; ok && j < nmax; ++j) {
            const uint32_t ld = kv_base + static_cast<uint32_t>(j + 1 < nmax ? 2 * j + 2 : 2 * j + 1);
            const uint32_t st = ld % C::kStages;
            if (!wait_load(st)) { ok = false; break; }
            for (int i = 0; i < 2; ++i) {
              if (j >= n[i]) continue;
              if (!mbar_wait(&p_full[i], p_cnt[i] & 1, abort_flag)) { ok = false; break; }
              ++p_cnt[i];
              tc_fence_after();
              const uint32_t p_addr = C::kPInTmem ? tmem + (i ? C::kColP1 : C::kColP0)
                                                  : sP0 + i * C::kPBytes;
              issue_pv<HD, kPageKV>(tmem + (i ? C::kColO1 : C::kColO0), p_addr,
                                   sKV0 + st * C::kTileBytes, j > 0);
              umma_commit(&pv_done[i]);
            }
            if (!ok) break;
            umma_commit(&kv_empty[st]);  // V_j is free once both P_i,j V_j have completed
          }
        }
        kv_base += 2 * nmax;
      }
      // every MMA issued by this thread completes before TMEM is released
      umma_commit(&drain[scores ? 0 : 1]);
      volatile int never = 0;
      mbar_wait(&drain[scores ? 0 : 1], 0, &never);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------------ softmax / epilogue
    const int wg = warp / 4;                       // which tile of the pair
    const int row = threadIdx.x % 128;             // TMEM lane == query row within the tile
    const uint32_t lane_off = static_cast<uint32_t>((warp % 4) * 32) << 16;
    const uint32_t tS = tmem + lane_off + (wg ? C::kColS1 : C::kColS0);
    const uint32_t tO = tmem + lane_off + (wg ? C::kColO1 : C::kColO0);
    uint8_t *pTile = sP + wg * C::kPBytes;
    uint8_t *oTile = C::kPInTmem ? sO + wg * C::kOStageBytes : pTile;
    const uint32_t tP = tmem + lane_off + (wg ? C::kColP1 : C::kColP0);
    const float sl2 = p.scale_log2;
    uint32_t s_ph = 0, pv_ph = 0;
    bool ok = true;
    // exponential turns with the warp of the other tile on this sub-partition (tile 0 first): wait
    // on my barrier, run the exponentials, arrive on the other's.  Both warps take one turn per
    // key block of the larger of the two tiles' block counts, so the turns always pair up.
    uint64_t *turn_mine = turn + (wg ? 4 : 0) + warp % 4;
    uint64_t *turn_other = turn + (wg ? 0 : 4) + warp % 4;
    uint32_t turn_ph = 0;
    auto take_turn = [&]() -> bool {
      if (!__all_sync(0xffffffffu, mbar_wait(turn_mine, turn_ph, abort_flag))) return false;
      turn_ph ^= 1;
      return true;
    };
    auto pass_turn = [&]() {
      __syncwarp();
      if (lane == 0) mbar_arrive(turn_other);
    };
    if (C::kExpTurns && wg == 1) pass_turn();
    for (int r = 0; ok; ++r) {
      const int u = unit_for_round<kGeneral>(p, tab, r, seq_order);
      if (u < 0) break;
      const WorkUnit w = decode_unit<kGeneral>(p, u, seq_order);
      const int pr = w.pair;
      const KvSpan kv = kv_span<kMode>(p, w.bh);
      const int n = tile_blocks(p, kv, pr, wg);
      // no turns in a unit with one tile only (a ragged last pair, a draft tree of <= 128 nodes):
      // both warps of a pair see the same block counts, so they skip the same units
      const int n_other = tile_blocks(p, kv, pr, wg ^ 1);
      const bool turns = C::kExpTurns && n > 0 && n_other > 0;
      if (n == 0) continue;
      const int qrow = pr * 2 * kBM + wg * kBM + row;
      const bool tree = kPaged && p.tree_mask != nullptr;
      const uint64_t tmask =
          (tree && qrow < p.N) ? p.tree_mask[static_cast<size_t>(w.bh / p.H) * p.N + qrow] : 0ull;
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
        // S_i's columns may now take the next block's scores
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_free[wg]);
        // masking only where a block reaches past this tile's first row's last visible key or
        // past the last key
        bool edge;
        if constexpr (kGeneral)
          edge = (p.causal && (j + 1) * kBN - 1 > kv.q_off + pr * 2 * kBM + wg * kBM) ||
                 ((j + 1) * kBN > kv.L) || (tree && (j + 1) * kBN > kv.q_off);
        else  // q_off = 0, L = N: only a causal tile's diagonal block and a ragged last block
          edge = (p.causal && j == n - 1) || ((j + 1) * kBN > p.N && (p.N % kBN) != 0);
        if (kPaged && tree && edge) {
          // context keys (< q_off) are visible; key q_off + u only if bit u of the node's mask is
          // set; nothing past L
#pragma unroll
          for (int c = 0; c < kBN; ++c) {
            const int u = j * kBN + c - kv.q_off;
            if (u >= 0 && (u >= kv.L - kv.q_off || !((tmask >> (u & 63)) & 1ull))) s[c] = -INFINITY;
          }
        } else if (edge) {
          const int lim = (p.causal ? min(kv.q_off + qrow + 1, kv.L) : kv.L) - j * kBN;  // visible
#pragma unroll
          for (int c = 0; c < kBN; ++c)
            if (c >= lim) s[c] = -INFINITY;
        }
        // row max: eight independent chains of 3-input max, then a short tree
        float mx[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) mx[q] = fmaxf(s[2 * q], s[2 * q + 1]);
#pragma unroll
        for (int c = 16; c < kBN; c += 16)
#pragma unroll
          for (int q = 0; q < 8; ++q) mx[q] = fmax3(mx[q], s[c + 2 * q], s[c + 2 * q + 1]);
        const float s_top =
            fmaxf(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], fmax3(mx[5], mx[6], mx[7])));
        // Lazy rescale: the reference max m_ref (log2 units) moves only when a block's max
        // exceeds it by more than 2^8 (always on the first block, where m_ref = -inf).
        const float m_blk = s_top * sl2;
        const bool need = m_blk > m_ref + kRescaleLog2;
        float alpha = 1.f;
        if (need) {
          alpha = ex2(m_ref - m_blk);  // 2^-inf = 0 on the first block
          m_ref = m_blk;
        }
        const float mneg = (m_ref == -INFINITY) ? 0.f : -m_ref;
        uint32_t pk[kBN / 2];
        if (turns && !take_turn()) { ok = false; break; }
        constexpr int kPoly = kPolyEvery<HD>;
        float lr_blk = 0.f;
        const float p_top = kPoly > 0 ? 0.f : ex2(fmaf(s_top, sl2, mneg));
        const float le = exp_row<kPoly>(s, sl2, mneg, pk, lr_blk);
        if (turns) pass_turn();
        // O is normalised by the sum of the bf16-rounded p that P V uses, so that it is a
        // convex combination of V rows even when one key dominates the row.  With MUFU only, the
        // rounding error that matters is the largest element's, so the fp32 sum is corrected by
        // exactly that element's rounding (same arithmetic as in exp_row); with the polynomial
        // share, exp_row sums the rounded values themselves.  The LSE keeps the fp32 sum.
        if constexpr (kPoly == 0)
          lr_blk = le + (__uint_as_float(pack_bf16x2(0.f, p_top) & 0xffff0000u) - p_top);
        l = l * alpha + le;
        lr = lr * alpha + lr_blk;
        if (j > 0) {
          // P_i,j-1 must have been consumed (and O_i completed through block j-1) before this
          // block's P overwrites the smem tile and before O_i is rescaled
          if (!__all_sync(0xffffffffu, mbar_wait(&pv_done[wg], pv_ph, abort_flag))) { ok = false; break; }
          pv_ph ^= 1;
          tc_fence_after();
        }
        // P first, then O's rescale.  A tcgen05.st reads its source registers asynchronously, so
        // they stay allocated until tcgen05.wait::st: wait right after each store, so that P's 64
        // registers and each rescaled chunk of O are free again before the next use (waiting only
        // once at the end held them all at once and made the d = 64 instance spill).
        if constexpr (C::kPInTmem) {
          tmem_st32(tP, pk);
          tmem_st32(tP + 32, pk + 32);
          tmem_wait_st();
        } else {
          if (kTmaO && !C::kPInTmem && p.o_tma && j == 0) {
            // the previous unit's O left this warp's rows of the P tile through tensor stores
            if (lane == 0) bulk_wait_group_read<0>();
            __syncwarp();
          }
          store_p_row(pTile, row, pk);
        }
        if (j > 0) {
          if (__any_sync(0xffffffffu, need)) {
            // rows that keep their reference use alpha = 1
#pragma unroll
            for (int cc = 0; cc < HD; cc += 32) {
              uint32_t o[32];
              tmem_ld32(tO + cc, o);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
              tmem_st32(tO + cc, o);
              tmem_wait_st();
            }
          }
        }
        if constexpr (!C::kPInTmem) fence_async_smem();  // generic-proxy P -> the tensor core
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[wg]);  // one arrival per warp
      }
      if (turns) {
        // the other tile's extra block (causal pairs: tile 1 has one more)
        for (int j = n; ok && j < n_other; ++j) {
          if (!take_turn()) ok = false;
          else pass_turn();
        }
      }
      if (!ok) break;
      // epilogue: O_i / l and LSE once the last P V of this tile has completed
      if (!__all_sync(0xffffffffu, mbar_wait(&pv_done[wg], pv_ph, abort_flag))) { ok = false; break; }
      pv_ph ^= 1;
      tc_fence_after();
      // a row with no visible key (possible only with a tree mask) gets O = 0
      const float inv = (kPaged && lr == 0.f) ? 0.f : 1.f / lr;
      const bool live = qrow < p.N;
      const size_t grow = kGeneral ? static_cast<size_t>(w.bh) * p.q_rows + p.q_row0 + qrow
                                   : static_cast<size_t>(w.bh) * p.N + qrow;
      if (kTmaO && p.o_tma) {
        // O / l as bf16 into this thread's row of the staging tile (the layout P uses: 64 columns
        // per 128-byte-swizzled chunk), then one tensor store per chunk of the warp's 32 rows.  With
        // P in TMEM (kPInTmem, not the configuration built) the staging tile is a buffer of its
        // own that still holds this warp's rows of the previous unit's O until those stores have
        // read it.
        if constexpr (C::kPInTmem) {
          if (lane == 0) bulk_wait_group_read<0>();
          __syncwarp();
        }
#pragma unroll
        for (int cc = 0; cc < HD; cc += 32) {
          uint32_t o[32];
          tmem_ld32(tO + cc, o);
          tmem_wait_ld();
          uint8_t *rowp = oTile + (cc / 64) * C::kChunkBytes + row * 128;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int u = (cc % 64) / 8 + e;
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(o[8 * e + 0]) * inv, __uint_as_float(o[8 * e + 1]) * inv);
            v.y = pack_bf16x2(__uint_as_float(o[8 * e + 2]) * inv, __uint_as_float(o[8 * e + 3]) * inv);
            v.z = pack_bf16x2(__uint_as_float(o[8 * e + 4]) * inv, __uint_as_float(o[8 * e + 5]) * inv);
            v.w = pack_bf16x2(__uint_as_float(o[8 * e + 6]) * inv, __uint_as_float(o[8 * e + 7]) * inv);
            *reinterpret_cast<uint4 *>(rowp + ((u ^ (row & 7)) * 16)) = v;
          }
        }
        fence_async_smem();
        __syncwarp();
        const int r0 = qrow - lane;  // the warp's first row; boxes reaching past N are clipped
        if (lane == 0 && r0 < p.N) {
#pragma unroll
          for (int ch = 0; ch < HD / 64; ++ch)
            tma_store_3d(&tm_o, oTile + ch * C::kChunkBytes + (row - lane) * 128, 64 * ch, r0, w.bh);
          bulk_commit_group();
        }
        if (live && p.lse) p.lse[grow] = (m_ref + lg2(l)) * kLn2;
        continue;
      }
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
    if (kTmaO && p.o_tma) {
      if (lane == 0) bulk_wait_group_all();  // the stores have read the P tile before the CTA exits
      __syncwarp();
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
