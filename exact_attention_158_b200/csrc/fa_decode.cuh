// fa_decode.cuh -- one decode step (query length 1) over a paged KV cache, split over the context.
//
// Paging: "LLM study notes" (devocean.sk.com), paged attention -- the KV cache is a pool of
// fixed-size blocks and a per-sequence block table maps logical block t to a physical block, so a
// sequence's keys are logically contiguous while physically scattered.  Here a block holds 16
// tokens of every head: pool [num_blocks, H, 16, d], so one (block, head) is a contiguous 16 x d
// slab (4 KB at d = 128).
//
// Split-KV: the context of each (sequence, head) is cut into chunks of kDecodeChunkPages blocks;
// each chunk runs the online softmax of "Flash Attention" (myungum), section 2 (running max m,
// running sum l, rescale of the partial output when m grows) and writes (unnormalised O, m, l) to
// the caller's workspace.  A second kernel merges the chunks with the same rule the pseudocode
// uses between key blocks: m = max_c m_c, l = sum_c 2^(m_c - m) l_c, O = sum_c 2^(m_c - m) O_c / l.
// Scores are kept in log2 units (scale * log2(e) folded into q), so exp becomes ex2.
//
// This path is bound by HBM bandwidth: every K/V byte is read once, with 16-byte vector loads
// that bypass L1, and the dot products run on the CUDA cores in fp32.
#pragma once
#include "sm100_ptx.cuh"

namespace fa {

constexpr int kPage = 16;
constexpr int kDecodeThreads = 128;      // 4 warps per (sequence, head, chunk)
constexpr int kDecodeChunkPages = 32;    // 512 tokens per chunk

struct DecodeParams {
  const uint16_t *q;
  const uint16_t *kp;
  const uint16_t *vp;
  const int32_t *table;
  const int32_t *lens;
  int max_blocks, num_blocks, H;
  float scale_log2;
  float *ws;    // [S*H][n_split][d + 2]: unnormalised O, m (log2 units), l
  int n_split;  // chunks per sequence at the table's maximum length
  void *o;
  int o_f32;
  float *lse;
  int SH;
};

__device__ __forceinline__ uint4 ld_stream_v4(const void *ptr) {
  uint4 r;
  asm("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];"
      : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
      : "l"(ptr));
  return r;
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4 &v, float (&f)[8]) {
  f[0] = __uint_as_float(v.x << 16);
  f[1] = __uint_as_float(v.x & 0xffff0000u);
  f[2] = __uint_as_float(v.y << 16);
  f[3] = __uint_as_float(v.y & 0xffff0000u);
  f[4] = __uint_as_float(v.z << 16);
  f[5] = __uint_as_float(v.z & 0xffff0000u);
  f[6] = __uint_as_float(v.w << 16);
  f[7] = __uint_as_float(v.w & 0xffff0000u);
}

__device__ __forceinline__ int clamp_len(int L, int max_blocks) {
  const int hi = max_blocks * kPage;
  return L < 1 ? 1 : (L > hi ? hi : L);
}

// grid (n_split, H, S); block 128.  Warp w takes the chunk's pages w, w+4, ...  Within a warp,
// LPR = d/8 lanes cover one key row (8 elements = 16 bytes each) and 32/LPR rows are read per
// warp-wide load, so one 16-row page takes 16*LPR/32 loads for K and as many for V.
template <int HD>
__global__ void __launch_bounds__(kDecodeThreads)
    fa_decode_partial_kernel(const DecodeParams p) {
  constexpr int LPR = HD / 8;
  constexpr int RPI = 32 / LPR;
  constexpr int NI = kPage / RPI;
  __shared__ float sm_acc[4][HD];
  __shared__ float sm_m[4], sm_l[4];

  const int c = blockIdx.x, h = blockIdx.y, s = blockIdx.z;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int L = clamp_len(p.lens[s], p.max_blocks);
  const int nblk = (L + kPage - 1) / kPage;
  const int pg0 = c * kDecodeChunkPages;
  if (pg0 >= nblk) return;  // this chunk lies past the sequence's end (uniform over the CTA)
  const int pg1 = min(nblk, pg0 + kDecodeChunkPages);
  const int dl = lane % LPR, slot = lane / LPR;

  float qf[8];
  bf16x8_to_f32(*reinterpret_cast<const uint4 *>(p.q + (static_cast<size_t>(s) * p.H + h) * HD + 8 * dl), qf);
#pragma unroll
  for (int e = 0; e < 8; ++e) qf[e] *= p.scale_log2;

  float m = -INFINITY, l = 0.f, acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;

  const int32_t *trow = p.table + static_cast<size_t>(s) * p.max_blocks;
  for (int pg = pg0 + warp; pg < pg1; pg += 4) {
    const int blk = trow[pg];
    if (blk < 0 || blk >= p.num_blocks) {  // caller broke the table contract: skip, report
      if (lane == 0) atomicExch(&g_device_status, 1 /* FA_ERR_INVALID_ARG */);
      continue;
    }
    const size_t base = (static_cast<size_t>(blk) * p.H + h) * kPage * HD;
    uint4 kr[NI], vr[NI];
#pragma unroll
    for (int i = 0; i < NI; ++i)
      kr[i] = ld_stream_v4(p.kp + base + (i * RPI + slot) * HD + 8 * dl);
#pragma unroll
    for (int i = 0; i < NI; ++i)
      vr[i] = ld_stream_v4(p.vp + base + (i * RPI + slot) * HD + 8 * dl);

    float sc[NI];
#pragma unroll
    for (int i = 0; i < NI; ++i) {
      float kf[8];
      bf16x8_to_f32(kr[i], kf);
      float dot = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) dot = fmaf(qf[e], kf[e], dot);
#pragma unroll
      for (int off = LPR / 2; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
      const int tok = pg * kPage + i * RPI + slot;
      sc[i] = tok < L ? dot : -INFINITY;
    }
    float pm = sc[0];
#pragma unroll
    for (int i = 1; i < NI; ++i) pm = fmaxf(pm, sc[i]);
#pragma unroll
    for (int off = LPR; off < 32; off <<= 1) pm = fmaxf(pm, __shfl_xor_sync(0xffffffffu, pm, off));
    const float mn = fmaxf(m, pm);  // finite: the page's first token is always live
    const float alpha = ex2(m - mn);
    m = mn;
    l *= alpha;
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] *= alpha;
#pragma unroll
    for (int i = 0; i < NI; ++i) {
      const float pi = ex2(sc[i] - mn);
      l += pi;
      float vf[8];
      bf16x8_to_f32(vr[i], vf);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] = fmaf(pi, vf[e], acc[e]);
    }
  }
  // lanes holding the same d-range but different rows: sum (they share the warp's m)
#pragma unroll
  for (int off = LPR; off < 32; off <<= 1) {
    l += __shfl_xor_sync(0xffffffffu, l, off);
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], off);
  }
  if (slot == 0) {
#pragma unroll
    for (int e = 0; e < 8; ++e) sm_acc[warp][8 * dl + e] = acc[e];
  }
  if (lane == 0) {
    sm_m[warp] = m;
    sm_l[warp] = l;
  }
  __syncthreads();
  float M = fmaxf(fmaxf(sm_m[0], sm_m[1]), fmaxf(sm_m[2], sm_m[3]));
  float f[4];
#pragma unroll
  for (int w = 0; w < 4; ++w) f[w] = ex2(sm_m[w] - M);  // warps without pages: 2^-inf = 0
  float *part = p.ws + (static_cast<size_t>(s * p.H + h) * p.n_split + c) * (HD + 2);
  for (int e = threadIdx.x; e < HD; e += kDecodeThreads)
    part[e] = f[0] * sm_acc[0][e] + f[1] * sm_acc[1][e] + f[2] * sm_acc[2][e] + f[3] * sm_acc[3][e];
  if (threadIdx.x == 0) {
    part[HD] = M;
    part[HD + 1] = f[0] * sm_l[0] + f[1] * sm_l[1] + f[2] * sm_l[2] + f[3] * sm_l[3];
  }
}

// One warp per (sequence, head): merge that unit's chunk partials, normalise, write O and LSE.
template <int HD>
__global__ void __launch_bounds__(128) fa_decode_combine_kernel(const DecodeParams p) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int u = blockIdx.x * 4 + warp;
  if (u >= p.SH) return;
  const int s = u / p.H;
  const int L = clamp_len(p.lens[s], p.max_blocks);
  const int nblk = (L + kPage - 1) / kPage;
  const int nsplit = (nblk + kDecodeChunkPages - 1) / kDecodeChunkPages;
  const float *part = p.ws + static_cast<size_t>(u) * p.n_split * (HD + 2);
  float M = -INFINITY;
  for (int c = 0; c < nsplit; ++c) M = fmaxf(M, part[c * (HD + 2) + HD]);
  float lsum = 0.f;
  float o[HD / 32];
#pragma unroll
  for (int k = 0; k < HD / 32; ++k) o[k] = 0.f;
  for (int c = 0; c < nsplit; ++c) {
    const float *pc = part + c * (HD + 2);
    const float f = ex2(pc[HD] - M);
    lsum = fmaf(f, pc[HD + 1], lsum);
#pragma unroll
    for (int k = 0; k < HD / 32; ++k) o[k] = fmaf(f, pc[lane + 32 * k], o[k]);
  }
  const float inv = 1.f / lsum;
  if (p.o_f32) {
    float *dst = static_cast<float *>(p.o) + static_cast<size_t>(u) * HD;
#pragma unroll
    for (int k = 0; k < HD / 32; ++k) dst[lane + 32 * k] = o[k] * inv;
  } else {
    uint16_t *dst = static_cast<uint16_t *>(p.o) + static_cast<size_t>(u) * HD;
#pragma unroll
    for (int k = 0; k < HD / 32; ++k) dst[lane + 32 * k] = static_cast<uint16_t>(pack_bf16x2(o[k] * inv, 0.f) & 0xffffu);
  }
  if (lane == 0 && p.lse) p.lse[u] = (M + lg2(lsum)) * 0.6931471805599453f;
}

}  // namespace fa
