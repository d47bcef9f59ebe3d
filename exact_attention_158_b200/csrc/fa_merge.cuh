// fa_merge.cuh -- merging attention partials computed over disjoint key ranges of one sequence,
// and writing the rows of a key-range partial that see none of its keys.
//
// Sequence-length parallelism ("FlashAttention-2 GPU work partitioning", section 3) carried
// across devices: each device holds one contiguous range of a sequence's keys and values and
// computes, for every query, O_r (normalised over the keys of its range that the query sees) and
// LSE_r.  The ranges' partials combine with the rescaling rule of the tiled algorithm ("Flash
// Attention" (myungum), section 2, steps 11-12), written for log-sum-exps:
//     M = max_r LSE_r,  w_r = exp(LSE_r - M),  O = sum_r w_r O_r / sum_r w_r,  LSE = M + ln sum_r w_r.
// A partial row that sees no key carries LSE = -inf and weight 0.  HBM bound: one pass over the
// partials.
#pragma once
#include "sm100_ptx.cuh"

namespace fa {

constexpr float kLn2Merge = 0.6931471805599453f;

// HD / 4 threads per row, 4 consecutive features each.  o_parts [G, rows, HD] fp32, lse_parts
// [G, rows]; o [rows, HD] (bf16 or fp32), lse [rows] or null.
template <int HD>
__global__ void __launch_bounds__(256) fa_merge_kernel(const float *__restrict__ o_parts,
                                                       const float *__restrict__ lse_parts, int G,
                                                       long long rows, void *o, int o_f32,
                                                       float *lse) {
  constexpr int kT = HD / 4;
  const long long gt = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long row = gt / kT;
  if (row >= rows) return;
  const int part = static_cast<int>(gt % kT);
  float M = -INFINITY;
  for (int g = 0; g < G; ++g) M = fmaxf(M, lse_parts[g * rows + row]);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float wsum = 0.f;
  if (M != -INFINITY) {
    constexpr float kLog2e = 1.4426950408889634f;
    for (int g = 0; g < G; ++g) {
      const float l = lse_parts[g * rows + row];
      if (l == -INFINITY) continue;  // that range holds no key this query sees
      const float w = ex2((l - M) * kLog2e);
      const float4 v = reinterpret_cast<const float4 *>(o_parts + (g * rows + row) * HD)[part];
      acc.x = fmaf(w, v.x, acc.x);
      acc.y = fmaf(w, v.y, acc.y);
      acc.z = fmaf(w, v.z, acc.z);
      acc.w = fmaf(w, v.w, acc.w);
      wsum += w;
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  if (o_f32) {
    reinterpret_cast<float4 *>(static_cast<float *>(o) + row * HD)[part] =
        make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  } else {
    uint2 w2;
    w2.x = pack_bf16x2(acc.x * inv, acc.y * inv);
    w2.y = pack_bf16x2(acc.z * inv, acc.w * inv);
    reinterpret_cast<uint2 *>(static_cast<uint16_t *>(o) + row * HD)[part] = w2;
  }
  if (part == 0 && lse) lse[row] = M == -INFINITY ? -INFINITY : M + lg2(wsum) * kLn2Merge;
}

// Rows [r0, r1) of every (b, h) of O [BH, rows, HD] and LSE [BH, rows]: O = 0, LSE = -inf (a query
// that sees none of the range's keys).  HD / 4 threads per row.
template <int HD>
__global__ void __launch_bounds__(256) fa_empty_rows_kernel(void *o, int o_f32, float *lse, int BH,
                                                            int rows, int r0, int r1) {
  constexpr int kT = HD / 4;
  const int span = r1 - r0;
  const long long gt = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long idx = gt / kT;
  if (idx >= static_cast<long long>(BH) * span) return;
  const int part = static_cast<int>(gt % kT);
  const long long row = (idx / span) * rows + r0 + idx % span;
  if (o_f32)
    reinterpret_cast<float4 *>(static_cast<float *>(o) + row * HD)[part] = make_float4(0.f, 0.f, 0.f, 0.f);
  else
    reinterpret_cast<uint2 *>(static_cast<uint16_t *>(o) + row * HD)[part] = make_uint2(0u, 0u);
  if (part == 0 && lse) lse[row] = -INFINITY;
}

}  // namespace fa
