// fa_lib.cu -- the C ABI declared in include/fa.h: argument checks, TMA descriptors, launches.
// Host code only decides shapes and launches; every step of the attention itself runs in the
// kernels of fa_prefill.cuh, fa_backward.cuh, fa_decode.cuh and fa_merge.cuh.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <climits>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "fa.h"
#include "fa_backward.cuh"
#include "fa_decode.cuh"
#include "fa_merge.cuh"
#include "fa_prefill.cuh"

namespace fa {
// One thread waits on a barrier that nothing arrives at; the bounded wait must give up.
__global__ void selftest_wait_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  abort_flag = 0;
  mbar_init(&bar, 1);
  fence_mbar_init();
  mbar_wait(&bar, 0, &abort_flag, limit_ns);  // records FA_ERR_TIMEOUT when it gives up
}

// MUFU throughput probe: every thread runs kEx2Chains independent chains x <- 2^x - 1.5 (which
// stays in [-1.5, 0.5]), so the exponentials, not their latency, bound the kernel.  The sink is
// written only if the sum takes a value it never takes, which keeps the work alive.
constexpr int kEx2Chains = 16;
__global__ void __launch_bounds__(256) ex2_rate_kernel(float *sink, int iters) {
  float x[kEx2Chains];
#pragma unroll
  for (int i = 0; i < kEx2Chains; ++i) x[i] = -1.f + 1e-2f * i + 1e-5f * threadIdx.x;
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int i = 0; i < kEx2Chains; ++i) x[i] = ex2(x[i]) - 1.5f;
  }
  float acc = 0.f;
#pragma unroll
  for (int i = 0; i < kEx2Chains; ++i) acc += x[i];
  if (acc == 1.0e30f) *sink = acc;
}

// HBM read probe: a grid-stride sweep over the buffer with the decode kernel's 16-byte streaming
// loads, four in flight per thread; the words are xor-folded so the loads stay live.
__global__ void __launch_bounds__(512) read_rate_kernel(const uint4 *buf, size_t n16, float *sink) {
  uint32_t acc = 0;
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  for (; i + 3 * stride < n16; i += 4 * stride) {
    uint4 a = ld_stream_v4(buf + i), b = ld_stream_v4(buf + i + stride);
    uint4 c = ld_stream_v4(buf + i + 2 * stride), d = ld_stream_v4(buf + i + 3 * stride);
    acc ^= a.x ^ a.y ^ a.z ^ a.w ^ b.x ^ b.y ^ b.z ^ b.w ^ c.x ^ c.y ^ c.z ^ c.w ^ d.x ^ d.y ^ d.z ^ d.w;
  }
  for (; i < n16; i += stride) {
    uint4 a = ld_stream_v4(buf + i);
    acc ^= a.x ^ a.y ^ a.z ^ a.w;
  }
  if (acc == 0x7fc01234u) *sink = __uint_as_float(acc);
}
}  // namespace fa

namespace {

constexpr int kVersion = 100;  // 0.1.0
constexpr int kMaxDevices = 64;

thread_local std::string t_last_error;

fa_status launch_failed(cudaError_t e) {
  t_last_error = cudaGetErrorString(e);
  return FA_ERR_LAUNCH;
}

struct DeviceInfo {
  bool probed = false;
  bool supported = false;
  int num_sms = 0;
  bool prefill_attr[6] = {};  // (d = 64, 128) x (square, paged, key range)
  bool bwd_attr[2] = {false, false};                    // d = 64, 128
};

std::mutex g_mutex;
DeviceInfo g_devices[kMaxDevices];

// Looks up (once per device) whether the current device is an sm_100 part and its SM count.
fa_status current_device(DeviceInfo **out, int *dev_out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return launch_failed(e);
  if (dev < 0 || dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceInfo &d = g_devices[dev];
  if (!d.probed) {
    int major = 0, minor = 0, sms = 0;
    if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return launch_failed(e);
    d.supported = (major == 10 && minor == 0);
    d.num_sms = sms;
    d.probed = true;
  }
  if (!d.supported) return FA_ERR_UNSUPPORTED;
  *out = &d;
  *dev_out = dev;
  return FA_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// [BH, N, d] bf16 viewed as a 3-D tensor (d innermost); boxes of 64 x box_rows x 1 with 128-byte
// swizzle, rows past N read as zeros (and not written by stores).
bool encode_bhnd(CUtensorMap *map, const void *base, int d, int N, int BH, int box_rows = 128) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                        static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(N) * d * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The backward's fp32 dQ accumulator [rows, d] as a 2-D tensor for bulk reductions: boxes of
// 32 features (128 bytes) x box_rows rows, 128-byte swizzle.
bool encode_dq_acc(CUtensorMap *map, float *base, int d, long long rows, int box_rows) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(d) * 4};
  cuuint32_t box[2] = {32, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

bool resolve_scale(float scale, int d, float *out) {
  if (std::isnan(scale) || std::isinf(scale)) return false;
  *out = scale > 0.f ? scale : 1.0f / std::sqrt(static_cast<float>(d));
  return true;
}

// The pools [num_blocks, H, 16, d] as a 4-D tensor (d, 16, H, num_blocks) read in 64 x 16 x 1 x 1
// boxes.  Used at d = 64, where that box is a whole 16-token page of one head (2 KB); d = 128 takes
// the 5-D page maps below.
bool encode_pool(CUtensorMap *map, const void *base, int d, int H, int num_blocks) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), 16, static_cast<cuuint64_t>(H),
                        static_cast<cuuint64_t>(num_blocks)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(16) * d * 2,
                           static_cast<cuuint64_t>(H) * 16 * d * 2};
  cuuint32_t box[4] = {64, 16, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The d = 128 V pool as a 5-D tensor (64 columns, 16 tokens, 2 column halves, H, num_blocks) read
// in 64 x 16 x 2 x 1 x 1 boxes: a whole 16-token page of one head (4 KB) per load, landing as
// [half][token][64 columns].  The half stride (128 bytes) is smaller than the token stride (256
// bytes): the box reorders the page so that each half is the 16 x 128-byte K-group pair the P V
// product reads for its 16 keys.
// The d = 128 K pool as a 5-D tensor (64 columns, 8 tokens, 2 column chunks, 2 token groups,
// num_blocks * H pages of one head) read in 64 x 8 x 2 x 2 x 1 boxes: a whole 16-token page of one
// head (4 KB) per load, landing as [token group][chunk][8 tokens][64 columns].  Eight such pages
// make a K tile whose 8-key groups (1 KB swizzle atoms) sit 2 KB apart for each 64-column chunk,
// the layout issue_qk reads for the paged mode.
bool encode_pool_k_pages(CUtensorMap *map, const void *base, int H, int num_blocks) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[5] = {64, 8, 2, 2, static_cast<cuuint64_t>(num_blocks) * H};
  cuuint64_t strides[4] = {256, 128, 8 * 256, 16 * 256};
  cuuint32_t box[5] = {64, 8, 2, 2, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void *>(base), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_pool_v_pages(CUtensorMap *map, const void *base, int H, int num_blocks) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[5] = {64, 16, 2, static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(num_blocks)};
  cuuint64_t strides[4] = {256, 128, 16 * 256, static_cast<cuuint64_t>(H) * 16 * 256};
  cuuint32_t box[5] = {64, 16, 2, 1, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void *>(base), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Static unit assignment of a causal square launch (fa::UnitTable).  The units are taken in groups
// of heads whose K and V total at most kGroupKvBytes (a quarter of L2), longest pair level first
// within a group, and each goes to the CTA that frees up first under the cost model "key blocks of
// both tiles + 1.5" (ties to the lowest CTA).  A group keeps at least kMinGroupHeads heads (with
// fewer, dozens of CTAs stream the same head's K/V at once, which measured slower) and there are
// no more groups than full rounds of units.  Returns false when the launch takes no table (d = 64,
// see fa::UnitTableOf; or one group: the level-major snake is then as good).
constexpr double kGroupKvBytes = 32.0 * 1024 * 1024;
constexpr int kMinGroupHeads = 16;

static bool build_unit_table(fa::UnitTable &t, int BH, int N, int num_pairs, int grid, int HD) {
  const int units = BH * num_pairs;
  if (HD != 128 || grid <= 0 || grid > fa::kMaxSchedCtas || units <= grid || units > fa::kMaxSchedUnits)
    return false;
  const double kv_head = 2.0 * N * HD * 2;  // bf16 K and V of one (b, h)
  int groups = static_cast<int>(std::ceil(BH * kv_head / kGroupKvBytes));
  groups = std::min({groups, units / grid, BH / kMinGroupHeads});
  if (groups <= 1) return false;
  auto tile_blocks = [&](int pr, int i) {
    const int q0 = pr * 2 * fa::kBM + i * fa::kBM;
    return q0 >= N ? 0 : (std::min(q0 + fa::kBM, N) - 1) / fa::kBN + 1;
  };
  std::vector<int> owner(units);
  std::vector<int> order;
  order.reserve(units);
  std::vector<std::pair<long, int>> heap;  // (finish time in half blocks, CTA): a min-heap
  for (int c = 0; c < grid; ++c) heap.push_back({0, c});
  auto later = [](const std::pair<long, int> &a, const std::pair<long, int> &b) { return a > b; };
  std::make_heap(heap.begin(), heap.end(), later);
  for (int g = 0, h0 = 0; g < groups; ++g) {
    const int gk = BH / groups + (g < BH % groups ? 1 : 0);
    for (int level = 0; level < num_pairs; ++level) {
      const int pr = num_pairs - 1 - level;
      const long cost = 2L * (tile_blocks(pr, 0) + tile_blocks(pr, 1)) + 3;
      for (int bh = h0; bh < h0 + gk; ++bh) {
        std::pop_heap(heap.begin(), heap.end(), later);
        const int u = level * BH + bh;
        owner[u] = heap.back().second;
        order.push_back(u);
        heap.back().first += cost;
        std::push_heap(heap.begin(), heap.end(), later);
      }
    }
    h0 += gk;
  }
  std::vector<int> count(grid + 1, 0);
  for (int u = 0; u < units; ++u) ++count[owner[u] + 1];
  for (int c = 0; c < grid; ++c) count[c + 1] += count[c];
  for (int c = 0; c <= grid; ++c) t.start[c] = static_cast<uint16_t>(count[c]);
  std::vector<int> fill(count.begin(), count.end() - 1);
  for (int u : order) t.unit[fill[owner[u]]++] = static_cast<uint16_t>(u);  // per CTA in run order
  t.count = units;
  return true;
}

// The table of the last causal square launch made by this thread, reused while the shape repeats.
struct UnitTableCache {
  int BH = -1, N = -1, grid = -1, HD = -1;
  bool valid = false;
  fa::UnitTable table{};
};

static const fa::UnitTable &unit_table(int BH, int N, int num_pairs, int grid, int HD) {
  static thread_local UnitTableCache cache;
  static const fa::UnitTable none{};
  if (cache.BH != BH || cache.N != N || cache.grid != grid || cache.HD != HD) {
    cache.BH = BH, cache.N = N, cache.grid = grid, cache.HD = HD;
    cache.valid = build_unit_table(cache.table, BH, N, num_pairs, grid, HD);
  }
  return cache.valid ? cache.table : none;
}

template <int HD, int kMode>
fa_status launch_prefill(DeviceInfo &dev, const CUtensorMap &tq, const CUtensorMap &tk,
                         const CUtensorMap &tv, fa::PrefillParams p, cudaStream_t stream,
                         const CUtensorMap *to = nullptr) {
  using C = fa::PrefillCfg<HD>;
  p.num_pairs = (p.N + 2 * fa::kBM - 1) / (2 * fa::kBM);
  p.num_units = p.BH * p.num_pairs;
  const int slot = (HD == 128 ? 1 : 0) + 2 * kMode;
  {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!dev.prefill_attr[slot]) {
      cudaError_t e = cudaFuncSetAttribute(fa::fa_prefill_kernel<HD, kMode>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(C::kSmemBytes));
      if (e != cudaSuccess) return launch_failed(e);
      dev.prefill_attr[slot] = true;
    }
  }
  const int grid = p.num_units < dev.num_sms ? p.num_units : dev.num_sms;
  // without an O map (p.o_tma = 0) the kernel never reads its O map argument
  typename fa::UnitTableOf<HD, kMode>::type tab{};
  if constexpr (!std::is_same_v<decltype(tab), fa::NoUnitTable>) {
    if (p.causal) tab = unit_table(p.BH, p.N, p.num_pairs, grid, HD);
  }
  fa::fa_prefill_kernel<HD, kMode><<<grid, fa::kPrefillThreads, C::kSmemBytes, stream>>>(
      tq, tk, tv, to != nullptr ? *to : tq, p, tab);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? FA_OK : launch_failed(e);
}

template <int HD>
fa_status launch_prefill_dense(DeviceInfo &dev, const void *q, const void *k, const void *v,
                               void *o, int o_f32, float *lse, int BH, int N, int causal,
                               float scale, cudaStream_t stream) {
  CUtensorMap tq, tk, tv;
  if (!encode_bhnd(&tq, q, HD, N, BH) || !encode_bhnd(&tk, k, HD, N, BH) ||
      !encode_bhnd(&tv, v, HD, N, BH)) {
    t_last_error = "cuTensorMapEncodeTiled failed";
    return FA_ERR_LAUNCH;
  }
  fa::PrefillParams p{};
  p.o = o;
  p.lse = lse;
  p.o_f32 = o_f32;
  p.BH = BH;
  p.N = N;
  p.causal = causal;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.q_rows = N;
  p.Nk = N;
  // bf16 O leaves through tensor stores of 32-row boxes
  CUtensorMap to;
  p.o_tma = (!o_f32 && encode_bhnd(&to, o, HD, N, BH, 32)) ? 1 : 0;
  return launch_prefill<HD, fa::kModeSquare>(dev, tq, tk, tv, p, stream, p.o_tma ? &to : nullptr);
}

// Backward workspace: dQ accumulator fp32 [BH, Np, d], then LSE2 and D fp32 [BH, Np] each, with
// Np = N rounded up to the 128-row block.
size_t bwd_padded_rows(int BH, int N) {
  return static_cast<size_t>(BH) * ((static_cast<size_t>(N) + fa::kBM - 1) / fa::kBM * fa::kBM);
}

template <int HD>
fa_status launch_bwd(DeviceInfo &dev, const void *q, const void *k, const void *v, const void *o,
                     int o_f32, const void *dout, const float *lse, void *dq, void *dk, void *dv,
                     int g_f32,
                     int BH, int N, int causal, float scale, void *workspace, cudaStream_t stream) {
  using C = fa::BwdCfg<HD>;
  CUtensorMap tq, tk, tv, tdo;
  if (!encode_bhnd(&tq, q, HD, N, BH) || !encode_bhnd(&tk, k, HD, N, BH) ||
      !encode_bhnd(&tv, v, HD, N, BH) || !encode_bhnd(&tdo, dout, HD, N, BH)) {
    t_last_error = "cuTensorMapEncodeTiled failed";
    return FA_ERR_LAUNCH;
  }
  {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!dev.bwd_attr[HD == 128]) {
      cudaError_t e = cudaFuncSetAttribute(fa::fa_bwd_kernel<HD>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(C::kSmemBytes));
      if (e != cudaSuccess) return launch_failed(e);
      dev.bwd_attr[HD == 128] = true;
    }
  }
  const int Np = (N + fa::kBM - 1) / fa::kBM * fa::kBM;
  const size_t prow = static_cast<size_t>(BH) * Np;
  float *dq_acc = static_cast<float *>(workspace);
  float *lse2 = dq_acc + prow * HD;
  float *dvec = lse2 + prow;
  constexpr int kRowThreads = HD / 8;
  const long long prep_threads = static_cast<long long>(prow) * kRowThreads;
  const unsigned prep_blocks = static_cast<unsigned>((prep_threads + 255) / 256);
  if (o_f32)
    fa::fa_bwd_prep_kernel<HD, true><<<prep_blocks, 256, 0, stream>>>(
        o, static_cast<const uint16_t *>(dout), lse, lse2, dvec, dq_acc, BH, N, Np);
  else
    fa::fa_bwd_prep_kernel<HD, false><<<prep_blocks, 256, 0, stream>>>(
        o, static_cast<const uint16_t *>(dout), lse, lse2, dvec, dq_acc, BH, N, Np);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return launch_failed(e);
  fa::BwdParams p{};
  p.lse2 = lse2;
  p.dvec = dvec;
  p.dq_acc = dq_acc;
  p.dk = dk;
  p.dv = dv;
  p.g_f32 = g_f32;
  p.BH = BH;
  p.N = N;
  p.Np = Np;
  p.nkb = Np / fa::kBN;
  p.causal = causal;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.scale = scale;
  CUtensorMap tdq;
  if (!encode_dq_acc(&tdq, dq_acc, HD, static_cast<long long>(prow), C::kBoxRows)) {
    t_last_error = "cuTensorMapEncodeTiled failed";
    return FA_ERR_LAUNCH;
  }
  // persistent: one CTA per SM at most, each taking pairs of key blocks (see the kernel)
  const long long pairs = static_cast<long long>(BH) * ((p.nkb + 1) / 2);
  const unsigned grid = static_cast<unsigned>(pairs < dev.num_sms ? pairs : dev.num_sms);
  fa::fa_bwd_kernel<HD><<<grid, fa::kBwdThreads, C::kSmemBytes, stream>>>(tq, tk, tv, tdo, tdq, p);
  if ((e = cudaGetLastError()) != cudaSuccess) return launch_failed(e);
  const long long post_threads = static_cast<long long>(BH) * N * kRowThreads;
  fa::fa_bwd_dq_kernel<HD><<<static_cast<unsigned>((post_threads + 255) / 256), 256, 0, stream>>>(
      dq_acc, dq, g_f32, scale, BH, N, Np);
  e = cudaGetLastError();
  return e == cudaSuccess ? FA_OK : launch_failed(e);
}

int decode_splits(int max_blocks) {
  return (max_blocks + fa::kDecodeChunkPages - 1) / fa::kDecodeChunkPages;
}

}  // namespace

extern "C" {

fa_status fa_fwd(const void *q, const void *k, const void *v, void *o, fa_out_dtype o_dtype,
                 float *lse, int B, int H, int N, int d, int causal, float scale,
                 fa_stream_t stream) {
  if (!q || !k || !v || !o) return FA_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || N < 1) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (o_dtype != FA_OUT_BF16 && o_dtype != FA_OUT_F32) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * H > INT_MAX) return FA_ERR_INVALID_ARG;
  // work units (pairs of 128-row query tiles) are counted in an int
  if (static_cast<long long>(B) * H * ((static_cast<long long>(N) + 2 * fa::kBM - 1) / (2 * fa::kBM)) >
      INT_MAX)
    return FA_ERR_INVALID_ARG;
  float sc;
  if (!resolve_scale(scale, d, &sc)) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return FA_ERR_ALIGNMENT;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return FA_ERR_ALIGNMENT;
  const int BH = B * H;
  const size_t rows = static_cast<size_t>(BH) * N;
  const size_t in_bytes = rows * d * 2;
  const size_t o_bytes = rows * d * (o_dtype == FA_OUT_F32 ? 4 : 2);
  if (overlaps(o, o_bytes, q, in_bytes) || overlaps(o, o_bytes, k, in_bytes) ||
      overlaps(o, o_bytes, v, in_bytes))
    return FA_ERR_INVALID_ARG;
  if (lse && (overlaps(lse, rows * 4, q, in_bytes) || overlaps(lse, rows * 4, k, in_bytes) ||
              overlaps(lse, rows * 4, v, in_bytes) || overlaps(lse, rows * 4, o, o_bytes)))
    return FA_ERR_INVALID_ARG;
  DeviceInfo *dev = nullptr;
  int dev_id = 0;
  fa_status st = current_device(&dev, &dev_id);
  if (st != FA_OK) return st;
  const int o_f32 = o_dtype == FA_OUT_F32;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (d == 128) return launch_prefill_dense<128>(*dev, q, k, v, o, o_f32, lse, BH, N, causal, sc, s);
  return launch_prefill_dense<64>(*dev, q, k, v, o, o_f32, lse, BH, N, causal, sc, s);
}

size_t fa_bwd_workspace_size(int B, int H, int N, int d) {
  if (B < 1 || H < 1 || N < 1 || (d != 64 && d != 128)) return 0;
  if (static_cast<long long>(B) * H > INT_MAX) return 0;
  return bwd_padded_rows(B * H, N) * (d + 2) * sizeof(float);
}

fa_status fa_bwd(const void *q, const void *k, const void *v, const void *o, fa_out_dtype o_dtype,
                 const void *dout, const float *lse, void *dq, void *dk, void *dv,
                 fa_out_dtype g_dtype, int B, int H, int N, int d, int causal, float scale,
                 void *workspace, size_t workspace_bytes, fa_stream_t stream) {
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv) return FA_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || N < 1) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (g_dtype != FA_OUT_BF16 && g_dtype != FA_OUT_F32) return FA_ERR_INVALID_ARG;
  if (o_dtype != FA_OUT_BF16 && o_dtype != FA_OUT_F32) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * H > INT_MAX) return FA_ERR_INVALID_ARG;
  const int BH = B * H;
  if (static_cast<long long>(BH) * ((N + fa::kBN - 1) / fa::kBN) > INT_MAX) return FA_ERR_INVALID_ARG;
  float sc;
  if (!resolve_scale(scale, d, &sc)) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return FA_ERR_ALIGNMENT;
  if (reinterpret_cast<uintptr_t>(lse) & 3u) return FA_ERR_ALIGNMENT;
  const size_t need = fa_bwd_workspace_size(B, H, N, d);
  if (!workspace || workspace_bytes < need) return FA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return FA_ERR_ALIGNMENT;
  const size_t rows = static_cast<size_t>(BH) * N;
  const size_t in_bytes = rows * d * 2, g_bytes = rows * d * (g_dtype == FA_OUT_F32 ? 4 : 2);
  const size_t o_bytes = rows * d * (o_dtype == FA_OUT_F32 ? 4 : 2);
  const void *ins[6] = {q, k, v, o, dout, lse};
  const size_t in_sizes[6] = {in_bytes, in_bytes, in_bytes, o_bytes, in_bytes, rows * 4};
  void *outs[4] = {dq, dk, dv, workspace};
  const size_t out_sizes[4] = {g_bytes, g_bytes, g_bytes, need};
  for (int a = 0; a < 4; ++a) {
    for (int b = 0; b < 6; ++b)
      if (overlaps(outs[a], out_sizes[a], ins[b], in_sizes[b])) return FA_ERR_INVALID_ARG;
    for (int b = a + 1; b < 4; ++b)
      if (overlaps(outs[a], out_sizes[a], outs[b], out_sizes[b])) return FA_ERR_INVALID_ARG;
  }
  DeviceInfo *dev = nullptr;
  int dev_id = 0;
  fa_status st = current_device(&dev, &dev_id);
  if (st != FA_OK) return st;
  const int g_f32 = g_dtype == FA_OUT_F32, o_f32 = o_dtype == FA_OUT_F32;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (d == 128)
    return launch_bwd<128>(*dev, q, k, v, o, o_f32, dout, lse, dq, dk, dv, g_f32, BH, N, causal,
                           sc, workspace, s);
  return launch_bwd<64>(*dev, q, k, v, o, o_f32, dout, lse, dq, dk, dv, g_f32, BH, N, causal, sc,
                        workspace, s);
}

size_t fa_decode_workspace_size(int num_seqs, int H, int d, int max_blocks_per_seq) {
  if (num_seqs < 1 || H < 1 || max_blocks_per_seq < 1 || (d != 64 && d != 128)) return 0;
  const size_t units = static_cast<size_t>(num_seqs) * H * decode_splits(max_blocks_per_seq);
  return units * (d + 2) * sizeof(float);
}

fa_status fa_decode_paged(const void *q, const void *k_pool, const void *v_pool,
                          const int32_t *block_table, int max_blocks_per_seq,
                          const int32_t *seq_lens, int num_blocks, void *o, fa_out_dtype o_dtype,
                          float *lse, int S, int H, int d, float scale, void *workspace,
                          size_t workspace_bytes, fa_stream_t stream) {
  if (!q || !k_pool || !v_pool || !block_table || !seq_lens || !o) return FA_ERR_INVALID_ARG;
  if (S < 1 || H < 1 || max_blocks_per_seq < 1 || num_blocks < 1) return FA_ERR_INVALID_ARG;
  if (o_dtype != FA_OUT_BF16 && o_dtype != FA_OUT_F32) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (static_cast<long long>(S) * H > INT_MAX / 4) return FA_ERR_INVALID_ARG;
  if (static_cast<long long>(max_blocks_per_seq) * fa::kPage > INT_MAX) return FA_ERR_INVALID_ARG;
  float sc;
  if (!resolve_scale(scale, d, &sc)) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_pool) || !aligned16(v_pool) || !aligned16(o))
    return FA_ERR_ALIGNMENT;
  if ((reinterpret_cast<uintptr_t>(block_table) & 3u) || (reinterpret_cast<uintptr_t>(seq_lens) & 3u))
    return FA_ERR_ALIGNMENT;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return FA_ERR_ALIGNMENT;
  const size_t need = fa_decode_workspace_size(S, H, d, max_blocks_per_seq);
  if (!workspace || workspace_bytes < need) return FA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return FA_ERR_ALIGNMENT;
  const size_t o_bytes = static_cast<size_t>(S) * H * d * (o_dtype == FA_OUT_F32 ? 4 : 2);
  if (overlaps(o, o_bytes, workspace, need) || (lse && overlaps(lse, static_cast<size_t>(S) * H * 4, workspace, need)))
    return FA_ERR_INVALID_ARG;
  DeviceInfo *dev = nullptr;
  int dev_id = 0;
  fa_status st = current_device(&dev, &dev_id);
  if (st != FA_OK) return st;

  fa::DecodeParams p;
  p.q = static_cast<const uint16_t *>(q);
  p.kp = static_cast<const uint16_t *>(k_pool);
  p.vp = static_cast<const uint16_t *>(v_pool);
  p.table = block_table;
  p.lens = seq_lens;
  p.max_blocks = max_blocks_per_seq;
  p.num_blocks = num_blocks;
  p.H = H;
  p.scale_log2 = sc * 1.4426950408889634f;
  p.ws = static_cast<float *>(workspace);
  p.n_split = decode_splits(max_blocks_per_seq);
  p.o = o;
  p.o_f32 = o_dtype == FA_OUT_F32;
  p.lse = lse;
  p.SH = S * H;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const dim3 grid1(p.n_split, H, S);
  const int grid2 = (p.SH + 3) / 4;
  if (d == 128) {
    fa::fa_decode_partial_kernel<128><<<grid1, fa::kDecodeThreads, 0, s>>>(p);
    fa::fa_decode_combine_kernel<128><<<grid2, 128, 0, s>>>(p);
  } else {
    fa::fa_decode_partial_kernel<64><<<grid1, fa::kDecodeThreads, 0, s>>>(p);
    fa::fa_decode_combine_kernel<64><<<grid2, 128, 0, s>>>(p);
  }
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? FA_OK : launch_failed(e);
}

}  // extern "C"

// ---------------------------------------------------------------------------------------------
// Allocation-free decode: the split-context scratch lives in a static device array.
// ---------------------------------------------------------------------------------------------
namespace {

// Held by every GPU that loads this library, for the life of the process.
static __device__ __align__(256) unsigned char g_noalloc_scratch[FA_NOALLOC_SCRATCH_BYTES];

std::mutex g_noalloc_mutex;
void *g_noalloc_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on `dev` (the current device), looked up once per device.
// In host code the array's name is only a host-side stand-in, never a device address.
fa_status noalloc_scratch(int dev, void **out) {
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (!g_noalloc_ptr[dev]) {
    void *ptr = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess) return launch_failed(e);
    if (!ptr) {
      t_last_error = "cudaGetSymbolAddress returned no address for the decode scratch";
      return FA_ERR_LAUNCH;
    }
    g_noalloc_ptr[dev] = ptr;
  }
  *out = g_noalloc_ptr[dev];
  return FA_OK;
}

}  // namespace

extern "C" {

fa_status fa_decode_paged_noalloc(const void *q, const void *k_pool, const void *v_pool,
                                  const int32_t *block_table, int max_blocks_per_seq,
                                  const int32_t *seq_lens, int num_blocks, void *o,
                                  fa_out_dtype o_dtype, float *lse, int S, int H, int d,
                                  float scale, fa_stream_t stream) {
  if (!q || !k_pool || !v_pool || !block_table || !seq_lens || !o) return FA_ERR_INVALID_ARG;
  if (S < 1 || H < 1 || max_blocks_per_seq < 1 || num_blocks < 1) return FA_ERR_INVALID_ARG;
  if (o_dtype != FA_OUT_BF16 && o_dtype != FA_OUT_F32) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (static_cast<long long>(S) * H > INT_MAX / 4) return FA_ERR_INVALID_ARG;
  if (static_cast<long long>(max_blocks_per_seq) * fa::kPage > INT_MAX) return FA_ERR_INVALID_ARG;
  float sc;
  if (!resolve_scale(scale, d, &sc)) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_pool) || !aligned16(v_pool) || !aligned16(o))
    return FA_ERR_ALIGNMENT;
  if ((reinterpret_cast<uintptr_t>(block_table) & 3u) || (reinterpret_cast<uintptr_t>(seq_lens) & 3u))
    return FA_ERR_ALIGNMENT;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return FA_ERR_ALIGNMENT;
  const size_t need = fa_decode_workspace_size(S, H, d, max_blocks_per_seq);
  if (need > FA_NOALLOC_SCRATCH_BYTES) {
    t_last_error = "fa_decode_paged_noalloc: these sizes need " + std::to_string(need) +
                   " bytes of scratch; the static array holds " +
                   std::to_string(FA_NOALLOC_SCRATCH_BYTES);
    return FA_ERR_WORKSPACE;
  }
  DeviceInfo *dev = nullptr;
  int dev_id = 0;
  fa_status st = current_device(&dev, &dev_id);
  if (st != FA_OK) return st;
  void *scratch = nullptr;
  if ((st = noalloc_scratch(dev_id, &scratch)) != FA_OK) return st;

  fa::DecodeParams p;
  p.q = static_cast<const uint16_t *>(q);
  p.kp = static_cast<const uint16_t *>(k_pool);
  p.vp = static_cast<const uint16_t *>(v_pool);
  p.table = block_table;
  p.lens = seq_lens;
  p.max_blocks = max_blocks_per_seq;
  p.num_blocks = num_blocks;
  p.H = H;
  p.scale_log2 = sc * 1.4426950408889634f;
  p.ws = static_cast<float *>(scratch);
  p.n_split = decode_splits(max_blocks_per_seq);
  p.o = o;
  p.o_f32 = o_dtype == FA_OUT_F32;
  p.lse = lse;
  p.SH = S * H;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const dim3 grid1(p.n_split, H, S);
  const int grid2 = (p.SH + 3) / 4;
  if (d == 128) {
    fa::fa_decode_partial_kernel<128><<<grid1, fa::kDecodeThreads, 0, s>>>(p);
    fa::fa_decode_combine_kernel<128><<<grid2, 128, 0, s>>>(p);
  } else {
    fa::fa_decode_partial_kernel<64><<<grid1, fa::kDecodeThreads, 0, s>>>(p);
    fa::fa_decode_combine_kernel<64><<<grid2, 128, 0, s>>>(p);
  }
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? FA_OK : launch_failed(e);
}

// Shared body of fa_prefill_paged and fa_tree_attention (tree_mask null: plain or causal chunk).
static fa_status prefill_paged_impl(const void *q, const void *k_pool, const void *v_pool,
                             const int32_t *block_table, int max_blocks_per_seq,
                                    const int32_t *seq_lens, int num_blocks,
                                    const uint64_t *tree_mask, void *o, fa_out_dtype o_dtype,
                                    float *lse, int S, int H, int Lq, int d, int causal,
                                    float scale, fa_stream_t stream) {
  if (!q || !k_pool || !v_pool || !block_table || !seq_lens || !o) return FA_ERR_INVALID_ARG;
  if (S < 1 || H < 1 || Lq < 1 || max_blocks_per_seq < 1 || num_blocks < 1) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (o_dtype != FA_OUT_BF16 && o_dtype != FA_OUT_F32) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (static_cast<long long>(S) * H * Lq > INT_MAX) return FA_ERR_INVALID_ARG;
  if (static_cast<long long>(max_blocks_per_seq) * fa::kPage > INT_MAX) return FA_ERR_INVALID_ARG;
  if (Lq > max_blocks_per_seq * fa::kPage) return FA_ERR_INVALID_ARG;
  // the d = 128 K map indexes (block, head) pages as block * H + head, block up to num_blocks
  if ((static_cast<long long>(num_blocks) + 1) * H > INT_MAX) return FA_ERR_INVALID_ARG;
  float sc;
  if (!resolve_scale(scale, d, &sc)) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_pool) || !aligned16(v_pool) || !aligned16(o))
    return FA_ERR_ALIGNMENT;
  if ((reinterpret_cast<uintptr_t>(block_table) & 3u) || (reinterpret_cast<uintptr_t>(seq_lens) & 3u))
    return FA_ERR_ALIGNMENT;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return FA_ERR_ALIGNMENT;
  const size_t rows = static_cast<size_t>(S) * H * Lq;
  const size_t q_bytes = rows * d * 2, o_bytes = rows * d * (o_dtype == FA_OUT_F32 ? 4 : 2);
  const size_t pool_bytes = static_cast<size_t>(num_blocks) * H * fa::kPage * d * 2;
  if (overlaps(o, o_bytes, q, q_bytes) || overlaps(o, o_bytes, k_pool, pool_bytes) ||
      overlaps(o, o_bytes, v_pool, pool_bytes))
    return FA_ERR_INVALID_ARG;
  if (lse && (overlaps(lse, rows * 4, o, o_bytes) || overlaps(lse, rows * 4, q, q_bytes) ||
              overlaps(lse, rows * 4, k_pool, pool_bytes) || overlaps(lse, rows * 4, v_pool, pool_bytes)))
    return FA_ERR_INVALID_ARG;
  DeviceInfo *dev = nullptr;
  int dev_id = 0;
  fa_status st = current_device(&dev, &dev_id);
  if (st != FA_OK) return st;
  CUtensorMap tq, tk, tv;
  const int BH = S * H;
  // d = 128: K and V pages arrive as one 4 KB box each (see encode_pool_k_pages / _v_pages)
  const bool pages = d == 128;
  if (!encode_bhnd(&tq, q, d, Lq, BH) ||
      !(pages ? encode_pool_k_pages(&tk, k_pool, H, num_blocks)
              : encode_pool(&tk, k_pool, d, H, num_blocks)) ||
      !(pages ? encode_pool_v_pages(&tv, v_pool, H, num_blocks)
              : encode_pool(&tv, v_pool, d, H, num_blocks))) {
    t_last_error = "cuTensorMapEncodeTiled failed";
    return FA_ERR_LAUNCH;
  }
  fa::PrefillParams p{};
  p.o = o;
  p.lse = lse;
  p.o_f32 = o_dtype == FA_OUT_F32;
  p.BH = BH;
  p.N = Lq;
  p.causal = causal;
  p.scale_log2 = sc * 1.4426950408889634f;
  p.seq_lens = seq_lens;
  p.block_table = block_table;
  p.max_blocks = max_blocks_per_seq;
  p.num_blocks = num_blocks;
  p.H = H;
  p.tree_mask = tree_mask;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  p.q_rows = Lq;
  // bf16 O leaves through tensor stores of 32-row boxes ([S * H, Lq, d] view)
  CUtensorMap to;
  p.o_tma = (o_dtype == FA_OUT_BF16 && encode_bhnd(&to, o, d, Lq, BH, 32)) ? 1 : 0;
  const CUtensorMap *top = p.o_tma ? &to : nullptr;
  if (d == 128) return launch_prefill<128, fa::kModePaged>(*dev, tq, tk, tv, p, s, top);
  return launch_prefill<64, fa::kModePaged>(*dev, tq, tk, tv, p, s, top);
}

fa_status fa_prefill_paged(const void *q, const void *k_pool, const void *v_pool,
                           const int32_t *block_table, int max_blocks_per_seq,
                           const int32_t *seq_lens, int num_blocks, void *o, fa_out_dtype o_dtype,
                           float *lse, int S, int H, int Lq, int d, int causal, float scale,
                           fa_stream_t stream) {
  return prefill_paged_impl(q, k_pool, v_pool, block_table, max_blocks_per_seq, seq_lens,
                            num_blocks, nullptr, o, o_dtype, lse, S, H, Lq, d, causal, scale,
                            stream);
}

fa_status fa_tree_attention(const void *q, const void *k_pool, const void *v_pool,
                            const int32_t *block_table, int max_blocks_per_seq,
                            const int32_t *seq_lens, int num_blocks, const uint64_t *tree_mask,
                            void *o, fa_out_dtype o_dtype, float *lse, int S, int H, int T, int d,
                            float scale, fa_stream_t stream) {
  if (!tree_mask) return FA_ERR_INVALID_ARG;
  if (T < 1 || T > 64) return FA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(tree_mask) & 7u) return FA_ERR_ALIGNMENT;
  if (S >= 1 && H >= 1 && (d == 64 || d == 128)) {
    const size_t o_bytes =
        static_cast<size_t>(S) * H * T * d * (o_dtype == FA_OUT_F32 ? 4 : 2);
    if (overlaps(o, o_bytes, tree_mask, static_cast<size_t>(S) * T * 8)) return FA_ERR_INVALID_ARG;
  }
  return prefill_paged_impl(q, k_pool, v_pool, block_table, max_blocks_per_seq, seq_lens,
                            num_blocks, tree_mask, o, o_dtype, lse, S, H, T, d, 0, scale, stream);
}

fa_status fa_fwd_keyrange(const void *q, const void *k, const void *v, void *o, fa_out_dtype o_dtype,
                          float *lse, int B, int H, int Nq, int q_row0, int Nk, int k_pos0, int d,
                          int causal, float scale, fa_stream_t stream) {
  if (!q || !k || !v || !o) return FA_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || Nq < 1 || Nk < 1 || q_row0 < 0 || q_row0 >= Nq || k_pos0 < 0)
    return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (o_dtype != FA_OUT_BF16 && o_dtype != FA_OUT_F32) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * H > INT_MAX) return FA_ERR_INVALID_ARG;
  // work units (pairs of 128-row query tiles) are counted in an int
  if (static_cast<long long>(B) * H * ((static_cast<long long>(Nq) + 2 * fa::kBM - 1) / (2 * fa::kBM)) >
      INT_MAX)
    return FA_ERR_INVALID_ARG;
  float sc;
  if (!resolve_scale(scale, d, &sc)) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return FA_ERR_ALIGNMENT;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return FA_ERR_ALIGNMENT;
  const int BH = B * H;
  const size_t qrows = static_cast<size_t>(BH) * Nq, krows = static_cast<size_t>(BH) * Nk;
  const size_t o_bytes = qrows * d * (o_dtype == FA_OUT_F32 ? 4 : 2);
  if (overlaps(o, o_bytes, q, qrows * d * 2) || overlaps(o, o_bytes, k, krows * d * 2) ||
      overlaps(o, o_bytes, v, krows * d * 2))
    return FA_ERR_INVALID_ARG;
  if (lse && (overlaps(lse, qrows * 4, o, o_bytes) || overlaps(lse, qrows * 4, q, qrows * d * 2) ||
              overlaps(lse, qrows * 4, k, krows * d * 2) || overlaps(lse, qrows * 4, v, krows * d * 2)))
    return FA_ERR_INVALID_ARG;
  DeviceInfo *dev = nullptr;
  int dev_id = 0;
  fa_status st = current_device(&dev, &dev_id);
  if (st != FA_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int o_f32 = o_dtype == FA_OUT_F32;
  // causal: rows before the range's first key see none of it
  const int q_start = causal ? std::max(q_row0, std::min(k_pos0, Nq)) : q_row0;
  if (q_start > q_row0) {
    const long long threads = static_cast<long long>(BH) * (q_start - q_row0) * (d / 4);
    const unsigned blocks = static_cast<unsigned>((threads + 255) / 256);
    if (d == 128)
      fa::fa_empty_rows_kernel<128><<<blocks, 256, 0, s>>>(o, o_f32, lse, BH, Nq, q_row0, q_start);
    else
      fa::fa_empty_rows_kernel<64><<<blocks, 256, 0, s>>>(o, o_f32, lse, BH, Nq, q_row0, q_start);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return launch_failed(e);
  }
  if (q_start >= Nq) return FA_OK;
  CUtensorMap tq, tk, tv;
  if (!encode_bhnd(&tq, q, d, Nq, BH) || !encode_bhnd(&tk, k, d, Nk, BH) ||
      !encode_bhnd(&tv, v, d, Nk, BH)) {
    t_last_error = "cuTensorMapEncodeTiled failed";
    return FA_ERR_LAUNCH;
  }
  fa::PrefillParams p{};
  p.o = o;
  p.lse = lse;
  p.o_f32 = o_f32;
  p.BH = BH;
  p.N = Nq - q_start;
  p.causal = causal;
  p.scale_log2 = sc * 1.4426950408889634f;
  p.q_row0 = q_start;
  p.q_rows = Nq;
  p.Nk = Nk;
  p.q_off = causal ? q_start - k_pos0 : 0;
  if (d == 128) return launch_prefill<128, fa::kModeRange>(*dev, tq, tk, tv, p, s);
  return launch_prefill<64, fa::kModeRange>(*dev, tq, tk, tv, p, s);
}

fa_status fa_merge_partials(const float *o_parts, const float *lse_parts, int G, long long rows,
                            int d, void *o, fa_out_dtype o_dtype, float *lse, fa_stream_t stream) {
  if (!o_parts || !lse_parts || !o) return FA_ERR_INVALID_ARG;
  if (G < 1 || rows < 1) return FA_ERR_INVALID_ARG;
  if (o_dtype != FA_OUT_BF16 && o_dtype != FA_OUT_F32) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (rows > (1ll << 40) / d) return FA_ERR_INVALID_ARG;
  if (!aligned16(o_parts) || !aligned16(o) || (reinterpret_cast<uintptr_t>(lse_parts) & 3u))
    return FA_ERR_ALIGNMENT;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return FA_ERR_ALIGNMENT;
  const size_t o_bytes = static_cast<size_t>(rows) * d * (o_dtype == FA_OUT_F32 ? 4 : 2);
  const size_t parts_bytes = static_cast<size_t>(G) * rows * d * 4;
  if (overlaps(o, o_bytes, o_parts, parts_bytes) ||
      overlaps(o, o_bytes, lse_parts, static_cast<size_t>(G) * rows * 4))
    return FA_ERR_INVALID_ARG;
  if (lse && (overlaps(lse, rows * 4, o_parts, parts_bytes) || overlaps(lse, rows * 4, o, o_bytes)))
    return FA_ERR_INVALID_ARG;
  DeviceInfo *dev = nullptr;
  int dev_id = 0;
  fa_status st = current_device(&dev, &dev_id);
  if (st != FA_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const long long threads = rows * (d / 4);
  const unsigned blocks = static_cast<unsigned>((threads + 255) / 256);
  const int o_f32 = o_dtype == FA_OUT_F32;
  if (d == 128)
    fa::fa_merge_kernel<128><<<blocks, 256, 0, s>>>(o_parts, lse_parts, G, rows, o, o_f32, lse);
  else
    fa::fa_merge_kernel<64><<<blocks, 256, 0, s>>>(o_parts, lse_parts, G, rows, o, o_f32, lse);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? FA_OK : launch_failed(e);
}

fa_status fa_get_device_status(fa_stream_t stream) {
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return launch_failed(e);
  int v = 0;
  if ((e = cudaMemcpyFromSymbol(&v, fa::g_device_status, sizeof v)) != cudaSuccess)
    return launch_failed(e);
  if (v != 0) {
    const int zero = 0;
    if ((e = cudaMemcpyToSymbol(fa::g_device_status, &zero, sizeof zero)) != cudaSuccess)
      return launch_failed(e);
  }
  return static_cast<fa_status>(v);
}

fa_status fa_selftest_wait_timeout(unsigned limit_us, fa_stream_t stream) {
  if (limit_us < 1 || limit_us > 2000000u) return FA_ERR_INVALID_ARG;
  DeviceInfo *dev = nullptr;
  int dev_id = 0;
  fa_status st = current_device(&dev, &dev_id);
  if (st != FA_OK) return st;
  fa::selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<uint64_t>(limit_us) * 1000ull);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? FA_OK : launch_failed(e);
}

fa_status fa_probe_ex2_rate(float *sink, int iters, long long *exps_out, fa_stream_t stream) {
  if (!sink || !exps_out || iters < 1 || iters > (1 << 24)) return FA_ERR_INVALID_ARG;
  DeviceInfo *dev = nullptr;
  int dev_id = 0;
  fa_status st = current_device(&dev, &dev_id);
  if (st != FA_OK) return st;
  const int blocks = 4 * dev->num_sms;  // 32 warps per SM: 8 per sub-partition
  fa::ex2_rate_kernel<<<blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(sink, iters);
  *exps_out = static_cast<long long>(blocks) * 256 * iters * fa::kEx2Chains;
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? FA_OK : launch_failed(e);
}

fa_status fa_probe_read_rate(const void *buf, size_t bytes, float *sink, fa_stream_t stream) {
  if (!buf || !sink || bytes < 16 || bytes % 16) return FA_ERR_INVALID_ARG;
  if (!aligned16(buf)) return FA_ERR_ALIGNMENT;
  DeviceInfo *dev = nullptr;
  int dev_id = 0;
  fa_status st = current_device(&dev, &dev_id);
  if (st != FA_OK) return st;
  fa::read_rate_kernel<<<4 * dev->num_sms, 512, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4 *>(buf), bytes / 16, sink);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? FA_OK : launch_failed(e);
}

const char *fa_status_string(fa_status status) {
  switch (status) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG: an argument is out of range";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED: head dim must be 64 or 128 on an sm_100 GPU";
    case FA_ERR_ALIGNMENT: return "FA_ERR_ALIGNMENT: tensors must be 16-byte aligned";
    case FA_ERR_LAUNCH: return "FA_ERR_LAUNCH: the CUDA launch failed (see fa_last_error_string)";
    case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT: a kernel abandoned a device-side wait";
    case FA_ERR_WORKSPACE: return "FA_ERR_WORKSPACE: decode workspace missing or too small";
  }
  return "unknown fa_status";
}

const char *fa_last_error_string(void) { return t_last_error.c_str(); }

fa_status fa_fwd_schedule(int B, int H, int N, int d, int num_ctas, int *start, int *unit,
                          int capacity, int *count) {
  if (count == nullptr || start == nullptr || unit == nullptr) return FA_ERR_INVALID_ARG;
  *count = 0;
  if (B < 1 || H < 1 || N < 1 || num_ctas < 1 || num_ctas > 1024) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  const long long BH = static_cast<long long>(B) * H;
  const long long pairs = (static_cast<long long>(N) + 2 * fa::kBM - 1) / (2 * fa::kBM);
  if (BH * pairs > INT_MAX) return FA_ERR_INVALID_ARG;
  const int units = static_cast<int>(BH * pairs);
  if (capacity < units) return FA_ERR_INVALID_ARG;
  const int grid = std::min(units, num_ctas);
  static thread_local fa::UnitTable t;
  if (!build_unit_table(t, static_cast<int>(BH), N, static_cast<int>(pairs), grid, d)) return FA_OK;
  for (int c = 0; c <= num_ctas; ++c) start[c] = c <= grid ? t.start[c] : units;
  for (int i = 0; i < units; ++i) unit[i] = t.unit[i];
  *count = units;
  return FA_OK;
}

int fa_version(void) { return kVersion; }

}  // extern "C"
