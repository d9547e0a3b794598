// Exact top-k selection per row (radix select on order-preserving keys).
// (DeepSeek-V4 CSA Step 2: keep the top-k indexer scores; ties to the lower
// index; indices emitted ascending, -1 padded.)
//
// One CTA per row.  Scores map to 32-bit keys whose unsigned order is the
// float order (-0 folded onto +0).  Three MSB-first histogram passes over
// 12, 12 and 8 key bits (4096-bin shared-memory histograms: a score's sign,
// exponent and top mantissa bits land in distinct bins, which keeps
// same-address atomics rare) find the k-th largest key K and how many of its
// ties to keep; a pass stops early once the threshold bucket is taken whole.
// A last pass in index order writes every key > K plus the first r ties, with
// output slots from a block-wide prefix count, so the list comes out
// ascending.  Rows up to kMaxCachedKeys are staged in shared memory once;
// longer rows are re-read from L2 on every pass.
#pragma once
#include "common.cuh"

namespace lcsa {

constexpr int kTopkThreads = 512;
constexpr int kMaxCachedKeys = 32768;   // 128 KiB of dynamic shared memory
constexpr int kTopkBins = 4096;

__device__ __forceinline__ uint32_t score_key(float s) {
  uint32_t u = __float_as_uint(s);
  if (u == 0x80000000u) u = 0u;                      // -0.0 == +0.0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive block scan (NT threads); also returns the block total.
template <int NT>
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* s_warp, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_warp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = lane < NT / 32 ? s_warp[lane] : 0u;
    uint32_t z = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t y = __shfl_up_sync(0xffffffffu, z, o);
      if (lane >= o) z += y;
    }
    if (lane < NT / 32) s_warp[lane] = z - w;       // exclusive warp offsets
    if (lane == 31) *total = z;
  }
  __syncthreads();
  return s_warp[warp] + x - v;
}

template <int NT>
__global__ void __launch_bounds__(NT)
topk_rows_kernel(const float* __restrict__ scores, long long ld, int n_cols,
                 const int32_t* __restrict__ n_valid, int k, int32_t* __restrict__ idx_out,
                 int cache_cap) {
  static_assert(kTopkBins == 8 * NT, "each thread owns 8 bins");
  extern __shared__ uint32_t s_keys[];
  __shared__ uint32_t s_hist[kTopkBins];
  __shared__ uint32_t s_warp[32];
  __shared__ uint32_t s_total;
  __shared__ uint32_t s_prefix, s_mask, s_kr;
  __shared__ int s_done;

  const int row = blockIdx.x;
  int n = n_cols;
  if (n_valid != nullptr) {
    n = n_valid[row];
    n = n < 0 ? 0 : (n > n_cols ? n_cols : n);
  }
  const float* src = scores + (long long)row * ld;
  int32_t* dst = idx_out + (long long)row * k;

  if (n <= k) {
    for (int i = threadIdx.x; i < k; i += NT) dst[i] = i < n ? i : -1;
    return;
  }
  const bool cached = n <= cache_cap;
  if (cached)
    for (int i = threadIdx.x; i < n; i += NT) s_keys[i] = score_key(__ldg(src + i));
  if (threadIdx.x == 0) { s_prefix = 0u; s_mask = 0u; s_kr = (uint32_t)k; s_done = 0; }

  for (int pass = 0; pass < 3; ++pass) {
    const int shift = pass == 0 ? 20 : (pass == 1 ? 8 : 0);
    const uint32_t dmask = pass == 2 ? 0xFFu : 0xFFFu;
    for (int i = threadIdx.x; i < kTopkBins; i += NT) s_hist[i] = 0u;
    __syncthreads();
    const uint32_t prefix = s_prefix, mask = s_mask;
    for (int i = threadIdx.x; i < n; i += NT) {
      const uint32_t key = cached ? s_keys[i] : score_key(__ldg(src + i));
      if ((key & mask) == prefix) atomicAdd(&s_hist[(key >> shift) & dmask], 1u);
    }
    __syncthreads();
    // Thread t owns bins [4095-8t-7, 4095-8t] (descending); a block scan of the
    // per-thread sums locates the bin where the count from the top reaches kr.
    const uint32_t kr = s_kr;
    uint32_t cnt[8], sum = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) { cnt[q] = s_hist[kTopkBins - 1 - 8 * threadIdx.x - q]; sum += cnt[q]; }
    const uint32_t excl = block_excl_scan<NT>(sum, s_warp, &s_total);
    if (excl < kr && excl + sum >= kr) {             // exactly one thread
      uint32_t c = excl;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (c + cnt[q] >= kr) {
          const uint32_t bin = (uint32_t)(kTopkBins - 1 - 8 * threadIdx.x - q);
          const uint32_t krem = kr - c;
          s_prefix = prefix | (bin << shift);
          s_mask = mask | (dmask << shift);
          s_kr = krem;
          s_done = (krem == cnt[q]) ? 1 : 0;       // whole bucket taken: no need to refine
          break;
        }
        c += cnt[q];
      }
    }
    __syncthreads();
    if (s_done) break;
  }

  // Index-order emission: keys above the bucket, plus the first kr of its ties.
  const uint32_t prefix = s_prefix, mask = s_mask, kr = s_kr;
  uint32_t gt_before = 0, eq_before = 0;
  for (int base = 0; base < n; base += NT) {
    const int i = base + threadIdx.x;
    uint32_t a = 0, e = 0;
    if (i < n) {
      const uint32_t key = (cached ? s_keys[i] : score_key(__ldg(src + i))) & mask;
      a = key > prefix;
      e = key == prefix;
    }
    const uint32_t ex = block_excl_scan<NT>(a | (e << 16), s_warp, &s_total);
    const uint32_t pa = ex & 0xffffu, pe = ex >> 16;
    if (a) {
      const uint32_t eqb = eq_before + pe;
      dst[gt_before + pa + (eqb < kr ? eqb : kr)] = i;
    } else if (e && eq_before + pe < kr) {
      dst[gt_before + pa + eq_before + pe] = i;
    }
    const uint32_t tot = s_total;
    gt_before += tot & 0xffffu;
    eq_before += tot >> 16;
    __syncthreads();                                   // s_warp / s_total reuse
  }
}

static cudaError_t launch_topk(const float* scores, int rows, int n_cols, long long ld, const int32_t* n_valid,
                               int k, int32_t* idx_out, cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  // Rows longer than k are staged in shared memory when they fit.
  const int cache_cap = n_cols <= k ? 0 : (n_cols < kMaxCachedKeys ? n_cols : kMaxCachedKeys);
  const size_t smem = (size_t)cache_cap * 4;
  cudaError_t e = cudaFuncSetAttribute(topk_rows_kernel<kTopkThreads>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxCachedKeys * 4);
  if (e != cudaSuccess) return e;
  count_launch();
  topk_rows_kernel<kTopkThreads><<<rows, kTopkThreads, smem, st>>>(scores, ld, n_cols, n_valid, k, idx_out,
                                                                   cache_cap);
  return cudaGetLastError();
}

}  // namespace lcsa
