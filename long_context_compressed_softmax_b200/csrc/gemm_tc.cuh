// Grouped output projection on tcgen05 tensor cores (DeepSeek-V4 "第四步，
// grouped output projection": with head dimension 512, the attention outputs
// of the n_h heads are split into g groups, each group is projected to an
// intermediate width d_g, and the concatenated groups are projected back to d).
//
// Both projections are one kernel: C[M, N] = A[M, K] . B[N, K]^T per group,
// BF16 operands, FP32 accumulation, BF16 output, where group j reads the A
// columns [j K, (j+1) K) (its heads' outputs, contiguous in a token's row), the
// B rows [j N, (j+1) N) (its projection) and writes the C columns
// [j N, (j+1) N).  The merge projection is the same kernel with one group.
//
// Persistent CTAs walk 128 x 256 output tiles (n fastest, so the CTAs in flight
// share A rows in L2; a group's B stays L2-resident).  Warp 0 streams A and B
// K-chunks of 64 by TMA into a 4-stage ring (128B swizzle), warp 1 issues the
// MMAs (M=128, N=256, K=16) into one of two TMEM accumulators, warps 2-5 drain
// the other accumulator (TMEM -> registers -> BF16 -> global) while the next
// tile accumulates.  Every wait is bounded; on expiry the CTA stops, records
// LCSA_DEV_TIMEOUT, drains its copies and frees TMEM.
#pragma once
#include <atomic>

#include "tc_ptx.cuh"

namespace lcsa {

constexpr int kGmBM = 128, kGmBN = 256, kGmBK = 64;
constexpr int kGmStages = 4;
constexpr int kGmThreads = 6 * 32;
constexpr uint32_t kGmABytes = kGmBM * kGmBK * 2;   // 16 KB
constexpr uint32_t kGmBBytes = kGmBN * kGmBK * 2;   // 32 KB
constexpr size_t kGmSmem = 1024 + kGmStages * (kGmABytes + kGmBBytes) + 128;

// Test hook: the next launch's producer in CTA 0 skips the stage fill of this
// k-chunk (no copy, no arrival), so every wait on it runs out (-1 = off).
inline std::atomic<int>& gemm_withhold_next() {
  static std::atomic<int> v{-1};
  return v;
}

struct GmGeom {
  int M, N, K;          // per group
  int groups;
  int m_tiles, n_tiles;
  long long ldc;        // C row stride (elements)
  int withhold;         // test hook: k-chunk whose stage CTA 0 never fills (-1 = none)
};

__global__ void __launch_bounds__(kGmThreads, 1)
gemm_bf16_kernel(const __grid_constant__ CUtensorMap a_map, const __grid_constant__ CUtensorMap b_map,
                 __nv_bfloat16* __restrict__ C, GmGeom g) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* s_a = smem;
  uint8_t* s_b = s_a + kGmStages * kGmABytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(s_b + kGmStages * kGmBBytes);
  uint64_t* full = bars;
  uint64_t* empty = full + kGmStages;
  uint64_t* acc_full = empty + kGmStages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drained = acc_empty + 2;            // MMA issuer: its MMAs have completed (abort path)
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long n_tiles_all = (long long)g.groups * g.m_tiles * g.n_tiles;
  const int k_chunks = g.K / kGmBK;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kGmStages; ++s) { tc::mbar_init(full + s, 1); tc::mbar_init(empty + s, 1); }
    for (int a = 0; a < 2; ++a) { tc::mbar_init(acc_full + a, 1); tc::mbar_init(acc_empty + a, 4); }
    tc::mbar_init(drained, 1);
    tc::fence_barrier_init();
    s_abort = 0;
  }
  if (warp == 1) { tc::tmem_alloc(&s_tmem, 512); tc::tmem_relinquish(); }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = s_tmem;
  volatile int* abort_flag = &s_abort;

  // tile t -> (group, m tile, n tile), n fastest
  auto tile_coords = [&](long long t, int* grp, int* mt, int* nt) {
    *nt = (int)(t % g.n_tiles);
    const long long r = t / g.n_tiles;
    *mt = (int)(r % g.m_tiles);
    *grp = (int)(r / g.m_tiles);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (tc::elect_one()) {
      tc::prefetch_tmap(&a_map);
      tc::prefetch_tmap(&b_map);
      long long it = 0;             // global k-chunk counter (ring position)
      bool ok = true;
      for (long long t = blockIdx.x; ok && t < n_tiles_all; t += gridDim.x) {
        int grp, mt, nt;
        tile_coords(t, &grp, &mt, &nt);
        for (int kc = 0; kc < k_chunks; ++kc, ++it) {
          const int s = (int)(it % kGmStages);
          const long long r = it / kGmStages;
          if (r > 0 && !tc::mbar_wait(empty + s, (uint32_t)((r - 1) & 1))) { ok = false; break; }
          if (*abort_flag) { ok = false; break; }
          if (it == g.withhold && blockIdx.x == 0) continue;     // test hook: this stage never fills
          tc::mbar_arrive_expect_tx(full + s, kGmABytes + kGmBBytes);
          tc::tma_load_2d(s_a + s * kGmABytes, &a_map, full + s, grp * g.K + kc * kGmBK, mt * kGmBM);
          tc::tma_load_2d(s_b + s * kGmBBytes, &b_map, full + s, kc * kGmBK, grp * g.N + nt * kGmBN);
        }
      }
      if (!ok) *abort_flag = 1;
      // drain: every issued copy lands before the CTA may exit
      for (long long j = it - kGmStages > 0 ? it - kGmStages : 0; j < it; ++j)
        tc::mbar_wait(full + (int)(j % kGmStages), (uint32_t)((j / kGmStages) & 1));
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (tc::elect_one()) {
      const uint32_t idesc = tc::idesc_bf16(kGmBM, kGmBN, 0, 0);
      long long it = 0;
      int ti = 0;                   // tiles of this CTA so far (accumulator ring)
      bool ok = true;
      for (long long t = blockIdx.x; ok && t < n_tiles_all; t += gridDim.x, ++ti) {
        const int a = ti & 1;
        if (ti >= 2 && !tc::mbar_wait(acc_empty + a, (uint32_t)(((ti >> 1) - 1) & 1))) { ok = false; break; }
        tc::tc_fence_after();
        for (int kc = 0; kc < k_chunks; ++kc, ++it) {
          const int s = (int)(it % kGmStages);
          if (*abort_flag || !tc::mbar_wait(full + s, (uint32_t)((it / kGmStages) & 1))) { ok = false; break; }
          tc::tc_fence_after();
          const uint32_t a_base = tc::smem_u32(s_a + s * kGmABytes);
          const uint32_t b_base = tc::smem_u32(s_b + s * kGmBBytes);
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            const uint64_t ad = tc::sdesc_sw128(a_base + ks * 32, 16, 1024);
            const uint64_t bd = tc::sdesc_sw128(b_base + ks * 32, 16, 1024);
            tc::mma_bf16_ss(tmem + (uint32_t)a * kGmBN, ad, bd, idesc, (kc | ks) ? 1u : 0u);
          }
          tc::mma_commit(empty + s);
        }
        if (!ok) break;
        tc::mma_commit(acc_full + a);
      }
      if (!ok) {
        *abort_flag = 1;
        // the MMAs already issued finish before TMEM is freed
        tc::mma_commit(drained);
        tc::mbar_wait(drained, 0);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2-5)
    const int quarter = warp & 3;                       // TMEM lanes [32 quarter, 32 quarter + 32)
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
    int ti = 0;
    for (long long t = blockIdx.x; t < n_tiles_all; t += gridDim.x, ++ti) {
      int grp, mt, nt;
      tile_coords(t, &grp, &mt, &nt);
      const int a = ti & 1;
      bool ok = !*abort_flag && tc::mbar_wait(acc_full + a, (uint32_t)((ti >> 1) & 1));
      if (!__all_sync(0xffffffffu, ok)) { *abort_flag = 1; break; }
      tc::tc_fence_after();
      const int row = mt * kGmBM + quarter * 32 + lane;
      __nv_bfloat16* crow = C + (long long)row * g.ldc + (long long)grp * g.N + (long long)nt * kGmBN;
      const int n_left = g.N - nt * kGmBN;               // valid columns of this tile (multiple of 8)
#pragma unroll 1
      for (int cb = 0; cb < kGmBN; cb += 32) {
        uint32_t v[32];
        tc::tmem_ld32(tmem + lane_addr + (uint32_t)(a * kGmBN + cb), v);
        tc::tmem_wait_ld();
        if (cb == kGmBN - 32) {                          // accumulator read out: hand it back
          tc::tc_fence_before();
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(acc_empty + a);
        }
        if (row < g.M) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            if (cb + 8 * q < n_left) {
              uint4 o;
              __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
              for (int e = 0; e < 4; ++e)
                h[e] = __floats2bfloat162_rn(__uint_as_float(v[8 * q + 2 * e]), __uint_as_float(v[8 * q + 2 * e + 1]));
              *reinterpret_cast<uint4*>(crow + cb + 8 * q) = o;
            }
          }
        }
      }
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 512);
  }
}

// C[M, groups*N] (row stride ldc) = per group j: A[:, jK:(j+1)K] . B[jN:(j+1)N, :]^T.
// A: [M, lda] BF16 (lda >= groups*K), B: [groups*N, K] BF16.
static cudaError_t launch_gemm_bf16(const void* A, long long lda, const void* B, __nv_bfloat16* C, long long ldc,
                                    int M, int N, int K, int groups, int sms, cudaStream_t st) {
  CUtensorMap am, bm;
  if (!make_tmap_2d(&am, A, 2, (uint64_t)M, (uint64_t)lda, (uint64_t)lda, kGmBK, kGmBM)) return cudaErrorInvalidValue;
  if (!make_tmap_2d(&bm, B, 2, (uint64_t)groups * N, (uint64_t)K, (uint64_t)K, kGmBK, kGmBN))
    return cudaErrorInvalidValue;
  GmGeom g;
  g.M = M; g.N = N; g.K = K; g.groups = groups;
  g.m_tiles = (M + kGmBM - 1) / kGmBM;
  g.n_tiles = (N + kGmBN - 1) / kGmBN;
  g.ldc = ldc;
  g.withhold = gemm_withhold_next().exchange(-1);
  const long long tiles = (long long)groups * g.m_tiles * g.n_tiles;
  const int grid = (int)(tiles < sms ? tiles : sms);
  cudaError_t e = cudaFuncSetAttribute(gemm_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGmSmem);
  if (e != cudaSuccess) return e;
  gemm_bf16_kernel<<<grid, kGmThreads, kGmSmem, st>>>(am, bm, C, g);
  count_launch();
  return cudaGetLastError();
}

}  // namespace lcsa
