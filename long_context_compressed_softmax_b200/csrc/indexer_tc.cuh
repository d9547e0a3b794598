// Lightning-Indexer scores on tcgen05 tensor cores (BF16, H_I = 64, D_I = 128).
// (DeepSeek-V4 CSA Step 2: a light indexer scores every compressed entry
// against the current query; s = sum_h w_h * relu(q_h . k_j).)
//
// GEMM view: M = 128 entries (A = k_I tile, K-major), N = 64 heads x up to 4
// query rows of one sequence (B = q_I, K-major), K = 128.  The accumulator
// sits in TMEM with one entry per lane, so the ReLU and the weighted head sum
// of the epilogue are per-thread register work: thread (lane j) reads the 64
// head columns of query q and emits s[q, j] with one coalesced store per warp.
//
// Warp roles (320 threads): warp 0 issues TMA loads (q once, then a 4-stage
// ring of k tiles), warp 1 allocates TMEM and issues the MMAs (double-buffered
// 256-column accumulators = all 512 columns), warps 2-9 drain accumulators.
// Every wait is bounded (tc::mbar_wait); on expiry the CTA stops, records
// LCSA_DEV_TIMEOUT, drains its in-flight copies and frees TMEM.
#pragma once
#include "tc_ptx.cuh"

namespace lcsa {

constexpr long long kIndexerChunkRows = 8192;
constexpr int kIxStages = 4;
constexpr int kIxTileE = 128;          // entries per tile (MMA M)
constexpr int kIxRows = 4;             // query rows per CTA (MMA N = 64 * rows)
constexpr int kIxThreads = 320;
constexpr uint32_t kIxQBytes = 2 * 256 * 128;          // 2 K-chunks x 256 rows x 128 B
constexpr uint32_t kIxKBytes = 2 * kIxTileE * 128;     // 2 K-chunks x 128 rows x 128 B
constexpr size_t kIxSmem = 1024 /*align slack*/ + kIxQBytes + kIxStages * kIxKBytes + kIxRows * 64 * 4 + 256;

struct IxGeom {
  int Tq, Nc, H;            // H = 64 heads
  int b0, nb, i0, ni;       // chunk rectangle: sequences [b0,b0+nb), rows [i0,i0+ni)
  int gps;                  // query groups per sequence = ceil(ni / 4)
  int splits;               // entry-range splits per group
  long long q_pos0;
  int m;
};

static bool indexer_tc_supported(const lcsa_indexer_args* a) {
  return a->dtype == LCSA_BF16 && a->H_I == 64 && a->D_I == 128;
}

__global__ void __launch_bounds__(kIxThreads, 1)
indexer_tc_kernel(const __grid_constant__ CUtensorMap q_map, const __grid_constant__ CUtensorMap k_map,
                  const float* __restrict__ w, float* __restrict__ scores, IxGeom g) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* s_q = smem;
  uint8_t* s_k = s_q + kIxQBytes;
  float* s_w = reinterpret_cast<float*>(s_k + kIxStages * kIxKBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(s_w + kIxRows * 64);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = k_full + kIxStages;
  uint64_t* acc_full = k_empty + kIxStages;
  uint64_t* acc_empty = acc_full + 2;
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- work unit
  const int n_groups = g.nb * g.gps;
  const int grp = n_groups - 1 - (int)blockIdx.x;          // heaviest groups first
  const int split = blockIdx.y;
  const int bl = grp / g.gps;
  const int b = g.b0 + bl;
  const int gi = grp - bl * g.gps;
  const int i_first = g.i0 + gi * kIxRows;
  int rows = g.i0 + g.ni - i_first;
  rows = rows < kIxRows ? rows : kIxRows;
  long long nv = (g.q_pos0 + i_first + rows - 1) / g.m;    // most entries any row of the group sees
  if (nv > g.Nc) nv = g.Nc;
  const int tiles_all = (int)((nv + kIxTileE - 1) / kIxTileE);
  const int per_split = (tiles_all + g.splits - 1) / g.splits;
  const int t_begin = split * per_split;
  int t_end = t_begin + per_split;
  t_end = t_end < tiles_all ? t_end : tiles_all;
  const int n_tiles = t_end > t_begin ? t_end - t_begin : 0;
  if (n_tiles == 0) return;                                // uniform across the CTA

  if (threadIdx.x == 0) {
    tc::mbar_init(q_full, 1);
    for (int s = 0; s < kIxStages; ++s) { tc::mbar_init(k_full + s, 1); tc::mbar_init(k_empty + s, 1); }
    for (int a = 0; a < 2; ++a) { tc::mbar_init(acc_full + a, 1); tc::mbar_init(acc_empty + a, 8); }
    tc::fence_barrier_init();
    s_abort = 0;
  }
  if (warp == 1) { tc::tmem_alloc(&s_tmem, 512); tc::tmem_relinquish(); }
  for (int e = threadIdx.x; e < kIxRows * 64; e += kIxThreads) {
    const int q = e >> 6, h = e & 63;
    s_w[e] = q < rows ? w[((long long)b * g.Tq + i_first + q) * 64 + h] : 0.f;
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = s_tmem;
  volatile int* abort_flag = &s_abort;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (tc::elect_one()) {
      tc::prefetch_tmap(&q_map);
      tc::prefetch_tmap(&k_map);
      const int qrow = (int)(((long long)b * g.Tq + i_first) * 64);
      tc::mbar_arrive_expect_tx(q_full, kIxQBytes);
      tc::tma_load_2d(s_q, &q_map, q_full, 0, qrow);
      tc::tma_load_2d(s_q + kIxQBytes / 2, &q_map, q_full, 64, qrow);
      int issued = 0;
      for (int n = 0; n < n_tiles; ++n) {
        const int s = n % kIxStages, r = n / kIxStages;
        if (r > 0 && !tc::mbar_wait(k_empty + s, (r - 1) & 1)) { *abort_flag = 1; break; }
        if (*abort_flag) break;
        const int krow = (int)((long long)b * g.Nc + (long long)(t_begin + n) * kIxTileE);
        uint8_t* dst = s_k + s * kIxKBytes;
        tc::mbar_arrive_expect_tx(k_full + s, kIxKBytes);
        tc::tma_load_2d(dst, &k_map, k_full + s, 0, krow);
        tc::tma_load_2d(dst + kIxKBytes / 2, &k_map, k_full + s, 64, krow);
        ++issued;
      }
      // drain: every issued copy must land before the CTA may exit
      for (int n = issued - kIxStages > 0 ? issued - kIxStages : 0; n < issued; ++n)
        tc::mbar_wait(k_full + n % kIxStages, (n / kIxStages) & 1);
      tc::mbar_wait(q_full, 0);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (tc::elect_one()) {
      const uint32_t idesc = tc::idesc_bf16(128, 64 * rows, 0, 0);
      bool ok = tc::mbar_wait(q_full, 0);
      for (int n = 0; ok && n < n_tiles; ++n) {
        const int s = n % kIxStages, r = n / kIxStages;
        const int a = n & 1, ra = n >> 1;
        if (*abort_flag) break;
        if (!tc::mbar_wait(k_full + s, r & 1)) { ok = false; break; }
        if (ra > 0 && !tc::mbar_wait(acc_empty + a, (ra - 1) & 1)) { ok = false; break; }
        tc::tc_fence_after();
        const uint32_t a_base = tc::smem_u32(s_k + s * kIxKBytes);
        const uint32_t b_base = tc::smem_u32(s_q);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t koff = (uint32_t)((ks & 3) * 32);
          const uint64_t ad = tc::sdesc_sw128(a_base + (ks >> 2) * (kIxKBytes / 2) + koff, 16, 1024);
          const uint64_t bd = tc::sdesc_sw128(b_base + (ks >> 2) * (kIxQBytes / 2) + koff, 16, 1024);
          tc::mma_bf16_ss(tmem + a * 256, ad, bd, idesc, ks > 0 ? 1u : 0u);
        }
        tc::mma_commit(k_empty + s);
        tc::mma_commit(acc_full + a);
      }
      if (!ok) *abort_flag = 1;
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int e = warp - 2;                 // 0..7
    const int quarter = warp & 3;           // TMEM lanes [32*quarter, 32*quarter+32)
    const int half = e >> 2;                // query rows {2*half, 2*half+1}
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
    for (int n = 0; n < n_tiles; ++n) {
      const int a = n & 1, ra = n >> 1;
      if (*abort_flag) break;
      if (!tc::mbar_wait(acc_full + a, ra & 1)) { *abort_flag = 1; break; }
      tc::tc_fence_after();
      uint32_t v[2][64];
#pragma unroll
      for (int qq = 0; qq < 2; ++qq) {
        const uint32_t col = tmem + lane_addr + (uint32_t)(a * 256 + (2 * half + qq) * 64);
        tc::tmem_ld32(col, v[qq]);
        tc::tmem_ld32(col + 32, v[qq] + 32);
      }
      tc::tmem_wait_ld();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(acc_empty + a);
      const long long j = (long long)(t_begin + n) * kIxTileE + quarter * 32 + lane;
#pragma unroll
      for (int qq = 0; qq < 2; ++qq) {
        const int q = 2 * half + qq;
        if (q < rows && j < g.Nc) {
          const float* wq = s_w + q * 64;
          float s = 0.f;
#pragma unroll
          for (int h = 0; h < 64; ++h) s = fmaf(wq[h], fmaxf(__uint_as_float(v[qq][h]), 0.f), s);
          const long long srow = (long long)bl * g.ni + (i_first - g.i0) + q;
          scores[srow * g.Nc + j] = s;
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

// Entry-range splits per query group when there are few groups (decode): the
// split count s (at most tiles / 8, so a CTA keeps >= 8 tiles) that minimises
// the waves of one-CTA-per-SM launches times the tiles per CTA, with a
// per-CTA start-up cost of about 6 tiles.  Many groups: no split.
static int indexer_splits(int n_groups, int tiles) {
  const int sms = sm_count();
  if (n_groups >= 4 * sms) return 1;
  const int max_splits = tiles / 8 > 1 ? tiles / 8 : 1;
  int best = 1;
  long long best_cost = -1;
  for (int s = 1; s <= max_splits; ++s) {
    const long long waves = ((long long)n_groups * s + sms - 1) / sms;
    const long long cost = waves * ((tiles + s - 1) / s + 6);
    if (best_cost < 0 || cost < best_cost) { best_cost = cost; best = s; }
  }
  return best;
}

// Scores for the chunk rectangle: sequences [b0, b0+nb), query rows [i0, i0+ni)
// of each; scores rows laid out [nb][ni][Nc].
static cudaError_t launch_indexer_tc_rect(const lcsa_indexer_args* a, float* scores, int b0, int nb, int i0, int ni,
                                         cudaStream_t st) {
  CUtensorMap qm, km;
  const uint64_t q_rows = (uint64_t)a->B * a->Tq * 64;
  const uint64_t k_rows = (uint64_t)a->B * a->Nc;
  if (!make_tmap_bf16_2d(&qm, a->q_idx, q_rows, 128, 128, 64, 256)) return cudaErrorInvalidValue;
  if (!make_tmap_bf16_2d(&km, a->k_idx, k_rows, 128, 128, 64, kIxTileE)) return cudaErrorInvalidValue;
  IxGeom g;
  g.Tq = a->Tq; g.Nc = a->Nc; g.H = 64;
  g.b0 = b0; g.nb = nb; g.i0 = i0; g.ni = ni;
  g.gps = (ni + kIxRows - 1) / kIxRows;
  g.q_pos0 = a->q_pos0; g.m = a->m;
  const int n_groups = nb * g.gps;
  long long nv = (a->q_pos0 + i0 + ni - 1) / a->m;
  if (nv > a->Nc) nv = a->Nc;
  const int tiles = (int)((nv + kIxTileE - 1) / kIxTileE);
  const int splits = indexer_splits(n_groups, tiles);
  g.splits = splits;
  cudaError_t e = cudaFuncSetAttribute(indexer_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kIxSmem);
  if (e != cudaSuccess) return e;
  dim3 grid(n_groups, splits);
  indexer_tc_kernel<<<grid, kIxThreads, kIxSmem, st>>>(qm, km, a->w, scores, g);
  count_launch();
  return cudaGetLastError();
}

}  // namespace lcsa
