// Core attention of CSA / HCA on tcgen05 tensor cores (BF16, H = 64 heads,
// D = 512, rotary R = 64).  DeepSeek-V4 hybrid attention, "第三步，core
// attention": multi-query attention of 64 heads over one shared K=V head; the
// key set is the selected compressed entries (CSA) or every visible entry
// (HCA), followed by the sliding window of raw tokens; a per-head sink logit
// joins the softmax denominator; the last 64 dims carry RoPE and the output
// is rotated back by -t.
//
// One CTA per (query, key-range split).  Per 64-key tile:
//   S = Q K^T   tcgen05 M=64 (heads), N=64 (keys), K=512; S lives in TMEM
//               lanes 16-31 of each sub-partition (double buffered)
//   softmax     one thread per head row, exp2 with a lazily updated running
//               max (O is rescaled only when the max grows by more than 2^8)
//   O += P V    tcgen05 M=64, N=2x256 (dims), K=64 keys; O lives in TMEM
//               lanes 0-15 of each sub-partition, all 512 columns
// The K tile doubles as V: the K-major view feeds S, the MN-major view of the
// same 128B-swizzled bytes feeds PV.
//
// Warps: 0-3 gather key rows with cp.async (16-byte pieces placed at their
// swizzled addresses; invalid rows zero-filled), 4 allocates TMEM and issues
// MMAs, 5-8 rotate Q, run the softmax and the epilogue.  Rotary slices of the
// keys come pre-rotated (rope.cuh).  All waits are bounded.
#pragma once
#include "tc_ptx.cuh"
#include "rope.cuh"

namespace lcsa {

constexpr int kAtKT = 64;                      // keys per tile
constexpr int kAtProdWarps = 8;                 // gather / TMA producers
constexpr int kAtProdThreads = kAtProdWarps * 32;
constexpr int kAtMmaWarp = kAtProdWarps;        // TMEM allocator and MMA issuer
constexpr int kAtSmWarp0 = kAtProdWarps + 1;    // first of the 4 softmax / epilogue warps
constexpr int kAtThreads = (kAtProdWarps + 5) * 32;
constexpr uint32_t kAtQBytes = 64 * 512 * 2;   // 64 KB
constexpr uint32_t kAtKBytes = kAtKT * 512 * 2;  // 64 KB
constexpr uint32_t kAtPBytes = 64 * kAtKT * 2;   // 8 KB
constexpr uint32_t kAtRegion = 64 * 128;       // one 64-dim column block of a 64-row tile
constexpr int kAtMaxIdx = 2048;                 // selected entries staged in shared memory per CTA
constexpr int kAtStages = 3;                    // K=V tile stages
constexpr size_t kAtSmem = 1024 + kAtStages * kAtKBytes + 2 * kAtPBytes + kAtStages * kAtKT * 2 * 8 +
                           kAtMaxIdx * 4 + 32 * 8 + 17 * 8;
constexpr float kLog2e = 1.4426950408889634f;

struct AtGeom {
  int Tq, Nc, k, Tkv;
  long long q_pos0, kv_pos0;
  int m, W;
  float scale_log2;
  double log_base;
  int sparse;
  int rot_slot;        // CSA rotary slices indexed by (query, slot) instead of by entry
  int splits;
  int out_bf16;
};

struct AtPtrs {
  const __nv_bfloat16* q;
  const __nv_bfloat16* ckv;
  const int32_t* idx;
  const __nv_bfloat16* kv;
  const __nv_bfloat16* rot_c;   // rotated slices of the entries
  const __nv_bfloat16* rot_w;   // rotated slices of the raw rows
  const float* sink;
  void* out;
  float* lse;
  float* o_part;                // splits > 1: [splits][rows][64][512]
  float* ml_part;               // splits > 1: [splits][rows][64][2]  (m in log2 units, l)
};

static bool attn_tc_supported(const lcsa_attn_args* a) {
  return a->dtype == LCSA_BF16 && a->H == 64 && a->D == 512 && a->R == 64;
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
__device__ __forceinline__ void named_bar(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }
// Arrive on `bar` (counted as one of its expected arrivals) once every
// cp.async this thread issued so far has landed.
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(tc::smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Key-set geometry of one query.
struct KeySet {
  int n_c, n_w, tiles_c, tiles;
  long long wlo;
};
__device__ __forceinline__ KeySet key_set(const AtGeom& g, const int32_t* idx_row, long long t) {
  KeySet s;
  if (g.sparse) {
    // idx rows are ascending with -1 padding at the end: count the valid prefix
    int lo = 0, hi = g.k;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (idx_row[mid] >= 0) lo = mid + 1; else hi = mid;
    }
    s.n_c = lo;
  } else {
    long long nv = t / g.m;
    s.n_c = (int)(nv < g.Nc ? nv : g.Nc);
  }
  long long wlo = t - g.W + 1;
  if (wlo < g.kv_pos0) wlo = g.kv_pos0;
  if (wlo < 0) wlo = 0;
  long long whi = t;
  if (whi > g.kv_pos0 + g.Tkv - 1) whi = g.kv_pos0 + g.Tkv - 1;
  s.n_w = whi >= wlo ? (int)(whi - wlo + 1) : 0;
  if (g.W == 0) s.n_w = 0;
  s.wlo = wlo;
  s.tiles_c = (s.n_c + kAtKT - 1) / kAtKT;
  s.tiles = s.tiles_c + (s.n_w + kAtKT - 1) / kAtKT;
  return s;
}

__global__ void __launch_bounds__(kAtThreads, 1)
attn_tc_kernel(AtPtrs P, AtGeom g, const __grid_constant__ CUtensorMap tm_ckv, const __grid_constant__ CUtensorMap tm_kv,
               const __grid_constant__ CUtensorMap tm_rotc, const __grid_constant__ CUtensorMap tm_rotw) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* s_k = smem;                                                  // kAtStages K=V tiles
  uint8_t* s_p = s_k + kAtStages * kAtKBytes;                           // 2 P buffers
  const uint8_t** s_tab = reinterpret_cast<const uint8_t**>(s_p + 2 * kAtPBytes);   // [stage][64][2] row pointers
  int32_t* s_idx = reinterpret_cast<int32_t*>(s_tab + kAtStages * kAtKT * 2);       // selected entries of this range
  float2* s_cs = reinterpret_cast<float2*>(s_idx + kAtMaxIdx);                      // [32] (cos, sin) at t
  uint64_t* bars = reinterpret_cast<uint64_t*>(s_cs + 32);
  uint64_t* q_ready = bars + 0;                 // softmax warps (4): Q is in TMEM
  uint64_t* q_full = bars + 15;                 // producers (async arrivals): Q staged in the last stage
  uint64_t* kv_full = bars + 1;                 // [kAtStages] producers (one arrival each; TMA bytes)
  uint64_t* kv_empty = kv_full + kAtStages;     // [kAtStages] MMA commit
  uint64_t* s_full = kv_empty + kAtStages;      // [2] MMA commit
  uint64_t* s_free = s_full + 2;                // [2] softmax warps (4)
  uint64_t* p_full = s_free + 2;                // [2] softmax warps (4)
  uint64_t* pv_done = p_full + 2;               // [2] MMA commit
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row = blockIdx.x;                 // b * Tq + i
  const int split = blockIdx.y;
  const int b = (int)(row / g.Tq), i = (int)(row - (long long)b * g.Tq);
  const long long t = g.q_pos0 + i;
  const int32_t* idx_row = g.sparse ? P.idx + row * g.k : nullptr;
  const KeySet ks = key_set(g, idx_row, t);
  const int per_split = (ks.tiles + g.splits - 1) / g.splits;
  const int t0 = split * per_split;
  const int t1 = t0 + per_split < ks.tiles ? t0 + per_split : ks.tiles;
  const int n_tiles = t1 > t0 ? t1 - t0 : 0;

  // ---------------------------------------------------------------- no keys
  if (n_tiles == 0) {
    for (int e = threadIdx.x; e < 64 * 512; e += kAtThreads) {
      const long long o = row * 64 * 512 + e;
      if (g.splits > 1) P.o_part[(long long)split * gridDim.x * 64 * 512 + o] = 0.f;
      else if (g.out_bf16) reinterpret_cast<__nv_bfloat16*>(P.out)[o] = __float2bfloat16_rn(0.f);
      else reinterpret_cast<float*>(P.out)[o] = 0.f;
    }
    if (threadIdx.x < 64) {
      const int h = threadIdx.x;
      if (g.splits > 1) {
        float* ml = P.ml_part + ((long long)split * gridDim.x + row) * 128 + 2 * h;
        ml[0] = -INFINITY; ml[1] = 0.f;
      } else if (P.lse) {
        P.lse[row * 64 + h] = P.sink ? P.sink[h] : -INFINITY;
      }
    }
    return;
  }

  if (threadIdx.x == 0) {
    tc::mbar_init(q_ready, 4);
    tc::mbar_init(q_full, kAtProdThreads);
    for (int s = 0; s < kAtStages; ++s) {
      tc::mbar_init(kv_full + s, kAtProdThreads);
      tc::mbar_init(kv_empty + s, 1);
    }
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(s_full + s, 1);
      tc::mbar_init(s_free + s, 4);
      tc::mbar_init(p_full + s, 4);
      tc::mbar_init(pv_done + s, 1);
    }
    tc::fence_barrier_init();
    s_abort = 0;
  }
  if (warp == kAtMmaWarp) { tc::tmem_alloc(&s_tmem, 512); tc::tmem_relinquish(); }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = s_tmem;
  volatile int* abort_flag = &s_abort;
  // TMEM map: lanes 0-15 of each sub-partition hold S[0] (cols 0-63), S[1]
  // (64-127) and Q (128-383, the A operand of S = Q K^T); lanes 16-31 hold O
  // (cols 0-511).
  constexpr uint32_t kTmQ = 128;
  constexpr uint32_t kTmO = 16u << 16;

  if (warp < kAtProdWarps) {
    // ============================================================ producers
    // Contiguous tiles (every HCA entry tile and every window tile) arrive as
    // eight 2D TMA boxes of 64 rows x 64 dims; CSA's selected rows are
    // gathered 16 bytes at a time with cp.async by all eight producer warps.
    const int tid = threadIdx.x;                    // 0..255
    const int piece = tid & 63;                     // 16-byte piece of a 1 KB row
    const int region = piece >> 3, c16 = piece & 7;
    const int kk0 = tid >> 6;                       // keys kk0, kk0+4, ..., kk0+60
    constexpr int kStep = kAtProdThreads / 64;
    // Q (64 heads x 1 KB) is staged in the last K stage, which tile 2 only
    // reuses once the softmax warps have moved Q into tensor memory.
    {
      const uint8_t* qrow0 = reinterpret_cast<const uint8_t*>(P.q + row * 64 * 512);
      const uint32_t qb = tc::smem_u32(s_k + (kAtStages - 1) * kAtKBytes) + region * kAtRegion + (c16 << 4);
#pragma unroll 8
      for (int u = 0; u < 64 / kStep; ++u) {
        const int h = kk0 + kStep * u;
        cp_async16((qb + h * 128) ^ ((uint32_t)(h & 7) << 4), qrow0 + (long long)h * 1024 + piece * 16, 16);
      }
      cp_async_arrive_noinc(q_full);
    }
    const int slot0 = t0 * kAtKT;
    if (g.sparse) {
      const int n_sel = (ks.n_c < t1 * kAtKT ? ks.n_c : t1 * kAtKT) - slot0;
      for (int e = tid; e < n_sel; e += kAtProdThreads) s_idx[e] = idx_row[slot0 + e];
      named_bar(1, kAtProdThreads);
    }
    if (tid == 0) {
      tc::prefetch_tmap(&tm_ckv);
      tc::prefetch_tmap(&tm_kv);
      tc::prefetch_tmap(&tm_rotc);
      tc::prefetch_tmap(&tm_rotw);
    }
    const uint8_t* dummy = reinterpret_cast<const uint8_t*>(P.q);
    for (int n = 0; n < n_tiles; ++n) {
      const int s = n % kAtStages;
      if (n >= kAtStages && !tc::mbar_wait_backoff(kv_empty + s, ((n - kAtStages) / kAtStages) & 1)) *abort_flag = 1;
      if (n == kAtStages - 1 && !tc::mbar_wait_backoff(q_ready, 0)) *abort_flag = 1;
      if (*abort_flag) break;
      const int gt = t0 + n;                        // tile index in the query's key list
      uint8_t* stage = s_k + s * kAtKBytes;
      if (gt >= ks.tiles_c || !g.sparse) {
        // ---- contiguous rows: TMA boxes
        if (tid == 0) {
          const CUtensorMap* mm;
          const CUtensorMap* mr;
          int y;
          if (gt < ks.tiles_c) {
            mm = &tm_ckv; mr = &tm_rotc;
            y = (int)((long long)b * g.Nc + (long long)gt * kAtKT);
          } else {
            mm = &tm_kv; mr = &tm_rotw;
            y = (int)((long long)b * g.Tkv + (ks.wlo - g.kv_pos0) + (long long)(gt - ks.tiles_c) * kAtKT);
          }
          tc::mbar_arrive_expect_tx(kv_full + s, kAtKBytes);
#pragma unroll
          for (int reg = 0; reg < 7; ++reg) tc::tma_load_2d(stage + reg * kAtRegion, mm, kv_full + s, reg * 64, y);
          tc::tma_load_2d(stage + 7 * kAtRegion, mr, kv_full + s, 0, y);
        } else {
          tc::mbar_arrive(kv_full + s);
        }
        continue;
      }
      // ---- gathered rows (CSA): per-tile row table, then 16-byte cp.async pieces
      const uint8_t** tab = s_tab + s * kAtKT * 2;
      if (tid < kAtKT) {
        const int kk = tid;
        const uint8_t* rm = nullptr;
        const uint8_t* rr = nullptr;
        const int slot = gt * kAtKT + kk;
        if (slot < ks.n_c) {
          const int j = s_idx[slot - slot0];
          if (j >= 0 && j < g.Nc) {
            rm = reinterpret_cast<const uint8_t*>(P.ckv + ((long long)b * g.Nc + j) * 512);
            rr = reinterpret_cast<const uint8_t*>(
                P.rot_c + (g.rot_slot ? (row * g.k + slot) : ((long long)b * g.Nc + j)) * 64);
          } else {
            report(LCSA_DEV_BAD_INDEX);
          }
        }
        tab[2 * kk] = rm;
        tab[2 * kk + 1] = rr;
      }
      named_bar(1, kAtProdThreads);
      const uint32_t kb = tc::smem_u32(stage) + region * kAtRegion + (c16 << 4);
      const int off = region == 7 ? c16 * 16 : piece * 16;
#pragma unroll 8
      for (int u = 0; u < 64 / kStep; ++u) {
        const int kk = kk0 + kStep * u;
        const uint8_t* base = tab[2 * kk + (region == 7 ? 1 : 0)];
        const uint32_t dst = (kb + kk * 128) ^ ((uint32_t)(kk & 7) << 4);
        cp_async16(dst, base ? base + off : dummy, base ? 16u : 0u);
      }
      cp_async_arrive_noinc(kv_full + s);
    }
    cp_async_wait_all();                            // nothing may land after the CTA exits
  } else if (warp == kAtMmaWarp) {
    // ============================================================ MMA issuer
    // S(n+1) and PV(n) are independent: whichever is ready is issued first.
    if (tc::elect_one()) {
      const uint32_t idesc_s = tc::idesc_bf16(64, kAtKT, 0, 0);    // A (TMEM) K-major, B K-major
      const uint32_t idesc_o = tc::idesc_bf16(64, 256, 0, 1);      // A K-major, B MN-major
      bool ok = tc::mbar_wait(q_ready, 0);
      int next_s = 0, next_pv = 0;
      uint64_t t_idle = 0;
      while (ok && next_pv < n_tiles) {
        bool did = false;
        if (next_s < n_tiles && next_s <= next_pv + 1) {
          const int st = next_s % kAtStages, sb = next_s & 1;
          if (tc::mbar_try_wait(kv_full + st, (next_s / kAtStages) & 1) &&
              (next_s < 2 || tc::mbar_try_wait(s_free + sb, ((next_s >> 1) - 1) & 1))) {
            tc::tc_fence_after();
            const uint32_t kb = tc::smem_u32(s_k + st * kAtKBytes);
#pragma unroll
            for (int kstep = 0; kstep < 32; ++kstep) {
              const uint32_t off = (uint32_t)((kstep >> 2) * kAtRegion + (kstep & 3) * 32);
              tc::mma_bf16_ts(tmem + sb * kAtKT, tmem + kTmQ + kstep * 8, tc::sdesc_sw128(kb + off, 16, 1024),
                              idesc_s, kstep > 0 ? 1u : 0u);
            }
            tc::mma_commit(s_full + sb);
            ++next_s;
            did = true;
          }
        }
        if (next_pv < next_s) {
          const int st = next_pv % kAtStages, sb = next_pv & 1;
          if (tc::mbar_try_wait(p_full + sb, (next_pv >> 1) & 1)) {
            tc::tc_fence_after();
            const uint32_t pb = tc::smem_u32(s_p + sb * kAtPBytes);
            const uint32_t kb = tc::smem_u32(s_k + st * kAtKBytes);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
#pragma unroll
              for (int kstep = 0; kstep < kAtKT / 16; ++kstep) {
                const uint64_t ad = tc::sdesc_sw128(pb + kstep * 32, 16, 1024);
                const uint64_t bd = tc::sdesc_sw128(kb + half * 4 * kAtRegion + kstep * 2048, kAtRegion, 1024);
                tc::mma_bf16_ss(tmem + kTmO + half * 256, ad, bd, idesc_o, (next_pv > 0 || kstep > 0) ? 1u : 0u);
              }
            }
            tc::mma_commit(kv_empty + st);
            tc::mma_commit(pv_done + sb);
            ++next_pv;
            did = true;
          }
        }
        if (did) {
          t_idle = 0;
        } else if (*abort_flag) {
          ok = false;
        } else {
          const uint64_t now = tc::globaltimer();
          if (t_idle == 0) t_idle = now;
          else if (now - t_idle > tc::kWaitLimitNs) { report(LCSA_DEV_TIMEOUT); ok = false; }
        }
      }
      if (!ok) *abort_flag = 1;
    }
  } else {
    // ============================================================ softmax / epilogue
    // Every head row h of this warp's 16-lane block is split over two threads:
    // thread (h % 16) takes keys 0-31 of each tile and dims 0-255 of O,
    // thread (h % 16) + 16 takes keys 32-63 and dims 256-511 (16x32bx2 TMEM
    // accesses).  Row maxima and sums meet through one shuffle.
    const int quarter = warp & 3;
    const int half = lane >> 4;                       // 0: keys 0-31 / dims 0-255, 1: keys 32-63 / dims 256-511
    const int h = quarter * 16 + (lane & 15);         // head row
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const int stid = threadIdx.x - kAtSmWarp0 * 32;   // 0..127
    // rotary table at position t (shared by the Q rotation and the -t output rotation)
    if (stid < 32) {
      float c, sn;
      rope_cs(t, stid, kRopeR, g.log_base, &c, &sn);
      s_cs[stid] = make_float2(c, sn);
    }
    named_bar(2, 128);
    // Q -> TMEM (A operand, lanes 0-15): head h's dims 256*half .. +255, two per
    // column; the rotary block (dims 448..511) is rotated at t on the way.
    if (!tc::mbar_wait(q_full, 0)) *abort_flag = 1;
    {
      const uint8_t* qs = s_k + (kAtStages - 1) * kAtKBytes + h * 128;
#pragma unroll 2
      for (int c = 0; c < 8; ++c) {                   // 32 dims = 16 columns per step
        const int cc = half * 8 + c;                  // 32-dim chunk of the row
        uint32_t r[16];
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const int chunk = (cc & 1) * 4 + v;         // 16-byte chunk within the 128-byte row of region cc/2
          const uint4 x = *reinterpret_cast<const uint4*>(qs + (cc >> 1) * kAtRegion + ((chunk ^ (h & 7)) << 4));
          r[4 * v] = x.x; r[4 * v + 1] = x.y; r[4 * v + 2] = x.z; r[4 * v + 3] = x.w;
        }
        if (cc >= 14) {
#pragma unroll
          for (int q2 = 0; q2 < 16; ++q2) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&r[q2]));
            const float2 cs = s_cs[(cc - 14) * 16 + q2];
            const __nv_bfloat162 o = __floats2bfloat162_rn(f.x * cs.x - f.y * cs.y, f.x * cs.y + f.y * cs.x);
            r[q2] = *reinterpret_cast<const uint32_t*>(&o);
          }
        }
        tc::tmem_st_16x32bx2_x16<128>(tmem + lane_base + kTmQ + c * 16, r);
      }
      tc::tmem_wait_st();
    }
    tc::tc_fence_before();
    __syncwarp();
    if (lane == 0) tc::mbar_arrive(q_ready);

    bool ok = true;
    float m_run = -INFINITY, l_run = 0.f;             // l_run: this thread's half of the row sum
    for (int n = 0; ok && n < n_tiles; ++n) {
      const int sb = n & 1;
      if (*abort_flag) { ok = false; break; }
      if (!tc::mbar_wait(s_full + sb, (n >> 1) & 1)) { ok = false; break; }
      tc::tc_fence_after();
      uint32_t v[32];
      tc::tmem_ld_16x32bx2_x32<32>(tmem + lane_base + sb * kAtKT, v);
      tc::tmem_wait_ld();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(s_free + sb);
      const int gt = t0 + n;
      int nvalid = gt < ks.tiles_c ? ks.n_c - gt * kAtKT : ks.n_w - (gt - ks.tiles_c) * kAtKT;
      nvalid = (nvalid < kAtKT ? nvalid : kAtKT) - 32 * half;   // valid keys among this thread's 32
      float tmax = -INFINITY;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float s = j < nvalid ? __uint_as_float(v[j]) : -INFINITY;
        v[j] = __float_as_uint(s);
        tmax = fmaxf(tmax, s);
      }
      tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 16)) * g.scale_log2;
      float alpha = 1.f;
      bool rescale = false;
      if (n == 0) {
        m_run = tmax;
      } else if (tmax > m_run + 8.f) {
        alpha = exp2f(m_run - tmax);
        m_run = tmax;
        rescale = true;
      }
      if (__any_sync(0xffffffffu, rescale)) {
        // O (lanes 16-31) is rescaled once PV(n-1) has finished; the 16x32bx2
        // accesses touch O's lanes only.
        if (!tc::mbar_wait(pv_done + ((n - 1) & 1), ((n - 1) >> 1) & 1)) ok = false;
        tc::tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < 256; c += 32) {
          uint32_t r[32];
          tc::tmem_ld_16x32bx2_x32<256>(tmem + lane_base + kTmO + c, r);
          tc::tmem_wait_ld();
#pragma unroll
          for (int q2 = 0; q2 < 32; ++q2) r[q2] = __float_as_uint(__uint_as_float(r[q2]) * alpha);
          tc::tmem_st_16x32bx2_x16<256>(tmem + lane_base + kTmO + c, r);
          tc::tmem_st_16x32bx2_x16<256>(tmem + lane_base + kTmO + c + 16, r + 16);
        }
        tc::tmem_wait_st();
      }
      l_run *= alpha;
      // P buffer sb is free once PV(n-2) is done
      if (n >= 2 && !tc::mbar_wait(pv_done + sb, ((n - 2) >> 1) & 1)) ok = false;
      {
        float psum = 0.f;
        uint8_t* prow = s_p + sb * kAtPBytes + h * 128;
        const float neg_m = -m_run;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t pk[4];
#pragma unroll
          for (int q2 = 0; q2 < 4; ++q2) {
            const float p0 = exp2f(fmaf(__uint_as_float(v[8 * c + 2 * q2]), g.scale_log2, neg_m));
            const float p1 = exp2f(fmaf(__uint_as_float(v[8 * c + 2 * q2 + 1]), g.scale_log2, neg_m));
            psum += p0 + p1;
            __nv_bfloat162 bp = __floats2bfloat162_rn(p0, p1);
            pk[q2] = *reinterpret_cast<uint32_t*>(&bp);
          }
          const int chunk = half * 4 + c;             // keys 8*chunk .. 8*chunk+7
          *reinterpret_cast<uint4*>(prow + ((chunk ^ (h & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
        l_run += psum;
      }
      tc::fence_proxy_async_smem();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(p_full + sb);
    }
    // ---------------------------------------------------------- epilogue
    if (ok && !tc::mbar_wait(pv_done + ((n_tiles - 1) & 1), ((n_tiles - 1) >> 1) & 1)) ok = false;
    tc::tc_fence_after();
    const float l_row = l_run + __shfl_xor_sync(0xffffffffu, l_run, 16);
    if (ok) {
      const long long orow = row * 64 + h;
      float scale_out;
      if (g.splits > 1) {
        scale_out = 1.f;
        if (half == 0) {
          float* ml = P.ml_part + ((long long)split * gridDim.x + row) * 128 + 2 * h;
          ml[0] = m_run;
          ml[1] = l_row;
        }
      } else {
        float M = m_run, l = l_row;
        if (P.sink) {
          const float s2 = P.sink[h] * kLog2e;
          const float Mn = fmaxf(M, s2);
          l = l * exp2f(M - Mn) + exp2f(s2 - Mn);
          scale_out = exp2f(M - Mn);
          M = Mn;
        } else {
          scale_out = 1.f;
        }
        scale_out = l > 0.f ? scale_out / l : 0.f;
        if (half == 0 && P.lse) P.lse[orow] = l > 0.f ? (M + log2f(l)) * 0.6931471805599453f : -INFINITY;
      }
#pragma unroll 1
      for (int c0 = 0; c0 < 256; c0 += 32) {
        uint32_t r[32];
        tc::tmem_ld_16x32bx2_x32<256>(tmem + lane_base + kTmO + c0, r);   // O dims c0.. (half 0) / 256+c0.. (half 1)
        tc::tmem_wait_ld();
        const int c = half * 256 + c0;
        float o[32];
#pragma unroll
        for (int q2 = 0; q2 < 32; ++q2) o[q2] = __uint_as_float(r[q2]) * scale_out;
        if (g.splits == 1 && c >= 448) {
#pragma unroll
          for (int q2 = 0; q2 < 32; q2 += 2) {
            const float2 cs = s_cs[(c - 448 + q2) >> 1];            // rotate by -t: (cos, -sin)
            const float a0 = o[q2], a1 = o[q2 + 1];
            o[q2] = a0 * cs.x + a1 * cs.y;
            o[q2 + 1] = -a0 * cs.y + a1 * cs.x;
          }
        }
        if (g.splits > 1) {
          store_vec<32>(P.o_part + ((long long)split * gridDim.x * 64 + orow) * 512 + c, o);
        } else if (g.out_bf16) {
          store_vec<32>(reinterpret_cast<__nv_bfloat16*>(P.out) + orow * 512 + c, o);
        } else {
          store_vec<32>(reinterpret_cast<float*>(P.out) + orow * 512 + c, o);
        }
      }
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == kAtMmaWarp) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 512);
  }
}

// Merge key-range splits: for (query, head) rows, M = max(m_s, sink), combine,
// normalise, rotate the rotary block by -t and store.
__global__ void __launch_bounds__(128)
attn_combine_kernel(const float* __restrict__ o_part, const float* __restrict__ ml_part, const float* __restrict__ sink,
                    void* out, float* lse, int splits, long long rows, int Tq, long long q_pos0, double log_base,
                    int out_bf16) {
  const long long rh = blockIdx.x;                // row * 64 + h
  const long long row = rh >> 6;
  const int h = (int)(rh & 63);
  const long long t = q_pos0 + row % Tq;
  float M = sink ? sink[h] * kLog2e : -INFINITY;
  for (int s = 0; s < splits; ++s) M = fmaxf(M, ml_part[((long long)s * rows + row) * 128 + 2 * h]);
  float l = sink ? exp2f(sink[h] * kLog2e - M) : 0.f;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  const int d0 = threadIdx.x * 4;
  for (int s = 0; s < splits; ++s) {
    const float* ml = ml_part + ((long long)s * rows + row) * 128 + 2 * h;
    if (ml[0] == -INFINITY) continue;
    const float f = exp2f(ml[0] - M);
    l += ml[1] * f;
    const float4 o = *reinterpret_cast<const float4*>(o_part + ((long long)s * rows * 64 + rh) * 512 + d0);
    acc[0] += o.x * f; acc[1] += o.y * f; acc[2] += o.z * f; acc[3] += o.w * f;
  }
  const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
  for (int q = 0; q < 4; ++q) acc[q] *= inv;
  if (d0 >= 448) {
#pragma unroll
    for (int q = 0; q < 4; q += 2) {
      float c, sn;
      rope_cs(t, (d0 - 448 + q) >> 1, kRopeR, log_base, &c, &sn);
      const float a0 = acc[q], a1 = acc[q + 1];
      acc[q] = a0 * c + a1 * sn;
      acc[q + 1] = -a0 * sn + a1 * c;
    }
  }
  if (out_bf16) store_vec<4>(reinterpret_cast<__nv_bfloat16*>(out) + rh * 512 + d0, acc);
  else store_vec<4>(reinterpret_cast<float*>(out) + rh * 512 + d0, acc);
  if (lse && threadIdx.x == 0) lse[rh] = l > 0.f ? (M + log2f(l)) * 0.6931471805599453f : -INFINITY;
}

// ------------------------------------------------------------------ host side
struct AtPlan {
  int splits;
  int rot_slot;
  size_t off_rot_c, off_rot_w, off_opart, off_ml, total;
};

static AtPlan attn_tc_plan(const lcsa_attn_args* a, int sparse) {
  AtPlan p;
  const long long rows = (long long)a->B * a->Tq;
  long long max_c;
  if (sparse) max_c = a->k;
  else {
    long long nv = (a->q_pos0 + a->Tq - 1) / a->m;
    max_c = nv < a->Nc ? nv : a->Nc;
  }
  const int max_tiles = (int)((max_c + kAtKT - 1) / kAtKT + (a->W + kAtKT - 1) / kAtKT + 1);
  int splits = 1;
  if (rows < 2 * 148) {
    splits = (int)((2 * 148 + rows - 1) / rows);
    const int cap = max_tiles / 4 > 1 ? max_tiles / 4 : 1;        // >= 4 tiles per split
    splits = splits < cap ? splits : cap;
  }
  // A CTA stages at most kAtMaxIdx selected entries: larger k needs more key-range splits.
  if (sparse && a->k > kAtMaxIdx) {
    const int need = (max_tiles + kAtMaxIdx / kAtKT - 1) / (kAtMaxIdx / kAtKT);
    splits = splits > need ? splits : need;
  }
  p.splits = splits;
  p.rot_slot = sparse && ((long long)a->Tq * a->k < (long long)a->Nc) ? 1 : 0;
  auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
  size_t off = 0;
  p.off_rot_c = off;
  off += al((p.rot_slot ? (size_t)rows * a->k : (size_t)a->B * a->Nc) * 64 * 2);
  p.off_rot_w = off;
  off += al((size_t)a->B * a->Tkv * 64 * 2);
  p.off_opart = off;
  if (splits > 1) off += al((size_t)splits * rows * 64 * 512 * 4);
  p.off_ml = off;
  if (splits > 1) off += al((size_t)splits * rows * 128 * 4);
  p.total = off + 256;
  return p;
}

static size_t attn_tc_workspace(const lcsa_attn_args* a, int sparse) { return attn_tc_plan(a, sparse).total; }

static cudaError_t launch_attn_tc(const lcsa_attn_args* a, int sparse, void* ws, cudaStream_t st) {
  const AtPlan pl = attn_tc_plan(a, sparse);
  uint8_t* w = reinterpret_cast<uint8_t*>(ws);
  const double log_base = log(a->rope_base > 0.f ? (double)a->rope_base : 10000.0);
  const long long rows = (long long)a->B * a->Tq;
  AtPtrs P;
  P.q = (const __nv_bfloat16*)a->q;
  P.ckv = (const __nv_bfloat16*)a->ckv;
  P.idx = sparse ? a->idx : nullptr;
  P.kv = (const __nv_bfloat16*)a->kv;
  P.rot_c = (const __nv_bfloat16*)(w + pl.off_rot_c);
  P.rot_w = (const __nv_bfloat16*)(w + pl.off_rot_w);
  P.sink = a->sink;
  P.out = a->out;
  P.lse = a->lse;
  P.o_part = (float*)(w + pl.off_opart);
  P.ml_part = (float*)(w + pl.off_ml);
  cudaError_t e;
  // rotary slices of the keys
  if (a->Nc > 0) {
    if (pl.rot_slot)
      e = launch_rope_rows(a->ckv, w + pl.off_rot_c, rows * a->k, 512, 1, 0, a->m, log_base, 1, a->idx,
                           (long long)a->Tq * a->k, a->Nc, st);
    else
      e = launch_rope_rows(a->ckv, w + pl.off_rot_c, (long long)a->B * a->Nc, 512, a->Nc, 0, a->m, log_base, 0,
                           nullptr, 0, a->Nc, st);
    if (e != cudaSuccess) return e;
  }
  if (a->Tkv > 0 && a->W > 0) {
    e = launch_rope_rows(a->kv, w + pl.off_rot_w, (long long)a->B * a->Tkv, 512, a->Tkv, a->kv_pos0, 1, log_base, 0,
                         nullptr, 0, 0, st);
    if (e != cudaSuccess) return e;
  }
  AtGeom g;
  g.Tq = a->Tq; g.Nc = a->Nc; g.k = sparse ? a->k : 0; g.Tkv = a->Tkv;
  g.q_pos0 = a->q_pos0; g.kv_pos0 = a->kv_pos0; g.m = a->m; g.W = a->W;
  const float scale = a->softmax_scale > 0.f ? a->softmax_scale : 1.0f / sqrtf(512.f);
  g.scale_log2 = scale * kLog2e;
  g.log_base = log_base;
  g.sparse = sparse;
  g.rot_slot = pl.rot_slot;
  g.splits = pl.splits;
  g.out_bf16 = a->out_dtype == LCSA_BF16;
  e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kAtSmem);
  if (e != cudaSuccess) return e;
  // Tensor maps for the contiguous tiles (64 rows x 64 dims, 128-byte swizzle).
  // A map whose tensor is absent is never read; it points at q instead.
  CUtensorMap m_ckv, m_kv, m_rotc, m_rotw;
  const uint64_t rows_rotc = pl.rot_slot ? (uint64_t)rows * a->k : (uint64_t)a->B * a->Nc;
  auto mk = [&](CUtensorMap* m, const void* base, uint64_t nrows, uint64_t cols) {
    if (base == nullptr || nrows == 0) return make_tmap_bf16_2d(m, a->q, (uint64_t)rows * 64, 512, 512, 64, 64);
    return make_tmap_bf16_2d(m, base, nrows, cols, cols, 64, 64);
  };
  if (!mk(&m_ckv, a->Nc > 0 ? a->ckv : nullptr, (uint64_t)a->B * a->Nc, 512) ||
      !mk(&m_kv, a->Tkv > 0 ? a->kv : nullptr, (uint64_t)a->B * a->Tkv, 512) ||
      !mk(&m_rotc, a->Nc > 0 ? (const void*)P.rot_c : nullptr, rows_rotc, 64) ||
      !mk(&m_rotw, (a->Tkv > 0 && a->W > 0) ? (const void*)P.rot_w : nullptr, (uint64_t)a->B * a->Tkv, 64))
    return cudaErrorInvalidValue;
  dim3 grid((unsigned)rows, pl.splits);
  attn_tc_kernel<<<grid, kAtThreads, kAtSmem, st>>>(P, g, m_ckv, m_kv, m_rotc, m_rotw);
  count_launch();
  e = cudaGetLastError();
  if (e != cudaSuccess || pl.splits == 1) return e;
  count_launch();
  attn_combine_kernel<<<(unsigned)(rows * 64), 128, 0, st>>>(P.o_part, P.ml_part, a->sink, a->out, a->lse,
                                                              pl.splits, rows, a->Tq, a->q_pos0, log_base,
                                                              g.out_bf16);
  return cudaGetLastError();
}

}  // namespace lcsa
