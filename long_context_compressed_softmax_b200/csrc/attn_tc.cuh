// Core attention of CSA / HCA on tcgen05 tensor cores (BF16, H = 64 heads,
// D = 512, rotary R = 64).  DeepSeek-V4 hybrid attention, "第三步，core
// attention": multi-query attention of 64 heads over one shared K=V head; the
// key set is the selected compressed entries (CSA) or every visible entry
// (HCA), followed by the sliding window of raw tokens; a per-head sink logit
// joins the softmax denominator; the last 64 dims carry RoPE and the output
// is rotated back by -t.
//
// Persistent kernel: one CTA per SM walks a static list of (query, key-range
// split) items, latest query positions (the longest key lists) first.  Per
// 64-key tile:
//   S = Q K^T   tcgen05 M=64 (heads), N=64 (keys), K=512, A (Q) from tensor
//               memory; S double buffered in TMEM lanes 0-15 of each
//               sub-partition
//   softmax     two threads per head row, exp2 with a lazily updated running
//               max (O is rescaled only when the max grows by more than 2^8)
//   O += P V    tcgen05 M=64, N=2x256 (dims), K=64 keys; O lives in TMEM
//               lanes 16-31 of each sub-partition, all 512 columns
// The K tile doubles as V: the K-major view feeds S, the MN-major view of the
// same 128B-swizzled bytes feeds PV.
//
// The stage ring carries, per item, a Q pseudo-tile (the 64 query heads by
// TMA plus the (cos, sin) row of the query position) and then the key tiles.
// The transition warps move the next item's Q into tensor memory as soon as
// the current item's last S = Q K^T has completed, then run the current
// item's epilogue (TMEM -> registers -> global) while the softmax warps
// already work on the next item.
//
// Warps: 0-7 produce (TMA boxes for contiguous rows, 16-byte cp.async
// gathers for selected entries), 8 allocates TMEM and issues MMAs, 9-12 run
// the softmax, 13-16 handle the item transitions (Q into tensor memory, the
// previous item's epilogue), so the softmax warps only ever see key tiles.
// Rotary slices of the keys come pre-rotated (rope.cuh).  Every wait is
// bounded; abort decisions among threads that share a named barrier are
// taken collectively at that barrier.
#pragma once
#include <atomic>

#include "tc_ptx.cuh"
#include "rope.cuh"
#include "fp8cache.cuh"

namespace lcsa {

constexpr int kAtKT = 64;                      // keys per tile
constexpr int kAtProdWarps = 8;                 // gather / TMA producers
constexpr int kAtProdThreads = kAtProdWarps * 32;
constexpr int kAtMmaWarp = kAtProdWarps;        // TMEM allocator and MMA issuer
constexpr int kAtSmWarp0 = kAtProdWarps + 1;    // first of the 4 softmax warps
constexpr int kAtXtWarp0 = kAtSmWarp0 + 4;      // first of the 4 transition warps (Q moves, epilogues)
constexpr int kAtGroupThreads = 128;            // threads of the softmax or of the transition group
constexpr int kAtThreads = (kAtProdWarps + 9) * 32;   // 544: 96 registers per thread
constexpr uint32_t kAtKBytes = kAtKT * 512 * 2;  // 64 KB: one key tile, or the 64 heads of one query
constexpr uint32_t kAtPBytes = 64 * kAtKT * 2;   // 8 KB
constexpr uint32_t kAtRegion = 64 * 128;       // one 128-byte column block of a 64-row tile
constexpr int kAtMaxIdx = 2048;                 // selected entries staged in shared memory per item
constexpr int kAtStages = 3;                    // stage ring (key tiles and Q pseudo-tiles)
constexpr uint32_t kAtCsBytes = 32 * 8;         // (cos, sin) of the 32 rotary pairs at one position
// shared-memory carve-up, offsets from the 1 KB aligned base
constexpr uint32_t kAtOffP = kAtStages * kAtKBytes;
constexpr uint32_t kAtOffTab = kAtOffP + 2 * kAtPBytes;
constexpr uint32_t kAtOffIdx = kAtOffTab + kAtStages * kAtKT * 2 * 8;
constexpr uint32_t kAtOffCs = kAtOffIdx + kAtMaxIdx * 4;               // [kAtStages] per stage, [2] per item
constexpr uint32_t kAtOffStats = kAtOffCs + (kAtStages + 2) * kAtCsBytes;   // [2][64] (row max, row sum)
constexpr uint32_t kAtOffScl = kAtOffStats + 2 * 64 * 8;             // [kAtStages][64] FP8 entry scales
constexpr uint32_t kAtOffKm = kAtOffScl + kAtStages * kAtKT * 4;        // [kAtStages][2] valid-row masks
constexpr uint32_t kAtOffBar = kAtOffKm + 32;
constexpr int kAtBars = 22;
constexpr size_t kAtSmem = 1024 + kAtOffBar + kAtBars * 8;
static_assert(kAtSmem <= 232448, "attention shared memory exceeds 227 KB");
constexpr int kAtCodeBytes = 448;               // FP8 entry cache: E4M3 bytes of dims 0..447 per entry
// FP8 entry tiles stage their raw codes (64 x 448 B) in the upper part of
// regions 3-6 of their own stage, below the rotary region 7.
constexpr uint32_t kAtCodeStage = 7 * kAtRegion - kAtKT * kAtCodeBytes;
static_assert(kAtCodeStage % 16 == 0 && kAtCodeStage >= 3 * kAtRegion, "FP8 code staging");
constexpr float kLog2e = 1.4426950408889634f;
// TMEM map: lanes 0-15 of each sub-partition hold S[0] (cols 0-63), S[1]
// (64-127) and Q (128-383, the A operand of S = Q K^T); lanes 16-31 hold O
// (cols 0-511).
constexpr uint32_t kTmQ = 128;
constexpr uint32_t kTmO = 16u << 16;

struct AtGeom {
  int B, Tq, Nc, k, Tkv;
  long long rows;      // B * Tq
  long long q_pos0, kv_pos0;
  int m, W;
  float scale_log2;
  int sparse;
  int rot_slot;        // CSA rotary slices indexed by (query, slot) instead of by entry
  int splits;
  int out_bf16;
  int out_v8;          // the output (or split partials) is 32-byte aligned: 32-byte stores
  int n_items;         // rows * splits
  int fp8;             // entries come from the FP8 cache (codes + scales + BF16 rotary slices)
};

struct AtPtrs {
  const __nv_bfloat16* ckv;
  const uint8_t* c8;            // FP8 entry cache: codes [B*Nc][448] (else null)
  const uint8_t* c8s;           // FP8 entry cache: scale bytes X + 127 [B*Nc]
  const int32_t* idx;
  const int32_t* nc;            // sparse: number of valid selected entries of each query row
  const float2* cs;             // [Tq][32] (cos, sin) at each query position
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
// Arrive on `bar` (counted as one of its expected arrivals) once every
// cp.async this thread issued so far has landed.
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(tc::smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// all but this thread's most recent cp.async group have landed
__device__ __forceinline__ void cp_async_wait_prev() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

// Key-set geometry of one query: n_c compressed entries (selected or
// visible), then the window of raw tokens.
struct KeySet {
  int n_c, n_w, tiles_c, tiles;
  long long wlo;
};
__device__ __forceinline__ KeySet key_set(const AtGeom& g, int n_c, long long t) {
  KeySet s;
  s.n_c = n_c;
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

// Work item `it`: query position rank it / (B * splits) counted from the
// last position down, then sequence, then split.
struct AtItem {
  long long row, t;
  int b, i, split;
  KeySet ks;
  int t0, n_tiles;     // tile range [t0, t0 + n_tiles) of the query's key list
};
__device__ __forceinline__ void at_item_rank(const AtGeom& g, int it, int* b, int* i, int* split) {
  const int per = g.B * g.splits;
  const int r = it / per, rem = it - r * per;
  *i = g.Tq - 1 - r;
  *b = rem / g.splits;
  *split = rem - *b * g.splits;
}
// Entry count of item `it` (a global load for CSA: issued one item ahead).
__device__ __forceinline__ int at_item_nc(const AtGeom& g, const AtPtrs& P, int it) {
  if (it >= g.n_items) return 0;
  int b, i, split;
  at_item_rank(g, it, &b, &i, &split);
  if (g.sparse) return __ldg(P.nc + (long long)b * g.Tq + i);
  const long long nv = (g.q_pos0 + i) / g.m;
  return (int)(nv < g.Nc ? nv : g.Nc);
}
__device__ __forceinline__ AtItem at_item(const AtGeom& g, int it, int n_c) {
  AtItem x;
  at_item_rank(g, it, &x.b, &x.i, &x.split);
  x.row = (long long)x.b * g.Tq + x.i;
  x.t = g.q_pos0 + x.i;
  x.ks = key_set(g, n_c, x.t);
  const int per_split = (x.ks.tiles + g.splits - 1) / g.splits;
  x.t0 = x.split * per_split;
  const int t1 = x.t0 + per_split < x.ks.tiles ? x.t0 + per_split : x.ks.tiles;
  x.n_tiles = t1 > x.t0 ? t1 - x.t0 : 0;
  return x;
}

// An item without keys: zero output, log-sum-exp of the sink alone.
__device__ void at_store_empty(const AtGeom& g, const AtPtrs& P, const AtItem& x, int tid) {
  for (int e = tid; e < 64 * 512; e += kAtGroupThreads) {
    const long long o = x.row * 64 * 512 + e;
    if (g.splits > 1) P.o_part[(long long)x.split * g.rows * 64 * 512 + o] = 0.f;
    else if (g.out_bf16) reinterpret_cast<__nv_bfloat16*>(P.out)[o] = __float2bfloat16_rn(0.f);
    else reinterpret_cast<float*>(P.out)[o] = 0.f;
  }
  if (tid < 64) {
    const int h = tid;
    if (g.splits > 1) {
      float* ml = P.ml_part + ((long long)x.split * g.rows + x.row) * 128 + 2 * h;
      ml[0] = -INFINITY;
      ml[1] = 0.f;
    } else if (P.lse) {
      P.lse[x.row * 64 + h] = P.sink ? P.sink[h] : -INFINITY;
    }
  }
}

// Q (staged by TMA in `qs`, 128B-swizzled 64-dim blocks) -> TMEM A operand
// (two dims per column).  Step c covers dims 64c .. 64c+63: thread (h % 16)
// writes dims 64c .. +31, thread (h % 16) + 16 dims 64c+32 .. +63 (16x32bx2
// with a 16-column offset), so both half-warps share the rotary block (dims
// 448..511, rotated at t with the (cos, sin) row `cs`).
__device__ __forceinline__ void at_q_to_tmem(const uint8_t* qs, const float2* cs, uint32_t taddr, int h, int half) {
  const uint8_t* qrow = qs + h * 128;
#pragma unroll 2
  for (int c = 0; c < 8; ++c) {
    uint32_t r[16];
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int chunk = half * 4 + v;             // 16-byte chunk within the 128-byte row of block c
      const uint4 x = *reinterpret_cast<const uint4*>(qrow + c * kAtRegion + ((chunk ^ (h & 7)) << 4));
      r[4 * v] = x.x; r[4 * v + 1] = x.y; r[4 * v + 2] = x.z; r[4 * v + 3] = x.w;
    }
    if (c == 7) {
#pragma unroll
      for (int q2 = 0; q2 < 16; ++q2) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&r[q2]));
        const float2 e = cs[half * 16 + q2];
        const __nv_bfloat162 o = __floats2bfloat162_rn(f.x * e.x - f.y * e.y, f.x * e.y + f.y * e.x);
        r[q2] = *reinterpret_cast<const uint32_t*>(&o);
      }
    }
    tc::tmem_st_16x32bx2_x16<16>(taddr + c * 32, r);
  }
  tc::tmem_wait_st();
}

// 32 consecutive values as 32-byte stores (p 32-byte aligned).
__device__ __forceinline__ void st_v8(void* p, const uint32_t* w) {
  asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(w[0]), "r"(w[1]), "r"(w[2]),
               "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
               : "memory");
}
__device__ __forceinline__ void store32_v8(float* p, const float* o) {
#pragma unroll
  for (int j = 0; j < 4; ++j) st_v8(p + 8 * j, reinterpret_cast<const uint32_t*>(o + 8 * j));
}
__device__ __forceinline__ void store32_v8(__nv_bfloat16* p, const float* o) {
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    uint32_t w[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const __nv_bfloat162 b2 = __floats2bfloat162_rn(o[16 * j + 2 * e], o[16 * j + 2 * e + 1]);
      w[e] = *reinterpret_cast<const uint32_t*>(&b2);
    }
    st_v8(p + 16 * j, w);
  }
}

// 16 consecutive FP32 values given as bit patterns, as 32-byte stores (p 32-byte aligned).
__device__ __forceinline__ void store16_v8_bits(float* p, const uint32_t* v) {
  st_v8(p, v);
  st_v8(p + 8, v + 8);
}
__device__ __forceinline__ void store16_v8_bits(__nv_bfloat16* p, const uint32_t* v) {
  uint32_t w[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]));
    w[e] = *reinterpret_cast<const uint32_t*>(&b2);
  }
  st_v8(p, w);
}

// Epilogue of one item, executed by the 128 transition threads.  Row
// statistics come from the softmax warps through shared memory; O -> sink,
// normalisation, -t rotation of the rotary block -> output (or split
// partials) straight from registers.  Piece k covers dims 32k .. 32k+31:
// thread (h % 16) takes dims 32k .. +15 and thread (h % 16) + 16 dims
// 32k+16 .. +31 (16x32bx2 with a 16-column offset), so each warp store
// instruction writes 16 rows x 2 adjacent 32-byte pieces (BF16).  The TMEM
// read of piece k+1 is in flight while piece k is scaled and stored;
// o_free[0] (dims 0-255, the first PV half of the next item) is arrived on
// after piece 7's read, o_free[1] after piece 15's.
__device__ bool at_epilogue(const AtGeom& g, const AtPtrs& P, uint64_t* pv_done, uint64_t* o_free /*[2]*/,
                            uint64_t* stats_full, const float2* stats, int item, const float2* cs, long long row,
                            int split, int last, uint32_t tmem, uint32_t lane_base, int h, int half, int xt, bool ok) {
  const int lane = xt & 31;
  if (!tc::mbar_wait(stats_full + (item & 1), (item >> 1) & 1)) ok = false;
  if (!tc::mbar_wait(pv_done + (last & 1), (last >> 1) & 1)) ok = false;
  tc::tc_fence_after();
  const float2 ml = stats[(item & 1) * 64 + h];         // (running max in log2 units, row sum)
  const long long orow = row * 64 + h;
  float scale_out = 1.f;
  if (g.splits > 1) {
    if (half == 0) {
      float* mlp = P.ml_part + ((long long)split * g.rows + row) * 128 + 2 * h;
      mlp[0] = ml.x;
      mlp[1] = ml.y;
    }
  } else {
    float M = ml.x, l = ml.y;
    if (P.sink) {
      const float s2 = P.sink[h] * kLog2e;
      const float Mn = fmaxf(M, s2);
      l = l * exp2f(M - Mn) + exp2f(s2 - Mn);
      scale_out = exp2f(M - Mn);
      M = Mn;
    }
    scale_out = l > 0.f ? scale_out / l : 0.f;
    if (half == 0 && P.lse) P.lse[orow] = l > 0.f ? (M + log2f(l)) * 0.6931471805599453f : -INFINITY;
  }
  float* of32 = g.splits > 1 ? P.o_part + ((long long)split * g.rows * 64 + orow) * 512
                             : (g.out_bf16 ? nullptr : reinterpret_cast<float*>(P.out) + orow * 512);
  __nv_bfloat16* obf = (g.splits == 1 && g.out_bf16) ? reinterpret_cast<__nv_bfloat16*>(P.out) + orow * 512 : nullptr;
  const uint32_t taddr = tmem + lane_base + kTmO;
  // piece k (0..15) = O columns 32k .. 32k+31: thread (h % 16) dims 32k .. +15,
  // thread (h % 16) + 16 dims 32k+16 .. +31 (16x32bx2 with a 16-column offset)
  uint32_t buf[2][16];
  tc::tmem_ld_16x32bx2_x16<16>(taddr, buf[0]);
#pragma unroll 2
  for (int k = 0; k < 16; ++k) {
    uint32_t* v = buf[k & 1];
    tc::tmem_wait_ld_regs16(v);
    if (k + 1 < 16) tc::tmem_ld_16x32bx2_x16<16>(taddr + (k + 1) * 32, buf[(k + 1) & 1]);
    if (k == 7 || k == 15) {
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(o_free + (k == 15 ? 1 : 0));  // that half of O may be overwritten
    }
    const int d0 = k * 32 + half * 16;                 // first output dim of this thread's piece
    // scaled in place (FP32 bit patterns in v)
#pragma unroll
    for (int q2 = 0; q2 < 16; ++q2) v[q2] = __float_as_uint(__uint_as_float(v[q2]) * scale_out);
    if (k >= 14 && g.splits == 1) {
#pragma unroll
      for (int q2 = 0; q2 < 16; q2 += 2) {
        const float2 e = cs[(d0 - 448 + q2) >> 1];      // rotate by -t: (cos, -sin)
        const float a0 = __uint_as_float(v[q2]), a1 = __uint_as_float(v[q2 + 1]);
        v[q2] = __float_as_uint(a0 * e.x + a1 * e.y);
        v[q2 + 1] = __float_as_uint(-a0 * e.y + a1 * e.x);
      }
    }
    if (g.out_v8) {
      if (obf) store16_v8_bits(obf + d0, v);
      else store16_v8_bits(of32 + d0, v);
    } else {
#pragma unroll
      for (int j = 0; j < 16; j += 8) {
        float o[8];
#pragma unroll
        for (int q2 = 0; q2 < 8; ++q2) o[q2] = __uint_as_float(v[j + q2]);
        if (obf) store_vec<8>(obf + d0 + j, o);
        else store_vec<8>(of32 + d0 + j, o);
      }
    }
  }
  return ok;
}

// kFp8: the entries come from the FP8 cache (a separate instantiation, so the
// BF16 kernel carries none of the expansion code).  kG4: BF16 selected rows
// arrive by TMA tile::gather4 instead of 16-byte cp.async (the measured
// alternative; cp.async is the default).
template <bool kFp8, bool kG4>
__global__ void __launch_bounds__(kAtThreads, 1)
attn_tc_kernel(AtPtrs P, AtGeom g, const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_ckv,
               const __grid_constant__ CUtensorMap tm_kv, const __grid_constant__ CUtensorMap tm_rotc,
               const __grid_constant__ CUtensorMap tm_rotw) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* s_k = smem;                                                        // kAtStages stages
  uint8_t* s_p = smem + kAtOffP;                                              // 2 P buffers
  const uint8_t** s_tab = reinterpret_cast<const uint8_t**>(smem + kAtOffTab);  // [stage][64][2] row pointers
  int32_t* s_idx = reinterpret_cast<int32_t*>(smem + kAtOffIdx);              // selected entries of the item
  float2* s_cs = reinterpret_cast<float2*>(smem + kAtOffCs);                  // [stage][32] with the Q pseudo-tile
  float2* s_cs_item = s_cs + kAtStages * 32;                                  // [2][32] for the epilogue
  float2* s_stats = reinterpret_cast<float2*>(smem + kAtOffStats);            // [2][64] softmax -> epilogue
  float* s_scl = reinterpret_cast<float*>(smem + kAtOffScl);                  // [stage][64] FP8 entry scales
  uint32_t* s_km = reinterpret_cast<uint32_t*>(smem + kAtOffKm);              // [stage][2] rows read (gathered tiles)
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kAtOffBar);
  uint64_t* q_ready = bars + 0;                 // transition warps (4): Q of the item is in TMEM
  uint64_t* kv_full = bars + 1;                 // [kAtStages] producers (one arrival each; TMA bytes)
  uint64_t* kv_empty = kv_full + kAtStages;     // [kAtStages] MMA commit (key tiles) / transition (Q)
  uint64_t* s_full = kv_empty + kAtStages;      // [2] MMA commit
  uint64_t* s_free = s_full + 2;                // [2] softmax warps (4)
  uint64_t* p_full = s_free + 2;                // [2] softmax warps (4)
  uint64_t* pv_done = p_full + 2;               // [2] MMA commit
  uint64_t* o_free = pv_done + 2;               // [2] transition warps (4): the epilogue has read O dims 0-255 / 256-511
  uint64_t* stats_full = o_free + 2;            // [2] by item parity, softmax warps (4): row statistics
  uint64_t* q_full = stats_full + 2;            // [2] by item parity, TMA bytes: Q and its (cos, sin) row
  uint64_t* s_done = q_full + 2;                // MMA commit after the last S of each item
  // Waiters that skip phases (the transition warps watch one event per item)
  // get barriers of their own, so that no parity wait can see a stale phase.
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = (int)gridDim.x;

  if (threadIdx.x == 0) {
    tc::mbar_init(q_ready, 4);
    for (int s = 0; s < kAtStages; ++s) {
      // every producer arrives where all of them fill tiles (gathered rows, FP8
      // expansion); otherwise thread 0 alone fills by TMA and arrives
      tc::mbar_init(kv_full + s, ((g.sparse && !kG4) || kFp8) ? kAtProdThreads : 1);
      tc::mbar_init(kv_empty + s, 1);
    }
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(s_full + s, 1);
      tc::mbar_init(s_free + s, 4);
      tc::mbar_init(p_full + s, 4);
      tc::mbar_init(pv_done + s, 1);
    }
    tc::mbar_init(o_free, 4);
    tc::mbar_init(o_free + 1, 4);
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(stats_full + s, 4);
      tc::mbar_init(q_full + s, 1);
    }
    tc::mbar_init(s_done, 1);
    tc::fence_barrier_init();
    s_abort = 0;
  }
  if (warp == kAtMmaWarp) { tc::tmem_alloc(&s_tmem, 512); tc::tmem_relinquish(); }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = s_tmem;
  volatile int* abort_flag = &s_abort;

  if (warp < kAtProdWarps) {
    // ============================================================ producers
    // Q and contiguous key tiles (every HCA entry tile and every window tile)
    // arrive as eight 2D TMA boxes of 64 rows x 64 dims; CSA's selected rows
    // are gathered 16 bytes at a time with cp.async by all producer warps
    // (which share named barrier 1 and leave only together), or with kG4 by
    // TMA gather, four rows per copy, warp w filling column block w.
    const int tid = threadIdx.x;                    // 0..kAtProdThreads-1
    if (tid == 0) {
      tc::prefetch_tmap(&tm_q);
      tc::prefetch_tmap(&tm_ckv);
      tc::prefetch_tmap(&tm_kv);
      tc::prefetch_tmap(&tm_rotc);
      tc::prefetch_tmap(&tm_rotw);
    }
    const uint8_t* dummy = reinterpret_cast<const uint8_t*>(P.cs);
    // Entry tiles that every producer fills (gathered rows, FP8 expansion)
    // make the producers leave only together, at named barrier 1.
    const bool coll = (g.sparse && !kG4) || kFp8;
    // TMA-gathered rows: every producer warp gathers; the lanes of a warp
    // share its abort decisions by warp votes.
    const bool gw = kG4 && g.sparse;
    // The threads that need a free stage wait for it (without sleeping):
    // thread 0, which issues every TMA copy, the 64 threads that build a
    // gathered tile's row table (the others are released by named barrier 1
    // after them) and the TMA-gathering warps.  Otherwise the other producers
    // have no work.
    const bool waits = tid == 0 || (coll && tid < kAtKT) || gw;
    bool bad = false;
    // The slot of the latest TMA fill of each stage and of each Q buffer
    // (thread 0), so that an abort waits for the copies still in flight
    // (registers: a run-time index into an array would put it on the stack).
    static_assert(kAtStages == 3, "one fill record per stage");
    int tx0 = -1, tx1 = -1, tx2 = -1, txq0 = -1, txq1 = -1;
    auto set_tx = [&](int st, int v) {
      if (st == 0) tx0 = v;
      else if (st == 1) tx1 = v;
      else tx2 = v;
    };
    // FP8 entry tiles are expanded one tile behind their copies: the stage of
    // the tile whose codes are in flight or landed but not yet expanded.
    int pend = -1;
    constexpr int kCodePer = kAtKT * (kAtCodeBytes / 16) / kAtProdThreads;   // 7
    constexpr int kRopePer = kAtKT * 8 / kAtProdThreads;                     // 2
    static_assert(kCodePer * kAtProdThreads == kAtKT * (kAtCodeBytes / 16), "code pieces per thread");
    static_assert(kRopePer * kAtProdThreads == kAtKT * 8, "rotary pieces per thread");
    // Expand the pending tile: its copies land (keep_newest: this thread's
    // latest group, the next tile's, may stay in flight), every producer has
    // read its codes before any BF16 row is written over them, then a proxy
    // fence and this thread's arrival on the tile's full barrier.  Collective
    // over the producers; false when one of them gave up.
    auto expand_pending = [&](bool keep_newest) -> bool {
      if (pend < 0) return true;
      if (keep_newest) cp_async_wait_prev();
      else cp_async_wait_all();
      if (!tc::bar_and(1, kAtProdThreads, !bad)) return false;
      uint8_t* stg = s_k + pend * kAtKBytes;
      uint4 cv[kCodePer];
#pragma unroll
      for (int u = 0; u < kCodePer; ++u) {
        const int q = tid + u * kAtProdThreads;                 // 16-code piece q % 28 of row q / 28
        cv[u] = *reinterpret_cast<const uint4*>(stg + kAtCodeStage + q * 16);
      }
      if (!tc::bar_and(1, kAtProdThreads, true)) return false;
#pragma unroll
      for (int u = 0; u < kCodePer; ++u) {
        const int q = tid + u * kAtProdThreads;
        const int kk = q / (kAtCodeBytes / 16), p = q - kk * (kAtCodeBytes / 16);
        uint4 lo, hi;
        e4m3x16_to_bf16(cv[u], s_scl[pend * kAtKT + kk], lo, hi);
        uint8_t* row = stg + (p >> 2) * kAtRegion + kk * 128;   // 16 codes = dims 16p .. 16p+15
        const int c0 = (p & 3) * 2;
        *reinterpret_cast<uint4*>(row + ((c0 ^ (kk & 7)) << 4)) = lo;
        *reinterpret_cast<uint4*>(row + (((c0 + 1) ^ (kk & 7)) << 4)) = hi;
      }
      tc::fence_proxy_async_smem();
      tc::mbar_arrive(kv_full + pend);
      pend = -1;
      return true;
    };
    int slot = 0, ni = 0;
    // CSA: the selected entries of the next item, loaded into registers while
    // the current item's tiles are gathered (its first gather then starts as
    // soon as a stage frees, without a dependent index load in front of it).
    constexpr int kPer = (kAtMaxIdx + kAtProdThreads - 1) / kAtProdThreads;
    int32_t e_pre[kPer];
    int pre_it = -1;
    auto load_idx = [&](const AtItem& y, int32_t* e_v) {
      const int s0 = y.t0 * kAtKT;
      const int32_t* idx_row = P.idx + y.row * g.k + s0;
      const int hi = y.ks.n_c < (y.t0 + y.n_tiles) * kAtKT ? y.ks.n_c : (y.t0 + y.n_tiles) * kAtKT;
#pragma unroll
      for (int u = 0; u < kPer; ++u) {
        const int e = tid + u * kAtProdThreads;
        e_v[u] = e < hi - s0 ? __ldg(idx_row + e) : 0;
      }
    };
    int nc_next = at_item_nc(g, P, blockIdx.x);
    for (int it = (coll || tid == 0 || gw) ? blockIdx.x : g.n_items; it < g.n_items; it += G) {
      const int nc_cur = nc_next;
      nc_next = at_item_nc(g, P, it + G);
      const AtItem x = at_item(g, it, nc_cur);
      if (x.n_tiles == 0) continue;
      {
        // ---- Q pseudo-tile: data on q_full[ni & 1]; the stage's kv_full
        // phase completes at once (nobody waits on it) to keep the ring's
        // phase count one per slot.
        const int st = slot % kAtStages;
        if (slot >= kAtStages && tid == 0 && !tc::mbar_wait(kv_empty + st, ((slot / kAtStages) - 1) & 1)) bad = true;
        if (*abort_flag) bad = true;
        if (gw) bad = __any_sync(0xffffffffu, bad);
        if (bad && !coll) break;
        if (tid == 0) {
          uint64_t* qf = q_full + (ni & 1);
          if (!bad) {
            set_tx(st, -1);                         // the stage's previous fill was consumed
            if (ni & 1) txq1 = ni; else txq0 = ni;
            tc::mbar_arrive_expect_tx(qf, kAtKBytes + kAtCsBytes);
#pragma unroll
            for (int reg = 0; reg < 8; ++reg)
              tc::tma_load_2d(s_k + st * kAtKBytes + reg * kAtRegion, &tm_q, qf, reg * 64, (int)(x.row * 64));
            tc::bulk_load(s_cs + st * 32, P.cs + (long long)x.i * 32, kAtCsBytes, qf);
          } else {
            tc::mbar_arrive(qf);
          }
        }
        if (coll || tid == 0) tc::mbar_arrive(kv_full + st);
        ++slot;
        ++ni;
      }
      const int slot0 = x.t0 * kAtKT;
      if (g.sparse && coll) {
        // Every read of the previous item's s_idx precedes the barrier of its
        // last gathered tile, which all producers have passed.  The entries
        // come from the registers filled during the previous item (all loads
        // issued before the first store when they were not prefetched).
        const int hi = x.ks.n_c < (x.t0 + x.n_tiles) * kAtKT ? x.ks.n_c : (x.t0 + x.n_tiles) * kAtKT;
        int32_t e_v[kPer];
        if (pre_it == it) {
#pragma unroll
          for (int u = 0; u < kPer; ++u) e_v[u] = e_pre[u];
        } else {
          load_idx(x, e_v);
        }
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
          const int e = tid + u * kAtProdThreads;
          if (e < hi - slot0) s_idx[e] = e_v[u];
        }
        // the next item's entries, in flight during this item's gathers
        pre_it = -1;
        if (it + G < g.n_items) {
          const AtItem y = at_item(g, it + G, nc_next);
          if (y.n_tiles > 0) {
            load_idx(y, e_pre);
            pre_it = it + G;
          }
        }
        if (!tc::bar_and(1, kAtProdThreads, !bad)) { bad = true; break; }
      }
      for (int n = 0; n < x.n_tiles; ++n, ++slot) {
        const int st = slot % kAtStages;
        const int gt = x.t0 + n;                    // tile index in the query's key list
        // TMA-gathered tile: lane l of each warp reads the entries of keys
        // 4 (l % 16) .. +3, the four-row group its copy fills, before the
        // stage wait
        const bool gath = gw && gt < x.ks.tiles_c;
        int32_t ev[4];
        if (gath) {
          const int sl0 = gt * kAtKT + 4 * (lane & 15);
          const int32_t* idx_row = P.idx + x.row * g.k;
#pragma unroll
          for (int j = 0; j < 4; ++j) ev[j] = sl0 + j < x.ks.n_c ? __ldg(idx_row + sl0 + j) : -1;
        }
        if (slot >= kAtStages && waits && !tc::mbar_wait(kv_empty + st, ((slot / kAtStages) - 1) & 1)) bad = true;
        if (*abort_flag) bad = true;
        if (gw) bad = __any_sync(0xffffffffu, bad);
        uint8_t* stage = s_k + st * kAtKBytes;
        if (gath) {
          // ---- selected rows by TMA gather: warp w < 7 fills entry column
          // block w, warp 7 the rotated slice, lanes 0-15 one four-row group
          // each; absent rows and bad indices take a row past the tensor's
          // end (zeros) and leave the tile's row mask.  Thread 0 arms the
          // stage for all 64 KB; a copy of another warp may land first (the
          // pending byte count goes below zero until then).
          if (bad) break;
          const int grp = lane & 15;
          const int oob_c = (int)((long long)g.B * g.Nc);
          const int oob_r = g.rot_slot ? (int)(g.rows * g.k) : oob_c;
          int yc[4], yr[4];
          uint32_t v = 0;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int sl = gt * kAtKT + 4 * grp + j;
            yc[j] = oob_c;
            yr[j] = oob_r;
            if (sl < x.ks.n_c) {
              if (ev[j] >= 0 && ev[j] < g.Nc) {
                yc[j] = (int)((long long)x.b * g.Nc + ev[j]);
                yr[j] = g.rot_slot ? (int)(x.row * g.k + sl) : yc[j];
                v |= 1u << j;
              } else if (tid < 16) {                // warp 0 reports
                report(LCSA_DEV_BAD_INDEX);
              }
            }
          }
          if (warp == 0) {
            const uint32_t km_lo = __reduce_or_sync(0xffffffffu, grp < 8 ? v << (4 * grp) : 0u);
            const uint32_t km_hi = __reduce_or_sync(0xffffffffu, grp >= 8 ? v << (4 * (grp - 8)) : 0u);
            if (tid == 0) {
              s_km[st * 2] = km_lo;
              s_km[st * 2 + 1] = km_hi;
              set_tx(st, slot);
              tc::mbar_arrive_expect_tx(kv_full + st, kAtKBytes);
            }
          }
          if (lane < 16) {
            uint8_t* dst = stage + warp * kAtRegion + grp * 4 * 128;
            if (warp < 7)
              tc::tma_gather4(dst, &tm_ckv, kv_full + st, warp * 64, yc[0], yc[1], yc[2], yc[3]);
            else
              tc::tma_gather4(dst, &tm_rotc, kv_full + st, 0, yr[0], yr[1], yr[2], yr[3]);
          }
          continue;
        }
        if (gt >= x.ks.tiles_c || !coll) {
          // ---- contiguous rows: TMA boxes
          if (pend >= 0 && !expand_pending(false)) { bad = true; break; }
          if (coll) {
            if (!tc::bar_and(1, kAtProdThreads, !bad)) { bad = true; break; }
          } else if (bad) {
            break;
          }
          if (tid == 0) {
            const CUtensorMap* mm;
            const CUtensorMap* mr;
            int y;
            if (gt < x.ks.tiles_c) {
              mm = &tm_ckv; mr = &tm_rotc;
              y = (int)((long long)x.b * g.Nc + (long long)gt * kAtKT);
            } else {
              mm = &tm_kv; mr = &tm_rotw;
              y = (int)((long long)x.b * g.Tkv + (x.ks.wlo - g.kv_pos0) + (long long)(gt - x.ks.tiles_c) * kAtKT);
            }
            set_tx(st, slot);
            tc::mbar_arrive_expect_tx(kv_full + st, kAtKBytes);
#pragma unroll
            for (int reg = 0; reg < 7; ++reg) tc::tma_load_2d(stage + reg * kAtRegion, mm, kv_full + st, reg * 64, y);
            tc::tma_load_2d(stage + 7 * kAtRegion, mr, kv_full + st, 0, y);
          } else if (coll) {
            tc::mbar_arrive(kv_full + st);
          }
          continue;
        }
        // ---- gathered rows (CSA) or FP8 entry rows: per-tile row table first
        const uint8_t** tab = s_tab + st * kAtKT * 2;
        if (tid < kAtKT) {
          const int kk = tid;
          const uint8_t* rm = nullptr;
          const uint8_t* rr = nullptr;
          float scl = 0.f;
          const int sl = gt * kAtKT + kk;
          if (sl < x.ks.n_c) {
            const int j = g.sparse ? s_idx[sl - slot0] : sl;      // dense: slot sl holds entry sl
            if (j >= 0 && j < g.Nc) {
              const long long e = (long long)x.b * g.Nc + j;
              rm = kFp8 ? P.c8 + e * kAtCodeBytes : reinterpret_cast<const uint8_t*>(P.ckv + e * 512);
              rr = reinterpret_cast<const uint8_t*>(P.rot_c + (g.rot_slot ? (x.row * g.k + sl) : e) * 64);
              if (kFp8) scl = ldexpf(1.f, (int)__ldg(P.c8s + e) - 127);
            } else {
              report(LCSA_DEV_BAD_INDEX);
            }
          }
          tab[2 * kk] = rm;
          tab[2 * kk + 1] = rr;
          s_scl[st * kAtKT + kk] = scl;
          // keys whose row is read: a bad index is skipped, not a zero key
          const uint32_t vm = __ballot_sync(0xffffffffu, rm != nullptr);
          if ((kk & 31) == 0) s_km[st * 2 + (kk >> 5)] = vm;
        }
        if (!tc::bar_and(1, kAtProdThreads, !bad)) { bad = true; break; }
        if (kFp8) {
          // FP8 entry rows: the 448 code bytes of each row land by 16-byte
          // cp.async in the stage's code staging area, the BF16 rotary rows at
          // their swizzled addresses in region 7 (absent rows: zeros); then
          // the previous FP8 tile is expanded while these copies are in flight.
          const uint32_t sb = tc::smem_u32(stage);
#pragma unroll
          for (int u = 0; u < kCodePer; ++u) {
            const int q = tid + u * kAtProdThreads;
            const int kk = q / (kAtCodeBytes / 16), p = q - kk * (kAtCodeBytes / 16);
            const uint8_t* base = tab[2 * kk];
            cp_async16(sb + kAtCodeStage + q * 16, base ? base + p * 16 : dummy, base ? 16u : 0u);
          }
#pragma unroll
          for (int u = 0; u < kRopePer; ++u) {
            const int q = tid + u * kAtProdThreads;
            const int kk = q >> 3, c16 = q & 7;
            const uint8_t* base = tab[2 * kk + 1];
            cp_async16(sb + 7 * kAtRegion + kk * 128 + ((c16 ^ (kk & 7)) << 4), base ? base + c16 * 16 : dummy,
                       base ? 16u : 0u);
          }
          cp_async_commit();
          if (pend >= 0 && !expand_pending(true)) { bad = true; break; }
          pend = st;
          continue;
        }
        // 16-byte piece q = tid + u * kAtProdThreads of the 64 x 1 KB tile:
        // key q / 64, piece q % 64 of its row (region = 64-dim block).
        const uint32_t sbase = tc::smem_u32(stage);
#pragma unroll 4
        for (int u = 0; u < (kAtKT * 64 + kAtProdThreads - 1) / kAtProdThreads; ++u) {
          const int q = tid + u * kAtProdThreads;
          if (q >= kAtKT * 64) break;
          const int kk = q >> 6, piece = q & 63;
          const int region = piece >> 3, c16 = piece & 7;
          const uint32_t kb = sbase + region * kAtRegion + (c16 << 4);
          const int off = region == 7 ? c16 * 16 : piece * 16;
          const uint8_t* base = tab[2 * kk + (region == 7 ? 1 : 0)];
          const uint32_t dst = (kb + kk * 128) ^ ((uint32_t)(kk & 7) << 4);
          cp_async16(dst, base ? base + off : dummy, base ? 16u : 0u);
        }
        cp_async_arrive_noinc(kv_full + st);
      }
      if (!bad && pend >= 0 && !expand_pending(false)) bad = true;   // no FP8 tile stays pending across items
      if (bad) break;
    }
    cp_async_wait_all();                            // nothing may land after the CTA exits
    if (bad) {
      *abort_flag = 1;
      // TMA fills still in flight land before the CTA exits (bounded waits:
      // each of these fills was armed with its full byte count)
      if (tid == 0) {
        const int txs[3] = {tx0, tx1, tx2};
#pragma unroll
        for (int s2 = 0; s2 < kAtStages; ++s2)
          if (txs[s2] >= 0) tc::mbar_wait(kv_full + s2, (txs[s2] / kAtStages) & 1);
        if (txq0 >= 0) tc::mbar_wait(q_full, (txq0 >> 1) & 1);
        if (txq1 >= 0) tc::mbar_wait(q_full + 1, (txq1 >> 1) & 1);
      }
    }
  } else if (warp == kAtMmaWarp) {
    // ============================================================ MMA issuer
    // S(n+1) and PV(n) are independent: whichever is ready is issued first.
    if (tc::elect_one()) {
      const uint64_t limit_ns = tc::wait_limit();                  // read once: the loop below polls
      const uint32_t idesc_s = tc::idesc_bf16(64, kAtKT, 0, 0);    // A (TMEM) K-major, B K-major
      const uint32_t idesc_o = tc::idesc_bf16(64, 256, 0, 1);      // A K-major, B MN-major
      bool ok = true;
      int slot = 0, tcount = 0, ni = 0;
      int nc_next = at_item_nc(g, P, blockIdx.x);
      for (int it = blockIdx.x; ok && it < g.n_items; it += G) {
        const int nc_cur = nc_next;
        nc_next = at_item_nc(g, P, it + G);
        const AtItem x = at_item(g, it, nc_cur);
        if (x.n_tiles == 0) continue;
        ++slot;                                     // the Q pseudo-tile
        if (!tc::mbar_wait(q_ready, ni & 1)) { ok = false; break; }
        tc::tc_fence_after();
        int next_s = 0, next_pv = 0;
        int pv_half = 0;                            // halves of PV(next_pv) already issued
        uint64_t t_idle = 0;
        while (next_pv < x.n_tiles) {
          bool did = false;
          if (next_s < x.n_tiles && next_s <= next_pv + 1) {
            const int gs = tcount + next_s, ss = slot + next_s;
            const int st = ss % kAtStages, sb = gs & 1;
            if (tc::mbar_try_wait(kv_full + st, (ss / kAtStages) & 1) &&
                (gs < 2 || tc::mbar_try_wait(s_free + sb, ((gs >> 1) - 1) & 1))) {
              tc::tc_fence_after();
              const uint32_t kb = tc::smem_u32(s_k + st * kAtKBytes);
#pragma unroll
              for (int kstep = 0; kstep < 32; ++kstep) {
                const uint32_t off = (uint32_t)((kstep >> 2) * kAtRegion + (kstep & 3) * 32);
                tc::mma_bf16_ts(tmem + sb * kAtKT, tmem + kTmQ + kstep * 8, tc::sdesc_sw128(kb + off, 16, 1024),
                                idesc_s, kstep > 0 ? 1u : 0u);
              }
              tc::mma_commit(s_full + sb);
              if (next_s == x.n_tiles - 1) tc::mma_commit(s_done);
              ++next_s;
              did = true;
            }
          }
          if (next_pv < next_s) {
            // PV(n): O[:, 256 half .. +255] += P V for both halves.  The first PV
            // of an item overwrites O, so each half waits for the previous
            // item's epilogue to have read that half (o_free[half]).
            const int gp = tcount + next_pv, sp = slot + next_pv;
            const int st = sp % kAtStages, sb = gp & 1;
            const bool first = next_pv == 0 && ni > 0;
            if ((pv_half > 0 || tc::mbar_try_wait(p_full + sb, (gp >> 1) & 1)) &&
                (!first || tc::mbar_try_wait(o_free + pv_half, (ni - 1) & 1))) {
              tc::tc_fence_after();
              const uint32_t pb = tc::smem_u32(s_p + sb * kAtPBytes);
              const uint32_t kb = tc::smem_u32(s_k + st * kAtKBytes);
              const int h_end = first && pv_half == 0 ? 1 : 2;   // a first PV goes one half at a time
#pragma unroll
              for (int half = 0; half < 2; ++half) {
                if (half < pv_half || half >= h_end) continue;  // unrolled: the issuing thread's hot loop
#pragma unroll
                for (int kstep = 0; kstep < kAtKT / 16; ++kstep) {
                  const uint64_t ad = tc::sdesc_sw128(pb + kstep * 32, 16, 1024);
                  const uint64_t bd = tc::sdesc_sw128(kb + half * 4 * kAtRegion + kstep * 2048, kAtRegion, 1024);
                  tc::mma_bf16_ss(tmem + kTmO + half * 256, ad, bd, idesc_o, (next_pv > 0 || kstep > 0) ? 1u : 0u);
                }
              }
              pv_half = h_end;
              if (pv_half == 2) {
                tc::mma_commit(kv_empty + st);
                tc::mma_commit(pv_done + sb);
                ++next_pv;
                pv_half = 0;
              }
              did = true;
            }
          }
          if (did) {
            t_idle = 0;
          } else if (*abort_flag) {
            ok = false;
            break;
          } else {
            const uint64_t now = tc::globaltimer();
            if (t_idle == 0) t_idle = now;
            else if (now - t_idle > limit_ns) { report(LCSA_DEV_TIMEOUT); ok = false; break; }
          }
        }
        slot += x.n_tiles;
        tcount += x.n_tiles;
        ++ni;
      }
      if (!ok) *abort_flag = 1;
    }
  } else if (warp < kAtXtWarp0) {
    // ============================================================ softmax
    // Every head row h of this warp's 16-lane block is split over two threads:
    // thread (h % 16) takes keys 0-31 of each tile, thread (h % 16) + 16 keys
    // 32-63 (16x32bx2 TMEM accesses).  Row maxima and sums meet through one
    // shuffle; the item's row statistics go to the epilogue through shared
    // memory.
    const int quarter = warp & 3;
    const int half = lane >> 4;                       // 0: keys 0-31 / O dims 0-255, 1: keys 32-63 / dims 256-511
    const int h = quarter * 16 + (lane & 15);         // head row
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    bool ok = true;
    int tcount = 0, ni = 0;
    int nc_next = at_item_nc(g, P, blockIdx.x);
    for (int it = blockIdx.x; it < g.n_items; it += G) {
      const int nc_cur = nc_next;
      nc_next = at_item_nc(g, P, it + G);
      const AtItem x = at_item(g, it, nc_cur);
      if (x.n_tiles == 0) continue;
      float m_run = -INFINITY, l_run = 0.f;           // l_run: this thread's half of the row sum
      for (int n = 0; n < x.n_tiles; ++n) {
        const int ga = tcount + n;                    // tile count over all items of this CTA
        const int sb = ga & 1;
        // warp-uniform exit: the shuffles and TMEM accesses below need all 32 lanes
        const bool good = ok && !*abort_flag && tc::mbar_wait(s_full + sb, (ga >> 1) & 1);
        if (!__all_sync(0xffffffffu, good)) { ok = false; break; }
        tc::tc_fence_after();
        uint32_t v[32];
        tc::tmem_ld_16x32bx2_x32<32>(tmem + lane_base + sb * kAtKT, v);
        tc::tmem_wait_ld();
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(s_free + sb);
        const int gt = x.t0 + n;
        int nvalid = gt < x.ks.tiles_c ? x.ks.n_c - gt * kAtKT : x.ks.n_w - (gt - x.ks.tiles_c) * kAtKT;
        nvalid = (nvalid < kAtKT ? nvalid : kAtKT) - 32 * half;   // valid keys among this thread's 32
        uint32_t km = nvalid >= 32 ? 0xffffffffu : (nvalid <= 0 ? 0u : (1u << nvalid) - 1u);
        if (g.sparse && gt < x.ks.tiles_c) {
          // gathered tile: the producers' row mask of its stage (slot = ga + ni + 1, one Q
          // slot per item before its tiles); the stage's fill completed before S, so this
          // wait returns at once and orders the mask's reads after the producers' writes
          const int sl = ga + ni + 1;
          if (!tc::mbar_wait(kv_full + sl % kAtStages, (sl / kAtStages) & 1)) ok = false;
          km &= s_km[(sl % kAtStages) * 2 + half];
        }
        float tmax = -INFINITY;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float s = (km >> j) & 1u ? __uint_as_float(v[j]) : -INFINITY;
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
          if (!tc::mbar_wait(pv_done + ((ga - 1) & 1), ((ga - 1) >> 1) & 1)) ok = false;
          tc::tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < 256; c += 16) {
            uint32_t r[16];
            tc::tmem_ld_16x32bx2_x16<256>(tmem + lane_base + kTmO + c, r);
            tc::tmem_wait_ld();
#pragma unroll
            for (int q2 = 0; q2 < 16; ++q2) r[q2] = __float_as_uint(__uint_as_float(r[q2]) * alpha);
            tc::tmem_st_16x32bx2_x16<256>(tmem + lane_base + kTmO + c, r);
          }
          tc::tmem_wait_st();
        }
        l_run *= alpha;
        // P buffer sb is free once the PV two tiles back is done
        if (ga >= 2 && !tc::mbar_wait(pv_done + sb, ((ga - 2) >> 1) & 1)) ok = false;
        {
          float psum = 0.f;
          uint8_t* prow = s_p + sb * kAtPBytes + h * 128;
          const float neg_m = m_run == -INFINITY ? 0.f : -m_run;   // no valid key yet: every p is 0
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
            const int chunk = half * 4 + c;           // keys 8*chunk .. 8*chunk+7
            *reinterpret_cast<uint4*>(prow + ((chunk ^ (h & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
          l_run += psum;
        }
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(p_full + sb);
      }
      const float l_row = l_run + __shfl_xor_sync(0xffffffffu, l_run, 16);
      if (half == 0) s_stats[(ni & 1) * 64 + h] = make_float2(m_run, l_row);
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(stats_full + (ni & 1));
      tcount += x.n_tiles;
      ++ni;
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
    }
    if (!ok) *abort_flag = 1;
  } else {
    // ============================================================ transitions
    // Per item: Q -> TMEM once the previous item's S MMAs have completed,
    // then the previous item's epilogue.  The four warps share named barrier
    // 2 and leave only together.
    const int quarter = warp & 3;
    const int half = lane >> 4;                       // Q dims / O dims 256*half .. +255
    const int h = quarter * 16 + (lane & 15);         // head row
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const int xt = threadIdx.x - kAtXtWarp0 * 32;     // 0..127
    bool ok = true;
    int slot = 0, tcount = 0, ni = 0;
    // the previous item, whose epilogue follows the next item's Q move
    bool pend = false;
    long long p_row = 0;
    int p_split = 0, p_last = 0;
    int nc_next = at_item_nc(g, P, blockIdx.x);
    for (int it = blockIdx.x; it < g.n_items; it += G) {
      const int nc_cur = nc_next;
      nc_next = at_item_nc(g, P, it + G);
      const AtItem x = at_item(g, it, nc_cur);
      if (x.n_tiles == 0) {
        at_store_empty(g, P, x, xt);
        continue;
      }
      const int qslot = slot++;
      const int qst = qslot % kAtStages;
      ok = tc::bar_and(2, kAtGroupThreads, ok);       // the previous epilogue is done with s_cs_item
      if (!ok) break;
      // Q is staged, and every S MMA of the previous item (the readers of Q's
      // TMEM columns) has completed.
      if (!tc::mbar_wait(q_full + (ni & 1), (ni >> 1) & 1)) ok = false;
      if (ni > 0 && !tc::mbar_wait(s_done, (ni - 1) & 1)) ok = false;
      tc::tc_fence_after();
      if (xt < 32) s_cs_item[(ni & 1) * 32 + xt] = s_cs[qst * 32 + xt];
      at_q_to_tmem(s_k + qst * kAtKBytes, s_cs + qst * 32, tmem + lane_base + kTmQ, h, half);
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(q_ready);
      ok = tc::bar_and(2, kAtGroupThreads, ok);       // every thread is done reading the Q stage
      if (!ok) break;
      if (xt == 0) tc::mbar_arrive(kv_empty + qst);   // the stage returns to the producers
      if (pend)
        ok = at_epilogue(g, P, pv_done, o_free, stats_full, s_stats, ni - 1, s_cs_item + ((ni - 1) & 1) * 32,
                         p_row, p_split, p_last, tmem, lane_base, h, half, xt, ok);
      pend = true;
      p_row = x.row;
      p_split = x.split;
      p_last = tcount + x.n_tiles - 1;
      slot += x.n_tiles;
      tcount += x.n_tiles;
      ++ni;
    }
    if (pend) {
      ok = tc::bar_and(2, kAtGroupThreads, ok);
      if (ok)
        ok = at_epilogue(g, P, pv_done, o_free, stats_full, s_stats, ni - 1, s_cs_item + ((ni - 1) & 1) * 32,
                         p_row, p_split, p_last, tmem, lane_base, h, half, xt, ok);
    }
    if (!ok) *abort_flag = 1;
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

// Per-call preparation: the valid prefix length of each CSA selection row
// (rows are ascending with -1 padding at the end) and the (cos, sin) row of
// every query position (angle in FP64).
__global__ void __launch_bounds__(256)
attn_prep_kernel(const int32_t* __restrict__ idx, int k, long long rows, int32_t* __restrict__ nc,
                 float2* __restrict__ cs, long long n_cs, long long q_pos0, double log_base) {
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx != nullptr && gid < rows) {
    const int32_t* r = idx + gid * k;
    int lo = 0, hi = k;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (r[mid] >= 0) lo = mid + 1; else hi = mid;
    }
    nc[gid] = lo;
  }
  if (gid < n_cs) {
    float c, s;
    rope_cs(q_pos0 + (gid >> 5), (int)(gid & 31), kRopeR, log_base, &c, &s);
    cs[gid] = make_float2(c, s);
  }
}

// ------------------------------------------------------------------ host side
struct AtPlan {
  int splits;
  int rot_slot;
  size_t off_rot_c, off_rot_w, off_nc, off_cs, off_opart, off_ml, total;
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
  // Few rows (decode): split each row's key range.  The split count s (>= 4
  // tiles per split) minimises, in units of one 64-key tile (~1.4 us), the
  // persistent CTAs' rounds x (tiles per item + ~1 tile of per-item cost)
  // plus the partial-output traffic of the combine (s x rows x 256 KB written
  // and read at ~6 TB/s).
  int splits = 1;
  const int sms = sm_count();
  if (rows < 2 * sms) {
    const int cap = max_tiles / 4 > 1 ? max_tiles / 4 : 1;
    double best = -1.0;
    for (int s = 1; s <= cap; ++s) {
      const long long rounds = (rows * s + sms - 1) / sms;
      const double cost = (double)rounds * (double)((max_tiles + s - 1) / s + 1) +
                          (s > 1 ? (double)s * (double)rows * 262144.0 / 6.0e6 / 1.4 : 0.0);
      if (best < 0.0 || cost < best) { best = cost; splits = s; }
    }
  }
  // An item stages at most kAtMaxIdx selected entries: larger k needs more key-range splits.
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
  p.off_nc = off;
  if (sparse) off += al((size_t)rows * 4);
  p.off_cs = off;
  off += al((size_t)a->Tq * kAtCsBytes);
  p.off_opart = off;
  if (splits > 1) off += al((size_t)splits * rows * 64 * 512 * 4);
  p.off_ml = off;
  if (splits > 1) off += al((size_t)splits * rows * 128 * 4);
  p.total = off + 256;
  return p;
}

static size_t attn_tc_workspace(const lcsa_attn_args* a, int sparse) { return attn_tc_plan(a, sparse).total; }

// How BF16 CSA tiles gather their selected rows: 0 = 16-byte cp.async by all
// producer warps (default), 1 = TMA tile::gather4.
inline std::atomic<int>& attn_gather_mode() {
  static std::atomic<int> m{0};
  return m;
}

// f8 != null: the entries come from the FP8 cache (a->ckv is not read).
static cudaError_t launch_attn_tc(const lcsa_attn_args* a, int sparse, void* ws, cudaStream_t st,
                                  const lcsa_fp8_entries* f8 = nullptr) {
  const AtPlan pl = attn_tc_plan(a, sparse);
  uint8_t* w = reinterpret_cast<uint8_t*>(ws);
  const double log_base = log(a->rope_base > 0.f ? (double)a->rope_base : 10000.0);
  const long long rows = (long long)a->B * a->Tq;
  // int32 item indices and TMA row coordinates
  if (rows * pl.splits * 64 > (long long)INT32_MAX - 64 * 1024) return cudaErrorInvalidValue;
  const bool g4 = sparse && f8 == nullptr && attn_gather_mode().load() == 1;
  // TMA-gathered rows: entry and rotary-slice row coordinates, and the row
  // past the end that absent rows read, are int32
  if (g4 && ((long long)a->B * a->Nc >= (long long)INT32_MAX || (pl.rot_slot && rows * a->k >= (long long)INT32_MAX)))
    return cudaErrorInvalidValue;
  AtPtrs P;
  P.ckv = (const __nv_bfloat16*)a->ckv;
  P.c8 = f8 ? f8->codes : nullptr;
  P.c8s = f8 ? f8->scales : nullptr;
  P.idx = sparse ? a->idx : nullptr;
  P.nc = (const int32_t*)(w + pl.off_nc);
  P.cs = (const float2*)(w + pl.off_cs);
  P.rot_c = (const __nv_bfloat16*)(w + pl.off_rot_c);
  P.rot_w = (const __nv_bfloat16*)(w + pl.off_rot_w);
  P.sink = a->sink;
  P.out = a->out;
  P.lse = a->lse;
  P.o_part = (float*)(w + pl.off_opart);
  P.ml_part = (float*)(w + pl.off_ml);
  cudaError_t e;
  // rotary slices of the keys (from the entries, or from the FP8 cache's BF16 rotary dims)
  if (a->Nc > 0) {
    const void* rsrc = f8 ? f8->rope : a->ckv;
    const int rld = f8 ? kRopeR : 512;
    if (pl.rot_slot)
      e = launch_rope_rows(rsrc, w + pl.off_rot_c, rows * a->k, rld, 1, 0, a->m, log_base, 1, a->idx,
                           (long long)a->Tq * a->k, a->Nc, st);
    else
      e = launch_rope_rows(rsrc, w + pl.off_rot_c, (long long)a->B * a->Nc, rld, a->Nc, 0, a->m, log_base, 0,
                           nullptr, 0, a->Nc, st);
    if (e != cudaSuccess) return e;
  }
  if (a->Tkv > 0 && a->W > 0) {
    e = launch_rope_rows(a->kv, w + pl.off_rot_w, (long long)a->B * a->Tkv, 512, a->Tkv, a->kv_pos0, 1, log_base, 0,
                         nullptr, 0, 0, st);
    if (e != cudaSuccess) return e;
  }
  {
    const long long n_cs = (long long)a->Tq * 32;
    const long long n = sparse && rows > n_cs ? rows : n_cs;
    count_launch();
    attn_prep_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(sparse ? a->idx : nullptr, a->k, rows,
                                                                  (int32_t*)(w + pl.off_nc), (float2*)(w + pl.off_cs),
                                                                  n_cs, a->q_pos0, log_base);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  AtGeom g;
  g.B = a->B; g.Tq = a->Tq; g.Nc = a->Nc; g.k = sparse ? a->k : 0; g.Tkv = a->Tkv;
  g.rows = rows;
  g.q_pos0 = a->q_pos0; g.kv_pos0 = a->kv_pos0; g.m = a->m; g.W = a->W;
  const float scale = a->softmax_scale > 0.f ? a->softmax_scale : 1.0f / sqrtf(512.f);
  g.scale_log2 = scale * kLog2e;
  g.sparse = sparse;
  g.rot_slot = pl.rot_slot;
  g.splits = pl.splits;
  g.out_bf16 = a->out_dtype == LCSA_BF16;
  g.out_v8 = (reinterpret_cast<uintptr_t>(pl.splits > 1 ? (const void*)P.o_part : a->out) & 31u) == 0 ? 1 : 0;
  g.n_items = (int)(rows * pl.splits);
  g.fp8 = f8 != nullptr;
  auto kern = g.fp8 ? attn_tc_kernel<true, false> : g4 ? attn_tc_kernel<false, true> : attn_tc_kernel<false, false>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kAtSmem);
  if (e != cudaSuccess) return e;
  // Tensor maps (128-byte swizzle): 64-row boxes, except the entry and
  // rotary-slice maps of TMA-gathered CSA, which read one row per box row.
  // A map whose tensor is absent is never read; it points at q instead.
  CUtensorMap m_q, m_ckv, m_kv, m_rotc, m_rotw;
  const uint64_t rows_rotc = pl.rot_slot ? (uint64_t)rows * a->k : (uint64_t)a->B * a->Nc;
  const uint32_t box_c = g4 ? 1 : 64;
  auto mk = [&](CUtensorMap* m, const void* base, uint64_t nrows, uint64_t cols, uint32_t box_rows) {
    if (base == nullptr || nrows == 0) return make_tmap_bf16_2d(m, a->q, (uint64_t)rows * 64, 512, 512, 64, box_rows);
    return make_tmap_bf16_2d(m, base, nrows, cols, cols, 64, box_rows);
  };
  bool okm = mk(&m_q, a->q, (uint64_t)rows * 64, 512, 64) &&
             mk(&m_ckv, (a->Nc > 0 && !f8) ? a->ckv : nullptr, (uint64_t)a->B * a->Nc, 512, box_c) &&
             mk(&m_kv, a->Tkv > 0 ? a->kv : nullptr, (uint64_t)a->B * a->Tkv, 512, 64) &&
             mk(&m_rotc, a->Nc > 0 ? (const void*)P.rot_c : nullptr, rows_rotc, 64, box_c) &&
             mk(&m_rotw, (a->Tkv > 0 && a->W > 0) ? (const void*)P.rot_w : nullptr, (uint64_t)a->B * a->Tkv, 64,
                64);
  if (!okm) return cudaErrorInvalidValue;
  const int grid = g.n_items < sm_count() ? g.n_items : sm_count();
  kern<<<grid, kAtThreads, kAtSmem, st>>>(P, g, m_q, m_ckv, m_kv, m_rotc, m_rotw);
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
