// Lightning-Indexer scores on the FP4 QK path (DeepSeek-V4 "FP4
// Quantization-Aware Training": the indexer computes its query-key scores in
// FP4; CSA Step 2 "Select": the Lightning Indexer runs in FP4 precision).
// H_I = 64, D_I = 128.
//
// The indexer keys live in HBM as MXFP4 (64 bytes of E2M1 codes + 4 scale
// bytes per entry, a quarter of BF16), which is what bounds long-context
// decode: every decode step streams all of them.  Per 128-entry tile:
//   TMA        packed codes -> shared memory (8-deep ring)
//   dequant    8 warps, two per tile (4 tiles in flight, 8 stages), write E4M3 in the
//              128B-swizzled K-major layout, each entry relative to its
//              largest block exponent (exact for blocks within 2^13 of it,
//              see mxfp4.cuh)
//   MMA        tcgen05 kind::f8f6f4, M = 128 entries, N = 64 heads x up to 4
//              query rows (E4M3 queries prepared by indexer_q8_kernel), K = 128
//   accumulators  512 TMEM columns split into 2-8 slots (64 x query rows
//              columns each), so the MMA runs up to 8 tiles ahead of the epilogue
//   epilogue   8 warps: w relu(x) formed as (w/2) x + (w/2) |x| on the FMA
//              pipe (the prepared head weights carry the query factors and
//              the 1/2), times the entry factor 2^(Xref - 6), one score per lane;
//              with 3-4 query rows each warp scores 2 rows of every tile,
//              with 1-2 rows the two warps of a lane quarter take alternate
//              tiles (one accumulator each).
// Warp roles (576 threads): 0 TMA producer, 1 TMEM allocator + MMA issuer,
// 2-9 epilogue, 10-17 dequantisers.  Every wait is bounded (tc::mbar_wait, or
// the non-suspending tc::mbar_wait_spin for the single-thread MMA issuer);
// on expiry the CTA stops, records LCSA_DEV_TIMEOUT, drains its in-flight
// copies and frees TMEM.
#pragma once
#include "tc_ptx.cuh"
#include "mxfp4.cuh"
#include "indexer_tc.cuh"

namespace lcsa {

constexpr int kI4CStages = 8;                  // packed-code ring
constexpr int kI4DqWarp0 = 10;
constexpr int kI4DqWarps = 8;                  // warps 2t, 2t+1 of the group expand tiles t, t+4, t+8, ...
constexpr int kI4Pairs = kI4DqWarps / 2;       // tiles being expanded at once
constexpr int kI4AStages = 2 * kI4Pairs;       // E4M3 key tiles: two per pair, so a pair never waits for the
                                               // MMA of the tile it just handed over
constexpr int kI4Threads = (kI4DqWarp0 + kI4DqWarps) * 32;   // 576
constexpr uint32_t kI4QBytes = 256 * 128;      // 4 query rows x 64 heads x 128 E4M3
constexpr uint32_t kI4ABytes = kIxTileE * 128; // 128 entries x 128 E4M3
constexpr uint32_t kI4CBytes = kIxTileE * 64;  // 128 entries x 64 code bytes
constexpr int kI4MaxAcc = 8;                   // TMEM accumulator slots (512 / (64 x query rows), up to 8)
constexpr int kI4Bars = 1 + 2 * kI4CStages + 2 * kI4AStages + 2 * kI4MaxAcc;
constexpr size_t kI4Smem = 1024 + kI4QBytes + kI4AStages * kI4ABytes + kI4CStages * kI4CBytes + kIxRows * 64 * 4 +
                           kI4Bars * 8;
static_assert(kI4Smem + 64 <= 232448, "shared memory of the FP4 indexer kernel");
// Piece order of the dequantisers: the lane of row r handles code block
// p = kI4Perm[(r >> 1) & 3] ^ i at step i, so that both the 64-byte-strided
// code reads and the swizzled 16-byte writes of 8 consecutive rows hit 8
// different bank groups (p -> kI4Perm[p] is multiplication by a primitive
// element of GF(4), so kI4Perm[k] and kI4Perm[k] ^ k are both permutations).
__device__ __constant__ int kI4Perm[4] = {0, 2, 3, 1};

// Instruction descriptor for kind::f8f6f4 with E4M3 A/B (format 0) and FP32 D.
__host__ __device__ __forceinline__ uint32_t idesc_e4m3(int M, int N) {
  uint32_t d = 0;
  d |= 1u << 4;
  d |= (uint32_t)((N >> 3) & 0x3F) << 17;
  d |= (uint32_t)((M >> 4) & 0x1F) << 24;
  return d;
}
__device__ __forceinline__ void mma_e4m3_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ int max_scale_byte(uint32_t sw) {
  const uint32_t a = max(sw & 0xFFu, (sw >> 8) & 0xFFu), b = max((sw >> 16) & 0xFFu, sw >> 24);
  return (int)max(a, b);
}

__global__ void __launch_bounds__(kI4Threads, 1)
indexer_fp4_kernel(const __grid_constant__ CUtensorMap q_map, const __grid_constant__ CUtensorMap c_map,
                   const uint32_t* __restrict__ k_scales, const float* __restrict__ w8,
                   float* __restrict__ scores, IxGeom g) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* s_q = smem;
  uint8_t* s_a = s_q + kI4QBytes;
  uint8_t* s_c = s_a + kI4AStages * kI4ABytes;
  float* s_w = reinterpret_cast<float*>(s_c + kI4CStages * kI4CBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(s_w + kIxRows * 64);
  uint64_t* q_full = bars;
  uint64_t* c_full = bars + 1;
  uint64_t* c_empty = c_full + kI4CStages;
  uint64_t* a_full = c_empty + kI4CStages;
  uint64_t* a_empty = a_full + kI4AStages;
  uint64_t* acc_full = a_empty + kI4AStages;
  uint64_t* acc_empty = acc_full + kI4MaxAcc;
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- work unit (as indexer_tc_kernel: heaviest query groups first)
  const int n_groups = g.nb * g.gps;
  const int grp = n_groups - 1 - (int)blockIdx.x;
  const int split = blockIdx.y;
  const int bl = grp / g.gps;
  const int b = g.b0 + bl;
  const int gi = grp - bl * g.gps;
  const int i_first = g.i0 + gi * kIxRows;
  int rows = g.i0 + g.ni - i_first;
  rows = rows < kIxRows ? rows : kIxRows;
  long long nv = (g.q_pos0 + i_first + rows - 1) / g.m;
  if (nv > g.Nc) nv = g.Nc;
  const int tiles_all = (int)((nv + kIxTileE - 1) / kIxTileE);
  const int per_split = (tiles_all + g.splits - 1) / g.splits;
  const int t_begin = split * per_split;
  int t_end = t_begin + per_split;
  t_end = t_end < tiles_all ? t_end : tiles_all;
  const int n_tiles = t_end > t_begin ? t_end - t_begin : 0;
  if (n_tiles == 0) return;
  const long long rect_row = (long long)bl * g.ni + (i_first - g.i0);   // first query row in the rectangle
  // TMEM accumulator slots: 64 x rows columns each, as many as fit in 512 (8, 4 or 2);
  // with 1-2 rows the epilogue halves take alternate tiles, so every slot stays with one half
  const int n_acc = rows == 1 ? 8 : rows == 2 ? 4 : 2;
  const uint32_t acc_cols = 512u / (uint32_t)n_acc;

  if (threadIdx.x == 0) {
    tc::mbar_init(q_full, 1);
    for (int s = 0; s < kI4CStages; ++s) { tc::mbar_init(c_full + s, 1); tc::mbar_init(c_empty + s, 2); }
    for (int s = 0; s < kI4AStages; ++s) { tc::mbar_init(a_full + s, 2); tc::mbar_init(a_empty + s, 1); }
    // rows > 2: all 8 epilogue warps read every accumulator; else 4 per accumulator
    for (int a = 0; a < kI4MaxAcc; ++a) {
      tc::mbar_init(acc_full + a, 1);
      tc::mbar_init(acc_empty + a, rows > 2 ? 8 : 4);
    }
    tc::fence_barrier_init();
    s_abort = 0;
  }
  if (warp == 1) { tc::tmem_alloc(&s_tmem, 512); tc::tmem_relinquish(); }
  for (int e = threadIdx.x; e < kIxRows * 64; e += kI4Threads) {
    const int q = e >> 6;
    s_w[e] = q < rows ? w8[(rect_row + q) * 64 + (e & 63)] : 0.f;
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = s_tmem;
  volatile int* abort_flag = &s_abort;
  const long long ent0 = (long long)b * g.Nc;          // first entry row of this sequence

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (tc::elect_one()) {
      tc::prefetch_tmap(&q_map);
      tc::prefetch_tmap(&c_map);
      tc::mbar_arrive_expect_tx(q_full, kI4QBytes);
      tc::tma_load_2d(s_q, &q_map, q_full, 0, (int)(rect_row * 64));
      int issued = 0;
      for (int n = 0; n < n_tiles; ++n) {
        const int s = n % kI4CStages, r = n / kI4CStages;
        if (r > 0 && !tc::mbar_wait(c_empty + s, (r - 1) & 1)) { *abort_flag = 1; break; }
        if (*abort_flag) break;
        tc::mbar_arrive_expect_tx(c_full + s, kI4CBytes);
        tc::tma_load_2d(s_c + s * kI4CBytes, &c_map, c_full + s, 0,
                        (int)(ent0 + (long long)(t_begin + n) * kIxTileE));
        ++issued;
      }
      for (int n = issued - kI4CStages > 0 ? issued - kI4CStages : 0; n < issued; ++n)
        tc::mbar_wait(c_full + n % kI4CStages, (n / kI4CStages) & 1);
      tc::mbar_wait(q_full, 0);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (tc::elect_one()) {
      const uint32_t idesc = idesc_e4m3(128, 64 * rows);
      bool ok = tc::mbar_wait(q_full, 0);
      const uint32_t b_base = tc::smem_u32(s_q);
      for (int n = 0; ok && n < n_tiles; ++n) {
        const int s = n % kI4AStages, r = n / kI4AStages;
        const int a = n % n_acc, ra = n / n_acc;
        if (*abort_flag) break;
        if (!tc::mbar_wait_spin(a_full + s, r & 1)) { ok = false; break; }
        if (ra > 0 && !tc::mbar_wait_spin(acc_empty + a, (ra - 1) & 1)) { ok = false; break; }
        tc::tc_fence_after();
        const uint32_t a_base = tc::smem_u32(s_a + s * kI4ABytes);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint64_t ad = tc::sdesc_sw128(a_base + ks * 32, 16, 1024);
          const uint64_t bd = tc::sdesc_sw128(b_base + ks * 32, 16, 1024);
          mma_e4m3_ss(tmem + (uint32_t)a * acc_cols, ad, bd, idesc, ks > 0 ? 1u : 0u);
        }
        tc::mma_commit(a_empty + s);
        tc::mma_commit(acc_full + a);
      }
      if (!ok) *abort_flag = 1;
    }
  } else if (warp < kI4DqWarp0) {
    // ------------------------------------------------------------ epilogue
    const int e = warp - 2;                 // 0..7
    const int quarter = warp & 3;           // TMEM lanes [32*quarter, 32*quarter+32)
    const int half = e >> 2;                // query rows {2*half, 2*half+1}
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
    // rows > 2: rows {2 half, 2 half + 1} of every tile; rows <= 2: every row
    // of the tiles n with n % 2 == half (accumulator `half`)
    const bool by_tile = rows <= 2;                      // CTA-uniform
    const int n_q = by_tile ? rows : min(2, max(0, rows - 2 * half));
    const int q0 = by_tile ? 0 : 2 * half;
    const int n_first = by_tile ? half : 0, n_step = by_tile ? 2 : 1;
    auto scale_word = [&](int n) -> uint32_t {           // this lane's entry of tile n
      const long long j = (long long)(t_begin + n) * kIxTileE + quarter * 32 + lane;
      return n < n_tiles && j < g.Nc ? __ldg(k_scales + ent0 + j) : 0x7F7F7F7Fu;
    };
    // scale words of the next three tiles this warp scores
    uint32_t sw1 = scale_word(n_first), sw2 = scale_word(n_first + n_step), sw3 = scale_word(n_first + 2 * n_step);
    for (int n = n_first; n_q > 0 && n < n_tiles; n += n_step) {
      const int a = n % n_acc, ra = n / n_acc;
      const long long j = (long long)(t_begin + n) * kIxTileE + quarter * 32 + lane;
      const uint32_t sw = sw1;
      sw1 = sw2; sw2 = sw3; sw3 = scale_word(n + 3 * n_step);
      // waits end on the same decision in every lane (a split warp would stall at the warp syncs)
      bool ok = !*abort_flag && tc::mbar_wait(acc_full + a, ra & 1);
      if (!__all_sync(0xffffffffu, ok)) { *abort_flag = 1; break; }
      tc::tc_fence_after();
      float sc[2] = {0.f, 0.f};
#pragma unroll
      for (int qq = 0; qq < 2; ++qq) {
        if (qq < n_q) {
          const uint32_t col = tmem + lane_addr + (uint32_t)a * acc_cols + (uint32_t)((q0 + qq) * 64);
          const uint32_t wq = tc::smem_u32(s_w + (q0 + qq) * 64);
          // w relu(x) = (w/2) x + (w/2) |x| on the FMA pipe (the prepared weights
          // carry the 1/2); eight partial sums: heads h = 4i + c, x and |x| terms
          float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int hb = 0; hb < 64; hb += 32) {     // 32 heads at a time
            uint32_t v[32];
            tc::tmem_ld32(col + hb, v);
            tc::tmem_wait_ld();
            if (qq == n_q - 1 && hb == 32) {       // accumulator read out: hand it back to the MMA warp
              tc::tc_fence_before();
              __syncwarp();
              if (lane == 0) tc::mbar_arrive(acc_empty + a);
            }
#pragma unroll
            for (int h = 0; h < 32; h += 4) {
              const float4 w4 = tc::lds128f(wq + (hb + h) * 4);
              const float x0 = __uint_as_float(v[h]), x1 = __uint_as_float(v[h + 1]);
              const float x2 = __uint_as_float(v[h + 2]), x3 = __uint_as_float(v[h + 3]);
              acc[0] = fmaf(w4.x, x0, acc[0]); acc[4] = fmaf(w4.x, fabsf(x0), acc[4]);
              acc[1] = fmaf(w4.y, x1, acc[1]); acc[5] = fmaf(w4.y, fabsf(x1), acc[5]);
              acc[2] = fmaf(w4.z, x2, acc[2]); acc[6] = fmaf(w4.z, fabsf(x2), acc[6]);
              acc[3] = fmaf(w4.w, x3, acc[3]); acc[7] = fmaf(w4.w, fabsf(x3), acc[7]);
            }
          }
          sc[qq] = ((acc[0] + acc[4]) + (acc[1] + acc[5])) + ((acc[2] + acc[6]) + (acc[3] + acc[7]));
        }
      }
      const float f = pow2f(max_scale_byte(sw) - 127 - 6);
      if (j < g.Nc) {
#pragma unroll
        for (int qq = 0; qq < 2; ++qq)
          if (qq < n_q) scores[(rect_row + q0 + qq) * g.Nc + j] = sc[qq] * f;
      }
    }
  } else {
    // ------------------------------------------------------------ dequantisers
    // warps 2t and 2t+1 of the group expand tiles n = t, t + 4, ... into E4M3
    // stage n % 8; the lane of warp 2t + hh handles entry rows lane + 32 (2 hh + jr)
    const int dq = (warp - kI4DqWarp0) >> 1, hh = (warp - kI4DqWarp0) & 1;
    const int pb = kI4Perm[(lane >> 1) & 3];
    // per-lane constants: step i reads code block p = pb ^ i at byte offset
    // (pb ^ i) * 16 of the row and writes its two 16-byte E4M3 chunks 2p, 2p+1
    // at swizzled offsets ((2p + h) ^ (row & 7)) * 16 = st_base ^ (32 i) ^ (16 h)
    const uint32_t ld_base = (uint32_t)pb << 4;
    const uint32_t st_base = ((uint32_t)(2 * pb) ^ (uint32_t)(lane & 7)) << 4;
    // byte i of prmt(w, 0, psel) = scale byte of block pb ^ i
    const uint32_t psel = (uint32_t)pb | ((uint32_t)(pb ^ 1) << 4) | ((uint32_t)(pb ^ 2) << 8) | ((uint32_t)(pb ^ 3) << 12);
    auto scale_words = [&](int n, uint32_t* sw) {
#pragma unroll
      for (int jr = 0; jr < 2; ++jr) {
        const long long j = (long long)(t_begin + n) * kIxTileE + lane + 32 * (2 * hh + jr);
        sw[jr] = n < n_tiles && j < g.Nc ? __ldg(k_scales + ent0 + j) : 0x7F7F7F7Fu;
      }
    };
    uint32_t cur[2], nxt[2];                    // this warp's next two tiles
    scale_words(dq, cur);
    scale_words(dq + kI4Pairs, nxt);
    for (int n = dq; n < n_tiles; n += kI4Pairs) {
      const int cs = n % kI4CStages, rc = n / kI4CStages;
      const int as = n % kI4AStages, ra = n / kI4AStages;
      uint32_t sw[2];
#pragma unroll
      for (int jr = 0; jr < 2; ++jr) { sw[jr] = cur[jr]; cur[jr] = nxt[jr]; }
      scale_words(n + 2 * kI4Pairs, nxt);
      bool ok = !*abort_flag && tc::mbar_wait(c_full + cs, rc & 1);
      ok = ok && (ra == 0 || tc::mbar_wait(a_empty + as, (ra - 1) & 1));
      if (!__all_sync(0xffffffffu, ok)) { *abort_flag = 1; break; }
#pragma unroll
      for (int jr = 0; jr < 2; ++jr) {
        const int r = lane + 32 * (2 * hh + jr);
        const uint32_t w = sw[jr];
        const uint32_t xref = (uint32_t)max_scale_byte(w);
        const uint32_t src = tc::smem_u32(s_c) + cs * kI4CBytes + r * 64;      // 64-byte aligned
        const uint32_t dst = tc::smem_u32(s_a) + as * kI4ABytes + r * 128;     // 128-byte aligned
        uint4 c[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) c[i] = tc::lds128(src | (ld_base ^ (uint32_t)(16 * i)));
        // byte i of dl: xref - (scale byte of block pb ^ i), never borrowing
        const uint32_t dl = xref * 0x01010101u - __byte_perm(w, 0, psel);
        // every block within 2^11 of the entry's largest: table by exponent-field arithmetic
        const bool fast = ((dl | (dl + 0x04040404u)) & 0xF0F0F0F0u) == 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t d = (dl >> (8 * i)) & 0xFFu;
          uint32_t lo, hi;
          if (fast) {
            lo = 0x6C686000u - d * 0x08080800u;
            hi = 0x7C787470u - d * 0x08080808u;
          } else {
            e4m3_table(6 - (int)d, lo, hi);
          }
          const uint2 e0 = e2m1x8_to_e4m3(c[i].x, lo, hi), e1 = e2m1x8_to_e4m3(c[i].y, lo, hi);
          const uint2 e2 = e2m1x8_to_e4m3(c[i].z, lo, hi), e3 = e2m1x8_to_e4m3(c[i].w, lo, hi);
          const uint32_t o = st_base ^ (uint32_t)(32 * i);
          tc::sts128(dst | o, make_uint4(e0.x, e0.y, e1.x, e1.y));
          tc::sts128(dst | (o ^ 16u), make_uint4(e2.x, e2.y, e3.x, e3.y));
        }
      }
      tc::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) { tc::mbar_arrive(c_empty + cs); tc::mbar_arrive(a_full + as); }
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// Block-scaled variant for query groups of one or two rows (decode), taken
// when lcsa_set_fp4_mma(1) asks for it: the codes go to the tensor cores as
// they are, exact for any spread of block scales.  On B200 it is not the
// faster one: 67.7 us against 65.5 us for the staging kernel on 8 sequences
// x 262144 entries (ALU pipe 15 % busy instead of 55 %, tensor pipe 12 %,
// DRAM 27 %), so the per-tile chain of one CTA per SM, not the
// dequantisation, bounds both.  Per 128-entry tile:
//   TMA        64-byte code rows -> 128-byte swizzled lines, each run of 16
//              codes padded to 16 bytes (the 4-bit operand layout of
//              tcgen05), 12-deep ring; 8 KB of HBM per tile
//   scales     8 warps (two per TMEM lane quarter, alternate tiles) write
//              each entry's four UE8M0 block scales to TMEM; each loads the
//              scale words of its next 8 tiles ahead
//   MMA        tcgen05 kind::mxf8f6f4 with block scaling: A = E2M1 keys with
//              their scales, B = E4M3 queries with scale 1, K = 32 per
//              instruction (one scale per row), FP32 accumulate, so every
//              product E2M1 x 2^(X_b - 127) x E4M3 is exact whatever the
//              spread of an entry's block scales
//   epilogue   8 warps, the two halves take alternate tiles (as the E4M3 path
//              with 1-2 rows), no entry factor
// TMEM: accumulators in columns [0, 384) (six of 64 or three of 128), the B
// scales in [384, 400), seven A-scale buffers of 16 columns from 400.  A
// scale buffer holds one group of 4 columns per K-step; the MMA reads the
// scale of row m at lane m, column (group + m / 32), so each lane writes its
// own entry's scale of block k in every column of group k, in every byte.
// Warp roles (576 threads): 0 TMA producer, 1 TMEM allocator + MMA issuer,
// 2-9 epilogue, 10-17 scale writers.  Waits are bounded as in the E4M3 path.

// Key path of the FP4 indexer call.  0: every rectangle takes the E4M3
// staging kernel (default: measured the faster on B200, 544 against 564 us
// for 64 decode queries over 262144 entries); 1: calls of one or two rows
// take the block-scaled kernel.
inline std::atomic<int>& fp4_mma_mode_ref() {
  static std::atomic<int> mode{0};
  return mode;
}
inline int fp4_mma_mode() { return fp4_mma_mode_ref().load(std::memory_order_relaxed); }

constexpr int kMxStages = 12;
constexpr int kMxSf = 7;                       // A-scale buffers in TMEM
constexpr int kMxScaleWarp0 = 10;
constexpr int kMxThreads = (kMxScaleWarp0 + 8) * 32;          // 576
constexpr int kMxSfAhead = 8;                  // scale words in flight per writer warp (its own tiles)
constexpr uint32_t kMxQBytes = 128 * 128;      // up to 2 query rows x 64 heads x 128 E4M3
constexpr uint32_t kMxCBytes = kIxTileE * 128; // one unpacked code tile in shared memory
constexpr uint32_t kMxCTx = kIxTileE * 64;     // bytes the copy of a tile credits (packed)
constexpr uint32_t kMxAccCols = 384;
constexpr uint32_t kMxSfB = 384;               // B scales (all 1)
constexpr uint32_t kMxSfA = 400;               // A-scale buffers
static_assert(kMxAccCols <= kMxSfB && kMxSfB + 16 <= kMxSfA && kMxSfA + 16 * kMxSf <= 512,
              "TMEM columns of the block-scaled indexer");
constexpr int kMxBars = 1 + 2 * kMxStages + 2 * kMxSf + 2 * 6;
constexpr size_t kMxSmem = 1024 + kMxQBytes + kMxStages * kMxCBytes + kIxRows * 64 * 4 + kMxBars * 8;
static_assert(kMxSmem + 64 <= 232448, "shared memory of the block-scaled indexer kernel");

// Instruction descriptor, kind::mxf8f6f4 with block scaling: A E2M1 (5),
// B E4M3 (0), both K-major, UE8M0 scales (bit 23), M = 128.  Bits 4-5 (the
// B scale-factor byte) are 1: the B scales are 1 in every byte.
__host__ __device__ __forceinline__ uint32_t idesc_mx_e2m1_e4m3(int N) {
  uint32_t d = 0;
  d |= 1u << 4;
  d |= 5u << 7;
  d |= (uint32_t)((N >> 3) & 0x3F) << 17;
  d |= 1u << 23;
  d |= (uint32_t)(128 >> 4) << 24;
  return d;
}
__device__ __forceinline__ void mma_mx_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale.scale_vec::1X [%0], %1, %2, %3, [%4], [%5], p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(sfa_tmem), "r"(sfb_tmem), "r"(accumulate)
      : "memory");
}

__global__ void __launch_bounds__(kMxThreads, 1)
indexer_mx_kernel(const __grid_constant__ CUtensorMap q_map, const __grid_constant__ CUtensorMap c_map,
                  const uint32_t* __restrict__ k_scales, const float* __restrict__ w8, float* __restrict__ scores,
                  IxGeom g) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* s_q = smem;
  uint8_t* s_c = s_q + kMxQBytes;
  float* s_w = reinterpret_cast<float*>(s_c + kMxStages * kMxCBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(s_w + kIxRows * 64);
  uint64_t* q_full = bars;
  uint64_t* c_full = bars + 1;
  uint64_t* c_empty = c_full + kMxStages;
  uint64_t* sf_full = c_empty + kMxStages;
  uint64_t* sf_empty = sf_full + kMxSf;
  uint64_t* acc_full = sf_empty + kMxSf;
  uint64_t* acc_empty = acc_full + 6;
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- work unit (as the E4M3 path; one group per sequence, 1-2 rows)
  const int n_groups = g.nb * g.gps;
  const int grp = n_groups - 1 - (int)blockIdx.x;
  const int split = blockIdx.y;
  const int bl = grp / g.gps;
  const int b = g.b0 + bl;
  const int gi = grp - bl * g.gps;
  const int i_first = g.i0 + gi * kIxRows;
  int rows = g.i0 + g.ni - i_first;
  rows = rows < 2 ? rows : 2;
  long long nv = (g.q_pos0 + i_first + rows - 1) / g.m;
  if (nv > g.Nc) nv = g.Nc;
  const int tiles_all = (int)((nv + kIxTileE - 1) / kIxTileE);
  const int per_split = (tiles_all + g.splits - 1) / g.splits;
  const int t_begin = split * per_split;
  int t_end = t_begin + per_split;
  t_end = t_end < tiles_all ? t_end : tiles_all;
  const int n_tiles = t_end > t_begin ? t_end - t_begin : 0;
  if (n_tiles == 0) return;
  const long long rect_row = (long long)bl * g.ni + (i_first - g.i0);
  const uint32_t acc_cols = 64u * (uint32_t)rows;
  const int n_acc = (int)(kMxAccCols / acc_cols);     // 6 or 3 accumulators

  if (threadIdx.x == 0) {
    tc::mbar_init(q_full, 1);
    for (int s = 0; s < kMxStages; ++s) { tc::mbar_init(c_full + s, 1); tc::mbar_init(c_empty + s, 1); }
    for (int s = 0; s < kMxSf; ++s) { tc::mbar_init(sf_full + s, 4); tc::mbar_init(sf_empty + s, 1); }
    for (int a = 0; a < 6; ++a) { tc::mbar_init(acc_full + a, 1); tc::mbar_init(acc_empty + a, 4); }
    tc::fence_barrier_init();
    s_abort = 0;
  }
  if (warp == 1) { tc::tmem_alloc(&s_tmem, 512); tc::tmem_relinquish(); }
  for (int e = threadIdx.x; e < kIxRows * 64; e += kMxThreads) {
    const int q = e >> 6;
    s_w[e] = q < rows ? w8[(rect_row + q) * 64 + (e & 63)] : 0.f;
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = s_tmem;
  volatile int* abort_flag = &s_abort;
  const long long ent0 = (long long)b * g.Nc;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (tc::elect_one()) {
      tc::prefetch_tmap(&q_map);
      tc::prefetch_tmap(&c_map);
      tc::mbar_arrive_expect_tx(q_full, kMxQBytes);
      tc::tma_load_2d(s_q, &q_map, q_full, 0, (int)(rect_row * 64));
      int issued = 0;
      for (int n = 0; n < n_tiles; ++n) {
        const int s = n % kMxStages, r = n / kMxStages;
        if (r > 0 && !tc::mbar_wait(c_empty + s, (r - 1) & 1)) { *abort_flag = 1; break; }
        if (*abort_flag) break;
        tc::mbar_arrive_expect_tx(c_full + s, kMxCTx);
        tc::tma_load_2d(s_c + s * kMxCBytes, &c_map, c_full + s, 0,
                        (int)(ent0 + (long long)(t_begin + n) * kIxTileE));
        ++issued;
      }
      for (int n = issued - kMxStages > 0 ? issued - kMxStages : 0; n < issued; ++n)
        tc::mbar_wait(c_full + n % kMxStages, (n / kMxStages) & 1);
      tc::mbar_wait(q_full, 0);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (tc::elect_one()) {
      const uint32_t idesc = idesc_mx_e2m1_e4m3(64 * rows);
      bool ok = tc::mbar_wait(q_full, 0);
      const uint32_t b_base = tc::smem_u32(s_q);
      for (int n = 0; ok && n < n_tiles; ++n) {
        const int s = n % kMxStages, rs = n / kMxStages;
        const int f = n % kMxSf, rf = n / kMxSf;
        const int a = n % n_acc, ra = n / n_acc;
        if (*abort_flag) break;
        if (!tc::mbar_wait_spin(c_full + s, rs & 1)) { ok = false; break; }
        if (!tc::mbar_wait_spin(sf_full + f, rf & 1)) { ok = false; break; }
        if (ra > 0 && !tc::mbar_wait_spin(acc_empty + a, (ra - 1) & 1)) { ok = false; break; }
        tc::tc_fence_after();
        const uint32_t a_base = tc::smem_u32(s_c + s * kMxCBytes);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint64_t ad = tc::sdesc_sw128(a_base + ks * 32, 16, 1024);
          const uint64_t bd = tc::sdesc_sw128(b_base + ks * 32, 16, 1024);
          mma_mx_ss(tmem + (uint32_t)a * acc_cols, ad, bd, idesc, tmem + kMxSfA + 16u * (uint32_t)f + 4u * ks,
                    tmem + kMxSfB, ks > 0 ? 1u : 0u);
        }
        tc::mma_commit(c_empty + s);
        tc::mma_commit(sf_empty + f);
        tc::mma_commit(acc_full + a);
      }
      if (!ok) *abort_flag = 1;
    }
  } else if (warp < kMxScaleWarp0) {
    // ------------------------------------------------------------ epilogue
    const int e = warp - 2;                 // 0..7
    const int quarter = warp & 3;           // TMEM lanes [32*quarter, 32*quarter+32)
    const int half = e >> 2;                // takes the tiles n with n % 2 == half
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
    for (int n = half; n < n_tiles; n += 2) {
      const int a = n % n_acc, ra = n / n_acc;
      const long long j = (long long)(t_begin + n) * kIxTileE + quarter * 32 + lane;
      bool ok = !*abort_flag && tc::mbar_wait(acc_full + a, ra & 1);
      if (!__all_sync(0xffffffffu, ok)) { *abort_flag = 1; break; }
      tc::tc_fence_after();
      float sc[2] = {0.f, 0.f};
#pragma unroll
      for (int qq = 0; qq < 2; ++qq) {
        if (qq < rows) {
          const uint32_t col = tmem + lane_addr + (uint32_t)a * acc_cols + (uint32_t)(qq * 64);
          const uint32_t wq = tc::smem_u32(s_w + qq * 64);
          // w relu(x) = (w/2) x + (w/2) |x| (the prepared weights carry the 1/2)
          float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int hb = 0; hb < 64; hb += 32) {
            uint32_t v[32];
            tc::tmem_ld32(col + hb, v);
            tc::tmem_wait_ld();
            if (qq == rows - 1 && hb == 32) {      // accumulator read out: hand it back to the MMA warp
              tc::tc_fence_before();
              __syncwarp();
              if (lane == 0) tc::mbar_arrive(acc_empty + a);
            }
#pragma unroll
            for (int h = 0; h < 32; h += 4) {
              const float4 w4 = tc::lds128f(wq + (hb + h) * 4);
              const float x0 = __uint_as_float(v[h]), x1 = __uint_as_float(v[h + 1]);
              const float x2 = __uint_as_float(v[h + 2]), x3 = __uint_as_float(v[h + 3]);
              acc[0] = fmaf(w4.x, x0, acc[0]); acc[4] = fmaf(w4.x, fabsf(x0), acc[4]);
              acc[1] = fmaf(w4.y, x1, acc[1]); acc[5] = fmaf(w4.y, fabsf(x1), acc[5]);
              acc[2] = fmaf(w4.z, x2, acc[2]); acc[6] = fmaf(w4.z, fabsf(x2), acc[6]);
              acc[3] = fmaf(w4.w, x3, acc[3]); acc[7] = fmaf(w4.w, fabsf(x3), acc[7]);
            }
          }
          sc[qq] = ((acc[0] + acc[4]) + (acc[1] + acc[5])) + ((acc[2] + acc[6]) + (acc[3] + acc[7]));
        }
      }
      if (j < g.Nc) {
#pragma unroll
        for (int qq = 0; qq < 2; ++qq)
          if (qq < rows) scores[(rect_row + qq) * g.Nc + j] = sc[qq];
      }
    }
  } else {
    // ------------------------------------------------------------ scale writers
    // lane l of this warp owns TMEM lane 32 * quarter + l = entry row of the
    // tiles n with n % 2 == half
    const int quarter = warp & 3;
    const int half = (warp - kMxScaleWarp0) >> 2;
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
    auto scale_word = [&](int n) -> uint32_t {
      const long long j = (long long)(t_begin + n) * kIxTileE + quarter * 32 + lane;
      return n < n_tiles && j < g.Nc ? __ldg(k_scales + ent0 + j) : 0x7F7F7F7Fu;
    };
    uint32_t r[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) r[i] = 0x7F7F7F7Fu;
    if (half == 0) tc::tmem_st16(tmem + lane_addr + kMxSfB, r);   // B scales: 1 (UE8M0 127) in every byte
    // words of this warp's next kMxSfAhead tiles (a ring of registers, static
    // indices: the loop below is unrolled by its length)
    uint32_t ring[kMxSfAhead];
#pragma unroll
    for (int u = 0; u < kMxSfAhead; ++u) ring[u] = scale_word(half + 2 * u);
    bool live = true;
    for (int n0 = half; live && n0 < n_tiles; n0 += 2 * kMxSfAhead) {
#pragma unroll
    for (int u = 0; u < kMxSfAhead; ++u) {
      const int n = n0 + 2 * u;
      if (n >= n_tiles) { live = false; break; }
      const int f = n % kMxSf, rf = n / kMxSf;
      const uint32_t sw = ring[u];
      ring[u] = scale_word(n + 2 * kMxSfAhead);
      bool ok = !*abort_flag && (rf == 0 || tc::mbar_wait(sf_empty + f, (rf - 1) & 1));
      if (!__all_sync(0xffffffffu, ok)) { *abort_flag = 1; live = false; break; }
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint32_t x = ((sw >> (8 * k)) & 0xFFu) * 0x01010101u;
        r[4 * k] = x; r[4 * k + 1] = x; r[4 * k + 2] = x; r[4 * k + 3] = x;
      }
      tc::tmem_st16(tmem + lane_addr + kMxSfA + 16u * (uint32_t)f, r);
      tc::tmem_wait_st();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(sf_full + f);
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

// Scores of the chunk rectangle (sequences [b0, b0+nb), rows [i0, i0+ni)),
// rows laid out [nb][ni][Nc].  q8 / w8: the prepared queries of the rectangle.
// Calls of one or two rows per sequence (few_rows) take the block-scaled
// kernel when the codes are 32-byte aligned, others the E4M3 staging kernel.
static cudaError_t launch_indexer_fp4_rect(const uint8_t* k_codes, const uint8_t* k_scales, int B, int Nc,
                                           long long q_pos0, int m, const uint8_t* q8, const float* w8,
                                           float* scores, int b0, int nb, int i0, int ni, bool few_rows,
                                           cudaStream_t st) {
  CUtensorMap qm, cm;
  const bool mx = few_rows && ni <= 2 && fp4_mma_mode() == 1 &&
                  make_tmap_u4x128_2d(&cm, k_codes, (uint64_t)B * Nc, kIxTileE);
  if (mx) {
    if (!make_tmap_2d(&qm, q8, 1, (uint64_t)nb * ni * 64, 128, 128, 128, 128)) return cudaErrorInvalidValue;
  } else {
    if (!make_tmap_2d(&qm, q8, 1, (uint64_t)nb * ni * 64, 128, 128, 128, 256)) return cudaErrorInvalidValue;
    if (!make_tmap_2d(&cm, k_codes, 1, (uint64_t)B * Nc, 64, 64, 64, kIxTileE, false)) return cudaErrorInvalidValue;
  }
  IxGeom g;
  g.Tq = 0; g.Nc = Nc; g.H = 64;
  g.b0 = b0; g.nb = nb; g.i0 = i0; g.ni = ni;
  g.gps = (ni + kIxRows - 1) / kIxRows;
  g.q_pos0 = q_pos0; g.m = m;
  const int n_groups = nb * g.gps;
  long long nv = (q_pos0 + i0 + ni - 1) / m;
  if (nv > Nc) nv = Nc;
  const int tiles = (int)((nv + kIxTileE - 1) / kIxTileE);
  const int splits = indexer_splits(n_groups, tiles);
  g.splits = splits;
  dim3 grid(n_groups, splits);
  if (mx) {
    cudaError_t e = cudaFuncSetAttribute(indexer_mx_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kMxSmem);
    if (e != cudaSuccess) return e;
    indexer_mx_kernel<<<grid, kMxThreads, kMxSmem, st>>>(qm, cm, reinterpret_cast<const uint32_t*>(k_scales), w8,
                                                          scores, g);
  } else {
    cudaError_t e = cudaFuncSetAttribute(indexer_fp4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kI4Smem);
    if (e != cudaSuccess) return e;
    indexer_fp4_kernel<<<grid, kI4Threads, kI4Smem, st>>>(qm, cm, reinterpret_cast<const uint32_t*>(k_scales), w8,
                                                           scores, g);
  }
  count_launch();
  return cudaGetLastError();
}

}  // namespace lcsa
