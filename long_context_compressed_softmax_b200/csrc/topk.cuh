// Exact top-k selection per row (radix select on order-preserving keys).
// (DeepSeek-V4 CSA Step 2: keep the top-k indexer scores; ties to the lower
// index; indices emitted ascending, -1 padded.)
//
// One CTA (16 warps) per row; the row is split into 16 contiguous warp
// segments.  Scores map to 32-bit keys whose unsigned order is the float
// order (-0 folded onto +0).
//   1. A 4096-bin histogram of the keys' top 12 bits (sign, exponent, three
//      mantissa bits) gives the bin holding the k-th largest key.
//   2. One sweep counts, per warp segment, the keys above that bin and
//      compacts the bin's (key, index) pairs into a candidate list.
//   3. The exact threshold key and the number of its ties to keep are found
//      on the candidates alone (12- and 8-bit histograms); a bin too full for
//      the list falls back to the same histograms over the whole row.
//   4. Each warp emits its segment in index order with ballots: every key
//      above the threshold plus the first r ties, at slots given by per-warp
//      prefix counts, so the list comes out ascending without block scans.
// Rows up to kMaxCachedKeys are staged in shared memory during pass 1;
// longer rows are re-read from L2 in each pass.
#pragma once
#include "common.cuh"
#include "tc_ptx.cuh"

namespace lcsa {

constexpr int kTopkThreads = 512;
constexpr int kMaxCachedKeys = 32768;   // 128 KiB of dynamic shared memory
constexpr int kTopkBins = 4096;
constexpr int kTopkCand = 2048;         // candidate list capacity

__device__ __forceinline__ uint32_t score_key(float s) {
  uint32_t u = __float_as_uint(s);
  if (u == 0x80000000u) u = 0u;                      // -0.0 == +0.0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive block scan (NT threads); *total receives the block sum.
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

struct TopkState {
  uint32_t prefix, mask, kr;
  int done;
};

// In a histogram of `nbins` (4096 or 256) bins scanned from the top, find the
// bin where the running count reaches st->kr and refine *st to it.  All NT
// threads call this; it ends with a barrier.
template <int NT>
__device__ __forceinline__ void topk_pick_bin(const uint32_t* hist, int nbins, int shift, uint32_t dmask,
                                              TopkState* st, uint32_t* s_warp, uint32_t* s_total,
                                              uint32_t* s_bincnt) {
  const uint32_t kr = st->kr;
  const int per = nbins / NT;                        // 8 bins per thread, or 0 (one bin for the first nbins threads)
  uint32_t cnt[8], sum = 0;
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    int bin = -1;
    if (per > 0) bin = q < per ? nbins - 1 - per * (int)threadIdx.x - q : -1;
    else bin = (q == 0 && (int)threadIdx.x < nbins) ? nbins - 1 - (int)threadIdx.x : -1;
    cnt[q] = bin >= 0 ? hist[bin] : 0u;
    sum += cnt[q];
  }
  const uint32_t excl = block_excl_scan<NT>(sum, s_warp, s_total);
  if (excl < kr && excl + sum >= kr) {               // exactly one thread
    uint32_t c = excl;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      if (c + cnt[q] >= kr) {
        const int bin = per > 0 ? nbins - 1 - per * (int)threadIdx.x - q : nbins - 1 - (int)threadIdx.x;
        st->prefix |= (uint32_t)bin << shift;
        st->mask |= dmask << shift;
        st->kr = kr - c;
        st->done = (kr - c == cnt[q]) ? 1 : 0;       // the whole bin is taken: no need to refine
        *s_bincnt = cnt[q];
        break;
      }
      c += cnt[q];
    }
  }
  __syncthreads();
}

// Visit every key of [lo, hi) (a warp segment) in index order per lane:
// lane L handles elements base+4L .. base+4L+3 of each 128-element step, and
// kUnroll steps are loaded before any is used, so a thread keeps 4*kUnroll
// scores in flight.  f(i, key, valid) is called for all 4*kUnroll slots of a
// group; vec4 requires src 16-byte aligned and lo % 4 == 0.
constexpr int kUnroll = 4;
template <typename F>
__device__ __forceinline__ void segment_visit(const float* __restrict__ src, const uint32_t* keys, bool cached,
                                              bool vec4, int lo, int hi, F&& f) {
  const int lane = threadIdx.x & 31;
  for (int base = lo; base < hi; base += 128 * kUnroll) {
    uint32_t kk[kUnroll][4];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int i0 = base + u * 128 + 4 * lane;
      if (vec4 && i0 + 3 < hi) {
        if (cached) {
          const uint4 v = *reinterpret_cast<const uint4*>(keys + i0);
          kk[u][0] = v.x; kk[u][1] = v.y; kk[u][2] = v.z; kk[u][3] = v.w;
        } else {
          const float4 v = __ldg(reinterpret_cast<const float4*>(src + i0));
          kk[u][0] = score_key(v.x); kk[u][1] = score_key(v.y); kk[u][2] = score_key(v.z); kk[u][3] = score_key(v.w);
        }
      } else {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int i = i0 + q;
          kk[u][q] = i < hi ? (cached ? keys[i] : score_key(__ldg(src + i))) : 0u;
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int i = base + u * 128 + 4 * lane + q;
        f(u, i, kk[u][q], i < hi);
      }
  }
}

template <int NT>
__global__ void __launch_bounds__(NT)
topk_rows_kernel(const float* __restrict__ scores, long long ld, int n_cols,
                 const int32_t* __restrict__ n_valid, int k, int32_t* __restrict__ idx_out,
                 int cache_cap) {
  static_assert(kTopkBins == 8 * NT, "each thread owns 8 bins");
  constexpr int W = NT / 32;
  extern __shared__ uint32_t s_keys[];
  __shared__ uint32_t s_hist[kTopkBins];
  __shared__ uint32_t s_ckey[kTopkCand];
  __shared__ int32_t s_cidx[kTopkCand];
  __shared__ uint32_t s_warp[32];
  __shared__ uint32_t s_total, s_bincnt, s_ncand;
  __shared__ uint32_t s_above[W], s_eq[W];           // per-warp-segment counts
  __shared__ TopkState s_st;

  const int row = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
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
  const bool vec4 = (reinterpret_cast<uintptr_t>(src) & 15u) == 0;
  // contiguous warp segments [seg_lo, seg_hi), lengths multiples of 128
  const int seg_len = ((n + W - 1) / W + 127) & ~127;
  const int seg_lo = warp * seg_len < n ? warp * seg_len : n;
  const int seg_hi = seg_lo + seg_len < n ? seg_lo + seg_len : n;

  for (int i = threadIdx.x; i < kTopkBins; i += NT) s_hist[i] = 0u;
  if (threadIdx.x == 0) { s_st.prefix = 0u; s_st.mask = 0u; s_st.kr = (uint32_t)k; s_st.done = 0; s_ncand = 0u; }
  if (threadIdx.x < W) { s_above[threadIdx.x] = 0u; s_eq[threadIdx.x] = 0u; }
  __syncthreads();

  // ---- pass 1: top-12-bit histogram (stages the row in shared memory)
  segment_visit(src, s_keys, false, vec4, seg_lo, seg_hi, [&](int, int i, uint32_t key, bool valid) {
    if (valid) {
      if (cached) s_keys[i] = key;
      atomicAdd(&s_hist[key >> 20], 1u);
    }
  });
  __syncthreads();
  topk_pick_bin<NT>(s_hist, kTopkBins, 20, 0xFFFu, &s_st, s_warp, &s_total, &s_bincnt);
  const uint32_t prefix1 = s_st.prefix, mask1 = s_st.mask;
  const bool fits = s_bincnt <= (uint32_t)kTopkCand;

  // ---- pass 2: per-segment counts above the bin; compact the bin's candidates
  {
    uint32_t above = 0;
    segment_visit(src, s_keys, cached, vec4, seg_lo, seg_hi, [&](int, int i, uint32_t key, bool valid) {
      if (!valid) return;
      const uint32_t mk = key & mask1;
      above += mk > prefix1;
      if (fits && mk == prefix1) {
        const uint32_t slot = atomicAdd(&s_ncand, 1u);
        s_ckey[slot] = key;
        s_cidx[slot] = i;
      }
    });
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) above += __shfl_xor_sync(0xffffffffu, above, o);
    if (lane == 0) s_above[warp] = above;
  }
  __syncthreads();

  // ---- resolve the exact threshold: on the candidates, or over the whole row
  const int ncand = fits ? (int)s_ncand : 0;
  for (int level = 0; level < 2; ++level) {
    if (s_st.done) break;                             // uniform: read after a barrier
    const int shift = level == 0 ? 8 : 0;
    const uint32_t dmask = level == 0 ? 0xFFFu : 0xFFu;
    const int nbins = level == 0 ? kTopkBins : 256;
    for (int i = threadIdx.x; i < nbins; i += NT) s_hist[i] = 0u;
    __syncthreads();
    const uint32_t prefix = s_st.prefix, mask = s_st.mask;
    if (fits) {
      for (int c = threadIdx.x; c < ncand; c += NT) {
        const uint32_t key = s_ckey[c];
        if ((key & mask) == prefix) atomicAdd(&s_hist[(key >> shift) & dmask], 1u);
      }
    } else {
      segment_visit(src, s_keys, cached, vec4, seg_lo, seg_hi, [&](int, int, uint32_t key, bool valid) {
        if (valid && (key & mask) == prefix) atomicAdd(&s_hist[(key >> shift) & dmask], 1u);
      });
    }
    __syncthreads();
    topk_pick_bin<NT>(s_hist, nbins, shift, dmask, &s_st, s_warp, &s_total, &s_bincnt);
  }
  const uint32_t prefix = s_st.prefix, mask = s_st.mask, kr = s_st.kr;

  // ---- per-segment counts of the threshold bin's keys above / equal to it
  if (fits) {
    for (int c = threadIdx.x; c < ncand; c += NT) {
      const uint32_t key = s_ckey[c] & mask;
      const int w = s_cidx[c] / seg_len;
      if (key > prefix) atomicAdd(&s_above[w], 1u);
      else if (key == prefix) atomicAdd(&s_eq[w], 1u);
    }
  } else {
    uint32_t above = 0, eq = 0;
    segment_visit(src, s_keys, cached, vec4, seg_lo, seg_hi, [&](int, int, uint32_t key, bool valid) {
      if (valid && (key & mask1) == prefix1) {
        const uint32_t mk = key & mask;
        above += mk > prefix;
        eq += mk == prefix;
      }
    });
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      above += __shfl_xor_sync(0xffffffffu, above, o);
      eq += __shfl_xor_sync(0xffffffffu, eq, o);
    }
    if (lane == 0) { s_above[warp] += above; s_eq[warp] = eq; }
  }
  __syncthreads();

  // ---- emission: every warp walks its own segment in index order; within a
  // 128-element step lane L owns elements 4L..4L+3, so a warp scan of the
  // per-lane counts gives each lane its running position.
  uint32_t run_a = 0, run_e = 0;
  for (int w = 0; w < warp; ++w) { run_a += s_above[w]; run_e += s_eq[w]; }
  {
    uint32_t fa[kUnroll], fe[kUnroll];              // per step: bit q set if element q is above / a tie
    segment_visit(src, s_keys, cached, vec4, seg_lo, seg_hi, [&](int u, int i, uint32_t key, bool valid) {
      const int q = i & 3;
      if (q == 0) { fa[u] = 0u; fe[u] = 0u; }
      if (valid) {
        const uint32_t mk = key & mask;
        fa[u] |= (uint32_t)(mk > prefix) << q;
        fe[u] |= (uint32_t)(mk == prefix) << q;
      }
      if (q == 3) {
        // packed counts (a in the low half, e in the high half) of this lane's four elements
        const uint32_t mine = __popc(fa[u]) | (__popc(fe[u]) << 16);
        uint32_t incl = mine;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        const uint32_t tot = __shfl_sync(0xffffffffu, incl, 31);
        uint32_t ga = run_a + ((incl - mine) & 0xffffu), ge = run_e + ((incl - mine) >> 16);
        const int i0 = i - 3;
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
          if ((fa[u] >> qq) & 1u) { dst[ga + (ge < kr ? ge : kr)] = i0 + qq; ++ga; }
          else if ((fe[u] >> qq) & 1u) { if (ge < kr) dst[ga + ge] = i0 + qq; ++ge; }
        }
        run_a += tot & 0xffffu;
        run_e += tot >> 16;
      }
    });
  }
}

// ---------------------------------------------------------------------------
// Rows of up to kMaxCachedKeys scores with 16-byte aligned rows: persistent
// CTAs, two per SM, one row at a time each.
//   1. A 512-score sample gives a value range [lo, hi]; the bucket
//      clamp((v - lo) * 2048 / (hi - lo)) is monotone in v and spreads
//      typical score rows over many of its 2048 buckets.
//   2. Pass 1 streams the row from global memory once: bucket histogram,
//      and the bucket of every score kept as a 16-bit code in shared memory.
//   3. The bucket holding the k-th score (bpiv) and the rank kr inside it
//      come from the histogram; its scores (few) are compacted in index
//      order into a list (scores re-read from global memory).
//   4. The list's exact top kr (ties to the lower index) is marked: one warp
//      ranks lists of up to 32; larger lists use 11/11/10-bit radix levels on
//      the keys; a bucket too full for the list is resolved over the row.
//   5. Selected list entries get code 2048, the others 0, so the selection
//      is exactly {code > bpiv}; one ordered compaction pass emits it.
// ---------------------------------------------------------------------------
// CTA size: 512 threads (two CTAs per SM) for long rows, 256 (four per SM)
// when the code buffer is at most 32 KB.
constexpr int kTk2Bins = 2048;
constexpr int kTk2List = 1024;
constexpr uint16_t kTk2Sel = 2048;                  // code of a selected score of the pivot bucket

// Two 16-bit codes per 32-bit word (codes <= 2048 < 2^15): adding
// 0x7FFF - b to each half sets the half's bit 15 exactly when its code is
// above b, with no carry between the halves; 0x8000 - b sets it when the code
// is at least b.  Flags of a word land at bits 15 and 31.
constexpr uint32_t kTk2Hi = 0x80008000u;
__device__ __forceinline__ uint32_t half_add(uint32_t b0) { return b0 | (b0 << 16); }
// flags (bits 15, 31) of the two codes of w -> bits 0, 1
__device__ __forceinline__ uint32_t pair_bits(uint32_t t) { return ((t >> 15) | (t >> 30)) & 3u; }

// Block-wide k-th largest key (ranks counted from 1) among cnt keys given by
// get(c, &key) -> valid; refines *st over three digit levels so that on
// return st->prefix is the exact key and st->kr the number of its copies to
// keep.  All threads call it; it ends with a barrier.
template <int kTk2Threads, typename Get>
__device__ __forceinline__ void tk2_radix(Get&& get, int cnt, uint32_t* hist, TopkState* st, uint32_t* s_warp,
                                          uint32_t* s_total, uint32_t* s_bincnt) {
  for (int level = 0; level < 3; ++level) {
    const int shift = level == 0 ? 21 : (level == 1 ? 10 : 0);
    const uint32_t dmask = level == 2 ? 0x3FFu : 0x7FFu;
    const int nbins = level == 2 ? 1024 : 2048;
    for (int i = threadIdx.x; i < nbins; i += kTk2Threads) hist[i] = 0u;
    __syncthreads();
    const uint32_t prefix = st->prefix, mask = st->mask;
    for (int c = threadIdx.x; c < cnt; c += kTk2Threads) {
      uint32_t key;
      if (get(c, &key) && (key & mask) == prefix) atomicAdd(&hist[(key >> shift) & dmask], 1u);
    }
    __syncthreads();
    topk_pick_bin<kTk2Threads>(hist, nbins, shift, dmask, st, s_warp, s_total, s_bincnt);
  }
}

// Ordered compaction helper: lane L holds 4 consecutive elements (bits of
// `f`); returns the number of set bits of lanes below L, and the warp total.
__device__ __forceinline__ uint32_t warp_excl_count4(uint32_t f, uint32_t* total) {
  const int lane = threadIdx.x & 31;
  const uint32_t lt = (1u << lane) - 1u;
  uint32_t before = 0, tot = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint32_t b = __ballot_sync(0xffffffffu, (f >> q) & 1u);
    before += __popc(b & lt);
    tot += __popc(b);
  }
  *total = tot;
  return before;
}

template <int kTk2Threads>
__global__ void __launch_bounds__(kTk2Threads, 1024 / kTk2Threads)
topk_smem_kernel(const float* __restrict__ scores, long long ld, int n_cols, const int32_t* __restrict__ n_valid,
                 int k, int32_t* __restrict__ idx_out, int rows, int chunk, const int32_t* __restrict__ map,
                 long long map_ld, int code_cap) {
  // code_cap: capacity of the code buffer (the longest row this launch may
  // see, from the caller); a longer row is reported and left unselected.
  constexpr int kTk2Warps = kTk2Threads / 32;
  // chunk > 0: virtual row v is columns [c*chunk, (c+1)*chunk) of row v / C
  // (C = ceil(n_cols / chunk), c = v % C), n_valid counted from c*chunk.
  // map != NULL: the emitted value of column i is map[row * map_ld + i].
  extern __shared__ __align__(16) uint16_t s_code[];   // bucket code of every score of the row
  __shared__ __align__(16) uint32_t s_hist[kTk2Bins];
  __shared__ uint32_t s_lkey[kTk2List];
  __shared__ int32_t s_lidx[kTk2List];
  __shared__ uint32_t s_warp[32];
  __shared__ uint32_t s_total, s_bincnt, s_nlist;
  __shared__ uint32_t s_wa[kTk2Warps], s_we[kTk2Warps];
  __shared__ float s_lo[kTk2Warps], s_hi[kTk2Warps];
  __shared__ TopkState s_st;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

  const int C = chunk > 0 ? (n_cols + chunk - 1) / chunk : 1;
  // valid-count word of (virtual) row v, loaded two rows ahead of its use
  auto raw_n = [&](int v) { return (n_valid != nullptr && v < rows) ? n_valid[v / C] : n_cols; };
  // scores of (virtual) row v and how many of them count, from its count word
  auto setup = [&](int v, int raw, const float** src_out) {
    const int r = v / C, c = v - r * C;              // real row and column chunk
    const int c0 = chunk > 0 ? c * chunk : 0;
    const int width = chunk > 0 ? (n_cols - c0 < chunk ? n_cols - c0 : chunk) : n_cols;
    int n = raw < 0 ? 0 : (raw > n_cols ? n_cols : raw);
    n -= c0;
    *src_out = scores + (long long)r * ld + c0;
    return n < 0 ? 0 : (n > width ? width : n);
  };
  // this thread's sample score of a row (issued one row ahead)
  auto sample = [&](const float* src, int n) {
    return n > k ? __ldg(src + (int)(((long long)threadIdx.x * n) / kTk2Threads)) : 0.f;
  };
  const int G = (int)gridDim.x;
  int raw_cur = raw_n(blockIdx.x), raw_nxt = raw_n(blockIdx.x + G);
  float smp_next = 0.f;
  if ((int)blockIdx.x < rows) {
    const float* s0;
    const int n0 = setup(blockIdx.x, raw_cur, &s0);
    smp_next = sample(s0, n0);
  }
  for (int row = blockIdx.x; row < rows; row += G) {
    const float* src;
    const int n = setup(row, raw_cur, &src);
    const float smp = smp_next;
    int32_t* dst = idx_out + (long long)row * k;
    const int32_t* mrow = map ? map + (long long)row * map_ld : nullptr;
    // the next row of this CTA, and the count word of the one after it
    const bool has_next = row + G < rows;
    const float* src2 = nullptr;
    const int n2 = has_next ? setup(row + G, raw_nxt, &src2) : 0;
    raw_cur = raw_nxt;
    raw_nxt = raw_n(row + 2 * G);
    const bool skip = n <= k || n > code_cap;          // nothing to select (or no room for the codes)
    if (has_next && skip) smp_next = sample(src2, n2);
    if (skip) {
      if (n > code_cap && threadIdx.x == 0) report(LCSA_DEV_BAD_INDEX);
      for (int i = threadIdx.x; i < k; i += kTk2Threads) dst[i] = (i < n && n <= k) ? (mrow ? mrow[i] : i) : -1;
      continue;                                        // no shared memory touched: no barrier needed
    }
    // ---- bucket range from the sample
    {
      const float v = smp;
      float mn = v, mx = v;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      }
      if (lane == 0) { s_lo[warp] = mn; s_hi[warp] = mx; }
    }
    for (int i = threadIdx.x; i < kTk2Bins; i += kTk2Threads) s_hist[i] = 0u;
    if (threadIdx.x == 0) { s_st.prefix = 0u; s_st.mask = 0u; s_st.kr = (uint32_t)k; s_st.done = 0; }
    __syncthreads();
    float lo = s_lo[0], hi = s_hi[0];
#pragma unroll
    for (int w = 1; w < kTk2Warps; ++w) { lo = fminf(lo, s_lo[w]); hi = fmaxf(hi, s_hi[w]); }
    // one bucket for everything when the sampled range is empty or not finite
    const float s0 = (hi > lo && hi - lo < INFINITY) ? (float)kTk2Bins / (hi - lo) : 0.f;
    const float scale = fabsf(lo * s0) < 1e30f ? s0 : 0.f;   // the offset below stays finite
    // bucket = (v - lo) * scale - 1/2 rounded to an integer and clamped to
    // [0, kTk2Bins - 1], taken from the low mantissa bits of a float in
    // [2^23, 2^23 + kTk2Bins - 1] (where one ulp is 1): one FMA, two clamps
    // and a mask.  A correctly rounded FMA of a function increasing in v is
    // non-decreasing in v, and so is the clamp: the bucket order never
    // contradicts the score order.  NaN-free rows (an infinite score clamps
    // to an end bucket).
    constexpr float kTwo23 = 8388608.f;
    const float c0 = scale == 0.f ? kTwo23 : kTwo23 - lo * scale - 0.5f;
    auto bucket = [&](float v) -> uint32_t {
      const float y = fminf(fmaxf(fmaf(v, scale, c0), kTwo23), kTwo23 + (float)(kTk2Bins - 1));
      return __float_as_uint(y) & 0x7FFFFFu;
    };
    // contiguous warp segments [seg_lo, seg_hi), lengths multiples of 256:
    // lane L owns elements 8L .. 8L+7 of each 256-element step
    const int seg = ((n + kTk2Warps - 1) / kTk2Warps + 255) & ~255;
    const int seg_lo = warp * seg < n ? warp * seg : n;
    const int seg_hi = seg_lo + seg < n ? seg_lo + seg : n;

    // ---- pass 1: stream the row, bucket histogram and codes
#pragma unroll 2
    for (int base = seg_lo; base < seg_hi; base += 256) {
      const int i0 = base + 8 * lane;
      if (i0 + 7 < seg_hi) {
        const float4 v0 = __ldg(reinterpret_cast<const float4*>(src + i0));
        const float4 v1 = __ldg(reinterpret_cast<const float4*>(src + i0 + 4));
        const uint32_t b[8] = {bucket(v0.x), bucket(v0.y), bucket(v0.z), bucket(v0.w),
                               bucket(v1.x), bucket(v1.y), bucket(v1.z), bucket(v1.w)};
#pragma unroll
        for (int q = 0; q < 8; ++q) atomicAdd(&s_hist[b[q]], 1u);
        *reinterpret_cast<uint4*>(s_code + i0) =
            make_uint4(b[0] | (b[1] << 16), b[2] | (b[3] << 16), b[4] | (b[5] << 16), b[6] | (b[7] << 16));
      } else {
        for (int q = 0; q < 8; ++q)
          if (i0 + q < seg_hi) {
            const uint32_t bq = bucket(__ldg(src + i0 + q));
            atomicAdd(&s_hist[bq], 1u);
            s_code[i0 + q] = (uint16_t)bq;
          }
      }
    }
    // the next row's scores into L2 while this row is resolved and emitted
    if (threadIdx.x == 0 && has_next && n2 > k && n2 <= code_cap && n2 >= 4)
      tc::bulk_prefetch_l2(src2, (uint32_t)(n2 & ~3) * 4u);
    __syncthreads();
    // bucket of the k-th score, by one warp: lane L sums buckets
    // 2047-64L .. 1984-64L, a warp scan from the top finds the lane and that
    // lane the bucket; rank kr inside it, its count cnt
    if (warp == 0) {
      const int top = kTk2Bins - 1 - 64 * lane;
      uint32_t sum = 0;
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        const uint4 v = *reinterpret_cast<const uint4*>(s_hist + top - 63 + 4 * q);
        sum += v.x + v.y + v.z + v.w;
      }
      uint32_t incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const uint32_t excl = incl - sum;
      // the lane whose 64 buckets hold the k-th score (exactly one)
      const uint32_t hit = __ballot_sync(0xffffffffu, excl < (uint32_t)k && incl >= (uint32_t)k);
      const int hl = __ffs(hit) - 1;
      const uint32_t cum0 = __shfl_sync(0xffffffffu, excl, hl);
      // its buckets, two per lane from the top: lane L takes 2L and 2L+1
      const int t0 = kTk2Bins - 1 - 64 * hl - 2 * lane;
      const uint32_t c0 = s_hist[t0], c1 = s_hist[t0 - 1];
      const uint32_t pair = c0 + c1;
      uint32_t pin = pair;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, pin, o);
        if (lane >= o) pin += y;
      }
      const uint32_t pex = cum0 + pin - pair;         // scores in buckets above t0
      if (pex < (uint32_t)k && pex + pair >= (uint32_t)k) {   // exactly one lane
        if (pex + c0 >= (uint32_t)k) { s_st.prefix = (uint32_t)t0; s_st.kr = (uint32_t)k - pex; s_bincnt = c0; }
        else { s_st.prefix = (uint32_t)(t0 - 1); s_st.kr = (uint32_t)k - pex - c0; s_bincnt = c1; }
      }
      if (lane == 0) s_nlist = 0u;
    }
    __syncthreads();
    const uint32_t bpiv = s_st.prefix, kr = s_st.kr, cnt = s_bincnt;
    const bool fits = cnt <= (uint32_t)kTk2List;

    // ---- per-warp counts above the pivot bucket; its scores into the list
    // (unordered: ranks use the column as the tie break)
    {
      uint32_t a = 0;
      const uint32_t gt2 = half_add(0x7FFFu - bpiv), ge2 = half_add(0x8000u - bpiv);
      for (int base = seg_lo; base < seg_hi; base += 256) {
        const int i0 = base + 8 * lane;
        uint32_t f = 0;
        if (i0 + 7 < seg_hi) {
          // eight codes at once: the count above bpiv and the flags of bpiv
          const uint4 c = *reinterpret_cast<const uint4*>(s_code + i0);
          const uint32_t g0 = (c.x + gt2) & kTk2Hi, g1 = (c.y + gt2) & kTk2Hi;
          const uint32_t g2 = (c.z + gt2) & kTk2Hi, g3 = (c.w + gt2) & kTk2Hi;
          a += (uint32_t)__popc(g0 | (g1 >> 1) | (g2 >> 2) | (g3 >> 3));
          if (fits) {
            const uint32_t e0 = (c.x + ge2) & ~g0 & kTk2Hi, e1 = (c.y + ge2) & ~g1 & kTk2Hi;
            const uint32_t e2 = (c.z + ge2) & ~g2 & kTk2Hi, e3 = (c.w + ge2) & ~g3 & kTk2Hi;
            f = pair_bits(e0) | (pair_bits(e1) << 2) | (pair_bits(e2) << 4) | (pair_bits(e3) << 6);
          }
        } else {
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const uint32_t cq = i0 + q < seg_hi ? s_code[i0 + q] : 0u;
            a += (i0 + q < seg_hi && cq > bpiv) ? 1u : 0u;
            f |= (uint32_t)(fits && i0 + q < seg_hi && cq == bpiv) << q;
          }
        }
        if (!__any_sync(0xffffffffu, f != 0u)) continue;
        const uint32_t mine = (uint32_t)__popc(f);
        uint32_t incl = mine;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        uint32_t base_slot = 0;
        if (lane == 31) base_slot = atomicAdd(&s_nlist, incl);
        uint32_t pos = __shfl_sync(0xffffffffu, base_slot, 31) + incl - mine;
        while (f) {
          const int q = __ffs(f) - 1;
          f &= f - 1u;
          s_lkey[pos] = score_key(__ldg(src + i0 + q));
          s_lidx[pos] = i0 + q;
          ++pos;
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
      if (lane == 0) s_wa[warp] = a;
    }
    __syncthreads();

    if (fits) {
      // ---- exact top kr of the list in (key desc, column asc) order
      if (cnt <= 32) {
        if (warp == 0) {
          const bool have = lane < (int)cnt;
          const uint32_t key = have ? s_lkey[lane] : 0u;
          const int32_t col = have ? s_lidx[lane] : 0;
          uint32_t rank = 0;
          for (int j = 0; j < (int)cnt; ++j) {
            const uint32_t kj = __shfl_sync(0xffffffffu, key, j);
            const int32_t cj = __shfl_sync(0xffffffffu, col, j);
            rank += (kj > key || (kj == key && cj < col)) ? 1u : 0u;
          }
          if (have) s_code[col] = rank < kr ? kTk2Sel : (uint16_t)0;
          if (have && rank < kr) atomicAdd(&s_wa[col / seg], 1u);
        }
      } else if (cnt <= (uint32_t)kTk2Threads) {
        const int t = threadIdx.x;
        if (t < (int)cnt) {
          const uint32_t key = s_lkey[t];
          const int32_t col = s_lidx[t];
          uint32_t rank = 0;
          for (int j = 0; j < (int)cnt; ++j) {
            const uint32_t kj = s_lkey[j];
            rank += (kj > key || (kj == key && s_lidx[j] < col)) ? 1u : 0u;
          }
          s_code[col] = rank < kr ? kTk2Sel : (uint16_t)0;
          if (rank < kr) atomicAdd(&s_wa[col / seg], 1u);
        }
      } else {
        if (threadIdx.x == 0) { s_st.prefix = 0u; s_st.mask = 0u; s_st.kr = kr; }
        __syncthreads();
        tk2_radix<kTk2Threads>([&](int c, uint32_t* key) { *key = s_lkey[c]; return true; }, (int)cnt, s_hist, &s_st,
                               s_warp, &s_total, &s_bincnt);
        const uint32_t T = s_st.prefix, rT = s_st.kr;  // keep every key > T and the rT lowest columns of T
        for (int c = threadIdx.x; c < (int)cnt; c += kTk2Threads) {
          const uint32_t key = s_lkey[c];
          const int32_t col = s_lidx[c];
          bool sel = key > T;
          if (key == T) {
            uint32_t before = 0;
            for (int j = 0; j < (int)cnt; ++j) before += (s_lkey[j] == T && s_lidx[j] < col) ? 1u : 0u;
            sel = before < rT;
          }
          s_code[col] = sel ? kTk2Sel : (uint16_t)0;
          if (sel) atomicAdd(&s_wa[col / seg], 1u);
        }
      }
    } else {
      // ---- the pivot bucket overflows the list: exact key over the row
      // (scores of the pivot bucket re-read from global memory)
      if (threadIdx.x == 0) { s_st.prefix = 0u; s_st.mask = 0u; s_st.kr = kr; }
      __syncthreads();
      tk2_radix<kTk2Threads>(
          [&](int c, uint32_t* key) {
            if (s_code[c] != bpiv) return false;
            *key = score_key(__ldg(src + c));
            return true;
          },
          n, s_hist, &s_st, s_warp, &s_total, &s_bincnt);
      const uint32_t T = s_st.prefix, rT = s_st.kr;
      // ties of T per warp segment, in index order
      uint32_t e = 0;
      for (int i = seg_lo + lane; i < seg_hi; i += 32)
        if (s_code[i] == bpiv) e += score_key(__ldg(src + i)) == T;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) e += __shfl_xor_sync(0xffffffffu, e, o);
      if (lane == 0) s_we[warp] = e;
      __syncthreads();
      uint32_t tie_off = 0;
      for (int w = 0; w < warp; ++w) tie_off += s_we[w];
      uint32_t sel_cnt = 0;
      for (int base = seg_lo; base < seg_hi; base += 32) {
        const int i = base + lane;
        const bool in = i < seg_hi && s_code[i] == bpiv;
        const uint32_t key = in ? score_key(__ldg(src + i)) : 0u;
        const bool tie = in && key == T;
        const uint32_t tb = __ballot_sync(0xffffffffu, tie);
        const bool sel = in && (key > T || (tie && tie_off + __popc(tb & ((1u << lane) - 1u)) < rT));
        if (in) s_code[i] = sel ? kTk2Sel : (uint16_t)0;
        sel_cnt += sel;
        tie_off += __popc(tb);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sel_cnt += __shfl_xor_sync(0xffffffffu, sel_cnt, o);
      if (lane == 0) s_wa[warp] += sel_cnt;
    }
    __syncthreads();

    if (has_next) smp_next = sample(src2, n2);         // next row's sample, in flight during the emission
    // ---- emission: the selection is {code > bpiv}, written in index order
    {
      const uint32_t gt2 = half_add(0x7FFFu - bpiv);
      uint32_t pos = 0;
      for (int w = 0; w < warp; ++w) pos += s_wa[w];
      for (int base = seg_lo; base < seg_hi; base += 256) {
        const int i0 = base + 8 * lane;
        uint32_t f = 0;
        if (i0 + 7 < seg_hi) {
          const uint4 c = *reinterpret_cast<const uint4*>(s_code + i0);
          f = pair_bits((c.x + gt2) & kTk2Hi) | (pair_bits((c.y + gt2) & kTk2Hi) << 2) |
              (pair_bits((c.z + gt2) & kTk2Hi) << 4) | (pair_bits((c.w + gt2) & kTk2Hi) << 6);
        } else {
#pragma unroll
          for (int q = 0; q < 8; ++q) f |= (uint32_t)(i0 + q < seg_hi && s_code[i0 + q] > bpiv) << q;
        }
        const uint32_t mine = (uint32_t)__popc(f);
        uint32_t incl = mine;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        uint32_t p = pos + incl - mine;
        while (f) {
          const int q = __ffs(f) - 1;
          f &= f - 1u;
          dst[p++] = mrow ? mrow[i0 + q] : i0 + q;
        }
        pos += __shfl_sync(0xffffffffu, incl, 31);
      }
    }
    __syncthreads();                                    // codes and counters are reused by the next row
  }
}

static bool topk_smem_ok(const float* scores, int n_cols, long long ld) {
  return n_cols <= kMaxCachedKeys && (ld & 3) == 0 && (reinterpret_cast<uintptr_t>(scores) & 15u) == 0;
}

// Rows longer than kMaxCachedKeys, in two exact phases: the top k of every
// 32768-column chunk, then the top k of the union of those (in column order,
// so ties still go to the lower column: an entry that loses inside its chunk
// has k chunk-mates ahead of it in the global order too).
constexpr int kTkChunk = kMaxCachedKeys;
static int topk_long_chunks(int n_cols, int k) {
  if (n_cols <= kMaxCachedKeys || (k & 3) != 0) return 0;     // candidate rows must stay 16-byte aligned
  const int C = (n_cols + kTkChunk - 1) / kTkChunk;
  return (long long)C * k <= kMaxCachedKeys ? C : 0;
}
static size_t topk_long_scratch(int rows, int n_cols, int k) {
  const int C = topk_long_chunks(n_cols, k);
  if (C == 0) return 0;
  auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
  const size_t per = (size_t)rows * C * k * 4;
  return 3 * al(per) + al((size_t)rows * 4);
}

// Union of the chunk selections, compacted in column order: scores, columns
// and the count per row.  One block per (row, chunk); a chunk's offset
// follows from the row's count alone.
__global__ void __launch_bounds__(256)
topk_gather_kernel(const float* __restrict__ scores, long long ld, int n_cols, const int32_t* __restrict__ n_valid,
                   int k, int C, const int32_t* __restrict__ local, float* __restrict__ cs, int32_t* __restrict__ ci,
                   int32_t* __restrict__ cn) {
  const int r = blockIdx.x / C, c = blockIdx.x - (blockIdx.x / C) * C;
  int n = n_cols;
  if (n_valid != nullptr) {
    n = n_valid[r];
    n = n < 0 ? 0 : (n > n_cols ? n_cols : n);
  }
  auto count = [&](int cc) {
    int nc = n - cc * kTkChunk;
    nc = nc < 0 ? 0 : (nc > kTkChunk ? kTkChunk : nc);
    return nc < k ? nc : k;
  };
  int off = 0;
  for (int cc = 0; cc < c; ++cc) off += count(cc);
  const int cnt = count(c);
  const int32_t* lrow = local + ((long long)r * C + c) * k;
  for (int j = threadIdx.x; j < cnt; j += blockDim.x) {
    const int col = c * kTkChunk + lrow[j];
    cs[(long long)r * C * k + off + j] = scores[(long long)r * ld + col];
    ci[(long long)r * C * k + off + j] = col;
  }
  if (c == C - 1 && threadIdx.x == 0) cn[r] = off + cnt;
}

template <int NT>
static cudaError_t launch_topk_smem_nt(const float* scores, int rows, int n_cols, long long ld,
                                       const int32_t* n_valid, int k, int32_t* idx_out, int chunk,
                                       const int32_t* map, long long map_ld, cudaStream_t st, int cap8) {
  const size_t smem = (size_t)(cap8 > 8 ? cap8 : 8) * 2;
  cudaError_t e = cudaFuncSetAttribute(topk_smem_kernel<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kMaxCachedKeys * 2);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148, per_sm = 1;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, topk_smem_kernel<NT>, NT, smem) != cudaSuccess ||
      per_sm < 1)
    per_sm = 1;
  const long long slots = (long long)sms * per_sm;
  const int grid = rows < slots ? rows : (int)slots;
  count_launch();
  topk_smem_kernel<NT><<<grid, NT, smem, st>>>(scores, ld, n_cols, n_valid, k, idx_out, rows, chunk, map, map_ld,
                                               cap8);
  return cudaGetLastError();
}

static cudaError_t launch_topk_smem(const float* scores, int rows, int n_cols, long long ld, const int32_t* n_valid,
                                    int k, int32_t* idx_out, int chunk, const int32_t* map, long long map_ld,
                                    cudaStream_t st, int n_max = -1) {
  const int width = chunk > 0 ? chunk : n_cols;
  const int cap = n_max >= 0 && n_max < width ? n_max : width;   // longest row of this launch
  const int cap8 = (cap + 7) & ~7;
  if (cap8 <= 16384)
    return launch_topk_smem_nt<256>(scores, rows, n_cols, ld, n_valid, k, idx_out, chunk, map, map_ld, st, cap8);
  return launch_topk_smem_nt<512>(scores, rows, n_cols, ld, n_valid, k, idx_out, chunk, map, map_ld, st, cap8);
}

// `scratch` (topk_long_scratch bytes, 256-byte aligned) enables the two-phase
// path for long rows; without it long rows use topk_rows_kernel.
// n_max >= 0: no row of this call has more than n_max valid columns (sizes
// the shared-memory code buffer; -1 = n_cols).
static cudaError_t launch_topk(const float* scores, int rows, int n_cols, long long ld, const int32_t* n_valid,
                               int k, int32_t* idx_out, cudaStream_t st, void* scratch = nullptr,
                               size_t scratch_bytes = 0, int n_max = -1) {
  if (rows == 0) return cudaSuccess;
  if (topk_smem_ok(scores, n_cols, ld))
    return launch_topk_smem(scores, rows, n_cols, ld, n_valid, k, idx_out, 0, nullptr, 0, st, n_max);
  const int C = topk_long_chunks(n_cols, k);
  const size_t need = topk_long_scratch(rows, n_cols, k);
  if (C > 0 && scratch != nullptr && need > 0 && scratch_bytes >= need && (ld & 3) == 0 &&
      (reinterpret_cast<uintptr_t>(scores) & 15u) == 0) {
    auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
    const size_t per = al((size_t)rows * C * k * 4);
    uint8_t* w = reinterpret_cast<uint8_t*>(scratch);
    int32_t* local = reinterpret_cast<int32_t*>(w);
    float* cs = reinterpret_cast<float*>(w + per);
    int32_t* ci = reinterpret_cast<int32_t*>(w + 2 * per);
    int32_t* cn = reinterpret_cast<int32_t*>(w + 3 * per);
    cudaError_t e = launch_topk_smem(scores, rows * C, n_cols, ld, n_valid, k, local, kTkChunk, nullptr, 0, st);
    if (e != cudaSuccess) return e;
    count_launch();
    topk_gather_kernel<<<rows * C, 256, 0, st>>>(scores, ld, n_cols, n_valid, k, C, local, cs, ci, cn);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return launch_topk_smem(cs, rows, C * k, (long long)C * k, cn, k, idx_out, 0, ci, (long long)C * k, st);
  }
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
