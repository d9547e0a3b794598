// KV compression: learned softmax-weighted pooling of a window of tokens into
// one entry, per channel.  CSA: window 2m, stride m; HCA: window = stride = m.
// (DeepSeek-V4 hybrid attention: "深度解析 DeepSeek-V4", CSA Step 1 and HCA.)
//
// HBM-bound streaming kernel.  Each thread owns one 16-byte channel vector of
// one entry and walks the entry's window in chunks of 8 tokens: the chunk's
// 16 loads (kv + gate) are issued together, the chunk max is taken first and
// the running (max, sum, weighted-sum) state is rescaled once per chunk, so a
// token costs one exp per element.  Consecutive entries of a block share
// their overlapping CSA tokens through L1/L2, so DRAM reads each token once.
#pragma once
#include "tc_ptx.cuh"

namespace lcsa {

// Entries j = j0 .. j0+Nc-1 of every sequence; the token buffer holds T rows
// per sequence for positions kv_pos0 .. kv_pos0+T-1 (every token of every
// computed window must be inside it); entry j is written at row j of an
// output of out_rows rows per sequence.
template <typename Tin, typename Tout, bool kPerChannelGate>
__global__ void __launch_bounds__(256)
compress_kernel(const Tin* __restrict__ kv, const Tin* __restrict__ gate, Tout* __restrict__ out,
                int T, int D, int m, int window, int Nc, int entries_per_block,
                const float* __restrict__ rms_w, float rms_eps, long long j0, long long kv_pos0,
                long long out_rows) {
  constexpr int V = Elem<Tin>::kVec;
  const int tpe = D / V;                         // threads per entry
  const int e_local = threadIdx.x / tpe;
  const int c = threadIdx.x - e_local * tpe;     // channel vector index
  const int b = blockIdx.y;
  const int jr = blockIdx.x * entries_per_block + e_local;   // entry relative to j0
  const long long j = j0 + jr;
  extern __shared__ float s_ss[];                // [entries_per_block] sum of squares
  const bool active = (e_local < entries_per_block) && (jr < Nc);
  if (rms_w != nullptr && threadIdx.x < entries_per_block) s_ss[threadIdx.x] = 0.f;

  float acc[V], run_max[V], run_sum[V];
#pragma unroll
  for (int v = 0; v < V; ++v) { acc[v] = 0.f; run_max[v] = -INFINITY; run_sum[v] = 0.f; }

  if (active) {
    const long long hi = (j + 1) * m - kv_pos0;                     // buffer rows
    const long long lo = (j + 1) * m - window > 0 ? (j + 1) * m - window - kv_pos0 : -kv_pos0;
    const Tin* kvb = kv + ((long long)b * T) * D + (long long)c * V;
    const Tin* gb = kPerChannelGate ? gate + ((long long)b * T) * D + (long long)c * V
                                    : gate + (long long)b * T;
    for (long long t0 = lo; t0 < hi; t0 += 8) {
      const int n = (int)((hi - t0) < 8 ? (hi - t0) : 8);
      float x[8][V], g[8][V];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (u < n) {
          load16(kvb + (t0 + u) * D, x[u]);
          if constexpr (kPerChannelGate) {
            load16(gb + (t0 + u) * D, g[u]);
          } else {
            float gs = ld_scalar(gb + t0 + u);
#pragma unroll
            for (int v = 0; v < V; ++v) g[u][v] = gs;
          }
        }
      }
#pragma unroll
      for (int v = 0; v < V; ++v) {
        float cm = run_max[v];
#pragma unroll
        for (int u = 0; u < 8; ++u) if (u < n) cm = fmaxf(cm, g[u][v]);
        const float alpha = __expf(run_max[v] - cm);   // exp(-inf) = 0 on the first chunk
        float a = acc[v] * alpha, s = run_sum[v] * alpha;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          if (u < n) {
            const float p = __expf(g[u][v] - cm);
            s += p;
            a = fmaf(p, x[u][v], a);
          }
        }
        acc[v] = a; run_sum[v] = s; run_max[v] = cm;
      }
    }
#pragma unroll
    for (int v = 0; v < V; ++v) acc[v] = acc[v] / run_sum[v];
  }

  if (rms_w != nullptr) {
    __syncthreads();
    if (active) {
      float ss = 0.f;
#pragma unroll
      for (int v = 0; v < V; ++v) ss = fmaf(acc[v], acc[v], ss);
      atomicAdd(&s_ss[e_local], ss);
    }
    __syncthreads();
    if (active) {
      const float inv = rsqrtf(s_ss[e_local] / (float)D + rms_eps);
#pragma unroll
      for (int v = 0; v < V; ++v) acc[v] = acc[v] * inv * __ldg(rms_w + c * V + v);
    }
  }
  if (active) {
    Tout* o = out + ((long long)b * out_rows + j) * D + (long long)c * V;
    store_vec<V>(o, acc);
  }
}

// ---------------------------------------------------------------------------
// Streaming compressor for whole sequences (per-channel gates, window 2m or m,
// no RMSNorm): token rows reach shared memory by bulk copies.
//
// A CTA (about four per SM) owns a contiguous range of blocks (m tokens each)
// of one sequence and streams their token rows, kCmpRows at a time, through a
// kCmpStages-deep ring:
// one thread issues two cp.async.bulk copies per stage (kv rows, gate rows;
// contiguous in HBM) that complete on the stage's mbarrier, so the bytes in
// flight do not depend on registers or occupancy.  Each thread owns two
// channels of every row and folds the rows in order, up to 4 at a time (one
// rescale by the chunk's maximum), into a per-channel softmax state (running
// max, sum of weights, weighted sum):
//   HCA (window m): the entry is the state of its block;
//   CSA (window 2m): entry j pools blocks j-1 and j, the merge of two
//     neighbouring block states; the range starts one block early so that its
//     first entry has its predecessor.
// Every wait is bounded; a CTA whose wait gave up stops at the same stage on
// all threads (__syncthreads_and), waits (bounded) for its copies in flight
// and leaves.
// ---------------------------------------------------------------------------
constexpr int kCmpRows = 8;        // token rows per stage
constexpr int kCmpStages = 3;      // 48 KB per CTA at D = 512: four CTAs per SM

struct Soft2 {                     // softmax state of 2 channels
  float m[2], s[2], a[2];
  __device__ __forceinline__ void reset() {
    m[0] = m[1] = -INFINITY;
    s[0] = s[1] = a[0] = a[1] = 0.f;
  }
};

// Two consecutive channels of a staged row as FP32.
__device__ __forceinline__ float2 ld2(const __nv_bfloat16* p) {
  return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
}
__device__ __forceinline__ float2 ld2(const float* p) { return *reinterpret_cast<const float2*>(p); }

// Fold rows r .. r+n-1 (n <= 4) of a staged tile into st.
template <typename Tin>
__device__ __forceinline__ void fold_rows(Soft2& st, const Tin* kvs, const Tin* gs, int D, int r, int n) {
  float2 x[4], g[4];
#pragma unroll
  for (int u = 0; u < 4; ++u)
    if (u < n) {
      x[u] = ld2(kvs + (r + u) * D);
      g[u] = ld2(gs + (r + u) * D);
    }
#pragma unroll
  for (int v = 0; v < 2; ++v) {
    float cm = st.m[v];
#pragma unroll
    for (int u = 0; u < 4; ++u) if (u < n) cm = fmaxf(cm, v ? g[u].y : g[u].x);
    const float alpha = __expf(st.m[v] - cm);          // 0 while the state is empty
    float a = st.a[v] * alpha, sm = st.s[v] * alpha;
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (u < n) {
        const float p = __expf((v ? g[u].y : g[u].x) - cm);
        sm += p;
        a = fmaf(p, v ? x[u].y : x[u].x, a);
      }
    st.m[v] = cm; st.s[v] = sm; st.a[v] = a;
  }
}

// 2^x on the MUFU (flushes results below 2^-126 to zero: such weights are
// negligible next to the chunk maximum's weight of 1).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// a BF16 pair (channel c in the low half) as a packed FP32 pair
__device__ __forceinline__ f2x bf2f2(uint32_t w) { return pk2(bf_lo(w), bf_hi(w)); }

// Weights of 4 rows against the chunk reference -m log2e (ncml2) folded into
// (s2, a2): p = exp2(g log2e - m log2e), s += p, a += p x.
__device__ __forceinline__ void fold4_core(const uint32_t* x, const uint32_t* g, f2x ncml2, f2x& s2, f2x& a2) {
  constexpr float kL2e = 1.4426950408889634f;
  const f2x l2e2 = pk2(kL2e, kL2e);
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const float2 t = upk2(fma2(bf2f2(g[u]), l2e2, ncml2));
    const f2x p2 = pk2(ex2(t.x), ex2(t.y));
    s2 = add2(s2, p2);
    a2 = fma2(p2, bf2f2(x[u]), a2);
  }
}

__device__ __forceinline__ void load4_bf16(const __nv_bfloat16* kvs, const __nv_bfloat16* gs, int D, int r,
                                           uint32_t* x, uint32_t* g, uint32_t* mw) {
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    x[u] = *reinterpret_cast<const uint32_t*>(kvs + (r + u) * D);
    g[u] = *reinterpret_cast<const uint32_t*>(gs + (r + u) * D);
  }
  const __nv_bfloat162 m2 = __hmax2(__hmax2(*reinterpret_cast<const __nv_bfloat162*>(&g[0]),
                                            *reinterpret_cast<const __nv_bfloat162*>(&g[1])),
                                    __hmax2(*reinterpret_cast<const __nv_bfloat162*>(&g[2]),
                                            *reinterpret_cast<const __nv_bfloat162*>(&g[3])));
  *mw = *reinterpret_cast<const uint32_t*>(&m2);
}

// Fold rows r .. r+3 of a staged BF16 tile into st: the common chunk (4 rows
// of one block).  The chunk maximum of both channels is one packed BF16 max
// tree (exact); each weight is exp2(g log2e - m log2e).
__device__ __forceinline__ void fold4_bf16(Soft2& st, const __nv_bfloat16* kvs, const __nv_bfloat16* gs, int D,
                                           int r) {
  uint32_t x[4], g[4], mw;
  load4_bf16(kvs, gs, D, r, x, g, &mw);
  constexpr float kL2e = 1.4426950408889634f;
  const float cm0 = fmaxf(st.m[0], bf_lo(mw)), cm1 = fmaxf(st.m[1], bf_hi(mw));
  // 0 while the state is empty (m = -inf)
  const f2x al2 = pk2(ex2((st.m[0] - cm0) * kL2e), ex2((st.m[1] - cm1) * kL2e));
  f2x s2 = mul2(pk2(st.s[0], st.s[1]), al2), a2 = mul2(pk2(st.a[0], st.a[1]), al2);
  fold4_core(x, g, pk2(-cm0 * kL2e, -cm1 * kL2e), s2, a2);
  const float2 sf = upk2(s2), af = upk2(a2);
  st.s[0] = sf.x; st.s[1] = sf.y; st.a[0] = af.x; st.a[1] = af.y;
  st.m[0] = cm0; st.m[1] = cm1;
}

// A whole block of 4 rows into an empty state (m = 4): no rescale.
__device__ __forceinline__ void block4_bf16(Soft2& st, const __nv_bfloat16* kvs, const __nv_bfloat16* gs, int D,
                                            int r) {
  uint32_t x[4], g[4], mw;
  load4_bf16(kvs, gs, D, r, x, g, &mw);
  constexpr float kL2e = 1.4426950408889634f;
  const float cm0 = bf_lo(mw), cm1 = bf_hi(mw);
  f2x s2 = 0ull, a2 = 0ull;                                         // +0.0 in both lanes
  fold4_core(x, g, pk2(-cm0 * kL2e, -cm1 * kL2e), s2, a2);
  const float2 sf = upk2(s2), af = upk2(a2);
  st.s[0] = sf.x; st.s[1] = sf.y; st.a[0] = af.x; st.a[1] = af.y;
  st.m[0] = cm0; st.m[1] = cm1;
}
__device__ __forceinline__ void fold4(Soft2& st, const __nv_bfloat16* kvs, const __nv_bfloat16* gs, int D, int r) {
  fold4_bf16(st, kvs, gs, D, r);
}
__device__ __forceinline__ void block4(Soft2& st, const __nv_bfloat16* kvs, const __nv_bfloat16* gs, int D, int r) {
  block4_bf16(st, kvs, gs, D, r);
}
__device__ __forceinline__ void block4(Soft2& st, const float* kvs, const float* gs, int D, int r) {
  fold_rows<float>(st, kvs, gs, D, r, 4);
}
__device__ __forceinline__ void fold4(Soft2& st, const float* kvs, const float* gs, int D, int r) {
  fold_rows<float>(st, kvs, gs, D, r, 4);
}

// CSA with m = 4 on BF16 rows: the packed state of one block of 4 rows
// (both channels), with the block maximum kept as -m log2e, the reference
// its weights were taken against.
struct Blk2 {
  f2x nml2, s2, a2;
  __device__ __forceinline__ void reset() {       // empty: m = -inf, s = a = 0
    nml2 = pk2(INFINITY, INFINITY);
    s2 = a2 = 0ull;
  }
};
__device__ __forceinline__ void block4_packed(Blk2& st, const __nv_bfloat16* kvs, const __nv_bfloat16* gs, int D,
                                              int r) {
  uint32_t x[4], g[4], mw;
  load4_bf16(kvs, gs, D, r, x, g, &mw);
  constexpr float kL2e = 1.4426950408889634f;
  st.nml2 = mul2(pk2(bf_lo(mw), bf_hi(mw)), pk2(-kL2e, -kL2e));
  st.s2 = st.a2 = 0ull;
  fold4_core(x, g, st.nml2, st.s2, st.a2);
}
// Fold the 8 rows of a stage into a running packed state (HCA blocks of a
// multiple of 8 rows): one packed BF16 max tree over the 8 gate rows, one
// rescale of the state to the new maximum (0 while the state is empty), then
// the weights of the 8 rows against it.
__device__ __forceinline__ void fold8_packed(Blk2& st, const __nv_bfloat16* kvs, const __nv_bfloat16* gs, int D) {
  uint32_t x[8], g[8], mlo, mhi;
  load4_bf16(kvs, gs, D, 0, x, g, &mlo);
  load4_bf16(kvs, gs, D, 4, x + 4, g + 4, &mhi);
  const __nv_bfloat162 m2 = __hmax2(*reinterpret_cast<const __nv_bfloat162*>(&mlo),
                                    *reinterpret_cast<const __nv_bfloat162*>(&mhi));
  const uint32_t mw = *reinterpret_cast<const uint32_t*>(&m2);
  constexpr float kL2e = 1.4426950408889634f;
  const float2 cn = upk2(mul2(pk2(bf_lo(mw), bf_hi(mw)), pk2(-kL2e, -kL2e)));
  const float2 on = upk2(st.nml2);
  const f2x nml = pk2(fminf(on.x, cn.x), fminf(on.y, cn.y));   // the larger maximum
  const float2 df = upk2(fma2(st.nml2, pk2(-1.f, -1.f), nml));   // (m_old - m_new) log2e <= 0
  const f2x al2 = pk2(ex2(df.x), ex2(df.y));
  st.s2 = mul2(st.s2, al2);
  st.a2 = mul2(st.a2, al2);
  st.nml2 = nml;
  fold4_core(x, g, nml, st.s2, st.a2);
  fold4_core(x + 4, g + 4, nml, st.s2, st.a2);
}

// CSA entry of blocks (prev, cur) per channel: the block with the larger
// maximum weighs 1, the other exp2(-|dm| log2e) (0 when prev is empty).
__device__ __forceinline__ float2 csa_merge_packed(const Blk2& p, const Blk2& c) {
  const float2 d = upk2(fma2(p.nml2, pk2(-1.f, -1.f), c.nml2));     // (m_prev - m_cur) log2e
  const float f0 = ex2(-fabsf(d.x)), f1 = ex2(-fabsf(d.y));
  const bool p0 = d.x > 0.f, p1 = d.y > 0.f;
  const f2x fa = pk2(p0 ? 1.f : f0, p1 ? 1.f : f1), fb = pk2(p0 ? f0 : 1.f, p1 ? f1 : 1.f);
  const float2 num = upk2(fma2(p.a2, fa, mul2(c.a2, fb)));
  const float2 den = upk2(fma2(p.s2, fa, mul2(c.s2, fb)));
  return make_float2(__fdividef(num.x, den.x), __fdividef(num.y, den.y));
}

// Two output channels in one store.
__device__ __forceinline__ void st_pair(float* p, float a, float b) { *reinterpret_cast<float2*>(p) = make_float2(a, b); }
__device__ __forceinline__ void st_pair(__nv_bfloat16* p, float a, float b) {
  *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(a, b);
}

// Warp roles: warps 0 .. nw-1 fold (one channel pair per thread), warp nw
// issues the bulk copies.  Stage k lives in slot k % kCmpStages; `full` of a
// slot completes when its copies land, `empty` when every folding warp has
// arrived (one arrival per warp) after reading it.
constexpr int kCmpMaxThreads = 256 + 32;   // D <= 512: up to 8 folding warps and the copy warp

template <typename Tin, typename Tout, bool kCSA>
__global__ void __launch_bounds__(kCmpMaxThreads, 4)
compress_bulk_kernel(const Tin* __restrict__ kv, const Tin* __restrict__ gate, Tout* __restrict__ out, int T, int D,
                     int m, int Nc, int blocks_per_unit, int units_per_seq) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  const uint32_t row_bytes = (uint32_t)D * sizeof(Tin);
  const uint32_t tile_bytes = kCmpRows * row_bytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kCmpStages * 2 * tile_bytes);
  uint64_t* empty = full + kCmpStages;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nw = (int)(blockDim.x >> 5) - 1;                          // folding warps
  const int b = blockIdx.x / units_per_seq;
  const int unit = blockIdx.x - b * units_per_seq;
  const int jb = unit * blocks_per_unit;                              // first entry of this CTA
  const int je = jb + blocks_per_unit < Nc ? jb + blocks_per_unit : Nc;
  if (jb >= je) return;                                               // uniform over the CTA
  const int first = (kCSA && jb > 0) ? jb - 1 : jb;                   // first block streamed
  const long long ta = (long long)first * m;                          // first token row
  const int rows = (je - first) * m;
  const int K = (rows + kCmpRows - 1) / kCmpRows;                     // stages
  if (tid == 0) {
    for (int s = 0; s < kCmpStages; ++s) {
      tc::mbar_init(full + s, 1);
      tc::mbar_init(empty + s, nw);
    }
    tc::fence_barrier_init();
  }
  __syncthreads();

  if (warp == nw) {
    // ---------------------------------------------------------------- copies
    if (lane == 0) {
      const Tin* kvb = kv + ((long long)b * T + ta) * D;
      const Tin* gb = gate + ((long long)b * T + ta) * D;
      int k = 0;
      for (; k < K; ++k) {
        const int slot = k % kCmpStages;
        if (k >= kCmpStages && !tc::mbar_wait(empty + slot, ((k / kCmpStages) - 1) & 1)) break;
        const int r0 = k * kCmpRows;
        const int n = rows - r0 < kCmpRows ? rows - r0 : kCmpRows;
        uint8_t* dst = smem + slot * 2 * tile_bytes;
        tc::mbar_arrive_expect_tx(full + slot, 2u * n * row_bytes);
        tc::bulk_load(dst, kvb + (long long)r0 * D, n * row_bytes, full + slot);
        tc::bulk_load(dst + tile_bytes, gb + (long long)r0 * D, n * row_bytes, full + slot);
      }
      // every copy issued lands before the CTA may leave
      for (int q = k - kCmpStages > 0 ? k - kCmpStages : 0; q < k; ++q)
        tc::mbar_wait(full + q % kCmpStages, (q / kCmpStages) & 1);
    }
    return;
  }

  // ------------------------------------------------------------------ folding
  const int c = 2 * tid;                                              // this thread's channels c, c+1
  const bool has = c < D;
  if constexpr (kCSA && sizeof(Tin) == 2 && kCmpRows == 8) {
    if (m == 4) {
      // Blocks of 4 rows, two per stage (streaming starts on a block
      // boundary): each block folds into one of two states that take turns
      // as the current and the previous block, so an entry is one merge.
      const __nv_bfloat16* kvb16 = reinterpret_cast<const __nv_bfloat16*>(smem) + c;
      Blk2 s0, s1;
      s1.reset();                                                     // the block before `first`: empty
      const int nblk = je - first;
      for (int k = 0; k < K; ++k) {
        const int slot = k % kCmpStages;
        if (!__all_sync(0xffffffffu, tc::mbar_wait(full + slot, (k / kCmpStages) & 1))) break;
        const __nv_bfloat16* kvs = kvb16 + slot * 2 * tile_bytes / 2;
        const __nv_bfloat16* gs = kvs + tile_bytes / 2;
        const int q0 = 2 * k;                                         // block index within the range
        if (has) {
          block4_packed(s0, kvs, gs, D, 0);
          if (first + q0 >= jb) {
            const float2 o = csa_merge_packed(s1, s0);
            st_pair(out + ((long long)b * Nc + first + q0) * D + c, o.x, o.y);
          }
          if (q0 + 1 < nblk) {
            block4_packed(s1, kvs, gs, D, 4);
            const float2 o = csa_merge_packed(s0, s1);               // block first + q0 + 1 >= jb
            st_pair(out + ((long long)b * Nc + first + q0 + 1) * D + c, o.x, o.y);
          }
        }
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(empty + slot);                 // this warp is done with the slot
      }
      return;
    }
  }
  if constexpr (!kCSA && sizeof(Tin) == 2 && kCmpRows == 8) {
    if (m % kCmpRows == 0) {
      // HCA blocks of a multiple of 8 rows start on stage boundaries: one
      // fold per stage, an entry every m / 8 stages.
      const __nv_bfloat16* kvb16 = reinterpret_cast<const __nv_bfloat16*>(smem) + c;
      const int spb = m / kCmpRows;                                   // stages per block
      Blk2 st;
      st.reset();
      int blk = jb, in_blk = 0;
      for (int k = 0; k < K; ++k) {
        const int slot = k % kCmpStages;
        if (!__all_sync(0xffffffffu, tc::mbar_wait(full + slot, (k / kCmpStages) & 1))) break;
        const __nv_bfloat16* kvs = kvb16 + slot * 2 * tile_bytes / 2;
        if (has) fold8_packed(st, kvs, kvs + tile_bytes / 2, D);
        if (++in_blk == spb) {
          if (has) {
            const float2 a = upk2(st.a2), sm = upk2(st.s2);
            st_pair(out + ((long long)b * Nc + blk) * D + c, __fdividef(a.x, sm.x), __fdividef(a.y, sm.y));
          }
          st.reset();
          in_blk = 0;
          ++blk;
        }
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(empty + slot);                 // this warp is done with the slot
      }
      return;
    }
  }
  Soft2 st, prev;
  st.reset();
  prev.reset();
  int blk = first, pos = 0;                                           // current block, rows of it folded
  for (int k = 0; k < K; ++k) {
    const int slot = k % kCmpStages;
    if (!__all_sync(0xffffffffu, tc::mbar_wait(full + slot, (k / kCmpStages) & 1))) break;
    const Tin* kvs = reinterpret_cast<const Tin*>(smem + slot * 2 * tile_bytes) + c;
    const Tin* gs = reinterpret_cast<const Tin*>(smem + slot * 2 * tile_bytes + tile_bytes) + c;
    const int r1 = rows - k * kCmpRows < kCmpRows ? rows - k * kCmpRows : kCmpRows;
    for (int r = 0; r < r1;) {
      int n = r1 - r < 4 ? r1 - r : 4;
      n = m - pos < n ? m - pos : n;                                  // a chunk stays inside its block
      if (has) {
        if (n == 4) {
          if (pos == 0 && m == 4) block4(st, kvs, gs, D, r);          // the state is empty
          else fold4(st, kvs, gs, D, r);
        } else {
          fold_rows<Tin>(st, kvs, gs, D, r, n);
        }
      }
      r += n;
      pos += n;
      if (pos == m) {                                                 // block `blk` complete
        if (has && blk >= jb) {
          constexpr float kL2e = 1.4426950408889634f;
          float o[2];
#pragma unroll
          for (int v = 0; v < 2; ++v) {
            if (kCSA) {                                               // entry 0: prev is empty
              // one weight is 1 (the block with the larger max), the other exp2(-|dm| log2e)
              const float d = (prev.m[v] - st.m[v]) * kL2e;
              const float f = ex2(-fabsf(d));                         // 0 when prev is empty
              const bool pa = d > 0.f;
              const float fa = pa ? 1.f : f, fb = pa ? f : 1.f;
              o[v] = __fdividef(fmaf(prev.a[v], fa, st.a[v] * fb), fmaf(prev.s[v], fa, st.s[v] * fb));
            } else {
              o[v] = __fdividef(st.a[v], st.s[v]);
            }
          }
          st_pair(out + ((long long)b * Nc + blk) * D + c, o[0], o[1]);
        }
        if (kCSA) prev = st;
        st.reset();
        pos = 0;
        ++blk;
      }
    }
    __syncwarp();
    if (lane == 0) tc::mbar_arrive(empty + slot);                     // this warp is done with the slot
  }
}

// Whole-sequence CSA (window 2m) or HCA (window m) compression with
// per-channel gates and no RMSNorm on the bulk-copy kernel.  Returns false
// when the shape does not fit it (odd D, D > 512, or a stage ring above
// 200 KB of shared memory).
template <typename Tin, typename Tout>
static bool launch_compress_bulk(const void* kv, const void* gate, int B, int T, int D, int m, int window,
                                 void* out, cudaStream_t st, cudaError_t* err) {
  if ((D & 1) || D / 2 + 32 > kCmpMaxThreads || (window != m && window != 2 * m)) return false;
  const int Nc = T / m;
  // about four CTAs per SM, each a contiguous range of blocks of one sequence
  const int want = (4 * sm_count() + B - 1) / B;
  int ups = Nc < want ? Nc : want;
  const int bpu = (Nc + ups - 1) / ups;
  ups = (Nc + bpu - 1) / bpu;
  const size_t smem = 128 + (size_t)kCmpStages * 2 * kCmpRows * D * sizeof(Tin) + kCmpStages * 16;
  if (smem > 200 * 1024) return false;
  const int threads = ((D / 2 + 31) / 32) * 32 + 32;                  // folding warps + the copy warp
  auto kern = window == 2 * m ? compress_bulk_kernel<Tin, Tout, true> : compress_bulk_kernel<Tin, Tout, false>;
  *err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (*err != cudaSuccess) return true;
  count_launch();
  kern<<<B * ups, threads, smem, st>>>((const Tin*)kv, (const Tin*)gate, (Tout*)out, T, D, m, Nc, bpu, ups);
  *err = cudaGetLastError();
  return true;
}

template <typename Tin, typename Tout>
static cudaError_t launch_compress_t(const void* kv, const void* gate, int per_channel, int B, int T, int D,
                                     int m, int window, const float* rms_w, float rms_eps, void* out,
                                     cudaStream_t st, long long j0 = 0, int n_entries = -1, long long kv_pos0 = 0,
                                     long long out_rows = -1) {
  constexpr int V = Elem<Tin>::kVec;
  const int Nc = n_entries >= 0 ? n_entries : T / m;
  if (out_rows < 0) out_rows = Nc;
  if (Nc == 0 || B == 0) return cudaSuccess;
  if (per_channel && rms_w == nullptr && j0 == 0 && n_entries < 0 && kv_pos0 == 0) {
    cudaError_t e;
    if (launch_compress_bulk<Tin, Tout>(kv, gate, B, T, D, m, window, out, st, &e)) return e;
  }
  const int tpe = D / V;
  int epb = 256 / tpe;
  if (epb < 1) epb = 1;
  const int threads = epb * tpe <= 1024 ? (epb * tpe < 32 ? 32 : epb * tpe) : 1024;
  dim3 grid((Nc + epb - 1) / epb, B);
  const size_t smem = rms_w ? (size_t)epb * sizeof(float) : 0;
  count_launch();
  if (per_channel)
    compress_kernel<Tin, Tout, true><<<grid, threads, smem, st>>>(
        (const Tin*)kv, (const Tin*)gate, (Tout*)out, T, D, m, window, Nc, epb, rms_w, rms_eps, j0, kv_pos0,
        out_rows);
  else
    compress_kernel<Tin, Tout, false><<<grid, threads, smem, st>>>(
        (const Tin*)kv, (const Tin*)gate, (Tout*)out, T, D, m, window, Nc, epb, rms_w, rms_eps, j0, kv_pos0,
        out_rows);
  return cudaGetLastError();
}

static cudaError_t launch_compress(const void* kv, const void* gate, int per_channel, int B, int T, int D,
                                   int m, int window, lcsa_dtype dt, const float* rms_w, float rms_eps,
                                   void* out, lcsa_dtype odt, cudaStream_t st, long long j0 = 0,
                                   int n_entries = -1, long long kv_pos0 = 0, long long out_rows = -1) {
  if (dt == LCSA_BF16) {
    if (odt == LCSA_BF16)
      return launch_compress_t<__nv_bfloat16, __nv_bfloat16>(kv, gate, per_channel, B, T, D, m, window, rms_w,
                                                             rms_eps, out, st, j0, n_entries, kv_pos0, out_rows);
    return launch_compress_t<__nv_bfloat16, float>(kv, gate, per_channel, B, T, D, m, window, rms_w, rms_eps, out,
                                                   st, j0, n_entries, kv_pos0, out_rows);
  }
  if (odt == LCSA_BF16)
    return launch_compress_t<float, __nv_bfloat16>(kv, gate, per_channel, B, T, D, m, window, rms_w, rms_eps, out,
                                                   st, j0, n_entries, kv_pos0, out_rows);
  return launch_compress_t<float, float>(kv, gate, per_channel, B, T, D, m, window, rms_w, rms_eps, out, st, j0,
                                         n_entries, kv_pos0, out_rows);
}

}  // namespace lcsa
