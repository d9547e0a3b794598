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
#include "common.cuh"

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
// Streaming compressor for whole sequences (window 2m or m, no RMSNorm).
//
// Each thread owns 4 channels and walks a stream of tokens 4 at a time (a
// chunk): raw 8-byte (BF16) or 16-byte (FP32) vectors of kv and gate, the next
// chunk's loads issued before the current chunk is reduced.  A block of m
// tokens folds into a per-channel softmax state (running max, sum of weights,
// weighted sum): one exp per element plus one rescale per chunk.
//   CSA (window 2m): entry j pools blocks j-1 and j, so it is the merge of
//     two neighbouring block states; a thread walks kCsaRun consecutive
//     blocks (plus the block before them) and emits one entry per block.
//   HCA (window m): the lanes of a CTA split a block's m tokens, and their
//     states merge through shared memory.
// A warp reads 256 contiguous bytes of a token row per load (32 threads x 8
// bytes); the CTA covers whole rows.  The grid is persistent (two CTAs of 256
// threads per SM) and strides over work units.
// ---------------------------------------------------------------------------
constexpr int kCsaRun = 16;          // CSA blocks per thread
constexpr int kStreamThreads = 256;

template <typename Tin> struct Raw4;                      // 4 channels of one token
template <> struct Raw4<__nv_bfloat16> { using T = uint2; };
template <> struct Raw4<float> { using T = float4; };

// Channel v (0..3) of a raw 4-channel vector as FP32 (a BF16 value is the
// high half of its FP32 bit pattern).
__device__ __forceinline__ float chan(const uint2& r, int v) {
  const uint32_t w = v < 2 ? r.x : r.y;
  return __uint_as_float((v & 1) ? (w & 0xffff0000u) : (w << 16));
}
__device__ __forceinline__ float chan(const float4& r, int v) {
  return v == 0 ? r.x : (v == 1 ? r.y : (v == 2 ? r.z : r.w));
}

struct Soft4 {                 // softmax state of 4 channels
  float m[4], s[4], a[4];
  __device__ __forceinline__ void reset() {
#pragma unroll
    for (int v = 0; v < 4; ++v) { m[v] = -INFINITY; s[v] = 0.f; a[v] = 0.f; }
  }
};

// One chunk of a thread's token stream: n (<= 4) tokens from token t.
template <typename Tin, bool kPC>
struct Chunk4 {
  typename Raw4<Tin>::T x[4], g[4];
  float gs[4];                 // scalar gates (kPC = false)
  __device__ __forceinline__ void load(const typename Raw4<Tin>::T* kvp, const typename Raw4<Tin>::T* gp,
                                       const Tin* gsp, long long t, int n, int tpr) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (u < n) {
        x[u] = __ldg(kvp + (t + u) * tpr);
        if constexpr (kPC) g[u] = __ldg(gp + (t + u) * tpr);
        else gs[u] = ld_scalar(gsp + t + u);
      }
    }
  }
  // fold the chunk's n tokens into st: one rescale by the chunk maximum;
  // channel by channel, each value converted where it is used
  __device__ __forceinline__ void fold(Soft4& st, int n) const {
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      float cm = st.m[v];
#pragma unroll
      for (int u = 0; u < 4; ++u) if (u < n) cm = fmaxf(cm, gate_at(u, v));
      const float alpha = __expf(st.m[v] - cm);        // 0 while the state is empty
      float a = st.a[v] * alpha, sm = st.s[v] * alpha;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (u < n) {
          const float p = __expf(gate_at(u, v) - cm);
          sm += p;
          a = fmaf(p, chan(x[u], v), a);
        }
      }
      st.m[v] = cm; st.s[v] = sm; st.a[v] = a;
    }
  }
  __device__ __forceinline__ float gate_at(int u, int v) const {
    if constexpr (kPC) return chan(g[u], v);
    else return gs[u];
  }
};

// Pooled value of the union of two states' tokens (A may be empty).
__device__ __forceinline__ void merge_out(const Soft4& A, const Soft4& B, float* o) {
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    const float M = fmaxf(A.m[v], B.m[v]);
    const float fa = __expf(A.m[v] - M), fb = __expf(B.m[v] - M);
    o[v] = (A.a[v] * fa + B.a[v] * fb) / (A.s[v] * fa + B.s[v] * fb);
  }
}

// Walk nb blocks of `bl` tokens starting at token t0 in chunks of 4 tokens;
// two chunk buffers alternate, so the next chunk's loads are in flight while
// the current one is folded.  on_block(k, state) runs after block k.
template <typename Tin, bool kPC, typename F>
__device__ __forceinline__ void walk_blocks(const typename Raw4<Tin>::T* kvp, const typename Raw4<Tin>::T* gp,
                                            const Tin* gsp, int tpr, long long t0, int nb, int bl, F&& on_block) {
  if (nb <= 0 || bl <= 0) return;
  const int cpb = (bl + 3) >> 2;
  const int nq = nb * cpb;
  Chunk4<Tin, kPC> ca, cb;
  Soft4 st;
  st.reset();
  int k = 0, w = 0;                  // block and chunk-in-block of the chunk being folded
  int kl = 0, wl = 0;                // ... of the next chunk to load
  auto load = [&](Chunk4<Tin, kPC>& c) {
    const int n = bl - 4 * wl < 4 ? bl - 4 * wl : 4;
    c.load(kvp, gp, gsp, t0 + (long long)kl * bl + 4 * wl, n, tpr);
    if (++wl == cpb) { wl = 0; ++kl; }
  };
  auto fold = [&](const Chunk4<Tin, kPC>& c) {
    const int n = bl - 4 * w < 4 ? bl - 4 * w : 4;
    c.fold(st, n);
    if (++w == cpb) {
      on_block(k, st);
      st.reset();
      w = 0;
      ++k;
    }
  };
  load(ca);
  for (int q = 0; q < nq; q += 2) {
    if (q + 1 < nq) load(cb);
    fold(ca);
    if (q + 1 < nq) {
      if (q + 2 < nq) load(ca);
      fold(cb);
    }
  }
}

template <typename Tin, typename Tout, bool kPC, bool kCSA>
__global__ void __launch_bounds__(kStreamThreads, 2)
compress_stream_kernel(const Tin* __restrict__ kv, const Tin* __restrict__ gate, Tout* __restrict__ out, int T, int D,
                       int m, int Nc, int units_per_seq, long long n_units) {
  using R = typename Raw4<Tin>::T;
  const int tpr = D >> 2;                          // threads per token row
  const int nl = blockDim.x / tpr;                 // lanes (token streams) per CTA
  const int c = threadIdx.x % tpr, l = threadIdx.x / tpr;
  extern __shared__ float s_part[];                // HCA: [nl][tpr][12] lane states
  for (long long u = blockIdx.x; u < n_units; u += gridDim.x) {
    const int b = (int)(u / units_per_seq);
    const int r = (int)(u - (long long)b * units_per_seq);
    const R* kvp = reinterpret_cast<const R*>(kv + (long long)b * T * D) + c;
    const R* gp = kPC ? reinterpret_cast<const R*>(gate + (long long)b * T * D) + c : nullptr;
    const Tin* gsp = kPC ? nullptr : gate + (long long)b * T;
    Tout* ob = out + (long long)b * Nc * D + c * 4;
    if constexpr (kCSA) {
      if (l >= nl) continue;
      const int jb = (r * nl + l) * kCsaRun;
      const int je = jb + kCsaRun < Nc ? jb + kCsaRun : Nc;
      if (jb >= je) continue;
      const int first = jb > 0 ? jb - 1 : 0;       // the block before the run feeds entry jb
      Soft4 prev;
      prev.reset();
      walk_blocks<Tin, kPC>(kvp, gp, gsp, tpr, (long long)first * m, je - first, m, [&](int k, const Soft4& st) {
        const int j = first + k;
        if (j >= jb) {
          float o[4];
          merge_out(prev, st, o);                  // entry 0: prev is empty
          store_vec<4>(ob + (long long)j * D, o);
        }
        prev = st;
      });
    } else {
      // block r, lanes split its m tokens
      const int L = (m + nl - 1) / nl;
      const int lo = l * L < m ? l * L : m;
      const int hi = lo + L < m ? lo + L : m;
      Soft4 part;
      part.reset();
      if (l < nl)
        walk_blocks<Tin, kPC>(kvp, gp, gsp, tpr, (long long)r * m + lo, 1, hi - lo,
                              [&](int, const Soft4& st) { part = st; });
      if (l < nl) {
        float* sp = s_part + ((long long)l * tpr + c) * 12;
#pragma unroll
        for (int v = 0; v < 4; ++v) { sp[v] = part.m[v]; sp[4 + v] = part.s[v]; sp[8 + v] = part.a[v]; }
      }
      __syncthreads();
      if (l == 0) {
        Soft4 acc = part;
        for (int q = 1; q < nl; ++q) {
          const float* sp = s_part + ((long long)q * tpr + c) * 12;
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const float M = fmaxf(acc.m[v], sp[v]);
            if (M == -INFINITY) continue;          // both empty
            const float fa = __expf(acc.m[v] - M), fb = __expf(sp[v] - M);
            acc.s[v] = acc.s[v] * fa + sp[4 + v] * fb;
            acc.a[v] = acc.a[v] * fa + sp[8 + v] * fb;
            acc.m[v] = M;
          }
        }
        float o[4];
#pragma unroll
        for (int v = 0; v < 4; ++v) o[v] = acc.a[v] / acc.s[v];
        store_vec<4>(ob + (long long)r * D, o);
      }
      __syncthreads();                             // s_part is reused by the next unit
    }
  }
}

// Whole-sequence CSA (window 2m) or HCA (window m) compression without
// RMSNorm on the streaming kernel.  Returns false when the shape needs the
// per-entry kernel (D not a multiple of 4 or wider than 4 x 256 channels).
template <typename Tin, typename Tout>
static bool launch_compress_stream(const void* kv, const void* gate, int per_channel, int B, int T, int D, int m,
                                   int window, void* out, cudaStream_t st, cudaError_t* err) {
  const int tpr = D / 4;
  if (D % 4 != 0 || tpr > kStreamThreads || (window != m && window != 2 * m)) return false;
  const int Nc = T / m;
  const int nl = kStreamThreads / tpr;
  const bool csa = window == 2 * m;
  const int ups = csa ? (Nc + nl * kCsaRun - 1) / (nl * kCsaRun) : Nc;
  const long long n_units = (long long)B * ups;
  const long long cap = 2LL * sm_count();
  const int grid = (int)(n_units < cap ? n_units : cap);
  const size_t smem = csa ? 0 : (size_t)nl * tpr * 12 * sizeof(float);
  const int threads = nl * tpr;
  count_launch();
  if (csa) {
    if (per_channel)
      compress_stream_kernel<Tin, Tout, true, true><<<grid, threads, 0, st>>>(
          (const Tin*)kv, (const Tin*)gate, (Tout*)out, T, D, m, Nc, ups, n_units);
    else
      compress_stream_kernel<Tin, Tout, false, true><<<grid, threads, 0, st>>>(
          (const Tin*)kv, (const Tin*)gate, (Tout*)out, T, D, m, Nc, ups, n_units);
  } else {
    if (per_channel)
      compress_stream_kernel<Tin, Tout, true, false><<<grid, threads, smem, st>>>(
          (const Tin*)kv, (const Tin*)gate, (Tout*)out, T, D, m, Nc, ups, n_units);
    else
      compress_stream_kernel<Tin, Tout, false, false><<<grid, threads, smem, st>>>(
          (const Tin*)kv, (const Tin*)gate, (Tout*)out, T, D, m, Nc, ups, n_units);
  }
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
  if (rms_w == nullptr && j0 == 0 && n_entries < 0 && kv_pos0 == 0) {
    cudaError_t e;
    if (launch_compress_stream<Tin, Tout>(kv, gate, per_channel, B, T, D, m, window, out, st, &e)) return e;
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
