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

template <typename Tin, typename Tout>
static cudaError_t launch_compress_t(const void* kv, const void* gate, int per_channel, int B, int T, int D,
                                     int m, int window, const float* rms_w, float rms_eps, void* out,
                                     cudaStream_t st, long long j0 = 0, int n_entries = -1, long long kv_pos0 = 0,
                                     long long out_rows = -1) {
  constexpr int V = Elem<Tin>::kVec;
  const int Nc = n_entries >= 0 ? n_entries : T / m;
  if (out_rows < 0) out_rows = Nc;
  if (Nc == 0 || B == 0) return cudaSuccess;
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
