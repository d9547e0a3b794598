// FP32 CUDA-core kernels for the indexer scores and the core attention.
// They serve FP32 storage and shapes outside the tensor-core kernels'
// specialisation (H=64, D=512, R=64 / H_I=64, D_I=128), e.g. the small
// parity-sized layer.  Straightforward: one CTA per (query, entry tile) for the
// indexer, one CTA per (query, head) for attention, accurate FP64 rotary
// angles, FP32 accumulation.
#pragma once
#include "common.cuh"

namespace lcsa {

// ---------------------------------------------------------------------------
// Indexer: s[b,t,j] = sum_h w[b,t,h] * relu(q_I[b,t,h,:] . k_I[b,j,:]) for
// j < N_vis(t); scores row stride = Nc.  Grid (entry tiles of 64, rows).
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256)
indexer_scores_generic(const T* __restrict__ q_idx, const float* __restrict__ w, const T* __restrict__ k_idx,
                       float* __restrict__ scores, int Tq, int Nc, int H, int Dd, long long q_pos0, int m,
                       int row0) {
  extern __shared__ float sm[];
  const int row = row0 + blockIdx.y;          // global row over B*Tq
  const int b = row / Tq, i = row - b * Tq;
  const long long t = q_pos0 + i;
  long long nv = t / m;
  if (nv > Nc) nv = Nc;
  if (nv < 0) nv = 0;
  const int j0 = blockIdx.x * 64;
  if (j0 >= nv) return;
  float* sq = sm;                             // [H][Dd+1]
  float* sk = sm + H * (Dd + 1);              // [64][Dd+1]
  float* sw = sk + 64 * (Dd + 1);             // [H]
  const T* qb = q_idx + (long long)row * H * Dd;
  for (int e = threadIdx.x; e < H * Dd; e += blockDim.x) sq[(e / Dd) * (Dd + 1) + e % Dd] = ld_scalar(qb + e);
  for (int e = threadIdx.x; e < H; e += blockDim.x) sw[e] = w[(long long)row * H + e];
  const T* kb = k_idx + ((long long)b * Nc + j0) * Dd;
  const int nj = (int)(nv - j0 < 64 ? nv - j0 : 64);
  for (int e = threadIdx.x; e < nj * Dd; e += blockDim.x) sk[(e / Dd) * (Dd + 1) + e % Dd] = ld_scalar(kb + e);
  __syncthreads();
  // 4 threads per entry, each a strided subset of heads.
  const int jl = threadIdx.x >> 2, part = threadIdx.x & 3;
  float acc = 0.f;
  if (jl < nj) {
    for (int h = part; h < H; h += 4) {
      float d = 0.f;
      for (int x = 0; x < Dd; ++x) d = fmaf(sq[h * (Dd + 1) + x], sk[jl * (Dd + 1) + x], d);
      acc = fmaf(sw[h], fmaxf(d, 0.f), acc);
    }
  }
  acc += __shfl_xor_sync(0xffffffffu, acc, 1);
  acc += __shfl_xor_sync(0xffffffffu, acc, 2);
  if (jl < nj && part == 0) scores[(long long)blockIdx.y * Nc + j0 + jl] = acc;
}

// ---------------------------------------------------------------------------
// Attention, one CTA (128 threads) per (b, query row, head).  Keys are taken
// in tiles of 32: compressed entries first (CSA: the idx list; HCA: 0..nv-1),
// then the window rows.  Online softmax with the sink folded in at the end.
// ---------------------------------------------------------------------------
constexpr int kGenKT = 32;

template <typename T, typename To>
__global__ void __launch_bounds__(128)
attn_generic(const T* __restrict__ q, const T* __restrict__ ckv, const int32_t* __restrict__ idx,
             const T* __restrict__ kv, const float* __restrict__ sink, To* __restrict__ out,
             float* __restrict__ lse, int Tq, int H, int D, int R, int Nc, int k, int Tkv,
             long long q_pos0, long long kv_pos0, int m, int W, float scale, double log_base, int sparse) {
  extern __shared__ float sm[];
  float* sq = sm;                    // [D]
  float* so = sq + D;                // [D]
  float* skey = so + D;              // [kGenKT][D]
  __shared__ float s_logit[kGenKT];
  __shared__ int s_src[kGenKT];      // >= 0: entry index; < 0: -(window position)-1 ... see below
  __shared__ long long s_pos[kGenKT];

  const int h = blockIdx.x % H;
  const long long row = blockIdx.x / H;      // b*Tq + i
  const int b = (int)(row / Tq), i = (int)(row - (long long)b * Tq);
  const long long t = q_pos0 + i;
  const int tid = threadIdx.x;
  const int hp = R / 2;

  // rotated query
  const T* qh = q + (row * H + h) * D;
  for (int d = tid; d < D; d += 128) sq[d] = ld_scalar(qh + d);
  for (int d = tid; d < D; d += 128) so[d] = 0.f;
  __syncthreads();
  for (int p = tid; p < hp; p += 128) {
    float c, s;
    rope_cs(t, p, R, log_base, &c, &s);
    const int d0 = D - R + 2 * p;
    const float a = sq[d0], bb = sq[d0 + 1];
    sq[d0] = a * c - bb * s;
    sq[d0 + 1] = a * s + bb * c;
  }

  // key set sizes
  int n_c;
  long long nv = t / m;
  if (nv > Nc) nv = Nc;
  if (nv < 0) nv = 0;
  const int32_t* irow = sparse ? idx + row * k : nullptr;
  if (sparse) {
    int c = 0;
    while (c < k && irow[c] >= 0) ++c;
    n_c = c;
  } else {
    n_c = (int)nv;
  }
  long long wlo = t - W + 1;
  if (wlo < kv_pos0) wlo = kv_pos0;
  if (wlo < 0) wlo = 0;
  long long whi = t;
  if (whi > kv_pos0 + Tkv - 1) whi = kv_pos0 + Tkv - 1;
  const int n_w = whi >= wlo ? (int)(whi - wlo + 1) : 0;
  const int n_keys = n_c + n_w;

  float run_max = -INFINITY, run_sum = 0.f;
  for (int k0 = 0; k0 < n_keys; k0 += kGenKT) {
    const int nk = n_keys - k0 < kGenKT ? n_keys - k0 : kGenKT;
    __syncthreads();
    if (tid < nk) {
      const int kk = k0 + tid;
      if (kk < n_c) {
        int j = sparse ? irow[kk] : kk;
        if (j >= Nc) { report(LCSA_DEV_BAD_INDEX); j = -1; }
        s_src[tid] = j;
        s_pos[tid] = (long long)j * m;
      } else {
        const long long s = wlo + (kk - n_c);
        s_src[tid] = -2 - (int)(s - kv_pos0);            // window row r -> -2-r
        s_pos[tid] = s;
      }
    }
    __syncthreads();
    for (int e = tid; e < nk * D; e += 128) {
      const int kk = e / D, d = e - kk * D;
      const int src = s_src[kk];
      float v = 0.f;
      if (src >= 0) v = ld_scalar(ckv + ((long long)b * Nc + src) * D + d);
      else if (src <= -2) v = ld_scalar(kv + ((long long)b * Tkv + (-2 - src)) * D + d);
      skey[kk * D + d] = v;
    }
    __syncthreads();
    for (int e = tid; e < nk * hp; e += 128) {
      const int kk = e / hp, p = e - kk * hp;
      float c, s;
      rope_cs(s_pos[kk], p, R, log_base, &c, &s);
      float* x = skey + kk * D + D - R + 2 * p;
      const float a = x[0], bb = x[1];
      x[0] = a * c - bb * s;
      x[1] = a * s + bb * c;
    }
    __syncthreads();
    // logits: warp w handles keys w, w+4, ...
    const int warp = tid >> 5, lane = tid & 31;
    for (int kk = warp; kk < nk; kk += 4) {
      float d = 0.f;
      for (int x = lane; x < D; x += 32) d = fmaf(sq[x], skey[kk * D + x], d);
      d = warp_sum(d);
      if (lane == 0) s_logit[kk] = (s_src[kk] == -1) ? -INFINITY : d * scale;
    }
    __syncthreads();
    float tmax = run_max;
    for (int kk = 0; kk < nk; ++kk) tmax = fmaxf(tmax, s_logit[kk]);
    const float alpha = (run_max == -INFINITY) ? 0.f : __expf(run_max - tmax);
    float psum = 0.f;
    for (int d = tid; d < D; d += 128) so[d] *= alpha;
    for (int kk = 0; kk < nk; ++kk) {
      const float p = (tmax == -INFINITY) ? 0.f : __expf(s_logit[kk] - tmax);
      psum += p;
      for (int d = tid; d < D; d += 128) so[d] = fmaf(p, skey[kk * D + d], so[d]);
    }
    run_sum = run_sum * alpha + psum;
    run_max = tmax;
  }
  __syncthreads();
  // sink, normalisation, output rotation at -t
  float denom = run_sum;
  float mx = run_max;
  if (sink != nullptr) {
    const float sg = sink[h];
    if (sg > mx) {
      const float a = (mx == -INFINITY) ? 0.f : __expf(mx - sg);
      denom *= a;
      for (int d = tid; d < D; d += 128) so[d] *= a;
      mx = sg;
    }
    denom += __expf(sg - mx);
  }
  const float inv = denom > 0.f ? 1.f / denom : 0.f;
  __syncthreads();
  for (int d = tid; d < D; d += 128) so[d] *= inv;
  __syncthreads();
  for (int p = tid; p < hp; p += 128) {
    float c, s;
    rope_cs(-t, p, R, log_base, &c, &s);
    const int d0 = D - R + 2 * p;
    const float a = so[d0], bb = so[d0 + 1];
    so[d0] = a * c - bb * s;
    so[d0 + 1] = a * s + bb * c;
  }
  __syncthreads();
  To* oh = out + (row * H + h) * D;
  for (int d = tid; d < D; d += 128) st_scalar(oh + d, so[d]);
  if (lse != nullptr && tid == 0) lse[row * H + h] = denom > 0.f ? mx + logf(denom) : -INFINITY;
}

}  // namespace lcsa
