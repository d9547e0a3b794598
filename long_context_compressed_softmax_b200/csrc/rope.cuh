// Rotary pre-pass for the tensor-core attention: rotates the last 64 dims of
// key rows once per call and stores them as BF16 slices, so the attention
// kernel streams ready-made K=V rows (dims 0..447 from the cache, dims
// 448..511 from these slices).  DeepSeek-V4 partial RoPE: only the last 64
// dims of queries and KV entries are rotated; an entry is both key and value.
//
// One warp per 8 rows; lane p rotates pair (2p, 2p+1) of the slice by
// pos * base^(-2p/64) (angle formed and reduced in FP64, evaluated in FP32).
#pragma once
#include "common.cuh"

namespace lcsa {

constexpr int kRopeR = 64;

// Frequencies theta_i = base^(-2i/64), i < 32, computed once on the host in FP64.
struct RopeTheta {
  double t[kRopeR / 2];
};

// (cos, sin) of pos * theta: the angle is formed and reduced modulo 2*pi in FP64
// (Cody-Waite reduction with 2*pi split into two doubles, error ~1e-15 rad for
// |angle| < 2^40), then evaluated in FP32 on the reduced angle.
__device__ __forceinline__ void rope_cs_reduced(long long pos, double theta, float* c, float* s) {
  const double kTwoPiHi = 6.283185307179586;            // nearest double to 2*pi
  const double kTwoPiLo = 2.4492935982947064e-16;       // 2*pi - kTwoPiHi
  const double ang = (double)pos * theta;
  const double k = rint(ang * 0.15915494309189535);     // ang / (2*pi), rounded
  const double r = fma(-k, kTwoPiLo, fma(-k, kTwoPiHi, ang));
  sincosf((float)r, s, c);
}

// mode 0: row r of src (rows [0, n)), position = pos0 + r * pos_step
// mode 1: slot r of idx (flattened [B*Tq*k]); entry j = idx[r] of sequence
//         r / (Tq*k); position = j * pos_step; j < 0 -> zeros
constexpr int kRopeRowsPerWarp = 8;

__global__ void __launch_bounds__(256)
rope_rows_kernel(const __nv_bfloat16* __restrict__ src, __nv_bfloat16* __restrict__ dst, long long n_rows, int D,
                 long long rows_per_seq, long long pos0, long long pos_step, const RopeTheta theta, int mode,
                 const int32_t* __restrict__ idx, long long slots_per_seq, int Nc) {
  const int lane = threadIdx.x & 31;
  const double th = theta.t[lane];                       // this lane's frequency, once per warp
  const long long r0 = ((long long)blockIdx.x * 8 + (threadIdx.x >> 5)) * kRopeRowsPerWarp;
#pragma unroll 2
  for (int k = 0; k < kRopeRowsPerWarp; ++k) {
    const long long r = r0 + k;
    if (r >= n_rows) return;
    const __nv_bfloat16* row;
    long long pos;
    bool valid = true;
    if (mode == 0) {
      row = src + r * D;
      pos = pos0 + (r % rows_per_seq) * pos_step;
    } else {
      const long long b = r / slots_per_seq;
      const int j = idx[r];
      valid = j >= 0 && j < Nc;
      row = src + (b * Nc + (valid ? j : 0)) * (long long)D;
      pos = (long long)(valid ? j : 0) * pos_step;
    }
    __nv_bfloat162 out = __floats2bfloat162_rn(0.f, 0.f);
    if (valid) {
      const __nv_bfloat162 x = reinterpret_cast<const __nv_bfloat162*>(row + D - kRopeR)[lane];
      float c, s;
      rope_cs_reduced(pos, th, &c, &s);
      const float2 f = __bfloat1622float2(x);
      out = __floats2bfloat162_rn(f.x * c - f.y * s, f.x * s + f.y * c);
    }
    reinterpret_cast<__nv_bfloat162*>(dst + r * kRopeR)[lane] = out;
  }
}

static cudaError_t launch_rope_rows(const void* src, void* dst, long long n_rows, int D, long long rows_per_seq,
                                    long long pos0, long long pos_step, double log_base, int mode,
                                    const int32_t* idx, long long slots_per_seq, int Nc, cudaStream_t st) {
  if (n_rows <= 0) return cudaSuccess;
  RopeTheta theta;
  for (int i = 0; i < kRopeR / 2; ++i) theta.t[i] = exp(-2.0 * (double)i / (double)kRopeR * log_base);
  const long long rows_per_block = 8LL * kRopeRowsPerWarp;
  const long long blocks = (n_rows + rows_per_block - 1) / rows_per_block;
  count_launch();
  rope_rows_kernel<<<(unsigned)blocks, 256, 0, st>>>((const __nv_bfloat16*)src, (__nv_bfloat16*)dst, n_rows, D,
                                                     rows_per_seq, pos0, pos_step, theta, mode, idx,
                                                     slots_per_seq, Nc);
  return cudaGetLastError();
}

}  // namespace lcsa
