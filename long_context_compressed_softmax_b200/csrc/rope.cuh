// Rotary pre-pass for the tensor-core attention: rotates the last 64 dims of
// key rows once per call and stores them as BF16 slices, so the attention
// kernel streams ready-made K=V rows (dims 0..447 from the cache, dims
// 448..511 from these slices).  DeepSeek-V4 partial RoPE: only the last 64
// dims of queries and KV entries are rotated; an entry is both key and value.
//
// One warp per row; lane p rotates pair (2p, 2p+1) of the slice by
// pos * base^(-2p/64) (angle in FP64).
#pragma once
#include "common.cuh"

namespace lcsa {

constexpr int kRopeR = 64;

// mode 0: row r of src (rows [0, n)), position = pos0 + r * pos_step
// mode 1: slot r of idx (flattened [B*Tq*k]); entry j = idx[r] of sequence
//         r / (Tq*k); position = j * pos_step; j < 0 -> zeros
__global__ void __launch_bounds__(256)
rope_rows_kernel(const __nv_bfloat16* __restrict__ src, __nv_bfloat16* __restrict__ dst, long long n_rows, int D,
                 long long rows_per_seq, long long pos0, long long pos_step, double log_base, int mode,
                 const int32_t* __restrict__ idx, long long slots_per_seq, int Nc) {
  const long long r = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
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
    rope_cs(pos, lane, kRopeR, log_base, &c, &s);
    const float2 f = __bfloat1622float2(x);
    out = __floats2bfloat162_rn(f.x * c - f.y * s, f.x * s + f.y * c);
  }
  reinterpret_cast<__nv_bfloat162*>(dst + r * kRopeR)[lane] = out;
}

static cudaError_t launch_rope_rows(const void* src, void* dst, long long n_rows, int D, long long rows_per_seq,
                                    long long pos0, long long pos_step, double log_base, int mode,
                                    const int32_t* idx, long long slots_per_seq, int Nc, cudaStream_t st) {
  if (n_rows <= 0) return cudaSuccess;
  const long long blocks = (n_rows + 7) / 8;
  count_launch();
  rope_rows_kernel<<<(unsigned)blocks, 256, 0, st>>>((const __nv_bfloat16*)src, (__nv_bfloat16*)dst, n_rows, D,
                                                     rows_per_seq, pos0, pos_step, log_base, mode, idx,
                                                     slots_per_seq, Nc);
  return cudaGetLastError();
}

}  // namespace lcsa
