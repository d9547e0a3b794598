// FP8 entry cache: compressed entries stored as FP8 E4M3 with one
// power-of-two scale per entry, the rotary dims kept in BF16 (DeepSeek-V4,
// "DeepSeek V4 技术架构深度解析", 二、CSA + HCA / KV Cache优化细节: the RoPE dims
// in BF16, the rest in FP8).
//
// Entry row x[0..D): body x[0..D-R) -> codes (E4M3, one byte each), scale byte
// X + 127 with X the smallest integer such that max|body| <= 448 * 2^X, raised
// to at least -124 (an all-zero body takes -124); codes are the E4M3 numbers
// nearest to body / 2^X (ties to even, saturating at 448), a zero of either
// sign coded +0.  Rotary dims x[D-R..D) -> BF16 (round to nearest even).
// With X >= -124 every E4M3 * 2^X is exact in BF16, so the attention kernel
// expands the cache losslessly in shared memory.
#pragma once
#include <cuda_fp8.h>
#include <cuda_fp16.h>
#include "common.cuh"

namespace lcsa {

constexpr int kFp8ScaleFloor = -124;

// One warp per entry row.
template <typename Tin>
__global__ void __launch_bounds__(256)
quantize_entries_fp8_kernel(const Tin* __restrict__ x, long long rows, int D, int R, uint8_t* __restrict__ codes,
                            uint8_t* __restrict__ scales, __nv_bfloat16* __restrict__ rope) {
  const int lane = threadIdx.x & 31;
  const int body = D - R;
  for (long long r = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows;
       r += (long long)gridDim.x * (blockDim.x >> 5)) {
    const Tin* row = x + r * D;
    float amax = 0.f;
    for (int e = lane; e < body; e += 32) amax = fmaxf(amax, fabsf(Elem<Tin>::to_f(row[e])));
    amax = warp_max(amax);
    // smallest X with amax <= 448 * 2^X: amax = f * 2^e with f in [0.5, 1) and
    // 448 = 0.875 * 2^9, so X = e - 9 when f <= 0.875, else e - 8
    int X = kFp8ScaleFloor;
    if (amax > 0.f) {
      int e;
      const float f = frexpf(amax, &e);
      X = f <= 0.875f ? e - 9 : e - 8;
      X = X < kFp8ScaleFloor ? kFp8ScaleFloor : (X > 127 ? 127 : X);
    }
    const float inv = ldexpf(1.f, -X);             // exact power of two
    for (int p = lane; 2 * p < body; p += 32) {
      // +0.0f turns -0 into +0 (a zero is coded +0); tiny negatives keep their sign
      float a = (Elem<Tin>::to_f(row[2 * p]) + 0.f) * inv;
      float b = 2 * p + 1 < body ? (Elem<Tin>::to_f(row[2 * p + 1]) + 0.f) * inv : 0.f;
      // below 2^-12 the code is a zero of the value's sign (half the smallest
      // E4M3 subnormal is 2^-10); FP32 subnormal products never reach the cvt
      if (fabsf(a) < 0x1p-12f) a = copysignf(0.f, a);
      if (fabsf(b) < 0x1p-12f) b = copysignf(0.f, b);
      const __nv_fp8x2_storage_t c = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
      uint8_t* o = codes + r * body + 2 * p;
      o[0] = (uint8_t)(c & 0xff);
      if (2 * p + 1 < body) o[1] = (uint8_t)(c >> 8);
    }
    for (int e = lane; e < R; e += 32) rope[r * R + e] = __float2bfloat16_rn(Elem<Tin>::to_f(row[body + e]));
    if (lane == 0) scales[r] = (uint8_t)(X + 127);
  }
}

static cudaError_t launch_quantize_entries_fp8(const void* x, long long rows, int D, int R, lcsa_dtype dt,
                                               uint8_t* codes, uint8_t* scales, void* rope, cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  const long long want = (rows + 7) / 8;
  const int grid = (int)(want < 148LL * 32 ? want : 148LL * 32);
  count_launch();
  if (dt == LCSA_BF16)
    quantize_entries_fp8_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>((const __nv_bfloat16*)x, rows, D, R, codes,
                                                                       scales, (__nv_bfloat16*)rope);
  else
    quantize_entries_fp8_kernel<float><<<grid, 256, 0, st>>>((const float*)x, rows, D, R, codes, scales,
                                                              (__nv_bfloat16*)rope);
  return cudaGetLastError();
}

// 16 E4M3 codes (bytes of c, element k in byte k) times 2^X -> 16 BF16 values
// as two 16-byte chunks (elements 0-7 in lo, 8-15 in hi).  E4M3 -> FP16 is
// exact, the FP32 product by a power of two is exact, and the result is a
// BF16 number, so every step is exact.
__device__ __forceinline__ void e4m3x16_to_bf16(const uint4& c, float scale, uint4& lo, uint4& hi) {
  const uint32_t w[4] = {c.x, c.y, c.z, c.w};
  uint32_t o[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)((w[i] >> (16 * h)) & 0xffffu), __NV_E4M3);
      __half2 hv;
      hv = *reinterpret_cast<const __half2*>(&hr);
      const float2 f = __half22float2(hv);
      const __nv_bfloat162 b = __floats2bfloat162_rn(f.x * scale, f.y * scale);
      o[2 * i + h] = *reinterpret_cast<const uint32_t*>(&b);
    }
  }
  lo = make_uint4(o[0], o[1], o[2], o[3]);
  hi = make_uint4(o[4], o[5], o[6], o[7]);
}

}  // namespace lcsa
