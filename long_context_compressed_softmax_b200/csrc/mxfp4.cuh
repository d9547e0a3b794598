// MXFP4 (FP4 E2M1 values with one power-of-two scale per 32) for the FP4
// indexer QK path.  DeepSeek-V4 "FP4 Quantization-Aware Training": the
// Lightning Indexer computes its query-key scores in FP4 and the block scale
// factors are absorbed into a wider format on dequantisation, exactly; "三、
// FP4量化": the CSA indexer QK path goes from FP32 to FP4.
//
// Block format (OCP Microscaling MXFP4): 32 consecutive values share the
// scale 2^X, X = floor(log2 amax) - 2 clamped to [-127, 127] (UE8M0 byte
// X + 127; an all-zero block takes X = -127; a block holding Inf/NaN takes
// byte 255 and zero codes).  Value i is the E2M1 number nearest to x_i / 2^X,
// ties to an even mantissa bit, saturated at 6; sign bit = (x_i < 0).  Codes
// pack two per byte, element 2i in the low nibble.
//
// Staging for the tensor cores: an E2M1 magnitude times 2^s is an FP8 E4M3
// number exactly while s >= -7 (E4M3 spans 2^-9 .. 448, E2M1 needs 3 of its
// binades).  Each key entry (and each query head) is staged relative to its
// largest block exponent Xref: block b is written as E2M1 * 2^(X_b - Xref + 6)
// and the factor 2^(Xref - 6) is applied to the score.  Blocks within 2^13 of
// the largest are exact; smaller ones round to the E4M3 grid (nearest even).
#pragma once
#include <cuda_fp8.h>
#include "common.cuh"

namespace lcsa {

// 2^e as a float (0 below the subnormal range); e <= 127.
__device__ __forceinline__ float pow2f(int e) {
  if (e >= -126) return __uint_as_float((uint32_t)(e + 127) << 23);
  if (e >= -149) return __uint_as_float(1u << (e + 149));
  return 0.f;
}

// Shared exponent of a block from the bits of its largest magnitude (finite).
__device__ __forceinline__ int mx_scale_exponent(uint32_t amax_bits) {
  const int E = (int)(amax_bits >> 23);
  if (E == 0) return -127;                // zero or subnormal: floor(log2) - 2 < -127
  const int X = E - 127 - 2;
  return X < -127 ? -127 : X;
}

// E2M1 magnitude code (0..7) of a >= 0: nearest of {0,.5,1,1.5,2,3,4,6},
// ties to the even code, saturating.
__device__ __forceinline__ uint32_t e2m1_mag_code(float a) {
  return (uint32_t)(a > 0.25f) + (uint32_t)(a >= 0.75f) + (uint32_t)(a > 1.25f) + (uint32_t)(a >= 1.75f) +
         (uint32_t)(a > 2.5f) + (uint32_t)(a >= 3.5f) + (uint32_t)(a > 5.0f);
}

// 4-bit code of x in a block with exponent X (sign from the bits of x).
__device__ __forceinline__ uint32_t e2m1_code(float x, int X) {
  const uint32_t bits = __float_as_uint(x);
  const uint32_t mag = bits & 0x7FFFFFFFu;
  const uint32_t c = e2m1_mag_code(__uint_as_float(mag) * pow2f(-X));
  return c | ((bits >> 31) && mag ? 8u : 0u);
}

// E4M3 bytes of the 8 E2M1 magnitudes times 2^s (s <= 6), byte c of (lo, hi)
// = magnitude code c.  At s = 6 the magnitudes are 32, 64, 96, 128, 192, 256,
// 384; lower s subtract (6 - s) from every non-zero exponent field while they
// stay normal (s >= -5), below that each value is rounded by the converter.
__device__ __forceinline__ void e4m3_table(int s, uint32_t& lo, uint32_t& hi) {
  if (s >= -5) {
    const uint32_t d = (uint32_t)(6 - s) * 8u;
    lo = 0x6C686000u - d * 0x01010100u;
    hi = 0x7C787470u - d * 0x01010101u;
    return;
  }
  const float f = pow2f(s);
  const float mags[8] = {0.f, 0.5f, 1.f, 1.5f, 2.f, 3.f, 4.f, 6.f};
  uint32_t b[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) b[c] = (uint32_t)__nv_cvt_float_to_fp8(mags[c] * f, __NV_SATFINITE, __NV_E4M3);
  lo = b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24);
  hi = b[4] | (b[5] << 8) | (b[6] << 16) | (b[7] << 24);
}

// Eight E2M1 codes (one 32-bit word, element 0 in the low nibble) to eight
// E4M3 bytes in element order: a byte-permute table lookup on the magnitude
// codes, then each code's sign bit moved to bit 7 of its byte.
__device__ __forceinline__ uint2 e2m1x8_to_e4m3(uint32_t w, uint32_t lo, uint32_t hi) {
  const uint32_t m = w & 0x77777777u;
  uint32_t v0 = __byte_perm(lo, hi, m);
  uint32_t v1 = __byte_perm(lo, hi, m >> 16);
  const uint32_t w4 = w << 4;
  v0 |= __byte_perm(w4, w, 0x5140) & 0x80808080u;   // signs of codes 0,1,2,3
  v1 |= __byte_perm(w4, w, 0x7362) & 0x80808080u;   // signs of codes 4,5,6,7
  return make_uint2(v0, v1);
}

// ---------------------------------------------------------------------------
// Quantiser: n_blocks contiguous 32-value blocks -> codes [n_blocks * 16] and
// scales [n_blocks].  One warp per block, lane i holds value i.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256) mxfp4_quantize_kernel(const T* __restrict__ x, long long n_blocks,
                                                             uint8_t* __restrict__ codes,
                                                             uint8_t* __restrict__ scales) {
  const int lane = threadIdx.x & 31;
  const long long stride = ((long long)gridDim.x * blockDim.x) >> 5;
  for (long long blk = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5; blk < n_blocks; blk += stride) {
    const float v = Elem<T>::to_f(x[blk * 32 + lane]);
    const uint32_t amax = __reduce_max_sync(0xffffffffu, __float_as_uint(v) & 0x7FFFFFFFu);
    uint32_t code = 0, sbyte = 255;
    if (amax < 0x7F800000u) {
      const int X = mx_scale_exponent(amax);
      sbyte = (uint32_t)(X + 127);
      code = e2m1_code(v, X);
    }
    const uint32_t odd = __shfl_down_sync(0xffffffffu, code, 1);
    if ((lane & 1) == 0) codes[blk * 16 + (lane >> 1)] = (uint8_t)(code | (odd << 4));
    if (lane == 0) scales[blk] = (uint8_t)sbyte;
  }
}

// ---------------------------------------------------------------------------
// Query preparation for the FP4 indexer: every (row, head) of q [.., 64, 128]
// BF16 in the rectangle (sequences [b0, b0+nb), rows [i0, i0+ni)) is
// quantised to MXFP4 (4 blocks) and staged as E4M3 relative to its largest
// block exponent; the head weight absorbs the factor and a 1/2 (the scoring
// epilogue forms w relu(x) as (w/2) x + (w/2) |x|):
//   q8 [nb*ni*64, 128] E4M3,  w8 [nb*ni*64] = w * 2^(Xref - 7).
// One warp per (row, head); lane l holds dims [4l, 4l+4) (block l / 8).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) indexer_q8_kernel(const __nv_bfloat16* __restrict__ q,
                                                         const float* __restrict__ w, int Tq, int b0, int nb,
                                                         int i0, int ni, uint8_t* __restrict__ q8,
                                                         float* __restrict__ w8) {
  const int lane = threadIdx.x & 31;
  const long long unit = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;   // (rect row, head)
  if (unit >= (long long)nb * ni * 64) return;
  const int h = (int)(unit & 63);
  const long long rr = unit >> 6;
  const int bl = (int)(rr / ni), i = (int)(rr - (long long)bl * ni);
  const long long src_row = ((long long)(b0 + bl) * Tq + i0 + i) * 64 + h;
  const uint2 raw = __ldg(reinterpret_cast<const uint2*>(q + src_row * 128) + lane);
  float v[4];
  {
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.y));
    v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
  }
  uint32_t amax = 0;
#pragma unroll
  for (int k = 0; k < 4; ++k) amax = max(amax, __float_as_uint(v[k]) & 0x7FFFFFFFu);
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) amax = max(amax, __shfl_xor_sync(0xffffffffu, amax, o));   // block amax
  const int X = mx_scale_exponent(amax < 0x7F800000u ? amax : 0x7F000000u);
  int Xref = X;
#pragma unroll
  for (int o = 8; o < 32; o <<= 1) Xref = max(Xref, __shfl_xor_sync(0xffffffffu, Xref, o));
  uint32_t word = 0;
#pragma unroll
  for (int k = 0; k < 4; ++k) word |= e2m1_code(v[k], X) << (4 * k);
  uint32_t lo, hi;
  e4m3_table(X - Xref + 6, lo, hi);
  const uint2 e = e2m1x8_to_e4m3(word, lo, hi);     // codes 4-7 are zero
  reinterpret_cast<uint32_t*>(q8 + unit * 128)[lane] = e.x;
  if (lane == 0) w8[unit] = w[src_row] * pow2f(Xref - 7);
}

}  // namespace lcsa
