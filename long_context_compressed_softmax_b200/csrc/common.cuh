// Shared device helpers for liblcsa (sm_100a).
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <math.h>

#include "lcsa.h"

namespace lcsa {

// ---------------------------------------------------------------------------
// Per-device status word.  Kernels record the first problem they detect
// (bounded wait expired, index out of range) and skip the offending access;
// lcsa_get_device_status() reads and clears it.
// ---------------------------------------------------------------------------
__device__ int g_status;

// Limit of every bounded wait in the library's kernels (ns of %globaltimer);
// lcsa_set_wait_limit_ns changes it per device.
constexpr unsigned long long kDefaultWaitLimitNs = 2000000000ull;   // 2 s
__constant__ unsigned long long g_wait_limit_ns = kDefaultWaitLimitNs;   // constant cache: cheap to poll

__device__ __forceinline__ void report(int code) { atomicCAS(&g_status, 0, code); }

// Packed FP32 pairs: sm_100 executes add, mul and fma on the two FP32 lanes
// of a 64-bit register in one instruction.
typedef unsigned long long f2x;
__device__ __forceinline__ f2x pk2(float a, float b) {
  f2x r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ float2 upk2(f2x r) {
  float2 f;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(f.x), "=f"(f.y) : "l"(r));
  return f;
}
__device__ __forceinline__ f2x fma2(f2x a, f2x b, f2x c) {
  f2x r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ f2x add2(f2x a, f2x b) {
  f2x r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ f2x mul2(f2x a, f2x b) {
  f2x r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// Host-side count of kernel launches issued by the library.
inline unsigned long long& launch_counter() {
  static unsigned long long n = 0;
  return n;
}
inline void count_launch(int n = 1) { __atomic_fetch_add(&launch_counter(), (unsigned long long)n, __ATOMIC_RELAXED); }

// Streaming multiprocessors of the current device.
static int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

// ---------------------------------------------------------------------------
// Element load / store helpers (BF16 storage, FP32 arithmetic).
// ---------------------------------------------------------------------------
template <typename T> struct Elem;
template <> struct Elem<float> {
  static constexpr int kVec = 4;  // elements per 16-byte vector
  __device__ __forceinline__ static float to_f(float x) { return x; }
  __device__ __forceinline__ static float from_f(float x) { return x; }
};
template <> struct Elem<__nv_bfloat16> {
  static constexpr int kVec = 8;
  __device__ __forceinline__ static float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
  __device__ __forceinline__ static __nv_bfloat16 from_f(float x) { return __float2bfloat16_rn(x); }
};

// Load 16 bytes (kVec elements) as floats.
__device__ __forceinline__ void load16(const float* p, float* v) {
  float4 a = __ldg(reinterpret_cast<const float4*>(p));
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
}
__device__ __forceinline__ void load16(const __nv_bfloat16* p, float* v) {
  uint4 a = __ldg(reinterpret_cast<const uint4*>(p));
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&a);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(h[i]);
    v[2 * i] = f.x; v[2 * i + 1] = f.y;
  }
}
// Store n floats (n = 4 for float, 8 for bf16 -> one 16-byte store; n = 4 bf16 -> 8 bytes).
template <int N> __device__ __forceinline__ void store_vec(float* p, const float* v) {
  static_assert(N % 4 == 0, "");
#pragma unroll
  for (int i = 0; i < N; i += 4)
    *reinterpret_cast<float4*>(p + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
}
template <int N> __device__ __forceinline__ void store_vec(__nv_bfloat16* p, const float* v) {
  static_assert(N % 4 == 0, "");
  if constexpr (N % 8 == 0) {
#pragma unroll
    for (int i = 0; i < N; i += 8) {
      uint4 o;
      __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
      for (int q = 0; q < 4; ++q) h[q] = __floats2bfloat162_rn(v[i + 2 * q], v[i + 2 * q + 1]);
      *reinterpret_cast<uint4*>(p + i) = o;
    }
  } else {
#pragma unroll
    for (int i = 0; i < N; i += 4) {
      uint2 o;
      __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&o);
      h[0] = __floats2bfloat162_rn(v[i], v[i + 1]);
      h[1] = __floats2bfloat162_rn(v[i + 2], v[i + 3]);
      *reinterpret_cast<uint2*>(p + i) = o;
    }
  }
}

__device__ __forceinline__ float ld_scalar(const float* p) { return __ldg(p); }
__device__ __forceinline__ float ld_scalar(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ void st_scalar(float* p, float v) { *p = v; }
__device__ __forceinline__ void st_scalar(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

// Rotary angle for position `pos` and pair i of an R-dim slice: pos*base^(-2i/R),
// computed in FP64 (positions reach 2^20, so an FP32 product would lose the
// fractional turns), then cos/sin rounded to FP32.
__device__ __forceinline__ void rope_cs(long long pos, int i, int R, double log_base, float* c, float* s) {
  double theta = exp(-2.0 * (double)i / (double)R * log_base);
  double ang = (double)pos * theta;
  double sd, cd;
  sincos(ang, &sd, &cd);
  *c = (float)cd;
  *s = (float)sd;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

}  // namespace lcsa
