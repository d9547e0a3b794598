// liblcsa: C ABI entry points (declared in include/lcsa.h), argument
// validation and kernel dispatch.  This is the library's only translation
// unit; the kernels live in the included headers.
#include <cuda_runtime.h>
#include <stdio.h>
#include <string.h>

#include "lcsa.h"
#include "common.cuh"
#include "compress.cuh"
#include "topk.cuh"
#include "generic.cuh"
#include "rope.cuh"
#include "indexer_tc.cuh"
#include "attn_tc.cuh"
#include "indexer_fp4.cuh"
#include "gemm_tc.cuh"

using namespace lcsa;

namespace {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t esize(lcsa_dtype d) { return d == LCSA_BF16 ? 2 : 4; }
inline bool valid_dtype(lcsa_dtype d) { return d == LCSA_BF16 || d == LCSA_FP32; }
inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

inline lcsa_status from_cuda(cudaError_t e) { return e == cudaSuccess ? LCSA_OK : LCSA_ERR_CUDA; }

// A device must exist for any compute call (there is no CPU path).
inline bool have_device() {
  int n = 0;
  return cudaGetDeviceCount(&n) == cudaSuccess && n > 0;
}

lcsa_status compress_common(const void* kv, const void* gate, int per_channel, int B, int T, int D, int m,
                            int window, lcsa_dtype dt, const float* rms_w, float rms_eps, void* out,
                            lcsa_dtype odt, void* stream) {
  if (!valid_dtype(dt) || !valid_dtype(odt)) return LCSA_ERR_INVALID_ARG;
  if (B < 0 || T < 0 || D <= 0 || m <= 0) return LCSA_ERR_INVALID_ARG;
  const int vec = dt == LCSA_BF16 ? 8 : 4;
  if (D % vec != 0 || D / vec > 1024) return LCSA_ERR_INVALID_ARG;
  if (odt == LCSA_BF16 && D % 8 != 0 && dt == LCSA_BF16) return LCSA_ERR_INVALID_ARG;
  const int Nc = T / m;
  if ((long long)B * Nc == 0) return LCSA_OK;
  if (!kv || !gate || !out) return LCSA_ERR_INVALID_ARG;
  if (!aligned16(kv) || !aligned16(out) || (per_channel && !aligned16(gate))) return LCSA_ERR_INVALID_ARG;
  if (rms_w && (reinterpret_cast<uintptr_t>(rms_w) & 3u)) return LCSA_ERR_INVALID_ARG;
  if (!have_device()) return LCSA_ERR_CUDA;
  return from_cuda(launch_compress(kv, gate, per_channel, B, T, D, m, window, dt, rms_w, rms_eps, out, odt,
                                   (cudaStream_t)stream));
}

lcsa_status check_indexer(const lcsa_indexer_args* a) {
  if (!a) return LCSA_ERR_INVALID_ARG;
  if (!valid_dtype(a->dtype)) return LCSA_ERR_INVALID_ARG;
  if (a->B < 0 || a->Tq < 0 || a->Nc < 0 || a->H_I <= 0 || a->D_I <= 0 || a->m <= 0 || a->k <= 0)
    return LCSA_ERR_INVALID_ARG;
  if (a->q_pos0 < 0) return LCSA_ERR_INVALID_ARG;
  if ((long long)a->B * a->Tq == 0) return LCSA_OK;
  if (!a->q_idx || !a->w || !a->idx_out || (a->Nc > 0 && !a->k_idx)) return LCSA_ERR_INVALID_ARG;
  if (!aligned16(a->q_idx) || !aligned16(a->w) || !aligned16(a->idx_out) ||
      (a->k_idx && !aligned16(a->k_idx)) || (a->scores_out && !aligned16(a->scores_out)))
    return LCSA_ERR_INVALID_ARG;
  if ((a->D_I * esize(a->dtype)) % 16 != 0) return LCSA_ERR_INVALID_ARG;
  if (!indexer_tc_supported(a) && (size_t)(a->H_I * (a->D_I + 1) + 64 * (a->D_I + 1) + a->H_I) * 4 > 200 * 1024)
    return LCSA_ERR_UNSUPPORTED;
  return LCSA_OK;
}

// need_ckv = 0: the entries come from elsewhere (the FP8 cache), ckv is not read.
lcsa_status check_attn(const lcsa_attn_args* a, int sparse, int need_ckv = 1) {
  if (!a) return LCSA_ERR_INVALID_ARG;
  if (!valid_dtype(a->dtype) || !valid_dtype(a->out_dtype)) return LCSA_ERR_INVALID_ARG;
  if (a->B < 0 || a->Tq < 0 || a->H <= 0 || a->D <= 0 || a->R < 0 || a->R > a->D || (a->R & 1) ||
      a->Nc < 0 || a->Tkv < 0 || a->m <= 0 || a->W < 0)
    return LCSA_ERR_INVALID_ARG;
  if (sparse && a->k <= 0) return LCSA_ERR_INVALID_ARG;
  if (a->q_pos0 < 0) return LCSA_ERR_INVALID_ARG;
  if ((long long)a->B * a->Tq == 0) return LCSA_OK;
  if ((a->D * esize(a->dtype)) % 16 != 0) return LCSA_ERR_INVALID_ARG;
  if (!a->q || !a->out) return LCSA_ERR_INVALID_ARG;
  if (need_ckv && a->Nc > 0 && !a->ckv) return LCSA_ERR_INVALID_ARG;
  if (a->Tkv > 0 && !a->kv) return LCSA_ERR_INVALID_ARG;
  if (sparse && !a->idx) return LCSA_ERR_INVALID_ARG;
  if (!aligned16(a->q) || !aligned16(a->out) || (need_ckv && a->ckv && !aligned16(a->ckv)) ||
      (a->kv && !aligned16(a->kv)) || (sparse && !aligned16(a->idx)) || (a->lse && !aligned16(a->lse)) ||
      (a->sink && (reinterpret_cast<uintptr_t>(a->sink) & 3u)))
    return LCSA_ERR_INVALID_ARG;
  if (!attn_tc_supported(a) && (size_t)(2 + kGenKT) * a->D * 4 > 200 * 1024) return LCSA_ERR_UNSUPPORTED;
  return LCSA_OK;
}

template <typename T, typename To>
cudaError_t launch_attn_generic_t(const lcsa_attn_args* a, int sparse, cudaStream_t st) {
  const float scale = a->softmax_scale > 0.f ? a->softmax_scale : 1.0f / sqrtf((float)a->D);
  const double log_base = log(a->rope_base > 0.f ? (double)a->rope_base : 10000.0);
  const size_t smem = (size_t)(2 + kGenKT) * a->D * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(attn_generic<T, To>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  const long long blocks = (long long)a->B * a->Tq * a->H;
  count_launch();
  attn_generic<T, To><<<(unsigned)blocks, 128, smem, st>>>(
      (const T*)a->q, (const T*)a->ckv, a->idx, (const T*)a->kv, a->sink, (To*)a->out, a->lse, a->Tq, a->H,
      a->D, a->R, a->Nc, a->k, a->Tkv, a->q_pos0, a->kv_pos0, a->m, a->W, scale, log_base, sparse);
  return cudaGetLastError();
}

cudaError_t launch_attn_generic(const lcsa_attn_args* a, int sparse, cudaStream_t st) {
  if (a->dtype == LCSA_BF16)
    return a->out_dtype == LCSA_BF16 ? launch_attn_generic_t<__nv_bfloat16, __nv_bfloat16>(a, sparse, st)
                                     : launch_attn_generic_t<__nv_bfloat16, float>(a, sparse, st);
  return a->out_dtype == LCSA_BF16 ? launch_attn_generic_t<float, __nv_bfloat16>(a, sparse, st)
                                   : launch_attn_generic_t<float, float>(a, sparse, st);
}

template <typename T>
cudaError_t launch_indexer_generic_t(const lcsa_indexer_args* a, float* scores, int row0, int rows,
                                     cudaStream_t st) {
  const size_t smem = (size_t)(a->H_I * (a->D_I + 1) + 64 * (a->D_I + 1) + a->H_I) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(indexer_scores_generic<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((a->Nc + 63) / 64, rows);
  count_launch();
  indexer_scores_generic<T><<<grid, 256, smem, st>>>((const T*)a->q_idx, a->w, (const T*)a->k_idx, scores, a->Tq,
                                                     a->Nc, a->H_I, a->D_I, a->q_pos0, a->m, row0);
  return cudaGetLastError();
}

// n_valid per row of a chunk rectangle (rows ordered [b][i0..i0+ni)):
// min(Nc, floor(t/m)) with t = q_pos0 + i.
__global__ void nvalid_kernel(int32_t* nv, int rows, int i0, int ni, long long q_pos0, int m, int Nc) {
  const int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= rows) return;
  const int i = i0 + r % ni;
  long long v = (q_pos0 + i) / m;
  nv[r] = (int32_t)(v < Nc ? v : Nc);
}

// Rows of one indexer chunk: at most kIndexerChunkRows score rows at a time.
long long indexer_chunk_budget(int B, int Tq) {
  const long long rows = (long long)B * Tq;
  return rows < kIndexerChunkRows ? rows : kIndexerChunkRows;
}

// Workspace of a chunk of r rows: scores + visible counts + the two-phase
// top-k scratch + `extra_per_row` bytes per row for the score kernels.
size_t indexer_ws_need(long long r, int Nc, int k, size_t extra_per_row) {
  const size_t per_row = (size_t)(Nc > 0 ? Nc : 1) * 4;
  size_t n = align256((size_t)r * per_row) + align256((size_t)r * 4) + topk_long_scratch((int)r, Nc, k);
  if (extra_per_row) n += align256((size_t)r * 64 * 128) + align256((size_t)r * (extra_per_row - 64 * 128));
  return n;
}

// Indexer + top-k over chunk rectangles: whole sequences when a sequence fits
// the chunk, else row ranges of one sequence (a multiple of the 4-row query
// group).  `scores_fn(sc, b0, nb, i0, ni, extra)` writes the rectangle's
// scores [nb*ni][Nc] to sc; then the visible counts and the top-k follow.
template <typename F>
lcsa_status indexer_by_chunks(int B, int Tq, int Nc, int k, long long q_pos0, int m, int32_t* idx_out,
                              float* scores_out, void* workspace, size_t workspace_bytes, size_t extra_per_row,
                              cudaStream_t st, F&& scores_fn) {
  long long budget = indexer_chunk_budget(B, Tq);
  while (budget > 1 && indexer_ws_need(budget, Nc, k, extra_per_row) > workspace_bytes) budget >>= 1;
  if (!workspace || indexer_ws_need(budget, Nc, k, extra_per_row) > workspace_bytes) return LCSA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return LCSA_ERR_INVALID_ARG;
  const size_t per_row = (size_t)(Nc > 0 ? Nc : 1) * 4;
  char* base = (char*)workspace;
  float* sc_ws = (float*)base;
  int32_t* nv = (int32_t*)(base + align256((size_t)budget * per_row));
  char* tk_scratch = base + align256((size_t)budget * per_row) + align256((size_t)budget * 4);
  const size_t tk_bytes = topk_long_scratch((int)budget, Nc, k);
  void* extra = extra_per_row ? (void*)(tk_scratch + tk_bytes) : nullptr;
  int nb_step, ni_step;
  if (Tq <= budget) { nb_step = (int)(budget / Tq); ni_step = Tq; }
  else { nb_step = 1; ni_step = budget >= 4 ? (int)(budget & ~3LL) : (int)budget; }
  for (int b0 = 0; b0 < B; b0 += nb_step) {
    const int nb = B - b0 < nb_step ? B - b0 : nb_step;
    for (int i0 = 0; i0 < Tq; i0 += ni_step) {
      const int ni = Tq - i0 < ni_step ? Tq - i0 : ni_step;
      const long long row0 = (long long)b0 * Tq + i0;      // rectangle rows are contiguous
      const int nr = nb * ni;
      float* sc = scores_out ? scores_out + row0 * (long long)Nc : sc_ws;
      cudaError_t e = cudaSuccess;
      if (Nc > 0) {
        e = scores_fn(sc, b0, nb, i0, ni, extra);
        if (e != cudaSuccess) return LCSA_ERR_CUDA;
      }
      count_launch();
      nvalid_kernel<<<(nr + 255) / 256, 256, 0, st>>>(nv, nr, i0, ni, q_pos0, m, Nc);
      // the longest row of the rectangle is its last position's visible count
      const long long last_vis = (q_pos0 + i0 + ni - 1) / m;
      const int n_max = (int)(last_vis < Nc ? last_vis : Nc);
      e = launch_topk(sc, nr, Nc, Nc, nv, k, idx_out + row0 * k, st, tk_scratch, tk_bytes, n_max);
      if (e != cudaSuccess) return LCSA_ERR_CUDA;
    }
  }
  return LCSA_OK;
}

}  // namespace

// Shared with noalloc.cu (same library, not exported): the argument checks of
// lcsa_indexer_topk, and the workspace that one query row needs.
__attribute__((visibility("hidden"))) lcsa_status lcsa_internal_check_indexer(const lcsa_indexer_args* a) {
  return check_indexer(a);
}
__attribute__((visibility("hidden"))) size_t lcsa_internal_indexer_one_row_bytes(const lcsa_indexer_args* a) {
  return indexer_ws_need(1, a->Nc, a->k, 0);
}

extern "C" {

const char* lcsa_version(void) { return "lcsa 0.1 (sm_100a)"; }

uint64_t lcsa_kernel_launches(void) { return __atomic_load_n(&launch_counter(), __ATOMIC_RELAXED); }

const char* lcsa_status_string(lcsa_status s) {
  switch (s) {
    case LCSA_OK: return "ok";
    case LCSA_ERR_INVALID_ARG: return "invalid argument";
    case LCSA_ERR_UNSUPPORTED: return "unsupported combination";
    case LCSA_ERR_WORKSPACE: return "workspace missing or too small";
    case LCSA_ERR_CUDA: return "CUDA error";
    case LCSA_ERR_DEVICE: return "device reported an error";
  }
  return "unknown status";
}

lcsa_status lcsa_get_device_status(void* stream, int* code) {
  if (!code) return LCSA_ERR_INVALID_ARG;
  if (!have_device()) return LCSA_ERR_CUDA;
  cudaStream_t st = (cudaStream_t)stream;
  int v = 0;
  if (cudaStreamSynchronize(st) != cudaSuccess) return LCSA_ERR_CUDA;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(int)) != cudaSuccess) return LCSA_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_status, &zero, sizeof(int)) != cudaSuccess) return LCSA_ERR_CUDA;
  *code = v;
  return v == 0 ? LCSA_OK : LCSA_ERR_DEVICE;
}

lcsa_status lcsa_set_wait_limit_ns(uint64_t ns) {
  if (!have_device()) return LCSA_ERR_CUDA;
  const unsigned long long v = ns ? (unsigned long long)ns : kDefaultWaitLimitNs;
  return from_cuda(cudaMemcpyToSymbol(g_wait_limit_ns, &v, sizeof(v)));
}

void lcsa_test_withhold_stage(int chunk) { gemm_withhold_next().store(chunk < 0 ? -1 : chunk); }

lcsa_status lcsa_set_attn_gather(int mode) {
  if (mode != 0 && mode != 1) return LCSA_ERR_INVALID_ARG;
  attn_gather_mode().store(mode);
  return LCSA_OK;
}

lcsa_status lcsa_set_fp4_mma(int mode) {
  if (mode != 0 && mode != 1) return LCSA_ERR_INVALID_ARG;
  fp4_mma_mode_ref().store(mode);
  return LCSA_OK;
}

lcsa_status lcsa_csa_compress(const void* kv, const void* gate, int gate_per_channel, int B, int T, int D, int m,
                              lcsa_dtype dtype, const float* rms_weight, float rms_eps, void* out,
                              lcsa_dtype out_dtype, void* stream) {
  return compress_common(kv, gate, gate_per_channel, B, T, D, m, 2 * m, dtype, rms_weight, rms_eps, out,
                         out_dtype, stream);
}

lcsa_status lcsa_hca_compress(const void* kv, const void* gate, int gate_per_channel, int B, int T, int D, int m,
                              lcsa_dtype dtype, const float* rms_weight, float rms_eps, void* out,
                              lcsa_dtype out_dtype, void* stream) {
  return compress_common(kv, gate, gate_per_channel, B, T, D, m, m, dtype, rms_weight, rms_eps, out, out_dtype,
                         stream);
}

lcsa_status lcsa_compress_entries(const void* kv, const void* gate, int gate_per_channel, int B, int Tkv, int D,
                                  int64_t kv_pos0, int m, int window, int64_t j0, int n_entries, lcsa_dtype dtype,
                                  const float* rms_weight, float rms_eps, void* cache, int64_t cache_rows,
                                  lcsa_dtype out_dtype, void* stream) {
  if (!valid_dtype(dtype) || !valid_dtype(out_dtype)) return LCSA_ERR_INVALID_ARG;
  if (B < 0 || Tkv < 0 || D <= 0 || m <= 0 || window <= 0 || kv_pos0 < 0 || j0 < 0 || n_entries < 0 ||
      cache_rows < 0)
    return LCSA_ERR_INVALID_ARG;
  const int vec = dtype == LCSA_BF16 ? 8 : 4;
  if (D % vec != 0 || D / vec > 1024) return LCSA_ERR_INVALID_ARG;
  if (out_dtype == LCSA_BF16 && D % 8 != 0) return LCSA_ERR_INVALID_ARG;
  if ((long long)B * n_entries == 0) return LCSA_OK;
  if (j0 + n_entries > cache_rows) return LCSA_ERR_INVALID_ARG;
  // windows move right with j: the first one's start and the last one's end bound them all
  const long long first_lo = (j0 + 1) * (long long)m - window > 0 ? (j0 + 1) * (long long)m - window : 0;
  const long long last_hi = (j0 + n_entries) * (long long)m;
  if (first_lo < kv_pos0 || last_hi > kv_pos0 + Tkv) return LCSA_ERR_INVALID_ARG;
  if (!kv || !gate || !cache) return LCSA_ERR_INVALID_ARG;
  if (!aligned16(kv) || !aligned16(cache) || (gate_per_channel && !aligned16(gate))) return LCSA_ERR_INVALID_ARG;
  if (rms_weight && (reinterpret_cast<uintptr_t>(rms_weight) & 3u)) return LCSA_ERR_INVALID_ARG;
  if (!have_device()) return LCSA_ERR_CUDA;
  return from_cuda(launch_compress(kv, gate, gate_per_channel, B, Tkv, D, m, window, dtype, rms_weight, rms_eps,
                                   cache, out_dtype, (cudaStream_t)stream, j0, n_entries, kv_pos0, cache_rows));
}

size_t lcsa_topk_workspace(int rows, int n_cols, int k) {
  if (rows <= 0 || n_cols <= 0 || k <= 0) return 0;
  return topk_long_scratch(rows, n_cols, k);
}

lcsa_status lcsa_topk_from_scores(const float* scores, int rows, int n_cols, int64_t ld, const int32_t* n_valid,
                                  int k, int32_t* idx_out, void* workspace, size_t workspace_bytes,
                                  void* stream) {
  if (rows < 0 || n_cols < 0 || k <= 0 || ld < n_cols) return LCSA_ERR_INVALID_ARG;
  if (rows == 0) return LCSA_OK;
  if (!idx_out || (n_cols > 0 && !scores)) return LCSA_ERR_INVALID_ARG;
  if (!aligned16(idx_out) || (scores && (reinterpret_cast<uintptr_t>(scores) & 3u)) ||
      (n_valid && (reinterpret_cast<uintptr_t>(n_valid) & 3u)))
    return LCSA_ERR_INVALID_ARG;
  if (workspace && !aligned16(workspace)) return LCSA_ERR_INVALID_ARG;
  if (!have_device()) return LCSA_ERR_CUDA;
  return from_cuda(launch_topk(scores, rows, n_cols, (long long)ld, n_valid, k, idx_out, (cudaStream_t)stream,
                               workspace, workspace_bytes));
}

int lcsa_indexer_uses_tensor_cores(const lcsa_indexer_args* a) { return a && indexer_tc_supported(a) ? 1 : 0; }

size_t lcsa_indexer_topk_workspace(const lcsa_indexer_args* a) {
  if (!a || a->B <= 0 || a->Tq <= 0) return 0;
  return indexer_ws_need(indexer_chunk_budget(a->B, a->Tq), a->Nc, a->k, 0);
}

lcsa_status lcsa_indexer_topk(const lcsa_indexer_args* a, void* workspace, size_t workspace_bytes, void* stream) {
  lcsa_status s = check_indexer(a);
  if (s != LCSA_OK) return s;
  if ((long long)a->B * a->Tq == 0) return LCSA_OK;
  if (!have_device()) return LCSA_ERR_CUDA;
  cudaStream_t st = (cudaStream_t)stream;
  const bool tc = indexer_tc_supported(a);
  return indexer_by_chunks(a->B, a->Tq, a->Nc, a->k, a->q_pos0, a->m, a->idx_out, a->scores_out, workspace,
                           workspace_bytes, 0, st,
                           [&](float* sc, int b0, int nb, int i0, int ni, void*) -> cudaError_t {
                             const long long row0 = (long long)b0 * a->Tq + i0;
                             if (tc) return launch_indexer_tc_rect(a, sc, b0, nb, i0, ni, st);
                             if (a->dtype == LCSA_BF16)
                               return launch_indexer_generic_t<__nv_bfloat16>(a, sc, (int)row0, nb * ni, st);
                             return launch_indexer_generic_t<float>(a, sc, (int)row0, nb * ni, st);
                           });
}

// ------------------------------------------------------------------ FP4 indexer path
lcsa_status lcsa_quantize_mxfp4(const void* x, int64_t rows, int cols, lcsa_dtype dtype, uint8_t* codes,
                                uint8_t* scales, void* stream) {
  if (!valid_dtype(dtype) || rows < 0 || cols <= 0 || cols % 32 != 0) return LCSA_ERR_INVALID_ARG;
  if (rows == 0) return LCSA_OK;
  if (!x || !codes || !scales) return LCSA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(x) % esize(dtype) != 0) return LCSA_ERR_INVALID_ARG;
  if (!have_device()) return LCSA_ERR_CUDA;
  const long long n_blocks = rows * (long long)(cols / 32);
  const long long want = (n_blocks + 7) / 8;                       // 8 warps (blocks of 32 values) per CTA
  const int grid = (int)(want < 148LL * 64 ? want : 148LL * 64);
  count_launch();
  if (dtype == LCSA_BF16)
    mxfp4_quantize_kernel<__nv_bfloat16><<<grid, 256, 0, (cudaStream_t)stream>>>(
        (const __nv_bfloat16*)x, n_blocks, codes, scales);
  else
    mxfp4_quantize_kernel<float><<<grid, 256, 0, (cudaStream_t)stream>>>((const float*)x, n_blocks, codes, scales);
  return from_cuda(cudaGetLastError());
}

static lcsa_status check_indexer_mxfp4(const lcsa_indexer_mxfp4_args* a) {
  if (!a) return LCSA_ERR_INVALID_ARG;
  if (a->B < 0 || a->Tq < 0 || a->Nc < 0 || a->H_I <= 0 || a->D_I <= 0 || a->m <= 0 || a->k <= 0 || a->q_pos0 < 0)
    return LCSA_ERR_INVALID_ARG;
  if (a->H_I != 64 || a->D_I != 128) return LCSA_ERR_UNSUPPORTED;
  if ((long long)a->B * a->Tq == 0) return LCSA_OK;
  if (!a->q_idx || !a->w || !a->idx_out || (a->Nc > 0 && (!a->k_codes || !a->k_scales))) return LCSA_ERR_INVALID_ARG;
  if (!aligned16(a->q_idx) || !aligned16(a->w) || !aligned16(a->idx_out) ||
      (a->k_codes && !aligned16(a->k_codes)) || (a->k_scales && (reinterpret_cast<uintptr_t>(a->k_scales) & 3u)) ||
      (a->scores_out && !aligned16(a->scores_out)))
    return LCSA_ERR_INVALID_ARG;
  return LCSA_OK;
}

// prepared queries of one rectangle: E4M3 [rows*64, 128] + head weights [rows*64]
static constexpr size_t kQ8PerRow = 64 * 128 + 64 * 4;

size_t lcsa_indexer_topk_mxfp4_workspace(const lcsa_indexer_mxfp4_args* a) {
  if (!a || a->B <= 0 || a->Tq <= 0) return 0;
  return indexer_ws_need(indexer_chunk_budget(a->B, a->Tq), a->Nc, a->k, kQ8PerRow);
}

lcsa_status lcsa_indexer_topk_mxfp4(const lcsa_indexer_mxfp4_args* a, void* workspace, size_t workspace_bytes,
                                   void* stream) {
  lcsa_status s = check_indexer_mxfp4(a);
  if (s != LCSA_OK) return s;
  if ((long long)a->B * a->Tq == 0) return LCSA_OK;
  if (!have_device()) return LCSA_ERR_CUDA;
  cudaStream_t st = (cudaStream_t)stream;
  return indexer_by_chunks(
      a->B, a->Tq, a->Nc, a->k, a->q_pos0, a->m, a->idx_out, a->scores_out, workspace, workspace_bytes, kQ8PerRow,
      st, [&](float* sc, int b0, int nb, int i0, int ni, void* extra) -> cudaError_t {
        const long long nr = (long long)nb * ni;
        uint8_t* q8 = (uint8_t*)extra;
        float* w8 = (float*)(q8 + align256((size_t)nr * 64 * 128));
        count_launch();
        indexer_q8_kernel<<<(unsigned)((nr * 64 + 7) / 8), 256, 0, st>>>(
            (const __nv_bfloat16*)a->q_idx, a->w, a->Tq, b0, nb, i0, ni, q8, w8);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        // the kernel follows the call's row count, not the chunking, so a
        // smaller workspace gives the same scores
        return launch_indexer_fp4_rect(a->k_codes, a->k_scales, a->B, a->Nc, a->q_pos0, a->m, q8, w8, sc, b0, nb,
                                       i0, ni, a->Tq <= 2, st);
      });
}

// ------------------------------------------------------------------ grouped output projection
static lcsa_status check_out_proj(const lcsa_out_proj_args* a) {
  if (!a) return LCSA_ERR_INVALID_ARG;
  if (a->T < 0 || a->n_h <= 0 || a->c <= 0 || a->g <= 0 || a->d_g <= 0 || a->d <= 0) return LCSA_ERR_INVALID_ARG;
  if (a->n_h % a->g != 0) return LCSA_ERR_INVALID_ARG;
  const long long K = (long long)(a->n_h / a->g) * a->c;
  if (K % 64 != 0 || ((long long)a->g * a->d_g) % 64 != 0 || a->d_g % 8 != 0 || a->d % 8 != 0)
    return LCSA_ERR_INVALID_ARG;
  if (K > (1 << 30) || (long long)a->g * a->d_g > (1 << 30)) return LCSA_ERR_INVALID_ARG;
  if (a->T == 0) return LCSA_OK;
  if (!a->o || !a->w_group || !a->w_out || !a->y) return LCSA_ERR_INVALID_ARG;
  if (!aligned16(a->o) || !aligned16(a->w_group) || !aligned16(a->w_out) || !aligned16(a->y))
    return LCSA_ERR_INVALID_ARG;
  return LCSA_OK;
}

size_t lcsa_grouped_out_proj_workspace(const lcsa_out_proj_args* a) {
  if (!a || a->T <= 0 || a->g <= 0 || a->d_g <= 0) return 0;
  return align256((size_t)a->T * (size_t)a->g * (size_t)a->d_g * 2);
}

lcsa_status lcsa_grouped_out_proj(const lcsa_out_proj_args* a, void* workspace, size_t workspace_bytes,
                                  void* stream) {
  lcsa_status s = check_out_proj(a);
  if (s != LCSA_OK) return s;
  if (a->T == 0) return LCSA_OK;
  if (!workspace || workspace_bytes < lcsa_grouped_out_proj_workspace(a)) return LCSA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return LCSA_ERR_INVALID_ARG;
  if (!have_device()) return LCSA_ERR_CUDA;
  cudaStream_t st = (cudaStream_t)stream;
  const int K = a->n_h / a->g * a->c;
  const long long gd = (long long)a->g * a->d_g;
  __nv_bfloat16* mid = (__nv_bfloat16*)workspace;
  const int sms = sm_count();
  cudaError_t e = launch_gemm_bf16(a->o, (long long)a->n_h * a->c, a->w_group, mid, gd, a->T, a->d_g, K, a->g, sms,
                                   st);
  if (e != cudaSuccess) return LCSA_ERR_CUDA;
  e = launch_gemm_bf16(mid, gd, a->w_out, (__nv_bfloat16*)a->y, a->d, a->T, a->d, (int)gd, 1, sms, st);
  return from_cuda(e);
}

int lcsa_attn_uses_tensor_cores(const lcsa_attn_args* a) { return a && attn_tc_supported(a) ? 1 : 0; }

size_t lcsa_attn_workspace(const lcsa_attn_args* a, int sparse) {
  if (!a || a->B <= 0 || a->Tq <= 0 || !attn_tc_supported(a)) return 0;
  return attn_tc_workspace(a, sparse);
}

static lcsa_status attn_common(const lcsa_attn_args* a, int sparse, void* ws, size_t ws_bytes, void* stream) {
  lcsa_status s = check_attn(a, sparse);
  if (s != LCSA_OK) return s;
  if ((long long)a->B * a->Tq == 0) return LCSA_OK;
  if (!have_device()) return LCSA_ERR_CUDA;
  cudaStream_t st = (cudaStream_t)stream;
  if (attn_tc_supported(a)) {
    const size_t need = attn_tc_workspace(a, sparse);
    if (need > 0 && (!ws || ws_bytes < need)) return LCSA_ERR_WORKSPACE;
    if (ws && !aligned16(ws)) return LCSA_ERR_INVALID_ARG;
    return from_cuda(launch_attn_tc(a, sparse, ws, st));
  }
  return from_cuda(launch_attn_generic(a, sparse, st));
}

lcsa_status lcsa_csa_sparse_attn(const lcsa_attn_args* a, void* ws, size_t ws_bytes, void* stream) {
  return attn_common(a, 1, ws, ws_bytes, stream);
}

lcsa_status lcsa_hca_dense_attn(const lcsa_attn_args* a, void* ws, size_t ws_bytes, void* stream) {
  return attn_common(a, 0, ws, ws_bytes, stream);
}

// ------------------------------------------------------------------ FP8 entry cache
lcsa_status lcsa_quantize_entries_fp8(const void* x, int64_t rows, int D, int R, lcsa_dtype dtype, uint8_t* codes,
                                      uint8_t* scales, void* rope, void* stream) {
  if (!valid_dtype(dtype) || rows < 0 || D <= 0 || R < 0 || R >= D || (R & 1)) return LCSA_ERR_INVALID_ARG;
  if (rows == 0) return LCSA_OK;
  if (!x || !codes || !scales || (R > 0 && !rope)) return LCSA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(x) % esize(dtype) != 0 || (reinterpret_cast<uintptr_t>(rope) & 1u))
    return LCSA_ERR_INVALID_ARG;
  if (!have_device()) return LCSA_ERR_CUDA;
  return from_cuda(launch_quantize_entries_fp8(x, rows, D, R, dtype, codes, scales, rope, (cudaStream_t)stream));
}

static lcsa_status attn_fp8_common(const lcsa_attn_args* a, const lcsa_fp8_entries* f8, int sparse, void* ws,
                                   size_t ws_bytes, void* stream) {
  lcsa_status s = check_attn(a, sparse, 0);
  if (s != LCSA_OK) return s;
  if (!f8) return LCSA_ERR_INVALID_ARG;
  if (!attn_tc_supported(a)) return LCSA_ERR_UNSUPPORTED;
  if ((long long)a->B * a->Tq == 0) return LCSA_OK;
  if (a->Nc > 0 && (!f8->codes || !f8->scales || !f8->rope || !aligned16(f8->codes) || !aligned16(f8->rope)))
    return LCSA_ERR_INVALID_ARG;
  if (!have_device()) return LCSA_ERR_CUDA;
  const size_t need = attn_tc_workspace(a, sparse);
  if (need > 0 && (!ws || ws_bytes < need)) return LCSA_ERR_WORKSPACE;
  if (ws && !aligned16(ws)) return LCSA_ERR_INVALID_ARG;
  return from_cuda(launch_attn_tc(a, sparse, ws, (cudaStream_t)stream, f8));
}

lcsa_status lcsa_csa_sparse_attn_fp8(const lcsa_attn_args* a, const lcsa_fp8_entries* e, void* ws, size_t ws_bytes,
                                     void* stream) {
  return attn_fp8_common(a, e, 1, ws, ws_bytes, stream);
}

lcsa_status lcsa_hca_dense_attn_fp8(const lcsa_attn_args* a, const lcsa_fp8_entries* e, void* ws, size_t ws_bytes,
                                    void* stream) {
  return attn_fp8_common(a, e, 0, ws, ws_bytes, stream);
}

}  // extern "C"
