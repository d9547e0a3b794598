// lcsa_indexer_topk_noalloc: the indexer + top-k call for callers that cannot
// allocate device memory.
//
// Some callers have no way to obtain device memory at the point where they
// call us: code running inside a memory pool or arena they do not own, an
// inference runtime that forbids allocation after start-up, or a host thread
// that must not synchronise the device (cudaMalloc/cudaFree can synchronise).
// lcsa_indexer_topk needs a score workspace from its caller; this variant
// instead uses one fixed scratch array that lives in the library's device
// image, so the caller passes only inputs and outputs.
//
// The scratch is a file-scope __device__ array of kNoAllocScratchBytes
// (32 MiB).  Every GPU that loads the library holds it until the process
// exits.  Host code cannot use the array's name as a device address (in host
// code it names a host-side stand-in), so the call looks the device address
// up with cudaGetSymbolAddress in the current context.  That address belongs
// to the context (and the copy of the module loaded into it): after a
// cudaDeviceReset, or in another context, it is a different one.  So every
// call outside stream capture looks it up afresh and remembers it for the
// current context; a call made while its stream is being captured uses the
// address remembered for the current context, and fails with LCSA_ERR_CUDA if
// there is none yet.
#include <cuda.h>
#include <cuda_runtime.h>
#include <mutex>

#include "lcsa.h"

lcsa_status lcsa_internal_check_indexer(const lcsa_indexer_args* a);
size_t lcsa_internal_indexer_one_row_bytes(const lcsa_indexer_args* a);

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;
constexpr int kMaxContexts = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

struct ScratchEntry {
  CUcontext ctx;
  void* addr;
};
std::mutex g_mutex;
ScratchEntry g_cache[kMaxContexts] = {};
int g_cache_n = 0;

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

// The current driver context (through the runtime's driver entry point, so the
// library needs no -lcuda); nullptr when it cannot be determined.
CUcontext current_context() {
  static CtxGetCurrentFn fn = []() -> CtxGetCurrentFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<CtxGetCurrentFn>(p);
    return nullptr;
  }();
  CUcontext c = nullptr;
  if (fn == nullptr || fn(&c) != CUDA_SUCCESS) return nullptr;
  return c;
}

// Device address of the scratch array in the current context (see the file
// comment for when it is looked up and when it is taken from the cache).
lcsa_status scratch_for_current_context(cudaStream_t st, void** ptr) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return LCSA_ERR_CUDA;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) return LCSA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (cs == cudaStreamCaptureStatusNone) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return LCSA_ERR_CUDA;
    const CUcontext ctx = current_context();        // exists now: the lookup above made it current
    if (ctx != nullptr) {
      int i = 0;
      while (i < g_cache_n && g_cache[i].ctx != ctx) ++i;
      if (i < g_cache_n) g_cache[i].addr = p;
      else if (g_cache_n < kMaxContexts) g_cache[g_cache_n++] = ScratchEntry{ctx, p};
    }
    *ptr = p;
    return LCSA_OK;
  }
  const CUcontext ctx = current_context();
  for (int i = 0; ctx != nullptr && i < g_cache_n; ++i)
    if (g_cache[i].ctx == ctx) {
      *ptr = g_cache[i].addr;
      return LCSA_OK;
    }
  return LCSA_ERR_CUDA;    // no call outside capture has run in this context yet
}

}  // namespace

extern "C" lcsa_status lcsa_indexer_topk_noalloc(const lcsa_indexer_args* a, void* stream) {
  // the same argument checks as lcsa_indexer_topk, before anything touches the device
  const lcsa_status v = lcsa_internal_check_indexer(a);
  if (v != LCSA_OK) return v;
  if ((long long)a->B * a->Tq == 0) return LCSA_OK;
  // The scratch must hold what one query row needs: its Nc FP32 scores, its
  // visible count and, for rows longer than 32768 columns, the two-phase
  // top-k scratch of that row.
  if (lcsa_internal_indexer_one_row_bytes(a) > kNoAllocScratchBytes) return LCSA_ERR_WORKSPACE;
  void* scratch = nullptr;
  const lcsa_status s = scratch_for_current_context((cudaStream_t)stream, &scratch);
  if (s != LCSA_OK) return s;
  // Every scratch element a chunk reads is written earlier in the same chunk
  // (scores of the visible entries, per-row counts), so nothing is cleared.
  return lcsa_indexer_topk(a, scratch, kNoAllocScratchBytes, stream);
}
