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
// code it names a host-side stand-in), so the first call on each device looks
// up its device address with cudaGetSymbolAddress while that device is
// current and caches it.
#include <cuda_runtime.h>
#include <mutex>

#include "lcsa.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set up once per device).
lcsa_status scratch_for_current_device(void** ptr) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return LCSA_ERR_CUDA;
  if (dev >= kMaxDevices) return LCSA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return LCSA_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *ptr = g_scratch_addr[dev];
  return LCSA_OK;
}

inline size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

extern "C" lcsa_status lcsa_indexer_topk_noalloc(const lcsa_indexer_args* a, void* stream) {
  if (!a) return LCSA_ERR_INVALID_ARG;
  if ((long long)a->B * a->Tq == 0) return lcsa_indexer_topk(a, nullptr, 0, stream);
  // The scratch must hold at least one score row (Nc floats) plus its count.
  const size_t one_row = round256((size_t)(a->Nc > 0 ? a->Nc : 1) * 4) + round256(4);
  if (a->Nc < 0 || one_row > kNoAllocScratchBytes) return LCSA_ERR_WORKSPACE;
  void* scratch = nullptr;
  lcsa_status s = scratch_for_current_device(&scratch);
  if (s != LCSA_OK) return s;
  // Every scratch element a chunk reads is written earlier in the same chunk
  // (scores of the visible entries, per-row counts), so nothing is cleared.
  return lcsa_indexer_topk(a, scratch, kNoAllocScratchBytes, stream);
}
