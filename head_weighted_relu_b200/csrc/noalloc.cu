// noalloc.cu -- indexer_topk for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocator) at the point where
// they run the indexer: code inside a custom allocator or memory-pool hook,
// plugins whose host framework owns every device allocation, or programs
// that must not allocate after start-up.  indexer_topk_noalloc gives them the
// same computation with its scratch memory taken from a fixed array in this
// library's device image instead of a caller-provided workspace.
//
// The array below is part of the module: every GPU that loads this library
// holds it (kNoAllocScratchBytes) until the process exits.  Its host-side name
// is only a stand-in; the device address is looked up per device with
// cudaGetSymbolAddress, which is the only value ever handed to a kernel.
#include <mutex>

#include "hwr_indexer.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;  // 64 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

void* g_scratch_addr[kMaxDevices];
std::mutex g_scratch_mutex;

// Device address of the scratch array on the current device; looked up on
// the first call per device (with that device current) and cached for the
// life of the process (a cudaDeviceReset would invalidate it).
indexer_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return INDEXER_ECUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return INDEXER_ECUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return INDEXER_OK;
}

}  // namespace

extern "C" {

indexer_status indexer_topk_noalloc(const indexer_problem* p, const void* q, const void* k, const float* w,
                                    const float* q_scale, const float* k_scale, const void* pool_coef,
                                    int32_t* out_idx, int32_t* out_len, float* out_score, void* stream) {
  size_t need = 0;
  indexer_status st = indexer_workspace_bytes(p, &need);
  if (st != INDEXER_OK) return st;
  if (need > kNoAllocScratchBytes) return INDEXER_EWORKSPACE;
  void* scratch = nullptr;
  st = scratch_address(&scratch);
  if (st != INDEXER_OK) return st;
  return indexer_topk(p, q, k, w, q_scale, k_scale, pool_coef, out_idx, out_len, out_score, scratch,
                      kNoAllocScratchBytes, stream);
}

indexer_status indexer_noalloc_read_status(int32_t* flags, void* stream) {
  if (!flags) return INDEXER_EINVAL;
  void* scratch = nullptr;
  indexer_status st = scratch_address(&scratch);
  if (st != INDEXER_OK) return st;
  // the status word sits at the start of the scratch array, as at the start
  // of any indexer_topk workspace
  return indexer_read_status(scratch, flags, stream);
}

}  // extern "C"
