// lserve_page_select_noalloc: page selection for callers that cannot allocate
// device memory.
//
// lserve_page_select needs scratch space for the physical-page scores, which
// the caller normally provides as a workspace allocated with cudaMalloc (or
// a framework allocator).  Some callers cannot do that: code running inside a
// host callback or a driver-level hook, plug-ins whose host process owns
// every allocation, or a thread that must not take the allocator's locks.
// This entry point keeps the scores in a fixed-size array that lives in the
// library's own device memory instead, so the call allocates nothing.
//
// The array (kNoAllocScores floats, 4 MiB) is a file-scope __device__
// variable: every GPU that loads the library holds one copy until the process
// exits.  All calls on a device share it; the scores of the previous call
// stay there and are overwritten by the next one (each call writes every
// entry it reads, so nothing needs clearing).  Calls whose executions overlap
// on the GPU -- on different streams, or in different threads -- race on the
// array and may produce wrong selections.
#include <mutex>

#include "../../include/lserve.h"
#include "common.cuh"

namespace {

constexpr size_t kNoAllocScores = 1u << 20;  // B * H_kv * max_pages_per_seq limit

static __device__ __align__(256) float g_noalloc_scores[kNoAllocScores];

// Device address of the array on the current device.  The first call on each
// device looks it up (with that device current) and caches it.
float* noalloc_scores_ptr() {
  static std::mutex mu;
  static float* cache[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!cache[dev]) {
    float* ptr = nullptr;
    if (cudaGetSymbolAddress((void**)&ptr, g_noalloc_scores) != cudaSuccess) return nullptr;
    cache[dev] = ptr;
  }
  return cache[dev];
}

}  // namespace

extern "C" int lserve_page_select_noalloc(const lserve_paged_desc* desc, const void* q,
                                          const void* stats_pool, const int32_t* block_table,
                                          const int32_t* ctx_lens, const uint8_t* head_kind,
                                          int32_t top_k, int32_t* sel, int32_t* sel_count,
                                          void* stream) {
  if (!desc) return LSERVE_ERR_INVALID_ARG;
  const long long need = (long long)desc->batch * desc->num_kv_heads * desc->max_pages_per_seq;
  if (desc->batch < 1 || desc->num_kv_heads < 1 || desc->max_pages_per_seq < 1)
    return LSERVE_ERR_INVALID_ARG;
  if (need > (long long)kNoAllocScores) return LSERVE_ERR_UNSUPPORTED;
  float* scores = noalloc_scores_ptr();
  if (!scores) return LSERVE_ERR_CUDA;
  // the scores land in the static array instead of a caller workspace
  return lserve_page_select(desc, q, stats_pool, block_table, ctx_lens, head_kind, top_k, sel,
                            sel_count, scores, nullptr, 0, stream);
}
