// Internal interface of the block-sparse prefill (prefill.cu) used by api.cu.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/lserve.h"

namespace lserve {

size_t prefill_workspace_bytes(const lserve_prefill_desc* desc);

int prefill_entry(const lserve_prefill_desc* desc, const void* q, const void* k, const void* v,
                  const uint8_t* head_kind_host, float softmax_scale, void* out, float* lse,
                  void* workspace, size_t workspace_bytes, cudaStream_t stream);

// The prefill with the paged epilogue (pd != nullptr): this sequence's K / V
// into the pools through block_table and the retrieval heads' page statistics,
// written by the kernel itself.  The caller has validated pd against d.
int prefill_paged_entry(const lserve_prefill_desc* d, const lserve_paged_desc* pd, const void* q,
                        const void* k, const void* v, const uint8_t* head_kind_host,
                        float softmax_scale, void* out, float* lse, const int32_t* block_table,
                        void* k_pool, void* v_pool, void* stats_pool, void* workspace,
                        size_t workspace_bytes, cudaStream_t stream);

}  // namespace lserve
