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

}  // namespace lserve
