// Block-sparse prefill: placeholder until the tcgen05 kernel lands.
#include "prefill.h"

namespace lserve {

size_t prefill_workspace_bytes(const lserve_prefill_desc*) { return 0; }

int prefill_entry(const lserve_prefill_desc*, const void*, const void*, const void*, const uint8_t*,
                  float, void*, float*, void*, size_t, cudaStream_t) {
  return LSERVE_ERR_UNSUPPORTED;
}

}  // namespace lserve
