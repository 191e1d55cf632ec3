// C-ABI entry points of liblserve.so (declared in include/lserve.h): argument
// validation, tensor-map encoding, workspace carving and kernel launches.
#include <cudaTypedefs.h>

#include <cmath>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "prefill.h"

namespace lserve {

__device__ unsigned int g_status = 0;

namespace {

constexpr uint64_t kDefaultWaitLimit = 4000000000ull;  // ~2 s at 1.9 GHz
uint64_t g_wait_limit = kDefaultWaitLimit;

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int sm_count_current() {
  static std::mutex mu;
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  std::lock_guard<std::mutex> lock(mu);
  if (cache[dev] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cache[dev] = v;
  }
  return cache[dev];
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return (PFN_cuTensorMapEncodeTiled_v12000) nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }();
  return fn;
}

}  // namespace

// 2-D bf16 tensor map [rows][cols] (row pitch `pitch_elems`), 128-byte swizzle,
// box of box_rows x 64 columns.
bool make_map_2d(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint64_t pitch_elems,
                 uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {pitch_elems * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t set_smem_once(const void* kernel, int bytes) {
  struct Entry {
    const void* fn;
    int dev;
    int bytes;
  };
  static std::mutex mu;
  static Entry done[256];
  static int ndone = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < ndone; ++i)
    if (done[i].fn == kernel && done[i].dev == dev && done[i].bytes >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  if (ndone < 256) done[ndone++] = Entry{kernel, dev, bytes};
  return cudaSuccess;
}

// Contiguous bf16 tensor [d2][d1][d0] (rank 2 or 3), box b0 x b1 x b2, 128-byte swizzle.
bool make_map_tiled(CUtensorMap* m, const void* base, int rank, uint64_t d0, uint64_t d1, uint64_t d2,
                    uint32_t b0, uint32_t b1, uint32_t b2) {
  auto fn = encode_fn();
  if (!fn || rank < 2 || rank > 3) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
  cuuint32_t box[3] = {b0, b1, b2};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void*>(base), dims,
            strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Rows of quantized codes (row_bytes = D or D / 2 bytes): a 2-D byte view,
// box_rows whole rows a copy, swizzled by the row width (128, 64 or 32 bytes)
// so that the rows a warp reads at once fall in different shared-memory banks.
bool make_map_codes(CUtensorMap* m, const void* base, uint64_t rows, uint32_t row_bytes,
                    uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  CUtensorMapSwizzle sw;
  if (row_bytes == 128) sw = CU_TENSOR_MAP_SWIZZLE_128B;
  else if (row_bytes == 64) sw = CU_TENSOR_MAP_SWIZZLE_64B;
  else if (row_bytes == 32) sw = CU_TENSOR_MAP_SWIZZLE_32B;
  else return false;
  cuuint64_t dims[2] = {row_bytes, rows};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {row_bytes, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

uint64_t wait_limit() { return g_wait_limit; }
int current_sm_count() { return sm_count_current(); }

// Device address of g_status on the current device (cached per device).
unsigned int* device_status_word() {
  static std::mutex mu;
  static unsigned int* cache[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!cache[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_status) != cudaSuccess) return nullptr;
    cache[dev] = static_cast<unsigned int*>(ptr);
  }
  return cache[dev];
}

static __global__ void wait_timeout_probe_kernel(uint64_t cycles, unsigned int* status) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    // nobody arrives: the bounded wait must give up and raise the flag
    (void)mbar_wait(&bar, 0, cycles, status);
  }
}

cudaError_t launch_wait_timeout_probe(uint64_t cycles, unsigned int* status, cudaStream_t stream) {
  wait_timeout_probe_kernel<<<1, 32, 0, stream>>>(cycles, status);
  return cudaGetLastError();
}

}  // namespace lserve

using namespace lserve;

namespace {

bool valid_paged(const lserve_paged_desc* d) {
  if (!d) return false;
  if (d->batch < 1 || d->num_kv_heads < 1 || d->num_q_heads < d->num_kv_heads) return false;
  if (d->num_q_heads % d->num_kv_heads) return false;
  if (d->logical_page < 1 || d->physical_page < d->logical_page) return false;
  if (d->physical_page % d->logical_page) return false;
  if (d->max_pages_per_seq < 1 || d->num_pool_pages < 1) return false;
  return true;
}

int supported_paged(const lserve_paged_desc* d) {
  const int G = d->num_q_heads / d->num_kv_heads;
  if (d->head_dim != 64 && d->head_dim != 128) return LSERVE_ERR_UNSUPPORTED;
  if (G != 1 && G != 2 && G != 4 && G != 8) return LSERVE_ERR_UNSUPPORTED;
  if (d->logical_page != 8 && d->logical_page != 16 && d->logical_page != 32 && d->logical_page != 64)
    return LSERVE_ERR_UNSUPPORTED;
  // tiles of min(N_P, 64) tokens: N_P = 32, or a multiple of 64 up to 1024
  if (!(d->physical_page == 32 || (d->physical_page % 64 == 0 && d->physical_page <= 1024)))
    return LSERVE_ERR_UNSUPPORTED;
  const long long rows = (long long)d->num_pool_pages * d->num_kv_heads * d->physical_page;
  if (rows >= (1ll << 31)) return LSERVE_ERR_UNSUPPORTED;
  return LSERVE_OK;
}

size_t select_ws(const lserve_paged_desc* d) {
  return ((size_t)d->batch * d->num_kv_heads * d->max_pages_per_seq * 4 + 255) / 256 * 256;
}

size_t decode_ws(const lserve_paged_desc* d) {
  const int sms = current_sm_count();
  if (sms <= 0) return 0;
  const int G = d->num_q_heads / d->num_kv_heads;
  return decode_workspace_bytes(d->batch * d->num_kv_heads, decode_grid(sms), G, d->head_dim);
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? LSERVE_OK : LSERVE_ERR_CUDA; }

}  // namespace

extern "C" {

const char* lserve_status_string(int s) {
  switch (s) {
    case LSERVE_OK: return "ok";
    case LSERVE_ERR_INVALID_ARG: return "invalid argument";
    case LSERVE_ERR_UNSUPPORTED: return "unsupported shape or parameter";
    case LSERVE_ERR_WORKSPACE: return "workspace missing or too small";
    case LSERVE_ERR_CUDA: return "CUDA runtime error";
    case LSERVE_ERR_TIMEOUT: return "bounded device wait timed out";
    case LSERVE_ERR_BOUNDS: return "index out of range (page skipped)";
    default: return "unknown status";
  }
}

int lserve_bounds_checked(void) { return kCheckBounds ? 1 : 0; }

void lserve_set_wait_limit_cycles(uint64_t cycles) {
  g_wait_limit = cycles ? cycles : kDefaultWaitLimit;
}

size_t lserve_workspace_size(int op, const void* desc, int32_t top_k) {
  (void)top_k;  // no workspace depends on it
  if (!desc) return 0;
  switch (op) {
    case LSERVE_OP_STATS:  // the statistics kernel needs no workspace
      return 0;
    case LSERVE_OP_SELECT: {
      const auto* d = static_cast<const lserve_paged_desc*>(desc);
      return valid_paged(d) ? select_ws(d) : 0;
    }
    case LSERVE_OP_DECODE: {
      const auto* d = static_cast<const lserve_paged_desc*>(desc);
      if (!valid_paged(d) || supported_paged(d) != LSERVE_OK) return 0;
      return decode_ws(d);
    }
    case LSERVE_OP_PREFILL:
      return prefill_workspace_bytes(static_cast<const lserve_prefill_desc*>(desc));
    default:
      return 0;
  }
}

int lserve_read_device_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return LSERVE_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(v)) != cudaSuccess) return LSERVE_ERR_CUDA;
  const unsigned int zero = 0;
  if (cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)) != cudaSuccess) return LSERVE_ERR_CUDA;
  if (v & (1u << LSERVE_ERR_TIMEOUT)) return LSERVE_ERR_TIMEOUT;
  if (v & (1u << LSERVE_ERR_BOUNDS)) return LSERVE_ERR_BOUNDS;
  return LSERVE_OK;
}

int lserve_debug_wait_timeout(uint64_t cycles, void* stream) {
  if (cycles == 0 || cycles > (1ull << 40)) return LSERVE_ERR_INVALID_ARG;
  unsigned int* st = device_status_word();
  if (!st) return LSERVE_ERR_CUDA;
  return cuda_status(launch_wait_timeout_probe(cycles, st, static_cast<cudaStream_t>(stream)));
}

int lserve_page_stats(const lserve_paged_desc* desc, const void* k_pool, const int32_t* block_table,
                      const int32_t* ctx_lens, const uint8_t* head_kind, void* stats_pool,
                      int32_t first_logical_page, void* stream) {
  if (!valid_paged(desc)) return LSERVE_ERR_INVALID_ARG;
  if (!k_pool || !block_table || !ctx_lens || !head_kind || !stats_pool) return LSERVE_ERR_INVALID_ARG;
  if (!aligned(k_pool, 16) || !aligned(stats_pool, 16) || !aligned(block_table, 4) ||
      !aligned(ctx_lens, 4))
    return LSERVE_ERR_INVALID_ARG;
  if (first_logical_page < 0) return LSERVE_ERR_INVALID_ARG;
  const int st = supported_paged(desc);
  if (st != LSERVE_OK) return st;
  StatsParams p;
  p.k_pool = static_cast<const __nv_bfloat16*>(k_pool);
  p.block_table = block_table;
  p.ctx_lens = ctx_lens;
  p.head_kind = head_kind;
  p.stats_pool = static_cast<__nv_bfloat16*>(stats_pool);
  p.batch = desc->batch;
  p.num_kv_heads = desc->num_kv_heads;
  p.logical_page = desc->logical_page;
  p.physical_page = desc->physical_page;
  p.max_pages = desc->max_pages_per_seq;
  p.num_pool_pages = desc->num_pool_pages;
  p.first_logical_page = first_logical_page;
  p.status = device_status_word();
  if (!p.status) return LSERVE_ERR_CUDA;
  const int g = desc->physical_page / desc->logical_page;
  const long long max_lp = (long long)desc->max_pages_per_seq * g;
  if (max_lp >= (1ll << 30)) return LSERVE_ERR_UNSUPPORTED;
  return cuda_status(launch_page_stats(p, desc->head_dim, (int)max_lp, static_cast<cudaStream_t>(stream)));
}

int lserve_prefill_to_pages(const lserve_paged_desc* desc, int32_t seq_len, const void* k,
                            const void* v, const int32_t* block_table, const uint8_t* head_kind,
                            void* k_pool, void* v_pool, void* stats_pool, void* stream) {
  if (!valid_paged(desc)) return LSERVE_ERR_INVALID_ARG;
  if (seq_len < 0) return LSERVE_ERR_INVALID_ARG;
  if (!k || !v || !block_table || !head_kind || !k_pool || !v_pool || !stats_pool)
    return LSERVE_ERR_INVALID_ARG;
  if (!aligned(k, 16) || !aligned(v, 16) || !aligned(k_pool, 16) || !aligned(v_pool, 16) ||
      !aligned(stats_pool, 16) || !aligned(block_table, 4))
    return LSERVE_ERR_INVALID_ARG;
  const int st = supported_paged(desc);
  if (st != LSERVE_OK) return st;
  if ((long long)seq_len > (long long)desc->max_pages_per_seq * desc->physical_page)
    return LSERVE_ERR_INVALID_ARG;
  if (seq_len == 0) return LSERVE_OK;
  ToPagesParams p;
  p.k = static_cast<const __nv_bfloat16*>(k);
  p.v = static_cast<const __nv_bfloat16*>(v);
  p.block_table = block_table;
  p.head_kind = head_kind;
  p.k_pool = static_cast<__nv_bfloat16*>(k_pool);
  p.v_pool = static_cast<__nv_bfloat16*>(v_pool);
  p.stats_pool = static_cast<__nv_bfloat16*>(stats_pool);
  p.seq_len = seq_len;
  p.num_kv_heads = desc->num_kv_heads;
  p.logical_page = desc->logical_page;
  p.physical_page = desc->physical_page;
  p.max_pages = desc->max_pages_per_seq;
  p.num_pool_pages = desc->num_pool_pages;
  p.status = device_status_word();
  if (!p.status) return LSERVE_ERR_CUDA;
  return cuda_status(launch_prefill_to_pages(p, desc->head_dim, static_cast<cudaStream_t>(stream)));
}

int lserve_decode_append(const lserve_paged_desc* desc, const void* k_new, const void* v_new,
                         const int32_t* block_table, const int32_t* ctx_lens,
                         const uint8_t* head_kind, void* k_pool, void* v_pool, void* stats_pool,
                         void* stream) {
  if (!valid_paged(desc)) return LSERVE_ERR_INVALID_ARG;
  if (!k_new || !v_new || !block_table || !ctx_lens || !head_kind || !k_pool || !v_pool || !stats_pool)
    return LSERVE_ERR_INVALID_ARG;
  if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(k_pool, 16) || !aligned(v_pool, 16) ||
      !aligned(stats_pool, 16) || !aligned(block_table, 4) || !aligned(ctx_lens, 4))
    return LSERVE_ERR_INVALID_ARG;
  const int st = supported_paged(desc);
  if (st != LSERVE_OK) return st;
  AppendParams p;
  p.k_new = static_cast<const __nv_bfloat16*>(k_new);
  p.v_new = static_cast<const __nv_bfloat16*>(v_new);
  p.block_table = block_table;
  p.ctx_lens = ctx_lens;
  p.head_kind = head_kind;
  p.k_pool = static_cast<__nv_bfloat16*>(k_pool);
  p.v_pool = static_cast<__nv_bfloat16*>(v_pool);
  p.stats_pool = static_cast<__nv_bfloat16*>(stats_pool);
  p.batch = desc->batch;
  p.num_kv_heads = desc->num_kv_heads;
  p.logical_page = desc->logical_page;
  p.physical_page = desc->physical_page;
  p.max_pages = desc->max_pages_per_seq;
  p.num_pool_pages = desc->num_pool_pages;
  p.status = device_status_word();
  if (!p.status) return LSERVE_ERR_CUDA;
  return cuda_status(launch_decode_append(p, desc->head_dim, static_cast<cudaStream_t>(stream)));
}

int lserve_page_select(const lserve_paged_desc* desc, const void* q, const void* stats_pool,
                       const int32_t* block_table, const int32_t* ctx_lens, const uint8_t* head_kind,
                       int32_t top_k, int32_t* sel, int32_t* sel_count, float* phys_scores,
                       void* workspace, size_t workspace_bytes, void* stream) {
  if (!valid_paged(desc)) return LSERVE_ERR_INVALID_ARG;
  if (!q || !stats_pool || !block_table || !ctx_lens || !head_kind || !sel || !sel_count)
    return LSERVE_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(stats_pool, 16) || !aligned(sel, 4) || !aligned(sel_count, 4) ||
      !aligned(block_table, 4) || !aligned(ctx_lens, 4) || (phys_scores && !aligned(phys_scores, 4)))
    return LSERVE_ERR_INVALID_ARG;
  if (top_k < 1 || top_k > desc->max_pages_per_seq) return LSERVE_ERR_INVALID_ARG;
  const int st = supported_paged(desc);
  if (st != LSERVE_OK) return st;
  if (desc->max_pages_per_seq > kTopkMaxPages) return LSERVE_ERR_UNSUPPORTED;
  float* scores = phys_scores;
  if (!scores) {
    if (!workspace || workspace_bytes < select_ws(desc) || !aligned(workspace, 16))
      return LSERVE_ERR_WORKSPACE;
    scores = static_cast<float*>(workspace);
  }
  SelectParams p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.stats_pool = static_cast<const __nv_bfloat16*>(stats_pool);
  p.block_table = block_table;
  p.ctx_lens = ctx_lens;
  p.head_kind = head_kind;
  p.scores = scores;
  p.sel = sel;
  p.sel_count = sel_count;
  p.batch = desc->batch;
  p.num_q_heads = desc->num_q_heads;
  p.num_kv_heads = desc->num_kv_heads;
  p.logical_page = desc->logical_page;
  p.physical_page = desc->physical_page;
  p.max_pages = desc->max_pages_per_seq;
  p.num_pool_pages = desc->num_pool_pages;
  p.top_k = top_k;
  p.status = device_status_word();
  if (!p.status) return LSERVE_ERR_CUDA;
  return cuda_status(launch_page_select(p, desc->head_dim, static_cast<cudaStream_t>(stream)));
}

int lserve_sparse_decode_attn(const lserve_paged_desc* desc, const void* q, const void* k_pool,
                              const void* v_pool, const int32_t* block_table, const int32_t* ctx_lens,
                              const uint8_t* head_kind, const int32_t* sel, const int32_t* sel_count,
                              int32_t top_k, int32_t sink_tokens, int32_t local_tokens,
                              float softmax_scale, void* out, float* lse, void* workspace,
                              size_t workspace_bytes, void* stream) {
  return lserve_sparse_decode_attn_ex(desc, q, k_pool, v_pool, block_table, ctx_lens, head_kind, sel,
                                      sel_count, top_k, sink_tokens, local_tokens, softmax_scale, out,
                                      lse, 0u, workspace, workspace_bytes, stream);
}

}  // extern "C"

namespace {

// Validation and parameters shared by the bf16 and int8 decode entry points
// (everything except the KV pools).
int decode_params(const lserve_paged_desc* desc, const void* q, const int32_t* block_table,
                  const int32_t* ctx_lens, const uint8_t* head_kind, const int32_t* sel,
                  const int32_t* sel_count, int32_t top_k, int32_t sink_tokens, int32_t local_tokens,
                  float softmax_scale, void* out, float* lse, uint32_t flags, void* workspace,
                  size_t workspace_bytes, DecodeParams& p, int& grid) {
  if (!valid_paged(desc)) return LSERVE_ERR_INVALID_ARG;
  if (flags & ~(uint32_t)(LSERVE_DECODE_OVERLAP_PROLOGUE | LSERVE_DECODE_OUT_F32 |
                          LSERVE_DECODE_PREFETCH_KV))
    return LSERVE_ERR_INVALID_ARG;
  if (!q || !block_table || !ctx_lens || !head_kind || !sel || !sel_count || !out)
    return LSERVE_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(out, 16) || !aligned(block_table, 4) || !aligned(ctx_lens, 4) ||
      !aligned(sel, 4) || !aligned(sel_count, 4) || (lse && !aligned(lse, 4)))
    return LSERVE_ERR_INVALID_ARG;
  if (top_k < 1 || top_k > desc->max_pages_per_seq) return LSERVE_ERR_INVALID_ARG;
  if (sink_tokens < 0 || local_tokens < 0 || !std::isfinite(softmax_scale)) return LSERVE_ERR_INVALID_ARG;
  const int st = supported_paged(desc);
  if (st != LSERVE_OK) return st;
  const size_t need = decode_ws(desc);
  if (need == 0) return LSERVE_ERR_CUDA;
  if (!workspace || workspace_bytes < need || !aligned(workspace, 256)) return LSERVE_ERR_WORKSPACE;
  const int D = desc->head_dim, G = desc->num_q_heads / desc->num_kv_heads;
  const int P = desc->batch * desc->num_kv_heads;
  if (P > kDecodeMaxPairs) return LSERVE_ERR_UNSUPPORTED;
  const int tile_rows = decode_tile_rows(desc->physical_page);
  grid = decode_grid(current_sm_count());
  {
    // Small calls use fewer CTAs: from the host-side shapes, a pair attends at
    // most max(top_k, sink + local pages) pages, which bounds the tiles of the
    // call; at least kDecodeMinTiles tiles per CTA keeps each pair split over
    // fewer CTAs (fewer partials to merge) while large calls still fill the GPU.
    const long long NP = desc->physical_page;
    const long long stream_pages = (sink_tokens + NP - 1) / NP + (local_tokens + NP - 1) / NP + 1;
    const long long sel_pages = top_k < desc->max_pages_per_seq ? top_k : desc->max_pages_per_seq;
    long long per_pair = sel_pages > stream_pages ? sel_pages : stream_pages;
    if (per_pair > desc->max_pages_per_seq) per_pair = desc->max_pages_per_seq;
    const long long tiles_ub = (long long)P * per_pair * (desc->physical_page / tile_rows);
    const long long want = (tiles_ub + kDecodeMinTiles - 1) / kDecodeMinTiles;
    if (want < grid) grid = want < 1 ? 1 : (int)want;
  }
  p = DecodeParams{};
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.block_table = block_table;
  p.ctx_lens = ctx_lens;
  p.head_kind = head_kind;
  p.sel = sel;
  p.sel_count = sel_count;
  if (flags & LSERVE_DECODE_OUT_F32) p.out_f32 = static_cast<float*>(out);
  else p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  // workspace: the pairs' merge epochs, then one tagged partial slot per CTA
  // (decode_workspace_bytes sizes it for the device's largest grid)
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  p.epochs = reinterpret_cast<uint32_t*>(ws);
  p.parts = reinterpret_cast<unsigned long long*>(ws + ((size_t)P * 4 + 255) / 256 * 256);
  p.batch = desc->batch;
  p.num_q_heads = desc->num_q_heads;
  p.num_kv_heads = desc->num_kv_heads;
  p.physical_page = desc->physical_page;
  p.max_pages = desc->max_pages_per_seq;
  p.num_pool_pages = desc->num_pool_pages;
  p.top_k = top_k;
  p.sink = sink_tokens;
  p.local = local_tokens;
  p.tile_rows = tile_rows;
  p.tiles_per_page = desc->physical_page / tile_rows;
  p.consumer_warps = decode_consumer_warps();
  p.scale_log2 = softmax_scale * 1.4426950408889634f;
  p.wait_limit = wait_limit();
  p.overlap_prologue = (flags & LSERVE_DECODE_OVERLAP_PROLOGUE) ? 1 : 0;
  p.prefetch_kv = (p.overlap_prologue && (flags & LSERVE_DECODE_PREFETCH_KV)) ? 1 : 0;
  p.status = device_status_word();
  if (!p.status) return LSERVE_ERR_CUDA;
  return LSERVE_OK;
}

}  // namespace

extern "C" {

int lserve_sparse_decode_attn_ex(const lserve_paged_desc* desc, const void* q, const void* k_pool,
                                 const void* v_pool, const int32_t* block_table,
                                 const int32_t* ctx_lens, const uint8_t* head_kind,
                                 const int32_t* sel, const int32_t* sel_count, int32_t top_k,
                                 int32_t sink_tokens, int32_t local_tokens, float softmax_scale,
                                 void* out, float* lse, uint32_t flags, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  if (!k_pool || !v_pool || !aligned(k_pool, 16) || !aligned(v_pool, 16)) return LSERVE_ERR_INVALID_ARG;
  DecodeParams p;
  int grid = 0;
  const int st = decode_params(desc, q, block_table, ctx_lens, head_kind, sel, sel_count, top_k,
                               sink_tokens, local_tokens, softmax_scale, out, lse, flags, workspace,
                               workspace_bytes, p, grid);
  if (st != LSERVE_OK) return st;
  const int D = desc->head_dim, G = desc->num_q_heads / desc->num_kv_heads;
  const uint64_t rows = (uint64_t)desc->num_pool_pages * desc->num_kv_heads * desc->physical_page;
  // [rows][D/64][64] view: a tile of tile_rows x D is one contiguous TMA copy
  CUtensorMap kmap, vmap;
  if (!make_map_tiled(&kmap, k_pool, 3, 64, D / 64, rows, 64, D / 64, p.tile_rows) ||
      !make_map_tiled(&vmap, v_pool, 3, 64, D / 64, rows, 64, D / 64, p.tile_rows))
    return LSERVE_ERR_CUDA;
  return cuda_status(launch_decode(p, kmap, vmap, D, G, grid, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

namespace {
// decode over a quantized cache (bits = 8 or 4)
int decode_quant_entry(const lserve_paged_desc* desc, const void* q, const void* k_pool8,
                       const void* v_pool8, const float* k_scale, const float* v_scale,
                       const int32_t* block_table, const int32_t* ctx_lens,
                       const uint8_t* head_kind, const int32_t* sel, const int32_t* sel_count,
                       int32_t top_k, int32_t sink_tokens, int32_t local_tokens,
                       float softmax_scale, void* out, float* lse, uint32_t flags, void* workspace,
                       size_t workspace_bytes, void* stream, int bits) {
  if (!k_pool8 || !v_pool8 || !k_scale || !v_scale) return LSERVE_ERR_INVALID_ARG;
  if (!aligned(k_pool8, 16) || !aligned(v_pool8, 16) || !aligned(k_scale, 16) || !aligned(v_scale, 16))
    return LSERVE_ERR_INVALID_ARG;
  DecodeParams p;
  int grid = 0;
  const int st = decode_params(desc, q, block_table, ctx_lens, head_kind, sel, sel_count, top_k,
                               sink_tokens, local_tokens, softmax_scale, out, lse, flags, workspace,
                               workspace_bytes, p, grid);
  if (st != LSERVE_OK) return st;
  p.k8 = static_cast<const int8_t*>(k_pool8);
  p.v8 = static_cast<const int8_t*>(v_pool8);
  p.k_scale = k_scale;
  p.v_scale = v_scale;
  const int D = desc->head_dim, G = desc->num_q_heads / desc->num_kv_heads;
  const uint64_t rows = (uint64_t)desc->num_pool_pages * desc->num_kv_heads * desc->physical_page;
  CUtensorMap kmap, vmap;
  if (!make_map_codes(&kmap, k_pool8, rows, (uint32_t)(D * bits / 8), p.tile_rows) ||
      !make_map_codes(&vmap, v_pool8, rows, (uint32_t)(D * bits / 8), p.tile_rows))
    return LSERVE_ERR_CUDA;
  return cuda_status(launch_decode_quant(p, kmap, vmap, D, G, bits, grid,
                                         static_cast<cudaStream_t>(stream)));
}
}  // namespace

extern "C" {

int lserve_decode_step(const lserve_paged_desc* desc, const void* q, const void* k_new,
                       const void* v_new, void* k_pool, void* v_pool, void* stats_pool,
                       const int32_t* block_table, const int32_t* ctx_lens,
                       const uint8_t* head_kind, const int32_t* sel, const int32_t* sel_count,
                       int32_t top_k, int32_t sink_tokens, int32_t local_tokens,
                       const int32_t* recent_from, float softmax_scale, void* out, float* lse,
                       uint32_t flags, void* workspace, size_t workspace_bytes, void* stream) {
  if (!k_pool || !v_pool || !aligned(k_pool, 16) || !aligned(v_pool, 16)) return LSERVE_ERR_INVALID_ARG;
  if ((k_new == nullptr) != (v_new == nullptr)) return LSERVE_ERR_INVALID_ARG;
  if (k_new && (!stats_pool || !aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(stats_pool, 16)))
    return LSERVE_ERR_INVALID_ARG;
  if (recent_from && !aligned(recent_from, 4)) return LSERVE_ERR_INVALID_ARG;
  DecodeParams p;
  int grid = 0;
  const int st = decode_params(desc, q, block_table, ctx_lens, head_kind, sel, sel_count, top_k,
                               sink_tokens, local_tokens, softmax_scale, out, lse, flags, workspace,
                               workspace_bytes, p, grid);
  if (st != LSERVE_OK) return st;
  p.k_new = static_cast<const __nv_bfloat16*>(k_new);
  p.v_new = static_cast<const __nv_bfloat16*>(v_new);
  p.k_pool_w = static_cast<__nv_bfloat16*>(k_pool);
  p.v_pool_w = static_cast<__nv_bfloat16*>(v_pool);
  p.stats_w = static_cast<__nv_bfloat16*>(stats_pool);
  p.logical_page = desc->logical_page;
  p.recent_from = recent_from;
  const int D = desc->head_dim, G = desc->num_q_heads / desc->num_kv_heads;
  const uint64_t rows = (uint64_t)desc->num_pool_pages * desc->num_kv_heads * desc->physical_page;
  CUtensorMap kmap, vmap;
  if (!make_map_tiled(&kmap, k_pool, 3, 64, D / 64, rows, 64, D / 64, p.tile_rows) ||
      !make_map_tiled(&vmap, v_pool, 3, 64, D / 64, rows, 64, D / 64, p.tile_rows))
    return LSERVE_ERR_CUDA;
  return cuda_status(launch_decode(p, kmap, vmap, D, G, grid, static_cast<cudaStream_t>(stream)));
}

int lserve_sparse_decode_attn_kv8(const lserve_paged_desc* desc, const void* q, const void* k_pool8,
                                  const void* v_pool8, const float* k_scale, const float* v_scale,
                                  const int32_t* block_table, const int32_t* ctx_lens,
                                  const uint8_t* head_kind, const int32_t* sel,
                                  const int32_t* sel_count, int32_t top_k, int32_t sink_tokens,
                                  int32_t local_tokens, float softmax_scale, void* out, float* lse,
                                  uint32_t flags, void* workspace, size_t workspace_bytes,
                                  void* stream) {
  return decode_quant_entry(desc, q, k_pool8, v_pool8, k_scale, v_scale, block_table, ctx_lens,
                            head_kind, sel, sel_count, top_k, sink_tokens, local_tokens,
                            softmax_scale, out, lse, flags, workspace, workspace_bytes, stream, 8);
}

int lserve_sparse_decode_attn_kv4(const lserve_paged_desc* desc, const void* q, const void* k_pool4,
                                  const void* v_pool4, const float* k_scale, const float* v_scale,
                                  const int32_t* block_table, const int32_t* ctx_lens,
                                  const uint8_t* head_kind, const int32_t* sel,
                                  const int32_t* sel_count, int32_t top_k, int32_t sink_tokens,
                                  int32_t local_tokens, float softmax_scale, void* out, float* lse,
                                  uint32_t flags, void* workspace, size_t workspace_bytes,
                                  void* stream) {
  return decode_quant_entry(desc, q, k_pool4, v_pool4, k_scale, v_scale, block_table, ctx_lens,
                            head_kind, sel, sel_count, top_k, sink_tokens, local_tokens,
                            softmax_scale, out, lse, flags, workspace, workspace_bytes, stream, 4);
}

static int quantize_entry(const lserve_paged_desc* desc, const void* k_pool, const void* v_pool,
                              const int32_t* block_table, const int32_t* ctx_lens, void* k_pool8,
                              void* v_pool8, float* k_scale, float* v_scale, void* stream, int bits) {
  if (!valid_paged(desc)) return LSERVE_ERR_INVALID_ARG;
  if (!k_pool || !v_pool || !block_table || !ctx_lens || !k_pool8 || !v_pool8 || !k_scale || !v_scale)
    return LSERVE_ERR_INVALID_ARG;
  if (!aligned(k_pool, 16) || !aligned(v_pool, 16) || !aligned(k_pool8, 16) || !aligned(v_pool8, 16) ||
      !aligned(k_scale, 16) || !aligned(v_scale, 16) || !aligned(block_table, 4) ||
      !aligned(ctx_lens, 4))
    return LSERVE_ERR_INVALID_ARG;
  const int st = supported_paged(desc);
  if (st != LSERVE_OK) return st;
  if ((long long)desc->batch * desc->max_pages_per_seq > 0x7fffffffll || desc->num_kv_heads > 65535)
    return LSERVE_ERR_UNSUPPORTED;
  QuantParams p;
  p.k_pool = static_cast<const __nv_bfloat16*>(k_pool);
  p.v_pool = static_cast<const __nv_bfloat16*>(v_pool);
  p.block_table = block_table;
  p.ctx_lens = ctx_lens;
  p.k_pool8 = static_cast<int8_t*>(k_pool8);
  p.v_pool8 = static_cast<int8_t*>(v_pool8);
  p.k_scale = k_scale;
  p.v_scale = v_scale;
  p.batch = desc->batch;
  p.num_kv_heads = desc->num_kv_heads;
  p.physical_page = desc->physical_page;
  p.max_pages = desc->max_pages_per_seq;
  p.num_pool_pages = desc->num_pool_pages;
  p.status = device_status_word();
  if (!p.status) return LSERVE_ERR_CUDA;
  return cuda_status(launch_quantize_kv(p, desc->head_dim, bits, static_cast<cudaStream_t>(stream)));
}

int lserve_quantize_pages_kv8(const lserve_paged_desc* desc, const void* k_pool, const void* v_pool,
                              const int32_t* block_table, const int32_t* ctx_lens, void* k_pool8,
                              void* v_pool8, float* k_scale, float* v_scale, void* stream) {
  return quantize_entry(desc, k_pool, v_pool, block_table, ctx_lens, k_pool8, v_pool8, k_scale,
                        v_scale, stream, 8);
}

int lserve_quantize_pages_kv4(const lserve_paged_desc* desc, const void* k_pool, const void* v_pool,
                              const int32_t* block_table, const int32_t* ctx_lens, void* k_pool4,
                              void* v_pool4, float* k_scale, float* v_scale, void* stream) {
  return quantize_entry(desc, k_pool, v_pool, block_table, ctx_lens, k_pool4, v_pool4, k_scale,
                        v_scale, stream, 4);
}

int lserve_seqshard_bounds(int32_t ctx_len, int32_t physical_page, int32_t rank,
                           int32_t num_shards, int32_t* first_page, int32_t* end_page,
                           int32_t* local_len) {
  if (ctx_len < 0 || physical_page < 1 || num_shards < 1 || rank < 0 || rank >= num_shards ||
      !first_page || !end_page || !local_len)
    return LSERVE_ERR_INVALID_ARG;
  const long long M = ((long long)ctx_len + physical_page - 1) / physical_page;
  const long long lo = M * rank / num_shards, hi = M * (rank + 1) / num_shards;
  long long n = (long long)ctx_len - lo * physical_page;
  const long long cap = (hi - lo) * physical_page;
  n = n < 0 ? 0 : (n > cap ? cap : n);
  *first_page = (int32_t)lo;
  *end_page = (int32_t)hi;
  *local_len = (int32_t)n;
  return LSERVE_OK;
}

int32_t lserve_seqshard_sel_stride(const lserve_paged_desc* desc, int32_t top_k, int32_t sink_tokens,
                                   int32_t local_tokens) {
  if (!valid_paged(desc) || top_k < 1 || sink_tokens < 0 || local_tokens < 0) return 0;
  const long long NP = desc->physical_page;
  const long long stream = (sink_tokens + NP - 1) / NP + (local_tokens + NP - 1) / NP + 1;
  const long long s = stream > top_k ? stream : top_k;
  return s > 0x7fffffffll ? 0 : (int32_t)s;
}

int lserve_seqshard_candidates(const lserve_paged_desc* desc, int32_t rank, int32_t num_shards,
                               const int32_t* ctx_lens_global, const uint8_t* head_kind,
                               const int32_t* sel, const int32_t* sel_count, int32_t sel_top_k,
                               const float* phys_scores, int32_t top_k, float* cand_score,
                               int32_t* cand_page, void* stream) {
  if (!valid_paged(desc)) return LSERVE_ERR_INVALID_ARG;
  if (num_shards < 1 || rank < 0 || rank >= num_shards || top_k < 1 || sel_top_k < 1 ||
      sel_top_k > desc->max_pages_per_seq)
    return LSERVE_ERR_INVALID_ARG;
  if (!ctx_lens_global || !head_kind || !sel || !sel_count || !phys_scores || !cand_score || !cand_page)
    return LSERVE_ERR_INVALID_ARG;
  if (!aligned(ctx_lens_global, 4) || !aligned(sel, 4) || !aligned(sel_count, 4) ||
      !aligned(phys_scores, 4) || !aligned(cand_score, 4) || !aligned(cand_page, 4))
    return LSERVE_ERR_INVALID_ARG;
  ShardParams p = {};
  p.ctx_lens = ctx_lens_global;
  p.head_kind = head_kind;
  p.sel = sel;
  p.sel_count = sel_count;
  p.scores = phys_scores;
  p.cand_score = cand_score;
  p.cand_page = cand_page;
  p.batch = desc->batch;
  p.num_kv_heads = desc->num_kv_heads;
  p.physical_page = desc->physical_page;
  p.max_pages = desc->max_pages_per_seq;
  p.top_k = top_k;
  p.sel_stride = sel_top_k;
  p.rank = rank;
  p.num_shards = num_shards;
  p.status = device_status_word();
  if (!p.status) return LSERVE_ERR_CUDA;
  return cuda_status(launch_seqshard_candidates(p, static_cast<cudaStream_t>(stream)));
}

int lserve_seqshard_merge(const lserve_paged_desc* desc, int32_t rank, int32_t num_shards,
                          const int32_t* ctx_lens_global, const uint8_t* head_kind,
                          const float* cand_score_all, const int32_t* cand_page_all, int32_t top_k,
                          int32_t sink_tokens, int32_t local_tokens, int32_t* sel_out,
                          int32_t* sel_count_out, int32_t sel_stride, void* stream) {
  if (!valid_paged(desc)) return LSERVE_ERR_INVALID_ARG;
  if (num_shards < 1 || rank < 0 || rank >= num_shards || top_k < 1) return LSERVE_ERR_INVALID_ARG;
  if (!ctx_lens_global || !head_kind || !cand_score_all || !cand_page_all || !sel_out || !sel_count_out)
    return LSERVE_ERR_INVALID_ARG;
  if (!aligned(ctx_lens_global, 4) || !aligned(cand_score_all, 4) || !aligned(cand_page_all, 4) ||
      !aligned(sel_out, 4) || !aligned(sel_count_out, 4))
    return LSERVE_ERR_INVALID_ARG;
  const int32_t need = lserve_seqshard_sel_stride(desc, top_k, sink_tokens, local_tokens);
  if (need == 0 || sel_stride < need) return LSERVE_ERR_INVALID_ARG;
  if ((long long)num_shards * top_k * 9 > 200 * 1024) return LSERVE_ERR_UNSUPPORTED;
  ShardParams p = {};
  p.ctx_lens = ctx_lens_global;
  p.head_kind = head_kind;
  p.all_score = cand_score_all;
  p.all_page = cand_page_all;
  p.out_sel = sel_out;
  p.out_count = sel_count_out;
  p.batch = desc->batch;
  p.num_kv_heads = desc->num_kv_heads;
  p.physical_page = desc->physical_page;
  p.max_pages = desc->max_pages_per_seq;
  p.top_k = top_k;
  p.out_stride = sel_stride;
  p.rank = rank;
  p.num_shards = num_shards;
  p.sink = sink_tokens;
  p.local = local_tokens;
  p.status = device_status_word();
  if (!p.status) return LSERVE_ERR_CUDA;
  return cuda_status(launch_seqshard_merge(p, static_cast<cudaStream_t>(stream)));
}

int lserve_seqshard_combine(int32_t num_shards, int32_t rows, int32_t head_dim, const float* o_parts,
                            const float* lse_parts, void* out, float* lse, void* stream) {
  if (num_shards < 1 || rows < 1 || (head_dim != 64 && head_dim != 128)) return LSERVE_ERR_INVALID_ARG;
  if (!o_parts || !lse_parts || !out) return LSERVE_ERR_INVALID_ARG;
  if (!aligned(o_parts, 4) || !aligned(lse_parts, 4) || !aligned(out, 2) || (lse && !aligned(lse, 4)))
    return LSERVE_ERR_INVALID_ARG;
  CombineParams p;
  p.o_parts = o_parts;
  p.lse_parts = lse_parts;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.num_shards = num_shards;
  p.rows = rows;
  p.head_dim = head_dim;
  return cuda_status(launch_seqshard_combine(p, static_cast<cudaStream_t>(stream)));
}

int lserve_blocksparse_prefill(const lserve_prefill_desc* desc, const void* q, const void* k,
                               const void* v, const uint8_t* head_kind_host, float softmax_scale,
                               void* out, float* lse, void* workspace, size_t workspace_bytes,
                               void* stream) {
  return prefill_entry(desc, q, k, v, head_kind_host, softmax_scale, out, lse, workspace,
                       workspace_bytes, static_cast<cudaStream_t>(stream));
}

int lserve_blocksparse_prefill_paged(const lserve_prefill_desc* desc, const lserve_paged_desc* paged,
                                     const void* q, const void* k, const void* v,
                                     const uint8_t* head_kind_host, float softmax_scale, void* out,
                                     float* lse, const int32_t* block_table, void* k_pool,
                                     void* v_pool, void* stats_pool, void* workspace,
                                     size_t workspace_bytes, void* stream) {
  if (!desc || !valid_paged(paged)) return LSERVE_ERR_INVALID_ARG;
  if (!block_table || !k_pool || !v_pool || !stats_pool) return LSERVE_ERR_INVALID_ARG;
  if (!aligned(k_pool, 16) || !aligned(v_pool, 16) || !aligned(stats_pool, 16) ||
      !aligned(block_table, 4))
    return LSERVE_ERR_INVALID_ARG;
  if (paged->head_dim != desc->head_dim || paged->num_kv_heads != desc->num_kv_heads)
    return LSERVE_ERR_INVALID_ARG;
  const int st = supported_paged(paged);
  if (st != LSERVE_OK) return st;
  if ((long long)desc->seq_len > (long long)paged->max_pages_per_seq * paged->physical_page)
    return LSERVE_ERR_INVALID_ARG;
  return prefill_paged_entry(desc, paged, q, k, v, head_kind_host, softmax_scale, out, lse,
                             block_table, k_pool, v_pool, stats_pool, workspace, workspace_bytes,
                             static_cast<cudaStream_t>(stream));
}

}  // extern "C"
