// lserve_page_stats kernel: channel-wise k_min / k_max of every logical page
// of the retrieval heads (LServe explainer, 技術的詳細 › 動的スパーシティ; the logical
// / physical split of 階層的ページング).
//
// One warp per logical page.  A logical page of one head is N_L * D bf16 =
// N_L * D * 2 contiguous bytes inside its physical page; lanes read it with
// 16-byte non-allocating loads (8 channels per lane, D/8 lanes per row), all
// rows of the page in flight at once, reduce min/max in bf16 registers (exact)
// and then across the row groups with shuffles.  HBM-bound: reads the keys
// once and writes 2*D*2 bytes per logical page.
#include "common.cuh"
#include "kernels.h"

namespace lserve {

template <int D, int NL>
__global__ void __launch_bounds__(kStatsWarps * 32)
page_stats_kernel(StatsParams p) {
  constexpr int LPR = D / 8;        // lanes per key row
  constexpr int RPI = 32 / LPR;     // rows one warp-wide load covers
  constexpr int ITERS = (NL + RPI - 1) / RPI;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.z, h = blockIdx.y;
  if (p.head_kind[h] != 0) return;  // streaming heads need no statistics
  const int n = p.ctx_lens[b];
  const int lp = p.first_logical_page + blockIdx.x * kStatsWarps + warp;
  if (lp * NL >= n) return;
  const int g = p.physical_page / NL;
  const int m = lp / g, sub = lp - m * g;
  const int pid = p.block_table[(size_t)b * p.max_pages + m];
  if (kCheckBounds && (m >= p.max_pages || pid < 0 || pid >= p.num_pool_pages)) {
    raise_status(p.status, LSERVE_ERR_BOUNDS);
    return;
  }
  const int valid = min(NL, n - lp * NL);
  const int r0 = lane / LPR, c = (lane % LPR) * 8;
  const __nv_bfloat16* base = p.k_pool + (((size_t)pid * p.num_kv_heads + h) * p.physical_page +
                                          (size_t)sub * NL) * D + c;
  uint4 rows[ITERS];
#pragma unroll
  for (int i = 0; i < ITERS; ++i) {
    const int r = r0 + i * RPI;
    if (r < valid) rows[i] = ldg_nc_v4(base + (size_t)r * D);
  }
  const uint32_t kPosInf2 = 0x7F807F80u, kNegInf2 = 0xFF80FF80u;
  __nv_bfloat162 mn[4], mx[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    mn[k] = *reinterpret_cast<const __nv_bfloat162*>(&kPosInf2);
    mx[k] = *reinterpret_cast<const __nv_bfloat162*>(&kNegInf2);
  }
#pragma unroll
  for (int i = 0; i < ITERS; ++i) {
    if (r0 + i * RPI < valid) {
      const __nv_bfloat162* v = reinterpret_cast<const __nv_bfloat162*>(&rows[i]);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        mn[k] = __hmin2(mn[k], v[k]);
        mx[k] = __hmax2(mx[k], v[k]);
      }
    }
  }
#pragma unroll
  for (int o = LPR; o < 32; o <<= 1) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      uint32_t a = *reinterpret_cast<uint32_t*>(&mn[k]);
      uint32_t bb = *reinterpret_cast<uint32_t*>(&mx[k]);
      a = __shfl_xor_sync(0xffffffffu, a, o);
      bb = __shfl_xor_sync(0xffffffffu, bb, o);
      mn[k] = __hmin2(mn[k], *reinterpret_cast<__nv_bfloat162*>(&a));
      mx[k] = __hmax2(mx[k], *reinterpret_cast<__nv_bfloat162*>(&bb));
    }
  }
  if (lane < LPR) {
    __nv_bfloat16* out = p.stats_pool +
                         ((((size_t)pid * p.num_kv_heads + h) * g + sub) * 2) * D + c;
    *reinterpret_cast<uint4*>(out) = *reinterpret_cast<uint4*>(mn);
    *reinterpret_cast<uint4*>(out + D) = *reinterpret_cast<uint4*>(mx);
  }
}

cudaError_t launch_page_stats(const StatsParams& p, int D, int max_logical_pages,
                              cudaStream_t stream) {
  const int todo = max_logical_pages - p.first_logical_page;
  if (todo <= 0) return cudaSuccess;
  dim3 grid((todo + kStatsWarps - 1) / kStatsWarps, p.num_kv_heads, p.batch);
  dim3 block(kStatsWarps * 32);
#define LSERVE_STATS_CASE(DD, NN)                                  \
  if (D == DD && p.logical_page == NN) {                           \
    page_stats_kernel<DD, NN><<<grid, block, 0, stream>>>(p);      \
    return cudaGetLastError();                                     \
  }
  LSERVE_STATS_CASE(64, 8)
  LSERVE_STATS_CASE(64, 16)
  LSERVE_STATS_CASE(64, 32)
  LSERVE_STATS_CASE(64, 64)
  LSERVE_STATS_CASE(128, 8)
  LSERVE_STATS_CASE(128, 16)
  LSERVE_STATS_CASE(128, 32)
  LSERVE_STATS_CASE(128, 64)
#undef LSERVE_STATS_CASE
  return cudaErrorInvalidValue;
}

}  // namespace lserve
