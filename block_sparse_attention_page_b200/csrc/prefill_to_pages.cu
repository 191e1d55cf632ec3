// lserve_prefill_to_pages kernel: after the prefill of one sequence, move its
// K / V ([T][H_kv][D], the prefill's layout) into the paged pools through the
// block table and build the page statistics in the same pass over K
// (LServe explainer, 技術的詳細 › 動的スパーシティ: the k_min / k_max the page
// scores read; 階層的ページング: logical pages of N_L tokens inside physical pages
// of N_P tokens).
//
// One warp per (logical page, KV head): each row of the page is read once
// (16-byte loads, D/8 lanes per row, up to 8 rows per lane in flight), stored
// to its pool row for K and V, and -- for retrieval heads -- folded into the
// exact bf16 min / max of its channels, which are reduced across the row
// groups with shuffles and written to the statistics pool.  HBM-bound: K and V
// are read once and written once, the statistics add 2*D*2 bytes per logical
// page.
#include "common.cuh"
#include "kernels.h"

namespace lserve {

template <int D, int NL>
__global__ void __launch_bounds__(kToPagesWarps * 32) prefill_to_pages_kernel(ToPagesParams p) {
  constexpr int LPR = D / 8;     // lanes per row
  constexpr int RPI = 32 / LPR;  // rows one warp-wide access covers
  constexpr int ITERS = (NL + RPI - 1) / RPI;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y;
  const int lp = blockIdx.x * kToPagesWarps + warp;  // logical page of the sequence
  const int T = p.seq_len;
  if (lp * NL >= T) return;
  const int NP = p.physical_page, g = NP / NL;
  const int m = lp / g, sub = lp - m * g;
  const int pid = m < p.max_pages ? p.block_table[m] : -1;
  if (pid < 0 || pid >= p.num_pool_pages) {
    if (lane == 0) raise_status(p.status, LSERVE_ERR_BOUNDS);
    return;
  }
  const int valid = min(NL, T - lp * NL);
  const int r0 = lane / LPR, c = (lane % LPR) * 8;
  const size_t src_stride = (size_t)p.num_kv_heads * D;  // between tokens of [T][H_kv][D]
  const size_t src0 = ((size_t)lp * NL) * src_stride + (size_t)h * D + c;
  const size_t dst0 = ((((size_t)pid * p.num_kv_heads + h) * NP) + (size_t)sub * NL) * D + c;
  const bool stats = p.head_kind[h] == 0;  // streaming heads need no statistics
  const uint32_t kPosInf2 = 0x7F807F80u, kNegInf2 = 0xFF80FF80u;
  __nv_bfloat162 mn[4], mx[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    mn[k] = *reinterpret_cast<const __nv_bfloat162*>(&kPosInf2);
    mx[k] = *reinterpret_cast<const __nv_bfloat162*>(&kNegInf2);
  }
  constexpr int CH = ITERS < 8 ? ITERS : 8;  // rows in flight per lane
#pragma unroll
  for (int i0 = 0; i0 < ITERS; i0 += CH) {
    uint4 kr[CH], vr[CH];
#pragma unroll
    for (int i = 0; i < CH; ++i) {
      const int r = r0 + (i0 + i) * RPI;
      if (r < valid) {
        kr[i] = ldg_nc_v4(p.k + src0 + (size_t)r * src_stride);
        vr[i] = ldg_nc_v4(p.v + src0 + (size_t)r * src_stride);
      }
    }
#pragma unroll
    for (int i = 0; i < CH; ++i) {
      const int r = r0 + (i0 + i) * RPI;
      if (r < valid) {
        *reinterpret_cast<uint4*>(p.k_pool + dst0 + (size_t)r * D) = kr[i];
        *reinterpret_cast<uint4*>(p.v_pool + dst0 + (size_t)r * D) = vr[i];
        const __nv_bfloat162* v = reinterpret_cast<const __nv_bfloat162*>(&kr[i]);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          mn[k] = __hmin2(mn[k], v[k]);
          mx[k] = __hmax2(mx[k], v[k]);
        }
      }
    }
  }
  if (!stats) return;
  // reduce over the row groups of the warp (lanes with the same channels)
#pragma unroll
  for (int o = LPR; o < 32; o <<= 1) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      uint32_t a = *reinterpret_cast<uint32_t*>(&mn[k]);
      uint32_t z = *reinterpret_cast<uint32_t*>(&mx[k]);
      a = __shfl_xor_sync(0xffffffffu, a, o);
      z = __shfl_xor_sync(0xffffffffu, z, o);
      mn[k] = __hmin2(mn[k], *reinterpret_cast<__nv_bfloat162*>(&a));
      mx[k] = __hmax2(mx[k], *reinterpret_cast<__nv_bfloat162*>(&z));
    }
  }
  if (r0 == 0) {
    __nv_bfloat16* st = p.stats_pool + ((((size_t)pid * p.num_kv_heads + h) * g) + sub) * 2 * D + c;
    *reinterpret_cast<uint4*>(st) = *reinterpret_cast<uint4*>(mn);
    *reinterpret_cast<uint4*>(st + D) = *reinterpret_cast<uint4*>(mx);
  }
}

cudaError_t launch_prefill_to_pages(const ToPagesParams& p, int D, cudaStream_t stream) {
  const int nlog = (p.seq_len + p.logical_page - 1) / p.logical_page;
  dim3 grid((nlog + kToPagesWarps - 1) / kToPagesWarps, p.num_kv_heads);
#define LSERVE_TOPAGES_CASE(DD, NN)                                                  \
  if (D == DD && p.logical_page == NN) {                                             \
    prefill_to_pages_kernel<DD, NN><<<grid, kToPagesWarps * 32, 0, stream>>>(p);     \
    return cudaGetLastError();                                                       \
  }
  LSERVE_TOPAGES_CASE(64, 8)
  LSERVE_TOPAGES_CASE(64, 16)
  LSERVE_TOPAGES_CASE(64, 32)
  LSERVE_TOPAGES_CASE(64, 64)
  LSERVE_TOPAGES_CASE(128, 8)
  LSERVE_TOPAGES_CASE(128, 16)
  LSERVE_TOPAGES_CASE(128, 32)
  LSERVE_TOPAGES_CASE(128, 64)
#undef LSERVE_TOPAGES_CASE
  return cudaErrorInvalidValue;
}

}  // namespace lserve
