// lserve_decode_append kernel: the cache maintenance of one decode step.
//
// The new token of every sequence b (position ctx_lens[b], before the caller
// advances the length) is written into the paged K / V pools at page
// block_table[b][pos / N_P], row pos % N_P, for every KV head.  For the
// retrieval heads the channel-wise k_min / k_max of the logical page that
// holds it (LServe explainer, 技術的詳細 › 動的スパーシティ: the statistics the
// query-centric score S^j reads; 階層的ページング: logical pages of N_L tokens
// inside the physical page) are updated in place: a logical page's first
// token sets both to its key, later tokens take the elementwise min / max.
// Min and max of bf16 values are exact, so the result equals a full rebuild
// of the page's statistics.
//
// One warp per (sequence, KV head): D/8 lanes move the K row and D/8 the V
// row with 16-byte accesses; the K lanes also read-modify-write the two
// statistics rows.  Pairs are independent, so nothing races.
#include "common.cuh"
#include "kernels.h"

namespace lserve {

template <int D>
__global__ void __launch_bounds__(kAppendWarps * 32) decode_append_kernel(AppendParams p) {
  constexpr int LPR = D / 8;  // lanes per row, 8 channels each
  const int lane = threadIdx.x & 31;
  const int pair = blockIdx.x * kAppendWarps + (threadIdx.x >> 5);
  if (pair >= p.batch * p.num_kv_heads) return;
  const int b = pair / p.num_kv_heads, h = pair - b * p.num_kv_heads;
  const int pos = p.ctx_lens[b];
  const int NP = p.physical_page, NL = p.logical_page;
  const int m = pos / NP;
  if (pos < 0 || m >= p.max_pages) {
    if (lane == 0) raise_status(p.status, LSERVE_ERR_BOUNDS);
    return;
  }
  const int pid = p.block_table[(size_t)b * p.max_pages + m];
  if (pid < 0 || pid >= p.num_pool_pages) {
    if (lane == 0) raise_status(p.status, LSERVE_ERR_BOUNDS);
    return;
  }
  const int row = pos - m * NP;
  const size_t dst = ((((size_t)pid * p.num_kv_heads + h) * NP) + row) * D;
  const size_t src = (size_t)pair * D;
  if (lane >= 2 * LPR) return;
  const bool is_k = lane < LPR;
  const int c = (is_k ? lane : lane - LPR) * 8;
  const uint4 x = *reinterpret_cast<const uint4*>((is_k ? p.k_new : p.v_new) + src + c);
  *reinterpret_cast<uint4*>((is_k ? p.k_pool : p.v_pool) + dst + c) = x;
  if (!is_k || p.head_kind[h] != 0) return;
  // k_min / k_max of the logical page holding the token
  const int g = NP / NL;
  const int sub = row / NL;
  __nv_bfloat16* st = p.stats_pool + ((((size_t)pid * p.num_kv_heads + h) * g) + sub) * 2 * D + c;
  uint4 mn = x, mx = x;
  if (row % NL != 0) {  // not the page's first token: fold into the stored statistics
    const uint4 omn = *reinterpret_cast<const uint4*>(st);
    const uint4 omx = *reinterpret_cast<const uint4*>(st + D);
    const __nv_bfloat162* a = reinterpret_cast<const __nv_bfloat162*>(&omn);
    const __nv_bfloat162* z = reinterpret_cast<const __nv_bfloat162*>(&omx);
    const __nv_bfloat162* v = reinterpret_cast<const __nv_bfloat162*>(&x);
    __nv_bfloat162* rn = reinterpret_cast<__nv_bfloat162*>(&mn);
    __nv_bfloat162* rx = reinterpret_cast<__nv_bfloat162*>(&mx);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      rn[k] = __hmin2(a[k], v[k]);
      rx[k] = __hmax2(z[k], v[k]);
    }
  }
  *reinterpret_cast<uint4*>(st) = mn;
  *reinterpret_cast<uint4*>(st + D) = mx;
}

cudaError_t launch_decode_append(const AppendParams& p, int D, cudaStream_t stream) {
  const int pairs = p.batch * p.num_kv_heads;
  const int grid = (pairs + kAppendWarps - 1) / kAppendWarps;
  if (D == 128)
    decode_append_kernel<128><<<grid, kAppendWarps * 32, 0, stream>>>(p);
  else if (D == 64)
    decode_append_kernel<64><<<grid, kAppendWarps * 32, 0, stream>>>(p);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace lserve
