// lserve_page_select kernels (LServe explainer, 技術的詳細 › 動的スパーシティ, the
// equation for S^j; 階層的ページング, physical score = max of logical scores; the
// "Top-K物理ページ" node of the 統一ブロックスパースアテンション figure).
//
// 1. page_score_kernel: a stream over the statistics pool.  One warp scores
//    physical pages; D/8 lanes share a logical page, each holding 8 channels
//    of the G query heads (fp32) in registers.  Per channel the sign of q
//    picks k_max or k_min (q*max(.)/q*min(.) without a second product: the
//    larger of q*k_max and q*k_min is q times k_max when q >= 0, else times
//    k_min; bf16 x bf16 products are exact in fp32).  Lanes reduce with
//    shuffles, the max over the g logical pages gives the physical score.
// 2. page_topk_kernel: one CTA per (sequence, retrieval head) finds the K-th
//    largest score by an 8-bit radix select over order-preserving integer
//    keys, then compacts the winners in ascending page order with one block
//    scan; ties at the threshold go to the lowest page indices.
#include "common.cuh"
#include "kernels.h"

namespace lserve {

template <int D, int G>
__global__ void __launch_bounds__(kScoreWarps * 32)
page_score_kernel(SelectParams p) {
  constexpr int LPR = D / 8;      // lanes per logical page
  constexpr int LPI = 32 / LPR;   // logical pages per warp step
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.z, h = blockIdx.y;
  if (p.head_kind[h] != 0) return;
  const int n = p.ctx_lens[b];
  const int NP = p.physical_page, NL = p.logical_page, g = NP / NL;
  const int npages = min((n + NP - 1) / NP, p.max_pages);
  const int nlog = (n + NL - 1) / NL;
  const int m0 = (blockIdx.x * kScoreWarps + warp) * kScorePagesPerWarp;
  if (m0 >= npages) return;
  const int c = (lane % LPR) * 8;
  const int slot = lane / LPR;

  float qf[G][8];
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
    const uint4 w = *reinterpret_cast<const uint4*>(
        p.q + ((size_t)b * p.num_q_heads + (size_t)h * G + hh) * D + c);
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      qf[hh][2 * k] = bf16_lo(ww[k]);
      qf[hh][2 * k + 1] = bf16_hi(ww[k]);
    }
  }

  for (int mi = 0; mi < kScorePagesPerWarp; ++mi) {
    const int m = m0 + mi;
    if (m >= npages) break;
    const int pid = p.block_table[(size_t)b * p.max_pages + m];
    if (kCheckBounds && (pid < 0 || pid >= p.num_pool_pages)) {
      raise_status(p.status, LSERVE_ERR_BOUNDS);
      continue;
    }
    const __nv_bfloat16* st = p.stats_pool + (((size_t)pid * p.num_kv_heads + h) * g) * 2 * D + c;
    float best = -INFINITY;
    for (int s0 = 0; s0 < g; s0 += LPI) {
      const int sub = s0 + slot;
      const bool valid = sub < g && m * g + sub < nlog;
      float part = 0.f;
      if (valid) {
        const uint4 mn = ldg_nc_v4(st + (size_t)sub * 2 * D);
        const uint4 mx = ldg_nc_v4(st + (size_t)sub * 2 * D + D);
        const uint32_t wn[4] = {mn.x, mn.y, mn.z, mn.w};
        const uint32_t wx[4] = {mx.x, mx.y, mx.z, mx.w};
        float kn[8], kx[8];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          kn[2 * k] = bf16_lo(wn[k]);
          kn[2 * k + 1] = bf16_hi(wn[k]);
          kx[2 * k] = bf16_lo(wx[k]);
          kx[2 * k + 1] = bf16_hi(wx[k]);
        }
#pragma unroll
        for (int hh = 0; hh < G; ++hh) {
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const float qq = qf[hh][k];
            part = fmaf(qq, qq >= 0.f ? kx[k] : kn[k], part);
          }
        }
      }
#pragma unroll
      for (int o = 1; o < LPR; o <<= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
      if (valid) best = fmaxf(best, part);
    }
    best = warp_max(best);
    if (lane == 0) p.scores[((size_t)b * p.num_kv_heads + h) * p.max_pages + m] = best;
  }
}

// order-preserving map float -> uint32 (-0 and +0 map to the same key)
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f == 0.f ? 0.f : f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__global__ void __launch_bounds__(kTopkThreads) page_topk_kernel(SelectParams p) {
  extern __shared__ uint32_t keys[];  // [npages]
  __shared__ int hist[256];
  __shared__ int sh_digit, sh_above;
  __shared__ uint32_t warp_tot[kTopkThreads / 32];
  const int b = blockIdx.y, h = blockIdx.x, tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const size_t pair = (size_t)b * p.num_kv_heads + h;
  int32_t* sel = p.sel + pair * p.top_k;
  const int K = p.top_k;
  if (p.head_kind[h] != 0) {
    for (int i = tid; i < K; i += blockDim.x) sel[i] = -1;
    if (tid == 0) p.sel_count[pair] = 0;
    return;
  }
  const int n = p.ctx_lens[b];
  int M = (n + p.physical_page - 1) / p.physical_page;
  if (M > p.max_pages) {  // the block table cannot hold this many pages
    if (tid == 0) raise_status(p.status, LSERVE_ERR_BOUNDS);
    M = p.max_pages;
  }
  if (M <= K) {  // every page is kept
    for (int i = tid; i < K; i += blockDim.x) sel[i] = i < M ? i : -1;
    if (tid == 0) p.sel_count[pair] = M;
    return;
  }
  const float* sc = p.scores + pair * p.max_pages;
  for (int m = tid; m < M; m += blockDim.x) keys[m] = order_key(sc[m]);
  __syncthreads();

  // radix select of the K-th largest key, 8 bits at a time from the top
  uint32_t prefix = 0, mask = 0;
  int need = K;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for (int m = tid; m < M; m += blockDim.x) {
      const uint32_t k = keys[m];
      if ((k & mask) == prefix) atomicAdd(&hist[(k >> shift) & 255u], 1);
    }
    __syncthreads();
    if (warp == 0) {
      // lane L owns digits 255-8L .. 248-8L (descending)
      int cnt[8], tot = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        cnt[i] = hist[255 - 8 * lane - i];
        tot += cnt[i];
      }
      int incl = tot;  // inclusive scan over lanes (higher digits first)
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      int above = incl - tot;
      if (above < need && need <= incl) {  // exactly one lane
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (above < need && need <= above + cnt[i]) {
            sh_digit = 255 - 8 * lane - i;
            sh_above = above;
          }
          above += cnt[i];
        }
      }
    }
    __syncthreads();
    need -= sh_above;
    prefix |= (uint32_t)sh_digit << shift;
    mask |= 255u << shift;
    __syncthreads();
  }
  const uint32_t T = prefix;  // the K-th largest key; `need` keys equal to it are kept

  // block scan of (greater, equal) counts over contiguous per-thread chunks
  const int per = (M + blockDim.x - 1) / blockDim.x;
  const int lo = min(M, tid * per), hi = min(M, lo + per);
  uint32_t gt = 0, eq = 0;
  for (int m = lo; m < hi; ++m) {
    gt += keys[m] > T;
    eq += keys[m] == T;
  }
  uint32_t v = (gt << 16) | eq, incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x / 32;
    uint32_t x = lane < nw ? warp_tot[lane] : 0, xi = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, xi, o);
      if (lane >= o) xi += t;
    }
    if (lane < nw) warp_tot[lane] = xi - x;  // exclusive
  }
  __syncthreads();
  const uint32_t before = warp_tot[warp] + incl - v;
  uint32_t gt_before = before >> 16, eq_before = before & 0xFFFFu;
  for (int m = lo; m < hi; ++m) {
    const uint32_t k = keys[m];
    if (k > T) {
      sel[gt_before + min(eq_before, (uint32_t)need)] = m;
      ++gt_before;
    } else if (k == T) {
      if (eq_before < (uint32_t)need) sel[gt_before + eq_before] = m;
      ++eq_before;
    }
  }
  if (tid == 0) p.sel_count[pair] = K;
}

cudaError_t launch_page_select(const SelectParams& p, int D, cudaStream_t stream) {
  const int per_cta = kScoreWarps * kScorePagesPerWarp;
  dim3 grid((p.max_pages + per_cta - 1) / per_cta, p.num_kv_heads, p.batch);
  const int G = p.num_q_heads / p.num_kv_heads;
#define LSERVE_SCORE_CASE(DD, GG)                                          \
  if (D == DD && G == GG) {                                                \
    page_score_kernel<DD, GG><<<grid, kScoreWarps * 32, 0, stream>>>(p);   \
  } else
  LSERVE_SCORE_CASE(64, 1)
  LSERVE_SCORE_CASE(64, 2)
  LSERVE_SCORE_CASE(64, 4)
  LSERVE_SCORE_CASE(64, 8)
  LSERVE_SCORE_CASE(128, 1)
  LSERVE_SCORE_CASE(128, 2)
  LSERVE_SCORE_CASE(128, 4)
  LSERVE_SCORE_CASE(128, 8)
  return cudaErrorInvalidValue;
#undef LSERVE_SCORE_CASE
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t smem = (size_t)p.max_pages * sizeof(uint32_t);
  if (smem > 48 * 1024) {
    e = set_smem_once((const void*)page_topk_kernel, (int)smem);
    if (e != cudaSuccess) return e;
  }
  page_topk_kernel<<<dim3(p.num_kv_heads, p.batch), kTopkThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace lserve
