// lserve_page_select kernels (LServe explainer, 技術的詳細 › 動的スパーシティ, the
// equation for S^j; 階層的ページング, physical score = max of logical scores; the
// "Top-K物理ページ" node of the 統一ブロックスパースアテンション figure).
//
// 1. page_score_kernel: a stream over the statistics pool.  One warp scores
//    kScorePagesPerWarp physical pages, issuing all their stats loads (into
//    shared memory, by cp.async) before it reduces; D/8 lanes share a logical page, each holding 8 channels of
//    the group-folded query Qp = sum_h max(q_h, 0), Qn = sum_h min(q_h, 0)
//    (max(q*k_max, q*k_min) = max(q,0)*k_max + min(q,0)*k_min because
//    k_max >= k_min).  Lanes reduce with shuffles, the max over the g logical
//    pages gives the physical score.
// 2. page_topk_kernel: one CTA per (sequence, retrieval head) finds the K-th
//    largest score by an 8-bit radix select over order-preserving integer
//    keys (from the highest bit on which the keys differ), stopping once the
//    bucket holding it has at most kTopkCand keys,
//    which are ranked exactly by (score, page index); then it compacts the
//    winners in ascending page order with one block scan.  Ties go to the
//    lowest page indices.
#include "common.cuh"
#include "kernels.h"

namespace lserve {

// Scores of kScorePagesPerWarp physical pages per warp.  Every lane first issues
// all its 16-byte stats loads for those pages (up to kScoreSteps warp steps of
// LPI logical pages each, k_min and k_max), then reduces.  The sum over the G
// query heads of the group is folded into q before the stream: since
// k_max >= k_min, max(q*k_max, q*k_min) = max(q,0)*k_max + min(q,0)*k_min, so
//   S^j = sum_i Qp[i] * k_max^j[i] + Qn[i] * k_min^j[i]
// with Qp[i] = sum_h max(q_h[i], 0) and Qn[i] = sum_h min(q_h[i], 0).
// The stats loads go to shared memory by cp.async (16 bytes per lane and
// load, each lane to its own slots), not to registers: with 70 registers
// six 4-warp blocks (32 KB of staging each; shared memory is the limit) run
// per SM with ~192 KB of statistics in flight -- finer blocks than three
// 8-warp ones with the same bytes in flight: 3% faster on the 8B layer and on
// the mixed batch.  Staged in registers (127 of them) the kernel held two
// blocks per SM and reached half the HBM bandwidth.
constexpr int kScoreSmem = kScoreWarps * kScorePagesPerWarp * kScoreSteps * 2 * 32 * 16;

template <int D, int G>
__global__ void __launch_bounds__(kScoreWarps * 32, 7)
page_score_kernel(SelectParams p) {
  constexpr int LPR = D / 8;      // lanes per logical page (16 channels x 8 = 128)
  constexpr int LPI = 32 / LPR;   // logical pages per warp step
  constexpr int PW = kScorePagesPerWarp;
  constexpr int SB = kScoreSteps;  // warp steps per page loaded at once
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.z, h = blockIdx.y;
  // launched as a programmatic dependent: q and the statistics may come from
  // the kernel before, so nothing is read before it has completed
  pdl_launch_dependents();
  pdl_wait_prior_grid();
  if (p.head_kind[h] != 0) return;
  const int n = p.ctx_lens[b];
  const int NP = p.physical_page, NL = p.logical_page, g = NP / NL;
  const int npages = min((n + NP - 1) / NP, p.max_pages);
  const int nlog = (n + NL - 1) / NL;
  const int m0 = (blockIdx.x * kScoreWarps + warp) * PW;
  if (m0 >= npages) return;
  const int c = (lane % LPR) * 8;
  const int slot = lane / LPR;
  const size_t pair = (size_t)b * p.num_kv_heads + h;

  // block-table entries of the warp's pages: lane j holds page m0 + j
  int pid_l = -1;
  if (lane < PW && m0 + lane < npages) pid_l = p.block_table[(size_t)b * p.max_pages + m0 + lane];

  float qp[8], qn[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) qp[k] = qn[k] = 0.f;
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
    const uint4 w = *reinterpret_cast<const uint4*>(
        p.q + ((size_t)b * p.num_q_heads + (size_t)h * G + hh) * D + c);
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float lo = bf16_lo(ww[k]), hi = bf16_hi(ww[k]);
      qp[2 * k] += fmaxf(lo, 0.f);
      qn[2 * k] += fminf(lo, 0.f);
      qp[2 * k + 1] += fmaxf(hi, 0.f);
      qn[2 * k + 1] += fminf(hi, 0.f);
    }
  }

  int pid[PW];
  bool pok[PW];
#pragma unroll
  for (int j = 0; j < PW; ++j) {
    pid[j] = __shfl_sync(0xffffffffu, pid_l, j);
    pok[j] = m0 + j < npages && pid[j] >= 0 && pid[j] < p.num_pool_pages;
    if (kCheckBounds && m0 + j < npages && !pok[j] && lane == 0) raise_status(p.status, LSERVE_ERR_BOUNDS);
  }
  float best[PW];
#pragma unroll
  for (int j = 0; j < PW; ++j) best[j] = -INFINITY;

  const int steps = (g + LPI - 1) / LPI;
  for (int s0 = 0; s0 < steps; s0 += SB) {
    extern __shared__ uint4 sbuf[];  // [warp][PW][SB][k_min, k_max][lane]
    uint4* mine = sbuf + (size_t)warp * PW * SB * 2 * 32;
    bool ok[PW][SB];
#pragma unroll
    for (int j = 0; j < PW; ++j) {
      const __nv_bfloat16* st = p.stats_pool + (((size_t)pid[j] * p.num_kv_heads + h) * g) * 2 * D + c;
#pragma unroll
      for (int t = 0; t < SB; ++t) {
        const int sub = (s0 + t) * LPI + slot;
        ok[j][t] = pok[j] && s0 + t < steps && sub < g && (m0 + j) * g + sub < nlog;
        if (ok[j][t]) {
          cp_async_16(mine + ((j * SB + t) * 2 + 0) * 32 + lane, st + (size_t)sub * 2 * D);
          cp_async_16(mine + ((j * SB + t) * 2 + 1) * 32 + lane, st + (size_t)sub * 2 * D + D);
        }
      }
    }
    cp_async_wait_all();  // this lane's copies have landed (each lane reads only its own slots)
#pragma unroll
    for (int j = 0; j < PW; ++j) {
#pragma unroll
      for (int t = 0; t < SB; ++t) {
        float part = 0.f;
        if (ok[j][t]) {
          const uint4 vn = mine[((j * SB + t) * 2 + 0) * 32 + lane];
          const uint4 vx = mine[((j * SB + t) * 2 + 1) * 32 + lane];
          const uint32_t wn[4] = {vn.x, vn.y, vn.z, vn.w};
          const uint32_t wx[4] = {vx.x, vx.y, vx.z, vx.w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            part = fmaf(qp[2 * k], bf16_lo(wx[k]), part);
            part = fmaf(qp[2 * k + 1], bf16_hi(wx[k]), part);
            part = fmaf(qn[2 * k], bf16_lo(wn[k]), part);
            part = fmaf(qn[2 * k + 1], bf16_hi(wn[k]), part);
          }
        }
#pragma unroll
        for (int o = 1; o < LPR; o <<= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
        if (ok[j][t]) best[j] = fmaxf(best[j], part);
      }
    }
  }
#pragma unroll
  for (int j = 0; j < PW; ++j) {
    float v = best[j];
#pragma unroll
    for (int o = LPR; o < 32; o <<= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    // a page whose block-table entry is bad scores -inf (never chosen ahead of a valid one)
    if (lane == 0 && m0 + j < npages) p.scores[pair * p.max_pages + m0 + j] = v;
  }
}

__global__ void __launch_bounds__(kTopkThreads) page_topk_kernel(SelectParams p) {
  extern __shared__ uint32_t keys[];  // [npages]
  __shared__ int hist[256];
  __shared__ int sh_digit, sh_above, sh_bucket, sh_ncand;
  __shared__ int cand[kTopkCand];
  __shared__ uint32_t warp_tot[kTopkThreads / 32];
  __shared__ uint32_t warp_max[kTopkThreads / 32], warp_min[kTopkThreads / 32];
  const int b = blockIdx.y, h = blockIdx.x, tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const size_t pair = (size_t)b * p.num_kv_heads + h;
  int32_t* sel = p.sel + pair * p.top_k;
  pdl_launch_dependents();
  pdl_wait_prior_grid();  // the scores come from the kernel before
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
  uint32_t kmx = 0u, kmn = 0xFFFFFFFFu;
  for (int m = tid; m < M; m += blockDim.x) {
    const uint32_t k = order_key(sc[m]);
    keys[m] = k;
    kmx = max(kmx, k);
    kmn = min(kmn, k);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    kmx = max(kmx, __shfl_xor_sync(0xffffffffu, kmx, o));
    kmn = min(kmn, __shfl_xor_sync(0xffffffffu, kmn, o));
  }
  if (lane == 0) {
    warp_max[warp] = kmx;
    warp_min[warp] = kmn;
  }
  __syncthreads();
  for (int w = 0; w < (int)(blockDim.x / 32); ++w) {
    kmx = max(kmx, warp_max[w]);
    kmn = min(kmn, warp_min[w]);
  }

  // Radix select of the K-th largest key, at most 8 bits at a time from the
  // top, until the bucket that holds it has at most kTopkCand keys; those few
  // are then ranked exactly by (key, page index).  `need` keys of the bucket
  // are kept.  The high bits on which the largest and the smallest key agree
  // are common to every key and decide nothing, so the first digit is the
  // (up to) 8 bits just below them (scores of similar magnitude share their
  // top byte: starting at bit 31 would spend a pass on it).
  const int hb = kmx == kmn ? -1 : 31 - __clz(kmx ^ kmn);  // highest bit where keys differ
  uint32_t mask = hb >= 31 ? 0u : (0xFFFFFFFFu << (hb + 1));
  uint32_t prefix = kmx & mask;
  int need = K, bucket = M;
  for (int hi = hb; hi >= 0 && bucket > kTopkCand;) {
    const int shift = max(0, hi - 7);
    const uint32_t dmask = (2u << (hi - shift)) - 1u;  // this pass's digit: bits [shift, hi]
    for (int i = tid; i < 256; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    // warp-aggregated: the lanes holding the same digit add their count once
    // (most keys share their top digits, which would serialise plain atomics)
    for (int base = 0; base < M; base += blockDim.x) {
      const int m = base + tid;
      const uint32_t k = m < M ? keys[m] : 0u;
      const bool act = m < M && (k & mask) == prefix;
      const uint32_t digit = act ? (k >> shift) & dmask : 256u;
      const unsigned peers = __match_any_sync(0xffffffffu, digit);
      if (act && lane == __ffs(peers) - 1) atomicAdd(&hist[digit], __popc(peers));
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
            sh_bucket = cnt[i];
          }
          above += cnt[i];
        }
      }
    }
    __syncthreads();
    need -= sh_above;
    prefix |= (uint32_t)sh_digit << shift;
    mask |= dmask << shift;
    bucket = sh_bucket;
    hi = shift - 1;
  }
  uint8_t* chosen = reinterpret_cast<uint8_t*>(keys + M);  // [M], valid for bucket members
  const bool ranked = bucket <= kTopkCand;
  if (ranked) {
    if (tid == 0) sh_ncand = 0;
    __syncthreads();
    for (int m = tid; m < M; m += blockDim.x)
      if ((keys[m] & mask) == prefix) cand[atomicAdd(&sh_ncand, 1)] = m;
    __syncthreads();
    for (int i = tid; i < bucket; i += blockDim.x) {
      const int mi = cand[i];
      const uint32_t ki = keys[mi];
      int r = 0;  // bucket keys ahead of this one
      for (int j = 0; j < bucket; ++j) {
        const int mj = cand[j];
        const uint32_t kj = keys[mj];
        r += (kj > ki) || (kj == ki && mj < mi);
      }
      chosen[mi] = r < need;
    }
    __syncthreads();
  }
  // Otherwise every bit was used and the bucket's keys are all equal: the
  // `need` lowest page indices among them are kept.

  // Compaction in ascending page order: one block scan of (above, kept) counts
  // over contiguous per-thread chunks.
  const int per = (M + blockDim.x - 1) / blockDim.x;
  const int lo = min(M, tid * per), hi = min(M, lo + per);
  uint32_t na = 0, nk = 0;
  for (int m = lo; m < hi; ++m) {
    const uint32_t km = keys[m] & mask;
    na += km > prefix;
    nk += km == prefix && (!ranked || chosen[m]);
  }
  uint32_t v = (na << 16) | nk, incl = v;
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
  uint32_t a_before = before >> 16, k_before = before & 0xFFFFu;
  for (int m = lo; m < hi; ++m) {
    const uint32_t km = keys[m] & mask;
    if (km > prefix) {
      sel[a_before + min(k_before, (uint32_t)need)] = m;
      ++a_before;
    } else if (km == prefix && (!ranked || chosen[m])) {
      if (k_before < (uint32_t)need) sel[a_before + k_before] = m;
      ++k_before;
    }
  }
  if (tid == 0) p.sel_count[pair] = K;
}

// Both kernels are launched as programmatic dependents of the work before
// them on the stream: their blocks may be scheduled while that work drains
// and wait (griddepcontrol.wait) before reading anything it may write.
template <typename Kern>
static cudaError_t launch_dependent(Kern kern, dim3 grid, int threads, size_t smem,
                                    cudaStream_t stream, const SelectParams& p) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

cudaError_t launch_page_select(const SelectParams& p, int D, cudaStream_t stream) {
  const int per_cta = kScoreWarps * kScorePagesPerWarp;
  dim3 grid((p.max_pages + per_cta - 1) / per_cta, p.num_kv_heads, p.batch);
  const int G = p.num_q_heads / p.num_kv_heads;
  cudaError_t e = cudaSuccess;
#define LSERVE_SCORE_CASE(DD, GG)                                                          \
  if (D == DD && G == GG) {                                                                \
    e = set_smem_once((const void*)page_score_kernel<DD, GG>, kScoreSmem);                 \
    if (e == cudaSuccess)                                                                  \
      e = launch_dependent(page_score_kernel<DD, GG>, grid, kScoreWarps * 32, kScoreSmem, stream, p); \
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
  if (e != cudaSuccess) return e;
  const size_t smem = (size_t)p.max_pages * (sizeof(uint32_t) + 1);  // keys + kept flags
  if (smem > 48 * 1024) {
    e = set_smem_once((const void*)page_topk_kernel, (int)smem);
    if (e != cudaSuccess) return e;
  }
  return launch_dependent(page_topk_kernel, dim3(p.num_kv_heads, p.batch), kTopkThreads, smem, stream,
                          p);
}

}  // namespace lserve
