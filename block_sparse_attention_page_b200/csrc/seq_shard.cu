// Sequence-sharded decode: one long sequence spread over N GPUs, each holding a
// contiguous range of its physical pages (LServe explainer, 技術的詳細 ›
// 動的スパーシティ and 階層的ページング for the page scores and the top-K; the
// split itself is this library's reading: the pages leave it open).
//
// Shard r of N holds pages [floor(M*r/N), floor(M*(r+1)/N)) of a sequence of
// M = ceil(n / N_P) pages.  Per decode step:
//   1. lserve_page_select on the shard's own pages (scores + its own top-K);
//   2. seqshard_candidates_kernel: the shard's top-K as (score, global page)
//      proposals;                                     -> all-gather (caller)
//   3. seqshard_merge_kernel: the global top-K re-made from all N shards'
//      proposals -- the same order as the unsharded top-K (score descending,
//      lowest page index on ties), so the choice is the unsharded one bit for
//      bit -- and the chosen pages this shard holds, as shard-local ordinals;
//      streaming heads get their sink + local pages that fall in the shard;
//   4. lserve_sparse_decode_attn_ex over those pages, fp32 out + lse;
//                                                     -> all-gather (caller)
//   5. seqshard_combine_kernel: o = sum_r e^(lse_r - M) o_r / sum_r e^(lse_r - M).
// Every shard's top-K holds every page of that shard that can be in the
// global top-K (its rank inside the shard is at most its global rank), so the
// union of the proposals contains the global choice.
#include "common.cuh"
#include "kernels.h"

namespace lserve {

namespace {

__device__ __forceinline__ int shard_first_page(int M, int r, int N) {
  return (int)(((long long)M * r) / N);
}

constexpr int kMergeThreads = 256;
constexpr int kMergeWarps = kMergeThreads / 32;
constexpr int kRankMax = 512;  // up to this many proposals: ranked directly, no bisection

// Sum of v over the block.  Two alternating slot rows make one barrier per
// call enough: a row is written again only two calls later, after every
// thread has passed the barrier of the call in between.
__device__ __forceinline__ int block_sum(int v, int* red, int& phase) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  v = __reduce_add_sync(0xffffffffu, v);
  if (lane == 0) red[phase * kMergeWarps + warp] = v;
  __syncthreads();
  int t = 0;
#pragma unroll
  for (int w = 0; w < kMergeWarps; ++w) t += red[phase * kMergeWarps + w];
  phase ^= 1;
  return t;
}

}  // namespace

// One CTA per (sequence, KV head): proposal i is the shard's i-th chosen page
// (ascending, as lserve_page_select writes them) with its physical score.
__global__ void seqshard_candidates_kernel(ShardParams p) {
  const int h = blockIdx.x, b = blockIdx.y;
  const size_t pair = (size_t)b * p.num_kv_heads + h;
  const int n = p.ctx_lens[b];
  const int M = (n + p.physical_page - 1) / p.physical_page;
  const int lo = shard_first_page(M, p.rank, p.num_shards);
  const int hi = shard_first_page(M, p.rank + 1, p.num_shards);
  const int own = min(hi - lo, p.max_pages);
  const int kind = p.head_kind[h], cnt_in = p.sel_count[pair];  // independent loads, issued together
  const int cnt = kind == 0 ? max(0, min(cnt_in, min(p.sel_stride, p.top_k))) : 0;
  for (int i = threadIdx.x; i < p.top_k; i += blockDim.x) {
    float s = -INFINITY;
    int pg = -1;
    if (i < cnt) {
      const int m = p.sel[pair * p.sel_stride + i];
      if (m >= 0 && m < own) {
        s = p.scores[pair * p.max_pages + m];
        pg = lo + m;
      } else {
        raise_status(p.status, LSERVE_ERR_BOUNDS);
      }
    }
    p.cand_score[pair * p.top_k + i] = s;
    p.cand_page[pair * p.top_k + i] = pg;
  }
}

// One CTA per (sequence, KV head).  Retrieval heads: the global top-K of the
// N * top_k proposals in shared memory, found without sorting.  Up to
// kRankMax proposals, each one's rank is counted directly (the proposals that
// come before it in (score descending, page ascending) order; pages are
// unique, so ranks are too) -- no barrier inside.  Beyond that, the K-th
// largest score key T by bisection over the 32-bit key space (each step one
// block-wide count of keys >= the midpoint), then, among the proposals whose
// key equals T, the lowest pages by a bisection over the page index.
// Streaming heads: the sink pages [0, ceil(sink / N_P)) and the pages holding
// the last local_tokens tokens, those in this shard.
__global__ void __launch_bounds__(kMergeThreads) seqshard_merge_kernel(ShardParams p) {
  extern __shared__ uint32_t smem[];  // keys [C], pages [C], chosen flags [C]
  __shared__ int red[2 * kMergeWarps];
  __shared__ int scan[kMergeWarps];
  const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const size_t pair = (size_t)b * p.num_kv_heads + h;
  const int n = p.ctx_lens[b];
  const int NP = p.physical_page;
  const int M = (n + NP - 1) / NP;
  const int lo = shard_first_page(M, p.rank, p.num_shards);
  const int hi = shard_first_page(M, p.rank + 1, p.num_shards);
  int32_t* out = p.out_sel + pair * p.out_stride;

  if (p.head_kind[h] != 0) {
    const int ns = min((p.sink + NP - 1) / NP, M);
    const int ls = max(max(0, n - p.local) / NP, ns);
    const int n1 = max(0, min(ns, hi) - lo);          // sink pages in [lo, hi)
    const int l0 = max(ls, lo);
    const int n2 = max(0, min(M, hi) - l0);           // local pages in [lo, hi)
    int total = n1 + n2;
    if (total > p.out_stride) {
      if (tid == 0) raise_status(p.status, LSERVE_ERR_BOUNDS);
      total = p.out_stride;
    }
    for (int i = tid; i < p.out_stride; i += blockDim.x)
      out[i] = i < total ? (i < n1 ? i : l0 - lo + (i - n1)) : -1;
    if (tid == 0) p.out_count[pair] = total;
    return;
  }

  const int K = p.top_k;
  const int C = p.num_shards * K;
  uint32_t* key = smem;
  int* page = reinterpret_cast<int*>(smem + C);
  uint8_t* chosen = reinterpret_cast<uint8_t*>(smem + 2 * C);
  int nvalid = 0;
  for (int c = tid; c < C; c += blockDim.x) {
    const int r = c / K, i = c - r * K;
    const size_t idx = (((size_t)r * p.batch + b) * p.num_kv_heads + h) * K + i;
    int pg = p.all_page[idx];
    if (pg >= M) {  // a proposal past the sequence: ignored
      raise_status(p.status, LSERVE_ERR_BOUNDS);
      pg = -1;
    }
    page[c] = pg;
    key[c] = pg >= 0 ? order_key(p.all_score[idx]) : 0u;
    nvalid += pg >= 0;
  }
  int phase = 0;
  nvalid = block_sum(nvalid, red, phase);  // its barrier also publishes key / page
  const int keff = min(min(K, M), nvalid);

  if (C <= kRankMax) {
    for (int c = tid; c < C; c += blockDim.x) {
      const int pg = page[c];
      const uint32_t kc = key[c];
      int r = 0;  // proposals ahead of this one (the same j for all threads: broadcast reads)
      for (int j = 0; j < C; ++j) {
        const int pj = page[j];
        const uint32_t kj = key[j];
        r += pj >= 0 && (kj > kc || (kj == kc && pj < pg));
      }
      chosen[c] = pg >= 0 && r < keff;
    }
  } else {
    // T = the largest t with #{key >= t} >= keff (keff >= 1); every valid key >= 0
    uint32_t T = 0;
    uint32_t pstar = 0;
    if (keff > 0) {
      uint32_t tl = 0, th = 0xFFFFFFFFu;
      while (tl < th) {
        const uint32_t mid = tl + (uint32_t)(((uint64_t)th - tl + 1) >> 1);
        int c_ge = 0;
        for (int c = tid; c < C; c += blockDim.x) c_ge += page[c] >= 0 && key[c] >= mid;
        if (block_sum(c_ge, red, phase) >= keff) tl = mid;
        else th = mid - 1;
      }
      T = tl;
      int c_gt = 0;
      for (int c = tid; c < C; c += blockDim.x) c_gt += page[c] >= 0 && key[c] > T;
      const int gt = block_sum(c_gt, red, phase);
      // the need = keff - gt lowest pages among key == T: P* = the smallest
      // page bound with #{key == T, page <= P*} >= need
      const int need = keff - gt;
      uint32_t pl = 0, ph = (uint32_t)max(M - 1, 0);
      while (pl < ph) {
        const uint32_t mid = (pl + ph) >> 1;
        int c_le = 0;
        for (int c = tid; c < C; c += blockDim.x)
          c_le += page[c] >= 0 && key[c] == T && (uint32_t)page[c] <= mid;
        if (block_sum(c_le, red, phase) >= need) ph = mid;
        else pl = mid + 1;
      }
      pstar = pl;
    }
    for (int c = tid; c < C; c += blockDim.x) {
      const int pg = page[c];
      chosen[c] = keff > 0 && pg >= 0 && (key[c] > T || (key[c] == T && (uint32_t)pg <= pstar));
    }
  }
  __syncthreads();

  // This shard's own proposals, slots [rank*K, rank*K + K), are its pages in
  // ascending order: the chosen ones are compacted in place by one block scan
  // over contiguous per-thread chunks.
  const int base = p.rank * K;
  const int per = (K + blockDim.x - 1) / blockDim.x;
  const int i0 = min(K, tid * per), i1 = min(K, i0 + per);
  int mine = 0;
  for (int i = i0; i < i1; ++i) mine += chosen[base + i];
  int incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) scan[warp] = incl;
  __syncthreads();
  int before = incl - mine, total = 0;
#pragma unroll
  for (int w = 0; w < kMergeWarps; ++w) {
    const int t = scan[w];
    if (w < warp) before += t;
    total += t;
  }
  for (int i = i0; i < i1; ++i)
    if (chosen[base + i]) {
      const int local = page[base + i] - lo;
      if (before < p.out_stride && local >= 0 && local < hi - lo) out[before] = local;
      ++before;
    }
  if (total > p.out_stride) {
    if (tid == 0) raise_status(p.status, LSERVE_ERR_BOUNDS);
    total = p.out_stride;
  }
  for (int i = total + tid; i < p.out_stride; i += blockDim.x) out[i] = -1;
  if (tid == 0) p.out_count[pair] = total;
}

// One warp per output row (query head of a sequence): the N shards' (o, lse)
// merged by their softmax normalisers.  A lane holds D/32 channels; the
// partials of four shards are loaded together (independent loads) before they
// are summed.
__global__ void seqshard_combine_kernel(CombineParams p) {
  constexpr int kCpl = 4;  // channels per lane, D <= 128
  constexpr int kBatch = 4;  // shards whose partials are in flight at once
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + warp;
  if (row >= p.rows) return;
  const int cpl = p.head_dim / 32;
  float M = -INFINITY;
  for (int r = 0; r < p.num_shards; ++r) M = fmaxf(M, p.lse_parts[(size_t)r * p.rows + row]);
  float wsum = 0.f;
  float acc[kCpl] = {0.f, 0.f, 0.f, 0.f};
  for (int r0 = 0; r0 < p.num_shards; r0 += kBatch) {
    float w[kBatch], v[kBatch][kCpl];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int r = r0 + u;
      const float l = r < p.num_shards ? p.lse_parts[(size_t)r * p.rows + row] : -INFINITY;
      w[u] = (M == -INFINITY || l == -INFINITY) ? 0.f : expf(l - M);
      const float* src = p.o_parts + ((size_t)r * p.rows + row) * p.head_dim + lane;
#pragma unroll
      for (int j = 0; j < kCpl; ++j) v[u][j] = (r < p.num_shards && j < cpl) ? src[32 * j] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      wsum += w[u];
#pragma unroll
      for (int j = 0; j < kCpl; ++j) acc[j] += w[u] * v[u][j];
    }
  }
#pragma unroll
  for (int j = 0; j < kCpl; ++j)
    if (j < cpl)
      p.out[(size_t)row * p.head_dim + lane + 32 * j] = __float2bfloat16_rn(wsum > 0.f ? acc[j] / wsum : 0.f);
  if (lane == 0 && p.lse) p.lse[row] = wsum > 0.f ? M + logf(wsum) : -INFINITY;
}

cudaError_t launch_seqshard_candidates(const ShardParams& p, cudaStream_t stream) {
  seqshard_candidates_kernel<<<dim3(p.num_kv_heads, p.batch), 128, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_seqshard_merge(const ShardParams& p, cudaStream_t stream) {
  const size_t smem = ((size_t)p.num_shards * p.top_k * 9 + 15) / 16 * 16;
  if (smem > 48 * 1024) {
    const cudaError_t e = set_smem_once((const void*)seqshard_merge_kernel, (int)smem);
    if (e != cudaSuccess) return e;
  }
  seqshard_merge_kernel<<<dim3(p.num_kv_heads, p.batch), kMergeThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_seqshard_combine(const CombineParams& p, cudaStream_t stream) {
  constexpr int kRowsPerCta = 8;
  seqshard_combine_kernel<<<(p.rows + kRowsPerCta - 1) / kRowsPerCta, 32 * kRowsPerCta, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace lserve
