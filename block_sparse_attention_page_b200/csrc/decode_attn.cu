// lserve_sparse_decode_attn kernel (LServe explainer, 統一ブロックスパースアテンション
// figure: retrieval heads attend the top-K physical pages, streaming heads the
// Lambda-shaped sink + local pages; 技術的詳細 › 静的スパーシティ).
//
// Work split ("stream-K" over pages).  For every (sequence b, KV head h) pair
// the pages it attends are cut into tiles of up to 64 tokens (one physical page
// at N_P <= 64); the tiles of all pairs are laid end to end and the list is cut
// into equal contiguous ranges, one per CTA of a persistent grid (one CTA per
// SM).  Every SM therefore streams the same number of KV bytes, however unequal
// the pairs are (64 selected pages next to ~10 sink + local pages).
//
// Per CTA: 16 warps (four per SM sub-partition to hide latency).  Every warp
// owns 1/16 of each tile's tokens and keeps its own online-softmax state, so a
// tile needs no CTA-wide barrier: warps run ahead of one another and overlap
// their phases.
//   feeding : all threads resolve up to 256 tiles at once (pair, page ordinal,
//             block-table lookup); each stage of an S-deep ring is refilled by
//             the last warp to finish with it -- K and V by TMA (128-byte
//             swizzle), the pair's q by a 1-D bulk copy.
//   QK      : 8 lanes per token, each an eighth of D with q of the heads in
//             registers (from the stage's bf16 q); packed FFMA2; three shuffles
//             join the eighths.
//   softmax : base-2 online softmax in fp32 per warp (warp-uniform running max
//             per head, row sums per lane).
//   PV      : lane = channel quad, over the warp's tokens; o of all G heads in
//             registers across tiles.
// At a pair boundary the warps' states are merged in shared memory.  A pair
// covered by one CTA is finalised there; otherwise each CTA writes an
// unnormalised (o, m, l) partial and the last CTA to finish the pair (per-pair
// counter in the workspace) merges the partials with log-sum-exp weights and
// resets the counter to zero.
#include "common.cuh"
#include "kernels.h"

namespace lserve {

namespace {

constexpr int kWarps = 16;
constexpr int kMergeWarps = 8;        // warps whose state fits the merge buffer at once
constexpr int kThreads = kWarps * 32;
constexpr int kTable = 256;            // tile descriptor slots
constexpr int kRound = kTable - 8;     // descriptors resolved per round (8 slots of slack)

// Pages the pair attends (retrieval: the selection; streaming: sink + local).
__device__ __forceinline__ int pair_pages(const DecodeParams& p, int pair) {
  const int b = pair / p.num_kv_heads, h = pair - b * p.num_kv_heads;
  const int n = p.ctx_lens[b];
  const int NP = p.physical_page;
  const int npages = (n + NP - 1) / NP;
  if (p.head_kind[h] == 0) return min(max(p.sel_count[pair], 0), min(p.top_k, npages));
  const int ns = min((p.sink + NP - 1) / NP, npages);
  const int ls = max(max(0, n - p.local) / NP, ns);
  return ns + max(0, npages - ls);
}

template <int D, int G>
struct DecLayout {
  static constexpr int kTileK = kDecodeTileMax * D * 2;                  // K (or V) tile bytes
  static constexpr int kStageQ = G * D * 2;
  static constexpr int kStage = (2 * kTileK + kStageQ + 1023) / 1024 * 1024;
  static constexpr int kPs = kWarps * 2 * (kDecodeTileMax / kWarps) * G * 8;  // two tiles
  static constexpr int kOw = kMergeWarps * G * D * 4;
  static constexpr int kMl = kMergeWarps * G * 2 * 4;
  static constexpr int kOff = (kDecodeMaxPairs + 1) * 4;
  static constexpr int kTab = kTable * 16;
  static constexpr int kFixed = kPs + kOw + kMl + kOff + kTab + 512;
  static constexpr int kBudget = 227 * 1024 - 1024;
  static constexpr int kStagesFit = (kBudget - kFixed) / kStage;
  static constexpr int kStages = kStagesFit > 8 ? 8 : kStagesFit;
  // offsets (stages first: 1024-aligned for the swizzled TMA tiles)
  static constexpr int oPs = kStages * kStage;
  static constexpr int oOw = oPs + kPs;
  static constexpr int oMl = oOw + kOw;
  static constexpr int oOff = oMl + kMl;
  static constexpr int oTab = (oOff + kOff + 15) / 16 * 16;
  static constexpr int oInfo = oTab + kTab;
  static constexpr int oBar = oInfo + kStages * 8;
  static constexpr int oCnt = oBar + kStages * 8;
  static constexpr int oMisc = oCnt + kStages * 4;
  static constexpr int kBytes = oMisc + 128;
  static_assert(kStages >= 2, "decode ring needs two stages");
  static_assert(kBytes <= kBudget, "decode shared memory over budget");
};

// CTA whose range holds tile u: largest c with floor(U*c/NC) <= u.
__device__ __forceinline__ int cta_of(long long u, long long U, int NC) {
  return (int)(((u + 1) * NC + U - 1) / U) - 1;
}

// CTA c has at least one tile (when U < NC some ranges are empty)
__device__ __forceinline__ bool cta_busy(int c, long long U, int NC) {
  return U * (c + 1) / NC > U * c / NC;
}

// Bounded wait that gives up at once when another warp already timed out.
__device__ __forceinline__ bool stage_wait(uint64_t* bar, uint32_t parity, uint64_t limit,
                                           unsigned int* status, volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (*abort_flag) return false;
    if ((uint64_t)(clock64() - t0) > limit) {
      raise_status(status, LSERVE_ERR_TIMEOUT);
      *abort_flag = 1;
      return false;
    }
  }
  return true;
}

}  // namespace

template <int D, int G, int TR>
__global__ void __launch_bounds__(kThreads, 1)
decode_attn_kernel(const __grid_constant__ DecodeParams p, const __grid_constant__ CUtensorMap kmap,
                   const __grid_constant__ CUtensorMap vmap) {
  using L = DecLayout<D, G>;
  constexpr int S = L::kStages;
  constexpr int HB = G < 4 ? G : 4;      // heads whose q a QK lane holds at a time
  constexpr int NHB = G / HB;            // head blocks (2 for G = 8)
  constexpr int LPT = 8;                 // QK lanes per token
  constexpr int CPT = D / LPT;           // channels per QK lane (an eighth of D)
  constexpr int NOUT = (G * D + kThreads - 1) / kThreads;  // merged outputs per thread
  constexpr int NQ = D / 4;              // PV channel quads
  constexpr int LPQ = 32 / NQ;           // PV lane groups per warp (1 at D=128, 2 at D=64)
  constexpr int NBOX = D / 64;
  constexpr int TPW_MAX = kDecodeTileMax / kWarps;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float2* ps_all = reinterpret_cast<float2*>(smem + L::oPs);
  float* ow = reinterpret_cast<float*>(smem + L::oOw);
  float* mlw = reinterpret_cast<float*>(smem + L::oMl);
  int* off = reinterpret_cast<int*>(smem + L::oOff);
  int4* tab = reinterpret_cast<int4*>(smem + L::oTab);
  int2* info = reinterpret_cast<int2*>(smem + L::oInfo);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::oBar);
  int* done_cnt = reinterpret_cast<int*>(smem + L::oCnt);
  int* misc = reinterpret_cast<int*>(smem + L::oMisc);  // [0..15] scan, [16] last flag, [18] abort
  volatile int* abort_flag = misc + 18;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int P = p.batch * p.num_kv_heads;
  const int tpp = p.tiles_per_page;
  const int NC = gridDim.x, cta = blockIdx.x;
  const uint64_t lim = p.wait_limit;

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      done_cnt[s] = 0;
    }
    misc[18] = 0;
    fence_mbar_init();
  }
  if (tid == 32) {
    tma_prefetch_desc(&kmap);
    tma_prefetch_desc(&vmap);
  }

  // ---- plan: tiles per pair -> exclusive prefix off[0..P] in shared memory
  {
    const int per = (P + kThreads - 1) / kThreads;
    const int lo = min(P, tid * per), hi = min(P, lo + per);
    int sum = 0;
    for (int pr = lo; pr < hi; ++pr) {
      const int c = pair_pages(p, pr) * tpp;
      off[pr] = c;
      sum += c;
    }
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    if (lane == 31) misc[warp] = incl;
    __syncthreads();
    int base = 0;
    for (int w = 0; w < warp; ++w) base += misc[w];
    int run = base + incl - sum;
    for (int pr = lo; pr < hi; ++pr) {
      const int c = off[pr];
      off[pr] = run;
      run += c;
    }
    if (tid == kThreads - 1) off[P] = base + incl;
    __syncthreads();
  }
  const long long U = off[P];
  const int u0 = (int)(U * cta / NC), u1 = (int)(U * (cta + 1) / NC);
  const int ntiles = u1 - u0;

  // pairs with nothing to attend (n = 0): zero output, lse = -inf
  if (cta == 0) {
    for (int pr = tid; pr < P; pr += kThreads) {
      if (off[pr + 1] != off[pr]) continue;
      const int b = pr / p.num_kv_heads, h = pr - b * p.num_kv_heads;
      for (int g = 0; g < G; ++g) {
        const size_t qh = (size_t)b * p.num_q_heads + (size_t)h * G + g;
        for (int c = 0; c < D; ++c) p.out[qh * D + c] = __float2bfloat16_rn(0.f);
        if (p.lse) p.lse[qh] = -INFINITY;
      }
    }
  }

  // ---- tile descriptors: (pair, first row in the [pool rows][D] view, valid tokens)
  auto lookup = [&](int u) -> int4 {
    int lo = 0, hi = P - 1;  // last pair with off[pair] <= u
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (off[mid] <= u) lo = mid; else hi = mid - 1;
    }
    const int pair = lo;
    const int local = u - off[pair];
    const int li = local / tpp, sub = local - li * tpp;
    const int b = pair / p.num_kv_heads, h = pair - b * p.num_kv_heads;
    const int n = p.ctx_lens[b];
    const int NP = p.physical_page;
    const int npages = (n + NP - 1) / NP;
    int m;
    if (p.head_kind[h] == 0) {
      m = p.sel[(size_t)pair * p.top_k + li];
    } else {
      const int ns = min((p.sink + NP - 1) / NP, npages);
      const int ls = max(max(0, n - p.local) / NP, ns);
      m = li < ns ? li : ls + (li - ns);
    }
    int pid = -1;
    if (m >= 0 && m < npages && m < p.max_pages) pid = p.block_table[(size_t)b * p.max_pages + m];
    if (pid < 0 || pid >= p.num_pool_pages) {  // bad selection or block-table entry: skip the page
      raise_status(p.status, LSERVE_ERR_BOUNDS);
      return make_int4(pair, 0, 0, 0);
    }
    return make_int4(pair, (int)(((long long)pid * p.num_kv_heads + h) * NP + sub * TR),
                     max(0, min(TR, n - m * NP - sub * TR)), 0);
  };
  auto lookup_round = [&](int k0) {
    for (int i = tid; i < kRound && k0 + i < ntiles; i += kThreads) tab[(k0 + i) % kTable] = lookup(u0 + k0 + i);
  };
  // one thread: load tile k into stage k % S
  auto issue = [&](int k) {
    const int4 t = tab[k % kTable];
    const int s = k % S;
    uint8_t* st = smem + s * L::kStage;
    info[s] = make_int2(t.x, t.z);
    const int b = t.x / p.num_kv_heads, h = t.x - b * p.num_kv_heads;
    mbar_arrive_expect_tx(&full[s], 2 * TR * D * 2 + L::kStageQ);
    // one contiguous TR x D tile each: 3-D view (64 channels, D/64 halves, rows)
    tma_load_3d(st, &kmap, 0, 0, t.y, &full[s]);
    tma_load_3d(st + L::kTileK, &vmap, 0, 0, t.y, &full[s]);
    bulk_load_1d(st + 2 * L::kTileK, p.q + ((size_t)b * p.num_q_heads + (size_t)h * G) * D,
                 L::kStageQ, &full[s]);
  };
  lookup_round(0);
  __syncthreads();
  if (warp == 0 && lane < S && lane < ntiles) issue(lane);

  // ---- per-warp mapping and state
  constexpr int tpw = TR / kWarps;             // tokens of each tile this warp owns
  const int tok_l = lane / LPT, qtr = lane % LPT;  // QK: (token, eighth of D)
  const int tok = warp * tpw + tok_l;
  const bool qk_lane = tok_l < tpw;
  const int quad = lane % NQ, half = lane / NQ;  // PV: channel quad (+ token half at D=64)
  const int pv_chunk = (4 * quad) / 8;
  const int pv_box = pv_chunk / 8, pv_cc = pv_chunk % 8;
  const int pv_byte = (quad & 1) * 8;
  constexpr int pv_n = tpw / LPQ;
  const int pv_t0 = warp * tpw + half * pv_n;
  // byte offsets inside a stage, fixed for the lane: its key chunks, and the
  // value words of its tokens
  // (a token row is NBOX consecutive 128-byte swizzle rows: row NBOX*t + half)
  uint32_t koff[CPT / 8];
#pragma unroll
  for (int ch = 0; ch < CPT / 8; ++ch) {
    const int c = (lane % LPT) * (CPT / 8) + ch;
    koff[ch] = sw128_offset(NBOX * (warp * tpw + lane / LPT) + c / 8, c % 8);
  }
  uint32_t voff[pv_n];
#pragma unroll
  for (int j = 0; j < pv_n; ++j)
    voff[j] = L::kTileK + pv_byte + sw128_offset(NBOX * (pv_t0 + j) + pv_box, pv_cc);
  float2* ps = ps_all + warp * 2 * TPW_MAX * G;  // [tile 0/1][token][head]
  int cur_pair = -1;
  float m_w[G], l_part[NHB];
  float2 o_acc[G][2];
  float2 qreg[HB][CPT / 2];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m_w[g] = -INFINITY;
    o_acc[g][0] = o_acc[g][1] = make_float2(0.f, 0.f);
  }
#pragma unroll
  for (int i = 0; i < NHB; ++i) l_part[i] = 0.f;

  auto load_q = [&](const uint8_t* st, int hb) {  // bf16 q of the stage -> this lane's quarter
#pragma unroll
    for (int h = 0; h < HB; ++h) {
      const uint4* src = reinterpret_cast<const uint4*>(st + 2 * L::kTileK + ((hb * HB + h) * D + qtr * CPT) * 2);
#pragma unroll
      for (int i = 0; i < CPT / 8; ++i) {
        const uint4 w = src[i];
        qreg[h][4 * i + 0] = bf16x2_to_float2(w.x);
        qreg[h][4 * i + 1] = bf16x2_to_float2(w.y);
        qreg[h][4 * i + 2] = bf16x2_to_float2(w.z);
        qreg[h][4 * i + 3] = bf16x2_to_float2(w.w);
      }
    }
  };

  // End of a pair segment (every warp arrives here at the same tile index):
  // merge the warps, then finalise or publish + maybe merge across CTAs.
  auto flush = [&](int pair) {
    float lw[NHB];  // this warp's row sum per head h, held by lane 2h
#pragma unroll
    for (int hb = 0; hb < NHB; ++hb) {
      float lv = l_part[hb];
#pragma unroll
      for (int o = LPT; o < 32; o <<= 1) lv += __shfl_xor_sync(0xffffffffu, lv, o);
      lw[hb] = lv;
    }
    if constexpr (LPQ == 2) {
#pragma unroll
      for (int g = 0; g < G; ++g) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          o_acc[g][j].x += __shfl_xor_sync(0xffffffffu, o_acc[g][j].x, 16);
          o_acc[g][j].y += __shfl_xor_sync(0xffffffffu, o_acc[g][j].y, 16);
        }
      }
    }
    // merge the warps, kMergeWarps at a time, into per-thread (M, o, l) of the outputs
    float Mo[NOUT], Oo[NOUT], Lo[NOUT];
#pragma unroll
    for (int i = 0; i < NOUT; ++i) {
      Mo[i] = -INFINITY;
      Oo[i] = 0.f;
      Lo[i] = 0.f;
    }
#pragma unroll
    for (int r = 0; r < kWarps / kMergeWarps; ++r) {
      const int wl = warp - r * kMergeWarps;
      if (wl >= 0 && wl < kMergeWarps) {
#pragma unroll
        for (int hb = 0; hb < NHB; ++hb)
          if (lane < 2 * HB && (lane & 1) == 0) mlw[(wl * G + hb * HB + (lane >> 1)) * 2 + 1] = lw[hb];
#pragma unroll
        for (int g = 0; g < G; ++g)
          if (lane == g) mlw[(wl * G + g) * 2] = m_w[g];
        if (lane < NQ) {
#pragma unroll
          for (int g = 0; g < G; ++g)
            *reinterpret_cast<float4*>(ow + (wl * G + g) * D + 4 * quad) =
                make_float4(o_acc[g][0].x, o_acc[g][0].y, o_acc[g][1].x, o_acc[g][1].y);
        }
      }
      __syncthreads();
#pragma unroll
      for (int i = 0; i < NOUT; ++i) {
        const int j = tid + i * kThreads;
        if (j < G * D) {
          const int g = j / D, c = j - g * D;
#pragma unroll
          for (int w = 0; w < kMergeWarps; ++w) {
            const float mw = mlw[(w * G + g) * 2];
            if (mw == -INFINITY) continue;
            const float Mn = fmaxf(Mo[i], mw);
            const float sc = exp2f(Mo[i] - Mn), wt = exp2f(mw - Mn);
            Oo[i] = Oo[i] * sc + wt * ow[(w * G + g) * D + c];
            Lo[i] = Lo[i] * sc + wt * mlw[(w * G + g) * 2 + 1];
            Mo[i] = Mn;
          }
        }
      }
      __syncthreads();
    }
    const bool live = !*abort_flag;
    const int b = pair / p.num_kv_heads, h = pair - b * p.num_kv_heads;
    const int c_first = cta_of(off[pair], U, NC), c_last = cta_of(off[pair + 1] - 1, U, NC);
    int nseg = 0;  // CTAs with tiles of this pair (CTAs without tiles write nothing)
    for (int cc = c_first; cc <= c_last; ++cc) nseg += cta_busy(cc, U, NC) ? 1 : 0;
    const size_t slot = (size_t)cta + pair;
#pragma unroll
    for (int i = 0; i < NOUT; ++i) {
      const int j = tid + i * kThreads;
      if (j >= G * D || !live) continue;
      const int g = j / D, c = j - g * D;
      const size_t qh = (size_t)b * p.num_q_heads + (size_t)h * G + g;
      if (nseg == 1) {
        const bool empty_row = !(Lo[i] > 0.f);
        p.out[qh * D + c] = __float2bfloat16_rn(empty_row ? 0.f : Oo[i] / Lo[i]);
        if (c == 0 && p.lse)
          p.lse[qh] = empty_row ? -INFINITY : (Mo[i] + __log2f(Lo[i])) * 0.69314718055994530942f;
      } else {
        p.part_o[(slot * G + g) * D + c] = Oo[i];
        if (c == 0) *reinterpret_cast<float2*>(p.part_ml + (slot * G + g) * 2) = make_float2(Mo[i], Lo[i]);
      }
    }
    if (nseg > 1 && live) {
      __threadfence();
      __syncthreads();
      if (tid == 0) misc[16] = (atomicAdd(&p.counters[pair], 1u) == (unsigned)(nseg - 1)) ? 1 : 0;
      __syncthreads();
      if (misc[16]) {  // last segment to finish: merge every partial of the pair
        __threadfence();
#pragma unroll
        for (int i = 0; i < NOUT; ++i) {
          const int j = tid + i * kThreads;
          if (j >= G * D) continue;
          const int g = j / D, c = j - g * D;
          float M = -INFINITY, o = 0.f, lsum = 0.f;
#pragma unroll 4
          for (int cc = c_first; cc <= c_last; ++cc) {
            const bool busy = cta_busy(cc, U, NC);  // predicated, independent loads
            const size_t sl = (size_t)cc + pair;
            const float2 ml = busy ? *reinterpret_cast<const float2*>(p.part_ml + (sl * G + g) * 2)
                                   : make_float2(-INFINITY, 0.f);
            const float os = busy ? p.part_o[(sl * G + g) * D + c] : 0.f;
            const float Mn = fmaxf(M, ml.x);
            if (Mn == -INFINITY) continue;
            const float sc = exp2f(M - Mn), wt = exp2f(ml.x - Mn);
            o = o * sc + wt * os;
            lsum = lsum * sc + wt * ml.y;
            M = Mn;
          }
          const size_t qh = (size_t)b * p.num_q_heads + (size_t)h * G + g;
          const bool empty_row = !(lsum > 0.f);
          p.out[qh * D + c] = __float2bfloat16_rn(empty_row ? 0.f : o / lsum);
          if (c == 0 && p.lse)
            p.lse[qh] = empty_row ? -INFINITY : (M + __log2f(lsum)) * 0.69314718055994530942f;
        }
        if (tid == 0) p.counters[pair] = 0u;
      }
    }
    __syncthreads();  // ow / mlw / misc free again
  };

  // Each iteration takes one tile, or two consecutive tiles of the same pair:
  // one softmax update per 128 tokens and two independent token chains per lane.
  int next_round = kRound;
  for (int k = 0; k < ntiles;) {
    if (k + S + 1 >= next_round && next_round < ntiles) {  // next round of tile descriptors
      __syncthreads();
      lookup_round(next_round);
      __syncthreads();
      next_round += kRound;
    }
    const int s0 = k % S, s1 = (k + 1) % S;
    const bool has1 = k + 1 < ntiles;
    bool arrived = stage_wait(&full[s0], (k / S) & 1, lim, p.status, abort_flag);
    if (has1) arrived = stage_wait(&full[s1], ((k + 1) / S) & 1, lim, p.status, abort_flag) && arrived;
    const bool ok = __all_sync(0xffffffffu, arrived);
    const int2 inf0 = info[s0];
    const int2 inf1 = has1 ? info[s1] : make_int2(-1, 0);
    const uint8_t* st0 = smem + s0 * L::kStage;
    const uint8_t* st1 = smem + s1 * L::kStage;
    if (inf0.x != cur_pair) {  // same decision in every warp (stage info is shared)
      if (cur_pair >= 0) flush(cur_pair);
      cur_pair = inf0.x;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        m_w[g] = -INFINITY;
        o_acc[g][0] = o_acc[g][1] = make_float2(0.f, 0.f);
      }
#pragma unroll
      for (int i = 0; i < NHB; ++i) l_part[i] = 0.f;
      if constexpr (NHB == 1) load_q(st0, 0);
    }
    const int nt = (has1 && inf1.x == inf0.x) ? 2 : 1;
    int valid[2];
    valid[0] = ok ? inf0.y : 0;
    valid[1] = (ok && nt == 2) ? inf1.y : 0;
    const uint8_t* stg[2] = {st0, st1};

    // ---- QK: partial dots over this lane's eighth of D, joined by three shuffles
    float x[2][NHB];
#pragma unroll
    for (int hb = 0; hb < NHB; ++hb) {
      if constexpr (NHB > 1) load_q(st0, hb);
      float2 acc[2][HB];
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int h = 0; h < HB; ++h) acc[i][h] = make_float2(0.f, 0.f);
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        if (qk_lane && tok < valid[i]) {
#pragma unroll
          for (int ch = 0; ch < CPT / 8; ++ch) {
            const int c = qtr * (CPT / 8) + ch;  // 16-byte chunk of the key row
            const uint4 kw = *reinterpret_cast<const uint4*>(stg[i] + koff[ch]);
            (void)c;
            const float2 k0 = bf16x2_to_float2(kw.x), k1 = bf16x2_to_float2(kw.y);
            const float2 k2 = bf16x2_to_float2(kw.z), k3 = bf16x2_to_float2(kw.w);
#pragma unroll
            for (int h = 0; h < HB; ++h) {
              acc[i][h] = __ffma2_rn(qreg[h][4 * ch + 0], k0, acc[i][h]);
              acc[i][h] = __ffma2_rn(qreg[h][4 * ch + 1], k1, acc[i][h]);
              acc[i][h] = __ffma2_rn(qreg[h][4 * ch + 2], k2, acc[i][h]);
              acc[i][h] = __ffma2_rn(qreg[h][4 * ch + 3], k3, acc[i][h]);
            }
          }
        }
      }
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        // join the 8 eighths by reduce-scatter: after the xor-4 and xor-2 steps
        // lane e holds head e % 4 summed over 4 lanes, the xor-1 step completes it
        float d[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const int hh = h < HB ? h : 0;
          d[h] = h < HB ? acc[i][hh].x + acc[i][hh].y : 0.f;
        }
        const bool up4 = (qtr & 4) != 0, up2 = (qtr & 2) != 0;
        // step 1: keep heads {0,1} (low lanes) or {2,3} (high lanes), send the other two
        const float s0 = up4 ? d[0] : d[2], s1 = up4 ? d[1] : d[3];
        const float r0 = __shfl_xor_sync(0xffffffffu, s0, 4), r1 = __shfl_xor_sync(0xffffffffu, s1, 4);
        const float k0 = (up4 ? d[2] : d[0]) + r0, k1 = (up4 ? d[3] : d[1]) + r1;
        // step 2: keep one of the two
        const float sx = up2 ? k0 : k1;
        const float kx = (up2 ? k1 : k0) + __shfl_xor_sync(0xffffffffu, sx, 2);
        const float dot = kx + __shfl_xor_sync(0xffffffffu, kx, 1);
        // lane e now holds head ((e & 4) ? 2 : 0) + ((e & 2) ? 1 : 0) = (e >> 1) & 3
        x[i][hb] = dot;
      }
    }
    // each lane's head after the reduce-scatter; lanes whose head is >= HB hold nothing
    const int my_h = (qtr >> 1) & 3;
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int hb = 0; hb < NHB; ++hb)
        x[i][hb] = (qk_lane && tok < valid[i] && my_h < HB && (qtr & 1) == 0) ? x[i][hb] * p.scale_log2 : -INFINITY;
    // ---- warp max per head over both tiles, new running max
    float tmax[G];
#pragma unroll
    for (int hb = 0; hb < NHB; ++hb) {
      float mx = fmaxf(x[0][hb], x[1][hb]);
#pragma unroll
      for (int o = LPT; o < 32; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
#pragma unroll
      for (int h = 0; h < HB; ++h) tmax[hb * HB + h] = __shfl_sync(0xffffffffu, mx, 2 * h);
    }
    float alpha[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float mnew = fmaxf(m_w[g], tmax[g]);
      alpha[g] = mnew == -INFINITY ? 1.f : fast_ex2(m_w[g] - mnew);
      m_w[g] = mnew;
    }
#pragma unroll
    for (int hb = 0; hb < NHB; ++hb) {
      float m_h = 0.f, a_h = 1.f;  // this lane's head, picked without dynamic indexing
#pragma unroll
      for (int g = 0; g < HB; ++g) {
        if (g == my_h) {
          m_h = m_w[hb * HB + g];
          a_h = alpha[hb * HB + g];
        }
      }
      float lsum = l_part[hb] * a_h;
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const float pr = fast_ex2(x[i][hb] - m_h);  // x = -inf gives 0
        lsum += pr;
        if (qk_lane && (qtr & 1) == 0 && my_h < HB)
          ps[(i * TPW_MAX + tok_l) * G + hb * HB + my_h] = make_float2(pr, pr);
      }
      l_part[hb] = lsum;
    }
    __syncwarp();

    // ---- PV: lane = channel quad, over this warp's tokens of both tiles, all G heads
#pragma unroll
    for (int g = 0; g < G; ++g) {
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        o_acc[g][j].x *= alpha[g];
        o_acc[g][j].y *= alpha[g];
      }
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
#pragma unroll
      for (int j = 0; j < pv_n; ++j) {
        const int t = pv_t0 + j;
        if (t < valid[i]) {
          const uint2 vw = *reinterpret_cast<const uint2*>(stg[i] + voff[j]);
          const float2 v01 = bf16x2_to_float2(vw.x), v23 = bf16x2_to_float2(vw.y);
          const float2* pt = ps + (i * TPW_MAX + half * pv_n + j) * G;
          if constexpr (G >= 2) {
#pragma unroll
            for (int g2 = 0; g2 < G / 2; ++g2) {
              const float4 pq = reinterpret_cast<const float4*>(pt)[g2];
              const float2 pa = make_float2(pq.x, pq.y), pb = make_float2(pq.z, pq.w);
              o_acc[2 * g2][0] = __ffma2_rn(pa, v01, o_acc[2 * g2][0]);
              o_acc[2 * g2][1] = __ffma2_rn(pa, v23, o_acc[2 * g2][1]);
              o_acc[2 * g2 + 1][0] = __ffma2_rn(pb, v01, o_acc[2 * g2 + 1][0]);
              o_acc[2 * g2 + 1][1] = __ffma2_rn(pb, v23, o_acc[2 * g2 + 1][1]);
            }
          } else {
            const float2 pa = pt[0];
            o_acc[0][0] = __ffma2_rn(pa, v01, o_acc[0][0]);
            o_acc[0][1] = __ffma2_rn(pa, v23, o_acc[0][1]);
          }
        }
      }
    }
    __syncwarp();
    // ---- release the stage(s); the last warp to finish one refills it
    if (lane == 0) {
      __threadfence_block();
      for (int i = 0; i < nt; ++i) {
        const int kk = k + i, ss = kk % S;
        if (atomicAdd(&done_cnt[ss], 1) == kWarps - 1) {
          done_cnt[ss] = 0;
          if (kk + S < ntiles && !*abort_flag) {
            fence_proxy_async_smem();
            issue(kk + S);
          }
        }
      }
    }
    k += nt;
  }
  if (cur_pair >= 0) flush(cur_pair);
}

size_t decode_workspace_bytes(int pairs, int grid, int G, int D) {
  const size_t cnt = ((size_t)pairs * 4 + 255) / 256 * 256;
  const size_t slots = (size_t)grid + pairs;
  const size_t o = (slots * G * D * 4 + 255) / 256 * 256;
  return cnt + o + slots * G * 2 * 4;
}

int decode_grid(int sm_count) { return sm_count; }

cudaError_t launch_decode(const DecodeParams& p, const CUtensorMap& kmap, const CUtensorMap& vmap,
                          int D, int G, int grid, cudaStream_t stream) {
  cudaError_t e = cudaSuccess;
#define LSERVE_DECODE_CASE(DD, GG)                                                        \
  if (D == DD && G == GG) {                                                               \
    const int smem = DecLayout<DD, GG>::kBytes + 1024;                                    \
    if (p.tile_rows == 64) {                                                              \
      e = set_smem_once((const void*)decode_attn_kernel<DD, GG, 64>, smem);               \
      if (e != cudaSuccess) return e;                                                     \
      decode_attn_kernel<DD, GG, 64><<<grid, kThreads, smem, stream>>>(p, kmap, vmap);    \
    } else {                                                                              \
      e = set_smem_once((const void*)decode_attn_kernel<DD, GG, 32>, smem);               \
      if (e != cudaSuccess) return e;                                                     \
      decode_attn_kernel<DD, GG, 32><<<grid, kThreads, smem, stream>>>(p, kmap, vmap);    \
    }                                                                                     \
    return cudaGetLastError();                                                            \
  }
  LSERVE_DECODE_CASE(64, 1)
  LSERVE_DECODE_CASE(64, 2)
  LSERVE_DECODE_CASE(64, 4)
  LSERVE_DECODE_CASE(64, 8)
  LSERVE_DECODE_CASE(128, 1)
  LSERVE_DECODE_CASE(128, 2)
  LSERVE_DECODE_CASE(128, 4)
  LSERVE_DECODE_CASE(128, 8)
#undef LSERVE_DECODE_CASE
  (void)e;
  return cudaErrorInvalidValue;
}

}  // namespace lserve
