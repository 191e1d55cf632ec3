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
// Per CTA: one producer warp and W = 8 consumer warps, one CTA per SM.  (A
// two-CTAs-per-SM shape -- W = 4, 32-token tiles, at most 112 KB of shared
// memory each, so that the next call's CTAs are resident while this call
// runs -- measured 1.5x slower on the 8B layer and is not instantiated.)
//   producer : its lanes resolve 32 tiles at a time (pair, page ordinal,
//              block-table lookup); then, stage by stage of an S-deep ring, it
//              waits until every consumer warp has released the stage and
//              refills it -- K and V by TMA (128-byte swizzle), the pair's q by
//              a 1-D bulk copy.
//   consumers: every warp owns 1/W of each tile's tokens and keeps
//              its own online-softmax state, so a tile needs no CTA-wide
//              barrier.  An iteration takes one tile, or two consecutive tiles
//              of the same pair.
//     QK     : 8 lanes per token, each an eighth of D with q in registers;
//              packed FFMA2; the G x rows partial dots of a lane are joined by
//              a reduce-scatter over the 8 lanes, so that afterwards every lane
//              holds whole dots of ONE head.
//     softmax: base-2 online softmax in fp32; running max per head shared by
//              the warp, one exp2 per head and lane for the rescale.
//     PV     : lane = channel quad, over the warp's tokens; o of all G heads in
//              registers across tiles, rescaled only when a running max grew.
// Pair boundaries come from the tile plan in shared memory, so all consumer
// warps agree on them whatever the data.  At a boundary the warps' states are
// merged in shared memory.  A pair covered by one CTA is finalised there.  A
// pair split over CTAs c_f .. c_l is merged by c_f, the CTA holding its first
// tile (the pair closes c_f's range, so c_f reaches it last): every other CTA
// c of the pair holds it as its FIRST pair and writes its unnormalised
// (o, m, l) partial into its own workspace slot as tagged 8-byte words
// {value, tag}.  c_f polls only the small (m, l) words (one warp's worth of
// loads per poll: polling every o word as well put ~60 KB per poll on the
// SM's load path and slowed the merge), stages them in shared memory, then
// reads each o word once (checking its tag too) and merges with log-sum-exp
// weights.  No fence, counter or atomic is involved: a word is one
// single-copy atomic store, and the tag carries the pair and the pair's merge
// epoch (a per-pair counter that c_f advances at the end of every call,
// whatever happened), so words left by an earlier call -- even one that ended
// in a timeout -- never match.
#include <cstring>
#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace lserve {

namespace {

constexpr int kBarConsumers = 1;       // named barrier of the consumer warps
constexpr int kMaxGrid = 512;          // CTAs whose range starts the range table holds
constexpr unsigned kFull = 0xffffffffu;

// One output element: bf16 by default, float with LSERVE_DECODE_OUT_F32.
__device__ __forceinline__ void store_out(const DecodeParams& p, size_t i, float v) {
  if (p.out_f32) p.out_f32[i] = v;
  else p.out[i] = __float2bfloat16_rn(v);
}

// Recent pages of a retrieval pair (the option of attending every token since
// the selection): the pages [ra, rz] holding positions [recent_from[b], n);
// those the selection holds are attended as selected pages.  The selection is
// ascending, so its entries in [ra, rz] are among its last rz - ra + 1.
__device__ __forceinline__ bool recent_range(const DecodeParams& p, int b, int n, int& ra, int& rz,
                                             int& rf) {
  if (!p.recent_from || n <= 0) return false;
  rf = max(0, min(p.recent_from[b], n));
  if (rf >= n) return false;
  ra = rf / p.physical_page;
  rz = (n - 1) / p.physical_page;
  return true;
}
// First index of the ascending selection s[0..nsel) whose page is >= ra: the
// selected pages among the recent ones are s[i0 .. nsel) (all are <= rz).
__device__ __forceinline__ int sel_tail_start(const int32_t* s, int nsel, int ra) {
  int i = nsel;
  while (i > 0 && s[i - 1] >= ra) --i;
  return i;
}
// The r-th recent page (0-based, ascending) that the selection does not hold:
// ra + r, pushed up by one for every selected page at or below it.
__device__ __forceinline__ int recent_page(const int32_t* s, int i0, int nsel, int ra, int r) {
  int j = ra + r;
  for (int i = i0; i < nsel && s[i] <= j; ++i) ++j;
  return j;
}

// Selected pages of a retrieval pair the attention takes (the clamped count).
__device__ __forceinline__ int sel_pages(const DecodeParams& p, int pair, int npages) {
  return min(max(p.sel_count[pair], 0), min(p.top_k, npages));
}

// Pages the pair attends (retrieval: the selection, plus the recent pages it
// does not hold; streaming: sink + local).
__device__ __forceinline__ int pair_pages(const DecodeParams& p, int pair) {
  const int b = pair / p.num_kv_heads, h = pair - b * p.num_kv_heads;
  const int n = p.ctx_lens[b];
  const int kind = p.head_kind[h];
  const int sc = p.sel_count[pair];  // loaded with the other two (one round trip)
  const int NP = p.physical_page;
  const int npages = (n + NP - 1) / NP;
  if (kind == 0) {
    const int nsel = min(max(sc, 0), min(p.top_k, npages));
    int ra, rz, rf;
    if (!recent_range(p, b, n, ra, rz, rf)) return nsel;
    const int32_t* s = p.sel + (size_t)pair * p.top_k;
    return nsel + max(0, (rz - ra + 1) - (nsel - sel_tail_start(s, nsel, ra)));
  }
  const int ns = min((p.sink + NP - 1) / NP, npages);
  const int ls = max(max(0, n - p.local) / NP, ns);
  return ns + max(0, npages - ls);
}

// The appended token's rows: K and V into the pools, and for a retrieval
// head its logical page's k_min / k_max (a page's first token starts them),
// exact in bf16.  One warp per (sequence, KV head); lanes take 16-byte
// chunks (D / 8 of them per row).
template <int D>
__device__ __forceinline__ void append_rows(const DecodeParams& p, int pair, int lane) {
  const int b = pair / p.num_kv_heads, h = pair - b * p.num_kv_heads;
  const int n = p.ctx_lens[b];
  if (n <= 0) return;
  const int t = n - 1, NP = p.physical_page, m = t / NP;
  int pid = -1;
  if (m < p.max_pages) pid = p.block_table[(size_t)b * p.max_pages + m];
  if (pid < 0 || pid >= p.num_pool_pages) {
    if (lane == 0) raise_status(p.status, LSERVE_ERR_BOUNDS);
    return;
  }
  constexpr int C16 = D / 8;  // 16-byte chunks per row
  const size_t row = ((size_t)pid * p.num_kv_heads + h) * NP + (t - m * NP);
  const size_t src = ((size_t)b * p.num_kv_heads + h) * D;
  if (lane < C16) {
    const uint4 k = *reinterpret_cast<const uint4*>(p.k_new + src + lane * 8);
    *reinterpret_cast<uint4*>(p.k_pool_w + row * D + lane * 8) = k;
    if (p.head_kind[h] == 0) {
      const int g = NP / p.logical_page, sub = (t - m * NP) / p.logical_page;
      __nv_bfloat16* st = p.stats_w + (((size_t)pid * p.num_kv_heads + h) * g + sub) * 2 * D + lane * 8;
      uint4 lo = k, hi = k;
      if (t % p.logical_page != 0) {
        const uint4 a = *reinterpret_cast<const uint4*>(st), z = *reinterpret_cast<const uint4*>(st + D);
        const __nv_bfloat162* kk = reinterpret_cast<const __nv_bfloat162*>(&k);
        const __nv_bfloat162* aa = reinterpret_cast<const __nv_bfloat162*>(&a);
        const __nv_bfloat162* zz = reinterpret_cast<const __nv_bfloat162*>(&z);
        __nv_bfloat162* ll = reinterpret_cast<__nv_bfloat162*>(&lo);
        __nv_bfloat162* hh = reinterpret_cast<__nv_bfloat162*>(&hi);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          ll[i] = __hmin2(aa[i], kk[i]);
          hh[i] = __hmax2(zz[i], kk[i]);
        }
      }
      *reinterpret_cast<uint4*>(st) = lo;
      *reinterpret_cast<uint4*>(st + D) = hi;
    }
  } else if (lane < 2 * C16) {
    const int c = lane - C16;
    *reinterpret_cast<uint4*>(p.v_pool_w + row * D + c * 8) =
        *reinterpret_cast<const uint4*>(p.v_new + src + c * 8);
  }
}

// QB = 8 / 4: the quantized cache -- K / V tiles of 8- or 4-bit codes
// followed by the page's K and V channel scales (float32 [D] each); QB = 0:
// bf16 tiles.  TR tokens per tile, W consumer warps; W = 4 is the
// two-CTAs-per-SM shape (at most 112 KB of shared memory each), W = 8 takes a
// whole SM.
template <int D, int G, int QB, int TR, int W>
struct DecLayout {
  static constexpr int kRow = D * (QB == 0 ? 16 : QB) / 8;               // bytes per K (or V) row
  static constexpr int kTileK = TR * kRow;                               // K (or V) tile bytes
  // K, V channel scales: four segments of D/4 channels (one per lane quad
  // position of the MMA fragments) at a padded stride, so that the four
  // segments a warp reads at once fall in different shared-memory banks
  static constexpr int kScaleSeg = D;                                    // bytes: D/4 floats
  static constexpr int kScaleSegP = kScaleSeg + 32;
  static constexpr int kScales = QB ? 2 * 4 * kScaleSegP : 0;
  static constexpr int oScale = 2 * kTileK;                              // stage offsets
  static constexpr int oQ = oScale + kScales;
  static constexpr int kStageQ = G * D * 2;
  static constexpr int oNew = oQ + kStageQ;                              // appended K, V rows (bf16)
  static constexpr int kNew = QB ? 0 : 2 * D * 2;
  static constexpr int kStage = (oNew + kNew + 1023) / 1024 * 1024;
  static constexpr int kPs = 2 * TR * G * 8;                            // p of two tiles
  static constexpr int kOw = W * G * D * 4;                              // o per warp
  static constexpr int kMl = W * G * 2 * 4;                              // (m, l) per warp
  static constexpr int kOff = ((kDecodeMaxPairs + 1) * 4 + 15) / 16 * 16;
  static constexpr int kCst = ((kMaxGrid + 1) * 4 + 15) / 16 * 16;
  static constexpr int kFixed = kPs + kOw + kMl + kOff + kCst + 1024;
  static constexpr int kBudget = W <= 4 ? 112 * 1024 : 227 * 1024 - 1024;
  static constexpr int kStagesFit = (kBudget - kFixed) / kStage;
  static constexpr int kStages = kStagesFit > 8 ? 8 : kStagesFit;
  // offsets (stages first: 1024-aligned for the swizzled TMA tiles)
  static constexpr int oPs = kStages * kStage;
  static constexpr int oOw = oPs + kPs;
  static constexpr int oMl = oOw + kOw;
  static constexpr int oOff = (oMl + kMl + 15) / 16 * 16;
  static constexpr int oCst = oOff + kOff;
  static constexpr int oInfo = oCst + kCst;
  static constexpr int oFull = (oInfo + kStages * 4 + 7) / 8 * 8;
  static constexpr int oEmpty = oFull + kStages * 8;
  static constexpr int oMisc = (oEmpty + kStages * 8 + 15) / 16 * 16;
  static constexpr int kBytes = oMisc + 128;
  static_assert(kStages >= 2, "decode ring needs two stages");
  static_assert(kStages * kStage >= kMaxGrid * G * 8, "the idle ring stages the merge's (m, l) words");
  static_assert(oPs % 16 == 0 && oOw % 16 == 0 && oMl % 16 == 0 &&
                    oOff % 16 == 0 && oCst % 16 == 0 && oInfo % 4 == 0 && oFull % 8 == 0 &&
                    oEmpty % 8 == 0 && oMisc % 16 == 0,
                "decode shared-memory arrays must keep their alignment");
  static_assert(kBytes <= kBudget, "decode shared memory over budget");
};

// First tile of CTA c's range, floor(U * c / NC) (c = NC gives U), in 32-bit
// arithmetic: U = q * NC + r, so U * c / NC = q * c + r * c / NC with
// r * c < NC^2.
__device__ __forceinline__ int range_start(int U, int c, int NC) {
  const int q = U / NC, r = U - q * NC;
  return q * c + (r * c) / NC;
}
// cst[c] = range_start(U, c, NC).  CTA whose range holds tile u: the largest
// c < NC with cst[c] <= u (ranges can be empty when U < NC; the largest such c
// is the one that owns u).
__device__ __forceinline__ int cta_of(const int* cst, int u, int NC) {
  int lo = 0, hi = NC - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (cst[mid] <= u) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// CTA c has at least one tile
__device__ __forceinline__ bool cta_busy(const int* cst, int c) { return cst[c + 1] > cst[c]; }

// Pair that tile u belongs to: the last pair with off[pair] <= u (pairs without
// tiles share their offset with the next pair and are skipped).
__device__ __forceinline__ int pair_of(const int* off, int u, int P) {
  int lo = 0, hi = P - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (off[mid] <= u) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Tagged partial words: {float value, tag} as one 64-bit store / load.  The
// tag is the pair's merge epoch for this call (20 bits) over the pair (11 low
// bits; pairs are < 2048), with the top bit set so that a zeroed word never
// matches -- a word from another pair, or from any of the pair's previous
// 2^20 - 1 calls, differs.
__device__ __forceinline__ uint32_t part_tag(uint32_t epoch, int pair) {
  return 0x80000000u | ((epoch & 0xFFFFFu) << 11) | (uint32_t)pair;
}
__device__ __forceinline__ void st_word(unsigned long long* a, float v, uint32_t tag) {
  const unsigned long long w = ((unsigned long long)tag << 32) | __float_as_uint(v);
  asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(a), "l"(w) : "memory");
}
__device__ __forceinline__ unsigned long long ld_word(const unsigned long long* a) {
  unsigned long long w;
  asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];" : "=l"(w) : "l"(a) : "memory");
  return w;
}
// Two adjacent words (16-byte aligned) in one access; each word is still a
// single-copy atomic 8-byte element.
__device__ __forceinline__ void st_word2(unsigned long long* a, float v0, float v1, uint32_t tag) {
  const unsigned long long w0 = ((unsigned long long)tag << 32) | __float_as_uint(v0);
  const unsigned long long w1 = ((unsigned long long)tag << 32) | __float_as_uint(v1);
  asm volatile("st.relaxed.gpu.global.v2.b64 [%0], {%1, %2};" ::"l"(a), "l"(w0), "l"(w1) : "memory");
}
__device__ __forceinline__ void ld_word2(const unsigned long long* a, unsigned long long& w0,
                                         unsigned long long& w1) {
  asm volatile("ld.relaxed.gpu.global.v2.b64 {%0, %1}, [%2];" : "=l"(w0), "=l"(w1) : "l"(a) : "memory");
}
__device__ __forceinline__ bool word_ok(unsigned long long w, uint32_t tag) {
  return (uint32_t)(w >> 32) == tag;
}
__device__ __forceinline__ float word_val(unsigned long long w) {
  return __uint_as_float((uint32_t)w);
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

// ---- QK join: a lane's V = G * R partial dots (index v = g * R + r, r the
// row of 4 tokens) are summed over the 8 lanes of its token by halving the
// list at lane strides 4, 2, 1: the lane keeps one half and sends the other.
// A step whose half would be empty sums the single value instead.
// first index a lane holds after the join, for lane bits (qtr) of the token
__host__ __device__ constexpr int join_base(int V, int qtr) {
  return ((qtr & 4) && V >= 2 ? V / 2 : 0) + ((qtr & 2) && V >= 4 ? V / 4 : 0) +
         ((qtr & 1) && V >= 8 ? V / 8 : 0);
}
// the step at this lane stride split the list inside one head's R rows: the
// two lanes hold different rows of the same head (a step that did not split
// leaves both lanes with the same values)
__host__ __device__ constexpr bool row_bit(int V, int R, int stride) {
  return (V * stride / 8) >= 1 && (V * stride / 8) < R;
}
// lane (of the 8) that holds head g's first row after the join
__host__ __device__ constexpr int head_src(int V, int R, int g) {
  int src = 0;
  for (int q = 7; q >= 0; --q)
    if (join_base(V, q) == g * R) src = q;
  return src;
}

template <int N, int STRIDE>
__device__ __forceinline__ void join_step(const float (&in)[N], float (&out)[N >= 2 ? N / 2 : 1],
                                          bool up) {
  if constexpr (N >= 2) {
#pragma unroll
    for (int i = 0; i < N / 2; ++i) {
      const float send = up ? in[i] : in[i + N / 2];
      const float keep = up ? in[i + N / 2] : in[i];
      out[i] = keep + __shfl_xor_sync(kFull, send, STRIDE);
    }
  } else {
    out[0] = in[0] + __shfl_xor_sync(kFull, in[0], STRIDE);
  }
}

template <int V>
constexpr int join_out() { return V >= 8 ? V / 8 : 1; }

// Quantized codes -> fp16 pairs, exactly (|code| <= 127 fits fp16's 11-bit
// significand).  8-bit: a byte c placed as the low byte of the fp16 1024 + x
// (0x64xx: 1024 .. 1279, step 1) after flipping its sign bit gives
// 1024 + (c + 128); subtracting 1152 leaves c.  Word w (codes of channels
// 4m .. 4m+3, lowest byte first) gives the pairs (4m, 4m+1) and (4m+2, 4m+3).
__device__ __forceinline__ void codes8_to_f16(uint32_t w, uint32_t& p01, uint32_t& p23) {
  const uint32_t u = w ^ 0x80808080u;
  const uint32_t x = __byte_perm(u, 0x64646464u, 0x4140);
  const uint32_t y = __byte_perm(u, 0x64646464u, 0x4342);
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(p01) : "r"(x), "r"(0x64806480u));
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(p23) : "r"(y), "r"(0x64806480u));
}
// 4-bit: nibble c of channel 8m + j (lowest nibble first) flipped by 8 is
// c + 8 in 1..15; ORed into the fp16 1024 and less 1032 it is c.  Word w
// (channels 8m .. 8m+7) gives the pairs (8m + j, 8m + j + 4), j = 0..3.
__device__ __forceinline__ uint32_t codes4_pair(uint32_t u, int j) {
  const uint32_t x = ((u >> (4 * j)) & 0x000F000Fu) | 0x64006400u;
  uint32_t r;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(x), "r"(0x64086408u));
  return r;
}
// channel offset (inside a lane's run) of element e of pair p of QB-bit codes
__host__ __device__ constexpr int pair_channel(int QB, int p, int e) {
  return QB == 4 ? 8 * (p / 4) + (p % 4) + 4 * e : 2 * p + e;
}
__device__ __forceinline__ uint32_t f32x2_to_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ float f16_lo(uint32_t w) { return __half2float(__ushort_as_half((unsigned short)(w & 0xFFFFu))); }
__device__ __forceinline__ float f16_hi(uint32_t w) { return __half2float(__ushort_as_half((unsigned short)(w >> 16))); }
// 8x8 b16 matrix transposed across the warp (lane L holds row L/4, columns
// 2*(L%4) + {0,1} before and after)
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
  uint32_t r;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(r) : "r"(x));
  return r;
}
__device__ __forceinline__ void mma_16816_f16(float (&d)[4], uint32_t a0, uint32_t a2, uint32_t b0,
                                              uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9},"
      " {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_1688_f16(float (&d)[4], uint32_t a0, uint32_t b0) {
  asm("mma.sync.aligned.m16n8k8.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5}, {%6},"
      " {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(0u), "r"(b0));
}

// Warp-level tensor-core tiles (mma.sync, bf16 in, fp32 accumulate).  The
// fragment layouts are those of the PTX ISA for m16n8k16 / m16n8k8 row.col:
// lane L holds rows L/4 (and L/4 + 8) of A and C, columns 2*(L%4) + {0,1}.
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a2, uint32_t b0,
                                          uint32_t b1) {
  // rows 8..15 of A are zero (at most 8 query heads per KV head)
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9},"
      " {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_1688(float (&d)[4], uint32_t a0, uint32_t b0) {
  asm("mma.sync.aligned.m16n8k8.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5}, {%6},"
      " {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(0u), "r"(b0));
}
// four 8x8 bf16 matrices, transposed, from shared memory (lane L gives the
// address of row L%8 of matrix L/8)
__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}

template <int V>
__device__ __forceinline__ void join_dots(const float (&d)[V], float (&out)[join_out<V>()], int qtr) {
  constexpr int N1 = V >= 2 ? V / 2 : 1, N2 = N1 >= 2 ? N1 / 2 : 1;
  float a[N1], b[N2];
  join_step<V, 4>(d, a, (qtr & 4) != 0);
  join_step<N1, 2>(a, b, (qtr & 2) != 0);
  join_step<N2, 1>(b, out, (qtr & 1) != 0);
}

}  // namespace

template <int D, int G, int TR, int QB, int W>
__global__ void __launch_bounds__((W + 1) * 32, W <= 4 ? 2 : 1)
decode_attn_kernel(const __grid_constant__ DecodeParams p, const __grid_constant__ CUtensorMap kmap,
                   const __grid_constant__ CUtensorMap vmap) {
  using L = DecLayout<D, G, QB, TR, W>;
  constexpr bool Q8 = QB != 0;             // a quantized cache (8- or 4-bit codes)
  constexpr int kThreads = (W + 1) * 32;   // consumer warps + the producer warp
  constexpr int kConsumerThreads = W * 32;
  constexpr int S = L::kStages;
  constexpr int HB = G < 4 ? G : 4;      // heads whose q a QK lane holds at a time
  constexpr int NHB = G / HB;            // head blocks (2 for G = 8)
  constexpr int LPT = 8;                 // QK lanes per token
  constexpr int CPT = D / LPT;           // channels per QK lane (an eighth of D)
  constexpr int KCH = CPT / 8;           // 16-byte key chunks per QK lane
  constexpr int TPW = TR / W;            // tokens of a tile per consumer warp
  constexpr int R = TPW / 4;             // QK rows (4 tokens each) per warp and tile
  constexpr int V = G * R;               // partial dots per lane and tile
  constexpr int C = join_out<V>();       // dots per lane after the join
  constexpr int NQ = D / 4;              // PV channel quads
  constexpr int LPQ = 32 / NQ;           // PV lane groups per warp (1 at D=128, 2 at D=64)
  constexpr int PVN = TPW / LPQ;         // tokens per PV lane and tile
  constexpr int NBOX = D / 64;
  constexpr int NOUT = (G * D + kConsumerThreads - 1) / kConsumerThreads;
  static_assert(TPW % 4 == 0 && R >= 1, "a warp takes whole rows of 4 tokens");
  static_assert(C <= R && R % C == 0, "after the join a lane holds rows of one head");

  extern __shared__ __align__(16) uint8_t smem_raw[];
  // 1024-byte aligned base, kept as an offset into the shared array
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  float2* ps = reinterpret_cast<float2*>(smem + L::oPs);   // [tile 0/1][token][head] (p, p)
  float* ow = reinterpret_cast<float*>(smem + L::oOw);     // [warp][head][D]
  float2* mlw = reinterpret_cast<float2*>(smem + L::oMl);  // [warp][head] (m, l)
  int* off = reinterpret_cast<int*>(smem + L::oOff);
  int* cst = reinterpret_cast<int*>(smem + L::oCst);
  int* info = reinterpret_cast<int*>(smem + L::oInfo);     // valid tokens of the stage's tile
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::oFull);
  uint64_t* empty = reinterpret_cast<uint64_t*>(smem + L::oEmpty);
  // [0..15] scan, [18] abort, [24..27] zeros
  int* misc = reinterpret_cast<int*>(smem + L::oMisc);
  volatile int* abort_flag = misc + 18;
  const uint8_t* zero16 = reinterpret_cast<const uint8_t*>(misc + 24);  // 16 zero bytes

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int P = p.batch * p.num_kv_heads;
  const int tpp = p.tiles_per_page;
  const int NC = gridDim.x, cta = blockIdx.x;
  const uint64_t lim = p.wait_limit;

  // The next kernel may start as soon as SMs free up; without the prologue
  // overlap, this grid reads nothing before the previous kernel completes.
  pdl_launch_dependents();
  if (!p.overlap_prologue) pdl_wait_prior_grid();

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], W);
    }
    misc[18] = 0;
    misc[24] = misc[25] = misc[26] = misc[27] = 0;
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
      const int t = __shfl_up_sync(kFull, incl, o);
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
  const int U = off[P];
  for (int c = tid; c <= NC; c += kThreads) cst[c] = range_start(U, c, NC);
  const int u0 = range_start(U, cta, NC), u1 = range_start(U, cta + 1, NC);
  const int ntiles = u1 - u0;

  __syncthreads();  // range table, barrier init and plan visible to every warp

  // =========================== producer warp ===============================
  if (warp == W) {
    // descriptor of tile u: (pair, first row in the [pool rows][D] view, valid tokens)
    // valid is packed with the first token the tile attends (lo, recent pages)
    // and 1 + the row of the appended token (0: none): valid | lo << 8 | (row + 1) << 16
    auto lookup = [&](int u, int& pair, int& row, int& valid) {
      pair = pair_of(off, u, P);
      const int local = u - off[pair];
      const int li = local / tpp, sub = local - li * tpp;
      const int b = pair / p.num_kv_heads, h = pair - b * p.num_kv_heads;
      const int n = p.ctx_lens[b];
      const int NP = p.physical_page;
      const int npages = (n + NP - 1) / NP;
      int m, lo = 0;
      if (p.head_kind[h] == 0) {
        const int nsel = sel_pages(p, pair, npages);
        if (li < nsel) {
          m = p.sel[(size_t)pair * p.top_k + li];
        } else {  // the (li - nsel)-th recent page the selection does not hold
          m = -1;
          int ra, rz, rf;
          if (recent_range(p, b, n, ra, rz, rf)) {
            const int32_t* s = p.sel + (size_t)pair * p.top_k;
            const int j = recent_page(s, sel_tail_start(s, nsel, ra), nsel, ra, li - nsel);
            if (j <= rz) {
              m = j;
              lo = max(0, rf - m * NP);
            }
          }
        }
      } else {
        const int ns = min((p.sink + NP - 1) / NP, npages);
        const int ls = max(max(0, n - p.local) / NP, ns);
        m = li < ns ? li : ls + (li - ns);
      }
      int pid = -1;
      if (m >= 0 && m < npages && m < p.max_pages) pid = p.block_table[(size_t)b * p.max_pages + m];
      if (pid < 0 || pid >= p.num_pool_pages) {  // bad selection or block-table entry: skip the page
        raise_status(p.status, LSERVE_ERR_BOUNDS);
        row = 0;
        valid = 0;
        return;
      }
      row = (int)(((long long)pid * p.num_kv_heads + h) * NP + sub * TR);
      valid = max(0, min(TR, n - m * NP - sub * TR));
      const int lo_t = min(valid, max(0, lo - sub * TR));
      const int ta = p.k_new ? n - 1 - (m * NP + sub * TR) : -1;  // the appended token's row
      const int fix = (ta >= lo_t && ta < valid) ? ta : -1;
      valid |= (lo_t << 8) | ((fix + 1) << 16);
    };
    int issued = 0;
    bool alive = true;
    const uint64_t pol = l2_policy_evict_first();  // KV tiles: read once
    // the stage's tile (and for the quantized cache its page's scales): expect
    // every byte of the stage, then the copies that read no output of the
    // previous kernel
    auto issue_kv = [&](int s, int pr, int row, int val) {
      uint8_t* st = smem + s * L::kStage;
      if constexpr (Q8) {
        const size_t ph = (size_t)row / p.physical_page;  // pool page * H_kv + head
        mbar_arrive_expect_tx(&full[s], 2 * L::kTileK + 2 * 4 * L::kScaleSeg + L::kStageQ);
        // rows swizzled by their width (tensor maps of the code pools)
        tma_load_2d_hint(st, &kmap, 0, row, &full[s], pol);
        tma_load_2d_hint(st + L::kTileK, &vmap, 0, row, &full[s], pol);
#pragma unroll
        for (int sg = 0; sg < 4; ++sg) {
          bulk_load_1d(st + L::oScale + sg * L::kScaleSegP, p.k_scale + ph * D + sg * (D / 4),
                       L::kScaleSeg, &full[s]);
          bulk_load_1d(st + L::oScale + (4 + sg) * L::kScaleSegP, p.v_scale + ph * D + sg * (D / 4),
                       L::kScaleSeg, &full[s]);
        }
      } else {
        const bool has_new = (val >> 16) != 0;  // the tile holds the appended token
        mbar_arrive_expect_tx(&full[s], 2 * TR * D * 2 + L::kStageQ + (has_new ? L::kNew : 0));
        // one contiguous TR x D tile each: 3-D view (64 channels, D/64 halves, rows)
        tma_load_3d_hint(st, &kmap, 0, 0, row, &full[s], pol);
        tma_load_3d_hint(st + L::kTileK, &vmap, 0, 0, row, &full[s], pol);
      }
    };
    // the copies of what the previous kernel may write: q, the appended rows
    auto issue_rest = [&](int s, int pr, int val) {
      uint8_t* st = smem + s * L::kStage;
      const int b = pr / p.num_kv_heads, h = pr - b * p.num_kv_heads;
      if constexpr (!Q8) {
        if ((val >> 16) != 0) {  // its K / V rows from k_new / v_new, next to the tile
          const size_t src = ((size_t)b * p.num_kv_heads + h) * D;
          bulk_load_1d(st + L::oNew, p.k_new + src, D * 2, &full[s]);
          bulk_load_1d(st + L::oNew + D * 2, p.v_new + src, D * 2, &full[s]);
        }
      }
      bulk_load_1d(st + L::oQ, p.q + ((size_t)b * p.num_q_heads + (size_t)h * G) * D, L::kStageQ,
                   &full[s]);
    };
    for (int kb = 0; kb < ntiles && alive; kb += 32) {
      int tp = 0, trow = 0, tval = 0;
      if (kb + lane < ntiles) lookup(u0 + kb + lane, tp, trow, tval);
      const int nb = min(32, ntiles - kb);
      int j0 = 0;
      if (kb == 0) {
        // With LSERVE_DECODE_PREFETCH_KV the first stages' KV copies go out
        // before the previous kernel completes (it writes no page this call
        // reads); q and the appended rows may be its outputs and wait for it.
        const int kpre = p.prefetch_kv ? min(S, nb) : 0;
        for (int j = 0; j < kpre; ++j) {
          const int pr = __shfl_sync(kFull, tp, j), row = __shfl_sync(kFull, trow, j);
          const int val = __shfl_sync(kFull, tval, j);
          if (lane == 0) {
            info[j] = val;
            issue_kv(j, pr, row, val);
          }
        }
        pdl_wait_prior_grid();
        for (int j = 0; j < kpre; ++j) {
          const int pr = __shfl_sync(kFull, tp, j), val = __shfl_sync(kFull, tval, j);
          if (lane == 0) issue_rest(j, pr, val);
        }
        j0 = kpre;
        issued = kpre;
      }
      for (int j = j0; j < nb; ++j) {
        const int k = kb + j, s = k % S;
        const int pr = __shfl_sync(kFull, tp, j);
        const int row = __shfl_sync(kFull, trow, j);
        const int val = __shfl_sync(kFull, tval, j);
        int ok = 1;
        if (lane == 0) {
          if (k >= S) ok = stage_wait(&empty[s], ((k / S) - 1) & 1, lim, p.status, abort_flag);
          if (ok && !*abort_flag) {
            fence_proxy_async_smem();  // the consumers' reads of the stage come first
            info[s] = val;
            issue_kv(s, pr, row, val);
            issue_rest(s, pr, val);
          } else {
            ok = 0;
          }
        }
        if (!__shfl_sync(kFull, ok, 0)) {
          alive = false;
          break;
        }
        ++issued;
      }
    }
    // after a timeout: let the copies still in flight land before the CTA exits
    if (!alive && lane == 0)
      for (int k = max(0, issued - S); k < issued; ++k) mbar_wait(&full[k % S], (k / S) & 1, lim, p.status);
    // The appended tokens' rows go to the pools and statistics (pairs dealt
    // round-robin over the CTAs).  This launch reads those rows from k_new /
    // v_new instead, so its own TMA copies of them may see either content.
    if (p.k_new) {
      if (ntiles == 0) pdl_wait_prior_grid();  // the pools may be in use by the kernel before
      for (int pr = cta; pr < P; pr += NC) append_rows<D>(p, pr, lane);
    }
    return;
  }

  // =========================== consumer warps ==============================
  pdl_wait_prior_grid();  // no global write before the previous kernel completes
  // Split pairs at the ends of this CTA's range: the first pair, if it began
  // in an earlier CTA, gets a partial written to this CTA's slot; the last
  // pair, if it begins here and goes on into later CTAs, is merged here.
  const int first_pair = ntiles > 0 ? pair_of(off, u0, P) : -1;
  const int last_pair = ntiles > 0 ? pair_of(off, u1 - 1, P) : -1;
  const int merge_pair =
      (last_pair >= 0 && off[last_pair] >= u0 && off[last_pair + 1] > u1) ? last_pair : -1;
  const uint32_t e_first = (first_pair >= 0 && off[first_pair] < u0) ? __ldcg(p.epochs + first_pair) : 0u;
  const uint32_t e_merge = merge_pair >= 0 ? __ldcg(p.epochs + merge_pair) : 0u;
  // pairs with nothing to attend (n = 0): zero output, lse = -inf
  if (cta == 0) {
    for (int pr = tid; pr < P; pr += kConsumerThreads) {
      if (off[pr + 1] != off[pr]) continue;
      const int b = pr / p.num_kv_heads, h = pr - b * p.num_kv_heads;
      for (int g = 0; g < G; ++g) {
        const size_t qh = (size_t)b * p.num_q_heads + (size_t)h * G + g;
        for (int c = 0; c < D; ++c) store_out(p, qh * D + c, 0.f);
        if (p.lse) p.lse[qh] = -INFINITY;
      }
    }
  }
  const int tok_l = lane / LPT, qtr = lane % LPT;  // QK: (token of the row, eighth of D)
  const int jb = join_base(V, qtr);
  const int my_g = jb / R, my_r0 = jb % R;         // head and first row of the joined dots
  const int quad = lane % NQ, half = lane / NQ;    // PV: channel quad (+ token half at D=64)
  const int wt0 = warp * TPW;                      // first token of this warp in a tile
  const int pv_t0 = wt0 + half * PVN;
  // byte offsets inside a stage, fixed for the lane (a token row is NBOX
  // consecutive 128-byte swizzle rows)
  uint32_t koff[R][KCH];
  uint32_t voff[PVN];
  if constexpr (!Q8) {
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int ch = 0; ch < KCH; ++ch) {
        const int c = qtr * KCH + ch;  // 16-byte chunk of the key row
        koff[r][ch] = sw128_offset(NBOX * (wt0 + 4 * r + tok_l) + c / 8, c % 8);
      }
    const int chunk = (4 * quad) / 8;
#pragma unroll
    for (int j = 0; j < PVN; ++j)
      voff[j] = L::kTileK + (quad & 1) * 8 + sw128_offset(NBOX * (pv_t0 + j) + chunk / 8, chunk % 8);
  }

  float2 qreg[HB][CPT / 2];
  float m_run = -INFINITY, l_run = 0.f;  // this lane's head: running max, partial row sum
  float2 o_acc[G][2];
#pragma unroll
  for (int g = 0; g < G; ++g) o_acc[g][0] = o_acc[g][1] = make_float2(0.f, 0.f);

  // ---- tensor-core consumer (bf16 cache, G >= 4).  Each warp owns 8 tokens of every
  // tile.  S = q K^T is one m16n8k16 row block per tile: the rows are the G
  // query heads of the pair (rows G..15 zero), the 8 columns the warp's
  // tokens, k over D in D/16 steps.  The reduction over channels is order-free,
  // so k-step ks, lane quad position qq takes channels CPL*qq + 4*ks + {0..3}:
  // each lane reads its CPL contiguous channels of q and of its token's key
  // with 16-byte loads (no transpose).  O += P V with P (fp32 softmax weights
  // split into bf16 hi + lo parts, so the product keeps ~16 bits) as the A
  // operand straight from the S accumulator layout and V^T fragments by
  // ldmatrix.trans; O (rows = heads, 8 channels per n-tile) stays in
  // registers across the pair's tiles.
  constexpr bool kMma = !Q8 && G >= 4;  // G < 4: most MMA rows would be padding
  constexpr bool kQmma = Q8;             // the quantized cache: tensor cores for every G
  constexpr int KS = D / 16;   // QK k-steps
  constexpr int CPL = D / 4;   // channels per lane in the QK operands
  constexpr int NTl = D / 8;   // PV n-tiles (8 channels each)
  const int hr = lane >> 2, qq = lane & 3;  // fragment row (head) and quad position
  const bool real_row = hr < G;
  const int mt0 = warp * 8;                  // the warp's 8 tokens of a tile
  const bool has_tok = mt0 < TR;             // 32-token tiles: warps 4..7 hold none
  uint32_t kof[CPL / 8];                     // this lane's key chunks (token mt0 + hr)
  uint32_t vof[NTl / 4];                     // ldmatrix row addresses of V, per 4 n-tiles
#pragma unroll
  for (int i = 0; i < CPL / 8; ++i) {
    const int c = (CPL * qq) / 8 + i;
    kof[i] = sw128_offset(NBOX * (mt0 + hr) + c / 8, c % 8);
  }
#pragma unroll
  for (int j = 0; j < NTl / 4; ++j) {
    const int c = 4 * j + (lane >> 3);
    vof[j] = L::kTileK + sw128_offset(NBOX * (mt0 + (lane & 7)) + c / 8, c % 8);
  }
  uint32_t qa[KS][2];   // A fragments of q: (a0, a2) per k-step
  float om[NTl][4];     // O fragments (only [0], [1] are real rows)
#pragma unroll
  for (int n = 0; n < NTl; ++n) om[n][0] = om[n][1] = om[n][2] = om[n][3] = 0.f;
  const uint32_t smem_base = smem_u32(smem);

  auto load_q_mma = [&](const uint8_t* st) {
#pragma unroll
    for (int i = 0; i < CPL / 8; ++i) {
      uint4 w = make_uint4(0u, 0u, 0u, 0u);
      if (real_row) w = reinterpret_cast<const uint4*>(st + L::oQ + (hr * D + CPL * qq) * 2)[i];
      qa[2 * i][0] = w.x;
      qa[2 * i][1] = w.y;
      qa[2 * i + 1][0] = w.z;
      qa[2 * i + 1][1] = w.w;
    }
  };
  // S of the warp's 8 tokens of tile st (two accumulators: even / odd k-steps)
  auto qk_mma = [&](const uint8_t* st, float (&sa)[4], float (&sb)[4]) {
    uint32_t kw[CPL / 2];
#pragma unroll
    for (int i = 0; i < CPL / 8; ++i) {
      const uint4 w = *reinterpret_cast<const uint4*>(st + kof[i]);
      kw[4 * i] = w.x;
      kw[4 * i + 1] = w.y;
      kw[4 * i + 2] = w.z;
      kw[4 * i + 3] = w.w;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) sa[i] = sb[i] = 0.f;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      if (ks & 1) mma_16816(sb, qa[ks][0], qa[ks][1], kw[2 * ks], kw[2 * ks + 1]);
      else mma_16816(sa, qa[ks][0], qa[ks][1], kw[2 * ks], kw[2 * ks + 1]);
    }
  };
  // bf16 halves of V rows mt0 + 2*qq + {0,1} that lie past `valid` -> 0 (the
  // cache may hold anything there; p is 0 for them but 0 * NaN is not)
  auto vmask = [&](int valid) -> uint32_t {
    const int t = mt0 + 2 * qq;
    return (t < valid ? 0x0000FFFFu : 0u) | (t + 1 < valid ? 0xFFFF0000u : 0u);
  };
  // O += P V over the warp's tokens of one or two tiles
  auto pv_mma = [&](int s0, int s1, int nt, const float (&pr)[2][2], int valid0, int valid1) {
    uint32_t ah[2], al[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      ah[i] = float2_to_bf16x2(pr[i][0], pr[i][1]);
      al[i] = float2_to_bf16x2(pr[i][0] - bf16_lo(ah[i]), pr[i][1] - bf16_hi(ah[i]));
    }
    const bool part0 = mt0 + 8 > valid0, part1 = nt == 2 && mt0 + 8 > valid1;  // warp-uniform
    const uint32_t mk0 = vmask(valid0), mk1 = vmask(valid1);
    const uint32_t b0 = smem_base + s0 * L::kStage, b1 = smem_base + s1 * L::kStage;
#pragma unroll
    for (int j = 0; j < NTl / 4; ++j) {
      uint32_t v0[4];
      ldsm_x4_trans(v0, b0 + vof[j]);
      if (part0) {
#pragma unroll
        for (int r = 0; r < 4; ++r) v0[r] &= mk0;
      }
      if (nt == 2) {
        uint32_t v1[4];
        ldsm_x4_trans(v1, b1 + vof[j]);
        if (part1) {
#pragma unroll
          for (int r = 0; r < 4; ++r) v1[r] &= mk1;
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          mma_16816(om[4 * j + r], ah[0], ah[1], v0[r], v1[r]);
          mma_16816(om[4 * j + r], al[0], al[1], v0[r], v1[r]);
        }
      } else {
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          mma_1688(om[4 * j + r], ah[0], v0[r]);
          mma_1688(om[4 * j + r], al[0], v0[r]);
        }
      }
    }
  };

  // ---- tensor-core consumer of the quantized cache (QB = 8 or 4, every G).
  // The fragments are those above, in fp16: a lane's QK operand is its
  // token's run of CPL channels, whose codes convert to fp16 exactly; the
  // page's K channel scales go into q instead (q' = q * k_scale, rounded once
  // to fp16, per tile), so S = q' . code.  For PV the lane forms its token's
  // V' = code * v_scale (fp16) and movmatrix transposes each 8 x 8 block into
  // the B fragment.  Pair p of a lane's run holds channels pair_channel(QB, p,
  // 0 / 1); n-tile p of O therefore holds, in fragment columns 2*qq + e,
  // channel CPL*qq + pair_channel(QB, p, e).
  constexpr int QBB = QB ? QB : 8;
  constexpr int CB = CPL * QBB / 8;          // code bytes of a lane's run
  constexpr int NP2 = CPL / 2;               // pairs of a lane's run
  uint32_t qbf[CPL / 2];                     // q of head hr (bf16 pairs, natural order); 0 on padding rows
  // Byte `o` of code row t of a tile: the tensor map swizzles 16-byte chunks by
  // the row width (128-, 64- or 32-byte mode): chunk ^= (t * kRow / 128) & M.
  auto code_at = [&](const uint8_t* tile, int t, int o) -> const uint8_t* {
    constexpr int M = L::kRow == 128 ? 7 : (L::kRow == 64 ? 3 : 1);
    const int sw = ((t * L::kRow) >> 7) & M;
    return tile + t * L::kRow + ((((o >> 4) ^ sw)) << 4) + (o & 15);
  };
  // this lane's run of codes of token row t of the tile at `tile`, as fp16 pairs
  auto run_codes = [&](const uint8_t* tile, int t, uint32_t (&pr)[NP2]) {
    uint32_t w[CB / 4];
#pragma unroll
    for (int i = 0; i < CB / 16; ++i) {
      const uint4 v = *reinterpret_cast<const uint4*>(code_at(tile, t, CB * qq + 16 * i));
      w[4 * i] = v.x;
      w[4 * i + 1] = v.y;
      w[4 * i + 2] = v.z;
      w[4 * i + 3] = v.w;
    }
    if constexpr (CB % 16 == 8) {
      const uint2 v = *reinterpret_cast<const uint2*>(code_at(tile, t, CB * qq + CB - 8));
      w[CB / 4 - 2] = v.x;
      w[CB / 4 - 1] = v.y;
    }
#pragma unroll
    for (int m = 0; m < CB / 4; ++m) {
      if constexpr (QB == 8) {
        codes8_to_f16(w[m], pr[2 * m], pr[2 * m + 1]);
      } else {
        const uint32_t u = w[m] ^ 0x88888888u;
#pragma unroll
        for (int j = 0; j < 4; ++j) pr[4 * m + j] = codes4_pair(u, j);
      }
    }
  };
  // f(pair, scale of its channel 0, scale of its channel 1) for every pair of
  // this lane's run, the page's K (which = 0) or V (1) channel scales read 8
  // channels at a time
  auto for_scale_pairs = [&](const uint8_t* st, int which, auto&& f) {
    const float4* sp = reinterpret_cast<const float4*>(st + L::oScale + (4 * which + qq) * L::kScaleSegP);
#pragma unroll
    for (int m = 0; m < CPL / 8; ++m) {
      const float4 a = sp[2 * m], b = sp[2 * m + 1];
      const float c[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int pp = 4 * m + j;
        f(pp, c[pair_channel(QBB, pp, 0) - 8 * m], c[pair_channel(QBB, pp, 1) - 8 * m]);
      }
    }
  };
  auto q_chan = [&](int c) -> float {  // q of head hr, channel CPL*qq + c
    return (c & 1) ? bf16_hi(qbf[c / 2]) : bf16_lo(qbf[c / 2]);
  };
  auto load_q_qmma = [&](const uint8_t* st) {
#pragma unroll
    for (int i = 0; i < CPL / 8; ++i) {
      uint4 w = make_uint4(0u, 0u, 0u, 0u);
      if (real_row) w = reinterpret_cast<const uint4*>(st + L::oQ + (hr * D + CPL * qq) * 2)[i];
      qbf[4 * i] = w.x;
      qbf[4 * i + 1] = w.y;
      qbf[4 * i + 2] = w.z;
      qbf[4 * i + 3] = w.w;
    }
  };
  // S of the warp's 8 tokens of tile st over the quantized keys
  auto qk_qmma = [&](const uint8_t* st, float (&sa)[4], float (&sb)[4]) {
    uint32_t qf[NP2];
    for_scale_pairs(st, 0, [&](int pp, float s0, float s1) {
      qf[pp] = f32x2_to_f16x2(q_chan(pair_channel(QBB, pp, 0)) * s0, q_chan(pair_channel(QBB, pp, 1)) * s1);
    });
    uint32_t kc[NP2];
    run_codes(st, mt0 + hr, kc);
#pragma unroll
    for (int i = 0; i < 4; ++i) sa[i] = sb[i] = 0.f;
#pragma unroll
    for (int k2 = 0; k2 < KS; ++k2) {
      if (k2 & 1) mma_16816_f16(sb, qf[2 * k2], qf[2 * k2 + 1], kc[2 * k2], kc[2 * k2 + 1]);
      else mma_16816_f16(sa, qf[2 * k2], qf[2 * k2 + 1], kc[2 * k2], kc[2 * k2 + 1]);
    }
  };
  // V' = code * v_scale of the warp's token mt0 + hr of tile st, transposed into
  // the B fragments of the NP2 n-tiles
  auto v_frags = [&](const uint8_t* st, uint32_t (&vb)[NP2]) {
    uint32_t vc[NP2];
    run_codes(st + L::kTileK, mt0 + hr, vc);
    for_scale_pairs(st, 1, [&](int pp, float s0, float s1) {
      vb[pp] = movmatrix_t(hmul2(vc[pp], f32x2_to_f16x2(s0, s1)));
    });
  };
  auto pv_qmma = [&](const uint8_t* st0, const uint8_t* st1, int nt, const float (&pr)[2][2]) {
    uint32_t ah[2], al[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      ah[i] = f32x2_to_f16x2(pr[i][0], pr[i][1]);
      al[i] = f32x2_to_f16x2(pr[i][0] - f16_lo(ah[i]), pr[i][1] - f16_hi(ah[i]));
    }
    uint32_t v0[NP2];
    v_frags(st0, v0);
    if (nt == 2) {
      uint32_t v1[NP2];
      v_frags(st1, v1);
#pragma unroll
      for (int n = 0; n < NP2; ++n) {
        mma_16816_f16(om[n], ah[0], ah[1], v0[n], v1[n]);
        mma_16816_f16(om[n], al[0], al[1], v0[n], v1[n]);
      }
    } else {
#pragma unroll
      for (int n = 0; n < NP2; ++n) {
        mma_1688_f16(om[n], ah[0], v0[n]);
        mma_1688_f16(om[n], al[0], v0[n]);
      }
    }
  };

  auto load_q = [&](const uint8_t* st, int hb) {  // bf16 q of the stage -> this lane's eighth
#pragma unroll
    for (int h = 0; h < HB; ++h) {
      const uint4* src = reinterpret_cast<const uint4*>(st + L::oQ + ((hb * HB + h) * D + qtr * CPT) * 2);
#pragma unroll
      for (int i = 0; i < KCH; ++i) {
        const uint4 w = src[i];
        qreg[h][4 * i + 0] = bf16x2_to_float2(w.x);
        qreg[h][4 * i + 1] = bf16x2_to_float2(w.y);
        qreg[h][4 * i + 2] = bf16x2_to_float2(w.z);
        qreg[h][4 * i + 3] = bf16x2_to_float2(w.w);
      }
    }
  };

  // partial dots of tile st for the rows of this lane: d[g * R + r] (bf16 cache)
  auto qk_tile = [&](const uint8_t* st, float (&d)[V], int hb) {
    {
#pragma unroll
      for (int r = 0; r < R; ++r) {
        float2 acc[HB];
#pragma unroll
        for (int h = 0; h < HB; ++h) acc[h] = make_float2(0.f, 0.f);
#pragma unroll
        for (int ch = 0; ch < KCH; ++ch) {
          const uint4 kw = *reinterpret_cast<const uint4*>(st + koff[r][ch]);
          const float2 k0 = bf16x2_to_float2(kw.x), k1 = bf16x2_to_float2(kw.y);
          const float2 k2 = bf16x2_to_float2(kw.z), k3 = bf16x2_to_float2(kw.w);
#pragma unroll
          for (int h = 0; h < HB; ++h) {
            acc[h] = __ffma2_rn(qreg[h][4 * ch + 0], k0, acc[h]);
            acc[h] = __ffma2_rn(qreg[h][4 * ch + 1], k1, acc[h]);
            acc[h] = __ffma2_rn(qreg[h][4 * ch + 2], k2, acc[h]);
            acc[h] = __ffma2_rn(qreg[h][4 * ch + 3], k3, acc[h]);
          }
        }
#pragma unroll
        for (int h = 0; h < HB; ++h) d[(hb * HB + h) * R + r] = acc[h].x + acc[h].y;
      }
    }
  };

  // o += p v over this lane's tokens of tile st (tokens past `valid` read zeros)
  auto pv_tile = [&](const uint8_t* st, int i, int valid) {
#pragma unroll
    for (int j = 0; j < PVN; ++j) {
      const int t = pv_t0 + j;
      const uint8_t* vp = t < valid ? st + voff[j] : zero16;
      const uint2 vw = *reinterpret_cast<const uint2*>(vp);
      const float2 v01 = bf16x2_to_float2(vw.x), v23 = bf16x2_to_float2(vw.y);
      const float2* pt = ps + (i * TR + t) * G;
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
  };

  // End of a pair segment (every consumer warp arrives here at the same tile):
  // merge the warps, then finalise the pair, or publish this CTA's partial, or
  // (the pair's merging CTA) fold in the other CTAs' partials and finalise.
  // fin: the flush after the loop (the only one that can merge other CTAs' partials)
  auto flush = [&](int pair, auto fin) {
  constexpr bool kFinal = decltype(fin)::value;
    if constexpr (kMma || kQmma) {
      float lw = l_run;  // row sum of head hr over the warp's tokens: the row's 4 lanes
      lw += __shfl_xor_sync(kFull, lw, 1);
      lw += __shfl_xor_sync(kFull, lw, 2);
      if (real_row) {
        if (qq == 0) mlw[warp * G + hr] = make_float2(m_run, lw);
        float* orow = ow + (warp * G + hr) * D;
#pragma unroll
        for (int n = 0; n < NTl; ++n) {
          if constexpr (kQmma) {  // n-tile n = pair n of the lanes' runs
            orow[CPL * qq + pair_channel(QBB, n, 0)] = om[n][0];
            orow[CPL * qq + pair_channel(QBB, n, 1)] = om[n][1];
          } else {
            *reinterpret_cast<float2*>(orow + 8 * n + 2 * qq) = make_float2(om[n][0], om[n][1]);
          }
        }
      }
    } else {
    float lw = l_run;  // row sum of this lane's head over the warp's tokens
    if constexpr (row_bit(V, R, 4)) lw += __shfl_xor_sync(kFull, lw, 4);
    if constexpr (row_bit(V, R, 2)) lw += __shfl_xor_sync(kFull, lw, 2);
    if constexpr (row_bit(V, R, 1)) lw += __shfl_xor_sync(kFull, lw, 1);
    lw += __shfl_xor_sync(kFull, lw, 8);
    lw += __shfl_xor_sync(kFull, lw, 16);
    if constexpr (LPQ == 2) {
#pragma unroll
      for (int g = 0; g < G; ++g)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          o_acc[g][j].x += __shfl_xor_sync(kFull, o_acc[g][j].x, 16);
          o_acc[g][j].y += __shfl_xor_sync(kFull, o_acc[g][j].y, 16);
        }
    }
#pragma unroll
    for (int g = 0; g < G; ++g)
      if (lane == head_src(V, R, g)) mlw[warp * G + g] = make_float2(m_run, lw);
    if (lane < NQ) {
#pragma unroll
      for (int g = 0; g < G; ++g)
        *reinterpret_cast<float4*>(ow + (warp * G + g) * D + 4 * quad) =
            make_float4(o_acc[g][0].x, o_acc[g][0].y, o_acc[g][1].x, o_acc[g][1].y);
    }
    }
    const int b = pair / p.num_kv_heads, h = pair - b * p.num_kv_heads;
    // only the first and the last pair of a CTA's range can reach into other CTAs
    const bool whole = off[pair] >= u0 && off[pair + 1] <= u1;
    // the merged pair is the last of the range: only the flush after the loop merges
    const bool merger = kFinal && !whole && pair == merge_pair;
    const uint32_t tag = part_tag((merger ? e_merge : e_first) + 1u, pair);
    // Partial of a CTA (its workspace slot): o words [G][D], then (m, l) word
    // pairs [G][2].  A thread's NOUT outputs are the consecutive channels
    // c0 .. c0 + NOUT - 1 of one head g (NOUT <= 2: one 16-byte access).
    constexpr int kSlot = G * D + 2 * G;
    const int j0 = tid * NOUT;
    const bool has_out = j0 < G * D;
    const int g = (has_out ? j0 : 0) / D, c0 = (has_out ? j0 : 0) - g * D;
    const bool live = named_sync_and(kBarConsumers, kConsumerThreads, !*abort_flag);
    // this CTA's own (o, m, l) of the thread's outputs: the warps' states
    // weighted by 2^(m_w - max over warps)
    float o_[NOUT], M = -INFINITY, l = 0.f;
#pragma unroll
    for (int w = 0; w < W; ++w) M = fmaxf(M, mlw[w * G + g].x);
#pragma unroll
    for (int i = 0; i < NOUT; ++i) o_[i] = 0.f;
#pragma unroll
    for (int w = 0; w < W; ++w) {
      const float2 ml = mlw[w * G + g];
      const float wt = ml.x == -INFINITY ? 0.f : fast_ex2(ml.x - M);
      l += wt * ml.y;
#pragma unroll
      for (int i = 0; i < NOUT; ++i) o_[i] += wt * ow[(w * G + g) * D + c0 + i];
    }
    if (!whole && !merger && live && has_out) {  // a later segment of a split pair: publish
      unsigned long long* sl = p.parts + (size_t)cta * kSlot;
      if constexpr (NOUT == 1) {
        st_word(sl + g * D + c0, o_[0], tag);
      } else {
#pragma unroll
        for (int i = 0; i < NOUT; i += 2) st_word2(sl + g * D + c0 + i, o_[i], o_[i + 1], tag);
      }
      if (c0 == 0) st_word2(sl + G * D + 2 * g, M, l, tag);
    }
    bool got = true;
    if constexpr (kFinal) {
      if (merger && live) {
        // Fold in the partials of CTAs cta+1 .. c_last (those with tiles).
        // First the (m, l) word pairs, one (segment, head) entry per thread
        // (a warp's worth of small loads per poll), each polled until its tag
        // matches and staged in shared memory -- the stage ring, idle now.
        // Then every thread loads its o words, kBatch segments at a time
        // (stale words are loaded again together), and adds them with weights
        // 2^(m_s - M) of the common maximum M.
        const int c_last = cta_of(cst, off[pair + 1] - 1, NC);
        const int nseg = c_last - cta, nml = nseg * G;
        float2* mls = reinterpret_cast<float2*>(smem);  // [segment][head]: (m, l)
        const long long t_poll = clock64();
        for (int i = tid; i < nml; i += kConsumerThreads) {
          const int cc = cta + 1 + i / G, gg = i % G;
          float2 ml = make_float2(-INFINITY, 0.f);
          if (cta_busy(cst, cc)) {
            const unsigned long long* a = p.parts + (size_t)cc * kSlot + G * D + 2 * gg;
            unsigned long long wm, wl;
            while (true) {
              ld_word2(a, wm, wl);
              if (word_ok(wm, tag) && word_ok(wl, tag)) break;
              if ((uint64_t)(clock64() - t_poll) > lim) {
                got = false;
                break;
              }
            }
            ml = make_float2(word_val(wm), word_val(wl));
          }
          mls[i] = ml;
        }
        got = named_sync_and(kBarConsumers, kConsumerThreads, got);
        if (has_out && got) {
          float Mt = M;
          for (int sg = 0; sg < nseg; ++sg) Mt = fmaxf(Mt, mls[sg * G + g].x);
          if (Mt != -INFINITY) {
            const float a = exp2f(M - Mt);
#pragma unroll
            for (int i = 0; i < NOUT; ++i) o_[i] *= a;
            l *= a;
          }
          constexpr int kBatch = 16 / NOUT;  // segments whose o words are in flight at once
          for (int s0 = 0; s0 < nseg && got; s0 += kBatch) {
            unsigned long long wo[kBatch][NOUT];
            bool us[kBatch];
            auto load_o = [&](int u) {
              const unsigned long long* sl = p.parts + (size_t)(cta + 1 + s0 + u) * kSlot + g * D + c0;
              if constexpr (NOUT == 1) {
                wo[u][0] = ld_word(sl);
              } else {
#pragma unroll
                for (int i = 0; i < NOUT; i += 2) ld_word2(sl + i, wo[u][i], wo[u][i + 1]);
              }
            };
            auto seg_ok = [&](int u) {
              bool ok = true;
#pragma unroll
              for (int i = 0; i < NOUT; ++i) ok = ok && word_ok(wo[u][i], tag);
              return ok;
            };
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
              us[u] = s0 + u < nseg && cta_busy(cst, cta + 1 + s0 + u);
              if (us[u]) load_o(u);
            }
            while (true) {
              bool pending = false;
#pragma unroll
              for (int u = 0; u < kBatch; ++u) pending |= us[u] && !seg_ok(u);
              if (!pending) break;
              if ((uint64_t)(clock64() - t_poll) > lim) {
                got = false;
                break;
              }
#pragma unroll
              for (int u = 0; u < kBatch; ++u)
                if (us[u] && !seg_ok(u)) load_o(u);
            }
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
              if (!us[u] || !got) continue;
              const float2 ml = mls[(s0 + u) * G + g];
              if (ml.x == -INFINITY) continue;
              const float wt = exp2f(ml.x - Mt);
#pragma unroll
              for (int i = 0; i < NOUT; ++i) o_[i] += word_val(wo[u][i]) * wt;
              l += ml.y * wt;
            }
          }
          M = Mt;
        }
        if (!got && tid == 0) raise_status(p.status, LSERVE_ERR_TIMEOUT);
      }
    }
    if ((whole || merger) && live && got && has_out) {
      const size_t qh = (size_t)b * p.num_q_heads + (size_t)h * G + g;
      const bool empty_row = !(l > 0.f);
#pragma unroll
      for (int i = 0; i < NOUT; ++i) store_out(p, qh * D + c0 + i, empty_row ? 0.f : o_[i] / l);
      if (c0 == 0 && p.lse)
        p.lse[qh] = empty_row ? -INFINITY : (M + __log2f(l)) * 0.69314718055994530942f;
    }
    named_sync(kBarConsumers, kConsumerThreads);  // ow / mlw / ps free again
  };

  // Each iteration takes one tile, or two consecutive tiles of the same pair:
  // one softmax update per 2 * TPW tokens of the warp.
  int cur = -1, pend = 0;  // current pair, and the local index of its first tile after it
  bool need_q = false;
  for (int k = 0; k < ntiles;) {
    if (k >= pend) {  // first tile of a new pair (same decision in every consumer warp)
      if (cur >= 0) flush(cur, std::false_type{});
      cur = pair_of(off, u0 + k, P);
      pend = off[cur + 1] - u0;
      m_run = -INFINITY;
      l_run = 0.f;
      if constexpr (kMma || kQmma) {
#pragma unroll
        for (int n = 0; n < NTl; ++n) om[n][0] = om[n][1] = 0.f;
      } else {
#pragma unroll
        for (int g = 0; g < G; ++g) o_acc[g][0] = o_acc[g][1] = make_float2(0.f, 0.f);
      }
      need_q = true;
    }
    const int nt = (k + 1 < ntiles && k + 1 < pend) ? 2 : 1;
    const int s0 = k % S, s1 = (k + 1) % S;
    const bool ok0 = __all_sync(kFull, stage_wait(&full[s0], (k / S) & 1, lim, p.status, abort_flag));
    const bool ok1 =
        nt == 2 && __all_sync(kFull, stage_wait(&full[s1], ((k + 1) / S) & 1, lim, p.status, abort_flag));
    const int inf0 = ok0 ? info[s0] : 0, inf1 = ok1 ? info[s1] : 0;
    const int valid0 = inf0 & 0xFF, valid1 = inf1 & 0xFF;        // tokens [lo, valid) attended
    const int lo0 = (inf0 >> 8) & 0xFF, lo1 = (inf1 >> 8) & 0xFF;
    const uint8_t* st0 = smem + s0 * L::kStage;
    const uint8_t* st1 = smem + s1 * L::kStage;
    if constexpr (!Q8) {
      if (p.k_new) {
        // the appended token's K / V row of a tile comes from k_new / v_new (the
        // producer copied them next to the tile): the warp that owns the row
        // overwrites it in the stage (no other warp reads it)
        constexpr int TPO = (kMma ? 8 : TPW);  // tokens of a tile per owning warp
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int fx = ((i == 0 ? inf0 : inf1) >> 16) - 1;
          if (fx >= 0 && fx / TPO == warp && (i == 0 || nt == 2)) {
            uint8_t* st = smem + (i == 0 ? s0 : s1) * L::kStage;
            constexpr int C16 = D / 8;
            if (lane < 2 * C16) {
              const int c = lane % C16;
              const uint4 v = reinterpret_cast<const uint4*>(st + L::oNew)[lane];  // K chunks, then V
              *reinterpret_cast<uint4*>(st + (lane < C16 ? 0 : L::kTileK) +
                                        sw128_offset(NBOX * fx + c / 8, c % 8)) = v;
            }
            __syncwarp();
          }
        }
      }
    }
    if constexpr (kMma || kQmma) {
      if (need_q) {
        if constexpr (kQmma) load_q_qmma(st0);
        else load_q_mma(st0);
      }
      need_q = false;
      if (has_tok) {
        float sa[2][4], sb[2][4];
        if constexpr (kQmma) {
          qk_qmma(st0, sa[0], sb[0]);
          if (nt == 2) qk_qmma(st1, sa[1], sb[1]);
        } else {
          qk_mma(st0, sa[0], sb[0]);
          if (nt == 2) qk_mma(st1, sa[1], sb[1]);
        }
        float x[2][2];
#pragma unroll
        for (int i = 0; i < 2; ++i)
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int tok = mt0 + 2 * qq + j;
            const bool ok = i == 0 ? (tok >= lo0 && tok < valid0)
                                   : (nt == 2 && tok >= lo1 && tok < valid1);
            x[i][j] = ok ? (sa[i][j] + sb[i][j]) * p.scale_log2 : -INFINITY;
          }
        float mx = fmaxf(fmaxf(x[0][0], x[0][1]), fmaxf(x[1][0], x[1][1]));
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));
        const float m_new = fmaxf(m_run, mx);
        const float alpha = m_new == -INFINITY ? 1.f : fast_ex2(m_run - m_new);
        const float m_use = m_new == -INFINITY ? 0.f : m_new;
        m_run = m_new;
        float pr[2][2];
        float lsum = l_run * alpha;
#pragma unroll
        for (int i = 0; i < 2; ++i)
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            pr[i][j] = fast_ex2(x[i][j] - m_use);  // x = -inf gives 0
            lsum += pr[i][j];
          }
        l_run = lsum;
        if (__any_sync(kFull, alpha != 1.f)) {
#pragma unroll
          for (int n = 0; n < NTl; ++n) {
            om[n][0] *= alpha;
            om[n][1] *= alpha;
          }
        }
        if constexpr (kQmma) pv_qmma(st0, st1, nt, pr);
        else pv_mma(s0, s1, nt, pr, valid0, valid1);
      }
    } else {
    if constexpr (NHB == 1) {
      if (need_q) load_q(st0, 0);
    }
    need_q = false;

    // ---- QK: partial dots over this lane's eighth of D, joined over the 8 lanes
    float d0[V], d1[V];
#pragma unroll
    for (int hb = 0; hb < NHB; ++hb) {
      if constexpr (NHB > 1) load_q(st0, hb);
      qk_tile(st0, d0, hb);
      if (nt == 2) qk_tile(st1, d1, hb);
    }
    float x[2][C];
    join_dots<V>(d0, x[0], qtr);
    if (nt == 2) join_dots<V>(d1, x[1], qtr);
#pragma unroll
    for (int j = 0; j < C; ++j) {
      const int tok = wt0 + 4 * (my_r0 + j) + tok_l;
      x[0][j] = (tok >= lo0 && tok < valid0) ? x[0][j] * p.scale_log2 : -INFINITY;
      x[1][j] = (tok >= lo1 && tok < valid1) ? x[1][j] * p.scale_log2 : -INFINITY;
    }

    // ---- online softmax of this lane's head: warp max over its rows and tokens
    float mx = x[0][0];
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int j = 0; j < C; ++j) mx = fmaxf(mx, x[i][j]);
    if constexpr (row_bit(V, R, 4)) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 4));
    if constexpr (row_bit(V, R, 2)) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));
    if constexpr (row_bit(V, R, 1)) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 8));
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 16));
    const float m_new = fmaxf(m_run, mx);
    const float alpha = m_new == -INFINITY ? 1.f : fast_ex2(m_run - m_new);
    const float m_use = m_new == -INFINITY ? 0.f : m_new;
    m_run = m_new;
    float lsum = l_run * alpha;
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int j = 0; j < C; ++j) {
        const float pr = fast_ex2(x[i][j] - m_use);  // x = -inf gives 0
        lsum += pr;
        const int tok = wt0 + 4 * (my_r0 + j) + tok_l;
        if (i == 0 || nt == 2) ps[(i * TR + tok) * G + my_g] = make_float2(pr, pr);
      }
    l_run = lsum;
    __syncwarp();

    // ---- PV: rescale o only when some head's running max grew
    float a[G];
    bool grew = false;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      a[g] = __shfl_sync(kFull, alpha, head_src(V, R, g));
      grew |= a[g] != 1.f;
    }
    if (grew) {  // warp-uniform: a[] was broadcast
#pragma unroll
      for (int g = 0; g < G; ++g) {
        o_acc[g][0] = __fmul2_rn(o_acc[g][0], make_float2(a[g], a[g]));
        o_acc[g][1] = __fmul2_rn(o_acc[g][1], make_float2(a[g], a[g]));
      }
    }
    pv_tile(st0, 0, valid0);
    if (nt == 2) pv_tile(st1, 1, valid1);
    }
    __syncwarp();
    // ---- release the stage(s) to the producer
    if (lane == 0) {
      if (ok0) mbar_arrive(&empty[s0]);
      if (ok1) mbar_arrive(&empty[s1]);
    }
    k += nt;
  }
  if (cur >= 0) flush(cur, std::true_type{});
  // The merged pair's epoch advances whatever happened above (a timeout
  // included), so no word of this call matches a later call's tags.
  if (tid == 0 && merge_pair >= 0) {
    asm volatile("st.relaxed.gpu.global.b32 [%0], %1;" ::"l"(p.epochs + merge_pair), "r"(e_merge + 1u)
                 : "memory");
  }
}

size_t decode_workspace_bytes(int pairs, int grid, int G, int D) {
  const size_t ep = ((size_t)pairs * 4 + 255) / 256 * 256;  // epochs
  return ep + (size_t)grid * (G * D + 2 * G) * 8;             // one tagged partial per CTA
}

int decode_grid(int sm_count) { return sm_count; }

int decode_consumer_warps() { return 8; }

int decode_tile_rows(int physical_page) {
  return physical_page < kDecodeTileMax ? physical_page : kDecodeTileMax;
}

namespace {
// launched as a programmatic dependent of the previous work on the stream
template <int D, int G, int QB, int TR, int W>
cudaError_t launch_decode_w(const DecodeParams& p, const CUtensorMap& kmap, const CUtensorMap& vmap,
                            int grid, cudaStream_t stream) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3((W + 1) * 32);
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cfg.dynamicSmemBytes = DecLayout<D, G, QB, TR, W>::kBytes + 1024;
  auto kern = decode_attn_kernel<D, G, TR, QB, W>;
  const cudaError_t e = set_smem_once((const void*)kern, (int)cfg.dynamicSmemBytes);
  if (e != cudaSuccess) return e;
  return cudaLaunchKernelEx(&cfg, kern, p, kmap, vmap);
}

template <int D, int G, int QB>
cudaError_t launch_decode_t(const DecodeParams& p, const CUtensorMap& kmap, const CUtensorMap& vmap,
                            int grid, cudaStream_t stream) {
  if (p.consumer_warps != 8) return cudaErrorInvalidValue;
  if (p.tile_rows == 64) return launch_decode_w<D, G, QB, 64, 8>(p, kmap, vmap, grid, stream);
  return launch_decode_w<D, G, QB, 32, 8>(p, kmap, vmap, grid, stream);
}

template <int QB>
cudaError_t launch_decode_any(const DecodeParams& p, const CUtensorMap& kmap, const CUtensorMap& vmap,
                              int D, int G, int grid, cudaStream_t stream) {
  if (grid < 1 || grid > kMaxGrid) return cudaErrorInvalidValue;
  if (p.tile_rows != 64 && p.tile_rows != 32) return cudaErrorInvalidValue;
#define LSERVE_DECODE_CASE(DD, GG) \
  if (D == DD && G == GG) return launch_decode_t<DD, GG, QB>(p, kmap, vmap, grid, stream);
  LSERVE_DECODE_CASE(64, 1)
  LSERVE_DECODE_CASE(64, 2)
  LSERVE_DECODE_CASE(64, 4)
  LSERVE_DECODE_CASE(64, 8)
  LSERVE_DECODE_CASE(128, 1)
  LSERVE_DECODE_CASE(128, 2)
  LSERVE_DECODE_CASE(128, 4)
  LSERVE_DECODE_CASE(128, 8)
#undef LSERVE_DECODE_CASE
  return cudaErrorInvalidValue;
}
}  // namespace

cudaError_t launch_decode(const DecodeParams& p, const CUtensorMap& kmap, const CUtensorMap& vmap,
                          int D, int G, int grid, cudaStream_t stream) {
  return launch_decode_any<0>(p, kmap, vmap, D, G, grid, stream);
}

cudaError_t launch_decode_quant(const DecodeParams& p, const CUtensorMap& kmap,
                                const CUtensorMap& vmap, int D, int G, int bits, int grid,
                                cudaStream_t stream) {
  if (bits == 8) return launch_decode_any<8>(p, kmap, vmap, D, G, grid, stream);
  if (bits == 4) return launch_decode_any<4>(p, kmap, vmap, D, G, grid, stream);
  return cudaErrorInvalidValue;
}

}  // namespace lserve
