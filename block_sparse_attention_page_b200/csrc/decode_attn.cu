// lserve_sparse_decode_attn kernels (LServe explainer, 統一ブロックスパースアテンション
// figure: retrieval heads attend the top-K physical pages, streaming heads the
// Lambda-shaped sink + local pages; 技術的詳細 › 静的スパーシティ).
//
// Work split ("stream-K" over pages): for every (sequence b, KV head h) pair
// the pages it attends are cut into tiles of 32 tokens; the tiles of all
// pairs are laid end to end and the whole list is cut into equal contiguous
// ranges, one per consumer warp of a persistent grid (one CTA per SM).  Every
// warp therefore streams the same number of KV bytes no matter how unequal the
// pairs are (64 selected pages next to ~10 sink+local pages).
//
// Per warp: a ring of kDecodeStages (K tile, V tile) buffers filled by TMA
// (lane 0 issues cp.async.bulk.tensor, 128-byte swizzle so that lane t reading
// row t and lane c reading channels c are both bank-conflict free).
//   QK : lane = token; q of the G heads is broadcast from shared memory (fp32);
//        packed FFMA2 over channel pairs.
//   softmax: base-2 online softmax in fp32 (max and rescale warp-uniform,
//        row sums kept per lane and reduced once per pair segment).
//   PV : lane = D/32 channels, loop over the tile's valid tokens.
// At each pair boundary the warp writes its unnormalised (o, m, l) partial;
// decode_combine_kernel merges the partials of a pair with log-sum-exp weights.
#include "common.cuh"
#include "kernels.h"

namespace lserve {

namespace {

constexpr int kTileRows = kDecodeTile;

__device__ __forceinline__ int streaming_ordinal(int li, int ns, int ls) {
  return li < ns ? li : ls + (li - ns);
}

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

__device__ __forceinline__ int warp_incl_scan(int v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += t;
  }
  return v;
}

// For each lane's tile index (`active` lanes, all >= anchor_base), find the
// pair that holds it.  (anchor_pair, anchor_base) is warp-uniform: pair
// anchor_pair starts at tile anchor_base.  Pairs are examined 32 at a time.
__device__ void resolve_pairs(const DecodeParams& p, int P, int lane, long long my_tile, bool active,
                              int& anchor_pair, long long& anchor_base, int& out_pair,
                              long long& out_base) {
  bool need = active;
  while (__any_sync(0xffffffffu, need)) {
    const int pr = anchor_pair + lane;
    const int cnt = pr < P ? pair_pages(p, pr) * p.tiles_per_page : 0;
    const long long incl = (long long)warp_incl_scan(cnt, lane) + anchor_base;
    const long long excl = incl - cnt;
    const long long last = __shfl_sync(0xffffffffu, incl, 31);
    int pos = 0;
#pragma unroll
    for (int s = 16; s >= 1; s >>= 1) {
      const long long v = __shfl_sync(0xffffffffu, incl, pos + s - 1);
      if (v <= my_tile) pos += s;
    }
    const long long base_at = __shfl_sync(0xffffffffu, excl, pos);
    if (need && my_tile < last) {
      out_pair = anchor_pair + pos;
      out_base = base_at;
      need = false;
    }
    if (__any_sync(0xffffffffu, need)) {
      anchor_pair += 32;
      anchor_base = last;
      if (anchor_pair >= P) break;  // unreachable for tiles < total; keeps the loop finite
    }
  }
}

struct TileInfo {
  int row0;   // first row of the tile in the 2-D [pool rows][D] view
  int pair;
  int valid;  // valid tokens in the tile (0..32)
};

__device__ TileInfo tile_info(const DecodeParams& p, int pair, long long local) {
  TileInfo ti;
  ti.pair = pair;
  const int b = pair / p.num_kv_heads, h = pair - b * p.num_kv_heads;
  const int n = p.ctx_lens[b];
  const int NP = p.physical_page;
  const int npages = (n + NP - 1) / NP;
  const int li = (int)(local / p.tiles_per_page);
  const int sub = (int)(local - (long long)li * p.tiles_per_page);
  int m;
  if (p.head_kind[h] == 0) {
    m = p.sel[(size_t)pair * p.top_k + li];
  } else {
    const int ns = min((p.sink + NP - 1) / NP, npages);
    const int ls = max(max(0, n - p.local) / NP, ns);
    m = streaming_ordinal(li, ns, ls);
  }
  int pid = -1;
  if (m >= 0 && m < npages && m < p.max_pages) pid = p.block_table[(size_t)b * p.max_pages + m];
  if (pid < 0 || pid >= p.num_pool_pages) {  // bad selection entry or block table entry
    raise_status(p.status, LSERVE_ERR_BOUNDS);
    ti.row0 = 0;
    ti.valid = 0;
    return ti;
  }
  ti.row0 = (int)(((long long)pid * p.num_kv_heads + h) * NP + sub * kTileRows);
  ti.valid = max(0, min(kTileRows, n - m * NP - sub * kTileRows));
  return ti;
}

template <int D, int G>
struct DecodeLayout {
  static constexpr int kTileBytes = kTileRows * D * 2;        // one K (or V) tile
  static constexpr int kBoxBytes = kTileRows * 128;           // one 64-channel TMA box
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kQBytes = G * D * 4;                   // fp32 q of the pair
  static constexpr int kPBytes = kTileRows * G * 8;           // (p, p) pairs per token/head
  static constexpr int kInfoBytes = kDecodeStages * 8;
  static constexpr int kBarBytes = kDecodeStages * 8;
  static constexpr int kRaw = kDecodeStages * kStageBytes + kQBytes + kPBytes + kInfoBytes + kBarBytes;
  static constexpr int kWarpBytes = (kRaw + 1023) / 1024 * 1024;
};

}  // namespace

template <int D, int G>
__global__ void __launch_bounds__(8 * 32, 1)
decode_attn_kernel(const __grid_constant__ DecodeParams p, const __grid_constant__ CUtensorMap kmap,
                   const __grid_constant__ CUtensorMap vmap) {
  using L = DecodeLayout<D, G>;
  constexpr int NBOX = D / 64;
  constexpr int CPL = D / 32;  // channels per lane in PV
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ long long s_blk_excl[32];
  __shared__ long long s_total;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  const int P = p.batch * p.num_kv_heads;

  uint8_t* wb = smem + (size_t)warp * L::kWarpBytes;
  float* q_s = reinterpret_cast<float*>(wb + kDecodeStages * L::kStageBytes);
  float2* p_s = reinterpret_cast<float2*>(wb + kDecodeStages * L::kStageBytes + L::kQBytes);
  int2* info_s = reinterpret_cast<int2*>(wb + kDecodeStages * L::kStageBytes + L::kQBytes + L::kPBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(wb + kDecodeStages * L::kStageBytes + L::kQBytes +
                                               L::kPBytes + L::kInfoBytes);
  if (lane == 0) {
    for (int s = 0; s < kDecodeStages; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
  }
  if (threadIdx.x == 0) {
    tma_prefetch_desc(&kmap);
    tma_prefetch_desc(&vmap);
  }

  // ---- plan: per-block tile totals over the pairs (warp 0), shared via smem
  const int per = (P + 31) / 32;
  if (warp == 0) {
    const int lo = min(P, lane * per), hi = min(P, lo + per);
    long long sum = 0;
    for (int pr = lo; pr < hi; ++pr) sum += (long long)pair_pages(p, pr) * p.tiles_per_page;
    long long incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    s_blk_excl[lane] = incl - sum;
    if (lane == 31) s_total = incl;
    if (blockIdx.x == 0) {  // publish the exclusive prefix per pair for the combine pass
      long long base = 0;
      for (int w0 = 0; w0 < P; w0 += 32) {
        const int pr = w0 + lane;
        const int cnt = pr < P ? pair_pages(p, pr) * p.tiles_per_page : 0;
        const long long inc = (long long)warp_incl_scan(cnt, lane) + base;
        if (pr < P) p.pair_tiles[pr] = (int32_t)(inc - cnt);
        base = __shfl_sync(0xffffffffu, inc, 31);
      }
      if (lane == 0) p.pair_tiles[P] = (int32_t)base;
    }
  }
  __syncthreads();
  __syncwarp();

  const long long U = s_total;
  const long long gw = (long long)blockIdx.x * nwarps + warp;
  const long long t0 = U * gw / p.num_warps, t1 = U * (gw + 1) / p.num_warps;
  if (t0 >= t1) return;
  const int ntiles = (int)(t1 - t0);

  // anchor: last lane-block whose first tile is <= t0
  int anchor_pair = 0;
  long long anchor_base = 0;
  {
    const bool ok = lane * per < P && s_blk_excl[lane] <= t0;
    const unsigned bal = __ballot_sync(0xffffffffu, ok);
    const int L0 = 31 - __clz(bal);  // bal has bit 0 set (block 0 starts at 0)
    anchor_pair = L0 * per;
    anchor_base = s_blk_excl[L0];
  }

  // per-lane tile descriptors for the producer, 32 tiles per batch
  TileInfo my;
  auto load_batch = [&](int k0) {
    const long long tile = t0 + k0 + lane;
    const bool act = tile < t1;
    int pr = 0;
    long long pb = 0;
    resolve_pairs(p, P, lane, tile, act, anchor_pair, anchor_base, pr, pb);
    my.row0 = 0;
    my.pair = 0;
    my.valid = 0;
    if (act) my = tile_info(p, pr, tile - pb);
    // next batch starts from the pair of this batch's last tile
    const int last_lane = min(31, ntiles - 1 - k0);
    anchor_pair = __shfl_sync(0xffffffffu, pr, last_lane);
    anchor_base = __shfl_sync(0xffffffffu, pb, last_lane);
  };

  auto issue = [&](int k) {  // warp-uniform; lane 0 starts the copies of tile k
    if ((k & 31) == 0 && k > 0) load_batch(k);
    const int row0 = __shfl_sync(0xffffffffu, my.row0, k & 31);
    const int pair = __shfl_sync(0xffffffffu, my.pair, k & 31);
    const int valid = __shfl_sync(0xffffffffu, my.valid, k & 31);
    if (lane == 0) {
      const int s = k % kDecodeStages;
      uint8_t* kt = wb + s * L::kStageBytes;
      uint8_t* vt = kt + L::kTileBytes;
      info_s[s] = make_int2(pair, valid);
      fence_proxy_async_smem();
      mbar_arrive_expect_tx(&bars[s], L::kStageBytes);
#pragma unroll
      for (int bx = 0; bx < NBOX; ++bx) {
        tma_load_2d(kt + bx * L::kBoxBytes, &kmap, bx * 64, row0, &bars[s]);
        tma_load_2d(vt + bx * L::kBoxBytes, &vmap, bx * 64, row0, &bars[s]);
      }
    }
  };

  load_batch(0);
  for (int k = 0; k < kDecodeStages && k < ntiles; ++k) issue(k);

  // ---- consumer state
  int cur_pair = -1;
  float m_run[G], l_run[G];
  float2 o_acc[G][CPL / 2];
  const float4* q4 = reinterpret_cast<const float4*>(q_s);

  auto reset = [&](int pair) {
    const int b = pair / p.num_kv_heads, h = pair - b * p.num_kv_heads;
    const __nv_bfloat16* qg = p.q + ((size_t)b * p.num_q_heads + (size_t)h * G) * D;
    for (int i = lane; i < G * D / 2; i += 32) {
      const uint32_t w = reinterpret_cast<const uint32_t*>(qg)[i];
      q_s[2 * i] = bf16_lo(w);
      q_s[2 * i + 1] = bf16_hi(w);
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
      m_run[g] = -INFINITY;
      l_run[g] = 0.f;
#pragma unroll
      for (int j = 0; j < CPL / 2; ++j) o_acc[g][j] = make_float2(0.f, 0.f);
    }
    __syncwarp();
  };

  auto flush = [&](int pair) {
    const long long slot = gw + pair;
    float* po = p.partial + (size_t)slot * G * D;
    float* pml = p.partial + (size_t)(p.num_warps + P) * G * D + (size_t)slot * G * 2;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float lsum = warp_sum(l_run[g]);
      float* dst = po + (size_t)g * D + lane * CPL;
      if constexpr (CPL == 4) {
        *reinterpret_cast<float4*>(dst) =
            make_float4(o_acc[g][0].x, o_acc[g][0].y, o_acc[g][1].x, o_acc[g][1].y);
      } else {
        *reinterpret_cast<float2*>(dst) = o_acc[g][0];
      }
      if (lane == 0) *reinterpret_cast<float2*>(pml + 2 * g) = make_float2(m_run[g], lsum);
    }
  };

  // PV: lane's channels inside the swizzled V tile
  const int pv_chunk = (lane * CPL) / 8;               // 16-byte chunk index 0..D/8-1
  const int pv_box = pv_chunk / 8, pv_cc = pv_chunk % 8;
  const int pv_off = ((lane * CPL) % 8) * 2;           // byte offset inside the chunk

  for (int k = 0; k < ntiles; ++k) {
    const int s = k % kDecodeStages;
    if (!mbar_wait(&bars[s], (k / kDecodeStages) & 1, p.wait_limit, p.status)) return;
    const int2 inf = info_s[s];
    if (inf.x != cur_pair) {
      if (cur_pair >= 0) flush(cur_pair);
      cur_pair = inf.x;
      reset(cur_pair);
    }
    const int valid = inf.y;
    if (valid > 0) {
      const uint8_t* kt = wb + s * L::kStageBytes;
      const uint8_t* vt = kt + L::kTileBytes;
      // ---- QK: lane = token
      float2 acc[G];
#pragma unroll
      for (int g = 0; g < G; ++g) acc[g] = make_float2(0.f, 0.f);
#pragma unroll
      for (int c = 0; c < D / 8; ++c) {
        const uint4 kw = *reinterpret_cast<const uint4*>(kt + (c / 8) * L::kBoxBytes +
                                                         sw128_offset(lane, c % 8));
        const float2 k0 = bf16x2_to_float2(kw.x), k1 = bf16x2_to_float2(kw.y);
        const float2 k2 = bf16x2_to_float2(kw.z), k3 = bf16x2_to_float2(kw.w);
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float4 qa = q4[(g * D + c * 8) / 4];
          const float4 qb = q4[(g * D + c * 8) / 4 + 1];
          acc[g] = __ffma2_rn(make_float2(qa.x, qa.y), k0, acc[g]);
          acc[g] = __ffma2_rn(make_float2(qa.z, qa.w), k1, acc[g]);
          acc[g] = __ffma2_rn(make_float2(qb.x, qb.y), k2, acc[g]);
          acc[g] = __ffma2_rn(make_float2(qb.z, qb.w), k3, acc[g]);
        }
      }
      // ---- online softmax (base 2)
      const bool tok_ok = lane < valid;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float x = tok_ok ? (acc[g].x + acc[g].y) * p.scale_log2 : -INFINITY;
        const float mnew = fmaxf(m_run[g], warp_max(x));
        const float alpha = exp2f(m_run[g] - mnew);
        const float pr = exp2f(x - mnew);
        m_run[g] = mnew;
        l_run[g] = l_run[g] * alpha + pr;
#pragma unroll
        for (int j = 0; j < CPL / 2; ++j) {
          o_acc[g][j].x *= alpha;
          o_acc[g][j].y *= alpha;
        }
        p_s[lane * G + g] = make_float2(pr, pr);
      }
      __syncwarp();
      // ---- PV: lane = CPL channels
      const uint8_t* vrow = vt + pv_box * L::kBoxBytes + pv_off;
#pragma unroll 4
      for (int t = 0; t < valid; ++t) {
        const uint8_t* vaddr = vrow + sw128_offset(t, pv_cc);
        float2 v2[CPL / 2];
        if constexpr (CPL == 4) {
          const uint2 vw = *reinterpret_cast<const uint2*>(vaddr);
          v2[0] = bf16x2_to_float2(vw.x);
          v2[1] = bf16x2_to_float2(vw.y);
        } else {
          v2[0] = bf16x2_to_float2(*reinterpret_cast<const uint32_t*>(vaddr));
        }
        const float4* pp = reinterpret_cast<const float4*>(p_s + t * G);
#pragma unroll
        for (int g = 0; g < G; ++g) {
          float2 pg;
          if constexpr (G >= 2) {
            const float4 pq = pp[g / 2];
            pg = (g & 1) ? make_float2(pq.z, pq.w) : make_float2(pq.x, pq.y);
          } else {
            pg = p_s[t];
          }
#pragma unroll
          for (int j = 0; j < CPL / 2; ++j) o_acc[g][j] = __ffma2_rn(pg, v2[j], o_acc[g][j]);
        }
      }
    }
    __syncwarp();
    if (k + kDecodeStages < ntiles) issue(k + kDecodeStages);
  }
  if (cur_pair >= 0) flush(cur_pair);
}

// One warp per (pair, query head of the pair): merge the partials of the warps
// whose tile ranges overlap the pair.  Lanes take one segment each (32 at a
// time): the max and the weighted row sum are warp reductions, then every lane
// accumulates its D/32 channels over the segments with independent loads.
template <int D>
__global__ void __launch_bounds__(128)
decode_combine_kernel(const __grid_constant__ DecodeParams p, int G) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  const int P = p.batch * p.num_kv_heads;
  if (warp >= P * G) return;
  const int pair = warp / G, g = warp - pair * G;
  const int b = pair / p.num_kv_heads, h = pair - b * p.num_kv_heads;
  const long long U = p.pair_tiles[P];
  const long long T0 = p.pair_tiles[pair], T1 = p.pair_tiles[pair + 1];
  const int NW = p.num_warps;
  const float* po = p.partial;
  const float* pml = p.partial + (size_t)(NW + P) * G * D;
  constexpr int CPL = D / 32;
  float acc[CPL];
#pragma unroll
  for (int j = 0; j < CPL; ++j) acc[j] = 0.f;
  float M = -INFINITY, Lsum = 0.f;
  if (T1 > T0) {
    // first warp whose range holds tile T0: start(w) = floor(U*w/NW) <= T0 < start(w+1)
    long long w0 = (T0 * NW) / U;
    while (w0 + 1 < NW && (U * (w0 + 1)) / NW <= T0) ++w0;
    while (w0 > 0 && (U * w0) / NW > T0) --w0;
    // last warp whose range holds tile T1 - 1
    long long w1 = ((T1 - 1) * NW) / U;
    while (w1 + 1 < NW && (U * (w1 + 1)) / NW <= T1 - 1) ++w1;
    while (w1 > 0 && (U * w1) / NW > T1 - 1) --w1;
    for (long long base = w0; base <= w1; base += 32) {
      const long long ww = base + lane;
      float m_s = -INFINITY, l_s = 0.f;
      bool has = false;
      if (ww <= w1) {
        const long long s0 = (U * ww) / NW, s1 = (U * (ww + 1)) / NW;
        has = s1 > s0;  // warps with an empty range wrote nothing
        if (has) {
          const float2 ml = *reinterpret_cast<const float2*>(pml + ((size_t)(ww + pair) * G + g) * 2);
          m_s = ml.x;
          l_s = ml.y;
        }
      }
      const float Mc = warp_max(m_s);
      const float Mn = fmaxf(M, Mc);
      if (!(Mn > -INFINITY)) continue;
      const float rescale = exp2f(M - Mn);  // 0 when M was -inf
      const float w_s = has ? exp2f(m_s - Mn) : 0.f;
      Lsum = Lsum * rescale + warp_sum(w_s * l_s);
      for (int j = 0; j < CPL; ++j) acc[j] *= rescale;
      M = Mn;
      const int nseg = (int)min(32ll, w1 - base + 1);
      const float* src0 = po + ((size_t)(base + pair) * G + g) * D + lane * CPL;
      const size_t stride = (size_t)G * D;
      // slots of empty-range warps were never written: their weight is 0 and the
      // select below (not a multiply) keeps whatever they hold out of the sum
#pragma unroll 8
      for (int i = 0; i < 32; ++i) {
        if (i >= nseg) break;
        const float wi = __shfl_sync(0xffffffffu, w_s, i);
        float v[CPL];
        if constexpr (CPL == 4) {
          const float4 t4 = *reinterpret_cast<const float4*>(src0 + i * stride);
          v[0] = t4.x; v[1] = t4.y; v[2] = t4.z; v[3] = t4.w;
        } else {
          const float2 t2 = *reinterpret_cast<const float2*>(src0 + i * stride);
          v[0] = t2.x; v[1] = t2.y;
        }
#pragma unroll
        for (int j = 0; j < CPL; ++j) acc[j] = wi != 0.f ? fmaf(wi, v[j], acc[j]) : acc[j];
      }
    }
  }
  const size_t qh = (size_t)b * p.num_q_heads + (size_t)h * G + g;
  __nv_bfloat16* out = p.out + qh * D + lane * CPL;
  const bool empty = !(M > -INFINITY) || !(Lsum > 0.f);
  const float inv = empty ? 0.f : 1.f / Lsum;
  for (int j = 0; j < CPL; ++j) out[j] = __float2bfloat16_rn(acc[j] * inv);
  if (p.lse != nullptr && lane == 0)
    p.lse[qh] = empty ? -INFINITY : (M + log2f(Lsum)) * 0.69314718055994530942f;
}

size_t decode_smem_bytes(int D, int G) {
#define LSERVE_LAYOUT_CASE(DD, GG) \
  if (D == DD && G == GG) return (size_t)DecodeLayout<DD, GG>::kWarpBytes;
  LSERVE_LAYOUT_CASE(64, 1)
  LSERVE_LAYOUT_CASE(64, 2)
  LSERVE_LAYOUT_CASE(64, 4)
  LSERVE_LAYOUT_CASE(64, 8)
  LSERVE_LAYOUT_CASE(128, 1)
  LSERVE_LAYOUT_CASE(128, 2)
  LSERVE_LAYOUT_CASE(128, 4)
  LSERVE_LAYOUT_CASE(128, 8)
#undef LSERVE_LAYOUT_CASE
  return 0;
}

int decode_warps_per_cta(int D, int G) {
  const size_t per = decode_smem_bytes(D, G);
  if (per == 0) return 0;
  const size_t budget = 227 * 1024 - 1024;  // minus the 1 KiB alignment slack
  int w = (int)(budget / per);
  return w > 8 ? 8 : w;
}

int decode_num_ctas(int sm_count) { return sm_count; }

size_t decode_workspace_bytes(int pairs, int num_warps, int G, int D) {
  const size_t head = ((size_t)(pairs + 1) * 4 + 255) / 256 * 256;
  const size_t slots = (size_t)num_warps + pairs;
  return head + slots * G * D * 4 + slots * G * 2 * 4;
}

cudaError_t launch_decode(const DecodeParams& p_in, const CUtensorMap& kmap, const CUtensorMap& vmap,
                          int D, int G, int num_ctas, cudaStream_t stream) {
  DecodeParams p = p_in;
  const int wpc = decode_warps_per_cta(D, G);
  if (wpc <= 0) return cudaErrorInvalidValue;
  p.num_warps = num_ctas * wpc;
  const size_t smem = (size_t)wpc * decode_smem_bytes(D, G) + 1024;
  cudaError_t e = cudaSuccess;
#define LSERVE_DECODE_CASE(DD, GG)                                                              \
  if (D == DD && G == GG) {                                                                     \
    e = set_smem_once((const void*)decode_attn_kernel<DD, GG>, (int)smem);                      \
    if (e != cudaSuccess) return e;                                                             \
    decode_attn_kernel<DD, GG><<<num_ctas, wpc * 32, smem, stream>>>(p, kmap, vmap);            \
  } else
  LSERVE_DECODE_CASE(64, 1)
  LSERVE_DECODE_CASE(64, 2)
  LSERVE_DECODE_CASE(64, 4)
  LSERVE_DECODE_CASE(64, 8)
  LSERVE_DECODE_CASE(128, 1)
  LSERVE_DECODE_CASE(128, 2)
  LSERVE_DECODE_CASE(128, 4)
  LSERVE_DECODE_CASE(128, 8)
  return cudaErrorInvalidValue;
#undef LSERVE_DECODE_CASE
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int P = p.batch * p.num_kv_heads;
  const int warps = P * G;
  if (D == 128)
    decode_combine_kernel<128><<<(warps + 3) / 4, 128, 0, stream>>>(p, G);
  else
    decode_combine_kernel<64><<<(warps + 3) / 4, 128, 0, stream>>>(p, G);
  return cudaGetLastError();
}

}  // namespace lserve
