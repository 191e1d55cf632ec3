// lserve_blocksparse_prefill: causal block-sparse flash attention on the
// sm_100a tensor cores (LServe explainer, 統一ブロックスパースアテンション: retrieval
// heads dense causal, streaming heads the Lambda mask of sink + local blocks,
// ideal speedup 1/(1-r) at block sparsity r; abstract page: computation on
// less important tokens is skipped block-wise).
//
// One CTA per SM, persistent over work tiles (query head, 128-row query tile).
// Tiles are ordered by decreasing cost (dense heads, last query tiles first)
// and dealt to CTAs in a snake order, so every SM ends up with a similar
// number of key tiles.  The key-tile iterator visits only the non-empty tiles
// of the row (all j <= i for dense heads; sink tiles and the local window for
// streaming heads) -- the block skipping of the method.
//
// Warp roles (192 threads; 224 in the paged-epilogue variant):
//   warp 0     TMA producer: Q tile, then K and V tiles into two-stage rings
//              (3-D tensor maps over [T][H][D], 128-byte swizzle, no multicast)
//   warp 1     tensor-memory owner and single-thread MMA issuer:
//                S_j = Q K_j^T  -> TMEM (two fp32 128x128 buffers, ping-pong)
//                O  += P_j V_j  -> TMEM (fp32 128 x D), P from shared memory
//   warps 2-5  softmax: thread r owns query row r (TMEM lane r); loads S_j,
//              masks, keeps the running max / row sum in fp32, writes P_j as
//              bf16 into shared memory (swizzled like a TMA tile), rescales O
//              in TMEM only when the row max grows by more than 2^8, and runs
//              the epilogue O / l -> bf16 and the log-sum-exp.
//   warp 6     page writer (lserve_blocksparse_prefill_paged only): each key
//              tile of a KV head into the paged pools and its page
//              statistics, read from the kernel's own K / V inputs.
// MMA order S_0, S_1, PV_0, S_2, PV_1, ... keeps the tensor core on S_{j+1}
// while the softmax warps work on S_j.
#include <algorithm>
#include <cmath>
#include <cstring>

#include "common.cuh"
#include "kernels.h"
#include "prefill.h"
#include "tcgen05.cuh"

namespace lserve {

namespace {

constexpr int kBM = 128;            // query rows per tile (MMA M)
constexpr int kBN = 128;            // keys per key tile (MMA N of S, K of PV)
constexpr int kThreads = 224;  // 7 warps; warp 6 writes the paged cache (kPaged only)
constexpr float kRescaleLog2 = 8.0f;  // rescale O only when the max grows by > 2^8
constexpr int kMaxHeads = 256;

struct PrefillParams {
  __nv_bfloat16* out;
  float* lse;
  unsigned int* status;
  uint64_t wait_limit;
  float scale_log2;
  int T, H_q, H_kv, G;
  int mask_block, sink_blocks, local_blocks;
  int n_qt;               // query tiles per head
  int n_dense, n_stream;  // query heads whose KV head is retrieval / streaming
  uint8_t dense_heads[kMaxHeads];
  uint8_t stream_heads[kMaxHeads];
  uint8_t kv_kind[kMaxHeads];
  // the paired kernel: first query head of each pair (two heads of one KV head)
  int n_dense_pairs, n_stream_pairs;
  uint8_t dense_pairs[kMaxHeads / 2];
  uint8_t stream_pairs[kMaxHeads / 2];
  // paged epilogue (lserve_blocksparse_prefill_paged only)
  const __nv_bfloat16* pg_k_in;   // the prefill's K and V, [T][H_kv][D]
  const __nv_bfloat16* pg_v_in;
  __nv_bfloat16* pg_k_pool;
  __nv_bfloat16* pg_v_pool;
  __nv_bfloat16* pg_stats;
  const int32_t* pg_block_table;  // this sequence's page ordinal -> pool id
  int pg_np, pg_nl, pg_max_pages, pg_num_pool_pages;
};

template <int D>
struct Layout {
  static constexpr int kBox = kBM * 128;          // one 64-column swizzled box: 16 KiB
  static constexpr int kTile = kBox * (D / 64);   // a Q, K or V tile
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kTile;           // 2 stages
  static constexpr int kV = kK + 2 * kTile;       // 2 stages
  static constexpr int kP = kV + 2 * kTile;       // P: 128 x 128 bf16, 2 boxes
  static constexpr int kBar = kP + 2 * kBox;
  static constexpr int kNumBars = 17;
  static constexpr int kBytes = kBar + kNumBars * 8 + 16;
};

struct TileRef {
  int hq, qt;
};

__device__ __forceinline__ TileRef tile_at(const PrefillParams& p, int idx) {
  const int nd = p.n_dense * p.n_qt;
  if (idx < nd) return {p.dense_heads[idx % p.n_dense], p.n_qt - 1 - idx / p.n_dense};
  idx -= nd;
  return {p.stream_heads[idx % p.n_stream], p.n_qt - 1 - idx / p.n_stream};
}

// round r of CTA c: snake order over the cost-sorted tile list
__device__ __forceinline__ int cta_tile(int r, int c, int grid) {
  return r * grid + ((r & 1) ? grid - 1 - c : c);
}

// Key tiles a query tile visits: [0, a_end) then [b_begin, b_end).
struct KvRange {
  int a_end, b_begin, b_end;
  __device__ int count() const { return a_end + (b_end - b_begin); }
  __device__ int at(int j) const { return j < a_end ? j : b_begin + (j - a_end); }
};

__device__ __forceinline__ KvRange kv_range(const PrefillParams& p, int kind, int qt) {
  if (kind == 0) return {qt + 1, qt + 1, qt + 1};
  const int R = kBN / p.mask_block;  // mask blocks per tile
  const int st = min((p.sink_blocks * p.mask_block + kBN - 1) / kBN, qt + 1);
  const int first_kb = max(0, qt * R - p.local_blocks + 1);
  const int lt = max((first_kb * p.mask_block) / kBN, st);
  return {st, lt, qt + 1};
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, uint64_t limit,
                                          unsigned int* status) {
  const bool ok = mbar_wait(bar, parity, limit, status);
  return __all_sync(0xffffffffu, ok);
}

// Paged epilogue of key tile kt of KV head h, run by one warp: the rows
// [kt*kBN, min(kt*kBN + kBN, T)) of the prefill's K and V go to their pool
// rows through the block table, and for a retrieval head every logical page
// of the tile gets the bf16 min / max of its keys per channel (the values
// lserve_page_stats and lserve_prefill_to_pages write).  The rows are read
// from the kernel's own K / V inputs -- the tile loads of this kernel keep
// them in L2 -- with plain 16-byte loads (D/8 lanes a row, 32 / (D/8) rows a
// step) and stored the same way, so the writer never holds a ring stage and
// waits on nothing.
template <int D>
__device__ void page_out(const PrefillParams& p, int kt, int h, int lane) {
  constexpr int LPR = D / 8;     // lanes per row
  constexpr int RPI = 32 / LPR;  // rows of one warp-wide step
  const int t0 = kt * kBN, tend = min(t0 + kBN, p.T);
  const int NP = p.pg_np, NL = p.pg_nl, g = NP / NL;
  const int r0 = lane / LPR, c = (lane % LPR) * 8;
  const size_t src_stride = (size_t)p.H_kv * D;  // between tokens of [T][H_kv][D]
  // the tile's block-table entries (at most kBN / 32 pages), one lane each
  const int m0 = t0 / NP;
  int pid_l = -1;
  if (m0 + lane < p.pg_max_pages && (m0 + lane) * NP < tend) pid_l = p.pg_block_table[m0 + lane];
  const uint32_t kPosInf2 = 0x7F807F80u, kNegInf2 = 0xFF80FF80u;
  for (int lp = t0 / NL; lp * NL < tend; ++lp) {  // logical pages of the tile (N_L divides kBN)
    const int m = lp / g, sub = lp - m * g;
    const int pid = __shfl_sync(0xffffffffu, pid_l, m - m0);
    if (pid < 0 || pid >= p.pg_num_pool_pages) {  // bad entry: the page is skipped and flagged
      if (lane == 0) raise_status(p.status, LSERVE_ERR_BOUNDS);
      continue;
    }
    const int valid = min(NL, tend - lp * NL);
    const size_t src0 = (size_t)lp * NL * src_stride + (size_t)h * D + c;
    const size_t dst0 = (((size_t)pid * p.H_kv + h) * NP + (size_t)sub * NL) * D + c;
    __nv_bfloat162 mn[4], mx[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      mn[k] = *reinterpret_cast<const __nv_bfloat162*>(&kPosInf2);
      mx[k] = *reinterpret_cast<const __nv_bfloat162*>(&kNegInf2);
    }
    for (int r = r0; r < valid; r += RPI) {
      const uint4 kr = ldg_nc_v4(p.pg_k_in + src0 + (size_t)r * src_stride);
      const uint4 vr = ldg_nc_v4(p.pg_v_in + src0 + (size_t)r * src_stride);
      *reinterpret_cast<uint4*>(p.pg_k_pool + dst0 + (size_t)r * D) = kr;
      *reinterpret_cast<uint4*>(p.pg_v_pool + dst0 + (size_t)r * D) = vr;
      const __nv_bfloat162* v = reinterpret_cast<const __nv_bfloat162*>(&kr);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        mn[k] = __hmin2(mn[k], v[k]);
        mx[k] = __hmax2(mx[k], v[k]);
      }
    }
    if (p.kv_kind[h] != 0) continue;  // streaming heads need no statistics
    // reduce over the row groups of the warp (lanes holding the same channels)
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
      __nv_bfloat16* st = p.pg_stats + ((((size_t)pid * p.H_kv + h) * g) + sub) * 2 * D + c;
      *reinterpret_cast<uint4*>(st) = *reinterpret_cast<uint4*>(mn);
      *reinterpret_cast<uint4*>(st + D) = *reinterpret_cast<uint4*>(mx);
    }
  }
}

// The page writer warp: follows the CTA's work tiles (the producer's order)
// and, for every tile of a KV head's first query head, writes the pages of
// its diagonal key tile -- each key tile of a head is the diagonal tile of
// exactly one such work tile.  It reads only the kernel's inputs and writes
// only the paged cache, so nothing else in the kernel waits on it.
template <int D, typename TileAt>
__device__ void page_writer(const PrefillParams& p, int total, TileAt tile_of, int lane) {
  for (int r = 0;; ++r) {
    const int idx = cta_tile(r, blockIdx.x, gridDim.x);
    if (idx >= total) break;
    const TileRef t = tile_of(idx);
    if (t.hq % p.G == 0) page_out<D>(p, t.qt, t.hq / p.G, lane);
  }
}

}  // namespace

template <int D, bool kPaged>
__global__ void __launch_bounds__(kPaged ? kThreads : kThreads - 32, 1)
prefill_kernel(const __grid_constant__ PrefillParams p, const __grid_constant__ CUtensorMap qmap,
               const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap) {
  using L = Layout<D>;
  constexpr int NBOX = D / 64;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* k_full = bars + 2;   // [2]
  uint64_t* k_empty = bars + 4;  // [2]
  uint64_t* v_full = bars + 6;   // [2]
  uint64_t* v_empty = bars + 8;  // [2]
  uint64_t* s_full = bars + 10;  // [2]
  uint64_t* s_free = bars + 12;  // [2]
  uint64_t* p_full = bars + 14;
  uint64_t* p_free = bars + 15;
  uint64_t* o_free = bars + 16;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::kBar + L::kNumBars * 8);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
      mbar_init(&s_full[s], 1);
      mbar_init(&s_free[s], 128);
    }
    mbar_init(p_full, 128);
    mbar_init(p_free, 1);
    mbar_init(o_free, 128);
    fence_mbar_init();
  }
  if (warp == 1) {
    tc::alloc(tmem_holder, 512);
    tc::relinquish();
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t tmem_o = tmem + 2 * kBN;  // columns [256, 256 + D)

  const int total = (p.n_dense + p.n_stream) * p.n_qt;
  const int grid = gridDim.x;
  const uint64_t lim = p.wait_limit;

  if (kPaged && warp == 6) {
    // ------------------------------------------------------------ page writer
    page_writer<D>(p, total, [&](int idx) { return tile_at(p, idx); }, lane);
  } else if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&qmap);
      tma_prefetch_desc(&kmap);
      tma_prefetch_desc(&vmap);
      int q_use = 0, kv_use = 0;
      for (int r = 0;; ++r) {
        const int idx = cta_tile(r, blockIdx.x, grid);
        if (idx >= total) break;
        const TileRef t = tile_at(p, idx);
        const int hkv = t.hq / p.G;
        const KvRange kr = kv_range(p, p.kv_kind[hkv], t.qt);
        if (q_use > 0 && !mbar_wait(q_empty, (q_use - 1) & 1, lim, p.status)) break;
        mbar_arrive_expect_tx(q_full, L::kTile);
        for (int bx = 0; bx < NBOX; ++bx)
          tma_load_3d(smem + L::kQ + bx * L::kBox, &qmap, bx * 64, t.hq, t.qt * kBM, q_full);
        ++q_use;
        bool ok = true;
        const int nkv = kr.count();
        for (int j = 0; j < nkv && ok; ++j) {
          const int kt = kr.at(j);
          const int s = kv_use & 1, n = kv_use >> 1;
          if (n > 0 && !mbar_wait(&k_empty[s], (n - 1) & 1, lim, p.status)) { ok = false; break; }
          mbar_arrive_expect_tx(&k_full[s], L::kTile);
          for (int bx = 0; bx < NBOX; ++bx)
            tma_load_3d(smem + L::kK + s * L::kTile + bx * L::kBox, &kmap, bx * 64, hkv, kt * kBN,
                        &k_full[s]);
          if (n > 0 && !mbar_wait(&v_empty[s], (n - 1) & 1, lim, p.status)) { ok = false; break; }
          mbar_arrive_expect_tx(&v_full[s], L::kTile);
          for (int bx = 0; bx < NBOX; ++bx)
            tma_load_3d(smem + L::kV + s * L::kTile + bx * L::kBox, &vmap, bx * 64, hkv, kt * kBN,
                        &v_full[s]);
          ++kv_use;
        }
        if (!ok) break;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = tc::idesc_bf16_f32(kBM, kBN, false, false);
      constexpr uint32_t idesc_pv = tc::idesc_bf16_f32(kBM, D, false, true);
      const uint32_t q_addr = smem_u32(smem + L::kQ);
      const uint32_t p_addr = smem_u32(smem + L::kP);
      int q_use = 0, kv_base = 0, s_count = 0, pv_count = 0, tile_count = 0;
      bool ok = true;
      for (int r = 0; ok; ++r) {
        const int idx = cta_tile(r, blockIdx.x, grid);
        if (idx >= total) break;
        const TileRef t = tile_at(p, idx);
        const KvRange kr = kv_range(p, p.kv_kind[t.hq / p.G], t.qt);
        const int nkv = kr.count();
        if (!mbar_wait(q_full, q_use & 1, lim, p.status)) break;
        ++q_use;
        tc::fence_after();
        auto issue_s = [&](int j) -> bool {
          const int kvi = kv_base + j, s = kvi & 1, n = kvi >> 1;
          const int sb = s_count & 1, sn = s_count >> 1;
          if (sn > 0 && !mbar_wait(&s_free[sb], (sn - 1) & 1, lim, p.status)) return false;
          if (!mbar_wait(&k_full[s], n & 1, lim, p.status)) return false;
          tc::fence_after();
          const uint32_t k_addr = smem_u32(smem + L::kK + s * L::kTile);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk / 4) * L::kBox + (kk % 4) * 32;
            tc::mma_ss(tmem + sb * kBN, tc::smem_desc_sw128(q_addr + off, 16, 1024),
                       tc::smem_desc_sw128(k_addr + off, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
          }
          tc::commit(&s_full[sb]);
          tc::commit(&k_empty[s]);
          if (j == nkv - 1) tc::commit(q_empty);
          ++s_count;
          return true;
        };
        auto issue_pv = [&](int j) -> bool {
          const int kvi = kv_base + j, s = kvi & 1, n = kvi >> 1;
          if (!mbar_wait(p_full, pv_count & 1, lim, p.status)) return false;
          if (j == 0 && tile_count > 0 && !mbar_wait(o_free, (tile_count - 1) & 1, lim, p.status))
            return false;
          if (!mbar_wait(&v_full[s], n & 1, lim, p.status)) return false;
          tc::fence_after();
          const uint32_t v_addr = smem_u32(smem + L::kV + s * L::kTile);
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk) {
            const uint32_t poff = (kk / 4) * L::kBox + (kk % 4) * 32;
            tc::mma_ss(tmem_o, tc::smem_desc_sw128(p_addr + poff, 16, 1024),
                       tc::smem_desc_sw128(v_addr + kk * 16 * 128, L::kBox, 1024), idesc_pv,
                       (j > 0 || kk > 0) ? 1u : 0u);
          }
          tc::commit(&v_empty[s]);
          tc::commit(p_free);
          ++pv_count;
          return true;
        };
        ok = issue_s(0);
        for (int j = 1; j < nkv && ok; ++j) ok = issue_s(j) && issue_pv(j - 1);
        if (ok) ok = issue_pv(nkv - 1);
        kv_base += nkv;
        ++tile_count;
      }
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int quad = warp & 3;                 // TMEM lane quarter of this warp
    const int row = quad * 32 + lane;          // query row within the tile
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    uint8_t* p_row = smem + L::kP + row * 128;
    int s_count = 0, pv_count = 0;
    bool ok = true;
    for (int r = 0; ok; ++r) {
      const int idx = cta_tile(r, blockIdx.x, grid);
      if (idx >= total) break;
      const TileRef t = tile_at(p, idx);
      const int kind = p.kv_kind[t.hq / p.G];
      const KvRange kr = kv_range(p, kind, t.qt);
      const int nkv = kr.count();
      const int q = t.qt * kBM + row;
      float m = -INFINITY, l = 0.f;
      for (int j = 0; j < nkv; ++j) {
        const int kt = kr.at(j);
        const int sb = s_count & 1, sn = s_count >> 1;
        if (!warp_wait(&s_full[sb], sn & 1, lim, p.status)) { ok = false; break; }
        tc::fence_after();
        float x[kBN];
#pragma unroll
        for (int c = 0; c < kBN / 32; ++c) {
          uint32_t u[32];
          tc::ld32(tmem + lane_off + sb * kBN + c * 32, u);
          tc::wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) x[c * 32 + i] = __uint_as_float(u[i]);
        }
        tc::fence_before();
        mbar_arrive(&s_free[sb]);
        ++s_count;
        const bool need_mask = kt == t.qt || (kt + 1) * kBN > p.T || (kind == 1 && p.mask_block < kBN);
        if (need_mask) {
          const int qb = q / p.mask_block;
#pragma unroll
          for (int i = 0; i < kBN; ++i) {
            const int k = kt * kBN + i;
            const int kb = k / p.mask_block;
            const bool allowed = k <= q && k < p.T &&
                                 (kind == 0 || kb < p.sink_blocks || qb - kb < p.local_blocks);
            if (!allowed) x[i] = -INFINITY;
          }
        }
        // row max and (below) row sum as 8 independent partial chains: one
        // softmax warp per SM sub-partition leaves no other warp to hide a
        // 128-long dependent chain
        float mt8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) mt8[i] = x[i];
#pragma unroll
        for (int i = 8; i < kBN; ++i) mt8[i & 7] = fmaxf(mt8[i & 7], x[i]);
        const float mt = fmaxf(fmaxf(fmaxf(mt8[0], mt8[1]), fmaxf(mt8[2], mt8[3])),
                               fmaxf(fmaxf(mt8[4], mt8[5]), fmaxf(mt8[6], mt8[7])));
        const float m_new = fmaxf(m, mt * p.scale_log2);
        float alpha = 1.f;
        bool rescale = false;
        if (j == 0) {
          m = m_new;
        } else if (m_new > m + kRescaleLog2) {
          alpha = tc::ex2(m - m_new);
          m = m_new;
          rescale = true;
        }
        const float mu = (m == -INFINITY) ? 0.f : m;
        float rs8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) rs8[i] = 0.f;
#pragma unroll
        for (int i = 0; i < kBN; ++i) {
          x[i] = tc::ex2(fmaf(x[i], p.scale_log2, -mu));
          rs8[i & 7] += x[i];
        }
        const float rs = ((rs8[0] + rs8[1]) + (rs8[2] + rs8[3])) + ((rs8[4] + rs8[5]) + (rs8[6] + rs8[7]));
        l = l * alpha + rs;
        // P_j may overwrite P_{j-1} (and O may be rescaled) once PV_{j-1} is done
        if (pv_count > 0 && !warp_wait(p_free, (pv_count - 1) & 1, lim, p.status)) { ok = false; break; }
        tc::fence_after();
        if (rescale) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t u[32];
            tc::ld32(tmem_o + lane_off + c * 32, u);
            tc::wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) u[i] = __float_as_uint(__uint_as_float(u[i]) * alpha);
            tc::st32(tmem_o + lane_off + c * 32, u);
          }
          tc::wait_st();
        }
#pragma unroll
        for (int c = 0; c < kBN / 8; ++c) {
          uint4 w;
          w.x = float2_to_bf16x2(x[c * 8 + 0], x[c * 8 + 1]);
          w.y = float2_to_bf16x2(x[c * 8 + 2], x[c * 8 + 3]);
          w.z = float2_to_bf16x2(x[c * 8 + 4], x[c * 8 + 5]);
          w.w = float2_to_bf16x2(x[c * 8 + 6], x[c * 8 + 7]);
          *reinterpret_cast<uint4*>(p_row + (c / 8) * L::kBox + (((c % 8) ^ (row & 7)) << 4)) = w;
        }
        fence_proxy_async_smem();
        tc::fence_before();
        mbar_arrive(p_full);
        ++pv_count;
      }
      if (!ok) break;
      // ---- epilogue: O / l -> bf16, log-sum-exp
      if (!warp_wait(p_free, (pv_count - 1) & 1, lim, p.status)) break;
      tc::fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      __nv_bfloat16* orow = p.out + ((size_t)q * p.H_q + t.hq) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t u[32];
        tc::ld32(tmem_o + lane_off + c * 32, u);
        tc::wait_ld();
        if (q < p.T) {
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 w;
            w.x = float2_to_bf16x2(__uint_as_float(u[v * 8 + 0]) * inv, __uint_as_float(u[v * 8 + 1]) * inv);
            w.y = float2_to_bf16x2(__uint_as_float(u[v * 8 + 2]) * inv, __uint_as_float(u[v * 8 + 3]) * inv);
            w.z = float2_to_bf16x2(__uint_as_float(u[v * 8 + 4]) * inv, __uint_as_float(u[v * 8 + 5]) * inv);
            w.w = float2_to_bf16x2(__uint_as_float(u[v * 8 + 6]) * inv, __uint_as_float(u[v * 8 + 7]) * inv);
            *reinterpret_cast<uint4*>(orow + c * 32 + v * 8) = w;
          }
        }
      }
      if (p.lse != nullptr && q < p.T)
        p.lse[(size_t)t.hq * p.T + q] = l > 0.f ? (m + __log2f(l)) * 0.69314718055994530942f : -INFINITY;
      tc::fence_before();
      mbar_arrive(o_free);
    }
  }
  tc::fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after();
    tc::dealloc(tmem, 512);
  }
}

// --- the paired kernel ------------------------------------------------------------
// Two query heads of the same KV head and the same query tile form one work
// tile: their key-tile ranges are identical and they read the same K and V
// tiles.  Each head has its own softmax warpgroup, S and O in tensor memory,
// and its P written over the first half of its own S (bf16 pairs, the A operand
// of PV read from TMEM).  The tensor core alternates between the heads
// (S_A0 S_B0 PV_A0 S_A1 PV_B0 S_B1 PV_A1 ...), so one head's softmax always
// overlaps the other head's matrix products -- the single-tile kernel above
// leaves the tensor core waiting for its one softmax warpgroup.
//   warp 0        TMA producer: Q of both heads, K and V into two-stage rings
//   warp 1        tensor-memory owner (all 512 columns) and MMA issuer
//   warp 2        page writer (lserve_blocksparse_prefill_paged only), as in
//                 prefill_kernel
//   warp 3        idle (it only lends its registers)
//   warps 4-7     softmax of head A (thread r: query row r = TMEM lane r)
//   warps 8-11    softmax of head B
// An S commit also covers the PV issued before it: when a softmax warpgroup
// sees S_j, the PV that read its P_{j-1} (the same columns) has completed and
// O may be rescaled.
namespace {
constexpr int kPairThreads = 384;
constexpr int kPairRegsCtl = 88;    // warpgroup 0 after setmaxnreg
constexpr int kPairRegsSoft = 208;  // softmax warpgroups: 128*88 + 256*208 = 384*168

template <int D>
struct PairLayout {
  static constexpr int kBox = kBM * 128;
  static constexpr int kTile = kBox * (D / 64);
  static constexpr int kQ = 0;                  // Q_A, Q_B
  static constexpr int kK = kQ + 2 * kTile;     // 2 stages
  static constexpr int kV = kK + 2 * kTile;     // 2 stages
  static constexpr int kBar = kV + 2 * kTile;
  static constexpr int kNumBars = 19;
  static constexpr int kBytes = kBar + kNumBars * 8 + 16;
};

__device__ __forceinline__ TileRef pair_tile_at(const PrefillParams& p, int idx) {
  const int nd = p.n_dense_pairs * p.n_qt;
  if (idx < nd) return {p.dense_pairs[idx % p.n_dense_pairs], p.n_qt - 1 - idx / p.n_dense_pairs};
  idx -= nd;
  return {p.stream_pairs[idx % p.n_stream_pairs], p.n_qt - 1 - idx / p.n_stream_pairs};
}
}  // namespace

template <int D, bool kPaged>
__global__ void __launch_bounds__(kPairThreads, 1)
prefill_pair_kernel(const __grid_constant__ PrefillParams p, const __grid_constant__ CUtensorMap qmap,
                    const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap) {
  using L = PairLayout<D>;
  constexpr int NBOX = D / 64;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* k_full = bars + 2;    // [2]
  uint64_t* k_empty = bars + 4;   // [2]
  uint64_t* v_full = bars + 6;    // [2]
  uint64_t* v_empty = bars + 8;   // [2]
  uint64_t* s_full = bars + 10;   // [head]
  uint64_t* p_full = bars + 12;   // [head]
  uint64_t* pv_done = bars + 14;  // [head]: the tile's last PV has completed
  uint64_t* o_free = bars + 16;   // [head]: the epilogue has read O
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::kBar + L::kNumBars * 8);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], 128);
      mbar_init(&pv_done[s], 1);
      mbar_init(&o_free[s], 128);
    }
    fence_mbar_init();
  }
  if (warp == 1) {
    tc::alloc(tmem_holder, 512);
    tc::relinquish();
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = *tmem_holder;
  // columns: S_A [0, 128), S_B [128, 256), O_A [256, 256 + D), O_B [256 + D, 256 + 2D);
  // P_X over the first 64 columns of S_X
  auto tmem_s = [&](int x) { return tmem + x * kBN; };
  auto tmem_o = [&](int x) { return tmem + 2 * kBN + x * D; };

  const int total = (p.n_dense_pairs + p.n_stream_pairs) * p.n_qt;
  const int grid = gridDim.x;
  const uint64_t lim = p.wait_limit;

  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kPairRegsCtl));
    if (warp == 0 && lane == 0) {
      // ------------------------------------------------------------ TMA producer
      tma_prefetch_desc(&qmap);
      tma_prefetch_desc(&kmap);
      tma_prefetch_desc(&vmap);
      int q_use = 0, kv_use = 0;
      for (int r = 0;; ++r) {
        const int idx = cta_tile(r, blockIdx.x, grid);
        if (idx >= total) break;
        const TileRef t = pair_tile_at(p, idx);  // t.hq: head A, head B = t.hq + 1
        const int hkv = t.hq / p.G;
        const KvRange kr = kv_range(p, p.kv_kind[hkv], t.qt);
        if (q_use > 0 && !mbar_wait(q_empty, (q_use - 1) & 1, lim, p.status)) break;
        mbar_arrive_expect_tx(q_full, 2 * L::kTile);
        for (int x = 0; x < 2; ++x)
          for (int bx = 0; bx < NBOX; ++bx)
            tma_load_3d(smem + L::kQ + x * L::kTile + bx * L::kBox, &qmap, bx * 64, t.hq + x,
                        t.qt * kBM, q_full);
        ++q_use;
        bool ok = true;
        const int nkv = kr.count();
        for (int j = 0; j < nkv && ok; ++j) {
          const int kt = kr.at(j);
          const int s = kv_use & 1, n = kv_use >> 1;
          if (n > 0 && !mbar_wait(&k_empty[s], (n - 1) & 1, lim, p.status)) { ok = false; break; }
          mbar_arrive_expect_tx(&k_full[s], L::kTile);
          for (int bx = 0; bx < NBOX; ++bx)
            tma_load_3d(smem + L::kK + s * L::kTile + bx * L::kBox, &kmap, bx * 64, hkv, kt * kBN,
                        &k_full[s]);
          if (n > 0 && !mbar_wait(&v_empty[s], (n - 1) & 1, lim, p.status)) { ok = false; break; }
          mbar_arrive_expect_tx(&v_full[s], L::kTile);
          for (int bx = 0; bx < NBOX; ++bx)
            tma_load_3d(smem + L::kV + s * L::kTile + bx * L::kBox, &vmap, bx * 64, hkv, kt * kBN,
                        &v_full[s]);
          ++kv_use;
        }
        if (!ok) break;
      }
    } else if (kPaged && warp == 2) {
      // ------------------------------------------------------------ page writer
      page_writer<D>(p, total, [&](int idx) { return pair_tile_at(p, idx); }, lane);
    } else if (warp == 1 && lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      constexpr uint32_t idesc_s = tc::idesc_bf16_f32(kBM, kBN, false, false);
      constexpr uint32_t idesc_pv = tc::idesc_bf16_f32(kBM, D, false, true);
      const uint32_t q_addr = smem_u32(smem + L::kQ);
      int q_use = 0, kv_base = 0, pcount = 0, tile_count = 0;
      bool ok = true;
      for (int r = 0; ok; ++r) {
        const int idx = cta_tile(r, blockIdx.x, grid);
        if (idx >= total) break;
        const TileRef t = pair_tile_at(p, idx);
        const KvRange kr = kv_range(p, p.kv_kind[t.hq / p.G], t.qt);
        const int nkv = kr.count();
        if (!mbar_wait(q_full, q_use & 1, lim, p.status)) break;
        ++q_use;
        tc::fence_after();
        // S_x(j) = Q_x K_j^T; K_j is released after head B's product
        auto issue_s = [&](int x, int j) -> bool {
          const int kvi = kv_base + j, s = kvi & 1, n = kvi >> 1;
          if (x == 0) {
            if (!mbar_wait(&k_full[s], n & 1, lim, p.status)) return false;
            tc::fence_after();
          }
          const uint32_t k_addr = smem_u32(smem + L::kK + s * L::kTile);
          const uint32_t qa = q_addr + x * L::kTile;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk / 4) * L::kBox + (kk % 4) * 32;
            tc::mma_ss(tmem_s(x), tc::smem_desc_sw128(qa + off, 16, 1024),
                       tc::smem_desc_sw128(k_addr + off, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
          }
          tc::commit(&s_full[x]);
          if (x == 1) {
            tc::commit(&k_empty[s]);
            if (j == nkv - 1) tc::commit(q_empty);
          }
          return true;
        };
        // O_x += P_x(j) V_j, P from tensor memory; V_j is released after head B's product
        auto issue_pv = [&](int x, int j) -> bool {
          const int kvi = kv_base + j, s = kvi & 1, n = kvi >> 1;
          if (!mbar_wait(&p_full[x], pcount & 1, lim, p.status)) return false;
          if (j == 0 && tile_count > 0 && !mbar_wait(&o_free[x], (tile_count - 1) & 1, lim, p.status))
            return false;
          if (x == 0 && !mbar_wait(&v_full[s], n & 1, lim, p.status)) return false;
          tc::fence_after();
          const uint32_t v_addr = smem_u32(smem + L::kV + s * L::kTile);
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk)  // 16 keys = 8 columns of P per step
            tc::mma_ts(tmem_o(x), tmem_s(x) + kk * 8,
                       tc::smem_desc_sw128(v_addr + kk * 16 * 128, L::kBox, 1024), idesc_pv,
                       (j > 0 || kk > 0) ? 1u : 0u);
          if (x == 1) tc::commit(&v_empty[s]);
          if (j == nkv - 1) tc::commit(&pv_done[x]);
          return true;
        };
        ok = issue_s(0, 0) && issue_s(1, 0);
        for (int j = 0; j < nkv && ok; ++j) {
          ok = issue_pv(0, j);
          if (ok && j + 1 < nkv) ok = issue_s(0, j + 1);
          if (ok) ok = issue_pv(1, j);
          if (ok && j + 1 < nkv) ok = issue_s(1, j + 1);
          ++pcount;
        }
        kv_base += nkv;
        ++tile_count;
      }
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kPairRegsSoft));
    // ------------------------------------------------------------ softmax
    const int x = (warp - 4) >> 2;             // head of the pair
    const int quad = warp & 3;                 // TMEM lane quarter of this warp
    const int row = quad * 32 + lane;          // query row within the tile
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    int jcount = 0, tile_count = 0;
    bool ok = true;
    for (int r = 0; ok; ++r) {
      const int idx = cta_tile(r, blockIdx.x, grid);
      if (idx >= total) break;
      const TileRef t = pair_tile_at(p, idx);
      const int hq = t.hq + x;
      const int kind = p.kv_kind[t.hq / p.G];
      const KvRange kr = kv_range(p, kind, t.qt);
      const int nkv = kr.count();
      const int q = t.qt * kBM + row;
      float m = -INFINITY, l = 0.f;
      for (int j = 0; j < nkv; ++j) {
        const int kt = kr.at(j);
        // S_j (its commit also covers PV_{j-1}: P's columns and O are free)
        if (!warp_wait(&s_full[x], jcount & 1, lim, p.status)) { ok = false; break; }
        tc::fence_after();
        float xs[kBN];
#pragma unroll
        for (int c = 0; c < kBN / 32; ++c) {
          uint32_t u[32];
          tc::ld32(tmem_s(x) + lane_off + c * 32, u);
          tc::wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) xs[c * 32 + i] = __uint_as_float(u[i]);
        }
        const bool need_mask = kt == t.qt || (kt + 1) * kBN > p.T || (kind == 1 && p.mask_block < kBN);
        if (need_mask) {
          const int qb = q / p.mask_block;
#pragma unroll
          for (int i = 0; i < kBN; ++i) {
            const int k = kt * kBN + i;
            const int kb = k / p.mask_block;
            const bool allowed = k <= q && k < p.T &&
                                 (kind == 0 || kb < p.sink_blocks || qb - kb < p.local_blocks);
            if (!allowed) xs[i] = -INFINITY;
          }
        }
        float mt8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) mt8[i] = xs[i];
#pragma unroll
        for (int i = 8; i < kBN; ++i) mt8[i & 7] = fmaxf(mt8[i & 7], xs[i]);
        const float mt = fmaxf(fmaxf(fmaxf(mt8[0], mt8[1]), fmaxf(mt8[2], mt8[3])),
                               fmaxf(fmaxf(mt8[4], mt8[5]), fmaxf(mt8[6], mt8[7])));
        const float m_new = fmaxf(m, mt * p.scale_log2);
        float alpha = 1.f;
        bool rescale = false;
        if (j == 0) {
          m = m_new;
        } else if (m_new > m + kRescaleLog2) {
          alpha = tc::ex2(m - m_new);
          m = m_new;
          rescale = true;
        }
        const float mu = (m == -INFINITY) ? 0.f : m;
        float rs8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) rs8[i] = 0.f;
#pragma unroll
        for (int i = 0; i < kBN; ++i) {
          xs[i] = tc::ex2(fmaf(xs[i], p.scale_log2, -mu));
          rs8[i & 7] += xs[i];
        }
        l = l * alpha + (((rs8[0] + rs8[1]) + (rs8[2] + rs8[3])) + ((rs8[4] + rs8[5]) + (rs8[6] + rs8[7])));
        if (rescale) {  // PV_{j-1} has completed (see above): O may be rescaled
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t u[32];
            tc::ld32(tmem_o(x) + lane_off + c * 32, u);
            tc::wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) u[i] = __float_as_uint(__uint_as_float(u[i]) * alpha);
            tc::st32(tmem_o(x) + lane_off + c * 32, u);
          }
        }
        // P_j over the first kBN / 2 columns of S_j (S_j is in registers now)
#pragma unroll
        for (int c = 0; c < kBN / 64; ++c) {
          uint32_t u[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) u[i] = float2_to_bf16x2(xs[c * 64 + 2 * i], xs[c * 64 + 2 * i + 1]);
          tc::st32(tmem_s(x) + lane_off + c * 32, u);
        }
        tc::wait_st();
        tc::fence_before();
        mbar_arrive(&p_full[x]);
        ++jcount;
      }
      if (!ok) break;
      // ---- epilogue: O / l -> bf16, log-sum-exp
      if (!warp_wait(&pv_done[x], tile_count & 1, lim, p.status)) break;
      tc::fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      __nv_bfloat16* orow = p.out + ((size_t)q * p.H_q + hq) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t u[32];
        tc::ld32(tmem_o(x) + lane_off + c * 32, u);
        tc::wait_ld();
        if (q < p.T) {
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 w;
            w.x = float2_to_bf16x2(__uint_as_float(u[v * 8 + 0]) * inv, __uint_as_float(u[v * 8 + 1]) * inv);
            w.y = float2_to_bf16x2(__uint_as_float(u[v * 8 + 2]) * inv, __uint_as_float(u[v * 8 + 3]) * inv);
            w.z = float2_to_bf16x2(__uint_as_float(u[v * 8 + 4]) * inv, __uint_as_float(u[v * 8 + 5]) * inv);
            w.w = float2_to_bf16x2(__uint_as_float(u[v * 8 + 6]) * inv, __uint_as_float(u[v * 8 + 7]) * inv);
            *reinterpret_cast<uint4*>(orow + c * 32 + v * 8) = w;
          }
        }
      }
      if (p.lse != nullptr && q < p.T)
        p.lse[(size_t)hq * p.T + q] = l > 0.f ? (m + __log2f(l)) * 0.69314718055994530942f : -INFINITY;
      tc::fence_before();
      mbar_arrive(&o_free[x]);
      ++tile_count;
    }
  }
  tc::fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after();
    tc::dealloc(tmem, 512);
  }
}

// --- host side ------------------------------------------------------------------

static bool make_map_3d(CUtensorMap* m, const void* base, uint64_t T, uint64_t H, uint64_t D) {
  // [T][H][D] bf16, box = 64 channels x 1 head x 128 tokens, 128-byte swizzle
  return make_map_tiled(m, base, 3, D, H, T, 64, 1, 128);
}

size_t prefill_workspace_bytes(const lserve_prefill_desc* d) {
  (void)d;
  return 0;  // the schedule is closed-form; nothing to stage
}

int prefill_entry(const lserve_prefill_desc* d, const void* q, const void* k, const void* v,
                  const uint8_t* head_kind_host, float softmax_scale, void* out, float* lse,
                  void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  return prefill_paged_entry(d, nullptr, q, k, v, head_kind_host, softmax_scale, out, lse, nullptr,
                             nullptr, nullptr, nullptr, workspace, workspace_bytes, stream);
}

int prefill_paged_entry(const lserve_prefill_desc* d, const lserve_paged_desc* pd, const void* q,
                        const void* k, const void* v, const uint8_t* head_kind_host,
                        float softmax_scale, void* out, float* lse, const int32_t* block_table,
                        void* k_pool, void* v_pool, void* stats_pool, void* workspace,
                        size_t workspace_bytes, cudaStream_t stream) {
  (void)workspace;
  (void)workspace_bytes;
  if (!d || !q || !k || !v || !head_kind_host || !out) return LSERVE_ERR_INVALID_ARG;
  if (d->seq_len < 1 || d->num_kv_heads < 1 || d->num_q_heads < d->num_kv_heads ||
      d->num_q_heads % d->num_kv_heads)
    return LSERVE_ERR_INVALID_ARG;
  if (d->block_q != d->block_k || d->sink_blocks < 0 || d->local_blocks < 1)
    return LSERVE_ERR_INVALID_ARG;
  if (!(softmax_scale > 0.f) || !std::isfinite(softmax_scale)) return LSERVE_ERR_INVALID_ARG;
  auto al = [](const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15) == 0; };
  if (!al(q) || !al(k) || !al(v) || !al(out) || (lse && (reinterpret_cast<uintptr_t>(lse) & 3)))
    return LSERVE_ERR_INVALID_ARG;
  if (d->head_dim != 64 && d->head_dim != 128) return LSERVE_ERR_UNSUPPORTED;
  if (d->block_q != 64 && d->block_q != 128) return LSERVE_ERR_UNSUPPORTED;
  if (d->num_q_heads > kMaxHeads || d->num_kv_heads > kMaxHeads) return LSERVE_ERR_UNSUPPORTED;
  for (int h = 0; h < d->num_kv_heads; ++h)
    if (head_kind_host[h] > 1) return LSERVE_ERR_INVALID_ARG;

  PrefillParams p;
  memset(&p, 0, sizeof(p));
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.status = device_status_word();
  if (!p.status) return LSERVE_ERR_CUDA;
  p.wait_limit = wait_limit();
  p.scale_log2 = softmax_scale * 1.4426950408889634f;
  p.T = d->seq_len;
  p.H_q = d->num_q_heads;
  p.H_kv = d->num_kv_heads;
  p.G = d->num_q_heads / d->num_kv_heads;
  p.mask_block = d->block_q;
  p.sink_blocks = d->sink_blocks;
  p.local_blocks = d->local_blocks;
  p.n_qt = (d->seq_len + kBM - 1) / kBM;
  for (int h = 0; h < d->num_kv_heads; ++h) p.kv_kind[h] = head_kind_host[h];
  for (int hq = 0; hq < d->num_q_heads; ++hq) {
    if (head_kind_host[hq / p.G] == 0)
      p.dense_heads[p.n_dense++] = (uint8_t)hq;
    else
      p.stream_heads[p.n_stream++] = (uint8_t)hq;
  }
  const bool paired = p.G % 2 == 0;  // two query heads of one KV head per work tile
  if (paired) {
    for (int hq = 0; hq < d->num_q_heads; hq += 2) {
      if (head_kind_host[hq / p.G] == 0)
        p.dense_pairs[p.n_dense_pairs++] = (uint8_t)hq;
      else
        p.stream_pairs[p.n_stream_pairs++] = (uint8_t)hq;
    }
  }
  CUtensorMap qm, km, vm;
  if (!make_map_3d(&qm, q, d->seq_len, d->num_q_heads, d->head_dim) ||
      !make_map_3d(&km, k, d->seq_len, d->num_kv_heads, d->head_dim) ||
      !make_map_3d(&vm, v, d->seq_len, d->num_kv_heads, d->head_dim))
    return LSERVE_ERR_CUDA;
  if (pd) {
    p.pg_k_in = static_cast<const __nv_bfloat16*>(k);
    p.pg_v_in = static_cast<const __nv_bfloat16*>(v);
    p.pg_k_pool = static_cast<__nv_bfloat16*>(k_pool);
    p.pg_v_pool = static_cast<__nv_bfloat16*>(v_pool);
    p.pg_stats = static_cast<__nv_bfloat16*>(stats_pool);
    p.pg_block_table = block_table;
    p.pg_np = pd->physical_page;
    p.pg_nl = pd->logical_page;
    p.pg_max_pages = pd->max_pages_per_seq;
    p.pg_num_pool_pages = pd->num_pool_pages;
  }
  const int sms = current_sm_count();
  if (sms <= 0) return LSERVE_ERR_CUDA;
  const int tiles = (paired ? d->num_q_heads / 2 : d->num_q_heads) * p.n_qt;
  const int grid = tiles < sms ? tiles : sms;
  cudaError_t e;
  // more than half of the SM's shared memory: one CTA per SM, so the 512-column
  // tensor-memory allocation never waits on a co-resident CTA
  const int kOneCtaSmem = 118 * 1024;
  if (paired) {
    // 512 tensor-memory columns: one CTA per SM (its shared memory alone guarantees that)
    if (d->head_dim == 128) {
      const int smem = std::max(PairLayout<128>::kBytes + 1024, kOneCtaSmem);
      e = set_smem_once(pd ? (const void*)prefill_pair_kernel<128, true> : (const void*)prefill_pair_kernel<128, false>, smem);
      if (e != cudaSuccess) return LSERVE_ERR_CUDA;
      if (pd) prefill_pair_kernel<128, true><<<grid, kPairThreads, smem, stream>>>(p, qm, km, vm);
      else prefill_pair_kernel<128, false><<<grid, kPairThreads, smem, stream>>>(p, qm, km, vm);
    } else {
      const int smem = std::max(PairLayout<64>::kBytes + 1024, kOneCtaSmem);
      e = set_smem_once(pd ? (const void*)prefill_pair_kernel<64, true> : (const void*)prefill_pair_kernel<64, false>, smem);
      if (e != cudaSuccess) return LSERVE_ERR_CUDA;
      if (pd) prefill_pair_kernel<64, true><<<grid, kPairThreads, smem, stream>>>(p, qm, km, vm);
      else prefill_pair_kernel<64, false><<<grid, kPairThreads, smem, stream>>>(p, qm, km, vm);
    }
  } else if (d->head_dim == 128) {
    const int smem = std::max(Layout<128>::kBytes + 1024, kOneCtaSmem);
    e = set_smem_once(pd ? (const void*)prefill_kernel<128, true> : (const void*)prefill_kernel<128, false>, smem);
    if (e != cudaSuccess) return LSERVE_ERR_CUDA;
    if (pd) prefill_kernel<128, true><<<grid, kThreads, smem, stream>>>(p, qm, km, vm);
    else prefill_kernel<128, false><<<grid, kThreads - 32, smem, stream>>>(p, qm, km, vm);
  } else {
    const int smem = std::max(Layout<64>::kBytes + 1024, kOneCtaSmem);
    e = set_smem_once(pd ? (const void*)prefill_kernel<64, true> : (const void*)prefill_kernel<64, false>, smem);
    if (e != cudaSuccess) return LSERVE_ERR_CUDA;
    if (pd) prefill_kernel<64, true><<<grid, kThreads, smem, stream>>>(p, qm, km, vm);
    else prefill_kernel<64, false><<<grid, kThreads - 32, smem, stream>>>(p, qm, km, vm);
  }
  return cudaGetLastError() == cudaSuccess ? LSERVE_OK : LSERVE_ERR_CUDA;
}

}  // namespace lserve
