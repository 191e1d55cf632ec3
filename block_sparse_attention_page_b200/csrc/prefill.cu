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
//   warp 6     page writer (lserve_blocksparse_prefill_paged only): the
//              diagonal key tile of each KV head into the paged pools and the
//              page statistics, while the tile is in its ring stage.
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
  // paged epilogue (lserve_blocksparse_prefill_paged; pg_k_pool == nullptr: none)
  __nv_bfloat16* pg_k_pool;
  __nv_bfloat16* pg_v_pool;
  __nv_bfloat16* pg_stats;
  const int32_t* pg_block_table;  // this sequence's page ordinal -> pool id
  int pg_np, pg_nl, pg_box_rows, pg_max_pages, pg_num_pool_pages;
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
  static constexpr int kNumBars = 19;
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

// Paged epilogue of one key tile (row kt of KV head h), run by the whole
// producer warp while the tile is still in its ring stage: K and V rows
// [kt*kBN, min(kt*kBN + kBN, T)) go to the pools through the block table --
// whole boxes of pg_box_rows rows by TMA stores, the rows of a page that the
// sequence fills only partly by plain stores of its valid rows -- and, for a
// retrieval head, every logical page of the tile gets the bf16 min / max of
// its valid keys per channel (the same values lserve_page_stats and
// lserve_prefill_to_pages write).  Returns after the TMA stores have read the
// stage.  ks / vs: the stage's K and V tiles (NBOX swizzled 128-row boxes).
template <int D>
__device__ void page_out(const PrefillParams& p, const CUtensorMap* kpm, const CUtensorMap* vpm,
                         const uint8_t* ks, const uint8_t* vs, int kt, int h, int lane) {
  constexpr int NBOX = D / 64;
  constexpr int kBoxBytes = kBM * 128;
  constexpr int CPL = D / 32;  // channels of a lane in the statistics (4 or 2)
  const int t0 = kt * kBN, tend = min(t0 + kBN, p.T);
  const int NP = p.pg_np, NL = p.pg_nl, BR = p.pg_box_rows, g = NP / NL;
  // byte offset of channel c of tile row r in a stage (128-byte swizzle per box)
  auto off = [&](int r, int c) {
    const int chunk = (c % 64) / 8;
    return (uint32_t)((c / 64) * kBoxBytes + r * 128 + ((chunk ^ (r & 7)) << 4) + (c % 8) * 2);
  };
  bool issued = false;
  // the tile's block-table entries (at most kBN / 32 pages), one lane each, in one round trip
  const int m0 = t0 / NP;
  int pid_l = -1;
  if (m0 + lane < p.pg_max_pages && (m0 + lane) * NP < tend) pid_l = p.pg_block_table[m0 + lane];
  for (int m = m0; m * NP < tend; ++m) {
    const int a = max(t0, m * NP) - t0, e = min(tend, (m + 1) * NP) - t0;  // tile rows [a, e)
    const int pid = __shfl_sync(0xffffffffu, pid_l, m - m0);
    if (pid < 0 || pid >= p.pg_num_pool_pages) {
      if (lane == 0) raise_status(p.status, LSERVE_ERR_BOUNDS);
      continue;
    }
    const size_t prow = ((size_t)pid * p.H_kv + h) * NP + (size_t)(t0 + a - m * NP);  // pool row of a
    if ((e - a) % BR == 0) {
      if (lane == 0) {
        fence_proxy_async_smem();  // the copies below read what the tile loads wrote
        // evict-first: the pools are not read again by this kernel, the K / V
        // tiles that later query tiles re-read should keep their L2 lines
        const uint64_t pol = l2_policy_evict_first();
        for (int r = a; r < e; r += BR)
          for (int bx = 0; bx < NBOX; ++bx) {
            tma_store_3d_hint(kpm, 0, bx, (int32_t)(prow + (r - a)), ks + bx * kBoxBytes + r * 128, pol);
            tma_store_3d_hint(vpm, 0, bx, (int32_t)(prow + (r - a)), vs + bx * kBoxBytes + r * 128, pol);
          }
      }
      issued = true;
    } else {  // the sequence's last, partly filled page: its valid rows
      for (int i = lane; i < (e - a) * (D / 8); i += 32) {
        const int r = a + i / (D / 8), c = (i % (D / 8)) * 8;
        const size_t dst = (prow + (size_t)(r - a)) * D + c;
        *reinterpret_cast<uint4*>(p.pg_k_pool + dst) = *reinterpret_cast<const uint4*>(ks + off(r, c));
        *reinterpret_cast<uint4*>(p.pg_v_pool + dst) = *reinterpret_cast<const uint4*>(vs + off(r, c));
      }
    }
    if (p.kv_kind[h] != 0) continue;  // streaming heads need no statistics
    for (int lp = (t0 + a) / NL; lp * NL < t0 + e; ++lp) {
      const int ra = lp * NL - t0, rb = min((lp + 1) * NL, tend) - t0;
      const uint32_t kPosInf2 = 0x7F807F80u, kNegInf2 = 0xFF80FF80u;
      __nv_bfloat162 mn[CPL / 2], mx[CPL / 2];
#pragma unroll
      for (int k = 0; k < CPL / 2; ++k) {
        mn[k] = *reinterpret_cast<const __nv_bfloat162*>(&kPosInf2);
        mx[k] = *reinterpret_cast<const __nv_bfloat162*>(&kNegInf2);
      }
      for (int r = ra; r < rb; ++r) {
#pragma unroll
        for (int k = 0; k < CPL / 2; ++k) {
          const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(ks + off(r, lane * CPL + 2 * k));
          mn[k] = __hmin2(mn[k], v);
          mx[k] = __hmax2(mx[k], v);
        }
      }
      __nv_bfloat16* st = p.pg_stats + ((((size_t)pid * p.H_kv + h) * g) + (lp - m * g)) * 2 * D + lane * CPL;
#pragma unroll
      for (int k = 0; k < CPL / 2; ++k) {
        reinterpret_cast<__nv_bfloat162*>(st)[k] = mn[k];
        reinterpret_cast<__nv_bfloat162*>(st + D)[k] = mx[k];
      }
    }
  }
  if (issued && lane == 0) {
    bulk_commit();
    bulk_wait_read();  // the stage may be refilled
  }
  __syncwarp();
}

// The page writer warp: follows the CTA's work tiles as the producer deals
// them (the same tile order and key-tile counts), and for every tile of a KV
// head's first query head writes the pages of its diagonal key tile -- the
// row's last key tile -- as soon as that tile's K and V have landed, then
// arrives on pg_done[stage].  The producer waits on pg_done before it refills
// that stage, so the tile stays in shared memory until it is written.  The
// MMA and softmax warps never wait on it.
// kv_issued[s]: fills of stage s the producer has issued.  A parity wait only
// tells phases apart within one phase of the barrier's current one, so the
// writer (which may run ahead of the producer) first waits until its tile's
// fill has been issued; the producer cannot refill the stage after it until
// the writer releases it, so that fill's phase is then the barrier's current
// or just-completed one.
template <int D, typename L, typename TileAt>
__device__ void page_writer(const PrefillParams& p, const CUtensorMap* kpm, const CUtensorMap* vpm,
                            uint8_t* smem, uint64_t* k_full, uint64_t* v_full, uint64_t* pg_done,
                            const volatile uint32_t* kv_issued, int total, TileAt tile_of, int lane) {
  const uint64_t lim = p.wait_limit;
  // waits by lane 0 alone (the other lanes idle at the broadcast)
  auto wait_issued = [&](int s, uint32_t want) -> bool {
    bool ok = true;
    if (lane == 0) {
      const long long t0 = clock64();
      while (kv_issued[s] < want) {
        if ((uint64_t)(clock64() - t0) > lim) {
          raise_status(p.status, LSERVE_ERR_TIMEOUT);
          ok = false;
          break;
        }
      }
    }
    return __shfl_sync(0xffffffffu, ok, 0);
  };
  auto wait1 = [&](uint64_t* bar, uint32_t parity) -> bool {
    bool ok = true;
    if (lane == 0) ok = mbar_wait(bar, parity, lim, p.status);
    return __shfl_sync(0xffffffffu, ok, 0);
  };
  int kv_use = 0;
  for (int r = 0;; ++r) {
    const int idx = cta_tile(r, blockIdx.x, gridDim.x);
    if (idx >= total) break;
    const TileRef t = tile_of(idx);
    const int hkv = t.hq / p.G;
    kv_use += kv_range(p, p.kv_kind[hkv], t.qt).count();
    if (t.hq % p.G != 0) continue;
    const int kvi = kv_use - 1, s = kvi & 1, n = kvi >> 1;
    if (!wait_issued(s, (uint32_t)n + 1) || !wait1(&k_full[s], n & 1) || !wait1(&v_full[s], n & 1))
      break;
    page_out<D>(p, kpm, vpm, smem + L::kK + s * L::kTile, smem + L::kV + s * L::kTile, t.qt, hkv, lane);
    if (lane == 0) mbar_arrive(&pg_done[s]);
  }
  if (lane == 0) bulk_wait_all();  // the pools' TMA writes are complete
}

}  // namespace

template <int D, bool kPaged>
__global__ void __launch_bounds__(kPaged ? kThreads : kThreads - 32, 1)
prefill_kernel(const __grid_constant__ PrefillParams p, const __grid_constant__ CUtensorMap qmap,
               const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
               const __grid_constant__ CUtensorMap kpm, const __grid_constant__ CUtensorMap vpm) {
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
  uint64_t* pg_done = bars + 17;  // [2]: the page writer is done with the stage's tile
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::kBar + L::kNumBars * 8);
  volatile uint32_t* kv_issued = tmem_holder + 1;  // [2]: fills of each stage issued

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    if (kPaged) kv_issued[0] = kv_issued[1] = 0u;
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
      mbar_init(&s_full[s], 1);
      mbar_init(&s_free[s], 128);
      if (kPaged) mbar_init(&pg_done[s], 1);
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
    page_writer<D, L>(p, &kpm, &vpm, smem, k_full, v_full, pg_done, kv_issued, total,
                      [&](int idx) { return tile_at(p, idx); }, lane);
  } else if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    // Lane 0 alone; lanes 1-31 of warp 0 do nothing (they must not fall into
    // the softmax branch below).  With the paged epilogue, a stage that holds
    // a KV head's diagonal key tile (visited once, by the group's first query
    // head) is refilled only after the page writer has released it.
    if (lane == 0) {
      tma_prefetch_desc(&qmap);
      tma_prefetch_desc(&kmap);
      tma_prefetch_desc(&vmap);
      int q_use = 0, kv_use = 0;
      // stage 0 / 1 holds a diagonal tile the page writer has not released yet;
      // ep0 / ep1 count the writer's releases (the pg_done phases) per stage
      bool owe0 = false, owe1 = false;
      int ep0 = 0, ep1 = 0;
      auto wait_writer = [&](int s) -> bool {
        if (!mbar_wait(&pg_done[s], (s ? ep1 : ep0) & 1, lim, p.status)) return false;
        if (s) {
          ++ep1;
          owe1 = false;
        } else {
          ++ep0;
          owe0 = false;
        }
        return true;
      };
      bool ok = true;
      for (int r = 0; ok; ++r) {
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
        const int nkv = kr.count();
        for (int j = 0; j < nkv && ok; ++j) {
          const int kt = kr.at(j);
          const int s = kv_use & 1, n = kv_use >> 1;
          if (n > 0 && !mbar_wait(&k_empty[s], (n - 1) & 1, lim, p.status)) { ok = false; break; }
          if (kPaged && (s ? owe1 : owe0) && !wait_writer(s)) { ok = false; break; }
          mbar_arrive_expect_tx(&k_full[s], L::kTile);
          for (int bx = 0; bx < NBOX; ++bx)
            tma_load_3d(smem + L::kK + s * L::kTile + bx * L::kBox, &kmap, bx * 64, hkv, kt * kBN,
                        &k_full[s]);
          if (n > 0 && !mbar_wait(&v_empty[s], (n - 1) & 1, lim, p.status)) { ok = false; break; }
          mbar_arrive_expect_tx(&v_full[s], L::kTile);
          for (int bx = 0; bx < NBOX; ++bx)
            tma_load_3d(smem + L::kV + s * L::kTile + bx * L::kBox, &vmap, bx * 64, hkv, kt * kBN,
                        &v_full[s]);
          if (kPaged) {
            kv_issued[s] = (uint32_t)n + 1;  // for the page writer
            if (t.hq % p.G == 0 && kt == t.qt) {  // the writer's tile
              if (s) owe1 = true;
              else owe0 = true;
            }
          }
          ++kv_use;
        }
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
  static constexpr int kNumBars = 21;
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
                    const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                    const __grid_constant__ CUtensorMap kpm, const __grid_constant__ CUtensorMap vpm) {
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
  uint64_t* pg_done = bars + 19;  // [2]: the page writer is done with the stage's tile
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::kBar + L::kNumBars * 8);
  volatile uint32_t* kv_issued = tmem_holder + 1;  // [2]: fills of each stage issued

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    if (kPaged) kv_issued[0] = kv_issued[1] = 0u;
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
      if (kPaged) mbar_init(&pg_done[s], 1);
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
    if (!kPaged && warp == 0 && lane == 0) {
      // (the kernel without the paged epilogue)
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
    } else if (kPaged && warp == 0 && lane == 0) {
      // ------------------------------------------------------------ TMA producer
      // A stage holding a diagonal key tile of the paged epilogue is refilled
      // after the page writer (warp 2) releases it, as in prefill_kernel.
      tma_prefetch_desc(&qmap);
      tma_prefetch_desc(&kmap);
      tma_prefetch_desc(&vmap);
      int q_use = 0, kv_use = 0;
      bool owe0 = false, owe1 = false;  // as in prefill_kernel
      int ep0 = 0, ep1 = 0;
      auto wait_writer = [&](int s) -> bool {
        if (!mbar_wait(&pg_done[s], (s ? ep1 : ep0) & 1, lim, p.status)) return false;
        if (s) {
          ++ep1;
          owe1 = false;
        } else {
          ++ep0;
          owe0 = false;
        }
        return true;
      };
      bool ok = true;
      for (int r = 0; ok; ++r) {
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
        const int nkv = kr.count();
        for (int j = 0; j < nkv && ok; ++j) {
          const int kt = kr.at(j);
          const int s = kv_use & 1, n = kv_use >> 1;
          if (n > 0 && !mbar_wait(&k_empty[s], (n - 1) & 1, lim, p.status)) { ok = false; break; }
          if (kPaged && (s ? owe1 : owe0) && !wait_writer(s)) { ok = false; break; }
          mbar_arrive_expect_tx(&k_full[s], L::kTile);
          for (int bx = 0; bx < NBOX; ++bx)
            tma_load_3d(smem + L::kK + s * L::kTile + bx * L::kBox, &kmap, bx * 64, hkv, kt * kBN,
                        &k_full[s]);
          if (n > 0 && !mbar_wait(&v_empty[s], (n - 1) & 1, lim, p.status)) { ok = false; break; }
          mbar_arrive_expect_tx(&v_full[s], L::kTile);
          for (int bx = 0; bx < NBOX; ++bx)
            tma_load_3d(smem + L::kV + s * L::kTile + bx * L::kBox, &vmap, bx * 64, hkv, kt * kBN,
                        &v_full[s]);
          if (kPaged) {
            kv_issued[s] = (uint32_t)n + 1;  // for the page writer
            if (t.hq % p.G == 0 && kt == t.qt) {  // the writer's tile
              if (s) owe1 = true;
              else owe0 = true;
            }
          }
          ++kv_use;
        }
      }
    } else if (kPaged && warp == 2) {
      // ------------------------------------------------------------ page writer
      page_writer<D, L>(p, &kpm, &vpm, smem, k_full, v_full, pg_done, kv_issued, total,
                        [&](int idx) { return pair_tile_at(p, idx); }, lane);
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

static int gcd_int(int a, int b) {
  while (b) {
    const int t = a % b;
    a = b;
    b = t;
  }
  return a;
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
  // paged epilogue: the pools as [rows][D] (3-D: 64 channels, D/64 halves,
  // rows), box = 64 channels x 1 half x gcd(N_P, 128) rows, 128-byte swizzle
  // (a box is a row range of one swizzled 128-row box of the stage)
  CUtensorMap kpm = km, vpm = vm;
  if (pd) {
    const uint64_t rows = (uint64_t)pd->num_pool_pages * pd->num_kv_heads * pd->physical_page;
    const int br = gcd_int(pd->physical_page, kBN);
    if (!make_map_tiled(&kpm, k_pool, 3, 64, d->head_dim / 64, rows, 64, 1, (uint32_t)br) ||
        !make_map_tiled(&vpm, v_pool, 3, 64, d->head_dim / 64, rows, 64, 1, (uint32_t)br))
      return LSERVE_ERR_CUDA;
    p.pg_k_pool = static_cast<__nv_bfloat16*>(k_pool);
    p.pg_v_pool = static_cast<__nv_bfloat16*>(v_pool);
    p.pg_stats = static_cast<__nv_bfloat16*>(stats_pool);
    p.pg_block_table = block_table;
    p.pg_np = pd->physical_page;
    p.pg_nl = pd->logical_page;
    p.pg_box_rows = br;
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
      if (pd) prefill_pair_kernel<128, true><<<grid, kPairThreads, smem, stream>>>(p, qm, km, vm, kpm, vpm);
      else prefill_pair_kernel<128, false><<<grid, kPairThreads, smem, stream>>>(p, qm, km, vm, kpm, vpm);
    } else {
      const int smem = std::max(PairLayout<64>::kBytes + 1024, kOneCtaSmem);
      e = set_smem_once(pd ? (const void*)prefill_pair_kernel<64, true> : (const void*)prefill_pair_kernel<64, false>, smem);
      if (e != cudaSuccess) return LSERVE_ERR_CUDA;
      if (pd) prefill_pair_kernel<64, true><<<grid, kPairThreads, smem, stream>>>(p, qm, km, vm, kpm, vpm);
      else prefill_pair_kernel<64, false><<<grid, kPairThreads, smem, stream>>>(p, qm, km, vm, kpm, vpm);
    }
  } else if (d->head_dim == 128) {
    const int smem = std::max(Layout<128>::kBytes + 1024, kOneCtaSmem);
    e = set_smem_once(pd ? (const void*)prefill_kernel<128, true> : (const void*)prefill_kernel<128, false>, smem);
    if (e != cudaSuccess) return LSERVE_ERR_CUDA;
    if (pd) prefill_kernel<128, true><<<grid, kThreads, smem, stream>>>(p, qm, km, vm, kpm, vpm);
    else prefill_kernel<128, false><<<grid, kThreads - 32, smem, stream>>>(p, qm, km, vm, kpm, vpm);
  } else {
    const int smem = std::max(Layout<64>::kBytes + 1024, kOneCtaSmem);
    e = set_smem_once(pd ? (const void*)prefill_kernel<64, true> : (const void*)prefill_kernel<64, false>, smem);
    if (e != cudaSuccess) return LSERVE_ERR_CUDA;
    if (pd) prefill_kernel<64, true><<<grid, kThreads, smem, stream>>>(p, qm, km, vm, kpm, vpm);
    else prefill_kernel<64, false><<<grid, kThreads - 32, smem, stream>>>(p, qm, km, vm, kpm, vpm);
  }
  return cudaGetLastError() == cudaSuccess ? LSERVE_OK : LSERVE_ERR_CUDA;
}

}  // namespace lserve
