// Internal launch interface between the C-ABI layer (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace lserve {

constexpr int kStatsWarps = 8;   // warps per CTA of the stats kernel
constexpr int kScoreWarps = 4;   // warps per CTA of the score kernel (6 CTAs per SM)
constexpr int kScorePagesPerWarp = 4;
constexpr int kScoreSteps = 2;        // warp steps (of 32 / (D/8) logical pages) loaded at once
constexpr int kTopkThreads = 512;
constexpr int kTopkMaxPages = 32768;
constexpr int kTopkCand = 128;       // bucket size ranked pairwise

struct StatsParams {
  const __nv_bfloat16* k_pool;
  const int32_t* block_table;
  const int32_t* ctx_lens;
  const uint8_t* head_kind;
  __nv_bfloat16* stats_pool;
  unsigned int* status;
  int batch, num_kv_heads, logical_page, physical_page, max_pages, num_pool_pages;
  int first_logical_page;
};

struct SelectParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* stats_pool;
  const int32_t* block_table;
  const int32_t* ctx_lens;
  const uint8_t* head_kind;
  float* scores;          // [B][H_kv][max_pages]
  int32_t* sel;           // [B][H_kv][top_k]
  int32_t* sel_count;     // [B][H_kv]
  unsigned int* status;
  int batch, num_q_heads, num_kv_heads, logical_page, physical_page, max_pages, num_pool_pages;
  int top_k;
};

// Decode split: tiles of up to 64 tokens (a physical page, or a 64-token part of
// a larger one); the tiles of all (sequence, KV head) pairs are laid end to end
// and cut into equal contiguous ranges, one per CTA of a persistent grid.
constexpr int kDecodeTileMax = 64;
constexpr int kDecodeMaxPairs = 2048;   // B * H_kv
#ifndef LSERVE_DECODE_MIN_TILES
#define LSERVE_DECODE_MIN_TILES 4
#endif
constexpr int kDecodeMinTiles = LSERVE_DECODE_MIN_TILES;  // tiles per CTA the grid aims at, at least

struct DecodeParams {
  const __nv_bfloat16* q;
  const int32_t* block_table;
  const int32_t* ctx_lens;
  const uint8_t* head_kind;
  const int32_t* sel;
  const int32_t* sel_count;
  __nv_bfloat16* out;     // bf16 [B][H_q][D], or null when out_f32 is set
  float* out_f32;         // float [B][H_q][D] instead (LSERVE_DECODE_OUT_F32)
  float* lse;
  // Split pairs (workspace).  A CTA writes at most one partial: the part of
  // its first pair that began in an earlier CTA.  Each word is 8 bytes, a
  // float value in the low half and a tag in the high half (one single-copy
  // atomic store), so the merging CTA can poll the words themselves.
  uint32_t* epochs;              // [P]: epoch of the pair's last split merge
  unsigned long long* parts;     // [grid][G*D + 2*G]: o[G][D], m[G], l[G] words
  unsigned int* status;
  int batch, num_q_heads, num_kv_heads, physical_page, max_pages, num_pool_pages;
  int top_k, sink, local;
  int tile_rows;          // tokens per tile (decode_tile_rows)
  int tiles_per_page;
  int consumer_warps;     // 8: one CTA per SM; 4: two co-resident CTAs per SM
  float scale_log2;       // softmax_scale * log2(e)
  uint64_t wait_limit;
  int overlap_prologue;   // plan + first lookups may run before the preceding kernel ends
  int prefetch_kv;        // the first stages' KV copies too (the preceding kernel writes no page)
  // quantized cache (lserve_sparse_decode_attn_kv8 / _kv4): codes [pool rows]
  // [D] bytes (8-bit) or [D/2] bytes (4-bit, two per byte) and float scales
  // [num_pool_pages][H_kv][D]; null for the bf16 cache
  const int8_t* k8;
  const int8_t* v8;
  const float* k_scale;
  const float* v_scale;
  // lserve_decode_step: the new token of sequence b sits at position
  // ctx_lens[b] - 1; its K / V rows (k_new / v_new, bf16 [B][H_kv][D]) are
  // written to the pools and the retrieval heads' page statistics in this
  // launch and attended from k_new / v_new (null: no append)
  const __nv_bfloat16* k_new;
  const __nv_bfloat16* v_new;
  __nv_bfloat16* k_pool_w;
  __nv_bfloat16* v_pool_w;
  __nv_bfloat16* stats_w;
  int logical_page;
  // retrieval heads also attend positions [recent_from[b], ctx_lens[b]) (null: off)
  const int32_t* recent_from;
};

// lserve_decode_append: one warp per (sequence, KV head)
constexpr int kAppendWarps = 8;
struct AppendParams {
  const __nv_bfloat16* k_new;   // [B][H_kv][D]
  const __nv_bfloat16* v_new;   // [B][H_kv][D]
  const int32_t* block_table;
  const int32_t* ctx_lens;      // position of the new token of each sequence
  const uint8_t* head_kind;
  __nv_bfloat16* k_pool;
  __nv_bfloat16* v_pool;
  __nv_bfloat16* stats_pool;
  unsigned int* status;
  int batch, num_kv_heads, logical_page, physical_page, max_pages, num_pool_pages;
};
cudaError_t launch_decode_append(const AppendParams& p, int D, cudaStream_t stream);

// lserve_prefill_to_pages: one warp per (logical page, KV head)
constexpr int kToPagesWarps = 8;
struct ToPagesParams {
  const __nv_bfloat16* k;      // [T][H_kv][D]
  const __nv_bfloat16* v;      // [T][H_kv][D]
  const int32_t* block_table;  // [max_pages] of this sequence
  const uint8_t* head_kind;
  __nv_bfloat16* k_pool;
  __nv_bfloat16* v_pool;
  __nv_bfloat16* stats_pool;
  unsigned int* status;
  int seq_len, num_kv_heads, logical_page, physical_page, max_pages, num_pool_pages;
};
cudaError_t launch_prefill_to_pages(const ToPagesParams& p, int D, cudaStream_t stream);

// lserve_quantize_pages_kv8: one CTA per (page of a sequence, KV head, K or V)
struct QuantParams {
  const __nv_bfloat16* k_pool;
  const __nv_bfloat16* v_pool;
  const int32_t* block_table;
  const int32_t* ctx_lens;
  int8_t* k_pool8;
  int8_t* v_pool8;
  float* k_scale;   // [num_pool_pages][H_kv][D]
  float* v_scale;
  unsigned int* status;
  int batch, num_kv_heads, physical_page, max_pages, num_pool_pages;
};
cudaError_t launch_quantize_kv(const QuantParams& p, int D, int bits, cudaStream_t stream);

// Sequence-sharded decode (seq_shard.cu): shard `rank` of `num_shards` holds
// pages [floor(M*rank/N), floor(M*(rank+1)/N)) of each sequence.
struct ShardParams {
  const int32_t* ctx_lens;     // GLOBAL sequence lengths [B]
  const uint8_t* head_kind;    // [H_kv]
  // candidates: the shard's own selection
  const int32_t* sel;          // [B][H_kv][sel_stride] shard-local page ordinals
  const int32_t* sel_count;    // [B][H_kv]
  const float* scores;         // [B][H_kv][max_pages] shard-local physical scores
  float* cand_score;           // candidates' output [B][H_kv][top_k]
  int32_t* cand_page;          // global page ordinals, -1 = none
  const float* all_score;      // merge's input: the gathered proposals [N][B][H_kv][top_k]
  const int32_t* all_page;
  // merge: the shard's pages of the global choice
  int32_t* out_sel;            // [B][H_kv][out_stride] shard-local ordinals, ascending, -1 padded
  int32_t* out_count;          // [B][H_kv]
  unsigned int* status;
  int batch, num_kv_heads, physical_page, max_pages, top_k, sel_stride, out_stride;
  int rank, num_shards, sink, local;
};
struct CombineParams {
  const float* o_parts;        // [N][rows][D]
  const float* lse_parts;      // [N][rows]
  __nv_bfloat16* out;          // [rows][D]
  float* lse;                  // [rows] or null
  int num_shards, rows, head_dim;
};
cudaError_t launch_seqshard_candidates(const ShardParams& p, cudaStream_t stream);
cudaError_t launch_seqshard_merge(const ShardParams& p, cudaStream_t stream);
cudaError_t launch_seqshard_combine(const CombineParams& p, cudaStream_t stream);

cudaError_t launch_page_stats(const StatsParams& p, int D, int max_logical_pages,
                              cudaStream_t stream);
cudaError_t launch_page_select(const SelectParams& p, int D, cudaStream_t stream);
cudaError_t launch_decode(const DecodeParams& p, const CUtensorMap& kmap, const CUtensorMap& vmap,
                          int D, int G, int grid, cudaStream_t stream);
// the quantized-cache variants, bits = 8 or 4 (p.k8 / p.v8 / p.k_scale / p.v_scale
// set; no tensor maps)
cudaError_t launch_decode_quant(const DecodeParams& p, const CUtensorMap& kmap,
                                const CUtensorMap& vmap, int D, int G, int bits, int grid,
                                cudaStream_t stream);
size_t decode_workspace_bytes(int pairs, int grid, int G, int D);
int decode_grid(int sm_count);
int decode_consumer_warps();
int decode_tile_rows(int physical_page);

cudaError_t launch_wait_timeout_probe(uint64_t cycles, unsigned int* status, cudaStream_t stream);

// Raises a kernel's dynamic shared memory limit once per (kernel, device), so
// that later calls (e.g. during CUDA-graph capture) launch without it.
cudaError_t set_smem_once(const void* kernel, int bytes);

// host helpers shared by the entry points (api.cu)
bool make_map_2d(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint64_t pitch_elems,
                 uint32_t box_rows);
bool make_map_tiled(CUtensorMap* m, const void* base, int rank, uint64_t d0, uint64_t d1, uint64_t d2,
                    uint32_t b0, uint32_t b1, uint32_t b2);
bool make_map_codes(CUtensorMap* m, const void* base, uint64_t rows, uint32_t row_bytes,
                    uint32_t box_rows);
uint64_t wait_limit();
int current_sm_count();
unsigned int* device_status_word();

}  // namespace lserve
