/*
 * lserve.h -- C ABI of liblserve.so: the hot path of LServe-style unified
 * sparse attention on one NVIDIA B200 (sm_100a).
 *
 * Source of the method: the LServe explainer page "MLSys 2025論文解説: LServe —
 * 統一疎アテンションによる長文脈LLM推論の効率化" (arXiv 2502.14866) and the LServe
 * abstract page "LServe: Efficient Long-sequence LLM Serving with Unified Sparse
 * Attention".  Section names below are that explainer's.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - bf16 tensors are IEEE bfloat16 (uint16 storage).  All pointers except
 *    those named *_host are DEVICE pointers owned by the caller; the library
 *    keeps no reference after the call returns and allocates nothing.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Calls only enqueue work; results are ready when the stream is.
 *  - Every call validates its arguments on the host first.  On failure it
 *    returns a non-zero lserve_status and launches nothing.  A launch error
 *    reported by the CUDA runtime returns LSERVE_ERR_CUDA.
 *  - Kernels never trap.  Waits on hardware barriers are bounded; a wait that
 *    runs out sets a device status flag (LSERVE_ERR_TIMEOUT) that
 *    lserve_read_device_status() returns.  Block-table entries, selected page
 *    ordinals and page counts are checked per page: an entry out of range sets
 *    LSERVE_ERR_BOUNDS and the offending page is skipped (never read).
 *  - Stateless and thread-safe, apart from one cached driver entry point and
 *    a per-device cache of the SM count.
 *
 * Paged KV cache layout (the "page" and "block table" of hierarchical paging,
 * 技術的詳細 › 階層的ページング)
 *  - k_pool, v_pool : bf16 [num_pool_pages][H_kv][N_P][D]; one (page, head)
 *                     is N_P * D contiguous elements.
 *  - block_table    : int32 [B][max_pages_per_seq]; entry m is the pool id of
 *                     physical page m (tokens [m*N_P, (m+1)*N_P)) of sequence b.
 *  - ctx_lens       : int32 [B]; n_b, the number of valid tokens of sequence b.
 *                     Tokens at positions >= n_b of the last page are ignored.
 *  - head_kind      : uint8 [H_kv] (device) -- 0 = retrieval head, 1 = streaming
 *                     head (技術的詳細 › 静的スパーシティ).
 *  - stats_pool     : bf16 [num_pool_pages][H_kv][g][2][D], g = N_P / N_L;
 *                     [..][0][:] = k_min, [..][1][:] = k_max of logical page
 *                     (pool page, head, sub-page), indexed by the same pool id.
 *  - q              : bf16 [B][H_q][D]; query head hq uses KV head hq / G,
 *                     G = H_q / H_kv.
 */
#ifndef LSERVE_H_
#define LSERVE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LSERVE_OK = 0,
  LSERVE_ERR_INVALID_ARG = 1, /* null pointer, bad size, misaligned pointer      */
  LSERVE_ERR_UNSUPPORTED = 2, /* valid but not built: e.g. D not in {64, 128}    */
  LSERVE_ERR_WORKSPACE = 3,   /* workspace missing or smaller than required      */
  LSERVE_ERR_CUDA = 4,        /* the CUDA runtime reported an error              */
  LSERVE_ERR_TIMEOUT = 5,     /* a bounded device wait ran out                   */
  LSERVE_ERR_BOUNDS = 6       /* a page index was out of range (page skipped)   */
} lserve_status;

typedef enum { LSERVE_OP_STATS = 0, LSERVE_OP_SELECT = 1, LSERVE_OP_DECODE = 2, LSERVE_OP_PREFILL = 3 } lserve_op;

/* Shapes of the paged decode calls. */
typedef struct {
  int32_t batch;             /* B >= 1                                              */
  int32_t num_q_heads;       /* H_q, a multiple of H_kv                             */
  int32_t num_kv_heads;      /* H_kv >= 1; G = H_q / H_kv in {1, 2, 4, 8}           */
  int32_t head_dim;          /* D in {64, 128}                                      */
  int32_t logical_page;      /* N_L in {8, 16, 32, 64}                              */
  int32_t physical_page;     /* N_P = g * N_L; 32 or a multiple of 64, <= 1024      */
  int32_t max_pages_per_seq; /* row length of block_table                           */
  int32_t num_pool_pages;    /* first dimension of k_pool / v_pool / stats_pool     */
} lserve_paged_desc;

/* Shapes of the prefill call.  Q [T][H_q][D], K/V [T][H_kv][D], O [T][H_q][D]. */
typedef struct {
  int32_t seq_len;      /* T >= 1                                                   */
  int32_t num_q_heads;  /* H_q, a multiple of H_kv                                  */
  int32_t num_kv_heads; /* H_kv                                                     */
  int32_t head_dim;     /* D = 128 (64 also accepted)                               */
  int32_t block_q;      /* query block, == block_k, 128                             */
  int32_t block_k;      /* key block                                                */
  int32_t sink_blocks;  /* Lambda mask: leading blocks every streaming row sees     */
  int32_t local_blocks; /* Lambda mask: blocks [i - local + 1, i] (diagonal counts) */
} lserve_prefill_desc;

/*
 * lserve_page_stats -- channel-wise k_min / k_max of every logical page.
 * [技術的詳細 › 動的スパーシティ: k_min^j[i], k_max^j[i] are the min / max of channel
 *  i over the keys of logical page j; 階層的ページング: logical pages of N_L tokens
 *  inside physical pages of N_P = g * N_L tokens.]
 *
 * For each sequence b, RETRIEVAL head h (streaming heads are skipped) and
 * logical page j >= first_logical_page with j * N_L < n_b, writes k_min and
 * k_max over the valid tokens [j*N_L, min((j+1)*N_L, n_b)) into stats_pool at
 * pool id block_table[b][j / g], sub-page j % g.  Results are exact (min/max of
 * bf16 values).  first_logical_page = 0 rebuilds everything; a larger value
 * refreshes only the pages from there on (e.g. the page a decode step filled).
 * Reads ~n*D*2 bytes of K per (b, h), writes 1/(N_L/2) of that.
 */
int lserve_page_stats(const lserve_paged_desc* desc, const void* k_pool, const int32_t* block_table,
                      const int32_t* ctx_lens, const uint8_t* head_kind, void* stats_pool,
                      int32_t first_logical_page, void* stream);

/*
 * lserve_prefill_to_pages -- hand a prefilled sequence to the paged decode
 * cache: K / V into the pools and the page statistics, in one pass over K.
 * [技術的詳細 › 動的スパーシティ: k_min^j / k_max^j of logical page j; 階層的ページング:
 *  logical pages of N_L tokens inside physical pages of N_P tokens.  The pages
 *  do not say where the statistics are built; building them while K is read
 *  once saves lserve_page_stats' separate pass over the cache.]
 *
 * One sequence of seq_len tokens: k, v bf16 [seq_len][H_kv][D] (the layout
 * lserve_blocksparse_prefill reads), block_table int32 [max_pages_per_seq]
 * (this sequence's page ordinal -> pool id; must cover seq_len tokens).
 * Token t of head h goes to pool id block_table[t / N_P], row t % N_P, of
 * k_pool / v_pool; for retrieval heads every logical page j of the sequence
 * gets k_min / k_max over its valid tokens in stats_pool (pool id
 * block_table[j / g], sub-page j % g) -- exactly what lserve_page_stats writes.
 * desc->batch is not used.  A bad pool id skips that page and sets
 * LSERVE_ERR_BOUNDS.  seq_len = 0 does nothing.  No workspace.
 */
int lserve_prefill_to_pages(const lserve_paged_desc* desc, int32_t seq_len, const void* k,
                            const void* v, const int32_t* block_table, const uint8_t* head_kind,
                            void* k_pool, void* v_pool, void* stats_pool, void* stream);

/*
 * lserve_decode_append -- cache maintenance of one decode step: append each
 * sequence's new token to the paged KV pools and keep the page statistics.
 * [技術的詳細 › 動的スパーシティ: the k_min / k_max statistics of logical page j;
 *  階層的ページング: logical pages of N_L tokens inside physical pages.  The pages
 *  describe the statistics, not how they are kept during decode: here a page's
 *  statistics after an append equal those lserve_page_stats would build.]
 *
 * For every sequence b and KV head h the token at position pos = ctx_lens[b]
 * (the length BEFORE this step; the caller advances ctx_lens afterwards) is
 * written: k_new[b][h][:] into k_pool at pool id block_table[b][pos / N_P],
 * row pos % N_P, and v_new likewise into v_pool.  For retrieval heads the
 * statistics of logical page pos / N_L (sub-page (pos % N_P) / N_L of that
 * pool page) become k_min = k_max = k_new when pos % N_L == 0, else the
 * elementwise min / max of the stored values and k_new (exact in bf16).
 * Streaming heads' statistics are not touched.
 *   k_new, v_new  bf16 [B][H_kv][D], 16-byte aligned.
 * The block table must already hold the page of pos.  A position outside
 * [0, max_pages_per_seq * N_P) or a bad pool id skips that sequence and sets
 * LSERVE_ERR_BOUNDS (lserve_read_device_status).  No workspace.
 * The page being appended to must belong to one sequence only: two sequences
 * whose block tables name the same pool page at their append positions (a
 * shared prefix page) would update that page's K / V row and statistics from
 * two warps at once, and the result is undefined.  Pages shared read-only
 * (before the append position) are fine.
 */
int lserve_decode_append(const lserve_paged_desc* desc, const void* k_new, const void* v_new,
                         const int32_t* block_table, const int32_t* ctx_lens,
                         const uint8_t* head_kind, void* k_pool, void* v_pool, void* stats_pool,
                         void* stream);

/*
 * lserve_page_select -- query-centric page scores and top-K physical pages.
 * [技術的詳細 › 動的スパーシティ, the equation
 *    S^j = sum_{i=1..D} max(q[i] * k_max^j[i], q[i] * k_min^j[i]);
 *  階層的ページング: a physical page scores the max of its logical pages;
 *  統一ブロックスパースアテンション figure: "Top-K物理ページ"; Reusable Page Selection:
 *  the result may be reused for k consecutive decode steps (default 4).]
 *
 * For each (b, retrieval KV head h): S^j is summed over the G query heads of h
 * (GQA reading), in fp32 from exact bf16 x bf16 products; P^m = max over the
 * valid logical pages of physical page m; then the top_k largest P^m, ties to
 * the lowest m.  Outputs:
 *   sel         int32 [B][H_kv][top_k]: chosen page ORDINALS m (not pool ids),
 *               ascending, padded with -1.  Streaming heads: all -1.
 *   sel_count   int32 [B][H_kv]: min(top_k, ceil(n_b / N_P)); 0 for streaming.
 *   phys_scores float [B][H_kv][max_pages_per_seq] or NULL; entries past the
 *               sequence's pages and for streaming heads are left untouched.
 * workspace: lserve_workspace_size(LSERVE_OP_SELECT, desc, top_k) bytes (used
 * for the scores when phys_scores is NULL).  1 <= top_k <= max_pages_per_seq.
 */
int lserve_page_select(const lserve_paged_desc* desc, const void* q, const void* stats_pool,
                       const int32_t* block_table, const int32_t* ctx_lens, const uint8_t* head_kind,
                       int32_t top_k, int32_t* sel, int32_t* sel_count, float* phys_scores,
                       void* workspace, size_t workspace_bytes, void* stream);

/*
 * lserve_sparse_decode_attn -- one decode step of paged GQA attention over the
 * pages each head keeps.
 * [統一ブロックスパースアテンション figure: retrieval heads attend the top-K
 *  physical pages, streaming heads the Lambda-shaped sink + local blocks;
 *  技術的詳細 › 静的スパーシティ: sink tokens and recent local tokens.]
 *
 * Retrieval head h of sequence b attends every valid token of the pages
 * sel[b][h][0 .. sel_count[b][h]) (page ordinals, as lserve_page_select writes
 * them).  A streaming head attends the pages [0, ceil(sink_tokens / N_P)) and
 * every page holding one of the last local_tokens tokens.  Each of the G query
 * heads computes softmax(softmax_scale * q.k) . v in fp32 (split over pages,
 * merged by a log-sum-exp combine pass) and writes:
 *   out  bf16 [B][H_q][D]
 *   lse  float [B][H_q] natural-log sum of exp(scale * q.k), or NULL.
 * A head with no token to attend (n_b = 0) gets out = 0, lse = -inf.
 * workspace: lserve_workspace_size(LSERVE_OP_DECODE, desc, top_k) bytes,
 * 256-byte aligned and ZERO-FILLED once before its first use.  It holds the
 * partial results of pairs split over several thread blocks, each word tagged
 * with the pair and a per-pair merge epoch (20 bits) kept in the workspace
 * too; every call advances the epochs it uses, also when it ends in an error
 * (a timeout), so leftovers of earlier calls are not mistaken for this
 * call's -- only a word left in a slot 2^20 merges of that pair earlier and
 * never overwritten since could match again: the workspace never needs
 * re-zeroing.  Calls that may run concurrently need separate workspaces.
 * Limits: B * H_kv <= 2048; N_P = 32 or a multiple of 64.
 */
int lserve_sparse_decode_attn(const lserve_paged_desc* desc, const void* q, const void* k_pool,
                              const void* v_pool, const int32_t* block_table, const int32_t* ctx_lens,
                              const uint8_t* head_kind, const int32_t* sel, const int32_t* sel_count,
                              int32_t top_k, int32_t sink_tokens, int32_t local_tokens,
                              float softmax_scale, void* out, float* lse, void* workspace,
                              size_t workspace_bytes, void* stream);

/*
 * lserve_sparse_decode_attn_ex -- lserve_sparse_decode_attn with launch flags.
 * (No counterpart on the pages: a launch option of this library.)
 *
 * The kernel is launched as a programmatic dependent of the work before it on
 * the stream: its thread blocks may start while that work is still finishing,
 * and they wait for it to complete (with its memory visible) before reading
 * q or the KV pools and before writing anything.  flags:
 *   0                                  plan and page lookups also wait
 *                                      (lserve_sparse_decode_attn does this).
 *   LSERVE_DECODE_OVERLAP_PROLOGUE     the caller guarantees that the kernel
 *                                      just before this call on the stream
 *                                      writes none of block_table, ctx_lens,
 *                                      head_kind, sel, sel_count: the split
 *                                      plan and the first page lookups then
 *                                      run before that kernel completes
 *                                      (e.g. consecutive decode-attention
 *                                      calls of different layers).
 *   LSERVE_DECODE_OUT_F32              `out` is float [B][H_q][D] (the
 *                                      normalised output before bf16
 *                                      rounding), e.g. a shard's partial
 *                                      for lserve_seqshard_combine.
 *   LSERVE_DECODE_PREFETCH_KV          with LSERVE_DECODE_OVERLAP_PROLOGUE
 *                                      (ignored without it): the caller also
 *                                      guarantees that the kernel just before
 *                                      writes no KV-pool page (nor quantized
 *                                      code or scale) this call reads, so the
 *                                      first tiles' copies start before that
 *                                      kernel completes (consecutive layers'
 *                                      calls; a QKV projection that writes q
 *                                      and the new token only).  q and the
 *                                      appended rows still wait for it.
 * Any other bit: LSERVE_ERR_INVALID_ARG.  Everything else as
 * lserve_sparse_decode_attn.
 */
#define LSERVE_DECODE_OVERLAP_PROLOGUE 1u
#define LSERVE_DECODE_OUT_F32 2u
#define LSERVE_DECODE_PREFETCH_KV 4u
int lserve_sparse_decode_attn_ex(const lserve_paged_desc* desc, const void* q, const void* k_pool,
                                 const void* v_pool, const int32_t* block_table,
                                 const int32_t* ctx_lens, const uint8_t* head_kind,
                                 const int32_t* sel, const int32_t* sel_count, int32_t top_k,
                                 int32_t sink_tokens, int32_t local_tokens, float softmax_scale,
                                 void* out, float* lse, uint32_t flags, void* workspace,
                                 size_t workspace_bytes, void* stream);

/*
 * lserve_decode_step -- one decode step in one launch: append each sequence's
 * new token to the paged cache and attend.
 * [技術的詳細 › 動的スパーシティ (the k_min / k_max statistics a new token
 *  updates) and › Reusable Page Selection (a selection is reused for k steps;
 *  the pages do not say whether tokens appended meanwhile are seen -- this
 *  call offers both readings); the attention as lserve_sparse_decode_attn.]
 *
 * ctx_lens[b] counts the new token: it sits at position t = ctx_lens[b] - 1.
 *   k_new, v_new  bf16 [B][H_kv][D] (16-byte aligned), or both NULL (no append):
 *                 written to row t of the pools, and for retrieval heads into
 *                 the k_min / k_max of logical page t / N_L (exactly as
 *                 lserve_decode_append), in the same launch; the attention
 *                 reads the new token from k_new / v_new, never from the pool.
 *   recent_from   int32 [B] or NULL.  NULL: a retrieval head attends the valid
 *                 tokens of its selected pages (the new token only if its page
 *                 is selected).  Given: it also attends every position in
 *                 [recent_from[b], ctx_lens[b]) -- e.g. the length when its
 *                 selection was made -- each token once.
 * Streaming heads attend the sink + local pages of ctx_lens[b] tokens (the new
 * token always).  Everything else -- sel, outputs, workspace, flags -- as
 * lserve_sparse_decode_attn_ex; LSERVE_DECODE_OVERLAP_PROLOGUE also requires
 * that the kernel before writes no recent_from.  The block table must already
 * hold the page of position t; a sequence with ctx_lens[b] = 0 appends nothing.
 * The appended page must belong to one sequence (see lserve_decode_append).
 */
int lserve_decode_step(const lserve_paged_desc* desc, const void* q, const void* k_new,
                       const void* v_new, void* k_pool, void* v_pool, void* stats_pool,
                       const int32_t* block_table, const int32_t* ctx_lens,
                       const uint8_t* head_kind, const int32_t* sel, const int32_t* sel_count,
                       int32_t top_k, int32_t sink_tokens, int32_t local_tokens,
                       const int32_t* recent_from, float softmax_scale, void* out, float* lse,
                       uint32_t flags, void* workspace, size_t workspace_bytes, void* stream);

/*
 * lserve_quantize_pages_kv8 -- an int8 copy of the paged K / V cache.
 * [LServe abstract page: the unified sparse attention is combined with a
 *  quantized KV cache (QServe's KV4 in the end-to-end results); the pages give
 *  no quantization scheme.  This library's scheme: symmetric int8, one float32
 *  scale per (pool page, KV head, channel) over the page's valid tokens.]
 *
 * For every sequence b, page ordinal m < ceil(n_b / N_P) and KV head h, with
 * pool id pid = block_table[b][m] and valid = min(N_P, n_b - m*N_P) tokens,
 * and separately for K and V:
 *   amax_c  = max over the valid rows of |x[row][c]|
 *   code    = rint(x * (127 / amax_c)) clamped to [-127, 127]  (float32,
 *             IEEE-rounded quotient and product, ties to even; 0 if amax_c = 0)
 *   scale_c = amax_c / 127                                      (float32)
 *   k_pool8 / v_pool8  int8 [num_pool_pages][H_kv][N_P][D]: the codes; rows
 *                      past `valid` are written as 0;
 *   k_scale / v_scale  float [num_pool_pages][H_kv][D]: the scales.
 * The value the cache holds is code * scale_c.  Inputs k_pool / v_pool are the
 * bf16 pools (layout above); they are only read, so the page statistics built
 * from them (lserve_page_stats, lserve_prefill_to_pages) stay the selection's
 * input.  Pool pages no sequence references are not touched.  A bad pool id
 * skips that page and sets LSERVE_ERR_BOUNDS.  No workspace.  All pointers
 * 16-byte aligned.
 */
int lserve_quantize_pages_kv8(const lserve_paged_desc* desc, const void* k_pool, const void* v_pool,
                              const int32_t* block_table, const int32_t* ctx_lens, void* k_pool8,
                              void* v_pool8, float* k_scale, float* v_scale, void* stream);

/*
 * lserve_quantize_pages_kv4 -- a 4-bit copy of the paged K / V cache.
 * [LServe abstract page: the sparse attention combined with QServe's KV4 in
 *  the end-to-end results; the pages give no scheme.  This library's scheme:
 *  the int8 scheme above with codes -7..7.]
 *
 * As lserve_quantize_pages_kv8 with 7 in place of 127:
 *   code    = rint(x * (7 / amax_c)) clamped to [-7, 7]  (float32, ties to even)
 *   scale_c = amax_c / 7
 *   k_pool4 / v_pool4  uint8 [num_pool_pages][H_kv][N_P][D/2]: two codes per
 *                      byte as 4-bit two's complement, channel 2i in the low
 *                      nibble and 2i+1 in the high nibble; rows past `valid`
 *                      are 0;
 *   k_scale / v_scale  float [num_pool_pages][H_kv][D].
 * A quarter of the bf16 cache's bytes (plus the scales).  No workspace; all
 * pointers 16-byte aligned.
 */
int lserve_quantize_pages_kv4(const lserve_paged_desc* desc, const void* k_pool, const void* v_pool,
                              const int32_t* block_table, const int32_t* ctx_lens, void* k_pool4,
                              void* v_pool4, float* k_scale, float* v_scale, void* stream);

/*
 * lserve_sparse_decode_attn_kv8 -- lserve_sparse_decode_attn_ex over the int8
 * cache that lserve_quantize_pages_kv8 writes.
 * [Same pages as lserve_sparse_decode_attn; the quantized cache as above.]
 *
 * Every attended token contributes k = code_k * k_scale and v = code_v *
 * v_scale of its page; pages, softmax, outputs, lse, flags and workspace are
 * exactly those of lserve_sparse_decode_attn_ex with the same arguments.
 * Arithmetic: tensor cores in fp16 -- the codes are exact in fp16, q * k_scale
 * and code_v * v_scale are rounded to fp16 (11-bit significand; q * k_scale
 * must lie within fp16's range), products accumulate in fp32, the softmax is
 * fp32.  k_pool8 / v_pool8 int8 [num_pool_pages][H_kv][N_P][D],
 * k_scale / v_scale float [num_pool_pages][H_kv][D], all 16-byte aligned.
 * Each attended page moves N_P*D bytes of K codes and of V codes plus 2*D*4
 * bytes of scales: about half the bf16 call's traffic.
 */
int lserve_sparse_decode_attn_kv8(const lserve_paged_desc* desc, const void* q, const void* k_pool8,
                                  const void* v_pool8, const float* k_scale, const float* v_scale,
                                  const int32_t* block_table, const int32_t* ctx_lens,
                                  const uint8_t* head_kind, const int32_t* sel,
                                  const int32_t* sel_count, int32_t top_k, int32_t sink_tokens,
                                  int32_t local_tokens, float softmax_scale, void* out, float* lse,
                                  uint32_t flags, void* workspace, size_t workspace_bytes,
                                  void* stream);

/*
 * lserve_sparse_decode_attn_kv4 -- lserve_sparse_decode_attn_kv8 over the
 * 4-bit cache that lserve_quantize_pages_kv4 writes (k_pool4 / v_pool4 uint8
 * [num_pool_pages][H_kv][N_P][D/2], two codes per byte; scales as kv8).  Each
 * attended page moves N_P*D/2 bytes of K codes and of V codes plus 2*D*4
 * bytes of scales: about a quarter of the bf16 call's traffic.
 * [Same pages as lserve_sparse_decode_attn; the 4-bit cache as above.]
 */
int lserve_sparse_decode_attn_kv4(const lserve_paged_desc* desc, const void* q, const void* k_pool4,
                                  const void* v_pool4, const float* k_scale, const float* v_scale,
                                  const int32_t* block_table, const int32_t* ctx_lens,
                                  const uint8_t* head_kind, const int32_t* sel,
                                  const int32_t* sel_count, int32_t top_k, int32_t sink_tokens,
                                  int32_t local_tokens, float softmax_scale, void* out, float* lse,
                                  uint32_t flags, void* workspace, size_t workspace_bytes,
                                  void* stream);

/*
 * lserve_blocksparse_prefill -- causal block-sparse flash attention for one
 * sequence.
 * [統一ブロックスパースアテンション: retrieval heads "block-sparse attention, static
 *  pattern" (dense causal here), streaming heads the Lambda mask of sink and
 *  local blocks; the ideal speedup at block sparsity r is 1/(1-r).  Abstract
 *  page: computation on less important tokens is skipped block-wise.]
 *
 * Query block row i of a head whose KV head is retrieval visits key blocks
 * 0..i; a streaming head visits [0, sink_blocks) and [i-local_blocks+1, i].
 * Causal masking applies inside the diagonal block.  QK^T and PV run on the
 * tcgen05 tensor cores (bf16 in, fp32 accumulate in tensor memory); softmax in
 * fp32.  head_kind_host is a HOST array uint8 [H_kv].
 *   q   bf16 [T][H_q][D], k / v bf16 [T][H_kv][D] (16-byte aligned)
 *   out bf16 [T][H_q][D]; lse float [H_q][T] (natural log) or NULL.
 * workspace: lserve_workspace_size(LSERVE_OP_PREFILL, desc, 0) bytes.
 */
int lserve_blocksparse_prefill(const lserve_prefill_desc* desc, const void* q, const void* k,
                               const void* v, const uint8_t* head_kind_host, float softmax_scale,
                               void* out, float* lse, void* workspace, size_t workspace_bytes,
                               void* stream);

/*
 * lserve_blocksparse_prefill_paged -- lserve_blocksparse_prefill that also
 * hands the sequence to the paged decode cache from inside the same kernel:
 * K / V through the block table into the pools and the retrieval heads' page
 * statistics (what lserve_prefill_to_pages writes, without its second pass).
 * [統一ブロックスパースアテンション as lserve_blocksparse_prefill; 階層的ページング:
 *  logical pages of N_L tokens inside physical pages of N_P tokens; 技術的詳細 ›
 *  動的スパーシティ: k_min^j / k_max^j of logical page j.]
 *
 * desc, q, k, v, head_kind_host, softmax_scale, out, lse, workspace: as
 * lserve_blocksparse_prefill (out and lse are bit-identical to it).
 * paged: the cache (batch unused; head_dim and num_kv_heads equal desc's;
 * N_L, N_P as lserve_page_stats supports); block_table int32
 * [max_pages_per_seq] of THIS sequence (page ordinal -> pool id), covering
 * seq_len tokens; k_pool / v_pool bf16 [num_pool_pages][H_kv][N_P][D],
 * stats_pool bf16 [num_pool_pages][H_kv][g][2][D] (16-byte aligned).  Token t
 * of KV head h goes to pool id block_table[t / N_P], row t % N_P; rows past
 * seq_len are not written; retrieval heads (head_kind_host[h] == 0) get the
 * k_min / k_max of every logical page.  A warp of the prefill kernel writes
 * each key block of 128 tokens (the diagonal block of one work tile of its KV
 * head's first query head), reading it from k / v alongside the attention.
 * A bad pool id skips that page and sets LSERVE_ERR_BOUNDS.
 */
int lserve_blocksparse_prefill_paged(const lserve_prefill_desc* desc, const lserve_paged_desc* paged,
                                     const void* q, const void* k, const void* v,
                                     const uint8_t* head_kind_host, float softmax_scale, void* out,
                                     float* lse, const int32_t* block_table, void* k_pool,
                                     void* v_pool, void* stats_pool, void* workspace,
                                     size_t workspace_bytes, void* stream);

/*
 * lserve_page_select_noalloc -- lserve_page_select for callers that cannot
 * allocate device memory.  (The LServe pages have no counterpart: this is a
 * deployment convenience of this library.)
 *
 * Same arguments and results as lserve_page_select without phys_scores and
 * workspace.  The physical-page scores go to a fixed 4 MiB array inside the
 * library's device memory, so no cudaMalloc is needed -- useful where the
 * caller runs inside a host callback or a plug-in whose host process owns all
 * allocations.  Limits and caveats:
 *   - B * H_kv * max_pages_per_seq must be <= 1,048,576, else
 *     LSERVE_ERR_UNSUPPORTED is returned and nothing is launched;
 *   - each GPU that loads the library holds the array until the process exits;
 *   - every call on a device shares the array (the previous call's scores stay
 *     there and are overwritten): calls that overlap on the GPU race;
 *   - the first call on each device looks up the array's device address with
 *     that device current; make that first call before any stream capture;
 *   - the current device must be the one `stream` belongs to (the array used
 *     is the current device's), and its index must be below 64 (the library
 *     caches one address per device index; higher indices get LSERVE_ERR_CUDA).
 */
int lserve_page_select_noalloc(const lserve_paged_desc* desc, const void* q, const void* stats_pool,
                               const int32_t* block_table, const int32_t* ctx_lens,
                               const uint8_t* head_kind, int32_t top_k, int32_t* sel,
                               int32_t* sel_count, void* stream);

/* Bytes of workspace `op` needs for these shapes on the CURRENT device
 * (desc points to lserve_paged_desc, or lserve_prefill_desc for PREFILL).
 * Returns 0 for invalid shapes. */
/*
 * Sequence-sharded decode: one long sequence over N GPUs (one process each).
 * [LServe explainer, 技術的詳細 › 動的スパーシティ / 階層的ページング: page scores
 *  and the top-K; the split across GPUs is this library's reading -- the
 *  pages leave it open.]
 *
 * Shard r of N holds the contiguous physical pages [P_r, P_{r+1}) of each
 * sequence, P_r = floor(M * r / N), M = ceil(n / N_P) with n the GLOBAL
 * length; its own paged cache holds them as shard-local ordinals 0.. with a
 * shard-local length (lserve_seqshard_bounds).  One decode step per shard:
 *   1. lserve_page_select(shard desc, local lengths, phys_scores non-NULL);
 *   2. lserve_seqshard_candidates -> this shard's proposals [B][H_kv][top_k];
 *   3. all-gather the proposals over the N shards (caller: NCCL) into
 *      [N][B][H_kv][top_k], shard order;
 *   4. lserve_seqshard_merge -> this shard's part of the global choice;
 *   5. lserve_sparse_decode_attn_ex(shard desc, local lengths, head_kind all
 *      0 (every head reads the merged selection), top_k = sel_stride,
 *      flags LSERVE_DECODE_OUT_F32, lse non-NULL) -> float o, lse;
 *   6. all-gather o [N][B*H_q][D] and lse [N][B*H_q] (caller);
 *   7. lserve_seqshard_combine -> out bf16 [B][H_q][D].
 * The choice equals the unsharded lserve_page_select bit for bit (the scores
 * of a page do not depend on the shard; every page of the global top-K is in
 * its own shard's top-K); out differs from the unsharded call only by
 * rounding.  All calls are asynchronous on `stream`, allocate nothing, and
 * set LSERVE_ERR_BOUNDS in the device status for out-of-range ordinals.
 */

/* Host only: this shard's page range [*first_page, *end_page) and its
 * shard-local length (tokens of the sequence in those pages). */
int lserve_seqshard_bounds(int32_t ctx_len, int32_t physical_page, int32_t rank,
                           int32_t num_shards, int32_t* first_page, int32_t* end_page,
                           int32_t* local_len);

/* Host only: the row length of the merged selection, max(top_k,
 * ceil(sink/N_P) + ceil(local/N_P) + 1); 0 on invalid arguments. */
int32_t lserve_seqshard_sel_stride(const lserve_paged_desc* desc, int32_t top_k,
                                   int32_t sink_tokens, int32_t local_tokens);

/*
 * lserve_seqshard_candidates -- this shard's proposals.  desc is the SHARD's
 * descriptor (max_pages_per_seq = its block-table row length).  For each
 * (b, h), proposal i < sel_count[b][h] (retrieval heads) is
 *   cand_page  = P_r(b) + sel[b][h][i]          (global page ordinal)
 *   cand_score = phys_scores[b][h][sel[b][h][i]]
 * and the rest up to top_k are (-inf, -1); streaming heads propose nothing.
 * sel / sel_count / phys_scores as lserve_page_select wrote them with top_k =
 * sel_top_k (the row length of sel).  ctx_lens_global: int32 [B] device.
 * Outputs float / int32 [B][H_kv][top_k], device.
 */
int lserve_seqshard_candidates(const lserve_paged_desc* desc, int32_t rank, int32_t num_shards,
                               const int32_t* ctx_lens_global, const uint8_t* head_kind,
                               const int32_t* sel, const int32_t* sel_count, int32_t sel_top_k,
                               const float* phys_scores, int32_t top_k, float* cand_score,
                               int32_t* cand_page, void* stream);

/*
 * lserve_seqshard_merge -- this shard's part of the global page choice.
 * cand_score_all / cand_page_all: the all-gathered proposals [N][B][H_kv][top_k].
 * Retrieval heads: the min(top_k, M) proposals first in (score descending,
 * page ascending) order -- the unsharded top-K; those in [P_r, P_{r+1}) are
 * written as shard-local ordinals, ascending.  Streaming heads: the sink
 * pages [0, ceil(sink_tokens/N_P)) and every page holding one of the last
 * local_tokens tokens (global positions), those in the shard, shard-local.
 *   sel_out        int32 [B][H_kv][sel_stride], -1 padded;
 *   sel_count_out  int32 [B][H_kv].
 * sel_stride >= lserve_seqshard_sel_stride(desc, top_k, sink, local), else
 * LSERVE_ERR_INVALID_ARG; N * top_k * 9 bytes must fit in shared memory
 * (<= 200 KiB, else LSERVE_ERR_UNSUPPORTED).
 */
int lserve_seqshard_merge(const lserve_paged_desc* desc, int32_t rank, int32_t num_shards,
                          const int32_t* ctx_lens_global, const uint8_t* head_kind,
                          const float* cand_score_all, const int32_t* cand_page_all, int32_t top_k,
                          int32_t sink_tokens, int32_t local_tokens, int32_t* sel_out,
                          int32_t* sel_count_out, int32_t sel_stride, void* stream);

/*
 * lserve_seqshard_combine -- attention over disjoint token sets merged into
 * attention over their union (log-sum-exp weights), per row (query head):
 *   M = max_r lse[r], w_r = exp(lse[r] - M),
 *   out = sum_r w_r o[r] / sum_r w_r   (bf16),   lse_out = M + log(sum_r w_r).
 * Rows with every lse = -inf get out = 0, lse_out = -inf.
 *   o_parts float [N][rows][head_dim], lse_parts float [N][rows] (natural log),
 *   out bf16 [rows][head_dim], lse float [rows] or NULL; head_dim 64 or 128.
 */
int lserve_seqshard_combine(int32_t num_shards, int32_t rows, int32_t head_dim, const float* o_parts,
                            const float* lse_parts, void* out, float* lse, void* stream);

size_t lserve_workspace_size(int op, const void* desc, int32_t top_k);

/* Synchronises `stream`, returns the first device-side error flag raised since
 * the last call (LSERVE_ERR_TIMEOUT / LSERVE_ERR_BOUNDS) or LSERVE_OK, and
 * clears the flags of the current device. */
int lserve_read_device_status(void* stream);

/* Upper bound, in SM clock cycles, of every bounded device wait started after
 * this call (default 4e9, about two seconds).  0 restores the default. */
void lserve_set_wait_limit_cycles(uint64_t cycles);

/* Diagnostic: launches one CTA that waits on a hardware barrier nobody
 * arrives at, bounded by `cycles`; lserve_read_device_status() must then
 * report LSERVE_ERR_TIMEOUT.  Exercises the timeout path without a fault. */
int lserve_debug_wait_timeout(uint64_t cycles, void* stream);

const char* lserve_status_string(int status);

/* 1: page-level index checks are compiled into every kernel. */
int lserve_bounds_checked(void);

#ifdef __cplusplus
}
#endif

#endif /* LSERVE_H_ */
