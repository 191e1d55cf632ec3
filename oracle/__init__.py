"""CPU oracle for LServe-style unified sparse attention -- TEST INFRASTRUCTURE ONLY.

Plain, slow, fp64 numpy restatement of what the hot path computes, written
from the LServe explainer page ("MLSys 2025論文解説: LServe — 統一疎アテンション
による長文脈LLM推論の効率化", arXiv 2502.14866) and the LServe abstract page
("LServe: Efficient Long-sequence LLM Serving with Unified Sparse Attention").

Only tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may
import this package.  It shares no code with the CUDA library and imports
nothing from it.  Inputs arrive as bf16 bit patterns (uint16) and are widened
exactly to float64 here.

Section references used throughout (all on the LServe explainer page unless
stated otherwise):
  [TD-static]   技術的詳細 › 静的スパーシティ (streaming heads, Lambda mask)
  [TD-dynamic]  技術的詳細 › 動的スパーシティ, the equation for S^j
  [TD-paging]   技術的詳細 › 階層的ページング (N_P = g * N_L, max-reduction)
  [TD-unified]  技術的詳細 › 統一ブロックスパースアテンション (figure; 1/(1-r))
  [TD-reuse]    技術的詳細 › Reusable Page Selection (k = 4, Table 6)
  [Abstract]    LServe abstract page (block-wise skipping; constant page budget)

Readings where the pages are silent (each is listed in the design notes):
  R1 GQA: one page choice per KV head, ranked by the SUM over its G query
     heads of S^j.                                          (parity unpinned)
  R2 partial pages: only valid tokens count; empty logical pages are skipped.
  R3 retrieval heads use pure top-K, nothing force-included.
  R4 ties go to the lowest page index; selections are reported ascending.
  R5 streaming decode is page-granular: sink pages [0, ceil(S/N_P)) plus every
     page holding one of the last L tokens.
  R10 tokens appended during a reuse window: by default a retrieval head sees
     them only if their page is selected; as an option it also attends every
     token appended since its selection (attended_tokens with recent_from).
  R6 Lambda prefill: block row i sees blocks {0..sink-1} and
     [i - local + 1, i] (the diagonal counts as local).   (parity unpinned)
  R7 retrieval heads in prefill are dense causal.
  R8 softmax scale is a parameter (1/sqrt(D) in the harness); scores unscaled.
  R15 quantized KV cache (row f3): symmetric int8, one float32 scale per
     (pool page, KV head, channel) over the page's valid tokens, codes decided
     in float32 (quantize_kv8); attention attends code * scale.
     (parity unpinned by the pages: they name KV quantization, not a scheme)
  R18 4-bit KV cache (row f3): the R15 scheme with codes -7..7 (quantize_kv4),
     two codes per byte in the device layout.       (parity unpinned, as R15)
  R17 sequence-sharded decode (row f4): shard r of N holds the contiguous
     physical pages [floor(M*r/N), floor(M*(r+1)/N)); each shard proposes its
     own top-K, the global top-K is re-made from the proposals, and the
     shards' attention results are merged by their log-sum-exp.  Pinned to the
     unsharded selection and attention (the split changes no result).
"""
from .lserve import (  # noqa: F401
    widen_bf16,
    page_stats,
    head_scores,
    logical_scores,
    physical_scores,
    select_top_k,
    retrieval_pages,
    streaming_pages,
    page_tokens,
    attended_tokens,
    decode_attention,
    decode_pair,
    shard_bounds,
    shard_candidates,
    merge_candidates,
    shard_streaming_pages,
    lse_combine,
    kv_blocks,
    computed_blocks,
    theoretical_speedup,
    prefill_rows,
    prefill_block_rows,
    prefill_flops,
    quantize_kv,
    quantize_kv8,
    quantize_kv4,
    dequantize_kv8,
    dequantized_seq,
)
