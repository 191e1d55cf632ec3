"""Thin Python binding of liblserve.so (LServe-style unified sparse attention
hot path on B200 / sm_100a).

Every function here only marshals arguments -- torch tensors in, raw device
pointers and the current CUDA stream out -- and calls the C-ABI function of
the same name declared in include/lserve.h.  All computation happens in the
library's CUDA kernels.  There is no fallback: if liblserve.so is missing or
cannot be loaded, importing this package raises.

Layouts (see include/lserve.h):
  q            bf16 [B][H_q][D]
  k/v pool     bf16 [num_pool_pages][H_kv][N_P][D]
  stats pool   bf16 [num_pool_pages][H_kv][N_P/N_L][2][D]
  block_table  int32 [B][max_pages]     ctx_lens int32 [B]
  head_kind    uint8 [H_kv] (0 retrieval, 1 streaming)
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_TIMEOUT, ERR_BOUNDS = range(7)
OP_STATS, OP_SELECT, OP_DECODE, OP_PREFILL = range(4)

EXPORTED = [
    "lserve_page_stats", "lserve_page_select", "lserve_sparse_decode_attn",
    "lserve_blocksparse_prefill", "lserve_workspace_size", "lserve_read_device_status",
    "lserve_set_wait_limit_cycles", "lserve_debug_wait_timeout", "lserve_status_string",
    "lserve_bounds_checked", "lserve_page_select_noalloc", "lserve_sparse_decode_attn_ex",
    "lserve_decode_append", "lserve_prefill_to_pages", "lserve_quantize_pages_kv8",
    "lserve_sparse_decode_attn_kv8", "lserve_seqshard_bounds", "lserve_seqshard_sel_stride",
    "lserve_seqshard_candidates", "lserve_seqshard_merge", "lserve_seqshard_combine",
    "lserve_quantize_pages_kv4", "lserve_sparse_decode_attn_kv4", "lserve_decode_step",
    "lserve_blocksparse_prefill_paged",
]
DECODE_OVERLAP_PROLOGUE = 1
DECODE_OUT_F32 = 2
DECODE_PREFETCH_KV = 4


class LServeError(RuntimeError):
    def __init__(self, fn, status, msg):
        super().__init__(f"{fn} failed: status {status} ({msg})")
        self.status = status


class PagedDesc(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "batch", "num_q_heads", "num_kv_heads", "head_dim", "logical_page", "physical_page",
        "max_pages_per_seq", "num_pool_pages")]


class PrefillDesc(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "seq_len", "num_q_heads", "num_kv_heads", "head_dim", "block_q", "block_k",
        "sink_blocks", "local_blocks")]


def library_path() -> str:
    return os.path.join(_HERE, "liblserve.so")


def _load(path):
    if not os.path.exists(path):
        raise ImportError(f"{path} not built: run `python block_sparse_attention_page_b200/build.py`")
    lib = ctypes.CDLL(path)
    vp, i32, sz, u64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t, ctypes.c_uint64
    P = ctypes.POINTER
    lib.lserve_page_stats.argtypes = [P(PagedDesc), vp, vp, vp, vp, vp, i32, vp]
    lib.lserve_page_select.argtypes = [P(PagedDesc), vp, vp, vp, vp, vp, i32, vp, vp, vp, vp, sz, vp]
    lib.lserve_sparse_decode_attn.argtypes = [P(PagedDesc), vp, vp, vp, vp, vp, vp, vp, vp, i32, i32,
                                              i32, ctypes.c_float, vp, vp, vp, sz, vp]
    lib.lserve_sparse_decode_attn_ex.argtypes = [P(PagedDesc), vp, vp, vp, vp, vp, vp, vp, vp, i32,
                                                 i32, i32, ctypes.c_float, vp, vp, ctypes.c_uint32,
                                                 vp, sz, vp]
    lib.lserve_decode_append.argtypes = [P(PagedDesc), vp, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.lserve_prefill_to_pages.argtypes = [P(PagedDesc), i32, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.lserve_blocksparse_prefill.argtypes = [P(PrefillDesc), vp, vp, vp, vp, ctypes.c_float, vp, vp,
                                               vp, sz, vp]
    lib.lserve_blocksparse_prefill_paged.argtypes = [P(PrefillDesc), P(PagedDesc), vp, vp, vp, vp,
                                                     ctypes.c_float, vp, vp, vp, vp, vp, vp, vp, sz,
                                                     vp]
    lib.lserve_quantize_pages_kv8.argtypes = [P(PagedDesc), vp, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.lserve_sparse_decode_attn_kv8.argtypes = [P(PagedDesc), vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                                  vp, i32, i32, i32, ctypes.c_float, vp, vp,
                                                  ctypes.c_uint32, vp, sz, vp]
    lib.lserve_quantize_pages_kv4.argtypes = lib.lserve_quantize_pages_kv8.argtypes
    lib.lserve_decode_step.argtypes = [P(PagedDesc), vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i32,
                                       i32, i32, vp, ctypes.c_float, vp, vp, ctypes.c_uint32, vp,
                                       sz, vp]
    lib.lserve_sparse_decode_attn_kv4.argtypes = lib.lserve_sparse_decode_attn_kv8.argtypes
    lib.lserve_page_select_noalloc.argtypes = [P(PagedDesc), vp, vp, vp, vp, vp, i32, vp, vp, vp]
    pi32 = P(i32)
    lib.lserve_seqshard_bounds.argtypes = [i32, i32, i32, i32, pi32, pi32, pi32]
    lib.lserve_seqshard_sel_stride.argtypes = [P(PagedDesc), i32, i32, i32]
    lib.lserve_seqshard_sel_stride.restype = i32
    lib.lserve_seqshard_candidates.argtypes = [P(PagedDesc), i32, i32, vp, vp, vp, vp, i32, vp, i32,
                                               vp, vp, vp]
    lib.lserve_seqshard_merge.argtypes = [P(PagedDesc), i32, i32, vp, vp, vp, vp, i32, i32, i32, vp,
                                          vp, i32, vp]
    lib.lserve_seqshard_combine.argtypes = [i32, i32, i32, vp, vp, vp, vp, vp]
    lib.lserve_page_select_noalloc.restype = ctypes.c_int
    lib.lserve_workspace_size.argtypes = [ctypes.c_int, vp, i32]
    lib.lserve_workspace_size.restype = sz
    lib.lserve_read_device_status.argtypes = [vp]
    lib.lserve_set_wait_limit_cycles.argtypes = [u64]
    lib.lserve_set_wait_limit_cycles.restype = None
    lib.lserve_debug_wait_timeout.argtypes = [u64, vp]
    lib.lserve_status_string.argtypes = [ctypes.c_int]
    lib.lserve_status_string.restype = ctypes.c_char_p
    for name in ("lserve_page_stats", "lserve_page_select", "lserve_sparse_decode_attn",
                 "lserve_blocksparse_prefill", "lserve_read_device_status", "lserve_debug_wait_timeout",
                 "lserve_bounds_checked", "lserve_quantize_pages_kv8",
                 "lserve_sparse_decode_attn_kv8", "lserve_sparse_decode_attn_ex",
                 "lserve_decode_append", "lserve_prefill_to_pages", "lserve_seqshard_bounds",
                 "lserve_seqshard_candidates", "lserve_seqshard_merge", "lserve_seqshard_combine",
                 "lserve_quantize_pages_kv4", "lserve_sparse_decode_attn_kv4",
                 "lserve_decode_step"):
        getattr(lib, name).restype = ctypes.c_int
    return lib


lib = _load(library_path())


def _decode_flags(overlap_prologue, prefetch_kv):
    return ((DECODE_OVERLAP_PROLOGUE if overlap_prologue else 0) |
            (DECODE_PREFETCH_KV if prefetch_kv else 0))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(fn, status):
    if status != OK:
        raise LServeError(fn, status, lib.lserve_status_string(status).decode())


def status_string(status: int) -> str:
    return lib.lserve_status_string(status).decode()


def paged_desc(B, H_q, H_kv, D, N_L, N_P, max_pages, num_pool_pages) -> PagedDesc:
    return PagedDesc(B, H_q, H_kv, D, N_L, N_P, max_pages, num_pool_pages)


def prefill_desc(T, H_q, H_kv, D, block, sink_blocks, local_blocks) -> PrefillDesc:
    return PrefillDesc(T, H_q, H_kv, D, block, block, sink_blocks, local_blocks)


def workspace_size(op: int, desc, top_k: int = 0) -> int:
    return lib.lserve_workspace_size(op, ctypes.byref(desc), top_k)


def page_stats(desc, k_pool, block_table, ctx_lens, head_kind, stats_pool, first_logical_page=0,
               stream=None):
    _check("lserve_page_stats", lib.lserve_page_stats(
        ctypes.byref(desc), _ptr(k_pool), _ptr(block_table), _ptr(ctx_lens), _ptr(head_kind),
        _ptr(stats_pool), first_logical_page, _stream(stream)))


def page_select(desc, q, stats_pool, block_table, ctx_lens, head_kind, top_k, sel, sel_count,
                phys_scores=None, workspace=None, stream=None):
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("lserve_page_select", lib.lserve_page_select(
        ctypes.byref(desc), _ptr(q), _ptr(stats_pool), _ptr(block_table), _ptr(ctx_lens),
        _ptr(head_kind), top_k, _ptr(sel), _ptr(sel_count), _ptr(phys_scores), _ptr(workspace),
        ws_bytes, _stream(stream)))


def page_select_noalloc(desc, q, stats_pool, block_table, ctx_lens, head_kind, top_k, sel, sel_count,
                        stream=None):
    """lserve_page_select with the scores kept in the library's static device
    array instead of a caller workspace (for callers that cannot allocate)."""
    _check("lserve_page_select_noalloc", lib.lserve_page_select_noalloc(
        ctypes.byref(desc), _ptr(q), _ptr(stats_pool), _ptr(block_table), _ptr(ctx_lens),
        _ptr(head_kind), top_k, _ptr(sel), _ptr(sel_count), _stream(stream)))


def sparse_decode_attn(desc, q, k_pool, v_pool, block_table, ctx_lens, head_kind, sel, sel_count,
                       top_k, sink_tokens, local_tokens, softmax_scale, out, lse=None,
                       workspace=None, stream=None, overlap_prologue=False, out_f32=False,
                       prefetch_kv=False):
    """lserve_sparse_decode_attn; overlap_prologue=True or out_f32=True call
    lserve_sparse_decode_attn_ex with LSERVE_DECODE_OVERLAP_PROLOGUE (the caller
    guarantees the previous kernel on the stream writes none of block_table,
    ctx_lens, head_kind, sel, sel_count; with prefetch_kv also no KV page this
    call reads) or LSERVE_DECODE_OUT_F32 (`out` is a float32 tensor)."""
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    flags = _decode_flags(overlap_prologue, prefetch_kv) | (DECODE_OUT_F32 if out_f32 else 0)
    if flags:
        _check("lserve_sparse_decode_attn_ex", lib.lserve_sparse_decode_attn_ex(
            ctypes.byref(desc), _ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(block_table),
            _ptr(ctx_lens), _ptr(head_kind), _ptr(sel), _ptr(sel_count), top_k, sink_tokens,
            local_tokens, float(softmax_scale), _ptr(out), _ptr(lse), flags,
            _ptr(workspace), ws_bytes, _stream(stream)))
        return
    _check("lserve_sparse_decode_attn", lib.lserve_sparse_decode_attn(
        ctypes.byref(desc), _ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(block_table), _ptr(ctx_lens),
        _ptr(head_kind), _ptr(sel), _ptr(sel_count), top_k, sink_tokens, local_tokens,
        float(softmax_scale), _ptr(out), _ptr(lse), _ptr(workspace), ws_bytes, _stream(stream)))


def decode_append(desc, k_new, v_new, block_table, ctx_lens, head_kind, k_pool, v_pool, stats_pool,
                  stream=None):
    """lserve_decode_append: write each sequence's new K/V row at position
    ctx_lens[b] and update that logical page's k_min / k_max (retrieval heads)."""
    _check("lserve_decode_append", lib.lserve_decode_append(
        ctypes.byref(desc), _ptr(k_new), _ptr(v_new), _ptr(block_table), _ptr(ctx_lens),
        _ptr(head_kind), _ptr(k_pool), _ptr(v_pool), _ptr(stats_pool), _stream(stream)))


def prefill_to_pages(desc, seq_len, k, v, block_table, head_kind, k_pool, v_pool, stats_pool,
                     stream=None):
    """lserve_prefill_to_pages: one sequence's prefill K/V ([T][H_kv][D]) into the
    paged pools, with the retrieval heads' page statistics, in one pass."""
    _check("lserve_prefill_to_pages", lib.lserve_prefill_to_pages(
        ctypes.byref(desc), int(seq_len), _ptr(k), _ptr(v), _ptr(block_table), _ptr(head_kind),
        _ptr(k_pool), _ptr(v_pool), _ptr(stats_pool), _stream(stream)))


def quantize_pages_kv8(desc, k_pool, v_pool, block_table, ctx_lens, k_pool8, v_pool8, k_scale,
                       v_scale, stream=None, bits=8):
    """lserve_quantize_pages_kv8 (bits=8: int8 tensors shaped like the pools)
    or lserve_quantize_pages_kv4 (bits=4: uint8 [pool pages][H_kv][N_P][D/2],
    two codes per byte), with float32 per-(page, head, channel) scales
    ([pool pages][H_kv][D]) of every page the block table references."""
    name = {8: "lserve_quantize_pages_kv8", 4: "lserve_quantize_pages_kv4"}[bits]
    _check(name, getattr(lib, name)(
        ctypes.byref(desc), _ptr(k_pool), _ptr(v_pool), _ptr(block_table), _ptr(ctx_lens),
        _ptr(k_pool8), _ptr(v_pool8), _ptr(k_scale), _ptr(v_scale), _stream(stream)))


def sparse_decode_attn_kv8(desc, q, k_pool8, v_pool8, k_scale, v_scale, block_table, ctx_lens,
                           head_kind, sel, sel_count, top_k, sink_tokens, local_tokens,
                           softmax_scale, out, lse=None, workspace=None, stream=None,
                           overlap_prologue=False, bits=8, prefetch_kv=False):
    """lserve_sparse_decode_attn_kv8 / _kv4: sparse decode attention over the
    8-bit or 4-bit cache."""
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    flags = _decode_flags(overlap_prologue, prefetch_kv)
    name = {8: "lserve_sparse_decode_attn_kv8", 4: "lserve_sparse_decode_attn_kv4"}[bits]
    _check(name, getattr(lib, name)(
        ctypes.byref(desc), _ptr(q), _ptr(k_pool8), _ptr(v_pool8), _ptr(k_scale), _ptr(v_scale),
        _ptr(block_table), _ptr(ctx_lens), _ptr(head_kind), _ptr(sel), _ptr(sel_count), top_k,
        sink_tokens, local_tokens, float(softmax_scale), _ptr(out), _ptr(lse), flags,
        _ptr(workspace), ws_bytes, _stream(stream)))


def decode_step(desc, q, k_new, v_new, k_pool, v_pool, stats_pool, block_table, ctx_lens,
                head_kind, sel, sel_count, top_k, sink_tokens, local_tokens, softmax_scale, out,
                lse=None, recent_from=None, workspace=None, stream=None, overlap_prologue=False,
                prefetch_kv=False):
    """lserve_decode_step: append the new tokens (k_new / v_new, or None) and
    attend, in one launch; ctx_lens counts the new token."""
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    flags = _decode_flags(overlap_prologue, prefetch_kv)
    _check("lserve_decode_step", lib.lserve_decode_step(
        ctypes.byref(desc), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_pool), _ptr(v_pool),
        _ptr(stats_pool), _ptr(block_table), _ptr(ctx_lens), _ptr(head_kind), _ptr(sel),
        _ptr(sel_count), top_k, sink_tokens, local_tokens, _ptr(recent_from),
        float(softmax_scale), _ptr(out), _ptr(lse), flags, _ptr(workspace), ws_bytes,
        _stream(stream)))


def blocksparse_prefill(desc, q, k, v, head_kind_host, softmax_scale, out, lse=None, workspace=None,
                        stream=None):
    hk = (ctypes.c_uint8 * len(head_kind_host))(*[int(x) for x in head_kind_host])
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("lserve_blocksparse_prefill", lib.lserve_blocksparse_prefill(
        ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), ctypes.cast(hk, ctypes.c_void_p),
        float(softmax_scale), _ptr(out), _ptr(lse), _ptr(workspace), ws_bytes, _stream(stream)))


def blocksparse_prefill_paged(desc, paged_desc, q, k, v, head_kind_host, softmax_scale, out,
                              block_table, k_pool, v_pool, stats_pool, lse=None, workspace=None,
                              stream=None):
    """lserve_blocksparse_prefill_paged: the prefill, and from the same kernel
    this sequence's K/V into the paged pools (through block_table) with the
    retrieval heads' page statistics."""
    hk = (ctypes.c_uint8 * len(head_kind_host))(*[int(x) for x in head_kind_host])
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("lserve_blocksparse_prefill_paged", lib.lserve_blocksparse_prefill_paged(
        ctypes.byref(desc), ctypes.byref(paged_desc), _ptr(q), _ptr(k), _ptr(v),
        ctypes.cast(hk, ctypes.c_void_p), float(softmax_scale), _ptr(out), _ptr(lse),
        _ptr(block_table), _ptr(k_pool), _ptr(v_pool), _ptr(stats_pool), _ptr(workspace), ws_bytes,
        _stream(stream)))


# --- sequence-sharded decode (one long sequence over several GPUs) -------------

def seqshard_bounds(ctx_len: int, physical_page: int, rank: int, num_shards: int):
    """(first page, end page, shard-local length) of shard `rank` (host only)."""
    a, b, n = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
    _check("lserve_seqshard_bounds", lib.lserve_seqshard_bounds(
        ctx_len, physical_page, rank, num_shards, ctypes.byref(a), ctypes.byref(b), ctypes.byref(n)))
    return a.value, b.value, n.value


def seqshard_sel_stride(desc, top_k: int, sink_tokens: int, local_tokens: int) -> int:
    v = lib.lserve_seqshard_sel_stride(ctypes.byref(desc), top_k, sink_tokens, local_tokens)
    if v <= 0:
        raise LServeError("lserve_seqshard_sel_stride", ERR_INVALID_ARG, "invalid argument")
    return v


def seqshard_candidates(desc, rank, num_shards, ctx_lens_global, head_kind, sel, sel_count,
                        phys_scores, top_k, cand_score, cand_page, stream=None):
    """This shard's proposals from its own lserve_page_select result (`sel`'s
    last dimension is the top_k that call used)."""
    _check("lserve_seqshard_candidates", lib.lserve_seqshard_candidates(
        ctypes.byref(desc), rank, num_shards, _ptr(ctx_lens_global), _ptr(head_kind), _ptr(sel),
        _ptr(sel_count), sel.shape[-1], _ptr(phys_scores), top_k, _ptr(cand_score), _ptr(cand_page),
        _stream(stream)))


def seqshard_merge(desc, rank, num_shards, ctx_lens_global, head_kind, cand_score_all, cand_page_all,
                   top_k, sink_tokens, local_tokens, sel_out, sel_count_out, stream=None):
    """This shard's part of the global choice (`sel_out`'s last dimension is
    the row length, at least seqshard_sel_stride)."""
    _check("lserve_seqshard_merge", lib.lserve_seqshard_merge(
        ctypes.byref(desc), rank, num_shards, _ptr(ctx_lens_global), _ptr(head_kind),
        _ptr(cand_score_all), _ptr(cand_page_all), top_k, sink_tokens, local_tokens, _ptr(sel_out),
        _ptr(sel_count_out), sel_out.shape[-1], _stream(stream)))


def seqshard_combine(o_parts, lse_parts, out, lse=None, stream=None):
    """o_parts float [N][rows][D], lse_parts float [N][rows] -> out bf16 [rows][D]."""
    N, rows, D = o_parts.shape
    _check("lserve_seqshard_combine", lib.lserve_seqshard_combine(
        N, rows, D, _ptr(o_parts), _ptr(lse_parts), _ptr(out), _ptr(lse), _stream(stream)))


def process_group_all_gather(group=None):
    """all_gather(dst, src) over a torch.distributed process group: dst[r] of
    shape src.shape receives rank r's src (NCCL between GPUs; gloo too).  The
    output is handed over as the concatenation along the first dimension (the
    same memory as the [N, *src.shape] stack), the form every backend takes."""
    import torch.distributed as dist

    def all_gather(dst, src):
        dist.all_gather_into_tensor(dst.view((-1,) + tuple(src.shape[1:])), src, group=group)
    return all_gather


class SeqShardStep:
    """One shard's buffers and steps of a sequence-sharded decode step.

    desc describes this shard's own paged cache (block-table rows of
    max_pages_per_seq shard-local pages).  `all_gather(dst, src)` fills dst
    [N, *src.shape] with every shard's src in shard order; the default is
    torch.distributed.all_gather_into_tensor on `group` (NCCL between GPUs).
    Kernels and exchanges run on the current CUDA stream, in call order.
    """

    def __init__(self, desc, rank, num_shards, top_k, sink_tokens, local_tokens, device="cuda",
                 group=None, all_gather=None):
        B, H_q, H_kv, D = desc.batch, desc.num_q_heads, desc.num_kv_heads, desc.head_dim
        self.desc, self.rank, self.N = desc, rank, num_shards
        self.top_k, self.sink, self.local = top_k, sink_tokens, local_tokens
        self.k_local = min(top_k, desc.max_pages_per_seq)
        self.stride = seqshard_sel_stride(desc, top_k, sink_tokens, local_tokens)
        if self.stride > desc.max_pages_per_seq:
            raise LServeError("SeqShardStep", ERR_INVALID_ARG,
                              "merged selection row longer than the shard's block-table row")
        i32, f32 = torch.int32, torch.float32
        self.sel = torch.empty((B, H_kv, self.k_local), dtype=i32, device=device)
        self.cnt = torch.empty((B, H_kv), dtype=i32, device=device)
        self.scores = torch.empty((B, H_kv, desc.max_pages_per_seq), dtype=f32, device=device)
        self.cand_s = torch.empty((B, H_kv, top_k), dtype=f32, device=device)
        self.cand_p = torch.empty((B, H_kv, top_k), dtype=i32, device=device)
        self.all_s = torch.empty((num_shards, B, H_kv, top_k), dtype=f32, device=device)
        self.all_p = torch.empty((num_shards, B, H_kv, top_k), dtype=i32, device=device)
        self.sel_m = torch.empty((B, H_kv, self.stride), dtype=i32, device=device)
        self.cnt_m = torch.empty((B, H_kv), dtype=i32, device=device)
        self.all_heads = torch.zeros(H_kv, dtype=torch.uint8, device=device)
        self.o = torch.empty((B * H_q, D), dtype=f32, device=device)
        self.lse = torch.empty(B * H_q, dtype=f32, device=device)
        self.all_o = torch.empty((num_shards, B * H_q, D), dtype=f32, device=device)
        self.all_lse = torch.empty((num_shards, B * H_q), dtype=f32, device=device)
        self.ws_dec = alloc_workspace(workspace_size(OP_DECODE, desc, self.stride), device)
        self.all_gather = all_gather if all_gather is not None else process_group_all_gather(group)

    def select(self, q, stats_pool, block_table, ctx_lens_local, ctx_lens_global, head_kind):
        """Steps 1-4: the shard's scores and own top-K, its proposals, their
        exchange and the merge.  The result (sel_m, cnt_m) may be reused for
        several decode steps."""
        page_select(self.desc, q, stats_pool, block_table, ctx_lens_local, head_kind, self.k_local,
                    self.sel, self.cnt, phys_scores=self.scores)
        seqshard_candidates(self.desc, self.rank, self.N, ctx_lens_global, head_kind, self.sel, self.cnt,
                            self.scores, self.top_k, self.cand_s, self.cand_p)
        self.all_gather(self.all_s, self.cand_s)
        self.all_gather(self.all_p, self.cand_p)
        seqshard_merge(self.desc, self.rank, self.N, ctx_lens_global, head_kind, self.all_s, self.all_p,
                       self.top_k, self.sink, self.local, self.sel_m, self.cnt_m)

    def attend(self, q, k_pool, v_pool, block_table, ctx_lens_local, softmax_scale, out, lse=None):
        """Steps 5-7: attention over the shard's chosen pages (float partials),
        their exchange and the log-sum-exp combine into out bf16 [B][H_q][D]."""
        sparse_decode_attn(self.desc, q, k_pool, v_pool, block_table, ctx_lens_local, self.all_heads,
                           self.sel_m, self.cnt_m, self.stride, self.sink, self.local, softmax_scale,
                           self.o, self.lse, workspace=self.ws_dec, out_f32=True)
        self.all_gather(self.all_o, self.o)
        self.all_gather(self.all_lse, self.lse)
        seqshard_combine(self.all_o, self.all_lse, out.view(-1, out.shape[-1]),
                         None if lse is None else lse.view(-1))


def read_device_status(stream=None) -> int:
    return lib.lserve_read_device_status(_stream(stream))


def set_wait_limit_cycles(cycles: int) -> None:
    lib.lserve_set_wait_limit_cycles(cycles)


def debug_wait_timeout(cycles: int, stream=None):
    _check("lserve_debug_wait_timeout", lib.lserve_debug_wait_timeout(cycles, _stream(stream)))


def alloc_workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """Caller-owned workspace: 256-byte aligned (caching allocator) and
    zero-filled, as lserve_sparse_decode_attn requires before its first use."""
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device)
