"""fp64 oracle functions -- test infrastructure only (see package docstring).

Every function follows one step of the method in the page's order:
  stats (k_min/k_max per logical page) -> S^j -> physical max -> top-K ->
  attention over the chosen pages; and, for prefill, the block iterator ->
  causal softmax attention over the allowed blocks.
"""
from __future__ import annotations

import math

import numpy as np


def widen_bf16(u16) -> np.ndarray:
    """bf16 bit patterns -> float64 (exact: a bf16 is the top half of a float32)."""
    u = np.asarray(u16, dtype=np.uint16)
    return (u.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# --- decode: page statistics [TD-dynamic] ------------------------------------

def page_stats(k: np.ndarray, N_L: int):
    """Channel-wise k_min^j / k_max^j of each logical page j.

    [TD-dynamic]: k_min^j[i] and k_max^j[i] are the min and max of channel i
    over the keys of logical page j.  R2: a partial last page uses only its
    valid tokens.  k is [n][D] float64; returns two [ceil(n/N_L)][D] arrays.
    """
    n, D = k.shape
    J = -(-n // N_L)
    full = n // N_L
    kmin = np.empty((J, D))
    kmax = np.empty((J, D))
    pages = k[:full * N_L].reshape(full, N_L, D)   # page j = rows [j*N_L, (j+1)*N_L)
    kmin[:full] = pages.min(axis=1)
    kmax[:full] = pages.max(axis=1)
    if J > full:                                   # partial last page: valid rows only
        kmin[full] = k[full * N_L:].min(axis=0)
        kmax[full] = k[full * N_L:].max(axis=0)
    return kmin, kmax


# --- decode: query-centric score [TD-dynamic, Eq. S^j] --------------------------

def head_scores(q: np.ndarray, kmin: np.ndarray, kmax: np.ndarray) -> np.ndarray:
    """s[h, j] = sum_{i=1..D} max(q_h[i] * k_max^j[i], q_h[i] * k_min^j[i]).

    [TD-dynamic], the equation for S^j, for each query head h of q [G][D].
    """
    q3 = q[:, None, :]
    return np.maximum(q3 * kmax[None, :, :], q3 * kmin[None, :, :]).sum(axis=2)


def logical_scores(q: np.ndarray, kmin: np.ndarray, kmax: np.ndarray) -> np.ndarray:
    """S^j for one KV head: reading R1, the sum over its G query heads of s[h, j]."""
    return head_scores(q, kmin, kmax).sum(axis=0)


# --- decode: logical -> physical max [TD-paging] --------------------------------

def physical_scores(S: np.ndarray, g: int) -> np.ndarray:
    """P^m = max of S^j over the (valid) logical pages j in [m*g, m*g + g).

    [TD-paging]: a physical page of N_P = g * N_L tokens is scored by the
    max-reduction of the scores of the logical pages it contains.
    """
    M = -(-len(S) // g)
    return np.array([S[m * g:min((m + 1) * g, len(S))].max() for m in range(M)])


# --- decode: top-K physical pages [TD-unified figure "Top-K物理ページ"] --------------

def select_top_k(P: np.ndarray, K: int) -> list:
    """The K highest-scoring physical pages (all of them if there are <= K).

    Ordering by (score descending, index ascending) puts ties on the lowest
    index (R4); the chosen set is returned in ascending page order.  [Abstract]:
    the page budget K is a constant, independent of the context length.
    """
    order = sorted(range(len(P)), key=lambda m: (-P[m], m))
    return sorted(order[:min(K, len(P))])


def retrieval_pages(q, k, n, N_L, N_P, K):
    """Retrieval-head page choice for one (sequence, KV head):
    stats -> S^j -> P^m -> top-K.  Returns (sel, P, S)."""
    kmin, kmax = page_stats(k[:n], N_L)
    S = logical_scores(q, kmin, kmax)
    P = physical_scores(S, N_P // N_L)
    return select_top_k(P, K), P, S


def streaming_pages(n: int, N_P: int, sink: int, local: int) -> list:
    """Pages a streaming head attends at decode (reading R5 of the Lambda mask
    [TD-static]): the sink pages [0, ceil(sink/N_P)) plus every page holding one
    of the last `local` tokens; ascending, without duplicates."""
    npages = -(-n // N_P)
    sink_pages = set(range(min(-(-sink // N_P), npages)))
    first_local = max(0, n - local) // N_P
    return sorted(sink_pages | set(range(first_local, npages)))


def page_tokens(pages, n: int, N_P: int) -> np.ndarray:
    """Valid token positions of the given physical pages (R2)."""
    out = [np.arange(m * N_P, min((m + 1) * N_P, n)) for m in pages]
    return np.concatenate(out) if out else np.zeros(0, dtype=np.int64)


# --- decode attention [TD-unified; "Top-K物理ページ" / "Λ型マスク"] -----------------

def decode_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, tokens, scale: float):
    """softmax(scale * q k_t) weighted sum of v_t over the given tokens, per head.

    q [G][D], k/v [n][D]; returns (o [G][D], lse [G]) with lse the natural log
    of sum_t exp(scale * q.k_t).  An empty token set gives o = 0, lse = -inf.
    """
    tokens = np.asarray(tokens, dtype=np.int64)
    G, D = q.shape
    if tokens.size == 0:
        return np.zeros((G, D)), np.full(G, -np.inf)
    z = scale * (q @ k[tokens].T)              # [G][T]
    zmax = z.max(axis=1, keepdims=True)
    e = np.exp(z - zmax)
    lsum = e.sum(axis=1)
    o = (e @ v[tokens]) / lsum[:, None]
    return o, zmax[:, 0] + np.log(lsum)


def attended_tokens(pages, n: int, N_P: int, recent_from=None) -> np.ndarray:
    """Token positions a decode step attends: the valid tokens of the given
    physical pages (R2) and, when recent_from is given (reading R10's option:
    retrieval heads also see every token appended since their selection was
    made, whose pages the reused selection may not hold), every position in
    [recent_from, n) -- a set, ascending, each token once."""
    toks = page_tokens(pages, n, N_P)
    if recent_from is None:
        return toks
    lo = max(0, min(int(recent_from), n))
    return np.union1d(toks, np.arange(lo, n)).astype(np.int64)


def decode_pair(q, k, v, n, kind, N_L, N_P, K, sink, local, scale):
    """One (sequence, KV head) of a decode step: retrieval heads pick top-K
    pages by S^j, streaming heads take sink + local pages; then attention.
    Returns (o [G][D], lse [G], pages)."""
    if kind == 0:
        pages = retrieval_pages(q, k, n, N_L, N_P, K)[0]
    else:
        pages = streaming_pages(n, N_P, sink, local)
    o, lse = decode_attention(q, k, v, page_tokens(pages, n, N_P), scale)
    return o, lse, pages


# --- sequence-sharded decode (one long sequence over N GPUs) -------------------
# Reading R17: the pages leave the multi-GPU split of one sequence open.  Shard
# r of N holds the contiguous physical pages [floor(M*r/N), floor(M*(r+1)/N))
# of a sequence of M pages; each shard scores its own pages, proposes its own
# top-K, the proposals are exchanged, and the global choice is re-made from
# them.  Attention runs per shard over the chosen pages it holds; the shards'
# (o, lse) are then merged by their softmax normalisers.

def shard_bounds(M: int, N: int) -> list:
    """[P_0, ..., P_N] with P_r = floor(M * r / N): shard r holds pages [P_r, P_{r+1})."""
    return [(M * r) // N for r in range(N + 1)]


def shard_candidates(P_shard: np.ndarray, K: int, first_page: int) -> list:
    """A shard's proposals: its own top-K pages (select_top_k on its scores),
    as (score, global page index) pairs."""
    return [(float(P_shard[m]), first_page + m) for m in select_top_k(P_shard, K)]


def merge_candidates(cands, K: int, M: int) -> list:
    """The global top-K re-made from every shard's proposals: the same order as
    select_top_k -- score descending, then global page index ascending -- and
    min(K, M) pages, returned ascending."""
    order = sorted(cands, key=lambda c: (-c[0], c[1]))
    return sorted(c[1] for c in order[:min(K, M)])


def shard_streaming_pages(n: int, N_P: int, sink: int, local: int, lo: int, hi: int) -> list:
    """A streaming head's pages (R5) that fall in shard pages [lo, hi), as shard-local ordinals."""
    return [m - lo for m in streaming_pages(n, N_P, sink, local) if lo <= m < hi]


def lse_combine(o_parts, lse_parts):
    """Attention over disjoint token sets merged into attention over their union.

    With o_r the softmax-weighted mean of v over set r and lse_r the natural log
    of that set's sum of exp(logit): M = max_r lse_r, w_r = exp(lse_r - M),
    o = sum_r w_r o_r / sum_r w_r and lse = M + log(sum_r w_r).  Sets with
    lse_r = -inf weigh nothing; if every set is empty, o = 0 and lse = -inf.
    o_parts [N][G][D], lse_parts [N][G]; returns (o [G][D], lse [G]).
    """
    o_parts = np.asarray(o_parts, dtype=np.float64)
    lse_parts = np.asarray(lse_parts, dtype=np.float64)
    N, G, D = o_parts.shape
    o = np.zeros((G, D))
    lse = np.full(G, -np.inf)
    for g in range(G):
        M = lse_parts[:, g].max()
        if M == -np.inf:
            continue
        w = np.exp(lse_parts[:, g] - M)
        o[g] = (w[:, None] * o_parts[:, g]).sum(axis=0) / w.sum()
        lse[g] = M + math.log(w.sum())
    return o, lse


# --- prefill: block iterator [TD-static, TD-unified] ---------------------------

def kv_blocks(i: int, kind: int, sink_blocks: int, local_blocks: int) -> list:
    """KV blocks that query block row i visits.

    Retrieval heads (kind 0): every block j <= i (dense causal, R7).
    Streaming heads (kind 1): the Lambda mask [TD-static] -- sink blocks
    [0, sink_blocks) and local blocks [i - local_blocks + 1, i] (R6).
    """
    if kind == 0:
        return list(range(i + 1))
    sink = set(range(min(sink_blocks, i + 1)))
    local = set(range(max(0, i - local_blocks + 1), i + 1))
    return sorted(sink | local)


def computed_blocks(nblocks: int, kind: int, sink_blocks: int, local_blocks: int) -> int:
    """Number of (query block, key block) tiles one head computes."""
    return sum(len(kv_blocks(i, kind, sink_blocks, local_blocks)) for i in range(nblocks))


def theoretical_speedup(nonempty: int, total: int) -> float:
    """[TD-unified]: at block sparsity r = 1 - nonempty/total the ideal
    speedup over computing every block is 1 / (1 - r)."""
    r = 1.0 - nonempty / total
    return 1.0 / (1.0 - r)


def prefill_flops(T, H_q, H_kv, D, block, head_kind, sink_blocks, local_blocks) -> float:
    """Work counted as the pages count it: full block tiles, 2 matmuls of
    2*block*block*D flops each, per query head."""
    nb = -(-T // block)
    G = H_q // H_kv
    tiles = sum(G * computed_blocks(nb, int(head_kind[h]), sink_blocks, local_blocks)
                for h in range(H_kv))
    return tiles * 4.0 * block * block * D


# --- prefill attention [TD-unified; Abstract "skipped block-wise"] -------------

def prefill_rows(q: np.ndarray, k: np.ndarray, v: np.ndarray, kind: int, block: int,
                 sink_blocks: int, local_blocks: int, scale: float, rows):
    """Causal softmax attention of the given query rows of ONE query head over
    the keys of the blocks kv_blocks() allows (keys s <= t only).

    q [rows][D] holds the query vectors of `rows` (token positions);
    k, v [T][D] the head's keys/values.  Returns (o [rows][D], lse [rows]).
    """
    rows = np.asarray(rows, dtype=np.int64)
    T, D = k.shape
    o = np.empty((len(rows), D))
    lse = np.empty(len(rows))
    for r, t in enumerate(rows):
        i = int(t) // block
        keys = np.concatenate([np.arange(j * block, min((j + 1) * block, T))
                               for j in kv_blocks(i, kind, sink_blocks, local_blocks)])
        keys = keys[keys <= t]
        z = scale * (k[keys] @ q[r])
        zmax = z.max()
        e = np.exp(z - zmax)
        lsum = e.sum()
        o[r] = (e @ v[keys]) / lsum
        lse[r] = zmax + math.log(lsum)
    return o, lse


def prefill_block_rows(q: np.ndarray, k: np.ndarray, v: np.ndarray, kind: int, block: int,
                       sink_blocks: int, local_blocks: int, scale: float, rows):
    """The same attention as prefill_rows for rows that all lie in ONE query
    block i [TD-unified; TD-static]: every such row may see the same key blocks
    kv_blocks(i), so their logits are one matrix product over those blocks
    (keys s > t masked out of row t), followed by each row's softmax.  Used for
    the long-sequence checks, where a row-by-row gather of up to T keys would
    dominate the run time.

    q [rows][D]; k, v [T][D] (one head).  Returns (o [rows][D], lse [rows]).
    """
    rows = np.asarray(rows, dtype=np.int64)
    T, D = k.shape
    i = int(rows[0]) // block
    assert np.all(rows // block == i), "rows of one query block only"
    blocks = kv_blocks(i, kind, sink_blocks, local_blocks)
    keys = np.concatenate([np.arange(j * block, min((j + 1) * block, T)) for j in blocks])
    # the allowed blocks are ascending and their union is a few contiguous runs:
    # gather them as slices (views) rather than by index
    runs, start = [], keys[0]
    for a, b in zip(keys[:-1], keys[1:]):
        if b != a + 1:
            runs.append((start, a + 1))
            start = b
    runs.append((start, keys[-1] + 1))
    ks = k[runs[0][0]:runs[0][1]] if len(runs) == 1 else np.concatenate([k[a:b] for a, b in runs])
    vs = v[runs[0][0]:runs[0][1]] if len(runs) == 1 else np.concatenate([v[a:b] for a, b in runs])
    z = scale * (q @ ks.T)                      # [rows][keys]
    z[keys[None, :] > rows[:, None]] = -np.inf  # causal: keys s <= t only
    zmax = z.max(axis=1, keepdims=True)
    e = np.exp(z - zmax)
    lsum = e.sum(axis=1)
    o = (e @ vs) / lsum[:, None]
    lse = zmax[:, 0] + np.log(lsum)
    return o, lse


# --- quantized KV cache [R15, R18] -------------------------------------------
# The pages name KV-cache quantization (QServe KV4, combined with LServe's
# sparsity in the abstract page) but give no scheme.  R15 reading: symmetric
# int8 with one scale per (pool page, KV head, channel) over the page's valid
# tokens; R18: the same with 4-bit codes (-7..7).  The integer codes are
# decided in float32 exactly as written below so that both sides take the
# same decision; the attention attends the value code * scale (a real number,
# exact in float64 here; each side rounds it as its own arithmetic does).

def quantize_kv(x_bits: np.ndarray, qmax: int):
    """Codes and scales of one page of one KV head, symmetric with codes in
    [-qmax, qmax] (qmax = 127: 8-bit codes, R15; qmax = 7: 4-bit codes, R18).

    x_bits: bf16 bits [t][D] of the page's valid tokens (t >= 1).
    amax_c = max_t |x[t][c]| (exact in float32); inv_c = float32(qmax) /
    float32(amax_c); code = rint(float32(x) * inv_c) (float32 product, round
    half to even), clamped to [-qmax, qmax]; scale_c = float32(amax_c) /
    float32(qmax).  A channel with amax 0 gets codes 0 and scale 0.
    Returns (codes int8 [t][D], scale float32 [D]).
    """
    x = widen_bf16(x_bits).astype(np.float32)
    q = np.float32(qmax)
    amax = np.max(np.abs(x), axis=0).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        inv = np.where(amax > 0, q / amax, np.float32(0.0)).astype(np.float32)
    prod = (x * inv[None, :]).astype(np.float32)
    codes = np.clip(np.rint(prod), -qmax, qmax).astype(np.int8)
    scale = (amax / q).astype(np.float32)
    return codes, scale


def quantize_kv8(x_bits: np.ndarray):
    """8-bit codes (R15): quantize_kv with qmax = 127."""
    return quantize_kv(x_bits, 127)


def quantize_kv4(x_bits: np.ndarray):
    """4-bit codes (R18): quantize_kv with qmax = 7 (codes -7..7, so a code
    and its negation are both representable in a signed nibble)."""
    return quantize_kv(x_bits, 7)


def dequantize_kv8(codes: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """code * scale per element, float64 (exact: an 8-bit integer times a
    24-bit significand).  The same for 4-bit codes."""
    return codes.astype(np.float64) * scale.astype(np.float64)[None, :]


def dequantized_seq(x_bits: np.ndarray, N_P: int, bits: int = 8) -> np.ndarray:
    """A sequence's K or V ([n][D] bf16 bits) as the quantized cache holds it:
    each physical page of N_P tokens quantized on its own valid tokens with
    `bits`-bit codes, then dequantized (float64 [n][D])."""
    qmax = {8: 127, 4: 7}[bits]
    n = x_bits.shape[0]
    out = np.empty(x_bits.shape, dtype=np.float64)
    for t0 in range(0, n, N_P):
        c, s = quantize_kv(x_bits[t0:t0 + N_P], qmax)
        out[t0:t0 + N_P] = dequantize_kv8(c, s)
    return out
