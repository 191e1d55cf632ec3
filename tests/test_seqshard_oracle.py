"""Pins for the oracle's sequence-sharded decode (reading R17) and the exchange
protocol run as two gloo ranks on the CPU.

The sharded decode must change no result: the global top-K re-made from every
shard's own top-K is the unsharded top-K, and attention over disjoint token
sets merged by their log-sum-exp is attention over the union.  Both are
checked against routines that know nothing of shards: brute-force enumeration
of the top-K set, torch's scaled_dot_product_attention and scipy's logsumexp.
"""
import itertools
import math
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp
from scipy.special import logsumexp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402


def _brute_top_k(P, K):
    """The unique K-set (all pages if fewer) whose every member beats every
    non-member by (score descending, index ascending), found by enumeration."""
    M = len(P)
    K = min(K, M)
    won = []
    for X in itertools.combinations(range(M), K):
        rest = [m for m in range(M) if m not in X]
        if all(P[a] > P[b] or (P[a] == P[b] and a < b) for a in X for b in rest):
            won.append(list(X))
    assert len(won) == 1
    return won[0]


def _sharded_top_k(P, K, N):
    b = oracle.shard_bounds(len(P), N)
    cands = []
    for r in range(N):
        cands += oracle.shard_candidates(P[b[r]:b[r + 1]], K, b[r])
    return oracle.merge_candidates(cands, K, len(P))


def test_shard_bounds_partition_the_pages():
    assert oracle.shard_bounds(10, 4) == [0, 2, 5, 7, 10]
    assert oracle.shard_bounds(3, 4) == [0, 0, 1, 2, 3]      # fewer pages than shards
    for M in range(0, 40):
        for N in range(1, 9):
            b = oracle.shard_bounds(M, N)
            assert b[0] == 0 and b[-1] == M
            sizes = [b[r + 1] - b[r] for r in range(N)]
            assert min(sizes) >= 0 and max(sizes) - min(sizes) <= 1


@pytest.mark.parametrize("M", [1, 4, 7, 10])
def test_sharded_top_k_is_the_global_top_k(M):
    rng = np.random.default_rng(100 + M)
    for trial in range(5):
        P = rng.integers(0, 3, size=M).astype(np.float64)  # many exact ties
        if trial % 2:
            P = rng.standard_normal(M)
        for N in (1, 2, 3, 5):
            for K in range(1, M + 2):
                assert _sharded_top_k(P, K, N) == _brute_top_k(P, K), (P, N, K)


def test_sharded_top_k_ties_across_a_shard_boundary():
    # equal scores on both sides of the boundary: the lower global index wins
    P = np.array([0.0, 5.0, 5.0, 5.0, 5.0, 1.0])
    assert _sharded_top_k(P, 2, 2) == [1, 2]
    assert _sharded_top_k(P, 3, 2) == [1, 2, 3]
    assert _sharded_top_k(P, 3, 3) == [1, 2, 3]


@pytest.mark.parametrize("n,N_P,S,L,N", [(1000, 64, 64, 256, 2), (1000, 64, 64, 256, 4),
                                         (262144, 128, 128, 1024, 8), (300, 64, 64, 256, 8),
                                         (5, 64, 64, 256, 3)])
def test_shard_streaming_pages_cover_the_streaming_set_once(n, N_P, S, L, N):
    M = -(-n // N_P)
    b = oracle.shard_bounds(M, N)
    got = []
    for r in range(N):
        got += [b[r] + m for m in oracle.shard_streaming_pages(n, N_P, S, L, b[r], b[r + 1])]
    assert got == oracle.streaming_pages(n, N_P, S, L)


def _sdpa(q, k, v, scale):
    out = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None], torch.from_numpy(k)[None], torch.from_numpy(v)[None], scale=scale)
    return out[0].numpy()


@pytest.mark.parametrize("N", [1, 2, 3, 6])
def test_lse_combine_of_disjoint_sets_is_attention_over_the_union(N):
    rng = np.random.default_rng(7 + N)
    n, G, D = 97, 4, 16
    q, k, v = rng.standard_normal((G, D)), rng.standard_normal((n, D)), rng.standard_normal((n, D))
    scale = 1 / math.sqrt(D)
    tokens = rng.permutation(n)
    cuts = sorted(rng.integers(0, n, size=N - 1).tolist())
    parts = np.split(tokens, cuts)                      # some parts may be empty
    outs = [oracle.decode_attention(q, k, v, np.sort(t), scale) for t in parts]
    o, lse = oracle.lse_combine([x[0] for x in outs], [x[1] for x in outs])
    assert np.allclose(o, _sdpa(q, k, v, scale), rtol=1e-12, atol=1e-12)
    assert np.allclose(lse, logsumexp(scale * q @ k.T, axis=1), rtol=1e-13)


def test_lse_combine_closed_forms():
    o_parts = np.array([[[1.0, 2.0]], [[3.0, -4.0]]])
    # equal normalisers: the plain mean
    o, lse = oracle.lse_combine(o_parts, np.array([[0.5], [0.5]]))
    assert np.allclose(o, [[2.0, -1.0]]) and np.allclose(lse, [0.5 + math.log(2)])
    # an empty set (lse = -inf) weighs nothing
    o, lse = oracle.lse_combine(o_parts, np.array([[-np.inf], [1.25]]))
    assert np.allclose(o, [[3.0, -4.0]]) and np.allclose(lse, [1.25])
    # every set empty: zero output, -inf
    o, lse = oracle.lse_combine(np.zeros((3, 1, 2)), np.full((3, 1), -np.inf))
    assert np.all(o == 0) and lse[0] == -np.inf


# --- the exchange, as two gloo ranks ----------------------------------------------------

def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, ws, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws)
    try:
        rng = np.random.default_rng(5)                  # same full problem on every rank
        M, K, n_tok, G, D = 37, 8, 37 * 4, 2, 8
        P = np.round(rng.standard_normal(M), 1)         # rounded: ties across shards
        qv = rng.standard_normal((G, D))
        kk = rng.standard_normal((n_tok, D))
        vv = rng.standard_normal((n_tok, D))
        b = oracle.shard_bounds(M, ws)
        lo, hi = b[rank], b[rank + 1]
        # 1. this shard's proposals, padded to K, exchanged with all_gather
        mine = oracle.shard_candidates(P[lo:hi], K, lo)
        score = torch.full((K,), -math.inf, dtype=torch.float64)
        page = torch.full((K,), -1, dtype=torch.int64)
        for i, (s_, m_) in enumerate(mine):
            score[i], page[i] = s_, m_
        all_s = [torch.empty_like(score) for _ in range(ws)]
        all_p = [torch.empty_like(page) for _ in range(ws)]
        dist.all_gather(all_s, score)
        dist.all_gather(all_p, page)
        cands = [(float(s_), int(m_)) for S_, P_ in zip(all_s, all_p)
                 for s_, m_ in zip(S_.tolist(), P_.tolist()) if m_ >= 0]
        chosen = oracle.merge_candidates(cands, K, M)
        # 2. attention over the chosen pages this shard holds (4 tokens a page)
        toks = np.array([t for m in chosen if lo <= m < hi for t in range(4 * m, 4 * m + 4)], dtype=np.int64)
        o, lse = oracle.decode_attention(qv, kk, vv, toks, 0.3)
        all_o = [torch.empty(G, D, dtype=torch.float64) for _ in range(ws)]
        all_l = [torch.empty(G, dtype=torch.float64) for _ in range(ws)]
        dist.all_gather(all_o, torch.from_numpy(o))
        dist.all_gather(all_l, torch.from_numpy(lse))
        o_m, lse_m = oracle.lse_combine([x.numpy() for x in all_o], [x.numpy() for x in all_l])
        # the unsharded answer
        want = oracle.select_top_k(P, K)
        all_toks = np.array([t for m in want for t in range(4 * m, 4 * m + 4)], dtype=np.int64)
        o_ref, lse_ref = oracle.decode_attention(qv, kk, vv, all_toks, 0.3)
        q.put((rank, chosen == want, float(np.abs(o_m - o_ref).max()), float(np.abs(lse_m - lse_ref).max())))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_exchange_proposals_and_partials():
    ws = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, ws, port, q)) for r in range(ws)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(ws))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, same_sel, err_o, err_l in res:
        assert same_sel, rank
        assert err_o < 1e-12 and err_l < 1e-12, (rank, err_o, err_l)


# --- the exchange SeqShardStep uses by default, as two gloo ranks ---------------------

def _gather_main(rank, ws, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws)
    try:
        import block_sparse_attention_page_b200 as lserve
        ag = lserve.process_group_all_gather()
        # a rank's proposals (score, page) and partials, tagged by the rank
        score = torch.full((2, 3, 4), float(rank) + 0.5)
        page = torch.arange(24, dtype=torch.int32).reshape(2, 3, 4) + 100 * rank
        all_s = torch.empty((ws, 2, 3, 4))
        all_p = torch.empty((ws, 2, 3, 4), dtype=torch.int32)
        ag(all_s, score)
        ag(all_p, page)
        lse = torch.arange(5, dtype=torch.float32) - rank       # 1-D, like the lse partials
        all_l = torch.empty((ws, 5))
        ag(all_l, lse)
        ok = all(torch.all(all_s[r] == r + 0.5) and
                 torch.equal(all_p[r], torch.arange(24, dtype=torch.int32).reshape(2, 3, 4) + 100 * r) and
                 torch.equal(all_l[r], torch.arange(5, dtype=torch.float32) - r)
                 for r in range(ws))
        q.put((rank, bool(ok)))
    finally:
        dist.destroy_process_group()


def test_default_exchange_places_every_shard_in_order():
    ws = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_gather_main, args=(r, ws, port, q)) for r in range(ws)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(ws))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res == [(0, True), (1, True)]
