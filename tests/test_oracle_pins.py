"""Pins for the CPU oracle: checks against what the LServe pages and plain
mathematics fix, independent of the oracle's own formulas.

Each check is chosen so that a plausible slip in the oracle (a dropped term, a
wrong sign, a swapped min/max, an off-by-one page boundary, ties going the
wrong way) fails at least one of them.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _rng(seed):
    return np.random.default_rng(seed)


def _bf16_values(rng, shape, scale=1.0):
    """Random bf16-representable float64 values."""
    return oracle.widen_bf16(synth.to_bf16(rng.standard_normal(shape) * scale))


# --- bf16 widening --------------------------------------------------------------

def test_widen_bf16_known_encodings():
    # IEEE bfloat16: sign | 8-bit exponent (bias 127) | 7-bit fraction
    bits = np.array([0x3F80, 0xC000, 0x3FC0, 0x0000, 0x8000, 0x4049, 0x7F7F], dtype=np.uint16)
    want = [1.0, -2.0, 1.5, 0.0, -0.0, 3.140625, 3.3895313892515355e38]
    got = oracle.widen_bf16(bits)
    assert list(got) == want


# --- page statistics ------------------------------------------------------------

@pytest.mark.parametrize("n,N_L,D", [(64, 16, 8), (70, 16, 5), (1, 16, 3), (33, 1, 4)])
def test_page_stats_bounds_are_tight(n, N_L, D):
    """min/max are characterised by: every key of the page lies inside
    [k_min, k_max] channel-wise, and each bound is attained by one of them."""
    rng = _rng(n * 7 + D)
    k = _bf16_values(rng, (n, D))
    kmin, kmax = oracle.page_stats(k, N_L)
    J = -(-n // N_L)
    assert kmin.shape == (J, D) and kmax.shape == (J, D)
    for j in range(J):
        rows = k[j * N_L:min((j + 1) * N_L, n)]
        assert np.all(rows >= kmin[j]) and np.all(rows <= kmax[j])
        for i in range(D):
            assert kmin[j, i] in rows[:, i] and kmax[j, i] in rows[:, i]


def test_page_stats_partial_page_ignores_missing_tokens():
    # 17 tokens at N_L=16: the second logical page holds exactly token 16
    k = np.arange(17 * 2, dtype=np.float64).reshape(17, 2)
    kmin, kmax = oracle.page_stats(k, 16)
    assert np.array_equal(kmin[1], k[16]) and np.array_equal(kmax[1], k[16])
    assert np.array_equal(kmin[0], k[0]) and np.array_equal(kmax[0], k[15])


def test_page_stats_single_token_pages_are_the_keys():
    k = _bf16_values(_rng(3), (9, 6))
    kmin, kmax = oracle.page_stats(k, 1)
    assert np.array_equal(kmin, k) and np.array_equal(kmax, k)


# --- query-centric score S^j ---------------------------------------------------------

def test_score_is_max_of_linear_form_over_the_stats_box():
    """sum_i max(q_i kmax_i, q_i kmin_i) is the maximum of q.x over the box
    prod_i [kmin_i, kmax_i]; a linear form attains it at a corner, so brute
    force over all 2^D corners must agree."""
    rng = _rng(11)
    D = 6
    for trial in range(20):
        lo = rng.standard_normal(D)
        hi = lo + np.abs(rng.standard_normal(D))
        q = rng.standard_normal((1, D))
        if trial == 0:
            q[0, :3] = 0.0
        best = max(float(q[0] @ np.array(c)) for c in itertools.product(*zip(lo, hi)))
        s = oracle.head_scores(q, lo[None], hi[None])[0, 0]
        assert s == pytest.approx(best, rel=1e-12, abs=1e-12)


def test_score_worked_example():
    # q = (1, -2, 0.5); kmin = (-1, -1, 2); kmax = (3, 1, 4):
    # channel 1: max(1*3, 1*-1) = 3; channel 2: max(-2*1, -2*-1) = 2;
    # channel 3: max(0.5*4, 0.5*2) = 2; total 7
    s = oracle.head_scores(np.array([[1.0, -2.0, 0.5]]), np.array([[-1.0, -1.0, 2.0]]),
                           np.array([[3.0, 1.0, 4.0]]))
    assert s[0, 0] == 7.0


def test_score_upper_bounds_every_key_in_the_page():
    """The page describes S^j as an upper-bound estimate of q.k within the page."""
    rng = _rng(5)
    n, N_L, D, G = 16 * 12 + 5, 16, 32, 4
    k = _bf16_values(rng, (n, D), 2.0)
    q = _bf16_values(rng, (G, D))
    kmin, kmax = oracle.page_stats(k, N_L)
    s = oracle.head_scores(q, kmin, kmax)
    S = oracle.logical_scores(q, kmin, kmax)
    for j in range(kmin.shape[0]):
        rows = k[j * N_L:min((j + 1) * N_L, n)]
        dots = q @ rows.T                                   # [G][tokens]
        assert np.all(s[:, j] >= dots.max(axis=1) - 1e-12 * np.abs(dots).max())
        # the summed (GQA) score bounds the summed logit of every key
        assert S[j] >= dots.sum(axis=0).max() - 1e-12 * np.abs(dots).sum()


def test_score_special_cases():
    rng = _rng(9)
    kmin = rng.standard_normal((3, 8))
    kmax = kmin + 1.0
    assert np.all(oracle.head_scores(np.zeros((2, 8)), kmin, kmax) == 0.0)
    # a page of identical keys: the box is a point and the score is q.k exactly
    key = rng.standard_normal(8)
    q = rng.standard_normal((2, 8))
    s = oracle.head_scores(q, key[None], key[None])
    assert np.allclose(s[:, 0], q @ key, rtol=1e-14, atol=1e-14)


def test_logical_score_sums_query_heads():
    rng = _rng(21)
    q = rng.standard_normal((4, 8))
    kmin = rng.standard_normal((5, 8))
    kmax = kmin + 0.5
    per_head = [oracle.head_scores(q[h:h + 1], kmin, kmax)[0] for h in range(4)]
    assert np.allclose(oracle.logical_scores(q, kmin, kmax), np.sum(per_head, axis=0))


# --- logical -> physical max ----------------------------------------------------------

def test_physical_score_is_max_of_its_logical_pages():
    rng = _rng(4)
    S = rng.standard_normal(4 * 9 + 3)
    P = oracle.physical_scores(S, 4)
    assert len(P) == 10
    for m in range(10):
        part = S[m * 4:(m + 1) * 4]
        assert P[m] in part and np.all(P[m] >= part)
    assert np.array_equal(oracle.physical_scores(S, 1), S)


def test_physical_score_is_tighter_than_scoring_the_whole_physical_page():
    """Max over logical sub-boxes <= score of the physical page's own (looser) box."""
    rng = _rng(8)
    k = _bf16_values(rng, (256, 16))
    q = _bf16_values(rng, (2, 16))
    P = oracle.physical_scores(oracle.logical_scores(q, *oracle.page_stats(k, 16)), 4)
    Pbox = oracle.logical_scores(q, *oracle.page_stats(k, 64))
    assert np.all(P <= Pbox + 1e-12)


# --- top-K selection ---------------------------------------------------------------

def _valid_topk_sets(P, K):
    """All K-subsets X such that every chosen page beats every other page:
    higher score, or equal score and lower index."""
    M = len(P)
    out = []
    for X in itertools.combinations(range(M), min(K, M)):
        Xs = set(X)
        ok = all(P[x] > P[y] or (P[x] == P[y] and x < y)
                 for x in Xs for y in range(M) if y not in Xs)
        if ok:
            out.append(list(X))
    return out


@pytest.mark.parametrize("M", [1, 3, 7, 10])
def test_topk_brute_force_with_ties(M):
    rng = _rng(M)
    for trial in range(6):
        P = rng.integers(0, 4, size=M).astype(np.float64)  # many exact ties
        if trial % 2:
            P = rng.standard_normal(M)
        for K in range(1, M + 2):
            valid = _valid_topk_sets(P, K)
            assert len(valid) == 1
            assert oracle.select_top_k(P, K) == valid[0]


def test_topk_tie_goes_to_lowest_index():
    assert oracle.select_top_k(np.array([1.0, 2.0, 2.0, 2.0, 0.5]), 2) == [1, 2]
    assert oracle.select_top_k(np.array([3.0, 3.0, 3.0]), 5) == [0, 1, 2]


# --- streaming page set (reading R5) ---------------------------------------------------

@pytest.mark.parametrize("n,N_P,S,L", [(1000, 64, 64, 256), (2048, 64, 64, 256), (300, 64, 64, 256),
                                       (65536, 64, 128, 512), (262144, 128, 128, 1024),
                                       (8193, 64, 64, 512), (5, 64, 64, 256), (129, 64, 0, 1)])
def test_streaming_pages_cover_sink_and_local_tokens(n, N_P, S, L):
    pages = oracle.streaming_pages(n, N_P, S, L)
    toks = set(oracle.page_tokens(pages, n, N_P).tolist())
    need = set(range(min(S, n))) | set(range(max(0, n - L), n))
    assert need <= toks                       # every sink and local token attended
    for m in pages:                           # and no page without one of them
        assert any(t in need for t in range(m * N_P, min((m + 1) * N_P, n)))
    assert pages == sorted(set(pages))


def test_streaming_pages_worked_example():
    # n=1000, N_P=64, sink 64, local 256: sink page 0; the last 256 tokens are
    # 744..999, i.e. pages 11 (704..767) to 15 (960..999)
    assert oracle.streaming_pages(1000, 64, 64, 256) == [0, 11, 12, 13, 14, 15]


# --- decode attention ----------------------------------------------------------------

def _sdpa(q, k, v, scale, mask=None, causal=False):
    """torch's scaled_dot_product_attention in float64 on the CPU."""
    out = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None], torch.from_numpy(k)[None], torch.from_numpy(v)[None],
        attn_mask=None if mask is None else torch.from_numpy(mask)[None],
        is_causal=causal, scale=scale)
    return out[0].numpy()


def test_decode_all_pages_selected_equals_dense_attention():
    rng = _rng(17)
    n, D, G, N_P = 300, 32, 4, 64
    q = _bf16_values(rng, (G, D))
    k = _bf16_values(rng, (n, D))
    v = _bf16_values(rng, (n, D))
    scale = 1 / math.sqrt(D)
    # K >= #pages: every page selected, so sparse decode is dense decode
    o, lse, pages = oracle.decode_pair(q, k, v, n, 0, 16, N_P, 99, 0, 0, scale)
    assert pages == list(range(5))
    assert np.allclose(o, _sdpa(q, k, v, scale), rtol=1e-12, atol=1e-12)
    z = scale * q @ k.T
    from scipy.special import logsumexp
    assert np.allclose(lse, logsumexp(z, axis=1), rtol=1e-13)


def test_decode_streaming_short_context_is_dense():
    rng = _rng(18)
    n, D, G = 200, 16, 2
    q, k, v = (_bf16_values(rng, s) for s in [(G, D), (n, D), (n, D)])
    o, _, pages = oracle.decode_pair(q, k, v, n, 1, 16, 64, 1, 64, 256, 0.25)
    assert pages == [0, 1, 2, 3]
    assert np.allclose(o, _sdpa(q, k, v, 0.25), rtol=1e-12, atol=1e-12)


def test_decode_closed_forms():
    rng = _rng(19)
    D = 8
    q = rng.standard_normal((3, D))
    v = rng.standard_normal((5, D))
    # one valid key: the output is that value row
    o, _ = oracle.decode_attention(q, rng.standard_normal((5, D)), v, [3], 0.7)
    assert np.allclose(o, np.repeat(v[3:4], 3, axis=0), rtol=0, atol=1e-15)
    # identical keys: uniform weights, the output is the mean of V
    k = np.repeat(rng.standard_normal((1, D)), 5, axis=0)
    o, lse = oracle.decode_attention(q, k, v, range(5), 0.7)
    assert np.allclose(o, np.repeat(v.mean(axis=0, keepdims=True), 3, axis=0), atol=1e-14)
    assert np.allclose(lse, 0.7 * q @ k[0] + math.log(5), rtol=1e-14)
    # nothing to attend
    o, lse = oracle.decode_attention(q, k, v, [], 1.0)
    assert np.all(o == 0) and np.all(np.isneginf(lse))


def test_tiny_planted_pages_are_the_top_k():
    """The method exists to find the pages with the highest q.k: in the tiny
    workload the 8 pages holding a key planted at 4*qbar must be exactly the
    top-8 of the retrieval head, by a clear margin."""
    w = synth.tiny_decode()
    G = w.G
    q = oracle.widen_bf16(w.q[0, 0:G])
    k = oracle.widen_bf16(w.k_seq(0, 0))
    sel, P, _ = oracle.retrieval_pages(q, k, 2048, w.N_L, w.N_P, w.top_k)
    order = np.sort(P)[::-1]
    assert (order[7] - order[8]) / abs(order[7]) > 1e-3
    assert sel == w.planted_pages[(0, 0)]


# --- prefill -----------------------------------------------------------------------

def test_pages_speedup_example():
    g = _golden("speedup_example.json")
    assert oracle.theoretical_speedup(g["nonempty_blocks"], g["total_blocks"]) == \
        pytest.approx(g["speedup"], rel=0.005)


def test_block_counts_closed_forms():
    # dense causal over nb blocks visits nb(nb+1)/2 tiles
    for nb in [1, 2, 6, 32, 1024]:
        assert oracle.computed_blocks(nb, 0, 1, 4) == nb * (nb + 1) // 2
    # a 6-block causal triangle has 21 tiles, the total of the pages' example
    assert oracle.computed_blocks(6, 0, 1, 4) == _golden("speedup_example.json")["total_blocks"]
    # Lambda(1 sink, 4 local): rows 0..3 see 1..4 blocks, later rows 5
    assert oracle.computed_blocks(1024, 1, 1, 4) == 10 + 1020 * 5
    assert oracle.computed_blocks(32, 1, 1, 4) == 10 + 28 * 5
    # with at most sink+local blocks the Lambda mask is dense causal
    for nb in range(1, 6):
        assert all(oracle.kv_blocks(i, 1, 1, 4) == list(range(i + 1)) for i in range(nb))


def test_prefill_flops_of_the_128k_workload():
    hk = np.array([0, 0, 0, 0, 1, 1, 1, 1])
    f = oracle.prefill_flops(131072, 32, 8, 128, 128, hk, 1, 4)
    assert f == (16 * 524800 + 16 * 5110) * 4 * 128 ** 3


def test_prefill_dense_heads_equal_causal_attention():
    rng = _rng(23)
    T, D, B = 200, 16, 32
    q, k, v = (_bf16_values(rng, (T, D)) for _ in range(3))
    scale = 1 / math.sqrt(D)
    o, lse = oracle.prefill_rows(q, k, v, 0, B, 1, 4, scale, np.arange(T))
    assert np.allclose(o, _sdpa(q, k, v, scale, causal=True), rtol=1e-12, atol=1e-12)
    from scipy.special import logsumexp
    z = scale * q @ k.T
    z[np.triu_indices(T, 1)] = -np.inf
    assert np.allclose(lse, logsumexp(z, axis=1), rtol=1e-13)


def test_prefill_lambda_few_blocks_is_causal():
    rng = _rng(24)
    T, D, B = 5 * 16 - 3, 8, 16                 # 5 blocks, ragged tail
    q, k, v = (_bf16_values(rng, (T, D)) for _ in range(3))
    o, _ = oracle.prefill_rows(q, k, v, 1, B, 1, 4, 0.3, np.arange(T))
    assert np.allclose(o, _sdpa(q, k, v, 0.3, causal=True), rtol=1e-12, atol=1e-12)


def test_prefill_lambda_matches_masked_attention():
    """Reading R6 (parity unpinned by the pages): token s is visible to token t
    iff s <= t and (s is in the first block, or t's block minus s's block < 4)."""
    rng = _rng(25)
    T, D, B = 16 * 9 + 7, 8, 16
    q, k, v = (_bf16_values(rng, (T, D)) for _ in range(3))
    bt, bs = np.arange(T)[:, None] // B, np.arange(T)[None, :] // B
    visible = (np.arange(T)[None, :] <= np.arange(T)[:, None]) & ((bs == 0) | (bt - bs < 4))
    o, _ = oracle.prefill_rows(q, k, v, 1, B, 1, 4, 0.3, np.arange(T))
    assert np.allclose(o, _sdpa(q, k, v, 0.3, mask=visible), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("kind", [0, 1])
def test_prefill_block_rows_match_masked_attention(kind):
    """The block-at-a-time form against torch SDPA with the causal mask (dense
    heads) or the R6 Lambda mask (streaming heads), every block of a ragged
    sequence in full, and lse against scipy's logsumexp of the masked logits."""
    from scipy.special import logsumexp
    rng = _rng(26 + kind)
    T, D, B = 16 * 11 + 5, 8, 16
    q, k, v = (_bf16_values(rng, (T, D)) for _ in range(3))
    t_idx = np.arange(T)
    bt, bs = t_idx[:, None] // B, t_idx[None, :] // B
    visible = t_idx[None, :] <= t_idx[:, None]
    if kind == 1:
        visible &= (bs == 0) | (bt - bs < 4)
    want = _sdpa(q, k, v, 0.3, mask=visible)
    z = 0.3 * q @ k.T
    z[~visible] = -np.inf
    want_lse = logsumexp(z, axis=1)
    for i in range(-(-T // B)):
        rows = np.arange(i * B, min((i + 1) * B, T))
        o, lse = oracle.prefill_block_rows(q[rows], k, v, kind, B, 1, 4, 0.3, rows)
        assert np.allclose(o, want[rows], rtol=1e-12, atol=1e-12), i
        assert np.allclose(lse, want_lse[rows], rtol=1e-13, atol=1e-13), i
    # a scattered subset of one block's rows
    rows = np.array([16 * 9 + 1, 16 * 9 + 7, 16 * 9 + 15])
    o, _ = oracle.prefill_block_rows(q[rows], k, v, kind, B, 1, 4, 0.3, rows)
    assert np.allclose(o, want[rows], rtol=1e-12, atol=1e-12)


def test_prefill_block_rows_closed_forms():
    rng = _rng(28)
    T, D, B = 64, 8, 16
    q, k, v = (_bf16_values(rng, (T, D)) for _ in range(3))
    # row 0 sees only key 0: o = v[0], lse = scale * q0 . k0
    o, lse = oracle.prefill_block_rows(q[:1], k, v, 0, B, 1, 4, 0.5, [0])
    assert np.array_equal(o[0], v[0]) and lse[0] == pytest.approx(0.5 * q[0] @ k[0], rel=1e-15)
    # identical keys: the row is the mean of the values it may see
    kk = np.repeat(k[:1], T, axis=0)
    rows = np.arange(48, 64)
    o, _ = oracle.prefill_block_rows(q[rows], kk, v, 0, B, 1, 4, 0.5, rows)
    for r, t in enumerate(rows):
        assert np.allclose(o[r], v[:t + 1].mean(axis=0), rtol=1e-12, atol=1e-12)
    # rows of two different blocks are refused
    with pytest.raises(AssertionError):
        oracle.prefill_block_rows(q[[15, 16]], k, v, 0, B, 1, 4, 0.5, [15, 16])


def test_method_constants_in_workloads():
    c = _golden("method_constants.json")
    for make in synth.DECODE_CONFIGS.values():
        w = make() if make is not synth.mixed_batch_decode else None
        if w is None:
            continue
        assert w.N_L == c["logical_page"] and w.N_P % w.N_L == 0
        assert c["physical_page_range"][0] <= w.N_P <= c["physical_page_range"][1]
        assert np.mean(w.head_kind) == c["streaming_fraction"]


# --- quantized KV (R15) ---------------------------------------------------------

def _bits(x):
    return synth.to_bf16(np.asarray(x, dtype=np.float64))


def test_kv8_hand_example():
    # channel 0: amax 2 -> inv 63.5; 1 -> 63.5 -> 64 (half to even), -2 -> -127, 0.5 -> 31.75 -> 32
    x = _bits([[1.0, 0.0], [-2.0, 0.0], [0.5, 0.0]])
    codes, scale = oracle.quantize_kv8(x)
    assert codes[:, 0].tolist() == [64, -127, 32]
    assert codes[:, 1].tolist() == [0, 0, 0] and scale[1] == 0.0   # all-zero channel
    assert scale[0] == np.float32(2.0) / np.float32(127.0)


def test_kv8_round_trip_error_and_range():
    rng = np.random.default_rng(11)
    x = _bits(rng.normal(size=(64, 128)) * rng.uniform(0.5, 8, size=128))
    codes, scale = oracle.quantize_kv8(x)
    assert codes.min() >= -127 and codes.max() <= 127
    xf = oracle.widen_bf16(x)
    amax = np.abs(xf).max(axis=0)
    # the largest magnitude of each channel maps to +-127
    j = np.abs(xf).argmax(axis=0)
    assert np.all(np.abs(codes[j, np.arange(128)]) == 127)
    back = oracle.dequantize_kv8(codes, scale)
    # quantization error <= half a step (plus the float32 rounding of the
    # scale and of the product that decided the code)
    bound = amax / 127 / 2 * (1 + 1e-5)
    assert np.all(np.abs(back - xf) <= bound[None, :])


def test_kv8_is_odd_and_scale_invariant():
    rng = np.random.default_rng(12)
    x = _bits(rng.normal(size=(16, 64)))
    c1, s1 = oracle.quantize_kv8(x)
    c2, s2 = oracle.quantize_kv8(x ^ np.uint16(0x8000))          # negate every value
    assert np.array_equal(c2, -c1) and np.array_equal(s1, s2)
    c4, s4 = oracle.quantize_kv8(_bits(oracle.widen_bf16(x) * 4))  # exact power-of-two scaling
    assert np.array_equal(c4, c1) and np.allclose(s4, 4 * s1, rtol=0, atol=0)


def test_dequantized_seq_pages_are_independent():
    rng = np.random.default_rng(13)
    x = _bits(rng.normal(size=(150, 32)))
    whole = oracle.dequantized_seq(x, 64)
    for t0 in (0, 64, 128):
        c, s = oracle.quantize_kv8(x[t0:t0 + 64])
        assert np.array_equal(whole[t0:t0 + 64], oracle.dequantize_kv8(c, s))


def test_kv8_lossless_on_grid_values():
    # integers in [-127, 127] times a per-channel power of two, each channel
    # reaching +-127: the codes are the integers and the round trip is exact
    rng = np.random.default_rng(14)
    ints = rng.integers(-127, 128, size=(40, 16))
    ints[3] = 127
    ints[7, ::2] = -127
    step = 2.0 ** rng.integers(-6, 3, size=16)
    x = _bits(ints * step)
    codes, scale = oracle.quantize_kv8(x)
    assert np.array_equal(np.abs(codes.astype(np.int64)), np.abs(ints))
    assert np.array_equal(codes.astype(np.int64), ints)
    assert np.array_equal(oracle.dequantize_kv8(codes, scale), oracle.widen_bf16(x))


def test_kv4_hand_example():
    # channel 0: amax 2 -> inv 3.5; 1 -> 3.5 -> 4 (half to even), -2 -> -7, 0.5 -> 1.75 -> 2
    # channel 1: amax 7 -> inv 1; 2.5 -> 2 and 3.5 -> 4 (half to even), -7 -> -7
    x = _bits([[1.0, 2.5], [-2.0, 3.5], [0.5, -7.0]])
    codes, scale = oracle.quantize_kv4(x)
    assert codes[:, 0].tolist() == [4, -7, 2]
    assert codes[:, 1].tolist() == [2, 4, -7]
    assert scale[0] == np.float32(2.0) / np.float32(7.0) and scale[1] == np.float32(1.0)


def test_kv4_round_trip_error_and_range():
    rng = np.random.default_rng(15)
    x = _bits(rng.normal(size=(64, 128)) * rng.uniform(0.5, 8, size=128))
    codes, scale = oracle.quantize_kv4(x)
    assert codes.min() >= -7 and codes.max() <= 7
    xf = oracle.widen_bf16(x)
    amax = np.abs(xf).max(axis=0)
    j = np.abs(xf).argmax(axis=0)
    assert np.all(np.abs(codes[j, np.arange(128)]) == 7)
    back = oracle.dequantize_kv8(codes, scale)
    bound = amax / 7 / 2 * (1 + 1e-5)
    assert np.all(np.abs(back - xf) <= bound[None, :])
    # 4-bit codes are the 8-bit scheme with a coarser grid: same scales up to 127/7
    _, s8 = oracle.quantize_kv8(x)
    assert np.allclose(scale * 7, s8 * 127, rtol=1e-6)


def test_kv4_is_odd_and_lossless_on_its_grid():
    rng = np.random.default_rng(16)
    x = _bits(rng.normal(size=(16, 64)))
    c1, s1 = oracle.quantize_kv4(x)
    c2, s2 = oracle.quantize_kv4(x ^ np.uint16(0x8000))
    assert np.array_equal(c2, -c1) and np.array_equal(s1, s2)
    ints = rng.integers(-7, 8, size=(40, 16))
    ints[5] = 7
    step = 2.0 ** rng.integers(-6, 3, size=16)
    xg = _bits(ints * step)
    codes, scale = oracle.quantize_kv4(xg)
    assert np.array_equal(codes.astype(np.int64), ints)
    assert np.array_equal(oracle.dequantize_kv8(codes, scale), oracle.widen_bf16(xg))
    # a 4-bit dequantized sequence quantizes each page on its own
    whole = oracle.dequantized_seq(x, 8, bits=4)
    c, s = oracle.quantize_kv4(x[8:16])
    assert np.array_equal(whole[8:16], oracle.dequantize_kv8(c, s))


# --- tokens appended since the last selection (R10 option) -----------------------

def test_attended_tokens_recent_option_closed_forms():
    n, N_P = 300, 64                       # pages 0..4, the last holding tokens 256..299
    pages = [1, 3]
    base = oracle.page_tokens(pages, n, N_P)
    # no recent tokens, or none past n: the selected pages' tokens only
    assert np.array_equal(oracle.attended_tokens(pages, n, N_P), base)
    assert np.array_equal(oracle.attended_tokens(pages, n, N_P, recent_from=n), base)
    # every token recent: all n tokens, each once
    assert np.array_equal(oracle.attended_tokens(pages, n, N_P, recent_from=0), np.arange(n))
    # recent tokens inside a selected page add nothing
    assert np.array_equal(oracle.attended_tokens([1, 4], n, N_P, recent_from=290),
                          oracle.page_tokens([1, 4], n, N_P))
    # recent tokens outside the selection are added, in order
    got = oracle.attended_tokens(pages, n, N_P, recent_from=296)
    assert np.array_equal(got, np.concatenate([base, np.arange(296, 300)]))


def test_decode_with_every_token_recent_is_dense_attention():
    """recent_from = 0 turns any selection into dense attention over all n
    tokens (torch SDPA, fp64)."""
    rng = _rng(31)
    n, D, G = 150, 16, 3
    q, k, v = (_bf16_values(rng, s) for s in ((G, D), (n, D), (n, D)))
    toks = oracle.attended_tokens([0], n, 64, recent_from=0)
    o, _ = oracle.decode_attention(q, k, v, toks, 0.25)
    want = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[:, None], torch.from_numpy(k)[None].expand(G, n, D),
        torch.from_numpy(v)[None].expand(G, n, D), scale=0.25)[:, 0].numpy()
    assert np.allclose(o, want, rtol=1e-12, atol=1e-12)
