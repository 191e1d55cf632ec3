"""GPU parity of the block-sparse prefill (tcgen05 kernel) against the fp64
oracle: every row on small shapes (several query/key tiles, ragged tails, both
head kinds, 64- and 128-token mask blocks, D = 64 and 128), every row of 18 of
the 32 query heads of a 16K-token sequence (many work units per CTA), and the
128K-token workload's stratified sample (per query head: the first two and the
last two query blocks, 8 random blocks and 256 random rows)."""
import math

import numpy as np
import pytest
import torch

import block_sparse_attention_page_b200 as lserve
import oracle
import synth
from synth.device import PrefillBuffers, bf16_bits

from parity import LSE_ABS, OUT_MAX_ABS, OUT_MEAN_ABS

pytestmark = pytest.mark.gpu


def run_prefill(w, with_lse=True):
    pb = PrefillBuffers(w)
    d = lserve.prefill_desc(w.T, w.H_q, w.H_kv, w.D, w.block, w.sink_blocks, w.local_blocks)
    ws = lserve.alloc_workspace(lserve.workspace_size(lserve.OP_PREFILL, d))
    lserve.blocksparse_prefill(d, pb.q, pb.k, pb.v, list(w.head_kind), 1.0 / math.sqrt(w.D), pb.out,
                               pb.lse if with_lse else None, workspace=ws)
    torch.cuda.synchronize()
    assert lserve.read_device_status() == lserve.OK
    return oracle.widen_bf16(bf16_bits(pb.out)), pb.lse.cpu().numpy().astype(np.float64)


def check_rows(w, out, lse, rows_of_head, Q=None, K=None, V=None):
    Q = oracle.widen_bf16(w.q()) if Q is None else Q
    K = oracle.widen_bf16(w.k()) if K is None else K
    V = oracle.widen_bf16(w.v()) if V is None else V
    scale = 1.0 / math.sqrt(w.D)
    worst = 0.0
    for hq in range(w.H_q):
        hk = hq // w.G
        rows = np.asarray(rows_of_head(hq))
        o, ls = oracle.prefill_rows(Q[rows, hq], K[:, hk], V[:, hk], int(w.head_kind[hk]), w.block,
                                    w.sink_blocks, w.local_blocks, scale, rows)
        err = np.abs(out[rows, hq] - o)
        worst = max(worst, err.max())
        assert err.max() <= OUT_MAX_ABS, (hq, err.max(), rows[np.unravel_index(err.argmax(), err.shape)[0]])
        assert err.mean() <= OUT_MEAN_ABS, (hq, err.mean())
        assert np.max(np.abs(lse[hq, rows] - ls)) <= LSE_ABS, (hq, np.max(np.abs(lse[hq, rows] - ls)))
    return worst


def test_tiny_prefill_all_rows():
    w = synth.tiny_prefill()
    out, lse = run_prefill(w)
    check_rows(w, out, lse, lambda hq: np.arange(w.T))


SHAPES = [
    # T, H_q, H_kv, D, block, sink, local, head_kind
    (1000, 8, 2, 128, 128, 1, 4, [0, 1]),        # ragged tail, 8 query tiles
    (777, 4, 4, 128, 128, 1, 2, [1, 0, 1, 0]),   # MHA
    (1500, 8, 4, 64, 64, 2, 3, [0, 1, 1, 0]),    # D=64, 64-token mask blocks
    (640, 4, 1, 128, 64, 1, 4, [1]),             # streaming only, block 64
    (129, 2, 1, 128, 128, 1, 4, [0]),            # two query tiles, 1 row in the second
    (64, 4, 2, 64, 64, 1, 4, [0, 1]),            # shorter than one tile
    (640, 12, 2, 64, 64, 1, 4, [0, 1]),          # G=6: three head pairs per KV head
    (300, 16, 2, 128, 128, 1, 4, [1, 0]),        # G=8, ragged second tile
    (450, 6, 3, 64, 128, 2, 2, [0, 1, 0]),       # G=2, D=64, two sink blocks
]


@pytest.mark.parametrize("shape", SHAPES)
def test_prefill_shapes_all_rows(shape):
    T, H_q, H_kv, D, B, S, L, hk = shape
    w = synth.prefill_workload(T, H_q, H_kv, D, B, seed=77 + T, sink_blocks=S, local_blocks=L,
                               head_kind=hk)
    out, lse = run_prefill(w)
    check_rows(w, out, lse, lambda hq: np.arange(T))


def test_prefill_dense_heads_match_causal_attention():
    """All heads retrieval: the kernel is plain causal attention (library check)."""
    T, H, D = 700, 4, 128
    w = synth.prefill_workload(T, H, H, D, 128, seed=5, head_kind=[0] * H)
    out, _ = run_prefill(w, with_lse=False)
    q = torch.from_numpy(oracle.widen_bf16(w.q())).permute(1, 0, 2)
    k = torch.from_numpy(oracle.widen_bf16(w.k())).permute(1, 0, 2)
    v = torch.from_numpy(oracle.widen_bf16(w.v())).permute(1, 0, 2)
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True,
                                                           scale=1 / math.sqrt(D))
    err = np.abs(out - ref.permute(1, 0, 2).numpy())
    assert err.max() <= OUT_MAX_ABS and err.mean() <= OUT_MEAN_ABS


def test_prefill_repeated_calls_are_bitwise_identical():
    w = synth.prefill_workload(1300, 8, 2, 128, 128, seed=9)
    a, la = run_prefill(w)
    b, lb = run_prefill(w)
    assert np.array_equal(a, b) and np.array_equal(la, lb)


def check_blocks(w, out, lse, plan, K=None, V=None):
    """Compare the kernel's rows with the oracle's block-at-a-time form.

    plan: {query head: {query block: row positions inside that block}}.  The
    oracle reads each KV head's keys and values once (contiguous copies) and
    each query block's rows of Q only.  Returns (worst |err|, rows checked)."""
    K = oracle.widen_bf16(w.k()) if K is None else K
    V = oracle.widen_bf16(w.v()) if V is None else V
    scale = 1.0 / math.sqrt(w.D)
    worst, checked, errs_sum = 0.0, 0, 0.0
    for hk in range(w.H_kv):
        heads = [hq for hq in plan if hq // w.G == hk]
        if not heads:
            continue
        kh = np.ascontiguousarray(K[:, hk])
        vh = np.ascontiguousarray(V[:, hk])
        for i in sorted(set(b for hq in heads for b in plan[hq])):
            t0, t1 = i * w.block, min((i + 1) * w.block, w.T)
            q_blk = oracle.widen_bf16(w.q_rows(t0, t1))
            # the rows the group's query heads need from this block, stacked into
            # one call (they see the same key blocks)
            parts = [(hq, np.asarray(sorted(plan[hq][i]), dtype=np.int64))
                     for hq in heads if i in plan[hq]]
            rows = np.concatenate([r for _, r in parts])
            qs = np.concatenate([q_blk[r - t0, hq] for hq, r in parts])
            o_all, ls_all = oracle.prefill_block_rows(qs, kh, vh, int(w.head_kind[hk]), w.block,
                                                      w.sink_blocks, w.local_blocks, scale, rows)
            at = 0
            for hq, r in parts:
                o, ls = o_all[at:at + len(r)], ls_all[at:at + len(r)]
                at += len(r)
                err = np.abs(out[r, hq] - o)
                worst = max(worst, float(err.max()))
                errs_sum += float(err.sum())
                checked += len(r)
                assert err.max() <= OUT_MAX_ABS, (hq, i, err.max())
                assert err.mean() <= OUT_MEAN_ABS, (hq, i, err.mean())
                assert np.max(np.abs(lse[hq, r] - ls)) <= LSE_ABS, (hq, i)
    return worst, checked, errs_sum / max(1, checked * w.D)


def test_prefill_16k_all_rows_multi_round():
    """More (query head, 128-row tile) work units than the GPU has SMs
    (16,384 tokens x 32 query heads = 4,096 units, 2,048 head pairs), so every
    CTA of the persistent grid runs many rounds: all rows of all 16 Lambda
    query heads and of two dense query heads are checked."""
    w = synth.prefill_workload(16384, 32, 8, 128, 128, 1004, name="prefill_16k")
    out, lse = run_prefill(w)
    nb = -(-w.T // w.block)
    full = {i: np.arange(i * w.block, min((i + 1) * w.block, w.T)) for i in range(nb)}
    heads = [0, 13] + [hq for hq in range(w.H_q) if w.head_kind[hq // w.G] == 1]
    worst, checked, mean = check_blocks(w, out, lse, {hq: full for hq in heads})
    assert checked == len(heads) * w.T
    print(f"16K prefill: {checked} rows, worst |err| = {worst:.4g}, mean |err| = {mean:.3g}")


def test_prefill_128k_stratified_rows():
    """The 128K workload, per query head: the first two and the last two
    query blocks in full, 8 seeded-random blocks in full and 256 seeded-random
    rows (drawn per KV head and checked for each of its query heads; all 32
    query heads, dense and Lambda)."""
    w = synth.prefill_128k()
    out, lse = run_prefill(w)
    K, V = oracle.widen_bf16(w.k()), oracle.widen_bf16(w.v())
    nb = -(-w.T // w.block)
    rng = np.random.default_rng(20250214)
    plan = {}
    for hk in range(w.H_kv):
        # 256 random rows per KV head, checked for each of its query heads
        rows = rng.choice(w.T, 256, replace=False)
        for hq in range(hk * w.G, (hk + 1) * w.G):
            blocks = {0, 1, nb - 2, nb - 1}
            blocks |= set(int(x) for x in rng.choice(np.arange(2, nb - 2), 8, replace=False))
            rows_of = {i: set(range(i * w.block, min((i + 1) * w.block, w.T))) for i in blocks}
            for t in rows:
                rows_of.setdefault(int(t) // w.block, set()).add(int(t))
            plan[hq] = rows_of
    worst, checked, mean = check_blocks(w, out, lse, plan, K, V)
    print(f"128K prefill: {checked} rows, worst |err| = {worst:.4g}, mean |err| = {mean:.3g}")
    assert np.all(np.isfinite(out[::997]))


def test_prefill_rejects_bad_arguments():
    w = synth.tiny_prefill()
    pb = PrefillBuffers(w)
    bad = lserve.prefill_desc(w.T, w.H_q, w.H_kv, 96, w.block, 1, 4)
    with pytest.raises(lserve.LServeError) as e:
        lserve.blocksparse_prefill(bad, pb.q, pb.k, pb.v, list(w.head_kind), 0.1, pb.out)
    assert e.value.status == lserve.ERR_UNSUPPORTED
    with pytest.raises(lserve.LServeError):
        lserve.blocksparse_prefill(lserve.prefill_desc(w.T, w.H_q, w.H_kv, w.D, w.block, 1, 4), pb.q,
                                   pb.k, pb.v, [0, 2], 0.1, pb.out)
