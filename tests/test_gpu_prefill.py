"""GPU parity of the block-sparse prefill (tcgen05 kernel) against the fp64
oracle: every row on small shapes (several query/key tiles, ragged tails, both
head kinds, 64- and 128-token mask blocks, D = 64 and 128), and sampled rows on
the 128K-token workload."""
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


def test_prefill_128k_sampled_rows():
    w = synth.prefill_128k()
    out, lse = run_prefill(w)
    Q, K, V = (oracle.widen_bf16(x) for x in (w.q(), w.k(), w.v()))
    rng = np.random.default_rng(4)
    T = w.T
    fixed = np.array([0, 1, 127, 128, 129, 511, 512, 640, T // 2, T - 129, T - 128, T - 2, T - 1])

    def rows(hq):
        extra = rng.integers(0, T, 12)
        return np.unique(np.concatenate([fixed, extra]))
    worst = check_rows(w, out, lse, rows, Q, K, V)
    print("128K prefill: worst sampled |err| =", worst)
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
