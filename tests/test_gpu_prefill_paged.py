"""GPU parity of lserve_blocksparse_prefill_paged: the block-sparse prefill
whose kernel also hands the sequence to the paged decode cache (K / V through
the block table into the pools, the retrieval heads' page statistics).

- Its attention output and log-sum-exp equal lserve_blocksparse_prefill's bit
  for bit (the same kernel schedule; the page writer only reads the inputs).
- Every valid row of the pools holds the sequence's K / V at its block-table
  position; rows past the sequence and pages the table does not name keep
  their sentinel.
- The retrieval heads' statistics equal, bit for bit, the oracle's k_min /
  k_max of every logical page; the streaming heads' statistics stay untouched.
- The result equals what the separate pass lserve_prefill_to_pages writes.
Shapes cover the paired kernel (G even) and the one-head kernel (G = 1),
D = 64 and 128, physical pages of 32 to 256 tokens (N_P = 192: pages split
across 128-token key tiles), logical pages of 8 to 64 tokens and ragged
sequence ends."""
import math

import numpy as np
import pytest
import torch

import block_sparse_attention_page_b200 as lserve
import oracle
import synth
from synth.device import PrefillBuffers, bf16_bits, bf16_tensor

pytestmark = pytest.mark.gpu

CASES = [
    # T, H_q, H_kv, D, block, N_L, N_P, head_kind
    (1000, 8, 2, 128, 64, 16, 64, [0, 1]),          # G = 4 (paired kernel), ragged end
    (777, 2, 2, 64, 64, 8, 32, [0, 1]),              # G = 1 (one-head kernel), D = 64, N_P = 32
    (1280, 4, 4, 128, 128, 32, 128, [1, 0, 0, 1]),   # G = 1, N_P = 128, T a multiple of 128
    (700, 4, 2, 128, 128, 16, 192, [0, 1]),          # N_P = 192: pages across key tiles
    (2100, 8, 2, 64, 64, 64, 256, [0, 0]),           # N_P = 256, N_L = 64, D = 64
    (130, 2, 2, 128, 64, 16, 64, [1, 0]),            # G = 1, two key tiles, 2-token tail
    (900, 16, 2, 128, 128, 16, 64, [0, 1]),          # G = 8: four query-head pairs per KV head
]


def _run(T, H_q, H_kv, D, block, N_L, N_P, hk, seed):
    w = synth.prefill_workload(T, H_q, H_kv, D, block, seed, head_kind=hk)
    pb = PrefillBuffers(w)
    d = lserve.prefill_desc(w.T, w.H_q, w.H_kv, w.D, w.block, w.sink_blocks, w.local_blocks)
    ws = lserve.alloc_workspace(lserve.workspace_size(lserve.OP_PREFILL, d))
    scale = 1.0 / math.sqrt(D)
    npages = -(-T // N_P)
    max_pages, pool_pages = npages + 3, npages + 5
    perm = synth.permutation(synth.tensor_key(seed, 91), pool_pages)[:npages]
    bt = np.full(max_pages, -1, dtype=np.int32)
    bt[:npages] = perm
    pd = lserve.paged_desc(1, H_q, H_kv, D, N_L, N_P, max_pages, pool_pages)
    g = N_P // N_L
    nan = synth.BF16_NAN

    def pools():
        return (bf16_tensor(np.full((pool_pages, H_kv, N_P, D), nan, dtype=np.uint16)),
                bf16_tensor(np.full((pool_pages, H_kv, N_P, D), nan, dtype=np.uint16)),
                bf16_tensor(np.full((pool_pages, H_kv, g, 2, D), nan, dtype=np.uint16)))

    bt_dev = torch.from_numpy(bt).cuda()
    # the plain prefill and the separate hand-over pass
    lserve.blocksparse_prefill(d, pb.q, pb.k, pb.v, list(hk), scale, pb.out, pb.lse, workspace=ws)
    out_ref, lse_ref = bf16_bits(pb.out), pb.lse.cpu().numpy().copy()
    k2, v2, s2 = pools()
    lserve.prefill_to_pages(pd, T, pb.k, pb.v, bt_dev, torch.tensor(hk, dtype=torch.uint8, device="cuda"),
                            k2, v2, s2)
    # the fused call
    pb.out.zero_()
    pb.lse.zero_()
    k1, v1, s1 = pools()
    lserve.blocksparse_prefill_paged(d, pd, pb.q, pb.k, pb.v, list(hk), scale, pb.out, bt_dev, k1, v1,
                                     s1, lse=pb.lse, workspace=ws)
    torch.cuda.synchronize()
    assert lserve.read_device_status() == lserve.OK
    return (w, bt, g, out_ref, lse_ref, bf16_bits(pb.out), pb.lse.cpu().numpy(),
            [bf16_bits(x) for x in (k1, v1, s1)], [bf16_bits(x) for x in (k2, v2, s2)])


@pytest.mark.parametrize("case", CASES)
def test_prefill_paged_output_cache_and_stats(case):
    T, H_q, H_kv, D, block, N_L, N_P, hk = case
    w, bt, g, out_ref, lse_ref, out, lse, fused, sep = _run(*case, seed=9300 + T)
    # attention unchanged, bit for bit
    assert np.array_equal(out, out_ref)
    assert np.array_equal(lse, lse_ref)
    kp, vp, sp = fused
    K, V = w.k(), w.v()
    nan = synth.BF16_NAN
    npages = -(-T // N_P)
    for h in range(H_kv):
        for t in range(T):
            assert np.array_equal(kp[bt[t // N_P], h, t % N_P], K[t, h]), (h, t)
            assert np.array_equal(vp[bt[t // N_P], h, t % N_P], V[t, h]), (h, t)
        # rows past the sequence in its last page: untouched
        last = bt[npages - 1]
        for r in range(T - (npages - 1) * N_P, N_P):
            assert np.all(kp[last, h, r] == nan) and np.all(vp[last, h, r] == nan), (h, r)
        if hk[h] == 0:
            kmin, kmax = oracle.page_stats(oracle.widen_bf16(K[:, h]), N_L)
            want_min, want_max = synth.to_bf16(kmin), synth.to_bf16(kmax)
            for j in range(kmin.shape[0]):
                assert np.array_equal(sp[bt[j // g], h, j % g, 0], want_min[j]), (h, j)
                assert np.array_equal(sp[bt[j // g], h, j % g, 1], want_max[j]), (h, j)
        else:
            assert np.all(sp[:, h] == nan)
    # pool pages the table does not name: untouched
    unused = np.setdiff1d(np.arange(kp.shape[0]), bt[:npages])
    assert np.all(kp[unused] == nan) and np.all(vp[unused] == nan) and np.all(sp[unused] == nan)
    # the same cache as the separate pass
    for a, b in zip(fused, sep):
        assert np.array_equal(a, b)


def test_prefill_paged_bad_pool_id_is_skipped_and_flagged():
    T, H_q, H_kv, D, block, N_L, N_P = 500, 4, 2, 64, 64, 16, 64
    w = synth.prefill_workload(T, H_q, H_kv, D, block, 9400, head_kind=[0, 1])
    pb = PrefillBuffers(w)
    d = lserve.prefill_desc(T, H_q, H_kv, D, block, w.sink_blocks, w.local_blocks)
    npages = -(-T // N_P)
    pool_pages = npages + 2
    bt = torch.arange(npages, dtype=torch.int32, device="cuda")
    bt[2] = pool_pages + 7  # past the pool
    pd = lserve.paged_desc(1, H_q, H_kv, D, N_L, N_P, npages, pool_pages)
    kp = torch.zeros((pool_pages, H_kv, N_P, D), dtype=torch.bfloat16, device="cuda")
    vp = torch.zeros_like(kp)
    sp = torch.zeros((pool_pages, H_kv, N_P // N_L, 2, D), dtype=torch.bfloat16, device="cuda")
    lserve.blocksparse_prefill_paged(d, pd, pb.q, pb.k, pb.v, [0, 1], 1.0 / math.sqrt(D), pb.out, bt,
                                     kp, vp, sp)
    assert lserve.read_device_status() == lserve.ERR_BOUNDS
    assert lserve.read_device_status() == lserve.OK
    K = w.k()
    got = bf16_bits(kp)
    for t in range(T):
        if t // N_P != 2:
            assert np.array_equal(got[t // N_P, 0, t % N_P], K[t, 0])
