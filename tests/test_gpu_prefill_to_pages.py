"""GPU parity of lserve_prefill_to_pages (a prefilled sequence handed to the
paged decode cache): the pools must hold the prefill's K / V rows at the
block-table positions and the statistics must equal, bit for bit, the
oracle's k_min / k_max of every logical page of the retrieval heads; a decode
step on the filled cache then matches the oracle's decode of the same
sequence."""
import math

import numpy as np
import pytest
import torch

import block_sparse_attention_page_b200 as lserve
import oracle
import synth
from synth.device import bf16_bits, bf16_tensor

from parity import OUT_MAX_ABS, OUT_MEAN_ABS

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T,H_kv,D,N_L,N_P,hk", [
    (1000, 4, 128, 16, 64, [0, 1, 0, 1]),   # ragged last physical and logical page
    (777, 2, 64, 8, 32, [1, 0]),            # D = 64, N_P = 32
    (64, 2, 128, 64, 128, [0, 0]),          # one logical page = N_L = 64, half a physical page
])
def test_prefill_to_pages_equals_the_cache_and_stats(T, H_kv, D, N_L, N_P, hk):
    G = 4
    H_q = G * H_kv
    w = synth.prefill_workload(T, H_q, H_kv, D, 64, seed=8800 + T, head_kind=hk)
    K, V = w.k(), w.v()                           # bf16 bits [T][H_kv][D]
    npages = -(-T // N_P)
    max_pages = npages + 3
    pool_pages = npages + 5
    perm = synth.permutation(synth.tensor_key(8800 + T, 77), pool_pages)[:npages]
    bt = np.full(max_pages, -1, dtype=np.int32)
    bt[:npages] = perm
    d = lserve.paged_desc(1, H_q, H_kv, D, N_L, N_P, max_pages, pool_pages)
    g = N_P // N_L
    nan = synth.BF16_NAN
    k_pool = bf16_tensor(np.full((pool_pages, H_kv, N_P, D), nan, dtype=np.uint16))
    v_pool = bf16_tensor(np.full((pool_pages, H_kv, N_P, D), nan, dtype=np.uint16))
    stats = torch.zeros((pool_pages, H_kv, g, 2, D), dtype=torch.bfloat16, device="cuda")
    bt_dev = torch.from_numpy(bt).cuda()
    hk_dev = torch.tensor(hk, dtype=torch.uint8, device="cuda")
    lserve.prefill_to_pages(d, T, bf16_tensor(K), bf16_tensor(V), bt_dev, hk_dev, k_pool, v_pool, stats)
    torch.cuda.synchronize()
    assert lserve.read_device_status() == lserve.OK
    kp, vp, sp = bf16_bits(k_pool), bf16_bits(v_pool), bf16_bits(stats)
    for h in range(H_kv):
        for t in range(T):
            assert np.array_equal(kp[bt[t // N_P], h, t % N_P], K[t, h]), (h, t)
            assert np.array_equal(vp[bt[t // N_P], h, t % N_P], V[t, h]), (h, t)
        if hk[h] == 0:
            kmin, kmax = oracle.page_stats(oracle.widen_bf16(K[:, h]), N_L)
            want_min, want_max = synth.to_bf16(kmin), synth.to_bf16(kmax)
            for j in range(kmin.shape[0]):
                assert np.array_equal(sp[bt[j // g], h, j % g, 0], want_min[j]), (h, j)
                assert np.array_equal(sp[bt[j // g], h, j % g, 1], want_max[j]), (h, j)
        else:
            assert np.all(sp[:, h] == 0)

    # a decode step on the handed-over cache
    top_k, sink, local = 4, N_P, 2 * N_P
    q = synth.normal_bf16(synth.tensor_key(8800 + T, 78), (1, H_q, D))
    sel = torch.full((1, H_kv, top_k), -7, dtype=torch.int32, device="cuda")
    cnt = torch.full((1, H_kv), -7, dtype=torch.int32, device="cuda")
    lens = torch.tensor([T], dtype=torch.int32, device="cuda")
    bt2 = bt_dev.view(1, -1)
    ws_sel = lserve.alloc_workspace(lserve.workspace_size(lserve.OP_SELECT, d, top_k))
    q_dev = bf16_tensor(q)
    lserve.page_select(d, q_dev, stats, bt2, lens, hk_dev, top_k, sel, cnt, workspace=ws_sel)
    out = torch.empty((1, H_q, D), dtype=torch.bfloat16, device="cuda")
    ws = lserve.alloc_workspace(lserve.workspace_size(lserve.OP_DECODE, d, top_k))
    scale = 1.0 / math.sqrt(D)
    lserve.sparse_decode_attn(d, q_dev, k_pool, v_pool, bt2, lens, hk_dev, sel, cnt, top_k, sink,
                              local, scale, out, None, workspace=ws)
    torch.cuda.synchronize()
    assert lserve.read_device_status() == lserve.OK
    got = oracle.widen_bf16(bf16_bits(out))[0]
    for h in range(H_kv):
        qg = oracle.widen_bf16(q[0, h * G:(h + 1) * G])
        o, _, _ = oracle.decode_pair(qg, oracle.widen_bf16(K[:, h]), oracle.widen_bf16(V[:, h]), T,
                                     hk[h], N_L, N_P, top_k, sink, local, scale)
        err = np.abs(got[h * G:(h + 1) * G] - o)
        assert err.max() <= OUT_MAX_ABS and err.mean() <= OUT_MEAN_ABS, (h, err.max())


def test_prefill_to_pages_rejects_a_sequence_longer_than_the_table():
    d = lserve.paged_desc(1, 8, 2, 128, 16, 64, 2, 4)
    z = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    bt = torch.zeros(2, dtype=torch.int32, device="cuda")
    hk = torch.zeros(2, dtype=torch.uint8, device="cuda")
    with pytest.raises(lserve.LServeError) as e:
        lserve.prefill_to_pages(d, 129, z, z, bt, hk, z, z, z)
    assert e.value.status == lserve.ERR_INVALID_ARG
