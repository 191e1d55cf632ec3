"""GPU parity of lserve_decode_append (decode-time cache maintenance): appending
tokens one decode step at a time must leave the paged K/V pools holding the
longer sequences and the page statistics equal, bit for bit, to the oracle's
k_min / k_max of the longer sequences (the full rebuild of every logical page).
The appends cross logical- and physical-page boundaries, hit both head kinds,
and the attention path then runs on the appended cache."""
import numpy as np
import pytest
import torch

import block_sparse_attention_page_b200 as lserve
import oracle
import synth
from synth.device import DecodeBuffers, bf16_bits, bf16_tensor

from parity import check_pair, check_stats, desc_of, run_decode_path

pytestmark = pytest.mark.gpu

STEPS = 40


@pytest.mark.parametrize("D,N_L,N_P,lens0", [
    (128, 16, 64, [61, 127, 1000]),     # crosses 64 / 128 page ends, several logical pages
    (64, 8, 32, [0, 30, 257]),          # an empty sequence grows from nothing
])
def test_append_equals_full_rebuild(D, N_L, N_P, lens0):
    final = [n + STEPS for n in lens0]
    w = synth.decode_workload(len(lens0), 8, 2, D, N_L, N_P, 4, 2 * N_P, 4 * N_P, final,
                              seed=9100 + D, shuffle=True)
    buf = DecodeBuffers(w, pad=synth.BF16_NAN)
    d = desc_of(w)
    K = [[w.k_seq(b, h) for h in range(w.H_kv)] for b in range(w.B)]
    V = [[w.v_seq(b, h) for h in range(w.H_kv)] for b in range(w.B)]
    # the device pools start as the prefix: rows [n0, n0 + STEPS) are erased
    nan = torch.tensor(synth.BF16_NAN, dtype=torch.int16).item()
    for b, n0 in enumerate(lens0):
        for t in range(n0, n0 + STEPS):
            pid = int(w.block_table[b, t // N_P])
            buf.k_pool.view(torch.int16)[pid, :, t % N_P] = nan
            buf.v_pool.view(torch.int16)[pid, :, t % N_P] = nan
    lens = np.array(lens0, dtype=np.int32)
    lens_dev = torch.from_numpy(lens.copy()).cuda()
    lserve.page_stats(d, buf.k_pool, buf.block_table, lens_dev, buf.head_kind, buf.stats[0])
    for step in range(STEPS):
        kn = np.stack([np.stack([K[b][h][lens[b]] for h in range(w.H_kv)]) for b in range(w.B)])
        vn = np.stack([np.stack([V[b][h][lens[b]] for h in range(w.H_kv)]) for b in range(w.B)])
        lserve.decode_append(d, bf16_tensor(kn), bf16_tensor(vn), buf.block_table, lens_dev,
                             buf.head_kind, buf.k_pool, buf.v_pool, buf.stats[0])
        lens += 1
        lens_dev.copy_(torch.from_numpy(lens.copy()))
    torch.cuda.synchronize()
    assert lserve.read_device_status() == lserve.OK
    assert list(lens) == final
    # pools: every row of the longer sequences, bit for bit
    kp, vp = bf16_bits(buf.k_pool), bf16_bits(buf.v_pool)
    for b in range(w.B):
        for h in range(w.H_kv):
            for t in range(final[b]):
                pid = int(w.block_table[b, t // N_P])
                assert np.array_equal(kp[pid, h, t % N_P], K[b][h][t]), (b, h, t)
                assert np.array_equal(vp[pid, h, t % N_P], V[b][h][t]), (b, h, t)
    # statistics of the retrieval heads: the oracle's full rebuild; streaming: untouched
    res = {"stats": bf16_bits(buf.stats[0])}
    for b in range(w.B):
        for h in range(w.H_kv):
            if w.head_kind[h] == 0:
                check_stats(w, res, b, h, oracle.widen_bf16(K[b][h]))
            else:
                for m in range(w.npages(b)):
                    assert np.all(res["stats"][int(w.block_table[b, m]), h] == 0)
    # the attention path on the appended cache
    out = run_decode_path(buf)
    for b in range(w.B):
        for h in range(w.H_kv):
            check_pair(w, out, b, h)


def test_append_out_of_range_position_is_flagged():
    w = synth.decode_workload(2, 4, 2, 128, 16, 64, 4, 64, 256, [100, 200], seed=3)
    buf = DecodeBuffers(w)
    d = desc_of(w)
    before = bf16_bits(buf.k_pool).copy()
    bad = torch.tensor([w.max_pages * w.N_P, -1], dtype=torch.int32, device="cuda")
    z = torch.zeros((w.B, w.H_kv, w.D), dtype=torch.bfloat16, device="cuda")
    lserve.decode_append(d, z, z, buf.block_table, bad, buf.head_kind, buf.k_pool, buf.v_pool,
                         buf.stats[0])
    torch.cuda.synchronize()
    assert lserve.read_device_status() == lserve.ERR_BOUNDS
    assert np.array_equal(bf16_bits(buf.k_pool), before)
