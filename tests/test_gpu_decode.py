"""GPU parity of the decode half: page stats -> page select -> sparse decode
attention, through the C-ABI, against the fp64 oracle on the same seeded
inputs.  Shapes span several tiles per pair, ragged last pages, every
supported head dim / GQA ratio / page geometry, and the degenerate cases."""
import numpy as np
import pytest
import torch

import block_sparse_attention_page_b200 as lserve
import synth
from synth.device import DecodeBuffers, bf16_bits

from parity import check_pair, desc_of, run_decode_path

pytestmark = pytest.mark.gpu


def _all_pairs(w, res, errs=None):
    for b in range(w.B):
        for h in range(w.H_kv):
            check_pair(w, res, b, h, errs)


def test_tiny_workload_end_to_end():
    w = synth.tiny_decode()
    buf = DecodeBuffers(w, pad=synth.BF16_NAN)
    res = run_decode_path(buf)
    _all_pairs(w, res)
    # the planted pages are exactly the retrieval head's selection
    assert list(res["sel"][0, 0]) == w.planted_pages[(0, 0)]


CASES = [
    # B, H_q, H_kv, D, N_L, N_P, top_k, sink, local, lens, shuffle
    (3, 8, 2, 128, 16, 64, 4, 64, 256, [1000, 64, 5000], False),
    (2, 4, 4, 64, 8, 32, 5, 32, 100, [777, 4096], True),        # MHA (G=1)
    (2, 16, 2, 128, 16, 128, 6, 128, 1024, [129, 20000], False),  # G=8, g=8
    (2, 8, 4, 64, 32, 256, 3, 300, 600, [2500, 513], True),     # N_P=256
    (1, 8, 2, 128, 64, 128, 2, 64, 64, [9000], False),          # N_L=64
    (4, 4, 2, 128, 16, 64, 64, 64, 256, [1, 17, 63, 4095], False),  # all selected, tiny n
    (2, 8, 4, 128, 16, 64, 8, 4096, 4096, [3000, 8000], False),  # n <= sink + local
    (2, 16, 4, 64, 8, 32, 6, 32, 100, [777, 3001], True),       # G=4, D=64, 32-token tiles
    (2, 16, 2, 64, 16, 64, 5, 64, 200, [1500, 4097], False),    # G=8, D=64
    (2, 8, 2, 128, 16, 32, 7, 32, 64, [2000, 333], True),       # G=4, D=128, 32-token tiles
]


@pytest.mark.parametrize("case", CASES)
def test_decode_path_shapes(case):
    B, H_q, H_kv, D, N_L, N_P, K, S, L, lens, shuffle = case
    w = synth.decode_workload(B, H_q, H_kv, D, N_L, N_P, K, S, L, lens, seed=4242 + D + N_P,
                              shuffle=shuffle)
    buf = DecodeBuffers(w, pad=synth.BF16_NAN)
    res = run_decode_path(buf)
    _all_pairs(w, res)


def test_empty_sequence_gives_zero_output():
    w = synth.decode_workload(2, 8, 2, 128, 16, 64, 4, 64, 256, [0, 3000], seed=7)
    buf = DecodeBuffers(w)
    res = run_decode_path(buf)
    assert np.all(res["out"][0] == 0) and np.all(np.isneginf(res["lse"][0]))
    for h in range(2):
        check_pair(w, res, 1, h)


def test_llama3_8b_decode_full():
    w = synth.llama3_8b_decode()
    res = run_decode_path(DecodeBuffers(w))
    errs = []
    _all_pairs(w, res, errs)
    print("max |err|, mean |err|, max |o|:", max(e[0] for e in errs), max(e[1] for e in errs),
          max(e[2] for e in errs))


def test_long_decode_256k_full():
    w = synth.long_decode_256k()
    res = run_decode_path(DecodeBuffers(w))
    _all_pairs(w, res)
    for h in range(w.H_kv):
        if w.head_kind[h] == 0:  # every planted page is among the 32 selected
            assert set(w.planted_pages[(0, h)]) <= set(int(x) for x in res["sel"][0, h])


def test_mixed_batch_decode_all_pairs():
    """All 256 (sequence, KV head) pairs of the 32-sequence mixed-length batch
    over a shuffled page pool."""
    w = synth.mixed_batch_decode()
    res = run_decode_path(DecodeBuffers(w))
    errs = []
    _all_pairs(w, res, errs)
    assert len(errs) == w.B * w.H_kv
    assert np.all(np.isfinite(res["out"]))
    print("mixed batch: max |err|, mean |err|, max |o|:", max(e[0] for e in errs),
          max(e[1] for e in errs), max(e[2] for e in errs))


def test_llama2_7b_mha_decode_all_pairs():
    """The MHA (G = 1) shape of the pages' second model, all 128 pairs: every
    KV head has one query head; retrieval heads 0-15, streaming 16-31."""
    w = synth.llama2_7b_mha_decode()
    res = run_decode_path(DecodeBuffers(w))
    errs = []
    _all_pairs(w, res, errs)
    assert len(errs) == w.B * w.H_kv
    assert np.all(np.isfinite(res["out"]))


def test_shuffled_pool_equals_identity_layout():
    a = synth.decode_workload(4, 8, 2, 128, 16, 64, 8, 64, 256, [3000, 5000, 64, 9000], seed=99)
    b = synth.decode_workload(4, 8, 2, 128, 16, 64, 8, 64, 256, [3000, 5000, 64, 9000], seed=99,
                              shuffle=True)
    ra = run_decode_path(DecodeBuffers(a))
    rb = run_decode_path(DecodeBuffers(b))
    assert np.array_equal(ra["sel"], rb["sel"])
    assert np.array_equal(ra["out"], rb["out"])


def test_repeated_calls_are_bitwise_identical():
    w = synth.decode_workload(2, 32, 8, 128, 16, 64, 16, 128, 512, [20000, 33333], seed=3)
    buf = DecodeBuffers(w)
    r1 = run_decode_path(buf)
    r2 = run_decode_path(buf)
    assert np.array_equal(r1["out"], r2["out"]) and np.array_equal(r1["sel"], r2["sel"])
    assert np.array_equal(r1["lse"], r2["lse"])


def test_bad_selection_entries_are_skipped_and_flagged():
    w = synth.decode_workload(1, 8, 2, 128, 16, 64, 4, 64, 256, [3000], seed=11)
    buf = DecodeBuffers(w)
    run_decode_path(buf)
    d = desc_of(w)
    sel = buf.sel[0].clone()
    sel[0, 0, 1] = 10 ** 6          # past the sequence's pages
    sel[0, 0, 2] = -3
    ws = lserve.alloc_workspace(lserve.workspace_size(lserve.OP_DECODE, d, w.top_k))
    lserve.sparse_decode_attn(d, buf.q, buf.k_pool, buf.v_pool, buf.block_table, buf.ctx_lens,
                              buf.head_kind, sel, buf.sel_count[0], w.top_k, w.sink, w.local, 0.1,
                              buf.out, buf.lse, workspace=ws)
    assert lserve.read_device_status() == lserve.ERR_BOUNDS
    assert torch.isfinite(buf.out.float()).all()
    assert lserve.read_device_status() == lserve.OK   # the flag was cleared


def test_bounded_wait_times_out_without_fault():
    lserve.debug_wait_timeout(200000)
    assert lserve.read_device_status() == lserve.ERR_TIMEOUT
    # the context is still usable
    x = torch.ones(1024, device="cuda")
    assert float(x.sum()) == 1024.0
    assert lserve.read_device_status() == lserve.OK


def test_workspace_too_small_is_rejected_on_device_shapes():
    w = synth.tiny_decode()
    buf = DecodeBuffers(w)
    d = desc_of(w)
    need = lserve.workspace_size(lserve.OP_DECODE, d, w.top_k)
    assert need > 0
    ws = lserve.alloc_workspace(need - 256)
    with pytest.raises(lserve.LServeError) as e:
        lserve.sparse_decode_attn(d, buf.q, buf.k_pool, buf.v_pool, buf.block_table, buf.ctx_lens,
                                  buf.head_kind, buf.sel[0], buf.sel_count[0], w.top_k, w.sink,
                                  w.local, 0.1, buf.out, buf.lse, workspace=ws[:need - 512])
    assert e.value.status == lserve.ERR_WORKSPACE


def test_overlapped_prologue_across_layers_is_bitwise_identical():
    """Back-to-back decode calls of several layers, launched as programmatic
    dependents with the prologue overlap (plan and lookups before the previous
    layer's kernel ends), give exactly the outputs of plain calls."""
    import math
    w = synth.llama3_8b_decode()
    layers = 3
    buf = DecodeBuffers(w, layers=layers)
    d = desc_of(w)
    ws_sel = lserve.alloc_workspace(lserve.workspace_size(lserve.OP_SELECT, d, w.top_k))
    for l in range(layers):
        lserve.page_stats(d, buf.k_pools[l], buf.block_table, buf.ctx_lens, buf.head_kind, buf.stats[l])
        lserve.page_select(d, buf.q, buf.stats[l], buf.block_table, buf.ctx_lens, buf.head_kind,
                           w.top_k, buf.sel[l], buf.sel_count[l], workspace=ws_sel)
    ws = lserve.alloc_workspace(lserve.workspace_size(lserve.OP_DECODE, d, w.top_k))
    scale = 1.0 / math.sqrt(w.D)

    def run(overlap, prefetch=False):
        outs = [torch.zeros_like(buf.out) for _ in range(layers)]
        lses = [torch.zeros_like(buf.lse) for _ in range(layers)]
        for rep in range(2):
            for l in range(layers):
                lserve.sparse_decode_attn(d, buf.q, buf.k_pools[l], buf.v_pools[l], buf.block_table,
                                          buf.ctx_lens, buf.head_kind, buf.sel[l], buf.sel_count[l],
                                          w.top_k, w.sink, w.local, scale, outs[l], lses[l],
                                          workspace=ws, overlap_prologue=overlap, prefetch_kv=prefetch)
        torch.cuda.synchronize()
        assert lserve.read_device_status() == lserve.OK
        return outs, lses

    plain_o, plain_l = run(False)
    ov_o, ov_l = run(True)
    pf_o, pf_l = run(True, prefetch=True)   # the first tiles' copies before the previous layer ends
    for l in range(layers):
        assert torch.equal(plain_o[l], ov_o[l]) and torch.equal(plain_l[l], ov_l[l])
        assert torch.equal(plain_o[l], pf_o[l]) and torch.equal(plain_l[l], pf_l[l])
