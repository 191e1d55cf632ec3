"""GPU parity of the quantized-KV decode (the 8-bit and the 4-bit cache): the
page quantizer bit for bit against the oracle's quantize_kv8 / quantize_kv4,
and sparse decode attention over the quantized cache against the fp64 oracle
attending the dequantized keys and values (code * scale), on the same seeded
inputs and selections."""
import numpy as np
import pytest
import torch

import block_sparse_attention_page_b200 as lserve
import synth
from synth.device import DecodeBuffers

from parity import check_pair, check_quantized_pages, desc_of, run_decode_path, run_decode_path_kv8

pytestmark = pytest.mark.gpu

CASES = [
    # B, H_q, H_kv, D, N_L, N_P, top_k, sink, local, lens, shuffle
    (3, 8, 2, 128, 16, 64, 4, 64, 256, [1000, 64, 5000], False),
    (2, 4, 4, 64, 8, 32, 5, 32, 100, [777, 4096], True),          # MHA (G=1), N_P=32
    (2, 16, 2, 128, 16, 128, 6, 128, 1024, [129, 20000], False),  # G=8, N_P=128
    (2, 8, 4, 64, 32, 256, 3, 300, 600, [2500, 513], True),       # D=64, N_P=256
    (4, 4, 2, 128, 16, 64, 64, 64, 256, [1, 17, 63, 4095], False),  # all selected, tiny n
    (2, 16, 4, 64, 8, 32, 6, 32, 100, [777, 3001], True),         # G=4, D=64, N_P=32
]


BITS = [8, 4]


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("case", CASES)
def test_kv8_quantizer_and_decode_shapes(case, bits):
    B, H_q, H_kv, D, N_L, N_P, K, S, L, lens, shuffle = case
    w = synth.decode_workload(B, H_q, H_kv, D, N_L, N_P, K, S, L, lens, seed=5151 + D + N_P,
                              shuffle=shuffle)
    res = run_decode_path_kv8(DecodeBuffers(w, pad=synth.BF16_NAN), bits=bits)
    for b in range(w.B):
        for h in range(w.H_kv):
            check_quantized_pages(w, res, b, h)
            check_pair(w, res, b, h, kv8=True)


@pytest.mark.parametrize("bits", BITS)
def test_kv8_tiny_workload(bits):
    w = synth.tiny_decode()
    res = run_decode_path_kv8(DecodeBuffers(w, pad=synth.BF16_NAN), bits=bits)
    for h in range(w.H_kv):
        check_quantized_pages(w, res, 0, h)
        check_pair(w, res, 0, h, kv8=True)
    assert list(res["sel"][0, 0]) == w.planted_pages[(0, 0)]


@pytest.mark.parametrize("bits", BITS)
def test_kv8_llama3_8b_decode_full(bits):
    w = synth.llama3_8b_decode()
    res = run_decode_path_kv8(DecodeBuffers(w), bits=bits)
    errs = []
    for b in range(w.B):
        for h in range(w.H_kv):
            check_pair(w, res, b, h, errs, kv8=True)
    for b, h in [(0, 0), (w.B - 1, w.H_kv - 1)]:
        check_quantized_pages(w, res, b, h)
    print("max |err|, mean |err|, max |o|:", max(e[0] for e in errs), max(e[1] for e in errs),
          max(e[2] for e in errs))


@pytest.mark.parametrize("bits", BITS)
def test_kv8_mixed_batch_and_mha_sampled_pairs(bits):
    for make, seed in ((synth.mixed_batch_decode, 21), (synth.llama2_7b_mha_decode, 22)):
        w = make()
        res = run_decode_path_kv8(DecodeBuffers(w), bits=bits)
        rng = np.random.default_rng(seed)
        pairs = [(int(b), int(h)) for b, h in zip(rng.integers(0, w.B, 8), rng.integers(0, w.H_kv, 8))]
        pairs += [(0, 0), (w.B - 1, w.H_kv - 1)]
        for b, h in pairs:
            check_pair(w, res, b, h, kv8=True, check_stats_bits=False)
        check_quantized_pages(w, res, *pairs[0])
        assert np.all(np.isfinite(res["out"]))


@pytest.mark.parametrize("bits", BITS)
def test_kv8_overlap_flag_is_bitwise_identical_and_close_to_bf16(bits):
    w = synth.decode_workload(2, 32, 8, 128, 16, 64, 16, 128, 512, [20000, 33333], seed=3)
    buf = DecodeBuffers(w)
    r1 = run_decode_path_kv8(buf, bits=bits)
    r2 = run_decode_path_kv8(buf, overlap=True, bits=bits)
    assert np.array_equal(r1["out"], r2["out"]) and np.array_equal(r1["lse"], r2["lse"])
    # per-page scales keep the output near the bf16 cache's (same pages): int8
    # within 0.05, 4-bit codes (a step of amax / 7) within 0.5
    rb = run_decode_path(buf)
    assert np.array_equal(rb["sel"], r1["sel"])
    assert np.max(np.abs(rb["out"] - r1["out"])) < (0.05 if bits == 8 else 0.5)


@pytest.mark.parametrize("bits", BITS)
def test_kv8_empty_sequence_and_bad_pool_id(bits):
    w = synth.decode_workload(2, 8, 2, 128, 16, 64, 4, 64, 256, [0, 3000], seed=8)
    buf = DecodeBuffers(w)
    res = run_decode_path_kv8(buf, bits=bits)
    assert np.all(res["out"][0] == 0) and np.all(np.isneginf(res["lse"][0]))
    for h in range(2):
        check_pair(w, res, 1, h, kv8=True)
    # a block-table entry past the pool: that page is skipped and flagged
    d = desc_of(w)
    bt = buf.block_table.clone()
    bt[1, 3] = w.num_pool_pages + 5
    lserve.quantize_pages_kv8(d, buf.k_pool, buf.v_pool, bt, buf.ctx_lens, res["k8"], res["v8"],
                              res["k_scale"], res["v_scale"], bits=bits)
    assert lserve.read_device_status() == lserve.ERR_BOUNDS
    assert lserve.read_device_status() == lserve.OK
