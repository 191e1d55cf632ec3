"""Decode path at the largest shapes the library accepts, against the oracle:
the largest physical page (N_P = 1024, 16 tiles per page) with the smallest
logical page (N_L = 8, 128 logical pages per physical page), the most
(sequence, KV head) pairs one decode call takes (B * H_kv = 2048), and a
600K-token sequence whose 9,375 pages the top-K ranks down to 200."""
import numpy as np
import pytest

import synth
from parity import check_pair, run_decode_path
from synth.device import DecodeBuffers

pytestmark = pytest.mark.gpu


def test_largest_physical_page_smallest_logical_page():
    w = synth.decode_workload(2, 8, 2, 64, 8, 1024, 3, 1024, 2048, [9000, 20000], seed=61)
    res = run_decode_path(DecodeBuffers(w, pad=synth.BF16_NAN))
    for b in range(w.B):
        for h in range(w.H_kv):
            check_pair(w, res, b, h)


def test_most_pairs_in_one_call():
    B, H_kv = 256, 8                         # 2048 (sequence, KV head) pairs
    lens = synth.randint_array(synth.tensor_key(62, 9), B, 1, 700).tolist()
    w = synth.decode_workload(B, 4 * H_kv, H_kv, 64, 16, 64, 4, 64, 256, lens, seed=62)
    res = run_decode_path(DecodeBuffers(w))
    rng = np.random.default_rng(62)
    pairs = [(int(b), int(h)) for b, h in zip(rng.integers(0, B, 48), rng.integers(0, H_kv, 48))]
    pairs += [(0, 0), (B - 1, H_kv - 1), (int(np.argmax(lens)), 0), (int(np.argmin(lens)), 3)]
    for b, h in pairs:
        check_pair(w, res, b, h)
    assert np.all(np.isfinite(res["out"]))


def test_many_pages_large_top_k():
    w = synth.decode_workload(1, 4, 2, 64, 16, 64, 200, 64, 256, [600000], seed=63)
    assert w.max_pages == 9375
    res = run_decode_path(DecodeBuffers(w))
    for h in range(w.H_kv):
        check_pair(w, res, 0, h)
