"""The benchmark's byte and flop accounting (its own page and block counting,
so that the timed legs run nothing of the oracle) agrees with the oracle's
page sets and block iterator on many shapes."""
import numpy as np
import pytest

import bench
import oracle


@pytest.mark.parametrize("NP", [32, 64, 128, 256])
def test_streaming_pages_and_tokens_match_the_oracle(NP):
    rng = np.random.default_rng(NP)
    for _ in range(300):
        n = int(rng.integers(0, 20 * NP))
        sink = int(rng.integers(0, 4 * NP))
        local = int(rng.integers(1, 8 * NP))
        pages = bench.stream_pages(n, NP, sink, local)
        want = [int(m) for m in oracle.streaming_pages(n, NP, sink, local)]
        assert pages == want, (n, sink, local)
        assert bench.valid_tokens(pages, n, NP) == len(oracle.page_tokens(want, n, NP))


@pytest.mark.parametrize("T,block,sink,local", [
    (2048, 64, 1, 4), (131072, 128, 1, 4), (1000, 64, 0, 1), (777, 128, 3, 2), (5000, 64, 2, 9),
])
def test_prefill_flops_match_the_oracle(T, block, sink, local):
    hk = np.array([0, 1, 1, 0], dtype=np.uint8)
    got = bench.prefill_flops(T, 8, 4, 128, block, hk, sink, local)
    want = oracle.prefill_flops(T, 8, 4, 128, block, hk, sink, local)
    assert got == want
