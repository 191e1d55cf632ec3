"""CPU-side checks of the sequence-sharded decode calls: the host-only shard
arithmetic against the oracle's shard split, and argument validation of the
device calls before they touch the GPU."""
import ctypes

import pytest

import block_sparse_attention_page_b200 as lserve
import oracle

FAKE = ctypes.c_void_p(1 << 20)        # aligned, never dereferenced on failing paths
MISALIGNED = ctypes.c_void_p((1 << 20) + 2)


def _desc(**kw):
    d = dict(B=1, H_q=4, H_kv=2, D=64, N_L=16, N_P=64, max_pages=32, num_pool_pages=32)
    d.update(kw)
    return lserve.paged_desc(d["B"], d["H_q"], d["H_kv"], d["D"], d["N_L"], d["N_P"],
                             d["max_pages"], d["num_pool_pages"])


@pytest.mark.parametrize("n,N_P", [(0, 64), (1, 64), (1000, 64), (4096, 64), (262144, 128), (8191, 32)])
@pytest.mark.parametrize("N", [1, 2, 3, 4, 8])
def test_bounds_follow_the_oracle_split_and_cover_the_sequence(n, N_P, N):
    M = -(-n // N_P)
    want = oracle.shard_bounds(M, N)
    total = 0
    for r in range(N):
        lo, hi, nl = lserve.seqshard_bounds(n, N_P, r, N)
        assert (lo, hi) == (want[r], want[r + 1])
        # the shard's tokens: its pages' share of [0, n)
        assert nl == max(0, min(n, hi * N_P) - lo * N_P)
        if hi < M:
            assert nl == (hi - lo) * N_P                # only the last shard ends mid-page
        total += nl
    assert total == n


def test_bounds_reject_bad_arguments():
    out = [ctypes.c_int32() for _ in range(3)]
    refs = [ctypes.byref(x) for x in out]
    L = lserve.lib
    assert L.lserve_seqshard_bounds(-1, 64, 0, 2, *refs) == lserve.ERR_INVALID_ARG
    assert L.lserve_seqshard_bounds(10, 0, 0, 2, *refs) == lserve.ERR_INVALID_ARG
    assert L.lserve_seqshard_bounds(10, 64, 2, 2, *refs) == lserve.ERR_INVALID_ARG
    assert L.lserve_seqshard_bounds(10, 64, -1, 2, *refs) == lserve.ERR_INVALID_ARG
    assert L.lserve_seqshard_bounds(10, 64, 0, 0, *refs) == lserve.ERR_INVALID_ARG
    assert L.lserve_seqshard_bounds(10, 64, 0, 1, None, refs[1], refs[2]) == lserve.ERR_INVALID_ARG


def test_sel_stride_holds_the_top_k_and_the_streaming_pages():
    d = _desc(N_P=128, max_pages=2048)
    assert lserve.seqshard_sel_stride(d, 32, 128, 1024) == 32          # 1 + 8 + 1 <= 32
    assert lserve.seqshard_sel_stride(d, 4, 128, 1024) == 10           # 1 sink + 9 local pages
    assert lserve.seqshard_sel_stride(d, 4, 0, 0) == 4
    assert lserve.lib.lserve_seqshard_sel_stride(ctypes.byref(d), 0, 0, 0) == 0
    assert lserve.lib.lserve_seqshard_sel_stride(ctypes.byref(d), 4, -1, 0) == 0


def _cand(d, rank=0, N=2, sel_top_k=8, top_k=8, ptr=FAKE, sel=FAKE):
    return lserve.lib.lserve_seqshard_candidates(ctypes.byref(d), rank, N, FAKE, FAKE, sel, FAKE,
                                                 sel_top_k, ptr, top_k, FAKE, FAKE, None)


def _merge(d, rank=0, N=2, top_k=8, stride=8, sel_out=FAKE, sink=64, local=256):
    return lserve.lib.lserve_seqshard_merge(ctypes.byref(d), rank, N, FAKE, FAKE, FAKE, FAKE, top_k,
                                            sink, local, sel_out, FAKE, stride, None)


def test_candidates_validation():
    d = _desc()
    assert _cand(_desc(B=0)) == lserve.ERR_INVALID_ARG
    assert _cand(d, rank=2) == lserve.ERR_INVALID_ARG
    assert _cand(d, rank=-1) == lserve.ERR_INVALID_ARG
    assert _cand(d, N=0) == lserve.ERR_INVALID_ARG
    assert _cand(d, top_k=0) == lserve.ERR_INVALID_ARG
    assert _cand(d, sel_top_k=33) == lserve.ERR_INVALID_ARG    # longer than the block-table row
    assert _cand(d, ptr=None) == lserve.ERR_INVALID_ARG
    assert _cand(d, sel=MISALIGNED) == lserve.ERR_INVALID_ARG


def test_merge_validation():
    d = _desc()
    assert _merge(_desc(N_P=40)) == lserve.ERR_INVALID_ARG
    assert _merge(d, rank=2) == lserve.ERR_INVALID_ARG
    assert _merge(d, top_k=0) == lserve.ERR_INVALID_ARG
    # the row must hold top_k and the streaming pages: 1 sink + 4 local + 1 page
    assert _merge(d, top_k=4, stride=5) == lserve.ERR_INVALID_ARG
    assert _merge(d, top_k=8, stride=7) == lserve.ERR_INVALID_ARG
    assert _merge(d, sel_out=None) == lserve.ERR_INVALID_ARG
    assert _merge(d, sel_out=MISALIGNED) == lserve.ERR_INVALID_ARG
    # N * top_k proposals must fit in shared memory
    assert _merge(d, N=64, top_k=1024, stride=1024) == lserve.ERR_UNSUPPORTED


def test_combine_validation():
    L = lserve.lib
    assert L.lserve_seqshard_combine(0, 4, 128, FAKE, FAKE, FAKE, None, None) == lserve.ERR_INVALID_ARG
    assert L.lserve_seqshard_combine(2, 0, 128, FAKE, FAKE, FAKE, None, None) == lserve.ERR_INVALID_ARG
    assert L.lserve_seqshard_combine(2, 4, 96, FAKE, FAKE, FAKE, None, None) == lserve.ERR_INVALID_ARG
    assert L.lserve_seqshard_combine(2, 4, 128, None, FAKE, FAKE, None, None) == lserve.ERR_INVALID_ARG
    assert L.lserve_seqshard_combine(2, 4, 128, FAKE, FAKE, None, None, None) == lserve.ERR_INVALID_ARG
    assert L.lserve_seqshard_combine(2, 4, 128, FAKE, FAKE, FAKE, MISALIGNED, None) == lserve.ERR_INVALID_ARG


def test_decode_accepts_the_float_output_flag():
    d = _desc()
    st = lserve.lib.lserve_sparse_decode_attn_ex(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                                 FAKE, FAKE, 8, 64, 256, 0.125, FAKE, None,
                                                 lserve.DECODE_OUT_F32 | lserve.DECODE_OVERLAP_PROLOGUE,
                                                 None, 0, None)
    assert st in (lserve.ERR_WORKSPACE, lserve.ERR_CUDA)   # past the flag check
