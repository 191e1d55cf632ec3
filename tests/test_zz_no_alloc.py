"""The allocation-free page-selection entry point.

Some callers of this library cannot call cudaMalloc (a host callback, a
plug-in whose host process owns every allocation).  lserve_page_select_noalloc
serves them by keeping its scratch scores in a static array inside the
library.  This checks, through the C-ABI, that it selects exactly the pages
lserve_page_select selects (page indices are compared bit for bit, the
tolerance the selection tests use), on two calls in a row.  The file is named
so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import block_sparse_attention_page_b200 as lserve
import synth
from synth.device import DecodeBuffers

pytestmark = pytest.mark.gpu


def _select_both(w, buf, d, layer=0):
    lserve.page_stats(d, buf.k_pool, buf.block_table, buf.ctx_lens, buf.head_kind, buf.stats[layer])
    ws = lserve.alloc_workspace(lserve.workspace_size(lserve.OP_SELECT, d, w.top_k))
    sel_a = torch.full_like(buf.sel[layer], -9)
    cnt_a = torch.full_like(buf.sel_count[layer], -9)
    lserve.page_select(d, buf.q, buf.stats[layer], buf.block_table, buf.ctx_lens, buf.head_kind,
                       w.top_k, sel_a, cnt_a, workspace=ws)
    sel_b = torch.full_like(buf.sel[layer], -9)
    cnt_b = torch.full_like(buf.sel_count[layer], -9)
    st = lserve.lib.lserve_page_select_noalloc(
        ctypes.byref(d), ctypes.c_void_p(buf.q.data_ptr()), ctypes.c_void_p(buf.stats[layer].data_ptr()),
        ctypes.c_void_p(buf.block_table.data_ptr()), ctypes.c_void_p(buf.ctx_lens.data_ptr()),
        ctypes.c_void_p(buf.head_kind.data_ptr()), w.top_k, ctypes.c_void_p(sel_b.data_ptr()),
        ctypes.c_void_p(cnt_b.data_ptr()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == lserve.OK, lserve.status_string(st)
    torch.cuda.synchronize()
    assert lserve.read_device_status() == lserve.OK
    return sel_a.cpu().numpy(), cnt_a.cpu().numpy(), sel_b.cpu().numpy(), cnt_b.cpu().numpy()


def test_noalloc_select_matches_workspace_select_twice():
    for w in [synth.decode_workload(3, 16, 4, 128, 16, 64, 12, 64, 256, [5000, 300, 9000], seed=31),
              synth.tiny_decode()]:
        buf = DecodeBuffers(w)
        d = lserve.paged_desc(w.B, w.H_q, w.H_kv, w.D, w.N_L, w.N_P, w.max_pages, w.num_pool_pages)
        for _ in range(2):  # two calls in a row share the static scratch
            sa, ca, sb, cb = _select_both(w, buf, d)
            assert np.array_equal(sa, sb) and np.array_equal(ca, cb)
            assert (ca >= 0).all()
        # a different query between the calls changes the selection consistently
        buf.q.copy_(-buf.q)


def _noalloc(d, q, stats, bt, ctx, hk, top_k, sel, cnt):
    return lserve.lib.lserve_page_select_noalloc(
        ctypes.byref(d), ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(stats.data_ptr()),
        ctypes.c_void_p(bt.data_ptr()), ctypes.c_void_p(ctx.data_ptr()), ctypes.c_void_p(hk.data_ptr()),
        top_k, ctypes.c_void_p(sel.data_ptr()), ctypes.c_void_p(cnt.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_noalloc_select_allocates_nothing_and_accepts_the_limit():
    """A shape of exactly 1,048,576 scores (the array's size: 16 sequences x 2
    KV heads x a block table 32,768 pages wide) is accepted and selects what
    the workspace path selects; torch's allocator sees no change across the
    call (the call itself allocates no device memory)."""
    w = synth.decode_workload(16, 4, 2, 64, 16, 64, 16, 64, 256,
                              [3000, 64, 5000, 777, 4096, 1, 2500, 6000] * 2, seed=32)
    buf = DecodeBuffers(w)
    wide = 32768
    assert w.B * w.H_kv * wide == 1 << 20
    bt = torch.full((w.B, wide), -1, dtype=torch.int32, device=buf.block_table.device)
    bt[:, :w.max_pages] = buf.block_table
    d = lserve.paged_desc(w.B, w.H_q, w.H_kv, w.D, w.N_L, w.N_P, wide, w.num_pool_pages)
    lserve.page_stats(d, buf.k_pool, bt, buf.ctx_lens, buf.head_kind, buf.stats[0])
    ws = lserve.alloc_workspace(lserve.workspace_size(lserve.OP_SELECT, d, w.top_k))
    sel_a = torch.full_like(buf.sel[0], -9)
    cnt_a = torch.full_like(buf.sel_count[0], -9)
    lserve.page_select(d, buf.q, buf.stats[0], bt, buf.ctx_lens, buf.head_kind, w.top_k, sel_a,
                       cnt_a, workspace=ws)
    sel_b = torch.full_like(sel_a, -9)
    cnt_b = torch.full_like(cnt_a, -9)
    torch.cuda.synchronize()
    before = torch.cuda.memory_allocated()
    for _ in range(2):
        st = _noalloc(d, buf.q, buf.stats[0], bt, buf.ctx_lens, buf.head_kind, w.top_k, sel_b, cnt_b)
        assert st == lserve.OK, lserve.status_string(st)
    torch.cuda.synchronize()
    assert torch.cuda.memory_allocated() == before
    assert lserve.read_device_status() == lserve.OK
    assert torch.equal(sel_a, sel_b) and torch.equal(cnt_a, cnt_b)
    assert int(cnt_b.min()) >= 0


def test_noalloc_select_rejects_too_large_shapes():
    d = lserve.paged_desc(64, 32, 8, 128, 16, 64, 4096, 64 * 4096)   # 2M scores > 1M
    st = lserve.lib.lserve_page_select_noalloc(ctypes.byref(d), None, None, None, None, None, 8, None,
                                               None, None)
    assert st in (lserve.ERR_UNSUPPORTED, lserve.ERR_INVALID_ARG)
    fake = ctypes.c_void_p(1 << 20)
    st = lserve.lib.lserve_page_select_noalloc(ctypes.byref(d), fake, fake, fake, fake, fake, 8, fake,
                                               fake, None)
    assert st == lserve.ERR_UNSUPPORTED
