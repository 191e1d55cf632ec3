"""Decode-path cases whose answer is fixed exactly: an all-zero q (every score
is 0, so the top-K is the lowest page indices and attention is the plain mean
of V over the attended tokens), pages duplicated so that their scores tie bit
for bit (the lowest indices win, R4), and one call split differently over the
CTAs (the output does not depend on the split beyond rounding)."""
import math

import numpy as np
import pytest
import torch

import block_sparse_attention_page_b200 as lserve
import oracle
import synth
from parity import OUT_MAX_ABS, OUT_MEAN_ABS, check_outputs, desc_of, run_decode_path
from synth.device import DecodeBuffers, bf16_bits

pytestmark = pytest.mark.gpu


def _seq_from_pool(pool_bits, w, b, h):
    """Dense [n][D] bf16 bits of one (sequence, KV head) read back through the block table."""
    n = int(w.ctx_lens[b])
    rows = [pool_bits[w.block_table[b, m], h] for m in range(w.npages(b))]
    return np.concatenate(rows)[:n]


def test_zero_query_selects_the_first_pages_and_averages_v():
    w = synth.decode_workload(3, 8, 2, 128, 16, 64, 6, 64, 256, [1000, 64, 5000], seed=71)
    buf = DecodeBuffers(w)
    buf.q.zero_()
    res = run_decode_path(buf)
    G = w.G
    for b in range(w.B):
        n = int(w.ctx_lens[b])
        for h in range(w.H_kv):
            if w.head_kind[h] == 0:
                cnt = int(res["sel_count"][b, h])
                assert cnt == min(w.top_k, w.npages(b))
                assert [int(x) for x in res["sel"][b, h, :cnt]] == list(range(cnt))  # all tied at 0
                pages = list(range(cnt))
            else:
                pages = oracle.streaming_pages(n, w.N_P, w.sink, w.local)
            toks = oracle.page_tokens(pages, n, w.N_P)
            want = oracle.widen_bf16(w.v_seq(b, h))[toks].mean(axis=0)  # uniform weights
            err = np.abs(res["out"][b, h * G:(h + 1) * G] - want[None, :])
            assert err.max() <= OUT_MAX_ABS and err.mean() <= OUT_MEAN_ABS, (b, h, err.max())
            # every logit is 0: lse = log(number of tokens)
            assert np.allclose(res["lse"][b, h * G:(h + 1) * G], math.log(len(toks)), atol=1e-4)


def test_duplicated_pages_tie_to_the_lowest_indices():
    w = synth.decode_workload(1, 8, 2, 128, 16, 64, 6, 64, 256, [4000], seed=72)
    buf = DecodeBuffers(w)
    b, h, G = 0, 0, w.G                      # KV head 0 is a retrieval head
    assert w.head_kind[h] == 0
    n, M = int(w.ctx_lens[b]), w.npages(b)
    q = oracle.widen_bf16(w.q[b, h * G:(h + 1) * G])
    _, P, _ = oracle.retrieval_pages(q, oracle.widen_bf16(w.k_seq(b, h)), n, w.N_L, w.N_P, w.top_k)
    src = int(np.argmax(P[:M - 1]))          # the best full page
    dst = [m for m in (1, 5, 9, 17, 25, 33, 41, 49, 57, 61) if m != src]
    for m in dst:                            # its keys copied into ten other full pages
        buf.k_pool[int(w.block_table[b, m]), h].copy_(buf.k_pool[int(w.block_table[b, src]), h])
    torch.cuda.synchronize()
    res = run_decode_path(buf)
    k = oracle.widen_bf16(_seq_from_pool(bf16_bits(buf.k_pool), w, b, h))
    want, P2, _ = oracle.retrieval_pages(q, k, n, w.N_L, w.N_P, w.top_k)
    assert len({P2[m] for m in [src] + dst}) == 1          # the copies tie exactly
    cnt = int(res["sel_count"][b, h])
    assert [int(x) for x in res["sel"][b, h, :cnt]] == want  # lowest indices among the tied
    # the device's scores of the tied pages are bit-identical too
    sc = res["scores"][b, h]
    assert len({float(sc[m]) for m in [src] + dst}) == 1
    v = oracle.widen_bf16(w.v_seq(b, h))
    check_outputs(w, res, b, h, q, k, v, want)


def test_output_does_not_depend_on_the_split():
    """The same selection attended with a 4x wider selection row: the host
    sizes the grid from the row length (64 CTAs for rows of 16 pages, one per
    SM for rows of 64), so the pairs are split over the CTAs differently."""
    w = synth.decode_workload(1, 32, 8, 128, 16, 128, 16, 128, 1024, [131072], seed=73)
    buf = DecodeBuffers(w)
    res = run_decode_path(buf)
    d = desc_of(w)
    K2 = 4 * w.top_k
    sel2 = torch.full((w.B, w.H_kv, K2), -1, dtype=torch.int32, device="cuda")
    sel2[:, :, :w.top_k] = buf.sel[0]
    out2 = torch.empty_like(buf.out)
    lse2 = torch.empty_like(buf.lse)
    ws = lserve.alloc_workspace(lserve.workspace_size(lserve.OP_DECODE, d, K2))
    lserve.sparse_decode_attn(d, buf.q, buf.k_pool, buf.v_pool, buf.block_table, buf.ctx_lens,
                              buf.head_kind, sel2, buf.sel_count[0], K2, w.sink, w.local,
                              res["scale"], out2, lse2, workspace=ws)
    torch.cuda.synchronize()
    assert lserve.read_device_status() == lserve.OK
    a = res["out"]
    bb = oracle.widen_bf16(bf16_bits(out2))
    # The fp32 sums are merged in another order: apart by at most one bf16 unit
    # in the last place of the larger value, plus the fp32 rounding of the sums'
    # terms (|p v| up to ~0.1 here, p carried as bf16 hi + lo: ~2^-16 of a term)
    # for outputs that cancel to near zero.
    mag = np.maximum(np.maximum(np.abs(a), np.abs(bb)), 1e-30)
    ulp = 2.0 ** (np.floor(np.log2(mag)) - 7)
    d = np.abs(a - bb)
    assert np.all(d <= ulp + 2e-5), (d.max(), (d / ulp).max(), int((d > ulp).sum()))
    l2 = lse2.cpu().numpy().astype(np.float64)
    assert np.allclose(l2, res["lse"], rtol=1e-5, atol=1e-5)
    # and the second split meets the oracle on every pair
    res2 = dict(res, out=bb, lse=l2)
    G = w.G
    for h in range(w.H_kv):
        n = int(w.ctx_lens[0])
        q = oracle.widen_bf16(w.q[0, h * G:(h + 1) * G])
        k = oracle.widen_bf16(w.k_seq(0, h))
        v = oracle.widen_bf16(w.v_seq(0, h))
        pages = ([int(x) for x in res["sel"][0, h, :int(res["sel_count"][0, h])]] if w.head_kind[h] == 0
                 else oracle.streaming_pages(n, w.N_P, w.sink, w.local))
        check_outputs(w, res2, 0, h, q, k, v, pages)


def _decode(w, buf, d, ws, out, lse, scale):
    lserve.sparse_decode_attn(d, buf.q, buf.k_pool, buf.v_pool, buf.block_table, buf.ctx_lens,
                              buf.head_kind, buf.sel[0], buf.sel_count[0], w.top_k, w.sink, w.local,
                              scale, out, lse, workspace=ws)
    torch.cuda.synchronize()
    assert lserve.read_device_status() == lserve.OK


def test_workspace_leftovers_are_never_merged():
    """The decode workspace heals itself: split partials are tagged with their
    pair and a per-pair merge epoch, so words that an earlier call left behind
    (here: every partial word of the previous call kept with its tag, its value
    replaced by NaN, as a call that stopped before merging would leave them)
    are ignored, and a workspace last used by a call of another shape needs no
    re-zeroing.  Each later call gives bit for bit the first call's output."""
    w = synth.llama3_8b_decode()
    buf = DecodeBuffers(w)
    res = run_decode_path(buf)
    d = desc_of(w)
    w2 = synth.decode_workload(3, 16, 2, 128, 16, 64, 16, 64, 256, [20000, 3000, 40000], seed=74)
    d2 = desc_of(w2)
    nbytes = max(lserve.workspace_size(lserve.OP_DECODE, d, w.top_k),
                 lserve.workspace_size(lserve.OP_DECODE, d2, w2.top_k))
    ws = lserve.alloc_workspace(nbytes)
    out = torch.empty_like(buf.out)
    lse = torch.empty_like(buf.lse)
    _decode(w, buf, d, ws, out, lse, res["scale"])
    ref_o, ref_l = out.clone(), lse.clone()
    assert torch.equal(ref_o, buf.out)                       # same split as run_decode_path's call
    P = w.B * w.H_kv
    head = (P * 4 + 255) // 256 * 256                        # the epochs, then the partial words
    assert int(ws[:P * 4].view(torch.int32).max()) >= 1      # the call did merge split pairs
    words = ws[head:].view(torch.int64)
    nan_low = torch.tensor(0x7FC00000, dtype=torch.int64, device=ws.device)
    for _ in range(2):
        # keep every word's tag (high half), poison its value (low half)
        words.copy_((words & ~0xFFFFFFFF) | nan_low)
        out.fill_(0)
        _decode(w, buf, d, ws, out, lse, res["scale"])
        assert torch.equal(out, ref_o) and torch.equal(lse, ref_l)
    # the same workspace after a call of another shape (G = 8, two KV heads)
    buf2 = DecodeBuffers(w2)
    run_decode_path(buf2)
    lserve.sparse_decode_attn(d2, buf2.q, buf2.k_pool, buf2.v_pool, buf2.block_table,
                              buf2.ctx_lens, buf2.head_kind, buf2.sel[0], buf2.sel_count[0],
                              w2.top_k, w2.sink, w2.local, res["scale"], buf2.out, buf2.lse,
                              workspace=ws)
    out.fill_(0)
    _decode(w, buf, d, ws, out, lse, res["scale"])
    assert torch.equal(out, ref_o) and torch.equal(lse, ref_l)
