"""GPU parity of lserve_decode_step: the decode-time append fused into the
attention launch.  Each step appends every sequence's new token (pools and
page statistics) and attends over the longer sequence, the new token read
from k_new / v_new; page selection runs on every 4th step (the reuse interval)
and is reused in between.  Every step's outputs are checked against the fp64
oracle on the same pages -- by default a retrieval head sees only its
selected pages, with recent_from it also sees every token appended since its
selection -- and at the end the pools and statistics must equal the longer
sequences' (the oracle's full rebuild), bit for bit."""
import math

import numpy as np
import pytest
import torch

import block_sparse_attention_page_b200 as lserve
import oracle
import synth
from synth.device import DecodeBuffers, bf16_bits, bf16_tensor

from parity import LSE_ABS, OUT_MAX_ABS, OUT_MEAN_ABS, check_stats, desc_of

pytestmark = pytest.mark.gpu

REUSE = 4


def _run_steps(w, lens0, steps, recent):
    buf = DecodeBuffers(w, pad=synth.BF16_NAN)
    d = desc_of(w)
    K = [[w.k_seq(b, h) for h in range(w.H_kv)] for b in range(w.B)]
    V = [[w.v_seq(b, h) for h in range(w.H_kv)] for b in range(w.B)]
    nan = torch.tensor(synth.BF16_NAN, dtype=torch.int16).item()
    for b, n0 in enumerate(lens0):          # the device pools start as the prefix
        for t in range(n0, n0 + steps):
            pid = int(w.block_table[b, t // w.N_P])
            buf.k_pool.view(torch.int16)[pid, :, t % w.N_P] = nan
            buf.v_pool.view(torch.int16)[pid, :, t % w.N_P] = nan
    lens = np.array(lens0, dtype=np.int32)
    lens_dev = torch.from_numpy(lens.copy()).cuda()
    lserve.page_stats(d, buf.k_pool, buf.block_table, lens_dev, buf.head_kind, buf.stats[0])
    ws = lserve.alloc_workspace(lserve.workspace_size(lserve.OP_DECODE, d, w.top_k))
    scale = 1.0 / math.sqrt(w.D)
    G = w.G
    since = lens.copy()
    since_dev = torch.from_numpy(since.copy()).cuda()
    worst = 0.0
    for step in range(steps):
        if step % REUSE == 0:               # select on the cache as it is before this step's token
            lserve.page_select(d, buf.q, buf.stats[0], buf.block_table, lens_dev, buf.head_kind,
                               w.top_k, buf.sel[0], buf.sel_count[0], phys_scores=buf.scores)
            since = lens.copy()
            since_dev.copy_(torch.from_numpy(since.copy()))
        kn = np.stack([np.stack([K[b][h][lens[b]] for h in range(w.H_kv)]) for b in range(w.B)])
        vn = np.stack([np.stack([V[b][h][lens[b]] for h in range(w.H_kv)]) for b in range(w.B)])
        lens += 1
        lens_dev.copy_(torch.from_numpy(lens.copy()))
        lserve.decode_step(d, buf.q, bf16_tensor(kn), bf16_tensor(vn), buf.k_pool, buf.v_pool,
                           buf.stats[0], buf.block_table, lens_dev, buf.head_kind, buf.sel[0],
                           buf.sel_count[0], w.top_k, w.sink, w.local, scale, buf.out, buf.lse,
                           recent_from=since_dev if recent else None, workspace=ws)
        torch.cuda.synchronize()
        assert lserve.read_device_status() == lserve.OK
        out = oracle.widen_bf16(bf16_bits(buf.out))
        lse = buf.lse.cpu().numpy().astype(np.float64)
        sel = buf.sel[0].cpu().numpy()
        cnt = buf.sel_count[0].cpu().numpy()
        for b in range(w.B):
            n = int(lens[b])
            for h in range(w.H_kv):
                q = oracle.widen_bf16(w.q[b, h * G:(h + 1) * G])
                if w.head_kind[h] == 0:
                    pages = [int(x) for x in sel[b, h, :int(cnt[b, h])]]
                    assert pages == sorted(set(pages)) and all(0 <= m < -(-n // w.N_P) for m in pages)
                    toks = oracle.attended_tokens(pages, n, w.N_P,
                                                  int(since[b]) if recent else None)
                else:
                    toks = oracle.page_tokens(oracle.streaming_pages(n, w.N_P, w.sink, w.local),
                                              n, w.N_P)
                o, ls = oracle.decode_attention(q, oracle.widen_bf16(K[b][h][:n]),
                                                oracle.widen_bf16(V[b][h][:n]), toks, scale)
                got = out[b, h * G:(h + 1) * G]
                err = np.abs(got - o)
                worst = max(worst, float(err.max()))
                assert err.max() <= OUT_MAX_ABS and err.mean() <= OUT_MEAN_ABS, (step, b, h, err.max())
                gl = lse[b, h * G:(h + 1) * G]
                if np.all(np.isneginf(ls)):
                    assert np.all(np.isneginf(gl))
                else:
                    assert np.max(np.abs(gl - ls)) <= LSE_ABS, (step, b, h)
    # pools and statistics: those of the longer sequences
    kp, vp = bf16_bits(buf.k_pool), bf16_bits(buf.v_pool)
    final = [n + steps for n in lens0]
    for b in range(w.B):
        for h in range(w.H_kv):
            for t in range(final[b]):
                pid = int(w.block_table[b, t // w.N_P])
                assert np.array_equal(kp[pid, h, t % w.N_P], K[b][h][t]), (b, h, t)
                assert np.array_equal(vp[pid, h, t % w.N_P], V[b][h][t]), (b, h, t)
    res = {"stats": bf16_bits(buf.stats[0])}
    for b in range(w.B):
        for h in range(w.H_kv):
            if w.head_kind[h] == 0:
                check_stats(w, res, b, h, oracle.widen_bf16(K[b][h]))
    return worst


STEPS = 10


@pytest.mark.parametrize("recent", [False, True])
@pytest.mark.parametrize("H_q,H_kv,D,N_L,N_P,top_k,lens0", [
    (8, 2, 128, 16, 64, 4, [61, 127, 1000]),        # G=4 (tensor-core consumer), page ends crossed
    (4, 4, 64, 8, 32, 3, [1, 30, 257]),             # MHA (CUDA-core consumer), tiny sequences
    (16, 2, 128, 16, 128, 5, [120, 3000]),          # G=8, two 64-token tiles per page
])
def test_decode_step_matches_oracle(H_q, H_kv, D, N_L, N_P, top_k, lens0, recent):
    final = [n + STEPS for n in lens0]
    w = synth.decode_workload(len(lens0), H_q, H_kv, D, N_L, N_P, top_k, 2 * N_P, 4 * N_P, final,
                              seed=9300 + D + N_P, shuffle=True)
    worst = _run_steps(w, lens0, STEPS, recent)
    print(f"decode_step recent={recent}: worst |err| = {worst:.4g}")


def test_decode_step_without_append_equals_sparse_decode_attn():
    """k_new = v_new = NULL: lserve_decode_step is lserve_sparse_decode_attn_ex
    (same pages, same split, bit for bit)."""
    w = synth.llama3_8b_decode()
    buf = DecodeBuffers(w)
    d = desc_of(w)
    lserve.page_stats(d, buf.k_pool, buf.block_table, buf.ctx_lens, buf.head_kind, buf.stats[0])
    lserve.page_select(d, buf.q, buf.stats[0], buf.block_table, buf.ctx_lens, buf.head_kind,
                       w.top_k, buf.sel[0], buf.sel_count[0], phys_scores=buf.scores)
    ws = lserve.alloc_workspace(lserve.workspace_size(lserve.OP_DECODE, d, w.top_k))
    scale = 1.0 / math.sqrt(w.D)
    lserve.sparse_decode_attn(d, buf.q, buf.k_pool, buf.v_pool, buf.block_table, buf.ctx_lens,
                              buf.head_kind, buf.sel[0], buf.sel_count[0], w.top_k, w.sink, w.local,
                              scale, buf.out, buf.lse, workspace=ws)
    o2 = torch.empty_like(buf.out)
    l2 = torch.empty_like(buf.lse)
    lserve.decode_step(d, buf.q, None, None, buf.k_pool, buf.v_pool, None, buf.block_table,
                       buf.ctx_lens, buf.head_kind, buf.sel[0], buf.sel_count[0], w.top_k, w.sink,
                       w.local, scale, o2, l2, workspace=ws)
    torch.cuda.synchronize()
    assert lserve.read_device_status() == lserve.OK
    assert torch.equal(buf.out, o2) and torch.equal(buf.lse, l2)


def test_decode_step_every_token_recent_is_dense_attention():
    """recent_from = 0: every retrieval head attends all n tokens (one step,
    appending), which the oracle computes as dense attention; long windows
    cost the plan no more than the selection's length."""
    w = synth.decode_workload(2, 8, 2, 128, 16, 64, 4, 64, 256, [3001, 9000], seed=9400)
    buf = DecodeBuffers(w)
    d = desc_of(w)
    lens0 = np.array(w.ctx_lens, dtype=np.int32) - 1        # the last token is the appended one
    lserve.page_stats(d, buf.k_pool, buf.block_table, torch.from_numpy(lens0).cuda(), buf.head_kind,
                      buf.stats[0])
    lserve.page_select(d, buf.q, buf.stats[0], buf.block_table, torch.from_numpy(lens0).cuda(),
                       buf.head_kind, w.top_k, buf.sel[0], buf.sel_count[0], phys_scores=buf.scores)
    K = [[w.k_seq(b, h) for h in range(w.H_kv)] for b in range(w.B)]
    V = [[w.v_seq(b, h) for h in range(w.H_kv)] for b in range(w.B)]
    kn = np.stack([np.stack([K[b][h][lens0[b]] for h in range(w.H_kv)]) for b in range(w.B)])
    vn = np.stack([np.stack([V[b][h][lens0[b]] for h in range(w.H_kv)]) for b in range(w.B)])
    zero = torch.zeros(w.B, dtype=torch.int32, device="cuda")
    ws = lserve.alloc_workspace(lserve.workspace_size(lserve.OP_DECODE, d, w.top_k))
    scale = 1.0 / math.sqrt(w.D)
    lserve.decode_step(d, buf.q, bf16_tensor(kn), bf16_tensor(vn), buf.k_pool, buf.v_pool,
                       buf.stats[0], buf.block_table, buf.ctx_lens, buf.head_kind, buf.sel[0],
                       buf.sel_count[0], w.top_k, w.sink, w.local, scale, buf.out, buf.lse,
                       recent_from=zero, workspace=ws)
    torch.cuda.synchronize()
    assert lserve.read_device_status() == lserve.OK
    out = oracle.widen_bf16(bf16_bits(buf.out))
    G = w.G
    for b in range(w.B):
        n = int(w.ctx_lens[b])
        for h in range(w.H_kv):
            q = oracle.widen_bf16(w.q[b, h * G:(h + 1) * G])
            if w.head_kind[h] == 0:
                toks = np.arange(n)
            else:
                toks = oracle.page_tokens(oracle.streaming_pages(n, w.N_P, w.sink, w.local), n, w.N_P)
            o, _ = oracle.decode_attention(q, oracle.widen_bf16(K[b][h]), oracle.widen_bf16(V[b][h]),
                                           toks, scale)
            err = np.abs(out[b, h * G:(h + 1) * G] - o)
            assert err.max() <= OUT_MAX_ABS and err.mean() <= OUT_MEAN_ABS, (b, h, err.max())
