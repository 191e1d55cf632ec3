"""Sequence-sharded decode on one GPU (parity with the unsharded path and the
fp64 oracle).

N shards of every sequence are emulated on the one device: each shard gets
its own block-table rows (shard-local page ordinals) and local lengths, and
the all-gathers become writes into the gathered buffers.  No kernel waits for
another.  The merged choice must equal the unsharded lserve_page_select bit
for bit; the combined output must meet the attention tolerance against the
oracle over those pages.  A second test runs SeqShardStep in N host threads
(one CUDA stream each) with a host-side all-gather.
"""
import math
import threading

import numpy as np
import pytest
import torch

import block_sparse_attention_page_b200 as lserve
import oracle
import synth
from parity import check_outputs, desc_of, run_decode_path
from synth.device import DecodeBuffers, bf16_bits

pytestmark = pytest.mark.gpu


class _View:
    """Shard r's own paged cache: block-table rows of its pages and its lengths."""

    def __init__(self, w, r, N, stride):
        self.bounds = [lserve.seqshard_bounds(int(w.ctx_lens[b]), w.N_P, r, N) for b in range(w.B)]
        ml = max([stride, 1] + [hi - lo for lo, hi, _ in self.bounds])
        bt = np.full((w.B, ml), -1, dtype=np.int32)
        for b, (lo, hi, _) in enumerate(self.bounds):
            bt[b, :hi - lo] = w.block_table[b, lo:hi]
        self.bt = torch.from_numpy(bt).cuda()
        self.ctx = torch.tensor([n for _, _, n in self.bounds], dtype=torch.int32, device="cuda")
        self.desc = lserve.paged_desc(w.B, w.H_q, w.H_kv, w.D, w.N_L, w.N_P, ml, w.num_pool_pages)


def _stats(w, buf):
    lserve.page_stats(desc_of(w), buf.k_pool, buf.block_table, buf.ctx_lens, buf.head_kind, buf.stats[0])


def run_sharded(w, buf, N):
    """The sharded step with its exchanges emulated; returns host copies."""
    K, B, H_kv, H_q, D = w.top_k, w.B, w.H_kv, w.H_q, w.D
    scale = 1.0 / math.sqrt(D)
    stride = lserve.seqshard_sel_stride(desc_of(w), K, w.sink, w.local)
    views = [_View(w, r, N, stride) for r in range(N)]
    all_s = torch.full((N, B, H_kv, K), float("nan"), device="cuda")
    all_p = torch.full((N, B, H_kv, K), -7, dtype=torch.int32, device="cuda")
    for r, v in enumerate(views):
        sel = torch.full((B, H_kv, K), -7, dtype=torch.int32, device="cuda")
        cnt = torch.full((B, H_kv), -7, dtype=torch.int32, device="cuda")
        sc = torch.full((B, H_kv, v.desc.max_pages_per_seq), float("nan"), device="cuda")
        lserve.page_select(v.desc, buf.q, buf.stats[0], v.bt, v.ctx, buf.head_kind, K, sel, cnt,
                           phys_scores=sc)
        lserve.seqshard_candidates(v.desc, r, N, buf.ctx_lens, buf.head_kind, sel, cnt, sc, K,
                                   all_s[r], all_p[r])
    all_o = torch.full((N, B * H_q, D), float("nan"), device="cuda")
    all_l = torch.full((N, B * H_q), float("nan"), device="cuda")
    every_head = torch.zeros(H_kv, dtype=torch.uint8, device="cuda")
    merged = []
    for r, v in enumerate(views):
        sel_m = torch.full((B, H_kv, stride), -7, dtype=torch.int32, device="cuda")
        cnt_m = torch.full((B, H_kv), -7, dtype=torch.int32, device="cuda")
        lserve.seqshard_merge(v.desc, r, N, buf.ctx_lens, buf.head_kind, all_s, all_p, K, w.sink, w.local,
                              sel_m, cnt_m)
        ws = lserve.alloc_workspace(lserve.workspace_size(lserve.OP_DECODE, v.desc, stride))
        lserve.sparse_decode_attn(v.desc, buf.q, buf.k_pool, buf.v_pool, v.bt, v.ctx, every_head, sel_m,
                                  cnt_m, stride, w.sink, w.local, scale, all_o[r], all_l[r], workspace=ws,
                                  out_f32=True)
        merged.append((sel_m, cnt_m))
    out = torch.empty((B, H_q, D), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, H_q), dtype=torch.float32, device="cuda")
    lserve.seqshard_combine(all_o, all_l, out.view(B * H_q, D), lse.view(-1))
    torch.cuda.synchronize()
    st = lserve.read_device_status()
    assert st == lserve.OK, lserve.status_string(st)
    return dict(views=views, stride=stride,
                sel=[(s.cpu().numpy(), c.cpu().numpy()) for s, c in merged],
                out=oracle.widen_bf16(bf16_bits(out)), lse=lse.cpu().numpy().astype(np.float64),
                scale=scale)


def _check_against_unsharded(w, res, sh, pairs=None):
    N = len(sh["views"])
    G = w.G
    for b in range(w.B):
        n = int(w.ctx_lens[b])
        for h in range(w.H_kv):
            if pairs is not None and (b, h) not in pairs:
                continue
            got = []
            for r in range(N):
                lo, hi, _ = sh["views"][r].bounds[b]
                s, c = sh["sel"][r]
                cnt = int(c[b, h])
                assert 0 <= cnt <= sh["stride"]
                assert np.all(s[b, h, cnt:] == -1)
                loc = [int(x) for x in s[b, h, :cnt]]
                assert loc == sorted(set(loc)) and all(0 <= m < hi - lo for m in loc)
                if w.head_kind[h] == 1:
                    assert loc == oracle.shard_streaming_pages(n, w.N_P, w.sink, w.local, lo, hi)
                got += [lo + m for m in loc]
            if w.head_kind[h] == 0:
                cg = int(res["sel_count"][b, h])
                assert got == [int(x) for x in res["sel"][b, h, :cg]], (b, h)  # bit for bit
            else:
                assert got == oracle.streaming_pages(n, w.N_P, w.sink, w.local)
            q = oracle.widen_bf16(w.q[b, h * G:(h + 1) * G])
            k = oracle.widen_bf16(w.k_seq(b, h))
            v = oracle.widen_bf16(w.v_seq(b, h))
            check_outputs(w, sh, b, h, q, k, v, got)
            # and the unsharded call: the same attention up to rounding
            d = np.abs(sh["out"][b, h * G:(h + 1) * G] - res["out"][b, h * G:(h + 1) * G])
            assert d.max() <= 1e-2, (b, h, d.max())


@pytest.mark.parametrize("N", [1, 2, 3, 5])
def test_sharded_decode_matches_unsharded_and_oracle(N):
    # lengths: several shards, a 3-page sequence (empty shards at N = 5), an empty one
    w = synth.decode_workload(4, 8, 2, 128, 16, 64, 8, 64, 256, [1000, 2500, 130, 0], seed=41)
    buf = DecodeBuffers(w)
    res = run_decode_path(buf)           # also builds the statistics
    sh = run_sharded(w, buf, N)
    _check_against_unsharded(w, res, sh)
    assert np.all(sh["out"][3] == 0) and np.all(np.isneginf(sh["lse"][3]))


@pytest.mark.parametrize("G,D,N_P,K", [(1, 64, 32, 6), (8, 128, 128, 4), (4, 64, 64, 16)])
def test_sharded_decode_shapes(G, D, N_P, K):
    H_kv = 4
    w = synth.decode_workload(2, G * H_kv, H_kv, D, 16, N_P, K, 64, 256, [3000, 777], seed=43 + G)
    buf = DecodeBuffers(w)
    res = run_decode_path(buf)
    _check_against_unsharded(w, res, run_sharded(w, buf, 3))


def test_sharded_decode_many_proposals():
    """4 shards x top-136 = 544 proposals: more than the merge ranks directly,
    so the global choice comes from its bisection over score keys and pages."""
    w = synth.decode_workload(2, 8, 2, 128, 16, 64, 136, 64, 256, [20000, 9000], seed=53)
    buf = DecodeBuffers(w)
    res = run_decode_path(buf)
    _check_against_unsharded(w, res, run_sharded(w, buf, 4))


@pytest.mark.parametrize("N", [4, 8])
def test_long_decode_256k_sharded(N):
    w = synth.long_decode_256k()
    buf = DecodeBuffers(w)
    res = run_decode_path(buf)
    _check_against_unsharded(w, res, run_sharded(w, buf, N))


def test_combine_closed_forms():
    rows, D = 5, 64
    o = torch.randn((2, rows, D), device="cuda")
    lse = torch.zeros((2, rows), device="cuda")
    lse[0, 1], lse[1, 2] = -math.inf, -math.inf     # row 1 only from shard 1, row 2 only from shard 0
    lse[:, 3] = -math.inf                           # row 3: nothing attended anywhere
    lse[0, 4], lse[1, 4] = 2.0, 2.0 + math.log(3.0)  # row 4: weights 1 : 3
    out = torch.empty((rows, D), dtype=torch.bfloat16, device="cuda")
    lo = torch.empty(rows, device="cuda")
    lserve.seqshard_combine(o, lse, out, lo)
    torch.cuda.synchronize()
    o64 = o.double().cpu().numpy()
    got = out.double().cpu().numpy()
    want = np.stack([(o64[0, 0] + o64[1, 0]) / 2, o64[1, 1], o64[0, 2], np.zeros(D),
                     (o64[0, 4] + 3 * o64[1, 4]) / 4])
    assert np.abs(got - want).max() <= 2 ** -8 * np.abs(want).max() + 1e-6
    lo = lo.cpu().numpy()
    assert lo[0] == pytest.approx(math.log(2.0), abs=1e-6)
    assert lo[1] == 0.0 and lo[2] == 0.0 and np.isneginf(lo[3])
    assert lo[4] == pytest.approx(2.0 + math.log(4.0), abs=1e-6)


def test_seqshard_step_in_threads_equals_the_emulation():
    """SeqShardStep on N host threads (one stream each), the all-gather done on
    the host between the steps: bit-identical to the emulated sequence."""
    N = 3
    w = synth.decode_workload(2, 8, 2, 128, 16, 64, 8, 64, 256, [2000, 4100], seed=47)
    buf = DecodeBuffers(w)
    _stats(w, buf)
    torch.cuda.synchronize()
    ref = run_sharded(w, buf, N)
    stride = ref["stride"]
    bar = threading.Barrier(N, timeout=120)
    box = [None] * N

    def gather_for(rank):
        def ag(dst, src):
            torch.cuda.current_stream().synchronize()
            box[rank] = src
            bar.wait()
            for r in range(N):
                dst[r].copy_(box[r])
            torch.cuda.current_stream().synchronize()
            bar.wait()
        return ag

    outs = [None] * N
    errors = []

    def run(rank):
        try:
            v = _View(w, rank, N, stride)
            step = lserve.SeqShardStep(v.desc, rank, N, w.top_k, w.sink, w.local, all_gather=gather_for(rank))
            out = torch.empty((w.B, w.H_q, w.D), dtype=torch.bfloat16, device="cuda")
            lse = torch.empty((w.B, w.H_q), dtype=torch.float32, device="cuda")
            torch.cuda.synchronize()  # buffers and the zeroed workspace are ready before stream s runs
            s = torch.cuda.Stream()
            with torch.cuda.stream(s):
                step.select(buf.q, buf.stats[0], v.bt, v.ctx, buf.ctx_lens, buf.head_kind)
                step.attend(buf.q, buf.k_pool, buf.v_pool, v.bt, v.ctx, ref["scale"], out, lse)
            s.synchronize()
            outs[rank] = (bf16_bits(out), lse.cpu().numpy())
        except BaseException as e:  # reported by the main thread
            errors.append(e)
            bar.abort()

    threads = [threading.Thread(target=run, args=(r,)) for r in range(N)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=300)
    assert not errors, errors
    assert lserve.read_device_status() == lserve.OK
    for r in range(N):  # every shard ends with the whole result
        assert np.array_equal(oracle.widen_bf16(outs[r][0]), ref["out"])
        assert np.array_equal(outs[r][1].astype(np.float64), ref["lse"])
