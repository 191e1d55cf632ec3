"""Helpers for the GPU parity tests: run the CUDA path through the C-ABI and
compare it with the fp64 oracle on the same seeded inputs.

Tolerances (stated by the method's target and written here once):
  - page statistics and selected page indices: bit-exact (selections wherever
    the oracle's K-th / (K+1)-th score margin exceeds 1e-3 relative; inside
    that band any set whose scores are within 1e-3 of the boundary is valid);
  - attention outputs: max abs error <= 1e-2 and mean abs error <= 1e-3
    against the fp64 oracle; log-sum-exp within 2e-3 absolute.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import block_sparse_attention_page_b200 as lserve
import oracle
import synth
from synth.device import DecodeBuffers, bf16_bits

SEL_MARGIN = 1e-3
OUT_MAX_ABS = 1e-2
OUT_MEAN_ABS = 1e-3
LSE_ABS = 2e-3


def desc_of(w):
    return lserve.paged_desc(w.B, w.H_q, w.H_kv, w.D, w.N_L, w.N_P, w.max_pages, w.num_pool_pages)


def run_decode_path(buf: DecodeBuffers, layer: int = 0, scale=None):
    """stats -> select -> decode on the device; returns host copies."""
    w = buf.w
    d = desc_of(w)
    scale = 1.0 / math.sqrt(w.D) if scale is None else scale
    lserve.page_stats(d, buf.k_pools[layer], buf.block_table, buf.ctx_lens, buf.head_kind,
                      buf.stats[layer])
    lserve.page_select(d, buf.q, buf.stats[layer], buf.block_table, buf.ctx_lens, buf.head_kind,
                       w.top_k, buf.sel[layer], buf.sel_count[layer], phys_scores=buf.scores)
    ws = lserve.alloc_workspace(lserve.workspace_size(lserve.OP_DECODE, d, w.top_k))
    lserve.sparse_decode_attn(d, buf.q, buf.k_pools[layer], buf.v_pools[layer], buf.block_table,
                              buf.ctx_lens, buf.head_kind, buf.sel[layer], buf.sel_count[layer],
                              w.top_k, w.sink, w.local, scale, buf.out, buf.lse, workspace=ws)
    torch.cuda.synchronize()
    st = lserve.read_device_status()
    assert st == lserve.OK, lserve.status_string(st)
    return dict(
        stats=bf16_bits(buf.stats[layer]),
        scores=buf.scores.cpu().numpy(),
        sel=buf.sel[layer].cpu().numpy(),
        sel_count=buf.sel_count[layer].cpu().numpy(),
        out=oracle.widen_bf16(bf16_bits(buf.out)),
        lse=buf.lse.cpu().numpy().astype(np.float64),
        scale=scale,
    )


def run_decode_path_kv8(buf: DecodeBuffers, layer: int = 0, scale=None, overlap=False, bits=8):
    """stats -> select on the bf16 cache, then quantize the pools to `bits`-bit
    codes (8: int8 [pool][H_kv][N_P][D]; 4: uint8 [pool][H_kv][N_P][D/2], two
    codes per byte) and decode over the quantized cache; returns host copies
    (plus codes and scales)."""
    w = buf.w
    d = desc_of(w)
    scale = 1.0 / math.sqrt(w.D) if scale is None else scale
    lserve.page_stats(d, buf.k_pools[layer], buf.block_table, buf.ctx_lens, buf.head_kind,
                      buf.stats[layer])
    lserve.page_select(d, buf.q, buf.stats[layer], buf.block_table, buf.ctx_lens, buf.head_kind,
                       w.top_k, buf.sel[layer], buf.sel_count[layer], phys_scores=buf.scores)
    shape = w.pool_shape() if bits == 8 else w.pool_shape()[:-1] + (w.D // 2,)
    k8 = torch.full(shape, 99, dtype=torch.int8, device=buf.device)
    v8 = torch.full(shape, -99, dtype=torch.int8, device=buf.device)
    ks = torch.full((w.num_pool_pages, w.H_kv, w.D), float("nan"), dtype=torch.float32,
                    device=buf.device)
    vs = torch.full_like(ks, float("nan"))
    lserve.quantize_pages_kv8(d, buf.k_pools[layer], buf.v_pools[layer], buf.block_table,
                              buf.ctx_lens, k8, v8, ks, vs, bits=bits)
    ws = lserve.alloc_workspace(lserve.workspace_size(lserve.OP_DECODE, d, w.top_k))
    lserve.sparse_decode_attn_kv8(d, buf.q, k8, v8, ks, vs, buf.block_table, buf.ctx_lens,
                                  buf.head_kind, buf.sel[layer], buf.sel_count[layer], w.top_k,
                                  w.sink, w.local, scale, buf.out, buf.lse, workspace=ws,
                                  overlap_prologue=overlap, bits=bits)
    torch.cuda.synchronize()
    st = lserve.read_device_status()
    assert st == lserve.OK, lserve.status_string(st)
    return dict(
        stats=bf16_bits(buf.stats[layer]),
        scores=buf.scores.cpu().numpy(),
        sel=buf.sel[layer].cpu().numpy(),
        sel_count=buf.sel_count[layer].cpu().numpy(),
        out=oracle.widen_bf16(bf16_bits(buf.out)),
        lse=buf.lse.cpu().numpy().astype(np.float64),
        scale=scale,
        k8=k8, v8=v8, k_scale=ks, v_scale=vs, bits=bits,
    )


def unpack_codes4(packed: np.ndarray) -> np.ndarray:
    """uint8 [..][D/2] -> int8 [..][D]: channel 2i is the low nibble of byte i,
    2i+1 the high nibble, each a 4-bit two's complement code."""
    u = packed.astype(np.uint8)
    lo = (u & 0xF).astype(np.int8)
    hi = (u >> 4).astype(np.int8)
    lo = np.where(lo >= 8, lo - 16, lo).astype(np.int8)
    hi = np.where(hi >= 8, hi - 16, hi).astype(np.int8)
    out = np.empty(packed.shape[:-1] + (packed.shape[-1] * 2,), dtype=np.int8)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return out


def check_quantized_pages(w, res, b, h):
    """Codes and scales of every page of (b, h), K and V, bit for bit against
    the oracle's quantize_kv8 / quantize_kv4; rows past the valid tokens hold
    code 0."""
    n = int(w.ctx_lens[b])
    bits = res.get("bits", 8)
    quant = oracle.quantize_kv8 if bits == 8 else oracle.quantize_kv4
    for key in ("k8", "v8", "k_scale", "v_scale"):   # one device -> host copy per call
        if key + "_np" not in res:
            res[key + "_np"] = res[key].cpu().numpy()
            if bits == 4 and key in ("k8", "v8"):
                res[key + "_np"] = unpack_codes4(res[key + "_np"].view(np.uint8))
    for name, bits, codes_all, scale_all in (("K", w.k_seq(b, h), res["k8_np"], res["k_scale_np"]),
                                             ("V", w.v_seq(b, h), res["v8_np"], res["v_scale_np"])):
        for m in range(-(-n // w.N_P)):
            pid = int(w.block_table[b, m])
            t0, t1 = m * w.N_P, min((m + 1) * w.N_P, n)
            codes, sc = quant(bits[t0:t1])
            got_c = codes_all[pid, h]
            got_s = scale_all[pid, h]
            assert np.array_equal(got_c[:t1 - t0], codes), (name, b, h, m)
            assert np.all(got_c[t1 - t0:] == 0), (name, b, h, m)
            assert np.array_equal(got_s.view(np.uint32), sc.view(np.uint32)), (name, b, h, m)


def check_stats(w, res, b, h, k):
    """Bit-exact k_min/k_max of every logical page of (b, h) against the oracle."""
    n = int(w.ctx_lens[b])
    kmin, kmax = oracle.page_stats(k, w.N_L)
    g = w.g
    want_min = synth.to_bf16(kmin)
    want_max = synth.to_bf16(kmax)
    j = np.arange(kmin.shape[0])
    got = res["stats"][w.block_table[b, j // g], h, j % g]   # [logical page][2][D]
    bad = np.flatnonzero(np.any(got[:, 0] != want_min, axis=1) | np.any(got[:, 1] != want_max, axis=1))
    assert bad.size == 0, (b, h, int(bad[0]) if bad.size else None)
    return n


def check_selection(w, res, b, h, P):
    """Selection parity per the tie/margin rule; returns the GPU's page list."""
    K = w.top_k
    M = len(P)
    cnt = int(res["sel_count"][b, h])
    sel = res["sel"][b, h]
    assert cnt == min(K, M)
    assert np.all(sel[cnt:] == -1)
    got = [int(x) for x in sel[:cnt]]
    assert got == sorted(set(got)) and all(0 <= m < M for m in got)
    want = oracle.select_top_k(P, K)
    if M <= K:
        assert got == want
        return got
    order = np.sort(P)[::-1]
    pk, pk1 = order[K - 1], order[K]
    margin = (pk - pk1) / max(abs(pk), abs(pk1), 1e-30)
    if margin > SEL_MARGIN:
        assert got == want, (b, h, margin)
    else:
        delta = SEL_MARGIN * max(abs(pk), abs(pk1))
        inside = np.zeros(M, dtype=bool)
        inside[got] = True
        assert P[inside].min() >= P[~inside].max() - delta, (b, h)
    return got


def check_scores(res, b, h, P):
    got = res["scores"][b, h, :len(P)].astype(np.float64)
    tol = 1e-5 * np.abs(P).max() + 1e-3
    assert np.max(np.abs(got - P)) <= tol, (b, h, np.max(np.abs(got - P)), tol)


def check_outputs(w, res, b, h, q, k, v, pages, stats_out=None):
    n = int(w.ctx_lens[b])
    G = w.G
    o, lse = oracle.decode_attention(q, k, v, oracle.page_tokens(pages, n, w.N_P), res["scale"])
    got = res["out"][b, h * G:(h + 1) * G]
    err = np.abs(got - o)
    if stats_out is not None:
        stats_out.append((err.max(), err.mean(), np.abs(o).max()))
    assert err.max() <= OUT_MAX_ABS, (b, h, err.max())
    assert err.mean() <= OUT_MEAN_ABS, (b, h, err.mean())
    gl = res["lse"][b, h * G:(h + 1) * G]
    if np.all(np.isneginf(lse)):
        assert np.all(np.isneginf(gl))
    else:
        assert np.max(np.abs(gl - lse)) <= LSE_ABS, (b, h, gl, lse)


def check_pair(w, res, b, h, errs=None, check_stats_bits=True, kv8=False):
    """Full parity of one (sequence, KV head): stats, scores, selection, output.
    kv8: the attention read the quantized cache (res["bits"]: 8 or 4), so the
    oracle attends the dequantized keys and values (pages and statistics stay
    those of bf16 K)."""
    G = w.G
    n = int(w.ctx_lens[b])
    q = oracle.widen_bf16(w.q[b, h * G:(h + 1) * G])
    k_bits = w.k_seq(b, h)
    v_bits = w.v_seq(b, h)
    k = oracle.widen_bf16(k_bits)
    v = oracle.widen_bf16(v_bits)
    k_att, v_att = k, v
    if kv8:
        k_att = oracle.dequantized_seq(k_bits, w.N_P, res.get("bits", 8))
        v_att = oracle.dequantized_seq(v_bits, w.N_P, res.get("bits", 8))
    if w.head_kind[h] == 0:
        if n > 0:
            if check_stats_bits:
                check_stats(w, res, b, h, k)
            kmin, kmax = oracle.page_stats(k, w.N_L)
            P = oracle.physical_scores(oracle.logical_scores(q, kmin, kmax), w.g)
            check_scores(res, b, h, P)
            pages = check_selection(w, res, b, h, P)
        else:
            assert int(res["sel_count"][b, h]) == 0
            pages = []
    else:
        assert int(res["sel_count"][b, h]) == 0 and np.all(res["sel"][b, h] == -1)
        pages = oracle.streaming_pages(n, w.N_P, w.sink, w.local)
    check_outputs(w, res, b, h, q, k_att, v_att, pages, errs)
    return pages
