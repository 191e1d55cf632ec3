"""Seeded synthetic workloads for LServe-style unified sparse attention.

This module only draws random numbers and lays them out; it holds none of the
attention method's arithmetic.  Both the CUDA path's tests/benchmarks and the
CPU oracle's tests take their inputs from here.  The elementwise generator is
``synth.c`` (SplitMix64 counter hash -> Box-Muller -> bfloat16); small seeded
choices (lengths, permutations, planted positions, channel scales) use the
same SplitMix64 definition re-stated in Python below.

Workload shapes follow the five synthetic configurations of the LServe page
(arXiv 2502.14866 explainer): Llama-3-8B GQA decode, 256K long decode,
128K block-sparse prefill, a mixed-length batch over a shuffled page pool, and
a tiny case.  The pages measure accuracy on LongBench/RULER/NIAH with trained
models; none of that is available, so planted keys play the "needle" role.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "libsynth.so")
_SRC = os.path.join(_HERE, "synth.c")

M64 = (1 << 64) - 1
GOLDEN = 0x9E3779B97F4A7C15

# tensor tags: each tensor of a workload draws from its own keyed stream
TAG_Q, TAG_K, TAG_V, TAG_PQ, TAG_PK, TAG_PV = 1, 2, 3, 4, 5, 6
TAG_KSCALE, TAG_VSCALE, TAG_OUTLIER, TAG_LENS, TAG_PERM, TAG_PLANT = 7, 8, 9, 10, 11, 12

BF16_NAN = 0x7FC0


def build(force: bool = False) -> str:
    """Compile libsynth.so next to its source (gcc, OpenMP)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", _SRC, "-o", _SO, "-lm"])
    return _SO


_lib = None


def _L():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_SO)
        u64, i64, dp, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p
        lib.synth_mix64.restype = u64
        lib.synth_mix64.argtypes = [u64]
        lib.synth_normal.restype = ctypes.c_double
        lib.synth_normal.argtypes = [u64, u64]
        lib.synth_to_bf16.restype = ctypes.c_uint16
        lib.synth_to_bf16.argtypes = [ctypes.c_double]
        lib.synth_seq_key.restype = u64
        lib.synth_seq_key.argtypes = [u64, i64, i64, i64]
        lib.synth_fill_normal_bf16.restype = None
        lib.synth_fill_normal_bf16.argtypes = [u64, u64, i64, i64, dp, dp, vp, i64]
        lib.synth_fill_pool_seq.restype = None
        lib.synth_fill_pool_seq.argtypes = [u64, i64, i64, i64, i64, i64, vp, dp, dp, vp,
                                            ctypes.c_uint16, vp]
        lib.synth_fill_seq_dense.restype = None
        lib.synth_fill_seq_dense.argtypes = [u64, i64, i64, i64, i64, i64, i64, dp, dp, vp, vp]
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


# --- small seeded draws (same SplitMix64 definition as synth.c) -------------

def mix64(z: int) -> int:
    z &= M64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & M64
    return z ^ (z >> 31)


def draw(key: int, i: int) -> int:
    return mix64((key + (i + 1) * GOLDEN) & M64)


def uniform(key: int, i: int) -> float:
    return ((draw(key, i) >> 11) + 0.5) * 2.0 ** -53


def tensor_key(seed: int, tag: int) -> int:
    return mix64((seed * 0x100000001B3) ^ mix64(tag))


def uniform_array(key: int, n: int) -> np.ndarray:
    return np.array([uniform(key, i) for i in range(n)], dtype=np.float64)


def randint_array(key: int, n: int, lo: int, hi: int) -> np.ndarray:
    """Integers uniform on [lo, hi] inclusive (multiply-shift on the top bits)."""
    span = hi - lo + 1
    return np.array([lo + ((draw(key, i) >> 11) * span >> 53) for i in range(n)], dtype=np.int64)


def permutation(key: int, n: int) -> np.ndarray:
    keys = np.array([draw(key, i) for i in range(n)], dtype=np.uint64)
    return np.argsort(keys, kind="stable").astype(np.int64)


def to_bf16(x) -> np.ndarray:
    """float64 -> bf16 bits, via float32 RNE then bf16 RNE (same as synth.c)."""
    f = np.asarray(x, dtype=np.float64).astype(np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


def bf16_to_f64(u) -> np.ndarray:
    u = np.asarray(u, dtype=np.uint16)
    return (u.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def normal_bf16(key: int, shape, counter0: int = 0, scale=None, shift=None) -> np.ndarray:
    shape = tuple(int(s) for s in shape)
    cols = shape[-1]
    rows = int(np.prod(shape[:-1])) if len(shape) > 1 else 1
    out = np.empty(shape, dtype=np.uint16)
    sc = None if scale is None else np.ascontiguousarray(scale, dtype=np.float64)
    sh = None if shift is None else np.ascontiguousarray(shift, dtype=np.float64)
    _L().synth_fill_normal_bf16(key, counter0, rows, cols, _ptr(sc), _ptr(sh), _ptr(out), cols)
    return out


# --- decode workloads ----------------------------------------------------------

@dataclass
class DecodeWorkload:
    """A paged decode problem: q for one step, a K/V pool, block table, lengths.

    Layouts (bf16 stored as uint16 bits):
      q            [B][H_q][D]
      K/V pool     [num_pool_pages][H_kv][N_P][D]
      block_table  [B][max_pages] int32 pool ids (-1 past the sequence's pages)
      ctx_lens     [B] int32
      head_kind    [H_kv] uint8 (0 retrieval, 1 streaming)
    """
    name: str
    seed: int
    B: int
    H_q: int
    H_kv: int
    D: int
    N_L: int
    N_P: int
    top_k: int
    sink: int
    local: int
    ctx_lens: np.ndarray
    head_kind: np.ndarray
    block_table: np.ndarray
    num_pool_pages: int
    q: np.ndarray
    k_scale: np.ndarray | None = None      # [H_kv][D]
    v_scale: np.ndarray | None = None      # [H_kv][D]
    k_shift: np.ndarray | None = None      # [B][H_kv][D]
    shift_pages: np.ndarray | None = None  # [B][max_pages] uint8
    k_patches: list = field(default_factory=list)  # (b, h, t, bf16 row [D])
    planted_pages: dict = field(default_factory=dict)  # (b, h) -> page ordinals

    @property
    def G(self):
        return self.H_q // self.H_kv

    @property
    def g(self):
        return self.N_P // self.N_L

    @property
    def max_pages(self):
        return self.block_table.shape[1]

    def npages(self, b):
        return -(-int(self.ctx_lens[b]) // self.N_P)

    def _keys(self):
        return tensor_key(self.seed, TAG_K), tensor_key(self.seed, TAG_V)

    def k_seq(self, b: int, h: int) -> np.ndarray:
        """Dense [n][D] bf16 bits of K for sequence b, KV head h."""
        n = int(self.ctx_lens[b])
        out = np.empty((n, self.D), dtype=np.uint16)
        sh = None if self.k_shift is None else np.ascontiguousarray(self.k_shift[b])
        sp = None if self.shift_pages is None else np.ascontiguousarray(self.shift_pages[b])
        sc = None if self.k_scale is None else np.ascontiguousarray(self.k_scale)
        _L().synth_fill_seq_dense(self._keys()[0], b, self.H_kv, h, self.D, self.N_P, n,
                                  _ptr(sc), _ptr(sh), _ptr(sp), _ptr(out))
        for (pb, ph, t, row) in self.k_patches:
            if pb == b and ph == h:
                out[t] = row
        return out

    def v_seq(self, b: int, h: int) -> np.ndarray:
        n = int(self.ctx_lens[b])
        out = np.empty((n, self.D), dtype=np.uint16)
        sc = None if self.v_scale is None else np.ascontiguousarray(self.v_scale)
        _L().synth_fill_seq_dense(self._keys()[1], b, self.H_kv, h, self.D, self.N_P, n,
                                  _ptr(sc), None, None, _ptr(out))
        return out

    def pool_shape(self):
        return (self.num_pool_pages, self.H_kv, self.N_P, self.D)

    def fill_pools(self, k_pool: np.ndarray, v_pool: np.ndarray, pad: int = 0) -> None:
        """Fill caller-provided uint16 arrays of shape pool_shape() (may be pinned memory)."""
        assert k_pool.shape == self.pool_shape() and v_pool.shape == self.pool_shape()
        assert k_pool.dtype == np.uint16 and k_pool.flags.c_contiguous and v_pool.flags.c_contiguous
        kk, kv = self._keys()
        L = _L()
        sc_k = None if self.k_scale is None else np.ascontiguousarray(self.k_scale)
        sc_v = None if self.v_scale is None else np.ascontiguousarray(self.v_scale)
        for b in range(self.B):
            row = np.ascontiguousarray(self.block_table[b], dtype=np.int32)
            sh = None if self.k_shift is None else np.ascontiguousarray(self.k_shift[b])
            sp = None if self.shift_pages is None else np.ascontiguousarray(self.shift_pages[b])
            n = int(self.ctx_lens[b])
            L.synth_fill_pool_seq(kk, b, self.H_kv, self.D, self.N_P, n, _ptr(row), _ptr(sc_k),
                                  _ptr(sh), _ptr(sp), pad, _ptr(k_pool))
            L.synth_fill_pool_seq(kv, b, self.H_kv, self.D, self.N_P, n, _ptr(row), _ptr(sc_v),
                                  None, None, pad, _ptr(v_pool))
        for (b, h, t, row) in self.k_patches:
            pid = self.block_table[b][t // self.N_P]
            k_pool[pid, h, t % self.N_P] = row

    def make_pools(self, pad: int = 0):
        k = np.empty(self.pool_shape(), dtype=np.uint16)
        v = np.empty(self.pool_shape(), dtype=np.uint16)
        self.fill_pools(k, v, pad)
        return k, v

    def kv_bytes(self) -> int:
        return 2 * self.num_pool_pages * self.H_kv * self.N_P * self.D * 2


def _identity_table(B, max_pages, ctx_lens, N_P):
    bt = np.full((B, max_pages), -1, dtype=np.int32)
    for b in range(B):
        np_b = -(-int(ctx_lens[b]) // N_P)
        bt[b, :np_b] = b * max_pages + np.arange(np_b)
    return bt, B * max_pages


def _head_kind(H_kv):
    hk = np.zeros(H_kv, dtype=np.uint8)
    hk[H_kv // 2:] = 1   # KV heads [0, H/2) retrieval, [H/2, H) streaming
    return hk


def _qbar(q, b, h, G):
    return bf16_to_f64(q[b, h * G:(h + 1) * G]).mean(axis=0)


def decode_workload(B, H_q, H_kv, D, N_L, N_P, top_k, sink, local, ctx_lens, seed,
                    name="custom", shuffle=False, head_kind=None) -> DecodeWorkload:
    """A generic decode workload: q, K, V ~ N(0,1), identity or shuffled pool."""
    ctx_lens = np.asarray(ctx_lens, dtype=np.int32)
    max_pages = max(1, -(-int(ctx_lens.max()) // N_P)) if len(ctx_lens) else 1
    if shuffle:
        npg = [-(-int(n) // N_P) for n in ctx_lens]
        total = int(sum(npg))
        perm = permutation(tensor_key(seed, TAG_PERM), total)
        bt = np.full((B, max_pages), -1, dtype=np.int32)
        run = 0
        for b in range(B):
            bt[b, :npg[b]] = perm[run:run + npg[b]]
            run += npg[b]
        num_pool = max(total, 1)
    else:
        bt, num_pool = _identity_table(B, max_pages, ctx_lens, N_P)
    hk = _head_kind(H_kv) if head_kind is None else np.asarray(head_kind, dtype=np.uint8)
    q = normal_bf16(tensor_key(seed, TAG_Q), (B, H_q, D))
    return DecodeWorkload(name, seed, B, H_q, H_kv, D, N_L, N_P, top_k, sink, local, ctx_lens, hk,
                          bt, num_pool, q)


def tiny_decode() -> DecodeWorkload:
    """Tiny: B=1, 4 q / 2 KV heads, D=64, n=2048, N_L=16, N_P=64, top-K 8,
    KV head 0 retrieval, head 1 streaming (sink 64 + local 256); 8 planted keys
    (one token each in 8 distinct physical pages of KV head 0) set to 4*qbar."""
    seed = 1001
    w = decode_workload(1, 4, 2, 64, 16, 64, 8, 64, 256, [2048], seed, name="tiny")
    kp = tensor_key(seed, TAG_PLANT)
    pages = permutation(kp, 32)[:8]
    qb = _qbar(w.q, 0, 0, w.G)
    row = to_bf16(4.0 * qb)
    for i, m in enumerate(sorted(int(p) for p in pages)):
        t = m * 64 + int(draw(kp, 1000 + i) % 64)
        w.k_patches.append((0, 0, t, row))
    w.planted_pages[(0, 0)] = sorted(int(p) for p in pages)
    return w


def llama3_8b_decode() -> DecodeWorkload:
    """Llama-3-8B-shaped decode layer: B=4, n=64K, 32 q / 8 KV heads, D=128,
    N_L=16, N_P=64, top-K 64 pages, sink 128 + local 512 for the streaming half.
    K/V ~ N(0,1) * s_c with s_c ~ U[0.5, 2] per (KV head, channel); two outlier
    channels per KV head get s_c = 8 on K."""
    seed = 1002
    w = decode_workload(4, 32, 8, 128, 16, 64, 64, 128, 512, [65536] * 4, seed,
                        name="llama3_8b_decode")
    H, D = w.H_kv, w.D
    w.k_scale = 0.5 + 1.5 * uniform_array(tensor_key(seed, TAG_KSCALE), H * D).reshape(H, D)
    w.v_scale = 0.5 + 1.5 * uniform_array(tensor_key(seed, TAG_VSCALE), H * D).reshape(H, D)
    ko = tensor_key(seed, TAG_OUTLIER)
    for h in range(H):
        ch = permutation(mix64(ko ^ (h + 1)), D)[:2]
        w.k_scale[h, ch] = 8.0
    return w


def long_decode_256k() -> DecodeWorkload:
    """Long decode: B=1, n=256K, 32 q / 8 KV heads, D=128, N_L=16, N_P=128 (g=8),
    top-K 32, sink 128 + local 1024; 16 planted pages at ordinals
    floor((i + 1/2) * 2048 / 16) whose keys are N(0,1) + 2*qbar (retrieval heads)."""
    seed = 1003
    w = decode_workload(1, 32, 8, 128, 16, 128, 32, 128, 1024, [262144], seed,
                        name="long_decode_256k")
    npages = w.npages(0)
    planted = [int((i + 0.5) * npages / 16) for i in range(16)]
    w.shift_pages = np.zeros((1, w.max_pages), dtype=np.uint8)
    w.shift_pages[0, planted] = 1
    w.k_shift = np.zeros((1, w.H_kv, w.D), dtype=np.float64)
    for h in range(w.H_kv):
        if w.head_kind[h] == 0:
            w.k_shift[0, h] = 2.0 * _qbar(w.q, 0, h, w.G)
            w.planted_pages[(0, h)] = planted
    return w


def llama2_7b_mha_decode() -> DecodeWorkload:
    """Llama-2-7B-shaped (MHA, G = 1) decode layer: B=4, n=32K, 32 query = 32 KV
    heads, D=128, N_L=16, N_P=64, top-K 64 pages (4K tokens), sink 128 + local
    512 for the streaming half; K/V ~ N(0,1) * s_c, s_c ~ U[0.5, 2] per
    (KV head, channel)."""
    seed = 1006
    w = decode_workload(4, 32, 32, 128, 16, 64, 64, 128, 512, [32768] * 4, seed,
                        name="llama2_7b_mha_decode")
    H, D = w.H_kv, w.D
    w.k_scale = 0.5 + 1.5 * uniform_array(tensor_key(seed, TAG_KSCALE), H * D).reshape(H, D)
    w.v_scale = 0.5 + 1.5 * uniform_array(tensor_key(seed, TAG_VSCALE), H * D).reshape(H, D)
    return w


def mixed_batch_decode() -> DecodeWorkload:
    """Batched mixed-length decode: B=32, n_b ~ U{8192..131072}, 32 q / 8 KV
    heads, D=128, N_L=16, N_P=64, pages shuffled through the block table,
    top-K 32, sink 64 + local 512."""
    seed = 1005
    lens = randint_array(tensor_key(seed, TAG_LENS), 32, 8192, 131072)
    return decode_workload(32, 32, 8, 128, 16, 64, 32, 64, 512, lens, seed,
                           name="mixed_batch_decode", shuffle=True)


# --- prefill workloads ---------------------------------------------------------

@dataclass
class PrefillWorkload:
    """Q [T][H_q][D], K/V [T][H_kv][D], bf16 bits, ~N(0,1)."""
    name: str
    seed: int
    T: int
    H_q: int
    H_kv: int
    D: int
    block: int
    sink_blocks: int
    local_blocks: int
    head_kind: np.ndarray

    @property
    def G(self):
        return self.H_q // self.H_kv

    def q(self):
        return normal_bf16(tensor_key(self.seed, TAG_PQ), (self.T, self.H_q, self.D))

    def k(self):
        return normal_bf16(tensor_key(self.seed, TAG_PK), (self.T, self.H_kv, self.D))

    def v(self):
        return normal_bf16(tensor_key(self.seed, TAG_PV), (self.T, self.H_kv, self.D))

    def q_rows(self, t0, t1):
        """Rows [t0, t1) of Q without generating the rest."""
        return normal_bf16(tensor_key(self.seed, TAG_PQ), (t1 - t0, self.H_q, self.D),
                           counter0=t0 * self.H_q * self.D)


def prefill_workload(T, H_q, H_kv, D, block, seed, sink_blocks=1, local_blocks=4,
                     name="custom", head_kind=None) -> PrefillWorkload:
    hk = _head_kind(H_kv) if head_kind is None else np.asarray(head_kind, dtype=np.uint8)
    return PrefillWorkload(name, seed, T, H_q, H_kv, D, block, sink_blocks, local_blocks, hk)


def tiny_prefill() -> PrefillWorkload:
    """Tiny prefill half: T=2048, 4 q / 2 KV heads, D=64, 64x64 blocks."""
    return prefill_workload(2048, 4, 2, 64, 64, 1001, name="tiny")


def prefill_128k() -> PrefillWorkload:
    """Block-sparse prefill: T=128K, 32 q / 8 KV heads, D=128, 128x128 blocks;
    KV heads 0-3 dense causal, 4-7 Lambda (1 sink + 4 local blocks)."""
    return prefill_workload(131072, 32, 8, 128, 128, 1004, name="prefill_128k")


DECODE_CONFIGS = {
    "tiny": tiny_decode,
    "llama3_8b_decode": llama3_8b_decode,
    "long_decode_256k": long_decode_256k,
    "mixed_batch_decode": mixed_batch_decode,
    "llama2_7b_mha_decode": llama2_7b_mha_decode,
}
PREFILL_CONFIGS = {"tiny": tiny_prefill, "prefill_128k": prefill_128k}
