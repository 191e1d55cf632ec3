"""Benchmark of the LServe-style sparse attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Workload (synthetic, seeded): the Llama-3-8B-shaped decode layer -- batch 4,
64K context, 32 query / 8 KV heads, D=128, bf16 paged KV (N_L=16, N_P=64),
half the KV heads streaming (sink 128 + local 512), top-64 physical pages for
the retrieval heads, selection reused over 4 decode steps.  The layer is
replicated over 32 layers (Llama-3-8B depth), each with its own KV / stats /
selection buffers, so one step streams ~1.5 GB -- far more than the 126 MB L2.

A step is one decode token through the 32 layers: every 4th step runs
page selection (lserve_page_select) before attention in each layer, the
others reuse it; every step runs lserve_sparse_decode_attn per layer.  Steps
are replayed from two CUDA graphs (with / without selection).

Reported (one JSON line, rank 0):
  value      touched-HBM GB/s of the decode steps, summed over ranks
  us_per_layer_step, ms_per_step
  stages     each call timed alone: selection, attention, the full stats
             build, and the block-sparse prefill TFLOP/s on the 128K workload
  roofline   for the dominant call (decode attention) against the measured
             HBM copy bandwidth
  e2e        the same step with the step's q copied host->device and the
             output read back device->host inside the timed region
  cpu_baseline  the fp64 oracle on a bounded sample of the same step
Multi-GPU (torchrun): every rank runs its own replica (weak scaling, no
collective on the data path); time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

LAYERS = 32
REUSE = 4
DEFAULT_STEPS = 6000          # GPU arm: 32-layer steps
DEFAULT_REF_STEPS = 200      # reference arm: layer-steps of the oracle (~20 s on one core)
DEFAULT_WARMUP = 8
METRIC = "sparse decode attn µs/step & HBM GB/s; block-sparse prefill TFLOP/s"


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p.get("bf16_tflops_sustained",
                                                                        p["bf16_tflops"])), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# --- algorithmic byte / flop accounting (what the chosen sparsity touches) ----
# Plain counting of the pages and blocks the method touches (the reading the
# kernels implement), kept here so that the measurement legs run nothing of
# the oracle; tests/test_bench_accounting.py checks these counts against it.

def stream_pages(n, NP, sink, local):
    """Pages a streaming head attends at length n: the sink pages
    [0, ceil(sink / N_P)) and every page holding one of the last `local` tokens."""
    if n <= 0:
        return []
    npages = -(-n // NP)
    ns = min(-(-sink // NP), npages)
    ls = max(max(0, n - local) // NP, ns)
    return list(range(ns)) + list(range(ls, npages))


def valid_tokens(pages, n, NP):
    """Tokens of the given pages that lie below length n."""
    return sum(max(0, min(NP, n - m * NP)) for m in pages)


def prefill_flops(T, H_q, H_kv, D, block, head_kind, sink_blocks, local_blocks):
    """Work counted as the pages count it: full block tiles (two matmuls of
    2*block*block*D flops each) per query head; a retrieval KV head's rows
    visit blocks 0..i, a streaming head's the sink blocks and the local
    window [i - local + 1, i]."""
    nb = -(-T // block)
    G = H_q // H_kv
    tiles = 0
    for h in range(H_kv):
        if int(head_kind[h]) == 0:
            cnt = nb * (nb + 1) // 2
        else:
            cnt = 0
            for i in range(nb):
                s_hi = min(sink_blocks, i + 1)   # sink blocks [0, s_hi)
                l_lo = max(0, i - local_blocks + 1)  # local blocks [l_lo, i]
                cnt += s_hi + (i - l_lo + 1) - max(0, s_hi - l_lo)
        tiles += G * cnt
    return tiles * 4.0 * block * block * D


def decode_bytes(w, fused_append=False):
    """Bytes one decode step of one layer must move, amortising selection over
    the reuse interval.  KV: valid tokens of the attended pages, K and V, D*2
    bytes each.  Selection: the stats of every valid logical page of the
    retrieval heads (2*D*2 bytes), the q vectors, scores and selection.  With
    fused_append the attention launch also appends the step's token (its K / V
    rows and the statistics it updates, append_bytes)."""
    D, NP, NL = w.D, w.N_P, w.N_L
    kv = 0
    stats = 0
    for b in range(w.B):
        n = int(w.ctx_lens[b])
        npages = -(-n // NP)
        for h in range(w.H_kv):
            if w.head_kind[h] == 0:
                # top-K pages; the count of valid tokens depends only on whether the
                # partial last page is selected -- bound it by full pages
                k = min(w.top_k, npages)
                kv += k * NP * D * 2 * 2
                stats += (-(-n // NL)) * 2 * D * 2
            else:
                toks = valid_tokens(stream_pages(n, NP, w.sink, w.local), n, NP)
                kv += toks * D * 2 * 2
    q = w.B * w.H_q * D * 2
    out = w.B * w.H_q * D * 2
    sel_io = q + w.B * w.H_kv * (w.max_pages * 4 + w.top_k * 4 + 4)
    attn = kv + q + out + (append_bytes(w) if fused_append else 0)
    select = stats + sel_io
    return dict(attn=attn, select=select, step=attn + select / REUSE, kv=kv, stats=stats)


def decode_bytes_kv8(w, bits=8):
    """Bytes one decode-attention call over the quantized cache moves: the
    codes of the attended pages (K and V, D * bits / 8 bytes per token each),
    the two float32 channel-scale rows of every attended (page, head), q and
    the output."""
    D, NP = w.D, w.N_P
    kv = 0
    for b in range(w.B):
        n = int(w.ctx_lens[b])
        npages = -(-n // NP)
        for h in range(w.H_kv):
            if w.head_kind[h] == 0:
                k = min(w.top_k, npages)
                kv += k * NP * D * bits // 8 * 2 + k * 2 * D * 4
            else:
                pages = stream_pages(n, NP, w.sink, w.local)
                toks = valid_tokens(pages, n, NP)
                kv += toks * D * bits // 8 * 2 + len(pages) * 2 * D * 4
    return kv + 2 * w.B * w.H_q * D * 2


def quantize_bytes(w, bits=8):
    """lserve_quantize_pages_kv8 / _kv4: read the valid bf16 K/V rows of every
    page, write the codes (whole pages) and the float32 scales."""
    rd = wr = 0
    for b in range(w.B):
        n = int(w.ctx_lens[b])
        npages = -(-n // w.N_P)
        rd += 2 * n * w.H_kv * w.D * 2
        wr += 2 * npages * w.H_kv * (w.N_P * w.D * bits // 8 + w.D * 4)
    return rd + wr


def stats_build_bytes(w):
    """lserve_page_stats full build: read K of the retrieval heads, write stats."""
    rd = wr = 0
    for b in range(w.B):
        n = int(w.ctx_lens[b])
        for h in range(w.H_kv):
            if w.head_kind[h] == 0:
                rd += n * w.D * 2
                wr += (-(-n // w.N_L)) * 2 * w.D * 2
    return rd + wr


def kernel_traffic(kernel):
    """DRAM bytes (read + write) per launch of `kernel` from the committed ncu
    record (profiles/traffic.json), provided the kernel's source file still
    hashes to the one the counters were taken on; otherwise None."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f)[kernel]
        with open(os.path.join(ROOT, rec["source"]), "rb") as f:
            digest = hashlib.sha256(f.read()).hexdigest()
        if rec["source_sha256"] != digest:
            return None
        return float(rec["traffic_bytes_per_launch"])
    except (OSError, KeyError, ValueError, TypeError):
        return None


def append_bytes(w):
    """lserve_decode_append: read k_new / v_new and write one K and V row per
    (sequence, KV head); read + write the two statistics rows of the retrieval
    heads' current logical page."""
    rows = w.B * w.H_kv * w.D * 2
    retrieval = int(sum(1 for h in range(w.H_kv) if w.head_kind[h] == 0)) * w.B
    return 2 * 2 * rows + retrieval * 2 * w.D * 2 * 2


# --- clocks sampling ----------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index, uuid=None):
        if uuid is not None:
            uuid = str(uuid)
            uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        self.sel = ["-i", uuid] if uuid else ["-i", str(device_index)]
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "200"] + self.sel,
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = []
        for line in out.strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append(dict(sm=float(parts[1]), smax=float(parts[2]), power=float(parts[3]),
                                 hw=parts[5], hwt=parts[6], swt=parts[7], swp=parts[8]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        sm = np.array([r["sm"] for r in rows])
        reasons = set()
        for r in rows:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("swp", "sw_power_cap")):
                if r[key].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(rows[0]["smax"]),
                "reasons": sorted(reasons), "samples": len(rows),
                "power_w_max": float(max(r["power"] for r in rows))}


# --- distributed plumbing -------------------------------------------------------

def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(x, ws, device):
    if ws == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(bytes_per_rank_step, steps, ws, elapsed_max_s):
    """Weak scaling: every rank streams its own replica; the job's throughput is
    the bytes all ranks moved over the slowest rank's time (GB/s)."""
    return bytes_per_rank_step * steps * ws / elapsed_max_s / 1e9


# --- the CPU oracle baseline ----------------------------------------------------

def host_cpu():
    """The host's CPU model and core counts."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    try:
        usable = len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        usable = os.cpu_count()
    return {"model": model, "nproc": os.cpu_count(), "usable_cores": usable}


class OraclePair:
    """One (sequence, KV head) of the decode workload in the oracle's hands:
    q, K and V widened to float64, and for a retrieval head its page statistics
    (built once beforehand, as the GPU builds them once after the prefill).
    visit() is what one decode step costs this pair: the page selection
    (S^j -> P^m -> top-K) when `select` is set, and the attention over the
    attended pages -- the gather of their tokens included."""

    def __init__(self, w, b, h):
        import oracle
        G = w.G
        self.w, self.kind = w, int(w.head_kind[h])
        self.n = int(w.ctx_lens[b])
        self.q = oracle.widen_bf16(w.q[b, h * G:(h + 1) * G])
        self.k = oracle.widen_bf16(w.k_seq(b, h))
        self.v = oracle.widen_bf16(w.v_seq(b, h))
        self.stats = oracle.page_stats(self.k, w.N_L) if self.kind == 0 else None
        self.pages = None
        self.scale = 1.0 / math.sqrt(w.D)

    def visit(self, select):
        import oracle
        w = self.w
        if self.kind == 0:
            if select or self.pages is None:
                P = oracle.physical_scores(oracle.logical_scores(self.q, *self.stats), w.g)
                self.pages = oracle.select_top_k(P, w.top_k)
            pages = self.pages
        else:
            pages = oracle.streaming_pages(self.n, w.N_P, w.sink, w.local)
        oracle.decode_attention(self.q, self.k, self.v, oracle.page_tokens(pages, self.n, w.N_P),
                                self.scale)


def _one_thread():
    """Limit BLAS / OpenMP pools of this process to one thread."""
    try:
        from threadpoolctl import threadpool_limits
        return threadpool_limits(1)
    except Exception:
        return None


def oracle_layer_steps(pairs, t0, steps):
    """Run layer-steps t0 .. t0 + steps - 1 over the given pairs (selection on
    every REUSE-th step, as the GPU step reuses it); returns seconds."""
    start = time.perf_counter()
    for t in range(t0, t0 + steps):
        for pr in pairs:
            pr.visit(t % REUSE == 0)
    return time.perf_counter() - start


def oracle_single_thread(w, budget_s=8.0):
    """The oracle's decode step on one thread: whole layer-steps (all pairs),
    as many complete reuse windows as fit the budget.  Returns (s / layer-step,
    layer-steps timed)."""
    lim = _one_thread()
    pairs = [OraclePair(w, b, h) for b in range(w.B) for h in range(w.H_kv)]
    oracle_layer_steps(pairs, 0, 1)           # warm-up (selection made)
    steps, elapsed = 0, 0.0
    while elapsed < budget_s or steps < REUSE:
        elapsed += oracle_layer_steps(pairs, REUSE + steps, REUSE)
        steps += REUSE
    del lim
    return elapsed / steps, steps


def _bundles(w):
    """The workload's (sequence, KV head) pairs grouped into bundles of equal
    cost: a retrieval pair with a streaming pair (their visits cost ~10:1)."""
    P = w.B * w.H_kv
    retr = [p for p in range(P) if w.head_kind[p % w.H_kv] == 0]
    strm = [p for p in range(P) if w.head_kind[p % w.H_kv] != 0]
    out = [list(x) for x in zip(retr, strm)]
    rest = retr[len(out):] + strm[len(out):]
    return out + [[p] for p in rest]


def _oracle_worker(args):
    """One process of the all-core run (spawned): builds its bundles of pairs,
    waits for the others, then runs layer-steps [s0, s1) over them."""
    bundle_ids, s0, s1, barrier = args
    lim = _one_thread()
    import synth
    w = synth.llama3_8b_decode()
    bundles = _bundles(w)
    pairs = [OraclePair(w, p // w.H_kv, p % w.H_kv) for i in bundle_ids for p in bundles[i]]
    oracle_layer_steps(pairs, 0, 1)
    barrier.wait()
    elapsed = oracle_layer_steps(pairs, s0, s1 - s0)
    del lim
    return elapsed


def oracle_all_cores(w, t_single, budget_s=6.0):
    """The oracle's decode step on the host's cores: one spawned process per
    core, each holding whole bundles (a retrieval + a streaming pair).  With W
    processes and nb bundles: W <= nb -> a process takes the bundles i with
    i mod W = its index, for every layer-step; W = R * nb -> a process takes
    one bundle and a contiguous 1/R of the layer-steps.  Every process starts
    at a barrier; the S layer-steps take the slowest process's time.
    t_single (s per layer-step on one thread) sizes S to about budget_s.
    Returns (s / layer-step, processes, layer-steps)."""
    import multiprocessing as mp
    nb = len(_bundles(w))
    cores = host_cpu()["usable_cores"] or 1
    if cores >= nb:
        R = cores // nb
        nw = nb * R
    else:
        R, nw = 1, 1
        while nw * 2 <= cores and nb % (nw * 2) == 0:
            nw *= 2
    per = max(REUSE, int(budget_s * nw / t_single / R) // REUSE * REUSE)  # steps per process
    S = per * R
    tasks = []
    for i in range(nw):
        if R == 1:
            tasks.append(([b for b in range(nb) if b % nw == i], REUSE, REUSE + S))
        else:
            rep = i // nb
            tasks.append(([i % nb], REUSE + rep * per, REUSE + (rep + 1) * per))
    env_keys = ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")
    saved = {k: os.environ.get(k) for k in env_keys}
    for k in env_keys:
        os.environ[k] = "1"
    try:
        ctx = mp.get_context("spawn")
        mgr = ctx.Manager()
        barrier = mgr.Barrier(nw)
        with ctx.Pool(nw) as pool:
            res = pool.map(_oracle_worker, [t + (barrier,) for t in tasks], chunksize=1)
        mgr.shutdown()
    finally:
        for k, v in saved.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v
    return max(res) / S, nw, S


def oracle_prefill_sample(threads_one=True, budget_rows=64):
    """The oracle's block-sparse prefill on a bounded sample of the 128K
    workload: two dense and two Lambda query heads, per head two full query
    blocks (one early, one late) and `budget_rows` random rows.  The time of the
    whole workload is extrapolated from it by the number of (row, key) pairs
    each head kind computes.  Returns (extrapolated s, sample description)."""
    import oracle
    import synth
    lim = _one_thread() if threads_one else None
    w = synth.prefill_128k()
    K, V = oracle.widen_bf16(w.k()), oracle.widen_bf16(w.v())
    nb = -(-w.T // w.block)
    scale = 1.0 / math.sqrt(w.D)
    rng = np.random.default_rng(7)

    def keys_of(kind, rows):
        """(row, key) pairs the rows compute: keys s <= t of the blocks row t sees."""
        t = np.asarray(rows, dtype=np.float64)
        if kind == 0:
            return float(np.sum(t + 1))
        i = np.floor(t / w.block)
        sink_end = np.minimum(w.sink_blocks, i + 1) * w.block
        local_start = np.maximum(np.maximum(0, i - w.local_blocks + 1) * w.block, sink_end)
        return float(np.sum(np.minimum(sink_end, t + 1) + np.maximum(0, t + 1 - local_start)))

    t_kind, keys_kind = {0: 0.0, 1: 0.0}, {0: 0.0, 1: 0.0}
    heads = [hq for hq in range(w.H_q) if w.head_kind[hq // w.G] == 0][:2] + \
            [hq for hq in range(w.H_q) if w.head_kind[hq // w.G] == 1][:2]
    for hq in heads:
        hk, kind = hq // w.G, int(w.head_kind[hq // w.G])
        kh, vh = np.ascontiguousarray(K[:, hk]), np.ascontiguousarray(V[:, hk])
        groups = {}
        for i in (int(rng.integers(2, nb // 4)), int(rng.integers(3 * nb // 4, nb))):
            groups[i] = list(range(i * w.block, min((i + 1) * w.block, w.T)))
        for t in rng.choice(w.T, budget_rows, replace=False):
            groups.setdefault(int(t) // w.block, []).append(int(t))
        for i, rows in groups.items():
            rows = np.asarray(sorted(set(rows)))
            qb = oracle.widen_bf16(w.q_rows(int(rows[0]), int(rows[-1]) + 1))[rows - rows[0], hq]
            t0 = time.perf_counter()
            oracle.prefill_block_rows(qb, kh, vh, kind, w.block, w.sink_blocks, w.local_blocks,
                                      scale, rows)
            t_kind[kind] += time.perf_counter() - t0
            keys_kind[kind] += keys_of(kind, rows)
    del lim
    all_rows = np.arange(w.T)
    n_heads = {kind: sum(1 for hq in range(w.H_q) if w.head_kind[hq // w.G] == kind)
               for kind in (0, 1)}
    total = sum(t_kind[k] / keys_kind[k] * keys_of(k, all_rows) * n_heads[k] for k in (0, 1))
    sampled = sum(t_kind.values())
    return total, (f"extrapolated: 2 dense + 2 Lambda query heads x (2 full query blocks + "
                   f"{budget_rows} random rows) timed ({sampled:.1f} s), scaled to all "
                   f"{w.H_q} heads x {w.T} rows by the (row, key) pairs of each head kind")


def cpu_baseline(w, acct, tc_flops=None):
    """The fp64 oracle timed on this host: the decode step on one thread and on
    every core, and the prefill (extrapolated from a sample)."""
    host = host_cpu()
    t1, steps1 = oracle_single_thread(w)
    tn, nw, S = oracle_all_cores(w, t1)
    res = {"value": acct["step"] / tn / 1e9, "unit": "GB/s", "cores": nw, "kind": "oracle",
           "sample": f"{S} layer-steps of the bench workload (all {w.B * w.H_kv} pairs, selection "
                     f"every {REUSE}th step) over {nw} processes of one thread each, started "
                     f"together; the slowest process's time",
           "host": host,
           "single_thread": {"value": acct["step"] / t1 / 1e9, "unit": "GB/s", "cores": 1,
                             "us_per_layer_step": t1 * 1e6,
                             "sample": f"{steps1} whole layer-steps on one thread"},
           "us_per_layer_step": tn * 1e6}
    if tc_flops is not None:
        tp1, s1 = oracle_prefill_sample(True)
        tpn, _ = oracle_prefill_sample(False)
        res["prefill"] = {"single_thread": {"TFLOP/s": tc_flops / tp1 / 1e12, "s": tp1, "cores": 1},
                          "all_cores_blas": {"TFLOP/s": tc_flops / tpn / 1e12, "s": tpn,
                                             "cores": host["usable_cores"]},
                          "sample": s1}
    return res


def reference_steps(w, steps, warmup):
    """The oracle as timed steps of the reference arm: a step is one whole
    layer-step of the workload -- every (sequence, KV head) pair: its page
    selection on every REUSE-th step (as the GPU step reuses it) and its
    attention over the attended pages, their tokens gathered inside the step.
    The bf16 inputs are widened and the page statistics built once (as on the
    GPU), untimed; one thread.  Returns (seconds of the K timed steps, sample)."""
    lim = _one_thread()
    pairs = [OraclePair(w, b, h) for b in range(w.B) for h in range(w.H_kv)]
    oracle_layer_steps(pairs, 0, warmup)
    elapsed = oracle_layer_steps(pairs, warmup, steps)
    del lim
    nsel = sum(1 for t in range(warmup, warmup + steps) if t % REUSE == 0)
    return elapsed, (f"each step one whole layer-step ({len(pairs)} pairs; selection on {nsel} of "
                     f"the {steps} timed steps, every {REUSE}th), 1 thread")


def reference_arm(args):
    """The oracle as the reference arm: same metric / unit / config; a step is
    one layer of the GPU arm's 32-layer step."""
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    import synth
    w = synth.llama3_8b_decode()
    acct = decode_bytes(w)
    elapsed, sample = reference_steps(w, args.steps, args.warmup)
    per_layer_step = elapsed / args.steps
    value = acct["step"] / per_layer_step / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_layer_step * 1e3,
        "step": "one layer-step of the workload (the GPU arm's step is 32 of them)",
        "us_per_layer_step": per_layer_step * 1e6, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w),
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": sample + f"; {elapsed:.2f} s for {args.steps} steps",
                         "host": host_cpu()},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


def workload_config(w):
    return {"workload": f"{w.name}: B={w.B} n={int(w.ctx_lens[0])} H_q={w.H_q} H_kv={w.H_kv} D={w.D} "
                        f"N_L={w.N_L} N_P={w.N_P} top_k={w.top_k} sink={w.sink} local={w.local} "
                        f"reuse={REUSE}",
            "layers": LAYERS, "global_batch": w.B, "seq_len": int(w.ctx_lens[0]),
            "parallelism": "replica per GPU",
            "l2": f"inputs larger than L2: {LAYERS} layer replicas, each step streams all of them"}


# --- the CUDA path ----------------------------------------------------------------

def main():
    global LAYERS
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=DEFAULT_WARMUP)
    ap.add_argument("--impl", default="lserve", choices=["lserve", "reference"])
    ap.add_argument("--no-prefill", action="store_true", help="skip the prefill stage")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--layers", type=int, default=LAYERS,
                    help="layer replicas (fewer = a small case for profiling; < 32 may fit in L2)")
    ap.add_argument("--no-mha", action="store_true", help="skip the MHA decode stage")
    ap.add_argument("--no-kv8", action="store_true", help="skip the quantized-cache (8- and 4-bit) decode stages")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the long-decode and mixed-batch decode stages")
    ap.add_argument("--prefill-only", action="store_true",
                    help="run only the prefill stage (profiling)")
    ap.add_argument("--prefill-seq", type=int, default=None,
                    help="prefill sequence length (default: the 128K workload)")
    ap.add_argument("--profile", default=None,
                    help="set up one workload and launch one decode call --steps times, then exit "
                         "(a small case for ncu): WORKLOAD:CACHE with WORKLOAD in "
                         "8b|mha|256k|mixed and CACHE in bf16|kv8|kv4")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    if args.steps is None:
        args.steps = DEFAULT_REF_STEPS if args.impl == "reference" else DEFAULT_STEPS
    LAYERS = max(1, args.layers)
    if args.impl == "reference":
        return reference_arm(args)

    import torch
    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    import block_sparse_attention_page_b200 as lserve
    import synth
    from synth.device import DecodeBuffers

    hbm_peak, tc_peak, tc_sustained, peak_src = peaks()
    if args.profile:
        return profile_case(lserve, synth, dev, args.profile, args.steps)
    if args.prefill_only:
        res = prefill_stage(lserve, synth, dev, torch.cuda.Stream(device=dev), tc_peak, None,
                            args.prefill_seq)
        if rank == 0:
            print(json.dumps({"prefill": res}))
        return 0
    w = synth.llama3_8b_decode()
    buf = DecodeBuffers(w, device=dev, layers=LAYERS)
    d = lserve.paged_desc(w.B, w.H_q, w.H_kv, w.D, w.N_L, w.N_P, w.max_pages, w.num_pool_pages)
    scale = 1.0 / math.sqrt(w.D)
    ws_dec = lserve.alloc_workspace(lserve.workspace_size(lserve.OP_DECODE, d, w.top_k), device=dev)
    ws_sel = lserve.alloc_workspace(lserve.workspace_size(lserve.OP_SELECT, d, w.top_k), device=dev)
    # every layer's q and output are slices of one tensor each, so that a step's
    # inputs and results cross the host link as one copy each (e2e below)
    q_all = buf.q.unsqueeze(0).repeat(LAYERS, 1, 1, 1).contiguous()
    out_all = torch.empty((LAYERS,) + tuple(buf.out.shape), dtype=buf.out.dtype, device=dev)
    qs = [q_all[l] for l in range(LAYERS)]
    outs = [out_all[l] for l in range(LAYERS)]
    stream = torch.cuda.Stream(device=dev)
    acct = decode_bytes(w, fused_append=True)

    def stats_all():
        for l in range(LAYERS):
            lserve.page_stats(d, buf.k_pools[l], buf.block_table, buf.ctx_lens, buf.head_kind,
                              buf.stats[l])

    def select(l):
        lserve.page_select(d, qs[l], buf.stats[l], buf.block_table, buf.ctx_lens, buf.head_kind,
                           w.top_k, buf.sel[l], buf.sel_count[l], workspace=ws_sel)

    # The step's new token of every sequence is appended in the attention launch
    # (lserve_decode_step).  So that every step sees the same cache, the token
    # appended is each sequence's last one again, with its own K / V (position
    # n - 1, ctx_lens unchanged): the pools and statistics keep their contents.
    last = [(int(w.block_table[b, (int(w.ctx_lens[b]) - 1) // w.N_P]),
             (int(w.ctx_lens[b]) - 1) % w.N_P) for b in range(w.B)]
    k_last = [torch.stack([buf.k_pools[l][pid, :, r] for pid, r in last]).contiguous()
              for l in range(LAYERS)]
    v_last = [torch.stack([buf.v_pools[l][pid, :, r] for pid, r in last]).contiguous()
              for l in range(LAYERS)]

    def attn(l, overlap=False):
        # overlap: the kernel before this call is the previous layer's attention,
        # which writes none of the selection / block-table inputs nor this
        # layer's pools, so the split plan, the first page lookups and the first
        # tiles' copies may start while it finishes (PDL)
        lserve.decode_step(d, qs[l], k_last[l], v_last[l], buf.k_pools[l], buf.v_pools[l],
                           buf.stats[l], buf.block_table, buf.ctx_lens, buf.head_kind, buf.sel[l],
                           buf.sel_count[l], w.top_k, w.sink, w.local, scale, outs[l], None,
                           workspace=ws_dec, overlap_prologue=overlap, prefetch_kv=overlap)

    with torch.cuda.stream(stream):
        stats_all()
        for l in range(LAYERS):
            select(l)
            attn(l)
    torch.cuda.synchronize()
    assert lserve.read_device_status(stream) == lserve.OK

    def capture(fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            fn()
        return g

    g_sel = capture(lambda: [(select(l), attn(l)) for l in range(LAYERS)])
    g_reuse = capture(lambda: [attn(l, overlap=l > 0) for l in range(LAYERS)])
    g_select_only = capture(lambda: [select(l) for l in range(LAYERS)])
    g_stats = capture(stats_all)

    # the same cache maintenance as a launch of its own (lserve_decode_append),
    # timed alone for comparison
    lens_last = (buf.ctx_lens - 1).to(torch.int32)

    def append_all():
        for l in range(LAYERS):
            lserve.decode_append(d, k_last[l], v_last[l], buf.block_table, lens_last, buf.head_kind,
                                 buf.k_pools[l], buf.v_pools[l], buf.stats[l])
    with torch.cuda.stream(stream):
        append_all()
    torch.cuda.synchronize()
    assert lserve.read_device_status(stream) == lserve.OK
    g_append = capture(append_all)

    def run_steps(k0, k, ev=None):
        # ev: event pairs recorded around the attention-only replays, so that the
        # average attention launch is measured inside the timed region itself
        for t in range(k0, k0 + k):
            if t % REUSE == 0:
                g_sel.replay()
            elif ev is not None and t < len(ev):
                ev[t][0].record(stream)
                g_reuse.replay()
                ev[t][1].record(stream)
            else:
                g_reuse.replay()

    def timed(fn, reps=1):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        if ws > 1:
            torch.distributed.barrier()
        e0.record(stream)
        with torch.cuda.stream(stream):
            for _ in range(reps):
                fn()
        e1.record(stream)
        torch.cuda.synchronize()
        if ws > 1:
            torch.distributed.barrier()
        return e0.elapsed_time(e1) / 1e3

    # warm-up (untimed), then exactly K steps
    with torch.cuda.stream(stream):
        run_steps(0, args.warmup)
    torch.cuda.synchronize()
    sampler = ClockSampler(local, getattr(torch.cuda.get_device_properties(dev), "uuid", None))
    sampler.start() if rank == 0 else None
    time.sleep(0.3)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          if t % REUSE else None for t in range(args.steps)]
    elapsed = timed(lambda: run_steps(0, args.steps, ev))
    clocks = sampler.stop() if rank == 0 else None
    attn_in_region = [a.elapsed_time(b) / 1e3 for t, (a, b) in enumerate(e for e in ev if e)]
    t_attn_region = float(np.mean(attn_in_region)) / LAYERS if attn_in_region else None
    elapsed = max_over_ranks(elapsed, ws, dev)
    step_bytes = acct["step"] * LAYERS
    value = whole_job_value(step_bytes, args.steps, ws, elapsed)
    us_layer = elapsed / (args.steps * LAYERS) * 1e6

    # stages, each alone (graph replays, CUDA events on the launching stream)
    reps = 20
    t_attn = timed(lambda: g_reuse.replay(), reps) / (reps * LAYERS)
    if t_attn_region is not None:
        t_attn = t_attn_region  # the launches of the timed region themselves
    t_sel = timed(lambda: g_select_only.replay(), reps) / (reps * LAYERS)
    t_stats = timed(lambda: g_stats.replay(), 3) / (3 * LAYERS)
    t_app = timed(lambda: g_append.replay(), reps) / (reps * LAYERS)
    app_bytes = append_bytes(w)
    sb = stats_build_bytes(w)
    attn_gbs = acct["attn"] / t_attn / 1e9
    stages = {
        "attention": {"us": t_attn * 1e6, "GB/s": attn_gbs, "frac": attn_gbs / hbm_peak,
                      "bytes": acct["attn"]},
        "selection": {"us": t_sel * 1e6, "GB/s": acct["select"] / t_sel / 1e9,
                      "frac": acct["select"] / t_sel / 1e9 / hbm_peak, "bytes": acct["select"]},
        "stats_build": {"us": t_stats * 1e6, "GB/s": sb / t_stats / 1e9,
                        "frac": sb / t_stats / 1e9 / hbm_peak, "bytes": sb},
        "append": {"us": t_app * 1e6, "GB/s": app_bytes / t_app / 1e9, "bytes": app_bytes,
                   "note": "lserve_decode_append as a launch of its own, per layer (the bench's "
                           "step appends inside the attention launch, lserve_decode_step); "
                           "launch-latency bound (48 KB)"},
    }
    del g_stats, g_append

    # e2e: per step, copy the step's q (all layers, one pinned buffer) host->device
    # straight into the layers' q slices, run the step, read every layer's output
    # back to pinned host memory in one copy
    q_host = torch.empty(tuple(q_all.shape), dtype=torch.bfloat16).pin_memory()
    o_host = torch.empty(tuple(out_all.shape), dtype=torch.bfloat16).pin_memory()
    q_host.copy_(q_all.cpu())

    def e2e_step(t):
        q_all.copy_(q_host, non_blocking=True)
        (g_sel if t % REUSE == 0 else g_reuse).replay()
        o_host.copy_(out_all, non_blocking=True)

    e2e_steps = min(args.steps, 400)
    e2e = None
    if not args.no_e2e:
        with torch.cuda.stream(stream):
            for t in range(args.warmup):
                e2e_step(t)
        t_e2e = timed(lambda: [e2e_step(t) for t in range(e2e_steps)])
        t_e2e = max_over_ranks(t_e2e, ws, dev)
        h2d = q_host.numel() * 2
        d2h = o_host.numel() * 2
        e2e = {"value": whole_job_value(step_bytes, e2e_steps, ws, t_e2e), "unit": "GB/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": t_e2e / e2e_steps * 1e3}

    # one kernel per attention call, two per selection call (scores, top-K)
    launches = args.steps * LAYERS + (-(-args.steps // REUSE)) * LAYERS * 2
    result = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": elapsed / args.steps * 1e3,
        "us_per_layer_step": us_layer, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(w),
        "roofline": {"bound": "hbm", "kernel": "decode_attn_kernel (lserve_sparse_decode_attn)",
                     "achieved": attn_gbs, "peak": hbm_peak, "unit": "GB/s",
                     "frac": attn_gbs / hbm_peak, "traffic": kernel_traffic("decode_attn"),
                     "algorithmic_bytes": acct["attn"],
                     "peak_source": f"{peak_src} hbm_gbs (copy, burst); of {peak_src}",
                     "timing": "mean attention launch inside the timed region (CUDA events "
                               "around the attention-only graph replays)"},
        "stages": stages,
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clocks,
    }
    del g_sel, g_reuse, g_select_only
    buf = None
    torch.cuda.empty_cache()

    if not args.no_mha:
        result["stages"]["attention_mha"] = mha_stage(lserve, synth, dev, stream, hbm_peak, timed)
    if not args.no_configs:
        result["stages"]["long_decode_256k"] = decode_config_stage(
            lserve, synth, dev, stream, hbm_peak, timed, synth.long_decode_256k, 16,
            shards=4 if ws == 1 else 1)
        if ws > 1:  # the 256K sequence split over the ranks, NCCL exchanges timed
            result["stages"]["long_decode_256k_seq_sharded"] = seqshard_stage(
                lserve, synth, dev, stream, hbm_peak, timed, rank, ws, args.warmup)
        result["stages"]["mixed_batch_decode"] = decode_config_stage(
            lserve, synth, dev, stream, hbm_peak, timed, synth.mixed_batch_decode, 3)
    if not args.no_kv8:
        for bits in (8, 4):
            result["stages"][f"attention_kv{bits}"] = kv8_stage(
                lserve, synth, dev, stream, hbm_peak, timed, synth.llama3_8b_decode, 16,
                stages["attention"]["us"], bits)
            if not args.no_mha:
                result["stages"][f"attention_mha_kv{bits}"] = kv8_stage(
                    lserve, synth, dev, stream, hbm_peak, timed, synth.llama2_7b_mha_decode, 8,
                    result["stages"]["attention_mha"]["us"], bits)
    if not args.no_prefill:
        result["stages"]["prefill"] = prefill_stage(lserve, synth, dev, stream, tc_peak, timed,
                                                    args.prefill_seq)

    if rank == 0 and ws == 1 and not args.no_cpu_baseline:  # the oracle baseline: one GPU runs only
        pf = result["stages"].get("prefill", {}).get("flops")
        # the oracle's step attends without appending: its bytes leave the append out
        result["cpu_baseline"] = cpu_baseline(w, decode_bytes(w), pf)
    if rank == 0:
        print(json.dumps(result))
    if ws > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return 0


def mha_stage(lserve, synth, dev, stream, hbm_peak, timed, layers=8):
    """Decode attention on the Llama-2-7B-shaped MHA layer (G = 1), alone:
    `layers` replicas back to back (each touches ~155 MB, more than L2)."""
    import torch
    from synth.device import DecodeBuffers
    w = synth.llama2_7b_mha_decode()
    buf = DecodeBuffers(w, device=dev, layers=layers)
    d = lserve.paged_desc(w.B, w.H_q, w.H_kv, w.D, w.N_L, w.N_P, w.max_pages, w.num_pool_pages)
    wss = lserve.alloc_workspace(lserve.workspace_size(lserve.OP_SELECT, d, w.top_k), device=dev)
    wsd = lserve.alloc_workspace(lserve.workspace_size(lserve.OP_DECODE, d, w.top_k), device=dev)
    outs = [torch.empty_like(buf.out) for _ in range(layers)]
    scale = 1.0 / math.sqrt(w.D)
    with torch.cuda.stream(stream):
        for l in range(layers):
            lserve.page_stats(d, buf.k_pools[l], buf.block_table, buf.ctx_lens, buf.head_kind,
                              buf.stats[l])
            lserve.page_select(d, buf.q, buf.stats[l], buf.block_table, buf.ctx_lens, buf.head_kind,
                               w.top_k, buf.sel[l], buf.sel_count[l], workspace=wss)
    torch.cuda.synchronize()

    def attn_all():
        for l in range(layers):
            lserve.sparse_decode_attn(d, buf.q, buf.k_pools[l], buf.v_pools[l], buf.block_table,
                                      buf.ctx_lens, buf.head_kind, buf.sel[l], buf.sel_count[l],
                                      w.top_k, w.sink, w.local, scale, outs[l], None, workspace=wsd,
                                      overlap_prologue=l > 0, prefetch_kv=l > 0)
    with torch.cuda.stream(stream):
        attn_all()
    torch.cuda.synchronize()
    assert lserve.read_device_status(stream) == lserve.OK
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        attn_all()
    with torch.cuda.stream(stream):
        for _ in range(3):
            g.replay()
    reps = 20
    t = timed(lambda: g.replay(), reps) / (reps * layers)
    bts = decode_bytes(w)["attn"]
    del g
    return {"us": t * 1e6, "GB/s": bts / t / 1e9, "frac": bts / t / 1e9 / hbm_peak, "bytes": bts,
            "workload": f"{w.name}: B={w.B} n={int(w.ctx_lens[0])} H_q={w.H_q} H_kv={w.H_kv} "
                        f"D={w.D} N_L={w.N_L} N_P={w.N_P} top_k={w.top_k} sink={w.sink} "
                        f"local={w.local}"}


def decode_config_stage(lserve, synth, dev, stream, hbm_peak, timed, make, layers, shards=1):
    """Selection and decode attention of another decode workload, each timed
    alone: `layers` replicas of its KV / stats / selection (together more bytes
    than L2 holds), graph replays, attention launched as in the main step."""
    import torch
    from synth.device import DecodeBuffers
    w = make()
    buf = DecodeBuffers(w, device=dev, layers=layers)
    d = lserve.paged_desc(w.B, w.H_q, w.H_kv, w.D, w.N_L, w.N_P, w.max_pages, w.num_pool_pages)
    wss = lserve.alloc_workspace(lserve.workspace_size(lserve.OP_SELECT, d, w.top_k), device=dev)
    wsd = lserve.alloc_workspace(lserve.workspace_size(lserve.OP_DECODE, d, w.top_k), device=dev)
    outs = [torch.empty_like(buf.out) for _ in range(layers)]
    scale = 1.0 / math.sqrt(w.D)

    def select_all():
        for l in range(layers):
            lserve.page_select(d, buf.q, buf.stats[l], buf.block_table, buf.ctx_lens, buf.head_kind,
                               w.top_k, buf.sel[l], buf.sel_count[l], workspace=wss)

    def attn_all():
        for l in range(layers):
            lserve.sparse_decode_attn(d, buf.q, buf.k_pools[l], buf.v_pools[l], buf.block_table,
                                      buf.ctx_lens, buf.head_kind, buf.sel[l], buf.sel_count[l],
                                      w.top_k, w.sink, w.local, scale, outs[l], None, workspace=wsd,
                                      overlap_prologue=l > 0, prefetch_kv=l > 0)
    with torch.cuda.stream(stream):
        for l in range(layers):
            lserve.page_stats(d, buf.k_pools[l], buf.block_table, buf.ctx_lens, buf.head_kind,
                              buf.stats[l])
        select_all()
        attn_all()
    torch.cuda.synchronize()
    assert lserve.read_device_status(stream) == lserve.OK
    graphs = []
    for fn in (select_all, attn_all):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            fn()
        with torch.cuda.stream(stream):
            for _ in range(3):
                g.replay()
        graphs.append(g)
    reps = 20
    t_sel = timed(lambda: graphs[0].replay(), reps) / (reps * layers)
    t_att = timed(lambda: graphs[1].replay(), reps) / (reps * layers)
    acct = decode_bytes(w)
    extra = {}
    if shards > 1:
        extra["seq_sharded"] = seqshard_timing(lserve, w, buf, d, dev, stream, timed, layers, shards,
                                               scale)
    del graphs, buf
    torch.cuda.empty_cache()
    step = t_att + t_sel / REUSE
    return {**extra,
            "attention": {"us": t_att * 1e6, "GB/s": acct["attn"] / t_att / 1e9,
                          "frac": acct["attn"] / t_att / 1e9 / hbm_peak, "bytes": acct["attn"]},
            "selection": {"us": t_sel * 1e6, "GB/s": acct["select"] / t_sel / 1e9,
                          "frac": acct["select"] / t_sel / 1e9 / hbm_peak, "bytes": acct["select"]},
            "us_per_layer_step": step * 1e6, "GB/s_per_step": acct["step"] / step / 1e9,
            "layers": layers,
            "workload": f"{w.name}: B={w.B} n={int(w.ctx_lens.min())}..{int(w.ctx_lens.max())} "
                        f"H_q={w.H_q} H_kv={w.H_kv} D={w.D} N_L={w.N_L} N_P={w.N_P} "
                        f"top_k={w.top_k} sink={w.sink} local={w.local} reuse={REUSE}"}


def seqshard_timing(lserve, w, buf, d, dev, stream, timed, layers, N, scale):
    """Shard 0's part of an N-way sequence-sharded step of the same workload:
    the selection part (its own pages' scores and top-K, its proposals, the
    merge) and the attention part (attention over its chosen pages with float
    partials, the combine), per layer, graph replays over the layer replicas.
    Every shard's proposals and partials are computed once beforehand; the two
    all-gathers between the parts cross GPUs and are not timed here."""
    import torch
    K, B, H_kv, H_q, D = w.top_k, w.B, w.H_kv, w.H_q, w.D
    stride = lserve.seqshard_sel_stride(d, K, w.sink, w.local)
    views = []
    for r in range(N):
        bounds = [lserve.seqshard_bounds(int(w.ctx_lens[b]), w.N_P, r, N) for b in range(B)]
        ml = max([stride, 1] + [hi - lo for lo, hi, _ in bounds])
        bt = np.full((B, ml), -1, dtype=np.int32)
        for b, (lo, hi, _) in enumerate(bounds):
            bt[b, :hi - lo] = w.block_table[b, lo:hi]
        views.append((lserve.paged_desc(B, H_q, H_kv, D, w.N_L, w.N_P, ml, w.num_pool_pages),
                      torch.from_numpy(bt).to(dev),
                      torch.tensor([n for _, _, n in bounds], dtype=torch.int32, device=dev)))
    i32, f32 = torch.int32, torch.float32
    all_s = torch.empty((N, B, H_kv, K), dtype=f32, device=dev)
    all_p = torch.empty((N, B, H_kv, K), dtype=i32, device=dev)
    all_o = torch.empty((N, B * H_q, D), dtype=f32, device=dev)
    all_l = torch.empty((N, B * H_q), dtype=f32, device=dev)
    every_head = torch.zeros(H_kv, dtype=torch.uint8, device=dev)
    sel = [torch.empty((B, H_kv, K), dtype=i32, device=dev) for _ in range(N)]
    cnt = [torch.empty((B, H_kv), dtype=i32, device=dev) for _ in range(N)]
    sc = [torch.empty((B, H_kv, v[0].max_pages_per_seq), dtype=f32, device=dev) for v in views]
    sel_m = [torch.empty((B, H_kv, stride), dtype=i32, device=dev) for _ in range(N)]
    cnt_m = [torch.empty((B, H_kv), dtype=i32, device=dev) for _ in range(N)]
    wsd = [lserve.alloc_workspace(lserve.workspace_size(lserve.OP_DECODE, v[0], stride), device=dev)
           for v in views]
    outs = [torch.empty((B * H_q, D), dtype=torch.bfloat16, device=dev) for _ in range(layers)]

    def select_part(r, l):
        dr, bt, ctx = views[r]
        lserve.page_select(dr, buf.q, buf.stats[l], bt, ctx, buf.head_kind, K, sel[r], cnt[r],
                           phys_scores=sc[r])
        lserve.seqshard_candidates(dr, r, N, buf.ctx_lens, buf.head_kind, sel[r], cnt[r], sc[r], K,
                                   all_s[r], all_p[r])

    def merge_part(r):
        lserve.seqshard_merge(views[r][0], r, N, buf.ctx_lens, buf.head_kind, all_s, all_p, K, w.sink,
                              w.local, sel_m[r], cnt_m[r])

    def attend_part(r, l):
        dr, bt, ctx = views[r]
        lserve.sparse_decode_attn(dr, buf.q, buf.k_pools[l], buf.v_pools[l], bt, ctx, every_head,
                                  sel_m[r], cnt_m[r], stride, w.sink, w.local, scale, all_o[r], all_l[r],
                                  workspace=wsd[r], out_f32=True)

    with torch.cuda.stream(stream):
        for r in range(N):
            select_part(r, 0)
        for r in range(N):
            merge_part(r)
            attend_part(r, 0)
    torch.cuda.synchronize()
    assert lserve.read_device_status(stream) == lserve.OK

    def sel0():
        for l in range(layers):
            select_part(0, l)
            merge_part(0)

    def att0():
        for l in range(layers):
            attend_part(0, l)
            lserve.seqshard_combine(all_o, all_l, outs[l])
    graphs = []
    for fn in (sel0, att0):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            fn()
        with torch.cuda.stream(stream):
            for _ in range(3):
                g.replay()
        graphs.append(g)
    reps = 20
    t_sel = timed(lambda: graphs[0].replay(), reps) / (reps * layers)
    t_att = timed(lambda: graphs[1].replay(), reps) / (reps * layers)
    assert lserve.read_device_status(stream) == lserve.OK
    del graphs
    return {"shards": N, "timed_shard": 0, "selection_us": t_sel * 1e6, "attention_us": t_att * 1e6,
            "us_per_layer_step": (t_att + t_sel / REUSE) * 1e6,
            "not_timed": f"two all-gathers per step across GPUs: proposals {8 * B * H_kv * K} B and "
                         f"partials {4 * B * H_q * (D + 1)} B per shard"}


def profile_case(lserve, synth, dev, spec, launches):
    """One decode call of one workload, launched `launches` times after its
    set-up (statistics, selection, quantization): the small case the ncu
    captures in profiles/ run."""
    import torch
    from synth.device import DecodeBuffers
    wname, cache = spec.split(":")
    make = {"8b": synth.llama3_8b_decode, "mha": synth.llama2_7b_mha_decode,
            "256k": synth.long_decode_256k, "mixed": synth.mixed_batch_decode}[wname]
    w = make()
    buf = DecodeBuffers(w, device=dev)
    d = lserve.paged_desc(w.B, w.H_q, w.H_kv, w.D, w.N_L, w.N_P, w.max_pages, w.num_pool_pages)
    wss = lserve.alloc_workspace(lserve.workspace_size(lserve.OP_SELECT, d, w.top_k), device=dev)
    wsd = lserve.alloc_workspace(lserve.workspace_size(lserve.OP_DECODE, d, w.top_k), device=dev)
    lserve.page_stats(d, buf.k_pool, buf.block_table, buf.ctx_lens, buf.head_kind, buf.stats[0])
    lserve.page_select(d, buf.q, buf.stats[0], buf.block_table, buf.ctx_lens, buf.head_kind,
                       w.top_k, buf.sel[0], buf.sel_count[0], workspace=wss)
    scale = 1.0 / math.sqrt(w.D)
    bits = {"bf16": 0, "kv8": 8, "kv4": 4}[cache]
    if bits:
        shape = w.pool_shape() if bits == 8 else w.pool_shape()[:-1] + (w.D // 2,)
        k8 = torch.empty(shape, dtype=torch.int8, device=dev)
        v8 = torch.empty_like(k8)
        ks = torch.empty((w.num_pool_pages, w.H_kv, w.D), dtype=torch.float32, device=dev)
        vs = torch.empty_like(ks)
        lserve.quantize_pages_kv8(d, buf.k_pool, buf.v_pool, buf.block_table, buf.ctx_lens, k8, v8,
                                  ks, vs, bits=bits)
    for _ in range(max(1, launches)):
        if bits:
            lserve.sparse_decode_attn_kv8(d, buf.q, k8, v8, ks, vs, buf.block_table, buf.ctx_lens,
                                          buf.head_kind, buf.sel[0], buf.sel_count[0], w.top_k,
                                          w.sink, w.local, scale, buf.out, None, workspace=wsd,
                                          bits=bits)
        else:
            lserve.sparse_decode_attn(d, buf.q, buf.k_pool, buf.v_pool, buf.block_table,
                                      buf.ctx_lens, buf.head_kind, buf.sel[0], buf.sel_count[0],
                                      w.top_k, w.sink, w.local, scale, buf.out, None, workspace=wsd)
    torch.cuda.synchronize()
    assert lserve.read_device_status() == lserve.OK
    print(json.dumps({"profile": spec, "launches": launches}))
    return 0


def seqshard_stage(lserve, synth, dev, stream, hbm_peak, timed, rank, ws, warmup, layers=8,
                   steps=64):
    """The 256K long decode as one sequence split over the ws ranks (rank r
    holds the physical pages [floor(M r / ws), floor(M (r + 1) / ws)) of every
    layer, reading R17): per layer-step each rank attends its share of the
    chosen pages, all-gathers the float partials over NCCL and combines them;
    every REUSE-th step it first scores its own pages, all-gathers its top-K
    proposals and merges them (SeqShardStep, the exchanges on the stream).
    `layers` replicas, `steps` layer-steps timed (after `warmup`), eager
    launches, max over ranks.  Bytes: those of the whole unsharded step."""
    import torch
    from synth.device import DecodeBuffers
    w = synth.long_decode_256k()
    buf = DecodeBuffers(w, device=dev, layers=layers)
    B, H_q, H_kv, D, K = w.B, w.H_q, w.H_kv, w.D, w.top_k
    d = lserve.paged_desc(B, H_q, H_kv, D, w.N_L, w.N_P, w.max_pages, w.num_pool_pages)
    bounds = [lserve.seqshard_bounds(int(w.ctx_lens[b]), w.N_P, rank, ws) for b in range(B)]
    stride = lserve.seqshard_sel_stride(d, K, w.sink, w.local)
    ml = max([stride, 1] + [hi - lo for lo, hi, _ in bounds])
    bt = np.full((B, ml), -1, dtype=np.int32)
    for b, (lo, hi, _) in enumerate(bounds):
        bt[b, :hi - lo] = w.block_table[b, lo:hi]
    dr = lserve.paged_desc(B, H_q, H_kv, D, w.N_L, w.N_P, ml, w.num_pool_pages)
    bt_r = torch.from_numpy(bt).to(dev)
    ctx_r = torch.tensor([n for _, _, n in bounds], dtype=torch.int32, device=dev)
    shards = [lserve.SeqShardStep(dr, rank, ws, K, w.sink, w.local, device=dev)
              for _ in range(layers)]
    outs = [torch.empty((B, H_q, D), dtype=torch.bfloat16, device=dev) for _ in range(layers)]
    scale = 1.0 / math.sqrt(D)
    with torch.cuda.stream(stream):
        for l in range(layers):  # the statistics of this rank's pages
            lserve.page_stats(dr, buf.k_pools[l], bt_r, ctx_r, buf.head_kind, buf.stats[l])

    def step(t):
        for l in range(layers):
            if t % REUSE == 0:
                shards[l].select(buf.q, buf.stats[l], bt_r, ctx_r, buf.ctx_lens, buf.head_kind)
            shards[l].attend(buf.q, buf.k_pools[l], buf.v_pools[l], bt_r, ctx_r, scale, outs[l])

    with torch.cuda.stream(stream):
        for t in range(max(warmup, REUSE)):
            step(t)
    torch.cuda.synchronize()
    assert lserve.read_device_status(stream) == lserve.OK
    el = timed(lambda: [step(t) for t in range(steps)])
    el = max_over_ranks(el, ws, dev)
    per = el / (steps * layers)
    acct = decode_bytes(w)
    return {"ranks": ws, "us_per_layer_step": per * 1e6, "GB/s_per_step": acct["step"] / per / 1e9,
            "layers": layers, "steps": steps,
            "what": "SeqShardStep per layer: attention over the rank's chosen pages, NCCL "
                    "all-gather of (o, lse), combine; every 4th step also scores, all-gathers "
                    "proposals and merges; eager launches; the bytes of the unsharded step",
            "workload": f"{w.name}: B={B} n={int(w.ctx_lens[0])} split over {ws} ranks"}


def kv8_stage(lserve, synth, dev, stream, hbm_peak, timed, make, layers, bf16_us, bits=8):
    """Decode attention over the quantized cache (lserve_sparse_decode_attn_kv8
    or _kv4 for bits = 8 / 4), alone: the workload's pools quantized once
    (lserve_quantize_pages_kv8 / _kv4, timed too), then `layers` replicas of
    the quantized pools attended back to back (more bytes than L2 holds), the
    selection being the bf16 statistics'."""
    import torch
    from synth.device import DecodeBuffers
    w = make()
    buf = DecodeBuffers(w, device=dev, layers=1)
    d = lserve.paged_desc(w.B, w.H_q, w.H_kv, w.D, w.N_L, w.N_P, w.max_pages, w.num_pool_pages)
    wss = lserve.alloc_workspace(lserve.workspace_size(lserve.OP_SELECT, d, w.top_k), device=dev)
    wsd = lserve.alloc_workspace(lserve.workspace_size(lserve.OP_DECODE, d, w.top_k), device=dev)
    shape = w.pool_shape() if bits == 8 else w.pool_shape()[:-1] + (w.D // 2,)
    k8 = torch.empty(shape, dtype=torch.int8, device=dev)
    v8 = torch.empty_like(k8)
    ks = torch.empty((w.num_pool_pages, w.H_kv, w.D), dtype=torch.float32, device=dev)
    vs = torch.empty_like(ks)

    def quantize():
        lserve.quantize_pages_kv8(d, buf.k_pool, buf.v_pool, buf.block_table, buf.ctx_lens, k8, v8,
                                  ks, vs, stream=stream, bits=bits)
    with torch.cuda.stream(stream):
        lserve.page_stats(d, buf.k_pool, buf.block_table, buf.ctx_lens, buf.head_kind, buf.stats[0])
        lserve.page_select(d, buf.q, buf.stats[0], buf.block_table, buf.ctx_lens, buf.head_kind,
                           w.top_k, buf.sel[0], buf.sel_count[0], workspace=wss)
        quantize()
    torch.cuda.synchronize()
    assert lserve.read_device_status(stream) == lserve.OK
    t_q = timed(quantize, 3) / 3
    qb = quantize_bytes(w, bits)
    buf.k_pools = buf.v_pools = None  # the bf16 pools are not read below
    torch.cuda.empty_cache()
    pools = [(k8, v8, ks, vs)] + [(k8.clone(), v8.clone(), ks.clone(), vs.clone())
                                  for _ in range(layers - 1)]
    outs = [torch.empty_like(buf.out) for _ in range(layers)]
    scale = 1.0 / math.sqrt(w.D)

    def attn_all():
        for l, (a, b, c, e) in enumerate(pools):
            lserve.sparse_decode_attn_kv8(d, buf.q, a, b, c, e, buf.block_table, buf.ctx_lens,
                                          buf.head_kind, buf.sel[0], buf.sel_count[0], w.top_k,
                                          w.sink, w.local, scale, outs[l], None, workspace=wsd,
                                          overlap_prologue=l > 0, prefetch_kv=l > 0, bits=bits)
    with torch.cuda.stream(stream):
        attn_all()
    torch.cuda.synchronize()
    assert lserve.read_device_status(stream) == lserve.OK
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        attn_all()
    with torch.cuda.stream(stream):
        for _ in range(3):
            g.replay()
    reps = 20
    t = timed(lambda: g.replay(), reps) / (reps * layers)
    bts = decode_bytes_kv8(w, bits)
    del g, pools
    torch.cuda.empty_cache()
    return {"us": t * 1e6, "GB/s": bts / t / 1e9, "frac": bts / t / 1e9 / hbm_peak, "bytes": bts,
            "speedup_vs_bf16_cache": bf16_us / (t * 1e6),
            "quantize": {"us": t_q * 1e6, "GB/s": qb / t_q / 1e9, "frac": qb / t_q / 1e9 / hbm_peak,
                         "bytes": qb, "what": f"lserve_quantize_pages_kv{bits} of the whole cache"},
            "workload": f"{w.name} ({bits}-bit cache): B={w.B} n={int(w.ctx_lens[0])} H_q={w.H_q} "
                        f"H_kv={w.H_kv} D={w.D} N_P={w.N_P} top_k={w.top_k}"}


def prefill_stage(lserve, synth, dev, stream, tc_peak, timed, seq=None):
    """Block-sparse prefill on the 128K workload (or `seq` tokens of the same
    shape): TFLOP/s over computed blocks."""
    import torch
    w = synth.prefill_128k() if seq is None else synth.prefill_workload(
        seq, 32, 8, 128, 128, 1004, name=f"prefill_{seq}")
    if timed is None:
        def timed(fn, reps=1):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            e0.record(stream)
            with torch.cuda.stream(stream):
                for _ in range(reps):
                    fn()
            e1.record(stream)
            torch.cuda.synchronize()
            return e0.elapsed_time(e1) / 1e3
    d = lserve.prefill_desc(w.T, w.H_q, w.H_kv, w.D, w.block, w.sink_blocks, w.local_blocks)
    need = lserve.workspace_size(lserve.OP_PREFILL, d)
    try:
        from synth.device import PrefillBuffers
        pb = PrefillBuffers(w, device=dev)
        wsb = lserve.alloc_workspace(need, device=dev)
        scale = 1.0 / math.sqrt(w.D)

        def run():
            lserve.blocksparse_prefill(d, pb.q, pb.k, pb.v, list(w.head_kind), scale, pb.out, None,
                                       workspace=wsb, stream=stream)
        with torch.cuda.stream(stream):
            run()
        torch.cuda.synchronize()
        t = timed(run, 3) / 3
        # the prefilled sequence handed to the paged decode cache: K/V into the
        # pools and the retrieval heads' page statistics in one pass
        N_L, N_P = 16, 64
        npages = -(-w.T // N_P)
        pd = lserve.paged_desc(1, w.H_q, w.H_kv, w.D, N_L, N_P, npages, npages)
        kp = torch.empty((npages, w.H_kv, N_P, w.D), dtype=torch.bfloat16, device=dev)
        vp = torch.empty_like(kp)
        sp = torch.empty((npages, w.H_kv, N_P // N_L, 2, w.D), dtype=torch.bfloat16, device=dev)
        bt = torch.randperm(npages, generator=torch.Generator().manual_seed(5)).to(torch.int32).to(dev)
        hk = torch.from_numpy(np.ascontiguousarray(w.head_kind)).to(dev)

        def to_pages():
            lserve.prefill_to_pages(pd, w.T, pb.k, pb.v, bt, hk, kp, vp, sp, stream=stream)
        with torch.cuda.stream(stream):
            to_pages()
        torch.cuda.synchronize()
        t_tp = timed(to_pages, 3) / 3

        # the same hand-over fused into the prefill kernel (its epilogue)
        def paged():
            lserve.blocksparse_prefill_paged(d, pd, pb.q, pb.k, pb.v, list(w.head_kind), scale,
                                             pb.out, bt, kp, vp, sp, workspace=wsb, stream=stream)
        with torch.cuda.stream(stream):
            paged()
        torch.cuda.synchronize()
        t_pg = timed(paged, 3) / 3
        assert lserve.read_device_status(stream) == lserve.OK
        retr = int(sum(1 for h in range(w.H_kv) if w.head_kind[h] == 0))
        tp_bytes = 2 * 2 * w.T * w.H_kv * w.D * 2 + retr * (-(-w.T // N_L)) * 2 * w.D * 2
        del kp, vp, sp
    except lserve.LServeError as e:
        return {"unavailable": str(e)}
    flops = prefill_flops(w.T, w.H_q, w.H_kv, w.D, w.block, w.head_kind, w.sink_blocks,
                          w.local_blocks)
    tf = flops / t / 1e12
    return {"ms": t * 1e3, "TFLOP/s": tf, "frac": tf / tc_peak, "flops": flops,
            "to_pages": {"us": t_tp * 1e6, "GB/s": tp_bytes / t_tp / 1e9, "bytes": tp_bytes,
                         "what": "lserve_prefill_to_pages: K/V into the paged pools (N_P=64) "
                                 "+ page statistics (N_L=16), one pass"},
            "paged": {"ms": t_pg * 1e3, "TFLOP/s": flops / t_pg / 1e12,
                      "frac": flops / t_pg / 1e12 / tc_peak,
                      "what": "lserve_blocksparse_prefill_paged: the prefill with the same hand-over "
                              "(N_P=64, N_L=16) in its kernel's epilogue"},
            "workload": f"{w.name}: T={w.T} H_q={w.H_q} H_kv={w.H_kv} D={w.D} block={w.block} "
                        f"Lambda({w.sink_blocks},{w.local_blocks}) on KV heads 4-7"}


if __name__ == "__main__":
    sys.exit(main())
