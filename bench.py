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
DEFAULT_STEPS = 6000
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

def decode_bytes(w):
    """Bytes one decode step of one layer must move, amortising selection over
    the reuse interval.  KV: valid tokens of the attended pages, K and V, D*2
    bytes each.  Selection: the stats of every valid logical page of the
    retrieval heads (2*D*2 bytes), the q vectors, scores and selection."""
    import oracle
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
                pages = oracle.streaming_pages(n, NP, w.sink, w.local)
                toks = len(oracle.page_tokens(pages, n, NP))
                kv += toks * D * 2 * 2
    q = w.B * w.H_q * D * 2
    out = w.B * w.H_q * D * 2
    sel_io = q + w.B * w.H_kv * (w.max_pages * 4 + w.top_k * 4 + 4)
    attn = kv + q + out
    select = stats + sel_io
    return dict(attn=attn, select=select, step=attn + select / REUSE, kv=kv, stats=stats)


def decode_bytes_kv8(w):
    """Bytes one decode-attention call over the int8 cache moves: the codes of
    the attended pages (K and V, D bytes per token each), the two float32
    channel-scale rows of every attended (page, head), q and the output."""
    import oracle
    D, NP = w.D, w.N_P
    kv = 0
    for b in range(w.B):
        n = int(w.ctx_lens[b])
        npages = -(-n // NP)
        for h in range(w.H_kv):
            if w.head_kind[h] == 0:
                k = min(w.top_k, npages)
                kv += k * NP * D * 2 + k * 2 * D * 4
            else:
                pages = oracle.streaming_pages(n, NP, w.sink, w.local)
                toks = len(oracle.page_tokens(pages, n, NP))
                kv += toks * D * 2 + len(pages) * 2 * D * 4
    return kv + 2 * w.B * w.H_q * D * 2


def quantize_bytes(w):
    """lserve_quantize_pages_kv8: read the valid bf16 K/V rows of every page,
    write the int8 codes (whole pages) and the float32 scales."""
    rd = wr = 0
    for b in range(w.B):
        n = int(w.ctx_lens[b])
        npages = -(-n // w.N_P)
        rd += 2 * n * w.H_kv * w.D * 2
        wr += 2 * npages * w.H_kv * (w.N_P * w.D + w.D * 4)
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


def decode_traffic():
    """DRAM bytes (read + write) per decode-attention launch from the committed
    ncu summary, provided the kernel source is still the one it measured."""
    import hashlib
    summ = os.path.join(ROOT, "profiles", "decode_attn_llama3_8b_decode.md")
    src = os.path.join(ROOT, "block_sparse_attention_page_b200", "csrc", "decode_attn.cu")
    try:
        fields = {}
        with open(summ) as f:
            for line in f:
                if line.startswith("- ") and ":" in line:
                    k, v = line[2:].split(":", 1)
                    fields[k.strip()] = v.strip().strip("`")
        with open(src, "rb") as f:
            digest = hashlib.sha256(f.read()).hexdigest()
        if fields.get("decode_attn.cu sha256") != digest:
            return None
        return float(fields["traffic bytes per launch"])
    except (OSError, KeyError, ValueError):
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

def oracle_step_sample(w, budget_s=12.0, max_pairs=None):
    """Time the oracle's decode step (stats of the retrieval heads already
    built, as on the GPU; then S^j -> P^m -> top-K -> attention per pair) on a
    bounded sample of (sequence, KV head) pairs; returns seconds per layer-step
    extrapolated from the pairs timed, and what was sampled."""
    import oracle
    try:
        from threadpoolctl import threadpool_limits
        lim = threadpool_limits(1)
    except Exception:
        lim = None
    G = w.G
    scale = 1.0 / math.sqrt(w.D)
    pairs = [(b, h) for b in range(w.B) for h in range(w.H_kv)]
    t_sel = t_attn = 0.0
    done = 0
    t_start = time.perf_counter()
    for (b, h) in pairs:
        n = int(w.ctx_lens[b])
        q = oracle.widen_bf16(w.q[b, h * G:(h + 1) * G])
        k = oracle.widen_bf16(w.k_seq(b, h))
        v = oracle.widen_bf16(w.v_seq(b, h))
        if w.head_kind[h] == 0:
            kmin, kmax = oracle.page_stats(k, w.N_L)      # built once, not timed (GPU: not per step)
            t0 = time.perf_counter()
            P = oracle.physical_scores(oracle.logical_scores(q, kmin, kmax), w.g)
            pages = oracle.select_top_k(P, w.top_k)
            t1 = time.perf_counter()
            t_sel += t1 - t0
        else:
            t1 = time.perf_counter()
            pages = oracle.streaming_pages(n, w.N_P, w.sink, w.local)
        oracle.decode_attention(q, k, v, oracle.page_tokens(pages, n, w.N_P), scale)
        t_attn += time.perf_counter() - t1
        done += 1
        if time.perf_counter() - t_start > budget_s or (max_pairs and done >= max_pairs):
            break
    if lim is not None:
        lim.unregister() if hasattr(lim, "unregister") else None
    frac = done / len(pairs)
    per_step = (t_sel / REUSE + t_attn) / frac
    return per_step, f"{done} of {len(pairs)} (sequence, KV head) pairs of one layer-step, " \
                     f"selection amortised over {REUSE} steps, 1 thread"


def reference_steps(w, steps, warmup):
    """The oracle as timed steps of the reference arm: step t takes the
    (sequence, KV head) pair t mod P of one layer -- its page selection
    (S^j -> P^m -> top-K) on every REUSE-th visit, as the GPU step reuses it,
    and its attention every visit -- so a step is a bounded sample of the
    workload and K steps amount to K / P layer-steps.  The bf16 inputs are
    widened once and the page statistics built once (as on the GPU), untimed;
    one thread.  Returns (seconds of the K timed steps, layer-steps, sample)."""
    import oracle
    try:
        from threadpoolctl import threadpool_limits
        lim = threadpool_limits(1)
    except Exception:
        lim = None
    G = w.G
    scale = 1.0 / math.sqrt(w.D)
    cache = []
    for b in range(w.B):
        n = int(w.ctx_lens[b])
        for h in range(w.H_kv):
            q = oracle.widen_bf16(w.q[b, h * G:(h + 1) * G])
            k = oracle.widen_bf16(w.k_seq(b, h))
            v = oracle.widen_bf16(w.v_seq(b, h))
            stats = None
            if w.head_kind[h] == 0:
                stats = oracle.page_stats(k, w.N_L)
                pages = oracle.select_top_k(
                    oracle.physical_scores(oracle.logical_scores(q, *stats), w.g), w.top_k)
            else:
                pages = oracle.streaming_pages(n, w.N_P, w.sink, w.local)
            toks = oracle.page_tokens(pages, n, w.N_P)
            # the attended keys and values (the selection is the same at every visit)
            cache.append((q, stats, np.ascontiguousarray(k[toks]), np.ascontiguousarray(v[toks])))
    P = len(cache)

    def step(t):
        q, stats, ks, vs = cache[t % P]
        if stats is not None and (t // P) % REUSE == 0:
            oracle.select_top_k(oracle.physical_scores(oracle.logical_scores(q, *stats), w.g), w.top_k)
        oracle.decode_attention(q, ks, vs, np.arange(len(ks)), scale)

    for t in range(warmup):
        step(t)
    t0 = time.perf_counter()
    for t in range(warmup, warmup + steps):
        step(t)
    elapsed = time.perf_counter() - t0
    if lim is not None and hasattr(lim, "unregister"):
        lim.unregister()
    return elapsed, steps / P, (f"each step one (sequence, KV head) pair of one layer ({P} pairs, "
                                f"selection on every {REUSE}th visit of a pair), 1 thread")


def reference_arm(args):
    """The oracle as the reference arm: same metric / unit / config."""
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    import synth
    w = synth.llama3_8b_decode()
    acct = decode_bytes(w)
    elapsed, layer_steps, sample = reference_steps(w, args.steps, args.warmup)
    per_layer_step = elapsed / layer_steps
    value = acct["step"] / per_layer_step / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_layer_step * LAYERS * 1e3,
        "us_per_layer_step": per_layer_step * 1e6, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w),
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": sample + f"; {elapsed:.1f} s for {args.steps} steps"},
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
    ap.add_argument("--steps", type=int, default=DEFAULT_STEPS)
    ap.add_argument("--warmup", type=int, default=DEFAULT_WARMUP)
    ap.add_argument("--impl", default="lserve", choices=["lserve", "reference"])
    ap.add_argument("--no-prefill", action="store_true", help="skip the prefill stage")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--layers", type=int, default=LAYERS,
                    help="layer replicas (fewer = a small case for profiling; < 32 may fit in L2)")
    ap.add_argument("--no-mha", action="store_true", help="skip the MHA decode stage")
    ap.add_argument("--no-kv8", action="store_true", help="skip the int8-cache decode stages")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the long-decode and mixed-batch decode stages")
    ap.add_argument("--prefill-only", action="store_true",
                    help="run only the prefill stage (profiling)")
    ap.add_argument("--prefill-seq", type=int, default=None,
                    help="prefill sequence length (default: the 128K workload)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
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
    acct = decode_bytes(w)

    def stats_all():
        for l in range(LAYERS):
            lserve.page_stats(d, buf.k_pools[l], buf.block_table, buf.ctx_lens, buf.head_kind,
                              buf.stats[l])

    def select(l):
        lserve.page_select(d, qs[l], buf.stats[l], buf.block_table, buf.ctx_lens, buf.head_kind,
                           w.top_k, buf.sel[l], buf.sel_count[l], workspace=ws_sel)

    def attn(l, overlap=False):
        # overlap: the kernel before this call is the previous layer's attention,
        # which writes none of the selection / block-table inputs, so the split
        # plan and first page lookups may run while it finishes (PDL)
        lserve.sparse_decode_attn(d, qs[l], buf.k_pools[l], buf.v_pools[l], buf.block_table,
                                  buf.ctx_lens, buf.head_kind, buf.sel[l], buf.sel_count[l], w.top_k,
                                  w.sink, w.local, scale, outs[l], None, workspace=ws_dec,
                                  overlap_prologue=overlap)

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

    # decode-time cache maintenance (lserve_decode_append), timed alone: each
    # sequence's last token is written again with its own K/V (position n - 1,
    # inside the block table), which leaves the cache and statistics unchanged
    lens_last = (buf.ctx_lens - 1).to(torch.int32)
    last = [(int(w.block_table[b, (int(w.ctx_lens[b]) - 1) // w.N_P]),
             (int(w.ctx_lens[b]) - 1) % w.N_P) for b in range(w.B)]
    k_last = [torch.stack([buf.k_pools[l][pid, :, r] for pid, r in last]).contiguous()
              for l in range(LAYERS)]
    v_last = [torch.stack([buf.v_pools[l][pid, :, r] for pid, r in last]).contiguous()
              for l in range(LAYERS)]

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
                   "note": "lserve_decode_append per layer; launch-latency bound (16 KB of K/V)"},
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
                     "frac": attn_gbs / hbm_peak, "traffic": decode_traffic(),
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
            lserve, synth, dev, stream, hbm_peak, timed, synth.long_decode_256k, 16, shards=4)
        result["stages"]["mixed_batch_decode"] = decode_config_stage(
            lserve, synth, dev, stream, hbm_peak, timed, synth.mixed_batch_decode, 3)
    if not args.no_kv8:
        result["stages"]["attention_kv8"] = kv8_stage(lserve, synth, dev, stream, hbm_peak, timed,
                                                      synth.llama3_8b_decode, 16,
                                                      stages["attention"]["us"])
        if not args.no_mha:
            result["stages"]["attention_mha_kv8"] = kv8_stage(
                lserve, synth, dev, stream, hbm_peak, timed, synth.llama2_7b_mha_decode, 8,
                result["stages"]["attention_mha"]["us"])
    if not args.no_prefill:
        result["stages"]["prefill"] = prefill_stage(lserve, synth, dev, stream, tc_peak, timed,
                                                    args.prefill_seq)

    if rank == 0 and ws == 1 and not args.no_cpu_baseline:  # the oracle baseline: one GPU runs only
        per_step, sample = oracle_step_sample(w, budget_s=15.0)
        cpu_val = acct["step"] / per_step / 1e9
        result["cpu_baseline"] = {"value": cpu_val, "unit": "GB/s", "cores": 1, "kind": "oracle",
                                  "sample": sample}
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
                                      overlap_prologue=l > 0)
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
                                      overlap_prologue=l > 0)
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


def kv8_stage(lserve, synth, dev, stream, hbm_peak, timed, make, layers, bf16_us):
    """Decode attention over the int8 cache (lserve_sparse_decode_attn_kv8),
    alone: the workload's pools quantized once (lserve_quantize_pages_kv8,
    timed too), then `layers` replicas of the int8 pools attended back to back
    (more bytes than L2 holds), the selection being the bf16 statistics'."""
    import torch
    from synth.device import DecodeBuffers
    w = make()
    buf = DecodeBuffers(w, device=dev, layers=1)
    d = lserve.paged_desc(w.B, w.H_q, w.H_kv, w.D, w.N_L, w.N_P, w.max_pages, w.num_pool_pages)
    wss = lserve.alloc_workspace(lserve.workspace_size(lserve.OP_SELECT, d, w.top_k), device=dev)
    wsd = lserve.alloc_workspace(lserve.workspace_size(lserve.OP_DECODE, d, w.top_k), device=dev)
    k8 = torch.empty(w.pool_shape(), dtype=torch.int8, device=dev)
    v8 = torch.empty_like(k8)
    ks = torch.empty((w.num_pool_pages, w.H_kv, w.D), dtype=torch.float32, device=dev)
    vs = torch.empty_like(ks)

    def quantize():
        lserve.quantize_pages_kv8(d, buf.k_pool, buf.v_pool, buf.block_table, buf.ctx_lens, k8, v8,
                                  ks, vs, stream=stream)
    with torch.cuda.stream(stream):
        lserve.page_stats(d, buf.k_pool, buf.block_table, buf.ctx_lens, buf.head_kind, buf.stats[0])
        lserve.page_select(d, buf.q, buf.stats[0], buf.block_table, buf.ctx_lens, buf.head_kind,
                           w.top_k, buf.sel[0], buf.sel_count[0], workspace=wss)
        quantize()
    torch.cuda.synchronize()
    assert lserve.read_device_status(stream) == lserve.OK
    t_q = timed(quantize, 3) / 3
    qb = quantize_bytes(w)
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
                                          overlap_prologue=l > 0)
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
    bts = decode_bytes_kv8(w)
    del g, pools
    torch.cuda.empty_cache()
    return {"us": t * 1e6, "GB/s": bts / t / 1e9, "frac": bts / t / 1e9 / hbm_peak, "bytes": bts,
            "speedup_vs_bf16_cache": bf16_us / (t * 1e6),
            "quantize": {"us": t_q * 1e6, "GB/s": qb / t_q / 1e9, "frac": qb / t_q / 1e9 / hbm_peak,
                         "bytes": qb, "what": "lserve_quantize_pages_kv8 of the whole cache"},
            "workload": f"{w.name} (int8 cache): B={w.B} n={int(w.ctx_lens[0])} H_q={w.H_q} "
                        f"H_kv={w.H_kv} D={w.D} N_P={w.N_P} top_k={w.top_k}"}


def prefill_stage(lserve, synth, dev, stream, tc_peak, timed, seq=None):
    """Block-sparse prefill on the 128K workload (or `seq` tokens of the same
    shape): TFLOP/s over computed blocks."""
    import torch
    import oracle
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
        retr = int(sum(1 for h in range(w.H_kv) if w.head_kind[h] == 0))
        tp_bytes = 2 * 2 * w.T * w.H_kv * w.D * 2 + retr * (-(-w.T // N_L)) * 2 * w.D * 2
        del kp, vp, sp
    except lserve.LServeError as e:
        return {"unavailable": str(e)}
    flops = oracle.prefill_flops(w.T, w.H_q, w.H_kv, w.D, w.block, w.head_kind, w.sink_blocks,
                                 w.local_blocks)
    tf = flops / t / 1e12
    return {"ms": t * 1e3, "TFLOP/s": tf, "frac": tf / tc_peak, "flops": flops,
            "to_pages": {"us": t_tp * 1e6, "GB/s": tp_bytes / t_tp / 1e9, "bytes": tp_bytes,
                         "what": "lserve_prefill_to_pages: K/V into the paged pools (N_P=64) "
                                 "+ page statistics (N_L=16), one pass"},
            "workload": f"{w.name}: T={w.T} H_q={w.H_q} H_kv={w.H_kv} D={w.D} block={w.block} "
                        f"Lambda({w.sink_blocks},{w.local_blocks}) on KV heads 4-7"}


if __name__ == "__main__":
    sys.exit(main())
