"""Benchmark of the lightning-indexer hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    python -m torch.distributed.run --nnodes=1 --nproc-per-node N --master-addr 127.0.0.1 \
        --master-port P bench.py --gpus N ...

One step = one 200000-token prefill through a 47-layer model under the searched 1/4 IndexCache
pattern (12 Full layers), with the indexer of every Full layer run on H = 64 heads, d = 128,
top-k = 2048 over rho = 0.9 correlated FP8 E4M3 layers. The prefill is chunked by 8192 queries
the way a model runs it: chunk c passes through all 47 layers (one indexcache_run call: the 12
Full layers launch the fused indexer, the 35 Shared layers alias the last Full layer's index
buffer) before chunk c + 1 starts. Inputs (all 47 layers, 81 GB) are generated on the device
before timing and are far larger than L2. `value` counts the causal (query, key) pairs the
Full layers score and top-k per second. The same step under the all-F, FFFS and FSSS patterns
is timed once each (extra keys), as are the 8-layer 16384-token IndexCache stack with its 8 x 8
top-k overlap and the 47-layer decode step of 32 requests (extra keys "stack_16k", "decode").

At N > 1 every rank runs its own independently seeded copy of the workload (weak scaling, no
collective on the data path).

`--impl reference` times the oracle (the only reference implementation there is) on a bounded
sample of query rows of the same workload, on the host cores.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "indexer q·k pairs scored+top-k'd/s (prefill, decode); % of FP8 / HBM roofline"
UNIT = "pairs/s"

LONG = dict(L=200000, H=64, d=128, topk=2048, n_layers=47, chunk=8192, seed=5)
STACK = dict(L=16384, H=64, d=128, topk=2048, n_layers=8, pattern="FSFSFSFS", seed=2)
DECODE = dict(B=32, lo=10000, hi=200000, H=64, d=128, topk=2048, n_layers=47, seed=4)

FP8_PER_BF16 = 2.0  # nominal dense FP8 / BF16 tensor throughput ratio on B200
# Kernel launches of one dsa_indexer_prefill call with top-k 2048: sample pass, per-row sample
# threshold, lean pass, exact pass (exits at once when the lean pass marked no block), finish.
PREFILL_LAUNCHES_PER_CALL = 5
# decode: the histogram clear, the scoring kernel, the collection pass and the rank pass
DECODE_LAUNCHES_PER_CALL = 4


# ------------------------------------------------------------------------------------------
# multi-process plumbing
# ------------------------------------------------------------------------------------------

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world: int, backend: str):
    if world > 1 and not torch.distributed.is_initialized():
        import datetime
        torch.distributed.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=300))


def barrier(world: int, device=None):
    if world > 1:
        if device is not None and torch.distributed.get_backend() == "nccl":
            torch.distributed.barrier(device_ids=[device.index])
        else:
            torch.distributed.barrier()


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Largest value over all ranks (the job is as slow as its slowest rank)."""
    if world == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if torch.distributed.get_backend() == "nccl" else "cpu")
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, world: int, device=None) -> float:
    if world == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if torch.distributed.get_backend() == "nccl" else "cpu")
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return float(t.item())


def rank_seed(base: int, rank: int) -> int:
    """Each rank draws an independent batch of the same workload."""
    return base + 1000 * rank


# ------------------------------------------------------------------------------------------
# measurement helpers
# ------------------------------------------------------------------------------------------

def causal_pairs(L: int) -> int:
    return L * (L + 1) // 2


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", str(self.gpu_index)],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        if self.path and os.path.exists(self.path):
            for line in open(self.path):
                f = [x.strip() for x in line.split(",")]
                if len(f) >= 9:
                    rows.append(f)
            os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        under_load = [x for x in sm if smax and x > 0.5 * max(smax)] or sm
        return {"sm_mhz": float(np.median(under_load)) if under_load else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": reasons,
                "samples": len(rows),
                "power_w_max": max((float(r[3]) for r in rows if r[3].replace(".", "").isdigit()),
                                   default=None)}


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def numpy_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return 1




def patterns_47():
    from synth import SEARCHED_QUARTER_PATTERN
    n = LONG["n_layers"]
    return {"searched 1/4": SEARCHED_QUARTER_PATTERN, "all F": "F" * n,
            "FFFS": ("FFFS" * 12)[:n], "FSSS": ("FSSS" * 12)[:n]}


def peak_tflops(peaks, sustained: bool) -> float:
    key = "bf16_tflops_sustained" if sustained else "bf16_tflops"
    return FP8_PER_BF16 * float(peaks[key])


# ------------------------------------------------------------------------------------------
# the 200000-token, 47-layer prefill (headline)
# ------------------------------------------------------------------------------------------

class LongPrefill:
    """Device-resident inputs of all 47 layers and the chunk-major IndexCache step."""

    def __init__(self, device, seed):
        from synth import correlated_layers
        c = LONG
        self.device = device
        self.L, self.H, self.d, self.topk, self.chunk = c["L"], c["H"], c["d"], c["topk"], c["chunk"]
        self.layers = list(correlated_layers(self.L, self.H, self.d, c["n_layers"], seed, device=device))
        self.chunks = [(c0, min(self.L, c0 + self.chunk)) for c0 in range(0, self.L, self.chunk)]
        # per chunk, every layer's views: queries of the chunk, keys before the chunk's end
        self.views = [[{"q": l.q[c0:c1], "q_scale": l.q_scale[c0:c1], "w": l.w[c0:c1],
                        "k": l.k[:c1], "k_scale": l.k_scale[:c1]} for l in self.layers]
                      for c0, c1 in self.chunks]
        from sparse_attention_token_04_b200 import binding as B
        self.B = B
        self.ws = torch.empty(B.dsa_prefill_workspace_bytes(self.chunk, self.H, self.d, self.topk),
                              dtype=torch.uint8, device=device)
        B.dsa_workspace_init(self.ws)
        # the pages' single overwritten index cache: one chunk-sized buffer every F layer rewrites
        self.out = torch.empty(self.chunk, self.topk, dtype=torch.int32, device=device)

    def step(self, pattern, after_chunk_layer=None):
        """One prefill of all chunks through all layers. after_chunk_layer(ci, l) is called after
        layer l of chunk ci has been enqueued (host side), before the next layer can overwrite."""
        for ci, (c0, c1) in enumerate(self.chunks):
            views = [v if pattern[l] == "F" else None for l, v in enumerate(self.views[ci])]
            cb = None
            if after_chunk_layer is not None:
                cb = (lambda ci_: (lambda l, p: after_chunk_layer(ci_, l)))(ci)
            self.B.indexcache_run(pattern, views, self.topk, f_bufs=[self.out[: c1 - c0]],
                                  q_pos0=c0, workspace=self.ws, after_layer=cb)

    def pairs(self, pattern):
        return pattern.count("F") * causal_pairs(self.L)

    def calls(self, pattern):
        return pattern.count("F") * len(self.chunks)


def timed(stream, fn, n):
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(n):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1)


def run_long(args, world, rank, device, peaks, peak_kind):
    from synth import SEARCHED_QUARTER_PATTERN
    stream = torch.cuda.current_stream()
    lp = LongPrefill(device, rank_seed(LONG["seed"], rank))
    pattern = SEARCHED_QUARTER_PATTERN
    for _ in range(args.warmup):
        lp.step(pattern)
    torch.cuda.synchronize()
    status = lp.B.dsa_read_device_status(lp.ws)
    if status != (0, 0):
        raise RuntimeError(f"device status after warm-up: {status}")

    with ClockSampler(device.index) as clocks:
        barrier(world, device)
        torch.cuda.synchronize()
        ms_total = timed(stream, lambda: lp.step(pattern), args.steps)
        barrier(world, device)
    clk = clocks.summary()
    ms_max = max_over_ranks(ms_total, world, device)
    ms_per_step = ms_max / args.steps
    total_pairs = sum_over_ranks(lp.pairs(pattern) * args.steps, world, device)
    value = total_pairs / (ms_max / 1e3)

    # the same step under the other patterns, once each (S layers launch nothing)
    pat = {}
    for name, p in patterns_47().items():
        ms = ms_per_step if p == pattern else timed(stream, lambda: lp.step(p), 1)
        pat[name] = {"f_layers": p.count("F"), "ms": ms}
    all_f = pat["all F"]["ms"]
    for v in pat.values():
        v["speedup_vs_all_f"] = all_f / v["ms"]

    # per indexer layer: the 25 chunk calls of one F layer
    n_full = pattern.count("F")
    layer_ms = ms_per_step / n_full
    flops_layer = 2.0 * lp.H * lp.d * causal_pairs(lp.L)
    achieved = flops_layer / (layer_ms / 1e3) / 1e12
    fp8_peak = peak_tflops(peaks, sustained=True)

    e2e = run_long_e2e(args, world, lp, pattern, stream) if args.e2e_steps > 0 else None
    return lp, {
        "value": value, "ms_per_step": ms_per_step, "clocks": clk, "patterns": pat,
        "gpu_launches": PREFILL_LAUNCHES_PER_CALL * lp.calls(pattern) * args.steps,
        "roofline": {
            "kernel": "dsa_indexer_prefill (sample, threshold, lean, exact-fallback and finish "
                      "launches of the 25 chunk calls of one indexer layer, timed together)",
            "bound": "tensor", "achieved": achieved, "peak": fp8_peak, "unit": "TFLOP/s",
            "frac": achieved / fp8_peak, "traffic": PREFILL_LEAN_TRAFFIC_PER_LAYER,
            "peak_source": f"{peak_kind}: 2 x bf16_tflops_sustained (nominal FP8/BF16 ratio); the "
                           "timed step runs for seconds",
            "algorithmic_per_launch": f"2*H*d*L(L+1)/2 = {flops_layer:.4e} FLOP per indexer layer",
            "launch_ms": layer_ms,
            "traffic_source": PREFILL_LEAN_TRAFFIC_SOURCE},
        "e2e": e2e,
    }


def run_long_e2e(args, world, lp, pattern, stream):
    """The headline step end to end through the public API: every step copies the F layers'
    inputs from pinned host memory to the device and every F layer's index rows back.

    The copies are pipelined with the chunk-major compute, as a serving loop would: chunk c+1's
    query rows and new key rows go up on a copy stream while chunk c is scored (they are rows
    chunk c does not read), and each F layer's index rows of chunk c go down on a second copy
    stream as soon as that layer has run, from one of two alternating sets of per-layer chunk
    buffers (a set is rewritten only after its previous copies have landed). The step ends when
    its last rows are on the host."""
    f_layers = [l for l, c in enumerate(pattern) if c == "F"]
    f_index = {l: j for j, l in enumerate(f_layers)}
    names = ("q", "q_scale", "w", "k", "k_scale")
    host_in = {l: {n: getattr(lp.layers[l], n).cpu().pin_memory() for n in names} for l in f_layers}
    host_out = {l: torch.empty(lp.L, lp.topk, dtype=torch.int32).pin_memory() for l in f_layers}
    h2d = sum(t.numel() * t.element_size() for d in host_in.values() for t in d.values())
    d2h = sum(t.numel() * t.element_size() for t in host_out.values())
    n_chunks, n_full = len(lp.chunks), len(f_layers)
    bufs = [[torch.empty(lp.chunk, lp.topk, dtype=torch.int32, device=lp.device) for _ in range(n_full)]
            for _ in range(2)]
    up, down = torch.cuda.Stream(lp.device), torch.cuda.Stream(lp.device)
    ev_up = [torch.cuda.Event() for _ in range(n_chunks)]
    ev_run = [[torch.cuda.Event() for _ in range(n_full)] for _ in range(n_chunks)]
    ev_down = [[torch.cuda.Event() for _ in range(n_full)] for _ in range(2)]
    used = [False, False]

    def upload(ci):
        c0, c1 = lp.chunks[ci]
        with torch.cuda.stream(up):
            for l in f_layers:
                dev, host = lp.layers[l], host_in[l]
                for n in names:
                    getattr(dev, n)[c0:c1].copy_(host[n][c0:c1], non_blocking=True)
        ev_up[ci].record(up)

    def e2e_step():
        up.wait_stream(stream)  # the previous step's compute still reads these inputs
        used[0] = used[1] = False
        upload(0)
        for ci, (c0, c1) in enumerate(lp.chunks):
            if ci + 1 < n_chunks:
                upload(ci + 1)
            stream.wait_event(ev_up[ci])
            par = ci % 2
            if used[par]:
                for e in ev_down[par]:
                    stream.wait_event(e)
            used[par] = True
            fb = [b[: c1 - c0] for b in bufs[par]]

            def after(l, ptr, ci=ci, c0=c0, c1=c1, par=par, fb=fb):
                if pattern[l] != "F":
                    return
                j = f_index[l]
                ev_run[ci][j].record(stream)
                down.wait_event(ev_run[ci][j])
                with torch.cuda.stream(down):
                    host_out[l][c0:c1].copy_(fb[j], non_blocking=True)
                ev_down[par][j].record(down)

            views = [v if pattern[l] == "F" else None for l, v in enumerate(lp.views[ci])]
            lp.B.indexcache_run(pattern, views, lp.topk, f_bufs=fb, keep_all=True, q_pos0=c0,
                                workspace=lp.ws, after_layer=after)
        stream.wait_stream(down)

    e2e_step()
    torch.cuda.synchronize()
    barrier(world, lp.device)
    ms = max_over_ranks(timed(stream, e2e_step, args.e2e_steps), world, lp.device)
    pairs = sum_over_ranks(lp.pairs(pattern) * args.e2e_steps, world, lp.device)
    # the indices that came back are the device's: spot-check the last chunk of every F layer
    c0, c1 = lp.chunks[-1]
    par = (n_chunks - 1) % 2
    for l in f_layers:
        if not torch.equal(host_out[l][c0:c1], bufs[par][f_index[l]][: c1 - c0].cpu()):
            raise RuntimeError(f"e2e: host copy of layer {l} differs from the device buffer")
    del host_in, host_out, bufs
    return {"value": pairs / (ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "steps": args.e2e_steps,
            "ms_per_step": ms / args.e2e_steps,
            "copies": "pipelined with the compute on two copy streams (pinned host buffers)"}


# DRAM bytes (read + write) of the lean pass (prefill_indexer_kernel<64, 128, 1>, the dominant
# launch) over the 25 chunk calls of one 200000-token indexer layer, from one ncu capture of the
# current kernel and sample stride (dram__bytes_read.sum 2.139e9 + dram__bytes_write.sum
# 4.517e9): q read once (1.64 GB), key tiles re-read per chunk, and the appended candidates written.
PREFILL_LEAN_TRAFFIC_PER_LAYER = 2.139e9 + 4.517e9
PREFILL_LEAN_TRAFFIC_SOURCE = ("ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum of the 25 lean-pass launches "
                               "of one 200000-token layer (all 25 chunks, seed 5), summed; the call's other launches "
                               "add 2.7e10 B, 1.4e10 of them the sample threshold's re-reads")


# ------------------------------------------------------------------------------------------
# the 8-layer 16384-token IndexCache stack with its top-k overlap (extra key)
# ------------------------------------------------------------------------------------------

def run_stack16k(args, world, rank, device, peaks, peak_kind):
    from sparse_attention_token_04_b200 import binding as B
    from synth import correlated_layers
    c = STACK
    L, H, d, topk, pattern = c["L"], c["H"], c["d"], c["topk"], c["pattern"]
    n_full = pattern.count("F")
    stream = torch.cuda.current_stream()
    layers = [lay if pattern[l] == "F" else None for l, lay in
              enumerate(correlated_layers(L, H, d, c["n_layers"], rank_seed(c["seed"], rank), device=device))]
    inputs = [None if l is None else {"q": l.q, "q_scale": l.q_scale, "w": l.w, "k": l.k,
                                      "k_scale": l.k_scale} for l in layers]
    f_bufs = [torch.empty(L, topk, dtype=torch.int32, device=device) for _ in range(n_full)]
    ws = torch.empty(B.dsa_prefill_workspace_bytes(L, H, d, topk), dtype=torch.uint8, device=device)
    B.dsa_workspace_init(ws)
    ov_counts = torch.empty(c["n_layers"], c["n_layers"], dtype=torch.int64, device=device)
    ov_valid = torch.empty(1, dtype=torch.int64, device=device)
    ov = torch.empty(c["n_layers"], c["n_layers"], dtype=torch.float64, device=device)
    ov_ws = torch.zeros(256, dtype=torch.uint8, device=device)
    marks = []

    def on_layer(l, ptr):
        if pattern[l] == "F":
            ev = torch.cuda.Event(enable_timing=True)
            ev.record(stream)
            marks[-1].append(ev)

    def step(record=False):
        if record:
            ev = torch.cuda.Event(enable_timing=True)
            ev.record(stream)
            marks.append([ev])
        _, ptrs = B.indexcache_run(pattern, inputs, topk, f_bufs=f_bufs, workspace=ws,
                                   after_layer=on_layer if record else None)
        B.topk_overlap_ptrs(ptrs, L, topk, L, ov_counts, ov_valid, ov, workspace=ov_ws)
        if record:
            ev = torch.cuda.Event(enable_timing=True)
            ev.record(stream)
            marks[-1].append(ev)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if B.dsa_read_device_status(ws) != (0, 0):
        raise RuntimeError("device status after the 16384-token stack warm-up")
    barrier(world, device)
    ms = max_over_ranks(timed(stream, lambda: step(True), args.stack_steps), world, device)
    pf = [a.elapsed_time(b) for m in marks for a, b in zip(m[:n_full], m[1:n_full + 1])]
    ovm = [m[-2].elapsed_time(m[-1]) for m in marks]
    pf_ms, ov_ms = float(np.mean(pf)), float(np.mean(ovm))
    flops = 2.0 * H * d * causal_pairs(L)
    achieved = flops / (pf_ms / 1e3) / 1e12
    peak = peak_tflops(peaks, sustained=False)
    ov_bytes = c["n_layers"] * L * topk * 4
    pairs = sum_over_ranks(n_full * causal_pairs(L) * args.stack_steps, world, device)
    return {"workload": "IndexCache prefill stack: 8 layers, L=16384, H=64, d=128, k=2048, pattern "
                        "FSFSFSFS (4 indexer layers), rho=0.9 correlated FP8 E4M3 layers, then the "
                        "8x8 top-k overlap",
            "value": pairs / (ms / 1e3), "unit": UNIT, "ms_per_step": ms / args.stack_steps,
            "steps": args.stack_steps,
            "prefill_call": {"launch_ms": pf_ms, "achieved_tflops": achieved, "peak_tflops": peak,
                             "frac": achieved / peak,
                             "peak_source": f"{peak_kind}: 2 x bf16_tflops (burst): a 2 ms call in a "
                                            "short timed loop"},
            "overlap_kernel": {"launch_ms": ov_ms, "bytes_per_launch": ov_bytes,
                               "gbs": ov_bytes / (ov_ms / 1e3) / 1e9,
                               "frac_hbm": ov_bytes / (ov_ms / 1e3) / 1e9 / float(peaks["hbm_gbs"])},
            "gpu_launches": (PREFILL_LAUNCHES_PER_CALL * n_full + 2) * args.stack_steps}


# ------------------------------------------------------------------------------------------
# the 47-layer decode step (extra key)
# ------------------------------------------------------------------------------------------

def run_decode(args, world, rank, device, peaks):
    from sparse_attention_token_04_b200 import binding as B
    from synth import SEARCHED_QUARTER_PATTERN, decode_lengths, paged_decode_layers

    cfg = DECODE
    seed = rank_seed(cfg["seed"], rank)
    lens = decode_lengths(cfg["B"], cfg["lo"], cfg["hi"], seed)
    table, seq, gen = paged_decode_layers(lens, cfg["H"], cfg["d"], cfg["n_layers"], seed, device=device)
    pattern = SEARCHED_QUARTER_PATTERN
    layers = [lay if pattern[l] == "F" else None for l, lay in enumerate(gen)]
    inputs = [None if l is None else {"q": l.q, "q_scale": l.q_scale, "w": l.w, "k_cache": l.k_cache,
                                      "k_scale_cache": l.k_scale_cache} for l in layers]
    n_full = pattern.count("F")
    topk = cfg["topk"]
    f_bufs = [torch.empty(cfg["B"], topk, dtype=torch.int32, device=device) for _ in range(n_full)]
    max_len = table.shape[1] * 64
    ws = torch.empty(B.dsa_decode_workspace_bytes(cfg["B"], max_len, cfg["H"], cfg["d"], topk),
                     dtype=torch.uint8, device=device)
    B.dsa_workspace_init(ws)
    stream = torch.cuda.current_stream()
    marks = []

    def on_layer(l, ptr):
        if pattern[l] == "F":
            ev = torch.cuda.Event(enable_timing=True)
            ev.record(stream)
            marks[-1].append(ev)

    def step(record=False):
        if record:
            ev = torch.cuda.Event(enable_timing=True)
            ev.record(stream)
            marks.append([ev])
        B.indexcache_run(pattern, inputs, topk, mode=B.DSA_MODE_DECODE, f_bufs=f_bufs,
                         block_table=table, seq_lens=seq, workspace=ws,
                         after_layer=on_layer if record else None)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    status = B.dsa_read_device_status(ws)
    if status != (0, 0):
        raise RuntimeError(f"decode device status after warm-up: {status}")
    barrier(world, device)
    ms = max_over_ranks(timed(stream, lambda: step(True), args.decode_steps), world, device)
    keys = sum(lens)
    pairs = sum_over_ranks(keys * n_full * args.decode_steps, world, device)
    per = [a.elapsed_time(b) for evs in marks for a, b in zip(evs[:-1], evs[1:])]
    launch_ms = float(np.mean(per))
    H, d = cfg["H"], cfg["d"]
    bytes_per_launch = (keys * (d + 4) + cfg["B"] * (H * d + 4 * H + 4 + 4)
                        + sum(4 * math.ceil(n / 64) for n in lens) + cfg["B"] * topk * 4)
    gbs = bytes_per_launch / (launch_ms / 1e3) / 1e9
    return {"workload": "IndexCache decode step: 32 requests, one query each, cache lengths "
                        "U[10000,200000], H=64, d=128, k=2048, paged 64-token blocks, 47 layers, "
                        "searched 1/4 pattern (12 indexer layers)",
            "value": pairs / (ms / 1e3), "unit": UNIT, "ms_per_step": ms / args.decode_steps,
            "steps": args.decode_steps, "keys_per_layer": keys,
            "roofline": {"kernel": "dsa_indexer_decode (decode_clear_kernel + decode_indexer_kernel + "
                                   "decode_collect_kernel + decode_rank_kernel)",
                         "bound": "hbm", "achieved": gbs, "peak": float(peaks["hbm_gbs"]),
                         "unit": "GB/s", "frac": gbs / float(peaks["hbm_gbs"]),
                         "traffic": (None if DECODE_SCORING_DRAM_BYTES_PER_KEY is None
                                     else DECODE_SCORING_DRAM_BYTES_PER_KEY * keys),
                         "traffic_source": DECODE_TRAFFIC_SOURCE,
                         "algorithmic_per_launch": f"{bytes_per_launch} B (d+4 per key + per-request "
                                                   "q/w/scale/table/out)",
                         "launch_ms": launch_ms},
            "gpu_launches": DECODE_LAUNCHES_PER_CALL * n_full * args.decode_steps}


def run_mli_decode(args, world, rank, device, peaks):
    """The 47-layer decode step with the sparse-attention consumer on every layer, under plain
    IndexCache and under the lagged multi-layer-indexer mode at the same retention (searched 1/4
    pattern). The consumer is dsa_sparse_attention_decode: 128 query heads over the 2048 selected
    rows of a 576-wide bf16 latent cache (one cache shared by all layers, the indexer's paged
    layout), values the first 512 entries. Plain: each layer's consumer follows its own indexer on
    one stream. Lagged: every Full layer's indexer runs on a second stream while the consumers read
    the previous indexer layer's selection. The consumer alone is also timed, with its roofline."""
    from sparse_attention_token_04_b200 import binding as B
    from synth import SEARCHED_QUARTER_PATTERN, decode_lengths, paged_decode_layers

    cfg = DECODE
    seed = rank_seed(cfg["seed"], rank)
    lens = decode_lengths(cfg["B"], cfg["lo"], cfg["hi"], seed)
    table, seq, gen = paged_decode_layers(lens, cfg["H"], cfg["d"], cfg["n_layers"], seed, device=device)
    pattern = SEARCHED_QUARTER_PATTERN
    layers = [lay if pattern[l] == "F" else None for l, lay in enumerate(gen)]
    inputs = [None if l is None else {"q": l.q, "q_scale": l.q_scale, "w": l.w, "k_cache": l.k_cache,
                                      "k_scale_cache": l.k_scale_cache} for l in layers]
    topk, Bn, heads, dkv, dv = cfg["topk"], cfg["B"], 128, 576, 512
    n_slots = int(layers[0].k_cache.shape[0]) * 64
    g = torch.Generator(device=device)
    g.manual_seed(seed + 7)
    latent = torch.randn(n_slots, dkv, generator=g, device=device).to(torch.bfloat16)
    q_att = torch.randn(Bn, heads, dkv, generator=g, device=device).to(torch.bfloat16)
    scale = 1.0 / math.sqrt(dkv)
    bufs = [torch.empty(Bn, topk, dtype=torch.int32, device=device) for _ in range(2)]
    by_ptr = {b.data_ptr(): b for b in bufs}
    ws = torch.empty(B.dsa_decode_workspace_bytes(Bn, table.shape[1] * 64, cfg["H"], cfg["d"], topk),
                     dtype=torch.uint8, device=device)
    B.dsa_workspace_init(ws)
    att_ws = torch.empty(B.dsa_sparse_attention_workspace_bytes(Bn, topk), dtype=torch.uint8, device=device)
    B.dsa_workspace_init(att_ws)
    att_out = torch.empty(Bn, heads, dv, dtype=torch.float32, device=device)
    side = torch.cuda.Stream(device=device)
    stream = torch.cuda.current_stream()

    def consume(l, ptr):
        B.dsa_sparse_attention_decode(q_att, latent, table, seq, by_ptr[ptr], scale, out=att_out,
                                      workspace=att_ws)

    def plain():
        B.indexcache_run(pattern, inputs, topk, mode=B.DSA_MODE_DECODE, f_bufs=bufs[:1],
                         block_table=table, seq_lens=seq, workspace=ws, after_layer=consume)

    def lagged():
        B.indexcache_run_lagged(pattern, inputs, topk, side, mode=B.DSA_MODE_DECODE, f_bufs=bufs,
                                block_table=table, seq_lens=seq, workspace=ws, consume=consume)

    def consumers_only():
        for l in range(len(pattern)):
            consume(l, bufs[0].data_ptr())

    res = {}
    for name, fn in (("plain", plain), ("lagged", lagged), ("consumers_only", consumers_only)):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        res[name] = timed(stream, fn, args.mli_steps) / args.mli_steps
    # The consumer alone, L2 flushed (a 256 MiB write) before every call, each call timed by
    # its own events on the launching stream.
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    pairs = []
    for _ in range(max(args.mli_steps, 1) * 10):
        flush.zero_()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        consume(0, bufs[0].data_ptr())
        e1.record(stream)
        pairs.append((e0, e1))
    torch.cuda.synchronize()
    call_ms = sum(a.elapsed_time(b) for a, b in pairs) / len(pairs)
    del flush
    if B.dsa_read_device_status(ws) != (0, 0) or B.dsa_read_device_status(att_ws) != (0, 0):
        raise RuntimeError("device status after the lagged decode steps")
    att_bytes = Bn * topk * dkv * 2 + Bn * heads * dkv * 2 + Bn * heads * dv * 4 + Bn * topk * 4
    att_flop = 2.0 * Bn * heads * topk * (dkv + dv)
    gbs = att_bytes / (call_ms / 1e3) / 1e9
    tflops = att_flop / (call_ms / 1e3) / 1e12
    bf16_peak = float(peaks["bf16_tflops"])
    return {"workload": "47-layer decode step, 32 requests U[10000,200000], searched 1/4 pattern (12 "
                        "indexer layers), the sparse-attention consumer (dsa_sparse_attention_decode: 128 "
                        "heads over the 2048 selected rows of a 576-wide bf16 latent cache) on every layer",
            "plain_indexcache_ms": res["plain"], "lagged_mli_ms": res["lagged"],
            "consumers_alone_ms": res["consumers_only"],
            "speedup_lagged_vs_plain": res["plain"] / res["lagged"], "steps": args.mli_steps,
            "attention_call": {
                "kernel": "attention_split_kernel + attention_combine_kernel",
                "launch_ms": call_ms, "timing": f"{len(pairs)} calls, L2 flushed before each", "bound": "hbm",
                "algorithmic_per_launch": f"{att_bytes} B (2048 selected 1152-byte latent rows per request, "
                                          f"q, out, indices); {att_flop:.4e} FLOP",
                "achieved": gbs, "peak": float(peaks["hbm_gbs"]), "unit": "GB/s",
                "frac": gbs / float(peaks["hbm_gbs"]),
                "tflops": tflops, "tflops_frac_of_bf16_burst": tflops / bf16_peak}}


# DRAM bytes (read + write) per cached key of decode_indexer_kernel from one ncu capture of this
# workload, or None when the kernel changed after the capture.
DECODE_SCORING_DRAM_BYTES_PER_KEY = 5.019e8 / 3737801
DECODE_TRAFFIC_SOURCE = ("decode_indexer_kernel DRAM read+write per cached key from one ncu capture "
                         "of this workload (SpeedOfLight/MemoryWorkloadAnalysis sections), times the "
                         "keys of one launch")


# ------------------------------------------------------------------------------------------
# CPU baseline: the oracle on sampled rows of the same workload
# ------------------------------------------------------------------------------------------

def cpu_baseline_long(lp, seconds):
    """The C++ oracle, as it stands, on uniformly drawn query rows of the first indexer layer of
    the headline workload: single-threaded (the plain oracle) for half the time, then the same
    per-row function on nproc threads over rows. Every row it computes is also compared with
    the GPU's row."""
    import oracle.cpp_oracle as C
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from parity import check_row
    from sparse_attention_token_04_b200 import binding as B

    lay = lp.layers[0]
    k_h, ks_h = lay.k.cpu().numpy(), lay.k_scale.cpu().numpy()
    rng = np.random.default_rng(0)
    rows = sorted({int(t) for t in rng.integers(0, lp.L, size=2048)})
    gpu = {}
    out = torch.empty(lp.chunk, lp.topk, dtype=torch.int32, device=lp.device)
    for c0, c1 in lp.chunks:
        want = [t for t in rows if c0 <= t < c1]
        if not want:
            continue
        B.dsa_indexer_prefill(lay.q[c0:c1], lay.q_scale[c0:c1], lay.w[c0:c1], lay.k[:c1],
                              lay.k_scale[:c1], lp.topk, q_pos0=c0, out_idx=out[: c1 - c0],
                              want_score=False, workspace=lp.ws)
        sel = out[torch.tensor([t - c0 for t in want], device=lp.device)].cpu().numpy()
        for i, t in enumerate(want):
            gpu[t] = sel[i]
    order = [int(t) for t in rng.permutation(rows)]
    pos_all = torch.tensor(order, device=lp.device)
    q_h = lay.q[pos_all].cpu().numpy()
    qs_h = lay.q_scale[pos_all].cpu().numpy()
    w_h = lay.w[pos_all].cpu().numpy()
    nproc = os.cpu_count() or 1

    def run(first, count, threads):
        sl = slice(first, first + count)
        res = C.prefill_positions(q_h[sl], qs_h[sl], w_h[sl], k_h, ks_h, order[sl], lp.topk,
                                  n_threads=threads)
        for r in res:
            check_row(gpu[r.t], None, r, lp.topk)
        return sum(r.t + 1 for r in res)

    nxt = 0
    res = {}
    for name, threads, batch in (("single", 1, 1), ("all", nproc, nproc)):
        pairs = n = 0
        t0 = time.perf_counter()
        while nxt + batch <= len(order) and time.perf_counter() - t0 < seconds / 2:
            pairs += run(nxt, batch, threads)
            nxt += batch
            n += batch
        res[name] = (pairs, n, time.perf_counter() - t0)
    p1, n1, e1 = res["single"]
    pa, na, ea = res["all"]
    step_pairs = 12 * causal_pairs(lp.L)
    return {"value": p1 / e1, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"{n1} uniformly drawn query rows of indexer layer 0 of the 200000-token "
                      f"workload ({p1} causal pairs, {e1:.1f} s) through the plain single-threaded "
                      "C++ oracle; the GPU's rows checked against it",
            "all_cores": {"value": pa / ea, "unit": UNIT, "cores": nproc,
                          "sample": f"{na} more rows ({pa} pairs, {ea:.1f} s), the same per-row "
                                    f"oracle on {nproc} threads over rows; checked the same way"},
            "host_nproc": nproc,
            "extrapolated_step_s": {
                "single": extrapolated_seconds(step_pairs, p1, e1),
                "all_cores": extrapolated_seconds(step_pairs, pa, ea),
                "note": "one step of the headline workload (12 indexer layers x L(L+1)/2 causal pairs) "
                        "at the sampled rates: extrapolated, not run (a row's cost grows with its "
                        "position, and the rows are uniformly drawn)"}}


def extrapolated_seconds(total_pairs, sampled_pairs, sampled_seconds):
    """Seconds for total_pairs at the rate of a sample (None for an empty sample)."""
    if sampled_pairs <= 0 or sampled_seconds <= 0:
        return None
    return total_pairs * sampled_seconds / sampled_pairs


# ------------------------------------------------------------------------------------------
# our implementation
# ------------------------------------------------------------------------------------------

def run_ours(args, world, rank, local):
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    init_dist(world, "nccl")
    peaks, peak_kind = measured_peaks()

    lp, long = run_long(args, world, rank, device, peaks, peak_kind)
    cpu = None
    if rank == 0 and world == 1 and args.cpu_seconds > 0:
        cpu = cpu_baseline_long(lp, args.cpu_seconds)
    del lp
    torch.cuda.empty_cache()
    stack = run_stack16k(args, world, rank, device, peaks, peak_kind) if args.stack_steps > 0 else None
    decode = run_decode(args, world, rank, device, peaks) if args.decode_steps > 0 else None
    mli = run_mli_decode(args, world, rank, device, peaks) if args.mli_steps > 0 else None

    if rank == 0:
        c = LONG
        line = {
            "metric": METRIC, "value": long["value"], "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": long["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "fp8_e4m3", "data": "synthetic",
            "config": {"workload": "200000-token prefill through 47 layers, searched 1/4 IndexCache "
                                   "pattern (12 indexer layers), H=64, d=128, k=2048, rho=0.9 "
                                   "correlated FP8 E4M3 layers, chunks of 8192 queries (chunk-major: "
                                   "each chunk through all layers via one indexcache_run)",
                       "L": c["L"], "H": c["H"], "d": c["d"], "topk": c["topk"],
                       "n_layers": c["n_layers"], "chunk": c["chunk"],
                       "pattern": patterns_47()["searched 1/4"],
                       "pairs_per_step_per_gpu": 12 * causal_pairs(c["L"]),
                       "l2": "inputs larger than L2 (12 x 1.64 GB of q read per step)",
                       "parallelism": f"independent workload per GPU x{world}"},
            "roofline": long["roofline"],
            "patterns": long["patterns"],
            "gpu_launches": long["gpu_launches"] + (stack["gpu_launches"] if stack else 0)
            + (decode["gpu_launches"] if decode else 0),
            "clocks": long["clocks"],
            "e2e": long["e2e"],
            "stack_16k": stack,
            "decode": decode,
            "mli_decode": mli,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------------------
# reference arm: the oracle
# ------------------------------------------------------------------------------------------

def run_reference(args, world, rank):
    """The C++ oracle on the host cores (nproc threads over rows), on uniformly drawn query
    rows of the headline workload's shape: each step scores ref_rows rows at uniformly drawn
    positions of a 200000-key layer. The oracle's cost per row depends only on its position."""
    if rank != 0:
        return
    import oracle.cpp_oracle as C
    from synth import gaussian_layer

    c = LONG
    L, H, d, topk = c["L"], c["H"], c["d"], c["topk"]
    rng = np.random.default_rng(1)
    keys = gaussian_layer(L, 1, d, seed=c["seed"])
    pool = gaussian_layer(256, H, d, seed=c["seed"] + 1)
    k_h, ks_h = keys.k.numpy(), keys.k_scale.numpy()
    qp, qsp, wp = pool.q.numpy(), pool.q_scale.numpy(), pool.w.numpy()
    nproc = os.cpu_count() or 1
    rows_per_step = args.ref_rows if args.ref_rows > 0 else nproc

    def step():
        pos = rng.integers(0, L, size=rows_per_step)
        pick = rng.integers(0, qp.shape[0], size=rows_per_step)
        C.prefill_positions(qp[pick], qsp[pick], wp[pick], k_h, ks_h, pos, topk, n_threads=nproc,
                            want_scores=False)
        return int((pos + 1).sum())

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    pairs = 0
    for _ in range(args.steps):
        pairs += step()
    el = time.perf_counter() - t0
    value = pairs / el
    sample = f"{args.steps} steps x {rows_per_step} uniformly drawn query rows, C++ oracle on {nproc} threads"
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": el * 1e3 / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": "200000-token prefill through 47 layers, searched 1/4 IndexCache "
                                   "pattern (12 indexer layers), H=64, d=128, k=2048, chunks of 8192",
                       "sample": sample},
            "cpu_baseline": {"value": value, "unit": UNIT, "kind": "oracle", "cores": nproc,
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=2)
    ap.add_argument("--stack-steps", type=int, default=20)
    ap.add_argument("--decode-steps", type=int, default=20)
    ap.add_argument("--mli-steps", type=int, default=10)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-rows", type=int, default=0, help="rows per reference step (0: nproc)")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("at least 3 warm-up steps")
    world, rank, local = dist_env()
    if world != args.gpus:
        if world == 1 and args.gpus > 1:
            raise SystemExit("launch N > 1 with torch.distributed.run (one process per GPU)")
    if args.impl == "reference":
        run_reference(args, world, rank)
        return
    try:
        run_ours(args, world, rank, local)
    finally:
        if world > 1 and torch.distributed.is_initialized():
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
