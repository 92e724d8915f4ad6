"""Benchmark of the lightning-indexer hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    python -m torch.distributed.run --nnodes=1 --nproc-per-node N --master-addr 127.0.0.1 \
        --master-port P bench.py --gpus N ...

One step = one pass of the whole hot path over one synthetic batch: the 8-layer IndexCache
prefill stack (L = 16384 tokens, H = 64 heads, d = 128, top-k = 2048, pattern FSFSFSFS, layer
inputs correlated with rho = 0.9), i.e. four fused prefill indexer launches with streaming
top-k whose index buffers the four Shared layers alias, followed by the 8 x 8 top-k overlap
of all eight layers. Inputs are generated on the device before timing; at N > 1 every rank
runs its own independent stack (weak scaling, no collective on the data path).

The decode workload (32 requests, cache lengths uniform in [10000, 200000], 47 layers with
the searched 1/4 pattern = 12 indexer layers, paged 64-token blocks) is timed in the same run
and reported under "decode". The CPU baseline is the oracle on a bounded sample of rows.

`--impl reference` times the oracle (the only reference implementation there is) on the same
workload, a bounded sample of rows per step, on the host cores.
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

PREFILL = dict(L=16384, H=64, d=128, topk=2048, n_layers=8, pattern="FSFSFSFS", seed=2)
DECODE = dict(B=32, lo=10000, hi=200000, H=64, d=128, topk=2048, n_layers=47, seed=4)

FP8_PER_BF16 = 2.0  # nominal dense FP8 / BF16 tensor throughput ratio on B200


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


# ------------------------------------------------------------------------------------------
# workloads
# ------------------------------------------------------------------------------------------

def make_prefill_stack(device, seed):
    from synth import correlated_layers
    cfg = PREFILL
    layers = []
    for l, lay in enumerate(correlated_layers(cfg["L"], cfg["H"], cfg["d"], cfg["n_layers"], seed,
                                              device=device)):
        layers.append(lay if cfg["pattern"][l] == "F" else None)
    return layers


def make_decode_stack(device, seed):
    from synth import SEARCHED_QUARTER_PATTERN, decode_lengths, paged_decode_layers
    cfg = DECODE
    lens = decode_lengths(cfg["B"], cfg["lo"], cfg["hi"], seed)
    table, seq, gen = paged_decode_layers(lens, cfg["H"], cfg["d"], cfg["n_layers"], seed, device=device)
    layers = []
    for l, lay in enumerate(gen):
        layers.append(lay if SEARCHED_QUARTER_PATTERN[l] == "F" else None)
    return lens, table, seq, layers


def prefill_dicts(layers):
    return [None if l is None else {"q": l.q, "q_scale": l.q_scale, "w": l.w, "k": l.k,
                                    "k_scale": l.k_scale} for l in layers]


def decode_dicts(layers):
    return [None if l is None else {"q": l.q, "q_scale": l.q_scale, "w": l.w, "k_cache": l.k_cache,
                                    "k_scale_cache": l.k_scale_cache} for l in layers]


# ------------------------------------------------------------------------------------------
# our implementation
# ------------------------------------------------------------------------------------------

def run_ours(args, world, rank, local):
    from sparse_attention_token_04_b200 import binding as B

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    init_dist(world, "nccl")
    cfg = PREFILL
    L, H, d, topk, pattern = cfg["L"], cfg["H"], cfg["d"], cfg["topk"], cfg["pattern"]
    n_full = pattern.count("F")
    stream = torch.cuda.current_stream()

    layers = make_prefill_stack(device, rank_seed(cfg["seed"], rank))
    inputs = prefill_dicts(layers)
    f_bufs = [torch.empty(L, topk, dtype=torch.int32, device=device) for _ in range(n_full)]
    shape_ws = B.dsa_prefill_workspace_bytes(L, H, d, topk)
    ws = torch.empty(shape_ws, dtype=torch.uint8, device=device)
    B.dsa_workspace_init(ws)
    ov_counts = torch.empty(cfg["n_layers"], cfg["n_layers"], dtype=torch.int64, device=device)
    ov_valid = torch.empty(1, dtype=torch.int64, device=device)
    ov = torch.empty(cfg["n_layers"], cfg["n_layers"], dtype=torch.float64, device=device)
    ov_ws = torch.zeros(256, dtype=torch.uint8, device=device)

    layer_events = []

    def on_layer(l, ptr):
        if pattern[l] == "F" and layer_events is not None:
            ev = torch.cuda.Event(enable_timing=True)
            ev.record(stream)
            layer_events[-1].append(ev)

    def step(record=False):
        if record:
            ev0 = torch.cuda.Event(enable_timing=True)
            ev0.record(stream)
            layer_events.append([ev0])
        _, ptrs = B.indexcache_run(pattern, inputs, topk, f_bufs=f_bufs, workspace=ws,
                                   after_layer=on_layer if record else None)
        if record:
            evo = torch.cuda.Event(enable_timing=True)
            evo.record(stream)
        B.topk_overlap_ptrs(ptrs, L, topk, L, ov_counts, ov_valid, ov, workspace=ov_ws)
        if record:
            eve = torch.cuda.Event(enable_timing=True)
            eve.record(stream)
            layer_events[-1].extend([evo, eve])

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    status = B.dsa_read_device_status(ws)
    if status != (0, 0):
        raise RuntimeError(f"device status after warm-up: {status}")

    pairs_per_step = n_full * causal_pairs(L)
    # per prefill call: sample pass, sample threshold, lean pass, exact pass (exits at once when
    # no block needs it), finish; then the two overlap kernels
    launches_per_step = n_full * 5 + 2
    with ClockSampler(local) as clocks:
        barrier(world, device)
        torch.cuda.synchronize()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(args.steps):
            step(record=True)
        t1.record(stream)
        torch.cuda.synchronize()
        barrier(world, device)
    clk = clocks.summary()
    ms_total = t0.elapsed_time(t1)
    ms_max = max_over_ranks(ms_total, world, device)
    ms_per_step = ms_max / args.steps

    # per-launch times of the prefill indexer call and of the overlap
    pf_ms, ov_ms = [], []
    for evs in layer_events:
        marks = evs[:-2]
        for a, b in zip(marks[:-1], marks[1:]):
            pf_ms.append(a.elapsed_time(b))
        ov_ms.append(evs[-2].elapsed_time(evs[-1]))
    pf_avg = float(np.mean(pf_ms))
    ov_avg = float(np.mean(ov_ms))

    total_pairs = sum_over_ranks(pairs_per_step * args.steps, world, device)
    value = total_pairs / (ms_max / 1e3)

    peaks, peak_kind = measured_peaks()
    fp8_peak = FP8_PER_BF16 * float(peaks["bf16_tflops_sustained"])
    flops_per_launch = 2.0 * H * d * causal_pairs(L)
    achieved_tflops = flops_per_launch / (pf_avg / 1e3) / 1e12
    ov_bytes = cfg["n_layers"] * L * topk * 4
    ov_gbs = ov_bytes / (ov_avg / 1e3) / 1e9

    # end to end through the public API with host buffers (pinned), copies timed
    e2e = None
    if args.e2e_steps > 0:
        host_inputs = []
        for lay in inputs:
            host_inputs.append(None if lay is None else
                               {k: v.cpu().pin_memory() for k, v in lay.items()})
        host_out = [torch.empty(L, topk, dtype=torch.int32).pin_memory() for _ in range(n_full)]
        host_ov = torch.empty(cfg["n_layers"], cfg["n_layers"], dtype=torch.float64).pin_memory()
        h2d = sum(v.numel() * v.element_size() for lay in host_inputs if lay for v in lay.values())
        d2h = sum(t.numel() * t.element_size() for t in host_out) + host_ov.numel() * 8

        def e2e_step():
            for lay, hl in zip(inputs, host_inputs):
                if lay is not None:
                    for k in lay:
                        lay[k].copy_(hl[k], non_blocking=True)
            _, ptrs = B.indexcache_run(pattern, inputs, topk, f_bufs=f_bufs, workspace=ws)
            B.topk_overlap_ptrs(ptrs, L, topk, L, ov_counts, ov_valid, ov, workspace=ov_ws)
            for hb, db in zip(host_out, f_bufs):
                hb.copy_(db, non_blocking=True)
            host_ov.copy_(ov, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        barrier(world, device)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(world, device)
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, device)
        e2e_pairs = sum_over_ranks(pairs_per_step * args.e2e_steps, world, device)
        e2e = {"value": e2e_pairs / (e2e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h), "steps": args.e2e_steps,
               "ms_per_step": e2e_ms / args.e2e_steps}
        del host_inputs, host_out

    decode = run_decode(args, world, rank, device, peaks) if args.decode_steps > 0 else None

    cpu = None
    if rank == 0 and world == 1 and args.cpu_seconds > 0:
        cpu = cpu_baseline_prefill(layers, f_bufs, args.cpu_seconds)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "fp8_e4m3", "data": "synthetic",
            "config": {"workload": "IndexCache prefill stack: 8 layers, L=16384, H=64, d=128, "
                                   "k=2048, pattern FSFSFSFS (4 indexer layers), rho=0.9 "
                                   "correlated FP8 E4M3 layers, then the 8x8 top-k overlap",
                       "L": L, "H": H, "d": d, "topk": topk, "n_layers": cfg["n_layers"],
                       "pattern": pattern, "pairs_per_step_per_gpu": pairs_per_step,
                       "l2": "inputs larger than L2 (4 x 134 MB of q read per step)",
                       "parallelism": f"independent stack per GPU x{world}"},
            "roofline": {"kernel": "dsa_indexer_prefill (sample, threshold, lean, exact-fallback and "
                                   "finish launches, timed together)",
                         "bound": "tensor", "achieved": achieved_tflops, "peak": fp8_peak,
                         "unit": "TFLOP/s", "frac": achieved_tflops / fp8_peak, "traffic": None,
                         "peak_source": f"{peak_kind}: 2 x bf16_tflops_sustained (nominal FP8/BF16 ratio)",
                         "algorithmic_per_launch": f"2*H*d*L(L+1)/2 = {flops_per_launch:.4e} FLOP",
                         "launch_ms": pf_avg},
            "overlap_kernel": {"launch_ms": ov_avg, "bytes_per_launch": ov_bytes, "gbs": ov_gbs,
                               "frac_hbm": ov_gbs / float(peaks["hbm_gbs"])},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clk,
            "e2e": e2e,
            "decode": decode,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)


def run_decode(args, world, rank, device, peaks):
    from sparse_attention_token_04_b200 import binding as B
    from synth import SEARCHED_QUARTER_PATTERN

    cfg = DECODE
    lens, table, seq, layers = make_decode_stack(device, rank_seed(cfg["seed"], rank))
    inputs = decode_dicts(layers)
    pattern = SEARCHED_QUARTER_PATTERN
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
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.decode_steps):
        step(record=True)
    t1.record(stream)
    torch.cuda.synchronize()
    barrier(world, device)
    ms = max_over_ranks(t0.elapsed_time(t1), world, device)
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
            "roofline": {"kernel": "dsa_indexer_decode (decode_indexer_kernel + decode_collect_kernel + decode_rank_kernel)",
                         "bound": "hbm", "achieved": gbs, "peak": float(peaks["hbm_gbs"]),
                         "unit": "GB/s", "frac": gbs / float(peaks["hbm_gbs"]),
                         "traffic": DECODE_SCORING_DRAM_BYTES_PER_KEY * keys,
                         "traffic_source": "decode_indexer_kernel DRAM read+write per cached key from one ncu "
                                           "capture of this workload (SpeedOfLight/MemoryWorkloadAnalysis "
                                           "sections), times the keys of one launch",
                         "algorithmic_per_launch": f"{bytes_per_launch} B (d+4 per key + per-request q/w/scale/table/out)",
                         "launch_ms": launch_ms},
            "gpu_launches": 3 * n_full * args.decode_steps}


# DRAM bytes (read + write) per cached key of decode_indexer_kernel, from one ncu capture of the
# decode workload (32 requests, lengths U[10000, 200000]): 5.694 TB/s x 88.416 us = 5.034e8 B
# over 3,737,801 keys (132 B of key and scale per key are algorithmic; the rest is the scores it
# writes). Valid for the kernel as captured; a change to it makes this figure stale.
DECODE_SCORING_DRAM_BYTES_PER_KEY = 5.034e8 / 3737801


def cpu_baseline_prefill(layers, f_bufs, seconds):
    """The oracle, as it stands, on sampled rows of the first F layer; checks those rows of
    the GPU output on the way."""
    import oracle.dsa_oracle as O
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from parity import check_row

    lay = layers[0].numpy()
    L, topk = PREFILL["L"], PREFILL["topk"]
    gpu = f_bufs[0].cpu().numpy()
    rng = np.random.default_rng(0)
    pairs = 0
    rows = 0
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < seconds:
        t = int(rng.integers(0, L))
        r = O.prefill_rows(lay, topk, [t])[0]
        check_row(gpu[t], None, r, topk)
        pairs += t + 1
        rows += 1
    el = time.perf_counter() - t0
    return {"value": pairs / el, "unit": UNIT, "cores": numpy_threads(), "kind": "oracle",
            "sample": f"{rows} uniformly drawn query rows of indexer layer 0 of the same stack "
                      f"({pairs} causal pairs, {el:.1f} s); GPU rows checked against it",
            "host_nproc": os.cpu_count()}


# ------------------------------------------------------------------------------------------
# reference arm: the oracle
# ------------------------------------------------------------------------------------------

def run_reference(args, world, rank):
    if rank != 0:
        return
    import oracle.dsa_oracle as O
    from synth import correlated_layers

    cfg = PREFILL
    L, H, d, topk = cfg["L"], cfg["H"], cfg["d"], cfg["topk"]
    layer = next(iter(correlated_layers(L, H, d, 1, cfg["seed"], device="cpu"))).numpy()
    rng = np.random.default_rng(1)
    rows_per_step = args.ref_rows

    def step():
        n = 0
        for t in rng.integers(0, L, size=rows_per_step):
            O.prefill_rows(layer, topk, [int(t)])
            n += int(t) + 1
        return n

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    pairs = 0
    for _ in range(args.steps):
        pairs += step()
    el = time.perf_counter() - t0
    value = pairs / el
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": el * 1e3 / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": "IndexCache prefill stack: 8 layers, L=16384, H=64, d=128, "
                                   "k=2048, pattern FSFSFSFS (4 indexer layers), rho=0.9 "
                                   "correlated FP8 E4M3 layers, then the 8x8 top-k overlap",
                       "sample": f"{rows_per_step} uniformly drawn query rows of an indexer layer per step"},
            "cpu_baseline": {"value": value, "unit": UNIT, "kind": "oracle", "cores": numpy_threads(),
                             "sample": f"{args.steps} steps x {rows_per_step} query rows"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_long_prefill_patterns(args, local):
    """Long-context prefill under several IndexCache patterns: L = 200000, H = 64, d = 128,
    k = 2048, 47 rho = 0.9 correlated layers, chunks of 8192 queries against the whole causal
    prefix. Every layer's indexer pass (all 25 chunks) is timed once with CUDA events; an F/S
    pattern runs exactly its F layers (S layers alias their F buffer: no launch), so its wall
    time is the sum over its F layers. Prints one JSON line."""
    from sparse_attention_token_04_b200 import binding as B
    from synth import SEARCHED_QUARTER_PATTERN, correlated_layers

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    L, H, d, topk, n_layers, chunk = 200000, 64, 128, 2048, 47, 8192
    patterns = {
        "searched 1/4 (12 F)": SEARCHED_QUARTER_PATTERN,
        "all F (47 F)": "F" * n_layers,
        "FFFS (36 F)": ("FFFS" * 12)[:n_layers],
        "FSSS (12 F)": ("FSSS" * 12)[:n_layers],
    }
    ws = torch.empty(B.dsa_prefill_workspace_bytes(chunk, H, d, topk), dtype=torch.uint8, device=device)
    B.dsa_workspace_init(ws)
    out_idx = torch.empty(chunk, topk, dtype=torch.int32, device=device)
    stream = torch.cuda.current_stream()
    layer_ms = []
    for layer in correlated_layers(L, H, d, n_layers, seed=5, device=device):
        def one_pass():
            for c0 in range(0, L, chunk):
                c1 = min(L, c0 + chunk)
                B.dsa_indexer_prefill(layer.q[c0:c1], layer.q_scale[c0:c1], layer.w[c0:c1],
                                      layer.k[:c1], layer.k_scale[:c1], topk, q_pos0=c0,
                                      out_idx=out_idx[: c1 - c0], want_score=False, workspace=ws)
        if not layer_ms:
            one_pass()  # warm-up
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        one_pass()
        e1.record(stream)
        torch.cuda.synchronize()
        layer_ms.append(e0.elapsed_time(e1))
    status = B.dsa_read_device_status(ws)
    pairs = causal_pairs(L)
    flops = 2.0 * H * d * pairs
    peaks, _ = measured_peaks()
    fp8_peak = FP8_PER_BF16 * float(peaks["bf16_tflops_sustained"])
    res = {}
    for name, pat in patterns.items():
        f_layers = [i for i, c in enumerate(pat) if c == "F"]
        ms = float(sum(layer_ms[i] for i in f_layers))
        res[name] = {"f_layers": len(f_layers), "ms": ms,
                     "speedup_vs_all_f": float(sum(layer_ms)) / ms}
    mean_ms = float(np.mean(layer_ms))
    line = {"workload": "long-context prefill: L=200000, H=64, d=128, k=2048, 47 rho=0.9 "
                        "correlated FP8 layers, chunks of 8192 queries", "device_status": list(status),
            "per_layer_ms": {"mean": mean_ms, "min": float(min(layer_ms)), "max": float(max(layer_ms))},
            "per_layer_pairs_per_s": pairs / (mean_ms / 1e3),
            "per_layer_tflops": flops / (mean_ms / 1e3) / 1e12,
            "per_layer_frac_fp8": flops / (mean_ms / 1e3) / 1e12 / fp8_peak,
            "patterns": res}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--decode-steps", type=int, default=50)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-rows", type=int, default=8)
    ap.add_argument("--long-prefill-patterns", action="store_true",
                    help="time the 200000-token, 47-layer prefill under four F/S patterns instead")
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
    if args.long_prefill_patterns:
        run_long_prefill_patterns(args, local)
        return
    try:
        run_ours(args, world, rank, local)
    finally:
        if world > 1 and torch.distributed.is_initialized():
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
