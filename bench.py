#!/usr/bin/env python
"""Throughput of the routed-MoE FFN step on B200, one JSON line on rank 0.

Default workload: decode, one layer, one token per step (hidden 2048, 512
routed experts + 1 shared, intermediate 768, top-10, int4 group-32 experts,
Zipf(1.1) router prior, 200 fresh seeded tokens). A step is one full pass of
the step (route -> dispatch -> experts -> combine) over that step's token.

Timing: W untimed warm-up steps, then K timed steps. Every step is bracketed
by its own pair of CUDA events on the launching stream; between steps a
2 x L2-sized buffer is overwritten (outside the event pairs) so every step
streams its expert weights from HBM rather than L2. SM clocks and throttle
reasons are sampled during the timed region; a region that saw a slowdown
reason (or clocks held low with none) is run once more and the second run is
reported. Multi-GPU (torchrun):
every rank runs an independent replica on its own token stream (weak
scaling, no collective in the data path); the reported time is the max over
ranks.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload decode1]
    python bench.py --impl reference ...   # the fp64 CPU oracle on the host cores
"""
from __future__ import annotations

import argparse
import csv
import io
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from bit_quantized_moe_gemv_b200 import workload as wlm  # noqa: E402

METRIC = "MoE-layer tokens/s (decode b=1..4, 8K prefill); % of HBM / tensor roofline"
LEAD_CYCLES = 200000  # ~0.1 ms spin before each timed step (outside its events)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM bytes (read + write) per launch of the dominant kernel(s), from the ncu
# captures summarised in profiles/ (None while no capture of the current
# kernel exists).
NCU_TRAFFIC = {
    # decode_fused_kernel of one step (dram read + write of one launch)
    "decode1": (34066688, "profiles/decode_fused_decode1.md"),
    # gather_rows + predequant + the wide-tile, the dequantising and the
    # mma.sync GEMMs (gate/up and down) of one moe_expert_ffn call (the
    # launches the prefill roofline times)
    "prefill8k": (2759788032, "profiles/grouped_gemm_prefill8k.md"),
}


def max_over_ranks(x, world, device):
    """The largest value of x over all ranks: a job's time is its slowest
    rank's (collective on the ranks' process group; a no-op at N = 1)."""
    if world <= 1:
        return x
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def ncu_traffic(workload):
    t = NCU_TRAFFIC.get(workload)
    return (t[0], t[1]) if t else (None, None)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="decode1",
                    choices=["decode1", "verify4", "decode48", "prefill8k", "prefill32k"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="bound on each CPU-baseline sample")
    ap.add_argument("--no-graph", action="store_true", help="decode48: plain launches instead of a CUDA graph")
    ap.add_argument("--headline-only", action="store_true",
                    help="decode1 only (by default the decode1 line also carries prefill8k and decode48 results)")
    ap.add_argument("--clock-window", type=float, default=1.2,
                    help="seconds of back-to-back steps around the timed region while clocks are sampled")
    return ap.parse_args()


def workload_config(wl, world=1):
    """The `config` object of the JSON line (identical for both arms)."""
    q = {wlm.Q_INT4_SYM_G32: "int4 sym g32", wlm.Q_INT2_ASYM_G16: "int2 asym g16",
         wlm.Q_INT8_PER_CHANNEL: "int8 per-channel"}
    routed = ", ".join(f"experts {lo}-{(hi or wl.E) - 1} {q[t]}" for lo, hi, t in wl.routed_qtypes)
    desc = (f"{wl.name}: T={wl.T} tokens/step, H={wl.H}, I={wl.I}, E={wl.E} routed + 1 shared "
            f"({q[wl.shared_qtype]}), top-{wl.k}, {routed}, Zipf({wl.zipf_s}) router prior"
            + (f", {wl.uniform_frac:.0%} uniform rows" if wl.uniform_frac else "")
            + (", fresh token per step" if wl.T <= 4 else ""))
    return {"workload": desc, "global_batch": wl.T * world, "parallelism": f"replicas x{world}"}


def load_balance(counts, row_tile=128):
    """How the routed rows of one prefill step spread over the routed experts
    (the shared expert's T rows are not included): the row-count histogram,
    the 128-row tiles the grouped GEMM runs and how full they are, and the
    groups of more than one tile (those the pre-dequantised path may take)."""
    c = np.asarray(counts, dtype=np.int64)
    nz = c[c > 0]
    tiles = (c + row_tile - 1) // row_tile
    bins = {"0": (0, 0), "1-127": (1, 127), "128-1023": (128, 1023), "1024-8191": (1024, 8191),
            ">=8192": (8192, np.iinfo(np.int64).max)}
    return {"rows": int(c.sum()), "experts_empty": int(np.sum(c == 0)),
            "experts_below_one_tile": int(np.sum((c > 0) & (c < row_tile))),
            "rows_max": int(c.max()) if c.size else 0,
            "rows_median_nonempty": float(np.median(nz)) if nz.size else 0.0,
            "row_tiles": int(tiles.sum()), "tile_fill": float(c.sum() / max(1, tiles.sum() * row_tile)),
            "groups_over_one_tile": int(np.sum(c > row_tile)),
            "rows_histogram": {name: int(np.sum((c >= lo) & (c <= hi))) for name, (lo, hi) in bins.items()}}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f), "measured"
    return FALLBACK_PEAKS, "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.proc = None
        self.path = None
        self.out = None
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            self.out = os.fdopen(fd, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "200", "-i", str(gpu_index)], stdout=self.out,
                                         stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            if self.out is not None:
                self.out.close()
                os.unlink(self.path)
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            self.proc.wait()
        self.out.close()
        with open(self.path) as f:
            rows = [r for r in csv.reader(io.StringIO(f.read())) if len(r) >= 9]
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.strip().lower() == "active"})
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


REJECT_REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown")


def clock_rejections(clk):
    """Why a timed region's clock record rejects its number (empty: kept).

    A hardware or thermal slowdown reason, or an SM clock held well below its
    maximum with no reason active (a leftover clock lock). sw_power_cap alone
    is kept (and shows in the record's reasons)."""
    if not clk:
        return []
    why = [r for r in clk.get("reasons", []) if r in REJECT_REASONS]
    sm, mx = clk.get("sm_mhz"), clk.get("sm_max_mhz")
    if not clk.get("reasons") and sm and mx and sm < 0.8 * mx:
        why.append(f"sm clock {sm:.0f} of {mx:.0f} MHz with no reason active")
    return why


def keep_busy(step, seconds, sync):
    """Untimed steps back to back for about `seconds` (at least one): the
    load around the timed region while clocks are sampled."""
    if seconds <= 0:
        return 0
    t0, n = time.perf_counter(), 0
    while True:
        for _ in range(8):
            step()
            n += 1
        sync()
        if time.perf_counter() - t0 >= seconds:
            return n


def timed_region(run, rank, world, device, sampler=None, sync=None, filler=None, window=0.0):
    """Run `run()` (the K timed steps) as the timed region: a barrier and a
    device synchronize on both sides, clocks sampled on rank 0 meanwhile.

    A K-step region can be far shorter than the sampler's 200 ms period, so
    with `filler` (one untimed step of the same workload) the sampler runs
    over a window of about `window` seconds of back-to-back steps: half before
    the region, half after it, each side synchronised, so the timed steps
    themselves run alone. The record states the window and its sample count.

    If rank 0's clock record rejects the run, every rank runs it once more and
    the second run is kept; its record lists the first run's reasons under
    `first_run_rejected`. Returns (run's result, clock record or None)."""
    import torch
    sampler = ClockSampler if sampler is None else sampler
    if sync is None:
        sync = torch.cuda.synchronize if device is not None and device.type == "cuda" else (lambda: None)
    first = None
    for attempt in (0, 1):
        if world > 1:
            torch.distributed.barrier()
        sync()
        clocks = sampler(device.index if device is not None else 0) if rank == 0 else None
        t_win = time.perf_counter()
        n_fill = keep_busy(filler, window / 2, sync) if filler is not None else 0
        if world > 1:
            torch.distributed.barrier()
        sync()
        res = run()
        if world > 1:
            torch.distributed.barrier()
        sync()
        n_fill += keep_busy(filler, window / 2, sync) if filler is not None else 0
        t_win = time.perf_counter() - t_win
        clk = clocks.stop() if clocks else None
        if clk is not None:
            clk["window_s"] = t_win
            clk["window"] = ("the timed region inside back-to-back untimed steps of the same workload "
                             f"({n_fill} of them)" if filler is not None else "the timed region alone")
        why = clock_rejections(clk)
        if attempt == 0 and max_over_ranks(1.0 if why else 0.0, world, device) > 0:
            first = why or ["rejected on rank 0"]
            continue
        break
    if clk is not None:
        clk["first_run_rejected"] = first
        clk["rejections"] = clock_rejections(clk)
    return res, clk


# ------------------------------------------------------------------ CPU side
def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def time_oracle(wl, lay, bias, n_steps_max, seconds, step_offset=0):
    """Run the fp64 oracle layer step by step until `seconds` or n_steps_max.
    Returns (tokens, elapsed seconds, steps)."""
    import oracle
    tokens, steps, t0 = 0, 0, time.perf_counter()
    while steps < n_steps_max:
        xb = wlm.gen_x(wl, step=step_offset + steps)
        oracle.moe_layer(xb, lay.w_router, bias, wl.k, lay.experts, lay.shared)
        tokens += wl.T
        steps += 1
        if time.perf_counter() - t0 >= seconds and steps >= 2:
            break
    return tokens, time.perf_counter() - t0, steps


def time_oracle_tokens(wl, lay, bias, seconds, chunk=16):
    """The fp64 oracle layer over the first tokens of the workload's input,
    `chunk` tokens per call, until `seconds`. Returns (tokens, elapsed s)."""
    import oracle
    xb = wlm.gen_x(wl)
    tokens, t0 = 0, time.perf_counter()
    while tokens < wl.T:
        n = min(chunk, wl.T - tokens)
        b = bias[tokens:tokens + n] if np.ndim(bias) == 2 else bias
        oracle.moe_layer(xb[tokens:tokens + n], lay.w_router, b, wl.k, lay.experts, lay.shared)
        tokens += n
        if time.perf_counter() - t0 >= seconds:
            break
    return tokens, time.perf_counter() - t0


def cpu_baseline(wl, lay, bias, seconds):
    """The fp64 oracle on the host cores, timed on a bounded sample of the
    workload, as tokens/s of one layer (a layer stack: layer 0's rate divided
    by the layer count, every layer costing the same)."""
    if wl.T > 4:
        tokens, secs = time_oracle_tokens(wl, lay, bias, seconds)
        sample = (f"{tokens} of the {wl.T} tokens of the step through the fp64 oracle in 16-token calls "
                  f"({secs:.1f} s; each call dequantises the experts it touches, so the rate is below what a "
                  f"whole step would reach)")
    else:
        tokens, secs, steps = time_oracle(wl, lay, bias, 10 ** 6, seconds, step_offset=10 ** 5)
        sample = (f"{steps} layer-steps of {wl.T} token(s) through the fp64 oracle ({secs:.1f} s)"
                  + (f" on layer 0, scaled by 1/{wl.layers} layers" if wl.layers > 1 else ""))
    return {"value": tokens / secs / wl.layers, "unit": "tokens/s", "cores": cpu_threads(), "kind": "oracle",
            "sample": sample}


# ------------------------------------------------------------------ GPU arm
def run_ours(args, rank, world, peaks, peak_kind):
    import torch

    from bit_quantized_moe_gemv_b200 import _lib as L
    from bit_quantized_moe_gemv_b200.device import DeviceExperts, bf16_tensor

    wl = wlm.WORKLOADS[args.workload]
    dev = torch.device("cuda", torch.cuda.current_device())
    lay = wlm.gen_layer(wl)
    bias, stride = wlm.gen_bias(wl)
    experts, shared = DeviceExperts(lay.experts), DeviceExperts([lay.shared])
    w_r = torch.from_numpy(lay.w_router).to(dev)
    b = torch.from_numpy(np.ascontiguousarray(bias)).to(dev)
    n_steps = args.warmup + args.steps
    # each rank gets its own stream of fresh tokens (replicas)
    xs_host = np.stack([wlm.gen_x(wl, step=rank * n_steps + s) for s in range(n_steps)])
    xs = bf16_tensor(xs_host)
    idx = torch.empty((n_steps, wl.T, wl.k), dtype=torch.int32, device=dev)
    gw = torch.empty((n_steps, wl.T, wl.k), dtype=torch.float32, device=dev)
    out = torch.empty((n_steps, wl.T, wl.H), dtype=torch.bfloat16, device=dev)
    ws = L.new_workspace(wl.T, wl.H, wl.I, wl.E, wl.k, device=dev)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(2 * max(l2, 126 << 20), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step(s):
        L.layer(xs[s], wl.I, wl.E, wl.k, w_r, b, stride, experts.table, shared.table, idx[s], gw[s], out[s], ws,
                stream=stream)

    def timed_loop(first, count, flush_between=True, host_io=None):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(count)]
        for i in range(count):
            s = first + i
            # keep the GPU ahead of the host: a short spin before each timed
            # step, so the step's launch is queued before its start event runs
            # and the events time the device, not the host's submission (the
            # end-to-end loop keeps the host's cost: no spin there)
            if host_io is None:
                torch.cuda._sleep(LEAD_CYCLES)
            evs[i][0].record(stream)
            if host_io is None:
                step(s)
            else:
                xin, xout = host_io
                xs[s].copy_(xin[s], non_blocking=True)
                step(s)
                xout[s].copy_(out[s], non_blocking=True)
            evs[i][1].record(stream)
            if flush_between:
                flush.fill_(i & 0xff)
        torch.cuda.synchronize()
        return [a.elapsed_time(z) for a, z in evs]

    # warm-up (untimed), same protocol
    timed_loop(0, args.warmup)

    def measured():
        launches0 = L.launch_count()
        t0 = time.perf_counter()
        t = timed_loop(args.warmup, args.steps)
        return t, L.launch_count() - launches0, time.perf_counter() - t0

    def filler():
        step(args.warmup)
        flush.fill_(1)

    (times, launches, t_wall), clk = timed_region(measured, rank, world, dev, filler=filler,
                                                  window=args.clock_window)
    assert L.get_status(ws, stream) == 0, "device-side status set during the bench"

    total_ms = float(np.sum(times))
    total_ms = max_over_ranks(total_ms, world, dev)
    tokens_all = world * wl.T * args.steps
    value = tokens_all / (total_ms / 1e3)

    # warm-L2 figure (context only): same steps without the flush
    warm = timed_loop(args.warmup, min(args.steps, 50), flush_between=False)

    # e2e: pinned host tokens in, pinned host output back, every step
    xin = xs_host.copy()
    xin_t = torch.from_numpy(xin.view(np.int16)).view(torch.bfloat16).pin_memory()
    xout_t = torch.empty((n_steps, wl.T, wl.H), dtype=torch.bfloat16).pin_memory()
    e2e_times = timed_loop(args.warmup, args.steps, host_io=(xin_t, xout_t))
    e2e_ms = float(np.sum(e2e_times))
    e2e_ms = max_over_ranks(e2e_ms, world, dev)

    # routing heat over the timed steps' tokens (untimed pass): the library's
    # per-expert hit counters, checked against the steps' own picks
    heat = torch.zeros(wl.E, dtype=torch.int32, device=dev)
    for s in range(args.warmup, args.warmup + args.steps):
        L.layer(xs[s], wl.I, wl.E, wl.k, w_r, b, stride, experts.table, shared.table, idx[s], gw[s], out[s], ws,
                stream=stream, heat=heat)
    torch.cuda.synchronize()
    heat_h = heat.cpu().numpy().astype(np.int64)
    assert np.array_equal(heat_h, np.bincount(idx[args.warmup:].cpu().numpy().ravel(), minlength=wl.E))
    order = np.argsort(-heat_h, kind="stable")
    routing_heat = {"steps": args.steps, "picks": int(heat_h.sum()), "experts_hit": int(np.sum(heat_h > 0)),
                    "hottest": [[int(e), int(heat_h[e])] for e in order[:8]],
                    "share_of_hottest_8": float(heat_h[order[:8]].sum() / max(1, heat_h.sum())),
                    "bytes_of_hottest_8": 8 * float(wlm.per_token_layer_bytes(wl, 1) - wlm.per_token_layer_bytes(wl, 0))}

    # the four-call composition of the same timed steps (moe_route,
    # moe_dispatch, moe_expert_ffn, moe_combine; L2 flushed between steps),
    # with moe_expert_ffn also timed alone: at decode sizes it runs the fused
    # kernel's expert phases on the given routing
    E, k, T, H = wl.E, wl.k, wl.T, wl.H
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(T * k, dtype=torch.int32, device=dev)
    inv = torch.empty(T * k, dtype=torch.int32, device=dev)
    y_perm = torch.empty((T * k, H), dtype=torch.bfloat16, device=dev)
    out4 = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    # three timed segments per step, each behind a short spin so that its
    # launches are queued before its start event runs (the events then time
    # the device, not the host's submission of the next call)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    # one untimed pass first: the first launch of each kernel loads its code
    L.route(xs[args.warmup], w_r, b, stride, k, idx[args.warmup], gw[args.warmup], ws, stream=stream)
    L.dispatch(idx[args.warmup], E, counts, offsets, perm, inv, ws, stream=stream)
    L.expert_ffn(xs[args.warmup], wl.I, k, E, perm, offsets, counts, experts.table, y_perm, ws, stream=stream)
    L.combine(y_perm, inv, gw[args.warmup], wl.I, xs[args.warmup], shared.table, out4, ws, stream=stream)
    torch.cuda.synchronize()
    launches0 = L.launch_count()
    for i in range(args.steps):
        s = args.warmup + i
        torch.cuda._sleep(LEAD_CYCLES)
        ev[i][0].record(stream)
        L.route(xs[s], w_r, b, stride, k, idx[s], gw[s], ws, stream=stream)
        L.dispatch(idx[s], E, counts, offsets, perm, inv, ws, stream=stream)
        ev[i][1].record(stream)
        torch.cuda._sleep(LEAD_CYCLES)
        ev[i][2].record(stream)
        L.expert_ffn(xs[s], wl.I, k, E, perm, offsets, counts, experts.table, y_perm, ws, stream=stream)
        ev[i][3].record(stream)
        torch.cuda._sleep(LEAD_CYCLES)
        ev[i][4].record(stream)
        L.combine(y_perm, inv, gw[s], wl.I, xs[s], shared.table, out4, ws, stream=stream)
        ev[i][5].record(stream)
        flush.fill_(i & 0xff)
    torch.cuda.synchronize()
    four_launches = L.launch_count() - launches0
    assert L.get_status(ws, stream) == 0, "device-side status set by the four-call steps"

    # algorithmic bytes per step: distinct routed experts + shared + router
    idx_h = idx[args.warmup:].cpu().numpy()
    uniq = np.array([len(np.unique(s)) for s in idx_h.reshape(args.steps, -1)])
    bytes_per_step = np.array([wlm.per_token_layer_bytes(wl, u) for u in uniq])
    achieved_gbs = float(np.sum(bytes_per_step) / (np.sum(times) / 1e3) / 1e9)
    peak = float(peaks["hbm_gbs"])
    four_ms = np.array([e[0].elapsed_time(e[1]) + e[2].elapsed_time(e[3]) + e[4].elapsed_time(e[5]) for e in ev])
    ffn_ms = np.array([e[2].elapsed_time(e[3]) for e in ev])
    expert_bytes = uniq * float(wlm.per_token_layer_bytes(wl, 1) - wlm.per_token_layer_bytes(wl, 0))
    ffn_gbs = float(np.sum(expert_bytes) / (np.sum(ffn_ms) / 1e3) / 1e9)
    four_call = {
        "calls": "moe_route, moe_dispatch, moe_expert_ffn, moe_combine (the shared expert in moe_combine)",
        "ms_per_step": float(np.mean(four_ms)),
        "tokens_per_s": world * wl.T / (float(np.mean(four_ms)) / 1e3),
        "gpu_launches": int(four_launches),
        "expert_ffn": {"ms_per_call": float(np.mean(ffn_ms)), "bytes_per_call": float(np.mean(expert_bytes)),
                       "achieved": ffn_gbs, "peak": peak, "unit": "GB/s", "frac": ffn_gbs / peak,
                       "kernel": "decode_fused_kernel, experts only (the given routing)"},
        "l2": "flushed between steps, outside the events",
        "timing": "sum of three event-timed segments per step (route + dispatch, expert_ffn, combine)",
    }
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": total_ms / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f16",  # tensor-core operands (fp16 weights and activations), fp32 accumulation
        "data": "synthetic (seeded; random weights of the stated architecture)",
        "config": dict(workload_config(wl, world),
                       l2="flushed between steps (2 x L2 write, outside the timed events)"),
        "roofline": {
            "bound": "hbm",
            "kernel": "moe_layer step: decode_fused_kernel, one launch per step (events bracket the launch)"
                      if wl.T <= 4 else "moe_layer step (all launches of one step)",
            "achieved": achieved_gbs,
            "peak": peak,
            "unit": "GB/s",
            "frac": achieved_gbs / peak,
            "peak_source": f"{peak_kind} hbm_gbs",
            "algorithmic_bytes_per_step": float(np.mean(bytes_per_step)),
            "traffic": ncu_traffic(args.workload)[0],
            "traffic_source": ncu_traffic(args.workload)[1],
        },
        "warm_l2": {"ms_per_step": float(np.mean(warm)), "note": "context only, weights partly L2-resident"},
        "e2e": {"value": tokens_all / (e2e_ms / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": int(wl.T * wl.H * 2), "d2h_bytes_per_step": int(wl.T * wl.H * 2)},
        "gpu_launches": int(launches),
        "clocks": clk,
        "wall_s_timed_region": t_wall,
        "routing_heat": routing_heat,
        "four_call": four_call,
    }
    return line, wl, lay, bias


def run_stack(args, rank, world, peaks, peak_kind):
    """48-layer decode stack: one step = the step's 4 tokens (slots) through
    all 48 layers, each layer with its own weights and fresh tokens (layers
    are not chained, so every layer sees the specified routing). The whole
    stack (58 GB) is resident and far larger than L2, so no flush is needed.
    Weights are drawn on the device (workload.draw_layer_device).

    The 48 moe_layer launches of a step are captured once into a CUDA graph
    over static input/output buffers and replayed every step (no host launch
    overhead between layers); each step's tokens are staged into the static
    input buffer before its start event, its routing copied out after its end
    event. --no-graph times the plain launches instead."""
    import torch

    from bit_quantized_moe_gemv_b200 import _lib as L
    from bit_quantized_moe_gemv_b200.device import BlockExperts

    wl = wlm.WORKLOADS[args.workload]
    dev = torch.device("cuda", torch.cuda.current_device())
    NL, T, k, E, H, I = wl.layers, wl.T, wl.k, wl.E, wl.H, wl.I
    layers, tables = [], []
    for li in range(NL):
        d = wlm.draw_layer_device(wl, li, device=dev)
        layers.append(d)
        tables.append((BlockExperts(d["qtype"], d["gu"], d["dn"], I, H, device=dev),
                       BlockExperts(d["shared_qtype"], d["sgu"], d["sdn"], I, H, device=dev)))
    bias, stride = wlm.gen_bias(wl)
    b = torch.from_numpy(np.ascontiguousarray(bias)).to(dev)
    n_steps = args.warmup + args.steps
    g = torch.Generator(device=dev)
    g.manual_seed(1000003 * (rank + 1))
    xs = torch.randn((n_steps, NL, T, H), dtype=torch.float32, device=dev, generator=g).to(torch.bfloat16)
    idx = torch.empty((n_steps, NL, T, k), dtype=torch.int32, device=dev)
    gw = torch.empty((n_steps, NL, T, k), dtype=torch.float32, device=dev)
    out = torch.empty((n_steps, NL, T, H), dtype=torch.bfloat16, device=dev)
    ws = L.new_workspace(T, H, I, E, k, device=dev)
    stream = torch.cuda.current_stream()

    def layers_into(xb, ib, wb, ob):
        for li in range(NL):
            ex, sh = tables[li]
            L.layer(xb[li], I, E, k, layers[li]["w_router"], b, stride, ex.table, sh.table, ib[li], wb[li], ob[li],
                    ws, stream=torch.cuda.current_stream())

    graph, launches_per_step = None, NL
    if not args.no_graph:
        x_st = torch.empty((NL, T, H), dtype=torch.bfloat16, device=dev)
        i_st = torch.empty((NL, T, k), dtype=torch.int32, device=dev)
        w_st = torch.empty((NL, T, k), dtype=torch.float32, device=dev)
        o_st = torch.empty((NL, T, H), dtype=torch.bfloat16, device=dev)
        x_st.copy_(xs[0])
        layers_into(x_st, i_st, w_st, o_st)  # first calls outside the capture (one-time attribute set-up)
        torch.cuda.synchronize()
        n0 = L.launch_count()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            layers_into(x_st, i_st, w_st, o_st)
        launches_per_step = L.launch_count() - n0
        torch.cuda.synchronize()

    def step(s):
        if graph is None:
            layers_into(xs[s], idx[s], gw[s], out[s])
        else:
            graph.replay()

    def stage_in(s):
        if graph is not None:
            x_st.copy_(xs[s])

    def stage_out(s):
        if graph is not None:
            idx[s].copy_(i_st)
            gw[s].copy_(w_st)
            out[s].copy_(o_st)

    def timed_loop(first, count, host_io=None):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(count)]
        for i in range(count):
            s = first + i
            if host_io is None:
                stage_in(s)
                torch.cuda._sleep(LEAD_CYCLES)
            evs[i][0].record(stream)
            if host_io is not None:
                (x_st if graph is not None else xs[s]).copy_(host_io[0][s], non_blocking=True)
            step(s)
            if host_io is not None:
                host_io[1][s].copy_(o_st if graph is not None else out[s], non_blocking=True)
            evs[i][1].record(stream)
            stage_out(s)
        torch.cuda.synchronize()
        return [a.elapsed_time(z) for a, z in evs]

    timed_loop(0, args.warmup)

    def measured():
        launches0 = L.launch_count()
        t = timed_loop(args.warmup, args.steps)
        # graph replays launch the captured kernels without calling the library
        n = L.launch_count() - launches0 if graph is None else launches_per_step * args.steps
        return t, n

    (times, launches), clk = timed_region(measured, rank, world, dev, filler=lambda: step(args.warmup),
                                          window=args.clock_window)
    assert L.get_status(ws, stream) == 0, "device-side status set during the bench"
    total_ms = float(np.sum(times))
    total_ms = max_over_ranks(total_ms, world, dev)
    tokens_all = world * T * args.steps
    value = tokens_all / (total_ms / 1e3)

    xin = xs.cpu().pin_memory()
    xout = torch.empty((n_steps, NL, T, H), dtype=torch.bfloat16).pin_memory()
    e2e_ms = float(np.sum(timed_loop(args.warmup, args.steps, host_io=(xin, xout))))
    e2e_ms = max_over_ranks(e2e_ms, world, dev)

    idx_h = idx[args.warmup:].cpu().numpy().reshape(args.steps, NL, T * k)
    uniq = np.array([[len(np.unique(r)) for r in s] for s in idx_h])  # [steps, layers]
    bytes_per_step = np.array([sum(wlm.per_token_layer_bytes(wl, u) for u in row) for row in uniq])
    achieved_gbs = float(np.sum(bytes_per_step) / (np.sum(times) / 1e3) / 1e9)
    peak = float(peaks["hbm_gbs"])
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16",
        "data": "synthetic (seeded; random weights of the stated architecture, drawn on the device)",
        "config": dict(workload_config(wl, world), layers=NL,
                       l2="inputs larger than L2 (58 GB stack streamed every step)"),
        "roofline": {
            "bound": "hbm",
            "kernel": ("moe_layer x 48 layers, one CUDA graph per step (one fused decode launch per layer)"
                       if graph is not None else "moe_layer x 48 layers (one launch per layer)"),
            "achieved": achieved_gbs, "peak": peak, "unit": "GB/s", "frac": achieved_gbs / peak,
            "peak_source": f"{peak_kind} hbm_gbs",
            "algorithmic_bytes_per_step": float(np.mean(bytes_per_step)),
            "bytes_per_generated_token": float(np.mean(bytes_per_step)) / T,
            "distinct_experts_per_layer_step": float(np.mean(uniq)),
            "traffic": None,
        },
        "e2e": {"value": tokens_all / (e2e_ms / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": int(NL * T * H * 2), "d2h_bytes_per_step": int(NL * T * H * 2)},
        "gpu_launches": int(launches), "clocks": clk,
    }
    return line, wl, None, bias


def run_prefill(args, rank, world, peaks, peak_kind):
    """Prefill workload: one step = moe_layer over all T tokens of one layer.

    Weights (1.36 GB) and activations exceed L2, so no flush is needed. The
    tensor-core roofline is taken on the expert FFN alone (moe_expert_ffn:
    gather + gate/up GEMM + down GEMM), timed with its own events.
    """
    import torch

    from bit_quantized_moe_gemv_b200 import _lib as L
    from bit_quantized_moe_gemv_b200.device import DeviceExperts, bf16_tensor

    wl = wlm.WORKLOADS[args.workload]
    dev = torch.device("cuda", torch.cuda.current_device())
    lay = wlm.gen_layer(wl)
    bias, stride = wlm.gen_bias(wl)
    experts, shared = DeviceExperts(lay.experts), DeviceExperts([lay.shared])
    w_r = torch.from_numpy(lay.w_router).to(dev)
    b = torch.from_numpy(np.ascontiguousarray(bias)).to(dev)
    xh = wlm.gen_x(wl, step=rank)
    x = bf16_tensor(xh)
    T, k, E, H, I = wl.T, wl.k, wl.E, wl.H, wl.I
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    gw = torch.empty((T, k), dtype=torch.float32, device=dev)
    out = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    ws = L.new_workspace(T, H, I, E, k, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        L.layer(x, I, E, k, w_r, b, stride, experts.table, shared.table, idx, gw, out, ws, stream=stream)

    def timed(fn, n, lead=True):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        for a, z in evs:
            if lead:
                torch.cuda._sleep(LEAD_CYCLES)
            a.record(stream)
            fn()
            z.record(stream)
        torch.cuda.synchronize()
        return [a.elapsed_time(z) for a, z in evs]

    for _ in range(args.warmup):
        step()

    def measured():
        launches0 = L.launch_count()
        t = timed(step, args.steps)
        return t, L.launch_count() - launches0

    (times, launches), clk = timed_region(measured, rank, world, dev, filler=step, window=args.clock_window)
    assert L.get_status(ws, stream) == 0, "device-side status set during the bench"
    total_ms = float(np.sum(times))
    total_ms = max_over_ranks(total_ms, world, dev)
    value = world * T * args.steps / (total_ms / 1e3)

    # expert FFN alone (routed experts), on the routing of the last step
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(T * k, dtype=torch.int32, device=dev)
    inv = torch.empty(T * k, dtype=torch.int32, device=dev)
    L.dispatch(idx, E, counts, offsets, perm, inv, ws, stream=stream)
    balance = load_balance(counts.cpu().numpy())
    y = torch.empty((T * k, H), dtype=torch.bfloat16, device=dev)
    ffn = lambda: L.expert_ffn(x, I, k, E, perm, offsets, counts, experts.table, y, ws, stream=stream)  # noqa: E731
    ffn()
    ffn_ms = float(np.mean(timed(ffn, max(3, min(args.steps, 10)))))
    flops = 2.0 * 3 * H * I * T * k
    achieved = flops / (ffn_ms / 1e3) / 1e12
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))

    # e2e: host tokens in, host output back
    xin = torch.from_numpy(xh.view(np.int16)).view(torch.bfloat16).pin_memory()
    xout = torch.empty((T, H), dtype=torch.bfloat16).pin_memory()

    def e2e_step():
        x.copy_(xin, non_blocking=True)
        step()
        xout.copy_(out, non_blocking=True)

    e2e_ms = max_over_ranks(float(np.sum(timed(e2e_step, args.steps, lead=False))), world, dev)
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16",
        "data": "synthetic (seeded; random weights of the stated architecture)",
        "config": dict(workload_config(wl, world), l2="inputs larger than L2 (1.36 GB of expert weights)"),
        "roofline": {"bound": "tensor",
                     "kernel": "moe_expert_ffn (gather, pre-dequantisation, tcgen05 and mma.sync gate/up and down)",
                     "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                     "peak_source": f"{peak_kind} bf16_tflops", "flops_per_launch": flops, "ms_per_launch": ffn_ms,
                     "traffic": ncu_traffic(args.workload)[0], "traffic_source": ncu_traffic(args.workload)[1]},
        "load_balance": balance,
        "e2e": {"value": world * T * args.steps / (e2e_ms / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": int(T * H * 2), "d2h_bytes_per_step": int(T * H * 2)},
        "gpu_launches": int(launches), "clocks": clk,
    }
    return line, wl, lay, bias


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    peaks, peak_kind = load_peaks()

    if args.impl == "reference":
        if rank != 0:
            return 0
        wl = wlm.WORKLOADS[args.workload]
        lay = wlm.gen_layer(wl)
        bias, _ = wlm.gen_bias(wl)
        budget = 150.0
        _, s_warm, _ = time_oracle(wl, lay, bias, args.warmup, budget / 4)
        tokens, secs, steps = time_oracle(wl, lay, bias, args.steps, budget, step_offset=args.warmup)
        value = tokens / secs / wl.layers  # a layer stack: layer 0 timed, every layer costs the same
        line = {
            "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
            "config": dict(workload_config(wl, 1),
                           l2="flushed between steps (2 x L2 write, outside the timed events)"
                           if wl.T <= 4 else "inputs larger than L2 (1.36 GB of expert weights)"),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cpu_threads(), "kind": "oracle",
                             "sample": f"{steps} of {args.steps} requested steps ({wl.T} token(s) each), bounded to "
                                       f"{budget:.0f} s" + (f", layer 0 of {wl.layers} timed and scaled by "
                                                             f"1/{wl.layers}" if wl.layers > 1 else "")},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        }
        print(json.dumps(line), flush=True)
        return 0

    import torch
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    def run_one(name):
        a = argparse.Namespace(**vars(args))
        a.workload = name
        if name.startswith("prefill"):
            res = run_prefill(a, rank, world, peaks, peak_kind)
        elif wlm.WORKLOADS[name].layers > 1:
            res = run_stack(a, rank, world, peaks, peak_kind)
        else:
            res = run_ours(a, rank, world, peaks, peak_kind)
        ln, wl, lay, bias = res
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            if lay is None:  # layer stack: time the oracle on layer 0 and scale to all layers
                lay = wlm.gen_layer(wl, layer=0)
            ln["cpu_baseline"] = cpu_baseline(wl, lay, bias, args.cpu_seconds)
        import torch
        torch.cuda.empty_cache()
        return ln

    line = run_one(args.workload)
    if args.workload == "decode1" and not args.headline_only:
        # the metric's other halves, measured in the same process: the 8K
        # prefill and the 48-layer decode stack, each with its own roofline,
        # clocks, e2e and CPU baseline
        keep = ("value", "unit", "ms_per_step", "steps", "warmup", "config", "roofline", "e2e", "gpu_launches",
                "clocks", "cpu_baseline", "load_balance", "dtype")
        line["workloads"] = {}
        for name in ("prefill8k", "decode48"):
            sub = run_one(name)
            line["workloads"][name] = {key: sub[key] for key in keep if key in sub}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
