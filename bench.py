#!/usr/bin/env python
"""Benchmark of block-sparse attention driven by a per-input mask on B200.

One step = the whole hot path over one batch of synthetic input already in
HBM: block selection (pool, score, rank-select with pins/drops and head
skipping), the attention work plan, and flash attention over the selected
tiles.  Metric: effective TFLOP/s = 4 * 64 * 64 * d * (selected tiles) / step
time, i.e. 4*B*H_active*N^2*d*density / t.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload joint|sdxl|video|stack|tiny]
                  [--pattern content|radial|random|window] [--kv-heads H_kv] [--no-graph]
  python bench.py --impl reference ...     # the fp64 CPU oracle on a bounded sample

Timing: each step (every layer) is captured once as a CUDA graph and
replayed, K replays timed with CUDA events (--no-graph: eager launches);
the stage times (selection, plan, attention kernel) come from a second run
of K steps launched eagerly with events between the stages.

Multi-GPU (torchrun, one process per GPU): every rank runs its own
independent batch (seed = rank); value = all ranks' flops / max-over-ranks
time (weak scaling, no data-path collective).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import SEG_PAD, WORKLOADS, head_mask_for_layer, make_qkv  # noqa: E402

METRIC = "effective TFLOP/s of block-sparse attention; speedup vs dense at 30% density"
UNIT = "TFLOP/s"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def describe(w, rho, H_kv=None):
    segs = ", ".join("%s[%d,%d)" % ({0: "text", 1: "pad", 2: "image", 3: "other"}[k], s, s + l) for k, s, l in w.segments)
    return "%s: B%d H%d%s d%d N%d%s, density %.2f%s" % (
        w.name, w.B, w.H, (" (K/V heads %d)" % H_kv) if H_kv and H_kv != w.H else "", w.d, w.N,
        (" (" + segs + ")") if segs else "", rho,
        (", head mask %d of %d" % (int(head_mask_for_layer(w).sum()), w.H)) if w.head_mask or w.mask_runs else "")


def paired_tiles(idx, counts, head_mask, H, nB):
    """64 x 64 tiles the attention kernel computes for these lists: the planner pairs query blocks (a, a + s)
    with a // s even, s = 1, 2 or 4 per head (the smallest summed union, the smaller s on ties), and each pair
    walks the union of its two lists with a 128-row tile (two 64 x 64 tiles per union entry).  Host-side
    restatement of the planner's pairing, for reporting."""
    idx = np.asarray(idx).reshape(-1, nB, idx.shape[-1])
    cnt = np.asarray(counts).reshape(-1, nB)
    BH = cnt.shape[0]
    M = np.zeros((BH, nB, nB), bool)
    b_ix, i_ix, e_ix = np.nonzero(np.arange(idx.shape[-1])[None, None, :] < cnt[..., None])
    M[b_ix, i_ix, idx[b_ix, i_ix, e_ix]] = True
    active = np.ones(BH, bool) if head_mask is None else np.tile(np.asarray(head_mask, bool), BH // H)
    best = None
    for s in (1, 2, 4):
        a = np.array([i for i in range(nB) if (i // s) % 2 == 0])
        b = a + s
        partner = np.where((b < nB)[None, :, None], M[:, np.minimum(b, nB - 1)], False)
        u = (M[:, a] | partner).sum(axis=(1, 2))
        best = u if best is None else np.minimum(best, u)
    return int(2 * best[active].sum())


def grouped_kv(K, V, g):
    """K and V of the first head of each group of g query heads: the shared
    key/value heads of a grouped-query layout ([B, H / g, N, d])."""
    return np.ascontiguousarray(K[:, ::g]), np.ascontiguousarray(V[:, ::g])


# ------------------------------------------------------------------ ranks
def max_over_ranks(x, device):
    """The largest x over all ranks of the process group (x itself with one
    rank): a step's time is the slowest rank's."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def time_stats(times_ms):
    """Mean, median and 90th percentile (nearest rank) of per-step times, ms."""
    xs = sorted(float(x) for x in times_ms)
    if not xs:
        raise ValueError("no times")
    p90 = xs[max(0, -(-9 * len(xs) // 10) - 1)]
    return {"mean": round(statistics.mean(xs), 5), "median": round(statistics.median(xs), 5), "p90": round(p90, 5)}


def crossover(points):
    """Sparse/dense crossover from [(N, sparse_ms, dense_ms), ...].

    Returns (N*, kind): the smallest length from which the sparse step stays
    faster than dense, interpolated linearly in log N between the last point
    where it was not and the next ("interpolated"); the first N when sparse
    wins at every point ("at or below"); None when it never wins at the
    largest N ("above")."""
    pts = sorted(points)
    if not pts:
        raise ValueError("no points")
    r = [d / s for _, s, d in pts]  # speedup of sparse over dense
    if r[-1] < 1.0:
        return None, "above"
    last_loss = max((q for q in range(len(pts)) if r[q] < 1.0), default=None)
    if last_loss is None:
        return float(pts[0][0]), "at or below"
    na, nb = math.log(pts[last_loss][0]), math.log(pts[last_loss + 1][0])
    ra, rb = r[last_loss], r[last_loss + 1]
    return float(math.exp(na + (1.0 - ra) / (rb - ra) * (nb - na))), "interpolated"


def job_value(flops_per_rank, ms_max, world):
    """Whole-job effective TFLOP/s: every rank's flops over the slowest rank's
    time (each rank runs its own batch: weak scaling)."""
    return world * flops_per_rank / (ms_max * 1e-3) / 1e12


# ------------------------------------------------------------------ oracle (CPU) sample
_INPUTS = {}


def _inputs_once(w, seed):
    """The workload's Q, K, V (all heads, layer 0), generated once per (workload, seed)."""
    key = (w.name, w.N, w.H, w.d, seed)
    if key not in _INPUTS:
        _INPUTS.clear()
        _INPUTS[key] = make_qkv(w, seed=seed)
    return _INPUTS[key]


def oracle_sample(w, rho, target_s=10.0, seed=0, g=1):
    """Times the fp64 oracle on whole heads of the workload (selection for the
    head, then attention for all its query rows) until about target_s of CPU
    work; very long heads are cut to an evenly spaced subset of rows.  g > 1:
    each query head reads the key/value head of its group of g."""
    import oracle
    mask = head_mask_for_layer(w)
    heads = [int(h) for h in np.flatnonzero(mask)]
    cls = oracle.layout(list(w.segments), w.N)
    flops = 0.0
    t_total = 0.0
    sel_s, att_s = 0.0, 0.0  # unscaled: every timed selection, every timed attention row
    done_heads, done_rows = 0, 0
    Qa, Ka, Va = _inputs_once(w, seed)
    for h in heads:
        hk = g * (h // g)  # the key/value head of h's group (itself without grouping)
        Q, K, V = (np.ascontiguousarray(x[:1, hh:hh + 1]) for x, hh in ((Qa, h), (Ka, hk), (Va, hk)))
        t0 = time.perf_counter()
        sc = oracle.scores(oracle.pool(Q), oracle.pool(K)).reshape(-1, w.nB, w.nB)
        idx, cnt = oracle.select(sc, cls, 1, rho)
        t_sel = time.perf_counter() - t0
        left = max(target_s - t_total - t_sel, 0.5)
        rows = np.arange(w.N, dtype=np.int64)
        if done_heads == 0:  # calibrate on the first head
            t = time.perf_counter()
            probe = rows[:: max(1, w.N // 512)]
            oracle.attention(Q, K, V, 1, idx, cnt, rows=probe)
            per_row = (time.perf_counter() - t) / len(probe)
            if per_row * w.N > left:
                rows = np.unique(np.linspace(0, w.N - 1, max(256, int(left / per_row))).astype(np.int64))
        t = time.perf_counter()
        oracle.attention(Q, K, V, 1, idx, cnt, rows=rows)
        t_att = time.perf_counter() - t
        sel_s += t_sel
        att_s += t_att
        flops += float(np.sum(4.0 * w.d * 64 * cnt[0, rows // 64]))
        t_total += t_att + t_sel * len(rows) / w.N
        done_heads += 1
        done_rows += len(rows)
        if t_total >= target_s:
            break
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    return {
        "value": flops / t_total / 1e12,
        "unit": UNIT,
        "cores": cores,
        "kind": "oracle",
        "sample": "%d of %d heads of the workload: fp64 selection per head (charged pro rata to the rows run) + "
                  "fp64 attention for %d query rows in all (%.1f s)" % (done_heads, len(heads), done_rows, t_total),
        "split": {"select_ms_per_head": round(1e3 * sel_s / max(done_heads, 1), 3),
                  "attention_us_per_row": round(1e6 * att_s / max(done_rows, 1), 3)},
        "seconds": t_total,
    }


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Polls SM clock and clock-event reasons through NVML from a thread while
    the timed region runs (every 2 ms, so short regions still get samples)."""
    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, uuid):
        self.uuid = uuid
        self.samples = []
        self.thread = None
        self.handle = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            if uuid:
                u = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
                self.handle = pynvml.nvmlDeviceGetHandleByUUID(u)
            else:
                self.handle = pynvml.nvmlDeviceGetHandleByIndex(0)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.handle = None

    def _run(self):
        import threading
        nv = self.nvml
        while not self.stop_event.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM)
                try:
                    r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                except AttributeError:
                    r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.handle)
                self.samples.append((sm, r))
            except Exception:
                pass
            self.stop_event.wait(0.002)

    def start(self):
        if self.handle is None:
            return
        import threading
        self.stop_event = threading.Event()
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()

    def stop(self):
        if self.thread is None:
            return None
        self.stop_event.set()
        self.thread.join(timeout=2)
        if not self.samples:
            return None
        reasons = sorted(n for n, bit in self.REASONS.items() if any(r & bit for _, r in self.samples))
        return {"sm_mhz": statistics.median(s for s, _ in self.samples), "sm_max_mhz": float(self.max_mhz),
                "reasons": reasons, "samples": len(self.samples), "source": "nvml, 2 ms polling"}


# ------------------------------------------------------------------ traffic from the committed ncu summary
def traffic_from_profile(kernel_src, workload="joint"):
    """dram bytes per launch recorded under profiles/ for the attention kernel on
    this workload, if the kernel source has not changed since the capture (else
    None; also None when no workload is given)."""
    if workload is None:
        return None
    p = os.path.join(ROOT, "profiles", "sparse_attn_kernel_%s.md" % workload)
    if not os.path.exists(p):
        return None
    digest = hashlib.sha256(open(kernel_src, "rb").read()).hexdigest()[:16]
    vals = {}
    for line in open(p):
        if ":" in line and line.strip().startswith("- "):
            k, v = line.strip()[2:].split(":", 1)
            vals[k.strip()] = v.strip()
    if vals.get("attention.cu sha256 (first 16 hex)") != digest:
        return None
    try:
        return float(vals["dram bytes per launch (full size)"])
    except (KeyError, ValueError):
        return None


# ------------------------------------------------------------------ GPU arm
def run_ours(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    import prompt_aware_head_b200 as sa

    w = WORKLOADS[args.workload]
    rho = args.density if args.density else w.densities[0]
    B, H, N, d = w.B, w.H, w.N, w.d
    H_kv = args.kv_heads or H
    if H_kv < 1 or H % H_kv:
        raise SystemExit("--kv-heads must divide the workload's %d heads" % H)
    g = H // H_kv
    # one step runs every layer of the workload (64 for the head-masked stack), each with its own inputs and
    # head mask [HS AttentionMask: a mask per (layer, head)]
    n_layers = min(args.layers or w.layers, w.layers)
    masks = [head_mask_for_layer(w, l) for l in range(n_layers)]
    pins, devs = [], []
    for l in range(n_layers):
        Qh, Kh, Vh = make_qkv(w, seed=args.seed + rank, layer=l)
        if g > 1:
            Kh, Vh = grouped_kv(Kh, Vh, g)
        p = [torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory() for x in (Qh, Kh, Vh)]
        del Qh, Kh, Vh
        pins.append(p)
        devs.append(tuple(x.to(dev, non_blocking=False) for x in p))
    L = sa.Layout(list(w.segments), N)
    ws_bytes = sa.sa_workspace_size(B, H, N, d)
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device=dev)
    idx = torch.zeros((B, H, w.nB, L.cap), dtype=torch.int32, device=dev)
    counts = torch.zeros((B, H, w.nB), dtype=torch.int32, device=dev)
    O = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev)
    O_host = torch.empty(O.shape, dtype=torch.bfloat16).pin_memory()
    stream = torch.cuda.current_stream(dev)
    sa.sa_workspace_init(ws, ws_bytes, stream)
    layer_in_bytes = sum(x.numel() for x in devs[0]) * 2
    in_bytes = n_layers * layer_in_bytes
    flush = in_bytes < 2 * L2_BYTES
    scratch = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev) if flush else None
    k_budget = sa.sa_budget(rho, L.n_cand)
    dense_short = k_budget >= L.n_cand
    km_dev = None  # --pad-mask: the layout's padding tokens masked as keys inside kept tiles
    if args.pad_mask:
        km = np.ones((B, N), np.uint8)
        for kind, start, length in w.segments:
            if kind == SEG_PAD:
                km[:, start:start + length] = 0
        km_dev = torch.from_numpy(km).to(dev)

    def select(l, q, k, st=None):
        mask = masks[l]
        st = st or stream
        if args.pattern == "content":
            sa.sa_select_blocks_gqa(L, q, k, B, H, H_kv, d, rho, mask, w.min_active, idx, counts, None, ws, ws_bytes,
                                    st)
        elif args.pattern == "radial":
            sa.sa_pattern_mask(L, sa.SA_PAT_RADIAL, B, H, rho, mask, w.min_active, idx, counts, stream=st)
        elif args.pattern == "random":
            sa.sa_pattern_mask(L, sa.SA_PAT_RANDOM, B, H, rho, mask, w.min_active, idx, counts, stream=st,
                               seed=rank)
        else:
            sa.sa_pattern_mask(L, sa.SA_PAT_WINDOW_GLOBAL, B, H, rho, mask, w.min_active, idx, counts,
                               window_tokens=512, n_global_blocks=8, stream=st)

    def step(ev=None, st=None):
        """All layers on stream st; ev (if given) holds 4 events per layer: start, selected, planned, attended."""
        st = st or stream
        for l in range(n_layers):
            Q, K, V = devs[l]
            e = ev[4 * l:4 * l + 4] if ev is not None else None
            if e:
                e[0].record(st)
            select(l, Q, K, st)
            if e:
                e[1].record(st)
            sa.sa_attention_plan(idx, counts, B, H, N, d, L.cap, masks[l], w.min_active, ws, ws_bytes, st)
            if e:
                e[2].record(st)
            sa.sa_attention_run_masked(Q, K, V, B, H, H_kv, N, d, km_dev, masks[l], w.min_active, 0.0, O, ws,
                                       ws_bytes, st)
            if e:
                e[3].record(st)

    def captured(fn):
        """fn() captured once into a CUDA graph on a side stream (the library's calls take that stream).
        Thread-local capture: other threads of the process (the NCCL watchdog under torchrun) keep
        calling CUDA while this one captures."""
        cap = torch.cuda.Stream(dev)
        cap.wait_stream(stream)
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=cap, capture_error_mode="thread_local"):
            fn(cap)
        stream.wait_stream(cap)
        for _ in range(2):
            gr.replay()
        torch.cuda.synchronize()
        return gr

    # per layer: selection (pool, scores, rank; one kernel for a pattern or a budget that covers every
    # candidate), planner (rows, order), attention (+ zeroing of skipped heads, + packing of a key mask)
    launches_per_step = sum((1 if dense_short or args.pattern != "content" else 3) + 2 + 1
                            + (1 if int(H - m.sum()) else 0) + (1 if km_dev is not None else 0) for m in masks)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert sa.sa_check(ws, stream) == sa.SA_OK
    # selected tiles of every layer (the lists of each layer, re-made once outside the timed region)
    tiles = 0
    tiles_per_layer = []
    computed = 0
    for l in range(n_layers):
        select(l, *devs[l][:2], stream)
        _, _, st = sa.sa_density(counts, B, H, w.nB, masks[l], ws, ws_bytes, stream)
        tiles += st.tiles
        tiles_per_layer.append(st.tiles)
        computed += paired_tiles(idx.cpu().numpy(), counts.cpu().numpy(), masks[l], H, w.nB)
    flops_step = 4.0 * 64 * 64 * d * tiles

    uuid = None
    try:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    # The step (every layer) is captured once into a CUDA graph and replayed: a serving loop repeats the same
    # launches every step, and the graph takes the host's launch path out of the timed region.  The step time
    # comes from replays of that graph (events around each replay: an event record inside a graph breaks the
    # programmatic-dependent-launch overlap of the kernels it separates).  The stage times (the attention
    # kernel's among them, for the roofline) come from a second run of as many steps launched eagerly with
    # events at the stage boundaries.
    graph = captured(lambda st: step(None, st)) if not args.no_graph else None
    clocks = ClockSampler(uuid)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4 * n_layers)] for _ in range(args.steps)]
    outer = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]

    def stage_times(e):
        return (e[0].elapsed_time(e[-1]),
                sum(e[4 * l].elapsed_time(e[4 * l + 1]) for l in range(n_layers)),
                sum(e[4 * l + 1].elapsed_time(e[4 * l + 2]) for l in range(n_layers)),
                sum(e[4 * l + 2].elapsed_time(e[4 * l + 3]) for l in range(n_layers)))

    def eager_steps():
        for i in range(args.steps):
            if flush:
                scratch.fill_(float(i))  # 512 MB write between steps, outside the per-step events
            step(evs[i])

    clocks.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    if graph is not None:
        for i in range(args.steps):
            if flush:
                scratch.fill_(float(i))
            outer[i][0].record(stream)
            graph.replay()
            outer[i][1].record(stream)
    else:
        eager_steps()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    if graph is not None:  # the stage-time run
        eager_steps()
        torch.cuda.synchronize()
        t_step = [a.elapsed_time(b) for a, b in outer]
    clk = clocks.stop()
    stage_rows = [stage_times(e) for e in evs]
    if graph is None:
        t_step = [r[0] for r in stage_rows]
    _, t_sel, t_plan, t_att = (list(x) for x in zip(*stage_rows))
    ms_step = statistics.mean(t_step)
    ms_max = max_over_ranks(ms_step, dev)
    value = job_value(flops_step, ms_max, world)
    assert sa.sa_check(ws, stream) == sa.SA_OK

    # dense baseline (same library, all heads of every layer, same inputs), and torch SDPA
    dense_ms = sdpa_ms = None
    if not args.no_dense:
        Od = torch.empty_like(O)

        def dense_all(st=None):
            for l in range(n_layers):
                Q, K, V = devs[l]
                sa.sa_dense_attention_gqa(Q, K, V, B, H, H_kv, N, d, 0.0, Od, ws, ws_bytes, st or stream)

        for _ in range(3):
            dense_all()
        if graph is not None:  # launched the same way as the sparse step
            dgraph = captured(dense_all)
            dense_run = dgraph.replay
        else:
            dense_run = dense_all
        de = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(5)]
        for a, b in de:
            if flush:
                scratch.fill_(1.0)
            a.record(stream)
            dense_run()
            b.record(stream)
        torch.cuda.synchronize()
        dense_ms = statistics.mean(a.elapsed_time(b) for a, b in de)
        try:
            def sdpa_all(st=None):
                for l in range(n_layers):
                    Q, K, V = devs[l]
                    torch.nn.functional.scaled_dot_product_attention(Q, K, V, enable_gqa=g > 1)
            for _ in range(2):
                sdpa_all()
            sdpa_run = captured(sdpa_all).replay if graph is not None else sdpa_all
            se = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(3)]
            for a, b in se:
                if flush:
                    scratch.fill_(1.0)
                a.record(stream)
                sdpa_run()
                b.record(stream)
            torch.cuda.synchronize()
            sdpa_ms = statistics.mean(a.elapsed_time(b) for a, b in se)
        except Exception:
            sdpa_ms = None
        del Od

    # End to end through the public API with host buffers (pinned): every layer of every step copies its Q, K,
    # V in and its O out inside the timed region.  The copies are pipelined as a serving loop would run them:
    # unit u's inputs go in on a copy stream while unit u-1 computes, its O comes out on another copy stream
    # while unit u+1 computes (two device slots of Q/K/V and O; a slot is refilled only after the unit that
    # used it is done).  A unit is one layer of one step.
    e2e_steps = max(1, min(args.steps, 10))
    units = e2e_steps * n_layers
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    slots = [tuple(torch.empty_like(x) for x in devs[0]) + (O,),
             tuple(torch.empty_like(x) for x in devs[0]) + (torch.empty_like(O),)]
    in_done = [torch.cuda.Event() for _ in range(units)]
    comp_done = [torch.cuda.Event() for _ in range(units)]
    out_done = [torch.cuda.Event() for _ in range(units)]
    ee = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
    torch.cuda.synchronize()
    ee[0].record(s_in)
    for u in range(units):
        l = u % n_layers
        q, k, v, o = slots[u % 2]
        if u >= 2:
            s_in.wait_event(comp_done[u - 2])
        with torch.cuda.stream(s_in):
            q.copy_(pins[l][0], non_blocking=True)
            k.copy_(pins[l][1], non_blocking=True)
            v.copy_(pins[l][2], non_blocking=True)
        in_done[u].record(s_in)
        stream.wait_event(in_done[u])
        if u >= 2:
            stream.wait_event(out_done[u - 2])
        select(l, q, k)
        sa.sa_block_sparse_attention_masked(q, k, v, B, H, H_kv, N, d, idx, counts, L.cap, km_dev, masks[l],
                                            w.min_active, 0.0, o, ws, ws_bytes, stream)
        comp_done[u].record(stream)
        s_out.wait_event(comp_done[u])
        with torch.cuda.stream(s_out):
            O_host.copy_(o, non_blocking=True)
        out_done[u].record(s_out)
    ee[1].record(s_out)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(ee[0].elapsed_time(ee[1]) / e2e_steps, dev)
    assert sa.sa_check(ws, stream) == sa.SA_OK
    del slots

    pk, pk_kind = peaks()
    att_ms = statistics.mean(t_att)
    sel_ms = statistics.mean(t_sel)
    achieved = flops_step / (att_ms * 1e-3) / 1e12
    traffic = traffic_from_profile(os.path.join(ROOT, "prompt_aware_head_b200", "csrc", "attention.cu"),
                                   args.workload if n_layers == 1 and args.pattern == "content" else None)
    n_act = sum(int(m.sum()) for m in masks)
    # key heads some active query head reads, summed over layers
    n_kv_act = sum(len({h // g for h in np.flatnonzero(m)}) for m in masks)
    # a control pattern reads no Q or K: only its lists count
    sel_bytes = ((1.0 * B * (n_act + n_kv_act) * N * d * 2 if args.pattern == "content" else 0.0)
                 + 4.0 * tiles + 4.0 * B * n_act * w.nB)
    sel_gbs = sel_bytes / (sel_ms * 1e-3) / 1e9
    dense_flops = 4.0 * B * H * N * N * d * n_layers
    out = {
        "metric": METRIC,
        "value": round(value, 3),
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_max, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded; Q/K rank-8 sinusoidal position structure + noise, V ~ N(0,1); no weights)",
        "config": {
            "workload": describe(w, rho, H_kv) + (" x %d layers" % n_layers if n_layers > 1 else ""),
            "B": B, "H": H, "H_kv": H_kv, "N": N, "d": d, "layers": n_layers, "density_budget": rho,
            "lists": args.pattern,
            "active_heads": n_act,
            "density_realized": round(tiles / (B * n_act * w.nB ** 2), 5),
            "selected_tiles": int(tiles),
            "computed_tiles": computed,  # 64 x 64 tiles the paired 128-row walk computes (effective TFLOP/s counts
                                         # only the selected ones): pairing efficiency = selected / computed
            "pairing_efficiency": round(tiles / computed, 4) if computed else None,
            "l2": "flushed between steps (512 MB write outside the per-step events)" if flush
                  else "inputs larger than L2 (%.0f MB of Q/K/V)" % (in_bytes / 1e6),
            "key_mask": "padding tokens masked inside kept tiles" if km_dev is not None else None,
            "parallelism": "replicas x%d (independent batches, no collective)" % world,
            "launch": "each step captured once as a CUDA graph and replayed (dense and SDPA likewise); stage "
                      "times from a second run of as many steps launched eagerly with events between the stages"
                      if graph is not None else "eager launches",
        },
        "breakdown_ms": {"select": round(sel_ms, 5), "plan": round(statistics.mean(t_plan), 5),
                         "attention": round(att_ms, 5)},
        "time_stats_ms": {"step": time_stats(t_step), "select": time_stats(t_sel), "plan": time_stats(t_plan),
                          "attention": time_stats(t_att)},
        "speedup_vs_dense": round(dense_ms / ms_step, 3) if dense_ms else None,
        "attention_speedup_vs_dense": round(dense_ms / att_ms, 3) if dense_ms else None,
        "dense_ms": round(dense_ms, 5) if dense_ms else None,
        "dense_tflops": round(dense_flops / (dense_ms * 1e-3) / 1e12, 2) if dense_ms else None,
        "dense_roofline_frac": round(dense_flops / (dense_ms * 1e-3) / 1e12 / pk["bf16_tflops"], 4) if dense_ms
        else None,
        "torch_sdpa_dense_ms": round(sdpa_ms, 5) if sdpa_ms else None,
        "speedup_vs_torch_sdpa": round(sdpa_ms / ms_step, 3) if sdpa_ms else None,
        "roofline": {
            "kernel": "sparse_attn_kernel<%d>" % d,
            "bound": "tensor",
            "achieved": round(achieved, 2),
            "peak": pk["bf16_tflops"],
            "unit": "TFLOP/s",
            "frac": round(achieved / pk["bf16_tflops"], 4),
            "peak_kind": "%s burst dense bf16 (frac vs %s sustained %.1f: %.4f)" % (
                pk_kind, pk_kind, pk["bf16_tflops_sustained"], achieved / pk["bf16_tflops_sustained"]),
            "traffic": traffic,
        },
        "selection_roofline": {
            "bound": "hbm", "achieved": round(sel_gbs, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
            "frac": round(sel_gbs / pk["hbm_gbs"], 4), "algorithmic_bytes": int(sel_bytes),
        },
        "e2e": {"value": round(job_value(flops_step, e2e_ms, world), 3), "unit": UNIT,
                "h2d_bytes_per_step": int(in_bytes), "d2h_bytes_per_step": int(O.numel() * 2 * n_layers),
                "ms_per_step": round(e2e_ms, 4),
                "copies": "pinned host buffers; unit u+1's inputs in and unit u-1's O out overlap unit u "
                          "(a unit is one layer of one step)"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk,
    }
    if n_layers > 1:
        out["per_layer_ms"] = {"step": round(ms_max / n_layers, 5), "select": round(sel_ms / n_layers, 5),
                               "attention": round(att_ms / n_layers, 5),
                               "dense": round(dense_ms / n_layers, 5) if dense_ms else None}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = oracle_sample(w, rho, target_s=args.cpu_seconds, seed=args.seed + rank, g=g)
        cb.pop("seconds", None)
        if n_layers > 1:
            cb["sample"] += "; layer 0 of %d" % n_layers
        out["cpu_baseline"] = cb
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


def run_crossover(args):
    """Sparse step (select + plan + attention) against this library's dense
    kernel over sequence lengths, on one GPU: the joint config's heads and
    head size at its density, image tokens only (rows of 128 tokens)."""
    import torch
    import prompt_aware_head_b200 as sa
    from workloads import make_workload

    if int(os.environ.get("WORLD_SIZE", "1")) > 1:
        raise SystemExit("--crossover runs on one GPU")
    dev = torch.device("cuda", 0)
    base = WORKLOADS["joint"]
    rho = args.density if args.density else base.densities[0]
    stream = torch.cuda.current_stream(dev)
    scratch = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    points = []
    for N in (512, 1024, 1536, 2048, 3072, 4096, 6144, 8192, 12288, 16384, 24576, 32768):
        w = make_workload("joint", N=N, segments=(), grid=(N // 128, 128))
        B, H, d = w.B, w.H, w.d
        Q, K, V = (torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16) for x in make_qkv(w))
        L = sa.Layout([], N)
        ws_bytes = sa.sa_workspace_size(B, H, N, d)
        ws = torch.zeros(ws_bytes, dtype=torch.uint8, device=dev)
        sa.sa_workspace_init(ws, ws_bytes, stream)
        idx = torch.zeros((B, H, w.nB, L.cap), dtype=torch.int32, device=dev)
        counts = torch.zeros((B, H, w.nB), dtype=torch.int32, device=dev)
        O = torch.empty_like(Q)

        def sparse(st=None):
            sa.sa_select_blocks(L, Q, K, B, H, d, rho, None, 0, idx, counts, None, ws, ws_bytes, st or stream)
            sa.sa_block_sparse_attention(Q, K, V, B, H, N, d, idx, counts, L.cap, None, 0, 0.0, O, ws, ws_bytes,
                                         st or stream)

        def dense(st=None):
            sa.sa_dense_attention(Q, K, V, B, H, N, d, 0.0, O, ws, ws_bytes, st or stream)

        def as_graph(fn):  # both sides launched the same way as the bench's steps
            cap = torch.cuda.Stream(dev)
            cap.wait_stream(stream)
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=cap, capture_error_mode="thread_local"):
                fn(cap)
            stream.wait_stream(cap)
            return gr

        ms = []
        graphs = []
        for fn in (sparse, dense):
            for _ in range(args.warmup):
                fn()
            if not args.no_graph:
                graphs.append(as_graph(fn))
                fn = graphs[-1].replay
                fn()
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(args.steps)]
            for a, b in ev:
                scratch.fill_(1.0)  # flush L2 outside the events
                a.record(stream)
                fn()
                b.record(stream)
            torch.cuda.synchronize()
            ms.append(statistics.mean(a.elapsed_time(b) for a, b in ev))
        assert sa.sa_check(ws, stream) == sa.SA_OK
        points.append((N, ms[0], ms[1]))
        del graphs
        torch.cuda.synchronize()
        L.release()
        del Q, K, V, O, ws, idx, counts
    n_star, kind = crossover(points)
    print(json.dumps({
        "metric": "sparse/dense crossover sequence length", "value": round(n_star) if n_star else None,
        "unit": "tokens", "crossover": kind, "higher_is_better": False, "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "dtype": "bf16", "data": "synthetic (seeded)",
        "config": {"workload": "B1 H24 d128, image tokens only (rows of 128), density %.2f" % rho,
                   "l2": "flushed before every timed call (512 MB write outside the events)",
                   "sparse": "sa_select_blocks + sa_block_sparse_attention", "dense": "sa_dense_attention",
                   "launch": "each side captured as a CUDA graph and replayed" if not args.no_graph else "eager"},
        "points": [{"N": n, "sparse_ms": round(a, 5), "dense_ms": round(b, 5), "speedup": round(b / a, 3)}
                   for n, a, b in points],
    }), flush=True)


def run_reference(args):
    """The fp64 CPU oracle as it stands, timed on the host cores (rank 0 only)."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    w = WORKLOADS[args.workload]
    rho = args.density if args.density else w.densities[0]
    H_kv = args.kv_heads or w.H
    if H_kv < 1 or w.H % H_kv:
        raise SystemExit("--kv-heads must divide the workload's %d heads" % w.H)
    g = w.H // H_kv
    per_step = max(2.0, 120.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        oracle_sample(w, rho, target_s=min(per_step, 2.0), seed=args.seed, g=g)
    vals, secs, last = [], [], None
    for _ in range(args.steps):
        last = oracle_sample(w, rho, target_s=per_step, seed=args.seed, g=g)
        vals.append(last["value"])
        secs.append(last["seconds"])
    value = statistics.mean(vals)
    out = {
        "impl": "reference",
        "metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(1e3 * statistics.mean(secs), 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (same seeded generator)",
        "config": {"workload": describe(w, rho, H_kv), "B": w.B, "H": w.H, "H_kv": H_kv, "N": w.N, "d": w.d,
                   "density_budget": rho},
        "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": last["cores"], "kind": "oracle",
                         "sample": last["sample"], "split": last["split"]},
        "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="joint")
    ap.add_argument("--density", type=float, default=None)
    ap.add_argument("--pattern", choices=["content", "radial", "random", "window"], default="content",
                    help="block lists from the content selector (default), or a control pattern at the same pins: "
                         "radial band at the same k, random blocks at the same k, or a 512-token window + 8 global "
                         "blocks")
    ap.add_argument("--kv-heads", type=int, default=None,
                    help="grouped-query layout: K and V hold this many heads, each shared by H / kv-heads "
                         "consecutive query heads (default: as many as Q)")
    ap.add_argument("--seed", type=int, default=0, help="input seed (rank r draws seed + r)")
    ap.add_argument("--pad-mask", action="store_true",
                    help="mask the layout's padding tokens as keys inside the kept tiles (token-level key mask)")
    ap.add_argument("--layers", type=int, default=None,
                    help="layers per step for a multi-layer workload (default: all of them, 64 for the stack)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch each step's kernels eagerly instead of replaying a captured CUDA graph")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--crossover", action="store_true",
                    help="instead of the step benchmark: the sequence length from which the sparse step beats dense "
                         "(one GPU)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.crossover:
        run_crossover(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
