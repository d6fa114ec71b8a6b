"""Benchmark of the VSA2 hot path on B200: router -> per-sequence TopK -> block-sparse attention.

One step = one pass of the whole path over one batch of synthetic input of the 720p workload
(B=1, H=20, D=128, grid 56x48x80 = 215,040 tokens, 3360 tiles, top64, bf16): router pooling,
router scores, TopK, attention forward. With --workload 480p_train_top64 the step also runs the
backward pass (training step of the fine branch; the router gets no gradient).

Prints one JSON line (rank 0). `value` is the effective TFLOPS of the whole step: FLOPs of the
selected tile pairs only (4*64*64*D per pair forward, 2.5x that backward) over the step time,
summed over ranks, divided by the max step time over ranks.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import threading
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synthetic as S  # noqa: E402

METRIC = "VSA2 attn fwd ms & effective TFLOPS, 215K tok H20 D128 top64"
DEFAULT_WORKLOAD = "720p_top64"
# kernels of ours launched per call (memsets are not counted)
LAUNCHES = {"router": 2, "topk": 9, "topk_csc": 11, "fwd": 1, "bwd": 2}


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p["hbm_gbs"], p["bf16_tflops"], p.get("bf16_tflops_sustained", p["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# Committed ncu summaries that carry DRAM bytes per selected pair for one kernel source and
# workload shape: (summary file, kernel source, token grid).
TRAFFIC_PROFILES = {
    "fwd": ("attn_fwd_tc_720p_4heads.md", "attn_fwd_tc.cu", (56, 48, 80)),
    "bwd": ("attn_bwd_tc_480p_4heads.md", "attn_bwd_tc.cu", (28, 32, 52)),
}


def profiled_traffic(kind, wl, pairs):
    """DRAM bytes of one launch from the committed ncu summary, scaled by selected pairs; None
    when the kernel source changed since the counters were taken or for other workloads."""
    name, kernel_src, grid = TRAFFIC_PROFILES[kind]
    if wl.grid != grid or wl.head_dim != 128 or wl.topk != 64:
        return None
    try:
        txt = open(os.path.join(ROOT, "profiles", name)).read()
        src = open(os.path.join(ROOT, "trainable_block_sparse_fine_b200", "csrc", kernel_src), "rb").read()
    except OSError:
        return None
    per = re.search(r"dram_bytes_per_pair:\s*(\d+)", txt)
    sha = re.search(r"source_sha1:\s*([0-9a-f]{40})", txt)
    if not (per and sha) or hashlib.sha1(src).hexdigest() != sha.group(1):
        return None
    return int(per.group(1)) * pairs


def pair_flops(wl, pairs, backward):
    f = 4.0 * 64 * 64 * wl.head_dim * pairs
    return f * (3.5 if backward else 1.0)


class Clocks:
    """Samples the SM clock and the clock-event (throttle) reasons every 20 ms through NVML, in
    a thread, while the timed region runs (read-only queries; no setting is changed). Falls back
    to an `nvidia-smi -lms` subprocess when NVML cannot be opened."""

    PERIOD_S = 0.02

    def __init__(self, device_index):
        self.device_index = device_index
        self.samples = []  # (sm_mhz, max_mhz, reasons bitmask)
        self.proc = None
        self.lines = []
        self._stop = threading.Event()
        self._thread = None

    def _nvml_loop(self, nv, h):
        while True:
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
                get = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                    nv.nvmlDeviceGetCurrentClocksThrottleReasons
                self.samples.append((float(sm), float(mx), int(get(h))))
            except Exception:
                pass
            if self._stop.wait(self.PERIOD_S):
                return

    def __enter__(self):
        try:
            import pynvml as nv
            nv.nvmlInit()
            try:
                import torch
                idx = torch.cuda._get_nvml_device_index(self.device_index)
            except Exception:
                idx = self.device_index
            h = nv.nvmlDeviceGetHandleByIndex(idx)
            self._nv = nv
            self._thread = threading.Thread(target=self._nvml_loop, args=(nv, h), daemon=True)
            self._thread.start()
            return self
        except Exception:
            self._thread = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.device_index),
                 "--query-gpu=clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                 "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                 "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=2)
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
                self.lines = [l for l in out.splitlines() if l.strip()]
            except Exception:
                self.proc.kill()

    def summary(self):
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        sm, mx, reasons = [], 0.0, set()
        if self.samples:
            nv = self._nv
            bits = {"hw_slowdown": getattr(nv, "nvmlClocksEventReasonHwSlowdown", 0x8),
                    "hw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonHwThermalSlowdown", 0x40),
                    "sw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonSwThermalSlowdown", 0x20),
                    "sw_power_cap": getattr(nv, "nvmlClocksEventReasonSwPowerCap", 0x4)}
            for f_sm, f_mx, r in self.samples:
                sm.append(f_sm)
                mx = max(mx, f_mx)
                reasons.update(n for n in names if r & bits[n])
            src = "nvml"
        else:
            for l in self.lines:
                f = [x.strip() for x in l.split(",")]
                try:
                    sm.append(float(f[0]))
                    mx = max(mx, float(f[1]))
                except (ValueError, IndexError):
                    continue
                for n, v in zip(names, f[4:8]):
                    if v.lower() == "active":
                        reasons.add(n)
            src = "nvidia-smi"
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm),
                "source": src}


# ----------------------------------------------------------------------------------------------
# reference arm and CPU baseline: the fp64 oracle on a bounded sample
# ----------------------------------------------------------------------------------------------
def oracle_sample(wl, budget_s=20.0, tiles=None):
    """Time the oracle's hot path on head 0 of batch 0: router + TopK on the whole head, the
    forward (and backward) on a sample of query tiles; extrapolate to all tiles and heads."""
    from oracle import vsa2_oracle as O

    q, k, v = (S.make_slice(wl, n, 0, 0) for n in ("q", "k", "v"))
    t0 = time.perf_counter()
    sc = O.router_scores(q, k).astype(np.float32)
    t1 = time.perf_counter()
    sel = O.topk_select(sc, wl.topk)
    t2 = time.perf_counter()
    N = wl.num_tiles
    rng = np.random.default_rng(0)
    order = rng.permutation(N)
    done, t_att = 0, 0.0
    for i in order:
        ts = time.perf_counter()
        O.sparse_attn_fwd(q, k, v, sel["kv_off"], sel["kv_idx"], query_tiles=[int(i)])
        t_att += time.perf_counter() - ts
        done += 1
        if tiles is not None and done >= tiles:
            break
        if tiles is None and (t2 - t0) + t_att > budget_s:
            break
    per_head = (t1 - t0) + (t2 - t1) + t_att * N / done
    if wl.backward:
        per_head += 2.5 * t_att * N / done  # backward restated as 2.5x the forward GEMM work
    total_s = per_head * wl.heads * wl.batch
    pairs = wl.batch * wl.heads * N * wl.topk
    flops = pair_flops(wl, pairs, wl.backward)
    return {"seconds_per_step": total_s, "tflops": flops / total_s / 1e12, "router_s": t1 - t0, "topk_s": t2 - t1,
            "fwd_tiles_sampled": done, "tiles": N,
            "sample": f"head 0 of {wl.heads}: router+TopK whole head, forward on {done}/{N} query tiles; "
                      f"extrapolated to {wl.heads} heads"}


def cores():
    return len(os.sched_getaffinity(0))


def run_reference(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    steps = []
    for _ in range(args.warmup):
        oracle_sample(wl, tiles=2)
    for _ in range(args.steps):
        steps.append(oracle_sample(wl, tiles=8))
    sec = statistics.mean(s["seconds_per_step"] for s in steps)
    pairs = wl.batch * wl.heads * wl.num_tiles * wl.topk
    val = pair_flops(wl, pairs, wl.backward) / sec / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOPS", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name, "batch": wl.batch, "heads": wl.heads, "head_dim": wl.head_dim,
                       "grid": list(wl.grid), "tokens": wl.tokens, "topk": wl.topk},
            "cpu_baseline": {"value": val, "unit": "TFLOPS", "cores": cores(), "kind": "oracle",
                             "sample": steps[-1]["sample"]},
            "e2e": {"value": val, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------------------------
# our arm
# ----------------------------------------------------------------------------------------------
def time_next_rows(e, x, wl, steps, stream, l2_flush, ev, hbm, tc_peak):
    """The coarse branch (Eq. 1-3) and the gated merge (Eq. 4, 13-14), and for training
    workloads their gradients, each timed on its own after the step, with L2 flushed before every
    launch. They are not part of the fine-branch step that the headline metric times."""
    import torch

    dev = x["q"].device
    B, H, N, L, D = wl.batch, wl.heads, wl.num_tiles, wl.tokens, wl.head_dim
    esize = 2 if wl.dtype == "bf16" else 4
    logits = torch.randn(B, H, L, generator=torch.Generator(device=dev).manual_seed(1234), device=dev)
    oc = torch.empty(B, H, N, D, dtype=x["q"].dtype, device=dev)
    lse_c = torch.empty(B, H, N, dtype=torch.float32, device=dev)
    out = torch.empty_like(x["q"])
    for _ in range(3):
        e.coarse_attn(x["q"], x["k"], x["v"], oc, lse_c)
        e.gated_merge(x["v"], logits, oc, out)  # V stands in for the fine output (same shape and dtype)
    tc, tm = [], []
    for _ in range(steps):
        t = [ev() for _ in range(4)]
        l2_flush.zero_()
        t[0].record(stream)
        e.coarse_attn(x["q"], x["k"], x["v"], oc, lse_c)
        t[1].record(stream)
        l2_flush.zero_()
        t[2].record(stream)
        e.gated_merge(x["v"], logits, oc, out)
        t[3].record(stream)
        torch.cuda.synchronize()
        tc.append(t[0].elapsed_time(t[1]))
        tm.append(t[2].elapsed_time(t[3]))
    extra = {}
    if wl.backward:  # gradients of the merge and of the coarse branch, after the fine backward
        grads = [torch.zeros(B, H, L, D, dtype=torch.float32, device=dev) for _ in range(3)]
        for _ in range(3):
            _, d_oc = e.gated_merge_bwd(x["do"], logits, oc)
            e.coarse_attn_bwd(x["q"], x["k"], x["v"], oc, lse_c, d_oc, *grads)
        tmb, tcb = [], []
        for _ in range(steps):
            t = [ev() for _ in range(4)]
            l2_flush.zero_()
            t[0].record(stream)
            e.gated_merge_bwd(x["do"], logits, oc)
            t[1].record(stream)
            l2_flush.zero_()
            t[2].record(stream)
            e.coarse_attn_bwd(x["q"], x["k"], x["v"], oc, lse_c, d_oc, *grads)
            t[3].record(stream)
            torch.cuda.synchronize()
            tmb.append(t[0].elapsed_time(t[1]))
            tcb.append(t[2].elapsed_time(t[3]))
        mb_ms, cb_ms = statistics.mean(tmb), statistics.mean(tcb)
        mb_bytes = B * H * L * D * esize + 8 * B * H * L + B * H * N * D * (esize + 4)
        cb_flops = 2.5 * 4.0 * N * N * D * B * H
        extra = {
            "gated_merge_bwd": {"ms": mb_ms, "algorithmic_bytes": mb_bytes, "gbs": mb_bytes / (mb_ms * 1e-3) / 1e9,
                                "hbm_frac": mb_bytes / (mb_ms * 1e-3) / 1e9 / hbm},
            "coarse_attn_bwd": {"ms": cb_ms, "effective_tflops": cb_flops / (cb_ms * 1e-3) / 1e12,
                                "kernels": "pool + pad + attn_bwd_dq_tc_kernel + attn_bwd_dkdv_tc_kernel + "
                                           "coarse_pool_bwd_kernel"},
        }
    # the token permutation (§2.2): Q from raster to cube-major order, one read and one write
    tp = []
    for it in range(3 + steps):
        t = [ev() for _ in range(2)]
        l2_flush.zero_()
        t[0].record(stream)
        e.to_cube_major(x["q"], out=out)
        t[1].record(stream)
        torch.cuda.synchronize()
        if it >= 3:
            tp.append(t[0].elapsed_time(t[1]))
    p_ms = statistics.mean(tp)
    p_bytes = 2 * B * H * L * D * esize
    extra["permute"] = {"ms": p_ms, "algorithmic_bytes": p_bytes, "gbs": p_bytes / (p_ms * 1e-3) / 1e9,
                        "hbm_frac": p_bytes / (p_ms * 1e-3) / 1e9 / hbm, "kernel": "permute_kernel (Q)"}
    err = e.device_error()
    if err != 0:
        raise RuntimeError(f"device error {err} in the coarse branch")
    c_ms, m_ms = statistics.mean(tc), statistics.mean(tm)
    c_flops = 4.0 * N * N * D * B * H
    pool_bytes = 3 * B * H * L * D * esize
    m_bytes = 2 * B * H * L * D * esize + B * H * L * 4 + B * H * N * D * esize
    return {
        "coarse_attn": {"ms": c_ms, "effective_tflops": c_flops / (c_ms * 1e-3) / 1e12,
                        "frac_of_sustained_bf16": c_flops / (c_ms * 1e-3) / 1e12 / tc_peak,
                        "pool_bytes": pool_bytes, "pool_floor_ms": pool_bytes / (hbm * 1e9) * 1e3,
                        "kernels": "coarse_pool_kernel + coarse_csr_kernel + attn_fwd_tc_kernel<true>"},
        "gated_merge": {"ms": m_ms, "algorithmic_bytes": m_bytes, "gbs": m_bytes / (m_ms * 1e-3) / 1e9,
                        "hbm_frac": m_bytes / (m_ms * 1e-3) / 1e9 / hbm},
        **extra,
    }


def run_ours(args, wl):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    import trainable_block_sparse_fine_b200 as V
    from trainable_block_sparse_fine_b200.sharding import max_over_ranks

    dev = torch.device("cuda", local)
    # weak scaling: every rank runs the full workload on its own batch element (seed offset)
    wl_r = wl.with_(seed=wl.seed + rank)
    names = ("q", "k", "v", "do") if wl.backward else ("q", "k", "v")
    dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    # inputs in pinned host memory (the end-to-end leg copies them every step); each fp32 array
    # is dropped once converted, and the generator's worker pool is shared by the ranks of a node
    workers = max(1, min(16, len(os.sched_getaffinity(0)) // max(1, int(os.environ.get("LOCAL_WORLD_SIZE", world)))))
    pinned = {}
    for n in names:
        a32 = S.make_tensor(wl_r, n, workers=workers)
        pinned[n] = torch.from_numpy(a32).to(dt).pin_memory()
        del a32
    x = {n: pinned[n].to(dev) for n in names}
    e = V.VSA2(wl.batch, wl.heads, wl.head_dim, wl.grid, wl.dtype, wl.topk)
    stream = torch.cuda.current_stream()
    l2_flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    scores = torch.empty(wl.batch, wl.heads, wl.num_tiles, wl.num_tiles, dtype=torch.float32, device=dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)

    def step(timers=None):
        t = timers or {}
        if t: t["r0"].record(stream)
        e.router_scores(x["q"], x["k"], out=scores)
        if t: t["r1"].record(stream)
        sel = e.topk_select(scores, wl.topk, csc=wl.backward)
        if t: t["t1"].record(stream)
        o, lse = e.attn_fwd(x["q"], x["k"], x["v"], sel[0], sel[1])
        if t: t["f1"].record(stream)
        if wl.backward:
            grads = e.attn_bwd(x["q"], x["k"], x["v"], o, lse, x["do"], *sel)
            if t: t["b1"].record(stream)
            return o, grads
        return o, None

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    err = e.device_error()
    if err != 0:
        raise RuntimeError(f"device error {V.vsa2_status_string(err)} during warm-up")

    keys = ["r0", "r1", "t1", "f1"] + (["b1"] if wl.backward else [])
    per = {k: [] for k in ("router", "topk", "fwd", "bwd", "step")}
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with Clocks(local) as clk:
        for _ in range(args.steps):
            l2_flush.zero_()  # L2 flush between timed steps (outside the timed events)
            timers = {k: ev() for k in keys}
            step(timers)
            torch.cuda.synchronize()
            per["router"].append(timers["r0"].elapsed_time(timers["r1"]))
            per["topk"].append(timers["r1"].elapsed_time(timers["t1"]))
            per["fwd"].append(timers["t1"].elapsed_time(timers["f1"]))
            if wl.backward:
                per["bwd"].append(timers["f1"].elapsed_time(timers["b1"]))
            per["step"].append(timers["r0"].elapsed_time(timers[keys[-1]]))
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms = max_over_ranks(statistics.mean(per["step"]), dev)
    err = e.device_error()
    if err != 0:
        raise RuntimeError(f"device error {V.vsa2_status_string(err)} in the timed region")

    pairs = wl.batch * wl.heads * wl.num_tiles * wl.topk
    flops_rank = pair_flops(wl, pairs, wl.backward)
    value = flops_rank * world / (ms * 1e-3) / 1e12

    # end to end through the public API: H2D of the step's inputs, the step, D2H of its output
    h2d = sum(pinned[n].numel() * pinned[n].element_size() for n in names)
    out_host = torch.empty(x["q"].shape, dtype=dt, pin_memory=True)
    d2h = out_host.numel() * out_host.element_size()
    e2e_ms = []
    for it in range(0 if args.no_e2e else args.warmup + args.steps):
        l2_flush.zero_()
        a, b = ev(), ev()
        a.record(stream)
        if wl.backward:
            xs = {n: pinned[n].to(dev, non_blocking=True) for n in names}
            o = e.forward(xs["q"], xs["k"], xs["v"], wl.topk, csc=True)
            e.attn_bwd(xs["q"], xs["k"], xs["v"], o[0], o[1], xs["do"], *o[2])
            out_host.copy_(o[0], non_blocking=True)
        else:  # one call on host buffers; its PCIe copies overlap the kernels group by group
            e.forward_host(pinned["q"], pinned["k"], pinned["v"], wl.topk, o=out_host)
        b.record(stream)
        torch.cuda.synchronize()
        if it >= args.warmup:
            e2e_ms.append(a.elapsed_time(b))
    e2e = max_over_ranks(statistics.mean(e2e_ms) if e2e_ms else float("nan"), dev)

    hbm, bf16_burst, bf16_sus, peak_kind = load_peaks()
    next_rows = None
    if not args.no_next:
        next_rows = time_next_rows(e, x, wl, args.steps, stream, l2_flush, ev, hbm, bf16_sus)
    fwd_ms = statistics.mean(per["fwd"])
    fwd_tflops = pair_flops(wl, pairs, False) / (fwd_ms * 1e-3) / 1e12
    if wl.backward:  # the backward pass (dQ kernel + dK/dV kernel) dominates a training step
        bwd_ms = statistics.mean(per["bwd"])
        bwd_tflops = 2.5 * pair_flops(wl, pairs, False) / (bwd_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "kernel": "attn_bwd_dq_tc_kernel + attn_bwd_dkdv_tc_kernel (one call)",
                "achieved": bwd_tflops, "traffic": profiled_traffic("bwd", wl, pairs)}
    else:
        roof = {"bound": "tensor", "kernel": "attn_fwd_tc_kernel", "achieved": fwd_tflops,
                "traffic": profiled_traffic("fwd", wl, pairs)}
    router_ms = statistics.mean(per["router"])
    router_bytes = 2 * wl.batch * wl.heads * wl.tokens * wl.head_dim * (2 if wl.dtype == "bf16" else 4) \
        + wl.batch * wl.heads * wl.num_tiles ** 2 * 4
    launches = LAUNCHES["router"] + (LAUNCHES["topk_csc"] if wl.backward else LAUNCHES["topk"]) + LAUNCHES["fwd"] \
        + (LAUNCHES["bwd"] if wl.backward else 0)
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            c = oracle_sample(wl, budget_s=20.0)
            cpu = {"value": c["tflops"], "unit": "TFLOPS", "cores": cores(), "kind": "oracle", "sample": c["sample"],
                   "seconds_per_step": c["seconds_per_step"]}
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": world, "steps": args.steps,
            "warmup": max(3, args.warmup), "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16" if wl.dtype == "bf16" else "fp32", "data": "synthetic",
            "config": {"workload": wl.name, "batch": wl.batch, "heads": wl.heads, "head_dim": wl.head_dim,
                       "grid": list(wl.grid), "tokens": wl.tokens, "tiles": wl.num_tiles, "topk": wl.topk,
                       "selected_pairs_per_rank": pairs, "backward": wl.backward,
                       "l2": "256 MB buffer written between timed steps; inputs also exceed L2"},
            "stages_ms": {"router": router_ms, "topk": statistics.mean(per["topk"]), "fwd": fwd_ms,
                          **({"bwd": statistics.mean(per["bwd"])} if wl.backward else {})},
            "fwd_kernel": {"ms": fwd_ms, "effective_tflops": fwd_tflops},
            "router": {"ms": router_ms, "algorithmic_bytes": router_bytes,
                       "gbs": router_bytes / (router_ms * 1e-3) / 1e9, "hbm_frac": router_bytes / (router_ms * 1e-3) / 1e9 / hbm},
            **({"bwd_pass": {"ms": bwd_ms, "effective_tflops": bwd_tflops}} if wl.backward else {}),
            "roofline": {"bound": roof["bound"], "kernel": roof["kernel"], "achieved": roof["achieved"],
                         "peak": bf16_sus, "unit": "TFLOP/s", "frac": roof["achieved"] / bf16_sus,
                         "peak_kind": f"{peak_kind} sustained bf16", "traffic": roof["traffic"]},
            "cpu_baseline": cpu,
            "e2e": {"value": flops_rank * world / (e2e * 1e-3) / 1e12, "unit": "TFLOPS", "ms_per_step": e2e,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "api": "VSA2.forward + attn_bwd after H2D copies" if wl.backward else "vsa2_forward_host"},
            "gpu_launches": launches * args.steps,
            "clocks": clk.summary(),
            **({"next_rows": next_rows} if next_rows else {}),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=list(S.WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end (host buffers) measurement")
    ap.add_argument("--heads", type=int, default=None, help="override the head count (profiling runs)")
    ap.add_argument("--no-next", action="store_true", help="skip timing the coarse branch and the gated merge")
    args = ap.parse_args()
    wl = S.WORKLOADS[args.workload]
    if args.heads:
        wl = wl.with_(heads=args.heads)
    if args.impl == "reference":
        run_reference(args, wl)
    else:
        run_ours(args, wl)


if __name__ == "__main__":
    main()
