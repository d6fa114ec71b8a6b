"""Benchmark of the VSA2 hot path on B200: router -> per-sequence TopK -> block-sparse attention.

One step = one pass of the whole path over one batch of synthetic input: router pooling, router
scores, TopK, attention forward, and for the training workload the backward pass too (the
router gets no gradient). The configurations, each printed as one JSON line by rank 0:
  tiny              B=1, H=2, D=64, grid 8x16x16, top8, fp32 (forward)
  480p_top64        B=1, H=20, D=128, grid 28x32x52, top64, bf16 (forward)
  480p_top128       the same tensors, top128
  480p_train_top64  the same tensors, top64, forward + backward
  720p_top64        B=1, H=20, D=128, grid 56x48x80 (215,040 tokens, 3360 tiles), top64, bf16
                    (forward): the headline, printed last, with a digest of all lines.
`value` is the effective TFLOPS of the whole step: FLOPs of the selected tile pairs only
(4*64*64*D per pair forward, 2.5x that backward) over the step time, summed over ranks, divided
by the max step time over ranks. `roofline.frac` is against the measured burst bf16 peak.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME|all]
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
HEADLINE = "720p_top64"
# every configuration of the benchmark, in the order they run; the headline prints last
ALL_WORKLOADS = ["tiny", "480p_top64", "480p_top128", "480p_train_top64", HEADLINE]
# kernels of ours launched per call (memsets are not counted)
LAUNCHES = {"router": 2, "topk": 10, "topk_csc": 12, "fwd": 1, "bwd": 2}


def load_sm_max_mhz():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f).get("sm_max_mhz", 1965.0))
    except Exception:
        return 1965.0


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


def profiled_traffic(kind, wl, pairs, root=ROOT):
    """DRAM bytes of one launch from the committed ncu summary, scaled by selected pairs; None
    when the kernel source changed since the counters were taken or for other workloads."""
    name, kernel_src, grid = TRAFFIC_PROFILES[kind]
    if wl.grid != grid or wl.head_dim != 128 or wl.topk != 64:
        return None
    try:
        txt = open(os.path.join(root, "profiles", name)).read()
        src = open(os.path.join(root, "trainable_block_sparse_fine_b200", "csrc", kernel_src), "rb").read()
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
    forward (and backward) on a sample of query tiles; extrapolate to all tiles and heads.
    Returns the extrapolated step time and the seconds the sample actually took."""
    from oracle import vsa2_oracle as O

    q, k, v = (S.make_slice(wl, n, 0, 0) for n in ("q", "k", "v"))
    do = S.make_slice(wl, "do", 0, 0) if wl.backward else None
    t0 = time.perf_counter()
    sc = O.router_scores(q, k).astype(np.float32)
    t1 = time.perf_counter()
    sel = O.topk_select(sc, wl.topk)
    t2 = time.perf_counter()
    N = wl.num_tiles
    order = np.random.default_rng(0).permutation(N)
    done, t_att = 0, 0.0
    for i in order:
        ts = time.perf_counter()
        O.sparse_attn_fwd(q, k, v, sel["kv_off"], sel["kv_idx"], query_tiles=[int(i)])
        if wl.backward:
            O.sparse_attn_bwd(q, k, v, do, sel["kv_off"], sel["kv_idx"], query_tiles=[int(i)])
        t_att += time.perf_counter() - ts
        done += 1
        if tiles is not None and done >= tiles:
            break
        if tiles is None and (t2 - t0) + t_att > budget_s:
            break
    per_head = (t1 - t0) + (t2 - t1) + t_att * N / done
    total_s = per_head * wl.heads * wl.batch
    pairs = wl.batch * wl.heads * N * wl.topk
    flops = pair_flops(wl, pairs, wl.backward)
    what = "forward and backward" if wl.backward else "forward"
    return {"seconds_per_step": total_s, "tflops": flops / total_s / 1e12, "router_s": t1 - t0, "topk_s": t2 - t1,
            "sample_s": (t2 - t0) + t_att, "fwd_tiles_sampled": done, "tiles": N,
            "sample": f"head 0 of {wl.heads}: router+TopK whole head, {what} on {done}/{N} query tiles; "
                      f"step time extrapolated to all tiles and {wl.heads} heads"}


def cores():
    return len(os.sched_getaffinity(0))


def run_reference(args, wl):
    """The reference arm: the fp64 oracle, as it stands, on this host's cores. Each step is a
    bounded sample (router and TopK of one head, the attention of 8 of its query tiles);
    `ms_per_step` is the time that sample took, `value` the whole step's effective TFLOPS
    extrapolated from it."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    steps = []
    for _ in range(args.warmup):
        oracle_sample(wl, tiles=2)
    for _ in range(args.steps):
        steps.append(oracle_sample(wl, tiles=8))
    sec = statistics.mean(s["seconds_per_step"] for s in steps)
    sample_ms = statistics.mean(s["sample_s"] for s in steps) * 1e3
    pairs = wl.batch * wl.heads * wl.num_tiles * wl.topk
    val = pair_flops(wl, pairs, wl.backward) / sec / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOPS", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": sample_ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name, "batch": wl.batch, "heads": wl.heads, "head_dim": wl.head_dim,
                       "grid": list(wl.grid), "tokens": wl.tokens, "topk": wl.topk},
            "extrapolated_ms_per_full_step": sec * 1e3,
            "cpu_baseline": {"value": val, "unit": "TFLOPS", "cores": cores(), "kind": "oracle",
                             "sample": steps[-1]["sample"]},
            "e2e": {"value": val, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------------------------
# our arm
# ----------------------------------------------------------------------------------------------
def time_next_rows(e, x, wl, steps, stream, l2_flush, ev, hbm, tc_peak, sel=None):
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
    if sel is not None:
        # the fine forward with the gated merge in its epilogue (Eq. 12-14 in one pass), against the
        # forward followed by the merge kernel; both on the step's selection
        tf, ts = [], []
        for it in range(3 + steps):
            t = [ev() for _ in range(4)]
            l2_flush.zero_()
            t[0].record(stream)
            e.attn_fwd_gated(x["q"], x["k"], x["v"], sel[0], sel[1], logits, oc)
            t[1].record(stream)
            l2_flush.zero_()
            t[2].record(stream)
            o_f, _ = e.attn_fwd(x["q"], x["k"], x["v"], sel[0], sel[1])
            e.gated_merge(o_f, logits, oc, out=o_f)
            t[3].record(stream)
            torch.cuda.synchronize()
            if it >= 3:
                tf.append(t[0].elapsed_time(t[1]))
                ts.append(t[2].elapsed_time(t[3]))
        extra["fine_fwd_gated"] = {"ms": statistics.mean(tf), "fwd_then_merge_ms": statistics.mean(ts),
                                   "kernel": "attn_fwd_tc_kernel<0, true> (merge in the epilogue)"}
    if wl.dtype == "bf16" and D == 128:
        # the whole-attention path takes Qc, Kc (Eq. 1) from the router's pass over Q and K: the
        # router call with and without the tile means, and the coarse call that then reads only V
        sc = torch.empty(B, H, N, N, dtype=torch.float32, device=dev)
        tr, trp, tcf = [], [], []
        for it in range(3 + steps):
            t = [ev() for _ in range(6)]
            l2_flush.zero_()
            t[0].record(stream)
            e.router_scores(x["q"], x["k"], out=sc)
            t[1].record(stream)
            l2_flush.zero_()
            t[2].record(stream)
            e.router_scores(x["q"], x["k"], out=sc, coarse_pool=True)
            t[3].record(stream)
            l2_flush.zero_()
            t[4].record(stream)
            e.coarse_attn(x["q"], x["k"], x["v"], oc, lse_c, pooled_qk=True)
            t[5].record(stream)
            torch.cuda.synchronize()
            if it >= 3:
                tr.append(t[0].elapsed_time(t[1]))
                trp.append(t[2].elapsed_time(t[3]))
                tcf.append(t[4].elapsed_time(t[5]))
        del sc
        v_bytes = B * H * L * D * esize
        extra["coarse_attn_pooled_in_router"] = {
            "ms": statistics.mean(tcf), "router_ms": statistics.mean(tr),
            "router_with_tile_means_ms": statistics.mean(trp), "v_pool_bytes": v_bytes,
            "v_pool_floor_ms": v_bytes / (hbm * 1e9) * 1e3,
            "kernels": "router_pool_kernel<..., true> writes Qc, Kc; coarse_pool_kernel (V) + coarse_csr_kernel + "
                       "attn_fwd_tc_kernel<1>"}
    if (wl.dtype == "bf16" and D == 128 and wl.topk % 2 == 0 and not getattr(wl, "padded", False)
            and wl.grid[0] % 4 == 0 and wl.grid[1] % 4 == 0 and wl.grid[2] % 8 == 0):
        # 128-token tiles (4x4x8, 8-token router sub-cubes): the same tensors reordered by the
        # permutation kernels, the same sparsity (top k/2 of tiles twice as large); router + TopK
        # once, then the forward, which runs M=128 query tiles against whole 128-token KV tiles
        from trainable_block_sparse_fine_b200 import VSA2
        k2 = wl.topk // 2
        e2 = VSA2(B, H, D, wl.grid, "bf16", k2, tile=(4, 4, 8), pool=(2, 2, 2))
        x2 = {n: e2.to_cube_major(e.to_raster(x[n])) for n in ("q", "k", "v")}
        sc2 = e2.router_scores(x2["q"], x2["k"])
        off2, idx2 = e2.topk_select(sc2, k2, csc=False)[:2]
        del sc2
        t2 = []
        for it in range(3 + steps):
            t = [ev() for _ in range(2)]
            l2_flush.zero_()
            t[0].record(stream)
            e2.attn_fwd(x2["q"], x2["k"], x2["v"], off2, idx2)
            t[1].record(stream)
            torch.cuda.synchronize()
            if it >= 3:
                t2.append(t[0].elapsed_time(t[1]))
        if e2.device_error() != 0:
            raise RuntimeError("device error in the 128-token-tile forward")
        pairs2 = int(off2[..., -1].sum().item())
        f2 = 4.0 * 128 * 128 * D * pairs2
        ms2 = statistics.mean(t2)
        extra["fwd_128_token_tiles"] = {
            "ms": ms2, "topk": k2, "tile_pairs": pairs2, "effective_tflops": f2 / (ms2 * 1e-3) / 1e12,
            "frac_of_burst_bf16": f2 / (ms2 * 1e-3) / 1e12 / tc_peak,
            "kernel": "attn_fwd_b128_kernel (M=128 query tiles, whole 128-token KV tiles)"}
        del x2, off2, idx2, e2
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
                        "frac_of_burst_bf16": c_flops / (c_ms * 1e-3) / 1e12 / tc_peak,
                        "pool_bytes": pool_bytes, "pool_floor_ms": pool_bytes / (hbm * 1e9) * 1e3,
                        "kernels": "coarse_pool_kernel + coarse_csr_kernel + attn_fwd_tc_kernel<true>"},
        "gated_merge": {"ms": m_ms, "algorithmic_bytes": m_bytes, "gbs": m_bytes / (m_ms * 1e-3) / 1e9,
                        "hbm_frac": m_bytes / (m_ms * 1e-3) / 1e9 / hbm},
        **extra,
    }


def time_dense(x, wl, stream, l2_flush, ev, iters=2):
    """Dense softmax attention over the same Q, K, V (every tile pair), the comparison the pages
    make for their attention speed-up (paper §4, Fig. 8, against FlashAttention-3 on H800). Timed
    with torch's scaled_dot_product_attention on each backend it offers for these tensors; the
    fastest is reported. A library kernel, timed for context only: it is not part of the path."""
    import torch
    from torch.nn.attention import SDPBackend, sdpa_kernel

    B, H, L, D = wl.batch, wl.heads, wl.tokens, wl.head_dim
    flops = 4.0 * L * L * D * B * H
    out = {}
    for name, be in (("cudnn", SDPBackend.CUDNN_ATTENTION), ("flash", SDPBackend.FLASH_ATTENTION)):
        try:
            with sdpa_kernel([be]):
                torch.nn.functional.scaled_dot_product_attention(x["q"], x["k"], x["v"])
                torch.cuda.synchronize()
                ts = []
                for _ in range(iters):
                    l2_flush.zero_()
                    a, b = ev(), ev()
                    a.record(stream)
                    torch.nn.functional.scaled_dot_product_attention(x["q"], x["k"], x["v"])
                    b.record(stream)
                    torch.cuda.synchronize()
                    ts.append(a.elapsed_time(b))
            out[name] = statistics.mean(ts)
        except Exception as exc:  # a backend that does not take these shapes on this build
            out[name] = f"unavailable: {type(exc).__name__}"
    times = {k: v for k, v in out.items() if isinstance(v, float)}
    if not times:
        return {"backends": out}
    best = min(times, key=times.get)
    return {"ms": times[best], "backend": f"torch sdpa ({best})", "backends": out,
            "effective_tflops": flops / (times[best] * 1e-3) / 1e12, "flops": flops}


_inputs_cache = {}


def device_inputs(wl, names, rank, world, dev):
    """Pinned host copies (the end-to-end leg copies them every step) and device copies of the
    workload's tensors; workloads on the same grid and seed share them (480p top64, top128 and
    the training step use the same Q, K, V)."""
    import torch

    key = (wl.grid, wl.dtype, wl.head_dim, wl.batch, wl.heads, wl.seed + rank)
    have = _inputs_cache.get(key)
    if have is None:
        _inputs_cache.clear()
        torch.cuda.empty_cache()
        have = _inputs_cache[key] = ({}, {})
    pinned, x = have
    dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    # each fp32 array is dropped once converted; the generator's worker pool is shared by the
    # ranks of a node
    workers = max(1, min(16, len(os.sched_getaffinity(0)) // max(1, int(os.environ.get("LOCAL_WORLD_SIZE", world)))))
    wl_r = wl.with_(seed=wl.seed + rank)  # weak scaling: every rank its own batch element
    for n in names:
        if n not in pinned:
            a32 = S.make_tensor(wl_r, n, workers=workers)
            pinned[n] = torch.from_numpy(a32).to(dt).pin_memory()
            del a32
            x[n] = pinned[n].to(dev)
    return pinned, x


def fp32_fma_peak_tflops(sm_max_mhz):
    """CUDA-core fp32 peak: 148 SMs x 128 FP32 lanes x 2 FLOP per FMA x the maximum SM clock."""
    return 148 * 128 * 2 * sm_max_mhz * 1e6 / 1e12


def mufu_peak(sm_max_mhz):
    """ex2 rate of the SFU (MUFU) pipes: 16 per clock per SM (a probe measured this on B200) x 148
    SMs x the maximum SM clock, in exponentials per second."""
    return 16 * 148 * sm_max_mhz * 1e6


def measure(args, wl, dev, rank, world):
    """One workload: warm-up, K timed steps, the end-to-end leg, the next rows; returns the JSON
    line (rank 0) or None."""
    import torch
    import trainable_block_sparse_fine_b200 as V
    from trainable_block_sparse_fine_b200.sharding import max_over_ranks
    import torch.distributed as dist

    names = ("q", "k", "v", "do") if wl.backward else ("q", "k", "v")
    dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    pinned, x = device_inputs(wl, names, rank, world, dev)
    e = V.VSA2(wl.batch, wl.heads, wl.head_dim, wl.grid, wl.dtype, wl.topk)
    stream = torch.cuda.current_stream()
    l2_flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    scores = torch.empty(wl.batch, wl.heads, wl.num_tiles, wl.num_tiles, dtype=torch.float32, device=dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)

    last_sel = {}

    def step(timers=None):
        t = timers or {}
        if t: t["r0"].record(stream)
        e.router_scores(x["q"], x["k"], out=scores)
        if t: t["r1"].record(stream)
        sel = e.topk_select(scores, wl.topk, csc=wl.backward)
        last_sel["sel"] = sel
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
    with Clocks(dev.index) as clk:
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
    sm_max = load_sm_max_mhz()
    next_rows = None
    if not args.no_next and wl.dtype == "bf16":
        next_rows = time_next_rows(e, x, wl, args.steps, stream, l2_flush, ev, hbm, bf16_burst,
                                   sel=last_sel.get("sel") if wl.head_dim == 128 else None)
        if wl.name == HEADLINE and not wl.backward:
            dense = time_dense(x, wl, stream, l2_flush, ev)
            if "ms" in dense:
                # the pages' ratio covers every op of Fig. 2 but the QKV projections: coarse branch,
                # router, TopK, fine branch and gated merge (here the fine forward with the merge
                # in its epilogue)
                fused = next_rows.get("fine_fwd_gated", {}).get("ms")
                fold = next_rows.get("coarse_attn_pooled_in_router")
                # coarse branch: with Qc, Kc from the router's pass (the router's extra time for the
                # tile means counted), else the standalone call
                coarse_ms = (fold["ms"] + max(0.0, fold["router_with_tile_means_ms"] - fold["router_ms"])
                             if fold else next_rows["coarse_attn"]["ms"])
                vsa2_ms = statistics.mean(per["router"]) + statistics.mean(per["topk"]) + coarse_ms + \
                    (fused if fused is not None else statistics.mean(per["fwd"]) + next_rows["gated_merge"]["ms"])
                dense["vsa2_all_ops_ms"] = vsa2_ms
                dense["speedup_all_ops"] = dense["ms"] / vsa2_ms
                dense["speedup_fine_branch_step"] = dense["ms"] / statistics.mean(per["step"])
            next_rows["dense_attention"] = dense
    fwd_ms = statistics.mean(per["fwd"])
    fwd_tflops = pair_flops(wl, pairs, False) / (fwd_ms * 1e-3) / 1e12
    tc = wl.dtype == "bf16" and wl.head_dim == 128
    if wl.backward:  # the backward pass (dQ kernel + dK/dV kernel) dominates a training step
        bwd_ms = statistics.mean(per["bwd"])
        bwd_tflops = 2.5 * pair_flops(wl, pairs, False) / (bwd_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "kernel": "attn_bwd_dq_tc_kernel + attn_bwd_dkdv_tc_kernel (one call)",
                "achieved": bwd_tflops, "traffic": profiled_traffic("bwd", wl, pairs)}
    elif tc:
        roof = {"bound": "tensor", "kernel": "attn_fwd_tc_kernel", "achieved": fwd_tflops,
                "traffic": profiled_traffic("fwd", wl, pairs)}
    else:  # fp32 / D=64: the CUDA-core forward
        roof = {"bound": "alu", "kernel": "attn_fwd_simt_kernel", "achieved": fwd_tflops, "traffic": None}
    if roof["bound"] == "tensor":
        peak, kind = bf16_burst, f"{peak_kind} burst bf16 (dense, cuBLAS 8192^3)"
        extra_peak = {"frac_of_sustained": roof["achieved"] / bf16_sus, "sustained_peak": bf16_sus}
    else:
        peak, kind = fp32_fma_peak_tflops(sm_max), f"derived fp32 FMA: 148 SMs x 128 lanes x 2 x {sm_max:.0f} MHz"
        extra_peak = {"note": "latency-bound at this size: the longest CSR row runs serially in one CTA (four threads per query row)"}
    router_ms = statistics.mean(per["router"])
    esize = 2 if wl.dtype == "bf16" else 4
    router_bytes = 2 * wl.batch * wl.heads * wl.tokens * wl.head_dim * esize + wl.batch * wl.heads * wl.num_tiles ** 2 * 4
    router_ex2 = 2.0 * wl.batch * wl.heads * (wl.tokens // 16) ** 2
    launches = LAUNCHES["router"] + (LAUNCHES["topk_csc"] if wl.backward else LAUNCHES["topk"]) + LAUNCHES["fwd"] \
        + (LAUNCHES["bwd"] if wl.backward else 0)
    if rank != 0:
        return None
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        c = oracle_sample(wl, budget_s=args.cpu_budget if wl.name == HEADLINE else min(args.cpu_budget, 6.0))
        cpu = {"value": c["tflops"], "unit": "TFLOPS", "cores": cores(), "kind": "oracle", "sample": c["sample"],
               "seconds_per_step": c["seconds_per_step"]}
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if wl.dtype == "bf16" else "fp32", "data": "synthetic",
        "config": {"workload": wl.name, "batch": wl.batch, "heads": wl.heads, "head_dim": wl.head_dim,
                   "grid": list(wl.grid), "tokens": wl.tokens, "tiles": wl.num_tiles, "topk": wl.topk,
                   "selected_pairs_per_rank": pairs, "backward": wl.backward,
                   "l2": "256 MB buffer written between timed steps"},
        "stages_ms": {"router": router_ms, "topk": statistics.mean(per["topk"]), "fwd": fwd_ms,
                      **({"bwd": statistics.mean(per["bwd"])} if wl.backward else {})},
        "fwd_kernel": {"ms": fwd_ms, "effective_tflops": fwd_tflops,
                       **({"frac_of_burst": fwd_tflops / bf16_burst} if tc else {})},
        "router": {"ms": router_ms, "algorithmic_bytes": router_bytes,
                   "gbs": router_bytes / (router_ms * 1e-3) / 1e9,
                   "hbm_frac": router_bytes / (router_ms * 1e-3) / 1e9 / hbm,
                   "roofline": {"bound": "mufu", "achieved": router_ex2 / (router_ms * 1e-3),
                                "peak": mufu_peak(sm_max), "unit": "ex2/s",
                                "frac": router_ex2 / (router_ms * 1e-3) / mufu_peak(sm_max),
                                "exponentials": router_ex2}},
        **({"bwd_pass": {"ms": bwd_ms, "effective_tflops": bwd_tflops, "frac_of_burst": bwd_tflops / bf16_burst}}
           if wl.backward else {}),
        "roofline": {"bound": roof["bound"], "kernel": roof["kernel"], "achieved": roof["achieved"],
                     "peak": peak, "unit": "TFLOP/s", "frac": roof["achieved"] / peak, "peak_kind": kind,
                     **extra_peak, "traffic": roof["traffic"]},
        "cpu_baseline": cpu,
        "e2e": {"value": flops_rank * world / (e2e * 1e-3) / 1e12, "unit": "TFLOPS", "ms_per_step": e2e,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "api": "VSA2.forward + attn_bwd after H2D copies" if wl.backward else "vsa2_forward_host"},
        "gpu_launches": launches * args.steps,
        "clocks": clk.summary(),
        **({"next_rows": next_rows} if next_rows else {}),
    }
    return line


def measure_sharded(args, wl, dev, rank, world):
    """Strong scaling of one workload over the ranks (§8(e) of the design: the path shards by
    (b, h)). --shard heads: rank r runs the router, TopK and forward of its heads (sharding
    .shard_units) and nothing crosses ranks. --shard ulysses: rank r holds a contiguous 1/P of
    the cube-major tokens of every head (a sequence-sharded model); one all-to-all per tensor
    gathers whole sequences of H/P heads (App. E), the same path runs on them, and one
    all-to-all returns the output shard; the two exchanges are timed beside the path. One step
    = the whole workload over all ranks; the time is the max over ranks."""
    import torch
    import torch.distributed as dist
    import trainable_block_sparse_fine_b200 as V
    from trainable_block_sparse_fine_b200.sharding import max_over_ranks, shard_units
    from trainable_block_sparse_fine_b200.ulysses import heads_to_seq, seq_to_heads

    if wl.batch != 1 or wl.backward:
        raise SystemExit("--shard takes the forward workloads with batch 1")
    dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    workers = max(1, min(16, len(os.sched_getaffinity(0)) // max(1, int(os.environ.get("LOCAL_WORLD_SIZE", world)))))
    if args.shard == "heads":
        heads = [h for _, h in shard_units(wl.batch, wl.heads, rank, world)]
        x = {n: torch.from_numpy(S.make_tensor(wl, n, heads=heads, workers=workers)).to(dt).to(dev)
             for n in ("q", "k", "v")}
        hr = len(heads)
    else:
        if wl.heads % world or wl.tokens % world:
            raise SystemExit("--shard ulysses needs heads and tokens divisible by the rank count")
        if not dist.is_initialized():
            import socket
            with socket.socket() as sk:
                sk.bind(("127.0.0.1", 0))
                port = sk.getsockname()[1]
            dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                                    device_id=dev)
        ls = wl.tokens // world
        x = {}
        for n in ("q", "k", "v"):
            full = S.make_tensor(wl, n, workers=workers)
            x[n] = torch.from_numpy(full[:, :, rank * ls:(rank + 1) * ls]).to(dt).to(dev).contiguous()
            del full
        hr = wl.heads // world
    e = V.VSA2(wl.batch, hr, wl.head_dim, wl.grid, wl.dtype, wl.topk)
    stream = torch.cuda.current_stream()
    l2_flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)

    def step(t=None):
        if args.shard == "ulysses":
            if t: t[0].record(stream)
            xs = {n: seq_to_heads(x[n]) for n in ("q", "k", "v")}
            if t: t[1].record(stream)
        else:
            xs = x
        o, _, _ = e.forward(xs["q"], xs["k"], xs["v"])
        if args.shard == "ulysses":
            if t: t[2].record(stream)
            o = heads_to_seq(o)
            if t: t[3].record(stream)
        return o

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    parts = {"a2a_in": [], "path": [], "a2a_out": [], "step": []}
    if world > 1:
        dist.barrier()
    with Clocks(dev.index) as clk:
        for _ in range(args.steps):
            l2_flush.zero_()
            t = [ev() for _ in range(4)]
            if args.shard == "heads":
                t[0].record(stream)
                step()
                t[3].record(stream)
            else:
                step(t)
            torch.cuda.synchronize()
            parts["step"].append(t[0].elapsed_time(t[3]))
            if args.shard == "ulysses":
                parts["a2a_in"].append(t[0].elapsed_time(t[1]))
                parts["path"].append(t[1].elapsed_time(t[2]))
                parts["a2a_out"].append(t[2].elapsed_time(t[3]))
    if world > 1:
        dist.barrier()
    if e.device_error() != 0:
        raise RuntimeError("device error in the sharded run")
    ms = max_over_ranks(statistics.mean(parts["step"]), dev)
    pairs = wl.batch * wl.heads * wl.num_tiles * wl.topk
    value = pair_flops(wl, pairs, False) / (ms * 1e-3) / 1e12
    if rank != 0:
        return None
    line = {"metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": world, "steps": args.steps,
            "warmup": max(3, args.warmup), "ms_per_step": ms, "higher_is_better": True, "scaling": "strong",
            "vs_baseline": None, "dtype": "bf16" if wl.dtype == "bf16" else "fp32", "data": "synthetic",
            "config": {"workload": wl.name, "shard": args.shard, "heads_per_rank": hr, "tokens": wl.tokens,
                       "topk": wl.topk, "l2": "256 MB buffer written between timed steps"},
            "clocks": clk.summary()}
    if args.shard == "ulysses":
        line["ulysses_ms"] = {k: statistics.mean(v) for k, v in parts.items() if k != "step"}
        line["ulysses_bytes_per_rank"] = {
            "a2a_in": 3 * wl.heads * (wl.tokens // world) * wl.head_dim * (2 if wl.dtype == "bf16" else 4),
            "a2a_out": wl.heads * (wl.tokens // world) * wl.head_dim * (2 if wl.dtype == "bf16" else 4)}
    return line


def run_ours(args, wls):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    dev = torch.device("cuda", local)
    lines = []
    if args.shard != "batch":
        for wl in wls:
            if wl.backward:
                continue  # the sharded modes time the forward path
            line = measure_sharded(args, wl, dev, rank, world)
            if line is not None:
                print(json.dumps(line), flush=True)
        if dist.is_initialized():
            dist.barrier()
            dist.destroy_process_group()
        return
    for wl in wls:
        line = measure(args, wl, dev, rank, world)
        if line is not None:
            lines.append(line)
            if wl.name != HEADLINE:
                print(json.dumps(line), flush=True)
    if rank == 0 and lines:
        head = next((l for l in lines if l["config"]["workload"] == HEADLINE), lines[-1])
        if len(lines) > 1:  # one-line digest of every config, at the end of the headline line
            head["configs"] = {l["config"]["workload"]: {
                "ms_per_step": round(l["ms_per_step"], 4), "value": round(l["value"], 2),
                "roofline_frac": round(l["roofline"]["frac"], 4), "bound": l["roofline"]["bound"],
                "fwd_ms": round(l["fwd_kernel"]["ms"], 4), "router_ms": round(l["router"]["ms"], 4),
                "topk_ms": round(l["stages_ms"]["topk"], 4),
                **({"bwd_ms": round(l["bwd_pass"]["ms"], 4)} if "bwd_pass" in l else {})} for l in lines}
        print(json.dumps(head), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="all", choices=["all"] + list(S.WORKLOADS),
                    help="all (default): every configuration, one JSON line each, the headline last")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=20.0, help="seconds of oracle work for the CPU baseline")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end (host buffers) measurement")
    ap.add_argument("--heads", type=int, default=None, help="override the head count (profiling runs)")
    ap.add_argument("--no-next", action="store_true", help="skip timing the coarse branch and the gated merge")
    ap.add_argument("--shard", default="batch", choices=["batch", "heads", "ulysses"],
                    help="batch (default): weak scaling, every rank its own batch element; heads / ulysses: "
                         "strong scaling of one forward workload (a single --workload) split by heads, or "
                         "held sequence-sharded with Ulysses all-to-alls around the per-head path")
    args = ap.parse_args()
    names = ALL_WORKLOADS if args.workload == "all" else [args.workload]
    wls = [S.WORKLOADS[n] for n in names]
    if args.heads:
        wls = [wl.with_(heads=args.heads) for wl in wls]
    if args.impl == "reference":
        run_reference(args, S.WORKLOADS[HEADLINE] if args.workload == "all" else wls[0])
    else:
        run_ours(args, wls)


if __name__ == "__main__":
    main()
