"""Benchmark of the batch-1 Prox sparse-FFN decode step on B200.

python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                [--workload llama3_8b] [--s2 70] [--no-graph]

One step = the workload's 256 decode tokens, one at a time (batch 1), each a
full pass of the hot path: Stage-1 threshold + INT4 proxy GEMV, top-k select,
Stage-2 gate/up + W_down, output reduction.  The layer is a seeded synthetic
Llama-3-8B-shaped FFN (d_model 4096, d_ff 14336, bf16 weights N(0, 0.02^2),
Laplace inputs with 0.5% outlier channels x30), s1 = 50% (tau calibrated on
256 draws), s2 = 70% (k = 4301).  Consecutive tokens rotate over enough
identical copies of the layer that every token's weights were last touched
more than 2x L2 bytes earlier, so HBM, not L2, serves them.

Prints one JSON line (rank 0).  For N > 1 it runs one replica per GPU
(launched by torchrun); value = all ranks' tokens / the slowest rank's time.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import platform
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "batch-1 sparse-FFN tokens/s"
UNIT = "tokens/s"
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "stage2_traffic.json")


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="llama3_8b")
    ap.add_argument("--s2", type=int, default=70)
    ap.add_argument("--tokens", type=int, default=None, help="tokens per step (default: workload's)")
    ap.add_argument("--no-graph", action="store_true", help="launch eagerly instead of a CUDA graph")
    ap.add_argument("--no-extras", action="store_true", help="skip sweep/dense/e2e/cpu legs")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    return ap.parse_args()


# ---------------------------------------------------------------------------
# distributed plumbing (replicas only: no data-path collective)
# ---------------------------------------------------------------------------

class Dist:
    """One process per GPU (replicas): barrier and max-over-ranks of a time.
    backend "gloo" runs the same logic on CPU (tests)."""

    def __init__(self, want: int, backend: str = "nccl"):
        import torch
        self.rank = int(os.environ.get("RANK", "0"))
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        if want != self.world:
            raise SystemExit(f"--gpus {want} but WORLD_SIZE={self.world}; launch N>1 with torchrun")
        self.pg = None
        self.device = "cuda" if backend == "nccl" else "cpu"
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            kw = {}
            if backend == "nccl":
                torch.cuda.set_device(self.local)
                kw["device_id"] = torch.device("cuda", self.local)
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
            self.pg = dist

    def barrier(self):
        if self.pg:
            self.pg.barrier()

    def max(self, v: float) -> float:
        if not self.pg:
            return v
        import torch
        t = torch.tensor([v], dtype=torch.float64, device=self.device)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = str(gpu_index)
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(gpu_index).uuid)
            if uuid:
                self.idx = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            pass
        self.proc = None
        self.f = None

    def start(self):
        try:
            self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", self.idx], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.flush()
        self.f.seek(0)
        rows = [ln.strip().split(",") for ln in self.f.read().splitlines() if ln.strip()]
        self.f.close()
        os.unlink(self.f.name)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                smax.append(float(r[2]))
            except ValueError:
                continue
            for name, val in zip(names, r[5:9]):
                if val.strip().lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "samples": len(sm), "reasons": sorted(reasons)}


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------

def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            return json.load(fh), "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}, "fallback"


def stage2_source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "activation_sparse_swiglu_b200", "csrc")
    for name in ("stage2.cu", "select.cuh", "prox_device.cuh", "prox_internal.h"):
        with open(os.path.join(csrc, name), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(k: int, d: int):
    """DRAM bytes per Stage-2 launch from a committed ncu summary, scaled to k,
    or None when the kernel changed since the counters were taken."""
    if not os.path.exists(PROFILE_TRAFFIC):
        return None
    with open(PROFILE_TRAFFIC) as fh:
        rec = json.load(fh)
    if rec.get("source_hash") != stage2_source_hash():
        return None
    per_channel = rec["dram_bytes_per_launch"] / rec["k"]
    return per_channel * k


def bf16_dev(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def run_ours(args, dist):
    import torch
    import activation_sparse_swiglu_b200 as prox
    import synth

    dev = torch.cuda.current_device()
    props = torch.cuda.get_device_properties(dev)
    cfg = synth.get_config(args.workload)
    n_tok = args.tokens or cfg.n_tokens
    s1 = cfg.s1_percent[0]
    k = cfg.k(args.s2)
    d, f = cfg.d_model, cfg.d_ff
    lay = synth.make_layer(cfg, n_tokens=n_tok)
    x_cal = torch.from_numpy(lay.x_cal).cuda()
    tau = prox.calibrate_thresholds(x_cal, s1 / 100.0)

    # algorithmic bytes of one token (what the method must move)
    g = d // 128
    l2 = int(getattr(props, "L2_cache_size", 126 * 2 ** 20))
    approx_tok_bytes = 8 * d + (d // 2) * f + 4 * f * g + 6 * k * d
    n_copies = max(2, math.ceil(2 * l2 / approx_tok_bytes) + 1)
    wg, wu, wd = bf16_dev(lay.w_gate_bits), bf16_dev(lay.w_up_bits), bf16_dev(lay.w_down_bits)
    layers = [prox.Layer(wg, wu, wd, tau=tau, k=k, max_batch=1) for _ in range(n_copies)]
    del wg, wu, wd
    torch.cuda.empty_cache()
    info = layers[0].info()

    x = torch.from_numpy(lay.x_eval).cuda()
    out = torch.empty_like(x)
    stream = torch.cuda.Stream()

    def run_tokens(fn):
        for t in range(n_tok):
            fn(layers[t % n_copies], x[t], out[t])

    def prox_fn(L, xi, oi):
        L.forward(xi, oi)

    def dense_fn(L, xi, oi):
        L.dense(xi, oi)

    def make_step(fn):
        if args.no_graph:
            def step():
                with torch.cuda.stream(stream):
                    run_tokens(fn)
            return step, None
        with torch.cuda.stream(stream):
            run_tokens(fn)  # warm the launch path outside capture
        stream.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            run_tokens(fn)

        def step():
            with torch.cuda.stream(stream):
                graph.replay()
        return step, graph

    def timed(step, steps, warmup, sample_clocks=False):
        for _ in range(warmup):
            step()
        stream.synchronize()
        dist.barrier()
        torch.cuda.synchronize()
        sampler = ClockSampler(dev) if sample_clocks else None
        if sampler:
            sampler.start()
            time.sleep(0.3)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            step()
        e1.record(stream)
        e1.synchronize()
        torch.cuda.synchronize()
        clocks = sampler.stop() if sampler else None
        dist.barrier()
        ms = e0.elapsed_time(e1)
        return dist.max(ms), clocks

    # ---- headline: prox forward -------------------------------------------
    for L in layers:
        L.stats()
    step, graph = make_step(prox_fn)
    ms, clocks = timed(step, args.steps, args.warmup, sample_clocks=True)
    ms_per_step = ms / args.steps
    tok_s = dist.world * n_tok * args.steps / (ms / 1e3)
    sum_nx, ntoks = 0, 0
    for L in layers:
        s_, t_ = L.stats()
        sum_nx += s_
        ntoks += t_
    mean_nx = sum_nx / max(ntoks, 1)
    del graph
    err_words = [L.error_word() for L in layers]

    # algorithmic bytes per token at the measured n_x (all groups touched)
    tok_bytes = 4 * d + mean_nx * f + 4 * f * g + 6 * k * d + 4 * d
    result = {
        "metric": METRIC,
        "value": round(tok_s, 1),
        "unit": UNIT,
        "n_gpus": dist.world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic (seeded Laplace tokens, N(0,sigma^2) bf16 weights; no dataset)",
        "config": {
            "workload": cfg.workload_name(s1, args.s2),
            "d_model": d, "d_ff": f, "k": k, "s1_percent": s1, "s2_percent": args.s2,
            "tau_x": tau, "tokens_per_step": n_tok, "batch": 1,
            "weights": "bf16 gate/up/down + int4 group-128 proxies",
            "l2": (f"inputs larger than L2: {n_copies} rotating layer copies "
                   f"({n_copies * (info['weight_bytes'] + info['proxy_bytes']) / 1e9:.2f} GB), "
                   f"each token streams {tok_bytes / 1e6:.1f} MB"),
            "launch": "eager" if args.no_graph else "cuda graph per step, PDL-chained kernels",
            "parallelism": f"replicas x{dist.world}" if dist.world > 1 else "single GPU",
        },
        "gpu_launches": 3 * n_tok * args.steps,  # stage1, stage2 (with the cut), reduce
        "clocks": clocks,
        "realised_s1": round(1 - mean_nx / d, 4),
        "hbm_gbs_forward": round(tok_bytes * tok_s / dist.world / 1e9, 1),
        "bytes_per_token": int(tok_bytes),
        "device_error_words": err_words,
    }
    peaks, peak_kind = measured_peaks()
    result["forward_roofline"] = {
        "bound": "hbm", "achieved": result["hbm_gbs_forward"], "peak": peaks["hbm_gbs"],
        "unit": "GB/s", "frac": round(result["hbm_gbs_forward"] / peaks["hbm_gbs"], 4),
        "peak_source": peak_kind,
        "note": "whole prox_ffn_forward: algorithmic bytes per token x tokens/s"}

    # ---- per-kernel durations (serialised, events between kernels) ----------
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    for e in evs:
        e.record(stream)  # torch creates the CUDA event lazily, on first record
    stream.synchronize()
    t_s1, t_s2, t_red = [], [], []
    with torch.cuda.stream(stream):
        for rep in range(2):
            for t in range(min(n_tok, 96)):
                layers[t % n_copies].forward_profiled(x[t], out[t], evs)
                evs[3].synchronize()
                if rep:
                    t_s1.append(evs[0].elapsed_time(evs[1]))
                    t_s2.append(evs[1].elapsed_time(evs[2]))
                    t_red.append(evs[2].elapsed_time(evs[3]))
    s2_ms = statistics.mean(t_s2)
    s2_bytes = 6 * k * d + 4 * d
    achieved = s2_bytes / (s2_ms / 1e3) / 1e9
    traffic = profiled_traffic(k, d)
    result["roofline"] = {
        "kernel": "stage2_kernel (exact top-k cut, then gate/up + W_down over the k selected channels)",
        "bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
        "frac": round(achieved / peaks["hbm_gbs"], 4),
        "traffic": None if traffic is None else int(traffic),
        "algorithmic_bytes_per_launch": s2_bytes,
        "avg_launch_us": round(s2_ms * 1e3, 2),
        "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured"
        else "fallback 6.65 TB/s",
    }
    result["kernel_us"] = {"stage1": round(statistics.mean(t_s1) * 1e3, 2),
                           "stage2": round(s2_ms * 1e3, 2),
                           "reduce": round(statistics.mean(t_red) * 1e3, 2)}

    if not args.no_extras:
        # ---- dense bf16 baseline on the same buffers -------------------------
        dsteps = max(2, args.steps // 4)
        dstep, dgraph = make_step(dense_fn)
        dms, _ = timed(dstep, dsteps, 2)
        del dgraph
        dense_tok_s = dist.world * n_tok * dsteps / (dms / 1e3)
        result["dense_tokens_per_s"] = round(dense_tok_s, 1)
        result["speedup_vs_dense"] = round(tok_s / dense_tok_s, 3)
        result["dense_hbm_gbs"] = round((6 * d * f + 8 * d) * dense_tok_s / dist.world / 1e9, 1)

        # ---- FFN-sparsity sweep of the workload --------------------------------
        sweep = []
        for s2 in cfg.s2_percent:
            if s2 == args.s2:
                sweep.append({"s2_percent": s2, "k": k, "tokens_per_s": result["value"]})
                continue
            kk = cfg.k(s2)
            for L in layers:
                L.set_k(kk)
            sstep, sgraph = make_step(prox_fn)
            sms, _ = timed(sstep, dsteps, 2)
            del sgraph
            stok = dist.world * n_tok * dsteps / (sms / 1e3)
            sweep.append({"s2_percent": s2, "k": kk, "tokens_per_s": round(stok, 1),
                          "speedup_vs_dense": round(stok / dense_tok_s, 3)})
        for L in layers:
            L.set_k(k)
        result["sweep"] = sorted(sweep, key=lambda r: r["s2_percent"])

        # ---- the paper's Stage-2 threshold rule (Prox §4.1, App. A.7) --------------
        # tau_s = the s2-quantile of the calibration tokens' proxy scores; the
        # channel count then varies per token.
        ncal = min(64, lay.x_cal.shape[0])
        cal_scores = torch.cat([layers[0].proxy_scores(x_cal[i:i + 1]) for i in range(ncal)])
        tau_s = prox.calibrate_thresholds(cal_scores, args.s2 / 100.0)
        del cal_scores
        for L in layers:
            L.set_mask(prox.MASK_THRESHOLD, tau_s)
            L.stats()
        tstep, tgraph = make_step(prox_fn)
        tms, _ = timed(tstep, dsteps, 2)
        del tgraph
        sel = [L.stats(with_selected=True) for L in layers]
        ntk = max(1, sum(r[1] for r in sel))
        k_hat = sum(r[2] for r in sel) / ntk
        for L in layers:
            L.set_mask(prox.MASK_TOPK)
        ttok = dist.world * n_tok * dsteps / (tms / 1e3)
        r_s1, r_s2, r_e = prox.runtime_sparsity(sum(r[0] for r in sel), sum(r[2] for r in sel),
                                                ntk, d, f)
        result["threshold_rule"] = {
            "tau_s": tau_s, "calibration_tokens": ncal, "mean_channels": round(k_hat, 1),
            "realised_s1": round(r_s1, 4), "realised_s2": round(r_s2, 4),
            "realised_e": round(r_e, 4), "tokens_per_s": round(ttok, 1),
            "speedup_vs_dense": round(ttok / dense_tok_s, 3)}

        # ---- variants: GeGLU gate (Prox §5) and ablation A3 (Prox §5.2) ------------
        variants = {}
        for vname, setup in (("geglu_tanh", lambda L: L.set_activation(prox.ACT_GELU_TANH)),
                             ("geglu_erf", lambda L: L.set_activation(prox.ACT_GELU_ERF)),
                             ("a3_proxy_values", lambda L: L.set_stage2(prox.STAGE2_PROXY_VALUES))):
            for L in layers:
                setup(L)
            vstep, vgraph = make_step(prox_fn)
            vms, _ = timed(vstep, dsteps, 2)
            del vgraph
            for L in layers:
                L.set_activation(prox.ACT_SILU)
                L.set_stage2(prox.STAGE2_EXACT)
            variants[vname] = round(dist.world * n_tok * dsteps / (vms / 1e3), 1)
        result["variants_tokens_per_s"] = variants

        # ---- the paper's operating points (Prox §4.2 allocation, App. A.4) -------
        # (s1, s2) from the target e with alpha = 1/3, s_ref = 0.7, s1 in [0, 0.7];
        # tau_x calibrated for s1, top-k with k = round((1 - s2) d_ff).
        ops = []
        for e_t in (0.4, 0.5, 0.6, 0.7):
            o_s1, o_s2 = prox.allocate_sparsity(e_t)
            o_tau = prox.calibrate_thresholds(x_cal, o_s1)
            o_k = max(1, int(round((1.0 - o_s2) * f)))
            for L in layers:
                L.set_tau(o_tau)
                L.set_k(o_k)
                L.stats()
            ostep, ograph = make_step(prox_fn)
            oms, _ = timed(ostep, dsteps, 2)
            del ograph
            rs = [L.stats(with_selected=True) for L in layers]
            _, _, o_e = prox.runtime_sparsity(sum(r[0] for r in rs), sum(r[2] for r in rs),
                                              max(1, sum(r[1] for r in rs)), d, f)
            otok = dist.world * n_tok * dsteps / (oms / 1e3)
            ops.append({"e_target": e_t, "s1": round(o_s1, 4), "s2": round(o_s2, 4), "k": o_k,
                        "realised_e": round(o_e, 4), "tokens_per_s": round(otok, 1),
                        "speedup_vs_dense": round(otok / dense_tok_s, 3)})
        for L in layers:
            L.set_tau(tau)
            L.set_k(k)
        result["operating_points"] = ops

        # ---- alpha on B200 (Prox App. A.3): Stage 1 vs a bf16 GEMV over the same
        # kept input rows.  Stage 1 runs both proxy projections, so
        # alpha = t_stage1 / (2 t_gemv).  The GEMV is cuBLAS (torch.matmul) on the
        # kept rows stored input-major [n_x, F] (x @ W) and output-major [F, n_x]
        # (W^T x); the faster one is the denominator.  alpha_roofline takes a GEMV
        # that streams its 2 n_x F bytes at the measured HBM peak instead.
        n_x = max(1, int(round(mean_nx)))
        slice_bytes = 2 * n_x * f
        n_win = max(2, math.ceil(2 * l2 / slice_bytes) + 1)
        w_src = bf16_dev(lay.w_gate_bits)

        def time_gemv(wins, fn):
            with torch.cuda.stream(stream):
                for i in range(3 * n_win):
                    fn(wins[i % n_win])
                g0 = torch.cuda.Event(enable_timing=True)
                g1 = torch.cuda.Event(enable_timing=True)
                reps = 20 * n_win
                g0.record(stream)
                for i in range(reps):
                    fn(wins[i % n_win])
                g1.record(stream)
            g1.synchronize()
            return g0.elapsed_time(g1) * 1e3 / reps

        xs = torch.randn(1, n_x, device="cuda").to(torch.bfloat16)
        xcol = xs.reshape(n_x, 1).contiguous()
        ys = torch.empty(1, f, device="cuda", dtype=torch.bfloat16)
        ycol = torch.empty(f, 1, device="cuda", dtype=torch.bfloat16)
        wins = [w_src[:n_x].clone() for _ in range(n_win)]
        gemv_in_us = time_gemv(wins, lambda w: torch.matmul(xs, w, out=ys))
        del wins
        wins = [w_src[:n_x].t().contiguous() for _ in range(n_win)]
        gemv_out_us = time_gemv(wins, lambda w: torch.matmul(w, xcol, out=ycol))
        del wins, w_src, xs, xcol, ys, ycol
        gemv_us = min(gemv_in_us, gemv_out_us)
        gemv_roof_us = slice_bytes / (peaks["hbm_gbs"] * 1e9) * 1e6
        t1_us = result["kernel_us"]["stage1"]
        proxy_bytes = n_x * f // 2 + 2 * f * g  # one projection: codes of the kept rows + scales
        result["alpha"] = {
            "n_x": n_x, "stage1_us": t1_us,
            "bf16_gemv_us": {"input_major": round(gemv_in_us, 2),
                             "output_major": round(gemv_out_us, 2),
                             "at_hbm_peak": round(gemv_roof_us, 2)},
            "alpha_time": round(t1_us / (2 * gemv_us), 4),
            "alpha_roofline": round(t1_us / (2 * gemv_roof_us), 4),
            "alpha_bytes": round(proxy_bytes / slice_bytes, 4),
            "bf16_gemv_gbs": round(slice_bytes / (gemv_us * 1e-6) / 1e9, 1),
            "note": ("Stage 1 (both INT4 proxies + scores, event-timed alone) over 2 x the "
                     f"faster cuBLAS bf16 GEMV of the same {n_x} kept rows x {f} channels, "
                     f"{n_win} rotating weight windows (> L2)")}

        # ---- end to end through the host-buffer entry point ----------------------
        xh = [torch.from_numpy(np.ascontiguousarray(lay.x_eval[c::n_copies])).pin_memory()
              for c in range(n_copies)]
        oh = [torch.empty_like(t).pin_memory() for t in xh]

        def e2e_step():
            for c in range(n_copies):
                layers[c].forward_host(xh[c], oh[c], stream=stream)

        ems, _ = timed(e2e_step, dsteps, 1)
        e2e_tok_s = dist.world * n_tok * dsteps / (ems / 1e3)
        result["e2e"] = {"value": round(e2e_tok_s, 1), "unit": UNIT,
                         "h2d_bytes_per_step": n_tok * d * 4, "d2h_bytes_per_step": n_tok * d * 4,
                         "path": "prox_ffn_forward_host (pinned host buffers, copies in the timed "
                                 "region, one stream sync per layer copy)"}

        # ---- HBM copy bandwidth with our own copy kernel ---------------------------
        nbytes = 1 << 30
        a = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        b = torch.empty_like(a)
        with torch.cuda.stream(stream):
            for _ in range(3):
                prox.copy(a, b, stream=stream)
            c0 = torch.cuda.Event(enable_timing=True)
            c1 = torch.cuda.Event(enable_timing=True)
            c0.record(stream)
            for _ in range(10):
                prox.copy(a, b, stream=stream)
            c1.record(stream)
        c1.synchronize()
        result["copy_kernel_gbs"] = round(2 * nbytes * 10 / (c0.elapsed_time(c1) / 1e3) / 1e9, 1)
        del a, b

    # ---- CPU baseline: the oracle on the host cores (rank 0, N = 1) -------------
    if dist.rank == 0 and dist.world == 1 and not args.no_extras:
        result["cpu_baseline"] = cpu_baseline(lay, tau, k, args.cpu_seconds)
    for L in layers:
        L.close()
    return result


def _oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        return max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:
        return os.cpu_count() or 1


def _cpu_model():
    try:
        with open("/proc/cpuinfo") as fh:
            for line in fh:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return platform.processor() or "unknown"


def cpu_baseline(lay, tau, k, seconds):
    """The fp64 oracle on the host: all cores for `seconds`, then a shorter
    single-thread sample of the same workload."""
    from oracle import prox_oracle as orc
    qg, sg = orc.quantize_proxy(lay.w_gate)
    qu, su = orc.quantize_proxy(lay.w_up)

    def timed(limit_s):
        n, t0 = 0, time.perf_counter()
        while True:
            x = lay.x_eval[n % lay.x_eval.shape[0]]
            orc.prox_ffn(x, lay.w_gate, lay.w_up, lay.w_down, qg, sg, qu, su, tau=tau, k=k)
            n += 1
            el = time.perf_counter() - t0
            if (el >= limit_s and n >= 2) or n >= lay.x_eval.shape[0]:
                return n, el

    n, el = timed(seconds)
    out = {"value": round(n / el, 3), "unit": UNIT, "cores": _oracle_threads(), "kind": "oracle",
           "cpu": _cpu_model(), "nproc": os.cpu_count(),
           "sample": f"{n} tokens of the same workload through the fp64 numpy oracle "
                     f"({el:.1f} s; proxy packing done once beforehand, not timed)"}
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            n1, el1 = timed(seconds / 3)
        out["single_thread"] = {"value": round(n1 / el1, 3), "unit": UNIT, "cores": 1,
                                "sample": f"{n1} tokens ({el1:.1f} s), BLAS limited to one thread"}
    except ImportError:
        pass
    return out


# ---------------------------------------------------------------------------
# reference arm: the fp64 oracle on the host cores
# ---------------------------------------------------------------------------

def run_reference(args, dist):
    import synth
    from oracle import prox_oracle as orc
    cfg = synth.get_config(args.workload)
    s1 = cfg.s1_percent[0]
    k = cfg.k(args.s2)
    lay = synth.make_layer(cfg, n_tokens=cfg.n_tokens)
    tau = orc.calibrate_tau(lay.x_cal, s1 / 100.0)
    qg, sg = orc.quantize_proxy(lay.w_gate)
    qu, su = orc.quantize_proxy(lay.w_up)
    per_step = 1

    def step(i):
        for j in range(per_step):
            x = lay.x_eval[(i * per_step + j) % lay.x_eval.shape[0]]
            orc.prox_ffn(x, lay.w_gate, lay.w_up, lay.w_down, qg, sg, qu, su, tau=tau, k=k)

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(args.warmup + i)
    el = time.perf_counter() - t0
    tok_s = args.steps * per_step / el
    cores = _oracle_threads()
    return {
        "impl": "reference",
        "metric": METRIC, "value": round(tok_s, 3), "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(el / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded Laplace tokens, N(0,sigma^2) bf16 weights; no dataset)",
        "config": {"workload": cfg.workload_name(s1, args.s2), "d_model": cfg.d_model,
                   "d_ff": cfg.d_ff, "k": k, "tokens_per_step": per_step, "batch": 1},
        "cpu_baseline": {"value": round(tok_s, 3), "unit": UNIT, "cores": cores, "kind": "oracle",
                         "cpu": _cpu_model(), "nproc": os.cpu_count(),
                         "sample": f"{per_step} token per step of the same workload through the "
                                   f"fp64 numpy oracle"},
        "e2e": {"value": round(tok_s, 3), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    args = parse_args()
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        if rank != 0:
            return
        print(json.dumps(run_reference(args, None)), flush=True)
        return
    import torch
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    dist = Dist(args.gpus)
    if dist.world == 1:
        torch.cuda.set_device(0)
    try:
        res = run_ours(args, dist)
        if dist.rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        dist.close()


if __name__ == "__main__":
    main()
