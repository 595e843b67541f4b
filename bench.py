"""Benchmark of the batch-1 Prox sparse-FFN decode step on B200.

python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                [--workload llama3_8b] [--s2 70] [--tokens T] [--no-graph]
                [--no-extras] [--legs a,b,...] [--record-traffic NCU_CSV]

One step = the workload's 256 decode tokens, one at a time (batch 1), each a
full pass of the hot path in one kernel launch: Stage-1 threshold + INT4 proxy
GEMV + scores, exact top-k cut, Stage-2 gate/up + W_down over the selected
channels, output sum (the CTAs exchange tagged words, no grid barrier).  The layer is a seeded synthetic
Llama-3-8B-shaped FFN (d_model 4096, d_ff 14336, bf16 weights N(0, 0.02^2),
Laplace inputs with 0.5% outlier channels x30), s1 = 50% (tau calibrated on 256
draws), s2 = 70% (k = 4301).  Consecutive tokens rotate over enough identical
copies of the layer that every token's weights were last touched more than
2x L2 bytes earlier, so HBM, not L2, serves them.

Besides the headline line it measures (unless --no-extras): the dense bf16
baseline, the s2 sweep, the score-threshold rule, GeGLU and A3 variants, the
cost-model operating points, alpha, an end-to-end number through the public
API with host buffers, the copy-kernel bandwidth, the tiny layer's latency, the
Qwen3-14B-shaped layer at three input sparsities, the 32-layer stack end to
end, the Llama-3-70B-shaped layer at batch 1..16 against dense, and the fp64
oracle on the host cores.

Prints one JSON line (rank 0).  For N > 1 it runs one replica per GPU
(launched by torchrun); value = all ranks' tokens / the slowest rank's time.

--record-traffic CSV reads an ncu CSV with dram__bytes_read.sum and
dram__bytes_write.sum of token_kernel launches of this workload and writes
profiles/token_traffic.json, stamped with the hash of the kernel sources; the
bench reports that traffic only while the sources hash the same.
"""

from __future__ import annotations

import argparse
import csv
import hashlib
import json
import math
import os
import platform
import re
import statistics
import subprocess
import sys
import tempfile
import time
import traceback

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "batch-1 sparse-FFN tokens/s"
UNIT = "tokens/s"
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "token_traffic.json")
PER_TOKEN_STAGE1 = 4  # include/prox.h PROX_BATCH_PER_TOKEN_STAGE1
CSRC = os.path.join(ROOT, "activation_sparse_swiglu_b200", "csrc")
SPEC_HBM_GBS = 8000.0  # B200 HBM3e spec bandwidth (DGX figure), for the spec fraction
ALL_LEGS = ("dense", "sweep", "threshold", "variants", "operating_points", "alpha", "e2e",
            "copy", "tiny", "qwen3_14b", "stack32", "llama3_70b", "cpu")


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="llama3_8b")
    ap.add_argument("--s2", type=int, default=70)
    ap.add_argument("--tokens", type=int, default=None, help="tokens per step (default: workload's)")
    ap.add_argument("--no-graph", action="store_true", help="launch eagerly instead of a CUDA graph")
    ap.add_argument("--no-extras", action="store_true", help="headline only")
    ap.add_argument("--legs", default=",".join(ALL_LEGS), help="extra legs to run")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--record-traffic", default=None, metavar="NCU_CSV")
    return ap.parse_args(argv)


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


TOKEN_KERNEL_SOURCES = ("token.cu", "token_args.cuh", "stage1.cuh", "stage2.cuh", "select.cuh",
                        "prox_device.cuh")


_COMMENT = re.compile(r"//[^\n]*|/\*.*?\*/", re.S)


def _code_only(text: str) -> str:
    """A C++/CUDA source without its comments and blank lines (the kernel
    sources hold no comment markers inside string literals)."""
    return "\n".join(line.rstrip() for line in _COMMENT.sub("", text).splitlines() if line.strip())


def kernel_source_hash() -> str:
    """Hash of the per-token kernel's code (its source files, comments
    stripped); a traffic record counts only while the code hashes the same as
    when it was taken, so any change to the code voids it and a comment edit
    does not."""
    h = hashlib.sha256()
    for name in TOKEN_KERNEL_SOURCES:
        with open(os.path.join(CSRC, name), encoding="utf-8") as fh:
            h.update(name.encode())
            h.update(_code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str):
    """DRAM bytes per token_kernel launch from the committed ncu record, or
    None when the kernels changed since the counters were taken or the record
    is of another workload."""
    if not os.path.exists(PROFILE_TRAFFIC):
        return None
    with open(PROFILE_TRAFFIC) as fh:
        rec = json.load(fh)
    if rec.get("source_hash") != kernel_source_hash() or rec.get("workload") != workload:
        return None
    return rec


def record_traffic(csv_path: str, workload: str, alg_bytes: float, command: str):
    """Writes profiles/token_traffic.json from an ncu --csv metrics log."""
    per = {}
    with open(csv_path) as fh:
        lines = [ln for ln in fh if ln.startswith('"')]
    for row in csv.DictReader(lines):
        if "token_kernel" not in row.get("Kernel Name", ""):
            continue
        name = row.get("Metric Name")
        if name not in ("dram__bytes_read.sum", "dram__bytes_write.sum"):
            continue
        unit = row.get("Metric Unit", "byte").lower()
        scale = {"byte": 1, "kbyte": 1e3, "mbyte": 1e6, "gbyte": 1e9}.get(unit, 1)
        val = float(row["Metric Value"].replace(",", "")) * scale
        per.setdefault(row["ID"], {})[name] = val
    launches = [v for _, v in sorted(per.items(), key=lambda kv: int(kv[0]))
                if len(v) == 2]
    if not launches:
        raise SystemExit(f"no token_kernel dram metrics in {csv_path}")
    tot = [v["dram__bytes_read.sum"] + v["dram__bytes_write.sum"] for v in launches]
    rec = {"kernel": "token_kernel", "workload": workload, "launches": len(launches),
           "dram_bytes_per_launch": int(statistics.median(tot)),
           "dram_read_bytes_median": int(statistics.median(v["dram__bytes_read.sum"] for v in launches)),
           "dram_write_bytes_median": int(statistics.median(v["dram__bytes_write.sum"] for v in launches)),
           "algorithmic_bytes_per_launch": int(alg_bytes),
           "source_hash": kernel_source_hash(), "command": command}
    with open(PROFILE_TRAFFIC, "w") as fh:
        json.dump(rec, fh, indent=1)
        fh.write("\n")
    return rec


def bf16_dev(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def token_bytes(d, f, k, n_x):
    """Algorithmic bytes of one token: x, the kept rows of both INT4 proxies,
    two fp16 scale rows per group, the k channel records and W_down rows, out."""
    g = d // 128
    return 4 * d + n_x * f + 4 * f * g + 6 * k * d + 4 * d


class Timer:
    """CUDA-graph step builder and device timing on one side stream."""

    def __init__(self, dist, stream, graph=True):
        self.dist = dist
        self.stream = stream
        self.graph = graph

    def make_step(self, body):
        import torch
        s = self.stream
        if not self.graph:
            def step():
                with torch.cuda.stream(s):
                    body()
            return step, None
        with torch.cuda.stream(s):
            body()  # warm the launch path outside capture
        s.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            body()

        def step():
            with torch.cuda.stream(s):
                g.replay()
        return step, g

    def time(self, step, steps, warmup, clocks_dev=None):
        import torch
        s = self.stream
        for _ in range(warmup):
            step()
        s.synchronize()
        self.dist.barrier()
        torch.cuda.synchronize()
        sampler = ClockSampler(clocks_dev) if clocks_dev is not None else None
        if sampler:
            sampler.start()
            time.sleep(0.3)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(s)
        for _ in range(steps):
            step()
        e1.record(s)
        e1.synchronize()
        torch.cuda.synchronize()
        clocks = sampler.stop() if sampler else None
        self.dist.barrier()
        return self.dist.max(e0.elapsed_time(e1)), clocks

    def tokens_per_s(self, body, n_tok, steps, warmup=2):
        step, g = self.make_step(body)
        ms, _ = self.time(step, steps, warmup)
        del g
        return self.dist.world * n_tok * steps / (ms / 1e3), ms / steps


def phase_breakdown(layers, xs, outs, n, stream):
    """Median over tokens of the per-phase times (us) of the token kernel,
    launched alone (no programmatic overlap): each phase ends when its last
    CTA reaches the stamp; times are from the first CTA's entry."""
    import torch
    import activation_sparse_swiglu_b200 as prox
    P = layers[0].info()["stage1_ctas"]
    ph = torch.zeros((P, 24), dtype=torch.int64, device="cuda")
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    for e in evs:
        e.record(stream)
    stream.synchronize()
    # slot -> name (include/prox.h, prox_ffn_forward_profiled); 13 is a count
    names = {8: "stage1_compact", 9: "stage1_loop", 2: "stage1_partials",
             16: "partials_phase", 3: "partials_in", 10: "scored", 17: "scores_phase",
             14: "histogram_complete", 15: "topk_cut", 18: "counts_phase", 4: "selected",
             11: "stage2_ring", 12: "stage2_gate_up", 5: "stage2", 19: "rows_phase",
             6: "rows_in", 7: "out"}
    per, kt = [], []
    with torch.cuda.stream(stream):
        for t in range(n + 4):
            ph.zero_()
            layers[t % len(layers)].forward_profiled(xs[t % xs.shape[0]], outs[t % xs.shape[0]],
                                                     evs, phase_ns=ph, stream=stream)
            evs[1].synchronize()
            if t >= 4:
                per.append(np.nanmax(prox.phase_times_us(ph), axis=0))
                kt.append(evs[0].elapsed_time(evs[1]) * 1e3)
    per = np.stack(per)
    out = {nm: round(float(np.nanmedian(per[:, i])), 2) for i, nm in names.items()}
    out["kernel_event_us"] = round(statistics.median(kt), 2)
    return out


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

class Bench:
    def __init__(self, args, dist):
        import torch
        import activation_sparse_swiglu_b200 as prox
        import synth
        self.torch, self.prox, self.synth = torch, prox, synth
        self.args, self.dist = args, dist
        self.dev = torch.cuda.current_device()
        self.props = torch.cuda.get_device_properties(self.dev)
        self.l2 = int(getattr(self.props, "L2_cache_size", 126 * 2 ** 20))
        self.stream = torch.cuda.Stream()
        self.timer = Timer(dist, self.stream, graph=not args.no_graph)
        self.peaks, self.peak_kind = measured_peaks()
        self.result = {}

    # -- headline ----------------------------------------------------------
    def headline(self):
        torch, prox, synth, args = self.torch, self.prox, self.synth, self.args
        cfg = synth.get_config(args.workload)
        self.cfg = cfg
        n_tok = args.tokens or cfg.n_tokens
        self.n_tok = n_tok
        s1 = cfg.s1_percent[0]
        k = cfg.k(args.s2)
        d, f = cfg.d_model, cfg.d_ff
        self.k, self.d, self.f, self.s1 = k, d, f, s1
        lay = synth.make_layer(cfg, n_tokens=n_tok)
        self.lay = lay
        self.x_cal = torch.from_numpy(lay.x_cal).cuda()
        tau = prox.calibrate_thresholds(self.x_cal, s1 / 100.0)
        self.tau = tau
        approx = token_bytes(d, f, k, d // 2)
        n_copies = max(2, math.ceil(2 * self.l2 / approx) + 1)
        self.n_copies = n_copies
        wg, wu, wd = bf16_dev(lay.w_gate_bits), bf16_dev(lay.w_up_bits), bf16_dev(lay.w_down_bits)
        self.layers = [prox.Layer(wg, wu, wd, tau=tau, k=k, max_batch=1) for _ in range(n_copies)]
        del wg, wu, wd
        torch.cuda.empty_cache()
        info = self.layers[0].info()
        self.x = torch.from_numpy(lay.x_eval).cuda()
        self.out = torch.empty_like(self.x)
        layers, x, out, s = self.layers, self.x, self.out, self.stream

        def body():
            for t in range(n_tok):
                layers[t % n_copies].forward(x[t], out[t], stream=s)
        self.body = body

        for L in layers:
            L.stats()
        step, graph = self.timer.make_step(body)
        ms, clocks = self.timer.time(step, args.steps, args.warmup, clocks_dev=self.dev)
        del graph
        ms_per_step = ms / args.steps
        tok_s = self.dist.world * n_tok * args.steps / (ms / 1e3)
        self.tok_s = tok_s
        sum_nx, ntoks = 0, 0
        for L in layers:
            s_, t_ = L.stats()
            sum_nx += s_
            ntoks += t_
        mean_nx = sum_nx / max(ntoks, 1)
        self.mean_nx = mean_nx
        err_words = [L.error_word() for L in layers]
        tb = token_bytes(d, f, k, mean_nx)
        self.tok_bytes = tb
        us_per_tok = ms_per_step * 1e3 / n_tok
        achieved = tb / (us_per_tok * 1e-6) / 1e9
        peak = self.peaks["hbm_gbs"]
        traffic = profiled_traffic(cfg.workload_name(s1, args.s2))
        r = self.result
        r.update({
            "metric": METRIC,
            "value": round(tok_s, 1),
            "unit": UNIT,
            "n_gpus": self.dist.world,
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
                       f"each token streams {tb / 1e6:.1f} MB"),
                "launch": "eager" if args.no_graph else
                          "cuda graph per step, one cooperative PDL-chained kernel per token",
                "parallelism": f"replicas x{self.dist.world}" if self.dist.world > 1 else "single GPU",
            },
            "gpu_launches": n_tok * args.steps,  # token_kernel: the whole step of one token
            "clocks": clocks,
            "realised_s1": round(1 - mean_nx / d, 4),
            "us_per_token": round(us_per_tok, 3),
            "bytes_per_token": int(tb),
            "device_error_words": err_words,
        })
        r["roofline"] = {
            "kernel": "token_kernel (Stage 1, exact top-k cut, Stage 2 gate/up + W_down, "
                      "output sum: the whole step of one token)",
            "bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4),
            "frac_of_spec_8tbs": round(achieved / SPEC_HBM_GBS, 4),
            "traffic": None if traffic is None else traffic["dram_bytes_per_launch"],
            "algorithmic_bytes_per_launch": int(tb),
            "avg_launch_us": round(us_per_tok, 3),
            "peak_source": (f"{self.peak_kind} (MEASURED_PEAKS.json hbm_gbs, burst copy)"
                            if self.peak_kind == "measured" else "fallback 6.65 TB/s"),
            "note": "average launch duration = the timed region / launches (every launch in "
                    "it is this kernel); traffic = ncu dram read+write of one launch of the "
                    "same workload, null once the kernel sources changed",
        }
        try:
            r["phases_us"] = phase_breakdown(layers, x, out, 32, s)
        except Exception as e:  # diagnostic only
            r["phases_us"] = {"error": repr(e)}

    # -- extras --------------------------------------------------------------
    def leg_dense(self):
        layers, x, out, s, n = self.layers, self.x, self.out, self.stream, self.n_tok
        nc = self.n_copies

        def body():
            for t in range(n):
                layers[t % nc].dense(x[t], out[t], stream=s)
        dsteps = max(2, self.args.steps // 4)
        tok, _ = self.timer.tokens_per_s(body, n, dsteps)
        self.dense_tok_s = tok
        d, f = self.d, self.f
        self.result["dense_tokens_per_s"] = round(tok, 1)
        self.result["speedup_vs_dense"] = round(self.tok_s / tok, 3)
        self.result["dense_hbm_gbs"] = round((6 * d * f + 8 * d) * tok / self.dist.world / 1e9, 1)

    def _dense(self):
        return getattr(self, "dense_tok_s", None)

    def _vs_dense(self, tok):
        dn = self._dense()
        return None if not dn else round(tok / dn, 3)

    def leg_sweep(self):
        cfg, layers = self.cfg, self.layers
        dsteps = max(2, self.args.steps // 4)
        sweep = []
        for s2 in cfg.s2_percent:
            if s2 == self.args.s2:
                sweep.append({"s2_percent": s2, "k": self.k, "tokens_per_s": self.result["value"],
                              "speedup_vs_dense": self._vs_dense(self.tok_s)})
                continue
            kk = cfg.k(s2)
            for L in layers:
                L.set_k(kk)
            tok, _ = self.timer.tokens_per_s(self.body, self.n_tok, dsteps)
            tb = token_bytes(self.d, self.f, kk, self.mean_nx)
            sweep.append({"s2_percent": s2, "k": kk, "tokens_per_s": round(tok, 1),
                          "speedup_vs_dense": self._vs_dense(tok),
                          "hbm_frac": round(tb * tok / 1e9 / self.peaks["hbm_gbs"], 4)})
        for L in layers:
            L.set_k(self.k)
        self.result["sweep"] = sorted(sweep, key=lambda r: r["s2_percent"])

    def leg_threshold(self):
        prox, layers = self.prox, self.layers
        dsteps = max(2, self.args.steps // 4)
        ncal = min(64, self.lay.x_cal.shape[0])
        cal_scores = layers[0].proxy_scores(self.x_cal[:ncal], stream=self.stream)
        tau_s = prox.calibrate_thresholds(cal_scores, self.args.s2 / 100.0, stream=self.stream)
        del cal_scores
        for L in layers:
            L.set_mask(prox.MASK_THRESHOLD, tau_s)
            L.stats()
        tok, _ = self.timer.tokens_per_s(self.body, self.n_tok, dsteps)
        sel = [L.stats(with_selected=True) for L in layers]
        for L in layers:
            L.set_mask(prox.MASK_TOPK)
        ntk = max(1, sum(r[1] for r in sel))
        r_s1, r_s2, r_e = prox.runtime_sparsity(sum(r[0] for r in sel), sum(r[2] for r in sel),
                                                ntk, self.d, self.f)
        self.result["threshold_rule"] = {
            "tau_s": tau_s, "calibration_tokens": ncal,
            "mean_channels": round(sum(r[2] for r in sel) / ntk, 1),
            "realised_s1": round(r_s1, 4), "realised_s2": round(r_s2, 4),
            "realised_e": round(r_e, 4), "tokens_per_s": round(tok, 1),
            "speedup_vs_dense": self._vs_dense(tok)}

    def leg_variants(self):
        prox, layers = self.prox, self.layers
        dsteps = max(2, self.args.steps // 4)
        variants = {}
        for vname, setup in (("geglu_tanh", lambda L: L.set_activation(prox.ACT_GELU_TANH)),
                             ("geglu_erf", lambda L: L.set_activation(prox.ACT_GELU_ERF)),
                             ("a3_proxy_values", lambda L: L.set_stage2(prox.STAGE2_PROXY_VALUES))):
            for L in layers:
                setup(L)
            tok, _ = self.timer.tokens_per_s(self.body, self.n_tok, dsteps)
            for L in layers:
                L.set_activation(prox.ACT_SILU)
                L.set_stage2(prox.STAGE2_EXACT)
            variants[vname] = round(tok, 1)
        self.result["variants_tokens_per_s"] = variants

    def _operating_points(self, alpha):
        prox, layers = self.prox, self.layers
        dsteps = max(2, self.args.steps // 4)
        ops = []
        for e_t in (0.4, 0.5, 0.6, 0.7):
            try:
                o_s1, o_s2 = prox.allocate_sparsity(e_t, alpha=alpha)
            except prox.ProxError as exc:
                ops.append({"e_target": e_t, "alpha": alpha, "unreachable": str(exc)})
                continue
            o_tau = prox.calibrate_thresholds(self.x_cal, o_s1)
            o_k = max(1, int(round((1.0 - o_s2) * self.f)))
            for L in layers:
                L.set_tau(o_tau)
                L.set_k(o_k)
                L.stats()
            tok, _ = self.timer.tokens_per_s(self.body, self.n_tok, dsteps)
            rs = [L.stats(with_selected=True) for L in layers]
            _, _, o_e = prox.runtime_sparsity(sum(r[0] for r in rs), sum(r[2] for r in rs),
                                              max(1, sum(r[1] for r in rs)), self.d, self.f,
                                              alpha=alpha)
            ops.append({"e_target": e_t, "alpha": alpha, "s1": round(o_s1, 4), "s2": round(o_s2, 4),
                        "k": o_k, "realised_e": round(o_e, 4), "tokens_per_s": round(tok, 1),
                        "speedup_vs_dense": self._vs_dense(tok)})
        for L in layers:
            L.set_tau(self.tau)
            L.set_k(self.k)
        return ops

    def leg_operating_points(self):
        # (s1, s2) from the target e with the paper's alpha = 1/3, s_ref = 0.7,
        # s1 in [0, 0.7] (Prox §4.2, App. A.4); tau_x calibrated for s1, top-k
        # with k = round((1 - s2) d_ff).  The same targets at the alpha measured
        # on this GPU follow in leg_alpha.
        self.result["operating_points"] = self._operating_points(1.0 / 3.0)

    def leg_alpha(self):
        # alpha on B200 (Prox App. A.3): Stage 1 vs a bf16 GEMV over the same kept
        # input rows.  Stage 1 runs both proxy projections, so alpha = t_stage1 /
        # (2 t_gemv).  t_stage1 is the Stage-1 phase of the token kernel (first
        # CTA entry to the last CTA's Stage-1 stamp); the GEMV is cuBLAS
        # (torch.matmul) on the kept rows stored input-major and output-major, the
        # faster one the denominator; alpha_roofline takes a GEMV that streams its
        # 2 n_x F bytes at the measured HBM peak instead.
        torch = self.torch
        ph = self.result.get("phases_us", {})
        t1_us = ph.get("scored")
        if t1_us is None:
            return
        d, f, s = self.d, self.f, self.stream
        n_x = max(1, int(round(self.mean_nx)))
        slice_bytes = 2 * n_x * f
        n_win = max(2, math.ceil(2 * self.l2 / slice_bytes) + 1)
        w_src = bf16_dev(self.lay.w_gate_bits)

        def time_gemv(wins, fn):
            with torch.cuda.stream(s):
                for i in range(3 * n_win):
                    fn(wins[i % n_win])
                g0 = torch.cuda.Event(enable_timing=True)
                g1 = torch.cuda.Event(enable_timing=True)
                reps = 20 * n_win
                g0.record(s)
                for i in range(reps):
                    fn(wins[i % n_win])
                g1.record(s)
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
        gemv_roof_us = slice_bytes / (self.peaks["hbm_gbs"] * 1e9) * 1e6
        g = d // 128
        proxy_bytes = n_x * f // 2 + 2 * f * g
        alpha = t1_us / (2 * gemv_us)
        self.result["alpha"] = {
            "n_x": n_x, "stage1_us": t1_us,
            "bf16_gemv_us": {"input_major": round(gemv_in_us, 2),
                             "output_major": round(gemv_out_us, 2),
                             "at_hbm_peak": round(gemv_roof_us, 2)},
            "alpha_time": round(alpha, 4),
            "alpha_roofline": round(t1_us / (2 * gemv_roof_us), 4),
            "alpha_bytes": round(proxy_bytes / slice_bytes, 4),
            "bf16_gemv_gbs": round(slice_bytes / (gemv_us * 1e-6) / 1e9, 1),
            "note": ("Stage-1 part of the token kernel (entry to the last CTA's scores: both INT4 "
                     "proxies, the partial exchange and the scores; launched alone) over 2 x "
                     f"the faster cuBLAS bf16 GEMV of the same {n_x} kept rows x "
                     f"{f} channels, {n_win} rotating weight windows (> L2)")}
        # The paper's allocation at the alpha measured here (Prox §4.2).
        self.result["operating_points_measured_alpha"] = self._operating_points(
            max(1e-3, round(alpha, 4)))

    def leg_e2e(self):
        # End to end through the public API: every step copies its 256 inputs
        # from pinned host memory, runs them through Layer.forward rotating the
        # layer copies per token (as the headline, so L2 serves nothing), and
        # copies the outputs back; the CUDA events bracket the copies too.
        torch, layers, s, n, nc = self.torch, self.layers, self.stream, self.n_tok, self.n_copies
        d = self.d
        xh = torch.from_numpy(np.ascontiguousarray(self.lay.x_eval[:n])).pin_memory()
        oh = torch.empty_like(xh).pin_memory()
        xd = torch.empty((n, d), dtype=torch.float32, device="cuda")
        od = torch.empty_like(xd)

        def step():
            with torch.cuda.stream(s):
                xd.copy_(xh, non_blocking=True)
                for t in range(n):
                    layers[t % nc].forward(xd[t], od[t], stream=s)
                oh.copy_(od, non_blocking=True)
        dsteps = max(2, self.args.steps // 4)
        ms, _ = self.timer.time(step, dsteps, 2)
        tok = self.dist.world * n * dsteps / (ms / 1e3)
        self.result["e2e"] = {"value": round(tok, 1), "unit": UNIT,
                              "h2d_bytes_per_step": n * d * 4, "d2h_bytes_per_step": n * d * 4,
                              "path": "Layer.forward per token (ctypes -> prox_ffn_forward), "
                                      "layer copies rotated per token as in the headline, "
                                      "pinned host->device copy of the step's inputs and "
                                      "device->host copy of its outputs inside the timed region"}

    def leg_copy(self):
        torch, prox, s = self.torch, self.prox, self.stream
        nbytes = 1 << 30
        a = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        b = torch.empty_like(a)
        with torch.cuda.stream(s):
            for _ in range(3):
                prox.copy(a, b, stream=s)
            c0 = torch.cuda.Event(enable_timing=True)
            c1 = torch.cuda.Event(enable_timing=True)
            c0.record(s)
            for _ in range(10):
                prox.copy(a, b, stream=s)
            c1.record(s)
        c1.synchronize()
        gbs = 2 * nbytes * 10 / (c0.elapsed_time(c1) / 1e3) / 1e9
        self.result["copy_kernel_gbs"] = round(gbs, 1)
        self.result["copy_kernel_frac_of_spec_8tbs"] = round(gbs / SPEC_HBM_GBS, 4)
        del a, b

    # -- other workloads -------------------------------------------------------
    def _layer_leg(self, name, s1, s2=70, n_tok=64, batch=None, dense=True):
        torch, prox, synth = self.torch, self.prox, self.synth
        cfg = synth.get_config(name)
        d, f = cfg.d_model, cfg.d_ff
        k = cfg.k(s2)
        lay = synth.make_layer(cfg, n_tokens=n_tok, n_cal=256)
        x_cal = torch.from_numpy(lay.x_cal).cuda()
        tau = prox.calibrate_thresholds(x_cal, s1 / 100.0)
        approx = token_bytes(d, f, k, d // 2)
        nc = max(2, math.ceil(2 * self.l2 / approx) + 1)
        wg, wu, wd = bf16_dev(lay.w_gate_bits), bf16_dev(lay.w_up_bits), bf16_dev(lay.w_down_bits)
        layers = [prox.Layer(wg, wu, wd, tau=tau, k=k, max_batch=1) for _ in range(nc)]
        del wg, wu, wd
        x = torch.from_numpy(lay.x_eval).cuda()
        out = torch.empty_like(x)
        s = self.stream
        return cfg, lay, layers, x, out, s, k, tau, nc

    def leg_tiny(self):
        # The tiny layer (config 1): the whole layer lives in L2, so this is a
        # latency number, not an HBM-roofline one.
        torch = self.torch
        cfg, lay, layers, x, out, s, k, tau, nc = self._layer_leg("tiny", 50, n_tok=64)
        n = x.shape[0]

        def body():
            for t in range(n):
                layers[t % nc].forward(x[t], out[t], stream=s)

        def dbody():
            for t in range(n):
                layers[t % nc].dense(x[t], out[t], stream=s)
        steps = max(4, self.args.steps)
        tok, ms = self.timer.tokens_per_s(body, n, steps)
        dtok, _ = self.timer.tokens_per_s(dbody, n, steps)
        ph = phase_breakdown(layers, x, out, 16, s)
        self.result["tiny"] = {
            "workload": cfg.workload_name(50, 70), "tokens_per_s": round(tok, 1),
            "us_per_token": round(1e6 / tok, 2), "dense_tokens_per_s": round(dtok, 1),
            "speedup_vs_dense": round(tok / dtok, 3), "phases_us": ph,
            "note": "the whole layer fits in L2: latency-bound, no HBM roofline claimed"}
        for L in layers:
            L.close()
        torch.cuda.empty_cache()

    def leg_qwen3_14b(self):
        # Config 3: the Qwen3-14B-shaped layer at s1 40 / 50 / 60 %, s2 70 %.
        torch, prox = self.torch, self.prox
        cfg, lay, layers, x, out, s, k, tau, nc = self._layer_leg("qwen3_14b", 50, n_tok=128)
        d, f = cfg.d_model, cfg.d_ff
        x_cal = torch.from_numpy(lay.x_cal).cuda()
        n = x.shape[0]

        def body():
            for t in range(n):
                layers[t % nc].forward(x[t], out[t], stream=s)

        def dbody():
            for t in range(n):
                layers[t % nc].dense(x[t], out[t], stream=s)
        steps = max(2, self.args.steps // 4)
        dtok, _ = self.timer.tokens_per_s(dbody, n, steps)
        rows = []
        for s1 in cfg.s1_percent:
            t1 = prox.calibrate_thresholds(x_cal, s1 / 100.0)
            for L in layers:
                L.set_tau(t1)
                L.stats()
            tok, _ = self.timer.tokens_per_s(body, n, steps)
            st = [L.stats() for L in layers]
            mean_nx = sum(a for a, _ in st) / max(1, sum(b for _, b in st))
            tb = token_bytes(d, f, k, mean_nx)
            rows.append({"s1_percent": s1, "tau_x": t1, "realised_s1": round(1 - mean_nx / d, 4),
                         "tokens_per_s": round(tok, 1), "us_per_token": round(1e6 / tok, 2),
                         "bytes_per_token": int(tb),
                         "hbm_frac": round(tb * tok / 1e9 / self.peaks["hbm_gbs"], 4),
                         "speedup_vs_dense": round(tok / dtok, 3)})
        self.result["qwen3_14b"] = {"workload": f"qwen3_14b ffn layer d_model={d} d_ff={f} s2=70% k={k}",
                                    "dense_tokens_per_s": round(dtok, 1), "rows": rows,
                                    "layer_copies": nc}
        for L in layers:
            L.close()
        torch.cuda.empty_cache()

    def leg_stack32(self):
        # Config 4: 32 Llama-3-8B-shaped layers (independent seeded weights
        # N(0, 0.02^2), drawn on the GPU with torch's Philox generator, seed
        # 4000 + layer), RMSNorm between layers, tau_x per layer at s1 50 % by
        # the sequential calibration of Prox App. A.7 (Algorithm 1) on 256
        # calibration tokens, top-k at s2 70 %; 128 tokens, each through all 32
        # layers in order, timed end to end (one CUDA graph per step).
        torch, prox, synth = self.torch, self.prox, self.synth
        from activation_sparse_swiglu_b200.stack import Stack
        cfg = synth.get_config("stack32")
        d, f, nl = cfg.d_model, cfg.d_ff, cfg.n_layers
        k = cfg.k(70)
        lay0 = synth.make_layer("llama3_8b", n_tokens=cfg.n_tokens, n_cal=256)
        stack = None
        try:
            stack = Stack([], k=k, max_batch=256)
            for li in range(nl):
                g = torch.Generator(device="cuda")
                g.manual_seed(4000 + li)
                w = [(torch.randn(shape, generator=g, device="cuda") * cfg.sigma).to(torch.bfloat16)
                     for shape in ((d, f), (d, f), (f, d))]
                stack.layers.append(prox.Layer(*w, tau=0.0, k=k, max_batch=256))
                stack.taus.append(0.0)
                del w
            torch.cuda.empty_cache()
            x_cal = torch.from_numpy(lay0.x_cal).cuda()
            taus, _ = stack.calibrate(x_cal, cfg.s1_percent[0] / 100.0, stream=self.stream)
            x = torch.from_numpy(lay0.x_eval).cuda()
            n = x.shape[0]
            ys = [torch.empty(d, device="cuda") for _ in range(2)]
            xs = [torch.empty(d, device="cuda") for _ in range(2)]
            outs = torch.empty_like(x)
            s = self.stream
            L = stack.layers

            def body():
                for t in range(n):
                    xin = x[t]
                    for li in range(nl):
                        dst = outs[t] if li == nl - 1 else ys[li & 1]
                        L[li].forward(xin, dst, stream=s)
                        if li + 1 < nl:
                            prox.rmsnorm(dst, out=xs[li & 1], stream=s)
                            xin = xs[li & 1]
            steps = max(2, self.args.steps // 10)
            for Ly in L:
                Ly.stats()
            tok, ms = self.timer.tokens_per_s(body, n, steps, warmup=1)
            st = [Ly.stats() for Ly in L]
            mean_nx = [a / max(1, b) for a, b in st]
            tb = sum(token_bytes(d, f, k, m) for m in mean_nx)
            us = 1e6 / tok
            self.result["stack32"] = {
                "workload": f"stack of {nl} llama3_8b-shaped layers d_model={d} d_ff={f} "
                            f"s1=50% s2=70% k={k}, RMSNorm between layers",
                "tokens_per_s": round(tok, 2), "us_per_token": round(us, 1),
                "us_per_layer": round(us / nl, 2),
                "bytes_per_token": int(tb),
                "hbm_frac": round(tb / (us * 1e-6) / 1e9 / self.peaks["hbm_gbs"], 4),
                "realised_s1_mean": round(1 - statistics.mean(mean_nx) / d, 4),
                "tau_x_first_last": [taus[0], taus[-1]],
                "launches_per_token": 2 * nl - 1,
                "weights": "seeded on the GPU (torch Philox, seed 4000 + layer), N(0, 0.02^2) bf16",
                "calibration": "Algorithm 1 (Prox App. A.7), 256 tokens, tau_x at s1 50 % per layer"}
        finally:
            if stack is not None:
                stack.close()
            torch.cuda.empty_cache()

    def leg_llama3_70b(self):
        # Config 5: the Llama-3-70B-shaped layer, per-token masks at batch
        # 1, 2, 4, 8, 16 against the dense baseline at the same batch.
        torch, prox, synth = self.torch, self.prox, self.synth
        cfg = synth.get_config("llama3_70b")
        d, f = cfg.d_model, cfg.d_ff
        k = cfg.k(70)
        lay = synth.make_layer(cfg, n_tokens=64, n_cal=256)
        x_cal = torch.from_numpy(lay.x_cal).cuda()
        tau = prox.calibrate_thresholds(x_cal, 0.5)
        wg, wu, wd = bf16_dev(lay.w_gate_bits), bf16_dev(lay.w_up_bits), bf16_dev(lay.w_down_bits)
        nc = 2
        layers = [prox.Layer(wg, wu, wd, tau=tau, k=k, max_batch=16) for _ in range(nc)]
        del wg, wu, wd
        torch.cuda.empty_cache()
        x = torch.from_numpy(lay.x_eval).cuda()
        out = torch.empty_like(x)
        s = self.stream
        rows = []
        steps = max(2, self.args.steps // 10)
        C = (f + 511) // 512
        for B in cfg.batch_sizes:
            nb = 64 // B  # batches per step

            def chain(B=B, nb=nb):  # B single-token launches per batch
                for i in range(nb):
                    layers[i % nc].forward(x[i * B:(i + 1) * B], out[i * B:(i + 1) * B], stream=s)

            def union(B=B, nb=nb):  # one batched step per batch: union loads
                for i in range(nb):
                    layers[i % nc].forward_batch(x[i * B:(i + 1) * B], out[i * B:(i + 1) * B], stream=s)

            def dense(B=B, nb=nb):  # batched dense, every weight read once
                for i in range(nb):
                    layers[i % nc].dense_batch(x[i * B:(i + 1) * B], out[i * B:(i + 1) * B], stream=s)
            # the union sizes of this step's batches (bytes the union path reads)
            n_rows, n_ch = [], []
            for i in range(nb):
                layers[i % nc].forward_batch(x[i * B:(i + 1) * B], out[i * B:(i + 1) * B], stream=s)
                r_, c_ = layers[i % nc].batch_union_sizes(stream=s)
                n_rows.append(r_)
                n_ch.append(c_)
            mean_rows, mean_ch = float(np.mean(n_rows)), float(np.mean(n_ch))
            if B <= PER_TOKEN_STAGE1:  # each token reads its own kept rows
                xk = np.abs(lay.x_eval[:nb * B]) >= np.float32(tau)
                mean_rows = float(xk.sum()) / nb
            union_bytes = mean_rows * C * 512 + mean_ch * 6 * d + 8 * B * d
            dense_bytes = 6.0 * d * f + 8 * B * d
            tok_c, _ = self.timer.tokens_per_s(chain, nb * B, steps)
            tok_u, _ = self.timer.tokens_per_s(union, nb * B, steps)
            tok_d, _ = self.timer.tokens_per_s(dense, nb * B, steps)
            rows.append({
                "batch": B,
                "union_tokens_per_s": round(tok_u, 1),
                "chain_tokens_per_s": round(tok_c, 1),
                "dense_tokens_per_s": round(tok_d, 1),
                "speedup_vs_dense": round(tok_u / tok_d, 3),
                "chain_speedup_vs_dense": round(tok_c / tok_d, 3),
                "stage1_rows_frac": round(mean_rows / d, 4),
                "union_channels_frac": round(mean_ch / f, 4),
                "union_bytes_per_batch": int(union_bytes),
                "union_hbm_gbs": round(union_bytes * tok_u / B / 1e9, 1),
                "dense_hbm_gbs": round(dense_bytes * tok_d / B / 1e9, 1),
                "us_per_batch": round(B * 1e6 / tok_u, 1)})
        best = [r["batch"] for r in rows if r["speedup_vs_dense"] > 1.0]
        crossover = {"last_batch_union_beats_dense": max(best) if best else None}
        self.result["llama3_70b"] = {
            "workload": f"llama3_70b ffn layer d_model={d} d_ff={f} s1=50% s2=70% k={k}, "
                        "per-token masks",
            "paths": "union = prox_ffn_forward_batch (one batched step, union loads of the "
                     "bf16 weights; Stage 1 per token for B <= 4, over the union rows above); chain = "
                     "prox_ffn_forward (B batch-1 launches); dense = prox_dense_ffn_batch (every "
                     "weight read once); bytes: union rows x proxy row + union channels x 6 d "
                     "(gate/up record + W_down row) + x/out; dense 6 d d_ff + x/out",
            "rows": rows, "crossover": crossover, "layer_copies": nc}
        for L in layers:
            L.close()
        torch.cuda.empty_cache()

    def leg_cpu(self):
        if self.dist.rank == 0 and self.dist.world == 1:
            self.result["cpu_baseline"] = cpu_baseline(self.lay, self.tau, self.k,
                                                       self.args.cpu_seconds)

    def run(self):
        self.headline()
        if self.args.no_extras:
            return self.result
        legs = [l for l in self.args.legs.split(",") if l]
        errors = {}
        for leg in ALL_LEGS:
            if leg not in legs:
                continue
            try:
                getattr(self, "leg_" + leg)()
            except Exception as e:  # a failed extra leg is reported, not fatal
                errors[leg] = f"{type(e).__name__}: {e}"
                traceback.print_exc(file=sys.stderr)
                self.torch.cuda.synchronize()
        if errors:
            self.result["leg_errors"] = errors
        for L in self.layers:
            L.close()
        return self.result


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
    if args.record_traffic:
        import synth
        cfg = synth.get_config(args.workload)
        k = cfg.k(args.s2)
        d, f = cfg.d_model, cfg.d_ff
        alg = token_bytes(d, f, k, d // 2)
        cmd = " ".join(sys.argv[1:])
        rec = record_traffic(args.record_traffic, cfg.workload_name(cfg.s1_percent[0], args.s2),
                             alg, f"bench.py {cmd}")
        print(json.dumps(rec))
        return
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
        res = Bench(args, dist).run()
        if dist.rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        dist.close()


if __name__ == "__main__":
    main()
