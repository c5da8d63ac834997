#!/usr/bin/env python
"""Benchmark of the Prox sparse SwiGLU FFN decode path on B200.

One step = the whole hot path (Stage 1 + Stage 2, every row of the path) over
one batch of synthetic decode tokens: by default the 4096 x 12288 layer
(Qwen3-8B shape, bf16 N(0, 0.02^2) weights with INT4 proxies), 512 Laplace
tokens with 0.1% x20 outlier coordinates, processed at batch 1, thresholds
calibrated on 512 vectors for 50% input keep and 70% channel sparsity.

Timing: the 512 per-token calls are captured in one CUDA graph and replayed;
the layer is held in 4 identical copies in HBM and token t reads copy t % 4,
so every token streams its weights from HBM rather than from the 126 MB L2.
CUDA events bracket the K timed steps (after W warm-up steps) with a barrier
and a device synchronisation on both sides; the max over ranks is reported.
Under torchrun each rank is an independent replica (no collective on the
data path); value = all ranks' tokens / the slowest rank's time.

Prints ONE JSON line (rank 0). --impl reference times the fp64 CPU oracle on
the host cores on a bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "sparse SwiGLU FFN µs/token/layer @70% sparsity; achieved HBM GB/s vs peak"

WORKLOADS = {
    # name: d_model, d_ff, sigma, tokens, calibration vectors, outlier fraction
    "qwen3-8b-ffn": dict(d=4096, f=12288, sigma=0.02, tokens=512, n_cal=512, outlier=0.001),
    "tiny-ffn": dict(d=256, f=768, sigma=0.02, tokens=64, n_cal=256, outlier=0.0),
    "large-ffn": dict(d=8192, f=28672, sigma=0.015, tokens=256, n_cal=256, outlier=0.0),
    # 36 pre-norm layers (RMSNorm eps 1e-6, unit gain, fp32 residual stream),
    # each with its own weights and depth-sequentially calibrated thresholds
    "qwen3-8b-stack36": dict(d=4096, f=12288, sigma=0.02, tokens=128, n_cal=128, outlier=0.0,
                             layers=36),
}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="qwen3-8b-ffn")
    ap.add_argument("--keep-x", type=float, default=0.5)
    ap.add_argument("--keep-s", type=float, default=0.3)
    ap.add_argument("--effective-sparsity", type=float, default=None,
                    help="target effective sparsity e: keep ratios from the budget split "
                         "(prox_allocate, alpha 1/3, s1 <= 0.7) instead of --keep-x/--keep-s")
    ap.add_argument("--proxy", choices=["int4", "bf16"], default="int4",
                    help="proxy kind: the method's INT4 proxy or the bf16-proxy ablation")
    ap.add_argument("--batch", type=int, default=1,
                    help="tokens per forward call (each token keeps its own masks)")
    ap.add_argument("--engine", choices=["auto", "simt", "tc"], default="auto",
                    help="Stage-2 engine: automatic, CUDA cores, or the tensor-core union GEMM "
                         "(passes of >= 4 tokens)")
    ap.add_argument("--stage1-engine", choices=["auto", "simt", "tc"], default="auto",
                    help="Stage-1 proxy products: automatic, CUDA cores, or tensor cores "
                         "(passes of >= 4 tokens, INT4 proxy)")
    ap.add_argument("--copies", type=int, default=4, help="rotating weight copies (L2 defeat)")
    ap.add_argument("--no-dense", action="store_true", help="skip the dense cuBLAS reference")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU-oracle baseline")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the compact records of the other workloads (sparsity and "
                         "batch sweeps, the 8192 x 28672 layer, the 36-layer stack)")
    ap.add_argument("--sec-steps", type=int, default=3, help="timed steps of each secondary record")
    return ap.parse_args()


def launches_per_call(args, d, batch):
    """Kernels one forward call of `batch` tokens launches: per pass, Stage 1
    and one Stage-2 kernel (CUDA cores) or two (tensor-core union engine:
    by default passes of 8 tokens, or of 4 when d_model >= 8192; of >= 4
    when forced)."""
    from free_ffn_activation_b200 import prox as P
    per_pass = P.max_batch_per_pass(d)
    passes = -(-batch // per_pass)
    tb = 1
    while tb < min(batch, per_pass):
        tb *= 2
    tc = (tb >= 8 or (tb >= 4 and d >= 8192)) if args.engine == "auto" else (args.engine == "tc" and tb >= 4)
    return passes * (3 if tc else 2)


def summary_fields(path):
    """'- key: value' lines of a profiles/ summary as a dict."""
    fields = {}
    for line in open(path):
        if ":" in line and line.startswith("- "):
            k, v = line[2:].split(":", 1)
            fields[k.strip()] = v.strip().strip("`")
    return fields


def traffic_from_summary(fields, mean_bytes=None):
    """DRAM bytes per launch from a summary's fields, scaled from the captured
    launch's algorithmic bytes to `mean_bytes` (traffic grows with the kept
    rows); None if the fields are missing."""
    try:
        traffic = float(fields["dram bytes per launch (read + write)"])
        captured = float(fields["algorithmic bytes of the captured launch"].split()[0])
    except (KeyError, ValueError, IndexError):
        return None
    return traffic * mean_bytes / captured if mean_bytes else traffic


def stage2_traffic(workload, batch, mean_bytes=None):
    """DRAM bytes per launch of the Stage-2 kernel from the committed ncu summary,
    if it covers this workload and was captured from the current kernel source
    (else None), scaled from the captured token to `mean_bytes` algorithmic bytes."""
    if workload != "qwen3-8b-ffn" or batch != 1:
        return None
    import hashlib
    src = os.path.join(ROOT, "free_ffn_activation_b200", "csrc", "k_stage2.cu")
    summ = os.path.join(ROOT, "profiles", "k_stage2_qwen3-8b-ffn_b1.md")
    if not os.path.exists(summ):
        return None
    digest = hashlib.sha256(open(src, "rb").read()).hexdigest()
    fields = summary_fields(summ)
    if fields.get("k_stage2.cu sha256") != digest:
        return None
    return traffic_from_summary(fields, mean_bytes)


def stamp_phases(st, sampled, slot):
    """Mean phase durations (us) over the sampled calls from their
    %globaltimer stamps (slot names in prox_internal.cuh's StampSlot).
    stage1 + stage2 is the time from one call's Stage 1 passing its wait for
    the previous kernel to the next call's: Stage 1 runs until Stage 2 passes
    its wait, Stage 2 until the next Stage 1 does."""
    import numpy as np
    st = st.astype(np.uint64)
    NONE = np.uint64(0xFFFFFFFFFFFFFFFF)

    def us(a, b):
        return (float(b) - float(a)) / 1e3

    rows = {k: [] for k in ("stage1", "stage2", "s1_wait_spread", "s1_prologue", "s1_stream",
                            "s1_reduce", "s1_lists", "s1_exit_to_s2_go", "s2_go_spread",
                            "s2_list", "s2_first_data", "s2_stream_window", "s2_tail",
                            "s2_exit_to_next_s1_go", "call")}
    for c in sampled:
        if c + 1 not in slot:
            continue
        a, b = st[slot[c]], st[slot[c + 1]]
        if a[1] == NONE or a[9] == NONE or b[1] == NONE:
            continue
        rows["stage1"].append(us(a[1], a[9]))
        rows["stage2"].append(us(a[9], b[1]))
        rows["call"].append(us(a[1], b[1]))
        rows["s1_wait_spread"].append(us(a[1], a[2]))
        rows["s1_prologue"].append(us(a[1], a[3]))
        rows["s1_stream"].append(us(a[3], a[4]))
        rows["s1_reduce"].append(us(a[4], a[5]))
        rows["s1_lists"].append(us(a[5], a[6]))
        rows["s1_exit_to_s2_go"].append(us(a[6], a[9]))
        rows["s2_go_spread"].append(us(a[9], a[10]))
        rows["s2_exit_to_next_s1_go"].append(us(a[15], b[1]))
        if a[11] != 0 and a[12] != NONE:
            rows["s2_list"].append(us(a[9], a[11]))
            rows["s2_first_data"].append(us(a[11], a[13]))
            rows["s2_stream_window"].append(us(a[12], a[14]))
            rows["s2_tail"].append(us(a[14], a[15]))
    out = {k: (float(np.mean(v)) if v else None) for k, v in rows.items()}
    out["pairs"] = len(rows["call"])
    return out


def max_over_ranks(x, world, dev):
    """Largest x over the ranks: the job's time is its slowest rank's."""
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs)"
    return 6650.0, "fallback 6.65 TB/s"


class ClockSampler:
    """nvidia-smi clock / throttle samples while the timed region runs."""

    def __init__(self, index: int):
        self.index = index
        self.samples = []
        self.proc = None

    def __enter__(self):
        q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
             "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
             "clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={q}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 7:
                self.samples.append(parts)

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}

        def num(v):
            try:
                return float(v)
            except ValueError:
                return None
        sm = [num(s[0]) for s in self.samples if num(s[0]) is not None]
        mx = [num(s[1]) for s in self.samples if num(s[1]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for s in self.samples for k in range(4)
                          if s[3 + k].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# reference arm: the fp64 CPU oracle, timed on the host cores
# ---------------------------------------------------------------------------

def band_count(s_abs, tau_s, rel=1e-3):
    """Channels whose |s~| lies within rel * tau_s of tau_s (the mask band)."""
    import numpy as np
    return int(np.count_nonzero(np.abs(np.asarray(s_abs, dtype=np.float64) - tau_s) <= rel * tau_s))


def cpu_oracle_time(w, x, tau_x, tau_s, seconds):
    """The fp64 oracle on a bounded sample of the workload's tokens `x`, at the
    given thresholds (the GPU arm's): returns (us/token, threads, sample string,
    oracle band count, channels compared, realised keep_x, keep_s)."""
    import numpy as np

    import oracle
    from free_ffn_activation_b200 import synth as S
    L = S.make_layer(S.LayerSpec(w["d"], w["f"], sigma=w["sigma"], seed=0))
    Por = oracle.make_proxy(L)
    cores = os.cpu_count() or 1
    done, t_used, threads = 0, 0.0, 1
    band, kx, ks = 0, 0.0, 0.0
    while done < x.shape[0] and t_used < seconds:
        n = min(max(1, cores), x.shape[0] - done)
        t0 = time.perf_counter()
        out = oracle.forward(x[done:done + n], tau_x, tau_s, L, Por, want=("mask_x", "mask_s", "s_proxy"))
        t_used += time.perf_counter() - t0
        threads = out["threads"]
        band += band_count(np.abs(out["s_proxy"]), tau_s)
        kx += float(out["mask_x"].sum())
        ks += float(out["mask_s"].sum())
        done += n
    # the same path on one thread, over the first two tokens of the sample
    t0 = time.perf_counter()
    oracle.forward(x[0:2], tau_x, tau_s, L, Por, n_threads=1, want=())
    us_one = (time.perf_counter() - t0) / 2 * 1e6
    sample = (f"{done} of {x.shape[0]} tokens of the {w['d']}x{w['f']} layer at the GPU arm's "
              f"thresholds, all stages, fp64, {threads} threads (one thread, 2 tokens: "
              f"{us_one:.0f} us/token); realised keep_x {kx / (done * w['d']):.4f}, "
              f"keep_s {ks / (done * w['f']):.4f}")
    return t_used / done * 1e6, threads, sample, band, done * w["f"]


def run_reference(args, w, rank, world):
    """The fp64 CPU oracle as the reference arm: thresholds calibrated by the
    oracle on the same calibration vectors as the GPU arm (n_cal of them), then
    W untimed and K timed steps, each over a bounded sample of the workload's
    tokens (the whole workload would take minutes per step)."""
    if rank != 0:
        return
    import numpy as np

    import oracle
    from free_ffn_activation_b200 import synth as S
    L = S.make_layer(S.LayerSpec(w["d"], w["f"], sigma=w["sigma"], seed=0))
    Por = oracle.make_proxy(L)
    x_cal = S.make_tokens(w["n_cal"], w["d"], seed=0, stream="x_cal", outlier_frac=w["outlier"])
    t0 = time.perf_counter()
    tau_x, tau_s = oracle.calibrate(x_cal, Por, args.keep_x, args.keep_s)
    cal_s = time.perf_counter() - t0
    x = S.make_tokens(w["tokens"], w["d"], seed=0, stream="x_eval", outlier_frac=w["outlier"])
    cores = os.cpu_count() or 1
    per_step = min(w["tokens"], max(16, cores))
    times, threads, done = [], 1, 0
    for it in range(args.warmup + args.steps):
        rows = [(done + k) % w["tokens"] for k in range(per_step)]
        done += per_step
        t0 = time.perf_counter()
        out = oracle.forward(x[rows], tau_x, tau_s, L, Por, want=())
        dt = time.perf_counter() - t0
        threads = out["threads"]
        if it >= args.warmup:
            times.append(dt)
    ms_step = float(np.mean(times)) * 1e3
    us = ms_step * 1e3 / per_step
    sample = (f"{per_step} of {w['tokens']} tokens per step (consecutive, wrapping), "
              f"{args.steps} timed steps after {args.warmup}, all stages, fp64, {threads} threads; "
              f"thresholds calibrated by the oracle on {w['n_cal']} vectors ({cal_s:.1f} s)")
    line = {
        "impl": "reference", "metric": METRIC, "value": us, "unit": "us/token/layer",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, "d_model": w["d"], "d_ff": w["f"], "batch": 1,
                   "tokens_per_step": per_step, "workload_tokens": w["tokens"],
                   "n_cal": w["n_cal"], "keep_x": args.keep_x, "keep_s": args.keep_s,
                   "tau_x": tau_x, "tau_s": tau_s},
        "cpu_baseline": {"value": us, "unit": "us/token/layer", "cores": threads,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": us, "unit": "us/token/layer", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# secondary records: the other workloads of the benchmark, in the same run
# ---------------------------------------------------------------------------

def graph_us_per_token(P, torch, dev, stream, calls, ntok, steps, warmup):
    """Capture `calls` (a list of zero-argument launch functions, one forward
    call each) in one CUDA graph and return device us per token over `steps`
    timed replays after `warmup` (CUDA events on the launching stream)."""
    def one():
        for fn in calls:
            fn()
    with torch.cuda.stream(stream):
        one()
    torch.cuda.synchronize(dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        one()
    for _ in range(warmup):
        with torch.cuda.stream(stream):
            g.replay()
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        with torch.cuda.stream(stream):
            g.replay()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    del g
    return e0.elapsed_time(e1) / steps * 1e3 / ntok


def sparse_calls(P, structs, x, y, ws, Bt, tau_x, tau_s, stream):
    d = x.shape[1]
    R = len(structs)
    ntok = x.shape[0]
    return [(lambda c=c: P.ffn_forward_raw(structs[c % R], x.data_ptr() + c * Bt * d * 2, Bt,
                                           tau_x, tau_s, y.data_ptr() + c * Bt * d * 4,
                                           ws.data_ptr(), ws.numel(), stream.cuda_stream))
            for c in range(ntok // Bt)]


def dense_calls(torch, layers, x, Bt):
    """torch bf16 F.linear x3 + silu*mul (cuBLAS) per call of Bt tokens."""
    import torch.nn.functional as F
    wd_t = [lay.w_down.t().contiguous() for lay in layers]
    yd = torch.empty(x.shape, dtype=torch.bfloat16, device=x.device)
    R = len(layers)

    def call(c):
        lay = layers[c % R]
        xt = x[c * Bt:(c + 1) * Bt]
        yd[c * Bt:(c + 1) * Bt] = F.linear(F.silu(F.linear(xt, lay.w_gate_cm)) * F.linear(xt, lay.w_up_cm),
                                           wd_t[c % R])
    return [(lambda c=c: call(c)) for c in range(x.shape[0] // Bt)], wd_t


def touched_per_call(P, base, x, Bt, tau_x, tau_s):
    """Mean weight bytes one call of Bt tokens touches, and the realised
    per-token keep ratios (an untimed forward)."""
    d, f = base.d_model, base.d_ff
    out = P.ffn_forward(base, x, tau_x, tau_s)
    n = x.shape[0] // Bt
    kx = out.mask_x.view(n, Bt, d).amax(dim=1).sum(dim=1).double().cpu().numpy()
    ks = out.mask_s.view(n, Bt, f).amax(dim=1).sum(dim=1).double().cpu().numpy()
    tb = sum(P.touched_bytes(d, f, int(a), int(b)) for a, b in zip(kx, ks)) / n
    return tb, out.mask_x.float().mean().item(), out.mask_s.float().mean().item()


def secondary_records(args, dev, base, layers, structs, x, x_cal, dense_b1_us, peak):
    """Compact records of the sparsity sweep and batch sweep on the same layer,
    the 8192 x 28672 layer at batch 1 and 16, and the 36-layer stack (fewer
    timed steps than the primary measurement; same protocol)."""
    import torch

    from free_ffn_activation_b200 import prox as P
    from free_ffn_activation_b200 import synth as S
    out = {"steps": args.sec_steps, "warmup": 2}
    stream = torch.cuda.Stream(dev)
    d, f = base.d_model, base.d_ff
    ntok = x.shape[0]
    y = torch.empty((ntok, d), dtype=torch.float32, device=dev)

    def sparse_point(tx, ts, Bt):
        ws = P.workspace(d, f, Bt, dev)
        us = graph_us_per_token(P, torch, dev, stream, sparse_calls(P, structs, x, y, ws, Bt, tx, ts, stream),
                                ntok, args.sec_steps, 2)
        tb, kx, ks = touched_per_call(P, base, x, Bt, tx, ts)
        return {"us_per_token": us, "keep_x": kx, "keep_s": ks,
                "path_GBps": tb / (us * Bt * 1e-6) / 1e9}

    # sparsity sweep at batch 1 (input keep fixed at 50%)
    sweep = []
    for keep_s in (1.0, 0.7, 0.5, 0.4, 0.3, 0.2, 0.1):
        tx, ts = P.calibrate(base, x_cal, args.keep_x, keep_s)
        r = sparse_point(tx, ts, 1)
        r.update({"channel_sparsity": round(1.0 - keep_s, 3), "dense_us_per_token": dense_b1_us,
                  "speedup": dense_b1_us / r["us_per_token"]})
        sweep.append(r)
    out["qwen3-8b-ffn sparsity sweep, batch 1"] = sweep
    # batch sweep at 70% channel sparsity (each token its own masks)
    tx, ts = P.calibrate(base, x_cal, args.keep_x, args.keep_s)
    bsw = []
    for Bt in (1, 2, 4, 8):
        r = sparse_point(tx, ts, Bt)
        calls, _ = dense_calls(torch, layers, x, Bt)
        du = graph_us_per_token(P, torch, dev, stream, calls, ntok, args.sec_steps, 2)
        r.update({"batch": Bt, "dense_us_per_token": du, "speedup": du / r["us_per_token"]})
        bsw.append(r)
    out["qwen3-8b-ffn batch sweep, 70% channel sparsity"] = bsw
    del y
    torch.cuda.empty_cache()

    # the 8192 x 28672 layer (1.41 GB of bf16 weights: larger than L2 as it is)
    wl = WORKLOADS["large-ffn"]
    Ll = S.make_layer(S.LayerSpec(wl["d"], wl["f"], sigma=wl["sigma"], seed=0))
    big = P.ProxLayer.from_weights(Ll["w_up_cm"], Ll["w_gate_cm"], Ll["w_down"], device=dev)
    del Ll
    xl = P.as_bf16(S.make_tokens(wl["tokens"], wl["d"], seed=0, stream="x_eval"), dev).contiguous()
    xlc = P.as_bf16(S.make_tokens(wl["n_cal"], wl["d"], seed=0, stream="x_cal"), dev)
    txl, tsl = P.calibrate(big, xlc, args.keep_x, args.keep_s)
    yl = torch.empty((wl["tokens"], wl["d"]), dtype=torch.float32, device=dev)
    bl = []
    for Bt in (1, 16):
        ws = P.workspace(wl["d"], wl["f"], Bt, dev)
        us = graph_us_per_token(P, torch, dev, stream,
                                sparse_calls(P, [big.cstruct()], xl, yl, ws, Bt, txl, tsl, stream),
                                wl["tokens"], args.sec_steps, 2)
        tb, kx, ks = touched_per_call(P, big, xl, Bt, txl, tsl)
        calls, _ = dense_calls(torch, [big], xl, Bt)
        du = graph_us_per_token(P, torch, dev, stream, calls, wl["tokens"], args.sec_steps, 2)
        bl.append({"batch": Bt, "us_per_token": us, "dense_us_per_token": du,
                   "speedup": du / us, "keep_x": kx, "keep_s": ks,
                   "path_GBps": tb / (us * Bt * 1e-6) / 1e9, "path_frac": tb / (us * Bt * 1e-6) / 1e9 / peak})
    out["large-ffn 8192x28672, 70% channel sparsity"] = bl
    del big, xl, yl
    torch.cuda.empty_cache()

    # the 36-layer stack (per token, every layer; 128 decode tokens)
    ws_ = WORKLOADS["qwen3-8b-stack36"]
    out["qwen3-8b-stack36, 70% channel sparsity per layer, batch 1"] = stack_measure(
        args, ws_, dev, 1, 0, steps=args.sec_steps, warmup=1, e2e=False)
    return out


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def run_ours(args, w, rank, world, local_rank):
    import numpy as np
    import torch
    import torch.distributed as dist

    from free_ffn_activation_b200 import prox as P
    from free_ffn_activation_b200 import synth as S

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    d, f, ntok = w["d"], w["f"], w["tokens"]
    # each rank an independent replica with its own token stream
    L = S.make_layer(S.LayerSpec(d, f, sigma=w["sigma"], seed=0))
    x_np = S.make_tokens(ntok, d, seed=rank, stream="x_eval", outlier_frac=w["outlier"])
    xc_np = S.make_tokens(w["n_cal"], d, seed=0, stream="x_cal", outlier_frac=w["outlier"])
    pk = P.PROXY_BF16 if args.proxy == "bf16" else P.PROXY_INT4
    base = P.ProxLayer.from_weights(L["w_up_cm"], L["w_gate_cm"], L["w_down"], device=dev,
                                    proxy_kind=pk)
    xc = P.as_bf16(xc_np, dev)
    tau_x, tau_s = P.calibrate(base, xc, args.keep_x, args.keep_s)
    R = max(1, args.copies)
    layers = [base] + [P.ProxLayer(*(None if t is None else t.clone() for t in (
        base.w_up_cm, base.w_gate_cm, base.w_down, base.q_up, base.q_gate, base.s_up, base.s_gate)),
        proxy_kind=pk) for _ in range(R - 1)]
    structs = [lay.cstruct() for lay in layers]
    x = P.as_bf16(x_np, dev).contiguous()
    y = torch.empty((ntok, d), dtype=torch.float32, device=dev)
    Bt = max(1, args.batch)
    assert ntok % Bt == 0 and Bt <= P.max_batch_per_pass(d), "batch must divide the tokens and fit one pass"
    ngrp = ntok // Bt
    ws = P.workspace(d, f, Bt, dev)
    wsb = ws.numel()

    # realised keep ratios (untimed); at batch > 1 the weights a call touches
    # are those of the union of its tokens' masks
    out = P.ffn_forward(base, x, tau_x, tau_s)
    mxu = out.mask_x.view(ngrp, Bt, d).amax(dim=1)
    msu = out.mask_s.view(ngrp, Bt, f).amax(dim=1)
    kx = mxu.sum(dim=1).double().cpu().numpy()          # per call
    ks = msu.sum(dim=1).double().cpu().numpy()
    touched = np.array([P.touched_bytes(d, f, int(a), int(b), pk) for a, b in zip(kx, ks)])
    stage2_bytes = 3 * ks * d * 2
    kx_tok = out.mask_x.sum(dim=1).double().mean().item()
    ks_tok = out.count_s.double().mean().item()
    # the mask band (channels whose |s~| lies within 1e-3 tau_s of tau_s) on the
    # benchmark's own tokens, from the device's proxy state (untimed)
    nband = 0
    for c in range(ngrp):
        s_dev, _ = P.proxy_state(base, x[c * Bt:(c + 1) * Bt], tau_x)
        nband += int(((s_dev.abs() - tau_s).abs() <= 1e-3 * tau_s).sum().item())
    band = {"rel": 1e-3, "device_band": nband, "channels": ntok * f,
            "device_band_frac": nband / (ntok * f)}

    stream = torch.cuda.Stream(dev)
    sp = stream.cuda_stream
    xrow = d * 2
    yrow = d * 4
    xp, yp, wp = x.data_ptr(), y.data_ptr(), ws.data_ptr()
    # phase stamps (%globaltimer, prox_test_set_stamps) on pairs of adjacent
    # calls, every 8th pair: the second call of a pair gives the time from
    # the first call's Stage 2 to the next call's Stage 1
    sampled = sorted({c for c0 in range(0, ngrp, 8) for c in (c0, c0 + 1) if c < ngrp})
    slot = {c: k for k, c in enumerate(sampled)}
    stamps = P.stamp_buffer(len(sampled), dev)

    def one_step():
        # the timed step: the public forward per call; the sampled calls are
        # captured with the stamp hook set, so the timed graph is the one
        # whose phases are read below
        for c in range(ngrp):
            t = c * Bt
            if c in slot:
                P.test_set_stamps(stamps[slot[c]].data_ptr())
            P.ffn_forward_raw(structs[c % R], xp + t * xrow, Bt, tau_x, tau_s, yp + t * yrow,
                              wp, wsb, sp)
            if c in slot:
                P.test_set_stamps(0)

    with torch.cuda.stream(stream):
        one_step()
    torch.cuda.synchronize(dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        one_step()
    # parity spot-check of the graph's output against direct calls with the same
    # tokens per call (calls of another batch size sum the proxy in another
    # order, so a channel within rounding of tau_s may legitimately differ)
    ref_y = torch.cat([P.ffn_forward(base, x[c * Bt:(c + 1) * Bt], tau_x, tau_s,
                                     want_masks=False).y for c in range(max(1, 8 // Bt))])
    g.replay()
    torch.cuda.synchronize(dev)
    nchk = ref_y.shape[0]
    assert torch.allclose(y[:nchk], ref_y, rtol=1e-4, atol=1e-5), "graph output differs"

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    for _ in range(args.warmup):
        g.replay()
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clk:
        e0.record(stream)
        for _ in range(args.steps):
            with torch.cuda.stream(stream):
                g.replay()
            torch.cuda.current_stream(dev).wait_stream(stream)
        e1.record(stream)
        barrier()
        # one more replay of the same graph with the stamp slots reset
        P.reset_stamps(stamps)
        torch.cuda.synchronize(dev)
        with torch.cuda.stream(stream):
            g.replay()
        torch.cuda.synchronize(dev)
    status = P.last_device_status(ws)[1]
    ms_total = e0.elapsed_time(e1)
    ms_total = max_over_ranks(ms_total, world, dev)
    ms_step = ms_total / args.steps
    us_tok = ms_step * 1e3 / (ntok * world)
    us_tok_rank = ms_step * 1e3 / ntok

    peak, peak_src = load_peaks()
    ph = stamp_phases(stamps.cpu().numpy(), sampled, slot)
    pair = [c for c in sampled if c + 1 in slot]
    s1_us, s2_us = ph["stage1"], ph["stage2"]
    s2_bytes = float(np.mean(stage2_bytes[pair]))
    s2_gbs = s2_bytes / (s2_us * 1e-6) / 1e9
    s1_bytes = float(np.mean((touched - stage2_bytes)[pair]))
    s1_gbs = s1_bytes / (s1_us * 1e-6) / 1e9
    path_gbs = float(np.mean(touched)) / (us_tok_rank * Bt * 1e-6) / 1e9  # per call
    s2_stream_gbs = None
    if ph.get("s2_stream_window"):
        s2_stream_gbs = s2_bytes / (ph["s2_stream_window"] * 1e-6) / 1e9

    # e2e through the public API with host buffers: pinned x in, y out
    x_host = x.cpu().pin_memory()
    y_host = torch.empty((ntok, d), dtype=torch.float32).pin_memory()
    e2e_steps = max(1, min(args.steps, 5))

    def e2e_step():
        with torch.cuda.stream(stream):
            x.copy_(x_host, non_blocking=True)
            for c in range(ngrp):
                t = c * Bt
                P.ffn_forward_raw(structs[c % R], xp + t * xrow, Bt, tau_x, tau_s,
                                  yp + t * yrow, wp, wsb, sp)
            y_host.copy_(y, non_blocking=True)

    for _ in range(2):
        e2e_step()
    barrier()
    f0 = torch.cuda.Event(enable_timing=True)
    f1 = torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    f1.record(stream)
    barrier()
    e2e_ms = f0.elapsed_time(f1) / e2e_steps
    e2e_ms = max_over_ranks(e2e_ms, world, dev)
    e2e_us = e2e_ms * 1e3 / (ntok * world)

    # dense bf16 reference on the same GPU, same protocol (cuBLAS GEMV)
    dense = None
    if not args.no_dense:
        import torch.nn.functional as F
        wd_t = [lay.w_down.t().contiguous() for lay in layers]
        xs = x
        yd = torch.empty((ntok, d), dtype=torch.bfloat16, device=dev)

        def dense_step():
            for c in range(ngrp):
                t = c * Bt
                lay = layers[c % R]
                xt = xs[t:t + Bt]
                u = F.linear(xt, lay.w_up_cm)
                gg = F.linear(xt, lay.w_gate_cm)
                yd[t:t + Bt] = F.linear(F.silu(gg) * u, wd_t[c % R])

        with torch.cuda.stream(stream):
            dense_step()
        torch.cuda.synchronize(dev)
        gd = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gd, stream=stream):
            dense_step()
        for _ in range(args.warmup):
            gd.replay()
        barrier()
        d0 = torch.cuda.Event(enable_timing=True)
        d1 = torch.cuda.Event(enable_timing=True)
        d0.record(stream)
        for _ in range(args.steps):
            with torch.cuda.stream(stream):
                gd.replay()
        d1.record(stream)
        barrier()
        dense_us = d0.elapsed_time(d1) / args.steps * 1e3 / ntok
        dense_bytes = 3 * d * f * 2
        dense = {"us_per_token": dense_us,
                 "GBps": dense_bytes / (dense_us * 1e-6) / 1e9,
                 "speedup_of_sparse": dense_us / us_tok_rank,
                 "kind": "torch F.linear x3 + silu*mul (cuBLAS), bf16, same graph/L2 protocol"}
        del gd

    secondary = None
    if world == 1 and not args.no_secondary and args.workload == "qwen3-8b-ffn" and Bt == 1 \
            and args.proxy == "int4" and dense is not None:
        t_sec = time.perf_counter()
        try:
            secondary = secondary_records(args, dev, base, layers, structs, x, xc,
                                          dense["us_per_token"], peak)
        except Exception as exc:  # a secondary record never voids the primary one
            secondary = {"error": f"{type(exc).__name__}: {exc}"}
        secondary["wall_s"] = time.perf_counter() - t_sec

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        us_cpu, cores, sample, oband, ochan = cpu_oracle_time(w, x_np, tau_x, tau_s, args.cpu_seconds)
        cpu = {"value": us_cpu, "unit": "us/token/layer", "cores": cores, "kind": "oracle",
               "sample": sample}
        band["oracle_band"] = oband
        band["oracle_channels"] = ochan
        band["oracle_band_frac"] = oband / max(1, ochan)

    if rank == 0:
        line = {
            "metric": METRIC, "value": us_tok, "unit": "us/token/layer", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": args.workload, "d_model": d, "d_ff": f, "batch": Bt,
                       "proxy": args.proxy, "engine": args.engine,
                       "stage1_engine": args.stage1_engine,
                       "tokens_per_step": ntok, "keep_x": args.keep_x, "keep_s": args.keep_s,
                       "tau_x": tau_x, "tau_s": tau_s,
                       "l2": f"{R} rotating weight copies ({R * (3 * d * f * 2 + (d * f + 8 * d if pk == P.PROXY_INT4 else 4 * d * f)) / 1e9:.2f} GB > L2)",
                       "parallelism": f"replicas x{world}"},
            "roofline": {"bound": "hbm", "kernel": "k_stage2 (exact up/gate/down)",
                         "achieved": s2_gbs, "peak": peak, "unit": "GB/s",
                         "frac": s2_gbs / peak, "traffic": stage2_traffic(args.workload, Bt, s2_bytes) if args.proxy == "int4" else None, "peak_source": peak_src,
                         "bytes_per_launch": s2_bytes, "us_per_launch": s2_us,
                         "timing": "in the timed graph: from Stage 2 passing its wait for Stage 1 "
                                   "to the next call's Stage 1 passing its wait (globaltimer stamps)",
                         "stream_GBps": s2_stream_gbs},
            "stage1": {"kernel": f"k_stage1 ({args.proxy} proxy + channel mask)", "us_per_launch": s1_us,
                       "bytes_per_launch": s1_bytes, "GBps": s1_gbs, "frac": s1_gbs / peak},
            "phases_us": ph,
            "device_status": status,
            "band": band,
            "effective_sparsity": None if args.effective_sparsity is None else {
                "target": args.effective_sparsity,
                "realised": (1.0 - ks_tok / f) - 2.0 / 3.0 * (kx_tok / d) / 3.0,
                "s1": 1.0 - args.keep_x, "s2": 1.0 - args.keep_s},
            "path": {"touched_MB_per_call": float(np.mean(touched)) / 1e6,
                     "GBps": path_gbs, "frac_of_peak": path_gbs / peak,
                     "keep_x": kx_tok / d, "keep_s": ks_tok / f,
                     "union_keep_x": float(np.mean(kx)) / d, "union_keep_s": float(np.mean(ks)) / f},
            "dense_ref": dense,
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_us, "unit": "us/token/layer",
                    "h2d_bytes_per_step": ntok * d * 2, "d2h_bytes_per_step": ntok * d * 4},
            "gpu_launches": launches_per_call(args, d, Bt) * (ntok // Bt) * args.steps,
            "clocks": clk.summary(),
            "secondary": secondary,
        }
        print(json.dumps(line), flush=True)
    del g


def stack_measure(args, w, dev, world, rank, steps, warmup, e2e=True, dense=True, clk=None):
    """The layer stack: a step is `tokens` decode tokens, each through all
    layers (prox_ffn_block per layer: pre-norm, Prox FFN, residual add). The
    whole stack is far larger than L2, so every layer streams from HBM.
    Returns a dict of the measurements (max over ranks)."""
    import torch
    import torch.distributed as dist

    from free_ffn_activation_b200 import prox as P
    from free_ffn_activation_b200 import synth as S

    d, f, ntok, nl = w["d"], w["f"], w["tokens"], w["layers"]
    eps = 1e-6
    layers = []
    for ell in range(nl):
        L = S.make_layer(S.LayerSpec(d, f, sigma=w["sigma"], seed=0, layer=ell))
        layers.append(P.ProxLayer.from_weights(L["w_up_cm"], L["w_gate_cm"], L["w_down"],
                                               device=dev))
        del L
    structs = [lay.cstruct() for lay in layers]
    # thresholds, depth-sequentially: layer l's from the calibration vectors
    # after layers 0..l-1 (each layer keeps 50% of inputs and 30% of channels)
    h_cal = torch.from_numpy(S.bf16_to_f32(S.make_tokens(w["n_cal"], d, seed=0,
                                                          stream="x_cal"))).to(dev)
    taus = []
    for lay in layers:
        tx, ts = P.calibrate(lay, P.rmsnorm_bf16(h_cal, eps), args.keep_x, args.keep_s)
        taus.append((tx, ts))
        P.ffn_block(lay, h_cal, tx, ts, eps, h_out=h_cal, want_masks=False)
    h0 = torch.from_numpy(S.bf16_to_f32(S.make_tokens(ntok, d, seed=rank,
                                                       stream="x_eval"))).to(dev)
    h = torch.empty_like(h0)
    xbuf = torch.empty((ntok, d), dtype=torch.bfloat16, device=dev)
    ws = P.workspace(d, f, 1, dev)
    wsb, wp = ws.numel(), ws.data_ptr()
    stream = torch.cuda.Stream(dev)
    sp = stream.cuda_stream
    hrow, xrow = d * 4, d * 2

    def one_step():
        h.copy_(h0)
        for t in range(ntok):
            hp, xp = h.data_ptr() + t * hrow, xbuf.data_ptr() + t * xrow
            for ell in range(nl):
                P.ffn_block_raw(structs[ell], hp, 1, taus[ell][0], taus[ell][1], eps, hp, xp,
                                wp, wsb, sp)

    with torch.cuda.stream(stream):
        one_step()
    torch.cuda.synchronize(dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        one_step()
    for _ in range(warmup):
        with torch.cuda.stream(stream):
            g.replay()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with (clk if clk is not None else _Null()):
        e0.record(stream)
        for _ in range(steps):
            with torch.cuda.stream(stream):
                g.replay()
        e1.record(stream)
        torch.cuda.synchronize(dev)
    ms_total = max_over_ranks(e0.elapsed_time(e1), world, dev)
    ms_step = ms_total / steps
    us_tok = ms_step * 1e3 / ntok                     # all layers, per token (per rank)
    status = P.last_device_status(ws)[1]
    del g
    # touched bytes: realised keep ratios of the step's tokens, layer by layer
    hh = h0.clone()
    touched = 0.0
    for ell, lay in enumerate(layers):
        hh, _, out = P.ffn_block(lay, hh, taus[ell][0], taus[ell][1], eps)
        kx = out.mask_x.sum(dim=1).double().mean().item()
        ks = out.count_s.double().mean().item()
        touched += P.touched_bytes(d, f, int(round(kx)), int(round(ks)))
    peak, peak_src = load_peaks()
    res = {"ms_per_step": ms_step, "us_per_token": us_tok, "us_per_layer": us_tok / nl,
           "layers": nl, "tokens_per_step": ntok, "steps": steps, "warmup": warmup,
           "device_status": status,
           "path": {"touched_MB_per_token": touched / 1e6,
                    "GBps": touched / (us_tok * 1e-6) / 1e9,
                    "frac_of_peak": touched / (us_tok * 1e-6) / 1e9 / peak,
                    "peak_source": peak_src}}

    if e2e:
        # host h in, host h out, the public call per layer
        h_host = h0.cpu().pin_memory()
        out_host = torch.empty((ntok, d), dtype=torch.float32).pin_memory()

        def e2e_step():
            with torch.cuda.stream(stream):
                h.copy_(h_host, non_blocking=True)
                for t in range(ntok):
                    hp, xp = h.data_ptr() + t * hrow, xbuf.data_ptr() + t * xrow
                    for ell in range(nl):
                        P.ffn_block_raw(structs[ell], hp, 1, taus[ell][0], taus[ell][1], eps, hp,
                                        xp, wp, wsb, sp)
                out_host.copy_(h, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize(dev)
        f0 = torch.cuda.Event(enable_timing=True)
        f1 = torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        e2e_step()
        f1.record(stream)
        torch.cuda.synchronize(dev)
        res["e2e_us_per_token"] = max_over_ranks(f0.elapsed_time(f1), world, dev) * 1e3 / ntok

    if dense:
        import torch.nn.functional as F
        wd_t = [lay.w_down.t().contiguous() for lay in layers]
        hd = torch.empty_like(h0)

        def dense_step():
            hd.copy_(h0)
            for t in range(ntok):
                ht = hd[t:t + 1]
                for ell, lay in enumerate(layers):
                    xt = (ht * torch.rsqrt(ht.pow(2).mean(dim=1, keepdim=True) + eps)).to(torch.bfloat16)
                    u = F.linear(xt, lay.w_up_cm)
                    gg = F.linear(xt, lay.w_gate_cm)
                    ht.add_(F.linear(F.silu(gg) * u, wd_t[ell]).float())

        with torch.cuda.stream(stream):
            dense_step()
        torch.cuda.synchronize(dev)
        gd = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gd, stream=stream):
            dense_step()
        for _ in range(warmup):
            with torch.cuda.stream(stream):
                gd.replay()
        torch.cuda.synchronize(dev)
        d0 = torch.cuda.Event(enable_timing=True)
        d1 = torch.cuda.Event(enable_timing=True)
        d0.record(stream)
        for _ in range(steps):
            with torch.cuda.stream(stream):
                gd.replay()
        d1.record(stream)
        torch.cuda.synchronize(dev)
        dense_us = max_over_ranks(d0.elapsed_time(d1), world, dev) / steps * 1e3 / ntok
        res["dense_ref"] = {"us_per_token": dense_us, "speedup_of_sparse": dense_us / us_tok,
                            "kind": "torch RMSNorm + F.linear x3 + silu*mul (cuBLAS), bf16, same protocol"}
        del gd, wd_t
    del layers, structs
    torch.cuda.empty_cache()
    return res


class _Null:
    def __enter__(self):
        return self

    def __exit__(self, *exc):
        return False


def run_stack(args, w, rank, world, local_rank):
    import torch

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    with ClockSampler(local_rank) as clk:
        r = stack_measure(args, w, dev, world, rank, args.steps, args.warmup, clk=clk)
    if rank == 0:
        d, f, ntok, nl = w["d"], w["f"], w["tokens"], w["layers"]
        line = {
            "metric": "sparse SwiGLU FFN stack µs/token (all layers) @70% sparsity",
            "value": r["us_per_token"] / world,
            "unit": "us/token", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": r["ms_per_step"], "higher_is_better": False, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": args.workload, "layers": nl, "d_model": d, "d_ff": f,
                       "batch": 1, "tokens_per_step": ntok, "keep_x": args.keep_x,
                       "keep_s": args.keep_s, "rmsnorm_eps": 1e-6,
                       "l2": f"{nl} distinct layers ({nl * (3 * d * f * 2 + d * f + 8 * d) / 1e9:.1f} GB > L2)",
                       "parallelism": f"replicas x{world}"},
            "us_per_layer": r["us_per_layer"],
            "path": r["path"],
            "dense_ref": r.get("dense_ref"),
            "device_status": r["device_status"],
            "e2e": {"value": r["e2e_us_per_token"] / world, "unit": "us/token",
                    "h2d_bytes_per_step": ntok * d * 4, "d2h_bytes_per_step": ntok * d * 4},
            "gpu_launches": 3 * nl * ntok * args.steps,
            "clocks": clk.summary(),
        }
        print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.effective_sparsity is not None:
        # the pages' compute budget: e = s2 - 2 alpha (1 - s1) / 3 with alpha = 1/3
        from free_ffn_activation_b200 import prox as P
        s1, s2 = P.allocate(args.effective_sparsity)
        args.keep_x, args.keep_s = 1.0 - s1, 1.0 - s2
    w = WORKLOADS[args.workload]
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if "layers" in w:
            if rank == 0:
                print(json.dumps({"impl": "reference", "unavailable":
                                  "the layer stack has no CPU-oracle arm (single-layer workloads have one)"}))
            return
        run_reference(args, w, rank, world)
        return
    from free_ffn_activation_b200 import prox as P
    engines = {"auto": P.ENGINE_AUTO, "simt": P.ENGINE_SIMT, "tc": P.ENGINE_TC}
    P.set_stage2_engine(engines[args.engine])
    P.set_stage1_engine(engines[args.stage1_engine])
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        if "layers" in w:
            run_stack(args, w, rank, world, local_rank)
        else:
            run_ours(args, w, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
