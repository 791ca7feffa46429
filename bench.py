"""Benchmark: exact attention forward + backward on B200 (libfa, sm_100a).

One step = the whole hot path on one batch: fa_fwd (O, LSE) then fa_bwd
(dQ, dK, dV) on the long-context causal workload B=1, H=16, N=32768, d=128,
bf16, scale 1/sqrt(d), seeded N(0, 1) inputs.  FLOPs follow the usual
convention: forward 4*B*H*N^2*d, backward 2.5x that, both halved for causal.

Prints one JSON line (rank 0).  `value` is device-timed throughput (CUDA
events around exactly --steps steps, inputs resident in HBM, max over ranks);
`e2e` is the same metric through the C ABI with host buffers (pinned
host->device copy of Q, K, V, dO and device->host copy of O, LSE, dQ, dK, dV
inside the timed region).  Multi-GPU (torchrun): every rank runs its own
batch of heads (no collective on the data path), weak scaling.

--impl reference times the fp64 CPU oracle (the correctness reference) on a
bounded sample of the same job (forward and backward of one head) on the host
cores.  The GPU line also carries `per_config`: forward and backward timings of
every workload of the evaluation (the five configurations, the sweep's twelve
runs included), and `cpu_baseline.per_config`: the oracle's wall time and
GFLOPS on a bounded sample of each.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = dict(name="long-context fwd+bwd causal", B=1, H=16, N=32768, d=128, causal=True, seed_workload=4)
METRIC = "attention fwd/bwd TFLOPS (bf16, 1xB200) and % of dense BF16 tensor peak"
DATASHEET_BF16_TFLOPS = 2250.0


def flops(B, H, N, d, causal):
    f = 4.0 * B * H * N * N * d * (0.5 if causal else 1.0)
    return f, 2.5 * f


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            p = json.load(fh)
        return dict(burst=float(p["bf16_tflops"]), sustained=float(p["bf16_tflops_sustained"]),
                    hbm=float(p["hbm_gbs"]), source="measured")
    except (OSError, KeyError, ValueError):
        return dict(burst=1590.0, sustained=1400.0, hbm=6650.0, source="fallback")


E2E_CHUNKS = 4  # head chunks of the end-to-end step (copies of one chunk overlap another's kernels)
PROBE_STEPS, PROBE_KEEP = 24, 16  # untimed steps with clock probes after the timed loop; kept (last)
KERNEL_SOURCES = ("fa_fwd.cuh", "fa_bwd.cuh", "sm100.cuh", "exp2_poly.cuh")


def kernel_source_hash():
    """SHA-256 over the kernel sources with comments and blank space removed (the code the
    compiler sees); a stored ncu traffic figure is only valid for the same hash."""
    import hashlib
    import re
    h = hashlib.sha256()
    for name in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "exact_attention_159_b200", "csrc", name)) as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()


def stored_traffic(kernel):
    """DRAM bytes per launch of `kernel` ("fwd" or "bwd") from the committed ncu summary of the bench
    workload, or None when the summary is missing or was taken on other kernel sources."""
    path = os.path.join(ROOT, "profiles", "dram_traffic_long_context_causal_B1_H16_N32768_d128.md")
    try:
        text = open(path).read()
    except OSError:
        return None
    import re
    src = re.search(r"kernel_source_sha256:\s*([0-9a-f]{64})", text)
    val = re.search(rf"{kernel}_traffic_bytes_per_launch:\s*([0-9]+)", text)
    if not src or not val or src.group(1) != kernel_source_hash():
        return None
    return int(val.group(1))


def config_dict(n_gpus):
    w = WORKLOAD
    return {"workload": f"{w['name']}: B={w['B']} H={w['H']} N={w['N']} d={w['d']}",
            "B": w["B"], "H": w["H"], "seq_len": w["N"], "head_dim": w["d"], "causal": w["causal"],
            "global_batch_heads": w["B"] * w["H"] * n_gpus, "parallelism": f"heads sharded x{n_gpus} (no collective)",
            "l2": "inputs larger than L2 (Q, K, V, dO 134 MB each vs 126 MB L2); no explicit flush"}


# --------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples during the timed region (SM clock, throttle reasons)."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = max(mx, float(f[2]))
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        loaded = sorted(sm)[len(sm) // 4:] or sm  # drop the idle head of the record
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------- multi-rank
def rank_seed(workload_seed, rank):
    """Seed of a rank's inputs: every rank draws its own heads (weak scaling)."""
    return workload_seed + 100 * rank


def max_over_ranks(values, world, device):
    """Element-wise max over ranks of per-rank timings (a collective only when world > 1)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t]


def job_tflops(flops_per_rank, world, ms_per_step):
    """Whole-job throughput: the work of every rank divided by the slowest rank's time."""
    return flops_per_rank * world / (ms_per_step * 1e-3) / 1e12


# ------------------------------------------------------------------ GPU arm
def run_gpu(args):
    import numpy as np
    import torch
    import torch.distributed as dist

    from exact_attention_159_b200 import api, build, inputs as I

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    build.build()
    w = WORKLOAD
    B, H, N, d, causal = w["B"], w["H"], w["N"], w["d"], w["causal"]
    scale = 1.0 / math.sqrt(d)
    # each rank draws its own heads (weak scaling): shift the seed by rank
    bits = I.attention_inputs(rank_seed(w["seed_workload"], rank), B, H, N, d, with_do=True)
    host = {k: torch.from_numpy(v.view(np.int16)).view(torch.bfloat16).pin_memory() for k, v in bits.items()}
    dev = {k: v.cuda() for k, v in host.items()}
    o = torch.empty_like(dev["q"])
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    dq, dk, dv = (torch.empty_like(dev["q"]) for _ in range(3))
    ws = torch.empty(api.fa_bwd_workspace_size(B, H, N, d), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    def step(prof=None):
        if prof is not None:
            api.fa_profile_next(0, prof[0], prof[1])
            api.fa_profile_next(1, prof[2], prof[3])
        api.fa_fwd(dev["q"], dev["k"], dev["v"], scale, causal, out=o, lse=lse)
        api.fa_bwd(dev["q"], dev["k"], dev["v"], o, dev["do"], lse, scale, causal, dq=dq, dk=dk, dv=dv,
                   workspace=ws)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        step()
    barrier()
    rc, detail = api.fa_last_device_status()
    if rc != 0:
        raise RuntimeError(f"device status {rc} ({detail:#x}) after warm-up")

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    for e4 in ev:  # torch creates the CUDA event handle at its first record
        for e in e4:
            e.record(stream)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier()
        t0.record(stream)
        for i in range(args.steps):
            step(ev[i])
        t1.record(stream)
        barrier()
    rc, detail = api.fa_last_device_status()
    if rc != 0:
        raise RuntimeError(f"device status {rc} ({detail:#x}) in the timed region")
    ms = t0.elapsed_time(t1)
    fwd_ms = [e[0].elapsed_time(e[1]) for e in ev]
    bwd_ms = [e[2].elapsed_time(e[3]) for e in ev]

    # The SM clock the kernels actually ran at, measured on the device right after the timed loop
    # (untimed): a probe kernel queued behind the forward and the backward of a few more steps,
    # with no synchronisation in between (an idle gap lets the power manager raise the clock).
    # Under the power cap it can sit well below what nvidia-smi's sampled clocks.sm reports.
    # The host work after the loop idles the GPU long enough for the clock to recover, so the pass
    # runs PROBE_STEPS steps and keeps the last PROBE_KEEP, once the power manager has settled.
    probe = torch.zeros((2 * PROBE_STEPS, 2), dtype=torch.int64, device="cuda")
    for i in range(PROBE_STEPS):
        api.fa_fwd(dev["q"], dev["k"], dev["v"], scale, causal, out=o, lse=lse)
        api.fa_sm_clock_probe(probe[2 * i], stream)
        api.fa_bwd(dev["q"], dev["k"], dev["v"], o, dev["do"], lse, scale, causal, dq=dq, dk=dk, dv=dv,
                   workspace=ws)
        api.fa_sm_clock_probe(probe[2 * i + 1], stream)
    torch.cuda.synchronize()
    eff_all = [1000.0 * c / ns if ns > 0 else 0.0 for c, ns in probe.tolist()]
    eff_mhz = [x for x in eff_all[-2 * PROBE_KEEP:] if x > 0]

    # end to end through host buffers
    h_out = {k: torch.empty(v.shape, dtype=v.dtype).pin_memory() for k, v in
             (("o", o), ("lse", lse), ("dq", dq), ("dk", dk), ("dv", dv))}
    h2d = sum(host[k].numel() * host[k].element_size() for k in ("q", "k", "v", "do"))
    d2h = sum(t.numel() * t.element_size() for t in h_out.values())

    # The heads are independent, so the end-to-end step streams them in chunks: the copy of chunk
    # c+1's inputs and of chunk c-1's results overlap the kernels of chunk c (copy engines on their
    # own streams, ordered by events).  Every byte still crosses PCIe inside the timed region.
    chunks = args.e2e_chunks
    n_chunks = chunks if (B == 1 and chunks >= 1 and H % chunks == 0) else 1
    hc = H // n_chunks
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ws_c = torch.empty(api.fa_bwd_workspace_size(B, hc, N, d), dtype=torch.uint8, device="cuda")

    def heads(t, c):
        return t[:, c * hc:(c + 1) * hc]

    prev_done = [None] * n_chunks  # chunk c's kernels of the previous step read its device inputs
    prev_out = [None] * n_chunks   # chunk c's copies to the host of the previous step read its outputs

    def e2e_step():
        ev_in = [torch.cuda.Event() for _ in range(n_chunks)]
        ev_done = [torch.cuda.Event() for _ in range(n_chunks)]
        ev_out = [torch.cuda.Event() for _ in range(n_chunks)]
        for c in range(n_chunks):
            if prev_done[c] is not None:
                s_in.wait_event(prev_done[c])
            with torch.cuda.stream(s_in):
                for k in ("q", "k", "v", "do"):
                    heads(dev[k], c).copy_(heads(host[k], c), non_blocking=True)
                ev_in[c].record(s_in)
        for c in range(n_chunks):
            stream.wait_event(ev_in[c])
            if prev_out[c] is not None:
                stream.wait_event(prev_out[c])
            q_, k_, v_, do_ = (heads(dev[x], c) for x in ("q", "k", "v", "do"))
            o_, lse_ = heads(o, c), heads(lse, c)
            api.fa_fwd(q_, k_, v_, scale, causal, out=o_, lse=lse_)
            api.fa_bwd(q_, k_, v_, o_, do_, lse_, scale, causal, dq=heads(dq, c), dk=heads(dk, c), dv=heads(dv, c),
                       workspace=ws_c)
            ev_done[c].record(stream)
            s_out.wait_event(ev_done[c])
            with torch.cuda.stream(s_out):
                for k, t in (("o", o), ("lse", lse), ("dq", dq), ("dk", dk), ("dv", dv)):
                    heads(h_out[k], c).copy_(heads(t, c), non_blocking=True)
                ev_out[c].record(s_out)
        prev_done[:] = ev_done
        prev_out[:] = ev_out

    e2e_steps = max(1, args.steps)
    e2e_step()
    stream.wait_stream(s_out)
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    e0.record(stream)
    s_in.wait_event(e0)  # the first copies start inside the timed region
    for _ in range(e2e_steps):
        e2e_step()
    stream.wait_stream(s_out)  # the timed region ends when the last results are on the host
    e1.record(stream)
    barrier()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps

    ms, e2e_ms = max_over_ranks([ms, e2e_ms], world, "cuda")
    f_fwd, f_bwd = flops(B, H, N, d, causal)
    ms_step = ms / args.steps
    value = job_tflops(f_fwd + f_bwd, world, ms_step)
    pk = peaks()
    fwd_avg = statistics.mean(fwd_ms)
    bwd_avg = statistics.mean(bwd_ms)
    fwd_tf = f_fwd / (fwd_avg * 1e-3) / 1e12
    bwd_tf = f_bwd / (bwd_avg * 1e-3) / 1e12
    dominant = "bwd" if bwd_avg >= fwd_avg else "fwd"
    ach = bwd_tf if dominant == "bwd" else fwd_tf
    result = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOPS", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) bf16)",
        "config": config_dict(world),
        "fwd_tflops": round(fwd_tf, 2), "bwd_tflops": round(bwd_tf, 2),
        "fwd_ms": round(fwd_avg, 4), "bwd_main_ms": round(bwd_avg, 4),
        "pct_dense_bf16_peak": {"step": round(100 * value / world / DATASHEET_BF16_TFLOPS, 2),
                                "fwd": round(100 * fwd_tf / DATASHEET_BF16_TFLOPS, 2),
                                "bwd": round(100 * bwd_tf / DATASHEET_BF16_TFLOPS, 2),
                                "denominator": "2250 TFLOPS datasheet dense bf16",
                                "fwd_of_measured_burst": round(100 * fwd_tf / pk["burst"], 2),
                                "bwd_of_measured_burst": round(100 * bwd_tf / pk["burst"], 2)},
        "roofline": {"bound": "tensor", "kernel": f"{dominant} attention kernel", "achieved": round(ach, 2),
                     "peak": pk["burst"], "unit": "TFLOP/s", "frac": round(ach / pk["burst"], 4),
                     "peak_kind": f"{pk['source']} burst bf16 GEMM (the timed region lasts "
                                  f"{ms * 1e-3:.2f} s, well under a seconds-long sustained loop)",
                     "frac_of_sustained": round(ach / pk["sustained"], 4),
                     "fwd_frac": round(fwd_tf / pk["burst"], 4), "bwd_frac": round(bwd_tf / pk["burst"], 4),
                     "traffic": stored_traffic(dominant),
                     "traffic_unit": "bytes per launch (ncu dram__bytes_read.sum + dram__bytes_write.sum)"},
        "e2e": {"value": round(job_tflops(f_fwd + f_bwd, world, e2e_ms), 2), "unit": "TFLOPS",
                "h2d_bytes_per_step": h2d * world, "d2h_bytes_per_step": d2h * world,
                "ms_per_step": round(e2e_ms, 3),
                "pipeline": f"{n_chunks} head chunks; pinned-host copies overlap the kernels on separate streams"},
        "gpu_launches": 4 * args.steps,
        "clocks": {**clk.summary(), "sm_mhz_effective": round(statistics.median(eff_mhz)) if eff_mhz else None,
                   "sm_mhz_effective_range": [round(min(eff_mhz)), round(max(eff_mhz))] if eff_mhz else None,
                   "sm_mhz_effective_how": f"device probe (clock64 cycles over 20 us of %globaltimer) queued behind "
                                           f"the forward and the backward of the last {PROBE_KEEP} of {PROBE_STEPS} "
                                           f"untimed steps run back to back after the timed loop"},
    }
    if not args.no_per_config:
        # every rank times the same extra shapes; rank 0 reports its own numbers (untimed by the main loop)
        try:
            result["per_config"] = gpu_per_config(api, reps=args.per_config_reps)
        except Exception as exc:  # the headline line above stands on its own
            result["per_config"] = {"error": f"{type(exc).__name__}: {exc}"}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(budget_s=args.cpu_seconds)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


# ------------------------------------------------------- per-config GPU timings
def configurations():
    """The evaluation's workloads, each with the passes its configuration names: (tag, workload id,
    B, H, N, d, causal, stress, backward).  Workload 5 is the twelve-run backward sweep."""
    from exact_attention_159_b200 import inputs as I
    out = []
    for wid, w in sorted(I.WORKLOADS.items()):
        out.append((w["name"], wid, w["B"], w["H"], w["N"], w["d"], w["causal"], w["stress"], w["bwd"]))
    for w in I.SWEEP:
        out.append((w["name"], 5, w["B"], w["H"], w["N"], w["d"], w["causal"], w["stress"], True))
    return out


def device_inputs(seed, B, H, N, d, stress, with_do):
    """Seeded N(0, 1) bf16 inputs drawn on the device with torch's generator (timing only: the same
    distributions and the same rescale-stress construction as the host generator, not its bits)."""
    import torch
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    shape = (B, H, N, d)
    t = {k: torch.randn(shape, generator=g, device="cuda", dtype=torch.float32) for k in ("q", "k", "v")}
    if stress:
        u = torch.randn(d, generator=g, device="cuda", dtype=torch.float64)
        u = (u / u.norm()).float()
        for k in ("q", "k"):
            a = torch.rand((B, H, N, 1), generator=g, device="cuda", dtype=torch.float32) * 8.0
            t[k] += a * u
    if with_do:
        t["do"] = torch.randn(shape, generator=g, device="cuda", dtype=torch.float32)
    return {k: v.to(torch.bfloat16) for k, v in t.items()}


def gpu_per_config(api, reps=5):
    """Forward and backward device time of every workload: `reps` calls each, the L2 flushed
    (a 256 MB write) before every timed call, CUDA events on the launching stream; medians."""
    import torch
    stream = torch.cuda.current_stream()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    rows = []
    for tag, wid, B, H, N, d, causal, stress, bwd in configurations():
        x = device_inputs(1000 * wid + 7, B, H, N, d, stress, bwd)
        scale = 1.0 / math.sqrt(d)
        o, lse = api.fa_fwd(x["q"], x["k"], x["v"], scale, causal)
        f_fwd, f_bwd = flops(B, H, N, d, causal)
        ws = torch.empty(api.fa_bwd_workspace_size(B, H, N, d), dtype=torch.uint8, device="cuda") if bwd else None
        grads = [torch.empty_like(x["q"]) for _ in range(3)] if bwd else None

        def timed(fn, prof_which=None):
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
            for e in ev[2:]:  # torch creates an event's handle at its first record
                e.record(stream)
            flush.zero_()
            if prof_which is not None:
                api.fa_profile_next(prof_which, ev[2], ev[3])
            ev[0].record(stream)
            fn()
            ev[1].record(stream)
            return ev

        def fwd_call():
            api.fa_fwd(x["q"], x["k"], x["v"], scale, causal, out=o, lse=lse)

        def bwd_call():
            api.fa_bwd(x["q"], x["k"], x["v"], o, x["do"], lse, scale, causal, dq=grads[0], dk=grads[1],
                       dv=grads[2], workspace=ws)

        fwd_call()
        if bwd:
            bwd_call()
        fe = [timed(fwd_call) for _ in range(reps)]
        be = [timed(bwd_call, 1) for _ in range(reps)] if bwd else []
        torch.cuda.synchronize()
        rc, detail = api.fa_last_device_status()
        if rc != 0:
            raise RuntimeError(f"device status {rc} ({detail:#x}) in the per-config timings ({tag})")
        f_ms = statistics.median(e[0].elapsed_time(e[1]) for e in fe)
        row = {"config": tag, "workload": wid, "B": B, "H": H, "N": N, "d": d, "causal": causal,
               "fwd_ms": round(f_ms, 4), "fwd_tflops": round(f_fwd / (f_ms * 1e-3) / 1e12, 2)}
        if bwd:
            b_ms = statistics.median(e[0].elapsed_time(e[1]) for e in be)
            m_ms = statistics.median(e[2].elapsed_time(e[3]) for e in be)
            row.update(bwd_ms=round(b_ms, 4), bwd_tflops=round(f_bwd / (b_ms * 1e-3) / 1e12, 2),
                       bwd_main_ms=round(m_ms, 4), bwd_main_tflops=round(f_bwd / (m_ms * 1e-3) / 1e12, 2))
        if wid == 4 and d == 128:
            # the cluster-pair (cta_group::2) variants of both kernels on the same inputs, for comparison;
            # a failure here is reported in the row and leaves the other timings in place
            try:
                api.fa_set_forward_variant(1)
                fwd_call()
                pe = [timed(fwd_call) for _ in range(reps)]
                api.fa_set_forward_variant(0)
                api.fa_set_backward_variant(1)
                if bwd:
                    bwd_call()
                pb = [timed(bwd_call, 1) for _ in range(reps)] if bwd else []
                torch.cuda.synchronize()
                p_ms = statistics.median(e[0].elapsed_time(e[1]) for e in pe)
                row.update(pair_fwd_ms=round(p_ms, 4), pair_fwd_tflops=round(f_fwd / (p_ms * 1e-3) / 1e12, 2))
                if bwd:
                    pm_ms = statistics.median(e[2].elapsed_time(e[3]) for e in pb)
                    row.update(pair_bwd_main_ms=round(pm_ms, 4),
                               pair_bwd_main_tflops=round(f_bwd / (pm_ms * 1e-3) / 1e12, 2))
            except Exception as exc:  # noqa: BLE001 -- reported in the JSON line
                row["pair_error"] = f"{type(exc).__name__}: {exc}"
            finally:
                api.fa_set_forward_variant(0)
                api.fa_set_backward_variant(0)
        rows.append(row)
        del x, o, lse, ws, grads
    return {"rows": rows, "inputs": "seeded N(0,1) bf16 drawn on the device (torch generator), stress "
                                    "construction for workload 3", "timing": f"median of {reps} calls, L2 flushed "
                                    "before each, CUDA events; bwd = the whole fa_bwd call (3 kernels), bwd_main "
                                    "= its main kernel; pair_* = the cluster-pair (cta_group::2) variants on workload 4",
            "flops": "fwd 4*B*H*N^2*d, bwd 2.5x, halved for causal"}


# ---------------------------------------------------------------- CPU oracle
def _visible_rows(N, causal):
    """Number of keys each query row sees (square problems)."""
    import numpy as np
    return np.arange(1, N + 1, dtype=np.float64) if causal else np.full(N, float(N))


def oracle_head(wid, B, H, N, d, stress, bwd):
    """fp64 operands of head (0, 0) of a workload (exact widenings of the seeded bf16 inputs)."""
    from exact_attention_159_b200 import inputs as I
    bits = I.head_inputs(wid, B, H, N, d, 0, 0, stress=stress, with_do=bwd)
    return {k: I.bf16_bits_to_f64(v) for k, v in bits.items()}


def oracle_sample(wid, B, H, N, d, causal, stress, bwd, fwd_budget_s, threads, n_bwd_rows=64, x=None):
    """The fp64 oracle on head (0, 0) of one workload: forward of every stride-th query row (stride
    chosen for ~fwd_budget_s), and, with bwd, the backward for 64 sampled query rows (dQ) and 64
    sampled key rows (dK, dV).  FLOPs are those of the outputs produced, each GEMM counted once:
    forward 4*d per visible (query, key) pair; backward 4*d per visible pair over every row (S and dP,
    which LSE and D need) + 2*d per visible pair of the dQ rows + 4*d per visible pair of the dK / dV
    rows (at full size these add up to the 10*d per pair, 2.5x the forward, of the convention)."""
    import numpy as np

    from oracle import oracle as OR

    if x is None:
        x = oracle_head(wid, B, H, N, d, stress, bwd)
    scale = 1.0 / math.sqrt(d)
    vis = _visible_rows(N, causal)
    probe = np.arange(0, N, max(1, N // 64))
    t = time.perf_counter()
    OR.fwd(x["q"], x["k"], x["v"], scale, causal, rows=probe, nthreads=threads)
    per_row = max(time.perf_counter() - t, 1e-4) / probe.size
    stride = max(1, int(math.ceil(N * per_row / fwd_budget_s)))
    rows = np.arange(stride // 2, N, stride)
    t = time.perf_counter()
    OR.fwd(x["q"], x["k"], x["v"], scale, causal, rows=rows, nthreads=threads)
    f_s = time.perf_counter() - t
    f_fl = float(4.0 * d * vis[rows].sum())
    out = {"fwd": {"seconds": round(f_s, 3), "gflops": round(f_fl / f_s / 1e9, 3), "flops": f_fl,
                   "sample": f"{rows.size} of {N} query rows (every {stride}th) of head (0,0)"}}
    if bwd:
        rng = np.random.default_rng(wid * 100 + N + d + int(causal))
        qr = np.unique(np.concatenate([[0, N - 1], rng.choice(N, size=min(N, n_bwd_rows), replace=False)]))
        kr = np.unique(np.concatenate([[0, N - 1], rng.choice(N, size=min(N, n_bwd_rows), replace=False)]))
        t = time.perf_counter()
        OR.bwd(x["q"], x["k"], x["v"], x["do"], scale, causal, qrows=qr, krows=kr, nthreads=threads)
        b_s = time.perf_counter() - t
        kvis = (N - kr).astype(np.float64) if causal else np.full(kr.size, float(N))
        b_fl = float(4.0 * d * vis.sum() + 2.0 * d * vis[qr].sum() + 4.0 * d * kvis.sum())
        out["bwd"] = {"seconds": round(b_s, 3), "gflops": round(b_fl / b_s / 1e9, 3), "flops": b_fl,
                      "sample": f"head (0,0): LSE and D of all {N} rows, dQ of {qr.size} query rows, "
                                f"dK and dV of {kr.size} key rows"}
    return out


def cpu_baseline(budget_s=15.0):
    """The oracle on every workload (head (0, 0), bounded samples); the headline value is the bench
    workload's forward + backward sample."""
    from oracle import oracle as OR

    threads = OR.default_threads()
    per = []
    head = None
    t0 = time.perf_counter()
    for tag, wid, B, H, N, d, causal, stress, bwd in configurations():
        fwd_budget = budget_s / 10.0 if wid == 4 else budget_s / 40.0
        r = oracle_sample(wid, B, H, N, d, causal, stress, bwd, fwd_budget, threads)
        row = {"config": tag, "workload": wid, "B": B, "H": H, "N": N, "d": d, "causal": causal, **r}
        per.append(row)
        if wid == 4:
            head = r
    fl = head["fwd"]["flops"] + head["bwd"]["flops"]
    sec = head["fwd"]["seconds"] + head["bwd"]["seconds"]
    return {"value": round(fl / sec / 1e12, 6), "unit": "TFLOPS", "cores": threads, "kind": "oracle",
            "sample": "fp64 oracle, head (0,0) of the bench workload: forward of "
                      f"{head['fwd']['sample'].split(' (')[0]}, and the backward ({head['bwd']['sample']}); "
                      "FLOPs of the outputs produced, each GEMM counted once",
            "seconds": round(sec, 2), "per_config": per, "per_config_seconds": round(time.perf_counter() - t0, 1)}


def run_reference(args):
    from oracle import oracle as OR

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    w = WORKLOAD
    threads = OR.default_threads()
    B, H, N, d, causal = w["B"], w["H"], w["N"], w["d"], w["causal"]
    fwd_budget = max(0.2, min(1.0, 30.0 / max(1, args.steps + args.warmup)))
    x = oracle_head(w["seed_workload"], B, H, N, d, False, True)
    samples = []
    for i in range(args.warmup + args.steps):
        r = oracle_sample(w["seed_workload"], B, H, N, d, causal, False, True, fwd_budget, threads, x=x)
        if i >= args.warmup:
            samples.append(r)
    fl = sum(r["fwd"]["flops"] + r["bwd"]["flops"] for r in samples)
    sec = sum(r["fwd"]["seconds"] + r["bwd"]["seconds"] for r in samples)
    value = fl / sec / 1e12
    sample = (f"fp64 oracle per step, head (0,0) of the workload: forward of {samples[0]['fwd']['sample'].split(' (')[0]}"
              f" and the backward ({samples[0]['bwd']['sample']}); FLOPs of the outputs produced, each GEMM counted once")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOPS", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(sec / max(1, args.steps) * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) bf16)", "config": config_dict(world),
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOPS", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def run_profile(args):
    """A few plain calls on one shape, for ncu captures: --profile fwd|bwd --shape B,H,N,d."""
    import numpy as np
    import torch

    from exact_attention_159_b200 import api, build, inputs as I

    B, H, N, d = (int(x) for x in args.shape.split(","))
    causal = bool(args.causal)
    torch.cuda.set_device(0)
    build.build()
    bits = I.attention_inputs(4, B, H, N, d, with_do=True)
    dev = {k: torch.from_numpy(v.view(np.int16)).view(torch.bfloat16).cuda() for k, v in bits.items()}
    scale = 1.0 / math.sqrt(d)
    o, lse = api.fa_fwd(dev["q"], dev["k"], dev["v"], scale, causal)
    calls = 3
    for _ in range(calls):
        if args.profile == "fwd":
            api.fa_fwd(dev["q"], dev["k"], dev["v"], scale, causal, out=o, lse=lse)
        else:
            api.fa_bwd(dev["q"], dev["k"], dev["v"], o, dev["do"], lse, scale, causal)
    torch.cuda.synchronize()
    rc, detail = api.fa_last_device_status()
    if rc != 0:
        raise RuntimeError(f"device status {rc} ({detail:#x})")
    print(f"profile {args.profile} B={B} H={H} N={N} d={d} causal={causal}: {calls + 1} calls ok")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true", help="skip the per-configuration GPU timings")
    ap.add_argument("--per-config-reps", type=int, default=5, help="timed calls per configuration")
    ap.add_argument("--profile", choices=["fwd", "bwd"], help="plain calls on --shape for ncu captures")
    ap.add_argument("--shape", default="1,16,16384,128", help="B,H,N,d for --profile")
    ap.add_argument("--causal", type=int, default=1, help="causal flag for --profile")
    ap.add_argument("--source-hash", action="store_true", help="print the kernel source hash and exit")
    ap.add_argument("--e2e-chunks", type=int, default=E2E_CHUNKS, help="head chunks of the end-to-end step")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)  # at least 3 untimed warm-up steps
    if args.source_hash:
        print(kernel_source_hash())
        return
    if args.profile:
        run_profile(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
