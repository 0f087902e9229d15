#!/usr/bin/env python
"""Benchmark of the online activation path on B200.

One step = one pass of the whole hot path over one batch resident in HBM:
residual alignment -> RMSNorm -> INT4 (rsq_align_norm_quant) and the
randomised Hadamard 2^12 -> INT4 (rht_quant), both on the same T x D bf16
batch (T = 16384 tokens per GPU, D = 4096, r = 32).  Token rows are
independent, so N GPUs process N independent shards with no collective on the
data path ("weak" scaling); the only collectives are the timing barrier and the
max-over-ranks of the elapsed time.

Prints ONE JSON line on rank 0.  `--impl reference` times the float64 CPU
oracle instead (rank 0 only, bounded samples).
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "tokens/s & HBM GB/s (frac of B200 peak), fused align+FWHT+INT4 quant, D=4096"
T_TOK, D, R, BITS, EPS = 16384, 4096, 32, 4, 1e-5
E2E_CHUNKS = 8
KERNEL_LOOP = 200  # isolated launches per kernel in the kernel-timing loop after the timed region
IN_STEP_MAX = 200  # steps with per-kernel events after the timed region
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 7700.0  # B200 HBM3e datasheet figure (HGX)
L2_BYTES = 126 * 10 ** 6
ARITHMETIC = ("bf16 I/O; alignment products on tcgen05 tensor cores as split-bf16 (hi/lo) operands with fp32 "
              "accumulation in TMEM; RMSNorm, absmax and quantiser in fp32 (sum of squares folded into fp64); "
              "Hadamard first stage as exact +-1 x bf16 tensor-core products, fp32 accumulate, fp32 butterflies")
CONTEXT = ("ReSpinQuant pages: ~0.2% online overhead of the alignment at r~32 relative to the base model's "
           "compute (hardware not stated for that figure; the end-to-end latency figures on the pages are "
           "from an H100)")


def algorithmic_bytes(T: int) -> dict:
    """Bytes each kernel must move per launch (the roofline numerators).

    align+norm+quant: read x (2 B/elem), write x_out (2 B/elem), write codes
    (D/2 B), write one fp32 scale per token; Q (D r fp32) and M (r^2 fp32)
    once per launch.  rht+quant: read x, write codes and scale; signs once."""
    per_tok_align = 2 * D * 2 + D * BITS // 8 + 4
    per_tok_rht = D * 2 + D * BITS // 8 + 4
    return {
        "align_norm_quant": T * per_tok_align + D * R * 4 + R * R * 4,
        "rht_quant": T * per_tok_rht + D,
        "per_token_align": per_tok_align,
        "per_token_rht": per_tok_rht,
    }


def workload_config(T: int, n: int) -> dict:
    b = algorithmic_bytes(T)
    ws = b["align_norm_quant"] + b["rht_quant"]
    return {
        "workload": f"hidden stream T={T}/GPU, D={D}, r={R}, bf16 I/O: residual align -> RMSNorm -> INT4, "
                    f"and randomised Hadamard 2^12 -> INT4",
        "T_per_gpu": T, "D": D, "r": R, "bits": BITS, "io_dtype": "bf16", "eps": EPS,
        "global_tokens": T * n, "parallelism": f"token-sharded replicas x{n}, no data-path collective",
        "l2": f"no flush: the bf16 input batch alone ({T * D * 2 / 1e6:.0f} MB) exceeds the {L2_BYTES / 1e6:.0f} MB L2; per-step traffic {ws / 1e6:.0f} MB",
    }


def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank value over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(tokens_per_rank: int, n_ranks: int, steps: int, elapsed_ms: float) -> float:
    """Tokens per second over the whole job: every rank processes its own shard
    of tokens_per_rank tokens per step; elapsed_ms is the max over ranks."""
    return tokens_per_rank * n_ranks * steps / (elapsed_ms / 1e3)


def shard_seed(rank: int) -> int:
    """Seed of this rank's token shard (Q, M and signs are shared by all ranks)."""
    return 1 + 1000 * rank


def peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d.get("bf16_tflops", 1590.0)),
                "source": "measured"}
    return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": 1590.0, "source": "fallback"}


def kernel_source_sha(files) -> str:
    """Hash of the kernel sources with comments and blank space removed, so a
    comment edit does not invalidate the recorded DRAM traffic but any change
    of code does."""
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), encoding="utf-8") as fh:
            src = fh.read()
        src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)   # block comments
        src = re.sub(r"//[^\n]*", " ", src)                  # line comments
        h.update(" ".join(src.split()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str):
    """dram bytes per launch from the committed ncu summary, if the kernel is unchanged."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f).get(kernel)
    if not rec:
        return None
    if rec.get("source_sha") != kernel_source_sha(rec.get("sources", [])):
        return None
    return rec.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.samples = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.index)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), [s.strip() for s in line.split(",")]))

    def stop(self, t0: float, t1: float) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=5)
        inside = [s for ts, s in self.samples if t0 <= ts <= t1]
        note = None
        if not inside:  # timed region shorter than the sampling period: nearest samples
            inside = [s for ts, s in sorted(self.samples, key=lambda p: min(abs(p[0] - t0), abs(p[0] - t1)))[:2]]
            note = "timed region shorter than the sampling period; nearest samples"
        sm, smax, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for s in inside:
            try:
                sm.append(float(s[1]))
                smax.append(float(s[2]))
                power.append(float(s[3]))
            except (ValueError, IndexError):
                continue
            for n, v in zip(names, s[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        out = {"sm_mhz": statistics.median(sm) if sm else None,
               "sm_max_mhz": max(smax) if smax else None,
               "reasons": sorted(reasons), "samples": len(sm),
               "power_w_max": max(power) if power else None}
        if note:
            out["note"] = note
        return out


def smi_id(dev) -> str:
    """nvidia-smi -i selector of a torch device (PCI bus id, robust to CUDA_VISIBLE_DEVICES)."""
    import torch
    p = torch.cuda.get_device_properties(dev)
    try:
        return f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
    except AttributeError:
        return str(dev.index)


def oracle_sample_rate(T_sample: int, threads: int, reps: int = 1) -> dict:
    """Time the float64 oracle (as it stands) on T_sample tokens of the workload,
    repeated reps times (inputs generated outside the timed region)."""
    import oracle
    from w3a3_quantization_online_b200 import inputs
    a, h = inputs.llama7b_case(T=T_sample)
    used = oracle.set_threads(threads)
    t0 = time.perf_counter()
    for _ in range(reps):
        oracle.align_norm_quant(a.x, a.Q, a.M, BITS, EPS, want_pre=False)
        oracle.rht_quant(h.x, h.signs, 1, BITS, want_pre=False)
    dt = time.perf_counter() - t0
    return {"seconds": dt, "tokens": T_sample * reps, "cores": used}


def cpu_baseline(target_s: float = 10.0) -> dict:
    """The oracle on the host cores: a sample of the workload sized to about
    target_s seconds (whole batches repeated once the sample reaches T tokens)."""
    cores = os.cpu_count() or 1
    oracle_sample_rate(max(8, cores), cores)  # thread pool start-up, page-in
    probe = oracle_sample_rate(min(T_TOK, 64 * cores), cores)
    per_tok = probe["seconds"] / probe["tokens"]
    T_s = int(max(cores, min(T_TOK, target_s / max(per_tok, 1e-9))))
    reps = 1
    if T_s == T_TOK:
        reps = max(1, int(round(target_s / max(per_tok * T_TOK, 1e-9))))
    r = oracle_sample_rate(T_s, cores, reps)
    # single-threaded: the same oracle on one core, a sample of about target_s / 2
    T_1 = int(max(8, min(T_TOK, (target_s / 2) / max(per_tok * r["cores"], 1e-9))))
    r1 = oracle_sample_rate(T_1, 1)
    return {"value": r["tokens"] / r["seconds"], "unit": "tokens/s", "cores": r["cores"], "kind": "oracle",
            "sample": f"{T_s} tokens of the same workload x {reps} pass(es) (both pipelines, float64 C "
                      f"oracle, OpenMP over tokens), {r['seconds']:.1f} s",
            "single_thread": {"value": r1["tokens"] / r1["seconds"], "unit": "tokens/s", "cores": r1["cores"],
                              "sample": f"{T_1} tokens of the same workload (both pipelines, float64 C oracle, "
                                        f"one thread), {r1['seconds']:.1f} s"}}


def run_reference(args) -> None:
    rank = int(os.environ.get("RANK", "0"))
    n = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    cores = os.cpu_count() or 1
    probe = oracle_sample_rate(max(8, cores), cores)
    per_tok = probe["seconds"] / probe["tokens"]
    budget = 120.0 / max(1, args.steps + args.warmup)
    tps = int(max(1, min(T_TOK, budget / max(per_tok, 1e-9))))
    import oracle
    from w3a3_quantization_online_b200 import inputs
    a, h = inputs.llama7b_case(T=tps)
    oracle.set_threads(cores)
    for _ in range(args.warmup):
        oracle.align_norm_quant(a.x, a.Q, a.M, BITS, EPS, want_pre=False)
        oracle.rht_quant(h.x, h.signs, 1, BITS, want_pre=False)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.align_norm_quant(a.x, a.Q, a.M, BITS, EPS, want_pre=False)
        oracle.rht_quant(h.x, h.signs, 1, BITS, want_pre=False)
    dt = time.perf_counter() - t0
    value = tps * args.steps / dt
    sample = f"{tps} tokens per step of the same workload (float64 C oracle, OpenMP over tokens)"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": n,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(T_TOK, n),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_gpu(args) -> None:
    import torch
    import torch.distributed as dist

    rank = int(os.environ.get("RANK", "0"))
    n = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if n != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={n}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if n > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    from w3a3_quantization_online_b200 import inputs, rsq

    T = args.tokens
    a = inputs.align_case(T, D, R, shard_seed(rank), dtype="bf16", bits=BITS, n_outliers=8,
                          outlier_scale=100.0, qm_seed=1)
    signs_np = inputs.random_signs(D, 1)
    x_host = torch.from_numpy(a.x).to(torch.bfloat16).pin_memory()
    x = x_host.to(dev)
    Q = torch.from_numpy(a.Q).to(dev)
    M = torch.from_numpy(a.M).to(dev)
    signs = torch.from_numpy(signs_np).to(dev)
    x_out = torch.empty_like(x)
    codes_a = torch.empty((T, D * BITS // 8), dtype=torch.uint8, device=dev)
    scales_a = torch.empty((T,), dtype=torch.float32, device=dev)
    codes_h = torch.empty_like(codes_a)
    scales_h = torch.empty_like(scales_a)
    stream = torch.cuda.Stream(device=dev)

    def step():
        rsq.rsq_align_norm_quant(x, Q, M, x_out, codes_a, scales_a, bits=BITS, eps=EPS, stream=stream)
        rsq.rht_quant(x, signs, 1, codes_h, scales_h, bits=BITS, stream=stream)

    def barrier():
        if n > 1:
            dist.barrier()

    # Clock samples cover the warm-up, the timed region and the kernel-timing
    # loop; the warm-up runs right before the timed region (no idle gap, so the
    # timed steps start at the clocks the warm-up brought up).
    sampler = ClockSampler(smi_id(dev))
    sampler.start()
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    torch.cuda.synchronize(dev)
    # nvidia-smi takes a moment to report its first sample: until it does (2 s at
    # most) the GPU keeps running untimed steps, so that the device is under load,
    # not idle, when the timed region starts and while the sampler comes up
    preroll, t_pre = 0, time.time()
    while not sampler.samples and sampler.proc is not None and time.time() - t_pre < 2.0:
        with torch.cuda.stream(stream):
            for _ in range(8):
                step()
        torch.cuda.synchronize(dev)
        preroll += 8

    # Timed region: exactly K steps back to back, as a user would call them
    # (each kernel may start early by programmatic dependent launch), between
    # one pair of CUDA events on the launching stream.
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    launches0 = rsq.launch_count()
    t_wall0 = time.time()
    with torch.cuda.stream(stream):
        e_start.record(stream)
        for k in range(args.steps):
            step()
        e_end.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    launches = rsq.launch_count() - launches0
    total_ms = e_start.elapsed_time(e_end)

    # Right after it, in the same clock window: the same steps with CUDA events
    # around each kernel, for per-kernel durations inside a step (an event
    # between the two kernels stops the second from starting early, so these
    # steps are not the timed ones).
    n_in = min(args.steps, IN_STEP_MAX)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n_in)]
    with torch.cuda.stream(stream):
        for k in range(n_in):
            ev[k][0].record(stream)
            rsq.rsq_align_norm_quant(x, Q, M, x_out, codes_a, scales_a, bits=BITS, eps=EPS, stream=stream)
            ev[k][1].record(stream)
            rsq.rht_quant(x, signs, 1, codes_h, scales_h, bits=BITS, stream=stream)
            ev[k][2].record(stream)
    torch.cuda.synchronize(dev)
    align_ms = [e[0].elapsed_time(e[1]) for e in ev]
    rht_ms = [e[1].elapsed_time(e[2]) for e in ev]

    # Kernel-timing loop right after the timed region: KERNEL_LOOP launches of
    # each kernel, each between its own pair of events (isolated launches, as
    # ncu times them), for a per-launch figure resting on many samples.
    def isolated(fn):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(KERNEL_LOOP)]
        with torch.cuda.stream(stream):
            for a0, a1 in evs:
                a0.record(stream)
                fn()
                a1.record(stream)
        torch.cuda.synchronize(dev)
        return [a0.elapsed_time(a1) for a0, a1 in evs]

    loop_ms = {
        "align_norm_quant": isolated(lambda: rsq.rsq_align_norm_quant(x, Q, M, x_out, codes_a, scales_a, bits=BITS,
                                                                      eps=EPS, stream=stream)),
        "rht_quant": isolated(lambda: rsq.rht_quant(x, signs, 1, codes_h, scales_h, bits=BITS, stream=stream)),
    }
    # Size-matched copy (context for the roofline, same clock window): a plain
    # device-to-device copy moving the same number of bytes (half read, half
    # written) as each kernel's algorithmic traffic, timed the same way.  At
    # these sizes a copy runs below the large-copy figure of the measured peak.
    ab0 = algorithmic_bytes(T)
    copy_ms = {}
    for name in ("align_norm_quant", "rht_quant"):
        half = (ab0[name] // 2) // 16 * 16
        c_src = torch.empty(half, dtype=torch.uint8, device=dev)
        c_dst = torch.empty(half, dtype=torch.uint8, device=dev)
        c_dst.copy_(c_src)
        copy_ms[name] = isolated(lambda: c_dst.copy_(c_src))
        del c_src, c_dst
    t_wall1 = time.time()
    clocks = sampler.stop(t_wall0, t_wall1)

    total_ms = max_over_ranks(total_ms, dev)
    ms_per_step = total_ms / args.steps
    value = whole_job_rate(T, n, args.steps, total_ms)

    # end to end through the C ABI with host buffers: pinned H2D of the batch,
    # both kernels, D2H of every output, all inside the timed region.  The batch
    # goes in E2E_CHUNKS row chunks on three streams (copy in, compute, copy
    # out), so the two PCIe directions and the kernels overlap; every byte of
    # every step still crosses PCIe inside the timed region.  The outputs of a
    # chunk (x_out rows, both code blocks, both scale blocks) sit next to each
    # other in one device buffer, so a chunk leaves in one copy.
    e2e_steps = max(3, min(args.steps, 20))
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    nch = E2E_CHUNKS
    rows = [(c * T // nch, (c + 1) * T // nch) for c in range(nch)]
    per_row = D * 2 + D * BITS // 8 + 4 + D * BITS // 8 + 4  # x_out, codes_a, scale_a, codes_h, scale_h
    obuf = torch.empty(T * per_row, dtype=torch.uint8, device=dev)
    obuf_h = torch.empty(T * per_row, dtype=torch.uint8).pin_memory()

    def chunk_outputs(r0, r1):
        n_r, base = r1 - r0, r0 * per_row
        parts, off = [], base
        for nbytes, dt, shape in ((n_r * D * 2, torch.bfloat16, (n_r, D)), (n_r * D * BITS // 8, torch.uint8, (n_r, D * BITS // 8)),
                                  (n_r * 4, torch.float32, (n_r,)), (n_r * D * BITS // 8, torch.uint8, (n_r, D * BITS // 8)),
                                  (n_r * 4, torch.float32, (n_r,))):
            parts.append(obuf[off:off + nbytes].view(dt).view(shape))
            off += nbytes
        return parts, base, off

    chunk_out = [chunk_outputs(r0, r1) for (r0, r1) in rows]
    ev_comp = [torch.cuda.Event() for _ in range(nch)]   # chunk's kernels done (x read, outputs written)
    ev_out = [torch.cuda.Event() for _ in range(nch)]    # chunk's outputs copied out
    ev_in = [torch.cuda.Event() for _ in range(nch)]     # chunk copied in
    started = [False]

    def e2e_step():
        for c, (r0, r1) in enumerate(rows):
            if started[0]:
                s_in.wait_event(ev_comp[c])  # the previous step's kernels have read x[c]
            with torch.cuda.stream(s_in):
                x[r0:r1].copy_(x_host[r0:r1], non_blocking=True)
                ev_in[c].record(s_in)
            stream.wait_event(ev_in[c])
            if started[0]:
                stream.wait_event(ev_out[c])  # the previous step's outputs of chunk c are out
            (xo_c, ca_c, sa_c, ch_c, sh_c), b0, b1 = chunk_out[c]
            rsq.rsq_align_norm_quant(x[r0:r1], Q, M, xo_c, ca_c, sa_c, bits=BITS, eps=EPS, stream=stream)
            rsq.rht_quant(x[r0:r1], signs, 1, ch_c, sh_c, bits=BITS, stream=stream)
            ev_comp[c].record(stream)
            s_out.wait_event(ev_comp[c])
            with torch.cuda.stream(s_out):
                obuf_h[b0:b1].copy_(obuf[b0:b1], non_blocking=True)
                ev_out[c].record(s_out)
        started[0] = True

    e2e_step()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    e0.record(s_in)
    for _ in range(e2e_steps):
        e2e_step()
    s_out.wait_event(ev_comp[-1])
    e1.record(s_out)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dev)
    e2e_value = whole_job_rate(T, n, e2e_steps, e2e_ms)
    h2d = x_host.numel() * 2
    d2h = obuf.numel()  # every chunk copies its whole output block
    assert d2h == x_out.numel() * 2 + codes_a.numel() + codes_h.numel() + 4 * (scales_a.numel() + scales_h.numel())

    if rank != 0:
        if n > 1:
            dist.destroy_process_group()
        return

    pk = peaks()
    ab = algorithmic_bytes(T)
    kern = {}
    for name, ms in (("align_norm_quant", align_ms), ("rht_quant", rht_ms)):
        lm = loop_ms[name]
        avg = statistics.mean(lm)
        gbs = ab[name] / (avg / 1e3) / 1e9
        in_step = statistics.mean(ms)
        kern[name] = {"avg_us": avg * 1e3, "median_us": statistics.median(lm) * 1e3, "min_us": min(lm) * 1e3,
                      "samples": len(lm), "achieved_gbs": gbs, "frac": gbs / pk["hbm_gbs"],
                      "frac_nominal": gbs / NOMINAL_HBM_GBS, "tokens_per_s": T / (avg / 1e3),
                      "in_step_avg_us": in_step * 1e3, "in_step_samples": len(ms),
                      "in_step_frac": ab[name] / (in_step / 1e3) / 1e9 / pk["hbm_gbs"],
                      "algorithmic_bytes_per_launch": ab[name]}
        cgbs = 2 * ((ab[name] // 2) // 16 * 16) / (statistics.mean(copy_ms[name]) / 1e3) / 1e9
        kern[name]["size_matched_copy_gbs"] = cgbs
        kern[name]["frac_of_size_matched_copy"] = gbs / cgbs
    dom = max(kern, key=lambda k: kern[k]["avg_us"])
    roof = {"bound": "hbm", "kernel": dom, "achieved": kern[dom]["achieved_gbs"], "peak": pk["hbm_gbs"],
            "unit": "GB/s", "frac": kern[dom]["frac"], "traffic": recorded_traffic(dom),
            "algorithmic_bytes_per_launch": ab[dom],
            "peak_source": f"{pk['source']} (STREAM-style copy, burst)",
            "frac_nominal": kern[dom]["frac_nominal"],
            "size_matched_copy": {"gbs": kern[dom]["size_matched_copy_gbs"],
                                  "frac": kern[dom]["frac_of_size_matched_copy"],
                                  "what": "device-to-device copy of the same byte count (half read, half written), "
                                          f"{KERNEL_LOOP} isolated launches; context, not the denominator"},
            "nominal_peak": {"value": NOMINAL_HBM_GBS, "unit": "GB/s", "source": "B200 HBM3e datasheet (HGX)"}}
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": n, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "arithmetic": ARITHMETIC,
        "data": "synthetic (seeded: N(0,1) activations with 8 outlier channels x100; random orthonormal Q, Cayley M, random signs)",
        "config": workload_config(T, n),
        "roofline": roof,
        "kernels": kern,
        "kernel_timing": f"avg_us: {KERNEL_LOOP} isolated launches of each kernel, each between its own pair "
                         "of CUDA events on the launching stream, right after the timed region (same clock "
                         "window); in_step_avg_us: CUDA events around each kernel of the steps that follow "
                         "the timed region (up to " + str(IN_STEP_MAX) + "; the timed steps themselves carry no "
                         "events between their kernels)",
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e2e_steps, "pipeline": f"{E2E_CHUNKS} row chunks on three streams: H2D, kernels, D2H"},
        "gpu_launches": launches,
        "clocks": clocks,
        "clock_preroll_steps": preroll,
        "context": CONTEXT,
    }
    if n == 1 and not args.no_secondary:
        line["secondary"] = secondary_metrics(dev, stream, pk)
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline()
    print(json.dumps(line), flush=True)
    if n > 1:
        dist.destroy_process_group()


def chain_metrics(dev, stream, T: int, steps: int, warmup: int, pk: dict) -> dict:
    """The 32-layer chain (config of the chain workload: D=4096, r=32, bf16,
    INT4, in place) at T rows, timed as one CUDA graph of the 32 layer calls."""
    import torch
    from w3a3_quantization_online_b200 import inputs, rsq
    x0, qs, ms, _, _ = inputs.chain_case(T=T)
    x = torch.from_numpy(x0).to(dev).to(torch.bfloat16)
    Qd = [torch.from_numpy(q).to(dev) for q in qs]
    Md = [torch.from_numpy(m).to(dev) for m in ms]
    codes = torch.empty((T, 2048), dtype=torch.uint8, device=dev)
    scales = torch.empty((T,), dtype=torch.float32, device=dev)
    L = len(qs)

    def chain():
        for i in range(L):
            rsq.rsq_align_norm_quant(x, Qd[i], Md[i], x, codes, scales, bits=4, stream=stream)

    with torch.cuda.stream(stream):
        chain()  # configure kernels outside capture
    torch.cuda.synchronize(dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        chain()
    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(steps):
            g.replay()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms_pass = e0.elapsed_time(e1) / steps
    per_layer_us = ms_pass * 1e3 / L
    bytes_layer = T * (2 * 4096 * 2 + 2048 + 4) + 4096 * 32 * 4 + 32 * 32 * 4
    gbs = bytes_layer / (per_layer_us * 1e-6) / 1e9
    del g
    return {"T": T, "layers": L, "us_per_layer": per_layer_us, "achieved_gbs": gbs, "frac": gbs / pk["hbm_gbs"],
            "tokens_per_s_per_layer": T / (per_layer_us * 1e-6), "passes": steps,
            "timing": "CUDA graph of the 32 in-place layer calls, CUDA events over the replays"}


def kernel_metrics(dev, stream, workload: str, steps: int, warmup: int, pk: dict) -> dict:
    """Back-to-back launches of each kernel of the W3A3 or down_proj workload."""
    import torch
    from w3a3_quantization_online_b200 import inputs, rsq
    if workload == "w3a3":
        a, h = inputs.w3a3_case(T=8192)
    elif workload == "downproj":
        a, h = None, inputs.down_proj_case(T=4096)
    else:
        raise SystemExit(f"unknown workload {workload}")
    res = {}
    if a is not None:
        x = torch.from_numpy(a.x).to(dev).to(torch.bfloat16)
        Q, M = torch.from_numpy(a.Q).to(dev), torch.from_numpy(a.M).to(dev)
        xo = torch.empty_like(x)
        c = torch.empty((a.T, a.D * a.bits // 8), dtype=torch.uint8, device=dev)
        sc = torch.empty((a.T,), dtype=torch.float32, device=dev)
        f = lambda: rsq.rsq_align_norm_quant(x, Q, M, xo, c, sc, bits=a.bits, stream=stream)
        byts = a.T * (2 * a.D * 2 + a.D * a.bits // 8 + 4) + a.D * a.r * 4
        res["align_norm_quant"] = (f, byts, a.T, f"T={a.T}, D={a.D}, r={a.r}, INT{a.bits}")
    xh = torch.from_numpy(h.x).to(dev).to(torch.bfloat16)
    sg = torch.from_numpy(h.signs).to(dev)
    ch = torch.empty((h.T, h.d * h.bits // 8), dtype=torch.uint8, device=dev)
    sh = torch.empty((h.T,), dtype=torch.float32, device=dev)
    fr = lambda: rsq.rht_quant(xh, sg, h.m, ch, sh, bits=h.bits, stream=stream)
    res["rht_quant"] = (fr, h.T * (h.d * 2 + h.d * h.bits // 8 + 4) + h.d, h.T,
                        f"T={h.T}, d={h.d} = {h.d // h.m}*{h.m}, INT{h.bits}")
    kern = {}
    for name, (f, byts, T, shape) in res.items():
        with torch.cuda.stream(stream):
            for _ in range(warmup):
                f()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        with torch.cuda.stream(stream):
            for _ in range(steps):
                f()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        us = e0.elapsed_time(e1) * 1e3 / steps
        kern[name] = {"shape": shape, "avg_us": us, "achieved_gbs": byts / (us * 1e-6) / 1e9,
                      "frac": byts / (us * 1e-6) / 1e9 / pk["hbm_gbs"], "tokens_per_s": T / (us * 1e-6),
                      "launches": steps, "timing": "back-to-back launches, CUDA events over the loop"}
    return kern


def _time_loop(stream, fn, steps: int, warmup: int) -> float:
    """Mean microseconds per call over `steps` back-to-back calls (CUDA events)."""
    import torch
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(steps):
            fn()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) * 1e3 / steps


def _hbm(byts: int, us: float, pk: dict, T: int, shape: str) -> dict:
    gbs = byts / (us * 1e-6) / 1e9
    return {"shape": shape, "avg_us": us, "bound": "hbm", "algorithmic_bytes_per_launch": byts, "achieved_gbs": gbs,
            "frac": gbs / pk["hbm_gbs"], "tokens_per_s": T / (us * 1e-6)}


def next_rows_metrics(dev, stream, pk: dict) -> dict:
    """The rows beyond the online path's core (each bounded to well under a
    second of GPU time): the SiLU-gated down_proj RHT, the attention-side
    Hadamards, the W4A4 GEMM and the offline (Q, M) construction."""
    import torch
    from w3a3_quantization_online_b200 import inputs, rsq
    out = {}
    # gated down_proj input, T = 4096, d = 12288: fused gate vs rht_quant of a stored product
    g = inputs.down_proj_gate_case(T=4096)
    a, b = (torch.from_numpy(v).to(dev).to(torch.bfloat16) for v in (g.a, g.b))
    sg = torch.from_numpy(g.signs).to(dev)
    ch = torch.empty((g.T, g.d // 2), dtype=torch.uint8, device=dev)
    sh = torch.empty((g.T,), dtype=torch.float32, device=dev)
    us = _time_loop(stream, lambda: rsq.rht_quant_silu_gate(a, b, sg, 12, ch, sh, bits=4, stream=stream), 50, 3)
    out["silu_gate_rht_quant"] = _hbm(g.T * (2 * g.d * 2 + g.d // 2 + 4) + g.d, us, pk, g.T,
                                      "T=4096, d=12288 = 1024*12, a and b bf16 in, INT4 out")
    del a, b, ch, sh
    # attention: 16384 tokens x 32 heads x 128
    c = inputs.attention_case(T=16384)
    x = torch.from_numpy(c.x).to(dev).to(torch.bfloat16)
    s = torch.from_numpy(c.signs).to(dev)
    xo = torch.empty_like(x)
    cq = torch.empty((c.T, c.d // 2), dtype=torch.uint8, device=dev)
    sq = torch.empty((c.T, 32), dtype=torch.float32, device=dev)
    st = torch.empty((c.T,), dtype=torch.float32, device=dev)
    us = _time_loop(stream, lambda: rsq.rht_heads(x, s, 32, xo, stream=stream), 50, 3)
    out["rht_heads"] = _hbm(c.T * c.d * 2 * 2 + c.d, us, pk, c.T, "T=16384, 32 heads x 128, bf16 in and out")
    us = _time_loop(stream, lambda: rsq.rht_heads_quant(x, s, 32, cq, sq, bits=4, stream=stream), 50, 3)
    out["rht_heads_quant"] = _hbm(c.T * (c.d * 2 + c.d // 2 + 32 * 4) + c.d, us, pk, c.T,
                                  "T=16384, 32 heads x 128, INT4 per (token, head)")
    us = _time_loop(stream, lambda: rsq.rht_head_mix_quant(x, s, 32, cq, st, bits=4, stream=stream), 50, 3)
    out["rht_head_mix_quant"] = _hbm(c.T * (c.d * 2 + c.d // 2 + 4) + c.d, us, pk, c.T,
                                     "T=16384, 32 heads x 128, INT4 per token")
    del x, xo, cq, sq, st
    # FlatQuant's Kronecker affine transform on the hidden stream: d = 4096 = 64 x 64, bf16, INT4
    f = inputs.flatquant_case()
    xf = torch.from_numpy(f.x).to(dev).to(torch.bfloat16)
    P1, P2 = torch.from_numpy(f.P1).to(dev), torch.from_numpy(f.P2).to(dev)
    cf = torch.empty((f.T, f.d // 2), dtype=torch.uint8, device=dev)
    sf = torch.empty((f.T,), dtype=torch.float32, device=dev)
    us = _time_loop(stream, lambda: rsq.kron_affine_quant(xf, P1, P2, cf, sf, bits=4, stream=stream), 20, 3)
    flops = 2.0 * f.T * f.d * (f.n1 + f.n2)
    peak64 = 148 * 64 * 2 * 1.965e9 / 1e12
    byts = f.T * (2 * f.d + f.d // 2 + 4) + 4 * (f.n1 * f.n1 + f.n2 * f.n2)
    out["kron_affine_quant"] = {"shape": "T=16384, d=4096 = 64 x 64, bf16 in, INT4 out, float64 products",
                                "avg_us": us, "bound": "alu", "algorithmic_fp64_flops": flops,
                                "achieved_tflops_fp64": flops / (us * 1e-6) / 1e12, "peak_tflops_fp64": peak64,
                                "frac": flops / (us * 1e-6) / 1e12 / peak64,
                                "achieved_gbs": byts / (us * 1e-6) / 1e9, "tokens_per_s": f.T / (us * 1e-6),
                                "peak_source": "148 SMs x 64 FP64 FMA/clock x 2 x 1.965 GHz (unit counts and max clock)"}
    del xf, cf, sf
    # W4A4 GEMM: the hidden stream through a 4096 x 4096 INT4 projection
    gm = inputs.gemm_case(16384, 4096, 4096, 21)
    ca, cw = torch.from_numpy(gm.codes_a).to(dev), torch.from_numpy(gm.codes_w).to(dev)
    sa, sw = torch.from_numpy(gm.scales_a).to(dev), torch.from_numpy(gm.scales_w).to(dev)
    y = torch.empty((gm.T, gm.N), dtype=torch.float16, device=dev)
    us = _time_loop(stream, lambda: rsq.w4a4_gemm(ca, sa, cw, sw, y=y, stream=stream), 20, 3)
    ops = 2.0 * gm.T * gm.N * gm.K
    peak_i8 = pk.get("bf16_tflops", 1590.0) * 2.0
    out["w4a4_gemm"] = {"shape": "T=16384, N=4096, K=4096, INT4 x INT4 -> fp16", "avg_us": us, "bound": "tensor",
                        "algorithmic_ops_per_launch": ops, "achieved_tops": ops / (us * 1e-6) / 1e12,
                        "peak_tops": peak_i8, "frac": ops / (us * 1e-6) / 1e12 / peak_i8,
                        "peak_source": "measured cuBLAS bf16 TFLOP/s (burst) x 2, the nominal int8 / bf16 dense ratio "
                                       "(4.5 / 2.25 PFLOP/s)"}
    # the same GEMM with the weights prepared once (int8), and the preparation itself
    w8 = torch.empty((gm.N, gm.K), dtype=torch.int8, device=dev)
    us_p = _time_loop(stream, lambda: rsq.w4a4_prepare_weights(cw, w8, stream=stream), 20, 3)
    us = _time_loop(stream, lambda: rsq.w4a4_gemm_s8w(ca, sa, w8, sw, y=y, stream=stream), 20, 3)
    out["w4a4_gemm_s8w"] = {"shape": "T=16384, N=4096, K=4096, INT4 activations x prepared int8 weights -> fp16",
                            "avg_us": us, "bound": "tensor", "algorithmic_ops_per_launch": ops,
                            "achieved_tops": ops / (us * 1e-6) / 1e12, "peak_tops": peak_i8,
                            "frac": ops / (us * 1e-6) / 1e12 / peak_i8,
                            "prepare_weights_us": us_p,
                            "note": "w4a4_prepare_weights runs once per weight matrix, not per call"}
    del ca, cw, y, w8
    # offline (Q, M) construction, D = 4096, r = 32
    R_in, R_out = inputs.near_hadamard_pair(4096, 77)
    Ri = torch.from_numpy(R_in.astype(np.float32)).to(dev)
    Ro = torch.from_numpy(R_out.astype(np.float32)).to(dev)
    ws = torch.empty(rsq.qm_workspace_bytes(4096, 32), dtype=torch.uint8, device=dev)
    iters = 16
    us = _time_loop(stream, lambda: rsq.qm_build(Ri, Ro, 32, iters=iters, workspace=ws, stream=stream), 3, 1)
    # float64 FMAs of the skinny products: per iteration and in the Ritz step 2 products with
    # each rotation (D^2 p each), plus the T_sub products (2 D^2 r)
    D, p_ = 4096, 64
    flops = 2.0 * (4 * iters + 2) * D * D * p_ + 2.0 * 2 * D * D * 32
    peak64 = 148 * 64 * 2 * 1.965e9 / 1e12
    out["qm_build"] = {"shape": "D=4096, r=32, 16 iterations", "avg_ms": us / 1e3, "bound": "alu",
                       "algorithmic_fp64_flops": flops, "achieved_tflops_fp64": flops / (us * 1e-6) / 1e12,
                       "peak_tflops_fp64": peak64, "frac": flops / (us * 1e-6) / 1e12 / peak64,
                       "peak_source": "148 SMs x 64 FP64 FMA/clock x 2 x 1.965 GHz (unit counts and max clock)"}
    torch.cuda.empty_cache()
    return out


def secondary_metrics(dev, stream, pk: dict) -> dict:
    """The other configurations, bounded to a few seconds of GPU time: W3A3
    (T=8192, D=8192, INT3: alignment and RHT 2^13), the down_proj RHT
    (T=4096, d=12288 Kronecker) and the 32-layer chain at T=16 and T=16384."""
    import torch
    out = {"w3a3": kernel_metrics(dev, stream, "w3a3", 100, 5, pk)}
    torch.cuda.empty_cache()
    out["downproj"] = kernel_metrics(dev, stream, "downproj", 100, 5, pk)
    torch.cuda.empty_cache()
    out["chain16"] = chain_metrics(dev, stream, 16, 50, 5, pk)
    out["chain16384"] = chain_metrics(dev, stream, 16384, 10, 3, pk)
    torch.cuda.empty_cache()
    out.update(next_rows_metrics(dev, stream, pk))
    return out


def run_secondary(args) -> None:
    """One secondary workload on its own line (rank 0, 1 GPU), with the
    requested steps: the 32-layer chain at decode (T=16) or prefill (T=16384)
    size, or the W3A3 / down_proj kernels."""
    import torch
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    pk = peaks()
    stream = torch.cuda.Stream(device=dev)
    out = {"workload": args.workload, "steps": args.steps, "warmup": args.warmup, "data": "synthetic"}
    if args.workload.startswith("chain"):
        T = 16 if args.workload == "chain16" else 16384
        out.update({"metric": "per-layer latency and HBM GB/s, 32-layer align+norm+INT4 chain, D=4096"})
        out.update(chain_metrics(dev, stream, T, args.steps, args.warmup, pk))
    else:
        out.update({"metric": "tokens/s and HBM GB/s per kernel",
                    "kernels": kernel_metrics(dev, stream, args.workload, args.steps, args.warmup, pk)})
    out["peak_gbs"] = pk["hbm_gbs"]
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["rsq", "reference"], default="rsq")
    ap.add_argument("--tokens", type=int, default=T_TOK, help="tokens per GPU (default 16384)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-secondary", action="store_true",
                    help="leave out the secondary workloads (W3A3, down_proj, 32-layer chain) of the headline line")
    ap.add_argument("--workload", default="hidden",
                    choices=["hidden", "chain16", "chain16384", "w3a3", "downproj"],
                    help="hidden = the headline step (default); the others print a secondary line")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    elif args.workload != "hidden":
        if int(os.environ.get("RANK", "0")) == 0:
            run_secondary(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
