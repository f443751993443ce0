#!/usr/bin/env python
"""Benchmark of jagged HSTU pointwise attention on B200.

One step = one training pass of one HSTU attention layer over the large jagged
workload (lognormal lengths, 256k tokens, d_model 1024 = 8 x 128, causal +
rab): forward (attention + LayerNorm(Y)*U) and full backward.  The metric is
useful TFLOP/s: 4*d per visible (i, j) pair and head for the forward, 8*d for
the backward (recomputation not counted).  M-FALCON candidates/s are measured
on the ranking workload (256 users x 2048 cached history, 1024 candidates,
b_m = 256) in the same run.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun each rank runs its own batch (weak scaling); the only
collective is the all-reduce of the rab / LayerNorm parameter gradients.
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

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from hstu_jagged_pointwise_b200 import workloads as W  # noqa: E402

METRIC = "jagged HSTU attn useful TFLOP/s fwd & fwd+bwd (% bf16 peak); M-FALCON cands/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "sm_max_mhz": 1965.0}


# ----------------------------------------------------------------------------
# workload accounting
# ----------------------------------------------------------------------------

def causal_pairs(lengths) -> int:
    L = np.asarray(lengths, dtype=np.int64)
    return int((L * (L + 1) // 2).sum())


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return FALLBACK_PEAKS, "fallback"


# DRAM bytes per launch measured by ncu (dram__bytes_read.sum + dram__bytes_write.sum)
# on the full-size workload, valid only while the kernel's sources are unchanged.
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dram_traffic.json")
KERNEL_SOURCES = {"attn_bwd_tc_kernel": "attn_bwd_tc.cu", "attn_fwd_tc_kernel": "attn_fwd_tc.cu"}
SHARED_SOURCES = ("ptx.cuh", "ew_bias.cuh", "hstu_rules.cuh", "internal.h")


def kernel_source_hash(name: str):
    import hashlib
    if name not in KERNEL_SOURCES:
        return None
    csrc = os.path.join(ROOT, "hstu_jagged_pointwise_b200", "csrc")
    h = hashlib.sha256()
    for f in (KERNEL_SOURCES[name],) + SHARED_SOURCES:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def measured_traffic(name: str, workload: str):
    """Bytes per launch from the committed ncu capture, or None when it does not
    describe this kernel source and workload."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    with open(TRAFFIC_FILE) as f:
        entry = json.load(f).get(name)
    if not entry or entry.get("workload") != workload:
        return None
    if entry.get("source_sha256") != kernel_source_hash(name):
        return None
    return int(entry["bytes_per_launch"])


def alu_fp32_peak_tflops(sm_mhz: float) -> float:
    # 148 SMs x 128 FP32 lanes x 2 FLOP (FFMA) per clock
    return 148 * 128 * 2 * sm_mhz * 1e6 / 1e12


# ----------------------------------------------------------------------------
# clocks during the timed region
# ----------------------------------------------------------------------------

class NvmlClockSampler:
    """SM clock and clock-event reasons every 10 ms through NVML (read-only queries)."""
    PERIOD_S = 0.01

    def __init__(self, device_index: int):
        import pynvml
        self.nv = pynvml
        pynvml.nvmlInit()
        props = torch.cuda.get_device_properties(device_index)
        bus = "%08X:%02X:%02X.0" % (getattr(props, "pci_domain_id", 0), props.pci_bus_id, props.pci_device_id)
        self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM))
        self.get_reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
        self.bits = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
                     "hw_thermal_slowdown": 0x40}
        self.samples, self.reasons = [], set()
        self.stop_flag = threading.Event()

    def _run(self):
        while not self.stop_flag.is_set():
            try:
                self.samples.append(float(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)))
                r = int(self.get_reasons(self.h))
                for name, bit in self.bits.items():
                    if r & bit:
                        self.reasons.add(name)
            except self.nv.NVMLError:
                pass
            time.sleep(self.PERIOD_S)

    def start(self):
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()

    def stop(self) -> dict:
        self.stop_flag.set()
        self.thread.join(timeout=2)
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples), "source": "nvml"}


def make_clock_sampler(device_index: int):
    try:
        return NvmlClockSampler(device_index)
    except Exception:
        return ClockSampler(device_index)


class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------
# distributed plumbing
# ----------------------------------------------------------------------------

def dist_init(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------------------
# CPU baseline (the fp64 oracle, as it stands)
# ----------------------------------------------------------------------------

def sub_workload(w, seqs):
    lens = [int(w.offsets[b + 1] - w.offsets[b]) for b in seqs]
    rows = np.concatenate([np.arange(w.offsets[b], w.offsets[b + 1]) for b in seqs])
    ts_list = [w.ts[w.offsets[b]:w.offsets[b + 1]] for b in seqs]
    s = W.make_causal(lens, H=w.H, d=w.d, dtype=w.dtype, seed=0, alpha=w.alpha, ts_list=ts_list,
                      with_grad=True)
    rt = torch.as_tensor(rows)
    for name in ("q", "k", "v", "u", "grad"):
        setattr(s, name, getattr(w, name)[rt])
    s.rab_pos, s.rab_time, s.gamma, s.beta = w.rab_pos, w.rab_time, w.gamma, w.beta
    return s


def oracle_sample(w, target_s: float = 12.0):
    """Bounded sample of the workload for the oracle: whole sequences (shortest first)
    whose estimated oracle time is about target_s seconds."""
    import oracle
    L = w.lengths
    order = np.argsort(L)
    def pick(rate, budget_s):
        seqs, flops = [], 0.0
        for b in order:
            f = 12 * w.d * w.H * causal_pairs([L[b]])
            if seqs and (flops + f) / rate > budget_s:
                break
            seqs.append(int(b))
            flops += f
        return seqs, flops

    def measure(seqs, flops):
        t0 = time.perf_counter()
        oracle.layer_bwd(sub_workload(w, seqs))
        return flops / max(time.perf_counter() - t0, 1e-3)

    # calibrate on the shortest sequence, then on about one and three seconds of work (short
    # sequences alone under-use the host threads, which would make the sample too small)
    rate = measure([int(order[0])], 12 * w.d * w.H * causal_pairs([L[order[0]]]))
    rate = measure(*pick(rate, 1.0))
    rate = measure(*pick(rate, 3.0))
    seqs, _ = pick(rate, target_s)
    return sub_workload(w, seqs), seqs


def time_oracle(sample):
    import oracle
    t0 = time.perf_counter()
    oracle.layer_bwd(sample)
    dt = time.perf_counter() - t0
    useful = 12 * sample.d * sample.H * causal_pairs(sample.lengths)
    return useful / dt / 1e12, dt, oracle.num_threads()


# ----------------------------------------------------------------------------
# our arm
# ----------------------------------------------------------------------------

def rank_workload(args, world, rank):
    """This rank's batch.  One GPU: the large layer (lognormal lengths summing to
    args.tokens).  N GPUs (weak scaling): one global batch of N * args.tokens tokens whose
    sequences are split across the ranks by shard.rank_sequences (whole sequences,
    balanced on sum(L^2)); each rank draws the dense tensors of its own sequences."""
    if world == 1:
        return W.large_layer(seed=args.seed, total=args.tokens)
    from hstu_jagged_pointwise_b200 import shard
    rng = np.random.Generator(np.random.PCG64(args.seed))
    lengths = W.lognormal_lengths(rng, args.tokens * world)
    mine = lengths[shard.rank_sequences(lengths, world, rank)]
    return W.make_causal(mine, H=8, d=128, dtype=torch.bfloat16, seed=args.seed + 404 + rank, with_grad=True,
                         alpha=float(lengths.max()), name=f"large_layer_T{args.tokens}_H8_d128")


def sum_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda")
    dist.all_reduce(t)
    return float(t.item())


def run_ours(args, world, rank, local):
    from hstu_jagged_pointwise_b200 import capi, ops, shard

    w = rank_workload(args, world, rank)
    dev = torch.device("cuda", local)
    H, d = w.H, w.d
    P_head = causal_pairs(w.lengths)
    P = P_head * H
    f_fwd, f_bwd = 4 * d * P, 8 * d * P
    host = {n: getattr(w, n).contiguous() for n in ("q", "k", "v", "u", "grad")}
    dv = {n: t.to(dev) for n, t in host.items()}
    off = torch.as_tensor(w.offsets).to(dev)
    ts = torch.as_tensor(w.ts).to(dev)
    rp, rt, g, b = (t.to(dev) for t in (w.rab_pos, w.rab_time, w.gamma, w.beta))
    layer = ops.Layer(off, ts, H, d, torch.bfloat16, w.alpha, w.max_len)
    fwd_out = dict(y=torch.empty_like(dv["q"]), o_pre=torch.empty_like(dv["q"]),
                   mean=torch.empty(w.T, dtype=torch.float32, device=dev),
                   rstd=torch.empty(w.T, dtype=torch.float32, device=dev))
    bwd_out = dict(dq=torch.empty_like(dv["q"]), dk=torch.empty_like(dv["k"]), dv=torch.empty_like(dv["v"]),
                   du=torch.empty_like(dv["u"]), d_rab_pos=torch.empty_like(rp), d_rab_time=torch.empty_like(rt),
                   d_gamma=torch.empty_like(g), d_beta=torch.empty_like(b))

    def step():
        layer.forward(dv["q"], dv["k"], dv["v"], dv["u"], rp, rt, g, b, out=fwd_out)
        layer.backward(dv["q"], dv["k"], dv["v"], dv["u"], rp, rt, g, b, fwd_out, dv["grad"], out=bwd_out)
        if world > 1:
            # the only exchange: data-parallel sum of the parameter gradients
            shard.allreduce_param_grads(bwd_out)

    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st = layer.check_device_error()
    if st != 0:
        raise RuntimeError(f"device status {capi.status_string(st)} after warm-up")

    # ---- device-timed region
    sampler = make_clock_sampler(local)
    capi.profile_enable(True)
    barrier(world)
    torch.cuda.synchronize()
    sampler.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clocks = sampler.stop()
    ms = e0.elapsed_time(e1) / args.steps
    kernels = capi.profile_read()
    capi.profile_enable(False)
    ms_max = max_over_ranks(ms, world)
    if layer.check_device_error() != 0:
        raise RuntimeError("device status set during the timed region")

    # forward alone (same stream, same inputs)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(args.steps):
        layer.forward(dv["q"], dv["k"], dv["v"], dv["u"], rp, rt, g, b, out=fwd_out)
    e1.record(stream)
    torch.cuda.synchronize()
    ms_fwd = max_over_ranks(e0.elapsed_time(e1) / args.steps, world)

    # Group LayerNorm variant of the same layer (LayerNorm kernels only differ)
    extra = {}
    if not args.no_gln:
        extra["gln"] = run_gln(args, world, w, dv, off, ts, rp, rt, fwd_out, bwd_out)
    if not args.no_proj:
        extra["projections"] = run_proj(args, world, rank)
    if not args.no_data:
        extra["data_step"] = run_data_step(args, world, rank, w)
    if not args.no_layer:
        extra["full_layer"] = run_full_layer(args, world, w, f_fwd + f_bwd)
    if not args.no_configs:
        extra["training_sl"] = run_training_sl(args, world, rank)
        extra["mtgr_medium"] = run_mtgr_medium(args, world, rank)

    # ---- end to end through the C ABI with host buffers
    if args.no_e2e:
        mf = None if args.no_mfalcon else run_mfalcon(args, world, rank, local)
        return finish(args, world, w, kernels, ms, ms_max, ms_fwd, None, None, None, mf, clocks, f_fwd, f_bwd, P, d,
                      extra)
    # Pipelined over three streams: the host->device copies of step k+1 and the
    # device->host copies of step k-1 run while step k computes (PCIe carries both
    # directions at once), on double-buffered device inputs and outputs.  Every copy is
    # one cudaMemcpyAsync from or to pinned host memory.
    small_names = (("rp", w.rab_pos), ("rt", w.rab_time), ("g", w.gamma), ("b", w.beta))
    pin = {n: t.pin_memory() for n, t in host.items()}
    pin.update({n: t.pin_memory() for n, t in small_names})
    pin["off"] = torch.as_tensor(w.offsets).pin_memory()
    pin["ts"] = torch.as_tensor(w.ts).pin_memory()
    out_names = list(bwd_out) + ["o_pre"]
    outs_h = [{n: torch.empty(bwd_out[n].shape if n in bwd_out else fwd_out[n].shape,
                              dtype=(bwd_out[n] if n in bwd_out else fwd_out[n]).dtype, pin_memory=True)
               for n in out_names} for _ in range(2)]
    dev_in = [dict(q=dv["q"], k=dv["k"], v=dv["v"], u=dv["u"], grad=dv["grad"], rp=rp, rt=rt, g=g, b=b, off=off,
                   ts=ts)]
    dev_in.append({n: torch.empty_like(t) for n, t in dev_in[0].items()})
    dev_fo = [fwd_out, {n: torch.empty_like(t) for n, t in fwd_out.items()}]
    dev_bo = [bwd_out, {n: torch.empty_like(t) for n, t in bwd_out.items()}]
    layers = [layer, ops.Layer(dev_in[1]["off"], dev_in[1]["ts"], H, d, torch.bfloat16, w.alpha, w.max_len)]
    h2d = sum(t.numel() * t.element_size() for t in pin.values())
    d2h = sum(t.numel() * t.element_size() for t in outs_h[0].values())
    s_h2d, s_d2h = torch.cuda.Stream(), torch.cuda.Stream()

    def run_pipeline(n_steps):
        """n_steps end-to-end steps: inputs from pinned host memory, outputs back to it."""
        in_ready = [torch.cuda.Event() for _ in range(n_steps)]
        done = [torch.cuda.Event() for _ in range(n_steps)]
        out_free = [torch.cuda.Event() for _ in range(n_steps)]

        def upload(k):
            with torch.cuda.stream(s_h2d):
                if k >= 2:
                    s_h2d.wait_event(done[k - 2])          # buffer k % 2 was read by step k - 2
                for n, t in pin.items():
                    dev_in[k % 2][n].copy_(t, non_blocking=True)
                in_ready[k].record(s_h2d)

        upload(0)
        for k in range(n_steps):
            if k + 1 < n_steps:
                upload(k + 1)
            stream.wait_event(in_ready[k])
            if k >= 2:
                stream.wait_event(out_free[k - 2])         # outputs k % 2 read back by step k - 2
            x, fo, bo, ly = dev_in[k % 2], dev_fo[k % 2], dev_bo[k % 2], layers[k % 2]
            ly.forward(x["q"], x["k"], x["v"], x["u"], x["rp"], x["rt"], x["g"], x["b"], out=fo)
            ly.backward(x["q"], x["k"], x["v"], x["u"], x["rp"], x["rt"], x["g"], x["b"], fo, x["grad"], out=bo)
            if world > 1:
                shard.allreduce_param_grads(bo)
            done[k].record(stream)
            with torch.cuda.stream(s_d2h):
                s_d2h.wait_event(done[k])
                for n, t in outs_h[k % 2].items():
                    t.copy_(fo[n] if n == "o_pre" else bo[n], non_blocking=True)
                out_free[k].record(s_d2h)
        stream.wait_stream(s_d2h)
        stream.wait_stream(s_h2d)

    run_pipeline(2)
    torch.cuda.synchronize()
    n_e2e = max(2, min(args.steps, 8))
    barrier(world)
    torch.cuda.synchronize()
    e0.record(stream)
    run_pipeline(n_e2e)
    e1.record(stream)
    torch.cuda.synchronize()
    for ly in layers:
        if ly.check_device_error() != 0:
            raise RuntimeError("device status set in the end-to-end leg")
    ms_e2e = max_over_ranks(e0.elapsed_time(e1) / n_e2e, world)

    # ---- M-FALCON candidates / s
    mf = None
    if not args.no_mfalcon:
        del pin, outs_h
        mf = run_mfalcon(args, world, rank, local)
    return finish(args, world, w, kernels, ms, ms_max, ms_fwd, ms_e2e, h2d, d2h, mf, clocks, f_fwd, f_bwd, P, d,
                  extra)


def run_proj(args, world, rank):
    """f1 (X -> U, V, Q, K with SiLU) and f2 of the large layer (262,144 tokens, d_model 1024),
    forward and backward, on the library's tcgen05 GEMM; the same products through
    torch.matmul (cuBLAS) are timed beside it for reference."""
    from hstu_jagged_pointwise_b200 import capi, ops
    dev = f"cuda:{torch.cuda.current_device()}"
    if args.tokens == 262144:
        w = W.projection_large(seed=args.seed + rank, device=dev)
    else:
        w = W.make_projection(args.tokens, 1024, 1024, 1024, seed=args.seed + rank, device=dev,
                              name=f"proj_T{args.tokens}_d1024")
    T, d_in, D, d_out = w.T, w.d_in, w.D, w.d_out
    blocks = [w.dact[:, i * D:(i + 1) * D].contiguous() for i in range(4)]
    outs = {}

    def step():
        outs["f1"] = ops.f1_fwd(w.x, w.w1, w.b1, D, out=outs.get("f1"))
        outs["f2"] = ops.f2_fwd(w.o_pre, w.w2, w.b2, residual=w.x, out=outs.get("f2"))
        outs["b1"] = ops.f1_bwd(w.x, w.w1, w.z, *blocks, out=outs.get("b1"))
        outs["b2"] = ops.f2_bwd(w.o_pre, w.w2, w.g_out, out=outs.get("b2"))

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    barrier(world)
    s = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    capi.profile_enable(True)
    e0.record(s)
    for _ in range(args.steps):
        step()
    e1.record(s)
    torch.cuda.synchronize()
    prof = capi.profile_read()
    capi.profile_enable(False)
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world)
    for o in outs.values():
        if int(o["status"].item()) != 0:
            raise RuntimeError("device status set in the projections")
    flops = 2 * T * (d_in * 4 * D + D * d_out) * 3            # forward + two backward products each
    n_g, t_g = prof["gemm_tc_kernel"]
    pk, _ = peaks()
    gemm_tf = flops / (t_g / args.steps * 1e-3) / 1e12

    # the same eight products through cuBLAS (torch.matmul), timed alone
    z4 = torch.empty(T, 4 * D, dtype=torch.bfloat16, device=w.x.device)
    dzb = torch.empty_like(z4)

    def lib_step():
        torch.matmul(w.x, w.w1.t(), out=z4)
        torch.matmul(w.o_pre, w.w2.t())
        torch.matmul(dzb, w.w1)
        torch.matmul(dzb.t(), w.x)
        torch.matmul(w.g_out, w.w2)
        torch.matmul(w.g_out.t(), w.o_pre)

    for _ in range(args.warmup):
        lib_step()
    torch.cuda.synchronize()
    e0.record(s)
    for _ in range(args.steps):
        lib_step()
    e1.record(s)
    torch.cuda.synchronize()
    ms_lib = e0.elapsed_time(e1) / args.steps
    return {"workload": w.name, "ms_per_step": round(ms, 4), "gemm_launches_per_step": n_g // args.steps,
            "gemm_ms_per_step": round(t_g / args.steps, 4), "gemm_tflops": round(gemm_tf, 1),
            "frac_bf16_sustained": round(gemm_tf / pk["bf16_tflops_sustained"], 4),
            "frac_bf16_burst": round(gemm_tf / pk["bf16_tflops"], 4),
            "other_kernels_ms_per_step": {k: round(v[1] / args.steps, 4) for k, v in prof.items()
                                          if k != "gemm_tc_kernel"},
            "cublas_same_products_ms": round(ms_lib, 4),
            "cublas_tflops": round(flops / (ms_lib * 1e-3) / 1e12, 1)}


def run_full_layer(args, world, w, attn_flops):
    """The whole layer on the same batch (d_model 1024): f1 -> attention -> Norm * U -> f2 + X,
    forward and backward, through ops.HSTULayer."""
    from hstu_jagged_pointwise_b200 import capi, ops
    dev = torch.device("cuda", torch.cuda.current_device())
    gen = torch.Generator(device=dev).manual_seed(args.seed + 55)
    dm, D = 1024, w.D
    x = torch.randn(w.T, dm, generator=gen, device=dev).to(torch.bfloat16)
    g_out = torch.randn(w.T, dm, generator=gen, device=dev).to(torch.bfloat16)
    prm = dict(w1=(torch.randn(4 * D, dm, generator=gen, device=dev) * dm ** -0.5).to(torch.bfloat16),
               b1=0.1 * torch.randn(4 * D, generator=gen, device=dev),
               w2=(torch.randn(dm, D, generator=gen, device=dev) * D ** -0.5).to(torch.bfloat16),
               b2=0.1 * torch.randn(dm, generator=gen, device=dev),
               rab_pos=w.rab_pos.to(dev), rab_time=w.rab_time.to(dev), ln_gamma=w.gamma.to(dev),
               ln_beta=w.beta.to(dev))
    layer = ops.HSTULayer(torch.as_tensor(w.offsets).to(dev), torch.as_tensor(w.ts).to(dev), dm, w.H, w.d,
                          w.alpha, w.max_len)

    def step():
        f = layer.forward(x, prm)
        layer.backward(f, g_out, prm)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    barrier(world)
    s = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    capi.profile_enable(True)
    e0.record(s)
    for _ in range(args.steps):
        step()
    e1.record(s)
    torch.cuda.synchronize()
    prof = capi.profile_read()
    capi.profile_enable(False)
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world)
    if layer.check_device_error() != 0:
        raise RuntimeError("device status set in the full layer")
    proj_flops = 3 * 2 * w.T * (dm * 4 * D + D * dm)
    flops = attn_flops + proj_flops
    pk, _ = peaks()
    tf = world * flops / (ms * 1e-3) / 1e12
    return {"workload": f"{w.name}_dmodel{dm}", "ms_per_step": round(ms, 4), "tflops": round(tf, 1),
            "pct_bf16_sustained": round(tf / world / pk["bf16_tflops_sustained"], 4),
            "kernel_ms_per_step": {k: round(v[1] / args.steps, 4) for k, v in sorted(prof.items(),
                                                                                      key=lambda kv: -kv[1][1])}}


def mtgr_pairs(w) -> int:
    """Visible (i, j) pairs of one head under the MTGR dynamic mixed mask (MTGR deep-dive
    section 2): static rows see the S static tokens; real-time row i sees S + (its index
    among the real-time tokens + 1); a candidate sees itself and the non-candidates with
    a strictly smaller timestamp."""
    off = np.asarray(w.offsets, np.int64)
    total = 0
    for b in range(len(off) - 1):
        L = int(off[b + 1] - off[b])
        S, R = int(w.n_static[b]), int(w.n_realtime[b])
        total += S * S + R * S + R * (R + 1) // 2
        ts = np.asarray(w.ts[off[b]:off[b + 1]], np.int64)
        hist = np.sort(ts[:S + R])
        total += int(np.searchsorted(hist, ts[S + R:], side="left").sum()) + (L - S - R)
    return total


def _timed(args, world, fn):
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    barrier(world)
    s = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    from hstu_jagged_pointwise_b200 import capi
    capi.profile_enable(True)
    e0.record(s)
    for _ in range(args.steps):
        fn()
    e1.record(s)
    torch.cuda.synchronize()
    prof = capi.profile_read()
    capi.profile_enable(False)
    return max_over_ranks(e0.elapsed_time(e1) / args.steps, world), prof


def _attn_leg(args, world, w, backward: bool, pairs_per_head: int):
    """One attention layer of workload w (forward, or forward + backward) timed on its own,
    with the useful TFLOP/s of the step and of the attention kernels."""
    from hstu_jagged_pointwise_b200 import ops
    dev = torch.device("cuda", torch.cuda.current_device())
    t = {n: getattr(w, n).to(dev) for n in ("q", "k", "v", "u", "rab_pos", "rab_time", "gamma", "beta")}
    if backward:
        t["grad"] = w.grad.to(dev)
    d = {n: torch.as_tensor(np.asarray(getattr(w, n), np.int32)).to(dev)
         for n in ("offsets", "n_static", "n_realtime") if getattr(w, n) is not None}
    layer = ops.Layer(d["offsets"], torch.as_tensor(w.ts).to(dev), w.H, w.d, w.dtype, w.alpha, w.max_len,
                      mask_kind=w.kind, n_static=d.get("n_static"), n_realtime=d.get("n_realtime"))
    fo = dict(y=torch.empty_like(t["q"]), o_pre=torch.empty_like(t["q"]),
              mean=torch.empty(w.T, dtype=torch.float32, device=dev),
              rstd=torch.empty(w.T, dtype=torch.float32, device=dev))
    bo = None
    if backward:
        bo = dict(dq=torch.empty_like(t["q"]), dk=torch.empty_like(t["k"]), dv=torch.empty_like(t["v"]),
                  du=torch.empty_like(t["u"]), d_rab_pos=torch.empty_like(t["rab_pos"]),
                  d_rab_time=torch.empty_like(t["rab_time"]), d_gamma=torch.empty_like(t["gamma"]),
                  d_beta=torch.empty_like(t["beta"]))

    def fwd():
        layer.forward(t["q"], t["k"], t["v"], t["u"], t["rab_pos"], t["rab_time"], t["gamma"], t["beta"], out=fo)

    def step():
        fwd()
        if backward:
            layer.backward(t["q"], t["k"], t["v"], t["u"], t["rab_pos"], t["rab_time"], t["gamma"], t["beta"], fo,
                           t["grad"], out=bo)

    ms, prof = _timed(args, world, step)
    if layer.check_device_error() != 0:
        raise RuntimeError(f"device status set in {w.name}")
    pk, _ = peaks()
    P = pairs_per_head * w.H
    f_fwd, f_bwd = 4 * w.d * P, 8 * w.d * P
    out = {"workload": w.name, "tokens": int(w.T), "sequences": int(w.B), "max_seq_len": int(w.max_len),
           "alpha": w.alpha, "visible_pairs": int(P), "ms_per_step": round(ms, 4)}
    flops = f_fwd + (f_bwd if backward else 0)
    tf = world * flops / (ms * 1e-3) / 1e12
    out["tflops_step"] = round(tf, 2)
    out["pct_bf16_sustained_step"] = round(tf / world / pk["bf16_tflops_sustained"], 4)
    for name, units in (("attn_fwd_tc_kernel", f_fwd), ("attn_bwd_tc_kernel", f_bwd)):
        if name in prof:
            n, tot = prof[name]
            kt = units / (tot / n * 1e-3) / 1e12
            out[name] = {"ms_per_launch": round(tot / n, 4), "tflops": round(kt, 2),
                         "frac_bf16_burst": round(kt / pk["bf16_tflops"], 4),
                         "frac_bf16_sustained": round(kt / pk["bf16_tflops_sustained"], 4)}
    return out


def run_training_sl(args, world, rank):
    """The training shape (64 Zipf(1.2) sequences in [16, 4096], Stochastic Length at
    alpha 1.6, cap 776; 4 heads x 128; causal + rab): forward and backward."""
    w = W.training_sl(seed=args.seed + rank)
    return _attn_leg(args, world, w, True, causal_pairs(w.lengths))


def run_mtgr_medium(args, world, rank):
    """MTGR-Medium-style users (128 rows of 24 profile + U[200, 3000] behaviour + 0-64
    real-time + 20-200 candidates; 6 heads x 128) under the dynamic mixed mask: forward."""
    w = W.mtgr_medium(seed=args.seed + rank)
    return _attn_leg(args, world, w, False, mtgr_pairs(w))


def run_data_step(args, world, rank, w):
    """The data step on the large layer's raw batch: Stochastic Length (cap 776 = 4096^0.8),
    the gathers of the kept rows (d_model 1024 bf16 features and int64 timestamps), and the
    token-balanced split into 8 bins."""
    from hstu_jagged_pointwise_b200 import capi, ops
    dev = torch.device("cuda", torch.cuda.current_device())
    off = torch.as_tensor(w.offsets).to(dev)
    gen = torch.Generator(device=dev).manual_seed(args.seed + 91)
    feats = torch.randn(w.T, 1024, generator=gen, device=dev).to(torch.bfloat16)
    ts = torch.as_tensor(w.ts).to(dev)
    cap = W.stochastic_length_cap(4096, 1.6)
    n_out = int(np.minimum(np.diff(w.offsets), cap).sum())   # the sampled size does not depend on the seed
    state = {}

    def step(i):
        o = ops.sl_sample(off, cap, seed=args.seed + i, out_capacity=w.T)
        n = n_out
        state["f"] = ops.gather_rows(feats, o["gather"], n, out=state.get("f"))
        state["t"] = ops.gather_rows(ts, o["gather"], n, out=state.get("t"))
        state["p"] = ops.pack_balanced(o["offsets"], 8)
        state["o"] = o

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    if int(state["o"]["offsets"][-1].item()) != n_out:
        raise RuntimeError("sampled size differs from the sum of min(L, cap)")
    s = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    capi.profile_enable(True)
    e0.record(s)
    for i in range(args.steps):
        step(i)
    e1.record(s)
    torch.cuda.synchronize()
    prof = capi.profile_read()
    capi.profile_enable(False)
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world)
    if int(state["o"]["status"].item()) != 0:
        raise RuntimeError("device status set by the Stochastic Length sampler")
    n_g, t_g = prof["gather_rows_kernel"]
    gbytes = n_out * (2 * (1024 * 2 + 8) + 2 * 4)            # rows read and written, the index read twice
    pk, _ = peaks()
    return {"workload": f"{w.name}_raw", "sl_cap": cap, "tokens_in": w.T, "tokens_out": n_out,
            "ms_per_step": round(ms, 4), "sl_sample_ms": round(prof["sl_sample_kernels"][1] / args.steps, 4),
            "gather_ms": round(t_g / args.steps, 4),
            "gather_gbs": round(gbytes / (t_g / args.steps * 1e-3) / 1e9, 1),
            "gather_frac_hbm": round(gbytes / (t_g / args.steps * 1e-3) / 1e9 / pk["hbm_gbs"], 4)}


def run_gln(args, world, w, dv, off, ts, rp, rt, fwd_out, bwd_out):
    """The layer with Group LayerNorm (4 groups, seeded random token ids, one gamma/beta row
    per group): forward + backward steps timed, and the LayerNorm kernels' HBM rates."""
    from hstu_jagged_pointwise_b200 import capi, ops
    G = 4
    dev = dv["q"].device
    gen = torch.Generator().manual_seed(args.seed + 77)
    tg = torch.randint(0, G, (w.T,), generator=gen, dtype=torch.uint8).to(dev)
    g = (1 + 0.1 * torch.randn(G, w.D, generator=gen)).to(dev)
    b = (0.1 * torch.randn(G, w.D, generator=gen)).to(dev)
    layer = ops.Layer(off, ts, w.H, w.d, torch.bfloat16, w.alpha, w.max_len, n_groups=G, token_group=tg)
    bo = dict(bwd_out, d_gamma=torch.empty_like(g), d_beta=torch.empty_like(b))

    def step():
        layer.forward(dv["q"], dv["k"], dv["v"], dv["u"], rp, rt, g, b, out=fwd_out)
        layer.backward(dv["q"], dv["k"], dv["v"], dv["u"], rp, rt, g, b, fwd_out, dv["grad"], out=bo)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    barrier(world)
    s = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    capi.profile_enable(True)
    e0.record(s)
    for _ in range(args.steps):
        step()
    e1.record(s)
    torch.cuda.synchronize()
    prof = capi.profile_read()
    capi.profile_enable(False)
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world)
    if layer.check_device_error() != 0:
        raise RuntimeError("device status set in the Group LayerNorm step")
    pk, _ = peaks()
    out = {"groups": G, "token_groups": "uniform random", "ms_per_step": round(ms, 4)}
    for name, nbytes in (("ln_fwd_kernel", (6 * w.D + 9) * w.T), ("ln_bwd_kernel", (10 * w.D + 9) * w.T)):
        n, t = prof[name]
        gbs = nbytes / (t / n * 1e-3) / 1e9
        out[name] = {"ms_per_launch": round(t / n, 4), "gbs": round(gbs, 1), "frac_hbm": round(gbs / pk["hbm_gbs"], 4)}
    return out


def finish(args, world, w, kernels, ms, ms_max, ms_fwd, ms_e2e, h2d, d2h, mf, clocks, f_fwd, f_bwd, P, d,
           extra=None):
    H = w.H
    # ---- roofline of the dominant kernel
    pk, pk_src = peaks()
    sm_mhz = pk.get("sm_max_mhz", 1965.0)
    kinfo = {}
    algo = {
        "attn_fwd_tc_kernel": ("tensor", f_fwd, "TFLOP/s"),
        "attn_bwd_dkv_simt_kernel": ("alu", 6 * d * P, "TFLOP/s"),
        "attn_bwd_dq_simt_kernel": ("alu", 2 * d * P, "TFLOP/s"),
        "attn_bwd_tc_kernel": ("tensor", f_bwd, "TFLOP/s"),
        "dq_convert_kernel": ("hbm", 6 * w.D * w.T, "GB/s"),
        "ln_fwd_kernel": ("hbm", (6 * w.D + 8) * w.T, "GB/s"),
        "ln_bwd_kernel": ("hbm", (10 * w.D + 8) * w.T, "GB/s"),
    }
    launches_total = 0
    for name, (n, tot) in kernels.items():
        per_step = n / args.steps
        launches_total += n
        avg = tot / n
        e = {"launches_per_step": per_step, "ms_per_launch": round(avg, 4),
             "share": round(tot / max(ms * args.steps, 1e-9), 4)}
        if name in algo:
            bound, units, unit = algo[name]
            if unit == "TFLOP/s":
                ach = units / (avg * 1e-3) / 1e12
                peak = pk["bf16_tflops_sustained"] if bound == "tensor" else alu_fp32_peak_tflops(sm_mhz)
            else:
                ach = units / (avg * 1e-3) / 1e9
                peak = pk["hbm_gbs"]
            e.update(bound=bound, achieved=round(ach, 2), peak=round(peak, 1), unit=unit,
                     frac=round(ach / peak, 4))
        kinfo[name] = e
    dominant = max(kernels.items(), key=lambda kv: kv[1][1])[0]
    dk = kinfo[dominant]
    roof = {"kernel": dominant, "bound": dk.get("bound"), "achieved": dk.get("achieved"),
            "peak": dk.get("peak"), "unit": dk.get("unit"), "frac": dk.get("frac"),
            "traffic": measured_traffic(dominant, w.name),
            "peak_source": f"{pk_src} ({'bf16_tflops_sustained' if dk.get('bound') == 'tensor' else ('hbm_gbs' if dk.get('bound') == 'hbm' else 'FP32 FFMA from unit counts x sm_max_mhz')})"}

    flops_step = f_fwd + f_bwd
    # useful FLOPs of all ranks (their shards differ slightly in size) over the slowest rank's time
    all_flops = sum_over_ranks(float(flops_step), world)
    all_fwd = sum_over_ranks(float(f_fwd), world)
    value = all_flops / (ms_max * 1e-3) / 1e12
    fwd_tflops = all_fwd / (ms_fwd * 1e-3) / 1e12
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_max, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded lognormal lengths, N(0,1) activations, N(0,0.02) rab tables)",
        "config": {"workload": w.name, "global_batch_tokens": int(sum_over_ranks(float(w.T), world)),
                   "sequences_per_gpu": w.B,
                   "max_seq_len": w.max_len, "H": H, "d": d, "mask": "causal+rab_pos+rab_time",
                   "parallelism": f"dp{world}", "l2": "inputs larger than L2 (512 MiB per tensor)"},
        "pct_bf16_peak_fwd_bwd": round(value / world / pk["bf16_tflops_sustained"], 4),
        "fwd_tflops": round(fwd_tflops, 3),
        "pct_bf16_peak_fwd": round(fwd_tflops / world / pk["bf16_tflops_sustained"], 4),
        "peak_source": pk_src,
        "e2e": None if ms_e2e is None else {
            "value": round(all_flops / (ms_e2e * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
            "ms_per_step": round(ms_e2e, 3), "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)},
        "gpu_launches": int(launches_total),
        "roofline": roof,
        "kernels": kinfo,
        "clocks": clocks,
    }
    if mf is not None:
        line["mfalcon"] = mf
    line.update(extra or {})
    return line, w


def run_mfalcon(args, world, rank, local):
    from hstu_jagged_pointwise_b200 import ops
    w = W.mfalcon_ranking(seed=args.seed + rank)
    dev = torch.device("cuda", local)
    d = {n: getattr(w, n).to(dev) for n in ("hist_k", "hist_v", "cand_q", "cand_k", "cand_v", "cand_u")}
    small = {n: getattr(w, n).to(dev) for n in ("rab_pos", "rab_time", "gamma", "beta")}
    ho = torch.as_tensor(w.hist_offsets).to(dev)
    co = torch.as_tensor(w.cand_offsets).to(dev)
    hts = torch.as_tensor(w.hist_ts).to(dev)
    cts = torch.as_tensor(w.cand_ts).to(dev)
    m = ops.MFalcon(ho, hts, co, cts, w.H, w.d, w.alpha, w.b_m, int(np.diff(w.hist_offsets).max()),
                    int(np.diff(w.cand_offsets).max()))
    out = dict(y=torch.empty_like(d["cand_q"]), o_pre=torch.empty_like(d["cand_q"]))

    def go():
        m.score(d["hist_k"], d["hist_v"], d["cand_q"], d["cand_k"], d["cand_v"], d["cand_u"], small["rab_pos"],
                small["rab_time"], small["gamma"], small["beta"], out=out)

    for _ in range(args.warmup):
        go()
    torch.cuda.synchronize()
    barrier(world)
    s = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for _ in range(args.steps):
        go()
    e1.record(s)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world)
    if m.check_device_error() != 0:
        raise RuntimeError("device status set in M-FALCON")
    n_c = w.T
    nh, nc = np.diff(w.hist_offsets).astype(np.int64), np.diff(w.cand_offsets).astype(np.int64)
    pairs = int(w.H * np.sum(nc * (nh + 1)))
    pk, _ = peaks()
    tfl = 4 * w.d * pairs / (ms * 1e-3) / 1e12
    del d, out, m
    seq = run_mfalcon_seq(args, world, w, dev)
    return {"workload": w.name, "cands_per_s": round(world * n_c / (ms * 1e-3), 1), "ms_per_pass": round(ms, 4),
            "tflops": round(world * tfl, 3), "pct_bf16_peak": round(tfl / pk["bf16_tflops_sustained"], 4),
            "b_m": w.b_m, "full_sequence": seq}


def run_mfalcon_seq(args, world, w, dev):
    """The same users as one jagged row each, [history ; candidates], through the
    attention forward with the full-sequence M-FALCON mask: history rows causal,
    candidates against all history and themselves."""
    from hstu_jagged_pointwise_b200 import capi, ops
    ws = W.mfalcon_seq_from(w, seed=args.seed + 1)
    t = {n: getattr(ws, n).to(dev) for n in ("q", "k", "v", "u", "rab_pos", "rab_time", "gamma", "beta")}
    off = torch.as_tensor(ws.offsets).to(dev)
    ts = torch.as_tensor(ws.ts).to(dev)
    nr = torch.as_tensor(ws.n_realtime).to(dev)
    layer = ops.Layer(off, ts, ws.H, ws.d, ws.dtype, ws.alpha, ws.max_len, mask_kind="mfalcon_seq", n_realtime=nr)
    out = dict(y=torch.empty_like(t["q"]), o_pre=torch.empty_like(t["q"]),
               mean=torch.empty(ws.T, dtype=torch.float32, device=dev),
               rstd=torch.empty(ws.T, dtype=torch.float32, device=dev))

    def go():
        layer.forward(t["q"], t["k"], t["v"], t["u"], t["rab_pos"], t["rab_time"], t["gamma"], t["beta"], out=out)

    for _ in range(args.warmup):
        go()
    torch.cuda.synchronize()
    barrier(world)
    s = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for _ in range(args.steps):
        go()
    e1.record(s)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world)
    if layer.check_device_error() != 0:
        raise RuntimeError("device status set in the full-sequence M-FALCON forward")
    nh, nc = np.diff(w.hist_offsets).astype(np.int64), np.diff(w.cand_offsets).astype(np.int64)
    pairs = int(w.H * np.sum(nh * (nh + 1) // 2 + nc * (nh + 1)))
    pk, _ = peaks()
    tfl = 4 * w.d * pairs / (ms * 1e-3) / 1e12
    del out, layer

    # the KV-cache producer on the same batch: history rows of k, v, ts packed for the scorer
    hist_rows = int(nh.sum())
    cache = ops.mfalcon_cache_history(off, ts, nr, t["k"], t["v"], hist_rows=hist_rows)
    for _ in range(args.warmup):
        ops.mfalcon_cache_history(off, ts, nr, t["k"], t["v"], out=cache)
    torch.cuda.synchronize()
    barrier(world)
    capi.profile_enable(True)
    e0.record(s)
    for _ in range(args.steps):
        ops.mfalcon_cache_history(off, ts, nr, t["k"], t["v"], out=cache)
    e1.record(s)
    torch.cuda.synchronize()
    prof = capi.profile_read()
    capi.profile_enable(False)
    ms_c = max_over_ranks(e0.elapsed_time(e1) / args.steps, world)
    if int(cache["status"].item()) != 0:
        raise RuntimeError("device status set in the KV-cache producer")
    nb = hist_rows * (4 * ws.D * 2 + 16)     # read and write k, v rows (bf16) and the int64 timestamp
    n_copy, t_copy = prof.get("cache_copy_kernel", (1, ms_c))
    gbs = nb / (t_copy / n_copy * 1e-3) / 1e9
    return {"workload": f"{w.name}_one_row", "tokens": int(ws.T), "cands_per_s": round(world * w.T / (ms * 1e-3), 1),
            "ms_per_pass": round(ms, 4), "tflops": round(world * tfl, 3),
            "pct_bf16_peak": round(tfl / pk["bf16_tflops_sustained"], 4),
            "kv_cache_producer": {"rows": hist_rows, "ms_per_call": round(ms_c, 4),
                                  "copy_kernel_ms": round(t_copy / n_copy, 4), "bytes_per_call": nb,
                                  "copy_kernel_gbs": round(gbs, 1), "frac_hbm": round(gbs / pk["hbm_gbs"], 4)}}


# ----------------------------------------------------------------------------
# reference arm: the fp64 oracle on the host cores
# ----------------------------------------------------------------------------

def run_reference(args, world, rank):
    if rank != 0:
        return None
    w = W.large_layer(seed=args.seed, total=args.tokens)
    sample, seqs = oracle_sample(w, target_s=max(5.0, 60.0 / max(args.steps + args.warmup, 1)))
    for _ in range(args.warmup):
        time_oracle(sample)
    vals, secs = [], []
    threads = 1
    for _ in range(args.steps):
        v, dt, threads = time_oracle(sample)
        vals.append(v)
        secs.append(dt)
    value = statistics.median(vals)
    desc = (f"{len(seqs)} whole sequences ({int(sample.T)} tokens, shortest first) of {w.name}; "
            f"forward + LayerNorm + full backward in fp64")
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * statistics.median(secs), 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": w.name, "sample": desc},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-mfalcon", action="store_true")
    ap.add_argument("--no-gln", action="store_true", help="skip the Group LayerNorm variant")
    ap.add_argument("--no-proj", action="store_true", help="skip the f1 / f2 projections")
    ap.add_argument("--no-data", action="store_true", help="skip the Stochastic Length / packing data step")
    ap.add_argument("--no-layer", action="store_true", help="skip the whole-layer (f1, attention, f2) step")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the training-shape (Stochastic Length) and MTGR-Medium legs")
    ap.add_argument("--only-configs", action="store_true",
                    help="run only the training-shape and MTGR-Medium legs and print their JSON (profiling aid)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end leg")
    ap.add_argument("--tokens", type=int, default=262144,
                    help="total tokens of the large-layer workload (smaller values for profiling)")
    ap.add_argument("--only-proj", action="store_true",
                    help="run only the f1 / f2 projections leg and print its JSON (profiling aid)")
    ap.add_argument("--only-layer", action="store_true",
                    help="run only the whole-layer leg and print its JSON (profiling aid)")
    ap.add_argument("--only-mfalcon", action="store_true",
                    help="run only the M-FALCON legs (cached scorer, one-row forward, KV-cache producer) "
                         "and print their JSON (profiling aid)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    world, rank, local = dist_init(args.gpus) if args.impl == "ours" else (
        int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")), 0)
    if args.impl == "reference":
        line = run_reference(args, world, rank)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    if args.only_proj:
        torch.cuda.set_device(local)
        line = run_proj(args, world, rank)
        if rank == 0:
            print(json.dumps({"projections": line}), flush=True)
        return
    if args.only_configs:
        torch.cuda.set_device(local)
        line = {"training_sl": run_training_sl(args, world, rank), "mtgr_medium": run_mtgr_medium(args, world, rank)}
        if rank == 0:
            print(json.dumps(line), flush=True)
        return
    if args.only_mfalcon:
        torch.cuda.set_device(local)
        line = run_mfalcon(args, world, rank, local)
        if rank == 0:
            print(json.dumps({"mfalcon": line}), flush=True)
        return
    if args.only_layer:
        torch.cuda.set_device(local)
        w = W.large_layer(seed=args.seed + rank, total=args.tokens)
        P = causal_pairs(w.lengths) * w.H
        line = run_full_layer(args, world, w, 12 * w.d * P)
        if rank == 0:
            print(json.dumps({"full_layer": line}), flush=True)
        return
    line, w = run_ours(args, world, rank, local)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        sample, seqs = oracle_sample(w)
        v, dt, threads = time_oracle(sample)
        line["cpu_baseline"] = {"value": round(v, 6), "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                                "sample": f"{len(seqs)} whole sequences ({int(sample.T)} tokens, shortest first) "
                                          f"of {w.name}, fwd+LN+bwd in fp64, {dt:.1f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
