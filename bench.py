#!/usr/bin/env python3
"""Benchmark: ternary / 4-bit dequant-fused matmuls on B200, one JSON line on stdout.

A *step* is one pass of every matmul row of the hot path over one batch of synthetic
input, shaped like one denoising step of the pages' 4B MMDiT plus the text encoder's
4-bit linears and the small-M ternary GEMV:

  mmdit_9216x3072, mmdit_3072x12288, mmdit_12288x3072   Q2_0, 1536 tokens (tensor cores)
  lora_r4, lora_r32, lora_r64                           Q2_0 9216x3072 + rank-r branch
  encoder_up (9728x2560), encoder_down (2560x9728)      4-bit, 512 tokens
  gemv_m1, gemv_m4, gemv_m16                            Q2_0 3072x3072, M <= 16 (HBM-bound)

``value`` is the step's algorithmic FLOPs (2*M*N*K, plus 2*M*r*(K+N) for the branch) per
second of device time, over all ranks (weak scaling: every rank runs its own step).  L2
is flushed (256 MB write) before every timed step, outside the step's events.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
For N > 1 launch one process per GPU with torch.distributed.run.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "ternary GEMM TFLOP/s and weight GB/s at 1 B200; % of tensor/HBM roofline"
UNIT = "TFLOP/s"
STEP_ORDER = ["mmdit_9216x3072", "gemv_m1", "gemv_m4", "gemv_m16", "mmdit_3072x12288",
              "lora_r4", "lora_r32", "lora_r64", "mmdit_12288x3072", "encoder_up",
              "encoder_down"]
DOMINANT = ["mmdit_9216x3072", "mmdit_3072x12288", "mmdit_12288x3072"]
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "tc_gemm_q2_mmdit.md")
TC_SOURCE = os.path.join(ROOT, "bit_weight_quantized_tgemm_b200", "csrc", "gemm_tc.cuh")
# CPU seconds the reference arm spends over all its steps (warm-up included)
REFERENCE_SECONDS = 90.0


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="CPU work for the oracle baseline sample (rank 0, N=1 only)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", default="",
                    help="comma-separated subset of the step's matmuls (profiling runs)")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the end-to-end leg, the small-M stream and the CPU baseline")
    ap.add_argument("--parts", default="",
                    help="comma-separated subset of the extra parts to run (default: all)")
    ap.add_argument("--kernels", action="store_true",
                    help="run every kernel of the library once on its workload inside an NVTX "
                         "range named 'kernels' (for ncu --nvtx --nvtx-include kernels/), then exit")
    return ap.parse_args()


# ---- distributed plumbing ----------------------------------------------------------------

def dist_setup(args):
    import torch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(v: float, world: int) -> float:
    """The slowest rank's value (device times are compared as the max over ranks)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_value(world: int, step_flops: float, step_ms: float) -> float:
    """Whole-job TFLOP/s: every rank runs one step of `step_flops`; the job takes the
    slowest rank's `step_ms`."""
    return world * step_flops / (step_ms * 1e-3) / 1e12


def dist_done(world):
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


# ---- clocks during the timed region ---------------------------------------------------

class ClockSampler:
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.rows = []
        self.proc = None
        self.t0 = self.t1 = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(gpu_index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append((time.time(), line.strip()))

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def summary(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        inside = [r for (t, r) in self.rows if self.t0 is not None and self.t0 <= t <= self.t1 + 0.06]
        if not inside:
            inside = [r for (_, r) in self.rows[-3:]]
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in inside:
            parts = [p.strip() for p in r.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---- the workload ------------------------------------------------------------------------

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "tflops_burst": d["bf16_tflops"],
                "tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "tflops_burst": 1590.0, "tflops_sustained": 1400.0,
            "source": "fallback"}


def ncu_traffic():
    """Per-launch DRAM bytes of the tensor-core Q2 kernel from the committed ncu summary,
    or None if there is none or the kernel source changed since it was taken."""
    if not os.path.exists(TRAFFIC_FILE):
        return None, None
    want_sha = None
    traffic = None
    with open(TRAFFIC_FILE) as f:
        for line in f:
            if line.startswith("kernel_source_sha256:"):
                want_sha = line.split(":", 1)[1].strip()
            if line.startswith("traffic_bytes_per_launch_full:"):
                traffic = float(line.split(":", 1)[1].strip())
    with open(TC_SOURCE, "rb") as f:
        sha = hashlib.sha256(f.read()).hexdigest()
    if want_sha != sha:
        return None, "kernel changed since the ncu capture"
    return traffic, None


class Op:
    """One matmul of the step, its device buffers and a direct C-ABI call."""

    def __init__(self, w, rank: int, tg, torch):
        self.w = w
        self.name = w.name
        prob = w.make() if rank == 0 else _reseed(w, rank).make()
        self.prob = prob
        dev = torch.device("cuda")
        self.x = _to_dev(prob.x, torch.bfloat16, torch)
        M, N, K = w.M, w.N, w.K
        if w.kind == "q4":
            wq, sz, st = tg.q4_pack(torch.from_numpy(prob.codes).to(dev),
                                    torch.from_numpy(prob.s).to(dev), torch.from_numpy(prob.z).to(dev))
            self.wq, self.sc = wq, sz
            self.op = tg.OP_Q4
        else:
            wq, d, st = tg.q2_pack(torch.from_numpy(prob.codes).to(dev),
                                   torch.from_numpy(prob.scale).to(dev))
            self.wq, self.sc = wq, d
            self.op = tg.OP_Q2_LORA if w.kind == "q2_lora" else tg.OP_Q2
        torch.cuda.synchronize()
        if int(st.item()) != 0:
            raise RuntimeError(f"{w.name}: pack status {int(st.item())}")
        self.a = self.b = None
        if w.kind == "q2_lora":
            self.a = _to_dev(prob.a, torch.bfloat16, torch)
            self.b = _to_dev(prob.b, torch.bfloat16, torch)
        self.y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        self.flops = w.flops
        self.weight_bytes = w.weight_bytes
        self.ws_need = tg.workspace_size(self.op, M, N, K, w.r)
        # host copies for the end-to-end leg
        self.x_host = self.x.cpu().pin_memory()
        self.y_host = torch.empty_like(self.y, device="cpu").pin_memory()

    def bind(self, tg, ws, stream):
        """Pre-compute the C call so a step costs one ctypes call per op."""
        L = tg.lib()
        w = self.w
        wsp = ws.data_ptr() if ws is not None else None
        wsn = ws.numel() if ws is not None else 0
        if w.kind == "q4":
            fn = L.tgemm_q4
            args = (self.x.data_ptr(), self.wq.data_ptr(), self.sc.data_ptr(), self.y.data_ptr(),
                    w.M, w.N, w.K, tg.OUT_BF16, wsp, wsn, stream)
        elif w.kind == "q2_lora":
            fn = L.tgemm_q2_lora
            args = (self.x.data_ptr(), self.wq.data_ptr(), self.sc.data_ptr(), self.a.data_ptr(),
                    self.b.data_ptr(), w.r, self.y.data_ptr(), w.M, w.N, w.K, tg.OUT_BF16, wsp,
                    wsn, stream)
        else:
            fn = L.tgemm_q2
            args = (self.x.data_ptr(), self.wq.data_ptr(), self.sc.data_ptr(), self.y.data_ptr(),
                    w.M, w.N, w.K, tg.OUT_BF16, wsp, wsn, stream)
        self._fn, self._args = fn, args

    def __call__(self):
        st = self._fn(*self._args)
        if st != 0:
            raise RuntimeError(f"{self.name}: status {st}")


def _reseed(w, rank):
    """The same workload with rank-specific data (weak scaling: every rank its own batch)."""
    import dataclasses

    base = tuple(w.seed) if isinstance(w.seed, tuple) else (w.seed,)
    return dataclasses.replace(w, seed=base + (7919, rank))


def _to_dev(bits, dtype, torch):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(dtype).cuda()


# ---- CPU oracle baseline -------------------------------------------------------------------

class OracleSampler:
    """The CPU oracle on sampled outputs of the step's matmuls.

    Outputs y[m, n] are drawn from every matmul in proportion to its FLOPs and computed
    one at a time from the packed row (oracle.*_gemm_at); each counts 2*K FLOPs (plus the
    branch's 2*r*(K+1) for the low-rank ops)."""

    def __init__(self, items):
        import oracle as orc

        self.o = orc.get()
        self.packed = []
        for item in items:
            w = item.w if hasattr(item, "w") else item
            prob = item.prob if hasattr(item, "prob") else w.make()
            if w.kind == "q4":
                wq, sc, _ = self.o.q4_pack(prob.codes, prob.s, prob.z)
            else:
                wq, sc, _ = self.o.q2_pack(prob.codes, prob.scale)
            self.packed.append((w, prob, wq, sc))
        self.total = sum(w.flops for (w, *_) in self.packed)
        self.per_sample = None  # seconds per unit of `scale`, from calibration

    def _run(self, scale, rng):
        o = self.o
        flops = 0
        n_out = 0
        t0 = time.perf_counter()
        for (w, prob, wq, sc) in self.packed:
            n = max(1, int(round(scale * w.flops / self.total)))
            mi = rng.integers(0, w.M, n)
            ni = rng.integers(0, w.N, n)
            if w.kind == "q4":
                o.q4_gemm_at(prob.x, wq, sc, w.N, mi, ni)
            elif w.kind == "q2_lora":
                o.q2_gemm_at(prob.x, wq, sc, w.N, mi, ni, prob.a, prob.b)
            else:
                o.q2_gemm_at(prob.x, wq, sc, w.N, mi, ni)
            flops += n * (2 * w.K + (2 * w.r * (w.K + 1) if w.r else 0))
            n_out += n
        return flops, time.perf_counter() - t0, n_out

    def run(self, seconds: float, seed: int = 0):
        """Sample until about `seconds` of oracle time have been spent (a small calibration
        run fixes the first batch's size; each batch re-estimates the time per sample, so
        a batch that falls short because of fixed per-call costs is topped up)."""
        rng = np.random.default_rng(seed)
        if self.per_sample is None:
            _, t, _ = self._run(200, rng)
            self.per_sample = max(t, 1e-4) / 200
        f = n = 0
        t = 0.0
        for _ in range(8):
            scale = max(50.0, (seconds - t) / self.per_sample)
            fb, tb, nb = self._run(scale, rng)
            f, t, n = f + fb, t + tb, n + nb
            self.per_sample = max(tb, 1e-4) / scale
            if t >= 0.9 * seconds:
                break
        return {"flops": f, "seconds": t, "samples": n, "cores": self.o.num_threads()}


def oracle_sample(items, seconds: float, seed: int = 0):
    return OracleSampler(items).run(seconds, seed)


def step_config(world: int, step_flops: float, step_wbytes: float) -> dict:
    """The workload both arms report (the same object in both JSON lines)."""
    return {
        "workload": "mmdit_step: 1536-token ternary 9216x3072, 3072x12288, 12288x3072; "
                    "rank 4/32/64 branch on 9216x3072; 512-token 4-bit 9728x2560, "
                    "2560x9728; 3072x3072 ternary GEMV at M=1,4,16",
        "tokens": 1536, "encoder_tokens": 512, "out_dtype": "bf16",
        "step_gflop": step_flops / 1e9, "step_weight_mb": step_wbytes / 1e6,
        "l2": "flushed before every timed step (256 MB write, outside the step events)",
        "parallelism": f"independent replicas x{world} (weak scaling, no collective)",
    }


def reference_arm(args, world, rank):
    """The oracle as the reference arm: K timed steps, each a bounded sample."""
    if rank != 0:
        return
    from bit_weight_quantized_tgemm_b200 import synth

    items = [synth.ALL[n] for n in STEP_ORDER]
    sampler = OracleSampler(items)
    per_step = max(0.2, REFERENCE_SECONDS / max(1, args.steps + args.warmup))
    for i in range(args.warmup):
        sampler.run(per_step, seed=1000 + i)
    fl, sec, samples, cores = 0, 0.0, 0, 1
    for i in range(args.steps):
        r = sampler.run(per_step, seed=i + 1)
        fl += r["flops"]
        sec += r["seconds"]
        samples += r["samples"]
        cores = r["cores"]
    value = fl / sec / 1e12
    sample = (f"{samples} outputs y[m,n] over {args.steps} steps, drawn from the step's 11 "
              f"matmuls in proportion to their FLOPs, each computed on its own by the CPU oracle")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * sec / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": dict(step_config(world, sum(w.flops for w in items), sum(w.weight_bytes for w in items)),
                       sample=sample),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---- our arm -------------------------------------------------------------------------------

def ours(args, world, rank, local):
    import torch

    import bit_weight_quantized_tgemm_b200 as tg
    from bit_weight_quantized_tgemm_b200 import synth

    tg.set_path(tg.PATH_AUTO)
    torch.manual_seed(0)
    names = [n for n in args.only.split(",") if n] or STEP_ORDER
    for n in names:
        if n not in synth.ALL:
            raise SystemExit(f"unknown matmul {n!r}; choose from {', '.join(STEP_ORDER)}")
    extras = not args.no_extras and not args.only
    ops = [Op(synth.ALL[n], rank, tg, torch) for n in names]
    ws_bytes = max(o.ws_need for o in ops)
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    for o in ops:
        o.bind(tg, ws, stream)
    flush_buf = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device="cuda")
    step_flops = sum(o.flops for o in ops)
    step_wbytes = sum(o.weight_bytes for o in ops)

    def step():
        for o in ops:
            o()

    # warm-up (also loads kernels, encodes nothing persistent)
    for _ in range(args.warmup):
        flush_buf.zero_()
        step()
    torch.cuda.synchronize()
    if tg.device_error():
        raise RuntimeError("device error after warm-up")

    # ---- timed region: K steps, events around each step, L2 flushed before each
    K = args.steps
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(K)]
    for kind in range(6):
        tg.profile_read(kind, reset=True)
    clocks = ClockSampler(local)
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    clocks.mark_start()
    launches0 = tg.launch_count()
    # events around the dominant kernel's launches only (its roofline); the other kinds
    # are timed in a separate profiled pass below, so the step itself carries 6 extra
    # event records, not two per launch
    tg.profile_enable(1 << tg.KIND_TC_Q2)
    for i in range(K):
        flush_buf.zero_()
        evs[i][0].record()
        step()
        evs[i][1].record()
    torch.cuda.synchronize()
    barrier(world)
    clocks.mark_end()
    tg.profile_enable(False)
    launches = tg.launch_count() - launches0
    step_ms_local = sum(a.elapsed_time(b) for a, b in evs) / K
    step_ms = max_over_ranks(step_ms_local, world)
    clk = clocks.summary()
    prof = {k: tg.profile_read(k, reset=True) for k in range(6)}

    # ---- profiled pass (not the timed region): events around every launch, per kind
    P = max(3, min(K, 30))
    tg.profile_enable(True)
    for _ in range(P):
        flush_buf.zero_()
        step()
    torch.cuda.synchronize()
    tg.profile_enable(False)
    prof_all = {k: tg.profile_read(k, reset=True) for k in range(6)}

    # ---- dominant kernel roofline (tensor-core Q2 kernel, FLOP-weighted over its launches)
    tc_ms, tc_n = prof[tg.KIND_TC_Q2]
    dom_flops = sum(o.flops for o in ops if o.name in DOMINANT)
    peaks = load_peaks()
    timed_s = step_ms * K * 1e-3
    peak = peaks["tflops_sustained"] if timed_s > 1.0 else peaks["tflops_burst"]
    achieved = (dom_flops * K) / (tc_ms * 1e-3) / 1e12 if tc_ms > 0 else None
    traffic, traffic_note = ncu_traffic()
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": (achieved / peak) if achieved else None, "traffic": traffic,
                "kernel": "tc_gemm_kernel<Q2> (1536 tokens; 9216x3072, 3072x12288, 12288x3072)",
                "launches": tc_n,
                "peak_source": f"MEASURED_PEAKS.json bf16 "
                               f"{'sustained' if timed_s > 1.0 else 'burst'} (of {peaks['source']}); "
                               "f16 operands run at the bf16 rate"}
    if traffic_note:
        roofline["traffic_note"] = traffic_note
    gv_ms, gv_n = prof_all[tg.KIND_GEMV_Q2]
    gv_bytes = sum(o.weight_bytes for o in ops if o.name.startswith("gemv")) * P
    # lone calls (events around each launch, inside the step): latency, not bandwidth
    lone_gbs = gv_bytes / (gv_ms * 1e-3) / 1e9 if gv_ms else None
    roofline_small_m = {"bound": "hbm", "unit": "GB/s", "peak": peaks["hbm_gbs"],
                        "kernel": "gemv_kernel<Q2> (M=1,4,16; 3072x3072), packed-weight bytes",
                        "how": "lone calls in the step's profiled pass",
                        "achieved": lone_gbs,
                        "lone_call": {"achieved": lone_gbs,
                                      "frac": lone_gbs / peaks["hbm_gbs"] if lone_gbs else None}}

    # ---- per-kind kernel times per step, from the profiled pass
    kinds = ["tc_q2", "tc_q2_lora", "tc_q4", "gemv_q2", "gemv_q4", "prep"]
    kernel_time = {"steps": P, "how": "CUDA events around every launch, separate pass of P steps"}
    kernel_time.update({kinds[k]: {"us_per_step": prof_all[k][0] * 1e3 / P,
                                   "launches_per_step": prof_all[k][1] / P} for k in range(6)})

    # ---- end-to-end through the C ABI with host buffers (pinned), copies inside the region
    h2d = sum(o.x.numel() * 2 for o in ops)
    d2h = sum(o.y.numel() * 2 for o in ops)
    e2e_steps = max(5, min(K, 50)) if extras else 1
    # Host-to-device copies run on one stream, the matmuls on the compute stream and the
    # device-to-host copies on a third, ordered by events: op i waits for its x, op i's y is
    # copied back as soon as op i is done, and a step's copy into x (or out of y) waits
    # for the previous step's op i.  Both copy directions overlap the matmuls.
    s_c = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    in_ready = [torch.cuda.Event() for _ in ops]
    done = [torch.cuda.Event() for _ in ops]
    out_done = [torch.cuda.Event() for _ in ops]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    e0.record(s_c)
    s_in.wait_stream(s_c)
    s_out.wait_stream(s_c)
    for step_i in range(e2e_steps):
        with torch.cuda.stream(s_in):
            for i, o in enumerate(ops):
                if step_i:
                    s_in.wait_event(done[i])
                o.x.copy_(o.x_host, non_blocking=True)
                in_ready[i].record(s_in)
        for i, o in enumerate(ops):
            s_c.wait_event(in_ready[i])
            if step_i:
                s_c.wait_event(out_done[i])
            o()
            done[i].record(s_c)
            with torch.cuda.stream(s_out):
                s_out.wait_event(done[i])
                o.y_host.copy_(o.y, non_blocking=True)
                out_done[i].record(s_out)
    s_c.wait_stream(s_in)
    s_c.wait_stream(s_out)
    e1.record(s_c)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world)

    # ---- small-M stream: 64 distinct 3072x3072 weights (160 MB > L2), one graph of 64 GEMVs
    parts = {}
    if extras:
        for key, fn in (("gemv_stream", gemv_stream), ("gemv_branch", gemv_branch),
                        ("dual_out_projection", dual_out_projection),
                        ("token_sweep", token_sweep), ("mmdit_sequence", mmdit_sequence)):
            if args.parts and key not in args.parts.split(","):
                continue
            try:
                parts[key] = fn(tg, torch, stream)
            except Exception as exc:  # report, do not hide
                parts[key] = {"error": str(exc)}

    # the small-M roofline proper: back-to-back calls over weights that do not fit in L2
    gs = parts.get("gemv_stream", {})
    by_shape = {}
    for key, res in gs.items():
        if not isinstance(res, dict) or not all(f"m{m}" in res for m in (1, 4, 16)):
            continue
        us = sum(res[f"m{m}"]["auto"]["us_per_call"] for m in (1, 4, 16))
        gbs = 3 * res["weight_mb"] * 1e6 / (us * 1e-6) / 1e9
        by_shape[key] = {"achieved": gbs, "frac": gbs / peaks["hbm_gbs"],
                         **{f"m{m}_frac": res[f"m{m}"]["auto"]["weight_gbs"] / peaks["hbm_gbs"]
                            for m in (1, 4, 16)}}
    if "q2_3072x3072" in by_shape:
        roofline_small_m["kernel"] = ("small-M path as dispatched (gemv_kernel; gemv_stream_kernel for "
                                      "<= 8 tokens on large one-pass linears), Q2 M=1,4,16 on "
                                      "3072x3072, packed-weight bytes")
        roofline_small_m["achieved"] = by_shape["q2_3072x3072"]["achieved"]
        roofline_small_m["how"] = ("CUDA graph of back-to-back calls at M = 1, 4 and 16, each over its "
                                   "own weight copy (working set >= 4x L2): packed-weight bytes of the "
                                   "three calls / their summed per-call time")
        roofline_small_m["by_shape"] = by_shape
    if roofline_small_m["achieved"]:
        roofline_small_m["frac"] = roofline_small_m["achieved"] / peaks["hbm_gbs"]

    dev_err = tg.device_error()
    cpu = None
    if rank == 0 and world == 1 and extras and not args.no_cpu_baseline:
        r = oracle_sample(ops, args.cpu_seconds)
        cpu = {"value": r["flops"] / r["seconds"] / 1e12, "unit": UNIT, "cores": r["cores"],
               "kind": "oracle",
               "sample": f"{r['samples']} outputs y[m,n] drawn from the step's 11 matmuls in "
                         f"proportion to their FLOPs, each computed on its own "
                         f"({r['seconds']:.1f} s on {r['cores']} host threads)"}

    value = aggregate_value(world, step_flops, step_ms)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f16", "data": "synthetic",
        "config": step_config(world, step_flops, step_wbytes),
        "weight_gbs": world * step_wbytes / (step_ms * 1e-3) / 1e9,
        "e2e": {"value": world * step_flops / (e2e_ms * 1e-3) / 1e12, "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms,
                "how": "tgemm_* C-ABI calls; every step copies each x from pinned host memory "
                       "and each y back to pinned host memory, on two copy streams that overlap "
                       "the matmuls (event-ordered per op); device-timed"},
        "gpu_launches": launches,
        "clocks": clk,
        "roofline": roofline,
        "roofline_small_m": roofline_small_m,
        "kernel_time": kernel_time,
        "parts": parts,
        "device_error": dev_err,
        "cpu_baseline": cpu,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


def _time_calls(torch, fn, reps=20, warm=3):
    """Median device time (seconds) of fn() over `reps` single calls, L2 flushed before each."""
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device="cuda")
    for _ in range(warm):
        fn()
    times = []
    for _ in range(reps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b) * 1e-3)
    return statistics.median(times)


def _q2_device_weights(tg, torch, N, K, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    codes = torch.randint(0, 3, (N, K), dtype=torch.uint8, device="cuda", generator=g)
    scale = (torch.rand(N, K // 128, device="cuda", generator=g) * 0.02).half().float()
    wq, d, _ = tg.q2_pack(codes, scale)
    return wq, d


def dual_out_projection(tg, torch, stream):
    """The MMDiT's fused out projection split along its input axis (page 2, 'Slice weights,
    not activations'): 1536 tokens, N = 3072, K1 = 3072 (attention output) + K2 = 12288
    (MLP output), bf16 out; one fused call against two separate calls plus an add."""
    M, N, K1, K2 = 1536, 3072, 3072, 12288
    wq1, d1 = _q2_device_weights(tg, torch, N, K1, 5)
    wq2, d2 = _q2_device_weights(tg, torch, N, K2, 6)
    x1 = torch.randn(M, K1, device="cuda").bfloat16()
    x2 = torch.randn(M, K2, device="cuda").bfloat16()
    y = torch.empty(M, N, device="cuda", dtype=torch.bfloat16)
    ws = torch.empty(tg.dual_workspace_size(M, N, K1, K2), dtype=torch.uint8, device="cuda")
    fused = _time_calls(torch, lambda: tg.gemm_q2_dual(x1, wq1, d1, x2, wq2, d2, y=y, workspace=ws))
    y1 = torch.empty(M, N, device="cuda", dtype=torch.float32)
    y2 = torch.empty(M, N, device="cuda", dtype=torch.float32)

    def separate():
        tg.gemm_q2(x1, wq1, d1, out_dtype=tg.OUT_F32, y=y1)
        tg.gemm_q2(x2, wq2, d2, out_dtype=tg.OUT_F32, y=y2)
        torch.add(y1, y2, out=y1)
    sep = _time_calls(torch, separate)
    flop = 2 * M * N * (K1 + K2)
    return {"shape": f"{M} tokens x {N} x ({K1} + {K2})", "fused_us": fused * 1e6,
            "fused_tflops": flop / fused / 1e12, "two_calls_plus_add_us": sep * 1e6}


def token_sweep(tg, torch, stream):
    """The 9216 x 3072 ternary matmul at the pages' step token counts (256 + text rows at
    256^2, 384 = quarter-size first step, 1280 = 1024 patches + 256, 1536) and 4096."""
    N, K = 9216, 3072
    wq, d = _q2_device_weights(tg, torch, N, K, 7)
    out = {}
    for M in (256, 384, 1280, 1536, 4096):
        x = torch.randn(M, K, device="cuda").bfloat16()
        y = torch.empty(M, N, device="cuda", dtype=torch.bfloat16)
        ws = torch.empty(max(tg.workspace_size(tg.OP_Q2, M, N, K), 256), dtype=torch.uint8,
                         device="cuda")
        t = _time_calls(torch, lambda: tg.gemm_q2(x, wq, d, y=y, workspace=ws), reps=10)
        out[f"m{M}"] = {"us": t * 1e6, "tflops": 2 * M * N * K / t / 1e12}
    return out


def mmdit_sequence(tg, torch, stream):
    """All 81 token-path ternary linears of one MMDiT step (text conditioning projection,
    5 joint blocks x 2 streams x 4, 20 single blocks x (stacked linear1 + two-input
    linear2)), captured once in a CUDA graph and replayed, at the pages' token counts:
    1024 image + 512 text (full size), 1024 + 256, and 256 + 128 (the quarter-size first
    step). 0.91 GB of distinct packed weights per step, more than L2, so every replay
    reads them from HBM."""
    from bit_weight_quantized_tgemm_b200 import mmdit
    weights = mmdit.make_weights(mmdit.weight_shapes(), seed=11)
    sustained = load_peaks()["tflops_sustained"]
    ev = lambda: torch.cuda.Event(enable_timing=True)

    def timed(fn, n):
        a, b = ev(), ev()
        a.record()
        for _ in range(n):
            fn()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) * 1e-3 / n

    out = {}
    for img, txt, sliced in ((1024, 512, False), (1024, 512, True), (1024, 256, False),
                             (256, 128, False)):
        seq = mmdit.StepSequence(mmdit.step_linears(img, txt, slice_rows=sliced), weights)
        graph = seq.capture(warmup=2)
        n0 = tg.launch_count()
        seq.run()
        torch.cuda.synchronize()
        launches = tg.launch_count() - n0
        # graph replays and eager runs alternate, so both see the same (power-capped) clocks
        clocks = ClockSampler(torch.cuda.current_device())
        clocks.mark_start()
        g_t, e_t = [], []
        for _ in range(3):
            g_t.append(timed(graph.replay, 8))
            e_t.append(timed(seq.run, 8))
        clocks.mark_end()
        clk = clocks.summary()
        t, eager = statistics.median(g_t), statistics.median(e_t)
        key = f"img{img}_txt{txt}" + ("_row_slices" if sliced else "")
        out[key] = {"linears": len(seq.linears), "launches": launches, "gflop": seq.flops / 1e9,
                    "us": t * 1e6, "tflops": seq.flops / t / 1e12,
                    "frac_of_sustained": seq.flops / t / 1e12 / sustained,
                    "weight_gbs": seq.weight_bytes / t / 1e9, "eager_us": eager * 1e6,
                    "sm_mhz": clk.get("sm_mhz"), "reasons": clk.get("reasons")}
        del graph, seq
    del weights
    torch.cuda.empty_cache()
    return out


def _device_weights(tg, torch, fmt, N, K, g):
    """One packed weight matrix drawn on the device (codes uniform, scales as the recipe)."""
    if fmt == 0:
        codes = torch.randint(0, 3, (N, K), dtype=torch.uint8, device="cuda", generator=g)
        scale = (torch.rand(N, K // 128, device="cuda", generator=g) * 0.02).half().float()
        wq, sc, _ = tg.q2_pack(codes, scale)
    else:
        codes = torch.randint(0, 16, (N, K), dtype=torch.uint8, device="cuda", generator=g)
        s = (torch.rand(N, K // 64, device="cuda", generator=g) * 0.01).half().float()
        z = (7 + torch.rand(N, K // 64, device="cuda", generator=g)).half().float()
        wq, sc, _ = tg.q4_pack(codes, s, z)
    return wq, sc


def _graph_per_call(tg, torch, calls, fn):
    """Seconds per call of `calls` (argument tuples for fn) replayed from one CUDA graph."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for c in calls[:4]:
            assert fn(*c, s.cuda_stream) == 0
        s.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=s):
            for c in calls:
                fn(*c, s.cuda_stream)
    torch.cuda.synchronize()
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = 10
    a.record()
    for _ in range(reps):
        graph.replay()
    b.record()
    torch.cuda.synchronize()
    del graph
    return a.elapsed_time(b) / (reps * len(calls)) * 1e-3


# Small-M shapes (format, N, K): the GEMV workload's 3072^2, the MMDiT step's large
# linears, and the 4-bit encoder's up and down projections.
GEMV_SHAPES = [(0, 3072, 3072), (0, 12288, 3072), (0, 3072, 12288), (0, 21504, 3072),
               (1, 9728, 2560), (1, 2560, 9728)]


def gemv_stream(tg, torch, stream):
    """Back-to-back small-M calls (M = 1, 4, 16), replayed from a CUDA graph, each call over
    its own weight copy; the copies total at least 4x the L2 size, so every call reads its
    weights from HBM.  Per shape: the library's own choice ("auto"), and each form forced
    (per-pass and streaming kernels); weight GB/s = packed-weight bytes / time per call."""
    l2 = torch.cuda.get_device_properties(0).L2_cache_size
    L = tg.lib()
    out = {}
    for fmt, N, K in GEMV_SHAPES:
        wbytes = N * K // 4 + N * (K // 128) * 2 if fmt == 0 else N * K // 2 + N * (K // 64) * 4
        ncopies = max(24, -(-4 * l2 // wbytes))
        g = torch.Generator(device="cuda").manual_seed(123 + N + K)
        copies = [_device_weights(tg, torch, fmt, N, K, g) for _ in range(ncopies)]
        fn = L.tgemm_q2 if fmt == 0 else L.tgemm_q4
        key = f"{'q2' if fmt == 0 else 'q4'}_{N}x{K}"
        res = {"copies": ncopies, "working_set_mb": ncopies * wbytes / 1e6, "weight_mb": wbytes / 1e6}
        for M in (1, 4, 16):
            x = torch.randn(M, K, device="cuda").bfloat16()
            y = torch.empty(M, N, device="cuda", dtype=torch.bfloat16)
            calls = [(x.data_ptr(), wq.data_ptr(), sc.data_ptr(), y.data_ptr(), M, N, K,
                      tg.OUT_BF16, None, 0) for (wq, sc) in copies]
            row = {}
            for label, path in (("auto", tg.PATH_AUTO), ("pass", tg.PATH_SMALL_M_PASS),
                                ("stream", tg.PATH_SMALL_M_STREAM)):
                prev = tg.set_path(path)
                try:
                    t = _graph_per_call(tg, torch, calls, fn)
                finally:
                    tg.set_path(prev)
                row[label] = {"us_per_call": t * 1e6, "weight_gbs": wbytes / t / 1e9}
            pl = tg.gemv_plan(fmt, M, N, K, torch.cuda.get_device_properties(0).multi_processor_count)
            if pl:
                row["stream_plan"] = {"passes": pl["passes"], "ring": pl["S"], "tiles": pl["j_max"]}
            res[f"m{M}"] = row
        out[key] = res
        del copies
        torch.cuda.empty_cache()
    return out


def gemv_branch(tg, torch, stream):
    """Small-M calls with the rank-r branch (M = 1, 4, 16 on 9216 x 3072, r = 4, 32, 64):
    the kernel computing u = x A^T plus the per-pass kernel, back to back from a CUDA graph
    over weight copies totalling >= 4x L2; r0: the same calls without the branch."""
    N, K = 9216, 3072
    wbytes = N * K // 4 + N * (K // 128) * 2
    l2 = torch.cuda.get_device_properties(0).L2_cache_size
    ncopies = max(24, -(-4 * l2 // wbytes))
    g = torch.Generator(device="cuda").manual_seed(321)
    copies = [_device_weights(tg, torch, 0, N, K, g) for _ in range(ncopies)]
    L = tg.lib()
    out = {}
    for M in (1, 4, 16):  # the same calls without the branch
        x = torch.randn(M, K, device="cuda").bfloat16()
        y = torch.empty(M, N, device="cuda", dtype=torch.bfloat16)
        calls = [(x.data_ptr(), wq.data_ptr(), d.data_ptr(), y.data_ptr(), M, N, K, tg.OUT_BF16, None, 0)
                 for (wq, d) in copies]
        t = _graph_per_call(tg, torch, calls, L.tgemm_q2)
        out[f"r0_m{M}"] = {"us_per_call": t * 1e6, "weight_gbs": wbytes / t / 1e9}
    for r in (4, 32, 64):
        a = (torch.randn(r, K, device="cuda") * 1e-3).bfloat16()
        b = (torch.randn(N, r, device="cuda") * 1e-3).bfloat16()
        for M in (1, 4, 16):
            x = torch.randn(M, K, device="cuda").bfloat16()
            y = torch.empty(M, N, device="cuda", dtype=torch.bfloat16)
            ws = torch.empty(max(tg.workspace_size(tg.OP_Q2_LORA, M, N, K, r), 256),
                             dtype=torch.uint8, device="cuda")
            calls = [(x.data_ptr(), wq.data_ptr(), d.data_ptr(), a.data_ptr(), b.data_ptr(), r,
                      y.data_ptr(), M, N, K, tg.OUT_BF16, ws.data_ptr(), ws.numel())
                     for (wq, d) in copies]
            t = _graph_per_call(tg, torch, calls, L.tgemm_q2_lora)
            out[f"r{r}_m{M}"] = {"us_per_call": t * 1e6, "weight_gbs": wbytes / t / 1e9}
    del copies
    torch.cuda.empty_cache()
    return out


def kernel_tour(tg, torch):
    """Every kernel of the library once, each call inside an NVTX range 'kernels' after two
    warm-up calls outside it; inputs are drawn outside the ranges and freed after each
    workload (a small device footprint for profilers that replay kernels)."""
    import torch.cuda.nvtx as nvtx
    g = torch.Generator(device="cuda").manual_seed(99)
    dev = "cuda"

    def once(label, fn):
        for _ in range(2):
            fn()
        torch.cuda.synchronize()
        nvtx.range_push("kernels")
        fn()
        nvtx.range_pop()
        torch.cuda.synchronize()
        print(f"kernels: {label}", flush=True)

    def codes(N, K, hi):
        return torch.randint(0, hi, (N, K), dtype=torch.uint8, device=dev, generator=g)

    # load-time packing and the dequantization hooks
    c2, s2 = codes(9216, 3072, 3), (torch.rand(9216, 24, device=dev, generator=g) * 0.02).half().float()
    once("q2_pack 9216x3072", lambda: tg.q2_pack(c2, s2))
    c4 = codes(9728, 2560, 16)
    s4 = (torch.rand(9728, 40, device=dev, generator=g) * 0.01).half().float()
    z4 = (7 + torch.rand(9728, 40, device=dev, generator=g)).half().float()
    once("q4_pack 9728x2560", lambda: tg.q4_pack(c4, s4, z4))
    wgl = torch.randint(0, 256, (768, 3072), dtype=torch.uint8, device=dev, generator=g)
    sgl = (torch.rand(3072, 48, device=dev, generator=g) * 0.02).half().float()
    once("q2_from_gemlite 3072x3072 g=64", lambda: tg.q2_from_gemlite(wgl, sgl, -sgl, 64))
    wq2, d2, _ = tg.q2_pack(c2, s2)
    wq4, sz4, _ = tg.q4_pack(c4, s4, z4)
    once("q2_dequant 9216x3072", lambda: tg.q2_dequant(wq2, d2))
    once("q4_dequant 9728x2560", lambda: tg.q4_dequant(wq4, sz4))
    del c2, s2, c4, s4, z4, wgl, sgl

    def x(M, K):
        return torch.randn(M, K, device=dev, generator=g).bfloat16()

    prev = tg.set_path(tg.PATH_AUTO)
    try:
        # tensor-core path: activation prep + the tcgen05 kernel
        x1 = x(1536, 3072)
        once("tgemm_q2 1536x9216x3072", lambda: tg.gemm_q2(x1, wq2, d2))
        a = (torch.randn(32, 3072, device=dev, generator=g) * 1e-3).bfloat16()
        b = (torch.randn(9216, 32, device=dev, generator=g) * 1e-3).bfloat16()
        once("tgemm_q2_lora r=32 1536x9216x3072", lambda: tg.gemm_q2_lora(x1, wq2, d2, a, b))
        xe = x(512, 2560)
        once("tgemm_q4 512x9728x2560", lambda: tg.gemm_q4(xe, wq4, sz4))
        cw = codes(3072, 3072, 3)
        cs = (torch.rand(3072, 24, device=dev, generator=g) * 0.02).half().float()
        wa, da, _ = tg.q2_pack(cw, cs)
        cw2 = codes(3072, 12288, 3)
        cs2 = (torch.rand(3072, 96, device=dev, generator=g) * 0.02).half().float()
        wb, db, _ = tg.q2_pack(cw2, cs2)
        del cw, cs, cw2, cs2
        xa, xb = x(1536, 3072), x(1536, 12288)
        once("tgemm_q2_dual 1536x3072x(3072+12288)", lambda: tg.gemm_q2_dual(xa, wa, da, xb, wb, db))
        # small-M path: the per-pass kernel (also with the branch and two inputs), the
        # streaming kernel
        tg.set_path(tg.PATH_SMALL_M_PASS)
        x16 = x(16, 3072)
        once("gemv pass Q2 M=16 3072x3072", lambda: tg.gemm_q2(x16, wa, da))
        x4e = x(4, 2560)
        once("gemv pass 4-bit M=4 9728x2560", lambda: tg.gemm_q4(x4e, wq4, sz4))
        x4 = x(4, 3072)
        once("gemv pass Q2 branch r=32 M=4 9216x3072", lambda: tg.gemm_q2_lora(x4, wq2, d2, a, b))
        x4b = x(4, 12288)
        once("gemv pass Q2 two inputs M=4 3072x(3072+12288)", lambda: tg.gemm_q2_dual(x4, wa, da, x4b, wb, db))
        tg.set_path(tg.PATH_SMALL_M_STREAM)
        x1q = x(1, 3072)
        once("gemv stream Q2 M=1 9216x3072", lambda: tg.gemm_q2(x1q, wq2, d2))
        x1e = x(1, 2560)
        once("gemv stream 4-bit M=1 9728x2560", lambda: tg.gemm_q4(x1e, wq4, sz4))
    finally:
        tg.set_path(prev)
    assert tg.device_error() == 0


def main():
    args = parse_args()
    if args.kernels:
        import torch

        import bit_weight_quantized_tgemm_b200 as tg
        kernel_tour(tg, torch)
        return 0
    world, rank, local = (1, 0, 0)
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        reference_arm(args, world, rank)
        return 0
    world, rank, local = dist_setup(args)
    try:
        ours(args, world, rank, local)
    finally:
        dist_done(world)
    return 0


if __name__ == "__main__":
    sys.exit(main())
