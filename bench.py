"""Benchmark of the fused attention forward on B200 (one JSON line on rank 0).

Step = one pass of the non-causal d=128 prefill sweep over a 16k-token batch
(H=16; seq 512, 1024, 2048, 4096 with B = 16384/seq), each shape one
``attn_fwd`` call through the C ABI, inputs resident in HBM, L2 flushed (a
256 MiB write) before every call.  ``value`` is TFLOP/s = algorithmic FLOPs
(4*B*H*S*S*d per shape) / summed CUDA-event time of the calls, max over ranks.
The other workloads (causal sweep, GQA long sequence, split-KV decode) are
measured in the same run and reported under ``breakdown``.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
For N > 1 launch under torchrun; every rank runs the same per-GPU work
(weak scaling, no collective on the data path).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from scaled_dot_product_fa2_b200 import inputs  # noqa: E402

HEADLINE = inputs.PREFILL_NONCAUSAL
WORKLOAD_NAME = ("prefill non-causal d=128 H=16 seq {512,1024,2048,4096} B=16384/seq "
                 "(one call per shape per step)")
METRIC = "attn fwd TFLOP/s (bf16, d=128) and decode KV GB/s, as fraction of B200 roofline"
L2_FLUSH_BYTES = 256 << 20
# After each flush a short device-side spin keeps the GPU busy while the host
# enqueues the timed call, so the events bracket device work only (no idle gap
# from host-side launch overhead).
HOST_SLACK_CYCLES = 200_000
DECODE_BATCH = 12
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "prefill_traffic.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-breakdown", action="store_true", help="time the headline step only")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile", metavar="WORKLOAD", default=None,
                    help="run a few untimed calls of one named workload (for ncu captures) and exit")
    ap.add_argument("--profile-calls", type=int, default=3)
    return ap.parse_args()


# ------------------------------------------------------------------ helpers

def load_peaks():
    if os.path.exists(PEAKS_FILE):
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


#: the sources the prefill kernel is compiled from (its device code and the
#: PTX wrappers it uses); the recorded DRAM traffic is valid while they are unchanged
PREFILL_KERNEL_SOURCES = ("prefill.cuh", "ptx.cuh")


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "scaled_dot_product_fa2_b200", "csrc")
    for name in PREFILL_KERNEL_SOURCES:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def measured_traffic(workload_name: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel source; else None."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    with open(TRAFFIC_FILE) as f:
        t = json.load(f)
    if t.get("kernel_source_hash") != kernel_source_hash():
        return None
    return t.get("per_launch_bytes", {}).get(workload_name)


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu_index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]
        return False

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def setup_dist(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device(f"cuda:{local}"))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(world, x: float) -> float:
    """Largest x over all ranks (the slowest rank's time)."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(world: int, flops_per_rank_step: float, steps: int, max_ms: float) -> float:
    """Whole-job TFLOP/s: every rank did the same per-GPU work in at most max_ms."""
    return world * flops_per_rank_step * steps / (max_ms / 1e3) / 1e12


# ------------------------------------------------------------------ CPU oracle baseline

class CpuOracleSample:
    """Times the oracle (as it stands) on bounded random row samples of a
    workload, on all host cores."""

    def __init__(self, w):
        import numpy as np
        self.np = np
        self.w = w
        q, k, v = inputs.workload_inputs(w)
        self.qd, self.kd, self.vd = q.double().numpy(), k.double().numpy(), v.double().numpy()
        self.threads = os.cpu_count() or 1
        self.rng = np.random.default_rng(0)
        self.total_rows = w.B * w.Hq * w.Sq
        self.per_row = None

    def _flops(self, rows):
        w, np = self.w, self.np
        i = rows % w.Sq
        if w.causal == inputs.CAUSAL_TOP_LEFT:
            keys = np.minimum(i + 1, w.Sk)
        elif w.causal == inputs.CAUSAL_BOTTOM_RIGHT:
            keys = np.clip(i + w.Sk - w.Sq + 1, 0, w.Sk)
        else:
            keys = np.full_like(i, w.Sk)
        return float(4.0 * w.d * keys.sum())

    def _run(self, n):
        import oracle
        rows = self.np.sort(self.rng.choice(self.total_rows, size=n, replace=False))
        t0 = time.perf_counter()
        oracle.attn_rows(self.qd, self.kd, self.vd, self.w.eff_scale, self.w.causal, rows, nthreads=self.threads)
        return rows, time.perf_counter() - t0

    def sample(self, target_s: float):
        """Returns (TFLOP/s, threads, description, seconds) for about target_s of work."""
        if self.per_row is None:
            n = min(self.total_rows, 8 * self.threads)
            _, dt = self._run(n)
            self.per_row = dt / n
        n = int(min(self.total_rows, max(self.threads, target_s / max(self.per_row, 1e-9))))
        rows, dt = self._run(n)
        self.per_row = dt / n
        tflops = self._flops(rows) / dt / 1e12
        desc = (f"{n} random query rows of {self.w.name} (of {self.total_rows}), fp64 oracle on "
                f"{self.threads} threads, {dt:.1f} s")
        return tflops, self.threads, desc, dt


def oracle_per_config(target_s: float = 1.5):
    """The oracle as it stands on every configuration: the tiny and decode
    workloads in full, each prefill shape and the GQA workload on a seeded
    random row sample whose measured per-row time is scaled to the full row
    count (labelled "extrapolated")."""
    import oracle
    threads = os.cpu_count() or 1
    out = {}
    for w in [inputs.TINY] + list(inputs.DECODE):
        q, k, v = inputs.workload_inputs(w)
        qd, kd, vd = q.double().numpy(), k.double().numpy(), v.double().numpy()
        t0 = time.perf_counter()
        oracle.attn_fwd(qd, kd, vd, w.eff_scale, w.causal, nthreads=threads)
        dt = time.perf_counter() - t0
        rate = (w.flops() / dt / 1e12) if not w.decode else None
        entry = {"full_s": round(dt, 4), "how": "measured on the whole workload", "threads": threads}
        if w.decode:
            entry["gbs"] = round(w.decode_bytes() / dt / 1e9, 3)
        else:
            entry["tflops"] = round(rate, 6)
        out[w.name] = entry
    for w in list(inputs.PREFILL_NONCAUSAL) + list(inputs.PREFILL_CAUSAL) + [inputs.GQA_LONG]:
        sampler = CpuOracleSample(w)
        tf, cores, desc, dt = sampler.sample(target_s=target_s)
        full_s = sampler.per_row * sampler.total_rows
        out[w.name] = {"tflops": round(tf, 6), "full_s": round(full_s, 2), "threads": cores,
                       "how": f"extrapolated from {desc}"}
        del sampler
    return out


# ------------------------------------------------------------------ GPU timing

class GpuPrefill:
    def __init__(self, w, rank: int):
        q, k, v = inputs.make_qkv(w.B, w.Hq, w.Hkv, w.Sq, w.Sk, w.d, w.seed + 7919 * rank)
        self.w = w
        self.host = [t.pin_memory() for t in (q, k, v)]
        self.q, self.k, self.v = (t.cuda() for t in (q, k, v))
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty((w.B, w.Hq, w.Sq), dtype=torch.float32, device="cuda")
        self.o_host = torch.empty(self.o.shape, dtype=self.o.dtype).pin_memory()
        self.lse_host = torch.empty(self.lse.shape, dtype=torch.float32).pin_memory()

    def run(self):
        import scaled_dot_product_fa2_b200 as sdpa
        sdpa.attn_fwd(self.q, self.k, self.v, causal=self.w.causal, scale=self.w.scale, out=self.o, lse=self.lse)

    def copy_inputs(self):
        """q, k, v from pinned host memory, on the current stream."""
        self.q.copy_(self.host[0], non_blocking=True)
        self.k.copy_(self.host[1], non_blocking=True)
        self.v.copy_(self.host[2], non_blocking=True)

    def copy_outputs(self):
        """o and lse back to pinned host memory, on the current stream."""
        self.o_host.copy_(self.o, non_blocking=True)
        self.lse_host.copy_(self.lse, non_blocking=True)

    def h2d_bytes(self):
        return sum(t.numel() * t.element_size() for t in self.host)

    def d2h_bytes(self):
        return self.o.numel() * 2 + self.lse.numel() * 4


class GpuPrefillVarlen(GpuPrefill):
    """Causal prefill over padded sequences of seeded lengths (query and key
    lengths equal per sequence); FLOPs count the valid causal work only."""

    def __init__(self, w, rank: int):
        super().__init__(w, rank)
        self.lens = inputs.prefill_lengths(w)
        self.seqlens = torch.tensor(self.lens, dtype=torch.int32, device="cuda")

    def run(self):
        import scaled_dot_product_fa2_b200 as sdpa
        sdpa.attn_fwd_varlen(self.q, self.k, self.v, self.seqlens, self.seqlens, causal=self.w.causal,
                             scale=self.w.scale, out=self.o, lse=self.lse)

    def flops(self):
        return sum(2.0 * self.w.Hq * L * L * self.w.d for L in self.lens)


class GpuPrefillBias(GpuPrefill):
    """A prefill workload with an additive bias shared by all heads and batches
    ([1, 1, S, S] bf16, seeded N(0, 1))."""

    def __init__(self, w, rank: int):
        super().__init__(w, rank)
        g = torch.Generator().manual_seed(w.seed + 99)
        self.bias = torch.randn((1, 1, w.Sq, w.Sk), generator=g).bfloat16().cuda()

    def run(self):
        import scaled_dot_product_fa2_b200 as sdpa
        sdpa.attn_fwd(self.q, self.k, self.v, causal=self.w.causal, scale=self.w.scale, out=self.o, lse=self.lse,
                      bias=self.bias)


class GpuDecode:
    def __init__(self, w, rank: int, copies: int = 3):
        import scaled_dot_product_fa2_b200 as sdpa
        self.w = w
        q, k, v = inputs.make_qkv(w.B, w.Hq, w.Hkv, w.Sq, w.Sk, w.d, w.seed + 7919 * rank)
        self.q = q.cuda()
        # several cache copies (3 x 256 MiB > L2) so each call streams from HBM
        self.kv = []
        for c in range(copies):
            kk, vv = k.cuda(), v.cuda()
            if c:
                kk = kk.clone()
                vv = vv.clone()
            self.kv.append((kk, vv))
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty((w.B, w.Hq, w.Sq), dtype=torch.float32, device="cuda")
        self.ws = sdpa.decode_workspace(self.q, self.kv[0][0])
        self.i = 0

    def run(self):
        import scaled_dot_product_fa2_b200 as sdpa
        k, v = self.kv[self.i % len(self.kv)]
        self.i += 1
        sdpa.attn_decode_splitkv(self.q, k, v, causal=self.w.causal, scale=self.w.scale, workspace=self.ws,
                                 out=self.o, lse=self.lse)


class GpuDecodeVarlen(GpuDecode):
    """The decode workload over caches whose valid length differs per batch
    (seeded lengths in [1, capacity], held on the device)."""

    def __init__(self, w, rank: int, copies: int = 3):
        super().__init__(w, rank, copies)
        self.lens = inputs.decode_lengths(w)
        self.seqlens = torch.tensor(self.lens, dtype=torch.int32, device="cuda")

    def run(self):
        import scaled_dot_product_fa2_b200 as sdpa
        k, v = self.kv[self.i % len(self.kv)]
        self.i += 1
        sdpa.attn_decode_splitkv_varlen(self.q, k, v, self.seqlens, causal=self.w.causal, scale=self.w.scale,
                                        workspace=self.ws, out=self.o, lse=self.lse)

    def valid_bytes(self):
        w = self.w
        kv = sum(2 * w.Hkv * L * w.d * 2 for L in self.lens)
        return kv + 2 * w.B * w.Hq * w.Sq * w.d * 2 + w.B * w.Hq * w.Sq * 4


class GpuBackward(GpuPrefill):
    """attn_bwd on a prefill workload, with the forward's o and lse and a
    seeded dO resident on the device."""

    def __init__(self, w, rank: int):
        import scaled_dot_product_fa2_b200 as sdpa
        super().__init__(w, rank)
        sdpa.attn_fwd(self.q, self.k, self.v, causal=w.causal, scale=w.scale, out=self.o, lse=self.lse)
        g = torch.Generator().manual_seed(w.seed + 4242 + 7919 * rank)
        self.dout = torch.randn(self.q.shape, generator=g).bfloat16().cuda()
        self.dq = torch.empty_like(self.q)
        self.dk = torch.empty_like(self.k)
        self.dv = torch.empty_like(self.v)
        self.ws = torch.empty(max(16, sdpa.bwd_workspace_size(w.B, w.Hq, w.Sq)), dtype=torch.uint8, device="cuda")

    def run(self):
        import scaled_dot_product_fa2_b200 as sdpa
        sdpa.attn_bwd(self.q, self.k, self.v, self.o, self.lse, self.dout, causal=self.w.causal, scale=self.w.scale,
                      dq=self.dq, dk=self.dk, dv=self.dv, workspace=self.ws)


class GpuRopeAppend:
    """The step before a decode: split the packed QKV, rotate q and k, append
    k and v to the cache (one launch of the rotary/append kernel)."""

    def __init__(self, w, rank: int):
        self.w = w
        past = [0] * w.B if w.Sq > 1 else None
        packed, kc, vc, past_lens = inputs.make_rope_inputs(w.B, w.Sq, w.Hq, w.Hkv, w.d, w.Sk,
                                                            w.seed + 7919 * rank, past_lens=past)
        cos, sin = inputs.rope_tables(w.Sk, w.d)
        self.packed, self.kc, self.vc = packed.cuda(), kc.cuda(), vc.cuda()
        self.cos, self.sin, self.past = cos.cuda(), sin.cuda(), past_lens.cuda()
        self.q = torch.empty((w.B, w.Hq, w.Sq, w.d), dtype=torch.bfloat16, device="cuda")
        self.tot = torch.empty(w.B, dtype=torch.int32, device="cuda")

    def run(self):
        import scaled_dot_product_fa2_b200 as sdpa
        sdpa.attn_rope_append(self.packed, self.cos, self.sin, self.past, self.kc, self.vc, self.w.Hq, self.w.Hkv,
                              q_out=self.q, total_lens=self.tot)


def timed_calls(fns, flush, reps: int, warmup: int):
    """Per-call CUDA-event times (ms) on the current stream, L2 flushed before each call."""
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        for fn in fns:
            flush()
            fn()
    torch.cuda.synchronize()
    times = [[] for _ in fns]
    for _ in range(reps):
        for i, fn in enumerate(fns):
            flush()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            times[i].append((a, b))
    torch.cuda.synchronize()
    return [[a.elapsed_time(b) for a, b in ts] for ts in times]


def main():
    args = parse_args()
    if args.impl == "reference":
        # the CPU oracle arm needs no process group: rank 0 runs, the others exit
        return run_reference(args, int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")))
    world, rank, local = setup_dist(args)
    if args.profile:
        return run_profile_case(args)
    import scaled_dot_product_fa2_b200 as sdpa
    from scaled_dot_product_fa2_b200 import build
    if rank == 0:
        build.build()
    barrier(world)
    peaks, peaks_kind = load_peaks()

    flush_buf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    def flush():
        flush_buf.fill_(1)
        torch.cuda._sleep(HOST_SLACK_CYCLES)

    shapes = [GpuPrefill(w, rank) for w in HEADLINE]
    flops_step = sum(s.w.flops() for s in shapes)

    # warm-up (untimed)
    for _ in range(max(args.warmup, 3)):
        for s in shapes:
            flush()
            s.run()
    sdpa.check_device_error()

    # ---- timed region: exactly K steps, barrier + synchronize on both sides
    stream = torch.cuda.current_stream()
    events = []
    with ClockSampler(local) as clocks:
        barrier(world)
        torch.cuda.synchronize()
        wall0 = time.perf_counter()
        for _ in range(args.steps):
            for s in shapes:
                flush()
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record(stream)
                s.run()
                b.record(stream)
                events.append((s.w.name, a, b))
        torch.cuda.synchronize()
        barrier(world)
        wall = time.perf_counter() - wall0
    sdpa.check_device_error()
    per_shape_ms = {}
    for name, a, b in events:
        per_shape_ms.setdefault(name, []).append(a.elapsed_time(b))
    kernel_ms = sum(sum(v) for v in per_shape_ms.values())
    kernel_ms = max_over_ranks(world, kernel_ms)
    wall = max_over_ranks(world, wall)
    ms_per_step = kernel_ms / args.steps
    value = weak_scaling_value(world, flops_step, args.steps, kernel_ms)

    # ---- end to end through the public API with host buffers (pinned), same metric.
    # Every step copies each shape's q, k, v in, runs the forward and reads o
    # and lse back, as a serving loop would: the input copies, the forwards and
    # the read-backs go to three streams, so the two copy directions and the
    # compute of different shapes overlap (each shape's buffers are reused only
    # after their previous forward and read-back are done).
    h2d_s, d2h_s = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in shapes]    # inputs of shape i on the device
    ev_fwd = [torch.cuda.Event() for _ in shapes]   # forward of shape i done (inputs free, outputs ready)
    ev_out = [torch.cuda.Event() for _ in shapes]   # outputs of shape i read back (outputs free)

    def e2e_step(first: bool):
        for i, s in enumerate(shapes):
            with torch.cuda.stream(h2d_s):
                if not first:
                    h2d_s.wait_event(ev_fwd[i])
                s.copy_inputs()
                ev_in[i].record(h2d_s)
            stream.wait_event(ev_in[i])
            if not first:
                stream.wait_event(ev_out[i])
            s.run()
            ev_fwd[i].record(stream)
            with torch.cuda.stream(d2h_s):
                d2h_s.wait_event(ev_fwd[i])
                s.copy_outputs()
                ev_out[i].record(d2h_s)

    for it in range(2):
        e2e_step(first=(it == 0))
    torch.cuda.synchronize()
    barrier(world)
    e_a = torch.cuda.Event(enable_timing=True)
    e_b = torch.cuda.Event(enable_timing=True)
    e_a.record(stream)
    h2d_s.wait_event(e_a)
    d2h_s.wait_event(e_a)
    for _ in range(args.steps):
        e2e_step(first=False)
    stream.wait_stream(h2d_s)
    stream.wait_stream(d2h_s)
    e_b.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(world, e_a.elapsed_time(e_b))
    e2e_value = weak_scaling_value(world, flops_step, args.steps, e2e_ms)
    h2d = sum(s.h2d_bytes() for s in shapes)
    d2h = sum(s.d2h_bytes() for s in shapes)

    # ---- roofline of the dominant kernel (prefill_kernel, the only kernel of the step)
    peak_tf = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    achieved = flops_step * args.steps / (sum(sum(v) for v in per_shape_ms.values()) / 1e3) / 1e12
    big = HEADLINE[-1].name
    traffic = measured_traffic(big)
    roofline = {"bound": "tensor", "kernel": "prefill_kernel<128,5>", "achieved": round(achieved, 1),
                "peak": peak_tf, "unit": "TFLOP/s", "frac": round(achieved / peak_tf, 4),
                "peak_kind": f"{peaks_kind} bf16 dense (burst)", "traffic": traffic,
                "traffic_workload": big}

    breakdown = {}
    for s in shapes:
        ts = per_shape_ms[s.w.name]
        med = statistics.median(ts)
        breakdown[s.w.name] = {"ms": round(med, 4), "tflops": round(s.w.flops() / med / 1e9, 1),
                               "frac": round(s.w.flops() / med / 1e9 / peak_tf, 4)}
    del shapes
    if not args.no_breakdown:
        breakdown.update(measure_breakdown(flush, peak_tf, float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])),
                                           rank))
    sdpa.check_device_error()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = sweep_oracle_sample(target_s=8.0)
        if not args.no_breakdown:
            for name, entry in oracle_per_config().items():
                breakdown.setdefault(name, {})["oracle"] = entry

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
            "wall_ms_per_step": round(wall * 1e3 / args.steps, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded randn N(0,1), rounded to bf16)",
            "config": {"workload": WORKLOAD_NAME,
                       "global_batch_tokens": 16384 * 4 * world, "seq_len": [w.Sq for w in HEADLINE],
                       "heads": 16, "head_dim": 128, "causal": False, "parallelism": f"replicas x{world}",
                       "l2": "flushed (256 MiB write) before every call",
                       "host_slack": "device spin after each flush so the events bracket device time only"},
            "e2e": {"value": round(e2e_value, 2), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": len(HEADLINE) * args.steps,
            "roofline": roofline,
            "cpu_baseline": cpu,
            "clocks": clocks.summary(),
            "breakdown": breakdown,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def measure_breakdown(flush, peak_tf, hbm_gbs, rank, reps: int = 10):
    import scaled_dot_product_fa2_b200 as sdpa
    out = {}
    # the tiny causal workload (B=1, H=2, S=128, d=64): a launch-latency figure
    s = GpuPrefill(inputs.TINY, rank)
    ms = statistics.median(timed_calls([s.run], flush, reps, 3)[0])
    out[inputs.TINY.name] = {"ms": round(ms, 4), "tflops": round(inputs.TINY.flops() / ms / 1e9, 3)}
    del s
    for w in inputs.PREFILL_CAUSAL + [inputs.GQA_LONG]:
        s = GpuPrefill(w, rank)
        ms = statistics.median(timed_calls([s.run], flush, reps, 3)[0])
        tf = w.flops() / ms / 1e9
        out[w.name] = {"ms": round(ms, 4), "tflops": round(tf, 1), "frac": round(tf / peak_tf, 4)}
        del s
    # the non-causal seq-2048 shape with an additive bias shared by all heads
    # and batches ([1, 1, S, S] bf16, 8 MiB: it stays in L2, so this measures
    # the bias path's compute cost)
    wb = inputs.BY_NAME["prefill_noncausal_s2048"]
    sb = GpuPrefillBias(wb, rank)
    ms = statistics.median(timed_calls([sb.run], flush, reps, 3)[0])
    tf = wb.flops() / ms / 1e9
    out[wb.name + "_bias"] = {"ms": round(ms, 4), "tflops": round(tf, 1), "frac": round(tf / peak_tf, 4),
                              "bias": "[1, 1, S, S] bf16"}
    del sb

    sv = GpuPrefillVarlen(inputs.PREFILL_VARLEN, rank)
    ms = statistics.median(timed_calls([sv.run], flush, reps, 3)[0])
    tf = sv.flops() / ms / 1e9
    out[inputs.PREFILL_VARLEN.name] = {"ms": round(ms, 4), "tflops": round(tf, 1), "frac": round(tf / peak_tf, 4),
                                       "lengths": sv.lens}
    del sv

    # Decode streams 268 MB per call from one of three rotating cache copies
    # (768 MiB > L2), so no call finds its K/V in L2.  No write flush here: a
    # flush leaves up to an L2's worth of dirty lines that the decode's reads
    # would write back inside the timed call.
    def slack_only():
        torch.cuda._sleep(HOST_SLACK_CYCLES)

    # The calls are timed in batches of DECODE_BATCH between one pair of events
    # (a ~50 us call is only a few ticks of the event clock).
    for w in inputs.DECODE:
        s = GpuDecode(w, rank)

        def batch(s=s):
            for _ in range(DECODE_BATCH):
                s.run()

        ms = statistics.median(timed_calls([batch], slack_only, reps, 2)[0]) / DECODE_BATCH
        gbs = w.decode_bytes() / ms / 1e6
        out[w.name] = {"ms": round(ms, 4), "gbs": round(gbs, 1), "frac": round(gbs / hbm_gbs, 4),
                       "splits": sdpa.decode_num_splits(w.B, w.Hq, w.Hkv, w.Sq, w.Sk, w.d),
                       "launches_per_call": 2}
        del s
    for w in inputs.DECODE:
        s = GpuDecodeVarlen(w, rank)

        def batch(s=s):
            for _ in range(DECODE_BATCH):
                s.run()

        ms = statistics.median(timed_calls([batch], slack_only, reps, 2)[0]) / DECODE_BATCH
        gbs = s.valid_bytes() / ms / 1e6
        out[w.name + "_varlen"] = {"ms": round(ms, 4), "gbs": round(gbs, 1), "frac": round(gbs / hbm_gbs, 4),
                                   "lengths": s.lens, "launches_per_call": 2}
        del s
    # backward pass at seq 4096 (B=4, H=16, d=128): the forward's o, lse are
    # computed once outside the timing; FLOPs = 2.5 x the forward's (the five
    # matmuls S = QK^T, dP = dO V^T, dV, dK, dQ), halved for causal
    for name in ("prefill_noncausal_s4096", "prefill_causal_s4096"):
        s = GpuBackward(inputs.BY_NAME[name], rank)
        ms = statistics.median(timed_calls([s.run], flush, reps, 3)[0])
        tf = 2.5 * s.w.flops() / ms / 1e9
        out["bwd_" + name.replace("prefill_", "")] = {"ms": round(ms, 4), "tflops": round(tf, 1),
                                                       "frac": round(tf / peak_tf, 4), "launches_per_call": 3}
        del s
    # rotary/append over a 4096-token prompt: 805 MB moved per call (> L2), no flush needed
    s = GpuRopeAppend(inputs.ROPE_PROMPT, rank)
    ms = statistics.median(timed_calls([s.run], slack_only, reps, 3)[0])
    gbs = inputs.rope_bytes(s.w) / ms / 1e6
    out[s.w.name] = {"ms": round(ms, 4), "gbs": round(gbs, 1), "frac": round(gbs / hbm_gbs, 4),
                     "launches_per_call": 1}
    del s
    # one new token per sequence: 393 KB per call, a latency figure (L2-resident)
    s = GpuRopeAppend(inputs.ROPE_DECODE, rank)

    def batch(s=s):
        for _ in range(DECODE_BATCH):
            s.run()

    ms = statistics.median(timed_calls([batch], slack_only, reps, 2)[0]) / DECODE_BATCH
    out[s.w.name] = {"ms": round(ms, 4), "gbs": round(inputs.rope_bytes(s.w) / ms / 1e6, 1),
                     "launches_per_call": 1}
    del s
    torch.cuda.empty_cache()
    return out


def run_profile_case(args):
    """A few back-to-back calls of one workload with an L2 flush before each:
    the small, self-terminating command that ncu captures are taken on."""
    import scaled_dot_product_fa2_b200 as sdpa
    rope = {inputs.ROPE_PROMPT.name: inputs.ROPE_PROMPT, inputs.ROPE_DECODE.name: inputs.ROPE_DECODE}
    flush_buf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    if args.profile in rope:
        w = rope[args.profile]
        runner = GpuRopeAppend(w, 0)
    elif args.profile.startswith("bwd_"):
        # the backward pass of a prefill workload, e.g. bwd_prefill_noncausal_s4096
        w = inputs.BY_NAME[args.profile[len("bwd_"):]]
        runner = GpuBackward(w, 0)
    elif args.profile == inputs.PREFILL_VARLEN.name:
        w = inputs.PREFILL_VARLEN
        runner = GpuPrefillVarlen(w, 0)
    elif args.profile.endswith("_varlen"):
        # a decode workload over its seeded per-batch lengths, e.g. decode_sq4_varlen
        w = inputs.BY_NAME[args.profile[:-len("_varlen")]]
        runner = GpuDecodeVarlen(w, 0)
    elif args.profile.endswith("_bias"):
        # a prefill workload with the [1, 1, S, S] bias, e.g. prefill_noncausal_s2048_bias
        w = inputs.BY_NAME[args.profile[:-len("_bias")]]
        runner = GpuPrefillBias(w, 0)
    else:
        w = inputs.BY_NAME[args.profile]
        runner = GpuDecode(w, 0) if w.decode else GpuPrefill(w, 0)
    for _ in range(args.profile_calls):
        flush_buf.fill_(1)
        torch.cuda._sleep(HOST_SLACK_CYCLES)
        runner.run()
    sdpa.check_device_error()
    print(f"profile case {w.name}: {args.profile_calls} calls ok", flush=True)


def sweep_oracle_sample(target_s: float):
    """The oracle on a bounded sample of the headline workload itself: seeded
    random query rows of every shape of the sweep, about target_s seconds in
    all, split over the shapes in proportion to their FLOPs; TFLOP/s = the
    sampled rows' algorithmic FLOPs / the time taken."""
    total = sum(w.flops() for w in HEADLINE)
    fl = dt = 0.0
    nrows = []
    cores = os.cpu_count() or 1
    for w in HEADLINE:
        sampler = CpuOracleSample(w)
        t_share = target_s * w.flops() / total
        if sampler.per_row is None:
            n = min(sampler.total_rows, 8 * sampler.threads)
            _, d0 = sampler._run(n)
            sampler.per_row = d0 / n
        n = int(min(sampler.total_rows, max(sampler.threads, t_share / max(sampler.per_row, 1e-9))))
        rows, d = sampler._run(n)
        fl += sampler._flops(rows)
        dt += d
        nrows.append(f"{n} of {w.name}")
        cores = sampler.threads
        del sampler
    desc = (f"seeded random query rows of every shape of the sweep ({', '.join(nrows)}), fp64 oracle on "
            f"{cores} threads, {dt:.1f} s")
    return {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": desc,
            "seconds": round(dt, 2)}


def run_reference(args, world, rank):
    """The reference arm: the fp64 oracle as it stands, on the host cores, on
    a bounded sample of the same workload as this benchmark's own arm (every
    shape of the non-causal sweep), rank 0 only."""
    if rank != 0:
        return
    vals = []
    per_step = max(1.0, 60.0 / max(1, args.warmup + args.steps))
    for i in range(args.warmup + args.steps):
        c = sweep_oracle_sample(target_s=per_step)
        if i >= args.warmup:
            vals.append(c)
    tf = statistics.median(c["value"] for c in vals)
    last = vals[-1]
    line = {"impl": "reference", "metric": METRIC, "value": round(tf, 6), "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * statistics.median(c["seconds"] for c in vals), 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded randn N(0,1), rounded to bf16)",
            "config": {"workload": WORKLOAD_NAME + " (each step a seeded row sample of it)"},
            "cpu_baseline": {"value": round(tf, 6), "unit": "TFLOP/s", "cores": last["cores"],
                             "kind": "oracle", "sample": last["sample"]},
            "e2e": {"value": round(tf, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
