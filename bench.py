#!/usr/bin/env python
"""Throughput of exact causal attention, forward + backward, bf16, on B200.

One step is the whole hot path over one batch: ``fa_fwd`` (O, LSE), then the
three backward stages ``fa_bwd_prep`` (D, padded LSE, zeroed dQ accumulator),
``fa_bwd_main`` (recompute, dK, dV, dQ accumulation) and ``fa_bwd_dq``
(dQ to bf16), on B=2, Hq=Hkv=32, N=8192, d=128, causal, synthetic N(0,1)
inputs rounded to bf16. FLOPs follow the usual convention: forward 4*B*Hq*N^2*d, halved when
causal; backward 2.5 times the forward.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line on rank 0. ``value`` is the whole-job TFLOP/s with
inputs resident in HBM (max over ranks of the device time); ``e2e`` is the
same metric measured through the C ABI with pinned host buffers, including
the host-to-device copies of Q, K, V, dO and the device-to-host copies of O,
LSE, dQ, dK, dV. ``--impl reference`` times the fp64 CPU oracle on a bounded
sample of the same workload instead.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "attention fwd / fwd+bwd TFLOP/s, bf16 causal N=8k d=128, % of B200 BF16 peak"
SHAPE = dict(B=2, Hq=32, Hkv=32, N=8192, d=128)
CAUSAL = True
SEED = 1003
WORKLOAD_NAME = "causal bf16 attention forward+backward, B=2 Hq=32 Hkv=32 N=8192 d=128"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

SPEC_BF16_TFLOPS = 2250.0  # B200 dense bf16 tensor peak, vendor figure (context for pct_of_spec)

# Counters of one ncu capture per kernel, with the hash of the kernel sources
# they were taken on: DRAM bytes per launch (dram__bytes_read.sum +
# dram__bytes_write.sum) and sm__pipe_tensor_cycles_active (% of peak). They
# are reported only while the sources still hash to the same value.
PROFILED = {
    # ncu --metrics gpu__time_duration.sum,dram__bytes_read.sum,dram__bytes_write.sum,
    #     sm__pipe_tensor_cycles_active.avg.pct_of_peak_sustained_active at the benchmark shape
    "bwd_main": {"src": "37c76f4c2b2b572a", "dram_bytes": 825_743_872 + 498_451_456, "tensor_pipe_active_pct": 48.71},
    "fwd": {"src": "37c76f4c2b2b572a", "dram_bytes": 404_009_984 + 116_269_056, "tensor_pipe_active_pct": 51.60},
}


def fwd_flops(B, Hq, N, d, causal):
    f = 4.0 * B * Hq * N * N * d
    return f / 2 if causal else f


def bwd_flops(B, Hq, N, d, causal):
    return 2.5 * fwd_flops(B, Hq, N, d, causal)


def kernel_flops(B, Hq, N, d, causal):
    """Algorithmic FLOPs credited to each tensor-core kernel, and the FLOPs it executes.

    The backward's five products (S, dP, dV, dK, dQ) all run in the main
    kernel, each once: 2.5 times the forward, the convention's figure.
    """
    f = fwd_flops(B, Hq, N, d, causal)
    return {"fwd": (f, f), "bwd_main": (2.5 * f, 2.5 * f)}


def algorithmic_bytes(B, Hq, Hkv, N, d):
    """Bytes each kernel must move at least once (bf16 tensors, f32 LSE/D)."""
    q = B * Hq * N * d * 2
    kv = B * Hkv * N * d * 2
    rows = B * Hq * N * 4
    return {
        "fwd": q + 2 * kv + q + rows,                     # read Q, K, V; write O, LSE
        "bwd_prep": 2 * q + rows + 2 * rows + 2 * q,      # read O, dO, LSE; write D, LSE2, zero dQacc (f32)
        "bwd_main": 2 * q + 2 * kv + 2 * rows + 2 * kv + 2 * q * 2,  # read Q,dO,K,V,LSE2,D; write dK,dV; dQacc add
        "bwd_dq": 2 * q + q,                              # read dQacc (f32), write dQ
    }


def kernel_source_hash() -> str:
    """Hash of the kernel sources (the csrc/*.cuh files) the recorded counters depend on."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "exact_io_aware_61_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if not name.endswith(".cuh"):
            continue
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            data = json.load(f)
        return data, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ clocks

CLOCK_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
REASON_NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")


class ClockSampler:
    """Samples SM clock, power and throttle reasons with nvidia-smi while running."""

    def __init__(self, gpu_index: str):
        self.gpu_index = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_index, f"--query-gpu={CLOCK_FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=self.out, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) != 9:
                    continue
                try:
                    rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[5:9]))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return None
        max_power = max(r[2] for r in rows)
        loaded = [r for r in rows if r[2] >= 0.5 * max_power] or rows
        reasons = sorted({REASON_NAMES[i] for r in loaded for i, v in enumerate(r[3]) if v == "Active"})
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows), "samples_under_load": len(loaded),
                "power_w_max": max_power}


# --------------------------------------------------------------- CPU oracle

def oracle_sample(inp_np, block: int, scale: float):
    """Run the fp64 oracle forward + backward on one sampled block of query rows.

    Block ``block`` picks head ``block % (B*Hq)`` and the 512 query rows
    ``r0, r0+16, ...`` (every 16th row, so the rows see keys spread over the
    causal range). Returns the algorithmic FLOPs of that sample under the
    same convention as the GPU numbers (only visible keys counted).
    """
    import oracle.attention as ref  # test infrastructure: CPU-baseline leg only

    B, Hq, N, d = inp_np["q"].shape
    bh = block % (B * Hq)
    b, h = divmod(bh, Hq)
    rows = list(range(block % 16, N, 16))
    q, k, v, do = (inp_np[n] for n in ("q", "k", "v", "do"))
    ref.attention_forward_rows(q, k, v, scale, CAUSAL, b, h, rows)
    ref.attention_backward_rows(q, k, v, do, scale, CAUSAL, b, h, rows)
    visible = sum((r + 1) if CAUSAL else N for r in rows)
    return 4.0 * d * visible * 3.5


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def sample_inputs_numpy():
    """The benchmark workload's inputs in float64 (exact upcast of the bf16 values)."""
    from exact_io_aware_61_b200 import inputs as inp_mod

    inp = inp_mod.make_inputs(SHAPE["B"], SHAPE["Hq"], SHAPE["Hkv"], SHAPE["N"], SHAPE["d"], "bf16", SEED, grad=True)
    return {n: inp_mod.as_f64(t) for n, t in inp.items()}


def cpu_baseline(min_seconds=10.0, max_seconds=30.0):
    inp = sample_inputs_numpy()
    scale = SHAPE["d"] ** -0.5
    flops, blocks = 0.0, 0
    t0 = time.perf_counter()
    while True:
        flops += oracle_sample(inp, blocks, scale)
        blocks += 1
        el = time.perf_counter() - t0
        if el >= min_seconds or el + el / blocks > max_seconds:
            break
    return {"value": flops / el / 1e12, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{blocks} blocks of 512 query rows (every 16th row of one head), fp64 numpy forward + "
                      f"backward of the full workload's inputs, {el:.1f} s"}


# ----------------------------------------------------------------- helpers

def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Largest ``value`` over all ranks (identity for one rank)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist

    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int, device=None):
    if world > 1:
        import torch
        import torch.distributed as dist

        t = torch.zeros(1, device=device)
        dist.all_reduce(t)


def physical_gpu_index(local_rank: int) -> str:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [x.strip() for x in vis.split(",") if x.strip()]
        if local_rank < len(ids):
            return ids[local_rank]
    return str(local_rank)


# -------------------------------------------------------------- our arm

def run_ours(args, rank, world, local):
    import torch

    import exact_io_aware_61_b200 as fa
    from exact_io_aware_61_b200 import inputs as inp_mod

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta

        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    fa.load()
    from exact_io_aware_61_b200.shard import pair_range

    # The job is world x the benchmark workload; its (batch, KV head) pairs are
    # split over the ranks in contiguous ranges (no collective on the data
    # path), so every rank runs the benchmark shape on its own slice.
    Hq, Hkv, N, d = (SHAPE[k] for k in ("Hq", "Hkv", "N", "d"))
    shard = pair_range(SHAPE["B"] * world, Hq, Hkv, rank, world)
    B, Hq, Hkv = shard.local_shape()
    scale = d ** -0.5
    host = inp_mod.make_inputs(B, Hq, Hkv, N, d, "bf16", SEED + shard.p0, grad=True)
    q, k, v, do = (host[n].to(dev) for n in ("q", "k", "v", "do"))
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(fa.fa_bwd_workspace_size(B, Hq, Hkv, N, d), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        fa.fa_fwd(q, k, v, o, lse, CAUSAL, scale, stream)
        if ev is not None:
            ev[1].record(stream)
        fa.fa_bwd_prep(o, lse, do, ws, Hkv, stream)
        if ev is not None:
            ev[2].record(stream)
        fa.fa_bwd_main(q, k, v, do, dk, dv, ws, CAUSAL, scale, stream)
        if ev is not None:
            ev[3].record(stream)
        fa.fa_bwd_dq(dq, ws, Hkv, stream)
        if ev is not None:
            ev[4].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if fa.fa_last_device_status(stream) != fa.FA_OK:
        raise RuntimeError("device status reports a timeout during warm-up")

    events = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    sampler = ClockSampler(physical_gpu_index(local))
    sampler.start()
    barrier(world, dev)
    torch.cuda.synchronize(dev)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for i in range(args.steps):
        step(events[i])
    end.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world, dev)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    status = fa.fa_last_device_status(stream)
    if status != fa.FA_OK:
        raise RuntimeError(f"device status {fa.status_string(status)} in the timed region")

    elapsed_ms = start.elapsed_time(end)
    per_kernel = {name: statistics.mean(e[i].elapsed_time(e[i + 1]) for e in events)
                  for i, name in enumerate(("fwd", "bwd_prep", "bwd_main", "bwd_dq"))}
    max_ms = max_over_ranks(elapsed_ms, world, dev)

    f_fwd = fwd_flops(B, Hq, N, d, CAUSAL)
    f_bwd = bwd_flops(B, Hq, N, d, CAUSAL)
    step_flops = f_fwd + f_bwd
    value = world * step_flops * args.steps / (max_ms / 1e3) / 1e12
    bwd_ms = per_kernel["bwd_prep"] + per_kernel["bwd_main"] + per_kernel["bwd_dq"]

    # forward alone: its own timed region (no backward kernels in between)
    fwd_only = None
    if not args.no_fwd_only:
        for _ in range(args.warmup):
            fa.fa_fwd(q, k, v, o, lse, CAUSAL, scale, stream)
        fsampler = ClockSampler(physical_gpu_index(local))
        fsampler.start()
        barrier(world, dev)
        torch.cuda.synchronize(dev)
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_fwd = max(args.steps, 20)
        f0.record(stream)
        for _ in range(n_fwd):
            fa.fa_fwd(q, k, v, o, lse, CAUSAL, scale, stream)
        f1.record(stream)
        torch.cuda.synchronize(dev)
        barrier(world, dev)
        fclocks = fsampler.stop()
        fwd_ms = max_over_ranks(f0.elapsed_time(f1), world, dev) / n_fwd
        fwd_only = {"launches": n_fwd, "ms": fwd_ms,
                    "tflops": world * fwd_flops(B, Hq, N, d, CAUSAL) / fwd_ms / 1e9, "clocks": fclocks}

    # end to end through the C ABI: pinned host buffers, every step's uploads and
    # downloads inside the timed region. Two sets of device buffers and three
    # streams ordered by events let step i's uploads and step i-1's downloads
    # overlap step i's kernels, as a caller of the stream-ordered API would run it.
    e2e = None
    if not args.no_e2e:
        hq_, hk_, hv_, hdo_ = (host[n].pin_memory() for n in ("q", "k", "v", "do"))
        e2e_steps = max(3, min(args.steps, 10))
        bufs = [dict(q=torch.empty_like(q), k=torch.empty_like(k), v=torch.empty_like(v), do=torch.empty_like(do),
                     o=torch.empty_like(o), lse=torch.empty_like(lse), dq=torch.empty_like(dq),
                     dk=torch.empty_like(dk), dv=torch.empty_like(dv), ws=torch.empty_like(ws)) for _ in range(2)]
        outs = [[torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in (o, lse, dq, dk, dv)]
                for _ in range(2)]
        up, comp, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        computed = [torch.cuda.Event() for _ in range(2)]
        downloaded = [torch.cuda.Event() for _ in range(2)]
        for e in computed + downloaded:
            e.record(comp)

        def e2e_step(i):
            s = i % 2
            b = bufs[s]
            up.wait_event(computed[s])  # step i-2's kernels have read this set's inputs
            with torch.cuda.stream(up):
                for name, src in (("q", hq_), ("k", hk_), ("v", hv_), ("do", hdo_)):
                    b[name].copy_(src, non_blocking=True)
            comp.wait_stream(up)
            comp.wait_event(downloaded[s])  # step i-2's outputs have left this set
            fa.fa_fwd(b["q"], b["k"], b["v"], b["o"], b["lse"], CAUSAL, scale, comp)
            fa.fa_bwd_prep(b["o"], b["lse"], b["do"], b["ws"], Hkv, comp)
            fa.fa_bwd_main(b["q"], b["k"], b["v"], b["do"], b["dk"], b["dv"], b["ws"], CAUSAL, scale, comp)
            fa.fa_bwd_dq(b["dq"], b["ws"], Hkv, comp)
            computed[s].record(comp)
            down.wait_event(computed[s])
            with torch.cuda.stream(down):
                for dst, name in zip(outs[s], ("o", "lse", "dq", "dk", "dv")):
                    dst.copy_(b[name], non_blocking=True)
            downloaded[s].record(down)

        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize(dev)
        barrier(world, dev)
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(comp)
        up.wait_stream(comp)
        for i in range(e2e_steps):
            e2e_step(i)
        comp.wait_stream(down)
        s1.record(comp)
        torch.cuda.synchronize(dev)
        barrier(world, dev)
        e2e_ms = max_over_ranks(s0.elapsed_time(s1), world, dev)
        if fa.fa_last_device_status(comp) != fa.FA_OK:
            raise RuntimeError("device status reports a timeout in the end-to-end region")
        # the pipelined forward must give the plain path's output exactly (the
        # forward is deterministic); anything else is an ordering error
        last = outs[(e2e_steps - 1) % 2]
        if not (torch.equal(last[0], o.cpu()) and torch.equal(last[1], lse.cpu())):
            raise RuntimeError("pipelined end-to-end run does not reproduce the forward output")
        h2d = sum(t.numel() * t.element_size() for t in (hq_, hk_, hv_, hdo_))
        d2h = sum(t.numel() * t.element_size() for t in outs[0])
        e2e = {"value": world * step_flops * e2e_steps / (e2e_ms / 1e3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
               "ms_per_step": e2e_ms / e2e_steps}

    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()
    if rank != 0:
        return

    peaks, peak_src = load_peaks()
    peak_tf = float(peaks["bf16_tflops"])
    hbm = float(peaks["hbm_gbs"])
    nbytes = algorithmic_bytes(B, Hq, Hkv, N, d)
    kf = kernel_flops(B, Hq, N, d, CAUSAL)
    src_hash = kernel_source_hash()
    names = {"fwd": f"fa_fwd_bf16_2tile_kernel<{d}>" if d != 256 else "fa_fwd_bf16_kernel<256>",
             "bwd_prep": f"fa_bwd_prep_kernel<{d}>",
             "bwd_main": f"fa_bwd2_main_kernel<{d}>" if d != 256 else "fa_bwd256_main_kernel",
             "bwd_dq": "fa_bwd_dq_kernel"}
    kernels = {}
    for name, ms in per_kernel.items():
        e = {"kernel": names[name], "ms": round(ms, 4), "gbs": round(nbytes[name] / ms / 1e6, 1)}
        if name in kf:
            credited, executed = kf[name]
            e["tflops"] = round(credited / ms / 1e9, 2)
            e["executed_tflops"] = round(executed / ms / 1e9, 2)
            e["pct_of_peak"] = round(100 * credited / ms / 1e9 / peak_tf, 2)
        prof = PROFILED.get(name)
        if prof and prof.get("src") == src_hash:
            e["tensor_pipe_active_pct"] = prof.get("tensor_pipe_active_pct")
            e["dram_bytes"] = prof.get("dram_bytes")
        kernels[name] = e
    dominant = max(kf, key=lambda n: per_kernel[n])
    credited, executed = kf[dominant]
    achieved = credited / per_kernel[dominant] / 1e9
    prof = PROFILED.get(dominant)
    fresh = bool(prof) and prof.get("src") == src_hash
    traffic_val = prof.get("dram_bytes") if fresh else None
    tensor_active = prof.get("tensor_pipe_active_pct") if fresh else None

    out = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(max_ms / args.steps, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic: i.i.d. N(0,1) rounded to bf16, seeded",
        "config": {"workload": WORKLOAD_NAME, "B": B, "Hq": Hq, "Hkv": Hkv, "N": N, "d": d, "causal": CAUSAL,
                   "parallelism": f"(batch, KV head) pairs of a {SHAPE['B'] * world}-batch job split over {world} "
                                  f"rank(s), {shard.pairs} pairs each, no collective on the data path",
                   "l2": "no flush: every step streams > 1 GB and each of Q, K, V, O, dO is 134 MB (> 126 MB L2)"},
        "fwd_tflops": round(f_fwd / per_kernel["fwd"] / 1e9, 2),
        "bwd_tflops": round(f_bwd / bwd_ms / 1e9, 2),
        "pct_of_peak": {"fwd": round(100 * f_fwd / per_kernel["fwd"] / 1e9 / peak_tf, 2),
                        "bwd": round(100 * f_bwd / bwd_ms / 1e9 / peak_tf, 2),
                        "step": round(100 * value / world / peak_tf, 2),
                        "peak_tflops": peak_tf, "peak_source": f"{peak_src} bf16_tflops (burst)"},
        "pct_of_spec": {"fwd": round(100 * f_fwd / per_kernel["fwd"] / 1e9 / SPEC_BF16_TFLOPS, 2),
                        "bwd": round(100 * f_bwd / bwd_ms / 1e9 / SPEC_BF16_TFLOPS, 2),
                        "step": round(100 * value / world / SPEC_BF16_TFLOPS, 2),
                        "spec_tflops": SPEC_BF16_TFLOPS,
                        "spec_source": "vendor dense bf16 figure (the 2:4-sparse figure halved)"},
        "hbm_gbs": {"fwd": kernels["fwd"]["gbs"],
                    "bwd": round(sum(nbytes[n] for n in ("bwd_prep", "bwd_main", "bwd_dq")) / bwd_ms / 1e6, 1),
                    "peak_gbs": hbm},
        "kernels": kernels,
        "roofline": {"kernel": names[dominant], "bound": "tensor", "achieved": round(achieved, 2), "peak": peak_tf,
                     "unit": "TFLOP/s", "frac": round(achieved / peak_tf, 4), "traffic": traffic_val,
                     "tensor_pipe_active": tensor_active,
                     "algorithmic_flops": credited, "executed_flops": executed,
                     "algorithmic_bytes": nbytes[dominant],
                     "peak_note": f"{peak_src} (burst bf16 GEMM)", "hbm_peak_gbs": hbm},
        "gpu_launches": 4 * args.steps,
        "clocks": clocks,
        "kernel_src": src_hash,
    }
    if fwd_only is not None:
        peak = float(load_peaks()[0]["bf16_tflops"])
        out["fwd_only"] = {"launches": fwd_only["launches"], "ms": round(fwd_only["ms"], 4),
                           "tflops": round(fwd_only["tflops"], 2),
                           "pct_of_peak": round(100 * fwd_only["tflops"] / world / peak, 2),
                           "clocks": fwd_only["clocks"]}
    if e2e is not None:
        out["e2e"] = {k: (round(v, 4) if isinstance(v, float) else v) for k, v in e2e.items()}
    if world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline()
    print(json.dumps(out), flush=True)


# --------------------------------------------------------- reference arm

def run_kvcache(args, rank, world, local):
    """Time fa_fwd_kvcache (decode over a KV cache) on one GPU: HBM throughput
    of the bytes the method must move (K and V once, Q, O, LSE), against the
    measured copy bandwidth."""
    import torch

    import exact_io_aware_61_b200 as fa

    if world != 1:
        raise SystemExit("--kvcache runs on one GPU")
    B, Hq, Hkv, Nq, Nk, d = (int(x) for x in args.kvcache.split(","))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    fa.load()
    g = torch.Generator(device="cpu").manual_seed(SEED)
    q = torch.randn((B, Hq, Nq, d), generator=g).to(torch.bfloat16).to(dev)
    k = torch.randn((B, Hkv, Nk, d), generator=g).to(torch.bfloat16).to(dev)
    v = torch.randn((B, Hkv, Nk, d), generator=g).to(torch.bfloat16).to(dev)
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=dev)
    ws = torch.empty(max(fa.fa_fwd_kvcache_workspace_size(B, Hq, Hkv, Nq, Nk, d), 16), dtype=torch.uint8,
                     device=dev)
    stream = torch.cuda.current_stream(dev)
    scale = d ** -0.5
    kv_bytes = 2 * B * Hkv * Nk * d * 2
    flush = None if kv_bytes > 2 * 126e6 else torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        fa.fa_fwd_kvcache(q, k, v, o, lse, ws, True, scale, stream)
    torch.cuda.synchronize(dev)
    events = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    sampler = ClockSampler(physical_gpu_index(local))
    sampler.start()
    for e0, e1 in events:
        if flush is not None:
            flush.zero_()
        e0.record(stream)
        fa.fa_fwd_kvcache(q, k, v, o, lse, ws, True, scale, stream)
        e1.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    if fa.fa_last_device_status(stream) != fa.FA_OK:
        raise RuntimeError("device status reports a timeout")
    ms = statistics.median(e0.elapsed_time(e1) for e0, e1 in events)
    nbytes = kv_bytes + 2 * B * Hq * Nq * d * 2 + 4 * B * Hq * Nq
    peaks, src = load_peaks()
    gbs = nbytes / ms / 1e6
    print(json.dumps({
        "metric": "KV-cache forward (decode) HBM throughput", "value": round(gbs, 1), "unit": "GB/s",
        "higher_is_better": True, "ms": round(ms, 4), "steps": args.steps, "warmup": args.warmup,
        "config": {"workload": f"causal bf16 KV-cache forward, B={B} Hq={Hq} Hkv={Hkv} Nq={Nq} Nk={Nk} d={d}",
                   "l2": "no flush: K and V exceed twice the L2" if flush is None else
                   "256 MB buffer written between timed launches"},
        "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": round(gbs / peaks["hbm_gbs"], 4), "algorithmic_bytes": nbytes,
                     "peak_note": f"{src} copy bandwidth"},
        "tflops": round(4 * B * Hq * Nq * Nk * d / ms / 1e9, 2),
        "clocks": clocks, "dtype": "bf16", "data": "synthetic: i.i.d. N(0,1) rounded to bf16, seeded"}))


def run_fwd_shape(args, rank, world, local):
    """Time fa_fwd alone on one shape (B,Hq,Hkv,N,d,causal,dtype) on one GPU and
    report TFLOP/s against the measured bf16 peak."""
    import torch

    import exact_io_aware_61_b200 as fa

    if world != 1:
        raise SystemExit("--fwd runs on one GPU")
    B, Hq, Hkv, N, d, causal = (int(x) for x in args.fwd.split(",")[:6])
    dtype = args.fwd.split(",")[6] if args.fwd.count(",") >= 6 else "bf16"
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    fa.load()
    from exact_io_aware_61_b200 import inputs as inp_mod
    host = inp_mod.make_inputs(B, Hq, Hkv, N, d, dtype, SEED)
    q, k, v = (host[n].to(dev) for n in ("q", "k", "v"))
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    in_bytes = sum(t.numel() * t.element_size() for t in (q, k, v))
    flush = None if in_bytes > 2 * 126e6 else torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        fa.fa_fwd(q, k, v, o, lse, causal, d ** -0.5, stream)
    torch.cuda.synchronize(dev)
    events = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    sampler = ClockSampler(physical_gpu_index(local))
    sampler.start()
    for e0, e1 in events:
        if flush is not None:
            flush.zero_()
        e0.record(stream)
        fa.fa_fwd(q, k, v, o, lse, causal, d ** -0.5, stream)
        e1.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    if fa.fa_last_device_status(stream) != fa.FA_OK:
        raise RuntimeError("device status reports a timeout")
    ms = statistics.median(e0.elapsed_time(e1) for e0, e1 in events)
    tflops = fwd_flops(B, Hq, N, d, bool(causal)) / ms / 1e9
    peaks, src = load_peaks()
    print(json.dumps({
        "metric": "attention forward TFLOP/s", "value": round(tflops, 2), "unit": "TFLOP/s",
        "higher_is_better": True, "ms": round(ms, 4), "steps": args.steps, "warmup": args.warmup,
        "config": {"workload": f"{'causal' if causal else 'full'} {dtype} attention forward, "
                               f"B={B} Hq={Hq} Hkv={Hkv} N={N} d={d}",
                   "l2": "no flush: Q, K, V exceed twice the L2" if flush is None else
                   "256 MB buffer written between timed launches"},
        "pct_of_peak": round(100 * tflops / peaks["bf16_tflops"], 2), "peak_tflops": peaks["bf16_tflops"],
        "peak_note": f"{src} bf16 GEMM (burst)", "clocks": clocks, "dtype": dtype,
        "data": "synthetic: i.i.d. N(0,1), seeded"}))


def run_seqpar(args, rank, world, local):
    """Time the sequence-sharded causal forward (striped tokens, K/V ring, merge) and its backward.

    On one GPU the W ranks' work is emulated: the busiest rank's W blocks
    (``fa_fwd_partial`` against every rank's K/V shard, all held on this GPU)
    and its ``fa_merge_partials``, with no transfer. Under torch.distributed
    (one rank per GPU, W = world) each rank runs ``seqpar.ring_forward`` over
    NCCL; the time is the maximum over ranks. ``value`` is the TFLOP/s of one
    rank's own blocks (their visible score entries x 4 d, per query head),
    over that rank's time."""
    import torch

    import exact_io_aware_61_b200 as fa
    from exact_io_aware_61_b200 import seqpar

    B, Hq, Hkv, N, d, W = (int(x) for x in args.seqpar.split(","))
    if world > 1 and world != W:
        raise SystemExit("--seqpar: W must equal the number of ranks under torch.distributed")
    if N % W:
        raise SystemExit("--seqpar: N must be a multiple of W")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta

        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    fa.load()
    n = N // W
    scale = d ** -0.5
    g = torch.Generator(device="cpu").manual_seed(SEED)
    me = W - 1 if world == 1 else rank  # under the causal mask rank W-1 has the most visible keys
    if world == 1:
        q = torch.randn((B, Hq, n, d), generator=g).to(torch.bfloat16).to(dev)
        kv = [(torch.randn((B, Hkv, n, d), generator=g).to(torch.bfloat16).to(dev),
               torch.randn((B, Hkv, n, d), generator=g).to(torch.bfloat16).to(dev)) for _ in range(W)]
        o_parts = torch.empty((W, B, Hq, n, d), dtype=torch.bfloat16, device=dev)
        l_parts = torch.empty((W, B, Hq, n), dtype=torch.float32, device=dev)
        o = torch.empty_like(q)
        lse = torch.empty((B, Hq, n), dtype=torch.float32, device=dev)
        sched = seqpar.ring_schedule(me, W, True)
    else:
        g.manual_seed(SEED + rank)
        q, k, v = (torch.randn((B, h, n, d), generator=g).to(torch.bfloat16).to(dev) for h in (Hq, Hkv, Hkv))
    stream = torch.cuda.current_stream(dev)
    blk_ev = []

    def run(record=False):
        if world > 1:
            seqpar.ring_forward(q, k, v, causal=True, scale=scale)
            return
        for t, (src, diag) in enumerate(sched):
            if record:
                e = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                e[0].record(stream)
            fa.fa_fwd_partial(q, kv[src][0], kv[src][1], o_parts[t], l_parts[t], True, scale, diag, stream)
            if record:
                e[1].record(stream)
                blk_ev.append(("block", e))
        if record:
            e = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            e[0].record(stream)
        fa.fa_merge_partials(o_parts, l_parts, o, lse, stream)
        if record:
            e[1].record(stream)
            blk_ev.append(("merge", e))

    for _ in range(args.warmup):
        run()
    torch.cuda.synchronize(dev)
    barrier(world, dev)
    sampler = ClockSampler(physical_gpu_index(local))
    sampler.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        run(record=True)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    barrier(world, dev)
    if fa.fa_last_device_status(stream) != fa.FA_OK:
        raise RuntimeError("device status reports a timeout")
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world, dev)
    # visible (query, key) pairs of this rank's blocks: n(n+1)/2 on the
    # diagonal-0 blocks, n(n-1)/2 on the diagonal -1 ones
    pairs = sum(n * (n + 1) // 2 if diag == 0 else n * (n - 1) // 2 for _, diag in seqpar.ring_schedule(me, W, True))
    flops = 4.0 * B * Hq * d * pairs
    tflops = flops / ms / 1e9
    peaks, src = load_peaks()
    out = {
        "metric": "sequence-sharded causal attention forward, TFLOP/s of one rank", "value": round(tflops, 2),
        "unit": "TFLOP/s", "higher_is_better": True, "n_gpus": world, "ms_per_step": round(ms, 4),
        "steps": args.steps, "warmup": args.warmup, "dtype": "bf16", "data": "synthetic: i.i.d. N(0,1), seeded",
        "config": {"workload": f"causal bf16 attention forward over N={N} tokens striped across W={W} ranks, "
                               f"B={B} Hq={Hq} Hkv={Hkv} d={d}, {n} tokens per rank",
                   "mode": "one GPU: rank W-1's blocks and merge, no transfer" if world == 1 else
                           "torch.distributed ring over NCCL, max over ranks",
                   "l2": "no flush: the per-rank working set is not larger than L2 at every W"},
        "pct_of_peak": round(100 * tflops / peaks["bf16_tflops"], 2), "peak_note": f"{src} bf16 GEMM (burst)",
        "clocks": clocks,
    }
    # the backward of the same rank: prep, one fa_bwd_partial per block, dQ
    # and (for the keys the rank owns) dK, dV conversions; under
    # torch.distributed the whole ring_backward with its exchanges
    g.manual_seed(SEED + 7 + rank)
    do = torch.randn(q.shape, generator=g).to(torch.bfloat16).to(dev)
    if world == 1:
        bops = seqpar.LibraryBackwardOps(q, kv[0][0], True, scale, stream)
        accs = [(torch.zeros(kv[0][0].shape, dtype=torch.float32, device=dev),
                 torch.zeros(kv[0][1].shape, dtype=torch.float32, device=dev)) for _ in range(W)]
        dq, dk, dv = torch.empty_like(q), torch.empty_like(kv[0][0]), torch.empty_like(kv[0][1])
    else:
        o, lse = seqpar.ring_forward(q, k, v, causal=True, scale=scale)

    def run_bwd():
        if world > 1:
            seqpar.ring_backward(q, k, v, o, lse, do, causal=True, scale=scale)
            return
        bops.prep(o, lse, do)
        for src, diag in sched:
            bops.block(q, kv[src][0], kv[src][1], do, accs[src][0], accs[src][1], diag)
        bops.finish(dq)
        bops.to_bf16(accs[me][0], dk)
        bops.to_bf16(accs[me][1], dv)

    for _ in range(args.warmup):
        run_bwd()
    torch.cuda.synchronize(dev)
    barrier(world, dev)
    b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    b0.record(stream)
    for _ in range(args.steps):
        run_bwd()
    b1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world, dev)
    if fa.fa_last_device_status(stream) != fa.FA_OK:
        raise RuntimeError("device status reports a timeout")
    bwd_ms = max_over_ranks(b0.elapsed_time(b1) / args.steps, world, dev)
    out["bwd"] = {"ms_per_step": round(bwd_ms, 4), "tflops": round(2.5 * flops / bwd_ms / 1e9, 2),
                  "pct_of_peak": round(100 * 2.5 * flops / bwd_ms / 1e9 / peaks["bf16_tflops"], 2),
                  "flops_note": "2.5 x the rank's forward FLOPs (the usual backward convention)"}
    if world == 1:
        blk = [a.elapsed_time(b) for kind, (a, b) in blk_ev if kind == "block"]
        mrg = [a.elapsed_time(b) for kind, (a, b) in blk_ev if kind == "merge"]
        mbytes = (W + 1) * B * Hq * n * (2 * d + 4)
        merge_ms = statistics.median(mrg)
        out["kernels"] = {
            "fa_fwd_partial": {"ms_per_block": round(statistics.median(blk), 4),
                               "tflops": round(flops / W / statistics.median(blk) / 1e9, 2)},
            "fa_merge_partials": {"ms": round(merge_ms, 4), "algorithmic_bytes": mbytes,
                                  "gbs": round(mbytes / merge_ms / 1e6, 1),
                                  "frac_of_hbm": round(mbytes / merge_ms / 1e6 / peaks["hbm_gbs"], 4)},
        }
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


def varlen_lengths(total: int, lo: int, hi: int, seed: int):
    """Seeded sequence lengths, uniform in [lo, hi], the last one cut so that they sum to ``total``."""
    import random

    rng = random.Random(seed)
    lens = []
    while sum(lens) < total:
        lens.append(min(rng.randint(lo, hi), total - sum(lens)))
    return lens


def run_varlen(args, rank, world, local):
    """Time fa_fwd_varlen and fa_bwd_varlen on one GPU over a packed batch of
    sequences of mixed lengths (causal, each sequence's queries against its
    own keys). FLOPs: per sequence 4 * Hq * L * (L + 1) / 2 * d forward (its
    visible pairs), 2.5 times that backward."""
    import torch

    import exact_io_aware_61_b200 as fa
    from exact_io_aware_61_b200 import inputs as inp_mod

    if world != 1:
        raise SystemExit("--varlen runs on one GPU")
    total, lo, hi, Hq, Hkv, d = (int(x) for x in args.varlen.split(","))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    fa.load()
    lens = varlen_lengths(total, lo, hi, SEED)
    host = inp_mod.make_varlen_inputs(lens, lens, Hq, Hkv, d, "bf16", SEED, grad=True)
    q, k, v, do = (host[n].to(dev) for n in ("q", "k", "v", "do"))
    cu = host["cu_q"].to(dev)
    scale = d ** -0.5
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:-1], dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(max(fa.fa_bwd_varlen_workspace_size(len(lens), total, total, Hq, Hkv, d), 16),
                     dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    mx = max(lens)

    def fwd():
        fa.fa_fwd_varlen(q, k, v, o, lse, cu, cu, mx, True, scale, stream)

    def bwd():
        fa.fa_bwd_varlen(q, k, v, o, lse, do, dq, dk, dv, cu, cu, mx, mx, ws, True, scale, stream)

    for _ in range(args.warmup):
        fwd()
        bwd()
    torch.cuda.synchronize(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    sampler = ClockSampler(physical_gpu_index(local))
    sampler.start()
    for e0, e1, e2 in ev:
        e0.record(stream)
        fwd()
        e1.record(stream)
        bwd()
        e2.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    if fa.fa_last_device_status(stream) != fa.FA_OK:
        raise RuntimeError("device status reports an error")
    f_ms = statistics.median(a.elapsed_time(b) for a, b, _ in ev)
    b_ms = statistics.median(b.elapsed_time(c) for _, b, c in ev)
    fflops = sum(4.0 * Hq * L * (L + 1) / 2 * d for L in lens)
    peaks, src = load_peaks()
    f_tf, b_tf = fflops / f_ms / 1e9, 2.5 * fflops / b_ms / 1e9
    print(json.dumps({
        "metric": "variable-length causal attention fwd+bwd TFLOP/s", "value": round(3.5 * fflops / (f_ms + b_ms) / 1e9, 2),
        "unit": "TFLOP/s", "higher_is_better": True, "steps": args.steps, "warmup": args.warmup,
        "fwd_tflops": round(f_tf, 2), "bwd_tflops": round(b_tf, 2), "fwd_ms": round(f_ms, 4), "bwd_ms": round(b_ms, 4),
        "pct_of_peak": {"fwd": round(100 * f_tf / peaks["bf16_tflops"], 2),
                        "bwd": round(100 * b_tf / peaks["bf16_tflops"], 2)},
        "peak_note": f"{src} bf16 GEMM (burst)",
        "config": {"workload": f"causal bf16 packed batch of {len(lens)} sequences, {total} tokens, lengths uniform "
                               f"in [{lo}, {hi}] (seeded), Hq={Hq} Hkv={Hkv} d={d}",
                   "lengths": lens, "l2": "no flush: Q, K, V and the gradients exceed the L2"},
        "clocks": clocks, "dtype": "bf16", "data": "synthetic: i.i.d. N(0,1), seeded"}))


def run_reference(args, rank, world):
    if rank != 0:
        return  # rank 0 alone times the oracle; the others exit without work
    inp = sample_inputs_numpy()
    scale = SHAPE["d"] ** -0.5
    for i in range(args.warmup):
        oracle_sample(inp, i, scale)
    flops = 0.0
    t0 = time.perf_counter()
    for i in range(args.steps):
        flops += oracle_sample(inp, args.warmup + i, scale)
    el = time.perf_counter() - t0
    value = flops / el / 1e12
    cores = blas_threads()
    out = {
        "impl": "reference",
        "metric": METRIC,
        "value": value,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": 1e3 * el / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic: i.i.d. N(0,1) rounded to bf16, seeded",
        "config": {"workload": WORKLOAD_NAME, **SHAPE, "causal": CAUSAL,
                   "parallelism": "rank 0 only, host cores"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": "per step: 512 query rows (every 16th row of one head), fp64 numpy forward "
                                   "+ backward"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-fwd-only", action="store_true", help="skip the separate forward-only timed region")
    ap.add_argument("--fwd", default=None,
                    help="B,Hq,Hkv,N,d,causal[,dtype]: time the forward alone on that shape")
    ap.add_argument("--kvcache", default=None,
                    help="B,Hq,Hkv,Nq,Nk,d: time the KV-cache (decode) forward instead of the benchmark step")
    ap.add_argument("--seqpar", default=None,
                    help="B,Hq,Hkv,N,d,W: time the sequence-sharded causal forward over W striped ranks")
    ap.add_argument("--varlen", default=None,
                    help="total,lo,hi,Hq,Hkv,d: time the variable-length forward and backward on a packed batch")
    ap.add_argument("--shape", default=None,
                    help="B,Hq,Hkv,N,d of a smaller case for profiling (default: the benchmark workload)")
    args = ap.parse_args(argv)
    if args.shape:
        global WORKLOAD_NAME
        B, Hq, Hkv, N, d = (int(x) for x in args.shape.split(","))
        SHAPE.update(B=B, Hq=Hq, Hkv=Hkv, N=N, d=d)
        WORKLOAD_NAME = f"causal bf16 attention forward+backward, B={B} Hq={Hq} Hkv={Hkv} N={N} d={d}"
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    rank, world, local = dist_env()
    if world != args.gpus:
        if world == 1 and args.gpus > 1:
            ap.error(f"--gpus {args.gpus} needs a launch with torch.distributed.run (one rank per GPU)")
    if args.seqpar:
        run_seqpar(args, rank, world, local)
    elif args.varlen:
        run_varlen(args, rank, world, local)
    elif args.kvcache:
        run_kvcache(args, rank, world, local)
    elif args.fwd:
        run_fwd_shape(args, rank, world, local)
    elif args.impl == "reference":
        run_reference(args, rank, world)
    else:
        run_ours(args, rank, world, local)


if __name__ == "__main__":
    main()
