#!/usr/bin/env python
"""Benchmark of the MLA decode hot path on B200: one step = split-KV schedule
(mla_get_metadata) + attention kernel + LSE-combine kernel over one synthetic batch.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload serving_b256]
                    [--impl ours|reference]

Prints one JSON line (rank 0).  Device times come from CUDA events on the launching
stream, summed over exactly K timed steps; an L2 flush (a 256 MB write, twice the L2)
runs before every step outside the timed events.  Multi-GPU runs (torchrun) are
independent replicas of the same workload per GPU (weak scaling; the path has no
exchange step): value = all ranks' FLOPs / max-over-ranks time.

--impl reference times the float64 CPU oracle (the only reference that exists for this
path) on a bounded sample of the same workload.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from deepseek_mla_decode_b200.workloads import WORKLOADS, make_workload  # noqa: E402

D_QK, D_LATENT = 576, 512
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


# ---------------------------------------------------------------------------
# algorithmic work (per call)
# ---------------------------------------------------------------------------
def algorithmic_work(seqlens, s_q, H, causal):
    """FLOPs = 2 (576 + 512) per (sequence, query token, visible key, head);
    cache bytes = every visible cache row once (1152 B per (sequence, key));
    algorithmic bytes = cache bytes + q + out + lse."""
    flops = 0
    keys = 0
    for n in np.asarray(seqlens).tolist():
        keys += max(int(n), 0)
        for i in range(s_q):
            vis = n if not causal else max(0, min(n, n - s_q + i + 1))
            flops += max(vis, 0) * H * 2 * (D_QK + D_LATENT)
    B = len(seqlens)
    cache_bytes = keys * D_QK * 2
    q_bytes = B * s_q * H * D_QK * 2
    out_bytes = B * s_q * H * D_LATENT * 2 + B * s_q * H * 4
    return flops, cache_bytes, cache_bytes + q_bytes + out_bytes


def max_over_ranks(values, world, device, dist=None):
    """Element-wise max of `values` over all ranks of the process group (the identity
    on one rank).  Every rank must call it with the same number of values."""
    import torch

    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t]


def whole_job_rate(world, work_per_rank, ms):
    """Throughput of the whole job: every rank did `work_per_rank` in at most `ms`
    (the slowest rank's time), so the job did world * work in that time."""
    return world * work_per_rank / (ms * 1e-3)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, FALLBACK_BF16_TFLOPS, "fallback"


def kernel_source_hash():
    h = hashlib.sha256()
    for f in ("mla_decode_kernel.cu", "ptx_sm100.cuh", "mla_internal.h"):
        with open(os.path.join(ROOT, "deepseek_mla_decode_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload):
    """DRAM bytes per attention launch from a committed ncu summary, if it was taken on
    the current kernel source; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
        e = d[workload]
        if e.get("kernel_hash") == kernel_source_hash():
            return float(e["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML reads only)
# ---------------------------------------------------------------------------
class ClockSampler:
    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4, "hw_slowdown": 0x8,
        "sync_boost": 0x10, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
    }

    def __init__(self, device_index_uuid):
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml

            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByUUID(device_index_uuid)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                    nv.nvmlDeviceGetCurrentClocksThrottleReasons
                self.reasons |= fn(self.h)
            except Exception:
                pass
            time.sleep(0.01)

    def __enter__(self):
        if self.nv is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        return {
            "sm_mhz": float(statistics.median(self.samples)),
            "sm_max_mhz": self.max_mhz,
            "reasons": [k for k, v in self.REASONS.items() if self.reasons & v],
            "samples": len(self.samples),
        }


# ---------------------------------------------------------------------------
# the CPU oracle (baseline / reference arm only)
# ---------------------------------------------------------------------------
def time_oracle(inp, budget_s, start_seq=0):
    """Runs the float64 oracle over whole sequences of the workload until the budget is
    spent; returns (flops done, seconds, sequences)."""
    from oracle import mla_oracle as O

    qn_all, qp_all = inp.q_nope, inp.q_pe
    flops = 0
    t0 = time.perf_counter()
    nseq = 0
    b = start_seq
    while True:
        b %= inp.B
        n = int(inp.cache_seqlens[b])
        nblk = (n + 63) // 64
        kv_b = O.bf16_to_f64(inp.kv_cache[inp.block_table[b, :nblk]])
        O.mla_decode_ref(O.bf16_to_f64(qn_all[b : b + 1]), O.bf16_to_f64(qp_all[b : b + 1]), kv_b,
                         np.arange(nblk)[None, :], np.array([n]), inp.softmax_scale, inp.causal)
        f, _, _ = algorithmic_work([n], inp.s_q, inp.H, inp.causal)
        flops += f
        nseq += 1
        b += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            return flops, el, nseq


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count()


# ---------------------------------------------------------------------------
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="serving_b256", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle time for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    w = WORKLOADS[args.workload]

    if args.impl == "reference":
        if rank != 0:
            return
        inp = make_workload(args.workload)
        for i in range(args.warmup):
            time_oracle(inp, 0.0, start_seq=i)
        flops = 0
        secs = 0.0
        nseq = 0
        for k in range(args.steps):
            f, s, n = time_oracle(inp, 0.0, start_seq=args.warmup + k)
            flops += f
            secs += s
            nseq += n
        value = flops / secs / 1e12
        line = {
            "impl": "reference", "metric": f"MLA decode TFLOP/s ({w.name})", "value": value, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "s_q": w.s_q, "H": w.H, "causal": w.causal,
                       "lengths": w.lengths, "seed": w.seed},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
                             "sample": f"one whole sequence per step, {nseq} sequences of {w.name}"},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        }
        print(json.dumps(line))
        return

    import torch
    import torch.distributed as dist

    import deepseek_mla_decode_b200 as mla

    if world > 1:
        torch.cuda.set_device(local_rank)
        import datetime

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())

    inp = make_workload(args.workload)
    flops, cache_bytes, algo_bytes = algorithmic_work(inp.cache_seqlens, inp.s_q, inp.H, inp.causal)

    def to_dev_bf16(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)

    q_nope = to_dev_bf16(inp.q_nope)
    q_pe = to_dev_bf16(inp.q_pe)
    kv = to_dev_bf16(inp.kv_cache)
    table = torch.from_numpy(inp.block_table).to(dev)
    seqlens = torch.from_numpy(inp.cache_seqlens).to(dev)
    B, s_q, H = inp.B, inp.s_q, inp.H
    meta = torch.empty((mla.metadata_size(B, s_q, H) + 3) // 4, dtype=torch.int32, device=dev)
    ws = torch.empty(mla.workspace_size(B, s_q, H), dtype=torch.uint8, device=dev)
    out = torch.empty((B, s_q, H, 512), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, s_q, H), dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step(ev=None):
        mla.get_metadata(seqlens, s_q, H, metadata=meta, stream=stream)
        if ev is not None:
            ev[0].record(stream)
        mla.decode_attention(q_nope, q_pe, kv, table, seqlens, inp.softmax_scale, inp.causal, meta, ws, out, lse,
                             status=status, stream=stream)
        if ev is not None:
            ev[1].record(stream)
        mla.decode_combine(seqlens, table.shape[1], s_q, H, meta, ws, out, lse, status=status, stream=stream)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} during warm-up")

    K = args.steps
    ev_s = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ev_e = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ev_a = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(uuid)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with sampler:
        for k in range(K):
            flush.zero_()
            ev_s[k].record(stream)
            step(ev_a[k])
            ev_e[k].record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    step_ms = sum(ev_s[k].elapsed_time(ev_e[k]) for k in range(K))
    att_ms = sum(ev_a[k][0].elapsed_time(ev_a[k][1]) for k in range(K))
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} in the timed region")
    step_ms, att_ms = max_over_ranks([step_ms, att_ms], world, dev, dist)

    # ---- end to end through the public API with host buffers ---------------
    e2e = None
    if args.e2e_steps > 0:
        h = {k: torch.from_numpy(np.ascontiguousarray(v)).pin_memory() for k, v in
             (("q_nope", inp.q_nope.view(np.int16)), ("q_pe", inp.q_pe.view(np.int16)),
              ("kv", inp.kv_cache.view(np.int16)), ("table", inp.block_table), ("seq", inp.cache_seqlens))}
        h_out = torch.empty(out.shape, dtype=torch.bfloat16).pin_memory()
        h_lse = torch.empty(lse.shape, dtype=torch.float32).pin_memory()
        d = {k: torch.empty(v.shape, dtype=v.dtype, device=dev) for k, v in h.items()}
        h2d = sum(v.numel() * v.element_size() for v in h.values())
        d2h = h_out.numel() * 2 + h_lse.numel() * 4

        def e2e_step():
            for k in h:
                d[k].copy_(h[k], non_blocking=True)
            m = mla.get_metadata(d["seq"], s_q, H, metadata=meta, stream=stream)
            mla.decode(d["q_nope"].view(torch.bfloat16), d["q_pe"].view(torch.bfloat16), d["kv"].view(torch.bfloat16),
                       d["table"], d["seq"], inp.softmax_scale, inp.causal, m, workspace=ws, out=out, lse=lse,
                       status=status, stream=stream)
            h_out.copy_(out, non_blocking=True)
            h_lse.copy_(lse, non_blocking=True)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        e0.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = e0.elapsed_time(e1) / args.e2e_steps
        (e2e_ms,) = max_over_ranks([e2e_ms], world, dev, dist)
        e2e = {"value": whole_job_rate(world, flops, e2e_ms) / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h), "ms_per_step": e2e_ms}

    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return

    hbm_peak, tc_peak, tc_sustained, peak_src = load_peaks()
    ms = step_ms / K
    att_avg_s = att_ms / K * 1e-3
    value = whole_job_rate(world, flops, ms) / 1e12
    t_hbm = cache_bytes / (hbm_peak * 1e9)
    t_tc = flops / (tc_peak * 1e12)
    bound = "hbm" if t_hbm >= t_tc else "tensor"
    if bound == "hbm":
        achieved = algo_bytes / att_avg_s / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s", "frac": achieved / hbm_peak,
                "traffic": recorded_traffic(w.name), "peak_source": peak_src + " (burst copy)"}
    else:
        achieved = flops / att_avg_s / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": tc_peak, "unit": "TFLOP/s",
                "frac": achieved / tc_peak, "traffic": recorded_traffic(w.name),
                "peak_source": peak_src + " (burst bf16 GEMM)"}
    roof["kernel"] = "mla_decode_kernel (split-KV attention)"
    roof["kernel_avg_us"] = att_avg_s * 1e6
    roof["roofline_us"] = max(t_hbm, t_tc) * 1e6
    roof["pct_of_roofline"] = max(t_hbm, t_tc) / att_avg_s

    line = {
        "metric": f"MLA decode TFLOP/s ({w.name}: B={B}, s_q={s_q}, H={H})",
        "value": value,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": w.name, "B": B, "s_q": s_q, "H": H, "causal": w.causal, "lengths": w.lengths,
                   "seed": w.seed, "block_size": 64, "softmax_scale": inp.softmax_scale,
                   "l2": "256 MB write before every step, outside the timed events",
                   "parallelism": f"replicas x{world}"},
        "hbm_gbs": algo_bytes / (ms * 1e-3) / 1e9,
        "kernel_tflops": flops / att_avg_s / 1e12,
        "roofline": roof,
        "gpu_launches": 3 * K,
        "clocks": sampler.summary(),
    }
    if e2e is not None:
        line["e2e"] = e2e
    if world == 1 and not args.no_cpu_baseline:
        f, s, n = time_oracle(inp, args.cpu_budget)
        line["cpu_baseline"] = {"value": f / s / 1e12, "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
                                "sample": f"{n} whole sequences of {w.name} ({s:.1f} s, float64 numpy)"}
    print(json.dumps(line))
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
