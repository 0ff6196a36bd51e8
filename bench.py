#!/usr/bin/env python
"""Benchmark of the MLA decode hot path on B200: one step = split-KV schedule
(mla_get_metadata) + attention kernel + LSE-combine kernel over one synthetic batch.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload serving_b256]
                    [--impl ours|reference]

Prints one JSON line (rank 0).  Device times come from CUDA events on the launching
stream, summed over exactly K timed steps; an L2 flush (a 256 MB write, then a 256 MB
read that evicts the dirty lines) runs before every step outside the timed events.  The
line also carries the attention kernel's roofline figures for the other decode
configurations (per_workload).  Multi-GPU runs (torchrun) are
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
def algorithmic_work(seqlens, s_q, H, causal, row_bytes=D_QK * 2):
    """FLOPs = 2 (576 + 512) per (sequence, query token, visible key, head);
    cache bytes = every visible cache row once (row_bytes per (sequence, key): 1152 B
    for the bf16 cache, 656 B for the packed FP8 cache);
    algorithmic bytes = cache bytes + q + out + lse."""
    flops = 0
    keys = 0
    for n in np.asarray(seqlens).tolist():
        keys += max(int(n), 0)
        for i in range(s_q):
            vis = n if not causal else max(0, min(n, n - s_q + i + 1))
            flops += max(vis, 0) * H * 2 * (D_QK + D_LATENT)
    B = len(seqlens)
    cache_bytes = keys * row_bytes
    q_bytes = B * s_q * H * D_QK * 2
    out_bytes = B * s_q * H * D_LATENT * 2 + B * s_q * H * 4
    return flops, cache_bytes, cache_bytes + q_bytes + out_bytes


def ragged_work(seqlens, q_lens, H, causal, row_bytes=D_QK * 2):
    """algorithmic_work with q_lens[b] query tokens for sequence b (the last q_lens[b]
    cache positions): FLOPs over each token's visible keys, the cache rows of every
    sequence with at least one token once, q / out / lse of the tokens."""
    flops = 0
    keys = 0
    tokens = 0
    for n, ql in zip(np.asarray(seqlens).tolist(), np.asarray(q_lens).tolist()):
        if ql <= 0:
            continue
        keys += max(int(n), 0)
        tokens += ql
        for i in range(ql):
            vis = n if not causal else max(0, min(n, n - ql + i + 1))
            flops += max(vis, 0) * H * 2 * (D_QK + D_LATENT)
    cache_bytes = keys * row_bytes
    io_bytes = tokens * H * (D_QK * 2 + D_LATENT * 2 + 4)
    return flops, cache_bytes, cache_bytes + io_bytes


def bench_ragged(mla, dev, steps, warmup, flush, B=128, s_q=4, H=128, seed=1005):
    """Speculative-decoding verification with per-sequence accepted drafts: B = 128
    sequences, up to s_q = 4 query tokens each with q_lens[b] drawn uniformly from
    1..4, causal, lengths U[1024, 8192] as in the MTP workload.  Times two public
    calls (attention and LSE combine, after an L2 flush): mla_decode_ragged over the
    per-sequence schedule and mla_decode_tokens over the token schedule (one s_q = 1
    sequence per query token).  The roofline is the slower of the cache bytes at HBM
    bandwidth and the FLOPs at the bf16 peak.  Returns {name: entry}."""
    import torch
    from deepseek_mla_decode_b200.workloads import make_inputs

    rng = np.random.default_rng(seed + 7919)
    seqlens = rng.integers(1024, 8192 + 1, size=B, dtype=np.int64).astype(np.int32)
    q_lens = rng.integers(1, s_q + 1, size=B, dtype=np.int64).astype(np.int32)
    inp = make_inputs(B, s_q, H, seqlens, seed, causal=True)

    def bf16(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)

    q_nope, q_pe, kv = bf16(inp.q_nope), bf16(inp.q_pe), bf16(inp.kv_cache)
    table = torch.from_numpy(inp.block_table).to(dev)
    lens = torch.from_numpy(inp.cache_seqlens).to(dev)
    qls = torch.from_numpy(q_lens).to(dev)
    st = torch.cuda.current_stream()
    out = torch.empty((B, s_q, H, 512), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, s_q, H), dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    hbm, tc, _, src = load_peaks()
    flops, cache_bytes, _ = ragged_work(seqlens, q_lens, H, True)
    t_hbm, t_tc = cache_bytes / (hbm * 1e9), flops / (tc * 1e12)
    bound = "tensor" if t_tc >= t_hbm else "hbm"
    roof = max(t_hbm, t_tc)
    res = {}
    for name, call in (("mtp_b128_sq4_ragged", "mla_decode_tokens (token schedule; attention + combine)"),
                       ("mtp_b128_sq4_ragged_tiles", "mla_decode_ragged (per-sequence schedule; attention + combine)")):
        tokens = name == "mtp_b128_sq4_ragged"
        if tokens:
            meta = mla.get_metadata_tokens(lens, qls, s_q, H, True, stream=st)
            ws = torch.empty(mla.workspace_size(B * s_q, 1, H), dtype=torch.uint8, device=dev)
            fn = mla.decode_tokens
        else:
            meta = mla.get_metadata(lens, s_q, H, stream=st)
            ws = torch.empty(mla.workspace_size(B, s_q, H), dtype=torch.uint8, device=dev)
            fn = mla.decode_ragged
        for _ in range(warmup):
            fn(q_nope, q_pe, kv, table, lens, qls, inp.softmax_scale, True, meta, workspace=ws, out=out, lse=lse,
               status=status, stream=st)
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
        for e in ev:
            flush()
            e[0].record(st)
            fn(q_nope, q_pe, kv, table, lens, qls, inp.softmax_scale, True, meta, workspace=ws, out=out, lse=lse,
               status=status, stream=st)
            e[1].record(st)
        torch.cuda.synchronize()
        if int(status.item()) != 0:
            raise RuntimeError(f"device status {int(status.item())} in the ragged decode ({name})")
        ms = sum(e[0].elapsed_time(e[1]) for e in ev) / steps
        achieved = flops / (ms * 1e-3) / 1e12 if bound == "tensor" else cache_bytes / (ms * 1e-3) / 1e9
        res[name] = {"workload": f"ragged MTP verification B={B}, s_q<={s_q} (q_lens U[1, {s_q}], mean "
                                 f"{float(q_lens.mean()):.2f}), H={H}, causal, n U[1024, 8192]",
                     "kernel": call, "bound": bound, "achieved": achieved,
                     "peak": tc if bound == "tensor" else hbm, "unit": "TFLOP/s" if bound == "tensor" else "GB/s",
                     "frac": roof / (ms * 1e-3), "peak_source": f"{src}", "call_avg_us": ms * 1e3,
                     "roofline_us": roof * 1e6, "steps": steps}
        del ws
    return res


def prefill_work(S, H):
    """Operations of the causal quantised prefill: 2 (192 + 128) per (head, query,
    visible key), S (S + 1) / 2 visible pairs per head."""
    return 2.0 * (192 + 128) * H * S * (S + 1) / 2


def bench_prefill(mla, dev, steps, warmup, S=None, H=None):
    """Quantised causal prefill (64K tokens, 16 heads, head dim 192) on seeded device
    inputs (N(0, 1) bf16 from a seeded torch generator; the inputs and the quantised
    workspace exceed L2).  Returns the per-workload entry: quantiser and attention
    kernel times (CUDA events) and the attention kernel's tensor roofline against the
    8-bit dense peak (twice the bf16 peak)."""
    import torch
    from deepseek_mla_decode_b200.workloads import PREFILL_S, PREFILL_H, PREFILL_SEED

    S = S or PREFILL_S
    H = H or PREFILL_H
    g = torch.Generator(device=dev).manual_seed(PREFILL_SEED)
    q = torch.randn((S, H, 192), generator=g, device=dev).to(torch.bfloat16)
    k = torch.randn((S, H, 192), generator=g, device=dev).to(torch.bfloat16)
    v = torch.randn((S, H, 128), generator=g, device=dev).to(torch.bfloat16)
    ws = torch.empty(mla.sage_workspace_size(S, H), dtype=torch.uint8, device=dev)
    out = torch.empty((S, H, 128), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((S, H), dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    st = torch.cuda.current_stream()
    scale = 1.0 / math.sqrt(192.0)
    for _ in range(warmup):
        mla.sage_prefill(q, k, v, scale, workspace=ws, out=out, lse=lse, status=status, stream=st)
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    for e in ev:
        e[0].record(st)
        mla.sage_quantize(q, k, v, workspace=ws, stream=st)
        e[1].record(st)
        mla.sage_attention(S, H, scale, ws, out=out, lse=lse, status=status, stream=st)
        e[2].record(st)
    torch.cuda.synchronize()
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} in the prefill")
    quant_ms = sum(e[0].elapsed_time(e[1]) for e in ev) / steps
    att_ms = sum(e[1].elapsed_time(e[2]) for e in ev) / steps
    _, bf16_peak, _, src = load_peaks()
    peak = 2 * bf16_peak
    ops = prefill_work(S, H)
    achieved = ops / (att_ms * 1e-3) / 1e12
    return {"workload": f"causal prefill S={S}, H={H}, head dim 192 / 128", "kernel": "sage_attn_kernel",
            "bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
            "peak_source": f"{src} bf16 GEMM x 2 (dense 8-bit)", "kernel_avg_us": att_ms * 1e3,
            "roofline_us": ops / (peak * 1e12) * 1e6, "quantize_us": quant_ms * 1e3,
            "tokens_per_s": S / ((att_ms + quant_ms) * 1e-3), "steps": steps}


def bench_absorb(mla, dev, steps, warmup, flush, B=256, s_q=1, H=128):
    """The absorption GEMMs either side of the decode at the serving shape: q_nope =
    W_UK^T q_heads and y = W_UV o per head, on seeded device inputs (N(0, 1) rows, N(0,
    0.05^2) weights), each call timed with CUDA events after an L2 flush.  Memory-bound:
    the algorithmic bytes are the rows read and written plus the head weights."""
    import torch

    R = B * s_q
    g = torch.Generator(device=dev).manual_seed(4242)
    q_heads = torch.randn((B, s_q, H, 128), generator=g, device=dev).to(torch.bfloat16)
    o_lat = torch.randn((B, s_q, H, 512), generator=g, device=dev).to(torch.bfloat16)
    w_uk = (0.05 * torch.randn((H, 128, 512), generator=g, device=dev)).to(torch.bfloat16)
    w_uv = (0.05 * torch.randn((H, 128, 512), generator=g, device=dev)).to(torch.bfloat16)
    q_nope = torch.empty((B, s_q, H, 512), dtype=torch.bfloat16, device=dev)
    y = torch.empty((B, s_q, H, 128), dtype=torch.bfloat16, device=dev)
    st = torch.cuda.current_stream()
    for _ in range(warmup):
        mla.absorb_q(q_heads, w_uk, q_nope=q_nope, stream=st)
        mla.absorb_out(o_lat, w_uv, y=y, stream=st)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    for e in ev:
        flush()
        e[0].record(st)
        mla.absorb_q(q_heads, w_uk, q_nope=q_nope, stream=st)
        e[1].record(st)
        flush()
        e[2].record(st)
        mla.absorb_out(o_lat, w_uv, y=y, stream=st)
        e[3].record(st)
    torch.cuda.synchronize()
    hbm, _, _, src = load_peaks()
    wbytes = H * 128 * 512 * 2
    res = {}
    for name, i0, nbytes in (("absorb_q", 0, R * H * (128 + 512) * 2 + wbytes),
                             ("absorb_out", 2, R * H * (512 + 128) * 2 + wbytes)):
        ms = sum(e[i0].elapsed_time(e[i0 + 1]) for e in ev) / steps
        gbs = nbytes / (ms * 1e-3) / 1e9
        res[f"{name}_b{B}"] = {
            "workload": f"{name} B={B}, s_q={s_q}, H={H} (bf16, fp32 accumulation)",
            "kernel": f"absorb_kernel ({name})",
            "bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
            "peak_source": f"{src} HBM copy", "kernel_avg_us": ms * 1e3, "roofline_us": nbytes / (hbm * 1e9) * 1e6,
            "algorithmic_bytes": nbytes, "flops": 2 * R * H * 128 * 512, "steps": steps}
    return res


def metric_name(w):
    """The metric string both arms print, so their lines can be divided."""
    return f"MLA decode TFLOP/s ({w.name}: B={w.B}, s_q={w.s_q}, H={w.H})"


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
            time.sleep(0.002)

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
# device timing
# ---------------------------------------------------------------------------
class L2Flush:
    """Before every step, outside the timed events: a 256 MB write (twice the L2) and
    then a 256 MB read of another buffer.  The read evicts the dirty lines the write
    left, so their write-back does not land inside the next timed kernel, and the step
    starts with none of its own inputs in L2."""

    DESCRIPTION = ("256 MB write then 256 MB read before every step, outside the timed events "
                   "(inputs come from HBM; no dirty lines are written back inside the timed kernel)")

    def __init__(self, dev):
        import torch

        self.w = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        self.r = torch.ones(64 << 20, dtype=torch.float32, device=dev)
        self.sink = torch.empty((), dtype=torch.float32, device=dev)

    def __call__(self):
        import torch

        self.w.zero_()
        torch.sum(self.r, dim=0, out=self.sink)


class DeviceRun:
    """One workload resident on the device, stepped through the C ABI: schedule,
    attention and LSE combine, each bracketed by CUDA events on the launching stream."""

    def __init__(self, mla, inp, dev, fp8=False):
        import torch

        self.mla, self.inp, self.dev, self.fp8 = mla, inp, dev, fp8

        def bf16(bits):
            return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)

        self.q_nope, self.q_pe, self.kv = bf16(inp.q_nope), bf16(inp.q_pe), bf16(inp.kv_cache)
        self.table = torch.from_numpy(inp.block_table).to(dev)
        self.seqlens = torch.from_numpy(inp.cache_seqlens).to(dev)
        B, s_q, H = inp.B, inp.s_q, inp.H
        self.meta = torch.empty((mla.metadata_size(B, s_q, H) + 3) // 4, dtype=torch.int32, device=dev)
        self.ws = torch.empty(mla.workspace_size(B, s_q, H), dtype=torch.uint8, device=dev)
        self.out = torch.empty((B, s_q, H, 512), dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty((B, s_q, H), dtype=torch.float32, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.stream = torch.cuda.current_stream()
        if fp8:  # the packed FP8 cache, quantised once (outside every timed region)
            self.kv = mla.quantize_kv_fp8(self.kv)
            torch.cuda.synchronize()

    def _step(self, ev=None):
        m, i, st = self.mla, self.inp, self.stream
        if ev is not None:
            ev[0].record(st)
        m.get_metadata(self.seqlens, i.s_q, i.H, metadata=self.meta, stream=st)
        if ev is not None:
            ev[1].record(st)
        if self.fp8:
            m.decode_fp8_attention(self.q_nope, self.q_pe, self.kv, self.table, self.seqlens, i.softmax_scale,
                                   i.causal, self.meta, self.ws, self.out, self.lse, status=self.status, stream=st)
        else:
            m.decode_attention(self.q_nope, self.q_pe, self.kv, self.table, self.seqlens, i.softmax_scale, i.causal,
                               self.meta, self.ws, self.out, self.lse, status=self.status, stream=st)
        if ev is not None:
            ev[2].record(st)
        m.decode_combine(self.seqlens, self.table.shape[1], i.s_q, i.H, self.meta, self.ws, self.out, self.lse,
                         status=self.status, stream=st)
        if ev is not None:
            ev[3].record(st)

    def steps(self, n, flush, timed=False, per_launch=True):
        """n steps with an L2 flush before each; with timed=True returns the summed
        milliseconds of the step and, with per_launch, of each launch (device events).
        Events between the launches make each launch wait for the previous one to
        finish, so the per-launch pass is the serialised one; without them the
        attention and combine kernels start their setup while their predecessor
        finishes (programmatic dependent launch), as they do in a real decode step."""
        import torch

        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n)] if timed else None
        for k in range(n):
            flush()
            if timed and not per_launch:
                evs[k][0].record(self.stream)
                self._step(None)
                evs[k][3].record(self.stream)
            else:
                self._step(evs[k] if timed else None)
        if not timed:
            return None
        torch.cuda.synchronize()
        tot = {"step": 0.0, "metadata": 0.0, "attention": 0.0, "combine": 0.0}
        for e in evs:
            tot["step"] += e[0].elapsed_time(e[3])
            if per_launch:
                tot["metadata"] += e[0].elapsed_time(e[1])
                tot["attention"] += e[1].elapsed_time(e[2])
                tot["combine"] += e[2].elapsed_time(e[3])
        return tot

    def check_status(self, where):
        v = int(self.status.item())
        if v != 0:
            raise RuntimeError(f"device status {v} in {where}")

    def e2e(self, n):
        """n steps through the public mla_decode call with pinned host inputs copied in
        and out inside the timed region; returns (ms per step, H2D bytes, D2H bytes)."""
        import torch

        i, m, st = self.inp, self.mla, self.stream
        # the cache as the caller holds it: bf16 rows, or the packed FP8 rows
        kv_host = self.kv.cpu().numpy() if self.fp8 else i.kv_cache.view(np.int16)
        h = {k: torch.from_numpy(np.ascontiguousarray(v)).pin_memory() for k, v in
             (("q_nope", i.q_nope.view(np.int16)), ("q_pe", i.q_pe.view(np.int16)),
              ("kv", kv_host), ("table", i.block_table), ("seq", i.cache_seqlens))}
        h_out = torch.empty(self.out.shape, dtype=torch.bfloat16).pin_memory()
        h_lse = torch.empty(self.lse.shape, dtype=torch.float32).pin_memory()
        d = {k: torch.empty(v.shape, dtype=v.dtype, device=self.dev) for k, v in h.items()}
        h2d = sum(v.numel() * v.element_size() for v in h.values())
        d2h = h_out.numel() * 2 + h_lse.numel() * 4

        def one():
            for k in h:
                d[k].copy_(h[k], non_blocking=True)
            meta = m.get_metadata(d["seq"], i.s_q, i.H, metadata=self.meta, stream=st)
            if self.fp8:
                m.decode_fp8(d["q_nope"].view(torch.bfloat16), d["q_pe"].view(torch.bfloat16), d["kv"], d["table"],
                             d["seq"], i.softmax_scale, i.causal, meta, workspace=self.ws, out=self.out,
                             lse=self.lse, status=self.status, stream=st)
            else:
                m.decode(d["q_nope"].view(torch.bfloat16), d["q_pe"].view(torch.bfloat16), d["kv"].view(torch.bfloat16),
                         d["table"], d["seq"], i.softmax_scale, i.causal, meta, workspace=self.ws, out=self.out,
                         lse=self.lse, status=self.status, stream=st)
            h_out.copy_(self.out, non_blocking=True)
            h_lse.copy_(self.lse, non_blocking=True)

        for _ in range(2):
            one()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(st)
        for _ in range(n):
            one()
        e1.record(st)
        torch.cuda.synchronize()
        self.check_status("the end-to-end steps")
        return e0.elapsed_time(e1) / n, h2d, d2h


def roofline(inp, t, steps, fp8=False):
    """Roofline figures of the attention kernel from summed device milliseconds.

    Roofline time = max(cache bytes / HBM peak, FLOPs / bf16 peak); `achieved` is the
    algorithmic bytes (HBM-bound) or FLOPs (tensor-bound) per launch over the kernel's
    average duration; pct_of_roofline = roofline time / kernel time, and
    pct_of_roofline_decode the same over the whole mla_decode call (attention +
    combine)."""
    hbm_peak, tc_peak, _, peak_src = load_peaks()
    flops, cache_bytes, algo_bytes = algorithmic_work(inp.cache_seqlens, inp.s_q, inp.H, inp.causal,
                                                      656 if fp8 else D_QK * 2)
    att_s = t["attention"] / steps * 1e-3
    t_hbm = cache_bytes / (hbm_peak * 1e9)
    t_tc = flops / (tc_peak * 1e12)
    if t_hbm >= t_tc:
        achieved = algo_bytes / att_s / 1e9
        r = {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s", "frac": achieved / hbm_peak,
             "peak_source": f"{peak_src} (burst copy)"}
    else:
        achieved = flops / att_s / 1e12
        r = {"bound": "tensor", "achieved": achieved, "peak": tc_peak, "unit": "TFLOP/s", "frac": achieved / tc_peak,
             "peak_source": f"{peak_src} (burst bf16 GEMM)"}
    r["kernel"] = "mla_decode_kernel<fp8> (split-KV attention, FP8 cache)" if fp8 else \
        "mla_decode_kernel (split-KV attention)"
    r["kernel_avg_us"] = att_s * 1e6
    r["roofline_us"] = max(t_hbm, t_tc) * 1e6
    r["pct_of_roofline"] = max(t_hbm, t_tc) / att_s
    r["step_us"] = t["step"] / steps * 1e3
    r["step_without_metadata_us"] = (t["step"] - t["metadata"]) / steps * 1e3
    r["pct_of_roofline_decode"] = max(t_hbm, t_tc) / ((t["attention"] + t["combine"]) / steps * 1e-3)
    return r


# ---------------------------------------------------------------------------
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="serving_b256", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--prefill-steps", type=int, default=5,
                    help="timed runs of the quantised 64K-token prefill (0 = skip)")
    ap.add_argument("--prefill-shape", default="65536,16", help="S,H of the quantised prefill")
    ap.add_argument("--ragged-steps", type=int, default=30,
                    help="timed calls of the ragged-query-count MTP verification (0 = skip)")
    ap.add_argument("--absorb-steps", type=int, default=30,
                    help="timed calls of each absorption GEMM at the serving shape (0 = skip)")
    ap.add_argument("--kv-format", default="bf16", choices=["bf16", "fp8"],
                    help="cache of the headline run: bf16 rows, or the packed FP8 rows (quantised once, untimed)")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle time for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--per-workload-steps", type=int, default=30,
                    help="timed steps for each of the other decode configurations (0 = skip)")
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
            "impl": "reference", "metric": metric_name(w), "value": value, "unit": "TFLOP/s",
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
    flusher = L2Flush(dev)

    inp = make_workload(args.workload)
    flops, cache_bytes, algo_bytes = algorithmic_work(inp.cache_seqlens, inp.s_q, inp.H, inp.causal)
    B, s_q, H = inp.B, inp.s_q, inp.H
    fp8 = args.kv_format == "fp8"
    if fp8:
        flops, cache_bytes, algo_bytes = algorithmic_work(inp.cache_seqlens, inp.s_q, inp.H, inp.causal, 656)
    run = DeviceRun(mla, inp, dev, fp8=fp8)

    run.steps(args.warmup, flusher)
    torch.cuda.synchronize()
    run.check_status("warm-up")

    K = args.steps
    uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(uuid)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with sampler:
        t = run.steps(K, flusher, timed=True, per_launch=False)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    run.check_status("the timed region")
    # second pass of K steps: events around every launch (serialised launches) give
    # the per-kernel times, the attention kernel's among them for the roofline
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    tk = run.steps(K, flusher, timed=True, per_launch=True)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    run.check_status("the per-launch pass")
    step_ms, meta_ms, att_ms, comb_ms, step_ser_ms = max_over_ranks(
        [t["step"], tk["metadata"], tk["attention"], tk["combine"], tk["step"]], world, dev, dist)

    # ---- end to end through the public API with host buffers ---------------
    e2e = None
    if args.e2e_steps > 0:
        e2e_ms, h2d, d2h = run.e2e(args.e2e_steps)
        if world > 1:
            dist.barrier()
        (e2e_ms,) = max_over_ranks([e2e_ms], world, dev, dist)
        e2e = {"value": whole_job_rate(world, flops, e2e_ms) / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h), "ms_per_step": e2e_ms}

    # ---- the other decode configurations: attention-kernel figures ----------
    per_workload = {}
    if world == 1 and args.per_workload_steps > 0:
        del run
        torch.cuda.empty_cache()
        for name in ("decode_b64", "mtp_b128_sq2", "serving_b256", "long_b4"):
            if name == args.workload and not fp8:
                continue
            wi = make_workload(name)
            ri = DeviceRun(mla, wi, dev)
            ri.steps(args.warmup, flusher)
            ti = ri.steps(args.per_workload_steps, flusher, timed=True)
            torch.cuda.synchronize()
            ri.check_status(name)
            per_workload[name] = roofline(wi, ti, args.per_workload_steps)
            del ri
            torch.cuda.empty_cache()
        # the four full-size decode configurations over the packed FP8 cache (656-byte rows)
        for name in ("serving_b256", "decode_b64", "mtp_b128_sq2", "long_b4"):
            if name == args.workload and fp8:
                continue
            wi = make_workload(name)
            ri = DeviceRun(mla, wi, dev, fp8=True)
            ri.steps(args.warmup, flusher)
            ti = ri.steps(args.per_workload_steps, flusher, timed=True)
            torch.cuda.synchronize()
            ri.check_status(name + " (fp8)")
            per_workload[name + "_fp8"] = roofline(wi, ti, args.per_workload_steps, fp8=True)
            del ri
            torch.cuda.empty_cache()

    if world == 1 and args.ragged_steps > 0:
        per_workload.update(bench_ragged(mla, dev, args.ragged_steps, args.warmup, flusher))
        torch.cuda.empty_cache()

    if world == 1 and args.absorb_steps > 0:
        per_workload.update(bench_absorb(mla, dev, args.absorb_steps, args.warmup, flusher))
        torch.cuda.empty_cache()

    if world == 1 and args.prefill_steps > 0:
        pS, pH = (int(x) for x in args.prefill_shape.split(","))
        per_workload[f"prefill_s{pS}_h{pH}"] = bench_prefill(mla, dev, args.prefill_steps, 2, pS, pH)
        torch.cuda.empty_cache()

    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return

    ms = step_ms / K
    value = whole_job_rate(world, flops, ms) / 1e12
    roof = roofline(inp, {"attention": att_ms, "step": step_ser_ms, "metadata": meta_ms, "combine": comb_ms}, K,
                    fp8=fp8)
    per_workload[w.name + ("_fp8" if fp8 else "")] = {
        k: roof[k] for k in ("bound", "kernel_avg_us", "roofline_us", "pct_of_roofline", "frac", "step_us",
                             "step_without_metadata_us", "pct_of_roofline_decode")}
    roof["traffic"] = recorded_traffic(w.name + ("_fp8" if fp8 else ""))

    line = {
        "metric": metric_name(w) + (" [FP8 cache]" if fp8 else ""),
        "value": value,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if not fp8 else "bf16 (e4m3 cache)",
        "data": "synthetic",
        "config": {"workload": w.name, "kv_format": args.kv_format, "B": B, "s_q": s_q, "H": H, "causal": w.causal,
                   "lengths": w.lengths,
                   "seed": w.seed, "block_size": 64, "softmax_scale": inp.softmax_scale,
                   "l2": L2Flush.DESCRIPTION,
                   "parallelism": f"replicas x{world}"},
        "hbm_gbs": algo_bytes / (ms * 1e-3) / 1e9,
        "kernel_tflops": flops / (att_ms / K * 1e-3) / 1e12,
        "metadata_us": meta_ms / K * 1e3,
        "combine_us": comb_ms / K * 1e3,
        "step_serialised_us": step_ser_ms / K * 1e3,
        "step_without_metadata_us": (step_ser_ms - meta_ms) / K * 1e3,
        "timing": ("value / ms_per_step: K steps with events only at step boundaries; metadata_us, "
                   "roofline.kernel_avg_us, combine_us: a second pass of K steps with events around "
                   "every launch (those events serialise the launches)"),
        "roofline": roof,
        "per_workload": per_workload,
        "gpu_launches": 3 * K,
        "clocks": sampler.summary(),
    }
    if e2e is not None:
        line["e2e"] = e2e
    if world == 1 and not args.no_cpu_baseline:
        f, s_, n = time_oracle(inp, args.cpu_budget)
        line["cpu_baseline"] = {"value": f / s_ / 1e12, "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
                                "sample": f"{n} whole sequences of {w.name} ({s_:.1f} s, float64 numpy)"}
    print(json.dumps(line))
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
