"""Throughput of exact tiled attention on B200: prefill TFLOP/s and split-KV decode KV GB/s.

python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mfa|reference] [--workload NAME]

One step = one pass of the hot path over one batch: the prefill forward of the named workload
(default: causal, B=2, H=8, N=4096, D=128, fp16). The same JSON line also carries the other
workloads (non-causal, sliding window, GQA + softcap prefill, packed variable-length prefill,
block-sparse prefill, chunked prefill over a paged cache, paged split-KV decode, and the backward
of the two B=2 H=8 N=4096 workloads), each timed the same way. Inputs are seeded synthetic tensors resident in HBM; L2 is flushed (a 256 MiB
write) before every timed step, outside the timed kernel. Times are CUDA events on the launching
stream; with N > 1 (torchrun, one process per GPU) the problem is sharded by (sequence, kv-head)
units with no exchange -- by default a batch N times the workload's, each GPU owning its slice
(weak scaling; --scaling strong splits the workload's own units instead) -- the max over ranks is
reported, and a decode line spreads every sequence's splits over the GPUs with one NCCL
all-gather of the partial results before the combine.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import mfa_inputs as mi  # noqa: E402

MAIN = "causal_b2_h8_n4096_d128_fp16"
# The pages' own forward timings on an Apple M1 Max (f16, "mlx-mfa 2.5.2", Performance tables:
# the dense causal table and the sliding-window table), for the workloads of the same shape.
# Context only: another machine, another kernel.
PAGES_M1_MAX_MS = {
    "causal_b2_h8_n4096_d128_fp16": 11.5,
    "causal_b2_h8_n8192_d128_fp16": 44.1,
    "window512_b2_h8_n8192_d128_fp16": 6.2,
    "window256_b2_h8_n8192_d128_fp16": 3.6,
}
PAGES_SOURCE = "mlx-mfa 2.5.2, Performance tables (Apple M1 Max, f16, ms per forward)"
METRIC = "attention TFLOP/s (prefill) and KV GB/s (split-KV decode) vs B200 peak"
NOMINAL_TFLOPS = 2250.0
NOMINAL_GBS = 8000.0
L2_FLUSH_BYTES = 256 << 20


# --------------------------------------------------------------------------- work accounting
def visible_pairs(case, Nq=None, Nk=None) -> int:
    """Visible (query, key) pairs of one head, summed row by row from the interval form."""
    Nq = case.Nq if Nq is None else int(Nq)
    Nk = case.Nk if Nk is None else int(Nk)
    i = np.arange(Nq, dtype=np.int64)
    a = i + (Nk - Nq)
    lo = np.zeros_like(a) if case.win_l < 0 else np.maximum(0, a - case.win_l)
    hi = np.full_like(a, Nk - 1)
    if case.causal:
        hi = np.minimum(hi, a)
    if case.win_r >= 0:
        hi = np.minimum(hi, a + case.win_r)
    return int(np.maximum(0, hi - lo + 1).sum())


def prefill_flops(case) -> float:
    return 4.0 * case.D * case.B * case.Hq * visible_pairs(case)


def prefill_bytes(case) -> float:
    e = 2
    return (e * case.B * case.Hq * case.Nq * case.D * 2 + e * 2 * case.B * case.Hkv * case.Nk * case.D
            + 4 * case.B * case.Hq * case.Nq)


def sparse_pairs(case, mask) -> int:
    """Visible (query, key) pairs summed over batch and heads: the causal / window interval of
    each row intersected with the key blocks its 128-row mask row has on."""
    blk = mi.SPARSE_BLOCK
    i = np.arange(case.Nq, dtype=np.int64)
    a = i + (case.Nk - case.Nq)
    lo = np.zeros_like(a) if case.win_l < 0 else np.maximum(0, a - case.win_l)
    hi = np.full_like(a, case.Nk - 1)
    if case.causal:
        hi = np.minimum(hi, a)
    if case.win_r >= 0:
        hi = np.minimum(hi, a + case.win_r)
    nkb = mask.shape[3]
    kb_lo = np.arange(nkb, dtype=np.int64) * blk
    kb_hi = np.minimum(kb_lo + blk - 1, case.Nk - 1)
    # overlap[i, kb] of row i's interval with key block kb
    ov = np.maximum(0, np.minimum(hi[:, None], kb_hi[None, :]) - np.maximum(lo[:, None], kb_lo[None, :]) + 1)
    total = 0
    for b in range(mask.shape[0]):
        for h in range(mask.shape[1]):
            on = mask[b, h][i // blk].astype(bool)          # [Nq, nkb]
            total += int((ov * on).sum())
    return total


def varlen_flops(case) -> float:
    nq, nk = case.lens()
    return 4.0 * case.D * case.Hq * sum(visible_pairs(case, a, b) for a, b in zip(nq, nk))


def varlen_bytes(case) -> float:
    nq, nk = case.lens()
    tq, tk = int(nq.sum()), int(nk.sum())
    return 2 * tq * case.Hq * case.D * 2 + 2 * 2 * tk * case.Hkv * case.D + 4 * tq * case.Hq


def decode_tokens(case, lens):
    """(cached tokens some query row sees, visible (row, token) pairs) summed over sequences:
    row t of a sequence of length L sees tokens [L - Nq + t - win_l, L - Nq + t] (causal) or
    [L - Nq + t - win_l, L - 1], clipped to [0, L)."""
    toks = pairs = 0
    for L in (int(x) for x in lens):
        lo_all = L
        for t in range(case.Nq):
            hi = min(L - case.Nq + t, L - 1) if case.causal else L - 1
            lo = max(0, L - case.Nq + t - case.win_l) if case.win_l >= 0 else 0
            pairs += max(0, hi - lo + 1)
            lo_all = min(lo_all, lo)
        toks += L - lo_all
    return toks, pairs


def decode_bytes(case, lens) -> float:
    kv = float(decode_tokens(case, lens)[0]) * case.Hkv * case.D * 2 * 2
    return kv + case.B * case.Hq * case.Nq * case.D * 2 * 2 + 4 * case.B * case.Hq * case.Nq


def decode_flops(case, lens) -> float:
    return 4.0 * case.D * case.Hq * float(decode_tokens(case, lens)[1])


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return {"tflops": d["bf16_tflops"], "tflops_sustained": d["bf16_tflops_sustained"],
                "gbs": d["hbm_gbs"], "source": "measured"}
    return {"tflops": 1590.0, "tflops_sustained": 1400.0, "gbs": 6650.0, "source": "fallback"}


KERNEL_SOURCES = {
    "mfa_fwd_kernel": ("fwd_kernel.cuh", "sm100.cuh"),
    "mfa_decode_phase1_kernel": ("decode_kernel.cuh", "sm100.cuh"),
}


def kernel_source_hash(kernel: str = "mfa_fwd_kernel") -> str:
    """Hash of the source files a kernel is built from (a changed kernel invalidates its record)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "tiled_exact_attention_mfa_b200", "csrc")
    for f in KERNEL_SOURCES[kernel]:
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def ncu_traffic(workload: str, kernel: str):
    """DRAM bytes per launch from the committed ncu summary, or None when the kernel sources
    changed since that capture."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.txt")
    if not os.path.exists(path):
        return None
    cur = kernel_source_hash(kernel)
    for line in open(path):
        parts = line.split()
        if len(parts) == 4 and not line.startswith("#") and parts[0] == workload and parts[1] == kernel:
            return float(parts[3]) if parts[2] == cur else None
    return None


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.proc = None
        self.gpu = gpu_index

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu), "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "samples": len(sm), "reasons": sorted(reasons)}


def parallelism(name: str, world: int, scaling: str) -> str:
    c = mi.workloads()[name]
    units = c.B * c.Hkv
    if scaling == "strong":
        return (f"sharded: the {units} (sequence, kv-head) units of the workload split over "
                f"{world} GPU(s), no exchange")
    return (f"sharded: a batch of {world} x {c.B} sequences, {units} (sequence, kv-head) units "
            f"per GPU on {world} GPU(s), no exchange")


def main_config(name: str, world: int, scaling: str = "weak") -> dict:
    """The `config` of the headline line, shared by the GPU arm and the reference arm."""
    c = mi.workloads()[name]
    return {"workload": name, "B": c.B, "Hq": c.Hq, "Hkv": c.Hkv, "N": c.Nq, "D": c.D,
            "causal": c.causal, "window": [c.win_l, c.win_r], "softcap": c.softcap,
            "dtype": mi.DTYPE_NAMES[c.dtype],
            "l2": "flushed before every timed step (256 MiB write)",
            "parallelism": parallelism(name, world, scaling)}


def pages_context(name: str) -> dict:
    """The pages' M1 Max time for this workload's shape, when they print one."""
    if name not in PAGES_M1_MAX_MS:
        return {}
    return {"pages_m1_max_ms": PAGES_M1_MAX_MS[name], "pages_source": PAGES_SOURCE}


# --------------------------------------------------------------------------- GPU arm
def upload(bits, dtype, dev):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.float16 if dtype == mi.FP16 else torch.bfloat16).to(dev)


def time_steps(fn, steps, warmup, flush, stream):
    """Run warmup untimed steps, then `steps` timed ones with an L2 flush before each.
    Returns per-step kernel milliseconds (CUDA events on `stream`) and the bracketed total."""
    import torch
    for _ in range(warmup):
        flush()
        fn()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    b0.record(stream)
    for s, e in ev:
        flush()
        s.record(stream)
        fn()
        e.record(stream)
    b1.record(stream)
    torch.cuda.synchronize()
    return [s.elapsed_time(e) for s, e in ev], b0.elapsed_time(b1)


def spread(ms):
    """Median and 10th / 90th percentiles of one rank's per-step times (ms)."""
    xs = sorted(ms)
    if not xs:
        return {}

    def pct(q):  # linear interpolation between order statistics
        pos = q * (len(xs) - 1)
        lo = int(pos)
        hi = min(lo + 1, len(xs) - 1)
        return xs[lo] + (xs[hi] - xs[lo]) * (pos - lo)
    return {"ms_median": round(pct(0.5), 5), "ms_p10": round(pct(0.1), 5),
            "ms_p90": round(pct(0.9), 5)}


def spread_of(r):
    return {k: r[k] for k in ("ms_median", "ms_p10", "ms_p90") if k in r}


def max_over_ranks(x: float, world: int, device: str = "cuda") -> float:
    """Largest per-rank time: the job takes as long as its slowest rank."""
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, world: int, max_ms: float) -> float:
    """Whole-job rate: the units all ranks processed divided by the slowest rank's time (per s)."""
    return units_per_rank * world / (max_ms * 1e-3)


def bench_prefill(case, steps, warmup, flush, stream, with_e2e, world, rank=0, scaling="weak"):
    """One prefill workload. With N > 1 ranks the problem is sharded by (sequence, kv head)
    units with no exchange: scaling "weak" makes the job N x the workload's batch, rank r owning
    batch rows [r B, (r + 1) B) (its own slice of the seeded inputs); "strong" splits the
    workload itself, rank r running its contiguous range of units. res["job_flops"] is the work of
    the whole job."""
    import torch
    import tiled_exact_attention_mfa_b200 as mfa
    from tiled_exact_attention_mfa_b200 import shard
    dev = torch.device("cuda")
    weak = scaling == "weak"
    q, k, v = case.batch_slice_tensors(rank) if (world > 1 and weak) else case.tensors()
    qt, kt, vt = (upload(x, case.dtype, dev) for x in (q, k, v))
    out = torch.empty_like(qt)
    lse = torch.empty(case.B, case.Hq, case.Nq, dtype=torch.float32, device=dev)
    scale = case.scale_f32()
    win = (case.win_l, case.win_r)
    kw = dict(scale=scale, causal=case.causal, window=win, softcap=case.softcap, stream=stream)

    if weak or world == 1:
        def step():
            mfa.mfa_fwd(qt, kt, vt, out, lse, **kw)
    else:
        def step():
            shard.fwd_sharded(qt, kt, vt, out, lse, world, rank, **kw)

    with torch.cuda.stream(stream):
        ms, bracket = time_steps(step, steps, warmup, flush, stream)
    res = {"ms": statistics.mean(ms), "ms_min": min(ms), **spread(ms), "bracket_ms": bracket,
           "flops": prefill_flops(case), "bytes": prefill_bytes(case)}
    res["job_flops"] = res["flops"] * (world if weak else 1)
    res["ms"] = max_over_ranks(res["ms"], world)

    if with_e2e:
        # the C-ABI call with host buffers (mfa_fwd_host): every step copies q, k, v from pinned
        # host memory, runs the forward and copies out and lse back, all inside the timed region
        torch_dt = qt.dtype
        hq = torch.from_numpy(q.view(np.int16)).view(torch_dt).pin_memory()
        hk = torch.from_numpy(k.view(np.int16)).view(torch_dt).pin_memory()
        hv = torch.from_numpy(v.view(np.int16)).view(torch_dt).pin_memory()
        ho = torch.empty(out.shape, dtype=torch_dt).pin_memory()
        hl = torch.empty(lse.shape, dtype=torch.float32).pin_memory()
        scratch = torch.empty(mfa.mfa_fwd_host_scratch_size(case.B, case.Hq, case.Hkv, case.Nq,
                                                            case.Nk, case.D),
                              dtype=torch.uint8, device=dev)

        if weak or world == 1:
            e_in = (hq, hk, hv, ho, hl)
        else:  # this rank's units: contiguous slices of the host tensors
            e_in = shard.prefill_shard_views(hq, hk, hv, ho, hl, world, rank)
            eq = e_in[0]
            scratch = torch.empty(mfa.mfa_fwd_host_scratch_size(eq.shape[0], eq.shape[1], 1,
                                                                case.Nq, case.Nk, case.D),
                                  dtype=torch.uint8, device=dev)

        def e2e_step():
            mfa.mfa_fwd_host(*e_in, scale=scale, causal=case.causal, window=win,
                             softcap=case.softcap, scratch=scratch, stream=stream)

        with torch.cuda.stream(stream):
            ems, _ = time_steps(e2e_step, max(3, steps // 2), 2, flush, stream)
        torch.cuda.synchronize()
        dev_parts = (out.cpu(), lse.cpu())
        if not (weak or world == 1):  # compare this rank's slices only
            dev_parts = shard.prefill_shard_views(qt.cpu(), kt.cpu(), vt.cpu(), *dev_parts, world,
                                                  rank)[3:]
            host_parts = e_in[3:]
        else:
            host_parts = (ho, hl)
        if not all(torch.equal(a, b) for a, b in zip(host_parts, dev_parts)):
            raise RuntimeError("host-buffer forward differs from the device forward")
        res["e2e_ms"] = max_over_ranks(statistics.mean(ems), world)
        # the PCIe floor on this machine, same run: the step's own pinned inputs copied in alone
        dq_, dk_, dv_ = (torch.empty_like(x, device=dev) for x in (hq, hk, hv))

        def h2d_only():
            dq_.copy_(hq, non_blocking=True)
            dk_.copy_(hk, non_blocking=True)
            dv_.copy_(hv, non_blocking=True)

        with torch.cuda.stream(stream):
            hms, _ = time_steps(h2d_only, 5, 2, flush, stream)
        res["h2d_alone_ms"] = statistics.mean(hms)
        res["h2d"] = int(sum(t.numel() * t.element_size() for t in e_in[:3]))
        res["d2h"] = int(sum(t.numel() * t.element_size() for t in e_in[3:]))
    return res


def bench_decode_sharded(case, steps, warmup, flush, stream, world, rank):
    """Split-KV decode with each sequence's splits spread over the ranks: rank r computes phase 1
    for its block of splits (it reads only those pages), the partial blocks are all-gathered over
    NCCL, and every rank runs the combine. The time of a step includes the exchange."""
    import torch
    import tiled_exact_attention_mfa_b200 as mfa
    from tiled_exact_attention_mfa_b200 import shard
    dev = torch.device("cuda")
    q, kp, vp, table, lens = case.tensors()
    qt, kt, vt = (upload(x, case.dtype, dev) for x in (q, kp, vp))
    tt, lt = torch.from_numpy(table).to(dev), torch.from_numpy(lens).to(dev)
    out = torch.empty_like(qt)
    lse = torch.empty(case.B, case.Hq, case.Nq, dtype=torch.float32, device=dev)
    plan = mfa.mfa_decode_plan(case.B, case.Nq, case.Hq, case.Hkv, case.D, table.shape[1], 16,
                               case.win_l)
    so, sm = shard.decode_partial_shapes(case.B, case.Nq, case.Hq, case.D, plan["max_splits"], world)
    po = torch.empty(so, dtype=torch.float32, device=dev)
    pm = torch.empty(sm, dtype=torch.float32, device=dev)

    def step():
        shard.decode_sharded(qt, kt, vt, tt, lt, out, lse, po, pm, world, rank,
                             scale=case.scale_f32(), causal=case.causal, softcap=case.softcap,
                             win_l=case.win_l)

    with torch.cuda.stream(stream):
        ms, bracket = time_steps(step, steps, warmup, flush, stream)
    return {"ms": max_over_ranks(statistics.mean(ms), world), "ms_min": min(ms), **spread(ms),
            "bracket_ms": bracket, "bytes": decode_bytes(case, lens),
            "exchange_bytes": int(4 * case.B * case.Hq * case.Nq * (case.D + 2) *
                                  shard.split_chunk(plan["max_splits"], world) * (world - 1))}


def host_call_us(case, stream, calls=200):
    """Host time of one forward call through the Python binding and the C ABI (argument checks,
    tensor maps from the library's cache, the launch), averaged over back-to-back calls."""
    import torch
    import tiled_exact_attention_mfa_b200 as mfa
    dev = torch.device("cuda")
    qt, kt, vt = (upload(x, case.dtype, dev) for x in case.tensors())
    out = torch.empty_like(qt)
    lse = torch.empty(case.B, case.Hq, case.Nq, dtype=torch.float32, device=dev)
    kw = dict(scale=case.scale_f32(), causal=case.causal, window=(case.win_l, case.win_r),
              softcap=case.softcap, stream=stream)
    for _ in range(10):
        mfa.mfa_fwd(qt, kt, vt, out, lse, **kw)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for _ in range(calls):
        mfa.mfa_fwd(qt, kt, vt, out, lse, **kw)
    dt = time.perf_counter() - t0
    torch.cuda.synchronize()
    return round(dt / calls * 1e6, 2)


def bench_varlen(case, steps, warmup, flush, stream, world):
    import torch
    import tiled_exact_attention_mfa_b200 as mfa
    dev = torch.device("cuda")
    q, k, v = case.tensors()
    cq, ck = case.cu_seqlens()
    qt, kt, vt = (upload(x, case.dtype, dev) for x in (q, k, v))
    cqt, ckt = torch.from_numpy(cq).to(dev), torch.from_numpy(ck).to(dev)
    out = torch.empty_like(qt)
    lse = torch.empty(case.Hq, qt.shape[0], dtype=torch.float32, device=dev)
    max_q = int(case.lens()[0].max())
    scale = case.scale_f32()

    def step():
        mfa.mfa_fwd_varlen(qt, kt, vt, cqt, ckt, max_q, out, lse, scale=scale, causal=case.causal,
                           window=(case.win_l, case.win_r), softcap=case.softcap, stream=stream)

    with torch.cuda.stream(stream):
        ms, bracket = time_steps(step, steps, warmup, flush, stream)
    return {"ms": max_over_ranks(statistics.mean(ms), world), "ms_min": min(ms), **spread(ms),
            "bracket_ms": bracket, "flops": varlen_flops(case), "bytes": varlen_bytes(case),
            "total_q": int(cq[-1])}


def bench_sparse(case, steps, warmup, flush, stream, world):
    import torch
    import tiled_exact_attention_mfa_b200 as mfa
    dev = torch.device("cuda")
    q, k, v, m = case.tensors()
    qt, kt, vt = (upload(x, case.dtype, dev) for x in (q, k, v))
    mt = torch.from_numpy(m).to(dev)
    out = torch.empty_like(qt)
    lse = torch.empty(case.B, case.Hq, case.Nq, dtype=torch.float32, device=dev)
    scale = case.scale_f32()

    def step():
        mfa.mfa_fwd_blocksparse(qt, kt, vt, mt, out, lse, scale=scale, causal=case.causal,
                                window=(case.win_l, case.win_r), softcap=case.softcap, stream=stream)

    with torch.cuda.stream(stream):
        ms, bracket = time_steps(step, steps, warmup, flush, stream)
    pairs = sparse_pairs(case, m)
    byts = 2 * case.B * case.Hq * case.Nq * case.D * 2 + 2 * 2 * case.B * case.Hkv * case.Nk * case.D \
        + 4 * case.B * case.Hq * case.Nq + m.size
    return {"ms": max_over_ranks(statistics.mean(ms), world), "ms_min": min(ms), **spread(ms),
            "bracket_ms": bracket, "flops": 4.0 * case.D * pairs, "bytes": float(byts),
            "density": float(m.mean())}


def bench_backward(case, steps, warmup, flush, stream, world):
    """mfa_bwd alone on the forward's outputs (computed once, outside the timed region).
    Algorithmic work: 5 matmuls over the visible pairs (S recomputed, dP, dV, dK, dQ)."""
    import torch
    import tiled_exact_attention_mfa_b200 as mfa
    dev = torch.device("cuda")
    q, k, v = case.tensors()
    qt, kt, vt = (upload(x, case.dtype, dev) for x in (q, k, v))
    win = (case.win_l, case.win_r)
    out, lse = mfa.mfa_fwd(qt, kt, vt, scale=case.scale_f32(), causal=case.causal, window=win,
                           softcap=case.softcap, stream=stream)
    dout = upload(case.dout(),
                  case.dtype, dev)
    dq, dk, dv = torch.empty_like(qt), torch.empty_like(kt), torch.empty_like(vt)
    ws = torch.empty(max(mfa.mfa_bwd_workspace_size(case.B, case.Hq, case.Nq), 256),
                     dtype=torch.uint8, device=dev)

    def step():
        mfa.mfa_bwd(qt, kt, vt, out, dout, lse, dq, dk, dv, scale=case.scale_f32(),
                    causal=case.causal, window=win, softcap=case.softcap, workspace=ws,
                    stream=stream)

    with torch.cuda.stream(stream):
        ms, bracket = time_steps(step, steps, warmup, flush, stream)
    return {"ms": max_over_ranks(statistics.mean(ms), world), "ms_min": min(ms), **spread(ms),
            "bracket_ms": bracket, "flops": 2.5 * prefill_flops(case),
            "bytes": 2.0 * prefill_bytes(case)}


BACKWARD_WORKLOADS = ("causal_b2_h8_n4096_d128_fp16", "noncausal_b2_h8_n4096_d128_fp16")


def bench_paged(case, steps, warmup, flush, stream, world):
    import torch
    import tiled_exact_attention_mfa_b200 as mfa
    dev = torch.device("cuda")
    q, kp, vp, table, lens, cq = case.tensors()
    qt, kt, vt = (upload(x, case.dtype, dev) for x in (q, kp, vp))
    tt, lt, ct = (torch.from_numpy(x).to(dev) for x in (table, lens, cq))
    out = torch.empty_like(qt)
    lse = torch.empty(case.Hq, qt.shape[0], dtype=torch.float32, device=dev)
    nq = np.diff(cq)
    max_q = int(nq.max())
    scale = case.scale_f32()

    def step():
        mfa.mfa_fwd_paged(qt, kt, vt, tt, lt, ct, max_q, out, lse, scale=scale, causal=case.causal,
                          window=(case.win_l, case.win_r), softcap=case.softcap, stream=stream)

    with torch.cuda.stream(stream):
        ms, bracket = time_steps(step, steps, warmup, flush, stream)
    pairs = sum(visible_pairs(case_like(case), a, b) for a, b in zip(nq, lens))
    kv_bytes = float(np.sum(lens)) * case.Hkv * case.D * 2 * 2
    return {"ms": max_over_ranks(statistics.mean(ms), world), "ms_min": min(ms), **spread(ms),
            "bracket_ms": bracket, "flops": 4.0 * case.D * case.Hq * pairs,
            "bytes": kv_bytes + 2 * 2 * float(cq[-1]) * case.Hq * case.D, "total_q": int(cq[-1])}


def case_like(case):
    """The masking fields of a workload (for visible_pairs with explicit lengths)."""
    return mi.PrefillCase("x", 1, 1, 1, 0, 0, case.D, case.dtype, case.causal, case.win_l, case.win_r)


def bench_decode(case, steps, warmup, flush, stream, world):
    import torch
    import tiled_exact_attention_mfa_b200 as mfa
    dev = torch.device("cuda")
    q, kp, vp, table, lens = case.tensors()
    qt, kt, vt = (upload(x, case.dtype, dev) for x in (q, kp, vp))
    tt = torch.from_numpy(table).to(dev)
    lt = torch.from_numpy(lens).to(dev)
    out = torch.empty_like(qt)
    lse = torch.empty(case.B, case.Hq, case.Nq, dtype=torch.float32, device=dev)
    ws_bytes = mfa.mfa_decode_workspace_size(case.B, case.Nq, case.Hq, case.Hkv, case.D, table.shape[1])
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    scale = case.scale_f32()

    def step():
        mfa.mfa_decode_splitkv(qt, kt, vt, tt, lt, out, lse, scale=scale, causal=case.causal,
                               softcap=case.softcap, workspace=ws, win_l=case.win_l,
                               stream=stream)

    with torch.cuda.stream(stream):
        ms, bracket = time_steps(step, steps, warmup, flush, stream)
    return {"ms": max_over_ranks(statistics.mean(ms), world), "ms_min": min(ms), **spread(ms),
            "bracket_ms": bracket, "bytes": decode_bytes(case, lens),
            "flops": decode_flops(case, lens), "seq_len_sum": int(np.sum(lens)),
            "visible_tokens": int(decode_tokens(case, lens)[0])}


def run_gpu(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
        dist.barrier()
    import tiled_exact_attention_mfa_b200 as mfa
    pk = peaks()
    stream = torch.cuda.Stream()
    flush_buf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")

    def flush():
        flush_buf.fill_(1)

    W = mi.workloads()
    clocks = ClockSampler(local)
    clocks.start()
    main_case = W[args.workload]
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    main = bench_prefill(main_case, args.steps, args.warmup, flush, stream, not args.no_e2e, world,
                         rank, args.scaling)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    others = []
    # the secondary workloads run at N = 1 only: a scaling run measures the headline, and every
    # rank would otherwise build all their inputs (page pools of GBs) in host memory at once
    if not args.only_main and world == 1:
        for name, case in W.items():
            if name == args.workload:
                continue
            sk, wu = max(3, min(args.steps, 10)), max(3, args.warmup)
            if isinstance(case, (mi.VarlenCase, mi.SparseCase, mi.PagedPrefillCase)):
                if isinstance(case, mi.VarlenCase):
                    r = bench_varlen(case, sk, wu, flush, stream, world)
                elif isinstance(case, mi.PagedPrefillCase):
                    r = bench_paged(case, sk, wu, flush, stream, world)
                else:
                    r = bench_sparse(case, sk, wu, flush, stream, world)
                tf = r["flops"] * world / (r["ms"] * 1e-3) / 1e12
                gbs = r["bytes"] * world / (r["ms"] * 1e-3) / 1e9
                t_floor = max(r["flops"] / (pk["tflops"] * 1e12), r["bytes"] / (pk["gbs"] * 1e9))
                others.append({**spread_of(r), "workload": name, "ms": round(r["ms"], 4), "unit": "TFLOP/s",
                               "value": round(tf, 1), "GB/s": round(gbs, 1),
                               **({"total_q": r["total_q"]} if "total_q" in r else
                                  {"block_density": round(r["density"], 4)}),
                               "frac_of_measured_tensor_peak": round(tf / pk["tflops"], 4),
                               "frac_of_nominal_tensor_peak": round(tf / NOMINAL_TFLOPS, 4),
                               "frac_of_roofline": round(t_floor / (r["ms"] * 1e-3), 4)})
            elif isinstance(case, mi.DecodeCase):
                r = bench_decode(case, sk, wu, flush, stream, world)
                tb = r["bytes"] * world / (r["ms"] * 1e-3) / 1e9
                others.append({**spread_of(r), "workload": name, "ms": round(r["ms"], 4), "unit": "GB/s",
                               "value": round(tb, 1), "bound": "hbm",
                               "frac_of_measured_peak": round(tb / pk["gbs"], 4),
                               "frac_of_nominal_peak": round(tb / NOMINAL_GBS, 4),
                               "seq_len_sum": r["seq_len_sum"],
                               **({"window_left": case.win_l,
                                   "visible_tokens": r["visible_tokens"]}
                                  if case.win_l >= 0 else {}),
                               "traffic_phase1": ncu_traffic(name, "mfa_decode_phase1_kernel"),
                               "tflops": round(r["flops"] * world / (r["ms"] * 1e-3) / 1e12, 2)})
            else:
                r = bench_prefill(case, sk, wu, flush, stream, False, world)
                if name == "causal_b1_h2_n128_d64_fp16":
                    r["host_us"] = host_call_us(case, stream)
                tf = r["flops"] * world / (r["ms"] * 1e-3) / 1e12
                gbs = r["bytes"] * world / (r["ms"] * 1e-3) / 1e9
                t_floor = max(r["flops"] / (pk["tflops"] * 1e12), r["bytes"] / (pk["gbs"] * 1e9))
                others.append({**spread_of(r), "workload": name, "ms": round(r["ms"], 4), "unit": "TFLOP/s",
                               "value": round(tf, 1), "GB/s": round(gbs, 1),
                               "frac_of_measured_tensor_peak": round(tf / pk["tflops"], 4),
                               "frac_of_nominal_tensor_peak": round(tf / NOMINAL_TFLOPS, 4),
                               "frac_of_roofline": round(t_floor / (r["ms"] * 1e-3), 4),
                               "traffic": ncu_traffic(name, "mfa_fwd_kernel"),
                               **({"host_us_per_call": r["host_us"]} if "host_us" in r else {}),
                               **pages_context(name)})
            getattr(case, "_cache", {}).clear()  # the workload's host inputs are not needed again
    if not args.only_main and world > 1:
        # the decode workload with every sequence's splits spread over the GPUs (strong
        # scaling of one decode step, with its one exchange: the all-gather of the partials)
        name = "decode_b8_hq32_hkv8_d128_bf16_len8k_128k"
        sk, wu = max(3, min(args.steps, 10)), max(3, args.warmup)
        r = bench_decode_sharded(W[name], sk, wu, flush, stream, world, rank)
        tb = r["bytes"] / (r["ms"] * 1e-3) / 1e9
        others.append({**spread_of(r), "workload": name + ":splits_over_gpus", "ms": round(r["ms"], 4),
                       "unit": "GB/s", "value": round(tb, 1), "bound": "hbm",
                       "frac_of_measured_peak_x_gpus": round(tb / (pk["gbs"] * world), 4),
                       "exchange_bytes_per_gpu": r["exchange_bytes"], "scaling": "strong",
                       "parallelism": f"splits of every sequence over {world} GPUs, NCCL all-gather "
                                      "of the (o, m, l) partials, combine on every GPU"})
    if not args.only_main:
        for name in BACKWARD_WORKLOADS:
            sk, wu = max(3, min(args.steps, 10)), max(3, args.warmup)
            r = bench_backward(W[name], sk, wu, flush, stream, world)
            tf = r["flops"] * world / (r["ms"] * 1e-3) / 1e12
            others.append({**spread_of(r), "workload": name + ":backward", "ms": round(r["ms"], 4),
                           "unit": "TFLOP/s", "value": round(tf, 1),
                           "frac_of_measured_tensor_peak": round(tf / pk["tflops"], 4),
                           "frac_of_nominal_tensor_peak": round(tf / NOMINAL_TFLOPS, 4),
                           "flops_convention": "2.5 x forward (S, dP, dV, dK, dQ over visible pairs)"})
    clk = clocks.stop()
    tflops = main["job_flops"] / (main["ms"] * 1e-3) / 1e12
    per_gpu_tflops = tflops / world
    line = {
        "metric": METRIC,
        "value": round(tflops, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(main["ms"], 5),
        **spread_of(main),
        "higher_is_better": True,
        "scaling": args.scaling,
        "vs_baseline": None,
        "dtype": mi.DTYPE_NAMES[main_case.dtype],
        "data": "synthetic (seeded N(0,1) Q/K/V, SplitMix64 + Box-Muller)",
        "config": main_config(args.workload, world, args.scaling),
        "context": {**pages_context(args.workload),
                    "note": "the pages' own timing on Apple hardware, for context; not a target"},
        "roofline": {"bound": "tensor", "achieved": round(per_gpu_tflops, 2),
                     "peak": pk["tflops"], "unit": "TFLOP/s",
                     "frac": round(per_gpu_tflops / pk["tflops"], 4),
                     "peak_source": f"{pk['source']} bf16 burst (fp16 dense rate is the same)",
                     "frac_of_nominal": round(per_gpu_tflops / NOMINAL_TFLOPS, 4),
                     "kernel": "mfa_fwd_kernel",
                     "traffic": ncu_traffic(args.workload, "mfa_fwd_kernel")},
        "gpu_launches": args.steps,
        "clocks": clk,
        "workloads": others,
    }
    if "e2e_ms" in main:
        line["e2e"] = {"value": round(main["job_flops"] / (main["e2e_ms"] * 1e-3) / 1e12, 3),
                       "unit": "TFLOP/s", "ms_per_step": round(main["e2e_ms"], 4),
                       "h2d_bytes_per_step": main["h2d"], "d2h_bytes_per_step": main["d2h"],
                       "h2d_alone_ms": round(main["h2d_alone_ms"], 4),
                       "call": "mfa_fwd_host (C ABI, pinned host buffers; copies in / kernels / "
                               "copies out pipelined over runs of about 12 MiB of (batch, kv-head) units)"}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(main_case, budget_s=args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


# --------------------------------------------------------------------------- oracle timing
def oracle_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(case, budget_s: float = 15.0):
    """The fp64 oracle as it stands, on whole (b, h) heads of the workload until ~budget_s."""
    import oracle
    q, k, v = case.tensors()
    w = lambda x: mi.widen(x, case.dtype)
    qd, kd, vd = w(q), w(k), w(v)
    G = case.Hq // case.Hkv
    pairs = visible_pairs(case)
    t0 = time.perf_counter()
    heads = 0
    for b in range(case.B):
        for h in range(case.Hq):
            oracle.attention(qd[b:b + 1, h:h + 1], kd[b:b + 1, h // G:h // G + 1],
                             vd[b:b + 1, h // G:h // G + 1], case.scale_f32(), case.causal,
                             case.win_l, case.win_r, case.softcap)
            heads += 1
            if time.perf_counter() - t0 > budget_s:
                break
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    flops = 4.0 * case.D * pairs * heads
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": oracle_threads(),
            "kind": "oracle", "sample": f"{heads} of {case.B * case.Hq} (b,h) heads of {case.name}, "
                                        f"all {case.Nq} rows each, fp64 numpy, {dt:.1f} s"}


def run_reference(args):
    """The reference arm: the fp64 oracle as it stands, timed over whole steps of the named
    workload (every head, every row) on the host cores. Rank 0 alone runs it."""
    import oracle
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    case = mi.workloads()[args.workload]
    q, k, v = case.tensors()
    w = lambda x: mi.widen(x, case.dtype)
    qd, kd, vd = w(q), w(k), w(v)

    def step():
        oracle.attention(qd, kd, vd, case.scale_f32(), case.causal, case.win_l, case.win_r,
                         case.softcap)

    for _ in range(args.warmup):
        step()
    ms = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        step()
        ms.append((time.perf_counter() - t0) * 1e3)
    mean_ms = statistics.mean(ms)
    value = prefill_flops(case) / (mean_ms * 1e-3) / 1e12
    sample = (f"whole steps: all {case.B * case.Hq} (b,h) heads x {case.Nq} rows of {case.name} "
              f"per step, fp64 numpy, {mean_ms / 1e3:.2f} s per step")
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(mean_ms, 3), **spread(ms), "higher_is_better": True,
            "scaling": args.scaling, "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": main_config(args.workload, world, args.scaling),
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": oracle_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_profile(args):
    """One workload alone (prefill or decode), for profiler captures: no e2e, no CPU baseline,
    no other workloads. Prints the mean per-step milliseconds."""
    import torch
    torch.cuda.set_device(0)
    stream = torch.cuda.Stream()
    flush_buf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    name, _, part = args.profile.partition(":")
    case = mi.workloads()[name]
    if part == "backward":
        r = bench_backward(case, args.steps, args.warmup, lambda: flush_buf.fill_(1), stream, 1)
    elif isinstance(case, mi.DecodeCase):
        r = bench_decode(case, args.steps, args.warmup, lambda: flush_buf.fill_(1), stream, 1)
    elif isinstance(case, mi.VarlenCase):
        r = bench_varlen(case, args.steps, args.warmup, lambda: flush_buf.fill_(1), stream, 1)
    elif isinstance(case, mi.SparseCase):
        r = bench_sparse(case, args.steps, args.warmup, lambda: flush_buf.fill_(1), stream, 1)
    elif isinstance(case, mi.PagedPrefillCase):
        r = bench_paged(case, args.steps, args.warmup, lambda: flush_buf.fill_(1), stream, 1)
    else:
        r = bench_prefill(case, args.steps, args.warmup, lambda: flush_buf.fill_(1), stream, False, 1)
    print(json.dumps({"profile": args.profile, "ms": round(r["ms"], 5)}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["mfa", "reference"], default="mfa")
    ap.add_argument("--workload", default=MAIN,
                    choices=sorted(n for n, c in mi.workloads().items() if isinstance(c, mi.PrefillCase)))
    ap.add_argument("--only-main", action="store_true", help="skip the other workloads")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--scaling", choices=["weak", "strong"], default="weak",
                    help="N > 1: weak = a batch N times the workload's, sharded by (sequence, "
                         "kv-head) units; strong = the workload's own units split over the GPUs")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--profile", default=None,
                    choices=sorted(mi.workloads()) + [n + ":backward" for n in BACKWARD_WORKLOADS],
                    help="time one workload alone (for profiler captures) and exit")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.profile:
        run_profile(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
