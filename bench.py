"""Benchmark: exact attention on B200 through the C-ABI library.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload long|gpt2|frame|decode] [--no-extra] [--no-cpu-baseline]
                    [--backward-only | --bound-only] [--verbose]

Headline (one JSON line on rank 0): prefill attention TFLOP/s on the largest
single-GPU workload, long-context GQA causal prefill (B=1, Hq=32, Hkv=8,
N=16384, d=128, bf16; 2.2 TFLOP per step).  One step is one attn_fwd call
(tile plan lookup, TMA/tcgen05 kernel: S = QK^T, mask on partial tiles,
online softmax, PV, O and LSE out).  Unless --no-extra, the same line carries
one entry per other workload -- GPT-2 causal prefill (B=8, H=12, N=1024,
d=64), frame block-sparse prefill (24 heads, 24 frames x 1040 tokens, d=128),
GQA decode (B=64, Hq=32, Hkv=8, d=128, lengths U[1024, 8192]) in KV GB/s --
each with its roofline fraction, the fp64 oracle's rate on the host cores
(cpu_baseline) and the end-to-end rate with host buffers (e2e), plus the
backward on the GPT-2 shape and the bound-based forward on the long-context
workload.  The main legs come last in the line.  --verbose prints every
leg's full record to stderr.  --impl reference times the fp64 oracle on the
host cores.

FLOPs are algorithmic: 4*d per allowed (query, key) pair.  Bytes for decode
are algorithmic: the K and V rows below each sequence's length, read once.

Timing: W untimed warm-up steps, then exactly K steps between a barrier and a
device synchronise on both sides; each step is bracketed by CUDA events on the
launching stream (the mean and the median per step are reported), and L2 is
flushed (a 256 MiB write) before every prefill step; the decode cache
(1.26 GB) is larger than L2.  Multi-GPU: one process per GPU, each rank runs
its own copy of the workload (weak scaling), the reported time is the max over
ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synthetic  # noqa: E402

MIB = 1 << 20

# ------------------------------------------------------------------ workloads
WORKLOADS = {
    "tiny": dict(kind="prefill", B=1, Hq=2, Hkv=2, N=256, d=64, mask="none", dtype="f32", seed=1001,
                 desc="tiny non-causal fp32: B=1, H=2, N=256, d=64"),
    "gpt2": dict(kind="prefill", B=8, Hq=12, Hkv=12, N=1024, d=64, mask="causal", dtype="bf16", seed=1002,
                 desc="GPT-2 causal prefill: B=8, H=12, N=1024, d=64, bf16"),
    "long": dict(kind="prefill", B=1, Hq=32, Hkv=8, N=16384, d=128, mask="causal", dtype="bf16", seed=1003,
                 desc="long-context GQA causal prefill: B=1, Hq=32, Hkv=8, N=16384, d=128, bf16"),
    "frame": dict(kind="prefill", B=1, Hq=24, Hkv=24, N=24960, d=128, mask="frame", frames=24, frame_len=1040,
                  dtype="bf16", seed=1004,
                  desc="frame block-sparse: B=1, H=24, 24 frames x 1040 tokens, d=128, bf16"),
    "decode": dict(kind="decode", B=64, Hq=32, Hkv=8, Lmax=8192, d=128, dtype="bf16", seed=1005, len_seed=2005,
                   desc="GQA decode: B=64, Hq=32, Hkv=8, d=128, lengths U[1024,8192]"),
}


def allowed_pairs(w) -> int:
    """Allowed (query, key) pairs per head of a prefill workload."""
    N = w["N"]
    if w["mask"] == "none":
        return N * N
    if w["mask"] == "causal":
        return N * (N + 1) // 2
    F, L = w["frames"], w["frame_len"]
    live = 1 + (2 if F > 1 else 0) + 3 * max(0, F - 2)  # key frames {0, f-1, f}
    return live * L * L


def prefill_flops(w) -> int:
    return 4 * w["d"] * allowed_pairs(w) * w["B"] * w["Hq"]


def plan_stats(w) -> dict:
    """The tile plan of a prefill workload (host only, per head): Q tiles, KV
    tile visits and how many of those carry an element predicate, before the
    pair builder's two-segment re-cut; beside it, the classes of a plain
    128 x 128 grid over the same mask.  The share of partial tiles among live
    ones is the figure step 3 of the TPU attention guide measures and removes
    by choosing the tile boundaries."""
    import exact_io_aware_sm_b200 as eio
    mk, bm = mask_of(w)
    N = w["N"]
    qt, kt = eio.plan(mk, bm, N, N)
    visits = int(qt[:, 3].sum())
    partial = sum(int(kt[r[2]:r[2] + r[3], 2].sum()) for r in qt)
    cls = eio.classify(mk, bm, N, N, 128, 128)
    full, part = int((cls == 1).sum()), int((cls == 2).sum())
    return {"q_tiles": len(qt), "kv_tile_visits": visits, "partial_visits": partial,
            "partial_share": partial / max(visits, 1),
            "grid128_live": full + part, "grid128_partial": part,
            "grid128_partial_share": part / max(full + part, 1)}


def decode_kv_bytes(lens, Hkv, d, elem=2) -> int:
    return int(np.sum(lens)) * Hkv * d * elem * 2


def attention_matrix_elements(N, H, B) -> int:
    """Elements of S (or P) for B*H heads of N x N (FlashAttention page, section 1)."""
    return N * N * H * B


def kv_cache_bytes_per_token(layers, heads, head_dim, elem=2) -> int:
    """K and V for one token (inference page, "Actual KV Cache Size")."""
    return 2 * elem * layers * heads * head_dim


def io_elements(N, d, M):
    """HBM accesses in elements: standard ~N^2, tiled ~N^2 d^2 / M (FlashAttention page, section 5)."""
    return N * N, N * N * d * d / M


# ------------------------------------------------------------------ peaks / traffic
def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return {"hbm_gbs": j["hbm_gbs"], "bf16_tflops": j["bf16_tflops"],
                "bf16_tflops_sustained": j.get("bf16_tflops_sustained", j["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def _code_only(src: str) -> str:
    """C/C++ source with comments removed and whitespace runs collapsed, so
    that an edit to comments or layout alone does not count as a change."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c in "\"'":  # string or character literal: kept whole
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        else:
            out.append(c)
            i += 1
    return re.sub(r"\s+", " ", "".join(out)).strip()


def kernel_source_sha(fn):
    """Hash of a kernel's code together with the local headers it includes
    (recursively), so that a change to a shared device helper also counts;
    comments and whitespace are excluded (see _code_only)."""
    csrc = os.path.join(ROOT, "exact_io_aware_sm_b200", "csrc")
    h, seen, todo = hashlib.sha256(), set(), [fn]
    while todo:
        name = todo.pop(0)
        path = os.path.join(csrc, name)
        if name in seen or not os.path.exists(path):
            continue
        seen.add(name)
        with open(path, "rb") as f:
            data = f.read().decode()
        h.update(name.encode() + b"\0" + _code_only(data).encode())
        todo += re.findall(r'^#include "([^"/]+)"', data, flags=re.M)
    return h.hexdigest()[:16]


def recorded_traffic(key):
    """DRAM bytes per launch from a committed ncu summary, or None when the
    kernel source changed since the counters were taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        j = json.load(f)
    e = j.get(key)
    if not e or e.get("source_sha") != kernel_source_sha(e["source"]):
        return None
    return e["dram_bytes_per_launch"]


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML (read only)."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting"}

    def __init__(self, index):
        self.samples, self.reasons, self.ok = [], set(), False
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                util = nv.nvmlDeviceGetUtilizationRates(self.h).gpu
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((mhz, util))
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.005)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0, "source": "nvml" if self.ok else "unavailable"}
        loaded = [m for m, u in self.samples if u > 0] or [m for m, _ in self.samples]
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples), "source": "nvml"}


# ------------------------------------------------------------------ distributed
def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, ms_max: float, world: int) -> float:
    """Units per second for the whole job: every rank processes
    `units_per_rank` in a step and the step takes the slowest rank's time."""
    return world * units_per_rank / (ms_max * 1e-3)


def rank_seed(seed: int, rank: int) -> int:
    """Each rank works on its own batch (weak scaling): distinct seeds."""
    return seed + 100000 * rank


# ------------------------------------------------------------------ inputs
def host_prefill_inputs(w, seed):
    dt = w["dtype"]
    B, N, Hq, Hkv, d = w["B"], w["N"], w["Hq"], w["Hkv"], w["d"]
    q = synthetic.tensor(seed, synthetic.TID_Q, (B, N, Hq, d), dt)
    k = synthetic.tensor(seed, synthetic.TID_K, (B, N, Hkv, d), dt)
    v = synthetic.tensor(seed, synthetic.TID_V, (B, N, Hkv, d), dt)
    return q, k, v


def to_torch(x, device=None, pin=False):
    import torch
    t = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16) if x.dtype == np.uint16 else torch.from_numpy(x)
    if pin:
        return t.pin_memory()
    return t.to(device) if device is not None else t


def mask_of(w):
    import exact_io_aware_sm_b200 as eio
    if w["mask"] == "none":
        return eio.MASK_NONE, None
    if w["mask"] == "causal":
        return eio.MASK_CAUSAL, None
    return eio.MASK_BLOCK, eio.frame_block_map(w["frames"], w["frame_len"])


# ------------------------------------------------------------------ timing core
def time_steps(step, K, W, world, flush=None):
    """W warm-ups, then K steps each bracketed by events on the current stream.
    Returns (mean ms, median ms, wall seconds of the timed region)."""
    import torch
    for _ in range(W):
        if flush:
            flush()
        step()
    torch.cuda.synchronize()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    barrier(world)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for i in range(K):
        if flush:
            flush()
        starts[i].record()
        step()
        ends[i].record()
    torch.cuda.synchronize()
    barrier(world)
    wall = time.perf_counter() - t0
    ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    return sum(ms) / K, statistics.median(ms), wall


def time_e2e_pipelined(h2d, run, d2h, steps, warmup, world, flush=None):
    """End-to-end steps through the public API with host buffers.  Every step
    copies its inputs host -> device (h2d: (pinned host tensor, [two device
    buffers]) pairs), runs the call (run(k) on buffer set k) and reads its
    results back device -> host (d2h: ([two device buffers], [two pinned host
    tensors]) pairs).  The three parts go on three streams with two buffer
    sets, so step i+1's input copy overlaps step i's call and step i-1's
    read-back, as a serving loop would run them.  Returns ms per step (device
    time from the first copy to the last read-back)."""
    import torch
    s_in, s_run, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_run = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def one(i):
        k = i % 2
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev_run[k])  # buffer set k no longer read
            for h, d in h2d:
                d[k].copy_(h, non_blocking=True)
            ev_in[k].record(s_in)
        with torch.cuda.stream(s_run):
            s_run.wait_event(ev_in[k])
            if i >= 2:
                s_run.wait_event(ev_out[k])  # results of set k read back
            if flush:
                flush()
            run(k)
            ev_run[k].record(s_run)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_run[k])
            for d, h in d2h:
                h[k].copy_(d[k], non_blocking=True)
            ev_out[k].record(s_out)

    for i in range(warmup):
        one(i)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(s_in)
    for i in range(warmup, warmup + steps):
        one(i)
    s_out.wait_stream(s_in)
    s_out.wait_stream(s_run)
    t1.record(s_out)
    torch.cuda.synchronize()
    barrier(world)
    return t0.elapsed_time(t1) / steps


def capture_graph(step):
    """Capture one call of `step` (library call, warm: plan and workspace
    cached) into a CUDA graph; replaying it removes the per-call host work."""
    import torch
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    torch.cuda.synchronize()
    return g


def make_flush():
    import torch
    buf = torch.empty(256 * MIB, dtype=torch.uint8, device="cuda")

    def flush():
        buf.fill_(1)
    return flush


def bench_prefill(w, args, world, rank, peaks, with_e2e=True):
    import torch

    import exact_io_aware_sm_b200 as eio
    seed = rank_seed(w["seed"], rank)
    q, k, v = host_prefill_inputs(w, seed)
    tq, tk, tv = (to_torch(x, "cuda") for x in (q, k, v))
    mk, bm = mask_of(w)
    scale = 1.0 / math.sqrt(w["d"])
    o = torch.empty_like(tq)
    lse = torch.empty((w["B"], w["Hq"], w["N"]), dtype=torch.float32, device="cuda")

    def step():
        eio.attn_fwd(tq, tk, tv, o=o, lse=lse, scale=scale, mask_kind=mk, block_map=bm)

    flush = make_flush()
    # Eager calls first (warms the plan cache), then the same call replayed
    # from a CUDA graph: the graph time is the kernel's, the eager time adds
    # the host-side call overhead when the GPU would otherwise idle.
    eager_ms, _, _ = time_steps(step, args.steps, args.warmup, world, flush)
    graph = capture_graph(step)
    ms, med, wall = time_steps(graph.replay, args.steps, args.warmup, world, flush)
    eio.sync_status()
    ms, med = max_over_ranks(ms, world), max_over_ranks(med, world)
    eager_ms = max_over_ranks(eager_ms, world)
    flops = prefill_flops(w)
    tflops = whole_job_rate(flops, ms, world) / 1e12
    peak = peaks["bf16_tflops"]
    out = {
        "ms_per_step": ms, "ms_median": med, "tflops": tflops, "flops_per_step": flops,
        "roofline": {"bound": "tensor", "achieved": flops / (ms * 1e-3) / 1e12, "peak": peak,
                     "unit": "TFLOP/s", "frac": flops / (ms * 1e-3) / 1e12 / peak,
                     "peak_source": f"{peaks['source']} bf16 burst",
                     "kernel": "prefill_bf16_kernel",
                     "traffic": recorded_traffic(f"prefill_{args_key(w)}")},
        "gpu_launches": args.steps,
        "wall_s": wall,
        "eager_ms_per_step": eager_ms,
        "timing": "CUDA graph replay of one attn_fwd call per step; eager_ms_per_step is the plain call",
    }
    # The exponentials: one per allowed (query, key) pair, on the MUFU unit
    # (16 per clock per SM on B200, measured; 148 SMs at the 1965 MHz boost
    # clock).  At d = 64 this bound is lower than the tensor-core one.
    n_exp = allowed_pairs(w) * w["B"] * w["Hq"]
    exp_peak = 16 * 148 * 1.965e9
    out["roofline_exp"] = {"bound": "alu", "unit": "Gexp/s", "achieved": n_exp / (ms * 1e-3) / 1e9,
                           "peak": exp_peak / 1e9, "frac": n_exp / (ms * 1e-3) / exp_peak,
                           "peak_source": "MUFU ex2 16/clk/SM x 148 SMs x 1965 MHz",
                           "attainable_tflops": flops / (n_exp / exp_peak) / 1e12}
    # attainable at this arithmetic intensity: min(peak, AI * HBM)
    alg_bytes = q.nbytes + k.nbytes + v.nbytes + q.nbytes + lse.numel() * 4  # Q, K, V in; O, LSE out
    ai = flops / alg_bytes
    out["roofline"]["attainable_tflops"] = min(peak, ai * peaks["hbm_gbs"] / 1e3)
    out["roofline"]["alg_bytes"] = int(alg_bytes)
    if with_e2e:
        hq_, hk_, hv_ = (to_torch(x, pin=True) for x in (q, k, v))
        dq, dk, dv = ([torch.empty_like(t) for _ in range(2)] for t in (tq, tk, tv))
        do, dl = [torch.empty_like(o) for _ in range(2)], [torch.empty_like(lse) for _ in range(2)]
        ho = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for _ in range(2)]
        hl = [torch.empty(lse.shape, dtype=torch.float32).pin_memory() for _ in range(2)]

        def run(i):
            eio.attn_fwd(dq[i], dk[i], dv[i], o=do[i], lse=dl[i], scale=scale, mask_kind=mk, block_map=bm)

        ems = time_e2e_pipelined([(hq_, dq), (hk_, dk), (hv_, dv)], run, [(do, ho), (dl, hl)],
                                 args.steps, 3, world, flush)
        eio.sync_status()
        ems = max_over_ranks(ems, world)
        out["e2e"] = {"value": whole_job_rate(flops, ems, world) / 1e12, "unit": "TFLOP/s",
                      "ms_per_step": ems,
                      "h2d_bytes_per_step": int(q.nbytes + k.nbytes + v.nbytes),
                      "d2h_bytes_per_step": int(o.numel() * o.element_size() + lse.numel() * 4),
                      "timing": "H2D, call and D2H on three streams with two buffer sets; L2 flushed "
                                "before each call"}
        del dq, dk, dv, do, dl
    del tq, tk, tv, o, lse
    torch.cuda.empty_cache()
    return out


def bench_backward(w, args, world, rank, peaks):
    """attn_bwd on a prefill workload (bf16; O and LSE from attn_fwd, computed
    once).  FLOPs: the five products of the backward over the allowed pairs,
    2.5x the forward's (the usual convention; the recomputation of S and P in
    both kernels is not counted)."""
    import torch

    import exact_io_aware_sm_b200 as eio
    seed = rank_seed(w["seed"], rank)
    q, k, v = host_prefill_inputs(w, seed)
    dout = synthetic.tensor(seed, 9, q.shape, w["dtype"])
    tq, tk, tv, tdo = (to_torch(x, "cuda") for x in (q, k, v, dout))
    mk, bm = mask_of(w)
    bm_ptr = None if bm is None else bm.ctypes.data
    scale = 1.0 / math.sqrt(w["d"])
    o, lse = eio.attn_fwd(tq, tk, tv, scale=scale, mask_kind=mk, block_map=bm)
    dq, dk, dv = torch.empty_like(tq), torch.empty_like(tk), torch.empty_like(tv)

    def step():
        eio.lib().attn_bwd(tq.data_ptr(), tk.data_ptr(), tv.data_ptr(), o.data_ptr(), lse.data_ptr(),
                           tdo.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), w["B"], w["Hq"], w["Hkv"],
                           w["N"], w["N"], w["d"], scale, mk, bm_ptr, torch.cuda.current_stream().cuda_stream)

    flush = make_flush()
    time_steps(step, 3, args.warmup, world, flush)
    graph = capture_graph(step)
    ms, med, _ = time_steps(graph.replay, args.steps, args.warmup, world, flush)
    eio.sync_status()
    ms, med = max_over_ranks(ms, world), max_over_ranks(med, world)
    flops = 2.5 * prefill_flops(w)
    tflops = whole_job_rate(flops, ms, world) / 1e12
    peak = peaks["bf16_tflops"]
    # The kernels run seven products (S and dP in both), 3.5x the forward.
    out = {"metric": "attention backward TFLOP/s", "value": tflops, "unit": "TFLOP/s", "ms_per_step": ms,
           "ms_median": med,
           "config": {"workload": w["desc"] + ", backward (dQ, dK, dV)"},
           "roofline": {"bound": "tensor", "achieved": flops / (ms * 1e-3) / 1e12, "peak": peak, "unit": "TFLOP/s",
                        "frac": flops / (ms * 1e-3) / 1e12 / peak, "peak_source": f"{peaks['source']} bf16 burst",
                        "executed_frac": 1.4 * flops / (ms * 1e-3) / 1e12 / peak,
                        "kernel": "bwd_dq + bwd_dkdv (one call)",
                        "traffic": recorded_traffic(f"backward_{args_key(w)}")},
           "gpu_launches": 2 * args.steps}
    del tq, tk, tv, tdo, o, lse, dq, dk, dv
    torch.cuda.empty_cache()
    return out


def bench_bound(w, args, world, rank, peaks):
    """attn_fwd_bound (bound-based softmax) on a prefill workload, next to the
    online forward: the key statistics (attn_key_stats) and the forward are
    timed separately, each as CUDA-graph replays with the L2 flushed between
    steps; the rate is reported with and without the statistics."""
    import torch

    import exact_io_aware_sm_b200 as eio
    seed = rank_seed(w["seed"], rank)
    q, k, v = host_prefill_inputs(w, seed)
    tq, tk, tv = (to_torch(x, "cuda") for x in (q, k, v))
    mk, bm = mask_of(w)
    scale = 1.0 / math.sqrt(w["d"])
    o = torch.empty_like(tq)
    lse = torch.empty((w["B"], w["Hq"], w["N"]), dtype=torch.float32, device="cuda")
    kbar = torch.empty((w["B"], w["Hkv"], w["d"]), dtype=torch.float32, device="cuda")
    radius = torch.empty((w["B"], w["Hkv"]), dtype=torch.float32, device="cuda")
    nfb = torch.zeros(1, dtype=torch.int32, device="cuda")

    def stats():
        eio.key_stats(tk, kbar, radius)

    def fwd():
        eio.attn_fwd_bound(tq, tk, tv, kbar, radius, o=o, lse=lse, scale=scale, mask_kind=mk, block_map=bm,
                           n_fallback=nfb)

    flush = make_flush()
    steps = args.steps
    stats()
    time_steps(fwd, 3, args.warmup, world, flush)
    g_stats, g_fwd = capture_graph(stats), capture_graph(fwd)
    ms_stats, _, _ = time_steps(g_stats.replay, steps, args.warmup, world, flush)
    ms_fwd, med_fwd, _ = time_steps(g_fwd.replay, steps, args.warmup, world, flush)
    med_fwd = max_over_ranks(med_fwd, world)
    eio.sync_status()
    ms_stats, ms_fwd = max_over_ranks(ms_stats, world), max_over_ranks(ms_fwd, world)
    nfb.zero_()
    fwd()  # one more call, to count its fallback rows
    eio.sync_status()
    flops = prefill_flops(w)
    peak = peaks["bf16_tflops"]
    out = {"metric": "prefill attn TFLOP/s (bound-based softmax)", "value": whole_job_rate(flops, ms_fwd, world) / 1e12,
           "unit": "TFLOP/s", "ms_per_step": ms_fwd, "ms_median": med_fwd, "key_stats_ms": ms_stats,
           "value_with_key_stats": whole_job_rate(flops, ms_fwd + ms_stats, world) / 1e12,
           "fallback_rows": int(nfb.item()),
           "config": {"workload": w["desc"] + ", attn_fwd_bound (key statistics precomputed)"},
           "roofline": {"bound": "tensor", "achieved": flops / (ms_fwd * 1e-3) / 1e12, "peak": peak, "unit": "TFLOP/s",
                        "frac": flops / (ms_fwd * 1e-3) / 1e12 / peak, "peak_source": f"{peaks['source']} bf16 burst",
                        "kernel": "prefill_bf16_kernel (bound mode)",
                        "traffic": recorded_traffic(f"prefill_bound_{args_key(w)}")},
           "gpu_launches": 3 * steps}
    del tq, tk, tv, o, lse
    torch.cuda.empty_cache()
    return out


def args_key(w):
    return f"{w['mask']}_d{w['d']}_n{w['N']}"


def bench_decode(w, args, world, rank, peaks, with_e2e=True):
    import torch

    import exact_io_aware_sm_b200 as eio
    seed = rank_seed(w["seed"], rank)
    B, Hq, Hkv, Lmax, d = w["B"], w["Hq"], w["Hkv"], w["Lmax"], w["d"]
    lens = synthetic.seqlens(w["len_seed"], B)
    q = synthetic.tensor(seed, synthetic.TID_Q, (B, Hq, d))
    kc = synthetic.kv_cache(seed, synthetic.TID_K, B, Lmax, Hkv, d, lens)
    vc = synthetic.kv_cache(seed, synthetic.TID_V, B, Lmax, Hkv, d, lens)
    tq, tk, tv = to_torch(q, "cuda"), to_torch(kc, "cuda"), to_torch(vc, "cuda")
    del kc, vc
    tl = torch.from_numpy(lens).cuda()
    scale = 1.0 / math.sqrt(d)
    o = torch.empty_like(tq)
    lse = torch.empty((B, Hq), dtype=torch.float32, device="cuda")

    def step():
        eio.attn_decode(tq, tk, tv, tl, o=o, lse=lse, scale=scale)

    steps = max(args.steps, 20)
    eager_ms, _, _ = time_steps(step, steps, args.warmup, world)
    graph = capture_graph(step)
    ms, med, wall = time_steps(graph.replay, steps, args.warmup, world)
    eio.sync_status()
    ms, med = max_over_ranks(ms, world), max_over_ranks(med, world)
    eager_ms = max_over_ranks(eager_ms, world)
    kvb = decode_kv_bytes(lens, Hkv, d)
    alg = kvb + q.nbytes * 2 + B * Hq * 4
    gbs = whole_job_rate(alg, ms, world) / 1e9
    peak = peaks["hbm_gbs"]
    out = {
        "metric": "decode KV GB/s", "value": gbs, "unit": "GB/s", "ms_per_step": ms, "ms_median": med,
        "config": {"workload": w["desc"], "sum_len": int(lens.sum()), "kv_bytes": kvb,
                   "l2": "cache (1.26 GB) larger than L2; no flush"},
        "roofline": {"bound": "hbm", "achieved": alg / (ms * 1e-3) / 1e9, "peak": peak, "unit": "GB/s",
                     "frac": alg / (ms * 1e-3) / 1e9 / peak, "peak_source": f"{peaks['source']} copy",
                     "kernel": "decode_split_kernel + decode_combine_kernel (one call)",
                     "traffic": recorded_traffic("decode")},
        "gpu_launches": 2 * steps, "steps": steps, "wall_s": wall,
        "eager_ms_per_step": eager_ms,
        "timing": "CUDA graph replay of one attn_decode call (split + combine) per step",
    }
    # Two new tokens per sequence (multi-token decode): the same cache bytes
    # serve both, so tokens per byte double if the time stays.
    q2 = to_torch(synthetic.tensor(seed + 7, synthetic.TID_Q, (B, 2, Hq, d)), "cuda")
    o2 = torch.empty_like(q2)
    l2 = torch.empty((B, Hq, 2), dtype=torch.float32, device="cuda")

    def step2():
        eio.attn_decode_multi(q2, tk, tv, tl, o=o2, lse=l2, scale=scale)

    if w["Hq"] // w["Hkv"] * 2 <= 8:
        time_steps(step2, 3, args.warmup, world)
        g2 = capture_graph(step2)
        ms2, _, _ = time_steps(g2.replay, steps, args.warmup, world)
        eio.sync_status()
        ms2 = max_over_ranks(ms2, world)
        out["multi_token_2"] = {"metric": "decode KV GB/s, 2 new tokens per sequence",
                                "value": whole_job_rate(kvb + q2.numel() * 4 + B * Hq * 8, ms2, world) / 1e9,
                                "unit": "GB/s", "ms_per_step": ms2,
                                "tokens_per_s": whole_job_rate(B * 2, ms2, world)}
    del q2, o2, l2
    if with_e2e:
        # A decode step's input is the new query; the cache stays resident.
        hq_ = to_torch(q, pin=True)
        dq = [torch.empty_like(tq) for _ in range(2)]
        do, dl = [torch.empty_like(o) for _ in range(2)], [torch.empty_like(lse) for _ in range(2)]
        ho = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for _ in range(2)]
        hl = [torch.empty(lse.shape, dtype=torch.float32).pin_memory() for _ in range(2)]

        def run(i):
            eio.attn_decode(dq[i], tk, tv, tl, o=do[i], lse=dl[i], scale=scale)

        ems = time_e2e_pipelined([(hq_, dq)], run, [(do, ho), (dl, hl)], steps, 3, world)
        eio.sync_status()
        ems = max_over_ranks(ems, world)
        out["e2e"] = {"value": whole_job_rate(alg, ems, world) / 1e9, "unit": "GB/s", "ms_per_step": ems,
                      "h2d_bytes_per_step": int(q.nbytes), "d2h_bytes_per_step": int(o.numel() * 2 + lse.numel() * 4),
                      "timing": "H2D, call and D2H on three streams with two buffer sets"}
    del tq, tk, tv
    torch.cuda.empty_cache()
    return out


# ------------------------------------------------------------------ CPU oracle
def row_allowed(w, i) -> int:
    """Allowed keys of query row i (per head) of a prefill workload."""
    N = w["N"]
    if w["mask"] == "none":
        return N
    if w["mask"] == "causal":
        return i + 1
    L = w["frame_len"]
    f = i // L
    return len({0, max(f - 1, 0), f}) * L


def oracle_prefill_call(w, seed, row_budget_flops=2e10):
    """One bounded pass of the fp64 oracle over the workload: the whole
    workload when it holds at most `row_budget_flops` algorithmic FLOPs, else
    a seeded uniform sample of (batch, head, query row) triples of about that
    size.  Returns a callable that runs the pass and returns its FLOPs, and a
    description of the sample."""
    import oracle
    q, k, v = host_prefill_inputs(w, seed)
    kinds = {"none": oracle.MASK_NONE, "causal": oracle.MASK_CAUSAL}
    ok = kinds.get(w["mask"], oracle.MASK_BLOCK)
    bm = oracle.frame_block_map(w["frames"], w["frame_len"]) if ok == oracle.MASK_BLOCK else None
    scale = 1.0 / math.sqrt(w["d"])
    total = prefill_flops(w)
    if total <= row_budget_flops:
        def run():
            oracle.attn_fwd(q, k, v, scale, ok, bm)
            return total
        return run, f"the whole workload ({w['B']} batch elements)"
    rng = np.random.default_rng(seed)
    per_row = 4 * w["d"] * allowed_pairs(w) / w["N"]  # mean FLOPs of one (b, h, i) row
    n = max(1, int(row_budget_flops / per_row))
    rows = np.stack([rng.integers(0, w["B"], n), rng.integers(0, w["Hq"], n), rng.integers(0, w["N"], n)],
                    axis=1).astype(np.int32)
    flops = sum(4 * w["d"] * row_allowed(w, int(i)) for i in rows[:, 2])

    def run():
        oracle.attn_rows(q, k, v, scale, rows, ok, bm)
        return flops
    return run, f"{n} seeded (batch, head, row) samples"


def oracle_prefill_sample(w, seed, min_seconds=8.0, max_passes=200):
    """Repeat bounded oracle passes until `min_seconds` of CPU work; returns
    (seconds, flops, description)."""
    run, desc = oracle_prefill_call(w, seed)
    dt, fl, n = 0.0, 0, 0
    while n < max_passes and (n == 0 or dt < min_seconds):
        t0 = time.perf_counter()
        fl += run()
        dt += time.perf_counter() - t0
        n += 1
    return dt, fl, f"{desc}, {n} passes, {dt:.1f} s"


def oracle_decode_call(w, seed, n_seq=8):
    """A bounded sample of the decode workload for the oracle: the first
    n_seq sequences, with the same seeded queries, caches and lengths as in
    the full batch.  Returns (run, description, algorithmic bytes per run)."""
    import oracle
    B, Hq, Hkv, Lmax, d = w["B"], w["Hq"], w["Hkv"], w["Lmax"], w["d"]
    n = min(n_seq, B)
    lens = synthetic.seqlens(w["len_seed"], B)[:n]
    q = synthetic.tensor(seed, synthetic.TID_Q, (n, Hq, d))
    kc = synthetic.kv_cache(seed, synthetic.TID_K, n, Lmax, Hkv, d, lens)
    vc = synthetic.kv_cache(seed, synthetic.TID_V, n, Lmax, Hkv, d, lens)
    scale = 1.0 / math.sqrt(d)

    def run():
        oracle.decode(q, kc, vc, lens, scale)

    nbytes = decode_kv_bytes(lens, Hkv, d) + q.nbytes * 2 + n * Hq * 4
    return run, f"the first {n} of {B} sequences ({int(lens.sum())} cached keys)", nbytes


def oracle_decode_baseline(w, seed, min_seconds=6.0):
    """The cpu_baseline of a decode line: the oracle's decode of a sample of
    the batch (oracle_decode_call), repeated for at least min_seconds."""
    import oracle
    oracle.build()
    cores = oracle.threads(cpu_cores())
    run, desc, nbytes = oracle_decode_call(w, seed)
    n, dt = 0, 0.0
    while dt < min_seconds:
        t0 = time.perf_counter()
        run()
        dt += time.perf_counter() - t0
        n += 1
    return {"value": nbytes * n / dt / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"{desc}, {n} passes, fp64, {dt:.1f} s", "cpu": cpu_model()}


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count()


def cpu_model() -> str:
    """The host CPU's model name (from /proc/cpuinfo), for the CPU baselines."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def oracle_prefill_baseline(w, seed, min_seconds=8.0):
    """The cpu_baseline of a prefill leg: the oracle on a bounded sample of
    the workload (oracle_prefill_call), repeated for at least min_seconds."""
    import oracle
    oracle.build()
    cores = oracle.threads(cpu_cores())
    dt, fl, desc = oracle_prefill_sample(w, seed, min_seconds=min_seconds)
    return {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": desc,
            "cpu": cpu_model()}


def run_reference(args, world, rank):
    """The oracle as the reference arm, on the same metric and workload: each
    step is one bounded pass over the workload (see oracle_prefill_call)."""
    w = WORKLOADS[args.workload]
    if rank != 0:
        return
    import oracle
    oracle.build()
    cores = oracle.threads(cpu_cores())  # all the host's cores, whatever OMP_NUM_THREADS the launcher set
    if w["kind"] == "decode":
        run_reference_decode(args, w, cores)
        return
    run, desc = oracle_prefill_call(w, w["seed"])
    for _ in range(min(args.warmup, 1)):
        run()
    dt, fl = 0.0, 0
    for _ in range(args.steps):
        t0 = time.perf_counter()
        fl += run()
        dt += time.perf_counter() - t0
    ms = 1e3 * dt / args.steps
    tflops = fl / dt / 1e12
    line = {
        "impl": "reference", "metric": "prefill attn TFLOP/s", "value": tflops, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": w["desc"], "sample": f"{desc} per step"},
        "cpu_baseline": {"value": tflops, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": f"{desc} per step, {args.steps} steps, fp64", "cpu": cpu_model()},
        "e2e": {"value": tflops, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_reference_decode(args, w, cores):
    """The reference arm on the decode workload: the oracle's decode over a
    bounded sample of sequences, in KV GB/s (algorithmic bytes)."""
    run, desc, nbytes = oracle_decode_call(w, w["seed"])
    for _ in range(min(args.warmup, 1)):
        run()
    dt = 0.0
    for _ in range(args.steps):
        t0 = time.perf_counter()
        run()
        dt += time.perf_counter() - t0
    gbs = nbytes * args.steps / dt / 1e9
    line = {
        "impl": "reference", "metric": "decode KV GB/s", "value": gbs, "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w["desc"], "sample": f"{desc} per step"},
        "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": f"{desc} per step, {args.steps} steps, fp64", "cpu": cpu_model()},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def sig(x, n=4):
    """x rounded to n significant digits (keeps the JSON line short)."""
    if not isinstance(x, float) or x == 0 or not math.isfinite(x):
        return x
    return round(x, -int(math.floor(math.log10(abs(x)))) + n - 1)


def short(d, keys):
    return {k: sig(d[k]) for k in keys if k in d and d[k] is not None}


ROOF_KEYS = ("bound", "achieved", "peak", "unit", "frac", "traffic")


def roof(r):
    """The roofline keys of the contract; traffic stays (null) when the ncu
    counters on record no longer match the kernel's code."""
    out = short(r, ROOF_KEYS)
    out["traffic"] = r.get("traffic")
    return out


def leg(workload, r, value, unit, cpu=None):
    """One workload's entry in the JSON line: the rate (the unit names the
    metric: TFLOP/s of prefill or backward attention, KV GB/s of decode), mean
    and median step times, the roofline of its dominant kernel, the oracle
    baseline and the end-to-end rate (both when measured)."""
    out = {"workload": workload, "value": sig(value), "unit": unit,
           "ms": sig(r["ms_per_step"]), "ms_median": sig(r.get("ms_median")), "roofline": roof(r["roofline"])}
    if "executed_frac" in r["roofline"]:
        out["roofline"]["executed_frac"] = sig(r["roofline"]["executed_frac"])
    if cpu is not None:
        out["cpu_baseline"] = short(cpu, ("value", "unit", "cores", "kind"))
    if r.get("e2e"):
        out["e2e"] = short(r["e2e"], ("value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step"))
    return out


SHORT_NAMES = {"gpt2": "GPT-2 causal B=8 H=12 N=1024 d=64",
               "long": "long GQA causal B=1 Hq=32 Hkv=8 N=16384 d=128",
               "frame": "frame block-sparse H=24 24x1040 d=128",
               "decode": "GQA decode B=64 Hq=32 Hkv=8 d=128 len U[1024,8192]"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="long", choices=["gpt2", "long", "frame", "decode"])
    ap.add_argument("--no-extra", action="store_true", help="skip the other workloads' legs")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--backward-only", action="store_true",
                    help="time only attn_bwd on the chosen prefill workload (one JSON line)")
    ap.add_argument("--bound-only", action="store_true",
                    help="time only attn_fwd_bound (and attn_key_stats) on the chosen prefill workload")
    ap.add_argument("--verbose", action="store_true",
                    help="also print every leg's full record (plans, eager times, second rooflines) to stderr")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3

    world, rank, local = dist_setup(args)
    if args.impl == "reference":
        run_reference(args, world, rank)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return

    import torch

    import exact_io_aware_sm_b200 as eio
    from exact_io_aware_sm_b200 import build as ebuild
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    ebuild.build()
    eio.lib()
    peaks = measured_peaks()
    w = WORKLOADS[args.workload]
    one = rank == 0 and world == 1 and not args.no_cpu_baseline  # the oracle baselines: one-GPU runs only

    sampler = ClockSampler(torch.cuda.current_device())
    if args.backward_only or args.bound_only:
        if args.workload == "decode":
            raise SystemExit("--backward-only / --bound-only need a prefill workload")
        with sampler:
            d = (bench_backward if args.backward_only else bench_bound)(w, args, world, rank, peaks)
        if rank == 0:
            d.update({"n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                      "higher_is_better": True, "scaling": "weak",
                      "dtype": "bf16", "data": "synthetic", "clocks": sampler.summary()})
            print(json.dumps(d), flush=True)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return

    detail = {}
    legs = {}
    with sampler:
        if args.workload == "decode":
            head = bench_decode(w, args, world, rank, peaks)
        else:
            head = bench_prefill(w, args, world, rank, peaks)
        detail[args.workload] = head
        if not args.no_extra:
            for name in ("gpt2", "long", "frame", "decode"):
                if name == args.workload:
                    continue
                wx = WORKLOADS[name]
                r = (bench_decode if name == "decode" else bench_prefill)(wx, args, world, rank, peaks)
                detail[name] = r
            g = WORKLOADS["gpt2"]
            detail["backward"] = bench_backward(g, args, world, rank, peaks)
            detail["bound"] = bench_bound(WORKLOADS["long"], args, world, rank, peaks)
    if args.verbose:
        for name, r in detail.items():
            if name in WORKLOADS and WORKLOADS[name]["kind"] == "prefill":
                r["plan"] = plan_stats(WORKLOADS[name])

    cpu = {}  # the oracle on a bounded sample of each workload, on the host cores, after the GPU legs
    if one:
        for name in detail:
            if name in WORKLOADS:
                seed = rank_seed(WORKLOADS[name]["seed"], 0)
                cpu[name] = (oracle_decode_baseline(WORKLOADS[name], seed) if name == "decode"
                             else oracle_prefill_baseline(WORKLOADS[name], seed))

    if rank == 0:
        if args.verbose:
            print("bench detail: " + json.dumps(detail), file=sys.stderr, flush=True)
        for name in ("gpt2", "frame", "long", "decode"):
            if name in detail and name != args.workload:
                r = detail[name]
                if name == "decode":
                    legs[name] = leg(SHORT_NAMES[name], r, r["value"], "GB/s", cpu.get(name))
                    if r.get("multi_token_2"):
                        legs[name]["multi_token_2"] = short(r["multi_token_2"], ("value", "unit", "ms_per_step"))
                else:
                    legs[name] = leg(SHORT_NAMES[name], r, r["tflops"], "TFLOP/s", cpu.get(name))
        if "backward" in detail:
            legs["backward"] = leg(SHORT_NAMES["gpt2"] + ", backward dQ dK dV, FLOPs 2.5x forward",
                                   detail["backward"], detail["backward"]["value"], "TFLOP/s")
        if "bound" in detail:
            b = detail["bound"]
            legs["bound"] = leg(SHORT_NAMES["long"] + ", bound-based softmax", b, b["value"], "TFLOP/s")
            legs["bound"]["key_stats_ms"] = sig(b["key_stats_ms"])
        order = ["backward", "bound", "gpt2", "frame", "long", "decode"]  # the main legs last
        if args.workload == "decode":
            metric, unit, value = "decode KV GB/s", "GB/s", head["value"]
            l2 = "cache (1.26 GB) larger than L2; no flush"
            launches = head["gpu_launches"]
        else:
            metric, unit, value = "prefill attn TFLOP/s", "TFLOP/s", head["tflops"]
            l2 = "flushed before every step (256 MiB write)"
            launches = head["gpu_launches"]
        hc = cpu.get(args.workload)
        line = {
            "metric": metric, "value": sig(value), "unit": unit, "n_gpus": world,
            "steps": head.get("steps", args.steps), "warmup": args.warmup,
            "ms_per_step": sig(head["ms_per_step"]), "ms_median": sig(head.get("ms_median")),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w["desc"], "parallelism": f"replicas x{world}", "l2": l2},
            "roofline": dict(roof(head["roofline"]), peak_source=head["roofline"]["peak_source"]),
            "cpu_baseline": hc, "e2e": short(head["e2e"], ("value", "unit", "h2d_bytes_per_step",
                                                            "d2h_bytes_per_step")),
            "gpu_launches": launches, "clocks": short(sampler.summary(), ("sm_mhz", "sm_max_mhz", "reasons")),
        }
        if hc is not None:
            line["cpu_baseline"] = dict(short(hc, ("value", "unit", "cores", "kind")), sample=hc["sample"],
                                        cpu=hc["cpu"])
        for name in order:
            if name in legs:
                line[name] = legs[name]
        print(json.dumps(line, separators=(",", ":")), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
