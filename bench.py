"""Benchmark of the Gated DeltaNet mixer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--also NAME ...] [--decode-workload NAME]

Prints ONE JSON line (rank 0).  The metric is the mixer layer's prefill
tokens/s and decode tokens/s on B200, with the fraction of roofline.

  value     prefill tokens/s of one mixer layer over all ranks on the headline
            workload (default: 8 packed sequences of 65536 tokens in all, 16
            key / 64 value heads of width 128 -- the largest single-GPU
            configuration).  Each rank runs its own copy (the mixer shares
            nothing across sequences), so scaling is weak.
  prefill   the same measurement (value, roofline, e2e, CPU baseline) for the
            other prefill workloads (--also).
  decode    one recurrent step for a batch of sequences on an fp32 state in
            HBM (and the bf16-state and 4-token variants).
  layer     the whole layer (in_proj GEMM, mixer, out_proj GEMM) with the
            9B model's hidden size 4096 on the 4 x 8192 workload, and each
            projection's tensor-core throughput against the bf16 peak.

Timing: W untimed warm-up steps, then K steps, each bracketed by CUDA events
on the launching stream; before every timed step a 256 MiB buffer is written
to flush L2 (outside the events).  Max over ranks.  `roofline` reports the
chunked core alone (events the library records around its launches, in a
second pass of the same steps).  `e2e` repeats the prefill through the public
call with every step's inputs copied from pinned host memory and its outputs
copied back inside the timed region (two buffer sets, copies of one step
overlapping the compute of the next).  `cpu_baseline` times the fp64 CPU
oracle on a bounded sample.

With --gpus N > 1 and no torchrun environment, the script starts N ranks
itself (torch.distributed.run on 127.0.0.1) and fails if the node has fewer
GPUs.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import socket
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from hybrid_linear_attention_05_b200.workloads import WORKLOADS, make_decode, make_prefill  # noqa: E402

METRIC = "GDN prefill tokens/s & decode tokens/s per layer at 1 B200; % of roofline"
DEFAULT_PREFILL = "prefill_varlen8_T65536_Hk16_Hv64_d128"
DEFAULT_ALSO = ["prefill_4x8192_Hk16_Hv32_d128", "prefill_T4096_Hk16_Hv16_d128"]
DEFAULT_DECODE = "decode_B256_Hk16_Hv32_d128"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# --------------------------------------------------------- multi-rank


def max_over_ranks(x: float, device=None) -> float:
    """Largest value of x over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: int, world: int, max_seconds: float) -> float:
    """Whole-job rate: the units every rank processed over the slowest rank's time."""
    return units_per_rank * world / max_seconds


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def launch_command(argv, n: int, port: int):
    """The command that runs this script as n ranks on this node."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=%d" % n,
            "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__), *argv]


# ------------------------------------------------------ profiled traffic

PROFILES = os.path.join(ROOT, "profiles", "ncu_traffic.tsv")
CSRC = os.path.join(ROOT, "hybrid_linear_attention_05_b200", "csrc")


def source_digest(name: str) -> str:
    with open(os.path.join(CSRC, name), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def profiled_traffic(source: str, workload: str):
    """DRAM bytes per launch recorded by an ncu capture of `source` on
    `workload`, or None when there is none or the source changed since."""
    if not os.path.exists(PROFILES):
        return None
    digest = source_digest(source)
    for line in open(PROFILES):
        parts = line.rstrip("\n").split("\t")
        if len(parts) >= 4 and not line.startswith("#"):
            if parts[0] == source and parts[1] == digest and parts[2] == workload:
                return float(parts[3])
    return None


# ------------------------------------------------------------ work counts


def prefill_counts(inp, chunk):
    """Algorithmic bytes and FLOPs of one prefill (whole call) and of the
    chunked core alone."""
    w = inp.w
    T, N, Hk, Hv, d = inp.T, inp.N, w.Hk, w.Hv, w.d
    e = 2 if w.dtype == "bf16" else 4
    state_in = 0 if inp.initial_state is None else N * Hv * d * d * 4
    state_out = N * Hv * d * d * 4
    # chunked core: normalised q, k, values, gates, z in; out and state out
    core_bytes = (T * (2 * Hk * d * e + Hv * d * e + Hv * 8 + Hv * d * e + Hv * d * e)
                  + state_in + state_out)
    core_flops = T * Hv * (10 * chunk * d + 6 * d * d)
    # whole call: mixed projection, a, b, z in, out, states, conv tail
    call_bytes = (T * (w.Cc * e + 2 * Hv * e + Hv * d * e + Hv * d * e) + state_in + state_out
                  + N * w.Cc * 3 * e)
    return dict(core_bytes=core_bytes, core_flops=core_flops, call_bytes=call_bytes,
                call_flops=core_flops)


def decode_counts(inp, state_bytes=4, T=1):
    """Algorithmic bytes of one decode step of T tokens for each of the
    workload's sequences (the token rows of `inp` are T per sequence)."""
    w = inp.w
    B, Hv, d = inp.mixed_qkv.shape[0] // T, w.Hv, w.d
    e = 2 if w.dtype == "bf16" else 4
    state = 2 * B * Hv * d * d * state_bytes
    conv = 2 * B * w.Cc * 3 * e
    io = B * T * (w.Cc * e + 2 * Hv * e + Hv * d * e + Hv * d * e)
    return dict(bytes=state + conv + io, flops=B * Hv * 6 * d * d)


# ------------------------------------------------------------- clocks


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append(dict(sm=float(parts[1]), smax=float(parts[2]), power=float(parts[3]),
                                 hw=parts[5], hwt=parts[6], swt=parts[7], pcap=parts[8]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        loaded = [r for r in rows if r["power"] > 200.0] or rows
        reasons = set()
        for r in loaded:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
                if r[key].lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in loaded),
                "sm_max_mhz": max(r["smax"] for r in rows), "reasons": sorted(reasons),
                "samples": len(rows), "samples_under_load": len(loaded)}


# ---------------------------------------------------------- CPU baseline


def cpu_oracle_prefill_sample(inp, budget_s=12.0):
    """Time the fp64 oracle on the first n tokens of the first sequence (all
    value heads, one host thread per head up to the core count), growing n
    until the run takes about budget_s/8, then one timed run at the size that
    fills the budget.  Returns (tokens/s, threads, description, seconds)."""
    import oracle
    w = inp.w
    threads = min(os.cpu_count() or 1, w.Hv)
    first = int(inp.cu_seqlens[1])

    def run(n):
        x0 = time.perf_counter()
        oracle.prefill(w.Hk, w.Hv, w.d, w.d, [0, n], inp.mixed_qkv[:n], inp.conv_w, inp.a[:n],
                       inp.b[:n], inp.A_log, inp.dt_bias, inp.z[:n], inp.norm_w,
                       None if inp.initial_state is None else inp.initial_state[:1],
                       None, scale=w.scale, nthreads=threads)
        return time.perf_counter() - x0

    n = min(32, first)
    dt = run(n)
    while dt < budget_s / 8 and n < first:
        n = min(first, n * 2)
        dt = run(n)
    n_final = min(first, max(n, int(n * (budget_s / max(dt, 1e-6)))))
    if n_final != n:
        dt = run(n_final)
        n = n_final
    return n / dt, threads, "first %d tokens of one sequence, all %d value heads" % (n, w.Hv), dt


def cpu_oracle_decode_sample(inp, budget_s=6.0):
    import oracle
    w = inp.w
    threads = os.cpu_count() or 1
    B_all = inp.mixed_qkv.shape[0]

    def run(B):
        x0 = time.perf_counter()
        oracle.decode(w.Hk, w.Hv, w.d, w.d, inp.mixed_qkv[:B], inp.conv_w, inp.a[:B], inp.b[:B],
                      inp.A_log, inp.dt_bias, inp.z[:B], inp.norm_w, inp.state[:B],
                      inp.conv_state[:B], scale=w.scale, nthreads=threads)
        return time.perf_counter() - x0

    B = min(8, B_all)
    dt = run(B)
    while dt < budget_s / 4 and B < B_all:
        B = min(B_all, B * 2)
        dt = run(B)
    return B / dt, threads, "%d of %d sequences, one token each" % (B, B_all)


# ------------------------------------------------------------- GPU arm

IMPL_NAMES = {1: "simt", 2: "tc", 3: "tc_split", 4: "tc_fused"}


def core_description(gdn, impl, nseg):
    """(kernel names, source file, launches per call) of the chunked core that
    `impl` runs, and the launches of the whole call."""
    if impl == gdn.GDN_IMPL_TC_FUSED:
        return "chunk_fused_kernel", "chunk_fused.cu", 1, 3  # + queue order, conv
    if impl == gdn.GDN_IMPL_TC_SPLIT:
        if nseg > 1:
            return ("chunk_keys_kernel + chunk_chain_kernel<xfer> + seg_scan_kernel + chunk_chain_kernel"
                    " (%d segments)" % nseg, "chunk_tc_split.cu", 4, 5)
        return "chunk_keys_kernel + chunk_chain_kernel", "chunk_tc_split.cu", 2, 3
    if impl == gdn.GDN_IMPL_TC:
        return "chunk_tc_kernel", "chunk_tc.cu", 1, 2
    return "chunk_simt_kernel", "chunk_simt.cu", 1, 2


def bench_prefill(name, args, world, dev, peaks, peak_kind, flush, stream, want_cp=False):
    """One prefill workload: the timed steps, the core's roofline, e2e and
    (single GPU, one sequence) the context-parallel pieces."""
    import torch
    import torch.distributed as dist
    from hybrid_linear_attention_05_b200 import api, gdn

    wp = WORKLOADS[name]
    inp = make_prefill(wp)
    dp = api.to_device(inp, device=dev, chunk=args.chunk)
    bufs = api.PrefillBuffers(dp)
    impl = gdn.gdn_prefill_resolve_impl(bufs.dims, inp.N, inp.T, dp.chunk, bufs.dtype_code,
                                        gdn.GDN_IMPL_AUTO, bufs.ws_bytes)
    nseg = gdn.gdn_prefill_auto_segments(bufs.dims, inp.N, inp.T) if impl == gdn.GDN_IMPL_TC_SPLIT else 1
    core_name, core_src, core_launches, call_launches = core_description(gdn, impl, nseg)

    def step(core_ev=None):
        api.prefill(dp, bufs=bufs, core_events=core_ev)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    # the headline steps run as a user would call them (no event between the
    # library's launches, which would keep a kernel from starting early)
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        evs[i][0].record(stream)
        step()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    step_ms = [a.elapsed_time(b) for a, b in evs]
    # the core's own time: the same steps again with the library recording
    # events around its core launches (for the roofline only)
    cevs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(args.steps)]
    for a, b in cevs:  # torch creates the CUDA event on first record; the library re-records it
        a.record(stream)
        b.record(stream)
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        step(core_ev=cevs[i])
    torch.cuda.synchronize()
    core_ms = [a.elapsed_time(b) for a, b in cevs]
    total_ms = max_over_ranks(sum(step_ms), dev)
    ms_per_step = total_ms / args.steps
    value = job_throughput(inp.T, world, ms_per_step * 1e-3)

    cnt = prefill_counts(inp, dp.chunk)
    core_avg_s = max_over_ranks(statistics.mean(core_ms), dev) * 1e-3
    hbm = peaks["hbm_gbs"]
    roofline = {
        "kernel": core_name,
        "bound": "hbm",
        "achieved": cnt["core_bytes"] / core_avg_s / 1e9,
        "peak": hbm,
        "unit": "GB/s",
        "frac": cnt["core_bytes"] / core_avg_s / 1e9 / hbm,
        "traffic": profiled_traffic(core_src, name),
        "peak_source": peak_kind,
        "algorithmic_bytes_per_launch": cnt["core_bytes"],
        "algorithmic_flops_per_launch": cnt["core_flops"],
        "kernel_us": core_avg_s * 1e6,
        "tensor_tflops": cnt["core_flops"] / core_avg_s / 1e12,
        "tensor_frac_of_burst": cnt["core_flops"] / core_avg_s / 1e12 / peaks["bf16_tflops"],
        "whole_call_hbm_frac": cnt["call_bytes"] / (ms_per_step * 1e-3) / 1e9 / hbm,
        "roofline_tokens_per_s": inp.T / max(cnt["call_bytes"] / (hbm * 1e9),
                                             cnt["call_flops"] / (peaks["bf16_tflops"] * 1e12)),
    }

    # ---------------- e2e: pinned host inputs -> device -> prefill -> host
    # Every step copies its inputs from pinned host memory, runs gdn_prefill
    # through the public call and reads its output and final state back.  Two
    # device buffer sets alternate between steps, and three streams (copy in,
    # compute, copy out) let step i+1's inputs cross PCIe while step i
    # computes and is read back, as a serving loop would; the timed region
    # spans all steps, from the first copy to the last read-back.
    host = {k: torch.from_numpy(np.ascontiguousarray(getattr(inp, k))).to(dp.dtype).pin_memory()
            for k in ("mixed_qkv", "a", "b", "z")}
    h_cu = torch.from_numpy(inp.cu_seqlens.astype(np.int32)).pin_memory()
    h_S0 = None if inp.initial_state is None else torch.from_numpy(inp.initial_state).pin_memory()
    slots = [(dp, bufs), (api.to_device(inp, device=dev, chunk=args.chunk), None)]
    slots[1] = (slots[1][0], api.PrefillBuffers(slots[1][0]))
    h_out = [torch.empty(bufs.out.shape, dtype=bufs.out.dtype).pin_memory() for _ in range(2)]
    h_S = [torch.empty(bufs.final_state.shape, dtype=torch.float32).pin_memory() for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in host.values()) + h_cu.numel() * 4 + (
        0 if h_S0 is None else h_S0.numel() * 4)
    d2h = h_out[0].numel() * h_out[0].element_size() + h_S[0].numel() * 4
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()  # noqa: E731
    in_ready = [ev(), ev()]      # inputs of a slot copied
    computed = [ev(), ev()]      # a slot's prefill done (its inputs free again)
    read_back = [ev(), ev()]     # a slot's outputs copied to the host

    def e2e_step(i):
        k = i & 1
        d, b = slots[k]
        with torch.cuda.stream(s_in):
            s_in.wait_event(computed[k])  # the step two back is done with these inputs
            for nm, t in host.items():
                getattr(d, nm).copy_(t, non_blocking=True)
            d.cu_seqlens.copy_(h_cu, non_blocking=True)
            if h_S0 is not None:
                d.initial_state.copy_(h_S0, non_blocking=True)
            in_ready[k].record(s_in)
        stream.wait_event(in_ready[k])
        stream.wait_event(read_back[k])  # the step two back has read these outputs
        api.prefill(d, bufs=b)
        computed[k].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(computed[k])
            h_out[k].copy_(b.out, non_blocking=True)
            h_S[k].copy_(b.final_state, non_blocking=True)
            read_back[k].record(s_out)

    for k in range(2):  # the events start recorded, so the first waits pass
        for e in (computed[k], read_back[k]):
            e.record(stream)
    for i in range(max(2, args.warmup)):
        e2e_step(i)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    s_in.wait_event(t0)
    for i in range(args.steps):
        e2e_step(i)
    for s_ in (s_in, s_out):
        e_ = torch.cuda.Event()
        e_.record(s_)
        stream.wait_event(e_)
    t1.record(stream)
    torch.cuda.synchronize()
    e2e_total = max_over_ranks(t0.elapsed_time(t1), dev)
    e2e = {"value": job_throughput(inp.T, world, e2e_total / args.steps * 1e-3), "unit": "tokens/s",
           "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
           "pipelined": "two buffer sets; copy-in, compute and copy-out streams"}
    del host, h_out, h_S, slots

    # ---------------- context-parallel pieces (one sequence, one GPU): the
    # kernels one rank runs for its part of a long sequence -- the map of the
    # part, the fold of the earlier parts' maps, the part's prefill -- each with
    # the L2 flushed before it.  The exchange between ranks (one all-gather of
    # the maps) is not part of these numbers.
    context_parallel = None
    if want_cp and world == 1 and inp.N == 1 and wp.d == 128 and wp.dtype == "bf16":
        W_cp = 8
        maps = api.state_map(dp, bufs)
        gathered = maps.expand(W_cp - 1, *maps.shape).contiguous()
        S_buf = torch.empty((1, wp.Hv, wp.d, wp.d), dtype=torch.float32, device=dev)

        def timed(fn):
            for _ in range(max(3, args.warmup)):
                fn()
            torch.cuda.synchronize()
            tot = 0.0
            for i in range(args.steps):
                flush.fill_(i & 0xFF)
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                fn()
                b.record(stream)
                torch.cuda.synchronize()
                tot += a.elapsed_time(b)
            return tot / args.steps * 1e3  # us

        map_us = timed(lambda: api.state_map(dp, bufs))
        fold_us = timed(lambda: api.state_fold(gathered, None, wp.Hk, wp.Hv, wp.d, out=S_buf))
        part_us = timed(lambda: api.prefill(dp, bufs=bufs, reuse_workspace=True))
        rank_us = map_us + fold_us + part_us
        context_parallel = {
            "parts": W_cp, "tokens_per_part": inp.T,
            "map_us": map_us, "fold_us": fold_us, "fold_maps": W_cp - 1,
            "prefill_after_map_us": part_us, "rank_us": rank_us,
            "rank_tokens_per_s": inp.T / (rank_us * 1e-6),
            "exchange_bytes_per_part": int(maps.numel() * 4),
            "note": "kernels of the last rank of a context-parallel prefill of one sequence of "
                    "%d x %d tokens, on one GPU; the all-gather of the maps is not included" % (W_cp, inp.T),
        }
        del maps, gathered, S_buf

    res = {
        "workload": name, "value": value, "unit": "tokens/s", "ms_per_step": ms_per_step,
        "config": {"workload": name, "sequences": inp.N, "tokens": inp.T,
                   "sequence_lengths": [int(x) for x in np.diff(inp.cu_seqlens)],
                   "key_heads": wp.Hk, "value_heads": wp.Hv, "head_dim": wp.d, "chunk": dp.chunk,
                   "impl": IMPL_NAMES.get(impl, str(impl)),
                   "l2": "flushed before every timed step (256 MiB write)"},
        "roofline": roofline, "e2e": e2e, "launches_per_step": call_launches,
    }
    if context_parallel:
        res["context_parallel"] = context_parallel
    del dp, bufs
    torch.cuda.empty_cache()
    return res, inp


LAYER_D_MODEL = 4096  # the 9B model's hidden size (its mixer shapes are the 4 x 8192 workload's)


def layer_counts(inp, d_model):
    """FLOPs and bytes of the two projections of one layer call."""
    w = inp.w
    T, Cc, HVd = inp.T, w.Cc, w.Hv * w.d
    n_in = Cc + HVd + 2 * w.Hv
    return dict(in_flops=2 * T * n_in * d_model, out_flops=2 * T * d_model * HVd,
                in_bytes=2 * (T * d_model + n_in * d_model + T * n_in),
                out_bytes=2 * (T * HVd + d_model * HVd + T * d_model))


def cpu_oracle_layer_sample(li, budget_s=5.0):
    """The fp64 oracle's whole layer on the first n tokens of the first
    sequence, n grown until the run takes about budget_s."""
    import oracle
    w, m = li.mixer.w, li.mixer
    threads = min(os.cpu_count() or 1, w.Hv)
    first = int(m.cu_seqlens[1])
    Cc, HVd = w.Cc, w.Hv * w.d

    def run(n):
        x0 = time.perf_counter()
        oracle.layer(w.Hk, w.Hv, w.d, w.d, [0, n], li.hidden[:n], li.w_in[:Cc], li.w_in[Cc:Cc + HVd],
                     li.w_in[Cc + HVd + w.Hv:], li.w_in[Cc + HVd:Cc + HVd + w.Hv], li.w_out, m.conv_w,
                     m.A_log, m.dt_bias, m.norm_w, None if m.initial_state is None else m.initial_state[:1],
                     None, scale=w.scale, nthreads=threads)
        return time.perf_counter() - x0

    n = min(32, first)
    dt = run(n)
    while dt < budget_s / 4 and n < first:
        n = min(first, n * 2)
        dt = run(n)
    return n / dt, threads, "first %d tokens of one sequence, d_model %d" % (n, li.d_model)


def bench_layer(name, args, world, dev, peaks, peak_kind, flush, stream):
    """The whole layer (in_proj, mixer, out_proj through gdn_layer_prefill) on
    a mixer workload with the 9B model's hidden size, and each projection's
    tensor-core throughput timed alone."""
    import torch
    from hybrid_linear_attention_05_b200 import api, gdn
    from hybrid_linear_attention_05_b200.workloads import make_layer

    wp = WORKLOADS[name]
    li = make_layer(wp, LAYER_D_MODEL)
    dl = api.layer_to_device(li, device=dev)
    lb = api.LayerBuffers(dl)
    T = li.mixer.T

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        ms = []
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            torch.cuda.synchronize()
            ms.append(a.elapsed_time(b))
        return max_over_ranks(statistics.mean(ms), dev)

    layer_ms = timed(lambda: api.layer_prefill(dl, bufs=lb))
    cnt = layer_counts(li.mixer, LAYER_D_MODEL)
    HVd = wp.Hv * wp.d
    n_in = dl.w_in.shape[0]
    y_in = torch.empty((T, n_in), dtype=torch.bfloat16, device=dev)
    o_in = torch.empty((T, HVd), dtype=torch.bfloat16, device=dev).normal_()
    in_ms = timed(lambda: gdn.gdn_linear(x=dl.hidden, w=dl.w_in, M=T, N=n_in, K=LAYER_D_MODEL,
                                         outs=[(y_in, n_in, n_in)]))
    out_ms = timed(lambda: gdn.gdn_linear(x=o_in, w=dl.w_out, M=T, N=LAYER_D_MODEL, K=HVd,
                                          outs=[(lb.y, LAYER_D_MODEL, LAYER_D_MODEL)]))
    peak = peaks["bf16_tflops"]
    proj = {}
    for key, ms, fl, by in (("in_proj", in_ms, cnt["in_flops"], cnt["in_bytes"]),
                            ("out_proj", out_ms, cnt["out_flops"], cnt["out_bytes"])):
        tf = fl / (ms * 1e-3) / 1e12
        proj[key] = {"kernel": "linear_tc_kernel", "bound": "tensor", "achieved": tf, "peak": peak,
                     "unit": "TFLOP/s", "frac": tf / peak, "peak_source": peak_kind + " (burst: timed alone)",
                     "kernel_us": ms * 1e3, "algorithmic_flops_per_launch": fl,
                     "algorithmic_bytes_per_launch": by}
    proj["in_proj"]["shape"] = "M %d, N %d (qkv %d | z %d | b %d | a %d), K %d" % (
        T, n_in, wp.Cc, HVd, wp.Hv, wp.Hv, LAYER_D_MODEL)
    proj["out_proj"]["shape"] = "M %d, N %d, K %d" % (T, LAYER_D_MODEL, HVd)
    res = {"workload": name + " + projections d_model %d" % LAYER_D_MODEL,
           "value": job_throughput(T, world, layer_ms * 1e-3), "unit": "tokens/s", "ms_per_step": layer_ms,
           "config": {"workload": name, "d_model": LAYER_D_MODEL, "tokens": T, "sequences": li.mixer.N,
                      "impl": "gdn_layer_prefill (in_proj GEMM, mixer, out_proj GEMM)",
                      "l2": "flushed before every timed step (256 MiB write)"},
           "projections": proj, "launches_per_step": 5}
    del dl, lb, y_in, o_in
    torch.cuda.empty_cache()
    return res, li


def bench_decode(args, world, dev, peaks, peak_kind, stream):
    import torch
    import torch.distributed as dist
    from hybrid_linear_attention_05_b200 import api

    hbm = peaks["hbm_gbs"]
    wd = WORKLOADS[args.decode_workload]
    dinp = make_decode(wd)

    def time_decode(state_dtype, T=1, src=None):
        dd = api.decode_to_device(src or dinp, device=dev, state_dtype=state_dtype)
        if T > 1:  # token rows b * T + t; the state and conv cache of the first B rows
            B = dd.B // T
            dd = api.DeviceDecode(Hk=dd.Hk, Hv=dd.Hv, d=dd.d, scale=dd.scale, B=B, mixed_qkv=dd.mixed_qkv,
                                  conv_w=dd.conv_w, a=dd.a, b=dd.b, A_log=dd.A_log, dt_bias=dd.dt_bias,
                                  z=dd.z, norm_w=dd.norm_w, state=dd.state[:B].contiguous(),
                                  conv_state=dd.conv_state[:B].contiguous())
        shape = (dd.B, dd.Hv, dd.d) if T == 1 else (dd.B, T, dd.Hv, dd.d)
        dout = torch.empty(shape, dtype=dd.mixed_qkv.dtype, device=dev)
        for _ in range(args.warmup):
            api.decode(dd, out=dout, T=T)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        dev_ms = []
        for i in range(args.steps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            api.decode(dd, out=dout, T=T)
            b.record(stream)
            dev_ms.append((a, b))
        torch.cuda.synchronize()
        d_total = max_over_ranks(sum(a.elapsed_time(b) for a, b in dev_ms), dev)
        state_mib = dd.state.numel() * dd.state.element_size() >> 20
        del dd
        return d_total / args.steps * 1e-3, state_mib

    d_step_s, state_mib = time_decode(torch.float32)
    dcnt = decode_counts(dinp)
    decode = {
        "metric": "GDN decode tokens/s per layer", "unit": "tokens/s",
        "value": job_throughput(dinp.mixed_qkv.shape[0], world, d_step_s), "ms_per_step": d_step_s * 1e3,
        "workload": args.decode_workload,
        "roofline": {"kernel": "decode_kernel", "bound": "hbm",
                     "achieved": dcnt["bytes"] / d_step_s / 1e9, "peak": hbm, "unit": "GB/s",
                     "frac": dcnt["bytes"] / d_step_s / 1e9 / hbm,
                     "traffic": profiled_traffic("decode.cu", args.decode_workload),
                     "peak_source": peak_kind, "algorithmic_bytes_per_launch": dcnt["bytes"]},
        "l2": "state (%d MiB) larger than L2" % state_mib,
    }
    # the same step with the recurrent state held in bf16 (half the state bytes)
    b_step_s, b_state_mib = time_decode(torch.bfloat16)
    bcnt = decode_counts(dinp, state_bytes=2)
    decode["bf16_state"] = {
        "value": job_throughput(dinp.mixed_qkv.shape[0], world, b_step_s), "unit": "tokens/s",
        "ms_per_step": b_step_s * 1e3,
        "roofline": {"kernel": "decode_kernel (bf16 state)", "bound": "hbm",
                     "achieved": bcnt["bytes"] / b_step_s / 1e9, "peak": hbm, "unit": "GB/s",
                     "frac": bcnt["bytes"] / b_step_s / 1e9 / hbm, "peak_source": peak_kind,
                     "algorithmic_bytes_per_launch": bcnt["bytes"]},
        "l2": "state (%d MiB) larger than L2" % b_state_mib,
    }
    # short multi-token decode: T = 4 tokens per sequence and step (fp32 state)
    T_mt = 4
    mt_inp = make_decode(wd, batch=dinp.mixed_qkv.shape[0] * T_mt)
    m_step_s, _ = time_decode(torch.float32, T=T_mt, src=mt_inp)
    mcnt = decode_counts(mt_inp, T=T_mt)
    decode["multi_token"] = {
        "tokens_per_sequence": T_mt,
        "value": job_throughput(dinp.mixed_qkv.shape[0] * T_mt, world, m_step_s), "unit": "tokens/s",
        "ms_per_step": m_step_s * 1e3,
        "roofline": {"kernel": "decode_multi_kernel (T = 4)", "bound": "hbm",
                     "achieved": mcnt["bytes"] / m_step_s / 1e9, "peak": hbm, "unit": "GB/s",
                     "frac": mcnt["bytes"] / m_step_s / 1e9 / hbm, "peak_source": peak_kind,
                     "algorithmic_bytes_per_launch": mcnt["bytes"]},
    }
    return decode, dinp


def run_ours(args, rank, world, local_rank):
    import torch
    from hybrid_linear_attention_05_b200 import gdn
    from hybrid_linear_attention_05_b200 import build as libbuild

    libbuild.build()
    gdn.lib()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    peaks, peak_kind = load_peaks()
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    with ClockSampler(local_rank) as clk:
        head, inp = bench_prefill(args.workload, args, world, dev, peaks, peak_kind, flush, stream)
        others = []
        for name in args.also:
            r, o_inp = bench_prefill(name, args, world, dev, peaks, peak_kind, flush, stream, want_cp=True)
            others.append((r, o_inp))
        decode, dinp = bench_decode(args, world, dev, peaks, peak_kind, stream)
        layer, linp = (None, None) if args.no_layer else bench_layer(
            args.layer_workload, args, world, dev, peaks, peak_kind, flush, stream)

    result = {
        "metric": METRIC,
        "value": head["value"], "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": WORKLOADS[args.workload].dtype,
        "data": "synthetic (seeded draws of the workload's shapes and distributions)",
        "config": {**head["config"], "parallelism": "replica per GPU (weak)"},
        "roofline": head["roofline"],
        "e2e": head["e2e"],
        "prefill": {r["workload"]: {k: v for k, v in r.items() if k != "workload"} for r, _ in others},
        "decode": decode,
        "layer": layer,
        # the library's kernels launched in the headline's timed steps
        "gpu_launches": head["launches_per_step"] * args.steps,
        "clocks": clk.summary(),
    }
    return result, inp, others, dinp, linp


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_PREFILL)
    ap.add_argument("--also", nargs="*", default=DEFAULT_ALSO,
                    help="further prefill workloads measured in the same run")
    ap.add_argument("--decode-workload", default=DEFAULT_DECODE)
    ap.add_argument("--chunk", type=int, default=None, help="override the workload's chunk length")
    ap.add_argument("--layer-workload", default="prefill_4x8192_Hk16_Hv32_d128",
                    help="mixer workload of the whole-layer line (hidden size %d)" % LAYER_D_MODEL)
    ap.add_argument("--no-layer", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--launcher-selftest", action="store_true",
                    help="start the ranks, join them on gloo and report them (no GPU work)")
    args = ap.parse_args()

    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        # one process per GPU: start the ranks ourselves
        if not args.launcher_selftest and args.impl == "ours":
            import torch
            have = torch.cuda.device_count()
            if have < args.gpus:
                print(json.dumps({"metric": METRIC, "error": "--gpus %d but this node has %d GPUs"
                                  % (args.gpus, have)}))
                sys.exit(1)
        cmd = launch_command(sys.argv[1:], args.gpus, _free_port())
        sys.exit(subprocess.call(cmd))

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        if rank == 0:
            print(json.dumps({"metric": METRIC, "error": "WORLD_SIZE %d differs from --gpus %d"
                              % (world, args.gpus)}))
        sys.exit(1)

    if args.launcher_selftest:
        import datetime
        import torch
        import torch.distributed as dist
        dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
        got = [None] * world
        dist.all_gather_object(got, (rank, local_rank, os.getpid()))
        if rank == 0:
            print(json.dumps({"world": world, "ranks": [g[0] for g in got],
                              "local_ranks": [g[1] for g in got], "pids": [g[2] for g in got]}))
        dist.destroy_process_group()
        return

    if args.impl == "reference":
        # The reference arm is the fp64 CPU oracle (there is no reference
        # implementation to install: the reference is a text of web pages).
        # Rank 0 runs it on the host cores; other ranks exit without work.
        if rank != 0:
            return
        wp = WORKLOADS[args.workload]
        inp = make_prefill(wp)
        vals, secs = [], []
        cores, sample = 1, ""
        for i in range(args.warmup + args.steps):
            v, cores, sample, dt = cpu_oracle_prefill_sample(inp, budget_s=3.0)
            if i >= args.warmup:
                vals.append(v)
                secs.append(dt)
        value = statistics.mean(vals)
        print(json.dumps({
            "impl": "reference", "metric": METRIC, "value": value,
            "unit": "tokens/s", "n_gpus": 0, "gpus_requested": args.gpus, "runs_on": "host CPU cores",
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": statistics.mean(secs) * 1e3, "step": "one bounded sample: " + sample,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded draws of the workload's shapes and distributions)",
            "config": {"workload": args.workload, "sequences": inp.N, "tokens": inp.T},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}))
        return

    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    result, inp, others, dinp, linp = run_ours(args, rank, world, local_rank)
    if rank == 0:
        if not args.no_cpu_baseline:
            v, cores, sample, _ = cpu_oracle_prefill_sample(inp, budget_s=10.0)
            result["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": cores,
                                      "kind": "oracle", "sample": sample}
            for r, o_inp in others:
                v, cores, sample, _ = cpu_oracle_prefill_sample(o_inp, budget_s=5.0)
                result["prefill"][r["workload"]]["cpu_baseline"] = {
                    "value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample}
            dv, dcores, dsample = cpu_oracle_decode_sample(dinp)
            result["decode"]["cpu_baseline"] = {"value": dv, "unit": "tokens/s", "cores": dcores,
                                                "kind": "oracle", "sample": dsample}
            if linp is not None:
                lv, lcores, lsample = cpu_oracle_layer_sample(linp)
                result["layer"]["cpu_baseline"] = {"value": lv, "unit": "tokens/s", "cores": lcores,
                                                   "kind": "oracle", "sample": lsample}
        print(json.dumps(result))
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
