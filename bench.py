"""Benchmark of the block-sparse attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

One step = one forward over one batch of the workload (the whole hot path:
one kernel launch that builds the per-tile block maps, streams Q/K/V with TMA,
runs both contractions on tcgen05 and the restricted softmax, merges the
chunks of cut tiles, and writes O and LSE), through bsa_forward_ws with a
workspace allocated once.  The pattern CSR is built once, outside the timed
region.  The default workload is the largest, causal_loglinear_32k.

Timing: W untimed warm-up steps; a soak of untimed steps (about 1.2 s, each
after its L2 flush) so that the clock samples see the loaded GPU; then K
timed steps.  Before every step the L2 is evicted by reading a 512 MB buffer
(a read leaves no dirty lines to write back during the step), and each step
is bracketed by CUDA events on the launching stream; the reported time is
the sum of the event intervals.  A barrier and a device synchronize surround
the timed loop; with N > 1 ranks (torchrun) every rank runs its own replica
(weak scaling, no collective in the data path) and the time is the max over
ranks.  Clock statistics are taken over the samples inside soak + timed loop.

Metric: useful TFLOP/s = 4 * bs^2 * d * (stored blocks over all heads) * B /
time, counting every stored block in full (diagonal causal blocks included).

`--impl reference` times the fp64 CPU oracle (the only reference there is) on
the host cores, each step a bounded sample of query rows of the same workload.
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
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "block-sparse attn fwd useful TFLOP/s & ms/fwd (1 B200), % of roofline"
DEFAULT_WORKLOAD = "causal_loglinear_32k"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNEL_DIR = os.path.join(ROOT, "block_sparse_attention_38_b200", "csrc")

# DRAM bytes (read + write) per launch from ncu captures of the kernel, keyed by
# workload, valid only for the kernel sources whose sha256 prefix is given
# (profiles/ holds the capture summaries).
NCU_TRAFFIC = {
    "loglinear_4k": (25427712 + 0, "b3f14ca92b384dc0"),
    "local_global_8k": (286169856 + 48533248, "b3f14ca92b384dc0"),
    "bernoulli_4k": (201544448 + 49105152, "b3f14ca92b384dc0"),
    "causal_loglinear_32k": (848413184 + 254313728, "e360f7440fb5438f"),
    "topk_4k": (25511680 + 0, "b3f14ca92b384dc0"),
    # the decode kernel, keyed by the hash of DECODE_SOURCES
    "decode_loglinear_32k": (175443200 + 3267584, "386e68dbdbbe3b74"),
    # the backward's three kernels together (dot + dK/dV + dQ), one backward
    "local_global_8k:backward": (134229248 + 4284160 + 336716800 + 111309568 + 330468096
                                 + 55514880, "418be616a808a425"),
}


def replica_seed(w, rank: int) -> int:
    """Seed of rank `rank`'s replica of workload w (rank 0 uses the workload's own seed)."""
    return w.seed + 1000 * rank


def max_over_ranks(values, world: int, device=None):
    """Element-wise maximum of `values` over all ranks (identity for one rank).

    Every rank calls it with the same number of values; the reduction runs on
    the process group's backend (NCCL with device tensors, gloo on the CPU)."""
    if world == 1:
        return [float(v) for v in values]
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.cpu()]


def whole_job_tflops(flops_per_rank: float, world: int, ms_per_step: float) -> float:
    """Aggregate useful TFLOP/s of `world` replicas that each did flops_per_rank in ms_per_step."""
    return flops_per_rank * world / (ms_per_step * 1e-3) / 1e12


def e2e_chunks(w, n_chunks: int = 0):
    """Contiguous input slices for the pipelined end-to-end step, as
    (index into [B, H, ...] tensors, first head, end head): whole batch
    entries when B > 1, else ranges of heads (the head range also selects the
    block-CSR rows h*M .. h_end*M).  By default inputs of 128 MB or more are
    cut in four; smaller ones stay whole, where the extra copies and launches
    issued per chunk cost more than the overlap gains (measured)."""
    if n_chunks <= 0:
        n_chunks = 4 if compulsory_bytes(w) >= 128e6 else 1
    if w.B > 1:
        n = min(n_chunks, w.B)
        cuts = [w.B * i // n for i in range(n + 1)]
        return [(slice(cuts[i], cuts[i + 1]), 0, w.H) for i in range(n)]
    n = min(n_chunks, w.H)
    cuts = [w.H * i // n for i in range(n + 1)]
    return [((slice(0, 1), slice(cuts[i], cuts[i + 1])), cuts[i], cuts[i + 1]) for i in range(n)]


def useful_flops(w, nnz_all_heads: int) -> float:
    return 4.0 * w.block_size * w.block_size * w.d * nnz_all_heads * w.B


def compulsory_bytes(w) -> float:
    return 4.0 * w.B * w.H * w.N * w.d * 2 + 4.0 * w.B * w.H * w.N


# The files each kernel is compiled from (its .cu and what it includes).
FORWARD_SOURCES = ("bsa_common.cuh", "bsa_forward.cu", "bsa_fwd_pp.cuh", "sm100_ptx.cuh")
DECODE_SOURCES = ("bsa_decode.cu", "sm100_ptx.cuh")
BACKWARD_SOURCES = ("bsa_backward.cu", "sm100_ptx.cuh")


def kernel_hash(sources=FORWARD_SOURCES) -> str:
    """sha256 prefix over a kernel's source files (sorted by name)."""
    h = hashlib.sha256()
    for name in sorted(sources):
        with open(os.path.join(KERNEL_DIR, name), "rb") as f:
            h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()[:16]


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms in the background."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        import tempfile

        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self, region=None):
        """Stop sampling; statistics over the samples taken inside `region`
        (wall-clock seconds (t0, t1), time.time() based) when given."""
        import datetime

        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                rows.append((ts, float(parts[2]), float(parts[3]), float(parts[4]), parts[6:10]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        inside = [r for r in rows if region is None or region[0] <= r[0] <= region[1]]
        use = inside or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in use for i in range(4) if r[4][i].lower() == "active"})
        return {"sm_mhz": statistics.median(r[1] for r in use), "sm_max_mhz": max(r[2] for r in rows),
                "sm_mhz_min": min(r[1] for r in use), "power_w_max": max(r[3] for r in use),
                "reasons": reasons, "samples": len(rows), "samples_in_timed_region": len(inside)}


L2_NOTE = "evicted before every timed step by a 512 MB read (no dirty lines left behind)"


class L2Flush:
    """Evicts the 126 MB L2 by reading a 512 MB buffer: a read leaves clean
    lines, so the timed kernel does not pay for writing back a flush's dirty
    lines."""

    def __init__(self, device):
        import torch

        self.buf = torch.zeros(128 * 1024 * 1024, dtype=torch.float32, device=device)

    def __call__(self):
        self.buf.sum()


def fwd_config(w, nnz: int, world: int, backward: bool = False) -> dict:
    """The `config` of a forward (or backward) line; both arms print the same one."""
    c = {"workload": w.name}
    if backward:
        c["pass"] = "backward"
    c.update({"B": w.B, "H": w.H, "N": w.N, "d": w.d, "block_size": w.block_size,
              "nnz_blocks": int(nnz), "causal": bool(w.causal), "l2": L2_NOTE,
              "parallelism": f"replicas x{world}"})
    if w.pattern.kind == workloads.TOPK:
        c["top_k"] = w.pattern.top_k
    return c


def decode_config(w, tokens_attended: int, world: int) -> dict:
    """The `config` of a decode line; both arms print the same one."""
    return {"workload": w.name, "B": w.B, "H": w.H, "L": w.L, "d": w.d,
            "block_size": w.block_size, "tokens_attended": int(tokens_attended),
            "append": bool(w.append), "l2": L2_NOTE, "parallelism": f"replicas x{world}"}


def soak(step, flush, seconds: float):
    """Untimed steps (each after its L2 flush) back to back for about
    `seconds`, right before the timed region: the clock samples then see the
    GPU under the same load as the timed steps.  Returns (steps, seconds)."""
    import torch

    if seconds <= 0:
        return 0, 0.0
    n = 0
    t0 = time.time()
    while True:
        for _ in range(8):
            flush()
            step()
            n += 1
        torch.cuda.synchronize()
        if time.time() - t0 >= seconds:
            return n, time.time() - t0


def cpu_model() -> str:
    """The host CPU's model name (from /proc/cpuinfo), or '' when unknown."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return ""


def causal_exact_flops(w, rp, ci) -> float:
    """4 d flops per (query, key) pair the causal mask keeps: a stored block
    j < i holds bs^2 pairs, the diagonal block bs (bs + 1) / 2."""
    bs, M = w.block_size, w.M
    pairs = 0
    for h in range(w.H):
        for i in range(M):
            for j in ci[rp[h * M + i]:rp[h * M + i + 1]]:
                pairs += bs * bs if j < i else (bs * (bs + 1) // 2 if j == i else 0)
    return 4.0 * w.d * pairs * w.B


def cpu_oracle_sample(w, q, k, v, rp, ci, seconds: float, rng_seed: int = 0, nthreads: int = 0):
    """Time the fp64 oracle on random query rows until `seconds` of work; returns
    (useful TFLOP/s, threads, rows done, seconds)."""
    import oracle

    rng = np.random.default_rng(rng_seed)
    total_rows = w.B * w.H * w.N
    lens = np.diff(rp).astype(np.int64)          # blocks per (h, block row)
    done_rows, flops, elapsed, threads = 0, 0.0, 0.0, 0
    batch = 256
    while elapsed < seconds:
        rows = rng.integers(0, total_rows, batch)
        h = (rows // w.N) % w.H
        r = (rows % w.N) // w.block_size
        t0 = time.perf_counter()
        _, _, threads = oracle.forward(q, k, v, rp, ci, w.block_size, w.scale, w.causal,
                                       rows=rows, nthreads=nthreads)
        elapsed += time.perf_counter() - t0
        flops += float((4.0 * w.block_size * w.d * lens[h * w.M + r]).sum())
        done_rows += batch
        if elapsed < seconds / 8:
            batch *= 2
    return flops / elapsed / 1e12, threads, done_rows, elapsed


def oracle_problem(w, q, k, v):
    """The oracle's view of workload w: (workload, q, k, v, row_ptr, col_idx).
    A top-k workload's pattern is the oracle's own selection, one CSR row per
    (b, h, block row), with the batch folded into the heads."""
    from oracle import patterns

    if w.pattern.kind != workloads.TOPK:
        rp, ci = patterns.csr(w.pattern)
        return w, q, k, v, rp, ci
    from oracle import topk as topk_oracle

    rp, ci = topk_oracle.topk_pattern(q.float().numpy(), k.float().numpy(), w.block_size,
                                      w.pattern.top_k, w.causal)
    wf = workloads.Workload(w.name, 1, w.B * w.H, w.N, w.d, w.block_size, w.pattern, w.seed,
                            causal=w.causal)
    shape = (1, w.B * w.H, w.N, w.d)
    return wf, q.reshape(shape), k.reshape(shape), v.reshape(shape), rp, ci


def run_reference(args, w, rank, world):
    """fp64 CPU oracle on the host cores, each step a bounded sample of rows."""
    if rank != 0:
        return
    w_in = w
    w, q, k, v, rp, ci = oracle_problem(w, *workloads.make_qkv(w))
    step_seconds = 2.0
    for i in range(args.warmup):
        cpu_oracle_sample(w, q, k, v, rp, ci, 0.2, rng_seed=1000 + i)
    vals, times, rows_done = [], [], 0
    threads = 0
    for i in range(args.steps):
        tf, threads, nrows, el = cpu_oracle_sample(w, q, k, v, rp, ci, step_seconds, rng_seed=i)
        vals.append(tf)
        times.append(el)
        rows_done += nrows
    value = statistics.median(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * statistics.mean(times), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": fwd_config(w_in, len(ci), world),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": f"{rows_done} random query rows of {w.name} over {args.steps} steps"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- backward
ORACLE_BACKWARD_MAX_N = 8192  # the dense oracle's N x N fp64 arrays stay within a few GB


def backward_flops(w, nnz_all_heads: int) -> float:
    """Useful flops of one backward: per stored block the five products
    S = QK^T, dP = dO V^T, dV = P^T dO, dQ = dS K, dK = dS^T Q (2 bs^2 d each)."""
    return 10.0 * w.block_size * w.block_size * w.d * nnz_all_heads * w.B


def backward_bytes(w) -> float:
    """Compulsory bytes: Q, K, V, O, dO read, dQ, dK, dV written (bf16), LSE
    read and D written and read (fp32)."""
    return 8.0 * w.B * w.H * w.N * w.d * 2 + 3 * 4.0 * w.B * w.H * w.N


def cpu_backward_sample(w, q, k, v, do, rp, ci, seconds: float, rng_seed: int = 0):
    """Time the fp64 backward oracle on random (b, h) pairs until `seconds` of
    work; returns (useful TFLOP/s, threads, pairs done, seconds)."""
    import torch

    from oracle import backward as obw

    rng = np.random.default_rng(rng_seed)
    M = w.M
    done, flops, elapsed = 0, 0.0, 0.0
    while elapsed < seconds:
        b, h = int(rng.integers(w.B)), int(rng.integers(w.H))
        rph = (rp[h * M:(h + 1) * M + 1] - rp[h * M]).astype(np.int32)
        cih = ci[rp[h * M]:rp[(h + 1) * M]]
        sl = (slice(b, b + 1), slice(h, h + 1))
        t0 = time.perf_counter()
        obw.backward(q[sl], k[sl], v[sl], do[sl], rph, cih, w.block_size, w.scale, w.causal)
        elapsed += time.perf_counter() - t0
        flops += 10.0 * w.block_size * w.block_size * w.d * len(cih)
        done += 1
    return flops / elapsed / 1e12, torch.get_num_threads(), done, elapsed


def run_backward(args, w, rank, world, local_rank):
    import torch

    import block_sparse_attention_38_b200 as bsa

    if w.pattern.kind == workloads.TOPK:
        raise SystemExit("--backward runs on host-built patterns")
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    bsa.library()
    q_h, k_h, v_h = workloads.make_qkv(w, seed=replica_seed(w, rank))
    g = torch.Generator().manual_seed(replica_seed(w, rank) + 77)
    do_h = torch.randn(q_h.shape, generator=g).to(torch.bfloat16)
    q, k, v, do = (t.to(dev) for t in (q_h, k_h, v_h, do_h))
    rp_np, ci_np = bsa.build_pattern_from(w.pattern)
    cp_np, ri_np = bsa.transpose_pattern(rp_np, ci_np, w.H, w.M)
    rp, ci, cp, ri = (torch.from_numpy(x).to(dev) for x in (rp_np, ci_np, cp_np, ri_np))
    O, L = bsa.forward(q, k, v, rp, ci, w.block_size, w.scale, w.causal)
    ws = torch.empty(int(bsa.library().bsa_backward_workspace_bytes(w.B, w.H, w.N)) // 4,
                     dtype=torch.float32, device=dev)
    flops = backward_flops(w, len(ci_np))
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        return bsa.backward(q, k, v, O, do, L, rp, ci, cp, ri, w.block_size, w.scale, w.causal,
                            workspace=ws)

    for _ in range(args.warmup):
        flush()
        step()
    torch.cuda.synchronize()
    bsa.backward_status(clear=True)
    visible = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    ids = [x.strip() for x in visible.split(",") if x.strip()]
    clocks = ClockSampler(ids[local_rank] if local_rank < len(ids) else str(local_rank))
    if rank == 0:
        clocks.start()
    region0 = time.time()
    soak_steps, soak_s = soak(step, flush, args.soak_seconds)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if world > 1:
        import torch.distributed as dist

        dist.barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush()
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clock_info = clocks.stop((region0, time.time())) if rank == 0 else None
    per_step = [s_.elapsed_time(e) for s_, e in zip(starts, ends)]
    total_ms = float(sum(per_step))
    if bsa.backward_status(clear=True) or bsa.device_status(clear=True):
        raise RuntimeError("backward kernels reported a device status")

    # End to end through the public API: Q, K, V, O, dO, LSE and the two CSR
    # copies from pinned host memory, the backward, dQ, dK, dV back to pinned
    # host memory, every step.
    hosts = [t.cpu().pin_memory() for t in (q, k, v, O, do, L)]
    hcsr = [torch.from_numpy(x).pin_memory() for x in (rp_np, ci_np, cp_np, ri_np)]
    devs = [torch.empty_like(t, device=dev) for t in hosts + hcsr]
    outs_h = [torch.empty(q.shape, dtype=torch.bfloat16).pin_memory() for _ in range(3)]
    h2d = sum(t.numel() * t.element_size() for t in hosts + hcsr)
    d2h = sum(t.numel() * t.element_size() for t in outs_h)

    def e2e_step():
        for dst, src in zip(devs, hosts + hcsr):
            dst.copy_(src, non_blocking=True)
        grads = bsa.backward(*devs[:6], *devs[6:], w.block_size, w.scale, w.causal, workspace=ws)
        for dst, src in zip(outs_h, grads):
            dst.copy_(src, non_blocking=True)
        return grads

    for _ in range(max(1, args.warmup)):
        e2e_step()
    torch.cuda.synchronize()
    e_steps = max(3, min(args.steps, 20))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(e_steps):
        grads = e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e_steps
    if not all(torch.equal(hh, gg.cpu()) for hh, gg in zip(outs_h, grads)):
        raise RuntimeError("end-to-end result differs from the device result")

    total_ms, e2e_ms = max_over_ranks([total_ms, e2e_ms], world, device=dev)
    if rank != 0:
        return
    ms = total_ms / args.steps
    peaks, peak_src = load_peaks()
    peak_tc = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    roof = {"bound": "tensor", "achieved": flops / (ms * 1e-3) / 1e12, "peak": peak_tc,
            "unit": "TFLOP/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    tr = NCU_TRAFFIC.get(w.name + ":backward")
    roof["traffic"] = tr[0] if tr and tr[1] == kernel_hash(BACKWARD_SOURCES) else None
    roof["peak_source"] = f"{peak_src} (MEASURED_PEAKS.json burst)" if peak_src == "measured" else "fallback"
    roof["kernel"] = "bsa::bwd::dot_kernel + tile_cost/order + dkdv_kernel + dq_kernel"
    roof["kernel_ms"] = ms
    cpu = None
    if world == 1 and not args.no_cpu_baseline and w.N > ORACLE_BACKWARD_MAX_N:
        cpu = {"value": None, "unit": "TFLOP/s", "cores": 0, "kind": "oracle",
               "sample": f"none: the dense fp64 backward oracle holds N x N arrays per (b, h), "
                         f"too large at N = {w.N}"}
    elif world == 1 and not args.no_cpu_baseline:
        tf, threads, npairs, el = cpu_backward_sample(w, q_h, k_h, v_h, do_h, rp_np, ci_np,
                                                      args.cpu_seconds)
        cpu = {"value": tf, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
               "sample": f"{npairs} random (b, h) backward passes of {w.name} ({el:.1f} s, fp64)"}
    line = {
        "metric": METRIC, "value": whole_job_tflops(flops, world, ms), "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": fwd_config(w, len(ci_np), world, backward=True),
        "roofline": roof,
        "cpu_baseline": cpu,
        "e2e": {"value": whole_job_tflops(flops, world, e2e_ms), "unit": "TFLOP/s",
                "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                "ms_per_step": e2e_ms},
        "gpu_launches": 5 * args.steps,  # D, tile costs, tile orders, dK/dV, dQ
        "clocks": clock_info,
        "soak": {"steps": soak_steps, "seconds": soak_s},
        "min_ms": min(per_step), "median_ms": statistics.median(per_step),
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ decode
def decode_tokens(w, lens, rp, ci) -> np.ndarray:
    """Cached tokens each (b, h) attends to in one decode step, [B, H]: the
    blocks j <= i of CSR row i = (seq_len - 1) // block_size, counted once,
    block i only up to the new token."""
    bs, M = w.block_size, w.M
    n = np.zeros((w.B, w.H), dtype=np.int64)
    for b in range(w.B):
        t = int(lens[b]) - 1
        i = t // bs
        for h in range(w.H):
            cols = set(int(j) for j in ci[rp[h * M + i]:rp[h * M + i + 1]])
            n[b, h] = sum(bs for j in cols if j < i) + (t - i * bs + 1 if i in cols else 0)
    return n


def decode_flops(w, tokens) -> float:
    return 4.0 * w.d * float(tokens.sum())


def decode_bytes(w, tokens) -> float:
    """Algorithmic HBM bytes of one step: the attended K and V rows; q, k_new
    and v_new read; the appended K and V rows written; O, LSE and seq_len."""
    per_token = 2.0 * w.d * 2
    vectors = w.B * w.H * w.d * 2.0 * (3 + (2 if w.append else 0) + 1)
    return per_token * float(tokens.sum()) + vectors + 4.0 * w.B * w.H + 4.0 * w.B


def cpu_decode_sample(w, q, kn, vn, K, V, lens, rp, ci, seconds: float, rng_seed: int = 0):
    """Time the fp64 decode oracle on random (b, h) pairs (CPU tensors) until
    `seconds` of work; returns (useful TFLOP/s, threads, pairs done, seconds)."""
    from oracle import decode as odec

    rng = np.random.default_rng(rng_seed)
    tokens = decode_tokens(w, lens, rp, ci)
    done, flops, elapsed, batch = 0, 0.0, 0.0, 4
    while elapsed < seconds:
        pairs = [(int(b), int(h)) for b, h in zip(rng.integers(0, w.B, batch),
                                                  rng.integers(0, w.H, batch))]
        t0 = time.perf_counter()
        odec.decode(q, K, V, lens, rp, ci, w.block_size, w.scale,
                    k_new=kn if w.append else None, v_new=vn if w.append else None, pairs=pairs)
        elapsed += time.perf_counter() - t0
        flops += sum(4.0 * w.d * tokens[b, h] for b, h in pairs)
        done += batch
        if elapsed < seconds / 8:
            batch *= 2
    import torch

    return flops / elapsed / 1e12, torch.get_num_threads(), done, elapsed


def run_decode(args, w, rank, world, local_rank):
    import torch

    import block_sparse_attention_38_b200 as bsa

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    bsa.library()
    q, kn, vn, K, V, lens = workloads.make_decode_inputs(w, device=dev, seed=replica_seed(w, rank))
    rp_np, ci_np = bsa.build_pattern_from(w.pattern)
    rp = torch.from_numpy(rp_np).to(dev)
    ci = torch.from_numpy(ci_np).to(dev)
    lens_np = lens.cpu().numpy()
    tokens = decode_tokens(w, lens_np, rp_np, ci_np)
    flops, nbytes = decode_flops(w, tokens), decode_bytes(w, tokens)
    O = torch.empty((w.B, w.H, w.d), dtype=torch.bfloat16, device=dev)
    L = torch.empty((w.B, w.H), dtype=torch.float32, device=dev)
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream(dev)
    kw = dict(k_new=kn, v_new=vn) if w.append else {}

    def step():
        bsa.decode(q, K, V, lens, rp, ci, w.block_size, w.scale, out=O, lse=L, **kw)

    for _ in range(args.warmup):
        flush()
        step()
    torch.cuda.synchronize()
    bsa.decode_status(clear=True)
    visible = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    ids = [x.strip() for x in visible.split(",") if x.strip()]
    clocks = ClockSampler(ids[local_rank] if local_rank < len(ids) else str(local_rank))
    if rank == 0:
        clocks.start()
    region0 = time.time()
    soak_steps, soak_s = soak(step, flush, args.soak_seconds)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if world > 1:
        import torch.distributed as dist

        dist.barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush()
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clock_info = clocks.stop((region0, time.time())) if rank == 0 else None
    per_step = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = float(sum(per_step))
    status = bsa.decode_status(clear=True)
    if status:
        raise RuntimeError(f"decode kernel reported device status {status:#x}")

    # End to end through the public API: the KV cache is device state; each
    # step brings the new token's q, k, v and the lengths from pinned host
    # memory, runs the step and returns O and LSE to pinned host memory.
    qp, knp, vnp = (t.cpu().pin_memory() for t in (q, kn, vn))
    lp = lens.cpu().pin_memory()
    Oh = torch.empty(O.shape, dtype=O.dtype).pin_memory()
    Lh = torch.empty(L.shape, dtype=L.dtype).pin_memory()
    qd, knd, vnd, ld = (torch.empty_like(t) for t in (q, kn, vn, lens))
    ins = [(qd, qp), (ld, lp)] + ([(knd, knp), (vnd, vnp)] if w.append else [])
    h2d = sum(src.numel() * src.element_size() for _, src in ins)
    d2h = Oh.numel() * Oh.element_size() + Lh.numel() * Lh.element_size()
    ekw = dict(k_new=knd, v_new=vnd) if w.append else {}

    def e2e_step():
        for dst, src in ins:
            dst.copy_(src, non_blocking=True)
        bsa.decode(qd, K, V, ld, rp, ci, w.block_size, w.scale, out=O, lse=L, **ekw)
        Oh.copy_(O, non_blocking=True)
        Lh.copy_(L, non_blocking=True)

    for _ in range(max(1, args.warmup)):
        e2e_step()
    torch.cuda.synchronize()
    e_steps = max(3, min(args.steps, 50))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e_steps
    if bsa.decode_status(clear=True):
        raise RuntimeError("decode kernel reported a device status in the end-to-end leg")
    if not torch.equal(Oh, O.cpu()):
        raise RuntimeError("end-to-end result differs from the device result")

    total_ms, e2e_ms = max_over_ranks([total_ms, e2e_ms], world, device=dev)
    if rank != 0:
        return
    ms = total_ms / args.steps
    peaks, peak_src = load_peaks()
    peak_tc = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    peak_hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    t_tc = flops / (peak_tc * 1e12)
    t_hbm = nbytes / (peak_hbm * 1e9)
    roof = {"bound": "hbm", "achieved": nbytes / (ms * 1e-3) / 1e9, "peak": peak_hbm,
            "unit": "GB/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    if roof["bound"] == "tensor":
        # against the GEMM rate held for seconds under the power cap (the
        # timed steps follow a soak of the same steps)
        sustained = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
        roof["frac_of_sustained_peak"] = roof["achieved"] / sustained
    tr = NCU_TRAFFIC.get(w.name)
    roof["traffic"] = tr[0] if tr and tr[1] == kernel_hash(DECODE_SOURCES) else None
    roof["peak_source"] = f"{peak_src} (MEASURED_PEAKS.json burst)" if peak_src == "measured" else "fallback"
    roof["roofline_frac_max_of_tc_hbm"] = max(t_tc, t_hbm) / (ms * 1e-3)
    roof["kernel"] = "bsa::decode::decode_kernel"
    roof["kernel_ms"] = ms
    roof["algorithmic_bytes"] = nbytes

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        Kc, Vc = K.cpu(), V.cpu()
        tf, threads, npairs, el = cpu_decode_sample(w, q.cpu(), kn.cpu(), vn.cpu(), Kc, Vc,
                                                    lens_np, rp_np, ci_np, args.cpu_seconds)
        cpu = {"value": tf, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
               "sample": f"{npairs} random (b, h) decode queries of {w.name} ({el:.1f} s, fp64)"}
    line = {
        "metric": METRIC, "value": whole_job_tflops(flops, world, ms), "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": decode_config(w, tokens.sum(), world),
        "roofline": roof,
        "cpu_baseline": cpu,
        "e2e": {"value": whole_job_tflops(flops, world, e2e_ms), "unit": "TFLOP/s",
                "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                "ms_per_step": e2e_ms},
        "gpu_launches": args.steps,
        "clocks": clock_info,
        "soak": {"steps": soak_steps, "seconds": soak_s},
        "min_ms": min(per_step), "median_ms": statistics.median(per_step),
    }
    print(json.dumps(line), flush=True)


def run_reference_backward(args, w, rank, world):
    """fp64 CPU backward oracle on the host cores, each step a bounded sample of (b, h)."""
    if rank != 0:
        return
    import torch

    from oracle import patterns

    if w.N > ORACLE_BACKWARD_MAX_N:
        print(json.dumps({"impl": "reference", "unavailable":
                          f"the dense fp64 backward oracle holds N x N arrays per (b, h), "
                          f"too large at N = {w.N}"}), flush=True)
        return
    q, k, v = workloads.make_qkv(w)
    g = torch.Generator().manual_seed(w.seed + 77)
    do = torch.randn(q.shape, generator=g).to(torch.bfloat16)
    rp, ci = patterns.csr(w.pattern)
    vals, times, done, threads = [], [], 0, 0
    for i in range(args.steps):
        tf, threads, n, el = cpu_backward_sample(w, q, k, v, do, rp, ci, 2.0, rng_seed=i)
        vals.append(tf)
        times.append(el)
        done += n
    value = statistics.median(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * statistics.mean(times), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": fwd_config(w, len(ci), world, backward=True),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": f"{done} random (b, h) backward passes of {w.name} over {args.steps} steps"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_reference_decode(args, w, rank, world):
    """fp64 CPU decode oracle on the host cores, each step a bounded sample of (b, h)."""
    if rank != 0:
        return
    from oracle import patterns

    q, kn, vn, K, V, lens = workloads.make_decode_inputs(w, device="cpu")
    rp, ci = patterns.csr(w.pattern)
    lens_np = lens.numpy()
    for i in range(args.warmup):
        cpu_decode_sample(w, q, kn, vn, K, V, lens_np, rp, ci, 0.2, rng_seed=1000 + i)
    vals, times, done, threads = [], [], 0, 0
    for i in range(args.steps):
        tf, threads, n, el = cpu_decode_sample(w, q, kn, vn, K, V, lens_np, rp, ci, 2.0, rng_seed=i)
        vals.append(tf)
        times.append(el)
        done += n
    value = statistics.median(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * statistics.mean(times), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": decode_config(w, decode_tokens(w, lens_np, rp, ci).sum(), world),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": f"{done} random (b, h) decode queries of {w.name} over {args.steps} steps"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_ours(args, w, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import block_sparse_attention_38_b200 as bsa

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    bsa.library()

    # Inputs: each rank its own replica (seed offset by rank).
    q_h, k_h, v_h = workloads.make_qkv(w, seed=replica_seed(w, rank))
    q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
    O = torch.empty_like(q)
    L = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream(dev)
    fws = torch.empty(bsa.forward_workspace_bytes(w.d), dtype=torch.uint8, device=dev)
    topk = w.pattern.kind == workloads.TOPK
    if topk:
        # The step chooses the pattern on the device from Q and K, then runs
        # the forward on it with the batch folded into the heads.
        fold = (1, w.B * w.H, w.N, w.d)
        ws = torch.empty(bsa.library().bsa_topk_workspace_bytes(w.B * w.H, w.N, w.d, w.block_size) // 8,
                         dtype=torch.float64, device=dev)
        rp, ci = bsa.topk_pattern(q, k, w.block_size, w.pattern.top_k, w.causal, workspace=ws)
        rp_np, ci_np = rp.cpu().numpy(), ci.cpu().numpy()

        def step(mid=None):
            rp_s, ci_s = bsa.topk_pattern(q, k, w.block_size, w.pattern.top_k, w.causal,
                                          workspace=ws)
            if mid is not None:
                mid.record(stream)
            bsa.forward(q.view(fold), k.view(fold), v.view(fold), rp_s, ci_s, w.block_size,
                        w.scale, w.causal, out=O.view(fold), lse=L.view(fold[:3]), workspace=fws)
        launches_per_step = 3  # block means, selection, forward
    else:
        rp_np, ci_np = bsa.build_pattern_from(w.pattern)
        rp = torch.from_numpy(rp_np).to(dev)
        ci = torch.from_numpy(ci_np).to(dev)

        def step(mid=None):
            if mid is not None:
                mid.record(stream)
            bsa.forward(q, k, v, rp, ci, w.block_size, w.scale, w.causal, out=O, lse=L,
                        workspace=fws)
        launches_per_step = 1
    nnz = int(len(ci_np))
    flops = useful_flops(w, nnz)

    for _ in range(args.warmup):
        flush()
        step()
    torch.cuda.synchronize()
    bsa.device_status(clear=True)

    visible = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    ids = [x.strip() for x in visible.split(",") if x.strip()]
    clocks = ClockSampler(ids[local_rank] if local_rank < len(ids) else str(local_rank))
    if rank == 0:
        clocks.start()
    region0 = time.time()
    soak_steps, soak_s = soak(step, flush, args.soak_seconds)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    mids = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush()
        starts[i].record(stream)
        step(mids[i])
        ends[i].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clock_info = clocks.stop((region0, time.time())) if rank == 0 else None
    per_step = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = float(sum(per_step))
    # the forward kernel alone (for a top-k step, after the selection kernels)
    fwd_ms_total = float(sum(m.elapsed_time(e) for m, e in zip(mids, ends)))
    status = bsa.device_status(clear=True)
    if status:
        raise RuntimeError(f"kernel reported device status {status:#x}")

    # End to end through the public API: pinned host inputs -> device, forward,
    # O and LSE back to pinned host memory, every step inside the timed region.
    # The step is pipelined over contiguous chunks of the inputs (whole batch
    # entries, or ranges of heads when B == 1): chunk i is copied in on one
    # stream while the forward of chunk i-1 runs on a second and the result of
    # chunk i-2 is copied out on a third.  Every byte still crosses the bus
    # within the step.
    qp, kp, vp = (t.pin_memory() for t in (q_h, k_h, v_h))
    rpp = torch.from_numpy(rp_np).pin_memory()
    cip = torch.from_numpy(ci_np).pin_memory()
    Oh = torch.empty(q_h.shape, dtype=torch.bfloat16).pin_memory()
    Lh = torch.empty((w.B, w.H, w.N), dtype=torch.float32).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in ((qp, kp, vp) if topk else (qp, kp, vp, rpp, cip)))
    d2h = Oh.numel() * Oh.element_size() + Lh.numel() * Lh.element_size()
    qd, kd, vd = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    rpd, cid = torch.empty_like(rp), torch.empty_like(ci)
    chunks = e2e_chunks(w)
    s_in, s_fw, s_out = (torch.cuda.Stream(dev) for _ in range(3))

    def e2e_step_topk():
        # host inputs in, pattern chosen on the device, forward, result out
        with torch.cuda.stream(stream):
            for dst, src in ((qd, qp), (kd, kp), (vd, vp)):
                dst.copy_(src, non_blocking=True)
            rp_s, ci_s = bsa.topk_pattern(qd, kd, w.block_size, w.pattern.top_k, w.causal,
                                          workspace=ws)
            bsa.forward(qd.view(fold), kd.view(fold), vd.view(fold), rp_s, ci_s, w.block_size,
                        w.scale, w.causal, out=O.view(fold), lse=L.view(fold[:3]), workspace=fws)
            Oh.copy_(O, non_blocking=True)
            Lh.copy_(L, non_blocking=True)

    def e2e_step():
        if topk:
            return e2e_step_topk()
        s_in.wait_stream(stream)
        with torch.cuda.stream(s_in):
            rpd.copy_(rpp, non_blocking=True)
            cid.copy_(cip, non_blocking=True)
        for sl, h0, h1 in chunks:
            with torch.cuda.stream(s_in):
                for dst, src in ((qd, qp), (kd, kp), (vd, vp)):
                    dst[sl].copy_(src[sl], non_blocking=True)
                ev_in = torch.cuda.Event()
                ev_in.record(s_in)
            s_fw.wait_event(ev_in)
            with torch.cuda.stream(s_fw):
                bsa.forward(qd[sl], kd[sl], vd[sl], rpd[h0 * w.M:h1 * w.M + 1], cid, w.block_size,
                            w.scale, w.causal, out=O[sl], lse=L[sl], workspace=fws)
                ev_fw = torch.cuda.Event()
                ev_fw.record(s_fw)
            s_out.wait_event(ev_fw)
            with torch.cuda.stream(s_out):
                Oh[sl].copy_(O[sl], non_blocking=True)
                Lh[sl].copy_(L[sl], non_blocking=True)
        stream.wait_stream(s_out)

    for _ in range(max(1, args.warmup)):
        e2e_step()
    torch.cuda.synchronize()
    e_steps = max(3, min(args.steps, 20))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e_steps
    status = bsa.device_status(clear=True)
    if status:
        raise RuntimeError(f"kernel reported device status {status:#x} in the end-to-end leg")
    ref_o = O.cpu()
    if not torch.equal(Oh, ref_o):
        raise RuntimeError("end-to-end result differs from the device result")

    total_ms, e2e_ms, fwd_ms_total = max_over_ranks([total_ms, e2e_ms, fwd_ms_total], world,
                                                    device=dev)
    if rank != 0:
        return

    ms = total_ms / args.steps
    fwd_ms = fwd_ms_total / args.steps
    value = whole_job_tflops(flops, world, ms)
    e2e_value = whole_job_tflops(flops, world, e2e_ms)
    peaks, peak_src = load_peaks()
    peak_tc = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    peak_hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    t_tc = flops / (peak_tc * 1e12)
    t_hbm = compulsory_bytes(w) / (peak_hbm * 1e9)
    if t_tc >= t_hbm:
        roof = {"bound": "tensor", "achieved": flops / (fwd_ms * 1e-3) / 1e12, "peak": peak_tc,
                "unit": "TFLOP/s"}
    else:
        roof = {"bound": "hbm", "achieved": compulsory_bytes(w) / (fwd_ms * 1e-3) / 1e9,
                "peak": peak_hbm, "unit": "GB/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    if roof["bound"] == "tensor":
        # against the GEMM rate held for seconds under the power cap (the
        # timed steps follow a soak of the same steps)
        sustained = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
        roof["frac_of_sustained_peak"] = roof["achieved"] / sustained
    tr = NCU_TRAFFIC.get(w.name)
    roof["traffic"] = tr[0] if tr and tr[1] == kernel_hash() else None
    roof["peak_source"] = f"{peak_src} (MEASURED_PEAKS.json burst)" if peak_src == "measured" else "fallback"
    roof["roofline_frac_max_of_tc_hbm"] = max(t_tc, t_hbm) / (fwd_ms * 1e-3)
    roof["kernel"] = "bsa::pp::fwd_kernel"
    roof["kernel_ms"] = fwd_ms

    # CPU baseline: the oracle, as it stands, on a bounded sample of rows.
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        wo, qo, ko, vo, orp, oci = oracle_problem(w, q_h, k_h, v_h)
        tf, threads, nrows, el = cpu_oracle_sample(wo, qo, ko, vo, orp, oci, args.cpu_seconds)
        cpu = {"value": tf, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
               "sample": f"{nrows} random query rows of {w.name} ({el:.1f} s, fp64)",
               "nproc": os.cpu_count(), "cpu_model": cpu_model()}
        if w.N <= 4096 and w.pattern.kind != workloads.TOPK:
            # the same oracle on one thread, a shorter sample
            tf1, _, n1, el1 = cpu_oracle_sample(wo, qo, ko, vo, orp, oci,
                                                min(3.0, args.cpu_seconds), nthreads=1)
            cpu["one_thread"] = {"value": tf1, "sample": f"{n1} random query rows ({el1:.1f} s)"}

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": fwd_config(w, nnz, world),
        "roofline": roof,
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": int(h2d),
                "d2h_bytes_per_step": int(d2h), "ms_per_step": e2e_ms},
        "gpu_launches": args.steps * launches_per_step,
        "clocks": clock_info,
        "soak": {"steps": soak_steps, "seconds": soak_s},
        "min_ms": min(per_step), "median_ms": statistics.median(per_step),
    }
    if w.causal:
        # the flops of the (query, key) pairs the causal mask keeps
        line["causal_exact_tflops"] = whole_job_tflops(causal_exact_flops(w, rp_np, ci_np),
                                                       world, ms)
    if topk:
        # the selection (block means + top-k select kernels) ahead of the forward
        line["selection_ms"] = ms - fwd_ms
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    choices=list(workloads.WORKLOADS) + list(workloads.DECODE_WORKLOADS))
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--soak-seconds", type=float, default=1.2,
                    help="untimed steps run back to back right before the timed ones, so that "
                         "the clock samples cover a loaded GPU")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--backward", action="store_true",
                    help="time the backward pass (dQ, dK, dV) instead of the forward")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    decode = args.workload in workloads.DECODE_WORKLOADS
    w = (workloads.DECODE_WORKLOADS if decode else workloads.WORKLOADS)[args.workload]
    run = run_decode if decode else (run_backward if args.backward else run_ours)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        ref = run_reference_decode if decode else (
            run_reference_backward if args.backward else run_reference)
        ref(args, w, rank, world)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist

        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        try:
            run(args, w, rank, world, local_rank)
        finally:
            dist.destroy_process_group()
    else:
        run(args, w, 0, 1, 0)


if __name__ == "__main__":
    main()
