"""Benchmark of librankcoll: effective GB/s of the simulated-rank collectives.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One STEP is one pass of the whole hot path over one batch of synthetic input:
8 simulated ranks x 2,097,152 fp32 elements (8 MiB) per rank ~N(0, 1e-2),
seed 1 (the ring / one-shot all-reduce workload), through
  all_reduce (one-shot), reduce_scatter (fp32 -> bf16, scale 1/8),
  all_gather (the bf16 shards), reduce (root 0), broadcast (root 0, in place),
  ring all_reduce (literal 14 steps), hierarchical all_reduce (2 x 4, fused).
Timing: the whole step is captured once into a CUDA graph and the K steps
replay it between one pair of CUDA events on the launching stream.  A split
per collective replays one graph per collective K more times, with an event
between consecutive collectives (`--graph per_op` makes that the headline).
Every collective of the step has its own inputs and outputs,
so between two reads of an op's inputs the other six move more than 500 MiB
(over 4x the 126 MB L2): the inputs come from HBM ("inputs larger than L2").
A second view times every collective alone after an L2 flush outside its
events (a 512 MiB write, then a 256 MiB read of another buffer, so L2 holds no
dirty lines of the flush's to write back).  CUDA event timestamps here tick
at about 2 us, so per-collective figures are means over many steps.

Effective GB/s = minimum bytes read + written / device time (decimal GB):
  all_reduce p*n*s_in + p*n*s_out; reduce_scatter p*n*s_in + n*s_out;
  all_gather n*s + p*n*s; reduce p*n*s_in + n*s_out; broadcast n*s + (p-1)*n*s;
  ring and hierarchical are charged the all_reduce minimum.
`value` is the step's total minimum bytes over the step's total device time.

`--impl reference` times the CPU oracle (single thread, host cores) on a
bounded sample of the same workload and prints the same metric.
With torchrun (N > 1) every rank runs its own replica of the step on its own
GPU (no data-path collective: the simulated ranks never leave one GPU); the
time is the max over ranks and `value` the sum of all replicas' bytes / that
time ("scaling": "weak").
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "effective GB/s and % of HBM peak for 8-rank all_reduce / reduce_scatter"
UNIT = "GB/s"
P, N = 8, 2097152
SEED = 1
SIGMA = 1e-2
# B200 HBM bandwidth as the pages quote it ("分布式训练/推理", section "从单卡到多卡：
# 瓶颈从 HBM 扩展到互联"): context beside the measured copy peak, not the roofline.
PAGES_HBM_GBS = 8000.0
FLUSH_BYTES = 512 << 20      # written, then...
CLEAN_BYTES = 256 << 20      # ...a separate buffer read, so L2 is left holding clean lines
WORKLOAD = ("ring/one-shot all_reduce workload: p=8 simulated ranks x 2,097,152 fp32 "
            "(8 MiB) per rank ~N(0,1e-2) seed 1; step = all_reduce, reduce_scatter fp32->bf16 "
            "x1/8, all_gather bf16, reduce, broadcast, ring all_reduce (literal), "
            "hierarchical all_reduce 2x4 (fused)")

# DRAM traffic per launch measured by ncu (dram__bytes_read.sum +
# dram__bytes_write.sum) for the kernel named, with the hash of the kernel's
# source file and the shared device helpers (common.cuh) when it was measured;
# a changed source reports null.  Captured on the launch after a call of the
# same collective on another buffer set, with ncu's cache control off, so the
# previous call's dirty outputs are written back inside the captured launch
# (bench.py --ncu-case OP --ncu-workload step).
NCU_TRAFFIC = {
    "ring_all_reduce": {"bytes": 67123200 + 63719168, "src": "f0a73279135321c7"},
    "all_reduce": {"bytes": 67107584 + 66091520, "src": "3194ac134632a10d"},
    "reduce_scatter": {"bytes": 67108864 + 5088256, "src": "3194ac134632a10d"},
    "all_gather": {"bytes": 4180224 + 28257536, "src": "02a6666765c86fcd"},
    "reduce": {"bytes": 67109888 + 8442880, "src": "3194ac134632a10d"},
    "broadcast": {"bytes": 8389120 + 54693888, "src": "02a6666765c86fcd"},
    "hier_all_reduce": {"bytes": 67109632 + 65382400, "src": "5eeac14585157d2b"},
}

# Each collective's duration inside the timed step graph, from one ncu
# launch list of the timed replays (NVTX range rc_timed_step; cache control
# off, so every kernel meets the L2 state the previous one left; mean of 3
# steps, us) and its DRAM bytes there.  ncu serialises the launches, so the
# absolute times run about 10% long; the bench reports each collective's
# share of this list times the live step time.
NCU_IN_STEP = {
    "all_reduce": {"us": 25.46, "dram": 67.1e6 + 65.8e6, "src": "3194ac134632a10d"},
    "reduce_scatter": {"us": 17.40, "dram": 67.1e6 + 13.8e6, "src": "3194ac134632a10d"},
    "all_gather": {"us": 9.80, "dram": 4.2e6 + 23.3e6, "src": "02a6666765c86fcd"},
    "reduce": {"us": 17.51, "dram": 67.1e6 + 14.1e6, "src": "3194ac134632a10d"},
    "broadcast": {"us": 12.83, "dram": 8.4e6 + 46.9e6, "src": "02a6666765c86fcd"},
    "ring_all_reduce": {"us": 26.09, "dram": 64.7e6 + 70.4e6, "src": "f0a73279135321c7"},
    "hier_all_reduce": {"us": 25.47, "dram": 67.1e6 + 64.7e6, "src": "5eeac14585157d2b"},
}


def busbw_all_reduce(size_bytes: float, p: int, t: float) -> float:
    """Bus bandwidth 2 s (p-1) / (p t) in bytes/s: "分布式训练/推理", section
    "带宽怎么核算：看 duration 之前先看 bytes" (s = bytes of one rank's tensor)."""
    return 2.0 * size_bytes * (p - 1) / (p * t)


def busbw_reduce_scatter(input_bytes: float, p: int, t: float) -> float:
    """Bus bandwidth s_input (p-1) / (p t), same section; s_input is the
    world_size x k input of one rank."""
    return input_bytes * (p - 1) / (p * t)


def ring_schedule_bytes(p: int, n: int, s: int) -> int:
    """Bytes the ring's schedule moves when every message goes through device
    memory: reduce-scatter 3(p-1) n s (each step reads the message and the
    receiver's chunk and writes the partial, p chunks of n/p), all-gather
    2(p-1) n s -- (5p-5) n s, 35 n s at p = 8 ("LLM Parallelism 基础", section
    "Ring AllReduce"; the minimum is 2 p n s)."""
    return (5 * p - 5) * n * s


def ring_model_seconds(size_bytes: float, p: int, bw: float) -> float:
    """Ring all-reduce time model 2 (N-1)/N * S/W ("分布式训练/推理", section
    "Ring all-reduce 的带宽账")."""
    return 2.0 * (p - 1) / p * size_bytes / bw


# minimum bytes of each collective in the step (p ranks, n elements per rank)
def step_ops(p=P, n=N):
    s_in, s_bf = 4, 2
    m = n // p
    return [
        ("all_reduce", p * n * s_in + p * n * s_in),
        ("reduce_scatter", p * n * s_in + n * s_bf),
        ("all_gather", n * s_bf + p * n * s_bf),
        ("reduce", p * n * s_in + n * s_in),
        ("broadcast", n * s_in + (p - 1) * n * s_in),
        ("ring_all_reduce", p * n * s_in + p * n * s_in),
        ("hier_all_reduce", p * n * s_in + p * n * s_in),
    ], m


KERNEL_OF = {
    "all_reduce": ("rc_reduce_front_kernel", "reduce.cu"),
    "reduce_scatter": ("rc_reduce_front_kernel", "reduce.cu"),
    "all_gather": ("rc_fanout_reg_kernel", "fanout.cu"),
    "reduce": ("rc_reduce_front_kernel", "reduce.cu"),
    "broadcast": ("rc_fanout_reg_kernel", "fanout.cu"),
    "ring_all_reduce": ("rc_ring_link_kernel", "ring.cu"),
    "hier_all_reduce": ("rc_hier_front_kernel", "hier.cu"),
}


def _src_hash(fname):
    """Hash of a kernel's source file plus the shared device helpers."""
    csrc = os.path.join(ROOT, "collective_rc_all_b200", "csrc")
    data = b""
    for f in (fname, "common.cuh"):
        with open(os.path.join(csrc, f), "rb") as fh:
            data += fh.read()
    return hashlib.sha256(data).hexdigest()[:16]


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"rc_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        sm, smax, reasons, samples = [], [], set(), 0
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                samples += 1
                try:
                    sm.append(float(parts[1]))
                    smax.append(float(parts[2]))
                except ValueError:
                    pass
                for nm, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(nm)
        try:
            os.remove(self.path)
        except OSError:
            pass
        return {"sm_mhz": float(np.median(sm)) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": samples}


# ------------------------------------------------------------------ multi-rank plumbing
def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def reduce_over_ranks(local_seconds: float, local_bytes: float, world: int, device=None):
    """Max of the ranks' device times and sum of their bytes (plumbing only:
    the timing scalars, not data).  Works with gloo (CPU) and nccl (GPU)."""
    if world <= 1:
        return local_seconds, local_bytes
    import torch
    import torch.distributed as dist
    t = torch.tensor([local_seconds], dtype=torch.float64, device=device)
    b = torch.tensor([local_bytes], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(b, op=dist.ReduceOp.SUM)
    return float(t.item()), float(b.item())


# ------------------------------------------------------------------ CPU oracle arm
def cpu_oracle_step_rate(budget_s: float = 12.0, n_sample: int = N // 8):
    """The oracle, as it stands (one thread), on a bounded sample of the step:
    the same seven collectives on n_sample elements per rank, repeated until
    budget_s has passed.  Returns (GB/s, reps, seconds, n_sample)."""
    import oracle
    import rc_inputs
    xs = rc_inputs.normal(P, n_sample, seed=SEED, sigma=SIGMA)
    ops, m = step_ops(P, n_sample)
    step_bytes = sum(b for _, b in ops)
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle.all_reduce(xs)
        rs = oracle.reduce_scatter(xs, "f32", "bf16", "sum", 1.0 / P)
        oracle.all_gather(rs, "bf16")
        oracle.reduce(xs, 0)
        oracle.broadcast(xs[0], P, 0)
        oracle.ring_all_reduce(xs)
        oracle.hier_all_reduce(xs, 4)
        reps += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    return step_bytes * reps / el / 1e9, reps, el, n_sample


def host_cpu():
    """The host's logical CPU count and model name (from /proc/cpuinfo)."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.lower().startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"host_cpu_count": os.cpu_count(), "host_cpu_model": model}


def run_reference(args):
    rank, _, world = dist_env()
    if rank != 0:
        return 0
    ops, _ = step_ops()
    per_step_budget = max(0.2, args.ref_seconds / max(1, args.steps + args.warmup))
    # warm-up steps (untimed), then K timed steps, each a bounded sample
    for _ in range(args.warmup):
        cpu_oracle_step_rate(budget_s=0.5 * per_step_budget)
    rates, total_s, total_reps = [], 0.0, 0
    for _ in range(args.steps):
        gbs, reps, el, ns = cpu_oracle_step_rate(budget_s=per_step_budget)
        rates.append(gbs)
        total_s += el
        total_reps += reps
    value = float(np.mean(rates))
    sample = (f"{total_reps} passes of the seven-collective step on {ns} elements per rank "
              f"(p=8, 1/8 of the workload), one thread, {total_s:.1f} s")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * total_s / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": WORKLOAD, "p": P, "n_per_rank": N, "l2": "n/a (host)"},
        "cpu_baseline": {"value": round(value, 3), "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": sample, **host_cpu()},
        "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ GPU arm
def run_ours(args):
    import torch
    import collective_rc_all_b200 as rc
    import rc_inputs

    rank, local_rank, world = dist_env()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    stream = torch.cuda.current_stream()
    ops, m = step_ops()
    step_bytes = sum(b for _, b in ops)

    # inputs: each replica draws its own batch (seed + rank); every collective
    # of the step gets its own copy of the inputs and its own outputs, so in
    # the back-to-back timing the inputs an op reads were last touched a whole
    # step (> 500 MiB of traffic, > 4x L2) earlier and come from HBM
    xs = rc_inputs.normal(P, N, seed=SEED + rank, sigma=SIGMA)
    send = [torch.from_numpy(x).to(dev) for x in xs]
    own = lambda: [t.clone() for t in send]
    f32 = lambda k: [torch.empty(N, dtype=torch.float32, device=dev) for _ in range(k)]
    bf16 = lambda k, n: [torch.empty(n, dtype=torch.bfloat16, device=dev) for _ in range(k)]
    def buffer_set():
        """Inputs (copies of the step's inputs) and outputs of every collective."""
        B = {"s_ar": own(), "s_rs": own(), "s_red": own(), "s_bc": own(), "s_ring": own(), "s_hier": own(),
             "y_ar": f32(P), "y_ring": f32(P), "y_hier": f32(P),
             "y_rs": bf16(P, m), "ag_in": bf16(P, m), "y_ag": bf16(P, N),
             "y_red": torch.empty(N, dtype=torch.float32, device=dev)}
        B["y_bc"] = [B["s_bc"][0]] + f32(P - 1)          # root 0 in place
        rc.rc_reduce_scatter(send, B["ag_in"], out_dtype="bf16", scale=1.0 / P)  # the all-gather's shards
        return B

    def calls_of(B):
        return {
            "all_reduce": lambda: rc.rc_all_reduce(B["s_ar"], B["y_ar"]),
            "reduce_scatter": lambda: rc.rc_reduce_scatter(B["s_rs"], B["y_rs"], out_dtype="bf16", scale=1.0 / P),
            "all_gather": lambda: rc.rc_all_gather(B["ag_in"], B["y_ag"]),
            "reduce": lambda: rc.rc_reduce(B["s_red"], B["y_red"], root=0),
            "broadcast": lambda: rc.rc_broadcast(B["s_bc"][0], B["y_bc"], root=0),
            "ring_all_reduce": lambda: rc.rc_ring_all_reduce(B["s_ring"], B["y_ring"], variant="literal"),
            "hier_all_reduce": lambda: rc.rc_hier_all_reduce(B["s_hier"], B["y_hier"], 4, variant="fused"),
        }

    B0 = buffer_set()
    y_ar, y_rs, y_ag, y_red, y_bc, y_ring, y_hier = (B0[k] for k in ("y_ar", "y_rs", "y_ag", "y_red", "y_bc",
                                                                     "y_ring", "y_hier"))
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    clean = torch.ones(CLEAN_BYTES // 4, dtype=torch.float32, device=dev)
    sink = torch.empty((), dtype=torch.float32, device=dev)

    def l2_flush():
        flush.zero_()
        torch.sum(clean, dim=0, out=sink)

    calls = calls_of(B0)
    names = [nm for nm, _ in ops]
    K, W = args.steps, args.warmup
    # back-to-back timing: every collective is captured once into its own CUDA
    # graph (one host launch per collective instead of the binding's argument
    # marshalling and checks, which take longer than a collective on the GPU),
    # and the whole step once more into one graph.  The headline replays the
    # step graph K times between one pair of events.  The split per
    # collective replays the per-collective graphs K times with an event
    # before every collective and one after the last.
    for nm in names:
        calls[nm]()  # first calls outside capture (one-time set-up)
    torch.cuda.synchronize()
    graphs, launches_per_graph = {}, {}
    for nm in names:
        g = torch.cuda.CUDAGraph()
        l0 = rc.rc_launch_count()
        with torch.cuda.graph(g, capture_error_mode="thread_local"):
            calls[nm]()
        launches_per_graph[nm] = rc.rc_launch_count() - l0
        graphs[nm] = g
    step_graph = None
    if args.graph == "step":
        step_graph = torch.cuda.CUDAGraph()
        l0 = rc.rc_launch_count()
        with torch.cuda.graph(step_graph, capture_error_mode="thread_local"):
            for nm in names:
                calls[nm]()
        launches_per_step = rc.rc_launch_count() - l0
    else:
        launches_per_step = sum(launches_per_graph.values())
    torch.cuda.synchronize()
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(K * len(names) + 1)]

    def one_step(k=None):
        for j, nm in enumerate(names):
            if k is not None:
                evs[k * len(names) + j].record(stream)
            graphs[nm].replay()

    # copy roofline of this library's own copy kernel (same run), 1 GiB
    copy_gbs = None
    copy_same_us = None
    if not args.no_copy_peak:
        cp_a = torch.empty(1 << 30, dtype=torch.uint8, device=dev)
        cp_b = torch.empty(1 << 30, dtype=torch.uint8, device=dev)
        for _ in range(3):
            rc.rc_copy(cp_a, cp_b)
        cps = []
        for _ in range(5):
            l2_flush()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            rc.rc_copy(cp_a, cp_b)
            b.record(stream)
            b.synchronize()
            cps.append(a.elapsed_time(b) * 1e-3)
        copy_gbs = 2 * (1 << 30) / min(cps) / 1e9
        del cp_a, cp_b
        # the same copy kernel moving exactly an all-reduce's algorithmic
        # bytes (64 MiB read + 64 MiB written), back to back on 4 separate
        # buffer pairs in one graph: the size-matched ceiling the 8 MiB-per-
        # rank collectives' back-to-back times compare with
        half = P * N * 4
        pairs = [(torch.empty(half, dtype=torch.uint8, device=dev),
                  torch.empty(half, dtype=torch.uint8, device=dev)) for _ in range(4)]
        for a_, b_ in pairs:
            rc.rc_copy(a_, b_)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, capture_error_mode="thread_local"):
            for a_, b_ in pairs:
                rc.rc_copy(a_, b_)
        for _ in range(3):
            g.replay()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(K):
            g.replay()
        b.record(stream)
        b.synchronize()
        copy_same_us = a.elapsed_time(b) * 1e-3 / (4 * K) * 1e6
        del g, pairs

    # the clock sampler starts before the warm-up, so the GPU is busy (not
    # idling at low clocks) when the timed region begins
    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)
    for _ in range(W):
        if step_graph is not None:
            step_graph.replay()
        else:
            one_step()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    if step_graph is not None:
        ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        # the NVTX range names the timed replays for a profiler's launch filter
        torch.cuda.nvtx.range_push("rc_timed_step")
        ea.record(stream)
        for _ in range(K):
            step_graph.replay()
        eb.record(stream)
        torch.cuda.nvtx.range_pop()
        torch.cuda.synchronize()
        step_s = ea.elapsed_time(eb) * 1e-3
        if world > 1:
            torch.distributed.barrier()
    # the split per collective (the headline too when --graph per_op)
    for k in range(K):
        one_step(k)
    evs[-1].record(stream)
    torch.cuda.synchronize()
    if step_graph is None:
        step_s = evs[0].elapsed_time(evs[-1]) * 1e-3
    # this library's kernels inside the headline's timed region: the kernels
    # the captured graph(s) hold, times the replays
    launches = K * launches_per_step
    # each collective back to back with itself: one graph of 4 calls of it
    # on 4 separate input/output sets (4 x its footprint > L2), replayed K
    # times -- its throughput as a stream of calls, every write-back paid
    rep_sets = [B0] + [buffer_set() for _ in range(3)]
    torch.cuda.synchronize()
    rep_s = {}
    for nm in names:
        fs = [calls_of(Bx)[nm] for Bx in rep_sets]
        for f in fs:
            f()   # one-time set-up outside capture
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, capture_error_mode="thread_local"):
            for f in fs:
                f()
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(K):
            g.replay()
        b.record(stream)
        b.synchronize()
        rep_s[nm] = a.elapsed_time(b) * 1e-3 / (K * len(fs))
        del g
    # in sequence: each collective after its predecessor in the step (the
    # last one precedes the first in a sequence of steps), live: one graph of
    # [X, Y] on each of the 4 sets, replayed K times, minus the repeated view
    # of X alone (the same 4 sets) -- what Y adds when it follows X
    seq_s = {}
    for i, y in enumerate(names):
        x = names[i - 1]
        fs = [f for Bx in rep_sets for f in (calls_of(Bx)[x], calls_of(Bx)[y])]
        for f in fs:
            f()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, capture_error_mode="thread_local"):
            for f in fs:
                f()
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(K):
            g.replay()
        b.record(stream)
        b.synchronize()
        seq_s[y] = (x, a.elapsed_time(b) * 1e-3 / (K * len(rep_sets)) - rep_s[x])
        del g
    del rep_sets
    time.sleep(0.3)
    clk = clocks.stop()
    if world > 1:
        torch.distributed.barrier()
    rc.rc_stream_status()

    # second view: every collective alone, L2 flushed (untimed) before it
    iso_k = min(K, 30)
    iso = {nm: [] for nm in names}
    for _ in range(iso_k):
        for nm in names:
            l2_flush()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            calls[nm]()
            b.record(stream)
            b.synchronize()
            iso[nm].append(a.elapsed_time(b) * 1e-3)
    rc.rc_stream_status()

    split_s = evs[0].elapsed_time(evs[-1]) * 1e-3
    per_op_s = {nm: 0.0 for nm in names}
    per_op_all = {nm: [] for nm in names}
    for k in range(K):
        for j, nm in enumerate(names):
            i = k * len(names) + j
            dt_ = evs[i].elapsed_time(evs[i + 1]) * 1e-3
            per_op_s[nm] += dt_
            per_op_all[nm].append(dt_)
    per_op_dist = {nm: sorted(v) for nm, v in per_op_all.items()}
    local_s = step_s
    tot_s, tot_bytes = reduce_over_ranks(local_s, step_bytes * K, world, device=dev)

    # ---- end to end through the same calls with host buffers (pinned)
    host_in = [torch.from_numpy(x).pin_memory() for x in xs]
    outs = [y_ar[0], y_rs, y_ag[0], y_red, y_bc[1], y_ring[0], y_hier[0]]
    flat_outs = [t for o in outs for t in (o if isinstance(o, list) else [o])]
    host_out = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in flat_outs]
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = sum(t.numel() * t.element_size() for t in host_out)
    e2e_k = max(3, K // 4)
    if args.no_e2e:
        e2e_k = 0

    # end to end: every step copies one set of inputs in from pinned host
    # memory, runs every collective of the step on it through the Python API,
    # and copies one copy of every result back.  PCIe is full duplex, so the
    # steps are pipelined: inputs are double-buffered on the device, the
    # host->device copy of step k+1 runs on its own stream while the
    # device->host copy of step k runs on another; step k+1's collectives wait
    # for its inputs and for the read-back of step k's results (which they
    # overwrite).
    send2 = [torch.empty_like(t) for t in send]
    bufs = [send, send2]

    def e2e_calls(buf):
        return {
            "all_reduce": lambda: rc.rc_all_reduce(buf, y_ar),
            "reduce_scatter": lambda: rc.rc_reduce_scatter(buf, y_rs, out_dtype="bf16", scale=1.0 / P),
            "all_gather": lambda: rc.rc_all_gather(y_rs, y_ag),
            "reduce": lambda: rc.rc_reduce(buf, y_red, root=0),
            "broadcast": lambda: rc.rc_broadcast(buf[0], [buf[0]] + y_bc[1:], root=0),
            "ring_all_reduce": lambda: rc.rc_ring_all_reduce(buf, y_ring, variant="literal"),
            "hier_all_reduce": lambda: rc.rc_hier_all_reduce(buf, y_hier, 4, variant="fused"),
        }

    calls_of = [e2e_calls(bufs[0]), e2e_calls(bufs[1])]
    h2d_s, d2h_s = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event(), torch.cuda.Event()]     # inputs of buffer i landed
    ev_used = [torch.cuda.Event(), torch.cuda.Event()]   # collectives done with buffer i
    ev_out = torch.cuda.Event()                          # results of the last step read back
    ev_used[0].record(stream)
    ev_used[1].record(stream)
    ev_out.record(stream)

    def e2e_step(k):
        i = k % 2
        with torch.cuda.stream(h2d_s):
            h2d_s.wait_event(ev_used[i])   # the step two back has finished reading buffer i
            for d, h in zip(bufs[i], host_in):
                d.copy_(h, non_blocking=True)
            ev_in[i].record(h2d_s)
        stream.wait_event(ev_in[i])
        stream.wait_event(ev_out)          # the previous results have been read back
        for nm in names:
            calls_of[i][nm]()
        ev_used[i].record(stream)
        with torch.cuda.stream(d2h_s):
            d2h_s.wait_event(ev_used[i])
            for h, d in zip(host_out, flat_outs):
                h.copy_(d, non_blocking=True)
            ev_out.record(d2h_s)

    e2e = None
    if e2e_k:
        for k in range(2):
            e2e_step(k)
        torch.cuda.synchronize()
        ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ea.record(stream)
        h2d_s.wait_event(ea)   # no copy of the timed steps starts before the clock
        d2h_s.wait_event(ea)
        for k in range(e2e_k):
            e2e_step(k)
        stream.wait_event(ev_out)
        eb.record(stream)
        eb.synchronize()
        e2e_s, e2e_bytes = reduce_over_ranks(ea.elapsed_time(eb) * 1e-3, step_bytes * e2e_k, world,
                                             device=dev)
        # the PCIe ceiling of this pipeline: one step's host->device copies and
        # one step's device->host copies running concurrently, as in the
        # pipeline, without the collectives
        torch.cuda.synchronize()
        pa, pb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        pa.record(stream)
        h2d_s.wait_event(pa)
        d2h_s.wait_event(pa)
        for _ in range(e2e_k):
            with torch.cuda.stream(h2d_s):
                for d, h in zip(bufs[0], host_in):
                    d.copy_(h, non_blocking=True)
            with torch.cuda.stream(d2h_s):
                for h, d in zip(host_out, flat_outs):
                    h.copy_(d, non_blocking=True)
        stream.wait_stream(h2d_s)
        stream.wait_stream(d2h_s)
        pb.record(stream)
        pb.synchronize()
        copies_s = pa.elapsed_time(pb) * 1e-3 / e2e_k
        e2e = {"value": round(e2e_bytes / e2e_s / 1e9, 2), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "pipelined": "H2D of step k+1 on one stream overlaps D2H of step k on another "
                            "(double-buffered device inputs)",
               "copies_only_ms_per_step": round(copies_s * 1e3, 4),
               "pcie_ceiling_gbs": round(step_bytes / copies_s / 1e9, 2)}

    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    peak, peak_kind = measured_peaks()
    value = tot_bytes / tot_s / 1e9
    per_op = {}
    for nm, b in ops:
        t = per_op_s[nm] / K
        dist = per_op_dist[nm]
        ti = float(np.mean(iso[nm]))
        trf = NCU_TRAFFIC.get(nm)
        per_op_traffic = trf["bytes"] if trf and trf["src"] == _src_hash(KERNEL_OF[nm][1]) else None
        per_op[nm] = {"us": round(t * 1e6, 2), "us_median": round(dist[len(dist) // 2] * 1e6, 2),
                      "ncu_dram_bytes": per_op_traffic, "algorithmic_bytes": b,
                      "gbs": round(b / t / 1e9, 1),
                      "frac_of_measured_hbm": round(b / t / 1e9 / peak, 4),
                      "frac_of_copy_kernel": round(b / t / 1e9 / copy_gbs, 4) if copy_gbs else None,
                      "repeated_us": round(rep_s[nm] * 1e6, 2),
                      "in_sequence_after": seq_s[nm][0],
                      "in_sequence_us": round(seq_s[nm][1] * 1e6, 2),
                      "in_sequence_frac_of_measured_hbm": round(b / seq_s[nm][1] / 1e9 / peak, 4),
                      "repeated_frac_of_measured_hbm": round(b / rep_s[nm] / 1e9 / peak, 4),
                      "repeated_frac_of_pages_8tbs": round(b / rep_s[nm] / 1e9 / PAGES_HBM_GBS, 4),
                      "isolated_us": round(ti * 1e6, 2),
                      "isolated_frac_of_measured_hbm": round(b / ti / 1e9 / peak, 4)}
    # in-step durations: each collective's share of the ncu launch list of the
    # timed step graph, times this run's step time (null once a kernel changed)
    ins = {nm: NCU_IN_STEP.get(nm) for nm in names}
    if all(v is not None and v["src"] == _src_hash(KERNEL_OF[nm][1]) for nm, v in ins.items()):
        tot_ncu = sum(v["us"] for v in ins.values())
        for nm, b in ops:
            t_in = ins[nm]["us"] / tot_ncu * (step_s / K)
            per_op[nm].update({"in_step_us": round(t_in * 1e6, 2),
                               "in_step_frac_of_measured_hbm": round(b / t_in / 1e9 / peak, 4),
                               "in_step_ncu_us": ins[nm]["us"], "in_step_ncu_dram_bytes": int(ins[nm]["dram"])})
    else:
        for nm in names:
            per_op[nm].update({"in_step_us": None, "in_step_frac_of_measured_hbm": None})
    if "all_reduce" in per_op:
        t_ar = per_op_s["all_reduce"] / K
        per_op["all_reduce"]["busbw_gib_s"] = round(busbw_all_reduce(N * 4, P, t_ar) / 2**30, 1)
    if "reduce_scatter" in per_op:
        t_rs = per_op_s["reduce_scatter"] / K
        per_op["reduce_scatter"]["busbw_gib_s"] = round(busbw_reduce_scatter(N * 4, P, t_rs) / 2**30, 1)
    if "ring_all_reduce" in per_op:
        t_ring = per_op_s["ring_all_reduce"] / K
        sched = ring_schedule_bytes(P, N, 4)
        per_op["ring_all_reduce"].update({
            "ring_model_us_at_measured_hbm": round(ring_model_seconds(N * 4, P, peak * 1e9) * 1e6, 2),
            "schedule_bytes": sched,
            "schedule_gbs": round(sched / t_ring / 1e9, 1),
            "schedule_gbs_repeated": round(sched / rep_s["ring_all_reduce"] / 1e9, 1)})
    dom = max(names, key=lambda nm: per_op_s[nm])
    dom_b = dict(ops)[dom]
    dom_t = per_op_s[dom] / K
    dom_rep = rep_s[dom]
    kname, kfile = KERNEL_OF[dom]
    tr = NCU_TRAFFIC.get(dom)
    traffic = tr["bytes"] if tr and tr.get("src") == _src_hash(kfile) else None

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        gbs, reps, el, ns = cpu_oracle_step_rate(budget_s=args.cpu_seconds)
        cpu = {"value": round(gbs, 3), "unit": UNIT, "cores": 1, "kind": "oracle",
               "sample": f"{reps} passes of the seven-collective step on {ns} elements per rank "
                         f"(p=8, 1/8 of the workload), one thread, {el:.1f} s", **host_cpu()}

    line = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
        "steps": K, "warmup": W, "ms_per_step": round(1e3 * tot_s / K, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "p": P, "n_per_rank": N,
                   "l2": ("inputs larger than L2: each collective of the step has its own inputs and "
                          "outputs, so between two reads of an op's inputs the other ops move > 500 MiB "
                          "(> 4x the 126 MB L2). " + (
                              "value: K replays of one CUDA graph of the whole step between one pair of "
                              "CUDA events; per_op.us: K "
                              "replays of one graph per collective, back to back, an event between "
                              "collectives" if step_graph is not None else
                              "value and per_op.us: K replays of one CUDA graph per collective, back to "
                              "back, an event between collectives") +
                          ". per_op.repeated_*: one graph of 4 calls of the collective on 4 separate "
                          "input/output sets, replayed K times. per_op.isolated_*: each collective alone (plain "
                          "call) after a 512 MiB "
                          "write + 256 MiB read L2 flush outside its events"),
                   "parallelism": f"replicas x{world}"},
        "roofline": {"bound": "hbm", "kernel": kname, "op": dom,
                     "achieved": round(dom_b / dom_rep / 1e9, 1), "peak": peak,
                     "peak_kind": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured" else "fallback",
                     "unit": "GB/s", "frac": round(dom_b / dom_rep / 1e9 / peak, 4),
                     "traffic": traffic, "algorithmic_bytes": dom_b,
                     "launch_us": round(dom_rep * 1e6, 2),
                     "launch_timing": ("average launch duration: CUDA events around K replays of one graph "
                                       "of 4 launches of the kernel on 4 separate input/output sets "
                                       "(4 x its inputs and outputs > L2), inside the clock-sampled region"),
                     "frac_of_pages_8tbs": round(dom_b / dom_rep / 1e9 / PAGES_HBM_GBS, 4),
                     "achieved_split_view": round(dom_b / dom_t / 1e9, 1),
                     "frac_split_view": round(dom_b / dom_t / 1e9 / peak, 4)},
        "split_ms_per_step": round(1e3 * split_s / K, 4),
        "per_op": per_op,
        "copy_kernel_gbs": round(copy_gbs, 1) if copy_gbs else None,
        "copy_134MB_back_to_back": ({"us": round(copy_same_us, 2),
                                     "gbs": round(2 * P * N * 4 / copy_same_us / 1e3, 1),
                                     "what": "this library's copy kernel moving 64 MiB -> 64 MiB (an 8 x 8 MiB "
                                             "all-reduce's algorithmic bytes), 4 buffer pairs in one graph, "
                                             "replayed back to back"}
                                    if copy_same_us else None),
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": int(launches),
        "clocks": clk,
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ sweep workload
def run_sweep(args):
    """The sweep configuration: p in {2,4,8,16}, per-rank sizes 1 KiB .. max in
    powers of 4, fp32/bf16/int32, all_reduce and reduce_scatter with sum and
    max, all_gather.  One JSON line per point: single-call device time (L2
    flushed before every call, outside the events; median and min of 200
    calls below 1 MiB per rank, 20 up to 64 MiB, 5 above), effective GB/s on the
    minimum-bytes basis, and for sizes <= 4 MiB the per-call time inside a
    CUDA graph of 20 back-to-back calls (the launch-latency term)."""
    import torch
    import collective_rc_all_b200 as rc

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    clean = torch.ones(CLEAN_BYTES // 4, dtype=torch.float32, device=dev)
    sink = torch.empty((), dtype=torch.float32, device=dev)
    peak, _ = measured_peaks()
    TT = {"f32": torch.float32, "bf16": torch.bfloat16, "i32": torch.int32}
    ESZ = {"f32": 4, "bf16": 2, "i32": 4}
    gen = torch.Generator(device=dev)
    sizes = [1 << k for k in range(10, 31, 2) if (1 << k) <= args.sweep_max_bytes]
    out = open(args.sweep_out, "w") if args.sweep_out else None

    def time_call(fn, footprint, reps):
        for _ in range(3):
            fn()
        ts = []
        for _ in range(reps):
            # always flush (untimed): without it the previous call's dirty
            # outputs are written back inside the timed call
            flush.zero_()
            torch.sum(clean, dim=0, out=sink)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            b.synchronize()
            ts.append(a.elapsed_time(b) * 1e-3)
        return float(np.median(ts)), float(min(ts))

    def time_graph(fn, calls=20):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, capture_error_mode="thread_local"):
            for _ in range(calls):
                fn()
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        ts = []
        for _ in range(10):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            g.replay()
            b.record(stream)
            b.synchronize()
            ts.append(a.elapsed_time(b) * 1e-3 / calls)
        del g
        return float(np.median(ts))

    for p in (2, 4, 8, 16):
        for nbytes in sizes:
            for dt in ("f32", "bf16", "i32"):
                s = ESZ[dt]
                n = nbytes // s
                gen.manual_seed(100 + p * 131 + nbytes % 10007)
                if dt == "i32":
                    send = [torch.randint(-(1 << 20), 1 << 20, (n,), generator=gen, device=dev,
                                          dtype=torch.int32) for _ in range(p)]
                else:
                    send = [(torch.rand(n, generator=gen, device=dev) * 2 - 1).to(TT[dt]) for _ in range(p)]
                y = [torch.empty(n, dtype=TT[dt], device=dev) for _ in range(p)]
                rs = [torch.empty(n // p, dtype=TT[dt], device=dev) for _ in range(p)]
                cases = [
                    ("all_reduce", "sum", lambda: rc.rc_all_reduce(send, y, op="sum"), 2 * p * n * s),
                    ("all_reduce", "max", lambda: rc.rc_all_reduce(send, y, op="max"), 2 * p * n * s),
                    ("reduce_scatter", "sum", lambda: rc.rc_reduce_scatter(send, rs, op="sum"), p * n * s + n * s),
                    ("reduce_scatter", "max", lambda: rc.rc_reduce_scatter(send, rs, op="max"), p * n * s + n * s),
                    ("all_gather", "-", lambda: rc.rc_all_gather(rs, y), n * s + p * n * s),
                ]
                reps = 200 if nbytes < (1 << 20) else (20 if nbytes <= (64 << 20) else 5)
                for coll, op, fn, byt in cases:
                    med, mn = time_call(fn, byt, reps)
                    row = {"p": p, "bytes_per_rank": nbytes, "dtype": dt, "coll": coll, "op": op,
                           "us": round(med * 1e6, 2), "us_min": round(mn * 1e6, 2),
                           "gbs": round(byt / med / 1e9, 1), "frac_of_measured_hbm": round(byt / med / 1e9 / peak, 4)}
                    if nbytes <= (4 << 20):
                        tg = time_graph(fn)
                        row["us_in_graph"] = round(tg * 1e6, 2)
                        row["gbs_in_graph"] = round(byt / tg / 1e9, 1)
                    line = json.dumps(row)
                    print(line, flush=True)
                    if out:
                        out.write(line + "\n")
                del send, y, rs
                torch.cuda.empty_cache()
    rc.rc_stream_status()
    if out:
        out.close()
    return 0


def zero1_bytes(p: int, n: int, s_grad: int, s_param: int) -> int:
    """Minimum bytes of one ZeRO-1 step over p ranks of n elements: every
    gradient read once, the fp32 master weights and both moments read and
    written once, every rank's parameters written once."""
    return p * n * s_grad + 2 * 3 * 4 * n + p * n * s_param


def run_zero1(args):
    """The sharded-optimizer workload (one JSON line): the ZeRO-1 AdamW step on
    a Llama-2-7B decoder layer (202,375,168 parameters) over 8 simulated
    ranks, fp32 gradients ~N(0, 1e-3), fp32 master weights and moments
    sharded 1/8 per rank.  Variants, each timed with CUDA events over K
    back-to-back steps after W warm-ups (every buffer is far larger than L2):
      fused_bf16     rc_zero1_step, bf16 parameters (the workload)
      fused_f32      rc_zero1_step, fp32 parameters
      unfused_f32    rc_reduce_scatter (fp32, x 1/8) + rc_adamw_step per
                     shard + rc_all_gather of the fp32 master shards
      owner_f32      the ShardedOptimizer form: per weight tensor, in-place
                     rc_all_reduce (x 1/8), rc_adamw_step by the owner
                     (tensor t % 8), rc_broadcast from the owner
    Effective GB/s always uses the fused step's minimum bytes (zero1_bytes)."""
    import torch
    import collective_rc_all_b200 as rc
    import rc_inputs

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    p, N = 8, args.zero1_elems
    if N % (8 * 4096) != 0:
        raise SystemExit("--zero1-elems must be a multiple of 8 * 4096")
    m = N // p
    hp = dict(rc_inputs.ZERO1_ADAMW)
    gen = torch.Generator(device=dev)
    gen.manual_seed(4)
    grads = [torch.randn(N, generator=gen, device=dev) * 1e-3 for _ in range(p)]
    gen.manual_seed(5)
    master = [torch.rand(m, generator=gen, device=dev) * 2 - 1 for _ in range(p)]
    ea = [torch.randn(m, generator=gen, device=dev) * 1e-3 for _ in range(p)]
    es = [(torch.randn(m, generator=gen, device=dev) * 1e-3).square() for _ in range(p)]
    p_bf16 = [torch.empty(N, dtype=torch.bfloat16, device=dev) for _ in range(p)]
    p_f32 = [torch.empty(N, dtype=torch.float32, device=dev) for _ in range(p)]
    gs = [torch.empty(m, dtype=torch.float32, device=dev) for _ in range(p)]
    # owner form: full-size fp32 state per tensor on its owner (views of flat arrays)
    shapes = [4096 * 4096] * 4 + [4096 * 11008] * 3
    if N != sum(shapes):  # a scaled-down case (profiling): the same seven tensors, scaled
        shapes = [s * N // sum(shapes) for s in shapes]
        shapes[-1] += N - sum(shapes)
    o_master = torch.rand(N, generator=gen, device=dev) * 2 - 1
    o_ea = torch.zeros(N, device=dev)
    o_es = torch.zeros(N, device=dev)
    offs = np.concatenate([[0], np.cumsum(shapes)]).astype(np.int64)

    def owner_step():
        for t, s in enumerate(shapes):
            a, b = int(offs[t]), int(offs[t + 1])
            gt = [g[a:b] for g in grads]
            owner = t % p
            rc.rc_all_reduce(gt, gt, scale=1.0 / p)
            rc.rc_adamw_step(o_master[a:b], o_ea[a:b], o_es[a:b], gt[owner], **hp)
            outs = [q[a:b] for q in p_f32]
            outs[owner] = o_master[a:b]
            rc.rc_broadcast(o_master[a:b], outs, root=owner)

    def unfused_step():
        rc.rc_reduce_scatter(grads, gs, out_dtype="f32", scale=1.0 / p)
        for r in range(p):
            rc.rc_adamw_step(master[r], ea[r], es[r], gs[r], **hp)
        rc.rc_all_gather(master, p_f32)

    variants = {
        "fused_bf16": (lambda: rc.rc_zero1_step(grads, p_bf16, master, ea, es, param_dtype="bf16", **hp), 2),
        "fused_f32": (lambda: rc.rc_zero1_step(grads, p_f32, master, ea, es, param_dtype="f32", **hp), 4),
        "unfused_f32": (unfused_step, 4),
        "owner_f32": (owner_step, 4),
    }
    K, W = args.steps, args.warmup
    peak, peak_kind = measured_peaks()
    res = {}
    clocks = ClockSampler(0)
    clocks.start()
    time.sleep(0.3)
    for name, (fn, sp) in variants.items():
        for _ in range(W):
            fn()
        torch.cuda.synchronize()
        l0 = rc.rc_launch_count()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(K):
            fn()
        b.record(stream)
        b.synchronize()
        t = a.elapsed_time(b) * 1e-3 / K
        byt = zero1_bytes(p, N, 4, sp)
        res[name] = {"ms": round(t * 1e3, 4), "min_bytes": byt, "gbs": round(byt / t / 1e9, 1),
                     "frac_of_measured_hbm": round(byt / t / 1e9 / peak, 4),
                     "launches_per_step": (rc.rc_launch_count() - l0) // K}
    clk = clocks.stop()
    rc.rc_stream_status()
    f = res["fused_bf16"]
    line = {
        "metric": "effective GB/s of the fused ZeRO-1 AdamW step (reduce-scatter, AdamW, all-gather in one pass)",
        "value": f["gbs"], "unit": UNIT, "n_gpus": 1, "steps": K, "warmup": W,
        "ms_per_step": f["ms"], "higher_is_better": True, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": f"ZeRO-1 AdamW step, {N:,} parameters (202,375,168 = one Llama-2-7B decoder layer), "
                               "p=8 simulated ranks, fp32 gradients ~N(0,1e-3), fp32 master weights "
                               "uniform[-1,1) and moments sharded 1/8, bf16 parameters on every rank",
                   "adamw": hp, "l2": "inputs larger than L2 (GBs per step)"},
        "roofline": {"bound": "hbm", "kernel": "rc_zero1_front_kernel", "achieved": f["gbs"], "peak": peak,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": f["frac_of_measured_hbm"],
                     "algorithmic_bytes": f["min_bytes"]},
        "variants": res,
        "clocks": clk,
    }
    print(json.dumps(line), flush=True)
    return 0


def moe_counts(p: int, t: int, k: int, experts: int, seed: int, zipf: float) -> np.ndarray:
    """Token-expert assignments per (source rank, destination rank) of one MoE
    layer: every rank routes t tokens to k distinct experts each, expert e
    lives on rank e // (experts // p), expert popularity ~ 1 / rank^zipf
    (zipf = 0: uniform).  Returns a p x p array of assignment counts."""
    rng = np.random.default_rng(seed)
    w = 1.0 / np.arange(1, experts + 1) ** zipf
    w = w[rng.permutation(experts)]
    w /= w.sum()
    per_rank = experts // p
    c = np.zeros((p, p), np.int64)
    for r in range(p):
        for _ in range(t):
            e = rng.choice(experts, size=k, replace=False, p=w)
            for x in e:
                c[r, x // per_rank] += 1
    return c


def run_a2a(args):
    """The MoE dispatch/combine workload (one JSON line): 8 simulated ranks
    (EP group), t = 4096 tokens per rank, top-2 routing, hidden 4096, bf16
    activations -- t*k*h*b = 64 MiB per rank and phase.  Variants: balanced
    routing (rc_all_to_all, equal splits) and skewed routing over 64 experts
    with popularity ~ 1/rank^1.2 (rc_all_to_all_v); each times the dispatch
    and the combine (the same exchange with the transposed counts) with CUDA
    events over K back-to-back rounds after W warm-ups.  Effective GB/s =
    (bytes read + written) / time; the cross-rank payload is reported too."""
    import torch
    import collective_rc_all_b200 as rc

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    p, t, k, h, E = 8, 4096, 2, 4096, 64
    b = 2
    peak, peak_kind = measured_peaks()
    K, W = args.steps, args.warmup
    res = {}
    clocks = ClockSampler(0)
    clocks.start()
    time.sleep(0.3)
    for name, zipf in (("balanced", None), ("skewed", 1.2)):
        if zipf is None:
            tok = np.full((p, p), t * k // p, np.int64)
        else:
            tok = moe_counts(p, t, k, E, seed=7, zipf=zipf)
        counts = tok * h
        send = [torch.empty(int(counts[r].sum()), dtype=torch.bfloat16, device=dev).normal_() for r in range(p)]
        mid = [torch.empty(int(counts[:, q].sum()), dtype=torch.bfloat16, device=dev) for q in range(p)]
        back = [torch.empty(int(counts[r].sum()), dtype=torch.bfloat16, device=dev) for r in range(p)]
        if zipf is None:
            dispatch = lambda: rc.rc_all_to_all(send, mid)
            combine = lambda: rc.rc_all_to_all(mid, back)
        else:
            dispatch = lambda: rc.rc_all_to_all_v(send, mid, counts)
            combine = lambda: rc.rc_all_to_all_v(mid, back, counts.T)
        for _ in range(W):
            dispatch()
            combine()
        torch.cuda.synchronize()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * K + 1)]
        for i in range(K):
            ev[2 * i].record(stream)
            dispatch()
            ev[2 * i + 1].record(stream)
            combine()
        ev[-1].record(stream)
        ev[-1].synchronize()
        td = sum(ev[2 * i].elapsed_time(ev[2 * i + 1]) for i in range(K)) * 1e-3 / K
        tc = sum(ev[2 * i + 1].elapsed_time(ev[2 * i + 2]) for i in range(K)) * 1e-3 / K
        payload = int(counts.sum()) * b                  # all blocks, one phase
        cross = int(counts.sum() - np.trace(counts)) * b  # blocks that change rank
        res[name] = {
            "dispatch_us": round(td * 1e6, 2), "combine_us": round(tc * 1e6, 2),
            "payload_bytes_per_phase": payload, "cross_rank_bytes_per_phase": cross,
            "max_rank_recv_bytes": int(counts.sum(axis=0).max()) * b,
            "dispatch_gbs": round(2 * payload / td / 1e9, 1), "combine_gbs": round(2 * payload / tc / 1e9, 1),
            "dispatch_frac_of_measured_hbm": round(2 * payload / td / 1e9 / peak, 4),
            "tokens_per_pair": tok.tolist() if zipf is not None else int(tok[0, 0]),
        }
        del send, mid, back
        torch.cuda.empty_cache()
    clk = clocks.stop()
    rc.rc_stream_status()
    bal = res["balanced"]
    line = {
        "metric": "effective GB/s of the MoE all-to-all dispatch (bytes read + written / time)",
        "value": bal["dispatch_gbs"], "unit": UNIT, "n_gpus": 1, "steps": K, "warmup": W,
        "ms_per_step": round((bal["dispatch_us"] + bal["combine_us"]) / 1e3, 4), "higher_is_better": True,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "MoE dispatch + combine: p=8 simulated ranks, t=4096 tokens per rank, top-2, "
                               "hidden 4096, bf16 (t*k*h*b = 64 MiB per rank and phase); skewed: 64 experts, "
                               "popularity ~ 1/rank^1.2, seed 7", "l2": "inputs larger than L2 (512 MiB per phase)"},
        "roofline": {"bound": "hbm", "kernel": "rc_a2a_kernel", "achieved": bal["dispatch_gbs"], "peak": peak,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": bal["dispatch_frac_of_measured_hbm"],
                     "algorithmic_bytes": 2 * bal["payload_bytes_per_phase"]},
        "variants": res,
        "clocks": clk,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_ddp(args):
    """The DDP gradient-synchronisation workload (one JSON line): 8 simulated
    ranks, two Llama-2-7B decoder layers (9 tensors each: W_q, W_k, W_v, W_o,
    W_gate, W_up, W_down and two norm weights), bf16 gradients in one flat
    buffer per rank in backward order.  A synthetic backward computes each
    rank's weight gradients as X^T dY (cuBLAS bf16 GEMMs, T tokens per rank)
    straight into the flat buffers, last tensor first, on the compute stream;
    the gradient bucketer averages them (x 1/8) on a high-priority
    communication stream.  Strategies of the pages' comparison:
      none           backward only (the reference time)
      naive          per-tensor all-reduce, all issued after backward
      flat_after     one all-reduce of everything after backward
      per_tensor     per-tensor all-reduce as soon as each gradient is ready
      bucket_25mb    25 MiB buckets as soon as each bucket is complete
    Reported per strategy (CUDA events, mean of K steps after W warm-ups):
    step time, backward time, and the exposed tail = end of the last
    all-reduce - end of backward."""
    import torch
    import collective_rc_all_b200 as rc

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    main_s = torch.cuda.current_stream()
    comm = torch.cuda.Stream(priority=-1)
    p, L, T, h, f = 8, 2, args.ddp_tokens, 4096, 11008
    layer = [("norm1", (h,)), ("q", (h, h)), ("k", (h, h)), ("v", (h, h)), ("o", (h, h)),
             ("norm2", (h,)), ("gate", (h, f)), ("up", (h, f)), ("down", (f, h))]
    fwd = [(f"l{l}.{nm}", shp) for l in range(L) for nm, shp in layer]
    bwd = fwd[::-1]                                       # gradients become ready in this order
    numel = [int(np.prod(s_)) for _, s_ in bwd]
    off = np.concatenate([[0], np.cumsum(numel)]).astype(np.int64)
    N = int(off[-1])
    grads = [torch.zeros(N, dtype=torch.bfloat16, device=dev) for _ in range(p)]
    gen = torch.Generator(device=dev)
    gen.manual_seed(11)
    X = [torch.randn(T, f, generator=gen, device=dev, dtype=torch.bfloat16) for _ in range(p)]
    dY = [torch.randn(T, f, generator=gen, device=dev, dtype=torch.bfloat16) for _ in range(p)]

    def grad_of(t, r):
        nm, shp = bwd[t]
        view = grads[r][int(off[t]):int(off[t + 1])]
        if len(shp) == 1:   # norm weight: sum over tokens of x * dy
            torch.sum(X[r][:, :h] * dY[r][:, :h], dim=0, out=view)
        else:               # weight (in, out): X[:, :in]^T @ dY[:, :out]
            torch.matmul(X[r][:, :shp[0]].t(), dY[r][:, :shp[1]], out=view.view(shp))

    strategies = {"none": None, "naive": (0, False), "flat_after": (2 ** 63, False),
                  "per_tensor": (0, True), "bucket_25mb": (25 << 20, True)}
    K, W = args.steps, args.warmup
    res = {}
    clocks = ClockSampler(0)
    clocks.start()
    time.sleep(0.3)
    for name, cfg in strategies.items():
        b = None if cfg is None else rc.Bucketer(grads, numel, cfg[0], comm_stream=comm)
        nb = len(b.buckets()) if b else 0

        def step():
            l0 = rc.rc_launch_count()
            for t in range(len(bwd)):
                for r in range(p):
                    grad_of(t, r)
                if b is not None and cfg[1]:
                    b.ready(t, main_s)
            e_bwd = torch.cuda.Event(enable_timing=True)
            e_bwd.record(main_s)
            if b is not None and not cfg[1]:
                for t in range(len(bwd)):
                    b.ready(t, main_s)
            if b is not None:
                b.flush(main_s)
            return e_bwd, rc.rc_launch_count() - l0

        for _ in range(W):
            step()
        torch.cuda.synchronize()
        tot, bw, launches = [], [], 0
        for _ in range(K):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(main_s)
            e_bwd, nl = step()
            e1.record(main_s)
            e1.synchronize()
            tot.append(e0.elapsed_time(e1))
            bw.append(e0.elapsed_time(e_bwd))
            launches = nl
        rc.rc_stream_status()
        res[name] = {"step_ms": round(float(np.mean(tot)), 4), "backward_ms": round(float(np.mean(bw)), 4),
                     "exposed_tail_ms": round(float(np.mean(tot) - np.mean(bw)), 4),
                     "buckets": nb, "all_reduce_kernels_per_step": int(launches)}
        if b is not None:
            b.close()
    clk = clocks.stop()
    base = res["none"]["step_ms"]
    for r_ in res.values():
        r_["slowdown_vs_backward_only"] = round(r_["step_ms"] / base, 4)
    ar_bytes = 2 * p * N * 2   # every gradient read and written once by the reduction
    best = min((k for k in res if k != "none"), key=lambda k: res[k]["step_ms"])
    line = {
        "metric": "exposed gradient-communication tail after backward, DDP bucketing strategies",
        "value": res[best]["exposed_tail_ms"], "unit": "ms", "n_gpus": 1, "steps": K, "warmup": W,
        "ms_per_step": res[best]["step_ms"], "higher_is_better": False, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": f"DDP gradient sync: p=8 simulated ranks, 2 Llama-2-7B decoder layers "
                               f"({N:,} parameters, 18 tensors), bf16 gradients from X^T dY GEMMs with "
                               f"T={T} tokens per rank, average (x 1/8) by bucketed in-place all-reduce on a "
                               f"high-priority stream", "best": best,
                   "all_reduce_bytes_per_step": ar_bytes},
        "strategies": res,
        "clocks": clk,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_configs(args):
    """Every named workload's calls, timed (one JSON line per call):
      uniform p=4 x 65,536 fp32         all_reduce, reduce_scatter, all_gather
      ring p=8 x 2,097,152 fp32         ring literal, ring one-shot, all_reduce
      ring p=8 x 2,097,152 bf16         ring literal, no-allocation ring, one-shot
      ring p in {2, 4, 16}, 8 MiB/rank  ring literal, one-shot (fp32 and bf16)
      hierarchical 2x4 x 4,194,304 bf16 fused, staged, flat all_reduce
      Llama-2-7B layer p=8              all_gather of bf16 shards, reduce_scatter
                                        fp32 -> bf16 x 1/8
    Each call alone after an L2 flush outside its events (median of reps),
    and back to back: one CUDA graph of 4 calls on 4 separate input/output
    sets (1 set for the layer, whose buffers dwarf L2), replayed; per call =
    time / calls.  GB/s on the minimum-bytes basis."""
    import torch
    import collective_rc_all_b200 as rc
    import rc_inputs

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    peak, peak_kind = measured_peaks()
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    clean = torch.ones(CLEAN_BYTES // 4, dtype=torch.float32, device=dev)
    sink = torch.empty((), dtype=torch.float32, device=dev)
    gen = torch.Generator(device=dev)
    TT = {"f32": torch.float32, "bf16": torch.bfloat16}

    def rand(n, dt, sigma=1.0):
        return (torch.randn(n, generator=gen, device=dev) * sigma).to(TT[dt])

    def iso(fn, reps=20):
        for _ in range(3):
            fn()
        ts = []
        for _ in range(reps):
            flush.zero_()
            torch.sum(clean, dim=0, out=sink)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            b.synchronize()
            ts.append(a.elapsed_time(b) * 1e-3)
        return float(np.median(ts))

    def b2b(fns, reps=20):
        for f in fns:
            f()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, capture_error_mode="thread_local"):
            for f in fns:
                f()
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            g.replay()
        b.record(stream)
        b.synchronize()
        del g
        return a.elapsed_time(b) * 1e-3 / (reps * len(fns))

    def emit(workload, call, byt, t_iso, t_b2b):
        row = {"workload": workload, "call": call, "min_bytes": byt,
               "isolated_us": round(t_iso * 1e6, 2), "isolated_gbs": round(byt / t_iso / 1e9, 1),
               "isolated_frac_of_measured_hbm": round(byt / t_iso / 1e9 / peak, 4),
               "back_to_back_us": round(t_b2b * 1e6, 2), "back_to_back_gbs": round(byt / t_b2b / 1e9, 1),
               "back_to_back_frac_of_measured_hbm": round(byt / t_b2b / 1e9 / peak, 4),
               "peak_gbs": peak, "peak_kind": peak_kind}
        print(json.dumps(row), flush=True)

    def sets(k, make):
        return [make() for _ in range(k)]

    # uniform p=4 x 65,536 fp32
    p, n = 4, 65536
    gen.manual_seed(0)
    S = sets(4, lambda: {"x": [rand(n, "f32") for _ in range(p)], "y": [torch.empty(n, device=dev) for _ in range(p)],
                         "rs": [torch.empty(n // p, device=dev) for _ in range(p)]})
    for call, mk, byt in (
            ("all_reduce", lambda d: (lambda: rc.rc_all_reduce(d["x"], d["y"])), 2 * p * n * 4),
            ("reduce_scatter", lambda d: (lambda: rc.rc_reduce_scatter(d["x"], d["rs"])), p * n * 4 + n * 4),
            ("all_gather", lambda d: (lambda: rc.rc_all_gather(d["rs"], d["y"])), n * 4 + p * n * 4)):
        emit("uniform p=4 x 65,536 fp32", call, byt, iso(mk(S[0]), 50), b2b([mk(d) for d in S]))
    del S

    # ring p=8 x 2,097,152 fp32 N(0, 1e-2)
    p, n = 8, 2097152
    gen.manual_seed(1)
    S = sets(4, lambda: {"x": [rand(n, "f32", 1e-2) for _ in range(p)], "y": [torch.empty(n, device=dev) for _ in range(p)]})
    for call, mk in (
            ("ring_all_reduce literal", lambda d: (lambda: rc.rc_ring_all_reduce(d["x"], d["y"], variant="literal"))),
            ("ring_all_reduce one-shot", lambda d: (lambda: rc.rc_ring_all_reduce(d["x"], d["y"], variant="oneshot"))),
            ("all_reduce", lambda d: (lambda: rc.rc_all_reduce(d["x"], d["y"])))):
        emit("ring p=8 x 2,097,152 fp32", call, 2 * p * n * 4, iso(mk(S[0])), b2b([mk(d) for d in S]))
    del S

    # ring p=8 x 2,097,152 bf16 (4 MiB per rank): fp32 partials in the link
    # kernel's shared memory, or (the no-allocation entry point's chain
    # kernel) in its fixed scratch (2 x 8 x 262,144 floats, exactly 16 MiB)
    p, n = 8, 2097152
    gen.manual_seed(1)
    S = sets(4, lambda: {"x": [rand(n, "bf16", 1e-2) for _ in range(p)],
                         "y": [torch.empty(n, dtype=torch.bfloat16, device=dev) for _ in range(p)]})
    rc.rc_reserve_workspace(2 * p * (n // p) * 4)
    for call, mk in (
            ("ring_all_reduce literal", lambda d: (lambda: rc.rc_ring_all_reduce(d["x"], d["y"], variant="literal"))),
            ("ring_all_reduce_noalloc", lambda d: (lambda: rc.rc_ring_all_reduce_noalloc(d["x"], d["y"]))),
            ("ring_all_reduce one-shot", lambda d: (lambda: rc.rc_ring_all_reduce(d["x"], d["y"], variant="oneshot")))):
        emit("ring p=8 x 2,097,152 bf16", call, 2 * p * n * 2, iso(mk(S[0])), b2b([mk(d) for d in S]))
    del S

    # the literal ring against the one-shot across p, 8 MiB per rank
    for p in (2, 4, 16):
        for dt in ("f32", "bf16"):
            n = (8 << 20) // (4 if dt == "f32" else 2)
            gen.manual_seed(1)
            S = sets(4, lambda: {"x": [rand(n, dt, 1e-2) for _ in range(p)],
                                 "y": [torch.empty(n, dtype=TT[dt], device=dev) for _ in range(p)]})
            for call, mk in (
                    ("ring_all_reduce literal", lambda d: (lambda: rc.rc_ring_all_reduce(d["x"], d["y"], variant="literal"))),
                    ("ring_all_reduce one-shot", lambda d: (lambda: rc.rc_ring_all_reduce(d["x"], d["y"], variant="oneshot")))):
                emit(f"ring p={p} x {n:,} {'fp32' if dt == 'f32' else 'bf16'}", call, 2 * p * n * (4 if dt == "f32" else 2),
                     iso(mk(S[0])), b2b([mk(d) for d in S]))
            del S
    torch.cuda.empty_cache()

    # hierarchical 2 x 4 x 4,194,304 bf16 N(0, 1)
    p, n = 8, 4194304
    gen.manual_seed(2)
    S = sets(4, lambda: {"x": [rand(n, "bf16") for _ in range(p)],
                         "y": [torch.empty(n, dtype=torch.bfloat16, device=dev) for _ in range(p)]})
    for call, mk in (
            ("hier_all_reduce fused", lambda d: (lambda: rc.rc_hier_all_reduce(d["x"], d["y"], 4, variant="fused"))),
            ("hier_all_reduce staged", lambda d: (lambda: rc.rc_hier_all_reduce(d["x"], d["y"], 4, variant="staged"))),
            ("all_reduce (flat)", lambda d: (lambda: rc.rc_all_reduce(d["x"], d["y"])))):
        emit("hierarchical 2x4 x 4,194,304 bf16", call, 2 * p * n * 2, iso(mk(S[0])), b2b([mk(d) for d in S]))
    del S
    torch.cuda.empty_cache()

    # Llama-2-7B decoder layer, p=8: all_gather of bf16 shards, reduce_scatter fp32 -> bf16 x 1/8
    N = rc_inputs.LLAMA2_7B_LAYER_ELEMS
    m = N // p
    gen.manual_seed(3)
    shards = [(torch.rand(m, generator=gen, device=dev) * 2 - 1).to(torch.bfloat16) for _ in range(p)]
    full = [torch.empty(N, dtype=torch.bfloat16, device=dev) for _ in range(p)]
    f = lambda: rc.rc_all_gather(shards, full)
    emit("Llama-2-7B layer p=8", "all_gather bf16", N * 2 + p * N * 2, iso(f, 5), b2b([f], 5))
    del full
    torch.cuda.empty_cache()
    gen.manual_seed(4)
    grads = [rand(N, "f32", 1e-3) for _ in range(p)]
    out = [torch.empty(m, dtype=torch.bfloat16, device=dev) for _ in range(p)]
    f = lambda: rc.rc_reduce_scatter(grads, out, out_dtype="bf16", scale=1.0 / p)
    emit("Llama-2-7B layer p=8", "reduce_scatter fp32->bf16 x1/8", p * N * 4 + N * 2, iso(f, 5), b2b([f], 5))
    rc.rc_stream_status()
    return 0


def run_pairs(args):
    """Each collective of the step after its predecessor, timed live: for
    every consecutive pair (X, Y) of the step's order, one CUDA graph of
    [X, Y] on 4 separate buffer sets, and one graph of [X] on the same sets,
    each replayed back to back; Y's in-sequence cost = T([X, Y]) - T([X])
    per call (everything the pair adds when Y follows X, the write-back of
    X's outputs that Y meets included).  One JSON line."""
    import torch
    import collective_rc_all_b200 as rc
    import rc_inputs
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    ops, m = step_ops()
    xs = rc_inputs.normal(P, N, seed=SEED, sigma=SIGMA)
    send = [torch.from_numpy(x).to(dev) for x in xs]

    def buffer_set():
        B = {k: [t.clone() for t in send] for k in ("ar", "rs", "red", "bc", "ring", "hier")}
        B.update({"y_ar": [torch.empty(N, device=dev) for _ in range(P)],
                  "y_ring": [torch.empty(N, device=dev) for _ in range(P)],
                  "y_hier": [torch.empty(N, device=dev) for _ in range(P)],
                  "y_rs": [torch.empty(m, dtype=torch.bfloat16, device=dev) for _ in range(P)],
                  "ag_in": [torch.empty(m, dtype=torch.bfloat16, device=dev) for _ in range(P)],
                  "y_ag": [torch.empty(N, dtype=torch.bfloat16, device=dev) for _ in range(P)],
                  "y_red": torch.empty(N, device=dev)})
        B["y_bc"] = [B["bc"][0]] + [torch.empty(N, device=dev) for _ in range(P - 1)]
        rc.rc_reduce_scatter(send, B["ag_in"], out_dtype="bf16", scale=1.0 / P)
        return B

    def call(nm, B):
        return {
            "all_reduce": lambda: rc.rc_all_reduce(B["ar"], B["y_ar"]),
            "reduce_scatter": lambda: rc.rc_reduce_scatter(B["rs"], B["y_rs"], out_dtype="bf16", scale=1.0 / P),
            "all_gather": lambda: rc.rc_all_gather(B["ag_in"], B["y_ag"]),
            "reduce": lambda: rc.rc_reduce(B["red"], B["y_red"], root=0),
            "broadcast": lambda: rc.rc_broadcast(B["bc"][0], B["y_bc"], root=0),
            "ring_all_reduce": lambda: rc.rc_ring_all_reduce(B["ring"], B["y_ring"], variant="literal"),
            "hier_all_reduce": lambda: rc.rc_hier_all_reduce(B["hier"], B["y_hier"], 4, variant="fused"),
        }[nm]

    sets = [buffer_set() for _ in range(4)]
    K = max(args.steps, 20)

    def timed(seq):
        for f in seq:
            f()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, capture_error_mode="thread_local"):
            for f in seq:
                f()
        for _ in range(max(3, args.warmup)):
            g.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(K):
            g.replay()
        b.record(stream)
        b.synchronize()
        del g
        return a.elapsed_time(b) * 1e-3 / (K * len(sets))

    peak, _ = measured_peaks()
    names = [nm for nm, _ in ops]
    alg = dict(ops)
    clocks = ClockSampler(0)
    clocks.start()
    single = {nm: timed([call(nm, B) for B in sets]) for nm in names}
    rows = {}
    for i, y in enumerate(names):
        x = names[i - 1]  # the step's predecessor (the last op precedes the first in a sequence of steps)
        pair = timed([f for B in sets for f in (call(x, B), call(y, B))])
        t_y = pair - single[x]
        rows[y] = {"after": x, "pair_us": round(pair * 1e6, 2), "after_alone_us": round(single[x] * 1e6, 2),
                   "in_sequence_us": round(t_y * 1e6, 2), "alone_back_to_back_us": round(single[y] * 1e6, 2),
                   "in_sequence_frac_of_measured_hbm": round(alg[y] / t_y / 1e9 / peak, 4)}
    clk = clocks.stop()
    rc.rc_stream_status()
    tot = sum(r["in_sequence_us"] for r in rows.values())
    print(json.dumps({"pairs": rows, "sum_in_sequence_us": round(tot, 2),
                      "sum_in_sequence_gbs": round(sum(alg.values()) / tot / 1e3, 1),
                      "peak": peak, "clocks": clk}), flush=True)
    return 0


NCU_WORKLOADS = {
    # name: (p, n per rank, dtype, description)
    "step": (8, 2097152, "f32", "8 ranks x 2,097,152 fp32 (8 MiB) per rank ~N(0,1e-2), the bench step's inputs"),
    "hier_bf16": (8, 4194304, "bf16", "8 ranks (2x4) x 4,194,304 bf16 (8 MiB) per rank ~N(0,1)"),
    "llama_eighth": (8, 202375168 // 8, "f32",
                     "1/8 of a Llama-2-7B decoder layer: 8 ranks x 25,296,896 elements"),
    "sweep_64mib": (8, (64 << 20) // 4, "f32", "8 ranks x 64 MiB fp32 per rank, uniform[-1,1)"),
}


def run_ncu_case(args):
    """Launches for a profiler, no timing: the collective `--ncu-case` on the
    workload `--ncu-workload`, called on S separate input/output sets in turn,
    twice around (4 sets when a set is under 256 MiB, else 2), so that the
    launches after the first S find the previous launch's outputs dirty in L2,
    as a collective in a sequence does.  With ncu --cache-control none, the
    launch numbered S (skip S) therefore counts those write-backs in its DRAM
    traffic.  Prints one line naming the launches."""
    import torch
    import collective_rc_all_b200 as rc
    op = args.ncu_case
    p, n, dt, desc = NCU_WORKLOADS[args.ncu_workload]
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    gen = torch.Generator(device=dev)
    gen.manual_seed(11)
    TT = {"f32": torch.float32, "bf16": torch.bfloat16}
    m = n // p
    odt = "bf16" if op in ("reduce_scatter", "all_gather") or dt == "bf16" else "f32"

    def one_set():
        d = {"x": [(torch.randn(n, generator=gen, device=dev)).to(TT[dt]) for _ in range(p)]}
        if op == "reduce_scatter":
            d["y"] = [torch.empty(m, dtype=TT[odt], device=dev) for _ in range(p)]
        elif op == "all_gather":
            d["x"] = [t[:m].to(torch.bfloat16) for t in d["x"]]
            d["y"] = [torch.empty(n, dtype=torch.bfloat16, device=dev) for _ in range(p)]
        elif op == "reduce":
            d["y"] = torch.empty(n, dtype=TT[dt], device=dev)
        elif op == "broadcast":
            d["y"] = [d["x"][0]] + [torch.empty(n, dtype=TT[dt], device=dev) for _ in range(p - 1)]
        else:
            d["y"] = [torch.empty(n, dtype=TT[dt], device=dev) for _ in range(p)]
        return d

    call = {
        "all_reduce": lambda d: rc.rc_all_reduce(d["x"], d["y"]),
        "reduce_scatter": lambda d: rc.rc_reduce_scatter(d["x"], d["y"], out_dtype=odt, scale=1.0 / p),
        "all_gather": lambda d: rc.rc_all_gather(d["x"], d["y"]),
        "reduce": lambda d: rc.rc_reduce(d["x"], d["y"], root=0),
        "broadcast": lambda d: rc.rc_broadcast(d["x"][0], d["y"], root=0),
        "ring_all_reduce": lambda d: rc.rc_ring_all_reduce(d["x"], d["y"], variant="literal"),
        "hier_all_reduce": lambda d: rc.rc_hier_all_reduce(d["x"], d["y"], 4, variant="fused"),
    }[op]
    set_bytes = 2 * p * n * (4 if dt == "f32" else 2)
    S = 4 if set_bytes < (256 << 20) else 2
    sets = [one_set() for _ in range(S)]
    torch.cuda.synchronize()
    l0 = rc.rc_launch_count()
    for _ in range(2):
        for d in sets:
            call(d)
    torch.cuda.synchronize()
    rc.rc_stream_status()
    print(json.dumps({"ncu_case": op, "workload": desc, "sets": S, "calls": 2 * S,
                      "launches": int(rc.rc_launch_count() - l0)}), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--ref-seconds", type=float, default=20.0,
                    help="total CPU budget of the reference arm (warm-up + timed steps)")
    # profiling aids: skip side phases (the timed step is always the whole step)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-copy-peak", action="store_true")
    ap.add_argument("--graph", choices=["step", "per_op"], default="step",
                    help="headline from one CUDA graph of the whole step, or from one graph per collective")
    # the sweep workload (not the driver's step): one JSON line per point
    ap.add_argument("--sweep", action="store_true")
    ap.add_argument("--sweep-max-bytes", type=int, default=1 << 30)
    ap.add_argument("--sweep-out", default="")
    # the sharded-optimizer workload (ZeRO-1 AdamW step): one JSON line
    ap.add_argument("--zero1", action="store_true")
    # the MoE dispatch / combine workload (all-to-all): one JSON line
    ap.add_argument("--a2a", action="store_true")
    # the DDP gradient-bucketing workload: one JSON line
    ap.add_argument("--ddp", action="store_true")
    # every named workload's calls, timed: one JSON line per call
    ap.add_argument("--configs", action="store_true")
    ap.add_argument("--ddp-tokens", type=int, default=1024, help="tokens per rank of the synthetic backward")
    ap.add_argument("--zero1-elems", type=int, default=202375168,
                    help="parameters of the ZeRO-1 workload (default: one Llama-2-7B decoder layer)")
    # each collective's live cost after its predecessor in the step
    ap.add_argument("--pairs", action="store_true")
    # launches for a profiler (no timing): one collective on one workload
    ap.add_argument("--ncu-case", default="", choices=[""] + [nm for nm, _ in step_ops()[0]])
    ap.add_argument("--ncu-workload", default="step", choices=sorted(NCU_WORKLOADS))
    args = ap.parse_args(argv)
    args.warmup = max(3, args.warmup)   # at least three untimed warm-up steps
    if args.ncu_case:
        return run_ncu_case(args)
    if args.pairs:
        return run_pairs(args)
    if args.impl == "reference":
        return run_reference(args)
    if args.sweep:
        return run_sweep(args)
    if args.zero1:
        return run_zero1(args)
    if args.a2a:
        return run_a2a(args)
    if args.ddp:
        return run_ddp(args)
    if args.configs:
        return run_configs(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
