"""Benchmark: paged decode attention effective KV GB/s and % of B200 HBM peak.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--block-size B]
                    [--partition-tokens P] [--impl ours|reference]

One step is one pass of the whole hot path over one batch: the copy-on-write
block copies of the step (workloads that share blocks), the append of each
sequence's new K/V row, then paged decode attention over every sequence's
context (which includes the new token).  The default workload is the batch-256
OPT-13B decode layer (40 heads x 128, bf16 KV, contexts uniform in [1, 2048],
block size 16).  The K/V pool is resident in HBM before the timed region starts
and is 43x larger than L2, so no L2 flush is needed between steps.

Multi-GPU: one process per GPU (torchrun); the path shards by sequence with no
exchange, so every rank runs its own replica of the workload and the job's
throughput is the sum of all ranks' bytes over the slowest rank's time.

`--impl reference` times the CPU oracle (float64 NumPy) on bounded samples of the
same workload instead; it is the only other place this script runs the oracle.
"""

import argparse
import json
import math
import multiprocessing as mp
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "paged decode attention effective KV GB/s and % of B200 HBM peak"
FALLBACK_HBM_GBS = 6650.0
WORKLOADS = ("opt13b", "llama7b", "cow", "longctx", "tiny", "gqa2", "gqa4", "gqa8", "gqa16", "gqa32", "gqa64", "swap")
DEFAULT_STEPS = {"opt13b": 500, "llama7b": 2000, "cow": 1000, "longctx": 500, "tiny": 200,
                 "gqa2": 500, "gqa4": 500, "gqa8": 500, "gqa16": 500, "gqa32": 300, "gqa64": 300, "swap": 20}


def parse():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", choices=WORKLOADS, default="opt13b")
    ap.add_argument("--block-size", type=int, default=16)
    ap.add_argument("--tune", action="store_true",
                    help="choose the partition size by timing the candidates on the workload before warm-up")
    ap.add_argument("--partition-tokens", type=int, default=None,
                    help="split-context partition size (default: the workload's, else the library's choice)")
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--eager", action="store_true",
                    help="launch every call from Python in the timed loop instead of replaying CUDA graphs")
    ap.add_argument("--no-targets", action="store_true",
                    help="default workload only: skip timing the long-context layer after it")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="CPU-baseline time budget")
    ap.add_argument("--q-len", type=int, default=1,
                    help="query tokens per sequence (>1: verify / chunked-prefill step through "
                         "paged_attn_multi_query; the last q_len positions are appended each step)")
    ap.add_argument("--num-seqs", type=int, default=None,
                    help="profiling aid: fewer sequences of the opt13b or gqa layers (a smaller case for ncu)")
    a = ap.parse_args()
    if a.steps is None:
        a.steps = DEFAULT_STEPS[a.workload]
    if a.warmup < 3:
        ap.error("--warmup must be >= 3")
    return a


def dist_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def job_throughput(bytes_per_step_per_rank, ms_per_step_by_rank):
    """Whole-job GB/s of independent replicas: all ranks' bytes over the slowest rank's time."""
    world = len(ms_per_step_by_rank)
    slowest = max(ms_per_step_by_rank)
    return bytes_per_step_per_rank * world / (slowest * 1e-3) / 1e9, slowest


def max_over_ranks(values, dist, device):
    """Element-wise max of a list of floats over all ranks (the timing rule for N > 1)."""
    import torch
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs, copy bandwidth)"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback 6.65 TB/s (no MEASURED_PEAKS.json)"


# ---------------------------------------------------------------------------
# CPU oracle timing (reference arm and cpu_baseline).  Worker processes are
# forked before this process touches CUDA, and never touch CUDA themselves.
# ---------------------------------------------------------------------------
_SAMPLE = None


def _cpu_worker_init():
    # one BLAS thread per worker process: cores used = number of processes
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(1)
    except ImportError:
        pass


def _oracle_task(i):
    import oracle
    c = _SAMPLE["cases"][i]
    t0 = time.perf_counter()
    oracle.paged_decode(c["q"], c["k"], c["v"], c["table"], c["ctx"], _SAMPLE["scale"], _SAMPLE["B"],
                        _SAMPLE["dtype"])
    return i, time.perf_counter() - t0


def oracle_sample_seqs(wname):
    """Sequences in the oracle's bounded sample: ``cpu_baseline`` and the reference
    arm time the same sample with the same function, so that the two agree."""
    return 2 if wname == "longctx" else 32


def make_cpu_sample(wname, block_size, n_seq, seed=7):
    """Bounded sample of the workload: its first ``n_seq`` context lengths and head
    geometry, with N(0,1) values placed through a random block table."""
    from paged_kv_cache_328_b200 import workloads as wl
    shapes = {"opt13b": (40, 128, "bf16", wl.opt13b_lengths()),
              "llama7b": (32, 128, "f16", wl.lognormal_lengths(64, wl.BASE_SEED + 2)),
              "cow": (40, 128, "f16", None), "longctx": (40, 128, "f16", wl.uniform_lengths(8, wl.BASE_SEED + 5,
                                                                                         16384, 32768)),
              "tiny": (2, 64, "f32", wl.tiny_lengths())}
    Hq = None
    if wname.startswith("gqa"):  # 8 K/V heads shared by `group` query heads each
        shapes[wname] = (8, 128, "bf16", wl.opt13b_lengths())
        Hq = 8 * int(wname[3:])
    H, D, dtype, ctx = shapes[wname]
    Hq = H if Hq is None else Hq
    if ctx is None:
        rng = np.random.default_rng(wl.BASE_SEED + 4)
        ctx = 512 + rng.integers(1, 257, size=128) + 1
    B = block_size if (wname == "opt13b" or wname.startswith("gqa")) else 16
    rng = np.random.default_rng(seed)
    cases = []
    for c in [int(x) for x in ctx[:n_seq]]:
        nblk = max(1, -(-c // B))
        nb = nblk + 2
        table = rng.permutation(nb)[:nblk].reshape(1, -1)
        if dtype == "f32":
            k = rng.standard_normal((nb, H, B, D), dtype=np.float32)
            v = rng.standard_normal((nb, H, B, D), dtype=np.float32)
            q = rng.standard_normal((1, Hq, D), dtype=np.float32)
        else:
            k = rng.integers(0, 1 << 16, size=(nb, H, B, D), dtype=np.uint16) & np.uint16(0xBFFF)
            v = rng.integers(0, 1 << 16, size=(nb, H, B, D), dtype=np.uint16) & np.uint16(0xBFFF)
            q = rng.integers(0, 1 << 16, size=(1, Hq, D), dtype=np.uint16) & np.uint16(0xBFFF)
            if dtype == "f16":  # keep magnitudes moderate: exponent field <= 15
                k, v, q = (x & np.uint16(0xBBFF) for x in (k, v, q))
        cases.append(dict(q=q, k=k, v=v, table=table, ctx=np.array([c]), nbytes=c * H * D * (2 if dtype != "f32"
                                                                                              else 4) * 2))
    return dict(cases=cases, scale=1.0 / math.sqrt(D), B=B, dtype=dtype, H=H, D=D)


def start_cpu_pool(sample):
    global _SAMPLE
    _SAMPLE = sample
    cores = os.cpu_count() or 1
    ctx = mp.get_context("fork")
    return ctx.Pool(cores, initializer=_cpu_worker_init), cores


def time_oracle(pool, sample, budget_s):
    """Run the oracle over the sample's sequences (repeating passes) until budget_s elapsed."""
    n = len(sample["cases"])
    done_bytes = 0
    tokens = 0
    t0 = time.perf_counter()
    passes = 0
    while True:
        for i, _ in pool.imap_unordered(_oracle_task, range(n)):
            done_bytes += sample["cases"][i]["nbytes"]
            tokens += int(sample["cases"][i]["ctx"][0])
        passes += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    wall = time.perf_counter() - t0
    return done_bytes, tokens, wall, passes


# ---------------------------------------------------------------------------
# Clock sampling during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.lines = []
        self.proc = None
        self.t_start = self.t_stop = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(gpu_index)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, ValueError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.perf_counter(), line.strip()))

    def mark(self, start):
        if start:
            self.t_start = time.perf_counter()
        else:
            self.t_stop = time.perf_counter()

    def summary(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        inside = [l for t, l in self.lines if self.t_start <= t <= self.t_stop + 0.15]
        window = "timed region"
        if not inside:  # timed region shorter than the sampling period: nearest samples
            inside = [l for t, l in self.lines if self.t_start - 0.3 <= t <= self.t_stop + 0.3]
            window = "timed region +-0.3 s"
        sm, mx, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for l in inside:
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm), "window": window}


# ---------------------------------------------------------------------------
# The GPU arm
# ---------------------------------------------------------------------------
def traffic_record(workload_key):
    """dram bytes per decode launch from a committed ncu capture, if the decode kernel's sources
    (listed in the record) are unchanged since the capture; else None."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        rec = json.load(open(path)).get(workload_key)
    except (OSError, ValueError):
        return None
    if not rec:
        return None
    h = hashlib.sha256()
    for f in rec.get("kernel_sources", []):
        h.update(open(os.path.join(ROOT, f), "rb").read())
    return rec["dram_bytes_per_launch"] if rec.get("csrc_sha256") == h.hexdigest() else None


NOMINAL_READ_GBS = 7700.0  # B200 (HGX) HBM3e nominal bandwidth, a read-only stream's ceiling


def spread(vals):
    """Mean, median and 10th / 90th percentiles of per-iteration times (ms)."""
    v = sorted(vals)

    def q(p):
        return v[min(len(v) - 1, int(round(p * (len(v) - 1))))]
    return {"mean": round(statistics.mean(v), 5), "median": round(statistics.median(v), 5),
            "p10": round(q(0.1), 5), "p90": round(q(0.9), 5)}


def unique_kv_bytes(w):
    """K+V bytes of the distinct pool rows the step's decode reads: each physical
    block counted once, with the longest prefix any sequence reads from it."""
    seen = {}
    for s_, c in enumerate(w.context_lens.tolist()):
        for j in range(-(-int(c) // w.B)):
            b = int(w.block_tables[s_, j])
            seen[b] = max(seen.get(b, 0), min(w.B, int(c) - j * w.B))
    return sum(seen.values()) * w.Hkv * w.D * w.elem_bytes * 2


def prepare(w, Lq, dev):
    """Device copies of the step's indices; with Lq > 1 the step appends and queries
    the last Lq positions of every context."""
    import torch
    if Lq > 1:
        sl = np.full((w.S, Lq), -1, dtype=np.int64)
        for s_ in range(w.S):
            c = int(w.context_lens[s_])
            for j in range(Lq):
                pos = c - Lq + j
                if pos >= 0:
                    sl[s_, j] = int(w.block_tables[s_, pos // w.B]) * w.B + pos % w.B
        w.slot_mapping = sl.reshape(-1)
        gq = torch.Generator(device=dev)
        gq.manual_seed(4242)
        w.q = torch.randn((w.S, Lq, w.H, w.D), generator=gq, device=dev).to(w.q.dtype)
        w.k_new = torch.randn((w.S * Lq, w.Hkv, w.D), generator=gq, device=dev).to(w.q.dtype)
        w.v_new = torch.randn((w.S * Lq, w.Hkv, w.D), generator=gq, device=dev).to(w.q.dtype)
    return dict(bt=torch.from_numpy(w.block_tables).to(dev), ctx=torch.from_numpy(w.context_lens).to(dev),
                slots=torch.from_numpy(w.slot_mapping).to(dev),
                pairs=torch.from_numpy(w.cow_pairs.reshape(-1, 2)).to(dev))


class Step:
    """One pass of the hot path over a workload: copy-on-write block copies (if
    any), the append of the step's new K/V rows, then paged attention."""

    def __init__(self, pkv, w, Lq, pt, ix, dev):
        import torch
        self.pkv, self.w, self.Lq, self.pt, self.ix = pkv, w, Lq, pt, ix
        self.out = torch.empty(tuple(w.q.shape), dtype=torch.float32, device=dev)
        self.stream = torch.cuda.current_stream(dev)
        if Lq > 1:
            nws = pkv.load().paged_attn_multi_query_workspace_size(w.S, Lq, w.H, w.Hkv, w.D, w.B, w.max_blocks, pt)
            self.ws = torch.empty(nws, dtype=torch.uint8, device=dev)
            self.pt_used = pt if pt else pkv.gqa_partition_tokens(w.S, w.H, w.Hkv, w.D, w.B, w.max_blocks, 0)
        else:
            self.ws = pkv.alloc_workspace(w.q, w.k_pool, ix["bt"], pt)
            self.pt_used = pkv.gqa_partition_tokens(w.S, w.H, w.Hkv, w.D, w.B, w.max_blocks, pt)
        self.split = self.pt_used < w.max_blocks * w.B
        self.launches = (1 if len(w.cow_pairs) else 0) + 1 + 2 + (1 if self.split else 0)

    def attend(self, q, bt, ctx, out):
        w = self.w
        if self.Lq > 1:
            return self.pkv.paged_attn_multi_query(q, w.k_pool, w.v_pool, bt, ctx, w.scale, out=out,
                                                   partition_tokens=self.pt, workspace=self.ws)
        return self.pkv.paged_attn_decode(q, w.k_pool, w.v_pool, bt, ctx, w.scale, out=out,
                                          partition_tokens=self.pt, workspace=self.ws)

    def __call__(self, dec_events=None):
        w, ix = self.w, self.ix
        if len(w.cow_pairs):
            self.pkv.kv_block_copy(w.k_pool, w.v_pool, ix["pairs"])
        self.pkv.kv_cache_append(w.k_new, w.v_new, w.k_pool, w.v_pool, ix["slots"])
        if dec_events is not None:
            dec_events[0].record(self.stream)
        self.attend(w.q, ix["bt"], ix["ctx"], self.out)
        if dec_events is not None:
            dec_events[1].record(self.stream)


def graph_chunk(steps):
    """Steps per captured graph: a divisor of the step count, so that the timed
    replays run exactly `steps` steps."""
    for m in (10, 8, 5, 4, 2):
        if steps % m == 0 and steps // m >= 3:
            return m
    return 1


def time_steps(step, steps, warmup, pkv, dev, local_rank, world, dist, eager=False):
    """W untimed steps, then K timed steps bracketed by a barrier and a synchronize
    on both sides, with the SM clocks sampled during the timed region.  Returns the
    total, per-step and per-attention-call times (CUDA events on the launching
    stream; the total is the max over ranks) and the clock summary.

    By default the steps run as CUDA graphs (the way a serving loop replays its
    decode step): M steps are captured once through the public API and replayed
    K / M times, each replay between two events; a graph of M attention calls is
    replayed after each of them (outside the steps' events), so that both see the
    same clocks under the power cap.  `eager` launches every call from Python
    instead, so the host's launch cost can show in the device timeline."""
    import torch
    stream = step.stream

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local_rank])

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    code, reason = pkv.get_device_error(dev)
    if code != 0:
        raise RuntimeError(f"device error word after warm-up: {code} reason {reason}")
    mk = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    m = 1 if eager else graph_chunk(steps)
    if not eager:
        g_step, g_call = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_step):
            for _ in range(m):
                step()
        with torch.cuda.graph(g_call):
            for _ in range(m):
                step.attend(step.w.q, step.ix["bt"], step.ix["ctx"], step.out)
        for _ in range(2):
            g_step.replay()
            g_call.replay()
        torch.cuda.synchronize()
        run_steps = g_step.replay
    clocks = ClockSampler(local_rank)
    time.sleep(0.3)
    n = steps // m
    ev = [(mk(), mk()) for _ in range(n)]       # around each step replay (or eager step)
    dec = [(mk(), mk()) for _ in range(n)]      # around each attention-call replay (or eager call)
    barrier()
    torch.cuda.synchronize()
    clocks.mark(True)
    for i in range(n):
        ev[i][0].record(stream)
        if eager:
            step(dec[i])
        else:
            run_steps()
        ev[i][1].record(stream)
        if not eager:
            dec[i][0].record(stream)
            g_call.replay()
            dec[i][1].record(stream)
    torch.cuda.synchronize()
    clocks.mark(False)
    barrier()
    per_step = [e0.elapsed_time(e1) / m for e0, e1 in ev]
    per_call = [e0.elapsed_time(e1) / m for e0, e1 in dec]
    total = sum(per_step) * m  # the K steps' device time
    if not eager:
        del g_step, g_call
    dec_mean = statistics.mean(per_call)
    if world > 1:
        total, dec_mean = max_over_ranks([total, dec_mean], dist, dev)
    code, reason = pkv.get_device_error(dev)
    if code != 0:
        raise RuntimeError(f"device error word after the timed steps: {code} reason {reason}")
    return dict(total_ms=total, step=spread(per_step), call=spread(per_call), call_mean=dec_mean,
                clocks=clocks.summary(),
                timing=("eager: every call launched from Python" if eager else
                        f"CUDA graphs of {m} steps (and of {m} attention calls) captured through the public "
                        f"API, replayed {n} times with an event between replays"))


def roofline(kind, kv_bytes, call_ms, peak, peak_src, traffic, call):
    achieved = kv_bytes / (call_ms * 1e-3) / 1e9
    return {
        "kernel": kind + " call (plan + persistent attention kernel + merge launches)",
        "bound": "hbm",
        "achieved": round(achieved, 1),
        "peak": peak,
        "peak_source": peak_src,
        "unit": "GB/s",
        "frac": round(achieved / peak, 4),
        "frac_of_nominal_read": round(achieved / NOMINAL_READ_GBS, 4),
        "nominal_read_gbs": NOMINAL_READ_GBS,
        "traffic": traffic,
        "algorithmic_bytes_per_launch": kv_bytes,
        "avg_launch_ms": round(call_ms, 5),
        "launch_ms": call,
    }


def run_gpu(a, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import paged_kv_cache_328_b200 as pkv
    from paged_kv_cache_328_b200 import workloads as wl

    sample = pool = None
    cores = 0
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        sample = make_cpu_sample(a.workload, a.block_size, n_seq=oracle_sample_seqs(a.workload))
        pool, cores = start_cpu_pool(sample)  # forked before any CUDA call

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    pkv.load()

    if a.num_seqs is not None and a.workload == "opt13b":
        w = wl.make_opt13b(B=a.block_size, device=dev, S=a.num_seqs)
        w.name += f"_S{a.num_seqs}"
    elif a.num_seqs is not None and a.workload.startswith("gqa"):
        w = wl.make_gqa(int(a.workload[3:]), device=dev, S=a.num_seqs, B=a.block_size)
        w.name += f"_S{a.num_seqs}"
    else:
        w = wl.make(a.workload, device=dev, B=a.block_size if a.workload in ("opt13b",) or
                    a.workload.startswith("gqa") else None)
    pt = w.partition_tokens if a.partition_tokens is None else a.partition_tokens
    Lq = a.q_len
    ix = prepare(w, Lq, dev)
    tuned = None
    if a.tune and Lq == 1:
        out = torch.empty(tuple(w.q.shape), dtype=torch.float32, device=dev)
        pt, times = pkv.tune_partition_tokens(w.q, w.k_pool, w.v_pool, ix["bt"], ix["ctx"], w.scale, reps=5,
                                              out=out)
        tuned = {str(k): round(v, 5) for k, v in times.items()}
    step = Step(pkv, w, Lq, pt, ix, dev)
    stream = step.stream
    t = time_steps(step, a.steps, a.warmup, pkv, dev, local_rank, world, dist, eager=a.eager)
    ms = t["total_ms"]
    dec_ms = t["call_mean"]
    out = step.out

    # ---- end to end through the public API with host buffers ---------------
    # Every step's inputs (q, the new K/V rows, tables, lengths, slots, copy pairs)
    # come from pinned host memory and its fp32 output goes back to pinned host
    # memory.  The loop is double-buffered the way a serving loop would run it:
    # the inputs of step i+1 cross the host link on one copy stream while step i
    # computes, and step i's output is read back on another while step i+1 computes.
    names = ("q", "k", "v", "bt", "ctx", "slots", "pairs")
    src = dict(q=w.q, k=w.k_new, v=w.v_new, bt=ix["bt"], ctx=ix["ctx"], slots=ix["slots"], pairs=ix["pairs"])
    pin = {n: src[n].cpu().pin_memory() for n in names}
    bufs = [{n: torch.empty_like(src[n]) for n in names} for _ in range(2)]
    outs = [torch.empty_like(out) for _ in range(2)]
    out_h = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    h2d = sum(x.numel() * x.element_size() for x in pin.values())
    d2h = out_h[0].numel() * out_h[0].element_size()
    h2d_stream, d2h_stream = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    in_ready = [torch.cuda.Event() for _ in range(2)]
    computed = [torch.cuda.Event() for _ in range(2)]
    read_back = [torch.cuda.Event() for _ in range(2)]

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local_rank])

    def e2e_h2d(i):
        b = bufs[i % 2]
        with torch.cuda.stream(h2d_stream):
            h2d_stream.wait_event(computed[i % 2])  # step i-2 is done with this buffer set
            for n in names:
                b[n].copy_(pin[n], non_blocking=True)
            in_ready[i % 2].record(h2d_stream)

    def e2e_compute(i):
        b, o = bufs[i % 2], outs[i % 2]
        stream.wait_event(in_ready[i % 2])
        stream.wait_event(read_back[i % 2])  # step i-2's output has been read back
        if len(w.cow_pairs):
            pkv.kv_block_copy(w.k_pool, w.v_pool, b["pairs"])
        pkv.kv_cache_append(b["k"], b["v"], w.k_pool, w.v_pool, b["slots"])
        step.attend(b["q"], b["bt"], b["ctx"], o)
        computed[i % 2].record(stream)

    def e2e_d2h(i):
        with torch.cuda.stream(d2h_stream):
            d2h_stream.wait_event(computed[i % 2])
            out_h[i % 2].copy_(outs[i % 2], non_blocking=True)
            read_back[i % 2].record(d2h_stream)

    def e2e_run(n_steps, t0=None):
        if t0 is not None:
            h2d_stream.wait_event(t0)
        e2e_h2d(0)
        for i in range(n_steps):
            if i + 1 < n_steps:
                e2e_h2d(i + 1)
            e2e_compute(i)
            e2e_d2h(i)
        stream.wait_event(read_back[(n_steps - 1) % 2])

    e2e_run(a.warmup)
    torch.cuda.synchronize()
    e_steps = max(3, a.steps // 2)
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    e2e_run(e_steps, t0=e0)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = e0.elapsed_time(e1) / e_steps
    if world > 1:
        e2e_ms = max_over_ranks([e2e_ms], dist, dev)[0]
    if not torch.equal(out_h[(e_steps - 1) % 2], out.cpu()):
        raise RuntimeError("end-to-end output differs from the device-timed step's output")

    kv_bytes = w.kv_bytes_attended()
    ms_step = ms / a.steps
    value, _ = job_throughput(kv_bytes, [ms_step] * world)
    peak, peak_src = measured_peaks()
    # the traffic record belongs to one kernel: multi-token queries run another one
    wkey = f"{w.name}" + (f"_pt{pt}" if pt else "") + (f"_L{Lq}" if Lq > 1 else "")
    kind = "paged_attn_multi_query" if Lq > 1 else "paged_attn_decode"
    result = {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": a.steps,
        "warmup": a.warmup,
        "ms_per_step": round(ms_step, 5),
        "step_ms": t["step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": w.dtype,
        "data": "synthetic",
        "config": {
            "workload": w.name, "num_seqs": w.S, "num_heads": w.H, "num_kv_heads": w.Hkv, "head_dim": w.D,
            "block_size": w.B,
            "context_tokens_per_step": int(w.context_lens.sum()), "kv_bytes_per_step": kv_bytes,
            "cow_pairs_per_step": int(len(w.cow_pairs)), "appended_tokens_per_step": int((w.slot_mapping >= 0).sum()),
            "query_tokens_per_sequence": Lq,
            "partition_tokens": step.pt_used,
            "l2": f"no flush: K/V pool {w.k_pool.numel() * w.k_pool.element_size() * 2 / 1e9:.2f} GB "
                  f"= {w.k_pool.numel() * w.k_pool.element_size() * 2 / 126e6:.0f}x L2",
            "parallelism": f"replicas x{world}",
            "timing": t["timing"],
        },
        "pct_of_hbm_peak": round(100.0 * value / world / peak, 2),
        "pct_of_hbm_peak_basis": "MEASURED_PEAKS.json hbm_gbs: a device-to-device copy counting read + write "
                                 "bytes; decode only reads, so a read stream can exceed it "
                                 "(roofline.frac_of_nominal_read is against the 7.7 TB/s nominal)",
        "seq_per_s": round(w.S * world / (ms_step * 1e-3), 1),
        "ctx_tokens_per_s": round(int(w.context_lens.sum()) * world / (ms_step * 1e-3), 1),
        "roofline": roofline(kind, kv_bytes, dec_ms, peak, peak_src, traffic_record(wkey), t["call"]),
        "e2e": {"value": round(kv_bytes * world / (e2e_ms * 1e-3) / 1e9, 1), "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 5),
                "note": "every step copies its inputs (q, new K/V rows, tables, lengths, slots, pairs) from "
                        "pinned host memory and reads its fp32 output back; double-buffered on two copy "
                        "streams so the copies overlap the neighbouring steps' kernels; the K/V cache "
                        "stays resident"},
        "gpu_launches": step.launches * a.steps,
        "clocks": t["clocks"],
    }
    if w.name == "cow":
        ub = unique_kv_bytes(w)
        result["config"]["cow_memory_saving"] = round(w.info["cow_saving"], 4)
        result["config"]["kv_bytes_unique_per_step"] = ub
        result["unique"] = {
            "value": round(ub * world / (ms_step * 1e-3) / 1e9, 1), "unit": "GB/s",
            "pct_of_hbm_peak": round(100.0 * ub / (ms_step * 1e-3) / 1e9 / peak, 2),
            "decode_call_gbs": round(ub / (dec_ms * 1e-3) / 1e9, 1),
            "note": "distinct pool rows read per step (shared prompt blocks once); the headline value counts "
                    "every sequence's logical context, and shared blocks re-read from L2 let it exceed HBM",
        }
    result["config"]["last_block_waste"] = round(wl.last_block_waste(w), 4)
    if tuned is not None:
        result["config"]["tuned_ms_per_call"] = tuned

    # ---- the long-context target, timed in the same process --------------------
    # The batch-256 layer and the long-context layer are the two configurations
    # with a throughput target; the default run times both under one clock sampler
    # each, so both numbers come from the same recorded line.
    if a.workload == "opt13b" and Lq == 1 and a.num_seqs is None and not a.no_targets:
        del step, out
        w2 = wl.make_longctx(device=dev)
        ix2 = prepare(w2, 1, dev)
        step2 = Step(pkv, w2, 1, w2.partition_tokens, ix2, dev)
        t2 = time_steps(step2, a.steps, a.warmup, pkv, dev, local_rank, world, dist, eager=a.eager)
        kv2 = w2.kv_bytes_attended()
        ms2 = t2["total_ms"] / a.steps
        v2, _ = job_throughput(kv2, [ms2] * world)
        result["targets"] = {"longctx": {
            "value": round(v2, 1), "unit": "GB/s", "ms_per_step": round(ms2, 5), "step_ms": t2["step"],
            "pct_of_hbm_peak": round(100.0 * v2 / world / peak, 2),
            "config": {"workload": w2.name, "num_seqs": w2.S, "num_heads": w2.H, "head_dim": w2.D,
                       "block_size": w2.B, "dtype": w2.dtype, "kv_bytes_per_step": kv2,
                       "context_tokens_per_step": int(w2.context_lens.sum()),
                       "partition_tokens": step2.pt_used, "steps": a.steps, "warmup": a.warmup},
            "roofline": roofline("paged_attn_decode", kv2, t2["call_mean"], peak, peak_src,
                                 traffic_record(f"{w2.name}_pt{w2.partition_tokens}"), t2["call"]),
            "gpu_launches": step2.launches * a.steps,
            "clocks": t2["clocks"],
        }}
        result["gpu_launches"] += step2.launches * a.steps

    if pool is not None:
        nbytes, tokens, wall, passes = time_oracle(pool, sample, a.cpu_seconds)
        pool.terminate()
        result["cpu_baseline"] = {
            "value": round(nbytes / wall / 1e9, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"{len(sample['cases'])} sequences x {sample['H']} heads of the workload's context lengths "
                      f"({passes} pass(es), {tokens} context tokens per head, {wall:.1f} s), float64 NumPy, "
                      f"one process per core",
        }
    if world > 1:
        dist.barrier(device_ids=[local_rank])
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


# ---------------------------------------------------------------------------
# Reference arm: the CPU oracle on bounded samples of the same workload
# ---------------------------------------------------------------------------
def run_reference(a, rank, world):
    if rank != 0:
        return
    if a.workload == "swap":
        print(json.dumps({"impl": "reference", "unavailable": "the reference arm times the oracle's attention; "
                          "the swap workload has no attention step"}), flush=True)
        return
    n_seq = oracle_sample_seqs(a.workload)
    sample = make_cpu_sample(a.workload, a.block_size, n_seq=n_seq)
    pool, cores = start_cpu_pool(sample)
    for _ in range(a.warmup):
        time_oracle(pool, sample, 0.0)
    step_bytes = sum(c["nbytes"] for c in sample["cases"])
    t0 = time.perf_counter()
    for _ in range(a.steps):
        time_oracle(pool, sample, 0.0)
    wall = time.perf_counter() - t0
    pool.terminate()
    value = step_bytes * a.steps / wall / 1e9
    res = {
        "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world, "steps": a.steps,
        "warmup": a.warmup, "ms_per_step": round(wall / a.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": {"workload": a.workload, "block_size": sample["B"], "parallelism": "cpu processes"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": f"{len(sample['cases'])} sequence(s) x {sample['H']} heads of the workload's "
                                   f"context lengths per step (the GPU arm's cpu_baseline sample), float64 NumPy, "
                                   f"one process per core"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(res), flush=True)


def run_swap(a, rank, world, local_rank):
    """Block-granular swap: every step moves 1024 random blocks of the batch-256
    layer's pool (B=16: 160 KB of K and 160 KB of V each) to pinned host memory and
    back into other free blocks.  Metric: bytes moved per direction per second."""
    import torch
    import paged_kv_cache_328_b200 as pkv
    from paged_kv_cache_328_b200 import workloads as wl
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    pkv.load()
    w = wl.make_opt13b(B=a.block_size, device=dev)
    n = 1024
    rng = np.random.default_rng(11)
    perm = rng.permutation(w.num_blocks)
    out_ids = torch.from_numpy(perm[:n].astype(np.int64)).to(dev)
    in_ids = torch.from_numpy(perm[n:2 * n].astype(np.int64)).to(dev)
    shape = (n,) + tuple(w.k_pool.shape[1:])
    hk = torch.empty(shape, dtype=w.k_pool.dtype).pin_memory()
    hv = torch.empty(shape, dtype=w.k_pool.dtype).pin_memory()
    st = torch.cuda.current_stream(dev)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    for _ in range(a.warmup):
        pkv.kv_blocks_to_host(w.k_pool, w.v_pool, out_ids, hk, hv)
        pkv.kv_blocks_from_host(hk, hv, w.k_pool, w.v_pool, in_ids)
    torch.cuda.synchronize()
    t_out = t_in = 0.0
    for _ in range(a.steps):
        ev[0].record(st)
        pkv.kv_blocks_to_host(w.k_pool, w.v_pool, out_ids, hk, hv)
        ev[1].record(st)
        pkv.kv_blocks_from_host(hk, hv, w.k_pool, w.v_pool, in_ids)
        ev[2].record(st)
        torch.cuda.synchronize()
        t_out += ev[0].elapsed_time(ev[1])
        t_in += ev[1].elapsed_time(ev[2])
    code, reason = pkv.get_device_error(dev)
    if code != 0:
        raise RuntimeError(f"device error word: {code} reason {reason}")
    moved = 2 * n * hk[0].numel() * hk.element_size()
    res = {"metric": "KV block swap GB/s (device <-> pinned host, one kernel per direction)",
           "value": round(moved / ((t_out + t_in) / 2 / a.steps * 1e-3) / 1e9, 2), "unit": "GB/s",
           "to_host_gbs": round(moved / (t_out / a.steps * 1e-3) / 1e9, 2),
           "from_host_gbs": round(moved / (t_in / a.steps * 1e-3) / 1e9, 2),
           "n_gpus": world, "steps": a.steps, "warmup": a.warmup,
           "ms_per_step": round((t_out + t_in) / a.steps, 4), "higher_is_better": True, "dtype": w.dtype,
           "data": "synthetic", "config": {"workload": "swap", "blocks_per_direction": n,
                                           "bytes_per_direction": moved, "block_size": w.B}}
    if rank == 0:
        print(json.dumps(res), flush=True)


def main():
    a = parse()
    rank, world, local_rank = dist_env()
    if a.gpus != world and world != 1:
        print(f"warning: --gpus {a.gpus} but WORLD_SIZE {world}", file=sys.stderr)
    if a.impl == "reference":
        run_reference(a, rank, world)
        return
    if a.workload == "swap":
        run_swap(a, rank, world, local_rank)
        return
    run_gpu(a, rank, world, local_rank)


if __name__ == "__main__":
    main()
