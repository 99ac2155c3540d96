#!/usr/bin/env python
"""Benchmark of the DeltaLog decode step on B200.

Workload (default): GDN decode, B=256 slots, H=32 heads, d_k=d_v=128, fp32
state (537 MB), bf16 q/k/v, merge interval M=8, synthetic seeded inputs.
One bench step = one pass of the whole hot path over the workload's 256-token
decode sequence for all B slots: 256/M merge cycles, each M-1 append
launches + 1 merge launch.  ``value`` = slot-tokens per second (B * tokens
per step * steps / time) summed over all ranks, inputs resident in HBM.

For the metric's headline the same line also carries, under "workloads",
KDA (B=128, H=32, d=128) and RWKV6 (B=128, H=64, d=64) at M=8 with their
eager-kernel and e2e figures (and once more with fp16 per-key log-gates),
and under "sweep" the headline at M = 4 and 16 (M = 1 is the "eager" key).  ``cpu_baseline`` times the fp64 oracle on the
host cores (one spawned worker process per core, each on its own sample of
the workload) and on one core alone.

``--impl reference`` times that same oracle sample as the reference arm
(rank 0 only).

Prints ONE JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import contextlib
import gc
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "state-update tokens/s (B*steps/s)"
UNIT = "tokens/s"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0   # burst cuBLAS bf16 GEMM, an earlier B200 measurement



@contextlib.contextmanager
def no_gc():
    """The Python collector off inside a timed region: a full collection can
    stall the launching thread for milliseconds, long enough to drain the
    GPU's queue of short launches."""
    was = gc.isenabled()
    gc.collect()
    gc.disable()
    try:
        yield
    finally:
        if was:
            gc.enable()

def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["deltalog", "reference"], default="deltalog")
    ap.add_argument("--op", choices=["gdn", "kda", "rwkv6"], default="gdn")
    ap.add_argument("--B", type=int, default=256)
    ap.add_argument("--H", type=int, default=32)
    ap.add_argument("--dk", dest="d", type=int, default=128, help="d_k = d_v")
    ap.add_argument("--M", type=int, default=8,
                    help="merge interval; 0 = the library's choice for the op and shape (dl_suggest_m)")
    ap.add_argument("--tokens", type=int, default=256, help="decode tokens per bench step")
    ap.add_argument("--pool", type=int, default=64, help="distinct input tokens kept on device")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-eager", action="store_true")
    ap.add_argument("--sweep", default="",
                    help="extra M values to time, e.g. 1,4,16 (default for the metric's headline: 4,16)")
    ap.add_argument("--headline-only", action="store_true",
                    help="time only the given workload (no other workloads of the metric, no M sweep)")
    ap.add_argument("--kernel", choices=["auto", "register"], default="auto",
                    help="dl_step kernel variant")
    ap.add_argument("--tiles", type=int, default=0, choices=[0, 1, 2, 4],
                    help="value tiles per head of the register step kernel (0 = automatic)")
    ap.add_argument("--no-pdl", action="store_true",
                    help="launch every step with plain stream ordering")
    ap.add_argument("--prefill-kernel", choices=["auto", "recurrent", "chunked"], default="auto",
                    help="kernel behind dl_prefill (with --prefill)")
    ap.add_argument("--pcie", action="store_true",
                    help="measure pinned host<->device copy bandwidth (the bound of the e2e line) "
                         "and print one JSON line")
    ap.add_argument("--prefill", type=int, default=0, metavar="L",
                    help="time the prefill hand-off (dl_prefill) of B prompts of L tokens instead "
                         "of decode; one JSON line, ALU roofline")
    ap.add_argument("--log-b-bf16", action="store_true",
                    help="store GDN/KDA log value factors b_i in bf16 (DL_OPT_LOG_B_BF16)")
    ap.add_argument("--log-lam-f16", action="store_true",
                    help="store KDA/RWKV6 per-key decay metadata as fp16 log-gates (DL_OPT_LOG_LAM_F16)")
    ap.add_argument("--slot-map", action="store_true",
                    help="run every token through the slot index map: batch row r on slot perm_t[r], "
                         "a fresh random permutation of the B slots per pool token")
    ap.add_argument("--admit-every", type=int, default=0, metavar="K",
                    help="re-admit one slot (dl_slot_load of a fresh state, round robin) every K "
                         "tokens inside the timed region (serving churn; 0 = off)")
    ap.add_argument("--graph", action="store_true",
                    help="replay each M-token cycle from a CUDA graph instead of launching from Python")
    ap.add_argument("--grid", default="",
                    help="B x M sweep, e.g. '1,16,64,256,1024x1,2,4,8,16,32': one JSON line per "
                         "point (CUDA graphs; M=1 is the eager kernel)")
    args = ap.parse_args()
    if args.grid or args.prefill or args.pcie:
        return args
    if args.admit_every and args.graph:
        ap.error("--admit-every runs the Python launch loop")
    args.m_auto = args.M == 0
    if args.m_auto:
        from recurrent_state_update_deltalog_b200 import suggest_m
        args.M = suggest_m(args.op, args.d, args.d)
        args.tokens = -(-args.tokens // args.M) * args.M
    if args.tokens % args.M:
        ap.error("--tokens must be a multiple of --M")
    return args


def workload_name(a):
    tail = "_logb_bf16" if getattr(a, "log_b_bf16", False) and a.op != "rwkv6" else ""
    tail += "_lam_f16" if getattr(a, "log_lam_f16", False) and a.op != "gdn" else ""
    return f"{a.op}_decode_b{a.B}_h{a.H}_d{a.d}_m{a.M}_bf16{tail}"


# ---------------------------------------------------------------------------
# algorithmic bytes (what the method must move; no cache effects)
# ---------------------------------------------------------------------------

def entry_bytes(op, dk, dv, es=2, bb=None, lb=4):
    """Bytes of one log entry: a_i (input dtype) + b_i + Lam_i.  bb: bytes of
    one b_i element (default: the input dtype for RWKV6, fp32 otherwise); lb:
    bytes of one per-key Lam element (4, or 2 for fp16 log-gates)."""
    a = dk * es
    b = dv * (bb or (es if op == "rwkv6" else 4))
    lam = 4 if op == "gdn" else lb * dk
    return a + b + lam


def launch_bytes(op, kind, B, H, dk, dv, n=0, es=2, bb=None, lb=4):
    """Algorithmic HBM bytes of one launch over all B*H (slot, head) units.

    kind: "append" (n entries in the log), "merge" (n entries before the step),
    "eager".  Per unit: state read 4*dk*dv (+ write on merge/eager), q/k/v in,
    o out, gates, the n log entries read (deferred only) and the appended entry
    (append only).  The RWKV6 bonus u[H, dk] is read once per launch.
    """
    unit = 4 * dk * dv
    if kind in ("merge", "eager"):
        unit += 4 * dk * dv
    unit += (2 * dk + dv) * es + dv * es                      # q|r, k, v in; o out
    unit += {"gdn": 8, "kda": 4 * dk + 4, "rwkv6": 4 * dk}[op]  # gates
    if kind != "eager":
        unit += n * entry_bytes(op, dk, dv, es, bb, lb)
    if kind == "append":
        unit += entry_bytes(op, dk, dv, es, bb, lb)
    total = unit * B * H
    if op == "rwkv6":
        total += H * dk * 4
    return total


def step_bytes(op, B, H, d, M, tokens, es=2, bb=None, lb=4):
    if M == 1:
        return tokens * launch_bytes(op, "eager", B, H, d, d, 0, es)
    per_cycle = sum(launch_bytes(op, "append", B, H, d, d, n, es, bb, lb) for n in range(M - 1))
    per_cycle += launch_bytes(op, "merge", B, H, d, d, M - 1, es, bb, lb)
    return per_cycle * (tokens // M)


def write_bytes_per_token(op, B, H, d, M, es=2, bb=None, lb=4):
    """Algorithmic HBM write bytes per slot-token (all heads), averaged over a cycle."""
    state_w = 4 * d * d
    io_w = d * es
    if M == 1:
        return H * (state_w + io_w)
    ent = entry_bytes(op, d, d, es, bb, lb)
    per_cycle = (M - 1) * (io_w + ent) + (io_w + state_w)
    return H * per_cycle / M


# ---------------------------------------------------------------------------
# multi-rank plumbing (one process per GPU; replicas, weak scaling)
# ---------------------------------------------------------------------------

def rank_seed(seed, rank):
    """Each rank is an independent replica with its own B slots and inputs."""
    return seed + 1000 * rank


def reduce_max(x, world, device):
    """Max of a per-rank float over all ranks (the job's time is its slowest rank)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(B, tokens, steps, world, max_ms):
    """Whole-job throughput: every rank's slot-tokens over the slowest rank's time."""
    return B * tokens * steps * world / (max_ms / 1e3)


# ---------------------------------------------------------------------------
# environment helpers
# ---------------------------------------------------------------------------

def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# the sources that define the decode step kernels and their launch geometry
STEP_KERNEL_SOURCES = ("kernels.cuh", "launch.cuh", "ptx.cuh")


def kernel_source_hash():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "recurrent_state_update_deltalog_b200", "csrc")
    for f in sorted(os.path.join(csrc, name) for name in STEP_KERNEL_SOURCES):
        with open(f, "rb") as fh:
            h.update(os.path.basename(f).encode())
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload):
    """DRAM bytes per launch of the dominant kernel from a committed ncu summary,
    or None when there is none or the kernel sources changed since."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
        e = d[workload]
        if e.get("source_hash") != kernel_source_hash():
            return None
        return e["bytes_per_launch"]
    except Exception:
        return None


class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.proc = None
        self.gpu = gpu_index

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu), "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            return None
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 8:
                continue
            try:
                sm.append(float(f[0]))
                mx = float(f[1])
            except ValueError:
                continue
            for nm, val in zip(names, f[4:8]):
                if val.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# the fp64 CPU oracle on the host cores: cpu_baseline and the reference arm
# ---------------------------------------------------------------------------

ORACLE_UNITS_PER_WORKER = 64    # (slot, head) units each worker decodes per run
ORACLE_MAX_WORKERS = 64         # host memory: ~150 MB of fp64 sample per worker


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def _oracle_worker(conn, seed, op, slots, H, d, tokens):
    """One worker process: draws its own sample (slots x H heads x tokens of the
    workload's distributions, with its own seed) once, then runs the fp64
    oracle on it whenever it is told to and replies with the seconds taken."""
    for var in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
        os.environ[var] = "1"
    import numpy as np
    from oracle import eager
    from synthetic import bonus, initial_state, sequence
    S0 = initial_state(seed, slots, H, d, d)
    seq = sequence(seed, op, slots, H, d, d, tokens, bf16=True)
    u = bonus(seed, H, d) if op == "rwkv6" else None
    conn.send("ready")
    while conn.recv() == "run":
        t = time.perf_counter()
        o, _, _ = eager(op, S0, seq, u=u)
        el = time.perf_counter() - t
        conn.send((el, bool(np.isfinite(o).all())))
    conn.close()


class OraclePool:
    """Spawned worker processes, one per core used, each holding one sample of
    the workload (ORACLE_UNITS_PER_WORKER units over one bench step of
    tokens).  A run is every worker decoding its sample at once; its time is
    wall-clock from the start signal to the last reply."""

    def __init__(self, a, workers):
        import multiprocessing as mp
        ctx = mp.get_context("spawn")
        self.workers = workers
        self.slots = max(1, ORACLE_UNITS_PER_WORKER // a.H)
        self.tokens = a.tokens
        self.conns, self.procs = [], []
        for w in range(workers):
            parent, child = ctx.Pipe()
            proc = ctx.Process(target=_oracle_worker, daemon=True,
                               args=(child, a.seed + 1 + w, a.op, self.slots, a.H, a.d, self.tokens))
            proc.start()
            child.close()
            self.conns.append(parent)
            self.procs.append(proc)
        for c in self.conns:
            if c.recv() != "ready":
                raise RuntimeError("oracle worker failed to start")

    @property
    def slot_tokens(self):
        return self.workers * self.slots * self.tokens

    def describe(self, a):
        return (f"{self.workers} worker process(es), each {self.slots} slots x {a.H} heads x {self.tokens} "
                f"tokens of {workload_name(a)} (fp64 eager recurrence; own seeded sample per worker)")

    def run(self):
        t = time.perf_counter()
        for c in self.conns:
            c.send("run")
        res = [c.recv() for c in self.conns]
        wall = time.perf_counter() - t
        if not all(ok for _, ok in res):
            raise RuntimeError("oracle produced non-finite outputs")
        return wall

    def close(self):
        for c in self.conns:
            try:
                c.send("stop")
                c.close()
            except OSError:
                pass
        for proc in self.procs:
            proc.join(timeout=30)


def cpu_baseline(a):
    """Oracle throughput on the host: every core (up to ORACLE_MAX_WORKERS)
    decoding its own sample at once, and one core alone on the same sample."""
    cores = min(host_cores(), ORACLE_MAX_WORKERS)
    one = OraclePool(a, 1)
    t1 = one.run()
    one.close()
    pool = OraclePool(a, cores)
    tn = pool.run()
    pool.close()
    return {"value": pool.slot_tokens / tn, "unit": UNIT, "cores": cores, "kind": "oracle",
            "cpu_model": cpu_model(), "host_cores": host_cores(), "sample": pool.describe(a),
            "seconds": round(tn, 3),
            "single_core": {"value": one.slot_tokens / t1, "unit": UNIT, "seconds": round(t1, 3),
                            "sample": one.describe(a)}}


def run_reference(a, rank):
    """The reference arm: the oracle as it stands on the host cores, each bench
    step one run of the cpu_baseline sample (rank 0 alone; other ranks exit)."""
    if rank != 0:
        return
    cores = min(host_cores(), ORACLE_MAX_WORKERS)
    pool = OraclePool(a, cores)
    for _ in range(a.warmup):
        pool.run()
    times = [pool.run() for _ in range(a.steps)]
    pool.close()
    total = sum(times)
    value = pool.slot_tokens * a.steps / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": a.gpus,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": 1e3 * total / a.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": workload_name(a), "op": a.op, "B": a.B, "H": a.H, "d_k": a.d,
                   "d_v": a.d, "M": a.M, "parallelism": "cpu"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "cpu_model": cpu_model(), "sample": "each step: " + pool.describe(a)},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

def run_gpu(a, rank, world, local_rank):
    import numpy as np
    import torch
    import torch.distributed as dist
    from recurrent_state_update_deltalog_b200 import DeltaLog
    from synthetic import bonus, initial_state, sequence

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    op, B, H, d, M = a.op, a.B, a.H, a.d, a.M
    seed = rank_seed(a.seed, rank)
    bb = 2 if a.log_b_bf16 else None           # b_i element bytes in the log
    lb = 2 if a.log_lam_f16 and op != "gdn" else 4   # per-key Lam element bytes in the log
    es = 2

    # inputs: a pool of distinct tokens resident in HBM (> L2), cycled
    S0 = torch.from_numpy(initial_state(seed, B, H, d, d)).to(dev)
    seq = sequence(seed, op, B, H, d, d, a.pool, bf16=True)
    first = "r" if op == "rwkv6" else "q"
    names = [first, "k", "v", "log_decay"] + ([] if op == "rwkv6" else ["beta"])
    host = {}
    dpool = {}
    for nm in names:
        t = torch.from_numpy(np.ascontiguousarray(seq[nm]))
        t = t.to(torch.bfloat16) if nm in (first, "k", "v") else t.float()
        host[nm] = t.pin_memory()
        dpool[nm] = t.to(dev)
    del seq
    u = torch.from_numpy(bonus(seed, H, d)).to(dev) if op == "rwkv6" else None
    out = torch.empty((a.pool, B, H, d), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)

    def tok_args(pool, i):
        return (pool[first][i], pool["k"][i], pool["v"][i], pool["log_decay"][i],
                pool["beta"][i] if op != "rwkv6" else None)

    perm_rng = np.random.default_rng(seed + 17)
    sidx = ([torch.from_numpy(perm_rng.permutation(B).astype(np.int32)).to(dev) for _ in range(a.pool)]
            if a.slot_map else None)

    def tok_map(i):
        return {"slot_idx": sidx[i]} if sidx else {}

    def make_handle(m):
        h = DeltaLog(B, H, d, d, m, op=op, dtype=torch.bfloat16)
        h.set_step_kernel(a.kernel)
        h.set_pdl(not a.no_pdl)
        h.set_value_tiles(a.tiles)
        if a.log_b_bf16 and m > 1:
            h.set_log_b_bf16(True)
        if a.log_lam_f16 and m > 1:
            h.set_log_lam_f16(True)
        h.load_state(S0)
        if u is not None:
            h.set_bonus(u)
        return h

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    def max_over_ranks(x):
        return reduce_max(x, world, dev)

    tok_counter = [0]
    used_kernel = [None]

    def run_step(h, m, eager=False, ev=None, rec=None):
        """One bench step: a.tokens decode tokens through dl_step (or dl_eager_step).
        With `ev`, each cycle's run of append launches (log lengths 0 .. m-2) is
        bracketed by one pair of events, kept in `rec`: the appends keep their
        programmatic-launch overlap inside the run, and the run ends where the
        merge (which never overlaps its predecessor's state) begins."""
        seg = None
        for j in range(a.tokens):
            i = tok_counter[0] % a.pool
            tok_counter[0] += 1
            args = tok_args(dpool, i)
            if eager:
                h.eager_step(*args, out=out[i], stream=stream, **tok_map(i))
                continue
            n = j % m
            if ev is not None and n == 0 and m > 1:
                seg = ev.pop()
                seg[0].record(stream)
            h.step(*args, out=out[i], stream=stream, **tok_map(i))
            if seg is not None and n == m - 2:
                seg[1].record(stream)
                rec.append((seg[0], seg[1], list(range(m - 1))))
                seg = None
            if a.admit_every and not eager and tok_counter[0] % a.admit_every == 0:
                b = (tok_counter[0] // a.admit_every) % B
                h.slot_load(b, S0[b], stream=stream)

    def build_graphs(h, m, eager):
        """One CUDA graph per m-token cycle of the input pool (8 tokens for the
        eager kernel); the log is empty at every cycle boundary, so each graph
        replays a complete append...merge cycle."""
        cyc = 8 if eager else m
        gs = torch.cuda.Stream(dev)
        graphs = []
        with torch.cuda.stream(gs):
            for c in range(max(1, a.pool // cyc)):
                gr = torch.cuda.CUDAGraph()
                with torch.cuda.graph(gr, stream=gs):
                    for j in range(cyc):
                        i = (c * cyc + j) % a.pool
                        fn = h.eager_step if eager else h.step
                        fn(*tok_args(dpool, i), out=out[i], stream=gs, **tok_map(i))
                graphs.append(gr)
        torch.cuda.synchronize(dev)
        return graphs, cyc

    def run_graph_step(graphs, cyc):
        for _ in range(a.tokens // cyc):
            graphs[tok_counter[0] % len(graphs)].replay()
            tok_counter[0] += 1

    def timed(m, eager=False, per_launch=False):
        """Time a.steps bench steps (or, with per_launch, a shorter second pass in
        which each cycle's run of append launches is bracketed by one pair of
        events: the average append duration of the dominant kernel)."""
        h = make_handle(m)
        if a.graph and not per_launch:
            graphs, cyc = build_graphs(h, m, eager)
            for _ in range(a.warmup):
                run_graph_step(graphs, cyc)
            start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            barrier()
            with no_gc():
                start.record(stream)
                for _ in range(a.steps):
                    run_graph_step(graphs, cyc)
                stop.record(stream)
                barrier()
            ms = start.elapsed_time(stop)
            if not eager:
                used_kernel[0] = h.last_step_kernel
            h.check_device(stream)
            del graphs
            h.close()
            return max_over_ranks(ms), None
        for _ in range(a.warmup):
            run_step(h, m, eager)
        steps = min(a.steps, 2) if per_launch else a.steps
        nev = steps * (a.tokens // m + 1) if per_launch else 0
        rec = []
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(nev)]
        start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        with no_gc():
            start.record(stream)
            for _ in range(steps):
                run_step(h, m, eager, ev if per_launch else None, rec)
            stop.record(stream)
            barrier()
        ms = start.elapsed_time(stop)
        launches = None
        if per_launch:
            launches = [(e0.elapsed_time(e1), ns) for e0, e1, ns in rec]
        if not eager:
            used_kernel[0] = h.last_step_kernel
        h.check_device(stream)
        h.close()
        return max_over_ranks(ms), launches

    peak, peak_kind = measured_peak()
    result = {}

    # headline: DeltaLog at M over the timed region (no events between launches);
    # in a B x M grid, M = 1 stands for the eager kernel
    eager_head = bool(getattr(a, "eager_headline", False))
    sampler = ClockSampler(local_rank)
    sampler.start()
    ms, _ = timed(M, eager=eager_head)
    clocks = sampler.stop()
    # per-launch durations of the dominant (append) kernel, second pass
    launches = timed(M, per_launch=True)[1] if M > 1 and not a.graph else None
    value = job_tokens_per_s(B, a.tokens, a.steps, world, ms)
    sb = step_bytes(op, B, H, d, M, a.tokens, bb=bb, lb=lb)
    result["value"] = value
    result["ms"] = ms

    if launches:
        count = sum(len(ns) for _, ns in launches)
        dur = sum(t for t, _ in launches) / count
        alg = sum(launch_bytes(op, "append", B, H, d, d, n, bb=bb, lb=lb) for _, ns in launches for n in ns) / count
        dominant = "deltalog_step_kernel (append)"
    else:   # average over every launch of the step (graph replay or M = 1)
        dur = ms / (a.steps * a.tokens)
        alg = sb / a.tokens
        dominant = "eager_step_kernel" if eager_head else "deltalog_step_kernel (all launches)"
    achieved = alg / (dur / 1e3) / 1e9
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "traffic": profiled_traffic(workload_name(a)),
                "kernel": dominant, "avg_launch_us": dur * 1e3,
                "alg_bytes_per_launch": alg, "peak_source": peak_kind,
                "frac_of_nominal_8000": achieved / 8000.0,
                "step_gbs": sb / (ms / a.steps / 1e3) / 1e9}

    extra = {}
    if not a.no_eager:
        ems, _ = timed(1, eager=True)
        eb = step_bytes(op, B, H, d, 1, a.tokens)
        extra["eager"] = {"value": B * a.tokens * a.steps * world / (ems / 1e3), "unit": UNIT,
                          "ms_per_step": ems / a.steps,
                          "gbs": eb / (ems / a.steps / 1e3) / 1e9,
                          "frac": eb / (ems / a.steps / 1e3) / 1e9 / peak,
                          "write_bytes_per_token": write_bytes_per_token(op, B, H, d, 1)}
        extra["speedup_vs_eager"] = value / extra["eager"]["value"]
    sweep = {}
    for mv in [int(x) for x in a.sweep.split(",") if x.strip()]:
        if a.tokens % mv:
            continue
        sms, _ = timed(mv)
        sbb = step_bytes(op, B, H, d, mv, a.tokens, bb=bb, lb=lb)
        gbs = sbb / (sms / a.steps / 1e3) / 1e9
        sweep[str(mv)] = {"value": B * a.tokens * a.steps * world / (sms / 1e3),
                          "ms_per_step": sms / a.steps, "gbs": gbs, "frac": gbs / peak,
                          "write_bytes_per_token": write_bytes_per_token(op, B, H, d, mv, bb=bb, lb=lb)}
    if sweep:
        extra["sweep"] = sweep

    # end to end: host (pinned) inputs -> dl_step_host -> host outputs, every token
    e2e = None
    if not a.no_e2e:
        h = make_handle(M)
        h.set_host_prefetch(True)   # host inputs are ready when each call is made
        hout = torch.empty((B, H, d), dtype=torch.bfloat16).pin_memory()

        def host_step():
            for j in range(a.tokens):
                i = tok_counter[0] % a.pool
                tok_counter[0] += 1
                h.step_host(*tok_args(host, i), out=hout, stream=stream)

        for _ in range(a.warmup):
            host_step()
        start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        with no_gc():
            start.record(stream)
            for _ in range(a.steps):
                host_step()
            stop.record(stream)
            barrier()
        e_ms = max_over_ranks(start.elapsed_time(stop))
        h.close()
        h2d = sum(host[nm][0].numel() * host[nm].element_size() for nm in names) * a.tokens
        d2h = hout.numel() * hout.element_size() * a.tokens   # written by the kernel over PCIe
        e2e = {"value": B * a.tokens * a.steps * world / (e_ms / 1e3), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "api": "dl_step_host, pinned host buffers: uploads prefetched on the handle's copy "
                      "stream, o written by the kernel into pinned host memory"}

    if rank != 0:
        return None
    line = {
        "metric": METRIC, "value": result["value"], "unit": UNIT, "n_gpus": world,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": result["ms"] / a.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": workload_name(a), "op": op, "B": B, "H": H, "d_k": d, "d_v": d,
                   "M": M, "state": "fp32", "inputs": "bf16", "tokens_per_step": a.tokens,
                   "step_kernel": used_kernel[0], "pdl": not a.no_pdl, "value_tiles": a.tiles or "auto",
                   "launch": "cuda graph per cycle" if a.graph else "python loop",
                   "m_choice": "dl_suggest_m" if getattr(a, "m_auto", False) else "given",
                   "admit_every_tokens": a.admit_every or None,
                   "slot_map": "random permutation per token" if a.slot_map else None,
                   "log_b": "bf16" if (a.log_b_bf16 or op == "rwkv6") else "fp32",
                   "log_lam": "fp32 scalar" if op == "gdn" else ("fp16 log-gates" if a.log_lam_f16 else "fp32"),
                   "input_pool_tokens": a.pool, "seed": a.seed,
                   "l2": (f"inputs larger than L2 (state {4 * B * H * d * d / 1e6:.0f} MB)"
                          if 4 * B * H * d * d > L2_BYTES else
                          f"state {4 * B * H * d * d / 1e6:.1f} MB fits in L2: HBM figures undercount"),
                   "parallelism": "replicas" if world == 1 else f"replicas x{world} (B per rank)"},
        "roofline": roofline,
        "gpu_launches": a.steps * a.tokens,
        "write_bytes_per_token": write_bytes_per_token(op, B, H, d, M, bb=bb, lb=lb),
        "clocks": clocks,
        "e2e": e2e,
    }
    line.update(extra)
    return line


# The metric's workloads beside its headline (GDN B=256 H=32 d=128, M=8):
# KDA and RWKV6 at their decode configurations, and the headline's M sweep.
METRIC_HEADLINE = {"op": "gdn", "B": 256, "H": 32, "d": 128, "M": 8}
METRIC_WORKLOADS = [{"op": "kda", "B": 128, "H": 32, "d": 128, "M": 8},
                    {"op": "rwkv6", "B": 128, "H": 64, "d": 64, "M": 8},
                    {"op": "kda", "B": 128, "H": 32, "d": 128, "M": 8, "log_lam_f16": True},
                    {"op": "rwkv6", "B": 128, "H": 64, "d": 64, "M": 8, "log_lam_f16": True}]
METRIC_SWEEP = "4,16"


def is_metric_headline(a):
    """The plain headline configuration (no serving or tuning switches)."""
    return (all(getattr(a, k) == v for k, v in METRIC_HEADLINE.items()) and not a.slot_map
            and not a.admit_every and not a.graph and not a.log_b_bf16 and not a.log_lam_f16
            and a.kernel == "auto"
            and a.tiles == 0 and not a.no_pdl and not getattr(a, "m_auto", False))


def workload_summary(line):
    """The figures of one workload's line that the headline line carries."""
    r = line["roofline"]
    out = {"value": line["value"], "unit": line["unit"], "ms_per_step": line["ms_per_step"],
           "step_gbs": r["step_gbs"], "step_frac": r["step_gbs"] / r["peak"],
           "append_frac": r["frac"], "avg_append_us": r["avg_launch_us"],
           "write_bytes_per_token": line["write_bytes_per_token"], "config": line["config"],
           "clocks": line["clocks"]}
    for key in ("eager", "speedup_vs_eager", "e2e"):
        if line.get(key) is not None:
            out[key] = line[key]
    return out


def run_decode(a, rank, world, local_rank):
    """The decode bench: the headline line, plus (for the metric's headline) the
    other workloads of the metric and the M sweep in extra keys of that line,
    and the oracle on the host cores beside it."""
    import copy
    headline = is_metric_headline(a)
    if headline and not a.sweep and not a.headline_only:
        a.sweep = METRIC_SWEEP
    line = run_gpu(a, rank, world, local_rank)
    if headline and not a.headline_only:
        extras = {}
        for w in METRIC_WORKLOADS:
            sub = copy.copy(a)
            for k, v in w.items():
                setattr(sub, k, v)
            sub.sweep = ""
            if sub.log_lam_f16:   # the same workload with compact snapshots: no second eager or e2e run
                sub.no_eager = sub.no_e2e = True
            sub_line = run_gpu(sub, rank, world, local_rank)
            if sub_line is not None:
                extras[sub_line["config"]["workload"]] = workload_summary(sub_line)
        if line is not None:
            line["workloads"] = extras
    if line is not None and not a.no_cpu and world == 1:
        line["cpu_baseline"] = cpu_baseline(a)
    return line


def run_grid(a, rank, world, local_rank):
    """B x M sweep (one JSON line per point): CUDA-graph replay, 512-token
    steps by default, M = 1 timed on the eager kernel."""
    import copy
    bs, ms = a.grid.split("x")
    for B in [int(x) for x in bs.split(",")]:
        for M in [int(x) for x in ms.split(",")]:
            p = copy.copy(a)
            p.B, p.M, p.graph = B, M, True
            p.no_e2e, p.no_cpu, p.no_eager, p.sweep = True, True, True, ""
            p.eager_headline = M == 1
            p.tokens = -(-a.tokens // M) * M   # whole merge cycles per step
            line = run_gpu(p, rank, world, local_rank)
            if line is not None:
                line["config"]["grid_point"] = {"B": B, "M": M, "kernel": "eager" if M == 1 else "deltalog"}
                line["step_gbs"] = line["roofline"]["step_gbs"]
                print(json.dumps(line), flush=True)


def prefill_flops(op, dk, dv):
    """fp32 flops of one prefill token per head: the contraction pass (S^T k and
    S^T q for GDN/KDA, S^T r for RWKV6; one FMA = 2 flops per state element
    each) and the update pass (decay multiply, 1 flop, and rank-1 FMA, 2)."""
    return (4 if op != "rwkv6" else 2) * dk * dv + 3 * dk * dv


def chunk_prefill_flops(op, d, C):
    """Flops of the chunk form per token and head (d_k = d_v = d, chunks of C
    tokens; a multiply-add counts 2).  Tensor-core products with the state,
    2 d^2 each: W S, (scaled Q) S and the state update for GDN/KDA; (scaled R)
    S and the update for RWKV6.  Per chunk, the C x C blocks: for GDN/KDA the
    strictly lower A (C(C-1)/2 dot products of length d), the lower P
    (C(C+1)/2), the forward substitution for the 2d columns of W and U
    (C(C-1)/2 multiply-adds each) and P B (C(C+1)/2 d); for RWKV6 the strictly
    lower P, its diagonal (u (.) k_t) . r_t (2 flops per key) and P V."""
    if op == "rwkv6":
        return 4 * d * d + 2 * (C + 1) * d
    return 6 * d * d + (5 * C - 1) * d


# dense tf32 : dense bf16 tensor throughput, nominal (1.1 and 2.25 PFLOP/s)
TF32_PER_BF16 = 1.1 / 2.25


def measured_bf16_tflops():
    """Burst bf16 GEMM TFLOP/s from the measured peaks, else the fallback."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, "fallback"


def fp32_peak_tflops(sm_mhz, sms=148):
    """fp32 SIMT peak: 128 FP32 lanes per SM, one FMA (2 flops) per lane per clock."""
    return sms * 128 * 2 * sm_mhz * 1e6 / 1e12


def eager_tokenwise(a, seq, names, first, u, stream, dev):
    """The prefill's prompts token by token through the eager decode kernel:
    tokens/s and ms of one pass (after one untimed pass)."""
    import numpy as np
    import torch
    from recurrent_state_update_deltalog_b200 import DeltaLog
    op, B, H, d, L = a.op, a.B, a.H, a.d, a.prefill
    he = DeltaLog(B, H, d, d, 1, op=op, dtype=torch.bfloat16)
    if u is not None:
        he.set_bonus(u)
    dseq = {nm: torch.from_numpy(np.ascontiguousarray(seq[nm])).to(
        dev, torch.bfloat16 if nm in (first, "k", "v") else torch.float32) for nm in names}
    oe = torch.empty((B, H, d), dtype=torch.bfloat16, device=dev)

    def eager_all():
        for t in range(L):
            he.eager_step(dseq[first][t], dseq["k"][t], dseq["v"][t], dseq["log_decay"][t],
                          dseq["beta"][t] if op != "rwkv6" else None, out=oe, stream=stream)

    eager_all()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with no_gc():
        e0.record(stream)
        eager_all()
        e1.record(stream)
        torch.cuda.synchronize(dev)
    eager_ms = e0.elapsed_time(e1)
    return {"value": B * L / (eager_ms / 1e3), "unit": "tokens/s", "ms": eager_ms}


def run_prefill(a, rank, world, local_rank):
    """Prefill hand-off: B prompts of L tokens packed token-major, every row
    from a zero state into its own slot; tokens/s = B * L / time.  Beside it,
    the same tokens pushed one by one through the eager decode kernel."""
    import numpy as np
    import torch
    from recurrent_state_update_deltalog_b200 import DeltaLog
    from synthetic import bonus, sequence

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    op, B, H, d, L = a.op, a.B, a.H, a.d, a.prefill
    seed = rank_seed(a.seed, rank)
    seq = sequence(seed, op, B, H, d, d, L, bf16=True)
    first = "r" if op == "rwkv6" else "q"
    names = [first, "k", "v", "log_decay"] + ([] if op == "rwkv6" else ["beta"])
    packed = {}
    for nm in names:        # [L, B, H, ...] -> rows one after another: [B * L, H, ...]
        arr = np.ascontiguousarray(np.swapaxes(seq[nm], 0, 1)).reshape((B * L,) + seq[nm].shape[2:])
        packed[nm] = torch.from_numpy(arr).to(dev, torch.bfloat16 if nm in (first, "k", "v") else torch.float32)
    cu = torch.arange(0, (B + 1) * L, L, dtype=torch.int32, device=dev)
    u = torch.from_numpy(bonus(seed, H, d)).to(dev) if op == "rwkv6" else None
    h = DeltaLog(B, H, d, d, a.M, op=op, dtype=torch.bfloat16)
    h.set_prefill_kernel(a.prefill_kernel)
    if u is not None:
        h.set_bonus(u)
    o = torch.empty((B * L, H, d), dtype=torch.bfloat16, device=dev)
    args = tuple(packed[nm] for nm in (first, "k", "v", "log_decay")) + (packed.get("beta"),)
    stream = torch.cuda.current_stream(dev)

    def once():
        h.prefill(*args, cu_seqlens=cu, zero_state=True, out=o, stream=stream)

    for _ in range(max(a.warmup, 3)):
        once()
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(local_rank)
    sampler.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with no_gc():
        e0.record(stream)
        for _ in range(a.steps):
            once()
        e1.record(stream)
        torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    ms = e0.elapsed_time(e1) / a.steps
    h.check_device()
    tok_s = B * L / (ms / 1e3)
    sm = (clocks or {}).get("sm_mhz") or 1965.0
    if h.last_prefill_kernel == "chunked":
        # every chunked kernel takes 32-token chunks
        C = 32
        per_th = chunk_prefill_flops(op, d, C)
        bf16, kind = measured_bf16_tflops()
        peak = bf16 * TF32_PER_BF16
        roof = {"bound": "tensor", "peak_note": f"tf32 dense: {kind} bf16 GEMM x {TF32_PER_BF16:.3f} "
                "(nominal 1.1 / 2.25 PFLOP/s)", "chunk_tokens": C}
    else:
        per_th = prefill_flops(op, d, d)
        peak = fp32_peak_tflops(1965.0)
        roof = {"bound": "alu", "peak_note": "fp32 SIMT at the 1965 MHz max clock: 148 SMs x 128 lanes x 2 flops"}
    flops = per_th * H * B * L / (ms / 1e3) / 1e12

    # baseline: the same prompts token by token through the eager decode kernel
    # (skipped with --no-eager)
    eager = None
    if not a.no_eager:
        eager = eager_tokenwise(a, seq, names, first, u, stream, dev)
    line = {
        "metric": "prefill tokens/s (B*L/s)", "value": tok_s, "unit": "tokens/s", "n_gpus": world,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": f"{op}_prefill_b{B}_l{L}_h{H}_d{d}_bf16", "op": op, "B": B, "L": L,
                   "H": H, "d_k": d, "d_v": d, "state": "fp32", "inputs": "bf16",
                   "start": "zero state", "kernel": h.last_prefill_kernel},
        "roofline": {"bound": roof["bound"], "achieved": flops, "peak": peak, "unit": "TFLOP/s",
                     "frac": flops / peak, "traffic": None, **{k: v for k, v in roof.items() if k != "bound"},
                     "flops_per_token_head": per_th, "sm_mhz": sm},
        "eager_tokenwise": eager,
        "clocks": clocks, "gpu_launches": a.steps,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_pcie(a, local_rank):
    """Pinned host <-> device copy bandwidth for the copy sizes the e2e line
    moves (20 back-to-back copies per size, CUDA events)."""
    import torch
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    out = {}
    for nbytes in (256 << 10, 2 << 20, 6 << 20, 64 << 20):
        hb = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
        db = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        res = {}
        for name, dst, src in (("h2d", db, hb), ("d2h", hb, db)):
            for _ in range(3):
                dst.copy_(src, non_blocking=True)
            torch.cuda.synchronize(dev)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(20):
                dst.copy_(src, non_blocking=True)
            e1.record()
            torch.cuda.synchronize(dev)
            res[name + "_gbs"] = nbytes * 20 / (e0.elapsed_time(e1) / 1e3) / 1e9
        out[f"{nbytes / 1e6:.2f}MB"] = res
    print(json.dumps({"metric": "pinned copy GB/s", "copies": out}), flush=True)


def main():
    a = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if a.impl == "reference":
        run_reference(a, rank)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        if a.grid:
            run_grid(a, rank, world, local_rank)
        elif a.prefill:
            run_prefill(a, rank, world, local_rank)
        elif a.pcie:
            if rank == 0:
                run_pcie(a, local_rank)
        else:
            line = run_decode(a, rank, world, local_rank)
            if line is not None:
                print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
