"""Benchmark: batched speculative-sampling verification on B200.

One step = one ``spec_verify`` call over one batch of synthetic inputs (every
row of the workload read once: target [B,k+1,V], draft [B,k,V]).  Metric:
verified draft positions per second (B*k per step) and logit GB/s, with the
verify kernel's achieved HBM bandwidth against the measured copy peak.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...   # the fp64 CPU oracle on host cores

Multi-GPU (torchrun, one process per GPU): every rank verifies its own
batch (independent replicas, no data-path collective); the JSON line reports
the units of all ranks over the slowest rank's device time.
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

L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
SPEC_HBM_GBS = 8000.0  # B200 HBM3e data-sheet bandwidth, for the fraction of the spec figure
PROFILE_DIR = os.path.join(ROOT, "profiles")
KSAMPLES = 40  # event-bracketed launches of the streaming kernel per workload

# sources that define the streaming kernel (the one the roofline figures describe)
KERNEL_SOURCES = [os.path.join(ROOT, "draft_token_verification_verify_b200", "csrc", f)
                  for f in ("sv_rows.cuh", "sv_common.cuh", "sv_ptx.cuh")]
# and the output projection kernel
HEAD_SOURCES = [os.path.join(ROOT, "draft_token_verification_verify_b200", "csrc", f)
                for f in ("sv_head.cuh", "sv_ptx.cuh")]

WORKLOAD_ORDER = ("batched", "greedy", "large", "single", "tiny")
GRAPH_WORKLOADS = ("single", "tiny")  # launch-bound: also timed from a CUDA-graph replay
# the further processors on top of a workload: (workload, feature), reported as
# "workload+feature" beside the five workloads
FEATURES = (("batched", "mask+penalty"), ("batched", "top_p"), ("single", "top_p"))
DESCR = {
    "tiny": "tiny stochastic verify B=1 k=4 V=32 fp32 T=1",
    "single": "single-sequence stochastic verify B=1 k=8 V=151936 bf16 T=1",
    "batched": "batched stochastic verify B=64 k=4 V=151936 bf16 T=0.7 top-k 50",
    "greedy": "batched greedy verify B=256 k=8 V=151936 bf16",
    "large": "large-batch stochastic verify B=512 k=3 V=128256 fp32 T in {0.5,1,1.5}",
}


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def rank_seed(rank: int) -> int:
    """Seed of a rank's batch: every rank verifies its own, independent batch."""
    return 1000 + rank


def max_over_ranks(ms: float, device=None) -> float:
    """The slowest rank's time (MAX all-reduce); unchanged without a process group."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return ms
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_rank: float, world: int, ms: float) -> float:
    """Whole-job throughput: the units of all ranks over the slowest rank's time."""
    return units_per_rank * world / (ms / 1000.0)


def measured_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_hash(sources=None) -> str:
    h = hashlib.sha256()
    for p in (KERNEL_SOURCES if sources is None else sources):
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str, kernel: str = "sv_rows_kernel", sources=None):
    """DRAM bytes per launch from the committed ncu summary of `kernel` on
    `workload`, if it was taken on the current kernel source (else None)."""
    path = os.path.join(PROFILE_DIR, f"{kernel}_{workload}.md")
    if not os.path.exists(path):
        return None
    vals = {}
    for line in open(path):
        if line.startswith("- ") and ":" in line:
            k, v = line[2:].split(":", 1)
            vals[k.strip()] = v.strip().strip("`")
    if vals.get("kernel_source_sha256_16") != kernel_source_hash(sources):
        return None
    try:
        return float(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi clock / throttle sampling while the GPU is busy."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], [], set()
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for name, val in zip(("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                                  "sw_power_cap"), f[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


def pctl(xs, q: float) -> float:
    """Nearest-rank percentile ``q`` (0..100) of a non-empty sequence."""
    s = sorted(xs)
    return s[min(len(s) - 1, max(0, math.ceil(q / 100.0 * len(s)) - 1))]


def launches_per_step(case, feature=None) -> int:
    """Kernels one spec_verify call launches: the streaming pass and the
    per-sequence kernel, plus the residual segment kernel for stochastic
    verification without top-k; the processors add their bitmap kernel, a
    nucleus without top-k its cut kernel."""
    stochastic_softmax = case.mode != "greedy" and not (0 < case.top_k < case.V)
    n = 3 if stochastic_softmax else 2
    if feature == "mask+penalty":
        n += 1
    if feature == "top_p" and stochastic_softmax:
        n += 1
    return n


def feature_tensors(feature, case, dev, seed):
    """Device tensors of a feature's options (kept alive by the caller)."""
    import torch

    if feature is None:
        return {}
    pr = workloads.make_processors(seed, case.B, case.V, top_p=(0.7, 0.95))
    t = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a).view(dt)).to(dev)
    if feature == "top_p":
        return {"top_p": t(pr.top_p, np.float32)}
    return {"vocab_mask": t(pr.mask, np.int32), "rep_ids": t(pr.rep_ids, np.int32),
            "rep_penalty": t(pr.rep_penalty, np.float32)}


def to_dev(a, device):
    import torch

    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(a).to(device)


def to_pinned(a):
    import torch

    a = np.ascontiguousarray(a)
    t = torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a)
    t = t.pin_memory()
    return t.view(torch.bfloat16) if a.dtype == np.uint16 else t


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


# Sequences per oracle step and worker: enough work per step that the barrier
# between steps does not dominate.
ORACLE_REPS = {"tiny": 2000, "single": 1, "batched": 1, "greedy": 4, "large": 1}


def _oracle_worker(name: str, worker: int, barrier, stop, out):
    """Spawned process: builds a one-sequence case of the workload (its own
    seed), then verifies it ORACLE_REPS[name] times per step, in lockstep with
    the parent through ``barrier``, until ``stop`` is set."""
    import oracle

    case = workloads.make_case(name, seed=7000 + worker, B=1)
    drafts = oracle.draft_tokens_for(case)
    greedy = case.mode == "greedy"
    reps = ORACLE_REPS[name]
    barrier.wait()  # set-up done
    steps = 0
    while True:
        barrier.wait()
        if stop.value:
            break
        for _ in range(reps):
            oracle.verify(case.target, None if greedy else case.draft, drafts,
                          None if greedy else case.uniforms, case.temperature, case.top_k, greedy)
        barrier.wait()
        steps += 1
    out.put((worker, steps))


class OracleRunner:
    """The fp64 oracle, as it stands, on every host core: one spawned process
    per core (spawn, so it is safe after CUDA has been initialised in this
    process), each verifying its own sequence of the workload; a step is one
    round of ORACLE_REPS sequences on every core, timed by the parent."""

    def __init__(self, name: str, workers: int):
        import multiprocessing as mp

        ctx = mp.get_context("spawn")
        self.name = name
        self.workers = workers
        self.barrier = ctx.Barrier(workers + 1)
        self.stop = ctx.Value("i", 0)
        self.out = ctx.Queue()
        self.procs = [ctx.Process(target=_oracle_worker, args=(name, w, self.barrier, self.stop, self.out))
                      for w in range(workers)]
        for p in self.procs:
            p.start()
        self.barrier.wait(timeout=300)  # every worker has its case

    def step(self):
        self.barrier.wait(timeout=300)
        self.barrier.wait(timeout=300)

    def close(self):
        self.stop.value = 1
        try:
            self.barrier.wait(timeout=60)
        except Exception:
            pass
        for p in self.procs:
            p.join(timeout=60)
            if p.is_alive():
                p.terminate()

    def sequences_per_step(self) -> int:
        return self.workers * ORACLE_REPS[self.name]


def cpu_baseline_single(name: str, case, drafts, budget_s: float, why: str):
    """The oracle on one thread, sequence after sequence of the batch (used when
    the multi-process run cannot be set up)."""
    import oracle

    greedy = case.mode == "greedy"
    done, t0 = 0, time.perf_counter()
    while done < case.B:
        sl = slice(done, done + 1)
        oracle.verify(case.target[sl], None if greedy else case.draft[sl], drafts[sl],
                      None if greedy else case.uniforms[sl], case.temperature[sl], case.top_k, greedy)
        done += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": done * case.k / dt, "unit": "positions/s", "cores": 1, "kind": "oracle",
            "sample": f"{done} of {workloads.WORKLOADS[name].B} sequences of the {name} workload "
                      f"({DESCR[name]}), single thread, {dt:.1f} s ({why})"}


def cpu_baseline(name: str, budget_s: float):
    """The oracle on every host core, for about ``budget_s`` seconds."""
    k = workloads.WORKLOADS[name].k
    run = OracleRunner(name, host_cores())
    try:
        run.step()  # warm-up
        steps, t0 = 0, time.perf_counter()
        while time.perf_counter() - t0 < budget_s:
            run.step()
            steps += 1
        dt = time.perf_counter() - t0
    finally:
        run.close()
    seqs = steps * run.sequences_per_step()
    return {"value": seqs * k / dt, "unit": "positions/s", "cores": run.workers, "kind": "oracle",
            "sample": f"{seqs} sequences of the {name} workload shape ({DESCR[name]}), one per core "
                      f"per step on {run.workers} processes, {dt:.1f} s"}


def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    name = args.workload
    k = workloads.WORKLOADS[name].k
    try:
        run = OracleRunner(name, host_cores())
        try:
            for _ in range(args.warmup):
                run.step()
            t0 = time.perf_counter()
            for _ in range(args.steps):
                run.step()
            dt = time.perf_counter() - t0
        finally:
            run.close()
        per_step, cores = run.sequences_per_step(), run.workers
        sample = (f"{per_step} sequence(s) of the {name} workload shape per step, one per core on "
                  f"{cores} processes")
    except Exception as exc:  # the multi-process run failed: the same steps on one thread
        import oracle

        case = workloads.make_case(name, seed=7000, B=1)
        drafts = oracle.draft_tokens_for(case)
        greedy = case.mode == "greedy"
        per_step, cores = ORACLE_REPS[name], 1

        def one_step():
            for _ in range(per_step):
                oracle.verify(case.target, None if greedy else case.draft, drafts,
                              None if greedy else case.uniforms, case.temperature, case.top_k, greedy)

        for _ in range(args.warmup):
            one_step()
        t0 = time.perf_counter()
        for _ in range(args.steps):
            one_step()
        dt = time.perf_counter() - t0
        sample = (f"{per_step} sequence(s) of the {name} workload shape per step, single thread "
                  f"(multi-process run failed: {type(exc).__name__})")
    value = args.steps * per_step * k / dt
    line = {
        "impl": "reference", "metric": "verified draft positions/sec", "value": value,
        "unit": "positions/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000 * dt / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": DESCR[name], "sample_per_step": f"{per_step} sequence(s)"},
        "cpu_baseline": {"value": value, "unit": "positions/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "positions/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def measure_workload(name, args, sv, dev, world, rank, local, e2e_leg=False, feature=None):
    """Time one workload: K steps bracketed by synchronize (and a barrier plus
    the max over ranks under torchrun), the streaming kernel alone from CUDA
    events over its own KSAMPLES launches, clocks sampled while the same steps
    run, and optionally the end-to-end leg and a CUDA-graph replay.  With a
    feature the proposer's draw and the verification take its options."""
    import torch

    case = workloads.make_case(name, seed=rank_seed(rank))
    ftens = feature_tensors(feature, case, dev, rank_seed(rank))
    B, k, V = case.B, case.k, case.V
    greedy = case.mode == "greedy"
    mode = (sv.SV_MODE_GREEDY if greedy else sv.SV_MODE_STOCHASTIC) | (
        sv.SV_DTYPE_BF16 if case.dtype == "bf16" else sv.SV_DTYPE_F32)
    logit_bytes = case.logit_bytes()

    target0 = to_dev(case.target, dev)
    draft0 = None if greedy else to_dev(case.draft, dev)
    unif = None if greedy else to_dev(case.uniforms, dev)
    temp = to_dev(case.temperature, dev)
    # the proposer's tokens, drawn on the GPU by the library's sampler (untimed)
    if greedy:
        drafts = sv.sample(to_dev(case.draft_proxy, dev), greedy=True)
    else:
        drafts = sv.sample(draft0, to_dev(case.draft_uniforms, dev), temp.repeat_interleave(k), case.top_k,
                           opts=sv.make_options(rows_per_sequence=k, **ftens) if ftens else None)
    torch.cuda.synchronize()

    # rotate input sets so that consecutive steps never hit in L2
    nsets = max(2, -(-4 * L2_BYTES // logit_bytes)) if logit_bytes < 4 * L2_BYTES else 1
    nsets = min(nsets, 64)
    targets = [target0] + [target0.clone() for _ in range(nsets - 1)]
    drafts_l = [draft0] + ([draft0.clone() for _ in range(nsets - 1)] if draft0 is not None else [None] * (nsets - 1))
    out_tok = torch.empty((B, k + 1), dtype=torch.int32, device=dev)
    out_n = torch.empty((B,), dtype=torch.int32, device=dev)
    status = torch.zeros((1,), dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()
    base_opts = sv.make_options(**ftens) if ftens else None
    wbytes = sv.spec_verify_workspace_size(B, k, V, case.top_k, mode, base_opts)
    wsp = torch.empty((max(wbytes, 1),), dtype=torch.uint8, device=dev)

    def step(i, ev0=None, ev1=None, on=None):
        opts = sv.make_options(event_start=ev0, event_stop=ev1, **ftens) if ev0 is not None else base_opts
        st = sv.spec_verify_ex(targets[i % nsets], drafts_l[i % nsets], drafts, unif, B, k, V, temp,
                               case.top_k, mode, out_tok, out_n, None, None, status, wsp, wbytes, opts,
                               stream if on is None else on)
        if st != sv.SV_OK:
            raise sv.SpecVerifyError(st, "spec_verify_ex")

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    if int(status.item()) != 0:
        raise SystemExit(f"{name}: device status {int(status.item())} during warm-up")

    # clock window: the same work back to back while nvidia-smi samples
    sampler = ClockSampler(local)
    sampler.start()
    t_end = time.perf_counter() + args.clock_window
    i = 0
    while time.perf_counter() < t_end:
        for _ in range(32):
            step(i)
            i += 1
        torch.cuda.synchronize()

    # ---- timed region: exactly K steps, no event between the launches ---------------
    t_start = torch.cuda.Event(enable_timing=True)
    t_stop = torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t_start.record(stream)
    for s_ in range(args.steps):
        step(s_)
    t_stop.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    elapsed_ms = max_over_ranks(t_start.elapsed_time(t_stop), dev)
    if int(status.item()) != 0:
        raise SystemExit(f"{name}: device status {int(status.item())} in the timed region")

    # ---- the streaming kernel alone: an event pair around it on KSAMPLES steps ------
    # (an event between the two launches of a step stops the second from starting
    # early, so these steps are timed apart from the K above)
    evk = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(KSAMPLES)]
    for a, b in evk:  # torch creates the CUDA event on first record
        a.record(stream)
        b.record(stream)
    torch.cuda.synchronize()
    for j_, (a, b) in enumerate(evk):
        step(args.steps + j_, a, b)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    kern_ms = [a.elapsed_time(b) for a, b in evk]
    if int(status.item()) != 0:
        raise SystemExit(f"{name}: device status {int(status.item())} in the kernel samples")

    value = job_rate(B * k * args.steps, world, elapsed_ms)
    gbs = job_rate(logit_bytes * args.steps, world, elapsed_ms) / 1e9
    kmean = sum(kern_ms) / len(kern_ms)
    peak, peak_src = measured_peak()
    achieved = logit_bytes / (kmean / 1000.0) / 1e9
    out = {
        "workload": DESCR[name] + (f", {feature}" if feature else ""), "B": B, "k": k, "V": V, "top_k": case.top_k, "mode": case.mode,
        "dtype": case.dtype, "value": value, "unit": "positions/s", "steps": args.steps,
        "ms_per_step": elapsed_ms / args.steps, "logit_gbs": gbs, "logit_bytes_per_step": logit_bytes,
        "l2": f"{nsets} rotating input set(s) of {logit_bytes / 1e6:.1f} MB"
              + (" (> 126 MB L2 in rotation)" if nsets * logit_bytes > L2_BYTES else ""),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": profiled_traffic(name), "peak_source": peak_src,
                     "kernel": "sv_rows_kernel", "kernel_ms_mean": kmean,
                     "kernel_ms_median": statistics.median(kern_ms),
                     "kernel_ms_p10": pctl(kern_ms, 10), "kernel_ms_p90": pctl(kern_ms, 90),
                     "kernel_samples": len(kern_ms),
                     "frac_of_spec": achieved / SPEC_HBM_GBS, "spec_gbs": SPEC_HBM_GBS},
        "gpu_launches": launches_per_step(case, feature) * args.steps,
        "clocks": clocks,
    }

    # ---- end to end through the public API, host (pinned) buffers -------------------
    if e2e_leg:
        h_target = to_pinned(case.target)
        h_draft = None if greedy else to_pinned(case.draft)
        h_tok = drafts.cpu().pin_memory()
        h_unif = None if greedy else to_pinned(case.uniforms)
        h_temp = to_pinned(case.temperature)
        o_tok = torch.empty((B, k + 1), dtype=torch.int32).pin_memory()
        o_n = torch.empty((B,), dtype=torch.int32).pin_memory()
        d_target, d_draft = targets[0], drafts_l[0]
        d_tok = torch.empty_like(drafts)
        d_unif = None if greedy else torch.empty_like(unif)
        d_temp = torch.empty_like(temp)
        h2d = sum(x.numel() * x.element_size() for x in (h_target, h_draft, h_tok, h_unif, h_temp)
                  if x is not None)
        d2h = o_tok.numel() * 4 + o_n.numel() * 4

        def e2e_step():
            d_target.copy_(h_target, non_blocking=True)
            if h_draft is not None:
                d_draft.copy_(h_draft, non_blocking=True)
                d_unif.copy_(h_unif, non_blocking=True)
            d_tok.copy_(h_tok, non_blocking=True)
            d_temp.copy_(h_temp, non_blocking=True)
            st = sv.spec_verify(d_target, d_draft, d_tok, d_unif, B, k, V, d_temp, case.top_k, mode,
                                out_tok, out_n, stream)
            if st != sv.SV_OK:
                raise sv.SpecVerifyError(st, "spec_verify")
            o_tok.copy_(out_tok, non_blocking=True)
            o_n.copy_(out_n, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        n_e2e = max(3, min(args.steps, 20))
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        a.record(stream)
        for _ in range(n_e2e):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(a.elapsed_time(b), dev)
        out["e2e"] = {"value": job_rate(B * k * n_e2e, world, e_ms), "unit": "positions/s",
                      "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": n_e2e}

    # ---- the same steps replayed from a CUDA graph (launch-bound workloads) ---------
    if args.graph or name in GRAPH_WORKLOADS:
        gs = torch.cuda.Stream(device=dev)
        gs.wait_stream(stream)
        per_graph = 16
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=gs):
            for i in range(per_graph):
                step(i, on=gs)
        rs = torch.cuda.current_stream()  # replay() launches the graph on the current stream
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        reps = max(3, args.steps // per_graph)
        ga, gb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ga.record(rs)
        for _ in range(reps):
            g.replay()
        gb.record(rs)
        torch.cuda.synchronize()
        g_ms = max_over_ranks(ga.elapsed_time(gb), dev) / (reps * per_graph)
        out["graph"] = {"value": job_rate(B * k, world, g_ms), "unit": "positions/s", "ms_per_step": g_ms,
                        "steps_per_graph": per_graph}
        del g
    out["_drafts"] = drafts.cpu().numpy()
    out["_case"] = case
    del targets, drafts_l, target0, draft0, wsp
    torch.cuda.empty_cache()
    return out


TREE_PARENTS = (0, 0, 1, 1, 2, 2, 3, 3)  # a binary tree of 8 candidate nodes


def measure_tree(args, sv, dev, world, rank):
    """Tree verification on the batched workload's shapes and value model: B
    sequences of a binary tree of 8 candidates (one target and one draft row
    per node plus the root), each node's token drawn on the GPU from its
    parent's processed draft row; K steps bracketed by synchronize."""
    import torch

    N = len(TREE_PARENTS)
    case = workloads.make_case("batched", seed=rank_seed(rank), k=N)
    B, V = case.B, case.V
    target = to_dev(case.target, dev)                                             # [B, N+1, V]
    draft = to_dev(np.concatenate([case.draft, case.draft[:, -1:]], axis=1), dev)
    par = torch.tensor(TREE_PARENTS, dtype=torch.int32, device=dev).repeat(B, 1)
    par_rows = torch.gather(draft, 1, par.long()[:, :, None].expand(B, N, V))      # [B, N, V]
    temp = to_dev(case.temperature, dev)
    toks = sv.sample(par_rows, to_dev(case.draft_uniforms, dev), temp.repeat_interleave(N), case.top_k)
    toks = toks.view(B, N).contiguous()
    del par_rows
    unif = to_dev(case.uniforms, dev)
    set_bytes = (target.numel() + draft.numel()) * target.element_size()
    nsets = max(2, -(-4 * L2_BYTES // set_bytes))
    nsets = min(nsets, 8)
    targets = [target] + [target.clone() for _ in range(nsets - 1)]
    drafts = [draft] + [draft.clone() for _ in range(nsets - 1)]
    out_tok = torch.empty((B, N + 1), dtype=torch.int32, device=dev)
    out_n = torch.empty((B,), dtype=torch.int32, device=dev)
    mode = sv.SV_MODE_STOCHASTIC | sv.SV_DTYPE_BF16
    stream = torch.cuda.current_stream()
    wbytes = sv.spec_verify_tree_workspace_size(B, N, V, case.top_k, mode)  # the list walk's records
    ws = torch.empty((max(wbytes, 1),), dtype=torch.uint8, device=dev)

    def step(i):
        st = sv.spec_verify_tree_ex(targets[i % nsets], drafts[i % nsets], toks, par, unif, B, N, V, temp,
                                    case.top_k, mode, out_tok, out_n, None, None, None,
                                    ws if wbytes else None, wbytes, stream)
        if st != sv.SV_OK:
            raise sv.SpecVerifyError(st, "spec_verify_tree_ex")

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    sampler = ClockSampler(rank)
    sampler.start()
    t_end = time.perf_counter() + getattr(args, "clock_window", 0.0)  # the same calls while clocks are sampled
    i = 0
    while time.perf_counter() < t_end:
        for _ in range(16):
            step(i)
            i += 1
        torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    a.record(stream)
    for i in range(args.steps):
        step(i)
    b.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    ms = max_over_ranks(a.elapsed_time(b), dev)
    n_host = out_n.cpu().numpy()
    return {"workload": f"batched tree verify B={B} N={N} (binary) V={V} bf16 T=0.7 top-k {case.top_k}",
            "value": job_rate(B * N * args.steps, world, ms), "unit": "verified candidate nodes/s",
            "ms_per_step": ms / args.steps, "mean_accepted": float(n_host.mean()),
            "gpu_launches": (4 if wbytes else 1) * args.steps, "clocks": clocks,
            "path": "streaming pass + list walk" if wbytes else "walk over the rows",
            "l2": f"{nsets} rotating input set(s) of {set_bytes / 1e6:.1f} MB"}


HEAD_SHAPE = (64, 4, 151936, 4096)  # B, k, V, H: the batched shape with a 4,096-wide hidden state
FALLBACK_BF16_TFLOPS_SUSTAINED = 1400.0  # a seconds-long cuBLAS bf16 loop under the 1 kW cap


def measured_bf16_peak():
    """The dense bf16 peak for a kernel timed inside a long loop: the
    sustained figure (the clocks settle under the power cap)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops_sustained"]), "measured (sustained)"
    except Exception:
        return FALLBACK_BF16_TFLOPS_SUSTAINED, "fallback (sustained)"


def measure_head(args, sv, dev, world, rank):
    """Greedy verification fused into the output projection: B x (k+1)
    hidden states [4,096] bf16 times a [V, 4,096] bf16 weight (1.24 GB, ten
    times L2: every step streams it from HBM), the logits reduced on chip.
    Draft tokens are random (the step's time does not depend on them).  The
    projection kernel is also timed alone between an event pair on KSAMPLES
    steps."""
    import torch

    B, k, V, H = HEAD_SHAPE
    case = workloads.make_head_case(rank_seed(rank), B, k, V, H)
    hidden = to_dev(case.hidden, dev)
    weight = to_dev(case.weight, dev)
    del case
    drafts = torch.from_numpy(np.random.default_rng(rank_seed(rank)).integers(0, V, (B, k)).astype(np.int32)).to(dev)
    out_tok = torch.empty((B, k + 1), dtype=torch.int32, device=dev)
    out_n = torch.empty((B,), dtype=torch.int32, device=dev)
    status = torch.zeros((1,), dtype=torch.int32, device=dev)
    wbytes = sv.spec_verify_head_workspace_size(B, k, V, H)
    ws = torch.empty((wbytes,), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step(ev0=None, ev1=None):
        opts = sv.make_options(event_start=ev0, event_stop=ev1) if ev0 is not None else None
        st = sv.spec_verify_head_greedy(hidden, weight, drafts, B, k, V, H, out_tok, out_n, None, ws, wbytes, opts,
                                        status, stream)
        if st != sv.SV_OK:
            raise sv.SpecVerifyError(st, "spec_verify_head_greedy")

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    sampler = ClockSampler(rank)
    sampler.start()
    t_end = time.perf_counter() + getattr(args, "clock_window", 0.0)
    while time.perf_counter() < t_end:
        for _ in range(8):
            step()
        torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    a.record(stream)
    for _ in range(args.steps):
        step()
    b.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(b), dev)
    evk = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(KSAMPLES)]
    for e0, e1 in evk:
        e0.record(stream)
        e1.record(stream)
    torch.cuda.synchronize()
    for e0, e1 in evk:
        step(e0, e1)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if int(status.item()) != 0:
        raise SystemExit(f"head: device status {int(status.item())}")
    kern_ms = [e0.elapsed_time(e1) for e0, e1 in evk]
    kmean = sum(kern_ms) / len(kern_ms)
    rows = B * (k + 1)
    flops = 2.0 * rows * V * H  # the logits of every position, no padding counted
    peak, src = measured_bf16_peak()
    achieved = flops / (kmean / 1000.0) / 1e12
    w_bytes = V * H * 2
    return {"workload": f"greedy verify fused into the output projection B={B} k={k} V={V} H={H} bf16",
            "value": job_rate(B * k * args.steps, world, ms), "unit": "positions/s",
            "ms_per_step": ms / args.steps, "gpu_launches": 2 * args.steps, "clocks": clocks,
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "peak_source": src, "kernel": "sv_head_kernel",
                         "traffic": profiled_traffic("head_greedy", "sv_head_kernel", HEAD_SOURCES),
                         "kernel_ms_mean": kmean, "kernel_ms_median": statistics.median(kern_ms),
                         "kernel_samples": len(kern_ms), "flops_per_launch": flops,
                         "weight_gbs": w_bytes / (kmean / 1000.0) / 1e9, "weight_bytes": w_bytes},
            "logits_written_bytes": 0,
            "l2": f"weight {w_bytes / 1e9:.2f} GB per step (> 126 MB L2)"}


def run_ours(args):
    import torch

    import draft_token_verification_verify_b200 as sv

    world, rank, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    sv.lib()

    if args.tree_only or args.head_only:
        r = (measure_tree if args.tree_only else measure_head)(args, sv, dev, world, local)
        if world > 1:
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()
        if rank == 0:
            print(json.dumps(r), flush=True)
        return 0
    name = args.workload
    head = measure_workload(name, args, sv, dev, world, rank, local, e2e_leg=not (args.no_e2e or args.feature),
                            feature=args.feature)
    others = {}
    if not args.headline_only:
        for other in WORKLOAD_ORDER:
            if other == name:
                continue
            r = measure_workload(other, args, sv, dev, world, rank, local)
            r.pop("_drafts")
            r.pop("_case")
            others[other] = r
        for base, feature in FEATURES:
            r = measure_workload(base, args, sv, dev, world, rank, local, feature=feature)
            r.pop("_drafts")
            r.pop("_case")
            others[f"{base}+{feature}"] = r
        others["tree"] = measure_tree(args, sv, dev, world, local)
        others["head_greedy"] = measure_head(args, sv, dev, world, local)
    case, drafts = head.pop("_case"), head.pop("_drafts")

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.feature:
        try:
            cpu = cpu_baseline(name, args.cpu_budget)
        except Exception as exc:  # the multi-process leg failed: one thread instead
            cpu = cpu_baseline_single(name, case, drafts, args.cpu_budget,
                                      f"multi-process run failed: {type(exc).__name__}")
        if cpu.get("cores", 1) > 1:  # the one-core figure beside the all-core one
            try:
                one = cpu_baseline_single(name, case, drafts, args.cpu_budget / 3,
                                          "one core, beside the all-core figure")
                cpu["single_core"] = {"value": one["value"], "unit": one["unit"], "sample": one["sample"]}
            except Exception as exc:
                cpu["single_core"] = {"unavailable": f"{type(exc).__name__}: {exc}"[:200]}

    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank != 0:
        return 0
    line = {
        "metric": "verified draft positions/sec", "value": head["value"], "unit": "positions/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": head["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": head["dtype"], "data": "synthetic",
        "config": {"workload": head["workload"], "B": head["B"], "k": head["k"], "V": head["V"],
                   "top_k": head["top_k"], "mode": head["mode"], "per_rank_batch": head["B"],
                   "parallelism": f"replicas x{world}", "l2": head["l2"],
                   "clocks_window": f"sampled over a {args.clock_window:.1f} s window of the same "
                                    "steps right before the timed region and during the kernel samples"},
        "logit_gbs": head["logit_gbs"],
        "logit_bytes_per_step": head["logit_bytes_per_step"],
        "roofline": head["roofline"],
        "gpu_launches": head["gpu_launches"],
        "clocks": head["clocks"],
        "e2e": head.get("e2e"),
        **({"graph": head["graph"]} if "graph" in head else {}),
        "cpu_baseline": cpu,
        "workloads": others,
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(workloads.WORKLOADS), default="batched")
    ap.add_argument("--clock-window", type=float, default=1.0)
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--graph", action="store_true",
                    help="also time the headline's steps replayed from a CUDA graph")
    ap.add_argument("--feature", choices=sorted({f for _, f in FEATURES}), default=None,
                    help="profile a feature alone: --workload with these options (no e2e or CPU leg)")
    ap.add_argument("--tree-only", action="store_true",
                    help="measure only the tree-verification line (one JSON line; for profiling)")
    ap.add_argument("--head-only", action="store_true",
                    help="measure only the output-projection greedy line (one JSON line; for profiling)")
    ap.add_argument("--headline-only", action="store_true",
                    help="measure only --workload (default: every workload, the headline first)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
