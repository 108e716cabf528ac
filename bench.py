"""Benchmark: one attention layer-step of paged decode (pa_cache_write of the
step's new K/V + pa_decode) on a seeded synthetic batch, through the C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

`--workload block_copy` measures copy-on-write's block copy (pa_copy_blocks)
instead, as "block copy GB/s" (bytes read + written per step / step time).

Prints one JSON line (rank 0).  `value` is KV GB/s: the step's algorithmic
attention bytes (every valid token's K and V once, shared prefix blocks
once, plus queries, outputs, table entries and lengths) divided by the step
time, summed over all ranks (replicas: the path has no cross-GPU exchange).
`--impl reference` times the CPU oracle on this host's cores instead.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import pa_workloads as W  # noqa: E402

METRIC = "paged decode attention KV GB/s"
DEFAULT_WORKLOAD = "gqa_bf16"

# DRAM bytes (read + write) per launch of the workload's dominant kernel from
# one ncu capture of that kernel, valid only for the kernel source that was
# profiled (keyed by its sha256): any edit to the source drops the figure to
# null until the kernel is captured again.
PROFILED_TRAFFIC = {
    # mean of two captured launches
    "gqa_bf16": {"source": "paged_kv_cache_452_b200/csrc/decode_tc.cu",
                 "sha256": "cd0f27a759d909e8a0ef8716d84b089fa243f970d0455572d34a677985fcd520",
                 "bytes": 293_273_344},
    # captured on the first 16 of fp8_long's 128 sequences (the full pools are
    # too large for a multi-pass capture) and scaled by the algorithmic bytes
    "fp8_long": {"source": "paged_kv_cache_452_b200/csrc/decode_tc.cu",
                 "sha256": "cd0f27a759d909e8a0ef8716d84b089fa243f970d0455572d34a677985fcd520",
                 "bytes": 4_874_331_623},
    "prefix_bf16": {"source": "paged_kv_cache_452_b200/csrc/decode_tc.cu",
                    "sha256": "cd0f27a759d909e8a0ef8716d84b089fa243f970d0455572d34a677985fcd520",
                    "bytes": 922_697_216},
    # mean of two captured launches
    "block_copy": {"source": "paged_kv_cache_452_b200/csrc/block_copy.cu",
                   "sha256": "14c4d4e16d7a6cfba5f9139645ec9d67aba270f8986a597db740b32a1a2c0f11",
                   "bytes": 488_925_056},
}


def profiled_traffic(workload):
    import hashlib
    e = PROFILED_TRAFFIC.get(workload)
    if not e:
        return None
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), e["source"])
    try:
        with open(path, "rb") as f:
            digest = hashlib.sha256(f.read()).hexdigest()
    except OSError:
        return None
    return e["bytes"] if digest == e["sha256"] else None


KV_BYTES = {"f32": 4, "bf16": 2, "e4m3": 1}
Q_BYTES = {"f32": 4, "bf16": 2}


def algorithmic_bytes(wl):
    """Bytes the attention of one step must move at least once (HBM)."""
    bs, hkv, d = wl.block_size, wl.num_kv_heads, wl.head_dim
    seq_lens = wl.context_lens + wl.q_lens
    tokens = int(seq_lens.sum())
    if wl.sharing is not None:  # the shared prefix is stored (and read) once
        tokens -= wl.prefix_len * max(0, int(wl.sharing.sum()) - 1)
    kv = tokens * 2 * hkv * d * KV_BYTES[wl.kv_dtype]
    rows = wl.num_new_tokens
    qo = 2 * rows * wl.num_q_heads * d * Q_BYTES[wl.q_dtype]
    table = int(sum(-(-int(n) // bs) for n in seq_lens)) * 4 + 4 * wl.num_seqs
    return kv + qo + table, kv


def logical_kv_bytes(wl):
    seq_lens = wl.context_lens + wl.q_lens
    return int(seq_lens.sum()) * 2 * wl.num_kv_heads * wl.head_dim * KV_BYTES[wl.kv_dtype]


def write_bytes(wl):
    t = wl.num_new_tokens
    return t * wl.num_kv_heads * wl.head_dim * 2 * (Q_BYTES[wl.q_dtype] + KV_BYTES[wl.kv_dtype]) + 8 * t


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f), "measured"
    except OSError:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons while the timed region runs."""
    FIELDS = ["clocks.sm", "clocks.max.sm", "clocks_event_reasons.hw_slowdown",
              "clocks_event_reasons.hw_thermal_slowdown", "clocks_event_reasons.sw_thermal_slowdown",
              "clocks_event_reasons.sw_power_cap"]

    def __init__(self, index):
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(index), "--query-gpu=" + ",".join(self.FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "50"],
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
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != len(self.FIELDS):
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[2:]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup(args, backend=None):
    """One process per GPU, launched by torchrun (RANK / LOCAL_RANK /
    WORLD_SIZE / MASTER_* from the environment).  Replicas only: the process
    group carries the start/stop barriers and the max-over-ranks of the
    timings, never the data path."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        if backend is None:
            backend = "nccl" if args.impl == "ours" else "gloo"
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def job_throughput(world, bytes_per_replica, ms):
    """Whole-job GB/s: every rank streamed `bytes_per_replica` per step and
    the step took `ms` (the max over ranks)."""
    return world * bytes_per_replica / (ms * 1e-3) / 1e9


def reduce_max(x, world, device):
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def oracle_prepare(wl, seqs):
    from oracle.workload import prepare  # test infrastructure: the CPU baseline only
    return prepare(wl, seqs)


def oracle_time(prep):
    """Wall time of the oracle's own arithmetic (cache writes + attention) on
    a prepared sample; the draws and pool replay are prepared beforehand."""
    from oracle.workload import compute
    t0 = time.perf_counter()
    compute(prep)
    return time.perf_counter() - t0


def oracle_sample(wl, budget_s):
    """Sequences of the batch whose oracle evaluation takes about budget_s,
    shortest first (the cost per token is scaled from a timing of the
    shortest sequence); their KV bytes."""
    import oracle
    tokens = (wl.context_lens + wl.q_lens).astype(np.int64)
    order = [int(s) for s in np.argsort(tokens, kind="stable")]
    t = oracle_time(oracle_prepare(wl, [order[0]]))
    per_token = t / max(1, int(tokens[order[0]]))
    seqs, est = [], 0.0
    for s in order:
        n = int(tokens[s])
        if seqs and est + per_token * n > budget_s:
            break
        seqs.append(s)
        est += per_token * n
    seqs.sort()
    kv = sum(int(wl.context_lens[s] + wl.q_lens[s]) for s in seqs) * 2 * wl.num_kv_heads * wl.head_dim * \
        KV_BYTES[wl.kv_dtype]
    return oracle_prepare(wl, seqs), len(seqs), kv, oracle.max_threads()


def cpu_baseline(wl, budget_s=15.0):
    prep, n, kv, cores = oracle_sample(wl, budget_s)
    t = oracle_time(prep)
    return {"value": kv / t / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"the {n} shortest of {wl.num_seqs} sequences of {wl.name}: their cache writes and "
                      f"all their query rows, fp64 C oracle, {t:.2f} s"}


def bench_reference(args):
    world, rank, _ = dist_setup(args)
    if rank != 0:  # the oracle runs once, on rank 0's host cores
        if world > 1:
            torch.distributed.destroy_process_group()
        return
    wl = W.make(args.workload, "full")
    if wl.kv_dtype == "e4m3":
        wl.fp8_scales_from_draws()
    per_step = max(0.05, min(args.ref_budget, 150.0 / (args.steps + args.warmup)))
    prep, n, kv, cores = oracle_sample(wl, per_step)
    for _ in range(args.warmup):
        oracle_time(prep)
    times = [oracle_time(prep) for _ in range(args.steps)]
    t = sum(times) / len(times)
    value = kv / t / 1e9
    sample = f"{n} of {wl.num_seqs} sequences of {wl.name} per step"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name, "sample_seqs": n},
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


def _time(fn, steps, stream):
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(steps):
        fn(i)
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps


# Untimed back-to-back replays just before the timed steps, so that the
# nvidia-smi samples (taken every 50 ms) see the GPU under this load: a timed
# region of 20 steps of 60 us is far shorter than one sampling interval.
CLOCK_WINDOW_S = 0.3


def _load(seconds, fn):
    t_end = time.perf_counter() + seconds
    i = 0
    while time.perf_counter() < t_end:
        for _ in range(32):
            fn(i)
            i += 1
        torch.cuda.synchronize()


def prefill_flops(wl):
    """QK^T and PV FLOPs of the step's prompt rows (q_len > 1): 4 * Hq * D
    per (query row, attended key), causal over prior context + chunk."""
    f = 0
    for c, q in zip(wl.context_lens.tolist(), wl.q_lens.tolist()):
        if q > 1:
            keys = q * c + q * (q + 1) // 2  # row i attends c + i + 1 keys
            f += 4 * wl.num_q_heads * wl.head_dim * keys
    return f


def _fusable(desc):
    """pa_decode_fused covers the tensor-core decode: bf16 queries, a bf16 or
    e4m3 pool, GQA group 2..8."""
    g = desc.num_q_heads // desc.num_kv_heads
    return desc.q_dtype == 1 and 2 <= g <= 8 and desc.kv_dtype in (1, 2)


class Measured:
    """One workload's graph-replayed step and attention, timed on one rank
    (max over ranks), with the clocks seen meanwhile."""

    def __init__(self, wl, device, args, world, rank, local):
        from paged_kv_cache_452_b200 import runner
        self.wl = wl
        b0 = runner.setup(wl, device)
        # the second copy of the pool, used alternately with the first so no
        # step finds the previous step's K/V in L2 (each copy is larger than L2)
        self.batches = [b0, runner.clone(b0)]
        stream = torch.cuda.current_stream()
        # eager warm-up through the public API, then one CUDA graph per pool
        # copy for the step (cache write + attention) and for the attention
        # alone, as a serving loop would replay them
        for i in range(args.warmup):
            runner.step(self.batches[i & 1])
        torch.cuda.synchronize()
        self.g_step, self.g_attend = [], []
        for b in self.batches:
            gs, ga = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
            with torch.cuda.graph(gs):
                runner.step(b)
            with torch.cuda.graph(ga):
                runner.attend(b)
            self.g_step.append(gs)
            self.g_attend.append(ga)
        # the same step as one launch (pa_decode_fused), where the path fuses it
        self.g_fused = []
        if int(wl.q_lens.max()) == 1 and _fusable(b0.desc):
            for b in self.batches:
                gf = torch.cuda.CUDAGraph()
                runner.step_fused(b)
                torch.cuda.synchronize()
                with torch.cuda.graph(gf):
                    runner.step_fused(b)
                self.g_fused.append(gf)
        # shared prefixes attended once for their sequences (pa_decode_prefix)
        self.g_pstep, self.g_pattend, self.plans = [], [], []
        if wl.sharing is not None or getattr(wl, "prefix_group", None) is not None:
            for b in self.batches:
                plan = runner.prefix_plan(b)
                if plan.groups.num_prefixes == 0:
                    break
                runner.step_prefix(b, plan)
                torch.cuda.synchronize()
                gs, ga = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
                with torch.cuda.graph(gs):
                    runner.step_prefix(b, plan)
                with torch.cuda.graph(ga):
                    runner.attend_prefix(b, plan)
                self.plans.append(plan)
                self.g_pstep.append(gs)
                self.g_pattend.append(ga)
        for i in range(args.warmup):
            self.g_step[i & 1].replay()
            self.g_attend[i & 1].replay()
            if self.g_fused:
                self.g_fused[i & 1].replay()
            if self.g_pstep:
                self.g_pstep[i & 1].replay()
                self.g_pattend[i & 1].replay()
        torch.cuda.synchronize()

        sampler = ClockSampler(local) if rank == 0 else None
        _load(CLOCK_WINDOW_S, lambda i: self.g_step[i & 1].replay())
        barrier(world)
        torch.cuda.synchronize()
        ms = _time(lambda i: self.g_step[i & 1].replay(), args.steps, stream)
        # the attention kernels alone: replays of a graph holding only them,
        # events on the replay stream
        attend_ms = _time(lambda i: self.g_attend[i & 1].replay(), args.steps, stream)
        fused_ms = _time(lambda i: self.g_fused[i & 1].replay(), args.steps, stream) if self.g_fused else None
        pstep_ms = _time(lambda i: self.g_pstep[i & 1].replay(), args.steps, stream) if self.g_pstep else None
        pattend_ms = _time(lambda i: self.g_pattend[i & 1].replay(), args.steps, stream) if self.g_pstep else None
        torch.cuda.synchronize()
        barrier(world)
        self.clocks = sampler.stop() if sampler else None
        self.ms = reduce_max(ms, world, device)
        self.attend_ms = reduce_max(attend_ms, world, device)
        self.fused_ms = reduce_max(fused_ms, world, device) if fused_ms is not None else None
        self.pstep_ms = reduce_max(pstep_ms, world, device) if pstep_ms is not None else None
        self.pattend_ms = reduce_max(pattend_ms, world, device) if pattend_ms is not None else None
        self.alg_bytes, self.kv_bytes = algorithmic_bytes(wl)

    def check(self):
        import paged_kv_cache_452_b200 as pa
        errs = [pa.workspace_error(b.workspace) for b in self.batches]
        errs += [pa.workspace_error(pl.workspace) for pl in self.plans]
        if any(errs):
            raise SystemExit(f"{self.wl.name}: kernel error word set: {errs}")

    def release(self):
        self.g_step.clear()
        self.g_attend.clear()
        self.g_fused.clear()
        self.g_pstep.clear()
        self.g_pattend.clear()
        self.plans.clear()
        self.batches.clear()
        torch.cuda.synchronize()
        torch.cuda.empty_cache()

    def summary(self, world, hbm, tc_peak):
        wl = self.wl
        rows = wl.num_new_tokens
        decode_rows = int((wl.q_lens == 1).sum())
        kv_gbs = self.alg_bytes / (self.attend_ms * 1e-3) / 1e9
        d = {"workload": wl.name, "num_seqs": wl.num_seqs, "query_rows": rows, "decode_rows": decode_rows,
             "kv_dtype": wl.kv_dtype, "num_q_heads": wl.num_q_heads, "num_kv_heads": wl.num_kv_heads,
             "head_dim": wl.head_dim, "block_size": wl.block_size,
             "context_tokens": int((wl.context_lens + wl.q_lens).sum()),
             "algorithmic_bytes": self.alg_bytes, "kv_bytes": self.kv_bytes,
             "attend_us": self.attend_ms * 1e3, "step_us": self.ms * 1e3,
             "kv_gbs": world * kv_gbs, "frac_of_measured_hbm": kv_gbs / hbm, "frac_of_8tbs": kv_gbs / 8000.0,
             "step_gbs": job_throughput(world, self.alg_bytes, self.ms),
             "tokens_per_s": world * rows / (self.ms * 1e-3),
             "decode_tokens_per_s": world * decode_rows / (self.ms * 1e-3),
             "clocks": self.clocks, "traffic": profiled_traffic(wl.name)}
        if self.fused_ms is not None:  # write + attention in one launch
            d["fused_step_us"] = self.fused_ms * 1e3
            d["fused_step_gbs"] = job_throughput(world, self.alg_bytes, self.fused_ms)
        if self.pstep_ms is not None:  # shared prefixes attended once (pa_decode_prefix)
            d["prefix_path_attend_us"] = self.pattend_ms * 1e3
            d["prefix_path_step_us"] = self.pstep_ms * 1e3
            d["prefix_path_kv_gbs"] = world * self.alg_bytes / (self.pattend_ms * 1e-3) / 1e9
        if wl.sharing is not None:  # the shared prefix counted once per sequence
            d["logical_kv_bytes"] = logical_kv_bytes(wl)
            d["effective_gbs"] = world * logical_kv_bytes(wl) / (self.attend_ms * 1e-3) / 1e9
        flops = prefill_flops(wl)
        if flops:
            # the step's bound: its bytes at the copy peak or its prompt-row
            # FLOPs at the sustained bf16 tensor peak, whichever is slower
            bound_us = max(self.alg_bytes / (hbm * 1e9), flops / (tc_peak * 1e12)) * 1e6
            d.update({"prefill_flops": flops, "bound_us": bound_us, "frac_of_bound": bound_us / (self.ms * 1e3)})
        return d


def e2e_measure(m, device, args, world):
    """End to end through the public API with host buffers: every step
    uploads its inputs from pinned host memory (one packed copy), runs cache
    write + attention (a CUDA graph captured from the public calls, replayed
    once per step) and reads its output back.  Uploads run on one stream and
    downloads on another, two device input sets used alternately, so a
    step's copies overlap its neighbours' kernels; the kernels stay in order
    on the main stream (two attention grids never run at once)."""
    import copy

    from paged_kv_cache_452_b200 import runner
    keys = ("q", "k_new", "v_new", "slots", "tables", "seq_lens")
    b0 = m.batches[0]
    layout, off = {}, 0
    for k in keys:
        t = getattr(b0, k)
        n = t.numel() * t.element_size()
        layout[k] = (off, n, t.dtype, tuple(t.shape))
        off += (n + 255) // 256 * 256
    host = torch.empty(off, dtype=torch.uint8).pin_memory()
    for k, (o, n, _, _) in layout.items():
        host[o:o + n].copy_(getattr(b0, k).detach().cpu().contiguous().view(-1).view(torch.uint8))
    stream = torch.cuda.current_stream()
    sets, devbufs, graphs = [], [], []
    for j in range(2):
        buf = torch.empty(off, dtype=torch.uint8, device=device)
        st = copy.copy(m.batches[j])  # pool copy j and its workspace
        for k, (o, n, dt, shape) in layout.items():
            setattr(st, k, buf[o:o + n].view(dt).view(shape))
        st.out = torch.empty_like(b0.out)
        buf.copy_(host)
        torch.cuda.synchronize()
        runner.step(st)  # the set's tensor maps and launch attributes are set up before capture
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            runner.step(st)
        sets.append(st)
        devbufs.append(buf)
        graphs.append(g)
    out_host = [torch.empty(b0.out.shape, dtype=b0.out.dtype).pin_memory() for _ in range(2)]
    d2h = out_host[0].numel() * out_host[0].element_size()
    up, down = torch.cuda.Stream(device), torch.cuda.Stream(device)
    landed = [torch.cuda.Event() for _ in range(2)]    # a set's inputs are on the device
    computed = [torch.cuda.Event() for _ in range(2)]  # a set's kernels have run
    read = [torch.cuda.Event() for _ in range(2)]      # a set's output is on the host
    for j in range(2):
        computed[j].record(stream)
        read[j].record(stream)

    def step(i):
        j = i & 1
        with torch.cuda.stream(up):
            up.wait_event(computed[j])  # the set's previous kernels no longer need its inputs
            devbufs[j].copy_(host, non_blocking=True)
            landed[j].record(up)
        stream.wait_event(landed[j])
        stream.wait_event(read[j])  # the set's previous output has been read
        graphs[j].replay()
        computed[j].record(stream)
        with torch.cuda.stream(down):
            down.wait_event(computed[j])
            out_host[j].copy_(sets[j].out, non_blocking=True)
            read[j].record(down)

    def timed(steps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        up.wait_event(e0)
        down.wait_event(e0)
        for i in range(steps):
            step(i)
        stream.wait_stream(up)
        stream.wait_stream(down)
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = reduce_max(timed(args.steps), world, device)
    # what came back is the step's output: the same bits as the kernel-only graph
    same = all(torch.equal(out_host[j].view(torch.int16), m.batches[0].out.cpu().view(torch.int16))
               for j in range(2)) if b0.out.dtype == torch.bfloat16 else True
    graphs.clear()
    return {"ms_per_step": e2e_ms, "h2d_bytes_per_step": off, "d2h_bytes_per_step": d2h, "output_matches": same}


PER_CONFIG = ("prefix_bf16", "fp8_long", "mixed_prefill_bs16", "mixed_prefill_bs32", "long_prefix_bf16")


def bench_ours(args):
    world, rank, local = dist_setup(args)
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    import paged_kv_cache_452_b200 as pa  # noqa: F401  (fails loudly without libpa.so)
    from paged_kv_cache_452_b200 import runner

    peaks, src = measured_peaks()
    hbm = float(peaks["hbm_gbs"])
    tc_peak = float(peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops", 1400.0)))

    wl = W.make(args.workload, "full")
    if args.max_seqs:
        wl = W.first_seqs(wl, args.max_seqs)
    m = Measured(wl, device, args, world, rank, local)
    stream = torch.cuda.current_stream()
    # the same step issued launch by launch from Python (no graph)
    eager_ms = reduce_max(_time(lambda i: runner.step(m.batches[i & 1]), args.steps, stream), world, device)
    e2e = e2e_measure(m, device, args, world)
    m.check()
    head = m.summary(world, hbm, tc_peak)
    cpu = cpu_baseline(wl, args.ref_budget) if (rank == 0 and not args.no_cpu_baseline) else None
    m.release()

    per_config = {wl.name: head}
    if not args.no_per_config:
        for name in PER_CONFIG:
            if name == wl.name:
                continue
            wl_c = W.make(name, "full")
            mc = Measured(wl_c, device, args, world, rank, local)
            mc.check()
            per_config[name] = mc.summary(world, hbm, tc_peak)
            mc.release()
            if rank == 0 and not args.no_cpu_baseline:
                per_config[name]["cpu_baseline"] = cpu_baseline(wl_c, min(args.ref_budget, 4.0))

    if rank != 0:
        if world > 1:
            torch.distributed.destroy_process_group()
        return
    achieved = m.alg_bytes / (m.attend_ms * 1e-3) / 1e9
    kernel = "decode_tc_kernel (pa_decode)" if int(wl.q_lens.max()) == 1 else \
        "decode_tc_kernel + prefill_umma_kernel (pa_decode_chunked_prefill)"
    line = {
        "metric": METRIC, "value": job_throughput(world, m.alg_bytes, m.ms), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": m.ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": wl.kv_dtype if wl.kv_dtype != "e4m3" else "fp8_e4m3",
        "data": "synthetic",
        "config": {"workload": wl.name, "num_seqs": wl.num_seqs, "num_q_heads": wl.num_q_heads,
                   "num_kv_heads": wl.num_kv_heads, "head_dim": wl.head_dim, "block_size": wl.block_size,
                   "context_tokens": head["context_tokens"], "kv_bytes": m.kv_bytes,
                   "algorithmic_bytes": m.alg_bytes, "parallelism": f"replicas x{world}",
                   "step": "pa_cache_write + pa_decode, replayed as a CUDA graph",
                   "l2": "2 pool copies used alternately, each larger than L2"},
        "decode_tokens_per_s": head["decode_tokens_per_s"],
        "fraction_of_8tbs": m.alg_bytes / (m.ms * 1e-3) / 1e9 / 8000.0,
        "eager_ms_per_step": eager_ms,
        "roofline": {"bound": "hbm", "kernel": kernel,
                     "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                     "peak_source": src, "traffic": profiled_traffic(wl.name), "kernel_ms": m.attend_ms},
        "e2e": {"value": job_throughput(world, m.alg_bytes, e2e["ms_per_step"]), "unit": "GB/s",
                "h2d_bytes_per_step": e2e["h2d_bytes_per_step"], "d2h_bytes_per_step": e2e["d2h_bytes_per_step"],
                "ms_per_step": e2e["ms_per_step"], "output_matches": e2e["output_matches"],
                "pipelining": "inputs uploaded as one packed copy on an upload stream, the step a CUDA graph "
                              "of the public calls, output read back on a download stream; two input sets"},
        # pa_cache_write + pa_decode's decode kernel (+ its prefill kernel for prompt rows)
        "gpu_launches": (3 if int(wl.q_lens.max()) > 1 else 2) * args.steps,
        "clocks": m.clocks,
    }
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if per_config:
        line["per_config"] = per_config
    print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


# Copy-on-write's device half (pa_copy_blocks), measured on its own: random
# pairs of blocks in the geometry of gqa_bf16's pool (8 kv heads, head_dim
# 128, 16 slots, bf16: 32 KiB per block per pool).
BLOCK_COPY = {"pairs": 4096, "num_kv_heads": 8, "head_dim": 128, "block_size": 16}
BLOCK_COPY_METRIC = "block copy GB/s"


def block_copy_geometry():
    c = BLOCK_COPY
    block_bytes = c["num_kv_heads"] * c["block_size"] * c["head_dim"] * 2
    # per step every pair reads and writes one block of each pool
    return c["pairs"], block_bytes, 2 * 2 * c["pairs"] * block_bytes


def block_copy_cpu(budget_s):
    """The oracle's copy (numpy, one host core) on a bounded sample of pairs."""
    import oracle
    n, block_bytes, _ = block_copy_geometry()
    c = BLOCK_COPY
    m = max(16, min(1024, n))  # 128 MiB of host blocks; passes repeat until budget_s
    shape = (2 * m, c["num_kv_heads"], c["block_size"], c["head_dim"])
    g = np.random.default_rng(0)
    k = g.integers(0, 1 << 16, size=shape, dtype=np.uint16)
    v = g.integers(0, 1 << 16, size=shape, dtype=np.uint16)
    perm = g.permutation(2 * m)
    pairs = list(zip(perm[:m].tolist(), perm[m:].tolist()))
    oracle.copy_blocks(k, v, pairs)  # warm
    t0 = time.perf_counter()
    reps = 0
    while True:
        oracle.copy_blocks(k, v, pairs)
        reps += 1
        t = time.perf_counter() - t0
        if t >= budget_s:
            break
    bytes_ = reps * 2 * 2 * m * block_bytes
    return {"value": bytes_ / t / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"{m} of {n} pairs per pass, {reps} passes, numpy block copies, {t:.2f} s"}


def bench_block_copy(args):
    world, rank, local = dist_setup(args)
    if args.impl == "reference":
        if rank == 0:
            per_step = max(0.05, min(args.ref_budget, 150.0 / (args.steps + args.warmup)))
            base = block_copy_cpu(per_step)
            line = {"impl": "reference", "metric": BLOCK_COPY_METRIC, "value": base["value"], "unit": "GB/s",
                    "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "higher_is_better": True,
                    "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                    "config": {"workload": "block_copy", **BLOCK_COPY}, "cpu_baseline": base,
                    "e2e": {"value": base["value"], "unit": "GB/s", "h2d_bytes_per_step": 0,
                            "d2h_bytes_per_step": 0}}
            print(json.dumps(line), flush=True)
        if world > 1:
            torch.distributed.destroy_process_group()
        return
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    import paged_kv_cache_452_b200 as pa

    n, block_bytes, alg_bytes = block_copy_geometry()
    c = BLOCK_COPY
    nb = 4 * n  # two pair sets, used alternately: 4 x 256 MiB of blocks per pool set
    desc = pa.CacheDesc.make(nb, c["block_size"], c["num_kv_heads"], c["num_kv_heads"], c["head_dim"],
                             "bf16", "bf16")
    k, v = pa.alloc_cache(desc, device)
    gen = torch.Generator(device=device).manual_seed(0)
    for t in (k, v):
        t.normal_(generator=gen)
    perm = np.random.default_rng(0).permutation(nb).astype(np.int32)
    src = [torch.from_numpy(perm[2 * j * n:(2 * j + 1) * n].copy()).to(device) for j in range(2)]
    dst = [torch.from_numpy(perm[(2 * j + 1) * n:(2 * j + 2) * n].copy()).to(device) for j in range(2)]
    stream = torch.cuda.current_stream()
    for i in range(args.warmup):
        pa.pa_copy_blocks(desc, src[i & 1], dst[i & 1], k, v)
    torch.cuda.synchronize()
    # parity spot check: each destination block equals its source
    for j in range(2):
        assert torch.equal(k[dst[j][:64].long()], k[src[j][:64].long()])
    graphs = []
    for j in range(2):
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr):
            pa.pa_copy_blocks(desc, src[j], dst[j], k, v)
        graphs.append(gr)
    for i in range(args.warmup):
        graphs[i & 1].replay()
    torch.cuda.synchronize()
    sampler = ClockSampler(local) if rank == 0 else None
    time.sleep(0.2 if sampler else 0)
    barrier(world)
    torch.cuda.synchronize()
    ms = _time(lambda i: graphs[i & 1].replay(), args.steps, stream)
    torch.cuda.synchronize()
    barrier(world)
    ms = reduce_max(ms, world, device)
    clocks = sampler.stop() if sampler else None
    # end to end through the public API: the pair lists come from pinned host
    # memory each step and one copied K block goes back to the host
    src_h = [s_.cpu().pin_memory() for s_ in src]
    dst_h = [d_.cpu().pin_memory() for d_ in dst]
    src_d = [torch.empty_like(s_) for s_ in src]
    dst_d = [torch.empty_like(d_) for d_ in dst]
    back = torch.empty(k[0].shape, dtype=k.dtype).pin_memory()
    h2d = 2 * n * 4
    d2h = back.numel() * back.element_size()

    def e2e_step(i):
        j = i & 1
        src_d[j].copy_(src_h[j], non_blocking=True)
        dst_d[j].copy_(dst_h[j], non_blocking=True)
        pa.pa_copy_blocks(desc, src_d[j], dst_d[j], k, v)
        back.copy_(k[int(perm[(2 * j + 1) * n])], non_blocking=True)

    for i in range(args.warmup):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = reduce_max(_time(e2e_step, args.steps, stream), world, device)
    graphs.clear()
    if rank != 0:
        if world > 1:
            torch.distributed.destroy_process_group()
        return
    peaks, psrc = measured_peaks()
    hbm = float(peaks["hbm_gbs"])
    achieved = alg_bytes / (ms * 1e-3) / 1e9
    line = {
        "metric": BLOCK_COPY_METRIC, "value": job_throughput(world, alg_bytes, ms), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "block_copy", **BLOCK_COPY, "block_bytes_per_pool": block_bytes,
                   "algorithmic_bytes": alg_bytes, "parallelism": f"replicas x{world}",
                   "step": "pa_copy_blocks over all pairs, replayed as a CUDA graph",
                   "l2": "two disjoint pair sets used alternately, 256 MiB read per step (> L2)"},
        "roofline": {"bound": "hbm", "kernel": "copy_blocks_kernel (pa_copy_blocks)", "achieved": achieved,
                     "peak": hbm, "unit": "GB/s", "frac": achieved / hbm, "peak_source": psrc,
                     "traffic": profiled_traffic("block_copy"), "kernel_ms": ms},
        "e2e": {"value": job_throughput(world, alg_bytes, e2e_ms), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": args.steps,
        "clocks": clocks,
    }
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = block_copy_cpu(min(args.ref_budget, 10.0))
    print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(W.WORKLOADS) + ["block_copy"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ref-budget", type=float, default=15.0, help="seconds of oracle work per sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="measure only --workload, not the other full-size workloads")
    ap.add_argument("--max-seqs", type=int, default=0,
                    help="only the first N sequences of --workload (a smaller case of the same mix, "
                         "for profiler captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.workload == "block_copy":
        bench_block_copy(args)
    elif args.impl == "reference":
        bench_reference(args)
    else:
        bench_ours(args)


if __name__ == "__main__":
    main()
