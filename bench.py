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
# one ncu capture (profiles/), valid only for the kernel source that was
# profiled: any edit to the source drops the figure to null.
PROFILED_TRAFFIC = {
    "gqa_bf16": {"source": "paged_kv_cache_452_b200/csrc/decode_tc.cu",
                 # the captured source with its header comment's CTA count corrected
                 # (a comment-only edit, same line count; the code is unchanged)
                 "sha256": "faab74a6d10b8ea93dd8d701d95eb0efa43c2f4d3fba534abb49367ada175fa1",
                 "bytes": 294_643_200},
    # profiles/copy_blocks_block_copy.md: mean of two launches
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
    """A prefix of the batch whose oracle evaluation takes about budget_s
    (scaled from a timing of the first sequence); its KV bytes."""
    import oracle
    t = oracle_time(oracle_prepare(wl, [0]))
    per_token = t / max(1, int(wl.context_lens[0] + wl.q_lens[0]))
    seqs, est = [], 0.0
    for s in range(wl.num_seqs):
        n = int(wl.context_lens[s] + wl.q_lens[s])
        if seqs and est + per_token * n > budget_s:
            break
        seqs.append(s)
        est += per_token * n
    kv = sum(int(wl.context_lens[s] + wl.q_lens[s]) for s in seqs) * 2 * wl.num_kv_heads * wl.head_dim * \
        KV_BYTES[wl.kv_dtype]
    return oracle_prepare(wl, seqs), len(seqs), kv, oracle.max_threads()


def cpu_baseline(wl, budget_s=15.0):
    prep, n, kv, cores = oracle_sample(wl, budget_s)
    t = oracle_time(prep)
    return {"value": kv / t / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"{n} of {wl.num_seqs} sequences of {wl.name}: their cache writes and all their "
                      f"query rows, fp64 C oracle, {t:.2f} s"}


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


def bench_ours(args):
    world, rank, local = dist_setup(args)
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    import paged_kv_cache_452_b200 as pa
    from paged_kv_cache_452_b200 import runner

    wl = W.make(args.workload, "full")
    # two copies of the pool, used alternately, so no step finds the previous
    # step's K/V in L2 (each copy is larger than L2 already)
    batches = [runner.setup(wl, device) for _ in range(2)]
    alg_bytes, kv_bytes = algorithmic_bytes(wl)
    stream = torch.cuda.current_stream()

    # eager warm-up through the public API, then one CUDA graph per pool copy
    # for the step (cache write + decode) and for the decode alone, as a
    # serving loop would replay them
    for i in range(args.warmup):
        runner.step(batches[i & 1])
    torch.cuda.synchronize()
    g_step, g_attend = [], []
    for b in batches:
        gs, ga = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(gs):
            runner.step(b)
        with torch.cuda.graph(ga):
            runner.attend(b)
        g_step.append(gs)
        g_attend.append(ga)
    for i in range(args.warmup):
        g_step[i & 1].replay()
        g_attend[i & 1].replay()
    torch.cuda.synchronize()

    sampler = ClockSampler(local) if rank == 0 else None
    time.sleep(0.2 if sampler else 0)
    barrier(world)
    torch.cuda.synchronize()
    ms = _time(lambda i: g_step[i & 1].replay(), args.steps, stream)
    torch.cuda.synchronize()
    barrier(world)
    ms = reduce_max(ms, world, device)
    # the dominant kernel, pa_decode's single launch, per launch: replays of a
    # graph holding only it, events on the replay stream
    attend_ms = reduce_max(_time(lambda i: g_attend[i & 1].replay(), args.steps, stream), world, device)
    clocks = sampler.stop() if sampler else None
    # the same step issued launch by launch from Python (no graph)
    eager_ms = reduce_max(_time(lambda i: runner.step(batches[i & 1]), args.steps, stream), world, device)

    # end to end through the public API with host buffers: every step copies
    # its inputs from pinned host memory, runs write + attention, and reads
    # its output back.  As a serving loop would, the copies of one step
    # overlap the kernels of its neighbours: uploads on one stream, the
    # kernels on the main stream, downloads on a third, two device input
    # sets used alternately (the pool and the workspace are shared; the
    # kernels stay in order on the main stream).
    import copy
    b0 = batches[0]
    keys = ("q", "k_new", "v_new", "slots", "tables", "seq_lens")
    host = {k: getattr(b0, k).cpu().pin_memory() for k in keys}
    out_host = [torch.empty(b0.out.shape, dtype=b0.out.dtype).pin_memory() for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out_host[0].numel() * out_host[0].element_size()
    sets = []
    for _ in range(2):
        st = copy.copy(b0)
        for k in keys:
            setattr(st, k, torch.empty_like(getattr(b0, k)))
        st.out = torch.empty_like(b0.out)
        sets.append(st)
    up, down = torch.cuda.Stream(device), torch.cuda.Stream(device)
    landed = [torch.cuda.Event() for _ in range(2)]    # a set's inputs are on the device
    computed = [torch.cuda.Event() for _ in range(2)]  # a set's kernels have run
    read = [torch.cuda.Event() for _ in range(2)]      # a set's output is on the host

    def e2e_step(i):
        j = i & 1
        st = sets[j]
        with torch.cuda.stream(up):
            up.wait_event(computed[j])  # the set's previous kernels no longer need its inputs
            for k, t in host.items():
                getattr(st, k).copy_(t, non_blocking=True)
            landed[j].record(up)
        stream.wait_event(landed[j])
        stream.wait_event(read[j])  # the set's previous output has been read
        runner.step(st)
        computed[j].record(stream)
        with torch.cuda.stream(down):
            down.wait_event(computed[j])
            out_host[j].copy_(st.out, non_blocking=True)
            read[j].record(down)

    def e2e_time(steps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        up.wait_event(e0)
        down.wait_event(e0)
        for i in range(steps):
            e2e_step(i)
        stream.wait_stream(up)
        stream.wait_stream(down)
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps

    for i in range(args.warmup):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = reduce_max(e2e_time(args.steps), world, device)

    errs = [pa.workspace_error(b.workspace) for b in batches]
    if any(errs):
        raise SystemExit(f"kernel error word set: {errs}")
    g_step.clear()  # release the graphs before the process group
    g_attend.clear()

    if rank != 0:
        if world > 1:
            torch.distributed.destroy_process_group()
        return
    peaks, src = measured_peaks()
    hbm = float(peaks["hbm_gbs"])
    achieved = alg_bytes / (attend_ms * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": job_throughput(world, alg_bytes, ms), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": wl.kv_dtype if wl.kv_dtype != "e4m3" else "fp8_e4m3",
        "data": "synthetic",
        "config": {"workload": wl.name, "num_seqs": wl.num_seqs, "num_q_heads": wl.num_q_heads,
                   "num_kv_heads": wl.num_kv_heads, "head_dim": wl.head_dim, "block_size": wl.block_size,
                   "context_tokens": int((wl.context_lens + wl.q_lens).sum()), "kv_bytes": kv_bytes,
                   "algorithmic_bytes": alg_bytes, "parallelism": f"replicas x{world}",
                   "step": "pa_cache_write + pa_decode, replayed as a CUDA graph",
                   "l2": "2 pool copies used alternately, each larger than L2"},
        "decode_tokens_per_s": world * wl.num_seqs / (ms * 1e-3),
        "fraction_of_8tbs": alg_bytes / (ms * 1e-3) / 1e9 / 8000.0,
        "eager_ms_per_step": eager_ms,
        "roofline": {"bound": "hbm", "kernel": "decode_tc_kernel (pa_decode)",
                     "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                     "peak_source": src, "traffic": profiled_traffic(wl.name), "kernel_ms": attend_ms},
        "e2e": {"value": job_throughput(world, alg_bytes, e2e_ms), "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "pipelining": "uploads and downloads on their own streams, two input sets"},
        # pa_cache_write + pa_decode's decode kernel (+ its prefill kernel for prompt rows)
        "gpu_launches": (3 if int(wl.q_lens.max()) > 1 else 2) * args.steps,
        "clocks": clocks,
    }
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl, args.ref_budget)
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
