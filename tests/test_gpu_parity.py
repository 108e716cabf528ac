"""CUDA path against the CPU oracle, through the C ABI.

Bit-exact: block tables and slot mappings (C++ pool vs pool model) and every
cache element written this step or at set-up (pa_cache_write vs the oracle's
write, e4m3 quantisation included).  Attention: max abs error against the
fp64 oracle within 1e-4 (fp32), 2e-2 (bf16), 6e-2 (e4m3, against the oracle
on the dequantised values).
"""
import numpy as np
import pytest
import torch

import pa_workloads as W
import paged_kv_cache_452_b200 as pa
from oracle.workload import expected
from paged_kv_cache_452_b200 import runner

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2, "e4m3": 6e-2}


def bits(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.float32:
        return t.view(torch.int32).numpy()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy()
    return t.numpy()


def check_cache(wl, b, exp):
    """Every position of every checked sequence: GPU pool bytes == oracle pool bytes."""
    bs = wl.block_size
    kc, vc = exp["k_cache"], exp["v_cache"]
    for s in exp["seqs"]:
        n = int(wl.context_lens[s] + wl.q_lens[s])
        if n == 0:
            continue
        pos = np.arange(n)
        blk = exp["tables"][s, pos // bs]
        cblk = exp["compact_tables"][s, pos // bs]
        off = pos % bs
        bi = torch.from_numpy(blk.astype(np.int64)).to(b.k_cache.device)
        oi = torch.from_numpy(off.astype(np.int64)).to(b.k_cache.device)
        gk = bits(b.k_cache[bi, :, oi, :])
        ok_ = kc[cblk, :, off, :]
        if wl.kv_dtype == "e4m3":
            gv = bits(b.v_cache[bi, :, :, oi])
            ov = vc[cblk, :, :, off]
        else:
            gv = bits(b.v_cache[bi, :, oi, :])
            ov = vc[cblk, :, off, :]
        assert np.array_equal(gk.view(ok_.dtype), ok_), f"K bytes differ in sequence {s}"
        assert np.array_equal(gv.view(ov.dtype), ov), f"V bytes differ in sequence {s}"


def poison_workspace(b):
    """NaN bytes in the partial-result scratch, so a read of a partial that
    this call did not write shows up in the output.  The error word and the
    arrival counters (the part of the workspace the contract zero-fills)
    stay zero."""
    counters = (b.seq_lens.shape[0] * b.desc.num_kv_heads * 4 + 255) // 256 * 256
    b.workspace.fill_(0xFF)
    b.workspace[:256 + counters].zero_()


def run_and_check(wl, device, seqs=None):
    b = runner.setup(wl, device)
    poison_workspace(b)
    runner.step(b)
    torch.cuda.synchronize()
    full_out = b.out.detach().cpu().to(torch.float64).numpy()
    bad = np.argwhere(~np.isfinite(full_out).all(axis=(1, 2))).ravel()
    assert bad.size == 0, f"{wl.name}: non-finite output rows {bad[:20].tolist()}"
    exp = expected(wl, seqs)
    assert np.array_equal(b.tables_host.numpy(), exp["tables"])
    assert np.array_equal(b.slots_host.numpy(), exp["step_slots"])
    assert b.num_cached == exp["num_cached"]
    check_cache(wl, b, exp)
    out = full_out[exp["rows"]]
    err = float(np.abs(out - exp["out"]).max()) if out.size else 0.0
    assert err <= TOL[wl.kv_dtype], f"{wl.name}: max abs error {err}"
    assert pa.workspace_error(b.workspace) == 0
    # the tcgen05 kernel's unit queue (header words 2 and 3) is back at zero
    assert b.workspace[:16].view(torch.int32)[2:4].tolist() == [0, 0]
    return b, err


SMALL = ["tiny_fp32", "gqa_bf16", "prefix_bf16", "fp8_long", "mixed_prefill_bs16", "mixed_prefill_bs32",
         "long_prefix_bf16"]


def outscoring_draws(wl, late_from, factor, seed=5):
    """Seeded N(0,1) draws for wl, keys of the cached context from position
    late_from on scaled by `factor`: scores there exceed the first 128 keys'
    by far more than 2^64 in the weights, so the tcgen05 prompt-row kernel's
    rows take their slow path (the reference moves, O and the sum are
    rescaled).  Sequences with equal prefix_group values share their first
    wl.prefix_len tokens' draws."""
    g = np.random.default_rng(seed)
    hkv, hq, d = wl.num_kv_heads, wl.num_q_heads, wl.head_dim
    shared = {}
    ks, vs = [], []
    for s in range(wl.num_seqs):
        n = int(wl.context_lens[s])
        k = g.standard_normal((n, hkv, d), dtype=np.float32)
        v = g.standard_normal((n, hkv, d), dtype=np.float32)
        grp = int(wl.prefix_group[s]) if wl.prefix_group is not None else -1
        if grp >= 0:
            if grp not in shared:
                shared[grp] = (k[:wl.prefix_len].copy(), v[:wl.prefix_len].copy())
            k[:wl.prefix_len], v[:wl.prefix_len] = shared[grp]
        k[late_from:] *= factor
        ks.append(k)
        vs.append(v)
    t = wl.num_new_tokens
    wl._fixed = {"k": ks, "v": vs, "k_new": g.standard_normal((t, hkv, d), dtype=np.float32),
                 "v_new": g.standard_normal((t, hkv, d), dtype=np.float32),
                 "q": g.standard_normal((t, hq, d), dtype=np.float32)}
    return wl


def test_prompt_rows_whose_later_keys_outscore_the_first_tile(cuda_device):
    # sequence 0: 64 prompt rows over 300 cached tokens, keys 200.. scaled;
    # sequence 1: 130 prompt rows over 40 cached tokens (unscaled)
    wl = outscoring_draws(W.custom("outscore", context_lens=[300, 40], q_lens=[64, 130], num_q_heads=8,
                                   num_kv_heads=2), late_from=200, factor=48.0)
    run_and_check(wl, cuda_device)


@pytest.mark.parametrize("name", SMALL)
def test_workload_small(name, cuda_device):
    run_and_check(W.make(name, "small"), cuda_device)


EDGE = {
    # empty context (attends only the new token), block boundaries, ragged tails
    "bounds_bs16": dict(context_lens=[0, 1, 15, 16, 17, 31, 32, 33, 47, 48]),
    "bounds_bs32": dict(context_lens=[0, 1, 31, 32, 33, 63, 64, 65], block_size=32),
    "bounds_fp8_bs16": dict(context_lens=[0, 15, 16, 17, 100], kv_dtype="e4m3"),
    "bounds_fp8_bs32": dict(context_lens=[0, 31, 32, 33, 200], kv_dtype="e4m3", block_size=32),
    "group2": dict(context_lens=[5, 80, 300], num_q_heads=4, num_kv_heads=2),
    "group8": dict(context_lens=[5, 80, 300], num_q_heads=16, num_kv_heads=2),
    "group8_fp8": dict(context_lens=[5, 80, 300], num_q_heads=16, num_kv_heads=2, kv_dtype="e4m3"),
    "head64": dict(context_lens=[3, 64, 129], head_dim=64),
    "head64_bs32": dict(context_lens=[3, 64, 129], head_dim=64, block_size=32),
    "mha_bf16": dict(context_lens=[7, 100], num_q_heads=4, num_kv_heads=4),  # group 1: CUDA cores
    "group16_bf16": dict(context_lens=[7, 100], num_q_heads=32, num_kv_heads=2),  # group > 8: CUDA cores
    "fp32_gqa": dict(context_lens=[9, 70], kv_dtype="f32", q_dtype="f32", num_q_heads=8, num_kv_heads=2),
    "fp8_f32_queries": dict(context_lens=[9, 70], kv_dtype="e4m3", q_dtype="f32"),
    "one_long": dict(context_lens=[5000], num_q_heads=8, num_kv_heads=8 // 4),  # split over many CTAs
    # fewer tiles than CTAs: empty CTAs sit between a sequence's contributors
    "fewer_tiles_than_ctas": dict(context_lens=[100, 3, 250], num_q_heads=4, num_kv_heads=1),
    "many_short": dict(context_lens=list(range(0, 700, 1)), num_q_heads=4, num_kv_heads=2, head_dim=64),
    "single": dict(context_lens=[1]),
    # batches with several tiles per worker warp, so contexts are cut at many
    # warp-range edges and merged from several pieces
    "split_uniform": dict(context_lens=[2000] * 20, num_q_heads=32, num_kv_heads=8),
    "split_ragged": dict(context_lens=[0, 1, 17, 3000, 5, 16, 4000, 33, 2500, 1, 64, 6000, 15, 31, 700],
                       num_q_heads=32, num_kv_heads=8),
    "split_group8_head64": dict(context_lens=[7999, 8000, 8001, 100, 7000, 8192], num_q_heads=16, num_kv_heads=2,
                              head_dim=64),
    "split_fp8": dict(context_lens=[3000] * 15 + [17], kv_dtype="e4m3", num_q_heads=32, num_kv_heads=8),
    "split_bs32": dict(context_lens=[4000] * 9 + [31, 32, 33], num_q_heads=32, num_kv_heads=8, block_size=32),
    # groups whose (max, sum) block is not a multiple of 16 bytes
    "split_group3": dict(context_lens=[5000] * 8 + [3, 40], num_q_heads=6, num_kv_heads=2),
    "split_group7_head64": dict(context_lens=[5000] * 8 + [0, 16], num_q_heads=14, num_kv_heads=2, head_dim=64),
    # e4m3 pools with one scale per kv head: heads about 3 000x apart, so a
    # head that used another head's scale would saturate or vanish; some
    # small scales saturate the codes at +-448 (the oracle does the same)
    "fp8_head_scales": dict(context_lens=[0, 5, 80, 300, 17], kv_dtype="e4m3", num_q_heads=16, num_kv_heads=4,
                            scale_mode="fixed", k_scale=[0.001, 0.01, 3.0, 0.5], v_scale=[2.0, 0.0007, 0.05, 1.0]),
    "fp8_head_scales_split": dict(context_lens=[3000] * 15 + [17], kv_dtype="e4m3", num_q_heads=32, num_kv_heads=8,
                                  scale_mode="fixed", k_scale=[0.001, 0.3, 3.0, 0.02, 0.01, 1.0, 0.1, 0.005],
                                  v_scale=[0.05, 2.0, 0.0007, 0.01, 0.3, 0.02, 1.5, 0.1]),
    "fp8_head_scales_from_draws_bs32": dict(context_lens=[31, 32, 33, 200], kv_dtype="e4m3", block_size=32,
                                            scale_mode="head"),
    # per-head scales on the CUDA-core path: fp32 queries, and a group above 8
    "fp8_head_scales_f32_queries": dict(context_lens=[9, 70], kv_dtype="e4m3", q_dtype="f32", num_q_heads=4,
                                        num_kv_heads=2, scale_mode="fixed", k_scale=[0.002, 2.0],
                                        v_scale=[3.0, 0.001]),
    "fp8_head_scales_group16": dict(context_lens=[7, 100], kv_dtype="e4m3", num_q_heads=32, num_kv_heads=2,
                                    scale_mode="fixed", k_scale=[0.002, 2.0], v_scale=[3.0, 0.001]),
}


@pytest.mark.parametrize("case", sorted(EDGE))
def test_edge_cases(case, cuda_device):
    run_and_check(W.custom(case, **EDGE[case]), cuda_device)


MIXED_EDGE = {
    # prefill chunks with no prior context, a 1-token chunk, chunks crossing blocks
    "mixed_edges": dict(context_lens=[0, 0, 17, 40, 3, 100], q_lens=[1, 20, 33, 1, 16, 1]),
    # chunks of exactly one, one less and one more than a unit of query
    # positions (64 rows / group 4 = 16 positions), over prior context that
    # ends mid-block and on a block edge
    "unit_bounds_g4": dict(context_lens=[0, 5, 16, 31, 7], q_lens=[16, 15, 17, 48, 1]),
    "mha_prefill": dict(context_lens=[3, 70, 0], q_lens=[64, 65, 130], num_q_heads=2, num_kv_heads=2),
    "group8_prefill": dict(context_lens=[0, 21, 9], q_lens=[8, 9, 40], num_q_heads=16, num_kv_heads=2),
    "group16_prefill": dict(context_lens=[0, 33], q_lens=[5, 37], num_q_heads=32, num_kv_heads=2),
    "group32_prefill": dict(context_lens=[0, 20, 100], q_lens=[9, 30, 1], num_q_heads=64, num_kv_heads=2),
    "head64_many_units": dict(context_lens=[3 * i for i in range(30)], q_lens=[70] * 30, num_q_heads=8,
                              num_kv_heads=2, head_dim=64),
    "head64_bs32_prefill": dict(context_lens=[0, 50, 7], q_lens=[70, 3, 1], head_dim=64, block_size=32),
    "group3_prefill": dict(context_lens=[4, 0], q_lens=[9, 22], num_q_heads=6, num_kv_heads=2),  # CUDA cores
    "prefill_only": dict(context_lens=[0, 200], q_lens=[33, 100]),
    "fp8_prefill": dict(context_lens=[0, 40], q_lens=[17, 30], kv_dtype="e4m3"),  # CUDA cores
    "fp8_head_scales_prefill": dict(context_lens=[0, 40, 9], q_lens=[17, 30, 1], kv_dtype="e4m3", num_q_heads=8,
                                    num_kv_heads=2, scale_mode="fixed", k_scale=[0.01, 1.0], v_scale=[0.3, 0.003]),
    # more prompt units than SMs: persistent CTAs chain several units
    "many_units": dict(context_lens=[7 * i for i in range(40)] + [5, 9], q_lens=[40] * 40 + [1, 1],
                       num_q_heads=8, num_kv_heads=2),
}


@pytest.mark.parametrize("case", sorted(MIXED_EDGE))
def test_mixed_edge_cases(case, cuda_device):
    run_and_check(W.custom(case, **MIXED_EDGE[case]), cuda_device)


def test_mixed_step_with_more_sequences_than_the_unit_table_holds(cuda_device):
    """8 502 sequences: the tcgen05 prefill kernel's per-sequence unit table no
    longer fits next to two K and two V stages, so the prompt rows fall back
    to the mma.sync prefill kernel (and the decode rows run at two CTAs per
    SM); the result must not change."""
    n = 8500
    wl = W.custom("many_sequences_mixed", context_lens=[5 + (i % 11) for i in range(n)] + [10, 40],
                  q_lens=[1] * n + [20, 33], num_q_heads=8, num_kv_heads=2)
    run_and_check(wl, cuda_device, seqs=[0, 1, 7, 4999, n - 1, n, n + 1])


def test_paged_output_equals_contiguous_output(cuda_device):
    """Paging changes nothing: the same draws through a shuffled free list and
    through an identity free list (contiguous blocks) give bit-identical
    outputs, because split points depend only on the lengths."""
    a = W.gqa_bf16("small")
    b = W.gqa_bf16("small")
    b.free_order = np.arange(b.num_blocks, dtype=np.int32)
    ra = runner.setup(a, cuda_device)
    rb = runner.setup(b, cuda_device)
    runner.step(ra)
    runner.step(rb)
    torch.cuda.synchronize()
    assert not torch.equal(ra.tables, rb.tables)
    assert torch.equal(ra.out.view(torch.int16), rb.out.view(torch.int16))


def test_prefix_sharing_leaves_output_unchanged(cuda_device):
    """Sequences that share prefix blocks give the same bits as with private
    copies of the prefix (the pages: KV byte-identical, output unchanged)."""
    a = W.prefix_bf16("small")
    b = W.prefix_bf16("small")
    b.sharing = None  # no token ids: every sequence gets private blocks
    b.prefix_len = a.prefix_len

    # same values: b draws its prefix from the shared stream too
    def prior_kv_f32(s, _a=a):
        return _a.prior_kv_f32(s)
    b.prior_kv_f32 = prior_kv_f32
    b.num_blocks = a.num_blocks + a.prefix_len // a.block_size * int(a.sharing.sum())
    b.free_order = np.arange(b.num_blocks, dtype=np.int32)
    ra = runner.setup(a, cuda_device)
    rb = runner.setup(b, cuda_device)
    runner.step(ra)
    runner.step(rb)
    torch.cuda.synchronize()
    shared = ra.tables[0, : a.prefix_len // a.block_size]
    assert torch.equal(ra.tables[1, : a.prefix_len // a.block_size], shared)
    assert not torch.equal(rb.tables[1, : a.prefix_len // a.block_size], rb.tables[0, : a.prefix_len // a.block_size])
    assert torch.equal(ra.out.view(torch.int16), rb.out.view(torch.int16))


def test_repeated_steps_are_deterministic(cuda_device):
    wl = W.fp8_long("small")
    b = runner.setup(wl, cuda_device)
    runner.step(b)
    first = b.out.clone()
    for _ in range(3):
        runner.attend(b)
    torch.cuda.synchronize()
    assert torch.equal(first.view(torch.int16), b.out.view(torch.int16))


def test_bad_table_entry_is_flagged_not_faulted(cuda_device):
    wl = W.gqa_bf16("small")
    b = runner.setup(wl, cuda_device)
    runner.step(b)
    b.tables[0, 0] = wl.num_blocks + 5  # past the pool: the kernel flags it and reads block 0
    runner.attend(b)
    torch.cuda.synchronize()
    assert pa.workspace_error(b.workspace) == 2


def test_context_longer_than_table_row_is_flagged(cuda_device):
    wl = W.gqa_bf16("small")
    b = runner.setup(wl, cuda_device)
    runner.step(b)
    b.seq_lens[0] = b.tables.shape[1] * wl.block_size + 40  # beyond the row: flagged and clamped
    runner.attend(b)
    torch.cuda.synchronize()
    assert pa.workspace_error(b.workspace) == 3


def test_bad_table_entry_in_prompt_rows_is_flagged(cuda_device):
    wl = W.mixed_prefill(16, "small")
    b = runner.setup(wl, cuda_device)
    runner.step(b)
    torch.cuda.synchronize()
    assert pa.workspace_error(b.workspace) == 0
    b.tables[0, 0] = -1  # sequence 0 is a prefill chunk
    runner.attend(b)
    torch.cuda.synchronize()
    assert pa.workspace_error(b.workspace) == 2


FULL = [("gqa_bf16", None), ("prefix_bf16", [0, 1, 2, 127, 128, 129, 200, 255]), ("fp8_long", [0, 77]),
        ("mixed_prefill_bs16", [0, 7, 8, 100, 255]), ("mixed_prefill_bs32", [3, 100]), ("long_prefix_bf16", [0, 63])]


@pytest.mark.slow
@pytest.mark.parametrize("name,seqs", FULL)
def test_workload_full_size_sampled(name, seqs, cuda_device):
    """Full-size workload, launched exactly as bench.py does; the oracle checks
    sampled sequences (their rows, their cache bytes) and the full tables."""
    run_and_check(W.make(name, "full"), cuda_device, seqs)


def test_merge_wait_that_runs_out_is_reported_and_the_next_call_is_correct(cuda_device):
    """Failure detection without a GPU fault: the workspace's fault-injection
    word makes the later pieces of every cut context skip their count-in,
    so each merging warp's bounded wait runs out (after 1 ms) and sets error
    word 1.  The call returns, the context stays usable, and once the
    workspace is zeroed again the next call gives the same bits as before."""
    import time
    wl = W.custom("merge_timeout", context_lens=[2000] * 20, num_q_heads=32, num_kv_heads=8)
    b = runner.setup(wl, cuda_device)
    runner.step(b)
    torch.cuda.synchronize()
    assert pa.workspace_error(b.workspace) == 0
    ref = b.out.clone()
    b.workspace.view(torch.int32)[1] = 1
    t0 = time.perf_counter()
    runner.attend(b)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert pa.workspace_error(b.workspace) == 1
    assert elapsed < 1.0, f"the injected wait should end after about 1 ms, took {elapsed:.3f} s"
    b.workspace.zero_()
    runner.attend(b)
    torch.cuda.synchronize()
    assert pa.workspace_error(b.workspace) == 0
    assert torch.equal(b.out.view(torch.int16), ref.view(torch.int16))
