"""pa_decode_prefix: each shared prefix attended once for all the sequences
that share it (a dense contraction on the tensor cores), merged with every
sequence's own suffix by a log-sum-exp combine ("49 vLLM / PagedAttention",
Почему это важно; "PagedAttention：KV cache 即虚拟内存（block manager &
碎片）", 深入原理, 共享 → prefix caching).

The result must be the oracle's attention over the whole context within the
bf16 tolerance, as pa_decode's is.  Cases: the prefix_bf16 workload, several
prefixes in one batch, more members than one 128-row tile holds, prefixes
that end inside a key chunk, a suffix of only the new token, block 32, head
dim 64, GQA groups 2 and 8, and replays from a CUDA graph.
"""
import numpy as np
import pytest
import torch

import pa_workloads as W
import paged_kv_cache_452_b200 as pa
from oracle.workload import expected
from paged_kv_cache_452_b200 import runner

pytestmark = pytest.mark.gpu

TOL = 2e-2


def _groups_case(name, n_groups, members, prefix_len, suffix_hi, private, seed=0, **kw):
    g = np.random.default_rng(seed)
    groups, ctx = [], []
    for grp in range(n_groups):
        for _ in range(members):
            groups.append(grp)
            ctx.append(prefix_len + int(g.integers(0, suffix_hi + 1)))
    for _ in range(private):
        groups.append(-1)
        ctx.append(int(g.integers(0, suffix_hi + prefix_len + 1)))
    return W.custom(name, context_lens=ctx, prefix_len=prefix_len, prefix_group=groups, **kw)


CASES = {
    "prefix_bf16": lambda: W.make("prefix_bf16", "small"),
    # every sequence shares the prefix: one prefix of 20 blocks, chunks of 256 + 64 keys
    "long_prefix_bf16": lambda: W.make("long_prefix_bf16", "small"),
    # 3 member tiles of 32 (group 4), a 20-block prefix: chunks of 256 + 64 keys
    "many_members": lambda: _groups_case("many_members", 1, 80, 320, 300, 10, num_q_heads=32, num_kv_heads=8),
    "two_prefixes": lambda: _groups_case("two_prefixes", 2, 7, 96, 150, 5, seed=1),
    # suffix of only the new token for some members (context == prefix)
    "new_token_only": lambda: _groups_case("new_token_only", 1, 6, 64, 0, 2, seed=2),
    "bs32_head64_group8": lambda: _groups_case("bs32_head64_group8", 2, 9, 96, 100, 3, seed=3, block_size=32,
                                               head_dim=64, num_q_heads=16, num_kv_heads=2),
    "group2": lambda: _groups_case("group2", 1, 70, 512, 40, 4, seed=4, num_q_heads=4, num_kv_heads=2),
    # long suffixes cut across warps: the merging warp folds contributors and prefix chunks
    "split_suffixes": lambda: _groups_case("split_suffixes", 1, 20, 1024, 3000, 4, seed=5, num_q_heads=32,
                                           num_kv_heads=8),
}


def _run(wl, device):
    b = runner.setup(wl, device)
    plan = runner.prefix_plan(b)
    runner.write_step(b)
    b.out.fill_(float("nan"))
    runner.attend_prefix(b, plan)
    torch.cuda.synchronize()
    return b, plan


@pytest.mark.parametrize("name", sorted(CASES))
def test_prefix_decode_matches_oracle(name, cuda_device):
    wl = CASES[name]()
    b, plan = _run(wl, cuda_device)
    assert plan.groups.num_prefixes >= 1, "the case must share a prefix"
    assert pa.workspace_error(plan.workspace) == 0
    exp = expected(wl)
    out = b.out.detach().cpu().double().numpy()[exp["rows"]]
    assert np.isfinite(out).all()
    err = float(np.abs(out - exp["out"]).max())
    assert err <= TOL, f"max abs error {err}"
    # the shared blocks really are shared: one physical run in every member's row
    g = plan.groups
    for p in range(g.num_prefixes):
        mem = g.prefix_members[int(g.prefix_start[p]):int(g.prefix_start[p + 1])].tolist()
        nblk = int(g.prefix_blocks[p])
        rows = b.tables_host[mem, :nblk]
        assert torch.equal(rows, rows[:1].expand_as(rows))


def test_prefix_chunk_whose_later_keys_outscore_its_first_tile(cuda_device):
    """The shared-prefix kernel's rows take the slow path inside a chunk: a
    640-token prefix (chunks of 256 keys), keys 160.. scaled."""
    from test_gpu_parity import outscoring_draws
    wl = outscoring_draws(W.custom("outscore_prefix", context_lens=[700, 660, 720, 645], num_q_heads=8,
                                   num_kv_heads=2, prefix_len=640, prefix_group=[0, 0, 0, 0]),
                          late_from=160, factor=48.0)
    b, plan = _run(wl, cuda_device)
    assert plan.groups.num_prefixes == 1
    assert pa.workspace_error(plan.workspace) == 0
    exp = expected(wl)
    out = b.out.detach().cpu().double().numpy()[exp["rows"]]
    assert np.isfinite(out).all()
    err = float(np.abs(out - exp["out"]).max())
    assert err <= TOL, f"max abs error {err}"


def test_prefix_decode_replayed_from_a_graph(cuda_device):
    wl = CASES["many_members"]()
    b, plan = _run(wl, cuda_device)
    first = b.out.clone()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        runner.attend_prefix(b, plan)
    for _ in range(4):
        b.out.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(b.out.view(torch.int16), first.view(torch.int16))
    assert pa.workspace_error(plan.workspace) == 0


def test_prefix_decode_without_groups_is_pa_decode(cuda_device):
    wl = W.make("gqa_bf16", "small")  # no shared blocks: pa_decode runs
    b, plan = _run(wl, cuda_device)
    assert plan.groups.num_prefixes == 0
    ref = b.out.clone()
    runner.attend(b)
    torch.cuda.synchronize()
    assert torch.equal(b.out.view(torch.int16), ref.view(torch.int16))


def test_prefix_longer_than_a_context_is_flagged(cuda_device):
    """A caller-made group whose prefix reaches a member's last token: the
    member's row is zero and error word 4 is set, without a fault."""
    wl = CASES["two_prefixes"]()
    b = runner.setup(wl, cuda_device)
    runner.write_step(b)
    plan = runner.prefix_plan(b)
    s = int(plan.groups.prefix_members[0])
    plan.dev["prefix_blocks"][0] = (int(b.seq_lens[s]) - 1) // wl.block_size + 1  # covers the new token
    plan.groups.max_prefix_blocks = max(plan.groups.max_prefix_blocks, int(plan.dev["prefix_blocks"][0]))
    plan.workspace = pa.alloc_workspace(pa.pa_decode_prefix_workspace_size(
        b.desc, b.seq_lens.shape[0], plan.groups.num_members, plan.groups.max_prefix_blocks), cuda_device)
    runner.attend_prefix(b, plan)
    torch.cuda.synchronize()
    assert pa.workspace_error(plan.workspace) == 4
    assert float(b.out[s].float().abs().max()) == 0.0


@pytest.mark.slow
@pytest.mark.parametrize("name,members,seqs", [
    ("prefix_bf16", 128, [0, 1, 63, 127, 128, 200, 255]),
    # a 32768-token prefix: eight chunks of 4096 keys (32-tile units), folded
    # eight deep into every member's suffix
    ("long_prefix_bf16", 64, [0, 31, 63]),
])
def test_prefix_decode_full_size_sampled(name, members, seqs, cuda_device):
    wl = W.make(name, "full")
    b, plan = _run(wl, cuda_device)
    assert plan.groups.num_prefixes == 1 and plan.groups.num_members == members
    assert pa.workspace_error(plan.workspace) == 0
    exp = expected(wl, seqs)
    out = b.out.detach().cpu().double().numpy()[exp["rows"]]
    err = float(np.abs(out - exp["out"]).max())
    assert err <= TOL, f"max abs error {err}"
