"""The step captured into a CUDA graph and replayed, against the CPU oracle.

A serving loop captures its per-step launches once and replays them ("vLLM
innenfra: slik gjør paged attention GPU-minnet til blokker på 16 tokens",
the paragraph on start-up profiling and CUDA-graph capture).  Here the step
(pa_cache_write of the new tokens, then pa_decode or
pa_decode_chunked_prefill) is captured once per pool copy, and the copies are
replayed alternately, six times in all, as bench.py replays them.  Every
replay must give the oracle's output within the attention tolerances, the
same bits as the first replay of that copy and as the other copy, and leave
the workspace's error word at zero: the split-K merge puts its arrival
counters back to zero itself, which is what lets a captured launch run again.
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


def _bits(t):
    return t.detach().cpu().contiguous().view(torch.int32 if t.dtype == torch.float32 else torch.int16)


def replay_and_check(wl, device, seqs=None, replays=6):
    b0 = runner.setup(wl, device)
    batches = [b0, runner.clone(b0)]
    for b in batches:  # tensor maps and launch attributes are set up before capture
        runner.step(b)
    torch.cuda.synchronize()
    graphs = []
    for b in batches:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            runner.step(b)
        graphs.append(g)
    exp = expected(wl, seqs)
    first = [None, None]
    for i in range(replays):
        j = i & 1
        b = batches[j]
        b.out.fill_(float("nan"))  # a replay that wrote nothing would show
        graphs[j].replay()
        torch.cuda.synchronize()
        assert pa.workspace_error(b.workspace) == 0, f"replay {i}: error word set"
        bits = _bits(b.out)
        if first[j] is None:
            first[j] = bits
            got = b.out.detach().cpu().double().numpy()[exp["rows"]]
            err = float(np.abs(got - exp["out"]).max())
            assert err <= TOL[wl.kv_dtype], f"replay {i}: max abs error {err}"
        else:
            assert torch.equal(bits, first[j]), f"replay {i} differs from the first replay of its copy"
    assert torch.equal(first[0], first[1]), "the two pool copies give different bits"
    graphs.clear()


@pytest.mark.parametrize("name", ["gqa_bf16", "prefix_bf16", "fp8_long", "mixed_prefill_bs16", "tiny_fp32"])
def test_graph_replayed_step_matches_oracle(name, cuda_device):
    replay_and_check(W.make(name, "small"), cuda_device)


def test_graph_replayed_step_with_contexts_cut_across_warps(cuda_device):
    # several tiles per worker warp, so every context is split and merged:
    # the arrival counters are used and must be back at zero for each replay
    wl = W.custom("graph_split", context_lens=[2000] * 20 + [0, 17], num_q_heads=32, num_kv_heads=8)
    replay_and_check(wl, cuda_device)


@pytest.mark.slow
def test_graph_replayed_step_full_size_sampled(cuda_device):
    replay_and_check(W.make("gqa_bf16", "full"), cuda_device, seqs=[0, 1, 31, 63])
