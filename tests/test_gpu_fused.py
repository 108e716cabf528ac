"""pa_decode_fused: the new token's cache write and the decode attention in
one launch, against the CPU oracle and against pa_cache_write + pa_decode.

The write must store exactly the bytes pa_cache_write stores (e4m3
quantisation with per-tensor or per-kv-head scales included), so the whole
pool after a fused step equals the pool after the two-launch step, bit for
bit, and every checked position equals the oracle's write.  The attention
reads the same tiles with the same split points, so the output is the same
bits as the two-launch step's, and within the benchmark spec's tolerances of the
oracle.
"""
import numpy as np
import pytest
import torch

import pa_workloads as W
import paged_kv_cache_452_b200 as pa
from oracle.workload import expected
from paged_kv_cache_452_b200 import runner

from test_gpu_parity import TOL, check_cache, poison_workspace

pytestmark = pytest.mark.gpu

CASES = {
    "gqa_bf16": None, "prefix_bf16": None, "fp8_long": None,
    # block edges: the new token opens a block, ends one, or is the only key
    "bounds_bs16": dict(context_lens=[0, 1, 15, 16, 17, 31, 32, 33, 47, 48]),
    "bounds_bs32_head64": dict(context_lens=[0, 1, 31, 32, 33, 63, 64, 65], block_size=32, head_dim=64),
    "bounds_fp8_bs32": dict(context_lens=[0, 31, 32, 33, 200], kv_dtype="e4m3", block_size=32),
    "group8": dict(context_lens=[5, 80, 300], num_q_heads=16, num_kv_heads=2),
    # contexts cut across warps: the last tile is in a later warp's range
    "split_uniform": dict(context_lens=[2000] * 20, num_q_heads=32, num_kv_heads=8),
    "fp8_head_scales": dict(context_lens=[0, 5, 80, 300, 17, 4000], kv_dtype="e4m3", num_q_heads=16,
                            num_kv_heads=4, scale_mode="fixed", k_scale=[0.001, 0.01, 3.0, 0.5],
                            v_scale=[2.0, 0.0007, 0.05, 1.0]),
}


def _workload(name):
    kw = CASES[name]
    return W.custom(name, **kw) if kw else W.make(name, "small")


@pytest.mark.parametrize("name", sorted(CASES))
def test_fused_step_equals_write_then_decode_and_oracle(name, cuda_device):
    wl = _workload(name)
    fused = runner.setup(wl, cuda_device)
    two = runner.setup(_workload(name), cuda_device)
    poison_workspace(fused)
    poison_workspace(two)
    runner.step_fused(fused)
    runner.step(two)
    torch.cuda.synchronize()
    assert pa.workspace_error(fused.workspace) == 0
    # the whole pools, unused slots included, and the outputs: same bits
    assert torch.equal(fused.k_cache.view(torch.uint8), two.k_cache.view(torch.uint8))
    assert torch.equal(fused.v_cache.view(torch.uint8), two.v_cache.view(torch.uint8))
    assert torch.equal(fused.out.view(torch.int16), two.out.view(torch.int16))
    exp = expected(wl)
    check_cache(wl, fused, exp)
    out = fused.out.detach().cpu().double().numpy()[exp["rows"]]
    err = float(np.abs(out - exp["out"]).max())
    assert err <= TOL[wl.kv_dtype], f"max abs error {err}"


def test_fused_step_replayed_from_a_graph(cuda_device):
    wl = W.make("fp8_long", "small")
    b = runner.setup(wl, cuda_device)
    runner.step_fused(b)
    torch.cuda.synchronize()
    first = b.out.clone()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        runner.step_fused(b)
    for _ in range(4):
        b.out.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(b.out.view(torch.int16), first.view(torch.int16))
    assert pa.workspace_error(b.workspace) == 0


def test_fused_step_refuses_paths_it_does_not_fuse(cuda_device):
    wl = W.make("tiny_fp32")
    b = runner.setup(wl, cuda_device)
    with pytest.raises(pa.PaError) as e:
        runner.step_fused(b)
    assert e.value.code == 2
