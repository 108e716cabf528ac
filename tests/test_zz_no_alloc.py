"""pa_decode_static, the entry point for callers that cannot allocate device
memory (no workspace: it uses a fixed scratch area built into the library).

Runs last (file name), so a failure here cannot hide any other test.  It
must pass alone in a fresh process and after the rest of the suite: the
scratch area keeps the previous call's contents, so two calls in a row are
checked against pa_decode with a caller workspace (the same kernels and the
same split points, so the same bits) and against the CPU oracle.
"""
import numpy as np
import pytest
import torch

import pa_workloads as W
import paged_kv_cache_452_b200 as pa
from oracle.workload import expected
from paged_kv_cache_452_b200 import runner

pytestmark = pytest.mark.gpu

TOL = {"bf16": 2e-2, "e4m3": 6e-2, "f32": 1e-4}

CASES = {
    "gqa_bf16": None, "fp8_long": None, "prefix_bf16": None,
    # group 8 over 6016 tiles: the largest partial slots, contexts cut at
    # many warp-range edges (still within the 8 MiB area)
    "group8": dict(context_lens=[3000] * 16, num_q_heads=16, num_kv_heads=2),
    # the CUDA-core path: fp32, and bf16 with a GQA group of 1
    "tiny_fp32": None,
    "mha_bf16": dict(context_lens=[7, 100, 0, 33], num_q_heads=4, num_kv_heads=4),
}


def _bits(t):
    return t.detach().cpu().contiguous().view(torch.int32 if t.dtype == torch.float32 else torch.int16)


@pytest.mark.parametrize("name", sorted(CASES))
def test_static_scratch_matches_workspace_path_and_oracle(name, cuda_device):
    kw = CASES[name]
    wl = W.custom(name, **kw) if kw else W.make(name, "small")
    b = runner.setup(wl, cuda_device)
    runner.step(b)  # pa_cache_write + pa_decode with a caller workspace
    torch.cuda.synchronize()
    assert pa.workspace_error(b.workspace) == 0
    ref = _bits(b.out)
    exp = expected(wl)
    for _ in range(2):  # the second call finds the first one's scratch contents
        b.out.fill_(float("nan"))
        pa.pa_decode_static(b.desc, b.q, b.k_cache, b.v_cache, b.tables, b.seq_lens, b.scale, b.out)
        torch.cuda.synchronize()
        assert torch.equal(_bits(b.out), ref), "static scratch and caller workspace differ"
        got = b.out.detach().cpu().double().numpy()[exp["rows"]]
        err = float(np.abs(got - exp["out"]).max())
        assert err <= TOL[wl.kv_dtype], err


def test_static_scratch_rejects_oversized_batch(cuda_device):
    # 16384 sequences x 64 kv heads need more arrival counters than the
    # 8 MiB area holds: refused by the host-side size check, before any
    # pointer is used (the test checks that precondition first)
    desc = pa.CacheDesc.make(64, 16, 64, 512, 128, "bf16", "bf16")
    assert pa.pa_decode_workspace_size(desc, 16384) > 8 << 20
    tiny = torch.empty(16, dtype=torch.uint8, device=cuda_device)
    with pytest.raises(pa.PaError) as e:
        pa.pa_decode_static(desc, tiny, tiny, tiny, torch.empty((16384, 1), dtype=torch.int32),
                            torch.empty(16384, dtype=torch.int32), 1.0, tiny)
    assert e.value.code == 2 and "static area holds" in str(e.value)


def test_static_scratch_rejects_unbuilt_shape(cuda_device):
    desc = pa.CacheDesc.make(16, 16, 8, 32, 96, "bf16", "bf16")  # head_dim 96 is not built
    tiny = torch.empty(16, dtype=torch.uint8, device=cuda_device)
    with pytest.raises(pa.PaError):
        pa.pa_decode_static(desc, tiny, tiny, tiny, torch.empty((1, 1), dtype=torch.int32),
                            torch.empty(1, dtype=torch.int32), 1.0, tiny)
