"""Fork and copy-on-write through the C ABI: the block copy kernel against
the oracle's copy, bit for bit, and forked sequences that diverge inside a
shared block, end to end (pool, copies, cache write, decode) against the
pool model and the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_452_b200 as pa
from oracle.pool_model import BlockPoolModel

pytestmark = pytest.mark.gpu

RAW = {"bf16": torch.int16, "f32": torch.int32, "e4m3": torch.uint8}


def raw(t):
    """A device pool as host storage bits."""
    return t.detach().cpu().contiguous().view(RAW[{torch.uint8: "e4m3", torch.bfloat16: "bf16"}.get(t.dtype, "f32")]).numpy()


@pytest.mark.parametrize("kv,nb,bs,hkv,d", [("bf16", 40, 16, 8, 128), ("f32", 33, 16, 2, 64),
                                             ("e4m3", 25, 32, 4, 128), ("bf16", 9, 16, 1, 64)])
def test_copy_blocks_matches_oracle_bit_for_bit(kv, nb, bs, hkv, d, cuda_device):
    desc = pa.CacheDesc.make(nb, bs, hkv, hkv, d, kv, "f32" if kv == "f32" else "bf16")
    k, v = pa.alloc_cache(desc, cuda_device)
    g = torch.Generator(device=cuda_device).manual_seed(nb)
    for t in (k, v):  # arbitrary bytes, NaN patterns included
        t.view(torch.uint8).copy_(torch.randint(0, 256, t.view(torch.uint8).shape, generator=g,
                                                device=cuda_device, dtype=torch.uint8))
    rng = np.random.default_rng(nb)
    perm = rng.permutation(nb)
    n = nb // 3
    pairs = list(zip(perm[:n].tolist(), perm[n:2 * n].tolist()))  # sources and destinations disjoint
    skipped = [(-1, int(perm[-1])), (int(perm[-1]), nb + 3), (int(perm[-2]), int(perm[-2]))]
    src = torch.tensor([p[0] for p in pairs + skipped], dtype=torch.int32, device=cuda_device)
    dst = torch.tensor([p[1] for p in pairs + skipped], dtype=torch.int32, device=cuda_device)
    k_exp, v_exp = raw(k), raw(v)
    oracle.copy_blocks(k_exp, v_exp, pairs)
    pa.pa_copy_blocks(desc, src, dst, k, v)
    torch.cuda.synchronize()
    assert np.array_equal(raw(k), k_exp) and np.array_equal(raw(v), v_exp)
    pa.pa_copy_blocks(desc, src[:0], dst[:0], k, v)  # nothing to copy
    with pytest.raises(pa.PaError):
        pa.pa_copy_blocks(desc, src, dst[:1], k, v)


def _bf16_bits(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_forks_that_diverge_inside_a_shared_block(cuda_device):
    """A 37-token parent (its third block holds 5 of 16 slots) is forked
    twice; each of the three appends its own token, so the two children
    copy the shared block before writing.  Two steps: pools compared byte
    for byte with the oracle, decode outputs within the bf16 tolerance."""
    nb, bs, hkv, hq, d = 24, 16, 2, 8, 128
    desc = pa.CacheDesc.make(nb, bs, hkv, hq, d, "bf16", "bf16")
    order = np.random.default_rng(5).permutation(nb).tolist()
    pool, model = pa.BlockPool(nb, bs, order), BlockPoolModel(nb, bs, order)
    k_dev, v_dev = pa.alloc_cache(desc, cuda_device, fill=float("nan"))
    k_ref, v_ref = oracle.new_caches(nb, hkv, bs, d, "bf16")
    rng = np.random.default_rng(6)
    scale = pa.default_scale(d)

    def write(k_bits, v_bits, slots):
        oracle.cache_write(k_bits, v_bits, np.array(slots, dtype=np.int64), k_ref, v_ref, "bf16", "bf16")
        kt = torch.from_numpy(k_bits.view(np.int16)).view(torch.bfloat16).to(cuda_device)
        vt = torch.from_numpy(v_bits.view(np.int16)).view(torch.bfloat16).to(cuda_device)
        st = torch.tensor(slots, dtype=torch.int64, device=cuda_device)
        pa.pa_cache_write(desc, kt, vt, st, k_dev, v_dev)

    pool.add_seq(0, 37)
    model.add_seq(0, 37)
    write(_bf16_bits(rng.standard_normal((37, hkv, d))), _bf16_bits(rng.standard_normal((37, hkv, d))),
          pool.slots(0, 0, 37))
    for child in (1, 2):
        pool.fork(0, child)
        model.fork(0, child)
    seqs = [0, 1, 2]
    ws = pa.alloc_workspace(pa.pa_decode_workspace_size(desc, 3), cuda_device)
    for step, order_ in enumerate(([1, 2, 0], [2, 0, 1])):
        slots = {}
        for s in order_:
            slots[s] = pool.append(s, 1)
            assert slots[s] == model.append(s, 1)
        copies = pool.take_copies()
        assert copies == model.take_copies()
        assert len(copies) == (2 if step == 0 else 0)
        for s in seqs:
            assert pool.block_table(s) == model.block_table(s)
            assert pool.ref_cnt(pool.block_table(s)[-1]) == model.ref_cnt[model.block_table(s)[-1]]
        if copies:
            oracle.copy_blocks(k_ref, v_ref, copies)
            pa.pa_copy_blocks(desc, torch.tensor([c[0] for c in copies], dtype=torch.int32, device=cuda_device),
                              torch.tensor([c[1] for c in copies], dtype=torch.int32, device=cuda_device),
                              k_dev, v_dev)
        write(_bf16_bits(rng.standard_normal((3, hkv, d))), _bf16_bits(rng.standard_normal((3, hkv, d))),
              [slots[s][0] for s in seqs])
        mb = max(len(model.block_table(s)) for s in seqs)
        tab = np.full((3, mb), -1, dtype=np.int32)
        for i, s in enumerate(seqs):
            tab[i, :len(model.block_table(s))] = model.block_table(s)
        lens = np.array([model.num_tokens(s) for s in seqs], dtype=np.int32)
        q = torch.randn((3, hq, d), generator=torch.Generator().manual_seed(step)).to(torch.bfloat16)
        out = torch.empty((3, hq, d), dtype=torch.bfloat16, device=cuda_device)
        pa.pa_decode(desc, q.to(cuda_device), k_dev, v_dev, torch.from_numpy(tab).to(cuda_device),
                     torch.from_numpy(lens).to(cuda_device), scale, out, ws)
        torch.cuda.synchronize()
        assert pa.workspace_error(ws) == 0
        assert np.array_equal(raw(k_dev).view(np.uint16), k_ref) and np.array_equal(raw(v_dev).view(np.uint16), v_ref)
        exp = oracle.attention(q.float().numpy(), np.arange(3), lens - 1, tab, k_ref, v_ref, "bf16", hq, scale)
        err = float(np.abs(out.float().cpu().numpy() - exp).max())
        assert err <= 2e-2, err
    # the parent's copy of the shared block is its own again; the children's
    # copies are theirs
    assert len({model.block_table(s)[2] for s in seqs}) == 3
