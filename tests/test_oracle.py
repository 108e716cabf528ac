"""Pins for the CPU oracle: each function is tied to something other than
itself -- a library routine (torch fp64 scaled_dot_product_attention, torch's
float8_e4m3fn cast), a closed form, brute force on tiny inputs, or an exact
invariant the pages state (paged output = dense output)."""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle

E4M3 = torch.float8_e4m3fn


def _torch_e4m3_value(codes):
    return torch.from_numpy(np.asarray(codes, dtype=np.uint8)).view(E4M3).to(torch.float64).numpy()


# ---------------------------------------------------------------- e4m3 codec

def test_e4m3_decode_matches_torch_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    mine = oracle.e4m3_decode(codes)
    ref = _torch_e4m3_value(codes)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(mine), nan)
    assert set(codes[nan].tolist()) == {0x7F, 0xFF}
    assert np.array_equal(mine[~nan], ref[~nan])
    assert np.array_equal(np.signbit(mine[~nan]), np.signbit(ref[~nan]))


def test_e4m3_decode_special_values():
    d = oracle.e4m3_decode
    assert d([0x7E])[0] == 448.0
    assert d([0xFE])[0] == -448.0
    assert d([0x01])[0] == 2.0 ** -9  # smallest subnormal
    assert d([0x07])[0] == 7 * 2.0 ** -9  # largest subnormal
    assert d([0x08])[0] == 2.0 ** -6  # smallest normal
    assert d([0x38])[0] == 1.0
    assert d([0x80])[0] == 0.0 and np.signbit(d([0x80])[0])


def test_e4m3_encode_roundtrip_all_finite_codes():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    vals = oracle.e4m3_decode(codes).astype(np.float32)
    assert np.array_equal(oracle.e4m3_encode(vals), codes)


def test_e4m3_encode_ties_to_even():
    enc = oracle.e4m3_encode
    assert enc([1.0 + 1 / 16])[0] == 0x38  # between 1.0 (m=0) and 1.125 (m=1) -> 1.0
    assert enc([1.0 + 3 / 16])[0] == 0x3A  # between 1.125 and 1.25 -> 1.25 (m=2)
    assert enc([2.0 ** -10])[0] == 0x00  # between 0 and 2^-9 -> 0
    assert enc([3 * 2.0 ** -10])[0] == 0x02  # between 2^-9 and 2^-8 -> 2^-8
    assert enc([432.0])[0] == 0x7E  # between 416 (m=5) and 448 (m=6) -> 448
    assert enc([-1.0 - 1 / 16])[0] == 0xB8


def test_e4m3_encode_saturates_and_nan():
    enc = oracle.e4m3_encode
    for v in [448.0, 448.5, 463.9, 464.0, 1e9, float("inf")]:
        assert enc([v])[0] == 0x7E
        assert enc([-v])[0] == 0xFE
    assert enc([float("nan")])[0] == 0x7F


def test_e4m3_encode_matches_torch_in_range():
    g = np.random.default_rng(7)
    x = np.concatenate([
        g.uniform(-448, 448, 20000),
        g.standard_normal(20000) * 0.01,
        # exact midpoints between neighbouring codes, both signs
        (oracle.e4m3_decode(np.arange(0, 0x7E)) + oracle.e4m3_decode(np.arange(1, 0x7F))) / 2,
        -(oracle.e4m3_decode(np.arange(0, 0x7E)) + oracle.e4m3_decode(np.arange(1, 0x7F))) / 2,
    ]).astype(np.float32)
    mine = oracle.e4m3_encode(x)
    ref = torch.from_numpy(x).to(E4M3).view(torch.uint8).numpy()
    assert np.array_equal(mine, ref)


# ---------------------------------------------------------------- cache write

def test_cache_write_index_by_hand():
    nb, hkv, bs, d = 3, 2, 4, 3
    kc = oracle.new_cache(nb, hkv, bs, d, "f32")
    vc = oracle.new_cache(nb, hkv, bs, d, "f32")
    t = 4
    k = np.arange(t * hkv * d, dtype=np.float32).reshape(t, hkv, d) + 1
    v = -k
    slots = np.array([5, -1, 11, 0], dtype=np.int64)
    oracle.cache_write(k, v, slots, kc, vc, "f32", "f32")
    # slot 5 -> block 1 offset 1; slot 11 -> block 2 offset 3; slot 0 -> block 0 offset 0
    expect = {(1, 1): 0, (2, 3): 2, (0, 0): 3}
    for b in range(nb):
        for o in range(bs):
            if (b, o) in expect:
                tok = expect[(b, o)]
                assert np.array_equal(kc[b, :, o, :], k[tok])
                assert np.array_equal(vc[b, :, o, :], v[tok])
            else:
                assert np.isnan(kc[b, :, o, :]).all() and np.isnan(vc[b, :, o, :]).all()
    with pytest.raises(ValueError):
        oracle.cache_write(k[:1], v[:1], np.array([12]), kc, vc, "f32", "f32")


def test_copy_blocks_by_hand():
    """Block 1 copied to block 3 (and block 0 to block 2), checked element by
    element against the values written by hand; the other blocks keep theirs."""
    nb, hkv, bs, d = 4, 2, 4, 3
    kc, vc = oracle.new_caches(nb, hkv, bs, d, "e4m3")  # V d-major, sentinel 0x7F
    for b in range(nb):
        for h in range(hkv):
            for o in range(bs):
                for e in range(d):
                    kc[b, h, o, e] = (b * 64 + h * 16 + o * 4 + e) % 127
                    vc[b, h, e, o] = (b * 32 + h * 8 + e * 4 + o + 1) % 127
    k0, v0 = kc.copy(), vc.copy()
    oracle.copy_blocks(kc, vc, [(1, 3), (0, 2)])
    for h in range(hkv):
        for o in range(bs):
            for e in range(d):
                assert kc[3, h, o, e] == (64 + h * 16 + o * 4 + e) % 127
                assert vc[3, h, e, o] == (32 + h * 8 + e * 4 + o + 1) % 127
                assert kc[2, h, o, e] == (h * 16 + o * 4 + e) % 127
                assert vc[2, h, e, o] == (h * 8 + e * 4 + o + 1) % 127
    assert np.array_equal(kc[:2], k0[:2]) and np.array_equal(vc[:2], v0[:2])
    oracle.copy_blocks(kc, vc, [])
    assert np.array_equal(kc[:2], k0[:2])


def test_copy_blocks_keeps_attention():
    """A table that points at the copy gives the same fp64 output as one that
    points at the original (what copy-on-write relies on)."""
    p = _paged_problem([40], 4, 2, 16, 16, seed=3, shuffle=True)
    kc, vc, tab = p["kc"], p["vc"], p["tables"]
    used = set(tab[0][tab[0] >= 0].tolist())
    free = [b for b in range(kc.shape[0]) if b not in used][:1]
    src = int(tab[0, 1])
    oracle.copy_blocks(kc, vc, [(src, free[0])])
    moved = tab.copy()
    moved[0, 1] = free[0]
    q = np.random.default_rng(4).standard_normal((1, 4, 16))
    oa = oracle.attention(q, [0], [39], tab, kc, vc, "f32", 4, 0.25)
    ob = oracle.attention(q, [0], [39], moved, kc, vc, "f32", 4, 0.25)
    assert np.array_equal(oa, ob)


def test_cache_write_bf16_is_bit_copy():
    nb, hkv, bs, d = 4, 2, 16, 8
    kc = oracle.new_cache(nb, hkv, bs, d, "bf16")
    vc = oracle.new_cache(nb, hkv, bs, d, "bf16")
    g = np.random.default_rng(1)
    k = torch.from_numpy(g.standard_normal((5, hkv, d), dtype=np.float32)).bfloat16()
    v = torch.from_numpy(g.standard_normal((5, hkv, d), dtype=np.float32)).bfloat16()
    kb = k.view(torch.int16).numpy().view(np.uint16)
    vb = v.view(torch.int16).numpy().view(np.uint16)
    slots = np.array([63, 0, 17, 31, 32])
    oracle.cache_write(kb, vb, slots, kc, vc, "bf16", "bf16")
    for t, s in enumerate(slots):
        assert np.array_equal(kc[s // bs, :, s % bs], kb[t])
        assert np.array_equal(vc[s // bs, :, s % bs], vb[t])


def test_cache_write_fp8_matches_torch_quantisation():
    nb, hkv, bs, d = 8, 2, 16, 32
    g = np.random.default_rng(2)
    k = torch.from_numpy(g.standard_normal((40, hkv, d), dtype=np.float32)).bfloat16()
    v = torch.from_numpy(3 * g.standard_normal((40, hkv, d), dtype=np.float32)).bfloat16()
    ks = float(np.float32(k.abs().max().item()) / np.float32(448))
    vs = float(np.float32(v.abs().max().item()) / np.float32(448))
    kc, vc = oracle.new_caches(nb, hkv, bs, d, "e4m3")
    slots = g.permutation(nb * bs)[:40]
    oracle.cache_write(k.view(torch.int16).numpy().view(np.uint16),
                       v.view(torch.int16).numpy().view(np.uint16), slots, kc, vc, "bf16", "e4m3",
                       ks, vs)
    kq = (k.float() / torch.tensor(ks, dtype=torch.float32)).to(E4M3).view(torch.uint8).numpy()
    vq = (v.float() / torch.tensor(vs, dtype=torch.float32)).to(E4M3).view(torch.uint8).numpy()
    for t, s in enumerate(slots):
        assert np.array_equal(kc[s // bs, :, s % bs], kq[t])
        assert np.array_equal(vc[s // bs, :, :, s % bs], vq[t])  # V is d-major for e4m3


def test_cache_write_fp8_v_is_d_major_by_hand():
    nb, hkv, bs, d = 2, 1, 4, 3
    kc, vc = oracle.new_caches(nb, hkv, bs, d, "e4m3")
    k = np.array([[[1.0, 2.0, 3.0]]], dtype=np.float32)
    oracle.cache_write(k, -k, np.array([6]), kc, vc, "f32", "e4m3", 1.0, 1.0)
    flat_v = vc.ravel()
    # slot 6 -> block 1, offset 2; element d sits at ((1*1+0)*3 + d)*4 + 2
    assert [flat_v[(3 + dd) * 4 + 2] for dd in range(3)] == [0xB8, 0xC0, 0xC4]  # -1, -2, -3
    assert [kc.ravel()[(1 * 4 + 2) * 3 + dd] for dd in range(3)] == [0x38, 0x40, 0x44]
    assert (flat_v == 0x7F).sum() == flat_v.size - 3


# ---------------------------------------------------------------- attention

def _paged_problem(lens, hq, hkv, d, bs, kv_dtype="f32", seed=0, shuffle=True, q_rows=None):
    """Random K/V per sequence, scattered into a pool through a random (or
    identity) block assignment; returns everything the checks need."""
    g = np.random.default_rng(seed)
    nblk = [-(-n // bs) for n in lens]
    nb = sum(nblk) + 3
    phys = np.random.default_rng(seed + 1000).permutation(nb) if shuffle else np.arange(nb)
    tables = np.full((len(lens), max(nblk)), -1, dtype=np.int32)
    pos = 0
    for s, m in enumerate(nblk):
        tables[s, :m] = phys[pos:pos + m]
        pos += m
    ks = [g.standard_normal((n, hkv, d)).astype(np.float32) for n in lens]
    vs = [g.standard_normal((n, hkv, d)).astype(np.float32) for n in lens]
    kc, vc = oracle.new_caches(nb, hkv, bs, d, kv_dtype)
    for s, n in enumerate(lens):
        slots = np.array([tables[s, p // bs] * bs + p % bs for p in range(n)], dtype=np.int64)
        oracle.cache_write(ks[s], vs[s], slots, kc, vc, "f32", kv_dtype)
    return dict(tables=tables, ks=ks, vs=vs, kc=kc, vc=vc)


def _sdpa(qrow, k, v, scale, hq, hkv, upto):
    """torch fp64 SDPA for one query row [Hq][D] over keys 0..upto."""
    qq = torch.from_numpy(qrow).double()[:, None, :]  # [Hq, 1, D]
    kk = torch.from_numpy(k[: upto + 1]).double().permute(1, 0, 2)  # [Hkv, n, D]
    vv = torch.from_numpy(v[: upto + 1]).double().permute(1, 0, 2)
    o = F.scaled_dot_product_attention(qq[None], kk[None], vv[None], scale=scale, enable_gqa=True)
    return o[0, :, 0, :].numpy()


@pytest.mark.parametrize("hq,hkv,d,bs", [(8, 2, 16, 4), (4, 4, 8, 16), (8, 1, 32, 32)])
def test_attention_matches_torch_sdpa_decode(hq, hkv, d, bs):
    lens = [1, 5, 16, 33, 70]
    P = _paged_problem(lens, hq, hkv, d, bs)
    g = np.random.default_rng(3)
    q = g.standard_normal((len(lens), hq, d))
    scale = 1 / math.sqrt(d)
    out = oracle.attention(q, np.arange(len(lens)), np.array(lens) - 1, P["tables"], P["kc"], P["vc"],
                           "f32", hq, scale)
    for s, n in enumerate(lens):
        ref = _sdpa(q[s], P["ks"][s], P["vs"][s], scale, hq, hkv, n - 1)
        np.testing.assert_allclose(out[s], ref, rtol=0, atol=1e-12)


def test_attention_over_a_bf16_cache_matches_torch_sdpa():
    """The bf16 load path: K/V rounded to bf16 by torch, written as bf16 bits,
    attended by the oracle = torch fp64 SDPA on torch's bf16 values."""
    lens = [3, 16, 41]
    hq, hkv, d, bs = 8, 2, 16, 16
    g = np.random.default_rng(31)
    nb = sum(-(-n // bs) for n in lens) + 2
    tables = np.full((len(lens), max(-(-n // bs) for n in lens)), -1, dtype=np.int32)
    phys = g.permutation(nb)
    kc, vc = oracle.new_caches(nb, hkv, bs, d, "bf16")
    kvals, vvals, pos = [], [], 0
    for s, n in enumerate(lens):
        m = -(-n // bs)
        tables[s, :m] = phys[pos:pos + m]
        pos += m
        k = torch.from_numpy(g.standard_normal((n, hkv, d), dtype=np.float32)).bfloat16()
        v = torch.from_numpy(g.standard_normal((n, hkv, d), dtype=np.float32)).bfloat16()
        slots = np.array([tables[s, p // bs] * bs + p % bs for p in range(n)])
        oracle.cache_write(k.view(torch.int16).numpy().view(np.uint16), v.view(torch.int16).numpy().view(np.uint16),
                           slots, kc, vc, "bf16", "bf16")
        kvals.append(k.double().numpy())
        vvals.append(v.double().numpy())
    q = g.standard_normal((len(lens), hq, d))
    out = oracle.attention(q, np.arange(len(lens)), np.array(lens) - 1, tables, kc, vc, "bf16", hq, 0.25)
    for s, n in enumerate(lens):
        ref = _sdpa(q[s], kvals[s], vvals[s], 0.25, hq, hkv, n - 1)
        np.testing.assert_allclose(out[s], ref, rtol=0, atol=1e-12)


def test_attention_matches_torch_sdpa_causal_rows():
    lens = [23, 50]
    hq, hkv, d, bs = 6, 3, 16, 8
    P = _paged_problem(lens, hq, hkv, d, bs, seed=4)
    g = np.random.default_rng(5)
    rows_seq, rows_pos = [], []
    for s, n in enumerate(lens):  # a chunk of queries at the last 7 positions
        for p in range(n - 7, n):
            rows_seq.append(s)
            rows_pos.append(p)
    q = g.standard_normal((len(rows_seq), hq, d))
    out = oracle.attention(q, rows_seq, rows_pos, P["tables"], P["kc"], P["vc"], "f32", hq, 0.3)
    for r, (s, p) in enumerate(zip(rows_seq, rows_pos)):
        ref = _sdpa(q[r], P["ks"][s], P["vs"][s], 0.3, hq, hkv, p)
        np.testing.assert_allclose(out[r], ref, rtol=0, atol=1e-12)


def test_paged_output_equals_dense_output_exactly():
    """Paging changes neither the output nor the compute: the same K/V stored
    through a shuffled table and through an identity (contiguous) table give
    bit-identical fp64 results."""
    lens = [3, 17, 64, 100]
    a = _paged_problem(lens, 8, 2, 16, 16, seed=9, shuffle=True)
    b = _paged_problem(lens, 8, 2, 16, 16, seed=9, shuffle=False)
    # same draws, different physical placement
    for s in range(len(lens)):
        assert np.array_equal(a["ks"][s], b["ks"][s])
    assert not np.array_equal(a["tables"], b["tables"])
    q = np.random.default_rng(10).standard_normal((len(lens), 8, 16))
    args = (np.arange(len(lens)), np.array(lens) - 1)
    oa = oracle.attention(q, *args, a["tables"], a["kc"], a["vc"], "f32", 8, 0.25)
    ob = oracle.attention(q, *args, b["tables"], b["kc"], b["vc"], "f32", 8, 0.25)
    assert np.array_equal(oa, ob)


def test_attention_brute_force_one_and_two_keys():
    d, bs = 4, 16
    P = _paged_problem([1, 2], 1, 1, d, bs, seed=11)
    q = np.random.default_rng(12).standard_normal((2, 1, d))
    out = oracle.attention(q, [0, 1], [0, 1], P["tables"], P["kc"], P["vc"], "f32", 1, 0.7)
    # one key: the output is that key's value row exactly
    assert np.array_equal(out[0, 0], P["vs"][0][0, 0].astype(np.float64))
    # two keys: weights are a logistic function of the logit difference
    k = P["ks"][1][:, 0].astype(np.float64)
    v = P["vs"][1][:, 0].astype(np.float64)
    s0 = 0.7 * (q[1, 0] @ k[0])
    s1 = 0.7 * (q[1, 0] @ k[1])
    w0 = 1 / (1 + math.exp(s1 - s0))
    np.testing.assert_allclose(out[1, 0], w0 * v[0] + (1 - w0) * v[1], rtol=0, atol=1e-15)


def test_gqa_head_mapping_contiguous_groups():
    """Query head h reads KV head h // (Hq / Hkv): give each KV head a
    constant V and check each query head returns its group's constant."""
    hq, hkv, d, bs, n = 6, 3, 4, 4, 9
    P = _paged_problem([n], hq, hkv, d, bs, seed=13)
    for b in range(P["vc"].shape[0]):
        for h in range(hkv):
            P["vc"][b, h] = np.where(np.isnan(P["vc"][b, h]), np.nan, float(h + 1))
    q = np.random.default_rng(14).standard_normal((1, hq, d))
    out = oracle.attention(q, [0], [n - 1], P["tables"], P["kc"], P["vc"], "f32", hq, 0.5)
    for h in range(hq):
        np.testing.assert_allclose(out[0, h], h // 2 + 1, rtol=0, atol=1e-14)


def test_fp8_attention_uses_dequantised_values():
    lens = [20, 37]
    hq, hkv, d, bs = 4, 2, 16, 16
    g = np.random.default_rng(15)
    P = _paged_problem(lens, hq, hkv, d, bs, seed=16)
    # requantise the cache to e4m3 with scales, then compare with SDPA on the
    # values torch decodes from the same codes
    ks, vs = 0.01, 0.02
    kc, vc = oracle.new_caches(*P["kc"].shape, "e4m3")
    for s, n in enumerate(lens):
        slots = np.array([P["tables"][s, p // bs] * bs + p % bs for p in range(n)])
        oracle.cache_write(P["ks"][s], P["vs"][s], slots, kc, vc, "f32", "e4m3", ks, vs)
    q = g.standard_normal((2, hq, d))
    out = oracle.attention(q, [0, 1], np.array(lens) - 1, P["tables"], kc, vc, "e4m3", hq, 0.25, ks, vs)
    for s, n in enumerate(lens):
        slots = [P["tables"][s, p // bs] * bs + p % bs for p in range(n)]
        kd = np.stack([_torch_e4m3_value(kc[x // bs, :, x % bs]) for x in slots]) * np.float64(np.float32(ks))
        vd = np.stack([_torch_e4m3_value(vc[x // bs, :, :, x % bs]) for x in slots]) * np.float64(np.float32(vs))
        ref = _sdpa(q[s], kd, vd, 0.25, hq, hkv, n - 1)
        np.testing.assert_allclose(out[s], ref, rtol=0, atol=1e-12)


# ------------------------------------------------- per-head fp8 scales

def test_per_head_quantisation_matches_torch():
    """One scale per kv head (amax of that head / 448): every code equals
    torch's e4m3 cast of x / scale_h in fp32."""
    nb, hkv, bs, d = 8, 4, 16, 32
    g = np.random.default_rng(21)
    mag = np.array([0.1, 1.0, 7.0, 300.0], dtype=np.float32)[None, :, None]  # very different heads
    k = torch.from_numpy(g.standard_normal((40, hkv, d), dtype=np.float32) * mag).bfloat16()
    v = torch.from_numpy(g.standard_normal((40, hkv, d), dtype=np.float32) * mag[:, ::-1]).bfloat16()
    ks = (k.float().abs().amax(dim=(0, 2)) / 448).numpy().astype(np.float32)
    vs = (v.float().abs().amax(dim=(0, 2)) / 448).numpy().astype(np.float32)
    assert len(set(ks.tolist())) == hkv
    kc, vc = oracle.new_caches(nb, hkv, bs, d, "e4m3")
    slots = g.permutation(nb * bs)[:40]
    oracle.cache_write(k.view(torch.int16).numpy().view(np.uint16), v.view(torch.int16).numpy().view(np.uint16),
                       slots, kc, vc, "bf16", "e4m3", ks, vs)
    kq = (k.float() / torch.from_numpy(ks)[None, :, None]).to(E4M3).view(torch.uint8).numpy()
    vq = (v.float() / torch.from_numpy(vs)[None, :, None]).to(E4M3).view(torch.uint8).numpy()
    for t, s in enumerate(slots):
        assert np.array_equal(kc[s // bs, :, s % bs], kq[t])
        assert np.array_equal(vc[s // bs, :, :, s % bs], vq[t])


def test_per_head_scales_all_equal_give_the_per_tensor_bits():
    lens = [23, 40]
    hq, hkv, d, bs = 8, 2, 16, 16
    P = _paged_problem(lens, hq, hkv, d, bs, seed=22)
    q = np.random.default_rng(23).standard_normal((2, hq, d))
    outs, caches = [], []
    for ks, vs in ((0.03, 0.05), (np.full(hkv, 0.03, np.float32), np.full(hkv, 0.05, np.float32))):
        kc, vc = oracle.new_caches(*P["kc"].shape, "e4m3")
        for s, n in enumerate(lens):
            slots = np.array([P["tables"][s, p // bs] * bs + p % bs for p in range(n)])
            oracle.cache_write(P["ks"][s], P["vs"][s], slots, kc, vc, "f32", "e4m3", ks, vs)
        caches.append((kc, vc))
        outs.append(oracle.attention(q, [0, 1], np.array(lens) - 1, P["tables"], kc, vc, "e4m3", hq, 0.25,
                                     ks, vs))
    assert np.array_equal(caches[0][0], caches[1][0]) and np.array_equal(caches[0][1], caches[1][1])
    assert np.array_equal(outs[0], outs[1])


def test_per_head_fp8_attention_uses_each_heads_scale():
    """GQA group 2 over 2 kv heads with different scales: SDPA on the values
    torch decodes from the same codes, each head times its own scale."""
    lens = [20, 37]
    hq, hkv, d, bs = 4, 2, 16, 16
    P = _paged_problem(lens, hq, hkv, d, bs, seed=24)
    ks = np.array([0.01, 0.004], dtype=np.float32)
    vs = np.array([0.02, 0.05], dtype=np.float32)
    kc, vc = oracle.new_caches(*P["kc"].shape, "e4m3")
    for s, n in enumerate(lens):
        slots = np.array([P["tables"][s, p // bs] * bs + p % bs for p in range(n)])
        oracle.cache_write(P["ks"][s], P["vs"][s], slots, kc, vc, "f32", "e4m3", ks, vs)
    q = np.random.default_rng(25).standard_normal((2, hq, d))
    out = oracle.attention(q, [0, 1], np.array(lens) - 1, P["tables"], kc, vc, "e4m3", hq, 0.25, ks, vs)
    for s, n in enumerate(lens):
        slots = [P["tables"][s, p // bs] * bs + p % bs for p in range(n)]
        kd = np.stack([_torch_e4m3_value(kc[x // bs, :, x % bs]) for x in slots]) * ks.astype(np.float64)[None, :, None]
        vd = np.stack([_torch_e4m3_value(vc[x // bs, :, :, x % bs]) for x in slots]) * vs.astype(np.float64)[None, :, None]
        ref = _sdpa(q[s], kd, vd, 0.25, hq, hkv, n - 1)
        np.testing.assert_allclose(out[s], ref, rtol=0, atol=1e-12)
    # and the scales matter: swapping them changes the output
    swapped = oracle.attention(q, [0, 1], np.array(lens) - 1, P["tables"], kc, vc, "e4m3", hq, 0.25,
                               ks[::-1].copy(), vs[::-1].copy())
    assert np.abs(swapped - out).max() > 1e-3
