"""Pins of the fp64 oracle to things other than itself (CPU only).

Each test names what fixes the expected value: the pages' worked example or
printed figures (fixtures under tests/golden/, with their citations), the
E4M3 format's closed forms, a library routine, brute force, or an invariant
the pages state.  Together they are chosen so that a dropped scale, a wrong
GQA head map, a transposed operand, an off-by-one in the gather or a wrong
block index fails at least one of them (see the planted-mistake tests at
the end).
"""

import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from oracle import codecs, paged, memory
from paged_kv_cache_416_b200.alloc import BlockAllocator
from paged_kv_cache_416_b200 import workloads as W
from paged_kv_cache_416_b200.workloads import raw

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# --------------------------------------------------------------------------
# the pages' worked example and printed figures
# --------------------------------------------------------------------------

def test_worked_example_block_table_and_gather():
    g = _golden("worked_example.json")
    bs, d = g["block_size"], g["head_dim"]
    alloc = BlockAllocator(g["pool_blocks"], bs, free_list=g["free_list"])
    n = g["num_tokens"]
    assert memory.blocks_needed(n, bs) == g["expected_blocks"]
    table = alloc.allocate(0, n)
    assert table == g["expected_block_table"]
    assert list(alloc.free) == g["expected_free_after"]
    # keys written through the table and read back are intact (bit-equal)
    rng = np.random.default_rng(0)
    keys = rng.standard_normal((n, 1, d)).astype(np.float32)
    pool = np.zeros((g["pool_blocks"], bs, 1, d), dtype=np.float32)
    slots = [oracle.slot_of(table, p, bs) for p in range(n)]
    assert slots == [alloc.slot(0, p) for p in range(n)]
    paged.write_kv(keys, keys, "f32", slots, pool, pool.copy(), "f32")
    back = paged.gather(pool, table, n)
    assert np.array_equal(back, keys) == g["expected_keys_intact"]
    # the rows live in the blocks the table names, at pos // bs, pos % bs
    assert np.array_equal(pool[41, :16], keys[:16]) and np.array_equal(pool[19, :8], keys[32:40])
    assert memory.paged_unused_slots([n], bs) == g["expected_unused_paged"]
    assert memory.reservation_unused_slots(n, g["reservation_tokens"]) == g["expected_unused_reserved"]


def test_printed_memory_figures():
    g = _golden("memory_figures.json")
    a = g["llama13b_one_sequence"]
    b13 = memory.kv_bytes(a["tokens"], a["layers"], a["kv_heads"], a["head_dim"], a["elem_bytes"])
    assert b13 == 2048 * 40 * 2 * 40 * 128 * 2
    assert round(b13 / 1e9, 1) == a["printed_gb"]
    b = g["llama31_70b_4096_tokens"]
    b70 = memory.kv_bytes(b["tokens"], b["layers"], b["kv_heads"], b["head_dim"], b["elem_bytes"])
    assert round(b70 / 1e9, 1) == b["printed_gb"]
    c = g["internal_fragmentation_4096"]
    waste = memory.reservation_unused_slots(c["used"], c["reserved"]) / c["reserved"]
    assert round(100 * waste) == c["printed_percent_wasted"]
    e = g["internal_fragmentation_1000"]
    assert memory.reservation_unused_slots(e["used"], e["reserved"]) == e["printed_unused"]


def test_paged_waste_is_below_one_block_per_sequence():
    rng = np.random.default_rng(3)
    lens = rng.integers(1, 5000, size=200)
    for bs in (16, 32):
        w = memory.paged_unused_slots(lens, bs)
        assert 0 <= w < bs * len(lens)
        assert w == sum((-(-int(n) // bs)) * bs - int(n) for n in lens)


# --------------------------------------------------------------------------
# codecs
# --------------------------------------------------------------------------

def test_e4m3_decode_closed_forms():
    dec = codecs.e4m3_decode
    assert dec(np.uint8(0x00)) == 0.0 and np.signbit(dec(np.uint8(0x80)))
    assert dec(np.uint8(0x01)) == 2.0 ** -9            # smallest subnormal
    assert dec(np.uint8(0x07)) == 7 * 2.0 ** -9        # largest subnormal
    assert dec(np.uint8(0x08)) == 2.0 ** -6            # smallest normal
    assert dec(np.uint8(0x38)) == 1.0                  # e = bias, m = 0
    assert dec(np.uint8(0x3C)) == 1.5
    assert dec(np.uint8(0x7E)) == 448.0                # largest finite
    assert dec(np.uint8(0xFE)) == -448.0
    assert np.isnan(dec(np.uint8(0x7F))) and np.isnan(dec(np.uint8(0xFF)))
    vals = codecs.e4m3_finite_values()
    assert len(vals) == 127 and np.all(np.diff(vals) > 0)
    # every normal binade holds 8 evenly spaced values
    for e in range(1, 16):
        seg = vals[8 * e: 8 * e + 8] if 8 * e + 8 <= 127 else vals[8 * e:]
        step = 2.0 ** (e - 7) / 8
        assert np.allclose(np.diff(seg), step)


def test_e4m3_roundtrip_every_finite_code():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    vals = codecs.e4m3_decode(codes).astype(np.float32)
    assert np.array_equal(codecs.e4m3_encode_f32(vals), codes)


def test_e4m3_encode_matches_library_cast():
    rng = np.random.default_rng(7)
    vals = codecs.e4m3_finite_values()
    mids = (vals[:-1] + vals[1:]) / 2  # exact ties
    x = np.concatenate([
        rng.standard_normal(400_000) * 3,
        rng.standard_normal(200_000) * 100,
        rng.uniform(-2.0 ** -6, 2.0 ** -6, 200_000),     # subnormal range
        mids, -mids, vals, -vals,
        np.nextafter(mids.astype(np.float32), np.float32(np.inf)),
        np.nextafter(mids.astype(np.float32), np.float32(-np.inf)),
        [0.0, -0.0, 463.99, -463.99, 448.0, 449.0],
    ]).astype(np.float32)
    x = x[np.abs(x) < 464.0]  # the library cast overflows to NaN beyond here
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = codecs.e4m3_encode_f32(x)
    assert np.array_equal(got, ref)


def test_e4m3_encode_saturates_and_nan():
    x = np.array([464.0, 480.0, 1e6, np.inf, -464.0, -np.inf, np.nan], dtype=np.float32)
    assert codecs.e4m3_encode_f32(x).tolist() == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE, 0x7F]


def test_16bit_decoders_match_library():
    rng = np.random.default_rng(1)
    w = rng.integers(0, 1 << 16, size=100_000, dtype=np.uint16)
    tf = torch.from_numpy(w.view(np.int16)).view(torch.float16).double().numpy()
    tb = torch.from_numpy(w.view(np.int16)).view(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(codecs.f16_bits_to_f64(w), tf)
    np.testing.assert_array_equal(codecs.bf16_bits_to_f64(w), tb)


# --------------------------------------------------------------------------
# attention: library routine, brute force, closed forms
# --------------------------------------------------------------------------

def _contiguous_case(rng, B, hq, hkv, d, bs, lens):
    """Pools holding each sequence's tokens in blocks 0.. in order
    (identity table), as fp64 values stored in float64 'raw' arrays."""
    nbs = [-(-n // bs) for n in lens]
    N = sum(nbs)
    kp = rng.standard_normal((N, bs, hkv, d))
    vp = rng.standard_normal((N, bs, hkv, d))
    tables = np.full((B, max(nbs)), -1, dtype=np.int64)
    o = 0
    for s, nb in enumerate(nbs):
        tables[s, :nb] = np.arange(o, o + nb)
        o += nb
    q = rng.standard_normal((B, hq, d))
    return q, kp, vp, tables


def _oracle_f64(q, kp, vp, tables, lens, scale, hkv):
    out = np.zeros_like(q)
    for s in range(q.shape[0]):
        out[s] = paged.decode_one(q[s], kp, vp, tables[s], int(lens[s]), scale, hkv)
    return out


@pytest.mark.parametrize("hq,hkv,d,bs", [(4, 4, 64, 16), (64, 8, 128, 16), (32, 8, 128, 32), (8, 1, 64, 16)])
def test_decode_matches_library_sdpa(hq, hkv, d, bs):
    rng = np.random.default_rng(hq * 131 + d)
    lens = [1, bs, bs + 1, 3 * bs - 5, 77]
    B = len(lens)
    q, kp, vp, tables = _contiguous_case(rng, B, hq, hkv, d, bs, lens)
    scale = 1.0 / math.sqrt(d)
    got = _oracle_f64(q, kp, vp, tables, lens, scale, hkv)
    for s, n in enumerate(lens):
        nb = -(-n // bs)
        K = torch.from_numpy(kp[tables[s, :nb]].reshape(-1, hkv, d)[:n]).permute(1, 0, 2)[None]
        V = torch.from_numpy(vp[tables[s, :nb]].reshape(-1, hkv, d)[:n]).permute(1, 0, 2)[None]
        Q = torch.from_numpy(q[s])[None, :, None, :]
        ref = F.scaled_dot_product_attention(Q, K, V, scale=scale, enable_gqa=True)[0, :, 0, :]
        np.testing.assert_allclose(got[s], ref.numpy(), rtol=1e-12, atol=1e-12)


def test_decode_matches_brute_force_on_tiny():
    """Pure-Python loops (math.exp), addressing each token through the table
    as the pages' sketch does, on scattered blocks."""
    rng = np.random.default_rng(11)
    hq, hkv, d, bs, N = 4, 2, 8, 4, 20
    lens = [1, 4, 5, 11]
    kp = rng.standard_normal((N, bs, hkv, d))
    vp = rng.standard_normal((N, bs, hkv, d))
    perm = rng.permutation(N)
    tables, o = [], 0
    for n in lens:
        nb = -(-n // bs)
        tables.append(list(perm[o:o + nb]) + [-1] * (3 - nb))
        o += nb
    q = rng.standard_normal((len(lens), hq, d))
    scale = 0.37
    got = _oracle_f64(q, kp, vp, np.array(tables), lens, scale, hkv)
    for s, n in enumerate(lens):
        for h in range(hq):
            kv = h // (hq // hkv)
            z = []
            for pos in range(n):
                b, off = tables[s][pos // bs], pos % bs
                z.append(scale * sum(q[s, h, i] * kp[b, off, kv, i] for i in range(d)))
            m = max(z)
            e = [math.exp(x - m) for x in z]
            tot = sum(e)
            for i in range(d):
                ref = sum(e[pos] / tot * vp[tables[s][pos // bs], pos % bs, kv, i] for pos in range(n))
                assert abs(got[s, h, i] - ref) < 1e-12


def test_decode_closed_forms():
    rng = np.random.default_rng(5)
    hq, hkv, d, bs = 4, 2, 16, 16
    q, kp, vp, tables = _contiguous_case(rng, 1, hq, hkv, d, bs, [40])
    t = tables[0]
    # one token: the output is that token's value row, exactly
    out = paged.decode_one(q[0], kp, vp, t, 1, 0.25, hkv)
    for h in range(hq):
        assert np.array_equal(out[h], vp[t[0], 0, h // 2])
    # q = 0: uniform weights, the mean of the value rows
    out = paged.decode_one(np.zeros((hq, d)), kp, vp, t, 40, 0.25, hkv)
    V = paged.gather(vp, t, 40)
    for h in range(hq):
        np.testing.assert_allclose(out[h], V[:, h // 2].mean(0), rtol=1e-12, atol=1e-13)
    # all keys equal: also the mean, whatever q is
    kp2 = kp.copy()
    kp2[t[:3]] = kp[t[0], 0]
    out = paged.decode_one(q[0], kp2, vp, t, 40, 0.25, hkv)
    for h in range(hq):
        np.testing.assert_allclose(out[h], V[:, h // 2].mean(0), rtol=1e-12, atol=1e-13)
    # one key far above the rest: its value row
    kp3 = np.zeros_like(kp)
    kp3[t[1], 5] = 1.0
    qd = np.ones((hq, d)) * 100.0
    out = paged.decode_one(qd, kp3, vp, t, 40, 1.0, hkv)
    for h in range(hq):
        np.testing.assert_allclose(out[h], vp[t[1], 5, h // 2], rtol=1e-12, atol=1e-12)
    # empty context: zeros
    assert not paged.decode_one(q[0], kp, vp, t, 0, 0.25, hkv).any()


def test_softmax_weights_sum_to_one():
    rng = np.random.default_rng(9)
    for n in (1, 2, 17, 4096):
        K = rng.standard_normal((n, 128)) * 3
        w = paged.attention_weights(rng.standard_normal(128), K, 1 / math.sqrt(128))
        assert abs(w.sum() - 1.0) < 1e-12 and (w >= 0).all()


# --------------------------------------------------------------------------
# paging invariants the pages state
# --------------------------------------------------------------------------

def test_physical_placement_does_not_change_the_result():
    """Blocks may sit wherever they are free: permuting physical ids (and
    moving the contents with them) gives the identical output."""
    rng = np.random.default_rng(21)
    hq, hkv, d, bs = 8, 2, 32, 16
    lens = [5, 16, 33, 100]
    q, kp, vp, tables = _contiguous_case(rng, 4, hq, hkv, d, bs, lens)
    base = _oracle_f64(q, kp, vp, tables, lens, 0.2, hkv)
    N = kp.shape[0]
    perm = rng.permutation(N)  # old id i -> new id perm[i]
    kp2, vp2 = np.empty_like(kp), np.empty_like(vp)
    kp2[perm], vp2[perm] = kp, vp
    t2 = np.where(tables >= 0, perm[np.maximum(tables, 0)], -1)
    assert np.array_equal(_oracle_f64(q, kp2, vp2, t2, lens, 0.2, hkv), base)


def test_shared_blocks_equal_unshared_copies():
    rng = np.random.default_rng(22)
    hq, hkv, d, bs = 4, 4, 16, 16
    # two sequences share 3 prefix blocks; the unshared version has copies
    kp = rng.standard_normal((12, bs, hkv, d))
    vp = rng.standard_normal((12, bs, hkv, d))
    shared = np.array([[0, 1, 2, 3], [0, 1, 2, 4]])
    kp[5:8], vp[5:8] = kp[0:3], vp[0:3]
    unshared = np.array([[0, 1, 2, 3], [5, 6, 7, 4]])
    q = rng.standard_normal((2, hq, d))
    lens = [60, 55]
    assert np.array_equal(_oracle_f64(q, kp, vp, shared, lens, 0.3, hkv),
                          _oracle_f64(q, kp, vp, unshared, lens, 0.3, hkv))


def test_unused_slots_and_table_entries_are_never_read():
    rng = np.random.default_rng(23)
    hq, hkv, d, bs = 4, 2, 16, 16
    q, kp, vp, tables = _contiguous_case(rng, 2, hq, hkv, d, bs, [20, 7])
    base = _oracle_f64(q, kp, vp, tables, [20, 7], 0.3, hkv)
    kp[tables[0, 1], 4:] = np.nan
    vp[tables[0, 1], 4:] = np.nan
    kp[tables[1, 0], 7:] = np.nan
    t = tables.copy()
    t[1, 1:] = 10**6  # past the sequence: never read
    assert np.array_equal(_oracle_f64(q, kp, vp, t, [20, 7], 0.3, hkv), base)


def test_copy_on_write_semantics():
    rng = np.random.default_rng(24)
    k = rng.integers(0, 1 << 16, size=(8, 16, 2, 8), dtype=np.uint16)
    v = rng.integers(0, 1 << 16, size=(8, 16, 2, 8), dtype=np.uint16)
    k0, v0 = k.copy(), v.copy()
    paged.copy_blocks(k, v, [[1, 5], [5, 6]])  # pairs read the state before any copy
    assert np.array_equal(k[5], k0[1]) and np.array_equal(v[5], v0[1])
    assert np.array_equal(k[6], k0[5]) and np.array_equal(v[6], v0[5])
    assert np.array_equal(k[1], k0[1])
    # a later write into the copy leaves the source untouched
    new = rng.integers(0, 1 << 16, size=(1, 2, 8), dtype=np.uint16)
    paged.write_kv(new, new, "bf16", [5 * 16 + 3], k, v, "bf16")
    assert np.array_equal(k[5, 3], new[0]) and np.array_equal(k[1], k0[1])


def test_allocator_copy_on_write_and_free():
    a = BlockAllocator(10, 4, free_list=range(10))
    a.allocate(0, 6)                      # blocks 0, 1 (second partial)
    a.fork(0, 1)
    a.fork(0, 2)
    assert a.refcount[0] == 3 and a.refcount[1] == 3
    s, cow = a.append_token(1)            # shared partial block -> copy first
    assert cow == (1, 2) and s == 2 * 4 + 2
    s, cow = a.append_token(2)
    assert cow == (1, 3)
    s, cow = a.append_token(0)            # last holder writes in place
    assert cow is None and s == 1 * 4 + 2 and a.refcount[1] == 1
    for _ in range(2):
        a.append_token(0)                 # fills block 1, then takes a new one
    assert a.tables[0] == [0, 1, 4] and a.lengths[0] == 9
    a.free_seq(1)
    assert a.refcount[0] == 2 and list(a.free)[-1] == 2
    a.free_seq(2)
    a.free_seq(0)
    assert a.used_blocks() == 0 and sorted(a.free) == list(range(10))


def test_write_kv_skips_padding_and_quantises_in_fp32():
    rng = np.random.default_rng(25)
    x = rng.standard_normal((3, 2, 8)).astype(np.float32)
    raw = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    kp = np.zeros((4, 4, 2, 8), dtype=np.uint8)
    vp = np.zeros((4, 4, 2, 8), dtype=np.uint8)
    paged.write_kv(raw, raw, "bf16", [5, -1, 15], kp, vp, "e4m3", k_scale=0.01, v_scale=0.02)
    xv = codecs.bf16_bits_to_f64(raw).astype(np.float32)
    assert np.array_equal(kp[1, 1], codecs.e4m3_encode_f32(xv[0] / np.float32(0.01)))
    assert np.array_equal(vp[3, 3], codecs.e4m3_encode_f32(xv[2] / np.float32(0.02)))
    assert kp.sum() == kp[1, 1].sum() + kp[3, 3].sum()  # the padding token wrote nothing


@pytest.mark.parametrize("in_dt", ["bf16", "f16"])
def test_write_kv_e4m3_matches_library_cast(in_dt):
    """The whole e4m3 branch of write_kv (decode of the 16-bit input, fp32
    division by the scale, RNE, saturation) against torch's own cast of
    (x.float() / scale).clamp(-448, 448) to float8_e4m3fn: random values at
    two scales, exact ties between neighbouring codes, values past the
    saturation boundary and infinities."""
    td = W.TORCH_DTYPE[in_dt]
    g = torch.Generator().manual_seed(31)
    hkv, d = 2, 64
    vals = torch.from_numpy(codecs.e4m3_finite_values())
    mids = (vals[:-1] + vals[1:]) / 2               # ties: 4 significant bits, exact in 16 bits
    edge = torch.tensor([440.0, 448.0, 456.0, 464.0, 480.0, 500.0, 1e4, float("inf"),
                         -float("inf"), 2.0 ** -9, 2.0 ** -10, 3 * 2.0 ** -11])
    for scale in (0.5, 0.0123):
        pieces = [torch.randn(4096, generator=g) * 3 * scale]
        if scale == 0.5:                            # a power of two keeps ties exact after /scale
            pieces += [mids * scale, -mids * scale, edge * scale, -edge * scale]
        x = torch.cat(pieces).to(td)
        n = -(-x.numel() // (hkv * d)) * hkv * d
        x = torch.cat([x, torch.zeros(n - x.numel(), dtype=td)]).reshape(-1, hkv, d)
        T = x.shape[0]
        xr = raw(x)
        kp = np.zeros((T, 1, hkv, d), dtype=np.uint8)
        vp = np.zeros((T, 1, hkv, d), dtype=np.uint8)
        paged.write_kv(xr, xr, in_dt, np.arange(T), kp, vp, "e4m3", k_scale=scale, v_scale=scale)
        ref = (x.float() / scale).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)
        assert np.array_equal(kp[:, 0], ref.numpy())
        assert np.array_equal(vp[:, 0], ref.numpy())


def test_fp8_decode_dequantises_with_the_scales():
    """An e4m3 cache decodes to code value * scale: attention over it equals
    attention over the dequantised fp64 cache (here checked via SDPA)."""
    rng = np.random.default_rng(26)
    hq, hkv, d, bs, n = 4, 2, 16, 16, 23
    kc = rng.integers(0, 0x7E, size=(2, bs, hkv, d), dtype=np.uint8) | (rng.integers(0, 2, size=(2, bs, hkv, d), dtype=np.uint8) << 7)
    vc = rng.integers(0, 0x7E, size=(2, bs, hkv, d), dtype=np.uint8)
    qf = rng.standard_normal((1, hq, d)).astype(np.float32)
    qraw = torch.from_numpy(qf).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    out = paged.decode(qraw, "bf16", kc, vc, "e4m3", np.array([[1, 0]]), [n], 0.25, hkv,
                       k_scale=0.003, v_scale=0.5)
    K = codecs.e4m3_decode(kc[[1, 0]]).reshape(-1, hkv, d)[:n] * 0.003
    V = codecs.e4m3_decode(vc[[1, 0]]).reshape(-1, hkv, d)[:n] * 0.5
    Q = codecs.bf16_bits_to_f64(qraw)
    ref = F.scaled_dot_product_attention(torch.from_numpy(Q)[:, :, None, :],
                                         torch.from_numpy(K).permute(1, 0, 2)[None],
                                         torch.from_numpy(V).permute(1, 0, 2)[None],
                                         scale=0.25, enable_gqa=True)[0, :, 0, :]
    np.testing.assert_allclose(out[0], ref.numpy(), rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------
# planted mistakes: each pin above catches at least one plausible error
# --------------------------------------------------------------------------

def _sdpa_pin_fails(monkeypatch, patch):
    patch(monkeypatch)
    try:
        test_decode_matches_library_sdpa(64, 8, 128, 16)
    except AssertionError:
        return True
    return False


def test_planted_wrong_gqa_map_is_caught(monkeypatch):
    def patch(mp):
        orig = paged.decode_one

        def bad(q_f64, k_vals, v_vals, table_row, n, scale, hkv):
            out = orig(q_f64, k_vals, v_vals, table_row, n, scale, hkv)
            hq = q_f64.shape[0]
            # strided instead of consecutive grouping
            for h in range(hq):
                kv = h % hkv
                K = paged.gather(k_vals, table_row, n)[:, kv]
                V = paged.gather(v_vals, table_row, n)[:, kv]
                out[h] = paged.attention_weights(q_f64[h], K, scale) @ V
            return out
        mp.setattr(paged, "decode_one", bad)
    assert _sdpa_pin_fails(monkeypatch, patch)


def test_planted_dropped_scale_is_caught(monkeypatch):
    def patch(mp):
        orig = paged.attention_weights
        mp.setattr(paged, "attention_weights", lambda q, K, scale: orig(q, K, 1.0))
    assert _sdpa_pin_fails(monkeypatch, patch)


def test_planted_gather_off_by_one_is_caught(monkeypatch):
    orig = paged.gather
    monkeypatch.setattr(paged, "gather", lambda pool, row, n: orig(pool, row, n + 1)[1:])
    with pytest.raises(AssertionError):
        test_decode_matches_brute_force_on_tiny()


def test_planted_e4m3_tie_rule_is_caught(monkeypatch):
    orig = codecs.e4m3_encode_f32

    def ties_away(x):
        x = np.asarray(x, dtype=np.float32)
        nudged = np.nextafter(x, np.copysign(np.float32(np.inf), x)).astype(np.float32)
        return orig(nudged)
    monkeypatch.setattr(codecs, "e4m3_encode_f32", ties_away)
    with pytest.raises(AssertionError):
        test_e4m3_encode_matches_library_cast()


def test_swap_out_and_back_in_restores_the_blocks():
    """Evicting blocks to a second pool and bringing them back into other
    slots leaves their bytes unchanged and touches nothing else."""
    rng = np.random.default_rng(27)
    dev_k = rng.integers(0, 1 << 16, size=(10, 4, 2, 8), dtype=np.uint16)
    dev_v = rng.integers(0, 1 << 16, size=(10, 4, 2, 8), dtype=np.uint16)
    host_k = np.zeros((6, 4, 2, 8), np.uint16)
    host_v = np.zeros((6, 4, 2, 8), np.uint16)
    k0, v0 = dev_k.copy(), dev_v.copy()
    paged.swap_blocks(dev_k, dev_v, host_k, host_v, [[3, 0], [7, 5]])
    assert np.array_equal(host_k[0], k0[3]) and np.array_equal(host_v[5], v0[7])
    assert not host_k[1:5].any()
    dev_k[[3, 7]] = 0
    paged.swap_blocks(host_k, host_v, dev_k, dev_v, [[0, 9], [5, 3]])
    assert np.array_equal(dev_k[9], k0[3]) and np.array_equal(dev_v[3], v0[7])
    assert np.array_equal(dev_k[:3], k0[:3]) and np.array_equal(dev_k[4:7], k0[4:7])


# --------------------------------------------------------------------------
# paged prefill (causal, chunked)
# --------------------------------------------------------------------------

def _prefill_case(rng, hq, hkv, d, bs, ctxs, nqs, dtype="f16"):
    B = len(ctxs)
    nbs = [-(-c // bs) for c in ctxs]
    N = sum(nbs) + 3
    perm = rng.permutation(N)
    tables, o = np.full((B, max(nbs)), -1, np.int64), 0
    for s, nb in enumerate(nbs):
        tables[s, :nb] = perm[o:o + nb]
        o += nb
    to = lambda x: torch.from_numpy(x.astype(np.float32)).to(torch.float16).view(torch.int16).numpy().view(np.uint16)
    kp = to(rng.standard_normal((N, bs, hkv, d)))
    vp = to(rng.standard_normal((N, bs, hkv, d)))
    qs = np.concatenate([[0], np.cumsum(nqs)])
    q = to(rng.standard_normal((int(qs[-1]), hq, d)))
    return q, kp, vp, tables, qs


def test_prefill_matches_library_sdpa_with_causal_offset():
    rng = np.random.default_rng(31)
    hq, hkv, d, bs = 8, 2, 32, 16
    ctxs, nqs = [50, 17, 33], [50, 5, 1]        # full prefill, a chunk, one token
    q, kp, vp, tables, qs = _prefill_case(rng, hq, hkv, d, bs, ctxs, nqs)
    got = paged.prefill(q, "f16", kp, vp, "f16", tables, ctxs, qs, 0.2, hkv)
    Q = codecs.f16_bits_to_f64(q)
    for s, (ctx, n) in enumerate(zip(ctxs, nqs)):
        nb = -(-ctx // bs)
        K = codecs.f16_bits_to_f64(kp[tables[s, :nb]]).reshape(-1, hkv, d)[:ctx]
        V = codecs.f16_bits_to_f64(vp[tables[s, :nb]]).reshape(-1, hkv, d)[:ctx]
        pos = ctx - n + np.arange(n)
        mask = torch.from_numpy(np.arange(ctx)[None, :] <= pos[:, None])  # [n, ctx]
        ref = F.scaled_dot_product_attention(
            torch.from_numpy(Q[qs[s]:qs[s + 1]]).permute(1, 0, 2)[None],
            torch.from_numpy(K).permute(1, 0, 2)[None], torch.from_numpy(V).permute(1, 0, 2)[None],
            attn_mask=mask, scale=0.2, enable_gqa=True)[0].permute(1, 0, 2)
        np.testing.assert_allclose(got[qs[s]:qs[s + 1]], ref.numpy(), rtol=1e-12, atol=1e-12)


def test_prefill_last_token_equals_decode_and_first_token_sees_itself_only():
    rng = np.random.default_rng(32)
    hq, hkv, d, bs = 4, 4, 16, 16
    ctxs, nqs = [40, 9], [40, 9]
    q, kp, vp, tables, qs = _prefill_case(rng, hq, hkv, d, bs, ctxs, nqs)
    pre = paged.prefill(q, "f16", kp, vp, "f16", tables, ctxs, qs, 0.25, hkv)
    last = q[[qs[1] - 1, qs[2] - 1]]
    dec = paged.decode(last, "f16", kp, vp, "f16", tables, ctxs, 0.25, hkv)
    np.testing.assert_allclose(pre[[qs[1] - 1, qs[2] - 1]], dec, rtol=1e-13, atol=1e-13)
    # a full prefill's first token attends only to itself: its value row
    v0 = codecs.f16_bits_to_f64(vp[tables[0, 0], 0])
    for h in range(hq):
        assert np.array_equal(pre[0, h], v0[h])


# ---- shared-prefix (cascade) decode -----------------------------------------
def test_shared_prefix_blocks_by_hand():
    # tables agree on their first two entries; bs 16
    t = np.array([[5, 6, 7, 8], [5, 6, 9, 10], [5, 11, 12, 13]], dtype=np.int32)
    assert paged.shared_prefix_blocks(t, [60, 60, 60], [0, 1], 16) == 2
    # the prefix ends before each member's last token: 33 tokens keep 2 blocks, 32 keep 1
    assert paged.shared_prefix_blocks(t, [33, 60, 60], [0, 1], 16) == 2
    assert paged.shared_prefix_blocks(t, [32, 60, 60], [0, 1], 16) == 1
    assert paged.shared_prefix_blocks(t, [60, 60, 60], [0, 1, 2], 16) == 1
    assert paged.shared_prefix_blocks(t, [60, 60, 60], [1], 16) == 0  # one member
    t2 = t.copy()
    t2[1, 0] = 99
    assert paged.shared_prefix_blocks(t2, [60, 60, 60], [0, 1], 16) == 0


def test_partial_attention_and_merge_by_brute_force():
    rng = np.random.default_rng(21)
    q = rng.standard_normal(4)
    K = rng.standard_normal((7, 4))
    V = rng.standard_normal((7, 3))
    z = [0.5 * sum(K[t, i] * q[i] for i in range(4)) for t in range(7)]
    lse = math.log(math.fsum(math.exp(x) for x in z))
    w = [math.exp(x - lse) for x in z]
    full = [math.fsum(w[t] * V[t, j] for t in range(7)) for j in range(3)]
    l, o = paged.partial_attention(q, K, V, 0.5)
    assert abs(l - lse) < 1e-12
    np.testing.assert_allclose(o, full, rtol=0, atol=1e-12)
    for cut in range(8):  # any split point, the empty parts included
        parts = [paged.partial_attention(q, K[:cut], V[:cut], 0.5),
                 paged.partial_attention(q, K[cut:], V[cut:], 0.5)]
        np.testing.assert_allclose(paged.merge_partials(parts), full, rtol=0, atol=1e-12)
    # an empty part carries no weight
    e = paged.partial_attention(q, K[:0], V[:0], 0.5)
    assert e[0] == -np.inf and not e[1].any()


@pytest.mark.parametrize("phase", ["fork", "tails"])
def test_shared_prefix_decode_equals_plain_decode(phase):
    w = W._shared_prefix(phase, 4, "cpu", prompts=3, samples=3, prefix=64, max_tail=40,
                         hq=8, hkv=2, d=32, bs=16)
    kp, vp = raw(w.k_pool), raw(w.v_pool)
    paged.copy_blocks(kp, vp, w.cow_pairs)  # the decode step: copy-on-write, then the write
    paged.write_kv(raw(w.new_k), raw(w.new_v), "bf16", w.slot_mapping, kp, vp, "bf16")
    args = (raw(w.q), "bf16", kp, vp, "bf16", w.block_tables, w.context_lens)
    got, pre = paged.shared_prefix_decode(*args, w.meta["group_start"], w.meta["group_seqs"],
                                          w.scale, w.num_kv_heads)
    ref = paged.decode(*args, w.scale, w.num_kv_heads)
    assert np.isfinite(ref).all()
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
    # every sample shares its prompt's full blocks: 64 + r tokens -> 4 blocks at bs 16
    assert (pre == 4).all()


# ---- planted mistakes in the prefill, shared-prefix and hash oracles -------
@pytest.mark.parametrize("bad", [
    lambda orig: (lambda ctx, n, i: orig(ctx, n, i) + 1),           # one future key seen
    lambda orig: (lambda ctx, n, i: max(orig(ctx, n, i) - 1, 1)),   # own key left out
    lambda orig: (lambda ctx, n, i: i + 1),                         # chunk taken as positions 0..n-1
])
def test_planted_prefill_position_mistakes_are_caught(monkeypatch, bad):
    monkeypatch.setattr(paged, "visible_keys", bad(paged.visible_keys))
    with pytest.raises(AssertionError):
        test_prefill_matches_library_sdpa_with_causal_offset()


def test_planted_merge_mistakes_are_caught(monkeypatch):
    orig_merge, orig_part = paged.merge_partials, paged.partial_attention

    def flipped(parts):  # weights exp(max - lse_i) instead of exp(lse_i - max)
        l = np.array([p[0] for p in parts])
        w = np.where(np.isfinite(l), np.exp(np.where(np.isfinite(l), l.max() - l, 0.0)), 0.0)
        return sum(wi * p[1] for wi, p in zip(w, parts)) / w.sum()

    def unnormalised(parts):  # the weighted sum not divided by the weights' sum
        l = np.array([p[0] for p in parts])
        w = np.exp(l - l.max())
        return sum(wi * p[1] for wi, p in zip(w, parts))

    def max_for_lse(q, K, V, scale):  # lse replaced by the part's max score
        lse, o = orig_part(q, K, V, scale)
        return (float(scale) * (K @ q)).max() if K.shape[0] else lse, o

    for name, fn in [("merge_partials", flipped), ("merge_partials", unnormalised),
                     ("partial_attention", max_for_lse)]:
        monkeypatch.setattr(paged, "merge_partials", orig_merge)
        monkeypatch.setattr(paged, "partial_attention", orig_part)
        monkeypatch.setattr(paged, name, fn)
        with pytest.raises(AssertionError):
            test_partial_attention_and_merge_by_brute_force()
        with pytest.raises(AssertionError):
            test_shared_prefix_decode_equals_plain_decode("tails")


def test_planted_shared_prefix_past_the_last_token_is_caught(monkeypatch):
    def no_cut(block_tables, context_lens, members, block_size):  # limit ctx // bs
        members = [int(m) for m in members]
        if len(members) < 2:
            return 0
        limit = min(int(context_lens[m]) // block_size for m in members)
        p = 0
        while p < limit and all(int(block_tables[m][p]) == int(block_tables[members[0]][p])
                                for m in members):
            p += 1
        return p
    monkeypatch.setattr(paged, "shared_prefix_blocks", no_cut)
    with pytest.raises(AssertionError):
        test_shared_prefix_blocks_by_hand()
