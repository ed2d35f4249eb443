"""Pins of the fp64 oracle against what the pages and mathematics fix (CPU only).

Each test ties one oracle function to something other than itself: a value printed or
hand-derived from the pages (tests/golden), a library routine (numpy, torch's CPU E4M3
conversion), a closed form, an invariant, or the pure-Python brute-force twin.
"""
import itertools
import math

import numpy as np
import pytest
import torch

from conftest import golden_lines
from oracle import brute
from paged_kv_cache_421_b200 import workloads as W


def _bf16_bits(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16).view(
        torch.int16).numpy().view(np.uint16)


def _bf16_vals(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# ------------------------------------------------------------------ sizing and slots
def test_slot_boundaries_golden(oracle_mod):
    rows = golden_lines("slot_boundaries.txt")
    bt = np.array([[7, 3, 9]], np.int32)
    ctx = 48
    slots = oracle_mod.slot_mapping(bt, np.array([ctx], np.int32), np.array([0, ctx], np.int32),
                                    16)
    for pos, slot in rows:
        assert slots[int(pos)] == int(slot), (pos, slot)


def test_blocks_and_bytes_golden(oracle_mod):
    n = 0
    for row in golden_lines("block_sizing.txt"):
        if row[0] == "blocks_needed":
            assert oracle_mod.blocks_needed(int(row[1]), int(row[2])) == int(row[3])
        else:
            bs, hkv, d, eb, want = map(int, row[1:])
            assert oracle_mod.block_bytes(bs, hkv, d, eb) == want
        n += 1
    assert n == 8


def test_waste_example_golden(oracle_mod):
    (used, reserved, waste, bs), = [tuple(map(int, r)) for r in golden_lines("waste_example.txt")]
    assert reserved - used == waste
    paged_slots = oracle_mod.blocks_needed(used, bs) * bs
    assert paged_slots >= used and paged_slots - used < bs
    assert oracle_mod.blocks_needed(used, bs) == 13


def test_cache_bytes_match_block_formula(oracle_mod):
    # the oracle's layout holds exactly num_blocks whole blocks
    for nb, bs, hkv, d in [(64, 16, 2, 64), (16384, 16, 8, 128)]:
        assert oracle_mod.cache_elems(nb, bs, hkv, d) * 2 == nb * oracle_mod.block_bytes(bs, hkv, d, 2)


@pytest.mark.parametrize("seed", range(6))
def test_slot_mapping_vs_brute(oracle_mod, seed):
    rng = np.random.default_rng(seed)
    bs = int(rng.choice([1, 2, 16]))
    B = int(rng.integers(1, 6))
    ctx = rng.integers(1, 41, size=B)
    ql = np.array([rng.integers(0, c + 1) for c in ctx])
    wl = W.make_workload("t", ctx, ql, 2, 1, 4, bs, 200, seed)
    got = oracle_mod.slot_mapping(wl.block_table, wl.seq_lens, wl.qsl, bs)
    want = brute.slot_mapping(wl.block_table.tolist(), wl.seq_lens.tolist(), wl.qsl.tolist(), bs)
    assert got.tolist() == want


def test_slots_injective_and_invertible(oracle_mod):
    wl = W.mixed_step()
    bs = wl.block_size
    hs = oracle_mod.slot_mapping(wl.hist_block_table, wl.hist_seq_lens, wl.hist_qsl, bs)
    ns = oracle_mod.slot_mapping(wl.block_table, wl.seq_lens, wl.qsl, bs)
    allslots = np.concatenate([hs, ns])
    assert np.unique(allslots).size == allslots.size
    # invert each new-token slot: block id must be the table entry of its logical block
    for r in range(wl.num_seqs):
        ql = int(wl.qsl[r + 1] - wl.qsl[r])
        for i in range(ql):
            s = int(ns[wl.qsl[r] + i])
            p = int(wl.seq_lens[r]) - ql + i
            assert s // bs == wl.block_table[r, p // bs] and s % bs == p % bs


def test_slot_mapping_rejects_bad_metadata(oracle_mod):
    bt = np.zeros((1, 2), np.int32)
    with pytest.raises(oracle_mod.OracleError):
        oracle_mod.slot_mapping(bt, np.array([3], np.int32), np.array([0, 4], np.int32), 16)
    with pytest.raises(oracle_mod.OracleError):  # position 40 needs a third logical block
        oracle_mod.slot_mapping(bt, np.array([41], np.int32), np.array([0, 1], np.int32), 16)


# ------------------------------------------------------------------ FP8 E4M3 codec
def test_e4m3_golden_points(oracle_mod):
    for row in golden_lines("e4m3_points.txt"):
        if row[0] == "decode":
            code, val = int(row[1], 16), row[2]
            got = oracle_mod.e4m3_decode(np.array([code]))[0]
            if val == "nan":
                assert math.isnan(got)
            else:
                assert got == float(val) and math.copysign(1, got) == math.copysign(1, float(val))
        elif row[0] == "encode":
            val, code = float(row[1]), int(row[2], 16)
            assert oracle_mod.e4m3_encode(np.array([val], np.float32))[0] == code, row


def test_e4m3_decode_all_codes_vs_torch(oracle_mod):
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle_mod.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().double().numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert nan.sum() == 2  # 0x7F and 0xFF
    assert np.array_equal(ours[~nan], ref[~nan])
    assert np.array_equal(np.signbit(ours[~nan]), np.signbit(ref[~nan]))


def test_e4m3_encode_all_bf16_vs_torch(oracle_mod):
    # every bf16 bit pattern as an fp32 input; torch rounds to nearest even but turns
    # magnitudes above 464 into NaN where the saturating encoder clamps to 448
    allbits = np.arange(65536, dtype=np.uint32)
    y = (allbits << 16).view(np.float32)
    ours = oracle_mod.e4m3_encode(y)
    ref = torch.from_numpy(y.copy()).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    finite = np.isfinite(y)
    inrange = finite & (np.abs(y) <= 464.0)
    assert np.array_equal(ours[inrange], ref[inrange])
    big = finite & (np.abs(y) > 464.0)
    assert np.all((ours[big] & 0x7F) == 0x7E)
    assert np.array_equal(ours[big] >> 7, (np.signbit(y[big])).astype(np.uint8))
    nanin = np.isnan(y)
    assert np.all((ours[nanin] & 0x7F) == 0x7F)


def test_e4m3_encode_random_fp32_vs_torch(oracle_mod):
    rng = np.random.default_rng(7)
    y = (rng.standard_normal(200000) * np.exp(rng.uniform(-12, 6, 200000))).astype(np.float32)
    y = y[np.abs(y) <= 464.0]
    ours = oracle_mod.e4m3_encode(y)
    ref = torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_e4m3_encode_is_nearest(oracle_mod):
    # brute force: |decode(encode(y)) - y| is minimal over all finite codes
    rng = np.random.default_rng(3)
    y = (rng.standard_normal(2000) * 50).astype(np.float32)
    vals = oracle_mod.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    enc = oracle_mod.e4m3_decode(oracle_mod.e4m3_encode(y))
    best = np.min(np.abs(np.abs(y.astype(np.float64))[:, None] - vals[None, :]), axis=1)
    assert np.all(np.abs(np.abs(enc) - np.abs(y)) == best)


# ------------------------------------------------------------------ cache write
def _oracle_cache(oracle_mod, wl, fill=True):
    n = oracle_mod.cache_elems(wl.num_blocks, wl.block_size, wl.num_kv_heads, wl.head_size)
    if wl.kv_dtype == W.BF16:
        cache = np.full(n, W.CACHE_FILL_BF16 if fill else 0, np.uint16)
    else:
        cache = np.full(n, W.CACHE_FILL_FP8 if fill else 0, np.uint8)
    ks = None if wl.k_scale is None else wl.k_scale.numpy()
    vs = None if wl.v_scale is None else wl.v_scale.numpy()
    for bt, sl, qs, k, v in [(wl.hist_block_table, wl.hist_seq_lens, wl.hist_qsl, wl.k_hist, wl.v_hist),
                             (wl.block_table, wl.seq_lens, wl.qsl, wl.k_new, wl.v_new)]:
        slots = oracle_mod.slot_mapping(bt, sl, qs, wl.block_size)
        oracle_mod.write_kv(cache, wl.kv_dtype, wl.num_blocks, wl.block_size, wl.num_kv_heads,
                            wl.head_size, W.bits(k), W.bits(v), slots, ks, vs)
    return cache


def test_write_bf16_roundtrip(oracle_mod):
    wl = W.tiny_decode()
    cache = _oracle_cache(oracle_mod, wl).reshape(wl.num_blocks, 2, wl.num_kv_heads,
                                                  wl.block_size, wl.head_size)
    k_src, v_src = (W.bits(t) for t in wl.kv_src())
    touched = np.zeros((wl.num_blocks, wl.block_size), bool)
    for r in range(wl.num_seqs):
        for p in range(int(wl.seq_lens[r])):
            b = wl.block_table[r, p // wl.block_size]
            o = p % wl.block_size
            row = wl.pos_rows[wl.pos_start[r] + p]
            assert np.array_equal(cache[b, 0, :, o, :], k_src[row])
            assert np.array_equal(cache[b, 1, :, o, :], v_src[row])
            touched[b, o] = True
    untouched = cache.transpose(0, 3, 1, 2, 4)[~touched]
    assert np.all(untouched == W.CACHE_FILL_BF16)


def test_write_bf16_vs_brute(oracle_mod):
    wl = W.make_workload("t", [5, 20], [3, 2], 2, 2, 4, 4, 16, 11)
    n = oracle_mod.cache_elems(16, 4, 2, 4)
    cache = np.zeros(n, np.uint16)
    slots = oracle_mod.slot_mapping(wl.block_table, wl.seq_lens, wl.qsl, 4)
    oracle_mod.write_kv(cache, W.BF16, 16, 4, 2, 4, W.bits(wl.k_new), W.bits(wl.v_new), slots)
    d = {}
    brute.write_kv_bf16(d, W.bits(wl.k_new).tolist(), W.bits(wl.v_new).tolist(),
                        slots.tolist(), 2, 4, 4)
    c5 = cache.reshape(16, 2, 2, 4, 4)
    for (b, kv, h, o, dd), val in d.items():
        assert c5[b, kv, h, o, dd] == val
    assert np.count_nonzero(c5) <= len(d)


def test_write_skips_negative_slots(oracle_mod):
    cache = np.zeros(oracle_mod.cache_elems(4, 4, 1, 2), np.uint16)
    k = np.array([[[1, 2]], [[3, 4]]], np.uint16)
    oracle_mod.write_kv(cache, W.BF16, 4, 4, 1, 2, k, k, np.array([-1, 5], np.int32))
    c = cache.reshape(4, 2, 1, 4, 2)
    assert c[1, 0, 0, 1].tolist() == [3, 4] and np.count_nonzero(c) == 4


def test_write_fp8_vs_torch_codec(oracle_mod):
    # FP8 pools keep K tiles token-major ([tok][d]) and V tiles dim-major ([d][tok])
    wl = W.make_workload("t", [9, 30], [9, 4], 4, 2, 8, 4, 32, 5, kv_dtype=W.FP8_E4M3)
    tiles = _oracle_cache(oracle_mod, wl).reshape(32, 2, 2, 4 * 8)
    k_src, v_src = wl.kv_src()
    for r in range(wl.num_seqs):
        for p in range(int(wl.seq_lens[r])):
            b = wl.block_table[r, p // 4]
            o = p % 4
            row = int(wl.pos_rows[wl.pos_start[r] + p])
            for kv, src, sc in [(0, k_src, wl.k_scale), (1, v_src, wl.v_scale)]:
                y = (src[row].float() / sc[:, None])  # fp32 IEEE division, per kv head
                ref = y.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
                got = tiles[b, 0].reshape(2, 4, 8)[:, o, :] if kv == 0 else \
                    tiles[b, 1].reshape(2, 8, 4)[:, :, o]
                assert np.array_equal(got, ref)


# ------------------------------------------------------------------ attention
def _attn_paged(oracle_mod, wl, cache):
    ks = None if wl.k_scale is None else wl.k_scale.numpy()
    vs = None if wl.v_scale is None else wl.v_scale.numpy()
    return oracle_mod.attention_paged(cache, wl.kv_dtype, wl.num_blocks, wl.block_size,
                                      wl.num_kv_heads, wl.head_size, W.bits(wl.q),
                                      wl.num_q_heads, wl.block_table, wl.seq_lens, wl.qsl,
                                      wl.scale, ks, vs)


def _attn_rows_all(oracle_mod, wl):
    k_src, v_src = wl.kv_src()
    T, Hq = wl.num_tokens, wl.num_q_heads
    tok = np.repeat(np.arange(T), Hq).astype(np.int32)
    hed = np.tile(np.arange(Hq), T).astype(np.int32)
    ks = None if wl.k_scale is None else wl.k_scale.numpy()
    vs = None if wl.v_scale is None else wl.v_scale.numpy()
    out, lse = oracle_mod.attention_rows(W.bits(k_src), W.bits(v_src), wl.pos_rows,
                                         wl.pos_start, wl.kv_dtype, W.bits(wl.q),
                                         wl.seq_lens, wl.qsl, wl.scale, tok, hed, ks, vs)
    return out.reshape(T, Hq, -1), lse.reshape(T, Hq)


@pytest.mark.parametrize("kv_dtype", [W.BF16, W.FP8_E4M3])
def test_paged_equals_unpaged(oracle_mod, kv_dtype):
    wl = W.make_workload("t", [1, 17, 40, 64, 23], [1, 1, 7, 16, 23], 8, 2, 32, 16, 64, 21,
                         kv_dtype=kv_dtype)
    cache = _oracle_cache(oracle_mod, wl)
    o1, l1 = _attn_paged(oracle_mod, wl, cache)
    o2, l2 = _attn_rows_all(oracle_mod, wl)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_prefix_sharing_paged_equals_unpaged(oracle_mod):
    wl = W.make_workload("t", [40, 35, 50], [1, 1, 1], 4, 2, 16, 16, 32, 9,
                         shared_prefix_tokens=32)
    assert np.array_equal(wl.block_table[:, :2], np.repeat(wl.block_table[:1, :2], 3, 0))
    cache = _oracle_cache(oracle_mod, wl)
    o1, l1 = _attn_paged(oracle_mod, wl, cache)
    o2, l2 = _attn_rows_all(oracle_mod, wl)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_attention_vs_numpy_textbook(oracle_mod):
    # contiguous textbook attention with numpy matmul + softmax on the gathered arrays
    wl = W.make_workload("t", [30, 45], [30, 5], 4, 2, 16, 8, 32, 13)
    cache = _oracle_cache(oracle_mod, wl)
    out, lse = _attn_paged(oracle_mod, wl, cache)
    k_src, v_src = (_bf16_vals(W.bits(t)) for t in wl.kv_src())
    q = _bf16_vals(W.bits(wl.q))
    G = wl.num_q_heads // wl.num_kv_heads
    for r in range(wl.num_seqs):
        rows = wl.pos_rows[wl.pos_start[r]:wl.pos_start[r + 1]]
        ql = int(wl.qsl[r + 1] - wl.qsl[r])
        ctx = int(wl.seq_lens[r])
        for i in range(ql):
            t = int(wl.qsl[r]) + i
            vis = ctx - ql + i + 1
            for h in range(wl.num_q_heads):
                K = k_src[rows[:vis], h // G]
                V = v_src[rows[:vis], h // G]
                s = wl.scale * (K @ q[t, h])
                w = np.exp(s - s.max())
                np.testing.assert_allclose(out[t, h], (w / w.sum()) @ V, rtol=1e-12, atol=1e-13)
                np.testing.assert_allclose(lse[t, h], s.max() + np.log(w.sum()), rtol=1e-13)


@pytest.mark.parametrize("case", range(8))
def test_attention_vs_brute(oracle_mod, case):
    rng = np.random.default_rng(100 + case)
    bs = int([1, 2, 16, 16, 2, 1, 16, 2][case])
    B = int(rng.integers(1, 4))
    ctx = rng.integers(1, 41, size=B)
    ql = np.array([rng.integers(0, c + 1) for c in ctx])
    hkv = int(rng.choice([1, 2]))
    G = int(rng.choice([1, 2, 3]))
    nb = int(sum(-(-c // bs) for c in ctx)) + 3
    wl = W.make_workload("t", ctx, ql, hkv * G, hkv, 4, bs, nb, 200 + case, scale=0.7)
    cache = _oracle_cache(oracle_mod, wl)
    out, _ = _attn_paged(oracle_mod, wl, cache)
    c5 = cache.reshape(nb, 2, hkv, bs, 4)

    def val(b, kv, h, o, d):
        return brute.bf16_bits_to_float(c5[b, kv, h, o, d])

    want = brute.attention(val, W.bits(wl.q).tolist(), hkv * G, hkv, 4, wl.block_table.tolist(),
                           wl.seq_lens.tolist(), wl.qsl.tolist(), bs, 0.7)
    if wl.num_tokens:
        np.testing.assert_allclose(out, np.array(want), rtol=1e-11, atol=1e-12)


def test_permutation_invariance_exhaustive(oracle_mod):
    # every assignment of 4 physical blocks (out of a 5-block pool) to the 4 logical blocks
    ctx, bs = 13, 4
    base = W.make_workload("t", [ctx], [2], 2, 1, 8, bs, 5, 31)
    k_src, v_src = wl_src = base.kv_src()
    ref = None
    for perm in itertools.permutations(range(5), 4):
        bt = np.array([perm], np.int32)
        cache = np.full(oracle_mod.cache_elems(5, bs, 1, 8), W.CACHE_FILL_BF16, np.uint16)
        allq = np.array([0, ctx], np.int32)
        slots = oracle_mod.slot_mapping(bt, np.array([ctx], np.int32), allq, bs)
        rows = base.pos_rows
        oracle_mod.write_kv(cache, W.BF16, 5, bs, 1, 8, W.bits(k_src)[rows], W.bits(v_src)[rows],
                            slots)
        out, lse = oracle_mod.attention_paged(cache, W.BF16, 5, bs, 1, 8, W.bits(base.q), 2, bt,
                                              base.seq_lens, base.qsl, base.scale)
        if ref is None:
            ref = (out, lse)
        assert np.array_equal(out, ref[0]) and np.array_equal(lse, ref[1])


def test_closed_form_single_key(oracle_mod):
    # one visible key: the output is that key's value row exactly
    wl = W.make_workload("t", [1, 9], [1, 9], 6, 3, 16, 4, 8, 17)
    cache = _oracle_cache(oracle_mod, wl)
    out, lse = _attn_paged(oracle_mod, wl, cache)
    v_src = _bf16_vals(W.bits(wl.kv_src()[1]))
    G = 2
    for t in [0, 1]:  # request 0's only token; request 1's first chunk query (0 computed)
        r = 0 if t == 0 else 1
        row = wl.pos_rows[wl.pos_start[r]]
        for h in range(6):
            assert np.array_equal(out[t, h], v_src[row, h // G])


def test_closed_form_equal_keys_mean(oracle_mod):
    # identical keys -> uniform weights -> mean of the values
    wl = W.make_workload("t", [37], [1], 2, 1, 8, 16, 4, 23)
    wl.k_hist[:] = wl.k_hist[0]
    wl.k_new[:] = wl.k_hist[0]
    cache = _oracle_cache(oracle_mod, wl)
    out, lse = _attn_paged(oracle_mod, wl, cache)
    v = _bf16_vals(W.bits(wl.kv_src()[1]))[wl.pos_rows]
    np.testing.assert_allclose(out[0, 0], v[:, 0].mean(axis=0), rtol=1e-13, atol=1e-14)
    s = wl.scale * _bf16_vals(W.bits(wl.q))[0, 0] @ _bf16_vals(W.bits(wl.k_hist))[0, 0]
    np.testing.assert_allclose(lse[0, 0], s + math.log(37), rtol=1e-13)


def test_closed_form_dominant_logit(oracle_mod):
    wl = W.make_workload("t", [20], [1], 1, 1, 8, 16, 4, 29, scale=1.0)
    wl.k_hist[:] = 0
    wl.k_new[:] = 0
    wl.k_hist[5] = 40.0
    wl.q[:] = 1.0
    cache = _oracle_cache(oracle_mod, wl)
    out, _ = _attn_paged(oracle_mod, wl, cache)
    v5 = _bf16_vals(W.bits(wl.v_hist))[5, 0]
    np.testing.assert_allclose(out[0, 0], v5, atol=1e-100 + 20 * math.exp(-320) + 1e-12)


def test_lse_merge_identity(oracle_mod):
    # attention over keys [0, m) and [m, n) separately, merged with their LSEs, equals
    # attention over [0, n): the split-KV reduce written as a partition of the softmax sum
    n, m, bs = 64, 32, 16
    wl = W.make_workload("t", [n], [1], 4, 2, 16, bs, 8, 41)
    cache = _oracle_cache(oracle_mod, wl)
    full, lse_full = _attn_paged(oracle_mod, wl, cache)
    bt = wl.block_table
    # part 1: same table, length m; part 2: a request whose table starts at block m / bs
    # and that sees the n - m remaining keys (the query is the same token)
    q = W.bits(wl.q)
    o1, l1 = oracle_mod.attention_paged(cache, W.BF16, 8, bs, 2, 16, q, 4, bt,
                                        np.array([m], np.int32), np.array([0, 1], np.int32),
                                        wl.scale)
    bt2 = np.zeros_like(bt)
    bt2[0, :bt.shape[1] - m // bs] = bt[0, m // bs:]
    o2, l2 = oracle_mod.attention_paged(cache, W.BF16, 8, bs, 2, 16, q, 4, bt2,
                                        np.array([n - m], np.int32), np.array([0, 1], np.int32),
                                        wl.scale)
    L = np.maximum(l1, l2)
    w1, w2 = np.exp(l1 - L), np.exp(l2 - L)
    merged = (w1[..., None] * o1 + w2[..., None] * o2) / (w1 + w2)[..., None]
    np.testing.assert_allclose(merged, full, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(L + np.log(w1 + w2), lse_full, rtol=1e-13)


def test_prefix_alias_golden(oracle_mod):
    rows = golden_lines("prefix_alias.txt")
    tables = {r[0]: [int(x) for x in r[1:]] for r in rows}
    bs, nb = 16, 9
    bt = np.zeros((2, 5), np.int32)
    bt[0, :3] = tables["A"]
    bt[1, :5] = tables["B"]
    rng = np.random.default_rng(5)
    n = oracle_mod.cache_elems(nb, bs, 1, 8)
    cache = _bf16_bits(rng.standard_normal(n))
    q = _bf16_bits(rng.standard_normal((1, 2, 8)))
    q2 = np.concatenate([q[:, :1], q[:, :1]], axis=0).reshape(2, 1, 8)  # same query, 2 reqs
    # both requests restricted to the shared prefix see identical keys
    o, _ = oracle_mod.attention_paged(cache, W.BF16, nb, bs, 1, 8, q2, 1, bt,
                                      np.array([32, 32], np.int32),
                                      np.array([0, 1, 2], np.int32), 0.3)
    assert np.array_equal(o[0], o[1])
    # a write into shared block B0 is seen through both tables
    k = _bf16_bits(np.full((1, 1, 8), 3.0))
    slots = oracle_mod.slot_mapping(bt[:1], np.array([5], np.int32), np.array([0, 1], np.int32), bs)
    assert slots[0] == tables["A"][0] * bs + 4
    oracle_mod.write_kv(cache, W.BF16, nb, bs, 1, 8, k, k, slots)
    o2, _ = oracle_mod.attention_paged(cache, W.BF16, nb, bs, 1, 8, q2, 1, bt,
                                       np.array([32, 32], np.int32),
                                       np.array([0, 1, 2], np.int32), 0.3)
    assert np.array_equal(o2[0], o2[1]) and not np.array_equal(o2[0], o[0])


def test_zero_query_requests_produce_nothing(oracle_mod):
    wl = W.make_workload("t", [10, 20, 5], [0, 2, 0], 2, 1, 8, 4, 16, 3)
    cache = _oracle_cache(oracle_mod, wl)
    out, _ = _attn_paged(oracle_mod, wl, cache)
    assert out.shape[0] == 2


def test_workload_shapes():
    # T and algorithmic KV bytes of the five serving steps
    wl = W.tiny_decode()
    assert wl.num_tokens == 4
    assert int(wl.seq_lens.sum()) * 2 * wl.num_kv_heads * wl.head_size * 2 == 58880
    wl = W.mixed_step()
    assert wl.num_tokens == 1072 and wl.q_lens.tolist()[-2:] == [512, 512]
    assert wl.seq_lens.tolist()[-2:] == [512, 2560]
    wl = W.prefix_share_decode()
    assert wl.num_tokens == 128
    assert np.all(wl.block_table[:, :64] == wl.block_table[0, :64])
    used = set(wl.block_table[0, :64].tolist())
    for r in range(128):
        nblk = -(-int(wl.seq_lens[r]) // 16)
        priv = set(wl.block_table[r, 64:nblk].tolist())
        assert not (priv & used)
        used |= priv


def test_write_fp8_divides_at_ties(oracle_mod):
    rows = [r for r in golden_lines("e4m3_points.txt") if r[0] == "divide"]
    assert len(rows) == 4
    xs = np.array([float(r[1]) for r in rows], np.float32)
    assert np.array_equal(_bf16_vals(_bf16_bits(xs)), xs.astype(np.float64))  # exact in bf16
    n = len(rows)
    k = _bf16_bits(xs).reshape(n, 1, 1)
    cache = np.zeros(oracle_mod.cache_elems(n, 1, 1, 1), np.uint8)
    scale = np.array([float(rows[0][2])], np.float32)
    oracle_mod.write_kv(cache, W.FP8_E4M3, n, 1, 1, 1, k, k, np.arange(n, dtype=np.int32),
                        scale, scale)
    c = cache.reshape(n, 2)
    for j, r in enumerate(rows):
        assert c[j, 0] == int(r[3], 16) and c[j, 1] == int(r[3], 16), r


# ------------------------------------------------------------------ block allocation
# allocate_slots as "Inside vLLM" reading notes, core point 1 describe it: count the new blocks
# (17 new tokens need ceil(17/16) = 2), check the free pool, take blocks from the head of the
# free-block queue ("vLLM architecture overview", section 2).  Expected values hand-computed.

def _alloc(om, rows, computed, new, queue, head, count, max_blocks=8, bs=16, capacity=None):
    q = np.array(queue, np.int32)
    if capacity is not None:
        assert q.size == capacity
    bt = np.full((len(computed), max_blocks), -9, np.int32)
    for r, row in enumerate(rows):
        bt[r, :len(row)] = row
    st = np.array([head, count], np.int32)
    got = om.allocate_slots(bt, computed, new, bs, q, st)
    return got, bt, st


def test_allocate_worked_example_17_tokens_take_two_blocks_from_head(oracle_mod):
    got, bt, st = _alloc(oracle_mod, [[]], [0], [17], [7, 3, 9, 1], 0, 4)
    assert got.tolist() == [2]
    assert bt[0, :3].tolist() == [7, 3, -9]
    assert st.tolist() == [2, 2]


def test_allocate_continues_a_partly_filled_block(oracle_mod):
    # (computed, new) -> new blocks: (16, 1) -> 1; (17, 15) -> 0 (positions 17..31 fit block 1);
    # (17, 16) -> 1; (0, 0) -> 0; (0, 16) -> 1; (0, 32) -> 2
    cases = [((16, 1), 1), ((17, 15), 0), ((17, 16), 1), ((0, 0), 0), ((0, 16), 1), ((0, 32), 2)]
    for (c, n), want in cases:
        have = -(-c // 16)
        got, bt, st = _alloc(oracle_mod, [[5] * have], [c], [n], [40, 41, 42], 0, 3)
        assert got.tolist() == [want], (c, n)
        assert bt[0, :have + want].tolist() == [5] * have + [40, 41, 42][:want]
        assert bt[0, have + want] == -9
        assert st.tolist() == [want, 3 - want]


def test_allocate_stops_at_first_request_it_cannot_place(oracle_mod):
    # pool of 3: requests need 2, 2, 1 -> the first is served, the second is not, and neither
    # is the third (first come, first served stops), leaving one block
    got, bt, st = _alloc(oracle_mod, [[], [], []], [0, 0, 0], [20, 32, 1], [4, 5, 6, 7], 0, 3)
    assert got.tolist() == [2, -1, -1]
    assert bt[0, :2].tolist() == [4, 5] and (bt[1:] == -9).all()
    assert st.tolist() == [2, 1]


def test_allocate_refuses_a_row_past_the_table(oracle_mod):
    got, bt, st = _alloc(oracle_mod, [[1, 2]], [32], [1], [9, 8], 0, 2, max_blocks=2)
    assert got.tolist() == [-1] and st.tolist() == [0, 2] and bt[0].tolist() == [1, 2]


def test_allocate_wraps_around_the_ring_and_free_appends_at_tail(oracle_mod):
    queue = np.array([20, 21, 0, 0, 24], np.int32)  # free ids at 4, 0, 1 (head 4, count 3)
    st = np.array([4, 3], np.int32)
    bt = np.full((1, 4), -9, np.int32)
    assert oracle_mod.allocate_slots(bt, [0], [17], 16, queue, st).tolist() == [2]
    assert bt[0, :2].tolist() == [24, 20] and st.tolist() == [1, 1]
    oracle_mod.free_blocks([30, 31, 32], queue, st)  # tail at (1 + 1) % 5 = 2: slots 2, 3, 4
    assert queue.tolist() == [20, 21, 30, 31, 32] and st.tolist() == [1, 4]
    bt2 = np.full((1, 4), -9, np.int32)
    assert oracle_mod.allocate_slots(bt2, [0], [64], 16, queue, st).tolist() == [4]
    assert bt2[0].tolist() == [21, 30, 31, 32] and st.tolist() == [0, 0]
    with pytest.raises(oracle_mod.OracleError):
        oracle_mod.free_blocks(list(range(6)), queue, st)  # more than the ring holds


def test_allocate_brute_force_invariants(oracle_mod):
    rng = np.random.default_rng(77)
    for _ in range(200):
        B = int(rng.integers(1, 12))
        cap = int(rng.integers(1, 40))
        queue = rng.permutation(1000)[:cap].astype(np.int32)
        head, count = int(rng.integers(0, cap)), int(rng.integers(0, cap + 1))
        computed = rng.integers(0, 80, B)
        new = rng.integers(0, 60, B)
        have = -(-computed // 16)
        bt = np.full((B, 10), -9, np.int32)
        for r in range(B):
            bt[r, :have[r]] = 100 + r
        before = bt.copy()
        st = np.array([head, count], np.int32)
        got = oracle_mod.allocate_slots(bt, computed, new, 16, queue, st)
        need = -(-(computed + new) // 16) - have
        taken = []
        served = True
        for r in range(B):
            fits = served and need[r] <= count - len(taken) and have[r] + need[r] <= 10
            served = fits
            assert got[r] == (need[r] if fits else -1)
            if fits:
                taken += bt[r, have[r]:have[r] + need[r]].tolist()
            assert (bt[r, :have[r]] == before[r, :have[r]]).all()
            k = have[r] + (need[r] if fits else 0)
            assert (bt[r, k:] == -9).all()
        assert taken == [int(queue[(head + j) % cap]) for j in range(len(taken))]
        assert st.tolist() == [(head + len(taken)) % cap, count - len(taken)]


# ------------------------------------------------------------------ sliding window
# The pages name the sliding window (architecture overview, section 2: SlidingWindowManager
# keeps only the window's blocks; section 6: SWA) without defining it; the reading taken: a
# query at position p sees keys max(0, p - W + 1) .. p.

@pytest.mark.parametrize("case", range(6))
def test_window_vs_brute(oracle_mod, case):
    rng = np.random.default_rng(700 + case)
    bs = int([1, 2, 16, 4, 16, 2][case])
    B = int(rng.integers(1, 4))
    ctx = rng.integers(1, 41, size=B)
    ql = np.array([rng.integers(1, c + 1) for c in ctx])
    window = int(rng.integers(1, 20))
    nb = int(sum(-(-c // bs) for c in ctx)) + 3
    wl = W.make_workload("t", ctx, ql, 2, 1, 4, bs, nb, 300 + case, scale=0.7)
    cache = _oracle_cache(oracle_mod, wl)
    out, _ = oracle_mod.attention_paged(cache, W.BF16, nb, bs, 1, 4, W.bits(wl.q), 2,
                                        wl.block_table, wl.seq_lens, wl.qsl, 0.7, window=window)
    c5 = cache.reshape(nb, 2, 1, bs, 4)

    def val(b, kv, h, o, d):
        return brute.bf16_bits_to_float(c5[b, kv, h, o, d])

    want = brute.attention(val, W.bits(wl.q).tolist(), 2, 1, 4, wl.block_table.tolist(),
                           wl.seq_lens.tolist(), wl.qsl.tolist(), bs, 0.7, window=window)
    np.testing.assert_allclose(out, np.array(want), rtol=1e-11, atol=1e-12)


def test_window_special_cases(oracle_mod):
    wl = W.make_workload("t", [37, 20], [5, 20], 4, 2, 8, 16, 8, 41)
    cache = _oracle_cache(oracle_mod, wl)
    full = _attn_paged(oracle_mod, wl, cache)
    args = (cache, W.BF16, wl.num_blocks, 16, 2, 8, W.bits(wl.q), 4, wl.block_table,
            wl.seq_lens, wl.qsl, wl.scale)
    # a window at least as long as every context is full attention, bit for bit
    for w in [37, 38, 1000]:
        o, l = oracle_mod.attention_paged(*args, window=w)
        assert np.array_equal(o, full[0]) and np.array_equal(l, full[1])
    # window 1: every query sees only its own position -> its own value row, lse = its score
    o, l = oracle_mod.attention_paged(*args, window=1)
    k_src, v_src = wl.kv_src()
    q = W.bits(wl.q)
    for r in range(2):
        ql = int(wl.qsl[r + 1] - wl.qsl[r])
        for i in range(ql):
            t = int(wl.qsl[r]) + i
            p = int(wl.seq_lens[r]) - ql + i
            row = wl.pos_rows[wl.pos_start[r] + p]
            for h in range(4):
                vrow = v_src[row, h // 2].float().numpy()
                np.testing.assert_array_equal(o[t, h], vrow.astype(np.float64))
                kk = k_src[row, h // 2].double().numpy()
                qq = np.array([brute.bf16_bits_to_float(int(x)) for x in q[t, h]])
                np.testing.assert_allclose(l[t, h], wl.scale * float(kk @ qq), rtol=1e-13)
    # the unpaged definition agrees under a window too
    k_bits, v_bits = W.bits(k_src), W.bits(v_src)
    T, Hq = wl.num_tokens, 4
    tok = np.repeat(np.arange(T), Hq).astype(np.int32)
    hed = np.tile(np.arange(Hq), T).astype(np.int32)
    for w in [1, 5, 16, 17]:
        o, _ = oracle_mod.attention_paged(*args, window=w)
        o2, _ = oracle_mod.attention_rows(k_bits, v_bits, wl.pos_rows, wl.pos_start, W.BF16,
                                          q, wl.seq_lens, wl.qsl, wl.scale, tok, hed, window=w)
        assert np.array_equal(o.reshape(T * Hq, -1), o2)


def test_window_equal_keys_mean_of_window(oracle_mod):
    # identical keys -> uniform weights over the window -> mean of the window's values
    wl = W.make_workload("t", [37], [1], 2, 1, 8, 16, 4, 23)
    wl.k_hist[:] = wl.k_hist[0]
    wl.k_new[:] = wl.k_hist[0]
    cache = _oracle_cache(oracle_mod, wl)
    k_src, v_src = wl.kv_src()
    for w in [1, 7, 16, 30]:
        o, _ = oracle_mod.attention_paged(cache, W.BF16, 4, 16, 1, 8, W.bits(wl.q), 2,
                                          wl.block_table, wl.seq_lens, wl.qsl, wl.scale, window=w)
        rows = wl.pos_rows[wl.pos_start[0] + np.arange(37 - w, 37)]
        want = v_src[rows, 0].double().numpy().mean(axis=0)
        np.testing.assert_allclose(o[0, 0], want, rtol=1e-12, atol=1e-13)


# ------------------------------------------------------------------ chunked local attention
# The architecture overview (section 2) also names ChunkedLocalAttentionManager without
# defining it; the reading taken: a query at position p sees keys floor(p / C) * C .. p.

@pytest.mark.parametrize("case", range(6))
def test_local_chunk_vs_brute(oracle_mod, case):
    rng = np.random.default_rng(800 + case)
    bs = int([1, 2, 16, 4, 16, 2][case])
    B = int(rng.integers(1, 4))
    ctx = rng.integers(1, 41, size=B)
    ql = np.array([rng.integers(1, c + 1) for c in ctx])
    chunk = int(rng.integers(1, 20))
    window = int(rng.choice([0, 0, 7]))
    nb = int(sum(-(-c // bs) for c in ctx)) + 3
    wl = W.make_workload("t", ctx, ql, 2, 1, 4, bs, nb, 400 + case, scale=0.7)
    cache = _oracle_cache(oracle_mod, wl)
    out, _ = oracle_mod.attention_paged(cache, W.BF16, nb, bs, 1, 4, W.bits(wl.q), 2,
                                        wl.block_table, wl.seq_lens, wl.qsl, 0.7,
                                        window=window, local_chunk=chunk)
    c5 = cache.reshape(nb, 2, 1, bs, 4)

    def val(b, kv, h, o, d):
        return brute.bf16_bits_to_float(c5[b, kv, h, o, d])

    want = brute.attention(val, W.bits(wl.q).tolist(), 2, 1, 4, wl.block_table.tolist(),
                           wl.seq_lens.tolist(), wl.qsl.tolist(), bs, 0.7, window=window,
                           local_chunk=chunk)
    np.testing.assert_allclose(out, np.array(want), rtol=1e-11, atol=1e-12)


def test_local_chunk_special_cases(oracle_mod):
    wl = W.make_workload("t", [37, 20], [5, 20], 4, 2, 8, 16, 8, 43)
    cache = _oracle_cache(oracle_mod, wl)
    full = _attn_paged(oracle_mod, wl, cache)
    args = (cache, W.BF16, wl.num_blocks, 16, 2, 8, W.bits(wl.q), 4, wl.block_table,
            wl.seq_lens, wl.qsl, wl.scale)
    # a chunk longer than every context is full attention; chunk 1 equals window 1
    for c in [37, 1000]:
        o, l = oracle_mod.attention_paged(*args, local_chunk=c)
        assert np.array_equal(o, full[0]) and np.array_equal(l, full[1])
    o1, l1 = oracle_mod.attention_paged(*args, local_chunk=1)
    ow, lw = oracle_mod.attention_paged(*args, window=1)
    assert np.array_equal(o1, ow) and np.array_equal(l1, lw)
    # the first query of a chunk (p % C == 0) sees exactly its own key
    k_src, v_src = wl.kv_src()
    o, _ = oracle_mod.attention_paged(*args, local_chunk=16)
    for r in range(2):
        ql = int(wl.qsl[r + 1] - wl.qsl[r])
        for i in range(ql):
            p = int(wl.seq_lens[r]) - ql + i
            if p % 16 == 0:
                t = int(wl.qsl[r]) + i
                row = wl.pos_rows[wl.pos_start[r] + p]
                np.testing.assert_array_equal(o[t, 0], v_src[row, 0].float().numpy().astype(np.float64))
    # paged agrees with unpaged under a local chunk
    T, Hq = wl.num_tokens, 4
    tok = np.repeat(np.arange(T), Hq).astype(np.int32)
    hed = np.tile(np.arange(Hq), T).astype(np.int32)
    for c in [3, 16, 17]:
        o, _ = oracle_mod.attention_paged(*args, local_chunk=c)
        o2, _ = oracle_mod.attention_rows(W.bits(k_src), W.bits(v_src), wl.pos_rows, wl.pos_start,
                                          W.BF16, W.bits(wl.q), wl.seq_lens, wl.qsl, wl.scale,
                                          tok, hed, local_chunk=c)
        assert np.array_equal(o.reshape(T * Hq, -1), o2)


# ------------------------------------------------------------------ context parallelism
# The architecture overview names decode context parallelism (DCP) without describing it.
# Reading taken: logical block j of a request lives on rank j mod world as that rank's local
# block j / world; each rank attends to its share and the shares merge by their LSEs.

def _dcp_local_tables(block_table, world):
    """Each rank's block table over the same physical pool: rank r's local block l is the
    global table's block l * world + r."""
    B, M = block_table.shape
    out = []
    for r in range(world):
        t = np.zeros((B, max(1, -(-M // world))), np.int32)
        own = block_table[:, r::world]
        t[:, :own.shape[1]] = own
        out.append(t)
    return out


def test_dcp_local_len_golden_and_partition(oracle_mod):
    # hand-counted: 40 keys in blocks of 16 over two ranks -> rank 0 holds blocks 0 and 2
    # (16 + 8 keys), rank 1 block 1 (16 keys); 17 keys over four ranks -> 16, 1, 0, 0
    assert list(oracle_mod.dcp_local_len([40], 16, 0, 2)) == [24]
    assert list(oracle_mod.dcp_local_len([40], 16, 1, 2)) == [16]
    assert [int(oracle_mod.dcp_local_len([17], 16, r, 4)[0]) for r in range(4)] == [16, 1, 0, 0]
    ctx = np.arange(0, 300)
    for world in [1, 2, 3, 5]:
        parts = np.stack([oracle_mod.dcp_local_len(ctx, 16, r, world) for r in range(world)])
        assert np.array_equal(parts.sum(axis=0), ctx)  # every key on exactly one rank
        # whole rounds of `world` blocks give every rank the same share
        full = ctx[ctx % (16 * world) == 0]
        for r in range(world):
            assert np.array_equal(oracle_mod.dcp_local_len(full, 16, r, world), full // world)
    assert np.array_equal(oracle_mod.dcp_local_len(ctx, 16, 0, 1), ctx)


@pytest.mark.parametrize("world", [1, 2, 3, 4])
def test_dcp_slots_match_the_global_slots_on_the_owner(oracle_mod, world):
    """With every rank's table drawn from one pool, the owner's local slot of a token is its
    global slot and every other rank skips it: the sharded write stores each token exactly
    once, where the unsharded write would."""
    wl = W.make_workload("t", [1, 16, 17, 40, 100, 333], [1, 1, 17, 5, 100, 64], 4, 2, 16, 16,
                         64, 87)
    glob = oracle_mod.slot_mapping(wl.block_table, wl.seq_lens, wl.qsl, 16)
    tables = _dcp_local_tables(wl.block_table, world)
    per_rank = np.stack([oracle_mod.dcp_slot_mapping(tables[r], wl.seq_lens, wl.qsl, 16, r, world)
                         for r in range(world)])
    assert np.all(per_rank >= -1)
    assert np.array_equal((per_rank >= 0).sum(axis=0), np.ones(wl.num_tokens))
    assert np.array_equal(per_rank.max(axis=0), glob)
    if world == 1:
        assert np.array_equal(per_rank[0], glob)


def test_merge_partials_closed_forms(oracle_mod):
    rng = np.random.default_rng(5)
    o = rng.standard_normal((1, 3, 8))
    l = rng.standard_normal((1, 3))
    out, lse = oracle_mod.merge_partials(o, l)          # one part: itself
    assert np.array_equal(out, o[0]) and np.allclose(lse, l[0], rtol=0, atol=1e-15)
    out, lse = oracle_mod.merge_partials(np.stack([o[0], o[0]]), np.stack([l[0], l[0]]))
    np.testing.assert_allclose(out, o[0], rtol=1e-15)  # two equal halves: same O, sum doubled
    np.testing.assert_allclose(lse, l[0] + math.log(2), rtol=1e-15)
    inf = np.full((2, 3), -np.inf)
    out, lse = oracle_mod.merge_partials(np.stack([o[0], 2 * o[0]]), inf)  # nothing seen
    assert np.all(out == 0) and np.all(lse == -np.inf)
    l2 = np.stack([l[0], np.full(3, -np.inf)])           # an empty part carries no weight
    out, lse = oracle_mod.merge_partials(np.stack([o[0], np.full((3, 8), np.nan)]), l2)
    assert np.array_equal(out, o[0]) and np.array_equal(lse, l[0])
    # weights follow e^lse: lse 0 and ln 3 give weights 1/4 and 3/4
    out, lse = oracle_mod.merge_partials(np.stack([np.ones((1, 2)), np.zeros((1, 2))]),
                                         np.array([[0.0], [math.log(3)]]))
    np.testing.assert_allclose(out, [[0.25, 0.25]], rtol=1e-15)
    np.testing.assert_allclose(lse, [math.log(4)], rtol=1e-15)


@pytest.mark.parametrize("world", [2, 3, 4])
def test_dcp_shards_merge_to_full_attention(oracle_mod, world):
    """Attention of each rank's share (its local table and local length, on the same pool),
    merged by the LSEs, is the unsharded attention; ranks that hold no key of a request add
    nothing (short contexts leave later ranks empty)."""
    ctx = [1, 5, 16, 17, 33, 64, 65, 200, 517]
    wl = W.make_workload("t", ctx, [1] * len(ctx), 8, 2, 16, 16, 80, 90 + world, scale=0.3)
    cache = _oracle_cache(oracle_mod, wl)
    full, lse_full = _attn_paged(oracle_mod, wl, cache)
    tables = _dcp_local_tables(wl.block_table, world)
    T, Hq, D = wl.num_tokens, wl.num_q_heads, wl.head_size
    parts_o = np.zeros((world, T, Hq, D))
    parts_l = np.full((world, T, Hq), -np.inf)
    for r in range(world):
        ll = oracle_mod.dcp_local_len(wl.seq_lens, 16, r, world)
        ql = np.where(ll > 0, 1, 0).astype(np.int32)   # requests with no local key: no rows
        qsl = np.concatenate([[0], np.cumsum(ql)]).astype(np.int32)
        rows = np.nonzero(ll > 0)[0]
        o, l = oracle_mod.attention_paged(cache, W.BF16, wl.num_blocks, 16, wl.num_kv_heads, D,
                                          W.bits(wl.q)[rows], Hq, tables[r], ll, qsl, wl.scale)
        parts_o[r, rows] = o
        parts_l[r, rows] = l
    assert np.any(parts_l == -np.inf)  # some shares are empty
    out, lse = oracle_mod.merge_partials(parts_o, parts_l)
    np.testing.assert_allclose(out, full, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, lse_full, rtol=1e-13)
