"""The OpenMP build of the oracle returns the plain build's bits (CPU only).

The OpenMP build runs the same C source with its independent units -- (request, kv head)
pairs of paged attention, selected rows of unpaged attention -- on several threads.  Each
unit's arithmetic is untouched, so every thread count must give identical bits; the benchmark
times both builds as its CPU baseline and the full-size GPU parity checks use the threaded one.
"""
import numpy as np
import pytest

from paged_kv_cache_421_b200 import workloads as W


def _oracle_cache(oracle, wl):
    n = oracle.cache_elems(wl.num_blocks, wl.block_size, wl.num_kv_heads, wl.head_size)
    cache = np.full(n, W.CACHE_FILL_BF16 if wl.kv_dtype == W.BF16 else W.CACHE_FILL_FP8,
                    np.uint16 if wl.kv_dtype == W.BF16 else np.uint8)
    ks = None if wl.k_scale is None else wl.k_scale.numpy()
    vs = None if wl.v_scale is None else wl.v_scale.numpy()
    for bt, sl, qs, k, v in [(wl.hist_block_table, wl.hist_seq_lens, wl.hist_qsl, wl.k_hist,
                              wl.v_hist),
                             (wl.block_table, wl.seq_lens, wl.qsl, wl.k_new, wl.v_new)]:
        slots = oracle.slot_mapping(bt, sl, qs, wl.block_size)
        oracle.write_kv(cache, wl.kv_dtype, wl.num_blocks, wl.block_size, wl.num_kv_heads,
                        wl.head_size, W.bits(k), W.bits(v), slots, ks, vs)
    return cache, ks, vs


@pytest.mark.parametrize("kv_dtype", [W.BF16, W.FP8_E4M3])
def test_openmp_attention_paged_is_bit_identical(oracle_mod, kv_dtype):
    rng = np.random.default_rng(31)
    ctx = rng.integers(1, 600, size=9)
    ql = np.array([1, 1, 3, 1, 0, 40, 1, 2, 1])
    ql = np.minimum(ql, ctx)
    wl = W.make_workload("omp", ctx, ql, 16, 4, 128, 16, 400, 31, kv_dtype=kv_dtype)
    cache, ks, vs = _oracle_cache(oracle_mod, wl)
    args = (cache, wl.kv_dtype, wl.num_blocks, 16, wl.num_kv_heads, wl.head_size, W.bits(wl.q),
            wl.num_q_heads, wl.block_table, wl.seq_lens, wl.qsl, wl.scale, ks, vs)
    o1, l1 = oracle_mod.attention_paged(*args)
    assert oracle_mod.threads_in_use(None) == 1
    for threads in (2, 5, 0):
        assert oracle_mod.threads_in_use(threads) >= 1
        o, l = oracle_mod.attention_paged(*args, threads=threads)
        assert np.array_equal(o.view(np.uint64), o1.view(np.uint64)), threads
        assert np.array_equal(l.view(np.uint64), l1.view(np.uint64)), threads
    # windows and local chunks go through the same units
    o1, _ = oracle_mod.attention_paged(*args, window=37, local_chunk=100)
    o, _ = oracle_mod.attention_paged(*args, window=37, local_chunk=100, threads=0)
    assert np.array_equal(o.view(np.uint64), o1.view(np.uint64))


def test_openmp_attention_rows_is_bit_identical(oracle_mod):
    wl = W.make_workload("omp-rows", [300, 77, 513], [1, 5, 1], 8, 2, 64, 16, 80, 32,
                         kv_dtype=W.FP8_E4M3)
    k_src, v_src = wl.kv_src()
    tokens = np.repeat(np.arange(wl.num_tokens, dtype=np.int32), wl.num_q_heads)
    heads = np.tile(np.arange(wl.num_q_heads, dtype=np.int32), wl.num_tokens)
    args = (W.bits(k_src), W.bits(v_src), wl.pos_rows, wl.pos_start, wl.kv_dtype, W.bits(wl.q),
            wl.seq_lens, wl.qsl, wl.scale, tokens, heads, wl.k_scale.numpy(),
            wl.v_scale.numpy())
    o1, l1 = oracle_mod.attention_rows(*args)
    o, l = oracle_mod.attention_rows(*args, threads=0)
    assert np.array_equal(o.view(np.uint64), o1.view(np.uint64))
    assert np.array_equal(l.view(np.uint64), l1.view(np.uint64))


def test_openmp_reports_errors_like_the_plain_build(oracle_mod):
    # a block id outside the pool is refused by both builds
    wl = W.make_workload("omp-bad", [40, 50], [1, 1], 4, 2, 64, 16, 10, 33)
    cache, _, _ = _oracle_cache(oracle_mod, wl)
    bt = wl.block_table.copy()
    bt[1, 2] = wl.num_blocks + 3
    for threads in (None, 0):
        with pytest.raises(oracle_mod.OracleError):
            oracle_mod.attention_paged(cache, wl.kv_dtype, wl.num_blocks, 16, wl.num_kv_heads,
                                       wl.head_size, W.bits(wl.q), wl.num_q_heads, bt,
                                       wl.seq_lens, wl.qsl, wl.scale, threads=threads)
