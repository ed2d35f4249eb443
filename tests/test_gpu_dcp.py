"""Row log-sum-exps exported by every attention kernel, the LSE merge of partial results, and
decode context parallelism with its ranks run one after another on one GPU (each rank's
kernels are independent launches over its own pool; only the exchange, an all-gather, is
left out and done by stacking), all against the oracle."""
import numpy as np
import pytest
import torch

import oracle
from gpu_common import TOL, GpuStep, assert_close, oracle_attention_all, oracle_cache
from paged_kv_cache_421_b200 import _binding as B
from paged_kv_cache_421_b200 import dcp, ops
from paged_kv_cache_421_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _wl(ctx, ql, hq, hkv, d, seed, kv_dtype=W.BF16):
    need = sum(-(-c // 16) for c in ctx)
    return W.make_workload("lse", ctx, ql, hq, hkv, d, 16, need + 8, seed, kv_dtype=kv_dtype)


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.int32)).cuda()


def _assert_lse(got, want, kv_dtype, what):
    # the output tolerance bounds the LSE too: scores are exact products of the stored
    # values, summed in fp32, and only the softmax sum's rounding reaches the LSE
    max_tol, mean_tol = TOL[kv_dtype]
    fin = np.isfinite(want)
    assert np.array_equal(np.isfinite(got), fin), f"{what}: -inf pattern differs"
    err = np.abs(got[fin].astype(np.float64) - want[fin])
    assert err.max() <= max_tol and err.mean() <= mean_tol, f"{what}: lse err {err.max():.3g}"


LSE_CASES = {
    "decode_d128": ([1, 17, 300, 2500], [1, 1, 1, 1], 32, 8, 128, W.BF16),
    "decode_d64": ([1, 17, 33, 64], [1, 1, 1, 1], 4, 2, 64, W.BF16),
    "decode_fp8": ([5000, 37, 900], [1, 1, 1], 32, 8, 128, W.FP8_E4M3),
    "mixed": ([900, 40, 1500, 77], [1, 40, 200, 1], 16, 4, 128, W.BF16),
    "chunk_d64": ([500, 130], [400, 64], 8, 2, 64, W.BF16),
    "long_chunk": ([2100], [500], 8, 2, 128, W.BF16),
}


@pytest.mark.parametrize("case", sorted(LSE_CASES))
def test_lse_out_matches_oracle(case):
    """Direct rows, decode split merges, fused chunk merges (<= 4 splits) and the reduce
    kernel (more splits) all export the row LSE."""
    ctx, ql, hq, hkv, d, kvd = LSE_CASES[case]
    wl = _wl(ctx, ql, hq, hkv, d, seed=len(case) * 7 + d, kv_dtype=kvd)
    st = GpuStep(wl, run_attention=False)
    want_o, want_l = oracle_attention_all(wl, oracle_cache(wl))
    q = wl.q.cuda().contiguous()
    for split in [0, 64, 1024]:
        lse = torch.full((wl.num_tokens, wl.num_q_heads), 7.0, device="cuda")
        out = ops.attention(st.cache, q, st.step["bt"], st.step["sl"], st.step["qsl"],
                            wl.seq_lens, wl.qsl, wl.scale, kv_split_tokens=split, lse_out=lse)
        torch.cuda.synchronize()
        assert_close(out.cpu().numpy(), want_o, kvd, f"{case} split={split}")
        _assert_lse(lse.cpu().numpy(), want_l, kvd, f"{case} split={split}")
        # the output itself is the same with and without the LSE export
        ref = st.attend(kv_split_tokens=split)
        assert torch.equal(out, ref)
    assert B.pa_device_error(reset=True) == 0


def test_empty_decode_rows_give_zero_and_minus_inf():
    wl = _wl([40, 300, 17], [1, 1, 1], 32, 8, 128, seed=11)
    st = GpuStep(wl, run_attention=False)
    want_o, want_l = oracle_attention_all(wl, oracle_cache(wl))
    sl = np.array([0, 300, 0], np.int32)
    for split in [0, 64]:
        lse = torch.zeros(3, 32, device="cuda")
        out = torch.full((3, 32, 128), 5.0, device="cuda")
        ops.attention(st.cache, wl.q.cuda().contiguous(), st.step["bt"], _dev(sl),
                      st.step["qsl"], sl, wl.qsl, wl.scale, out=out, kv_split_tokens=split,
                      lse_out=lse)
        torch.cuda.synchronize()
        o, l = out.cpu().numpy(), lse.cpu().numpy()
        assert np.all(o[[0, 2]] == 0) and np.all(l[[0, 2]] == -np.inf)
        assert_close(o[1:2], want_o[1:2], W.BF16, f"kept row split={split}")
        _assert_lse(l[1:2], want_l[1:2], W.BF16, f"kept row split={split}")
    assert B.pa_device_error(reset=True) == 0


@pytest.mark.parametrize("num_parts", [1, 3, 40])
@pytest.mark.parametrize("d", [64, 128])
def test_merge_partials_matches_oracle(num_parts, d):
    rng = np.random.default_rng(num_parts * 131 + d)
    rows = 37
    po = rng.standard_normal((num_parts, rows, d)).astype(np.float32)
    pl = (3 * rng.standard_normal((num_parts, rows))).astype(np.float32)
    empty = rng.random((num_parts, rows)) < 0.3
    pl[empty] = -np.inf
    pl[:, 5] = -np.inf                       # a row no part saw
    po[pl == -np.inf] = np.nan               # an empty part's output must not reach the result
    want_o, want_l = oracle.merge_partials(po.astype(np.float64), pl.astype(np.float64))
    out = torch.full((rows, d), 9.0, device="cuda")
    lse = torch.zeros(rows, device="cuda")
    dcp.merge(torch.from_numpy(po).cuda(), torch.from_numpy(pl).cuda(), out=out, lse_out=lse)
    torch.cuda.synchronize()
    o, l = out.cpu().numpy(), lse.cpu().numpy()
    assert np.all(np.isfinite(o))
    np.testing.assert_allclose(o, want_o, rtol=1e-4, atol=1e-5)
    fin = np.isfinite(want_l)
    assert np.array_equal(np.isfinite(l), fin) and np.all(l[~fin] == -np.inf)
    np.testing.assert_allclose(l[fin], want_l[fin], rtol=1e-5, atol=1e-5)
    assert np.all(o[5] == 0)


def _rank_pool(wl, rank, world, seed):
    """One rank's share: its own pool, block table and local lengths."""
    loc = dcp.local_seq_lens(wl.seq_lens, rank, world)
    nblk = [-(-int(n) // 16) for n in loc]
    width = max(1, max(nblk)) + 1
    num_blocks = sum(nblk) + 4
    ids = np.random.default_rng(seed).permutation(num_blocks).astype(np.int32)
    table = np.zeros((wl.num_seqs, width), np.int32)
    cur = 0
    for r, n in enumerate(nblk):
        table[r, :n] = ids[cur:cur + n]
        cur += n
    cache = ops.PagedKVCache(num_blocks, wl.num_kv_heads, wl.head_size, wl.kv_dtype,
                             k_scale=wl.k_scale, v_scale=wl.v_scale)
    if wl.kv_dtype == W.BF16:
        cache.buffer.view(torch.int16).fill_(W.CACHE_FILL_BF16)
    else:
        cache.buffer.fill_(W.CACHE_FILL_FP8)
    return loc, table, cache


def _oracle_rank_pool(wl, table, num_blocks, rank, world):
    """The oracle's copy of the same rank's pool after the same two writes."""
    n = oracle.cache_elems(num_blocks, 16, wl.num_kv_heads, wl.head_size)
    fill = W.CACHE_FILL_BF16 if wl.kv_dtype == W.BF16 else W.CACHE_FILL_FP8
    pool = np.full(n, fill, np.uint16 if wl.kv_dtype == W.BF16 else np.uint8)
    ks = None if wl.k_scale is None else wl.k_scale.cpu().numpy()
    vs = None if wl.v_scale is None else wl.v_scale.cpu().numpy()
    slots = []
    for sl, qs, k, v in [(wl.hist_seq_lens, wl.hist_qsl, wl.k_hist, wl.v_hist),
                         (wl.seq_lens, wl.qsl, wl.k_new, wl.v_new)]:
        s = oracle.dcp_slot_mapping(table, sl, qs, 16, rank, world)
        oracle.write_kv(pool, wl.kv_dtype, num_blocks, 16, wl.num_kv_heads, wl.head_size,
                        W.bits(k), W.bits(v), s, ks, vs)
        slots.append(s)
    return pool, slots


@pytest.mark.parametrize("world,kvd", [(2, W.BF16), (4, W.BF16), (3, W.FP8_E4M3)])
def test_dcp_ranks_merge_to_full_attention(world, kvd):
    ctx = [1, 5, 16, 17, 40, 100, 1000, 5000]
    wl = _wl(ctx, [1] * len(ctx), 32, 8, 128, seed=40 + world, kv_dtype=kvd)
    want_o, want_l = oracle_attention_all(wl, oracle_cache(wl))
    q = wl.q.cuda().contiguous()
    sl_dev, qsl_dev = _dev(wl.seq_lens), _dev(wl.qsl)
    hsl_dev, hqsl_dev = _dev(wl.hist_seq_lens), _dev(wl.hist_qsl)
    Th, T = int(wl.hist_qsl[-1]), wl.num_tokens
    outs, lses = [], []
    for rank in range(world):
        loc, table, cache = _rank_pool(wl, rank, world, seed=rank + 100 * world)
        bt = _dev(table)
        hslots = dcp.slot_mapping(bt, hsl_dev, hqsl_dev, Th, rank, world)
        ops.write_kv(cache, wl.k_hist.cuda().contiguous(), wl.v_hist.cuda().contiguous(), hslots)
        slots = dcp.slot_mapping(bt, sl_dev, qsl_dev, T, rank, world)
        ops.write_kv(cache, wl.k_new.cuda().contiguous(), wl.v_new.cuda().contiguous(), slots)
        o, l = dcp.partial_attention(cache, q, bt, _dev(loc), qsl_dev, loc, wl.qsl, wl.scale)
        torch.cuda.synchronize()
        # the rank's slots and pool bytes are the oracle's, bit for bit
        pool, (hs, ss) = _oracle_rank_pool(wl, table, cache.num_blocks, rank, world)
        assert np.array_equal(hslots.cpu().numpy(), hs) and np.array_equal(slots.cpu().numpy(), ss)
        assert np.array_equal(cache.buffer.cpu().numpy().view(pool.dtype), pool)
        outs.append(o)
        lses.append(l)
    lse = torch.empty(T, 32, device="cuda")
    merged = dcp.merge(torch.stack(outs), torch.stack(lses), lse_out=lse)
    torch.cuda.synchronize()
    assert_close(merged.cpu().numpy(), want_o, kvd, f"dcp world={world}")
    _assert_lse(lse.cpu().numpy(), want_l, kvd, f"dcp world={world}")
    assert any(bool(torch.any(torch.isinf(x))) for x in lses)  # some shares were empty
    assert B.pa_device_error(reset=True) == 0
