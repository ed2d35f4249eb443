"""Decode context parallelism on the host (no GPU): the per-rank key counts of the C ABI
against the oracle, argument errors, the planner's empty shares, and the one collective of
the step -- the all-gather of every rank's (out, lse) -- run as gloo ranks on CPU, with the
oracle standing in for each rank's attention and for the merge."""
import ctypes
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from conftest import ROOT
from paged_kv_cache_421_b200 import _binding as B
from paged_kv_cache_421_b200 import build as pa_build
from paged_kv_cache_421_b200 import dcp
from paged_kv_cache_421_b200 import workloads as W


@pytest.fixture(scope="module")
def lib():
    pa_build.build()
    return B.load()


def test_local_seq_lens_match_the_oracle(lib, oracle_mod):
    ctx = np.arange(0, 700)
    for world in [1, 2, 3, 4, 8]:
        for rank in range(world):
            got = dcp.local_seq_lens(ctx, rank, world)
            assert np.array_equal(got, oracle_mod.dcp_local_len(ctx, 16, rank, world)), (rank, world)


def test_local_seq_lens_argument_errors(lib):
    for args in [(5, 16, -1, 2), (5, 16, 2, 2), (5, 16, 0, 0), (5, 0, 0, 1)]:
        c, bs, rank, world = args
        with pytest.raises(B.PaError) as e:
            B.pa_dcp_local_seq_lens(np.array([c]), bs, rank, world)
        assert e.value.status == B.PA_ERR_INVALID_ARG
    with pytest.raises(B.PaError):
        B.pa_dcp_local_seq_lens(np.array([-1]), 16, 0, 1)


def test_dcp_calls_reject_bad_arguments_without_device(lib):
    p = ctypes.c_void_p(0x1000)  # never dereferenced: every call below fails on the host
    assert lib.pa_dcp_slot_mapping(p, 4, p, p, 1, 1, 16, 2, 2, p, None) == B.PA_ERR_INVALID_ARG
    assert lib.pa_dcp_slot_mapping(p, 4, p, p, 1, 1, 16, 0, 0, p, None) == B.PA_ERR_INVALID_ARG
    assert lib.pa_dcp_slot_mapping(None, 4, p, p, 1, 1, 16, 0, 2, p, None) == B.PA_ERR_INVALID_ARG
    assert lib.pa_dcp_slot_mapping(None, 4, None, None, 0, 0, 16, 0, 2, None, None) == B.PA_OK
    assert lib.pa_merge_partials(p, p, 0, 4, 128, p, None, None) == B.PA_ERR_INVALID_ARG
    assert lib.pa_merge_partials(p, p, 1025, 4, 128, p, None, None) == B.PA_ERR_INVALID_ARG
    assert lib.pa_merge_partials(p, p, 2, 4, 96, p, None, None) == B.PA_ERR_UNSUPPORTED
    assert lib.pa_merge_partials(None, p, 2, 4, 128, p, None, None) == B.PA_ERR_INVALID_ARG
    assert lib.pa_merge_partials(ctypes.c_void_p(0x1004), p, 2, 4, 128, p, None, None) == \
        B.PA_ERR_INVALID_ARG  # rows move as 16-byte vectors
    assert lib.pa_merge_partials(None, None, 2, 0, 128, None, None, None) == B.PA_OK


def test_planner_accepts_empty_shares_only_with_lse(lib):
    sl, qsl = np.array([0, 40, 0]), np.array([0, 1, 2, 3])
    args = (sl, qsl, 32, 8, 128, 4, 148, 1 << 20)
    with pytest.raises(B.PaError) as e:
        B.pa_plan_attention(*args)
    assert e.value.status == B.PA_ERR_METADATA
    p = B.pa_plan_attention(*args, with_lse=True)
    assert p["num_decode_seqs"] == 3 and p["decode_max_splits"] == 1
    assert p["decode_ctas"] == 3 * 8  # one CTA per (request, kv head), empty ones included
    # every request empty: still one block per split and one split
    p = B.pa_plan_attention(np.array([0, 0]), np.array([0, 1, 2]), 32, 8, 128, 4, 148, 0,
                            with_lse=True)
    assert p["decode_split_blocks"] >= 1 and p["decode_max_splits"] == 1
    # a chunk-kind request with no key stays an error (G = 4, q_len 3 -> 12 rows > 8)
    with pytest.raises(B.PaError) as e:
        B.pa_plan_attention(np.array([0]), np.array([0, 3]), 32, 8, 128, 4, 148, 0,
                            with_lse=True)
    assert e.value.status == B.PA_ERR_METADATA


def test_dcp_requires_a_decode_step():
    dcp.check_decode_step([0, 1, 2, 2], 32, 8)
    with pytest.raises(ValueError):
        dcp.check_decode_step([0, 2], 32, 8)
    with pytest.raises(ValueError):
        dcp.check_decode_step([0, 1], 64, 4)


# ------------------------------------------------------------------ the exchange, gloo ranks
def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


CTX = [1, 9, 16, 17, 40, 64, 130, 333]


def _workload():
    return W.make_workload("dcp", CTX, [1] * len(CTX), 8, 2, 64, 16, 48, 4218, scale=0.2)


def _share(oracle, wl, cache, rank, world):
    """The oracle's attention over one rank's share (its local table on the same pool);
    requests with no key on the rank give 0 and -inf."""
    bt = wl.block_table
    local = np.zeros((bt.shape[0], -(-bt.shape[1] // world)), np.int32)
    own = bt[:, rank::world]
    local[:, :own.shape[1]] = own
    ll = oracle.dcp_local_len(wl.seq_lens, 16, rank, world)
    rows = np.nonzero(ll > 0)[0]
    qsl = np.concatenate([[0], np.cumsum(ll > 0)]).astype(np.int32)
    T, Hq, D = wl.num_tokens, wl.num_q_heads, wl.head_size
    o = np.zeros((T, Hq, D))
    l = np.full((T, Hq), -np.inf)
    oo, lo = oracle.attention_paged(cache, W.BF16, wl.num_blocks, 16, wl.num_kv_heads, D,
                                    W.bits(wl.q)[rows], Hq, local, ll, qsl, wl.scale)
    o[rows], l[rows] = oo, lo
    return o, l


def _oracle_cache(oracle, wl):
    cache = np.full(oracle.cache_elems(wl.num_blocks, 16, wl.num_kv_heads, wl.head_size),
                    W.CACHE_FILL_BF16, np.uint16)
    for bt, sl, qs, k, v in [(wl.hist_block_table, wl.hist_seq_lens, wl.hist_qsl, wl.k_hist,
                              wl.v_hist), (wl.block_table, wl.seq_lens, wl.qsl, wl.k_new,
                                           wl.v_new)]:
        slots = oracle.slot_mapping(bt, sl, qs, 16)
        oracle.write_kv(cache, W.BF16, wl.num_blocks, 16, wl.num_kv_heads, wl.head_size,
                        W.bits(k), W.bits(v), slots)
    return cache


def _exchange_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import oracle
    from paged_kv_cache_421_b200 import dcp as dcp_mod
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = _workload()
        cache = _oracle_cache(oracle, wl)
        o, l = _share(oracle, wl, cache, rank, world)
        parts_o, parts_l = dcp_mod.exchange(torch.from_numpy(o.astype(np.float32)),
                                            torch.from_numpy(l.astype(np.float32)))
        # rank order, every rank's own contribution in its slot
        for r in range(world):
            ro, rl = _share(oracle, wl, cache, r, world)
            assert np.array_equal(parts_o[r].numpy(), ro.astype(np.float32))
            assert np.array_equal(parts_l[r].numpy(), rl.astype(np.float32))
        merged, lse = oracle.merge_partials(parts_o.numpy().astype(np.float64),
                                            parts_l.numpy().astype(np.float64))
        full, lse_full = oracle.attention_paged(cache, W.BF16, wl.num_blocks, 16,
                                                wl.num_kv_heads, wl.head_size, W.bits(wl.q),
                                                wl.num_q_heads, wl.block_table, wl.seq_lens,
                                                wl.qsl, wl.scale)
        err = float(np.abs(merged - full).max())
        lerr = float(np.abs(lse - lse_full).max())
        q.put((rank, err, lerr, bool(np.any(parts_l.numpy() == -np.inf))))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_dcp_exchange_gloo(world):
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_exchange_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    res = [q.get(timeout=10) for _ in range(world)]
    assert sorted(r[0] for r in res) == list(range(world))
    for _, err, lerr, some_empty in res:
        assert err < 1e-6 and lerr < 1e-5  # fp32 transport of fp64 shares
        assert some_empty  # short contexts leave later ranks without keys
