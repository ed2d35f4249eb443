"""Cascade attention over a shared prefix: host logic (CPU only, no device).

The "vLLM architecture overview" (section 2) shows two requests whose block tables start with
the same physical blocks, A = [B0, B3, B7] and B = [B0, B3, B1, B5, B8]: the prefix B0, B3 is
stored once and referenced by both.  Cascade attention (named in section 6) reads such a
prefix once for all the requests that share it.  Here: the helper that finds the shared
prefix in a step's block tables, against a brute-force count and the pages' example, and the
planner's handling of a call that asks for it.
"""
import numpy as np
import pytest

from conftest import golden_lines
from paged_kv_cache_421_b200 import _binding as B
from paged_kv_cache_421_b200 import workloads as W


@pytest.fixture(scope="module")
def lib():
    return B.load()


def brute_common_prefix(bt, seq_lens, qsl, bs=16):
    """Largest n: all requests with queries agree on their first n entries, and each of them
    has n * bs <= seq_len - q_len.  Tried n by n, from the longest row down."""
    ql = np.diff(qsl)
    live = [r for r in range(len(seq_lens)) if ql[r] > 0]
    if not live:
        return 0
    for n in range(bt.shape[1], -1, -1):
        if all(n * bs <= seq_lens[r] - ql[r] for r in live) and \
                all(np.array_equal(bt[r, :n], bt[live[0], :n]) for r in live):
            return n
    return 0


def test_pages_example_shares_two_blocks(lib):
    rows = {r[0]: [int(x) for x in r[1:]] for r in golden_lines("prefix_alias.txt")}
    a, b = rows["A"], rows["B"]
    bt = np.zeros((2, 5), np.int32)
    bt[0, :3], bt[1, :5] = a, b
    # one new token each; contexts long enough that both queries see both shared blocks
    seq_lens = np.array([3 * 16, 5 * 16], np.int32)
    qsl = np.array([0, 1, 2], np.int32)
    assert B.pa_common_prefix_blocks(bt, seq_lens, qsl) == 2
    # a request that has not yet computed its second shared block limits the prefix to one
    assert B.pa_common_prefix_blocks(bt, np.array([16 + 16, 80], np.int32), qsl) == 1
    # a request with no query this step does not constrain it: B alone shares with itself
    # the 4 whole blocks its 79 computed tokens fill
    assert B.pa_common_prefix_blocks(bt, np.array([3, 80], np.int32),
                                     np.array([0, 0, 1], np.int32)) == 4
    assert B.pa_common_prefix_blocks(bt, seq_lens, np.array([0, 0, 0], np.int32)) == 0


def test_common_prefix_matches_brute_force(lib):
    rng = np.random.default_rng(5)
    for _ in range(300):
        nreq = int(rng.integers(1, 7))
        maxb = int(rng.integers(1, 9))
        shared = rng.integers(0, 50, size=maxb)
        bt = np.tile(shared, (nreq, 1)).astype(np.int32)
        for r in range(nreq):  # each row diverges somewhere (or never)
            cut = int(rng.integers(0, maxb + 1))
            bt[r, cut:] = rng.integers(50, 100, size=maxb - cut)
        ql = rng.integers(0, 3, size=nreq)
        seq = np.array([int(rng.integers(q, maxb * 16 + 1)) if maxb * 16 >= q else q
                        for q in ql], np.int32)
        qsl = np.zeros(nreq + 1, np.int32)
        qsl[1:] = np.cumsum(ql)
        assert B.pa_common_prefix_blocks(bt, seq, qsl) == brute_common_prefix(bt, seq, qsl)


def test_common_prefix_argument_errors(lib):
    with pytest.raises(B.PaError) as e:
        B.pa_common_prefix_blocks(np.zeros((1, 2)), np.array([1]), np.array([0, 2]))
    assert e.value.status == B.PA_ERR_METADATA  # q_len > seq_len
    assert lib.pa_common_prefix_blocks(None, 4, None, None, 1, 16, None) == B.PA_ERR_INVALID_ARG


def test_prefix_share_workload_shares_its_prefix(lib):
    wl = W.prefix_share_decode()
    n = B.pa_common_prefix_blocks(wl.block_table, wl.seq_lens, wl.qsl)
    assert n == 64  # the 1024-token prefix of the workload, 64 aliased blocks


def _plan(wl, P, ws=1 << 34, **kw):
    return B.pa_plan_attention(wl.seq_lens, wl.qsl, wl.num_q_heads, wl.num_kv_heads,
                               wl.head_size, wl.max_blocks_per_seq, 148, ws,
                               common_prefix_tokens=P, **kw)


def test_plan_cascade_on_prefix_share_decode(lib):
    wl = W.prefix_share_decode()
    base = _plan(wl, 0)
    p = _plan(wl, 1024)
    T, Hq, D = wl.num_tokens, wl.num_q_heads, wl.head_size
    assert base["prefix_splits"] == 0 and base["prefix_ctas"] == 0
    # 128 tokens x 4 heads per kv head = 512 rows = 2 tcgen05 CTAs (256 rows) per kv head;
    # 1024 prefix keys = 8 tiles of 128; splits fill the SMs with at least two tiles each
    assert p["prefix_splits"] == 4 and p["prefix_split_blocks"] == 16
    assert p["prefix_ctas"] == 2 * 8 * 4
    # the decode kernel now walks only the suffixes
    assert p["decode_ctas"] <= base["decode_ctas"]
    per = lambda rows: -(-rows // 256) * 256  # noqa: E731  (256-byte aligned regions)
    rows = p["prefix_splits"] * T * Hq
    assert p["workspace_needed"] == (B.pa_attention_workspace_bytes(
        T, Hq, D, max(p["decode_max_splits"], p["chunk_max_splits"]))
        + per(rows * D * 4) + per(rows * 4))


def test_plan_cascade_refusals(lib):
    wl = W.prefix_share_decode()
    with pytest.raises(B.PaError) as e:  # not a multiple of the block size
        _plan(wl, 1000)
    assert e.value.status == B.PA_ERR_INVALID_ARG
    with pytest.raises(B.PaError) as e:  # longer than some request's computed tokens
        _plan(wl, (int(wl.seq_lens.min() - 1) // 16 + 1) * 16)
    assert e.value.status == B.PA_ERR_METADATA
    with pytest.raises(B.PaError) as e:  # with a sliding window
        _plan(wl, 1024, sliding_window=512)
    assert e.value.status == B.PA_ERR_UNSUPPORTED
    with pytest.raises(B.PaError) as e:  # no room for the prefix partials
        _plan(wl, 1024, ws=0)
    assert e.value.status == B.PA_ERR_WORKSPACE
    # a chunk-kind request in the step
    mixed = W.make_workload("m", [1100, 1100], [1, 40], 32, 8, 128, 16, 200, 1,
                            shared_prefix_tokens=1024)
    with pytest.raises(B.PaError) as e:
        _plan(mixed, 1024)
    assert e.value.status == B.PA_ERR_UNSUPPORTED


def test_plan_cascade_fits_a_small_workspace(lib):
    # fewer prefix splits when the workspace holds fewer partials, down to one
    wl = W.prefix_share_decode()
    T, Hq, D = wl.num_tokens, wl.num_q_heads, wl.head_size
    one = -(-T * Hq * D * 4 // 256) * 256 + -(-T * Hq * 4 // 256) * 256
    p = _plan(wl, 1024, ws=one)
    assert p["prefix_splits"] == 1 and p["workspace_needed"] <= one
    assert p["decode_max_splits"] == 1
