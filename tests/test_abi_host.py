"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every entry point
its header declares, sizes pools by the pages' block formula, plans launches consistently
and rejects bad arguments before touching the device."""
import ctypes
import os
import re

import numpy as np
import pytest

from conftest import ROOT, golden_lines
from paged_kv_cache_421_b200 import _binding as B
from paged_kv_cache_421_b200 import build as pa_build
from paged_kv_cache_421_b200 import workloads as W


@pytest.fixture(scope="module")
def lib():
    pa_build.build()
    return B.load()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "pa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\**\s*(pa_[a-z_0-9]+)\s*\(",
                       src, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ["pa_alloc_cache", "pa_write_kv", "pa_attention", "pa_slot_mapping",
                     "pa_cache_bytes", "pa_free_cache", "pa_attention_workspace_bytes"]:
        assert required in names
    assert sorted(B.EXPORTED) == names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_cache_bytes_follow_block_formula(lib):
    for row in golden_lines("block_sizing.txt"):
        if row[0] != "block_bytes":
            continue
        bs, hkv, d, eb, want = map(int, row[1:])
        dtype = B.PA_BF16 if eb == 2 else B.PA_FP8_E4M3
        assert B.pa_cache_bytes(1, bs, hkv, d, dtype) == want
        assert B.pa_cache_bytes(1000, bs, hkv, d, dtype) == 1000 * want
    assert B.pa_cache_bytes(0, 16, 8, 128, B.PA_BF16) == 0
    assert B.pa_cache_bytes(4, 16, 8, 128, 7) == 0


def test_workspace_formula(lib):
    assert B.pa_attention_workspace_bytes(8, 64, 128, 1) == 0
    ws = B.pa_attention_workspace_bytes(8, 64, 128, 10)
    parts = 10 * 8 * 64 * 129 * 4
    counters = 8 * 64 * 4
    assert ws >= parts + counters and ws < parts + counters + 768


def _plan(wl, num_sms=148, ws=None, split=0):
    if ws is None:
        ws = B.pa_attention_workspace_bytes(max(wl.num_tokens, 1), wl.num_q_heads, wl.head_size,
                                            1 << 16)
    return B.pa_plan_attention(wl.seq_lens, wl.qsl, wl.num_q_heads, wl.num_kv_heads,
                               wl.head_size, wl.max_blocks_per_seq, num_sms, ws,
                               kv_split_tokens=split)


@pytest.mark.parametrize("name", ["tiny_decode", "llama8b_decode", "mixed_step",
                                  "prefix_share_decode", "long70b_decode"])
def test_plan_invariants(lib, name):
    wl = W.CONFIGS[name]()
    p = _plan(wl)
    G = wl.num_q_heads // wl.num_kv_heads
    ql = wl.q_lens
    dec = (ql > 0) & (ql * G <= 8)
    assert p["num_decode_seqs"] == int(dec.sum())
    assert p["num_chunk_seqs"] == int(((ql > 0) & ~dec).sum())
    blocks = -(-wl.seq_lens.astype(np.int64) // 16)
    if p["num_decode_seqs"]:
        sb = p["decode_split_blocks"]
        ns = -(-blocks[dec] // sb)
        assert p["decode_max_splits"] == ns.max()
        assert p["decode_ctas"] == int(ns.sum()) * wl.num_kv_heads
        assert sb % 4 == 0 or sb == blocks[dec].max()
    if p["num_chunk_seqs"]:
        rows_per_cta = 256 if wl.head_size == 128 else 64  # tcgen05 CTA / mma.sync CTA
        assert p["chunk_max_qtiles"] == int(np.max(-(-(ql[~dec & (ql > 0)] * G) // rows_per_cta)))
    smax = max(p["decode_max_splits"], p["chunk_max_splits"])
    assert p["any_split"] == int(smax > 1)
    assert p["workspace_needed"] == B.pa_attention_workspace_bytes(wl.num_tokens, wl.num_q_heads,
                                                                    wl.head_size, smax)


def test_plan_long_context_is_split_for_occupancy(lib):
    wl = W.long70b_decode()
    p = _plan(wl)
    assert p["decode_max_splits"] > 1
    assert p["decode_ctas"] >= 148 * 4  # several waves of CTAs on 148 SMs
    # without workspace nothing is split
    p0 = _plan(wl, ws=0)
    assert p0["decode_max_splits"] == 1 and p0["workspace_needed"] == 0
    # a small workspace caps the split count
    ws3 = B.pa_attention_workspace_bytes(wl.num_tokens, wl.num_q_heads, wl.head_size, 3)
    p3 = _plan(wl, ws=ws3)
    assert p3["decode_max_splits"] <= 3 and p3["workspace_needed"] <= ws3


def test_plan_forced_split(lib):
    wl = W.tiny_decode()
    p = _plan(wl, split=16)
    assert p["decode_split_blocks"] == 1 and p["decode_max_splits"] == 4
    with pytest.raises(B.PaError) as e:
        _plan(wl, ws=0, split=16)
    assert e.value.status == B.PA_ERR_WORKSPACE
    with pytest.raises(B.PaError) as e:
        _plan(wl, split=24)  # not a multiple of the block size
    assert e.value.status == B.PA_ERR_INVALID_ARG


@pytest.mark.parametrize("sl,qsl", [
    ([5, 6], [0, 7, 8]),     # q_len > seq_len
    ([5, 6], [1, 2, 3]),     # does not start at 0
    ([5, 6], [0, 2, 1]),     # decreasing
    ([0, 6], [0, 1, 2]),     # a query with no context
    ([5, 2000], [0, 1, 2]),  # more blocks than the table holds
])
def test_plan_rejects_bad_metadata(lib, sl, qsl):
    with pytest.raises(B.PaError) as e:
        B.pa_plan_attention(np.array(sl), np.array(qsl), 8, 2, 128, 16, 148, 1 << 20)
    assert e.value.status == B.PA_ERR_METADATA


def test_plan_rejects_unsupported(lib):
    with pytest.raises(B.PaError) as e:
        B.pa_plan_attention(np.array([5]), np.array([0, 1]), 8, 2, 96, 16, 148, 0)
    assert e.value.status == B.PA_ERR_UNSUPPORTED
    with pytest.raises(B.PaError) as e:
        B.pa_plan_attention(np.array([5]), np.array([0, 1]), 8, 3, 128, 16, 148, 0)
    assert e.value.status == B.PA_ERR_INVALID_ARG


def test_argument_errors_without_device(lib):
    h = ctypes.c_void_p()
    # unsupported shapes and missing FP8 scales fail before any allocation
    assert lib.pa_alloc_cache(16, 16, 2, 96, B.PA_BF16, None, None, None, ctypes.byref(h)) == \
        B.PA_ERR_UNSUPPORTED
    assert lib.pa_alloc_cache(16, 8, 2, 128, B.PA_BF16, None, None, None, ctypes.byref(h)) == \
        B.PA_ERR_UNSUPPORTED
    assert lib.pa_alloc_cache(16, 16, 2, 64, B.PA_FP8_E4M3, None, None, None, ctypes.byref(h)) == \
        B.PA_ERR_UNSUPPORTED
    assert lib.pa_alloc_cache(16, 16, 2, 128, B.PA_FP8_E4M3, None, None, None, ctypes.byref(h)) == \
        B.PA_ERR_INVALID_ARG
    assert lib.pa_alloc_cache(0, 16, 2, 128, B.PA_BF16, None, None, None, ctypes.byref(h)) == \
        B.PA_ERR_INVALID_ARG
    assert lib.pa_alloc_cache(16, 16, 2, 128, B.PA_BF16, None, None, ctypes.c_void_p(0x1001),
                              ctypes.byref(h)) == B.PA_ERR_INVALID_ARG
    assert lib.pa_write_kv(None, None, None, None, 4, None) == B.PA_ERR_INVALID_ARG
    assert lib.pa_attention(None, None, 8, None, 4, None, None, None, None, 1, 1, 0.1, None, None,
                            0, None) == B.PA_ERR_INVALID_ARG
    assert lib.pa_slot_mapping(None, 4, None, None, 1, 1, 16, None, None) == B.PA_ERR_INVALID_ARG
    assert lib.pa_free_cache(None) == B.PA_OK
    assert B.pa_status_string(B.PA_ERR_METADATA) == "PA_ERR_METADATA"
    n_out, n_dup = ctypes.c_int(7), ctypes.c_int(7)
    assert lib.pa_validate_slots(None, None, 4, ctypes.byref(n_out), ctypes.byref(n_dup),
                                 None) == B.PA_ERR_INVALID_ARG
    fake = ctypes.c_void_p(0x1000)  # never dereferenced: the checks below fail first
    assert lib.pa_validate_slots(fake, None, -1, ctypes.byref(n_out), ctypes.byref(n_dup),
                                 None) == B.PA_ERR_INVALID_ARG
    assert lib.pa_validate_slots(fake, None, 4, None, ctypes.byref(n_dup), None) == \
        B.PA_ERR_INVALID_ARG
    # the bounded-wait test hook needs a wait limit of its own
    opts = B.pa_attention_opts()
    plan = B.pa_plan()
    sl = (ctypes.c_int * 1)(40)
    qs = (ctypes.c_int * 2)(0, 1)
    for skip, limit, status in [(1, 0, B.PA_ERR_INVALID_ARG), (-1, 10, B.PA_ERR_INVALID_ARG),
                                (1, -5, B.PA_ERR_INVALID_ARG), (1, 1000, B.PA_OK),
                                (0, 0, B.PA_OK)]:
        opts.test_skip_decode_load, opts.test_wait_limit_us = skip, limit
        assert lib.pa_plan_attention(sl, qs, 1, 1, 8, 2, 128, 16, 4, 148, 0, ctypes.byref(opts),
                                     ctypes.byref(plan)) == status, (skip, limit)


def test_allocator_argument_errors_without_device(lib):
    st = ctypes.c_void_p(0x1000)  # never dereferenced: every call below fails or returns early
    assert lib.pa_allocate_slots(None, 4, None, None, 0, 16, None, 8, st, None, None) == B.PA_OK
    assert lib.pa_allocate_slots(None, 4, None, None, 3, 16, None, 8, st, None, None) == \
        B.PA_ERR_INVALID_ARG
    assert lib.pa_allocate_slots(None, 4, None, None, -1, 16, None, 8, st, None, None) == \
        B.PA_ERR_INVALID_ARG
    assert lib.pa_allocate_slots(None, 4, None, None, 0, 0, None, 8, st, None, None) == \
        B.PA_ERR_INVALID_ARG
    assert lib.pa_allocate_slots(None, 4, None, None, 0, 16, None, 0, st, None, None) == \
        B.PA_ERR_INVALID_ARG
    assert lib.pa_free_blocks(None, 0, st, 8, st, None) == B.PA_OK
    assert lib.pa_free_blocks(None, 2, st, 8, st, None) == B.PA_ERR_INVALID_ARG
    assert lib.pa_free_blocks(st, 9, st, 8, st, None) == B.PA_ERR_INVALID_ARG
    assert lib.pa_free_blocks(st, 1, None, 8, st, None) == B.PA_ERR_INVALID_ARG


@pytest.mark.parametrize("window", [1, 16, 100, 1000, 5000])
def test_plan_with_sliding_window(lib, window):
    """Decode CTAs cover only the blocks from the window start of each request's first query
    row; chunk requests keep their split partition; a window past every context changes
    nothing."""
    wl = W.mixed_step()
    ws = B.pa_attention_workspace_bytes(wl.num_tokens, wl.num_q_heads, wl.head_size, 1 << 16)
    args = (wl.seq_lens, wl.qsl, wl.num_q_heads, wl.num_kv_heads, wl.head_size,
            wl.max_blocks_per_seq, 148, ws)
    p = B.pa_plan_attention(*args, sliding_window=window)
    full = B.pa_plan_attention(*args)
    G = wl.num_q_heads // wl.num_kv_heads
    dec = (wl.q_lens > 0) & (wl.q_lens * G <= 8)
    ctx, ql = wl.seq_lens.astype(np.int64), wl.q_lens.astype(np.int64)
    first = np.maximum(0, ctx - ql - window + 1) // 16
    eff = -(-ctx // 16) - first
    sb = p["decode_split_blocks"]
    assert p["decode_max_splits"] == int((-(-eff[dec] // sb)).max())
    assert p["decode_ctas"] == int((-(-eff[dec] // sb)).sum()) * wl.num_kv_heads
    assert p["decode_ctas"] <= full["decode_ctas"]
    assert p["num_chunk_seqs"] == full["num_chunk_seqs"]
    huge = B.pa_plan_attention(*args, sliding_window=int(ctx.max()) + 1)
    assert huge == full
    with pytest.raises(B.PaError) as e:
        B.pa_plan_attention(*args, sliding_window=-1)
    assert e.value.status == B.PA_ERR_INVALID_ARG


def test_struct_layouts_match_the_header(tmp_path):
    """The ctypes mirrors of pa_plan and pa_attention_opts have the header's sizes and field
    offsets (compiled with the host C compiler against include/pa.h)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no host C compiler")
    fields = {"pa_plan": [f[0] for f in B.pa_plan._fields_],
              "pa_attention_opts": [f[0] for f in B.pa_attention_opts._fields_]}
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "pa.h"', 'int main(void) {']
    for st, names in fields.items():
        lines.append(f'printf("{st} size %zu\\n", sizeof({st}));')
        for n in names:
            lines.append(f'printf("{st} {n} %zu\\n", offsetof({st}, {n}));')
    lines += ['return 0;', '}']
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    subprocess.run([cc, "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split("\n")
    got = {tuple(line.split()[:2]): int(line.split()[2]) for line in out if line.strip()}
    for st, cls in [("pa_plan", B.pa_plan), ("pa_attention_opts", B.pa_attention_opts)]:
        assert got[(st, "size")] == ctypes.sizeof(cls), st
        for n in fields[st]:
            assert got[(st, n)] == getattr(cls, n).offset, (st, n)


@pytest.mark.parametrize("chunk", [1, 16, 100, 1000, 8192])
def test_plan_with_local_chunk(lib, chunk):
    """Chunked local attention: decode CTAs cover only the blocks from the first key of each
    request's first query row, floor(p / C) * C; chunks at least as long as every context
    change nothing."""
    wl = W.mixed_step()
    ws = B.pa_attention_workspace_bytes(wl.num_tokens, wl.num_q_heads, wl.head_size, 1 << 16)
    args = (wl.seq_lens, wl.qsl, wl.num_q_heads, wl.num_kv_heads, wl.head_size,
            wl.max_blocks_per_seq, 148, ws)
    p = B.pa_plan_attention(*args, local_chunk=chunk)
    full = B.pa_plan_attention(*args)
    G = wl.num_q_heads // wl.num_kv_heads
    dec = (wl.q_lens > 0) & (wl.q_lens * G <= 8)
    ctx, ql = wl.seq_lens.astype(np.int64), wl.q_lens.astype(np.int64)
    p0 = ctx - ql
    eff = -(-ctx // 16) - (p0 - p0 % chunk) // 16
    sb = p["decode_split_blocks"]
    assert p["decode_max_splits"] == int((-(-eff[dec] // sb)).max())
    assert p["decode_ctas"] == int((-(-eff[dec] // sb)).sum()) * wl.num_kv_heads
    assert p["decode_ctas"] <= full["decode_ctas"]
    assert B.pa_plan_attention(*args, local_chunk=int(ctx.max()) + 1) == full
    with pytest.raises(B.PaError) as e:
        B.pa_plan_attention(*args, local_chunk=-1)
    assert e.value.status == B.PA_ERR_INVALID_ARG


def test_plan_random_metadata_stays_inside_the_workspace(lib):
    """Every plan the planner accepts indexes only the splits its workspace holds: for random
    batches, windows, local chunks, forced splits and workspace sizes, each request's split
    count (computed the way the kernels compute it) is at most the plan's maximum, and that
    maximum's workspace fits in the bytes given."""
    rng = np.random.default_rng(4217)
    accepted = 0
    for _ in range(300):
        n = int(rng.integers(1, 40))
        Hkv = int(rng.choice([1, 2, 8]))
        Hq = Hkv * int(rng.choice([1, 4, 8]))
        D = int(rng.choice([64, 128]))
        ql = rng.choice([0, 1, 1, 1, 2, 3, 17, 130, 600], size=n).astype(np.int64)
        ctx = ql + rng.integers(0, 20000, size=n)
        ctx = np.where(ctx == 0, 0, np.maximum(ctx, 1))
        qsl = np.concatenate([[0], np.cumsum(ql)])
        T = int(qsl[-1])
        maxb = int(max(1, (-(-ctx // 16)).max())) + int(rng.integers(0, 3))
        window = int(rng.choice([0, 0, 1, 77, 4096]))
        chunk = int(rng.choice([0, 0, 1, 100, 8192]))
        forced = int(rng.choice([0, 0, 0, 16, 256, 4096]))
        smax_ws = int(rng.choice([0, 1, 2, 5, 64, 1 << 12]))
        ws = B.pa_attention_workspace_bytes(max(T, 1), Hq, D, smax_ws) if smax_ws > 1 else 0
        try:
            p = B.pa_plan_attention(ctx, qsl, Hq, Hkv, D, maxb, 148, ws, kv_split_tokens=forced,
                                    sliding_window=window, local_chunk=chunk)
        except B.PaError as e:
            assert forced and e.status == B.PA_ERR_WORKSPACE, e
            continue
        accepted += 1
        G = Hq // Hkv
        blocks = -(-ctx // 16)
        smax = max(p["decode_max_splits"], p["chunk_max_splits"])
        assert p["decode_max_splits"] <= 1024
        if smax > 1:
            assert p["workspace_needed"] <= ws
        for r in range(n):
            if ql[r] == 0:
                continue
            if ql[r] * G <= 8:  # decode kind
                lim = int(ctx[r] - ql[r])
                lo = 0
                if window:
                    lo = max(lo, lim - window + 1)
                if chunk:
                    lo = max(lo, lim // chunk * chunk)
                ns = -(-(int(blocks[r]) - lo // 16) // p["decode_split_blocks"])
                assert 1 <= ns <= p["decode_max_splits"]
            else:
                ns = -(-int(blocks[r]) // p["chunk_split_blocks"])
                assert 1 <= ns <= p["chunk_max_splits"]
    assert accepted > 150


def _mixed(dec_ctx, chunk_ctx, chunk_ql, hq=32, hkv=8):
    ctx = np.array(list(dec_ctx) + list(chunk_ctx))
    ql = np.array([1] * len(dec_ctx) + list(chunk_ql))
    return ctx, np.concatenate([[0], np.cumsum(ql)])


def test_plan_chunk_ctas_beside_decode(lib):
    """A step with both kinds gives the tcgen05 chunk kernel fewer CTAs than items when their
    estimated schedule ends within the decode kernel's time, and one CTA per item otherwise:
    for a step of one kind only, for head_size 64, and when even the longest item outlasts the
    decodes.  More decode work never asks for more chunk CTAs."""
    def plan(ctx, qsl, d=128, kv_dtype=0, hq=32, hkv=8):
        mb = int(max(-(-int(c) // 16) for c in ctx))
        return B.pa_plan_attention(ctx, qsl, hq, hkv, d, mb, 148, 1 << 30, kv_dtype=kv_dtype)

    for kv_dtype, name in [(W.BF16, "mixed_step"), (W.FP8_E4M3, "mixed_step_fp8")]:
        wl = W.CONFIGS[name]()
        p = plan(wl.seq_lens, wl.qsl, kv_dtype=kv_dtype)
        items = p["chunk_ctas"] // wl.num_kv_heads
        assert 0 < p["chunk_ctas_per_kv_head"] < items, (name, p)
    for name in ["prefill_chunks", "llama8b_decode", "long70b_decode"]:  # one kind only
        wl = W.CONFIGS[name]()
        assert plan(wl.seq_lens, wl.qsl)["chunk_ctas_per_kv_head"] == 0, name
    ctx, qsl = _mixed([4000] * 32, [700, 900], [400, 300])
    assert plan(ctx, qsl, d=64)["chunk_ctas_per_kv_head"] == 0  # the mma.sync chunk kernel
    # a chunk whose longest item alone outlasts two short decodes: one CTA per item
    ctx, qsl = _mixed([100, 120], [16000, 900], [2000, 300])
    assert plan(ctx, qsl)["chunk_ctas_per_kv_head"] == 0
    # more decode bytes: never more chunk CTAs, and within [1, items)
    prev = None
    for n_dec in [16, 32, 64, 128]:
        ctx, qsl = _mixed([5000] * n_dec, [70, 430, 1033, 250, 764, 90],
                          [70, 130, 33, 200, 64, 90])
        p = plan(ctx, qsl)
        y = p["chunk_ctas_per_kv_head"]
        if y:
            assert 1 <= y < p["chunk_ctas"] // 8
            assert prev is None or prev == 0 or y <= prev, (n_dec, y, prev)
        prev = y
    assert prev > 0
