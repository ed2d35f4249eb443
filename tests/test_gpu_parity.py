"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Bit-exact for slot mapping and the cache contents; attention within the stated tolerance
(bf16 KV: max abs 2e-2, mean abs 2e-3 against fp64; FP8 E4M3 KV: 4e-2 / 4e-3)."""
import zlib

import numpy as np
import pytest
import torch

import oracle
from gpu_common import (GpuStep, assert_close, oracle_attention_all, oracle_attention_rows,
                        oracle_cache, sample_rows)
from paged_kv_cache_421_b200 import _binding as B
from paged_kv_cache_421_b200 import ops
from paged_kv_cache_421_b200 import workloads as W

pytestmark = pytest.mark.gpu

ALL_CONFIGS = ["tiny_decode", "llama8b_decode", "mixed_step", "prefix_share_decode",
               "long70b_decode", "long70b_decode_fp8", "mixed_step_fp8"]


@pytest.fixture(autouse=True)
def _clean_error_word():
    B.pa_device_error(reset=True)
    yield
    assert B.pa_device_error(reset=True) == 0, "a kernel recorded a device error"


_steps = {}
_oracles = {}


def step_of(name):
    if name not in _steps:
        _steps.clear()
        _oracles.clear()
        torch.cuda.empty_cache()
        wl = W.CONFIGS[name]()
        _steps[name] = GpuStep(wl)
    return _steps[name]


def oracle_of(name):
    """(cache, out, lse) of the oracle for the step of `name`: its own slot mapping and write of
    the history and the step, then exact attention over every row (all kv heads of every
    request, each gathered once)."""
    st = step_of(name)
    if name not in _oracles:
        cache = oracle_cache(st.wl)
        out, lse = oracle_attention_all(st.wl, cache)
        _oracles[name] = (cache, out, lse)
    return _oracles[name]


# ------------------------------------------------------------------ slot mapping + write
@pytest.mark.parametrize("name", ALL_CONFIGS)
def test_slot_mapping_bit_exact(name):
    st = step_of(name)
    wl = st.wl
    want_h = oracle.slot_mapping(wl.hist_block_table, wl.hist_seq_lens, wl.hist_qsl, 16)
    want = oracle.slot_mapping(wl.block_table, wl.seq_lens, wl.qsl, 16)
    assert np.array_equal(st.hist_slots.cpu().numpy(), want_h)
    assert np.array_equal(st.slots.cpu().numpy(), want)


@pytest.mark.parametrize("name", ALL_CONFIGS)
def test_cache_write_bit_exact_full_buffer(name):
    # the whole pool, never-written blocks included (they must keep the fill pattern)
    st = step_of(name)
    want = oracle_of(name)[0]
    got = st.cache_host()
    assert got.nbytes == want.nbytes
    assert np.array_equal(got, want.view(np.uint8)), "cache bytes differ from the oracle"


def test_fp8_write_divides_at_ties():
    # x / 7 lands exactly on an E4M3 midpoint; the GPU must divide (not multiply by 1/7)
    xs = torch.tensor([0.0888671875, 0.1708984375, 0.1982421875, -0.0888671875])
    want = [0x06, 0x0C, 0x0E, 0x86]
    n = xs.numel()
    scale = torch.full((1,), 7.0, device="cuda")
    cache = ops.PagedKVCache(1, 1, 128, B.PA_FP8_E4M3, k_scale=scale, v_scale=scale)
    k = torch.zeros(n, 1, 128, dtype=torch.bfloat16, device="cuda")
    k[:, 0, 0] = xs.to(torch.bfloat16).cuda()
    slots = torch.arange(n, dtype=torch.int32, device="cuda")
    ops.write_kv(cache, k, k, slots)
    got = cache.view()[0, 0, 0, :n, 0].cpu().tolist()
    assert got == want


# ------------------------------------------------------------------ attention
@pytest.mark.parametrize("name", ALL_CONFIGS)
def test_attention_all_rows(name):
    # every (token, q head) row of the step -- for the long-context configs every kv head of
    # every request, so every split and every split merge -- against the paged oracle
    st = step_of(name)
    want = oracle_of(name)[1]
    stats = assert_close(st.out.cpu().numpy(), want, st.wl.kv_dtype, name)
    print(name, stats, want.shape[0] * want.shape[1], "rows")


@pytest.mark.parametrize("name", ["mixed_step", "prefix_share_decode", "long70b_decode",
                                  "long70b_decode_fp8"])
def test_attention_sampled_rows(name):
    # sampled rows against the unpaged oracle, which reads each position's K/V from the source
    # rows instead of the cache: a second path to the same attention
    st = step_of(name)
    wl = st.wl
    n = {"mixed_step": 40, "prefix_share_decode": 40, "long70b_decode": 8,
         "long70b_decode_fp8": 4}[name]
    tokens, heads = sample_rows(wl, n)
    want, _ = oracle_attention_rows(wl, tokens, heads)
    got = st.out.cpu().numpy()[tokens, heads]
    stats = assert_close(got, want, wl.kv_dtype, name)
    print(name, stats, len(tokens), "rows")


@pytest.mark.parametrize("name", ["mixed_step", "mixed_step_fp8"])
def test_mixed_step_chunks_all_rows(name):
    # every row of both prefill chunks (the chunk kernel's causal diagonal tiles included),
    # against the unpaged oracle
    st = step_of(name)
    wl = st.wl
    t0 = int(wl.qsl[48])
    T = wl.num_tokens
    tok = np.repeat(np.arange(t0, T), 2).astype(np.int32)
    hed = np.tile(np.array([0, 31], np.int32), T - t0)
    want, _ = oracle_attention_rows(wl, tok, hed)
    assert_close(st.out.cpu().numpy()[tok, hed], want, wl.kv_dtype, "chunks")


@pytest.mark.parametrize("name", ["tiny_decode", "llama8b_decode", "prefix_share_decode"])
def test_split_invariance(name):
    # every forced KV partition against the oracle, and close to the unsplit result
    st = step_of(name)
    want = oracle_of(name)[1]
    base = st.attend(kv_split_tokens=1 << 20).cpu().numpy()  # one split per request
    assert_close(base, want, st.wl.kv_dtype, "one split")
    for kv_split in [16, 48, 112, 512]:
        got = st.attend(kv_split_tokens=kv_split).cpu().numpy()
        assert np.max(np.abs(got - base)) < 2e-3, kv_split
        assert_close(got, want, st.wl.kv_dtype, f"split {kv_split}")


@pytest.mark.parametrize("name", ["long70b_decode", "long70b_decode_fp8"])
def test_split_invariance_long(name):
    # the long-context steps at forced partitions from 1024 keys per split (up to 128 splits
    # of a request) to one split per request, every row against the oracle
    st = step_of(name)
    want = oracle_of(name)[1]
    for kv_split in [1024, 4096, 1 << 17]:
        got = st.attend(kv_split_tokens=kv_split).cpu().numpy()
        assert_close(got, want, st.wl.kv_dtype, f"{name} split {kv_split}")


# ------------------------------------------------------------------ edge cases
def _small(ctx, ql, hq, hkv, d, seed, kv_dtype=W.BF16, shared=0, nb=None):
    need = sum(-(-c // 16) for c in ctx)
    return W.make_workload("edge", ctx, ql, hq, hkv, d, 16, nb or need + 8, seed,
                           kv_dtype=kv_dtype, shared_prefix_tokens=shared)


EDGE_CASES = {
    "ctx1": ([1], [1], 8, 1, 128),
    "one_block_exact": ([16, 32], [1, 1], 4, 2, 128),
    "ragged_tail": ([17, 33, 63, 15], [1, 1, 1, 1], 32, 8, 128),
    "mha_group1": ([40, 77], [1, 1], 4, 4, 128),
    "spec_decode_qlen2_g4": ([50, 300], [2, 2], 8, 2, 128),
    "qlen3_g4_chunk_kind": ([50, 300], [3, 3], 8, 2, 128),
    "first_chunk_no_history": ([70], [70], 8, 2, 128),
    "chunk_d64": ([130, 64], [100, 64], 8, 2, 64),
    "decode_d64_g2": ([1, 17, 33, 64], [1, 1, 1, 1], 4, 2, 64),
    "zero_query_mixed": ([10, 20, 5, 40], [0, 2, 0, 1], 8, 2, 128),
    "long_chunk_tail": ([1000], [333], 16, 2, 128),
    "many_requests": ([int(x) for x in np.random.default_rng(3).integers(1, 200, 300)],
                      [1] * 300, 8, 2, 128),
    "g16_chunk": ([90, 40], [1, 1], 32, 2, 128),
    # chunk rows whose last q-tile has whole 32-row warps (stored as TMA boxes) next to a
    # partial warp (plain stores): 48, 704 and 488 rows at G 8
    "chunk_warp_store_paths": ([300, 90, 400], [6, 88, 61], 16, 2, 128),
    # G 3 divides neither 128 nor 32: Q staged and O stored by the warps
    "g3_chunk": ([200, 90], [50, 37], 6, 2, 128),
}


@pytest.mark.parametrize("case", sorted(EDGE_CASES))
def test_edge_case(case):
    ctx, ql, hq, hkv, d = EDGE_CASES[case]
    wl = _small(ctx, ql, hq, hkv, d, seed=zlib.crc32(case.encode()) % 1000)
    st = GpuStep(wl)
    assert np.array_equal(st.cache_host(), oracle_cache(wl).view(np.uint8))
    want, _ = oracle_attention_all(wl, oracle_cache(wl))
    assert_close(st.out.cpu().numpy(), want, wl.kv_dtype, case)
    for split in [16, 64]:
        assert_close(st.attend(kv_split_tokens=split).cpu().numpy(), want, wl.kv_dtype,
                     f"{case} split {split}")


@pytest.mark.parametrize("kv_dtype,q_lens", [(W.BF16, [1, 1, 1, 1]), (W.FP8_E4M3, [1, 1, 1, 1]),
                                             (W.BF16, [17, 9, 5, 60]),
                                             (W.FP8_E4M3, [17, 9, 5, 60])],
                         ids=["bf16-decode", "fp8-decode", "bf16-chunks", "fp8-chunks"])
def test_nan_garbage_in_unwritten_slots(kv_dtype, q_lens):
    # stale NaN patterns in the unused tail of partly filled blocks must not reach the output
    # (decode rows, and prefill chunks whose last key tile ends inside a block)
    wl = _small([17, 33, 5, 100], q_lens, 16, 2, 128, seed=9, kv_dtype=kv_dtype)
    st = GpuStep(wl, fill=False, garbage_tail=True)
    tokens = np.repeat(np.arange(wl.num_tokens), wl.num_q_heads)
    heads = np.tile(np.arange(wl.num_q_heads), wl.num_tokens)
    want, _ = oracle_attention_rows(wl, tokens, heads)
    assert_close(st.out.cpu().numpy().reshape(-1, 128), want, kv_dtype, "garbage tail")


@pytest.mark.parametrize("seed", range(10))
def test_random_small_steps(seed):
    rng = np.random.default_rng(1000 + seed)
    B_ = int(rng.integers(1, 12))
    hkv = int(rng.choice([1, 2, 4]))
    G = int(rng.choice([1, 2, 4, 8]))
    d = int(rng.choice([64, 128]))
    ctx = rng.integers(1, 700, size=B_)
    ql = np.array([int(rng.choice([0, 1, 1, 1, 2, int(rng.integers(1, c + 1))])) for c in ctx])
    ql = np.minimum(ql, ctx)
    if ql.sum() == 0:
        ql[0] = 1
    wl = _small(ctx, ql, hkv * G, hkv, d, seed=seed)
    st = GpuStep(wl)
    assert np.array_equal(st.cache_host(), oracle_cache(wl).view(np.uint8))
    want, _ = oracle_attention_all(wl, oracle_cache(wl))
    assert_close(st.out.cpu().numpy(), want, wl.kv_dtype, f"seed {seed}")


FP8_CHUNK_CASES = {
    # FP8 E4M3 cache with chunk-kind requests (q_len * group > 8): the tcgen05 chunk kernel's
    # kind::f8f6f4 path, alone and mixed with decodes
    "first_chunk": ([70], [70], 8, 2),
    "chunk_after_history": ([1000], [333], 16, 2),
    "spec_decode_g8_qlen2": ([300, 517], [2, 2], 64, 8),
    "qlen3_g4": ([50, 300], [3, 3], 8, 2),
    "mixed_decodes_and_chunk": ([2000, 3001, 600, 700], [1, 1, 200, 1], 32, 8),
    "ragged_chunk_tails": ([129, 255, 17], [129, 100, 17], 8, 1),
    # G 3 divides no 128-row TMA box of Q: the softmax warps load and split Q themselves
    "g3_no_q_map": ([200, 90], [50, 37], 6, 2),
}


@pytest.mark.parametrize("case", sorted(FP8_CHUNK_CASES))
def test_fp8_chunk_case(case):
    ctx, ql, hq, hkv = FP8_CHUNK_CASES[case]
    wl = _small(ctx, ql, hq, hkv, 128, seed=zlib.crc32(case.encode()) % 1000,
                kv_dtype=W.FP8_E4M3)
    st = GpuStep(wl)
    ocache = oracle_cache(wl)
    assert np.array_equal(st.cache_host(), ocache)
    want, want_lse = oracle_attention_all(wl, ocache)
    assert_close(st.out.cpu().numpy(), want, W.FP8_E4M3, case)
    # forced partitions: fused split merges (<= 4 splits) and the reduce kernel (more)
    for split in [64, 256]:
        assert_close(st.attend(kv_split_tokens=split).cpu().numpy(), want, W.FP8_E4M3,
                     f"{case} split {split}")


@pytest.mark.parametrize("seed", range(4))
def test_random_small_steps_fp8_with_chunks(seed):
    rng = np.random.default_rng(3000 + seed)
    B_ = int(rng.integers(1, 8))
    hkv = int(rng.choice([1, 2, 4]))
    G = int(rng.choice([1, 2, 4, 8]))
    ctx = rng.integers(1, 900, size=B_)
    ql = np.array([int(rng.choice([1, 2, int(rng.integers(1, c + 1))])) for c in ctx])
    ql = np.minimum(ql, ctx)
    wl = _small(ctx, ql, hkv * G, hkv, 128, seed=seed, kv_dtype=W.FP8_E4M3)
    st = GpuStep(wl)
    assert np.array_equal(st.cache_host(), oracle_cache(wl))
    want, _ = oracle_attention_all(wl, oracle_cache(wl))
    assert_close(st.out.cpu().numpy(), want, W.FP8_E4M3, f"fp8 chunks seed {seed}")


@pytest.mark.parametrize("kv_split_tokens", [0, 1024])
def test_fp8_decode_repeats_bit_identical(kv_split_tokens):
    # The FP8 decode kernel runs its scores and probabilities ahead of the V copies; any wait
    # that can pass on an older phase shows up as results that change from call to call.  Many
    # short requests with partial last tiles (and, at 1024-key splits, many split merges), each
    # called five times: every call bit-identical, and equal to the oracle within tolerance.
    rng = np.random.default_rng(4243 + kv_split_tokens)
    ctx = [int(x) for x in rng.integers(300, 3000, 48)]
    wl = W.make_workload("fp8-repeat", ctx, [1] * 48, 32, 8, 128, 16, 16 * 1024, 4243,
                         kv_dtype=W.FP8_E4M3)
    st = GpuStep(wl, kv_split_tokens=kv_split_tokens)
    first = st.out.cpu()
    for i in range(4):
        again = st.attend(kv_split_tokens=kv_split_tokens).cpu()
        assert torch.equal(again, first), f"call {i + 1} differs from the first"
    want, _ = oracle_attention_all(wl, oracle_cache(wl))
    assert_close(first.numpy(), want, W.FP8_E4M3, "fp8 repeat")


def test_random_small_steps_fp8():
    for seed in range(4):
        rng = np.random.default_rng(2000 + seed)
        ctx = rng.integers(1, 900, size=5)
        wl = _small(ctx, [1] * 5, 16, 2, 128, seed=seed, kv_dtype=W.FP8_E4M3)
        st = GpuStep(wl)
        assert np.array_equal(st.cache_host(), oracle_cache(wl))
        want, _ = oracle_attention_all(wl, oracle_cache(wl))
        assert_close(st.out.cpu().numpy(), want, W.FP8_E4M3, f"fp8 seed {seed}")
        for split in [16, 128]:
            assert_close(st.attend(kv_split_tokens=split).cpu().numpy(), want, W.FP8_E4M3,
                         f"fp8 seed {seed} split {split}")


def test_empty_step_is_a_no_op():
    wl = _small([5], [1], 4, 2, 128, seed=1)
    st = GpuStep(wl)
    out = torch.full((0, 4, 128), 1.0, device="cuda")
    B.pa_attention(st.cache.handle, st.wl.q.cuda(), 4, st.step["bt"], st.step["bt"].shape[1],
                   st.step["sl"], st.step["qsl"], np.array([5], np.int32),
                   np.array([0, 0], np.int32), 1, 0, 0.1, out)
    B.pa_write_kv(st.cache.handle, st.wl.k_new.cuda(), st.wl.v_new.cuda(), st.slots, 0)


def test_prefix_alias_write_visible_to_all_tables():
    wl = _small([40, 35, 50], [1, 1, 1], 4, 2, 64, seed=5, shared=32)
    st = GpuStep(wl)
    want, _ = oracle_attention_all(wl, oracle_cache(wl))
    assert_close(st.out.cpu().numpy(), want, W.BF16, "aliased")
    # overwrite token 3 of the first shared block through request 0's table
    slot = int(wl.block_table[0, 0]) * 16 + 3
    k = torch.full((1, 2, 64), 2.5, dtype=torch.bfloat16, device="cuda")
    ops.write_kv(st.cache, k, k, torch.tensor([slot], dtype=torch.int32, device="cuda"))
    view = st.cache.view()
    for r in range(3):
        assert torch.all(view[int(wl.block_table[r, 0]), :, :, 3, :] == 2.5)


# ------------------------------------------------------------------ error paths (no faults)
def test_bad_block_id_is_reported_not_faulted():
    wl = _small([40], [1], 4, 2, 128, seed=2)
    st = GpuStep(wl)
    bt = st.step["bt"].clone()
    bt[0, 1] = wl.num_blocks + 1000  # outside the pool: the kernel clamps and records code 3
    ops.attention(st.cache, wl.q.cuda(), bt, st.step["sl"], st.step["qsl"], wl.seq_lens, wl.qsl,
                  wl.scale)
    assert B.pa_device_error(reset=True) == 3
    assert B.pa_validate_block_table(st.cache.handle, bt, bt.shape[1], st.step["sl"], 1) == 1
    assert B.pa_validate_block_table(st.cache.handle, st.step["bt"], bt.shape[1],
                                     st.step["sl"], 1) == 0


@pytest.mark.parametrize("seed", range(4))
def test_slot_validator_counts_out_of_pool_and_duplicate_slots(seed):
    # seeded bad slot maps: some slots pushed past the pool, some copied onto other tokens'
    # slots, some skips; the expected counts are taken from the map itself
    rng = np.random.default_rng(500 + seed)
    wl = _small([int(x) for x in rng.integers(20, 300, 6)], [1] * 6, 8, 2, 128, seed=seed,
                nb=512)
    st = GpuStep(wl, run_attention=False)
    num_slots = wl.num_blocks * 16
    n = 4000
    slots = rng.choice(num_slots, n, replace=False).astype(np.int64)
    assert B.pa_validate_slots(st.cache.handle, torch.from_numpy(slots.astype(np.int32)).cuda(),
                               n) == (0, 0)
    pick = rng.choice(n, 300, replace=False)
    slots[pick[:100]] = num_slots + rng.integers(0, 10 * num_slots, 100)  # out of the pool
    slots[pick[100:150]] = -1                                             # skips
    untouched = np.setdiff1d(np.arange(n), pick)
    slots[pick[150:]] = slots[rng.choice(untouched, 150)]                 # copies of valid slots
    valid = slots[(slots >= 0) & (slots < num_slots)]
    want = (int(np.sum(slots >= num_slots)), int(valid.size - np.unique(valid).size))
    got = B.pa_validate_slots(st.cache.handle, torch.from_numpy(slots.astype(np.int32)).cuda(), n)
    assert got == want and want[1] > 0 and want[0] == 100


@pytest.mark.parametrize("kv_dtype", [W.BF16, W.FP8_E4M3])
def test_decode_wait_runs_out_and_is_reported(kv_dtype):
    # one decode CTA leaves one of its TMA loads unissued (test hook): its bounded wait gives up
    # after 1 ms, the kernel records code 1 and returns, and the context stays usable
    wl = _small([2000, 700], [1, 1], 8, 2, 128, seed=13, kv_dtype=kv_dtype)
    st = GpuStep(wl)
    want, _ = oracle_attention_all(wl, oracle_cache(wl))
    assert_close(st.out.cpu().numpy(), want, kv_dtype, "before")
    nb = ops.workspace_bytes_for(st.cache, wl.seq_lens, wl.qsl, wl.num_q_heads,
                                 wl.max_blocks_per_seq)
    ws = torch.empty(max(nb, 256), dtype=torch.uint8, device="cuda")
    out = torch.zeros(wl.num_tokens, wl.num_q_heads, 128, device="cuda")
    B.pa_attention_ex(st.cache.handle, wl.q.cuda(), wl.num_q_heads, st.step["bt"],
                      wl.max_blocks_per_seq, st.step["sl"], st.step["qsl"], wl.seq_lens, wl.qsl,
                      wl.num_seqs, wl.num_tokens, wl.scale, out, ws, ws.numel(),
                      test_skip_decode_load=4, test_wait_limit_us=1000)
    torch.cuda.synchronize()
    assert B.pa_device_error(reset=True) == 1
    # the next call runs normally
    assert_close(st.attend().cpu().numpy(), want, kv_dtype, "after")


def test_slot_beyond_table_is_reported():
    bt = torch.zeros(1, 2, dtype=torch.int32, device="cuda")
    sl = torch.tensor([40], dtype=torch.int32, device="cuda")
    qsl = torch.tensor([0, 1], dtype=torch.int32, device="cuda")
    slots = ops.slot_mapping(bt, sl, qsl, 1)
    assert slots.item() == -1
    assert B.pa_device_error(reset=True) == 2


def test_host_metadata_errors():
    wl = _small([40], [1], 4, 2, 128, seed=2)
    st = GpuStep(wl, run_attention=False)
    q = wl.q.cuda()
    out = torch.empty(1, 4, 128, device="cuda")
    with pytest.raises(B.PaError) as e:  # q_len > seq_len
        B.pa_attention(st.cache.handle, q, 4, st.step["bt"], st.step["bt"].shape[1],
                       st.step["sl"], st.step["qsl"], np.array([0], np.int32),
                       np.array([0, 1], np.int32), 1, 1, 0.1, out)
    assert e.value.status == B.PA_ERR_METADATA
    with pytest.raises(B.PaError) as e:  # forced split without workspace
        B.pa_attention_ex(st.cache.handle, q, 4, st.step["bt"], st.step["bt"].shape[1],
                          st.step["sl"], st.step["qsl"], wl.seq_lens, wl.qsl, 1, 1, 0.1, out,
                          kv_split_tokens=16)
    assert e.value.status == B.PA_ERR_WORKSPACE
