"""Cascade attention over a shared prefix, on the GPU, against the fp64 oracle.

Requests whose block tables start with the same physical blocks ("vLLM architecture
overview", section 2: A = [B0, B3, B7] and B = [B0, B3, B1, B5, B8] share B0, B3) let the call
read those blocks once for all of the step's queries (cascade attention, section 6): a prefix
pass attends every query row to the prefix, the decode kernel attends each request to its own
remaining keys and merges both by their LSEs.  The result is plain attention over the whole
context, so every output row is compared with the oracle's full attention (not with the
non-cascade GPU path), within the bf16 tolerance; the exported LSE with the oracle's LSE.
"""
import numpy as np
import pytest
import torch

from gpu_common import GpuStep, assert_close, oracle_attention_all, oracle_cache
from paged_kv_cache_421_b200 import _binding as B
from paged_kv_cache_421_b200 import ops
from paged_kv_cache_421_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean_error_word():
    B.pa_device_error(reset=True)
    yield
    assert B.pa_device_error(reset=True) == 0, "a kernel recorded a device error"


def _cascade(st, P, kv_split_tokens=0, lse=False, workspace_bytes=None):
    wl = st.wl
    lse_out = (torch.full((wl.num_tokens, wl.num_q_heads), float("nan"), device="cuda")
               if lse else None)
    ws = None
    if workspace_bytes is not None:
        ws = torch.empty(max(workspace_bytes, 256), dtype=torch.uint8, device="cuda")
    out = ops.attention(st.cache, wl.q.cuda().contiguous(), st.step["bt"], st.step["sl"],
                        st.step["qsl"], wl.seq_lens, wl.qsl, wl.scale,
                        kv_split_tokens=kv_split_tokens, lse_out=lse_out, workspace=ws,
                        common_prefix_tokens=P)
    torch.cuda.synchronize()
    return out.cpu().numpy(), (None if lse_out is None else lse_out.cpu().numpy())


def test_cascade_prefix_share_decode_all_rows():
    wl = W.prefix_share_decode()
    st = GpuStep(wl)
    P = 16 * B.pa_common_prefix_blocks(wl.block_table, wl.seq_lens, wl.qsl)
    assert P == 1024
    want, want_lse = oracle_attention_all(wl, oracle_cache(wl))
    got, lse = _cascade(st, P, lse=True)
    stats = assert_close(got, want, W.BF16, "cascade prefix_share_decode")
    print("cascade", stats)
    assert np.max(np.abs(lse - want_lse)) < 1e-3
    # and the same rows without cascade agree with it closely
    assert np.max(np.abs(got - st.out.cpu().numpy())) < 2e-3
    # forced splits of the suffix walk: the split merge takes the prefix partials too
    for split in [16, 64]:
        got, lse = _cascade(st, P, kv_split_tokens=split, lse=True)
        assert_close(got, want, W.BF16, f"cascade split {split}")
        assert np.max(np.abs(lse - want_lse)) < 1e-3


def _small(ctx, ql, hq, hkv, d, seed, shared, nb=None):
    need = -(-shared // 16) + sum(-(-c // 16) - shared // 16 for c in ctx)
    return W.make_workload("cascade-edge", ctx, ql, hq, hkv, d, 16, nb or need + 8, seed,
                           shared_prefix_tokens=shared)


CASES = {
    # name: (ctx, q_len, Hq, Hkv, D, shared prefix tokens)
    "one_block_prefix": ([17, 40, 100], [1, 1, 1], 8, 2, 128, 16),
    "suffix_of_one_token": ([65, 65, 80], [1, 1, 1], 8, 2, 128, 64),
    "prefix_not_tile_aligned": ([200, 130, 61], [1, 1, 1], 32, 8, 128, 48),
    "spec_decode_qlen2_g4": ([600, 520, 700], [2, 2, 2], 8, 2, 128, 512),
    "g8_long_prefix": ([2500, 2100], [1, 1], 64, 8, 128, 2048),
    "mha_group1": ([300, 400, 350], [1, 1, 1], 4, 4, 128, 256),
    "head_size_64": ([300, 180, 99], [1, 1, 1], 4, 2, 64, 96),
    "zero_query_first": ([300, 400, 350, 500], [0, 1, 0, 1], 8, 2, 128, 256),
    "many_requests": ([int(x) for x in 64 + np.random.default_rng(7).integers(1, 200, 300)],
                      [1] * 300, 8, 2, 128, 64),
}


@pytest.mark.parametrize("case", sorted(CASES))
def test_cascade_edge_case(case):
    ctx, ql, hq, hkv, d, shared = CASES[case]
    wl = _small(ctx, ql, hq, hkv, d, seed=len(case) * 7 + shared, shared=shared)
    st = GpuStep(wl)
    assert B.pa_common_prefix_blocks(wl.block_table, wl.seq_lens, wl.qsl) * 16 >= shared
    want, want_lse = oracle_attention_all(wl, oracle_cache(wl))
    for P in sorted({16, shared}):
        for split in [0, 16]:
            got, lse = _cascade(st, P, kv_split_tokens=split, lse=True)
            assert_close(got, want, W.BF16, f"{case} P {P} split {split}")
            assert np.max(np.abs(lse - want_lse)) < 1e-3, (case, P, split)


def test_cascade_fp8_cache():
    # the prefix pass on the FP8 chunk path, the suffixes on the FP8 decode path
    wl = W.make_workload("cascade-fp8", [700, 900, 1300, 650], [1, 1, 1, 1], 32, 8, 128, 16,
                         400, 61, kv_dtype=W.FP8_E4M3, shared_prefix_tokens=512)
    st = GpuStep(wl)
    want, want_lse = oracle_attention_all(wl, oracle_cache(wl))
    for split in [0, 64]:
        got, lse = _cascade(st, 512, kv_split_tokens=split, lse=True)
        assert_close(got, want, W.FP8_E4M3, f"fp8 cascade split {split}")
        assert np.max(np.abs(lse - want_lse)) < 2e-3


def test_cascade_with_a_workspace_for_one_prefix_split():
    wl = W.prefix_share_decode()
    st = GpuStep(wl, run_attention=False)
    T, Hq, D = wl.num_tokens, wl.num_q_heads, wl.head_size
    one = -(-T * Hq * D * 4 // 256) * 256 + -(-T * Hq * 4 // 256) * 256
    plan = B.pa_plan_attention(wl.seq_lens, wl.qsl, Hq, wl.num_kv_heads, D,
                               wl.max_blocks_per_seq, 148, one, common_prefix_tokens=1024)
    assert plan["prefix_splits"] == 1
    want, _ = oracle_attention_all(wl, oracle_cache(wl))
    got, _ = _cascade(st, 1024, workspace_bytes=one)
    assert_close(got, want, W.BF16, "one prefix split")


def test_cascade_refusals_launch_nothing():
    wl = _small([300, 400], [1, 1], 8, 2, 128, seed=3, shared=256)
    st = GpuStep(wl, run_attention=False)
    out = torch.full((wl.num_tokens, 8, 128), 7.0, device="cuda")
    # 304 > 299 computed tokens of the first request; 250 is not a whole number of blocks
    for P, status in [(304, B.PA_ERR_METADATA), (250, B.PA_ERR_INVALID_ARG)]:
        with pytest.raises(B.PaError) as e:
            ops.attention(st.cache, wl.q.cuda(), st.step["bt"], st.step["sl"], st.step["qsl"],
                          wl.seq_lens, wl.qsl, wl.scale, out=out, common_prefix_tokens=P)
        assert e.value.status == status
    torch.cuda.synchronize()
    assert torch.all(out == 7.0)
