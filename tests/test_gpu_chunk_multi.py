"""Steps with decode-kind and chunk-kind requests, where the tcgen05 chunk kernel runs beside the
decode kernel on fewer CTAs than it has (q-tile pair, split) items: each CTA walks several items
in turn, its mbarrier phases carried from item to item and Q restaged for each.  The planner
chooses the CTA count (pa_plan.chunk_ctas_per_kv_head); every case first checks that it chose
fewer CTAs than items, then compares every row with the oracle, and a repeated call with the
first bit for bit."""
import numpy as np
import pytest
import torch

from gpu_common import GpuStep, assert_close, oracle_attention_all, oracle_cache
from paged_kv_cache_421_b200 import _binding as B
from paged_kv_cache_421_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean_error_word():
    B.pa_device_error(reset=True)
    yield
    assert B.pa_device_error(reset=True) == 0, "a kernel recorded a device error"


def _decodes(n, lo, hi, seed):
    rng = np.random.default_rng(seed)
    return [int(x) for x in rng.integers(lo, hi, n)]


# name: (contexts, query lengths, q heads, kv heads, kv dtype, sliding window)
_DEC = _decodes(32, 3000, 5000, 7)
CASES = {
    # chunks of ragged lengths: items whose second q-tile is partly or wholly past the rows,
    # first chunks (no history) and chunks after history
    "ragged_bf16": (_DEC + [70, 430, 1033, 250, 764, 90], [1] * 32 + [70, 130, 33, 200, 64, 90],
                    32, 8, W.BF16, 0),
    "ragged_fp8": (_DEC + [70, 430, 1033, 250, 764, 90], [1] * 32 + [70, 130, 33, 200, 64, 90],
                   32, 8, W.FP8_E4M3, 0),
    # a sliding window: items whose rows start at different keys
    "window_bf16": (_DEC + [70, 430, 1033, 250, 764, 90], [1] * 32 + [70, 130, 33, 200, 64, 90],
                    32, 8, W.BF16, 2000),
    # a long chunk split four ways: the last CTA of each q-tile pair merges the splits itself,
    # inside a CTA that has other items before or after
    "fused_split_merge": (_DEC + [1800, 300], [1] * 32 + [64, 100], 32, 8, W.BF16, 0),
    # eight splits: partials merged by the reduce kernel after the chunk kernel
    "reduce_splits": (_DEC + [4000, 300], [1] * 32 + [64, 100], 32, 8, W.BF16, 0),
    # group 3, which divides no TMA box of 128 rows: Q staged by the softmax warps (bf16) or
    # loaded and split by them from global memory (FP8), item after item
    "g3_staged_q_bf16": (_DEC + [70, 430, 1033, 250, 764, 90], [1] * 32 + [70, 130, 33, 200, 64, 90],
                         24, 8, W.BF16, 0),
    "g3_staged_q_fp8": (_DEC + [70, 430, 1033, 250, 764, 90], [1] * 32 + [70, 130, 33, 200, 64, 90],
                        24, 8, W.FP8_E4M3, 0),
    # one kv head, group 8: many small items over many CTAs of the one kv head
    "one_kv_head_many_items": (_decodes(64, 7000, 9000, 11) + [40 + 13 * i for i in range(30)],
                               [1] * 64 + [40] * 30, 8, 1, W.BF16, 0),
}


@pytest.mark.parametrize("case", sorted(CASES))
def test_chunk_items_beside_decode(case):
    ctx, ql, hq, hkv, kv_dtype, window = CASES[case]
    need = sum(-(-c // 16) for c in ctx)
    wl = W.make_workload("multi-" + case, ctx, ql, hq, hkv, 128, 16, need + 8,
                         5000 + len(case), kv_dtype=kv_dtype)
    plan = B.pa_plan_attention(wl.seq_lens, wl.qsl, hq, hkv, 128, wl.block_table.shape[1],
                               torch.cuda.get_device_properties(0).multi_processor_count,
                               1 << 30, kv_dtype=kv_dtype, sliding_window=window)
    items_per_head = plan["chunk_ctas"] // hkv
    assert 0 < plan["chunk_ctas_per_kv_head"] < items_per_head, plan
    st = GpuStep(wl, run_attention=False)
    first = st.attend(sliding_window=window)
    want, _ = oracle_attention_all(wl, oracle_cache(wl), window=window)
    assert_close(first.cpu().numpy(), want, kv_dtype, case)
    again = st.attend(sliding_window=window)
    assert torch.equal(again, first), "a repeated call differs"
