"""pa_attention_noalloc against pa_attention and the oracle, through the C ABI.

Some callers cannot allocate device memory where they run attention -- a host framework that
owns all device memory and gives plugins no allocator, or a serving process whose memory
budget forbids allocation after start-up -- so they cannot pass pa_attention a workspace for
its split-KV partials.  pa_attention_noalloc keeps those partials in the library's fixed
static scratch instead.  These tests check that it returns what pa_attention returns with a
workspace of the scratch's size, and what the fp64 oracle computes, on two calls in a row (the
second one running over the scratch the first one left behind); that a step too large to
split within the scratch still runs, unsplit; and that argument errors come before anything
else.  The file is collected last and builds all it needs itself, so it passes alone in a
fresh process as well as after the other tests."""
import numpy as np
import pytest
import torch

from gpu_common import TOL, GpuStep, assert_close, oracle_attention_all, oracle_cache
from paged_kv_cache_421_b200 import _binding as B
from paged_kv_cache_421_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _with_pa_attention(st, workspace_bytes=None) -> torch.Tensor:
    """pa_attention with a workspace of `workspace_bytes` (default: the scratch's size)."""
    wl = st.wl
    T, Hq, D = wl.num_tokens, wl.num_q_heads, wl.head_size
    nb = B.PA_NOALLOC_SCRATCH_BYTES if workspace_bytes is None else workspace_bytes
    ws = torch.empty(max(nb, 256), dtype=torch.uint8, device="cuda")
    out = torch.full((T, Hq, D), float("nan"), device="cuda")
    B.pa_attention(st.cache.handle, wl.q.cuda(), Hq, st.step["bt"], wl.max_blocks_per_seq,
                   st.step["sl"], st.step["qsl"], wl.seq_lens, wl.qsl, wl.num_seqs, T, wl.scale,
                   out, ws, nb)
    torch.cuda.synchronize()
    return out


def _with_noalloc(st) -> torch.Tensor:
    wl = st.wl
    T, Hq, D = wl.num_tokens, wl.num_q_heads, wl.head_size
    out = torch.full((T, Hq, D), float("nan"), device="cuda")
    B.pa_attention_noalloc(st.cache.handle, wl.q.cuda(), Hq, st.step["bt"], wl.max_blocks_per_seq,
                           st.step["sl"], st.step["qsl"], wl.seq_lens, wl.qsl, wl.num_seqs, T,
                           wl.scale, out)
    torch.cuda.synchronize()
    return out


def _plan(wl, workspace_bytes):
    return B.pa_plan_attention(wl.seq_lens, wl.qsl, wl.num_q_heads, wl.num_kv_heads,
                               wl.head_size, wl.max_blocks_per_seq,
                               torch.cuda.get_device_properties(0).multi_processor_count,
                               workspace_bytes)


def test_noalloc_matches_pa_attention_and_oracle_on_two_calls_in_a_row():
    rng = np.random.default_rng(77)
    # call 1: long decodes (split into many KV partitions) and a causal chunk
    ctx1 = np.concatenate([rng.integers(3000, 9000, size=6), [700]])
    wl1 = W.make_workload("noalloc-1", ctx1, [1] * 6 + [200], 32, 8, 128, 16, 4096, 901)
    # call 2: a different batch (70B-like heads), over the scratch call 1 left behind
    ctx2 = rng.integers(5000, 20000, size=3)
    wl2 = W.make_workload("noalloc-2", ctx2, [1, 1, 1], 64, 8, 128, 16, 4096, 902)
    max_tol, mean_tol = TOL[W.BF16]
    for wl in (wl1, wl2):
        plan = _plan(wl, B.PA_NOALLOC_SCRATCH_BYTES)
        assert plan["any_split"] and plan["workspace_needed"] <= B.PA_NOALLOC_SCRATCH_BYTES
        st = GpuStep(wl, run_attention=False)
        want = _with_pa_attention(st).cpu().numpy()
        got = _with_noalloc(st).cpu().numpy()
        assert np.all(np.isfinite(got))
        err = np.abs(got.astype(np.float64) - want)
        assert err.max() <= max_tol and err.mean() <= mean_tol, (wl.name, err.max(), err.mean())
        # and against the fp64 oracle on every row
        ref, _ = oracle_attention_all(wl, oracle_cache(wl), threads=0)
        assert_close(got, ref, W.BF16, f"{wl.name} vs oracle")
    assert B.pa_device_error(reset=True) == 0


def test_noalloc_runs_a_step_too_large_to_split_within_its_scratch():
    # 2048 chunk tokens x 32 q heads: two splits of every row would need more than 64 MiB of
    # partials, so the planner keeps the chunk whole, exactly as pa_attention does with a
    # workspace of the scratch's size
    wl = W.make_workload("noalloc-big", [2048], [2048], 32, 8, 128, 16, 160, 903)
    assert (B.pa_attention_workspace_bytes(wl.num_tokens, 32, 128, 2)
            > B.PA_NOALLOC_SCRATCH_BYTES)
    plan = _plan(wl, B.PA_NOALLOC_SCRATCH_BYTES)
    assert not plan["any_split"] and plan["workspace_needed"] == 0
    st = GpuStep(wl, run_attention=False)
    want = _with_pa_attention(st).cpu().numpy()
    got = _with_noalloc(st).cpu().numpy()
    assert np.array_equal(got, want), "same plan, same kernels: same bits"
    ref, _ = oracle_attention_all(wl, oracle_cache(wl), threads=0)
    assert_close(got, ref, W.BF16, "unsplit chunk vs oracle")
    assert B.pa_device_error(reset=True) == 0


def test_noalloc_checks_arguments_before_anything_else():
    st = GpuStep(W.make_workload("noalloc-args", [40], [1], 64, 8, 128, 16, 16, 904),
                 run_attention=False)
    T, Hq = 4096, 64
    out = torch.zeros(T, Hq, 128, device="cuda")
    with pytest.raises(B.PaError) as e:  # null q with a large step: INVALID_ARG, as pa_attention
        B.pa_attention_noalloc(st.cache.handle, None, Hq, st.step["bt"], 3, st.step["sl"],
                               st.step["qsl"], np.array([T], np.int32),
                               np.array([0, T], np.int32), 1, T, 0.1, out)
    assert e.value.status == B.PA_ERR_INVALID_ARG
    q = torch.zeros(T, 60, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(B.PaError) as e:  # 60 q heads over 8 kv heads
        B.pa_attention_noalloc(st.cache.handle, q, 60, st.step["bt"], 3, st.step["sl"],
                               st.step["qsl"], np.array([T], np.int32),
                               np.array([0, T], np.int32), 1, T, 0.1, out)
    assert e.value.status == B.PA_ERR_INVALID_ARG
