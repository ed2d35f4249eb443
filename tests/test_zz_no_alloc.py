"""pa_attention_noalloc against pa_attention, through the C ABI.

Some callers cannot allocate device memory where they run attention -- a host framework that
owns all device memory and gives plugins no allocator, or a serving process whose memory
budget forbids allocation after start-up -- so they cannot pass pa_attention a workspace for
its split-KV partials.  pa_attention_noalloc keeps those partials in the library's fixed
static scratch instead.  These tests check that it returns what pa_attention returns, on two
calls in a row (the second one running over the scratch the first one left behind), and that
calls too large for the scratch are refused.  The file is collected last and builds all it
needs itself, so it passes alone in a fresh process as well as after the other tests."""
import numpy as np
import pytest
import torch

from gpu_common import TOL, GpuStep
from paged_kv_cache_421_b200 import _binding as B
from paged_kv_cache_421_b200 import ops
from paged_kv_cache_421_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _with_pa_attention(st) -> torch.Tensor:
    wl = st.wl
    T, Hq, D = wl.num_tokens, wl.num_q_heads, wl.head_size
    nb = ops.workspace_bytes_for(st.cache, wl.seq_lens, wl.qsl, Hq, wl.max_blocks_per_seq)
    ws = torch.empty(max(nb, 256), dtype=torch.uint8, device="cuda")
    out = torch.full((T, Hq, D), float("nan"), device="cuda")
    B.pa_attention(st.cache.handle, wl.q.cuda(), Hq, st.step["bt"], wl.max_blocks_per_seq,
                   st.step["sl"], st.step["qsl"], wl.seq_lens, wl.qsl, wl.num_seqs, T, wl.scale,
                   out, ws, ws.numel())
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


def test_noalloc_matches_pa_attention_on_two_calls_in_a_row():
    rng = np.random.default_rng(77)
    # call 1: long decodes (split into many KV partitions) and a causal chunk
    ctx1 = np.concatenate([rng.integers(3000, 9000, size=6), [700]])
    wl1 = W.make_workload("noalloc-1", ctx1, [1] * 6 + [200], 32, 8, 128, 16, 4096, 901)
    # call 2: a different batch (70B-like heads), over the scratch call 1 left behind
    ctx2 = rng.integers(5000, 20000, size=3)
    wl2 = W.make_workload("noalloc-2", ctx2, [1, 1, 1], 64, 8, 128, 16, 4096, 902)
    max_tol, mean_tol = TOL[W.BF16]
    for wl in (wl1, wl2):
        plan = B.pa_plan_attention(wl.seq_lens, wl.qsl, wl.num_q_heads, wl.num_kv_heads,
                                   wl.head_size, wl.max_blocks_per_seq,
                                   torch.cuda.get_device_properties(0).multi_processor_count,
                                   B.PA_NOALLOC_SCRATCH_BYTES)
        assert plan["any_split"] and plan["workspace_needed"] <= B.PA_NOALLOC_SCRATCH_BYTES
        st = GpuStep(wl, run_attention=False)
        want = _with_pa_attention(st).cpu().numpy()
        got = _with_noalloc(st).cpu().numpy()
        assert np.all(np.isfinite(got))
        err = np.abs(got.astype(np.float64) - want)
        assert err.max() <= max_tol and err.mean() <= mean_tol, (wl.name, err.max(), err.mean())
    assert B.pa_device_error(reset=True) == 0


def test_noalloc_refuses_calls_larger_than_its_scratch():
    # 2 splits x 2048 tokens x 64 heads x 129 floats > 64 MiB: refused before any launch
    st = GpuStep(W.make_workload("noalloc-big", [40], [1], 64, 8, 128, 16, 16, 903),
                 run_attention=False)
    T, Hq = 2048, 64
    q = torch.zeros(T, Hq, 128, dtype=torch.bfloat16, device="cuda")
    out = torch.zeros(T, Hq, 128, device="cuda")
    with pytest.raises(B.PaError) as e:
        B.pa_attention_noalloc(st.cache.handle, q, Hq, st.step["bt"], 3, st.step["sl"],
                               st.step["qsl"], np.array([T], np.int32),
                               np.array([0, T], np.int32), 1, T, 0.1, out)
    assert e.value.status == B.PA_ERR_WORKSPACE
