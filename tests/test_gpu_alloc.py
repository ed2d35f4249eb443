"""Device block allocation (allocate_slots and the free-block queue) against the oracle:
block tables, per-request counts and the queue state bit-exact, then the step's slot mapping
from the allocated tables."""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_421_b200 import _binding as B
from paged_kv_cache_421_b200 import ops

pytestmark = pytest.mark.gpu


def _case(rng, B_, cap, max_blocks, bs=16, fill_frac=None):
    queue = rng.permutation(4 * cap + 7)[:cap].astype(np.int32)
    head = int(rng.integers(0, cap))
    count = int(rng.integers(0, cap + 1)) if fill_frac is None else int(cap * fill_frac)
    computed = rng.integers(0, (max_blocks - 2) * bs, B_).astype(np.int32)
    new = np.where(rng.random(B_) < 0.7, 1, rng.integers(0, 3 * bs, B_)).astype(np.int32)
    bt = np.full((B_, max_blocks), -5, np.int32)
    for r in range(B_):
        h = -(-int(computed[r]) // bs)
        bt[r, :h] = rng.integers(0, 10000, h)
    return queue, head, count, computed, new, bt


def _run_both(queue, head, count, computed, new, bt, bs=16):
    want_bt, want_st = bt.copy(), np.array([head, count], np.int32)
    want = oracle.allocate_slots(want_bt, computed, new, bs, queue, want_st)
    d_bt = torch.from_numpy(bt).cuda()
    d_q = torch.from_numpy(queue).cuda()
    d_st = torch.tensor([head, count], dtype=torch.int32, device="cuda")
    d_out = torch.empty(len(computed), dtype=torch.int32, device="cuda")
    B.pa_allocate_slots(d_bt, bt.shape[1], torch.from_numpy(computed).cuda(),
                        torch.from_numpy(new).cuda(), len(computed), bs, d_q, queue.size, d_st,
                        d_out)
    torch.cuda.synchronize()
    assert B.pa_device_error(reset=True) == 0
    return (want, want_bt, want_st), (d_out.cpu().numpy(), d_bt.cpu().numpy(), d_st.cpu().numpy())


@pytest.mark.parametrize("seed", range(8))
def test_allocate_matches_oracle(seed):
    rng = np.random.default_rng(500 + seed)
    B_ = [1, 7, 300, 1023, 1024, 1025, 2500, 4096][seed]  # single and several 1024-request chunks
    cap = int(rng.integers(1, 4 * B_ + 2))
    queue, head, count, computed, new, bt = _case(rng, B_, cap, max_blocks=12)
    (w, wbt, wst), (g, gbt, gst) = _run_both(queue, head, count, computed, new, bt)
    assert np.array_equal(g, w)
    assert np.array_equal(gbt, wbt)
    assert np.array_equal(gst, wst)


def test_allocate_exhaustion_and_overflow_stop_service():
    rng = np.random.default_rng(9)
    for frac in [0.0, 0.05, 0.5, 1.0]:
        queue, head, count, computed, new, bt = _case(rng, 2000, 1500, max_blocks=6,
                                                      fill_frac=frac)
        new[700] = 200  # a row that overflows 6 blocks: service stops there at the latest
        (w, wbt, wst), (g, gbt, gst) = _run_both(queue, head, count, computed, new, bt)
        assert np.array_equal(g, w) and np.array_equal(gbt, wbt) and np.array_equal(gst, wst)
        assert (g[700:] == -1).all()


def test_free_then_allocate_and_slot_mapping():
    rng = np.random.default_rng(11)
    cap, B_, mb = 600, 40, 16
    ids = rng.permutation(cap).astype(np.int32)
    q = ops.BlockQueue(torch.from_numpy(ids[:400]).cuda(), capacity=cap)
    oq = np.zeros(cap, np.int32)
    oq[:400] = ids[:400]
    ost = np.array([0, 400], np.int32)
    bt = np.full((B_, mb), -1, np.int32)
    d_bt = torch.from_numpy(bt).cuda()
    computed = np.zeros(B_, np.int32)
    for step in range(6):
        new = rng.integers(1, 40, B_).astype(np.int32)
        got = ops.allocate_slots(d_bt, torch.from_numpy(computed).cuda(),
                                 torch.from_numpy(new).cuda(), q)
        want = oracle.allocate_slots(bt, computed, new, 16, oq, ost)
        assert np.array_equal(got.cpu().numpy(), want)
        assert np.array_equal(d_bt.cpu().numpy(), bt)
        assert np.array_equal(q.state.cpu().numpy(), ost)
        served = want >= 0
        # the step's slot mapping from the allocated tables (served requests only)
        sl = (computed + new)[served]
        qsl = np.concatenate([[0], np.cumsum(new[served])]).astype(np.int32)
        if served.any():
            rows = np.ascontiguousarray(bt[served])
            slots = ops.slot_mapping(torch.from_numpy(rows).cuda(), torch.from_numpy(sl).cuda(),
                                     torch.from_numpy(qsl).cuda(), int(qsl[-1]))
            assert np.array_equal(slots.cpu().numpy(), oracle.slot_mapping(rows, sl, qsl, 16))
        computed = np.where(served, computed + new, computed).astype(np.int32)
        # finished requests (every third, once past 200 tokens) give their blocks back
        for r in range(B_):
            if computed[r] > 200 and r % 3 == step % 3:
                nb = -(-int(computed[r]) // 16)
                back = bt[r, :nb].copy()
                ops.free_blocks(torch.from_numpy(back).cuda(), q)
                oracle.free_blocks(back, oq, ost)
                bt[r, :] = -1
                d_bt[r, :] = -1
                computed[r] = 0
        torch.cuda.synchronize()
        assert np.array_equal(q.queue.cpu().numpy(), oq)
        assert np.array_equal(q.state.cpu().numpy(), ost)
    assert B.pa_device_error(reset=True) == 0
