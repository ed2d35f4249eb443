"""Multi-rank host logic of the benchmark on CPU (gloo, world size 2).

The serving step shards by request batch: every rank runs its own batch with no collective
on the data path, and only the timing is combined (max over ranks).  These tests run the
same host code the GPU ranks run, with gloo on CPU."""
import json
import os
import socket
import subprocess
import sys

import torch.distributed as dist
import torch.multiprocessing as mp

from conftest import ROOT


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    sys.path.insert(0, ROOT)
    import bench
    got = bench.max_over_ranks(1.5 + rank, world, device="cpu")
    # every rank reports the same max, regardless of its own value
    q.put((rank, got))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_gloo():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=10) for _ in range(world))
    assert res == {0: 2.5, 1: 2.5}


def test_reference_arm_runs_on_rank0_only():
    # under torchrun the oracle arm runs and prints on rank 0; the other ranks exit quietly
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl",
           "reference", "--gpus", "2", "--steps", "1", "--warmup", "0", "--workload",
           "tiny_decode"]
    res = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2
    assert rec["cpu_baseline"]["kind"] == "oracle" and rec["value"] > 0
    assert rec["e2e"]["h2d_bytes_per_step"] == 0


def test_bench_byte_accounting():
    sys.path.insert(0, ROOT)
    import bench
    from paged_kv_cache_421_b200 import workloads as W
    wl = W.tiny_decode()
    assert bench.kv_bytes(wl) == 58880
    assert bench.decode_kv_bytes(wl) == 58880
    assert bench.unique_kv_bytes(wl) == 10 * 8192
    wl = W.mixed_step()
    assert bench.decode_kv_bytes(wl) == bench.kv_bytes(wl) - (512 + 2560) * 2 * 8 * 128 * 2
    wl = W.prefix_share_decode()
    assert bench.unique_kv_bytes(wl) < bench.kv_bytes(wl)
    args = bench.parse_args([])
    assert args.gpus == 1 and args.steps > 0 and args.warmup >= 3


def test_bench_flop_and_window_accounting():
    """The algorithmic FLOPs and windowed bytes bench.py reports, against brute-force counts
    of the unmasked (query, key) pairs and visible keys."""
    sys.path.insert(0, ROOT)
    import bench
    from paged_kv_cache_421_b200 import workloads as W
    wl = W.mixed_step()
    # the mixed step's prefill FLOPs: 4 D per unmasked pair per q head (about 21.5 GFLOP)
    pairs = 0
    for ctx, ql in zip(wl.seq_lens, wl.q_lens):
        if ql * (wl.num_q_heads // wl.num_kv_heads) > 8:
            pairs += sum(int(ctx) - int(ql) + i + 1 for i in range(int(ql)))
    assert bench.chunk_flops(wl) == pairs * wl.num_q_heads * 4 * wl.head_size
    assert abs(bench.chunk_flops(wl) / 1e9 - 21.48) < 0.01
    for window in [1, 100, 700, 5000]:
        pairs_w = 0
        for ctx, ql in zip(wl.seq_lens, wl.q_lens):
            if ql * 4 > 8:
                pairs_w += sum(min(int(ctx) - int(ql) + i + 1, window) for i in range(int(ql)))
        assert bench.chunk_flops(wl, window) == pairs_w * wl.num_q_heads * 4 * wl.head_size
        keys = 0
        for ctx, ql in zip(wl.seq_lens, wl.q_lens):
            first = max(0, int(ctx) - int(ql) - window + 1)  # window start of the first query
            keys += int(ctx) - first
        assert bench.kv_bytes(wl, window) == keys * 2 * wl.num_kv_heads * wl.head_size * 2
    # a window as long as every context changes nothing
    assert bench.kv_bytes(wl, int(wl.seq_lens.max())) == bench.kv_bytes(wl)
    assert bench.chunk_flops(wl, int(wl.seq_lens.max())) == bench.chunk_flops(wl)


def test_bench_local_chunk_accounting():
    """Chunked local attention: a query at position p sees p % C + 1 keys (its own chunk up to
    itself), and with a window W as well, the smaller of that and W."""
    sys.path.insert(0, ROOT)
    import bench
    from paged_kv_cache_421_b200 import workloads as W
    wl = W.mixed_step()
    big = 1 << 40
    for C, Wn in [(1, 0), (16, 0), (100, 0), (1000, 0), (100, 37), (1000, 5000), (64, 1)]:
        pairs = keys = 0
        for ctx, ql in zip(wl.seq_lens.astype(int), wl.q_lens.astype(int)):
            p0 = ctx - ql
            keys += ctx - p0 + min(p0, Wn - 1 if Wn else big, p0 % C)
            if ql * 4 > 8:
                pairs += sum(min(p % C + 1, Wn if Wn else big) for p in range(p0, ctx))
        assert bench.chunk_flops(wl, Wn, C) == pairs * wl.num_q_heads * 4 * wl.head_size
        assert bench.kv_bytes(wl, Wn, C) == keys * 2 * wl.num_kv_heads * wl.head_size * 2
    # chunks at least as long as every context change nothing
    assert bench.kv_bytes(wl, 0, int(wl.seq_lens.max()) + 1) == bench.kv_bytes(wl)
    assert bench.chunk_flops(wl, 0, int(wl.seq_lens.max()) + 1) == bench.chunk_flops(wl)
    assert bench.parse_args(["--local-chunk", "8192"]).local_chunk == 8192


def test_bench_launch_count_follows_the_launch_sequence():
    """gpu_launches counts what pa_attention launches: the counter clear for split decodes
    and for chunk splits merged inside the tcgen05 kernel (<= 4), the reduce otherwise."""
    sys.path.insert(0, ROOT)
    import bench

    def plan(dec, chunk, ds, cs):
        return {"num_decode_seqs": dec, "num_chunk_seqs": chunk, "decode_max_splits": ds,
                "chunk_max_splits": cs}
    assert bench.launches_for_plan(plan(4, 0, 1, 0), 128) == 3      # slots, write, decode
    assert bench.launches_for_plan(plan(4, 0, 3, 0), 128) == 4      # + counter clear
    assert bench.launches_for_plan(plan(4, 2, 1, 1), 128) == 4      # decode + chunk
    assert bench.launches_for_plan(plan(0, 2, 0, 3), 128) == 4      # fused merge: clear
    assert bench.launches_for_plan(plan(0, 2, 0, 9), 128) == 4      # reduce, no clear
    assert bench.launches_for_plan(plan(4, 2, 5, 9), 128) == 6      # everything
    assert bench.launches_for_plan(plan(0, 2, 0, 3), 64) == 4       # head_size 64: reduce
