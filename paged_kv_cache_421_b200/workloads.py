"""Seeded synthetic serving-step workloads.

This module only draws inputs: request lengths, a shuffled physical block pool handed out
as per-request block tables, and Q/K/V values.  It holds none of the hot path's arithmetic
(no slot computation, no cache write, no attention); both the CUDA library and the fp64
oracle consume what it produces.

A workload describes one batch step of a continuous-batching engine ("Inside vLLM" reading
notes, core point 2: all scheduled requests flattened into one super-sequence, decodes first
and prefill chunks after them):

* ``seq_lens[r]``: request r's total KV length including this step's new tokens;
* ``qsl``: query_start_loc, the prefix offsets of each request's new tokens ([B + 1]);
* ``block_table[r]``: physical block ids for request r's logical blocks, drawn in order from
  a seeded permutation of the pool (the free-block queue); rows are padded with block 0;
* a *history step* (``hist_*``): the earlier tokens of every request, laid out as a prefill
  step of its own, so that each side fills its own cache through its own slot mapping and
  write before the step under test;
* ``pos_rows``/``pos_start``: for each request and position, the row of
  ``cat(k_hist, k_new)`` that holds that position's K/V (an unpaged view of the same data).

Values: Q, K, V ~ N(0, 1) rounded to bf16.  FP8 scales (per kv head, separately for K and
V) are amax over all of that head's K (resp. V) values / 448.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np
import torch

BF16 = 0
FP8_E4M3 = 1

# Fill for never-written cache slots: finite and large (bf16 32768.0; E4M3 448), so a
# stray read shows up in the error instead of hiding.
CACHE_FILL_BF16 = 0x4700
CACHE_FILL_FP8 = 0x7E

SEED_BASE = 4210  # per-config seed = 4210 + config number


@dataclass
class Workload:
    name: str
    num_q_heads: int
    num_kv_heads: int
    head_size: int
    block_size: int
    num_blocks: int
    kv_dtype: int
    scale: float
    seq_lens: np.ndarray           # int32 [B]
    qsl: np.ndarray                # int32 [B+1]
    block_table: np.ndarray        # int32 [B][max_blocks]
    hist_seq_lens: np.ndarray      # int32 [Bh]
    hist_qsl: np.ndarray           # int32 [Bh+1]
    hist_block_table: np.ndarray   # int32 [Bh][max_blocks]
    pos_rows: np.ndarray           # int64 [sum seq_lens]
    pos_start: np.ndarray          # int64 [B+1]
    q: torch.Tensor                # bf16 [T][Hq][D]
    k_new: torch.Tensor            # bf16 [T][Hkv][D]
    v_new: torch.Tensor
    k_hist: torch.Tensor           # bf16 [Th][Hkv][D]
    v_hist: torch.Tensor
    k_scale: Optional[torch.Tensor] = None  # fp32 [Hkv]
    v_scale: Optional[torch.Tensor] = None
    meta: dict = field(default_factory=dict)

    @property
    def num_seqs(self) -> int:
        return int(self.seq_lens.size)

    @property
    def num_tokens(self) -> int:
        return int(self.qsl[-1])

    @property
    def q_lens(self) -> np.ndarray:
        return np.diff(self.qsl)

    @property
    def dtype_bytes(self) -> int:
        return 2 if self.kv_dtype == BF16 else 1

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_table.shape[1])

    def kv_src(self):
        """(k_src, v_src) = cat(history, new): the rows ``pos_rows`` index."""
        return (torch.cat([self.k_hist, self.k_new.to(self.k_hist.device)]),
                torch.cat([self.v_hist, self.v_new.to(self.v_hist.device)]))


def _randn_bf16(gen: torch.Generator, shape, device) -> torch.Tensor:
    return torch.randn(*shape, generator=gen, device=device, dtype=torch.float32).to(
        torch.bfloat16)


def make_workload(name: str, ctx_lens, q_lens, num_q_heads: int, num_kv_heads: int,
                  head_size: int, block_size: int, num_blocks: int, seed: int,
                  kv_dtype: int = BF16, shared_prefix_tokens: int = 0,
                  scale: Optional[float] = None, device="cpu",
                  max_blocks_per_seq: Optional[int] = None) -> Workload:
    """Build one step.  ``ctx_lens[r]`` is the total length after this step (new tokens
    included); ``q_lens[r]`` the number of new tokens.  With ``shared_prefix_tokens`` > 0
    every request's first tokens live in the same physical blocks (a whole number of
    blocks, written once by the history step), as after a prefix-cache hit."""
    rng = np.random.default_rng(seed)
    ctx = np.asarray(ctx_lens, np.int64)
    ql = np.asarray(q_lens, np.int64)
    B = ctx.size
    assert ql.size == B and np.all(ql >= 0) and np.all(ql <= ctx)
    assert shared_prefix_tokens % block_size == 0
    assert np.all(ctx - ql >= shared_prefix_tokens)

    # Block allocation, as the scheduler's allocator would hand them out: the pool is a
    # seeded permutation of all physical ids, consumed in order.
    pool = rng.permutation(num_blocks).astype(np.int32)
    need = [-(-int(c) // block_size) for c in ctx]  # allocator's block count per request
    n_shared = shared_prefix_tokens // block_size
    max_blocks = max(need) if max_blocks_per_seq is None else max_blocks_per_seq
    assert max_blocks >= max(need)
    total_needed = n_shared + sum(n - n_shared for n in need)
    assert total_needed <= num_blocks, "pool too small for this workload"
    block_table = np.zeros((B, max_blocks), np.int32)
    shared = pool[:n_shared]
    cursor = n_shared
    for r in range(B):
        block_table[r, :n_shared] = shared
        own = need[r] - n_shared
        block_table[r, n_shared:need[r]] = pool[cursor:cursor + own]
        cursor += own

    qsl = np.zeros(B + 1, np.int32)
    qsl[1:] = np.cumsum(ql)
    seq_lens = ctx.astype(np.int32)

    # History step: positions [0, ctx - q_len) of every request.  With a shared prefix its
    # tokens form one extra pseudo-request (index 0) over the shared blocks only.
    hist_ctx, hist_q, hist_bt = [], [], []
    if n_shared:
        hist_ctx.append(shared_prefix_tokens)
        hist_q.append(shared_prefix_tokens)
        row = np.zeros(max_blocks, np.int32)
        row[:n_shared] = shared
        hist_bt.append(row)
    for r in range(B):
        done = int(ctx[r] - ql[r])
        hist_ctx.append(done)
        hist_q.append(done - shared_prefix_tokens)
        hist_bt.append(block_table[r])
    hist_seq_lens = np.asarray(hist_ctx, np.int32)
    hist_qsl = np.zeros(len(hist_q) + 1, np.int32)
    hist_qsl[1:] = np.cumsum(hist_q)
    hist_block_table = np.stack(hist_bt).astype(np.int32)
    Th = int(hist_qsl[-1])
    T = int(qsl[-1])

    # Unpaged view: source row (in cat(k_hist, k_new)) of every (request, position).
    pos_start = np.zeros(B + 1, np.int64)
    pos_start[1:] = np.cumsum(ctx)
    pos_rows = np.empty(int(pos_start[-1]), np.int64)
    h0 = 1 if n_shared else 0
    for r in range(B):
        base = int(pos_start[r])
        if n_shared:
            pos_rows[base:base + shared_prefix_tokens] = np.arange(shared_prefix_tokens)
        own_hist = int(hist_q[h0 + r])
        start_h = int(hist_qsl[h0 + r])
        pos_rows[base + shared_prefix_tokens: base + shared_prefix_tokens + own_hist] = \
            np.arange(start_h, start_h + own_hist)
        done = int(ctx[r] - ql[r])
        pos_rows[base + done: base + int(ctx[r])] = Th + np.arange(int(qsl[r]), int(qsl[r + 1]))

    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    q = _randn_bf16(gen, (T, num_q_heads, head_size), dev)
    k_new = _randn_bf16(gen, (T, num_kv_heads, head_size), dev)
    v_new = _randn_bf16(gen, (T, num_kv_heads, head_size), dev)
    k_hist = _randn_bf16(gen, (Th, num_kv_heads, head_size), dev)
    v_hist = _randn_bf16(gen, (Th, num_kv_heads, head_size), dev)

    k_scale = v_scale = None
    if kv_dtype == FP8_E4M3:
        def amax(a, b):
            m = torch.zeros(num_kv_heads, device=dev, dtype=torch.float32)
            for t in (a, b):
                if t.shape[0]:
                    m = torch.maximum(m, t.float().abs().amax(dim=(0, 2)))
            return m
        k_scale = (amax(k_hist, k_new) / 448.0).clamp_min(1e-12)
        v_scale = (amax(v_hist, v_new) / 448.0).clamp_min(1e-12)

    if scale is None:
        scale = 1.0 / float(np.sqrt(head_size))
    return Workload(name=name, num_q_heads=num_q_heads, num_kv_heads=num_kv_heads,
                    head_size=head_size, block_size=block_size, num_blocks=num_blocks,
                    kv_dtype=kv_dtype, scale=scale, seq_lens=seq_lens, qsl=qsl,
                    block_table=block_table, hist_seq_lens=hist_seq_lens, hist_qsl=hist_qsl,
                    hist_block_table=hist_block_table, pos_rows=pos_rows,
                    pos_start=pos_start, q=q, k_new=k_new, v_new=v_new, k_hist=k_hist,
                    v_hist=v_hist, k_scale=k_scale, v_scale=v_scale,
                    meta={"seed": seed, "shared_prefix_tokens": shared_prefix_tokens})


# ---------------------------------------------------------------- the five serving steps
def tiny_decode(device="cpu") -> Workload:
    """4 decode requests, context {1, 17, 33, 64}; 4 q / 2 kv heads, head_dim 64,
    block 16, a 64-block pool; scale 1/sqrt(64)."""
    return make_workload("tiny_decode", [1, 17, 33, 64], [1, 1, 1, 1], 4, 2, 64, 16, 64,
                         SEED_BASE + 1, scale=1.0 / 8.0, device=device)


def llama8b_decode(device="cpu") -> Workload:
    """64 decode requests, context uniform in [512, 4096]; 32 q / 8 kv heads, head_dim 128,
    block 16; a 16384-block (1 GiB bf16) shuffled pool."""
    rng = np.random.default_rng(SEED_BASE + 2)
    ctx = rng.integers(512, 4096, size=64, endpoint=True)
    return make_workload("llama8b_decode", ctx, np.ones(64, np.int64), 32, 8, 128, 16, 16384,
                         SEED_BASE + 2, device=device)


def mixed_step(kv_dtype: int = BF16, device="cpu") -> Workload:
    """48 decodes (context uniform in [1024, 8192]) then two 512-token prefill chunks with 0
    and 2048 tokens already computed; 1072 tokens of a 2048-token budget; 32/8 heads,
    head_dim 128, block 16, a 65536-block pool; bf16 or FP8 E4M3 cache."""
    rng = np.random.default_rng(SEED_BASE + 3)
    dec = rng.integers(1024, 8192, size=48, endpoint=True)
    ctx = np.concatenate([dec, [512, 2048 + 512]])
    ql = np.concatenate([np.ones(48, np.int64), [512, 512]])
    assert ql.sum() <= 2048
    name = "mixed_step" + ("_fp8" if kv_dtype == FP8_E4M3 else "")
    return make_workload(name, ctx, ql, 32, 8, 128, 16, 65536, SEED_BASE + 3,
                         kv_dtype=kv_dtype, device=device)


def prefill_chunks(device="cpu") -> Workload:
    """The mixed step's two prefill chunks alone, the chunk kernel's share of that step: 512
    new tokens over 0 and over 2048 computed ones; 32/8 heads, head_dim 128, block 16."""
    return make_workload("prefill_chunks", [512, 2048 + 512], [512, 512], 32, 8, 128, 16,
                         65536, SEED_BASE + 6, device=device)


def prefix_share_decode(device="cpu") -> Workload:
    """128 decode requests sharing a 1024-token prefix (the same 64 physical blocks in every
    table) plus private suffixes of uniform [64, 512] tokens; 32/8 heads, head_dim 128."""
    rng = np.random.default_rng(SEED_BASE + 4)
    suffix = rng.integers(64, 512, size=128, endpoint=True)
    ctx = 1024 + suffix
    return make_workload("prefix_share_decode", ctx, np.ones(128, np.int64), 32, 8, 128, 16,
                         16384, SEED_BASE + 4, shared_prefix_tokens=1024, device=device)


def long70b_decode(kv_dtype: int = BF16, device="cpu") -> Workload:
    """8 decode requests, context uniform in [32768, 131072]; 64 q / 8 kv heads, head_dim
    128, block 16, a 65536-block pool; bf16 or FP8 E4M3 cache with per-kv-head scales."""
    rng = np.random.default_rng(SEED_BASE + 5)
    ctx = rng.integers(32768, 131072, size=8, endpoint=True)
    name = "long70b_decode" + ("_fp8" if kv_dtype == FP8_E4M3 else "")
    return make_workload(name, ctx, np.ones(8, np.int64), 64, 8, 128, 16, 65536,
                         SEED_BASE + 5, kv_dtype=kv_dtype, device=device)


CONFIGS = {
    "tiny_decode": tiny_decode,
    "llama8b_decode": llama8b_decode,
    "mixed_step": mixed_step,
    "prefix_share_decode": prefix_share_decode,
    "long70b_decode": long70b_decode,
    "long70b_decode_fp8": lambda device="cpu": long70b_decode(FP8_E4M3, device=device),
    "mixed_step_fp8": lambda device="cpu": mixed_step(FP8_E4M3, device=device),
    "prefill_chunks": prefill_chunks,
}


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> numpy uint16 bit patterns (host copy)."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
