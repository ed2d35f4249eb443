"""Shared helpers of the GPU parity tests: run a workload through the library's C ABI and
build the oracle's own view of the same step from the same seeded inputs."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from paged_kv_cache_421_b200 import ops
from paged_kv_cache_421_b200 import workloads as W

# parity tolerances against fp64 (bf16 in, fp32 accumulate): max abs 2e-2, mean abs 2e-3;
# doubled for an FP8 E4M3 cache
TOL = {W.BF16: (2e-2, 2e-3), W.FP8_E4M3: (4e-2, 4e-3)}


def _dev_i32(a) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, np.int32)).cuda()


class GpuStep:
    """Everything the device computed for one workload."""

    def __init__(self, wl: W.Workload, kv_split_tokens: int = 0, fill: bool = True,
                 garbage_tail: bool = False, run_attention: bool = True):
        torch.cuda.synchronize()
        self.wl = wl
        self.cache = ops.PagedKVCache(wl.num_blocks, wl.num_kv_heads, wl.head_size, wl.kv_dtype,
                                      k_scale=wl.k_scale, v_scale=wl.v_scale)
        if fill:
            if wl.kv_dtype == W.BF16:
                self.cache.buffer.view(torch.int16).fill_(W.CACHE_FILL_BF16)
            else:
                self.cache.buffer.fill_(W.CACHE_FILL_FP8)
        if garbage_tail:
            # NaN bit patterns everywhere a valid step never writes
            if wl.kv_dtype == W.BF16:
                self.cache.buffer.view(torch.int16).fill_(0x7FC0)
            else:
                self.cache.buffer.fill_(0x7F)
        self.hist = dict(bt=_dev_i32(wl.hist_block_table), sl=_dev_i32(wl.hist_seq_lens),
                         qsl=_dev_i32(wl.hist_qsl))
        self.step = dict(bt=_dev_i32(wl.block_table), sl=_dev_i32(wl.seq_lens),
                         qsl=_dev_i32(wl.qsl))
        Th = int(wl.hist_qsl[-1])
        self.hist_slots = ops.slot_mapping(self.hist["bt"], self.hist["sl"], self.hist["qsl"], Th)
        if Th:
            ops.write_kv(self.cache, wl.k_hist.cuda().contiguous(), wl.v_hist.cuda().contiguous(),
                         self.hist_slots)
        T = wl.num_tokens
        self.slots = ops.slot_mapping(self.step["bt"], self.step["sl"], self.step["qsl"], T)
        if T:
            ops.write_kv(self.cache, wl.k_new.cuda().contiguous(), wl.v_new.cuda().contiguous(),
                         self.slots)
        self.out = None
        if run_attention:
            self.out = ops.attention(self.cache, wl.q.cuda().contiguous(), self.step["bt"],
                                     self.step["sl"], self.step["qsl"], wl.seq_lens, wl.qsl,
                                     wl.scale, kv_split_tokens=kv_split_tokens)
        torch.cuda.synchronize()

    def attend(self, kv_split_tokens: int = 0, sliding_window: int = 0,
               local_chunk: int = 0) -> torch.Tensor:
        wl = self.wl
        out = ops.attention(self.cache, wl.q.cuda().contiguous(), self.step["bt"],
                            self.step["sl"], self.step["qsl"], wl.seq_lens, wl.qsl, wl.scale,
                            kv_split_tokens=kv_split_tokens, sliding_window=sliding_window,
                            local_chunk=local_chunk)
        torch.cuda.synchronize()
        return out

    def cache_host(self) -> np.ndarray:
        return self.cache.buffer.cpu().numpy()


def oracle_cache(wl: W.Workload) -> np.ndarray:
    """The oracle's cache after the history step and this step's write (flat, native dtype)."""
    n = oracle.cache_elems(wl.num_blocks, wl.block_size, wl.num_kv_heads, wl.head_size)
    if wl.kv_dtype == W.BF16:
        cache = np.full(n, W.CACHE_FILL_BF16, np.uint16)
    else:
        cache = np.full(n, W.CACHE_FILL_FP8, np.uint8)
    ks = None if wl.k_scale is None else wl.k_scale.cpu().numpy()
    vs = None if wl.v_scale is None else wl.v_scale.cpu().numpy()
    for bt, sl, qs, k, v in [(wl.hist_block_table, wl.hist_seq_lens, wl.hist_qsl, wl.k_hist,
                              wl.v_hist),
                             (wl.block_table, wl.seq_lens, wl.qsl, wl.k_new, wl.v_new)]:
        slots = oracle.slot_mapping(bt, sl, qs, wl.block_size)
        oracle.write_kv(cache, wl.kv_dtype, wl.num_blocks, wl.block_size, wl.num_kv_heads,
                        wl.head_size, W.bits(k), W.bits(v), slots, ks, vs)
    return cache


# The oracle's attention runs on its OpenMP build over every host core by default: the same
# bits as the single-threaded build (pinned by tests/test_oracle_openmp.py), in less time.
ORACLE_THREADS = 0


def oracle_attention_all(wl: W.Workload, cache: np.ndarray, window: int = 0,
                         local_chunk: int = 0, threads=ORACLE_THREADS):
    ks = None if wl.k_scale is None else wl.k_scale.cpu().numpy()
    vs = None if wl.v_scale is None else wl.v_scale.cpu().numpy()
    return oracle.attention_paged(cache, wl.kv_dtype, wl.num_blocks, wl.block_size,
                                  wl.num_kv_heads, wl.head_size, W.bits(wl.q), wl.num_q_heads,
                                  wl.block_table, wl.seq_lens, wl.qsl, wl.scale, ks, vs,
                                  window=window, local_chunk=local_chunk, threads=threads)


def oracle_attention_rows(wl: W.Workload, tokens, heads, threads=ORACLE_THREADS):
    k_src, v_src = wl.kv_src()
    ks = None if wl.k_scale is None else wl.k_scale.cpu().numpy()
    vs = None if wl.v_scale is None else wl.v_scale.cpu().numpy()
    return oracle.attention_rows(W.bits(k_src), W.bits(v_src), wl.pos_rows, wl.pos_start,
                                 wl.kv_dtype, W.bits(wl.q), wl.seq_lens, wl.qsl, wl.scale,
                                 np.asarray(tokens, np.int32), np.asarray(heads, np.int32), ks, vs,
                                 threads=threads)


def assert_close(got: np.ndarray, want: np.ndarray, kv_dtype: int, what: str = "") -> dict:
    max_tol, mean_tol = TOL[kv_dtype]
    err = np.abs(got.astype(np.float64) - want)
    stats = {"max_abs": float(err.max()) if err.size else 0.0,
             "mean_abs": float(err.mean()) if err.size else 0.0}
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    assert stats["max_abs"] <= max_tol, f"{what}: max abs err {stats['max_abs']:.3g} > {max_tol}"
    assert stats["mean_abs"] <= mean_tol, f"{what}: mean abs err {stats['mean_abs']:.3g} > {mean_tol}"
    return stats


def sample_rows(wl: W.Workload, n: int, seed: int = 0):
    """(tokens, heads) to check: the first and last token of every request plus random ones,
    each with a random head and with the first and last head."""
    rng = np.random.default_rng(seed)
    toks = set()
    for r in range(wl.num_seqs):
        a, b = int(wl.qsl[r]), int(wl.qsl[r + 1])
        if b > a:
            toks.update({a, b - 1, (a + b) // 2})
    toks = sorted(toks)
    if len(toks) > n:
        toks = sorted(rng.choice(toks, n, replace=False).tolist())
    tokens, heads = [], []
    for t in toks:
        for h in {0, wl.num_q_heads - 1, int(rng.integers(wl.num_q_heads))}:
            tokens.append(t)
            heads.append(h)
    return np.array(tokens, np.int32), np.array(heads, np.int32)
