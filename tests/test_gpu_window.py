"""Sliding-window attention (a query at position p sees keys max(0, p - W + 1) .. p) against
the oracle: decode and chunked-prefill rows, bf16 and FP8 pools, head sizes 64 and 128, and
forced KV splits whose ranges start below, inside and past the window."""
import zlib

import numpy as np
import pytest

from gpu_common import GpuStep, assert_close, oracle_attention_all, oracle_cache
from paged_kv_cache_421_b200 import _binding as B
from paged_kv_cache_421_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _wl(ctx, ql, hq, hkv, d, seed, kv_dtype=W.BF16):
    need = sum(-(-c // 16) for c in ctx)
    return W.make_workload("win", ctx, ql, hq, hkv, d, 16, need + 8, seed, kv_dtype=kv_dtype)


CASES = {
    "decode_g4": ([1, 17, 300, 1000, 2500], [1, 1, 1, 1, 1], 32, 8, 128),
    "decode_g8_long": ([9000, 4100], [1, 1], 64, 8, 128),
    "spec_decode_qlen2": ([300, 700], [2, 2], 8, 2, 128),
    "chunks": ([600, 333, 2000], [600, 100, 300], 8, 2, 128),
    "mixed": ([900, 40, 1500, 77], [1, 40, 200, 1], 16, 4, 128),
    "chunk_d64": ([500, 130], [400, 64], 8, 2, 64),
}


@pytest.mark.parametrize("case", sorted(CASES))
@pytest.mark.parametrize("window", [1, 16, 17, 100, 513, 4096])
def test_window_matches_oracle(case, window):
    ctx, ql, hq, hkv, d = CASES[case]
    wl = _wl(ctx, ql, hq, hkv, d, seed=zlib.crc32(repr((case, window)).encode()) % 997)
    st = GpuStep(wl, run_attention=False)
    want, _ = oracle_attention_all(wl, oracle_cache(wl), window=window)
    for split in [0, 16, 64, 512]:
        got = st.attend(kv_split_tokens=split, sliding_window=window).cpu().numpy()
        assert_close(got, want, wl.kv_dtype, f"{case} W={window} split={split}")
    assert B.pa_device_error(reset=True) == 0


@pytest.mark.parametrize("window", [16, 1000])
def test_window_fp8_decode(window):
    wl = _wl([5000, 37, 900], [1, 1, 1], 32, 8, 128, seed=5, kv_dtype=W.FP8_E4M3)
    st = GpuStep(wl, run_attention=False)
    want, _ = oracle_attention_all(wl, oracle_cache(wl), window=window)
    for split in [0, 64]:
        got = st.attend(kv_split_tokens=split, sliding_window=window).cpu().numpy()
        assert_close(got, want, wl.kv_dtype, f"fp8 W={window} split={split}")


def test_window_longer_than_context_is_full_attention():
    wl = _wl([300, 1200], [1, 64], 8, 2, 128, seed=3)
    st = GpuStep(wl, run_attention=False)
    full = st.attend().cpu().numpy()
    assert np.array_equal(st.attend(sliding_window=1200).cpu().numpy(), full)
    assert np.array_equal(st.attend(sliding_window=1 << 20).cpu().numpy(), full)


# chunked local attention: a query at position p sees keys floor(p / C) * C .. p
@pytest.mark.parametrize("case", sorted(CASES))
@pytest.mark.parametrize("chunk", [1, 16, 100, 1000])
def test_local_chunk_matches_oracle(case, chunk):
    ctx, ql, hq, hkv, d = CASES[case]
    wl = _wl(ctx, ql, hq, hkv, d, seed=zlib.crc32(repr((case, chunk, "c")).encode()) % 997)
    st = GpuStep(wl, run_attention=False)
    want, _ = oracle_attention_all(wl, oracle_cache(wl), local_chunk=chunk)
    for split in [0, 64]:
        got = st.attend(kv_split_tokens=split, local_chunk=chunk).cpu().numpy()
        assert_close(got, want, wl.kv_dtype, f"{case} C={chunk} split={split}")
    assert B.pa_device_error(reset=True) == 0


def test_local_chunk_with_window_and_fp8():
    wl = _wl([5000, 37, 900], [1, 1, 1], 32, 8, 128, seed=7, kv_dtype=W.FP8_E4M3)
    st = GpuStep(wl, run_attention=False)
    for window, chunk in [(0, 512), (300, 1024), (2000, 256)]:
        want, _ = oracle_attention_all(wl, oracle_cache(wl), window=window, local_chunk=chunk)
        got = st.attend(sliding_window=window, local_chunk=chunk).cpu().numpy()
        assert_close(got, want, wl.kv_dtype, f"fp8 W={window} C={chunk}")
    wl = _wl([600, 1500], [600, 300], 8, 2, 128, seed=8)
    st = GpuStep(wl, run_attention=False)
    want, _ = oracle_attention_all(wl, oracle_cache(wl), window=200, local_chunk=256)
    for split in [0, 64]:
        got = st.attend(kv_split_tokens=split, sliding_window=200, local_chunk=256).cpu().numpy()
        assert_close(got, want, wl.kv_dtype, f"chunks W=200 C=256 split={split}")
