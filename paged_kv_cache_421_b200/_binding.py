"""ctypes binding of libpa.so (include/pa.h).  Argument marshalling only.

Every function here has the name of the C entry point it calls and forwards device
pointers, sizes and the CUDA stream; all arithmetic of the hot path runs in the library's
kernels.  Torch tensors are accepted wherever the C call takes a device pointer (their
``data_ptr()`` is passed) and numpy arrays wherever it takes host memory.  A missing library
raises immediately: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpa.so")

PA_OK = 0
PA_ERR_INVALID_ARG = 1
PA_ERR_UNSUPPORTED = 2
PA_ERR_OOM = 3
PA_ERR_CUDA = 4
PA_ERR_WORKSPACE = 5
PA_ERR_METADATA = 6
PA_ERR_DEVICE = 7
PA_BF16 = 0
PA_FP8_E4M3 = 1

EXPORTED = [
    "pa_cache_bytes", "pa_alloc_cache", "pa_free_cache", "pa_cache_data", "pa_slot_mapping",
    "pa_write_kv", "pa_attention_workspace_bytes", "pa_attention", "pa_plan_attention",
    "pa_attention_ex", "pa_validate_block_table", "pa_device_error", "pa_status_string",
    "pa_last_cuda_error", "pa_attention_noalloc", "pa_allocate_slots", "pa_free_blocks",
    "pa_dcp_local_seq_lens", "pa_dcp_slot_mapping", "pa_merge_partials", "pa_validate_slots",
    "pa_common_prefix_blocks",
]
PA_NOALLOC_SCRATCH_BYTES = 64 << 20


class pa_plan(ctypes.Structure):
    _fields_ = [
        ("num_decode_seqs", ctypes.c_int),
        ("num_chunk_seqs", ctypes.c_int),
        ("decode_split_blocks", ctypes.c_int),
        ("decode_max_splits", ctypes.c_int),
        ("chunk_split_blocks", ctypes.c_int),
        ("chunk_max_splits", ctypes.c_int),
        ("chunk_max_qtiles", ctypes.c_int),
        ("decode_ctas", ctypes.c_int64),
        ("chunk_ctas", ctypes.c_int64),
        ("any_split", ctypes.c_int),
        ("workspace_needed", ctypes.c_size_t),
        ("reduce_rows_max", ctypes.c_int),
        ("prefix_splits", ctypes.c_int),
        ("prefix_split_blocks", ctypes.c_int),
        ("prefix_ctas", ctypes.c_int64),
        ("chunk_ctas_per_kv_head", ctypes.c_int),
    ]

    def as_dict(self) -> dict:
        return {name: getattr(self, name) for name, _ in self._fields_}


class pa_attention_opts(ctypes.Structure):
    _fields_ = [
        ("kv_split_tokens", ctypes.c_int),
        ("num_sms", ctypes.c_int),
        ("events", ctypes.c_void_p * 6),
        ("sliding_window", ctypes.c_int),
        ("local_chunk", ctypes.c_int),
        ("lse_out", ctypes.c_void_p),
        ("common_prefix_tokens", ctypes.c_int),
        ("test_skip_decode_load", ctypes.c_int),
        ("test_wait_limit_us", ctypes.c_int),
        ("kv_dtype", ctypes.c_int),
    ]


class PaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        name = _lib.pa_status_string(status).decode() if _lib else str(status)
        extra = ""
        if status == PA_ERR_CUDA and _lib:
            extra = f" (cudaError {_lib.pa_last_cuda_error()})"
        super().__init__(f"{where}: {name}{extra}")


_lib = None


def load() -> ctypes.CDLL:
    """Load libpa.so (built in-tree by ``python -m paged_kv_cache_421_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m paged_kv_cache_421_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, Z, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
    sig = {
        "pa_cache_bytes": (Z, [I, I, I, I, I]),
        "pa_alloc_cache": (I, [I, I, I, I, I, P, P, P, ctypes.POINTER(P)]),
        "pa_free_cache": (I, [P]),
        "pa_cache_data": (P, [P]),
        "pa_slot_mapping": (I, [P, I, P, P, I, I, I, P, P]),
        "pa_write_kv": (I, [P, P, P, P, I, P]),
        "pa_allocate_slots": (I, [P, I, P, P, I, I, P, I, P, P, P]),
        "pa_free_blocks": (I, [P, I, P, I, P, P]),
        "pa_attention_workspace_bytes": (Z, [I, I, I, I]),
        "pa_attention": (I, [P, P, I, P, I, P, P, P, P, I, I, F, P, P, Z, P]),
        "pa_plan_attention": (I, [P, P, I, I, I, I, I, I, I, I, Z,
                                  ctypes.POINTER(pa_attention_opts), ctypes.POINTER(pa_plan)]),
        "pa_attention_ex": (I, [P, P, I, P, I, P, P, P, P, I, I, F, P, P, Z,
                                ctypes.POINTER(pa_attention_opts), P]),
        "pa_validate_block_table": (I, [P, P, I, P, I, ctypes.POINTER(I), P]),
        "pa_validate_slots": (I, [P, P, I, ctypes.POINTER(I), ctypes.POINTER(I), P]),
        "pa_common_prefix_blocks": (I, [P, I, P, P, I, I, ctypes.POINTER(I)]),
        "pa_device_error": (I, [ctypes.POINTER(I), I]),
        "pa_status_string": (ctypes.c_char_p, [I]),
        "pa_last_cuda_error": (I, []),
        "pa_attention_noalloc": (I, [P, P, I, P, I, P, P, P, P, I, I, F, P, P]),
        "pa_dcp_local_seq_lens": (I, [P, I, I, I, I, P]),
        "pa_dcp_slot_mapping": (I, [P, I, P, P, I, I, I, I, I, P, P]),
        "pa_merge_partials": (I, [P, P, I, ctypes.c_int64, I, P, P, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _ptr(x) -> Optional[int]:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, "data_ptr"):
        return x.data_ptr()
    if isinstance(x, np.ndarray):
        return x.ctypes.data
    raise TypeError(f"cannot pass {type(x)} as a pointer")


def _host_i32(a) -> np.ndarray:
    if hasattr(a, "cpu"):
        a = a.cpu().numpy()
    return np.ascontiguousarray(a, dtype=np.int32)


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if hasattr(stream, "cuda_stream"):
        return stream.cuda_stream
    return int(stream)


def _check(status: int, where: str) -> None:
    if status != PA_OK:
        raise PaError(status, where)


# ------------------------------------------------------------------ thin wrappers
def pa_cache_bytes(num_blocks, block_size, num_kv_heads, head_size, kv_dtype) -> int:
    return int(load().pa_cache_bytes(num_blocks, block_size, num_kv_heads, head_size, kv_dtype))


def pa_alloc_cache(num_blocks, block_size, num_kv_heads, head_size, kv_dtype,
                   k_scale=None, v_scale=None, external_buf=None) -> int:
    h = ctypes.c_void_p()
    _check(load().pa_alloc_cache(num_blocks, block_size, num_kv_heads, head_size, kv_dtype,
                                 _ptr(k_scale), _ptr(v_scale), _ptr(external_buf),
                                 ctypes.byref(h)), "pa_alloc_cache")
    return h.value


def pa_free_cache(handle) -> None:
    _check(load().pa_free_cache(handle), "pa_free_cache")


def pa_cache_data(handle) -> int:
    return load().pa_cache_data(handle)


def pa_slot_mapping(block_table, max_blocks_per_seq, seq_lens, query_start_loc, num_seqs,
                    num_tokens, block_size, slot_mapping, stream=None) -> None:
    _check(load().pa_slot_mapping(_ptr(block_table), max_blocks_per_seq, _ptr(seq_lens),
                                  _ptr(query_start_loc), num_seqs, num_tokens, block_size,
                                  _ptr(slot_mapping), _stream(stream)), "pa_slot_mapping")


def pa_allocate_slots(block_table, max_blocks_per_seq, num_computed, num_new, num_seqs,
                      block_size, free_queue, queue_capacity, queue_state, num_allocated,
                      stream=None) -> None:
    _check(load().pa_allocate_slots(_ptr(block_table), max_blocks_per_seq, _ptr(num_computed),
                                    _ptr(num_new), num_seqs, block_size, _ptr(free_queue),
                                    queue_capacity, _ptr(queue_state), _ptr(num_allocated),
                                    _stream(stream)), "pa_allocate_slots")


def pa_free_blocks(block_ids, num_ids, free_queue, queue_capacity, queue_state,
                   stream=None) -> None:
    _check(load().pa_free_blocks(_ptr(block_ids), num_ids, _ptr(free_queue), queue_capacity,
                                 _ptr(queue_state), _stream(stream)), "pa_free_blocks")


def pa_write_kv(handle, k, v, slot_mapping, num_tokens, stream=None) -> None:
    _check(load().pa_write_kv(handle, _ptr(k), _ptr(v), _ptr(slot_mapping), num_tokens,
                              _stream(stream)), "pa_write_kv")


def pa_attention_workspace_bytes(num_tokens, num_q_heads, head_size, max_splits) -> int:
    return int(load().pa_attention_workspace_bytes(num_tokens, num_q_heads, head_size,
                                                   max_splits))


def pa_plan_attention(seq_lens_host, query_start_loc_host, num_q_heads, num_kv_heads,
                      head_size, max_blocks_per_seq, num_sms, workspace_bytes,
                      kv_split_tokens=0, block_size=16, sliding_window=0,
                      local_chunk=0, with_lse=False, common_prefix_tokens=0,
                      kv_dtype=0) -> dict:
    """with_lse: plan as a call that exports LSEs (which admits empty decode shares); the
    planner only tests the pointer for NULL, so a dummy non-NULL value stands in.  kv_dtype:
    the cache's element type (PA_BF16 / PA_FP8_E4M3)."""
    sl = _host_i32(seq_lens_host)
    qs = _host_i32(query_start_loc_host)
    opts = pa_attention_opts()
    opts.kv_split_tokens = kv_split_tokens
    opts.sliding_window = sliding_window
    opts.local_chunk = local_chunk
    opts.lse_out = 16 if with_lse else None
    opts.common_prefix_tokens = common_prefix_tokens
    opts.kv_dtype = kv_dtype
    plan = pa_plan()
    _check(load().pa_plan_attention(sl.ctypes.data, qs.ctypes.data, sl.size, int(qs[-1]),
                                    num_q_heads, num_kv_heads, head_size, block_size,
                                    max_blocks_per_seq, num_sms, workspace_bytes,
                                    ctypes.byref(opts), ctypes.byref(plan)), "pa_plan_attention")
    return plan.as_dict()


def pa_attention(handle, q, num_q_heads, block_table, max_blocks_per_seq, seq_lens,
                 query_start_loc, seq_lens_host, query_start_loc_host, num_seqs, num_tokens,
                 scale, out, workspace=None, workspace_bytes=0, stream=None) -> None:
    sl = _host_i32(seq_lens_host)
    qs = _host_i32(query_start_loc_host)
    _check(load().pa_attention(handle, _ptr(q), num_q_heads, _ptr(block_table),
                               max_blocks_per_seq, _ptr(seq_lens), _ptr(query_start_loc),
                               sl.ctypes.data, qs.ctypes.data, num_seqs, num_tokens,
                               float(scale), _ptr(out), _ptr(workspace), workspace_bytes,
                               _stream(stream)), "pa_attention")


def pa_attention_ex(handle, q, num_q_heads, block_table, max_blocks_per_seq, seq_lens,
                    query_start_loc, seq_lens_host, query_start_loc_host, num_seqs, num_tokens,
                    scale, out, workspace=None, workspace_bytes=0, kv_split_tokens=0,
                    num_sms=0, events=None, sliding_window=0, local_chunk=0, lse_out=None,
                    common_prefix_tokens=0, test_skip_decode_load=0, test_wait_limit_us=0,
                    stream=None) -> None:
    sl = _host_i32(seq_lens_host)
    qs = _host_i32(query_start_loc_host)
    opts = pa_attention_opts()
    opts.kv_split_tokens = kv_split_tokens
    opts.num_sms = num_sms
    opts.sliding_window = sliding_window
    opts.local_chunk = local_chunk
    opts.lse_out = _ptr(lse_out)
    opts.common_prefix_tokens = common_prefix_tokens
    opts.test_skip_decode_load = test_skip_decode_load
    opts.test_wait_limit_us = test_wait_limit_us
    for i, ev in enumerate(events or []):
        if ev is not None:
            opts.events[i] = ev.cuda_event if hasattr(ev, "cuda_event") else int(ev)
    _check(load().pa_attention_ex(handle, _ptr(q), num_q_heads, _ptr(block_table),
                                  max_blocks_per_seq, _ptr(seq_lens), _ptr(query_start_loc),
                                  sl.ctypes.data, qs.ctypes.data, num_seqs, num_tokens,
                                  float(scale), _ptr(out), _ptr(workspace), workspace_bytes,
                                  ctypes.byref(opts), _stream(stream)), "pa_attention_ex")


def pa_attention_noalloc(handle, q, num_q_heads, block_table, max_blocks_per_seq, seq_lens,
                         query_start_loc, seq_lens_host, query_start_loc_host, num_seqs,
                         num_tokens, scale, out, stream=None) -> None:
    """pa_attention for callers that cannot allocate device memory: the split-KV partials go
    to the library's fixed static scratch (PA_NOALLOC_SCRATCH_BYTES) instead of a workspace."""
    sl = _host_i32(seq_lens_host)
    qs = _host_i32(query_start_loc_host)
    _check(load().pa_attention_noalloc(handle, _ptr(q), num_q_heads, _ptr(block_table),
                                       max_blocks_per_seq, _ptr(seq_lens), _ptr(query_start_loc),
                                       sl.ctypes.data, qs.ctypes.data, num_seqs, num_tokens,
                                       float(scale), _ptr(out), _stream(stream)),
           "pa_attention_noalloc")


def pa_validate_block_table(handle, block_table, max_blocks_per_seq, seq_lens, num_seqs,
                            stream=None) -> int:
    bad = ctypes.c_int(0)
    _check(load().pa_validate_block_table(handle, _ptr(block_table), max_blocks_per_seq,
                                          _ptr(seq_lens), num_seqs, ctypes.byref(bad),
                                          _stream(stream)), "pa_validate_block_table")
    return bad.value


def pa_common_prefix_blocks(block_table_host, seq_lens_host, query_start_loc_host,
                            block_size=16) -> int:
    """Leading block-table entries that every request with queries shares, each request's
    queries seeing all of them (host arrays)."""
    bt = np.ascontiguousarray(block_table_host, dtype=np.int32)
    sl = _host_i32(seq_lens_host)
    qs = _host_i32(query_start_loc_host)
    n = ctypes.c_int(0)
    _check(load().pa_common_prefix_blocks(bt.ctypes.data, bt.shape[1], sl.ctypes.data,
                                          qs.ctypes.data, sl.size, block_size, ctypes.byref(n)),
           "pa_common_prefix_blocks")
    return n.value


def pa_validate_slots(handle, slot_mapping, num_tokens, stream=None) -> tuple:
    """(tokens whose slot lies outside the pool, tokens whose slot another token of the call
    also holds) for one call's slot mapping; negative slots are skips."""
    out_of_pool, dups = ctypes.c_int(0), ctypes.c_int(0)
    _check(load().pa_validate_slots(handle, _ptr(slot_mapping), num_tokens,
                                    ctypes.byref(out_of_pool), ctypes.byref(dups),
                                    _stream(stream)), "pa_validate_slots")
    return out_of_pool.value, dups.value


def pa_device_error(reset: bool = True) -> int:
    code = ctypes.c_int(0)
    _check(load().pa_device_error(ctypes.byref(code), int(reset)), "pa_device_error")
    return code.value


def pa_status_string(status: int) -> str:
    return load().pa_status_string(status).decode()


def pa_dcp_local_seq_lens(seq_lens_host, block_size, rank, world) -> np.ndarray:
    """Keys of each request that rank `rank` of a `world`-rank DCP group holds (host)."""
    sl = _host_i32(seq_lens_host)
    out = np.zeros(sl.size, np.int32)
    _check(load().pa_dcp_local_seq_lens(sl.ctypes.data, sl.size, block_size, rank, world,
                                        out.ctypes.data), "pa_dcp_local_seq_lens")
    return out


def pa_dcp_slot_mapping(block_table, max_blocks_per_seq, seq_lens, query_start_loc, num_seqs,
                        num_tokens, block_size, rank, world, slot_mapping, stream=None) -> None:
    _check(load().pa_dcp_slot_mapping(_ptr(block_table), max_blocks_per_seq, _ptr(seq_lens),
                                      _ptr(query_start_loc), num_seqs, num_tokens, block_size,
                                      rank, world, _ptr(slot_mapping), _stream(stream)),
           "pa_dcp_slot_mapping")


def pa_merge_partials(part_out, part_lse, num_parts, num_rows, head_size, out, lse_out=None,
                      stream=None) -> None:
    _check(load().pa_merge_partials(_ptr(part_out), _ptr(part_lse), num_parts, num_rows,
                                    head_size, _ptr(out), _ptr(lse_out), _stream(stream)),
           "pa_merge_partials")
