"""Paged KV cache oracle: plain fp64 CPU reference.

TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the benchmark's
CPU-baseline leg may import this package.  The product (``paged_kv_cache_421_b200``) never
imports, links or executes anything here, and nothing here imports the product: the two
share only the seeded input generator, which holds none of the method's arithmetic.

The arithmetic lives in ``pa_oracle.c`` (plain C, fp64), compiled with gcc by
:func:`build`; this module is argument marshalling over numpy arrays.  ``brute.py`` is a
second, pure-Python restatement used to pin this one on tiny inputs.

Sources (page title and section):
  * slot formula and block table lookup: "vLLM: from KV Cache to high-throughput serving",
    article 3 outline; "vLLM architecture overview", section 2;
  * per-block bytes and blocks needed (ceil(17/16) = 2): "Inside vLLM" reading notes,
    core point 1;
  * flattened super-sequence with per-request masking: "Inside vLLM" notes, core point 2;
  * causal chunks: chunked prefill, article 5 outline of the first page;
  * exact attention, LSE: FlashAttention, article 7 outline of the first page;
  * FP8 E4M3: named in article 6 outline; the codec follows the OCP 8-bit floating point
    specification.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pa_oracle.c")
_OUT_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_OUT_DIR, "liboracle.so")
# the same source built with OpenMP: independent (request, kv head) units and selected rows
# run on several threads, each with the arithmetic of the plain build
_OMP_LIB_PATH = os.path.join(_OUT_DIR, "liboracle_omp.so")

BF16 = 0
FP8_E4M3 = 1

_lib = None
_omp_lib = None

_CFLAGS = ["-O2", "-std=c99", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
           "-Wall", "-Wextra"]


def _compile(path: str, extra: list, force: bool) -> str:
    if (not force and os.path.exists(path)
            and os.path.getmtime(path) >= os.path.getmtime(_SRC)):
        return path
    tmp = path + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", *_CFLAGS, *extra, "-o", tmp, _SRC, "-lm"])
    os.replace(tmp, path)
    return path


def build(force: bool = False) -> str:
    """Compile pa_oracle.c into a shared library (gcc, strict IEEE: no fast-math, no FMA
    contraction, so the fp32 divide of the FP8 path is a correctly rounded divide), and the
    same source once more with OpenMP (liboracle_omp.so)."""
    os.makedirs(_OUT_DIR, exist_ok=True)
    _compile(_OMP_LIB_PATH, ["-fopenmp"], force)
    return _compile(_LIB_PATH, ["-Wno-unknown-pragmas"], force)


def _declare(lib):
    P = ctypes.c_void_p
    i32, i64, f64, u8 = ctypes.c_int, ctypes.c_int64, ctypes.c_double, ctypes.c_uint8
    lib.oracle_set_threads.restype = i32
    lib.oracle_set_threads.argtypes = [i32]
    lib.oracle_cache_elems.restype = i64
    lib.oracle_cache_elems.argtypes = [i32, i32, i32, i32]
    lib.oracle_block_bytes.restype = i64
    lib.oracle_block_bytes.argtypes = [i32, i32, i32, i32]
    lib.oracle_blocks_needed.restype = i64
    lib.oracle_blocks_needed.argtypes = [i64, i32]
    lib.oracle_e4m3_decode.restype = f64
    lib.oracle_e4m3_decode.argtypes = [u8]
    lib.oracle_e4m3_encode.restype = u8
    lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
    lib.oracle_e4m3_encode_array.restype = None
    lib.oracle_e4m3_encode_array.argtypes = [P, i64, P]
    lib.oracle_e4m3_decode_array.restype = None
    lib.oracle_e4m3_decode_array.argtypes = [P, i64, P]
    lib.oracle_slot_mapping.restype = i32
    lib.oracle_slot_mapping.argtypes = [P, i32, P, P, i32, i32, P]
    lib.oracle_allocate_slots.restype = i32
    lib.oracle_allocate_slots.argtypes = [P, i32, P, P, i32, i32, P, i32, P, P]
    lib.oracle_free_blocks.restype = i32
    lib.oracle_free_blocks.argtypes = [P, i32, P, i32, P]
    lib.oracle_write_kv_bf16.restype = None
    lib.oracle_write_kv_bf16.argtypes = [P, i32, i32, i32, i32, P, P, P, i32]
    lib.oracle_write_kv_fp8.restype = None
    lib.oracle_write_kv_fp8.argtypes = [P, i32, i32, i32, i32, P, P, P, P, P, i32]
    lib.oracle_attention_paged.restype = i32
    lib.oracle_attention_paged.argtypes = [P, i32, i32, i32, i32, i32, P, P, P, i32, P, i32,
                                           P, P, i32, f64, i32, i32, P, P]
    lib.oracle_dcp_local_len.restype = i32
    lib.oracle_dcp_local_len.argtypes = [i32, i32, i32, i32]
    lib.oracle_dcp_slot_mapping.restype = i32
    lib.oracle_dcp_slot_mapping.argtypes = [P, i32, P, P, i32, i32, i32, i32, P]
    lib.oracle_merge_partials.restype = None
    lib.oracle_merge_partials.argtypes = [P, P, i32, i64, i32, P, P]
    lib.oracle_attention_rows.restype = i32
    lib.oracle_attention_rows.argtypes = [P, P, i32, i32, P, P, i32, P, P, P, i32, P, P, i32,
                                          f64, i32, i32, P, P, i32, P, P]
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = _declare(ctypes.CDLL(build()))
    return _lib


def _load_omp():
    global _omp_lib
    if _omp_lib is None:
        build()
        _omp_lib = _declare(ctypes.CDLL(_OMP_LIB_PATH))
    return _omp_lib


def host_cores() -> int:
    """Host cores this process may run on."""
    return len(os.sched_getaffinity(0))


def _attention_lib(threads):
    """The plain (single-threaded) oracle for threads None or 1, else the OpenMP build set to
    that many threads (0: every host core this process may use)."""
    if threads is None or threads == 1:
        return _load()
    lib = _load_omp()
    lib.oracle_set_threads(host_cores() if threads == 0 else int(threads))
    return lib


def threads_in_use(threads) -> int:
    """Threads an attention call with this `threads` argument runs on."""
    return int(_attention_lib(threads).oracle_set_threads(0))


def _c(a: np.ndarray, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a) -> ctypes.c_void_p:
    return ctypes.c_void_p(0) if a is None else ctypes.c_void_p(a.ctypes.data)


class OracleError(RuntimeError):
    pass


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise OracleError(f"{what}: status {rc}")


# ---------------------------------------------------------------- sizing formulas
def block_bytes(block_size: int, num_kv_heads: int, head_size: int, dtype_bytes: int) -> int:
    """2 * block_size * num_kv_heads * head_size * dtype_bytes ("Inside vLLM", point 1)."""
    return int(_load().oracle_block_bytes(block_size, num_kv_heads, head_size, dtype_bytes))


def blocks_needed(n_tokens: int, block_size: int) -> int:
    """ceil(n_tokens / block_size) ("Inside vLLM", point 1: 17 new tokens -> 2 blocks)."""
    return int(_load().oracle_blocks_needed(n_tokens, block_size))


def cache_elems(num_blocks: int, block_size: int, num_kv_heads: int, head_size: int) -> int:
    return int(_load().oracle_cache_elems(num_blocks, block_size, num_kv_heads, head_size))


# ---------------------------------------------------------------- FP8 E4M3 codec
def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    c = _c(codes, np.uint8)
    out = np.empty(c.shape, np.float64)
    _load().oracle_e4m3_decode_array(_p(c), c.size, _p(out))
    return out


def e4m3_encode(y: np.ndarray) -> np.ndarray:
    """Encode fp32 values (round to nearest even, saturate to +-448, NaN stays NaN)."""
    a = _c(y, np.float32)
    out = np.empty(a.shape, np.uint8)
    _load().oracle_e4m3_encode_array(_p(a), a.size, _p(out))
    return out


# ---------------------------------------------------------------- slot mapping / write
def slot_mapping(block_table: np.ndarray, seq_lens: np.ndarray, qsl: np.ndarray,
                 block_size: int) -> np.ndarray:
    bt = _c(block_table, np.int32)
    sl = _c(seq_lens, np.int32)
    q = _c(qsl, np.int32)
    out = np.full(int(q[-1]), -1, np.int32)
    _check(_load().oracle_slot_mapping(_p(bt), bt.shape[1], _p(sl), _p(q), sl.size,
                                       block_size, _p(out)), "oracle_slot_mapping")
    return out


def allocate_slots(block_table: np.ndarray, num_computed, num_new, block_size: int,
                   queue: np.ndarray, state: np.ndarray) -> np.ndarray:
    """In place on block_table (int32 [B][max_blocks]) and state (int32 [head, count]); returns
    num_allocated (int32 [B], -1 for a request not served).  See oracle_allocate_slots."""
    assert block_table.dtype == np.int32 and block_table.flags.c_contiguous
    assert state.dtype == np.int32 and state.size == 2
    c = _c(np.asarray(num_computed), np.int32)
    n = _c(np.asarray(num_new), np.int32)
    q = _c(queue, np.int32)
    out = np.zeros(c.size, np.int32)
    _check(_load().oracle_allocate_slots(_p(block_table), block_table.shape[1], _p(c), _p(n),
                                         c.size, block_size, _p(q), q.size, _p(state), _p(out)),
           "oracle_allocate_slots")
    return out


def free_blocks(ids, queue: np.ndarray, state: np.ndarray) -> None:
    """In place on queue (int32 ring) and state (int32 [head, count])."""
    assert queue.dtype == np.int32 and state.dtype == np.int32
    i = _c(np.asarray(ids), np.int32)
    _check(_load().oracle_free_blocks(_p(i), i.size, _p(queue), queue.size, _p(state)),
           "oracle_free_blocks")


def write_kv(cache: np.ndarray, kv_dtype: int, num_blocks: int, block_size: int,
             num_kv_heads: int, head_size: int, k_bits: np.ndarray, v_bits: np.ndarray,
             slots: np.ndarray, k_scale=None, v_scale=None) -> None:
    """In-place write.  cache: uint16 (bf16 bits) or uint8 (E4M3 codes), flat, in the
    [block][K|V][kv head][token][dim] layout; k_bits/v_bits: uint16 bf16 bits [T][Hkv][D]."""
    assert cache.flags.c_contiguous
    k = _c(k_bits, np.uint16)
    v = _c(v_bits, np.uint16)
    s = _c(slots, np.int32)
    lib = _load()
    if kv_dtype == BF16:
        assert cache.dtype == np.uint16
        lib.oracle_write_kv_bf16(_p(cache), num_blocks, block_size, num_kv_heads, head_size,
                                 _p(k), _p(v), _p(s), s.size)
    else:
        assert cache.dtype == np.uint8
        ks = _c(k_scale, np.float32)
        vs = _c(v_scale, np.float32)
        lib.oracle_write_kv_fp8(_p(cache), num_blocks, block_size, num_kv_heads, head_size,
                                _p(k), _p(v), _p(ks), _p(vs), _p(s), s.size)


# ---------------------------------------------------------------- attention
def attention_paged(cache: np.ndarray, kv_dtype: int, num_blocks: int, block_size: int,
                    num_kv_heads: int, head_size: int, q_bits: np.ndarray, num_q_heads: int,
                    block_table: np.ndarray, seq_lens: np.ndarray, qsl: np.ndarray,
                    scale: float, k_scale=None, v_scale=None, window: int = 0,
                    local_chunk: int = 0, threads=None):
    """Exact attention over the paged cache.  Returns (out [T][Hq][D], lse [T][Hq]) fp64.
    window > 0: a query at position p sees keys max(0, p - window + 1) .. p;
    local_chunk > 0: only keys floor(p / local_chunk) * local_chunk .. p.
    threads: None / 1 single-threaded; n > 1 (0 = all host cores) the OpenMP build, which
    returns the same bits."""
    q = _c(q_bits, np.uint16)
    bt = _c(block_table, np.int32)
    sl = _c(seq_lens, np.int32)
    qs = _c(qsl, np.int32)
    T = int(qs[-1])
    out = np.zeros((T, num_q_heads, head_size), np.float64)
    lse = np.zeros((T, num_q_heads), np.float64)
    ks = None if k_scale is None else _c(k_scale, np.float32)
    vs = None if v_scale is None else _c(v_scale, np.float32)
    _check(_attention_lib(threads).oracle_attention_paged(
        _p(cache), kv_dtype, num_blocks, block_size, num_kv_heads, head_size, _p(ks), _p(vs),
        _p(q), num_q_heads, _p(bt), bt.shape[1], _p(sl), _p(qs), sl.size, float(scale),
        int(window), int(local_chunk), _p(out), _p(lse)), "oracle_attention_paged")
    return out, lse


def attention_rows(k_src: np.ndarray, v_src: np.ndarray, pos_rows: np.ndarray,
                   pos_start: np.ndarray, kv_dtype: int, q_bits: np.ndarray,
                   seq_lens: np.ndarray, qsl: np.ndarray, scale: float,
                   sel_tokens: np.ndarray, sel_heads: np.ndarray, k_scale=None, v_scale=None,
                   window: int = 0, local_chunk: int = 0, threads=None):
    """Unpaged exact attention for selected (token, q head) rows.

    k_src, v_src: uint16 bf16 bits [rows][Hkv][D]; request r's position p reads source row
    pos_rows[pos_start[r] + p].  Returns (out [nsel][D], lse [nsel]) in fp64.
    threads: as for attention_paged."""
    k = _c(k_src, np.uint16)
    v = _c(v_src, np.uint16)
    num_kv_heads, head_size = k.shape[1], k.shape[2]
    q = _c(q_bits, np.uint16)
    num_q_heads = q.shape[1]
    pr = _c(pos_rows, np.int64)
    ps = _c(pos_start, np.int64)
    sl = _c(seq_lens, np.int32)
    qs = _c(qsl, np.int32)
    st = _c(sel_tokens, np.int32)
    sh = _c(sel_heads, np.int32)
    out = np.zeros((st.size, head_size), np.float64)
    lse = np.zeros(st.size, np.float64)
    ks = None if k_scale is None else _c(k_scale, np.float32)
    vs = None if v_scale is None else _c(v_scale, np.float32)
    _check(_attention_lib(threads).oracle_attention_rows(
        _p(k), _p(v), num_kv_heads, head_size, _p(pr), _p(ps), kv_dtype, _p(ks), _p(vs),
        _p(q), num_q_heads, _p(sl), _p(qs), sl.size, float(scale), int(window),
        int(local_chunk), _p(st), _p(sh),
        st.size, _p(out), _p(lse)), "oracle_attention_rows")
    return out, lse


# ---------------------------------------------------------------- context parallelism
def dcp_local_len(seq_lens, block_size: int, rank: int, world: int) -> np.ndarray:
    """Keys rank `rank` of `world` holds of each request: block j of a request lives on rank
    j mod world (see oracle_dcp_local_len)."""
    lib = _load()
    return np.array([lib.oracle_dcp_local_len(int(c), block_size, rank, world)
                     for c in np.asarray(seq_lens).ravel()], np.int32)


def dcp_slot_mapping(local_table: np.ndarray, seq_lens: np.ndarray, qsl: np.ndarray,
                     block_size: int, rank: int, world: int) -> np.ndarray:
    """Slots of the step's new tokens on one rank: -1 where another rank owns the token's
    block (see oracle_dcp_slot_mapping).  seq_lens are total request lengths."""
    bt = _c(local_table, np.int32)
    sl = _c(seq_lens, np.int32)
    q = _c(qsl, np.int32)
    out = np.full(int(q[-1]), -2, np.int32)
    _check(_load().oracle_dcp_slot_mapping(_p(bt), bt.shape[1], _p(sl), _p(q), sl.size,
                                           block_size, rank, world, _p(out)),
           "oracle_dcp_slot_mapping")
    return out


def merge_partials(part_o: np.ndarray, part_lse: np.ndarray):
    """LSE merge of attention over disjoint key sets.  part_o [P][..., D], part_lse [P][...]
    (natural log); returns (out [..., D], lse [...]) in fp64."""
    o = _c(part_o, np.float64)
    l = _c(part_lse, np.float64)
    P, D = o.shape[0], o.shape[-1]
    rows = l[0].size
    assert o.size == P * rows * D and l.size == P * rows
    out = np.zeros(o.shape[1:], np.float64)
    lse = np.zeros(l.shape[1:], np.float64)
    _load().oracle_merge_partials(_p(o), _p(l), P, rows, D, _p(out), _p(lse))
    return out, lse
