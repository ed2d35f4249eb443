"""Pure-Python brute-force twin of the oracle, for tiny inputs only.

TEST INFRASTRUCTURE ONLY (same rule as the rest of ``oracle/``).  It is a second,
independent statement of the same definitions, in plain Python loops with Python floats
(IEEE double), used to pin the C oracle: slot = block_table[p // bs] * bs + p % bs, the cache
write, and exact softmax attention with per-request, causal visibility ("Inside vLLM"
reading notes, core points 1-2; chunked prefill and FlashAttention outlines of the first
page).  It computes softmax as a plain ratio of exponentials of the raw scores (no max
subtraction), which is exact at the tiny magnitudes it is used on.
"""
from __future__ import annotations

import math
import struct


def bf16_bits_to_float(bits: int) -> float:
    return struct.unpack("<f", struct.pack("<I", (int(bits) & 0xFFFF) << 16))[0]


def slot_of(block_table_row, pos: int, block_size: int) -> int:
    return int(block_table_row[pos // block_size]) * block_size + pos % block_size


def slot_mapping(block_table, seq_lens, qsl, block_size):
    slots = []
    for r in range(len(seq_lens)):
        q_len = int(qsl[r + 1]) - int(qsl[r])
        for i in range(q_len):
            pos = int(seq_lens[r]) - q_len + i
            slots.append(slot_of(block_table[r], pos, block_size))
    return slots


def write_kv_bf16(cache: dict, k, v, slots, num_kv_heads, head_size, block_size):
    """cache: dict keyed by (block, kv, head, token_in_block, d) -> bf16 bits."""
    for t, slot in enumerate(slots):
        if slot < 0:
            continue
        b, o = divmod(int(slot), block_size)
        for h in range(num_kv_heads):
            for d in range(head_size):
                cache[(b, 0, h, o, d)] = int(k[t][h][d])
                cache[(b, 1, h, o, d)] = int(v[t][h][d])


def attention(cache_value, q, num_q_heads, num_kv_heads, head_size, block_table, seq_lens,
              qsl, block_size, scale, window=0, local_chunk=0):
    """cache_value(block, kv, head, tok, d) -> float.  q: nested [T][Hq][D] bf16 bits.
    window > 0: the query at position p sees only positions p - window + 1 .. p;
    local_chunk > 0: only positions from the start of its chunk, floor(p / C) * C .. p.
    Returns out as nested lists [T][Hq][D] of floats."""
    group = num_q_heads // num_kv_heads
    T = int(qsl[-1])
    out = [[[0.0] * head_size for _ in range(num_q_heads)] for _ in range(T)]
    for r in range(len(seq_lens)):
        q_len = int(qsl[r + 1]) - int(qsl[r])
        ctx = int(seq_lens[r])
        for i in range(q_len):
            t = int(qsl[r]) + i
            visible = ctx - q_len + i + 1
            start = max(0, visible - window) if window > 0 else 0
            if local_chunk > 0:
                start = max(start, (visible - 1) // local_chunk * local_chunk)
            for h in range(num_q_heads):
                g = h // group
                qv = [bf16_bits_to_float(q[t][h][d]) for d in range(head_size)]
                weights = [0.0] * start
                for p in range(start, visible):
                    b = int(block_table[r][p // block_size])
                    o = p % block_size
                    dot = sum(qv[d] * cache_value(b, 0, g, o, d) for d in range(head_size))
                    weights.append(math.exp(scale * dot))
                total = sum(weights)
                for d in range(head_size):
                    acc = 0.0
                    for p in range(start, visible):
                        b = int(block_table[r][p // block_size])
                        o = p % block_size
                        acc += weights[p] * cache_value(b, 1, g, o, d)
                    out[t][h][d] = acc / total
    return out
