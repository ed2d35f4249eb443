"""Torch-tensor conveniences over the C ABI (allocation of outputs and workspace, stream
selection).  Every computation happens inside libpa.so; these helpers only size and
allocate tensors and forward pointers."""
from __future__ import annotations

from typing import Optional

import numpy as np
import torch

from . import _binding as B


class PagedKVCache:
    """One layer's paged K/V pool: [num_blocks][K|V][num_kv_heads][block_size][head_size].

    The device memory is a torch tensor handed to ``pa_alloc_cache`` as its external buffer,
    so torch's allocator owns it; the handle only adds the library's descriptors."""

    def __init__(self, num_blocks: int, num_kv_heads: int, head_size: int,
                 kv_dtype: int = B.PA_BF16, block_size: int = 16,
                 k_scale: Optional[torch.Tensor] = None, v_scale: Optional[torch.Tensor] = None,
                 device="cuda"):
        self.num_blocks, self.num_kv_heads, self.head_size = num_blocks, num_kv_heads, head_size
        self.block_size, self.kv_dtype = block_size, kv_dtype
        nbytes = B.pa_cache_bytes(num_blocks, block_size, num_kv_heads, head_size, kv_dtype)
        if nbytes == 0:
            raise B.PaError(B.PA_ERR_INVALID_ARG, "pa_cache_bytes")
        self.buffer = torch.empty(nbytes, dtype=torch.uint8, device=device)
        self.k_scale = None if k_scale is None else k_scale.to(device, torch.float32).contiguous()
        self.v_scale = None if v_scale is None else v_scale.to(device, torch.float32).contiguous()
        self.handle = B.pa_alloc_cache(num_blocks, block_size, num_kv_heads, head_size, kv_dtype,
                                       self.k_scale, self.v_scale, self.buffer)

    @property
    def nbytes(self) -> int:
        return self.buffer.numel()

    def view(self) -> torch.Tensor:
        """The pool as [num_blocks, 2, num_kv_heads, block_size, head_size] (bf16 or uint8).
        For an FP8 pool the V tiles ([:, 1]) are dim-major: read them as
        ``view()[:, 1].reshape(num_blocks, num_kv_heads, head_size, block_size)``."""
        dt = torch.bfloat16 if self.kv_dtype == B.PA_BF16 else torch.uint8
        return self.buffer.view(dt).view(self.num_blocks, 2, self.num_kv_heads, self.block_size,
                                         self.head_size)

    def close(self) -> None:
        if getattr(self, "handle", None):
            B.pa_free_cache(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def slot_mapping(block_table: torch.Tensor, seq_lens: torch.Tensor, qsl: torch.Tensor,
                 num_tokens: int, block_size: int = 16, out: Optional[torch.Tensor] = None,
                 stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty(num_tokens, dtype=torch.int32, device=block_table.device)
    B.pa_slot_mapping(block_table, block_table.shape[1], seq_lens, qsl, seq_lens.numel(),
                      num_tokens, block_size, out, stream)
    return out


class BlockQueue:
    """The free-block queue on the device: a ring of block ids plus (head, count)."""

    def __init__(self, block_ids: torch.Tensor, capacity: Optional[int] = None):
        n = block_ids.numel()
        cap = n if capacity is None else capacity
        assert cap >= n > 0
        self.queue = torch.zeros(cap, dtype=torch.int32, device=block_ids.device)
        self.queue[:n] = block_ids.to(torch.int32)
        self.state = torch.tensor([0, n], dtype=torch.int32, device=block_ids.device)

    @property
    def capacity(self) -> int:
        return self.queue.numel()


def allocate_slots(block_table: torch.Tensor, num_computed: torch.Tensor, num_new: torch.Tensor,
                   queue: BlockQueue, block_size: int = 16, out: Optional[torch.Tensor] = None,
                   stream=None) -> torch.Tensor:
    """Append each request's new blocks to its block-table row (in place); returns the blocks
    taken per request, -1 where the request was not served."""
    if out is None:
        out = torch.empty(num_computed.numel(), dtype=torch.int32, device=block_table.device)
    B.pa_allocate_slots(block_table, block_table.shape[1], num_computed, num_new,
                        num_computed.numel(), block_size, queue.queue, queue.capacity, queue.state,
                        out, stream)
    return out


def free_blocks(block_ids: torch.Tensor, queue: BlockQueue, stream=None) -> None:
    B.pa_free_blocks(block_ids, block_ids.numel(), queue.queue, queue.capacity, queue.state,
                     stream)


def write_kv(cache: PagedKVCache, k: torch.Tensor, v: torch.Tensor, slots: torch.Tensor,
             stream=None) -> None:
    assert k.is_contiguous() and v.is_contiguous() and k.dtype == torch.bfloat16
    B.pa_write_kv(cache.handle, k, v, slots, slots.numel(), stream)


def workspace_bytes_for(cache: PagedKVCache, seq_lens_host, qsl_host, num_q_heads: int,
                        max_blocks_per_seq: int, kv_split_tokens: int = 0,
                        num_sms: Optional[int] = None, sliding_window: int = 0,
                        local_chunk: int = 0, with_lse: bool = False,
                        common_prefix_tokens: int = 0) -> int:
    if num_sms is None:
        num_sms = torch.cuda.get_device_properties(cache.buffer.device).multi_processor_count
    qs = np.asarray(qsl_host)
    T = int(qs[-1])
    unlimited = B.pa_attention_workspace_bytes(max(T, 1), num_q_heads, cache.head_size, 1 << 16)
    plan = B.pa_plan_attention(seq_lens_host, qsl_host, num_q_heads, cache.num_kv_heads,
                               cache.head_size, max_blocks_per_seq, num_sms, unlimited,
                               kv_split_tokens=kv_split_tokens, block_size=cache.block_size,
                               sliding_window=sliding_window, local_chunk=local_chunk,
                               with_lse=with_lse, common_prefix_tokens=common_prefix_tokens,
                               kv_dtype=cache.kv_dtype)
    return int(plan["workspace_needed"])


def attention(cache: PagedKVCache, q: torch.Tensor, block_table: torch.Tensor,
              seq_lens: torch.Tensor, qsl: torch.Tensor, seq_lens_host, qsl_host, scale: float,
              out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
              kv_split_tokens: int = 0, events=None, sliding_window: int = 0,
              local_chunk: int = 0, lse_out: Optional[torch.Tensor] = None,
              common_prefix_tokens: int = 0, stream=None) -> torch.Tensor:
    """Paged attention of one step; with ``lse_out`` (fp32 [T][Hq]) each row's natural-log
    log-sum-exp is written too, and decode-kind requests may hold no key (0 and -inf).
    ``common_prefix_tokens`` > 0: the requests' block tables share that many leading tokens'
    blocks (see pa_common_prefix_blocks), read once for all of them (cascade attention)."""
    T, Hq, D = q.shape
    if out is None:
        out = torch.empty(T, Hq, D, dtype=torch.float32, device=q.device)
    if lse_out is not None:
        assert lse_out.dtype == torch.float32 and lse_out.is_contiguous()
        assert lse_out.numel() == T * Hq
    if workspace is None:
        nb = workspace_bytes_for(cache, seq_lens_host, qsl_host, Hq, block_table.shape[1],
                                 kv_split_tokens, sliding_window=sliding_window,
                                 local_chunk=local_chunk, with_lse=lse_out is not None,
                                 common_prefix_tokens=common_prefix_tokens)
        workspace = torch.empty(max(nb, 1), dtype=torch.uint8, device=q.device)
    B.pa_attention_ex(cache.handle, q, Hq, block_table, block_table.shape[1], seq_lens, qsl,
                      seq_lens_host, qsl_host, seq_lens.numel(), T, scale, out, workspace,
                      workspace.numel(), kv_split_tokens=kv_split_tokens, events=events,
                      sliding_window=sliding_window, local_chunk=local_chunk, lse_out=lse_out,
                      common_prefix_tokens=common_prefix_tokens, stream=stream)
    return out
