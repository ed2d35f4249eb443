"""Decode context parallelism (DCP): each request's KV sharded over a group of GPUs.

The "vLLM architecture overview" (section 8, the index of its FlashAttention document) names
DCP without describing it.  Reading taken: logical block j of a request lives on rank
j mod world, as that rank's local logical block j / world, so every rank's share is an
ordinary paged cache (``ops.PagedKVCache``) with its own block table.  One decode step on
each rank (one process per GPU, ``torch.distributed`` over NCCL):

1. ``slot_mapping`` + ``ops.write_kv``: the rank stores the new tokens whose block it owns;
2. ``partial_attention``: every query attends to the rank's share, exporting each row's
   natural-log LSE (a request with no key on this rank yields 0 and -inf);
3. ``exchange``: an all-gather of every rank's (out, lse), the one collective of the step;
4. ``merge``: the LSE merge of the shares (``pa_merge_partials``), which is exactly the
   attention over the whole context.

Only pure decode steps shard this way (every request has q_len 0 or 1, and the GQA group
fits the decode tile, num_q_heads / num_kv_heads <= 8): a query row of a longer chunk needs
a causal mask across shares, which a per-rank bottom-right mask does not express.  This
module is argument marshalling and the collective; the arithmetic runs in the library's
kernels.
"""
from __future__ import annotations

from typing import Optional, Tuple

import numpy as np
import torch
import torch.distributed as dist

from . import _binding as B
from . import ops


def local_seq_lens(seq_lens_host, rank: int, world: int, block_size: int = 16) -> np.ndarray:
    """Keys of each request (of total length seq_lens_host[r]) that rank `rank` holds."""
    return B.pa_dcp_local_seq_lens(seq_lens_host, block_size, rank, world)


def slot_mapping(local_block_table: torch.Tensor, seq_lens: torch.Tensor, qsl: torch.Tensor,
                 num_tokens: int, rank: int, world: int, block_size: int = 16,
                 out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Slots of the step's new tokens on this rank (seq_lens: device, total lengths); -1 for
    tokens another rank stores, which ``ops.write_kv`` skips."""
    if out is None:
        out = torch.empty(num_tokens, dtype=torch.int32, device=local_block_table.device)
    B.pa_dcp_slot_mapping(local_block_table, local_block_table.shape[1], seq_lens, qsl,
                          seq_lens.numel(), num_tokens, block_size, rank, world, out, stream)
    return out


def check_decode_step(qsl_host, num_q_heads: int, num_kv_heads: int) -> None:
    q_lens = np.diff(np.asarray(qsl_host, np.int64))
    if np.any(q_lens > 1) or num_q_heads // num_kv_heads > 8:
        raise ValueError("context parallelism shards decode steps only: q_len <= 1 and "
                         "num_q_heads / num_kv_heads <= 8")


def partial_attention(cache: ops.PagedKVCache, q: torch.Tensor, local_block_table: torch.Tensor,
                      local_seq_lens_dev: torch.Tensor, qsl: torch.Tensor,
                      local_seq_lens_host, qsl_host, scale: float,
                      out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                      workspace: Optional[torch.Tensor] = None,
                      stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """This rank's share of the step: (out [T][Hq][D], lse [T][Hq]) over its own keys."""
    T, Hq, _ = q.shape
    check_decode_step(qsl_host, Hq, cache.num_kv_heads)
    if lse is None:
        lse = torch.empty(T, Hq, dtype=torch.float32, device=q.device)
    out = ops.attention(cache, q, local_block_table, local_seq_lens_dev, qsl,
                        local_seq_lens_host, qsl_host, scale, out=out, workspace=workspace,
                        lse_out=lse, stream=stream)
    return out, lse


def exchange(out: torch.Tensor, lse: torch.Tensor,
             group=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """All-gather every rank's (out, lse) into [world][...] tensors, rank order."""
    world = dist.get_world_size(group)
    parts_out = torch.empty((world,) + tuple(out.shape), dtype=out.dtype, device=out.device)
    parts_lse = torch.empty((world,) + tuple(lse.shape), dtype=lse.dtype, device=lse.device)
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(parts_out, out.contiguous(), group=group)
        dist.all_gather_into_tensor(parts_lse, lse.contiguous(), group=group)
    else:  # gloo (CPU tensors): gather into views of the same buffers
        dist.all_gather(list(parts_out.unbind(0)), out.contiguous(), group=group)
        dist.all_gather(list(parts_lse.unbind(0)), lse.contiguous(), group=group)
    return parts_out, parts_lse


def merge(parts_out: torch.Tensor, parts_lse: torch.Tensor, out: Optional[torch.Tensor] = None,
          lse_out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """LSE merge of the shares: parts_out [P][T][Hq][D], parts_lse [P][T][Hq] -> out."""
    P, D = parts_out.shape[0], parts_out.shape[-1]
    rows = parts_lse[0].numel()
    assert parts_out.is_contiguous() and parts_lse.is_contiguous()
    assert parts_out.dtype == torch.float32 and parts_lse.dtype == torch.float32
    assert parts_out.numel() == P * rows * D
    if out is None:
        out = torch.empty(parts_out.shape[1:], dtype=torch.float32, device=parts_out.device)
    B.pa_merge_partials(parts_out, parts_lse, P, rows, D, out, lse_out, stream)
    return out


def attention(cache: ops.PagedKVCache, q: torch.Tensor, local_block_table: torch.Tensor,
              seq_lens_host, qsl: torch.Tensor, qsl_host, scale: float,
              group=None) -> torch.Tensor:
    """One decode step's attention over the whole context, this rank holding its share in
    `cache` (its local table in `local_block_table`); seq_lens_host are the requests' total
    lengths.  Every rank of `group` calls this with the same queries and gets the result.
    Kernels run on torch's current stream, which NCCL orders the all-gather against."""
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    loc = local_seq_lens(seq_lens_host, rank, world, cache.block_size)
    loc_dev = torch.from_numpy(loc).to(q.device)
    out, lse = partial_attention(cache, q, local_block_table, loc_dev, qsl, loc, qsl_host, scale)
    parts_out, parts_lse = exchange(out, lse, group)
    return merge(parts_out, parts_lse)
