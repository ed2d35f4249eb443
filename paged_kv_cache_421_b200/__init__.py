"""Paged KV cache and varlen paged attention for NVIDIA B200 (sm_100a).

The hot path -- block allocation, slot mapping, the KV-cache write and paged attention over a
flattened continuous-batching step -- runs in hand-written CUDA kernels behind the C ABI of
``libpa.so`` (``include/pa.h``).  ``_binding`` mirrors that ABI name for name; ``ops``
adds torch-tensor conveniences on top (output allocation, stream selection); ``workloads``
draws seeded synthetic serving steps; ``dcp`` runs decode attention with each request's KV
sharded over a group of GPUs (context parallelism).  PyTorch provides device memory and
streams only.
"""
from . import _binding  # noqa: F401
from ._binding import (PA_BF16, PA_FP8_E4M3, PaError, load, pa_alloc_cache,  # noqa: F401
                       pa_allocate_slots, pa_attention, pa_attention_ex,
                       pa_attention_noalloc, pa_attention_workspace_bytes, pa_cache_bytes,
                       pa_cache_data, pa_dcp_local_seq_lens, pa_dcp_slot_mapping,
                       pa_device_error, pa_free_blocks, pa_free_cache, pa_merge_partials,
                       pa_plan_attention, pa_slot_mapping, pa_status_string,
                       pa_validate_block_table, pa_write_kv)
