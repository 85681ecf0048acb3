"""One layer's paged KV cache on one GPU, driven through the C ABI.

A decode step of a serving loop, in the order the method needs it:

1. host: the C++ allocator gives every request a slot for its new token,
   taking a fresh block when the last one is full and copying a shared
   partial block first (copy-on-write pairs);
2. device: ``pa_copy_blocks`` for those pairs, then ``pa_reshape_and_cache``
   writes the new keys and values into their slots;
3. device: ``pa_decode`` attends every request's query over its whole
   cache through the block table.

Host-side staging uses pinned buffers and one copy per array.
"""

import numpy as np
import torch

from . import (PA_DECODE_AUTO, PaAlloc, pa_copy_blocks, pa_decode, pa_decode_workspace_size,
               pa_reshape_and_cache)


class PagedDecodeCache:
    def __init__(self, num_blocks, num_q_heads, num_kv_heads, head_dim, block_size, max_batch,
                 max_seq_len, initial_order=None, device="cuda", partition_tokens=0,
                 variant=PA_DECODE_AUTO):
        self.num_blocks = int(num_blocks)
        self.hq, self.hkv, self.d, self.bs = num_q_heads, num_kv_heads, head_dim, block_size
        self.max_batch = int(max_batch)
        self.max_seq_len = int(max_seq_len)
        self.max_blocks = -(-self.max_seq_len // block_size)
        self.device = torch.device(device)
        self.variant = variant
        self.partition_tokens = partition_tokens
        self.pool = torch.empty((self.num_blocks, 2, num_kv_heads, block_size, head_dim),
                                dtype=torch.bfloat16, device=self.device)
        self.alloc = PaAlloc(self.num_blocks, block_size, initial_order)
        nbytes, self.num_partitions = pa_decode_workspace_size(
            self.max_batch, num_q_heads, num_kv_heads, head_dim, block_size, self.max_seq_len,
            partition_tokens)
        self.workspace = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=self.device)
        # device-side step inputs
        self.d_tables = torch.zeros((self.max_batch, self.max_blocks), dtype=torch.int32, device=self.device)
        self.d_lens = torch.zeros(self.max_batch, dtype=torch.int32, device=self.device)
        self.d_slots = torch.zeros(self.max_batch, dtype=torch.int64, device=self.device)
        self.d_pairs = torch.zeros((self.max_batch, 2), dtype=torch.int32, device=self.device)
        # pinned host staging
        self.h_tables = torch.zeros((self.max_batch, self.max_blocks), dtype=torch.int32).pin_memory()
        self.h_lens = torch.zeros(self.max_batch, dtype=torch.int32).pin_memory()
        self.h_slots = torch.zeros(self.max_batch, dtype=torch.int64).pin_memory()
        self.h_pairs = torch.zeros((self.max_batch, 2), dtype=torch.int32).pin_memory()

    # ---------------------------------------------------------------- host
    def plan_append(self, seq_ids):
        """Allocator step for one new token per request (host only).

        Returns (slots int64 [B], pairs int32 [n, 2], tables int32 [B, MB],
        lens int32 [B]) as numpy arrays.
        """
        slots, pairs = self.alloc.append_batch(seq_ids, 1, as_numpy=True)
        tables, lens = self.alloc.block_tables(seq_ids, self.max_blocks)
        return slots, pairs, tables, lens

    def stage(self, slots, pairs, tables, lens, stream=None):
        """Copy one step's host metadata to the device (pinned, async)."""
        b = len(slots)
        npairs = len(pairs)
        self.h_slots[:b].numpy()[:] = slots
        self.h_tables[:b].numpy()[:] = tables
        self.h_lens[:b].numpy()[:] = lens
        if npairs:
            self.h_pairs[:npairs].numpy()[:] = pairs
        self.d_slots[:b].copy_(self.h_slots[:b], non_blocking=True)
        self.d_tables[:b].copy_(self.h_tables[:b], non_blocking=True)
        self.d_lens[:b].copy_(self.h_lens[:b], non_blocking=True)
        if npairs:
            self.d_pairs[:npairs].copy_(self.h_pairs[:npairs], non_blocking=True)
        return npairs

    # -------------------------------------------------------------- device
    def run(self, q, k_new, v_new, out, slots, tables, lens, pairs=None, max_seq_len=None):
        """Device part of a step on already-resident inputs (async)."""
        if pairs is not None and pairs.shape[0] > 0:
            pa_copy_blocks(self.pool, pairs)
        pa_reshape_and_cache(k_new, v_new, self.pool, slots)
        self.decode(q, out, tables, lens, max_seq_len)

    def decode(self, q, out, tables, lens, max_seq_len=None):
        pa_decode(out, q, self.pool, tables, lens, max_seq_len or self.max_seq_len,
                  1.0 / float(np.sqrt(self.d)), workspace=self.workspace, variant=self.variant,
                  partition_tokens=self.partition_tokens)

    def launches_per_step(self, npairs):
        """Kernels this library launches for one step."""
        return (1 if npairs else 0) + 1 + 1 + (1 if self.num_partitions > 1 else 0)
