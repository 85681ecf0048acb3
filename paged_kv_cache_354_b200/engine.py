"""One layer's paged KV cache on one GPU, driven through the C ABI.

A decode step of a serving loop, in the order the method needs it:

1. host: the C++ allocator gives every request a slot for its new token,
   taking a fresh block when the last one is full and copying a shared
   partial block first (copy-on-write pairs);
2. device: ``pa_copy_blocks`` for those pairs, then ``pa_reshape_and_cache``
   writes the new keys and values into their slots;
3. device: ``pa_decode`` attends every request's query over its whole
   cache through the block table.

Host-side staging: the allocator writes a step's slots, copy-on-write pairs,
block tables and lengths straight into one pinned buffer, which reaches the
device in a single copy.  The device part of a step (cache write, decode,
merge) can be recorded once into a CUDA graph and replayed every step.
"""

import ctypes

import numpy as np
import torch

from . import (PA_DECODE_AUTO, PaAlloc, _check, lib, pa_copy_blocks, pa_decode, pa_decode_append,
               pa_decode_workspace_size, pa_reshape_and_cache)


def _align(n, a=256):
    return (n + a - 1) // a * a


class PagedDecodeCache:
    def __init__(self, num_blocks, num_q_heads, num_kv_heads, head_dim, block_size, max_batch,
                 max_seq_len, initial_order=None, device="cuda", partition_tokens=0,
                 variant=PA_DECODE_AUTO, staging_sets=1):
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
        nbytes, self.num_partitions, self.schedule = pa_decode_workspace_size(
            self.max_batch, num_q_heads, num_kv_heads, head_dim, block_size, self.max_seq_len,
            partition_tokens, with_schedule=True)
        self.workspace = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=self.device)
        # A step's staging buffer: metadata written by the allocator and the
        # step's inputs, in one pinned block that reaches the device in one
        # copy.  Layout: slots int64[B] | lens int32[B] | pairs int32[B,2] |
        # tables int32[B,MB] | q bf16[B,Hq,D] | k bf16[B,Hkv,D] | v bf16[B,Hkv,D].
        # ``staging_sets`` pinned buffers rotate so a caller can fill the
        # next step's inputs while the device works on the current one.
        b, mb = self.max_batch, self.max_blocks
        self._layout = {}
        off = 0
        for name, dtype, shape in (("slots", torch.int64, (b,)), ("lens", torch.int32, (b,)),
                                   ("pairs", torch.int32, (b, 2)), ("tables", torch.int32, (b, mb)),
                                   ("q", torch.bfloat16, (b, num_q_heads, head_dim)),
                                   ("k", torch.bfloat16, (b, num_kv_heads, head_dim)),
                                   ("v", torch.bfloat16, (b, num_kv_heads, head_dim))):
            nbytes_f = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
            self._layout[name] = (off, dtype, shape, nbytes_f)
            off += _align(nbytes_f)
        self.stage_bytes = off
        self.meta_bytes = self._layout["q"][0]
        self.h_stage = [torch.zeros(off, dtype=torch.uint8).pin_memory() for _ in range(staging_sets)]
        self.d_stage = torch.zeros(off, dtype=torch.uint8, device=self.device)
        # device views the kernels (and a captured graph) read
        (self.s_slots, self.s_lens, self.s_pairs, self.s_tables, self.s_q, self.s_k,
         self.s_v) = (self._view(self.d_stage, n) for n in ("slots", "lens", "pairs", "tables", "q", "k", "v"))
        self._ncow = ctypes.c_int(0)
        self._ids = None
        self._ids_src = None
        self.graph = None

    def _view(self, buf, name):
        off, dtype, shape, nbytes_f = self._layout[name]
        return buf[off:off + nbytes_f].view(dtype).view(shape)

    def staged(self, name, j=0):
        """Host view of field ``name`` of pinned staging buffer ``j`` (fill
        q / k / v here; the allocator fills the metadata)."""
        return self._view(self.h_stage[j], name)

    def _hptr(self, name, j):
        return ctypes.c_void_p(self.h_stage[j].data_ptr() + self._layout[name][0])

    # ---------------------------------------------------------------- host
    def plan_append(self, seq_ids):
        """Allocator step for one new token per request (host only).

        Returns (slots int64 [B], pairs int32 [n, 2], tables int32 [B, MB],
        lens int32 [B]) as numpy arrays.
        """
        slots, pairs = self.alloc.append_batch(seq_ids, 1, as_numpy=True)
        tables, lens = self.alloc.block_tables(seq_ids, self.max_blocks)
        return slots, pairs, tables, lens

    def host_step(self, seq_ids, j=0):
        """Allocator step for one new token per request (host only), written
        straight into pinned staging buffer ``j``.  Returns the number of
        copy-on-write pairs.  ``seq_ids`` must hold max_batch requests."""
        if self._ids is None or self._ids_src is not seq_ids:
            self._ids = np.ascontiguousarray(np.asarray(seq_ids, dtype=np.int64))
            self._ids_src = seq_ids
            assert len(self._ids) == self.max_batch
        h = self.alloc._h
        ids = ctypes.c_void_p(self._ids.ctypes.data)
        b = self.max_batch
        _check(lib.pa_alloc_append_batch(h, ids, b, 1, self._hptr("slots", j), self._hptr("pairs", j), b,
                                         ctypes.byref(self._ncow)), "pa_alloc_append_batch")
        _check(lib.pa_alloc_block_tables(h, ids, b, self.max_blocks, self._hptr("tables", j),
                                         self._hptr("lens", j)), "pa_alloc_block_tables")
        return self._ncow.value

    def upload(self, j=0, with_inputs=True):
        """One host-to-device copy of staging buffer ``j`` (metadata, and the
        q / k / v inputs unless ``with_inputs`` is false); async, pinned."""
        n = self.stage_bytes if with_inputs else self.meta_bytes
        self.d_stage[:n].copy_(self.h_stage[j][:n], non_blocking=True)

    def capture(self, out):
        """Record the device part of a step -- the new tokens' cache write
        fused with the decode, and the merge -- on the staged device buffers
        into a CUDA graph; replay it with ``replay``.

        Call after one ``host_step`` + ``upload`` so the staged slots are
        real: the eager warm-up run writes the step's own K/V, which the
        replay writes again."""
        side = torch.cuda.Stream(device=self.device)
        side.wait_stream(torch.cuda.current_stream(self.device))
        with torch.cuda.stream(side):
            self._device_step(out)
        torch.cuda.current_stream(self.device).wait_stream(side)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self._device_step(out)
        self.graph = g
        return g

    def _device_step(self, out):
        self.append_decode(self.s_q, self.s_k, self.s_v, out, self.s_slots, self.s_tables, self.s_lens)

    def replay(self, npairs):
        """Device part of a staged step: copy-on-write copies (if any), then the graph."""
        if npairs:
            pa_copy_blocks(self.pool, self.s_pairs[:npairs])
        self.graph.replay()

    def capture_steps(self, out, h_out, zero_copy=True):
        """Record, for every staging buffer j, a whole step as one CUDA graph:
        the upload of buffer j and the fused cache write + decode + merge,
        with the output landing in the pinned host tensor ``h_out``.

        zero_copy: the kernels store the output straight into ``h_out``
        across PCIe as each (request, head) row becomes final, so the rows
        stream to the host while the decode still runs and only the merged
        rows are left at its end.  Otherwise the kernels write ``out`` on the
        device and the graph ends with one device-to-host copy of it.  Both
        sets of graphs may be recorded; ``replay_step`` uses the one named,
        or the last recorded.  Needs the graph of ``capture`` (its eager
        warm-up); steps with copy-on-write pairs run eagerly, since the
        copies must come between the upload and the decode."""
        assert self.graph is not None, "capture() first"
        self._out, self._h_out, self._zero_copy = out, h_out, zero_copy
        graphs = []
        for j in range(len(self.h_stage)):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                self.d_stage.copy_(self.h_stage[j], non_blocking=True)
                self._device_step(h_out if zero_copy else out)
                if not zero_copy:
                    h_out.copy_(out, non_blocking=True)
            graphs.append(g)
        if not hasattr(self, "step_graphs"):
            self.step_graphs = {}
        self.step_graphs[bool(zero_copy)] = graphs
        return graphs

    def replay_step(self, j, npairs, zero_copy=None):
        """A whole staged step (asynchronous): one graph launch, or, with
        copy-on-write pairs, the upload, the copies and the decode launched
        one by one.  ``h_out`` holds the output once the stream is
        synchronised."""
        zc = self._zero_copy if zero_copy is None else bool(zero_copy)
        if npairs:
            self.upload(j)
            pa_copy_blocks(self.pool, self.s_pairs[:npairs])
            if zc:
                self._device_step(self._h_out)
            else:
                self._device_step(self._out)
                self._h_out.copy_(self._out, non_blocking=True)
        else:
            self.step_graphs[zc][j].replay()

    # -------------------------------------------------------------- device
    def run(self, q, k_new, v_new, out, slots, tables, lens, pairs=None, max_seq_len=None):
        """Device part of a step on already-resident inputs (async): the
        copy-on-write copies, then the new tokens' cache write fused with the
        decode (pa_decode_append; the library's default path).  With an
        explicit partition size or variant the two calls run separately."""
        if pairs is not None and pairs.shape[0] > 0:
            pa_copy_blocks(self.pool, pairs)
        self.append_decode(q, k_new, v_new, out, slots, tables, lens, max_seq_len)

    def append_decode(self, q, k_new, v_new, out, slots, tables, lens, max_seq_len=None):
        if self.partition_tokens == 0 and self.variant == PA_DECODE_AUTO:
            pa_decode_append(out, q, self.pool, k_new, v_new, slots, tables, lens,
                             max_seq_len or self.max_seq_len, 1.0 / float(np.sqrt(self.d)),
                             workspace=self.workspace)
        else:
            pa_reshape_and_cache(k_new, v_new, self.pool, slots)
            self.decode(q, out, tables, lens, max_seq_len)

    def decode(self, q, out, tables, lens, max_seq_len=None):
        pa_decode(out, q, self.pool, tables, lens, max_seq_len or self.max_seq_len,
                  1.0 / float(np.sqrt(self.d)), workspace=self.workspace, variant=self.variant,
                  partition_tokens=self.partition_tokens)

    def launches_per_step(self, npairs):
        """Kernels this library launches for one step."""
        # the cache write is fused into the balanced decode; on the
        # per-partition grid (or with explicit choices) it runs first
        fused = self.partition_tokens == 0 and self.variant == PA_DECODE_AUTO and self.schedule == "balanced"
        cache_write = 0 if fused else 1
        return (1 if npairs else 0) + cache_write + 1 + (1 if self.num_partitions > 1 else 0)
