"""Python binding of libpa.so: paged KV cache and paged decode attention on B200.

Thin marshalling over the C ABI declared in ``include/pa.h``: every function
here has the C entry point's name and only turns tensors into pointers and
the current CUDA stream into a handle.  All work runs in the library's
kernels; there is no Python or CPU fallback.  Importing this package raises
if ``libpa.so`` is missing (build it with
``python paged_kv_cache_354_b200/_build.py``).

bf16 tensors are ``torch.bfloat16``; shapes follow ``include/pa.h``:
    kv_pool      [num_blocks, 2, num_kv_heads, block_size, head_dim]
    q, out       [batch, num_q_heads, head_dim]
    key, value   [num_tokens, num_kv_heads, head_dim]
    kv_cache     [batch, 2, num_kv_heads, max_len, head_dim]  (contiguous decode)
    block_tables int32 [batch, max_blocks_per_seq]; seq_lens int32 [batch]
    slot_mapping int64 [num_tokens]; block_pairs int32 [num_pairs, 2]
"""

import ctypes
import os

import numpy as np

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libpa.so")

PA_OK = 0
PA_ERR_INVALID = -1
PA_ERR_UNSUPPORTED = -2
PA_ERR_OOM = -3
PA_ERR_CUDA = -4
PA_ERR_NOT_FOUND = -5
PA_ERR_EXISTS = -6

PA_DEVERR_BLOCK_ID = 0x1
PA_DEVERR_SLOT = 0x2
PA_DEVERR_SEQ_LEN = 0x4
PA_DEVERR_WAIT_TIMEOUT = 0x8
PA_DEVERR_COPY_PAIR = 0x10

PA_DECODE_AUTO = 0
PA_DECODE_CUDA_CORE = 1
PA_DECODE_MMA = 2
PA_DECODE_TCGEN05 = 3

PA_SCHEDULE_BALANCED = -1  # partition_tokens value that asks for the balanced schedule

_c = ctypes
_P = _c.c_void_p
_I = _c.c_int
_I64 = _c.c_int64
_SZ = _c.c_size_t

# name -> (restype, argtypes); mirrors include/pa.h
_SIGNATURES = {
    "pa_version": (_I, []),
    "pa_last_error_string": (_c.c_char_p, []),
    "pa_device_error": (_I, [_P, _I]),
    "pa_reshape_and_cache": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _P]),
    "pa_copy_blocks": (_I, [_P, _P, _I, _I, _I, _I, _I, _P]),
    "pa_decode_workspace_size": (_I, [_I, _I, _I, _I, _I, _I, _P, _P]),
    "pa_decode_workspace_size_ex": (_I, [_I, _I, _I, _I, _I, _I, _I, _P, _P, _P]),
    "pa_decode": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _c.c_float, _P, _SZ, _P]),
    "pa_decode_ex": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _c.c_float, _P, _SZ,
                          _I, _I, _P]),
    "pa_decode_noalloc": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _c.c_float, _P]),
    "pa_decode_append": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _c.c_float, _P,
                              _SZ, _P]),
    "pa_decode_multi_workspace_size": (_I, [_I, _I, _I, _I, _I, _I, _I, _P]),
    "pa_decode_multi": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _I, _c.c_float, _P, _SZ,
                             _P]),
    "pa_decode_contiguous_workspace_size": (_I, [_I, _I, _I, _I, _I, _P]),
    "pa_decode_contiguous": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _c.c_float, _P, _SZ, _I, _P]),
    "pa_selftest_wait_timeout": (_I, [_I64, _P]),
    "pa_alloc_create": (_I, [_I, _I, _P, _P]),
    "pa_alloc_destroy": (_I, [_P]),
    "pa_alloc_add_seq": (_I, [_P, _I64]),
    "pa_alloc_fork": (_I, [_P, _I64, _I64]),
    "pa_alloc_append": (_I, [_P, _I64, _I, _P, _P, _I, _P]),
    "pa_alloc_append_batch": (_I, [_P, _P, _I, _I, _P, _P, _I, _P]),
    "pa_alloc_free_seq": (_I, [_P, _I64]),
    "pa_alloc_num_free": (_I, [_P, _P]),
    "pa_alloc_seq_len": (_I, [_P, _I64, _P]),
    "pa_alloc_refcount": (_I, [_P, _I, _P]),
    "pa_alloc_block_table": (_I, [_P, _I64, _P, _I, _P]),
    "pa_alloc_block_tables": (_I, [_P, _P, _I, _I, _P, _P]),
    "pa_alloc_dump": (_I, [_P, _P, _P, _P]),
    "pa_alloc_stats": (_I, [_P, _P]),
}


def _load():
    if not os.path.exists(_LIB_PATH):
        raise ImportError(
            f"{_LIB_PATH} is missing: build it with `python paged_kv_cache_354_b200/_build.py`"
        )
    lib = ctypes.CDLL(_LIB_PATH)
    for name, (res, args) in _SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()
LIB_PATH = _LIB_PATH


class PaError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        msg = lib.pa_last_error_string().decode(errors="replace")
        super().__init__(f"{where} returned {status}: {msg}")


class OutOfBlocks(PaError):
    pass


def _check(status, where):
    if status != PA_OK:
        if status == PA_ERR_OOM:
            raise OutOfBlocks(status, where)
        raise PaError(status, where)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _stream(stream):
    import torch

    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _require(t, dtype, name, pinned_ok=False):
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_cuda and not (pinned_ok and t.is_pinned()):
        raise TypeError(f"{name}: expected a CUDA tensor" + (" or a pinned host tensor" if pinned_ok else ""))
    if not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous tensor")


# --------------------------------------------------------------------------
# kernels
# --------------------------------------------------------------------------
def pa_version():
    return lib.pa_version()


def pa_device_error(clear=True):
    """OR of PA_DEVERR_* bits recorded by kernels on the current device."""
    code = ctypes.c_int32(0)
    _check(lib.pa_device_error(ctypes.byref(code), 1 if clear else 0), "pa_device_error")
    return code.value


def pa_reshape_and_cache(key, value, kv_pool, slot_mapping, stream=None):
    import torch

    _require(key, torch.bfloat16, "key")
    _require(value, torch.bfloat16, "value")
    _require(kv_pool, torch.bfloat16, "kv_pool")
    _require(slot_mapping, torch.int64, "slot_mapping")
    nb, two, hkv, bs, d = kv_pool.shape
    t = key.shape[0]
    if key.shape != (t, hkv, d) or value.shape != (t, hkv, d) or slot_mapping.shape != (t,):
        raise ValueError("pa_reshape_and_cache: shape mismatch")
    _check(lib.pa_reshape_and_cache(_ptr(key), _ptr(value), _ptr(kv_pool), _ptr(slot_mapping), t, nb,
                                    hkv, bs, d, _stream(stream)), "pa_reshape_and_cache")


def pa_copy_blocks(kv_pool, block_pairs, stream=None):
    import torch

    _require(kv_pool, torch.bfloat16, "kv_pool")
    nb, two, hkv, bs, d = kv_pool.shape
    n = 0 if block_pairs is None else block_pairs.shape[0]
    if n == 0:
        return
    _require(block_pairs, torch.int32, "block_pairs")
    _check(lib.pa_copy_blocks(_ptr(kv_pool), _ptr(block_pairs), n, nb, hkv, bs, d, _stream(stream)),
           "pa_copy_blocks")


def pa_decode_workspace_size(batch, num_q_heads, num_kv_heads, head_dim, block_size, max_seq_len,
                             partition_tokens=0, with_schedule=False):
    """(bytes, num_partitions) of the split-K scratch pa_decode needs; with
    ``with_schedule`` also "balanced" or "grid"."""
    nbytes = ctypes.c_size_t(0)
    parts = ctypes.c_int(0)
    balanced = ctypes.c_int(0)
    _check(lib.pa_decode_workspace_size_ex(batch, num_q_heads, num_kv_heads, head_dim, block_size,
                                           max_seq_len, partition_tokens, ctypes.byref(nbytes),
                                           ctypes.byref(parts), ctypes.byref(balanced)),
           "pa_decode_workspace_size")
    if with_schedule:
        return nbytes.value, parts.value, ("balanced" if balanced.value else "grid")
    return nbytes.value, parts.value


def pa_decode(out, q, kv_pool, block_tables, seq_lens, max_seq_len, scale, workspace=None,
              variant=PA_DECODE_AUTO, partition_tokens=0, stream=None):
    """Paged decode attention; writes ``out`` (bf16 [B, Hq, D]) in place.
    ``out`` is a CUDA tensor or a pinned host tensor (the kernels then store
    the rows across PCIe as they finish; read it after the stream syncs)."""
    import torch

    _require(out, torch.bfloat16, "out", pinned_ok=True)
    _require(q, torch.bfloat16, "q")
    _require(kv_pool, torch.bfloat16, "kv_pool")
    _require(block_tables, torch.int32, "block_tables")
    _require(seq_lens, torch.int32, "seq_lens")
    nb, two, hkv, bs, d = kv_pool.shape
    b, hq, dq = q.shape
    if out.shape != q.shape or dq != d or block_tables.shape[0] != b or seq_lens.shape != (b,):
        raise ValueError("pa_decode: shape mismatch")
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        _require(workspace, torch.uint8, "workspace")
        ws_ptr, ws_bytes = _ptr(workspace), workspace.numel()
    _check(lib.pa_decode_ex(_ptr(out), _ptr(q), _ptr(kv_pool), _ptr(block_tables), _ptr(seq_lens), b, hq,
                            hkv, d, bs, nb, block_tables.shape[1], int(max_seq_len), float(scale), ws_ptr,
                            ws_bytes, int(variant), int(partition_tokens), _stream(stream)), "pa_decode")


def pa_decode_multi_workspace_size(batch, num_query_tokens, num_q_heads, num_kv_heads, head_dim, block_size,
                                   max_seq_len):
    nbytes = ctypes.c_size_t(0)
    _check(lib.pa_decode_multi_workspace_size(batch, num_query_tokens, num_q_heads, num_kv_heads, head_dim,
                                              block_size, max_seq_len, ctypes.byref(nbytes)),
           "pa_decode_multi_workspace_size")
    return nbytes.value


def pa_decode_multi(out, q, kv_pool, block_tables, seq_lens, max_seq_len, scale, workspace, stream=None):
    """T causal query tokens per request: q, out bf16 [B, T, Hq, D]."""
    import torch

    _require(out, torch.bfloat16, "out", pinned_ok=True)
    _require(q, torch.bfloat16, "q")
    _require(kv_pool, torch.bfloat16, "kv_pool")
    _require(block_tables, torch.int32, "block_tables")
    _require(seq_lens, torch.int32, "seq_lens")
    _require(workspace, torch.uint8, "workspace")
    nb, two, hkv, bs, d = kv_pool.shape
    b, t, hq, dq = q.shape
    if out.shape != q.shape or dq != d or block_tables.shape[0] != b or seq_lens.shape != (b,):
        raise ValueError("pa_decode_multi: shape mismatch")
    _check(lib.pa_decode_multi(_ptr(out), _ptr(q), _ptr(kv_pool), _ptr(block_tables), _ptr(seq_lens), b, t, hq,
                               hkv, d, bs, nb, block_tables.shape[1], int(max_seq_len), float(scale),
                               _ptr(workspace), workspace.numel(), _stream(stream)), "pa_decode_multi")


def pa_decode_contiguous_workspace_size(batch, num_q_heads, num_kv_heads, head_dim, max_len):
    nbytes = ctypes.c_size_t(0)
    _check(lib.pa_decode_contiguous_workspace_size(batch, num_q_heads, num_kv_heads, head_dim, max_len,
                                                   ctypes.byref(nbytes)), "pa_decode_contiguous_workspace_size")
    return nbytes.value


def pa_decode_contiguous(out, q, kv_cache, seq_lens, scale, workspace, variant=PA_DECODE_AUTO, stream=None):
    """Decode over a contiguous per-request cache kv_cache bf16
    [B, 2, Hkv, max_len, D] (no block table); writes ``out`` in place."""
    import torch

    _require(out, torch.bfloat16, "out", pinned_ok=True)
    _require(q, torch.bfloat16, "q")
    _require(kv_cache, torch.bfloat16, "kv_cache")
    _require(seq_lens, torch.int32, "seq_lens")
    _require(workspace, torch.uint8, "workspace")
    b, two, hkv, max_len, d = kv_cache.shape
    bq, hq, dq = q.shape
    if two != 2 or out.shape != q.shape or dq != d or bq != b or seq_lens.shape != (b,):
        raise ValueError("pa_decode_contiguous: shape mismatch")
    _check(lib.pa_decode_contiguous(_ptr(out), _ptr(q), _ptr(kv_cache), _ptr(seq_lens), b, hq, hkv, d, max_len,
                                    float(scale), _ptr(workspace), workspace.numel(), int(variant),
                                    _stream(stream)), "pa_decode_contiguous")


PA_NOALLOC_SCRATCH_BYTES = 16 * 1024 * 1024


def pa_decode_noalloc(out, q, kv_pool, block_tables, seq_lens, max_seq_len, scale, stream=None):
    """pa_decode without a workspace argument, for callers that cannot
    allocate device memory: the split-K partials live in a fixed array of
    PA_NOALLOC_SCRATCH_BYTES inside the library (shared by all calls on a
    device; calls that overlap on the GPU race on it)."""
    import torch

    _require(out, torch.bfloat16, "out", pinned_ok=True)
    _require(q, torch.bfloat16, "q")
    _require(kv_pool, torch.bfloat16, "kv_pool")
    _require(block_tables, torch.int32, "block_tables")
    _require(seq_lens, torch.int32, "seq_lens")
    nb, two, hkv, bs, d = kv_pool.shape
    b, hq, dq = q.shape
    if out.shape != q.shape or dq != d or block_tables.shape[0] != b or seq_lens.shape != (b,):
        raise ValueError("pa_decode_noalloc: shape mismatch")
    _check(lib.pa_decode_noalloc(_ptr(out), _ptr(q), _ptr(kv_pool), _ptr(block_tables), _ptr(seq_lens), b,
                                 hq, hkv, d, bs, nb, block_tables.shape[1], int(max_seq_len), float(scale),
                                 _stream(stream)), "pa_decode_noalloc")


def pa_decode_append(out, q, kv_pool, key, value, slot_mapping, block_tables, seq_lens, max_seq_len, scale,
                     workspace=None, stream=None):
    """pa_reshape_and_cache of each request's newest token (key/value
    [B, Hkv, D], slot_mapping [B]) and pa_decode, in one pass."""
    import torch

    _require(out, torch.bfloat16, "out", pinned_ok=True)
    for t, dt, n in ((q, torch.bfloat16, "q"), (kv_pool, torch.bfloat16, "kv_pool"),
                     (key, torch.bfloat16, "key"), (value, torch.bfloat16, "value"),
                     (slot_mapping, torch.int64, "slot_mapping"), (block_tables, torch.int32, "block_tables"),
                     (seq_lens, torch.int32, "seq_lens")):
        _require(t, dt, n)
    nb, two, hkv, bs, d = kv_pool.shape
    b, hq, dq = q.shape
    if (out.shape != q.shape or dq != d or key.shape != (b, hkv, d) or value.shape != (b, hkv, d)
            or slot_mapping.shape != (b,) or block_tables.shape[0] != b or seq_lens.shape != (b,)):
        raise ValueError("pa_decode_append: shape mismatch")
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        _require(workspace, torch.uint8, "workspace")
        ws_ptr, ws_bytes = _ptr(workspace), workspace.numel()
    _check(lib.pa_decode_append(_ptr(out), _ptr(q), _ptr(kv_pool), _ptr(key), _ptr(value), _ptr(slot_mapping),
                                _ptr(block_tables), _ptr(seq_lens), b, hq, hkv, d, bs, nb, block_tables.shape[1],
                                int(max_seq_len), float(scale), ws_ptr, ws_bytes, _stream(stream)),
           "pa_decode_append")


def pa_selftest_wait_timeout(limit_ns, stream=None):
    _check(lib.pa_selftest_wait_timeout(int(limit_ns), _stream(stream)), "pa_selftest_wait_timeout")


# --------------------------------------------------------------------------
# host allocator
# --------------------------------------------------------------------------
class PaAlloc:
    """Handle on the C++ block allocator (pa_alloc_* calls).

    Method names match the allocator model used by the tests so one driver
    can run either.
    """

    def __init__(self, num_blocks, block_size, initial_order=None):
        self.num_blocks = int(num_blocks)
        self.block_size = int(block_size)
        h = ctypes.c_void_p()
        order = None
        if initial_order is not None:
            order = np.ascontiguousarray(np.asarray(initial_order, dtype=np.int32))
            if order.shape != (self.num_blocks,):
                raise ValueError("initial_order must list every block once")
        _check(lib.pa_alloc_create(self.num_blocks, self.block_size,
                                   order.ctypes.data_as(ctypes.c_void_p) if order is not None else None,
                                   ctypes.byref(h)), "pa_alloc_create")
        self._h = h
        self._cow = np.zeros(2 * 1024, dtype=np.int32)

    def close(self):
        if self._h:
            lib.pa_alloc_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def add_seq(self, seq_id):
        _check(lib.pa_alloc_add_seq(self._h, int(seq_id)), "pa_alloc_add_seq")

    def fork(self, parent, child):
        _check(lib.pa_alloc_fork(self._h, int(parent), int(child)), "pa_alloc_fork")

    def free_seq(self, seq_id):
        _check(lib.pa_alloc_free_seq(self._h, int(seq_id)), "pa_alloc_free_seq")

    def append(self, seq_id, num_tokens):
        return self.append_batch([seq_id], num_tokens)

    def append_batch(self, seq_ids, num_tokens, as_numpy=False):
        """(slots, cow_pairs) like the model: slots in (request, token) order."""
        ids = np.ascontiguousarray(np.asarray(seq_ids, dtype=np.int64))
        slots = np.empty(len(ids) * int(num_tokens), dtype=np.int64)
        ncow = ctypes.c_int(0)
        cap = max(1, len(ids))
        if self._cow.size < 2 * cap:
            self._cow = np.zeros(2 * cap, dtype=np.int32)
        _check(lib.pa_alloc_append_batch(self._h, ids.ctypes.data_as(ctypes.c_void_p), len(ids),
                                         int(num_tokens), slots.ctypes.data_as(ctypes.c_void_p),
                                         self._cow.ctypes.data_as(ctypes.c_void_p), cap,
                                         ctypes.byref(ncow)), "pa_alloc_append_batch")
        pairs = self._cow[: 2 * ncow.value].reshape(-1, 2).copy()
        if as_numpy:
            return slots, pairs
        return slots.tolist(), [tuple(int(x) for x in p) for p in pairs]

    def num_free(self):
        n = ctypes.c_int(0)
        _check(lib.pa_alloc_num_free(self._h, ctypes.byref(n)), "pa_alloc_num_free")
        return n.value

    def seq_len(self, seq_id):
        n = ctypes.c_int(0)
        _check(lib.pa_alloc_seq_len(self._h, int(seq_id), ctypes.byref(n)), "pa_alloc_seq_len")
        return n.value

    def refcount(self, block):
        n = ctypes.c_int(0)
        _check(lib.pa_alloc_refcount(self._h, int(block), ctypes.byref(n)), "pa_alloc_refcount")
        return n.value

    def block_table(self, seq_id):
        cap = self.num_blocks
        out = np.empty(cap, dtype=np.int32)
        n = ctypes.c_int(0)
        _check(lib.pa_alloc_block_table(self._h, int(seq_id), out.ctypes.data_as(ctypes.c_void_p), cap,
                                        ctypes.byref(n)), "pa_alloc_block_table")
        return out[: n.value].tolist()

    def block_tables(self, seq_ids, max_blocks_per_seq):
        """Padded int32 [n, max_blocks_per_seq] tables and int32 lengths (numpy)."""
        ids = np.ascontiguousarray(np.asarray(seq_ids, dtype=np.int64))
        tables = np.empty((len(ids), int(max_blocks_per_seq)), dtype=np.int32)
        lens = np.empty(len(ids), dtype=np.int32)
        _check(lib.pa_alloc_block_tables(self._h, ids.ctypes.data_as(ctypes.c_void_p), len(ids),
                                         int(max_blocks_per_seq), tables.ctypes.data_as(ctypes.c_void_p),
                                         lens.ctypes.data_as(ctypes.c_void_p)), "pa_alloc_block_tables")
        return tables, lens

    def dump(self):
        free = np.empty(self.num_blocks, dtype=np.int32)
        refs = np.empty(self.num_blocks, dtype=np.int32)
        n = ctypes.c_int(0)
        _check(lib.pa_alloc_dump(self._h, free.ctypes.data_as(ctypes.c_void_p), ctypes.byref(n),
                                 refs.ctypes.data_as(ctypes.c_void_p)), "pa_alloc_dump")
        return free[: n.value].tolist(), refs.tolist()

    def stats(self):
        """dict: tokens, logical_slots, physical_blocks, live_requests, free_blocks."""
        out = np.zeros(5, dtype=np.int64)
        _check(lib.pa_alloc_stats(self._h, out.ctypes.data_as(ctypes.c_void_p)), "pa_alloc_stats")
        keys = ("tokens", "logical_slots", "physical_blocks", "live_requests", "free_blocks")
        return dict(zip(keys, (int(x) for x in out)))

    def free_list(self):
        return self.dump()[0]

    def refcounts(self):
        return self.dump()[1]
