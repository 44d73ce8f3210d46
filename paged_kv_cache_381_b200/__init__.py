"""Paged KV-cache decode for B200 (sm_100a): Python binding of libpa.so.

Argument marshalling only -- every step of the path runs in the library's CUDA
kernels or its native host code.  PyTorch supplies device memory and streams.
The names follow the C ABI in include/pa.h:

    pa_cache_write(k, v, k_cache, v_cache, slot_mapping)
    pa_decode(out, q, k_cache, v_cache, block_tables, context_lens, scale, ...)
    pa_copy_blocks(k_cache, v_cache, pairs)
    pa_step(...)                  one layer-step from host buffers
    BlockManager / Scheduler      host bookkeeping (pa_bm_*, pa_sched_*)
"""

import ctypes

import numpy as np

from . import _native

PA_OK = 0
STATUS_NAMES = {0: "PA_OK", 1: "PA_ERR_INVALID_ARG", 2: "PA_ERR_UNSUPPORTED", 3: "PA_ERR_NO_BLOCKS",
                4: "PA_ERR_CUDA", 5: "PA_ERR_DEVICE"}
PA_ERR_NO_BLOCKS = 3
DEVERR_SLOT, DEVERR_BLOCK_ID, DEVERR_CONTEXT_LEN, DEVERR_TIMEOUT = 0x1, 0x2, 0x4, 0x8
DEVERR_SMEM_ALIGN = 0x10
KERNELS = ("cache_write", "decode", "reduce", "plan", "copy_blocks", "verify", "swap", "write_plan")
DEFAULT_PARTITION = 512


class PagedAttentionError(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)}")


class NoBlocksError(PagedAttentionError):
    pass


def _check(status, what):
    if status != PA_OK:
        if status == PA_ERR_NO_BLOCKS:
            raise NoBlocksError(status, what)
        raise PagedAttentionError(status, what)


def lib():
    return _native.load()


# ---------------------------------------------------------------------------
# device path
# ---------------------------------------------------------------------------

def _dtype_code(t):
    import torch
    codes = {torch.float32: 0, torch.float16: 1, torch.bfloat16: 2}
    if t.dtype not in codes:
        raise TypeError(f"unsupported dtype {t.dtype}")
    return codes[t.dtype]


def _stream(t, stream=None):
    import torch
    if stream is not None:
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _dev(t, name):
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")
    return ctypes.c_void_p(t.data_ptr())


def _cache_desc(k_cache):
    nb, bs, hkv, d = k_cache.shape
    return _native.CacheDesc(nb, bs, hkv, d, _dtype_code(k_cache))


def pa_cache_write(k, v, k_cache, v_cache, slot_mapping, stream=None):
    """Scatter new-token rows k, v [T, Hkv, D] into the pools through int64 slots."""
    import torch
    if slot_mapping.dtype != torch.int64:
        raise TypeError("slot_mapping must be int64")
    desc = _cache_desc(k_cache)
    T = int(slot_mapping.numel())
    st = lib().pa_cache_write(_dev(k, "k"), _dev(v, "v"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
                              _dev(slot_mapping, "slot_mapping"), T, ctypes.byref(desc), _stream(k_cache, stream))
    _check(st, "pa_cache_write")


def pa_copy_blocks(k_cache, v_cache, pairs, stream=None):
    """Copy whole blocks src -> dst in both pools; pairs: int32 [n, 2] on the device."""
    import torch
    if pairs.dtype != torch.int32:
        raise TypeError("pairs must be int32")
    desc = _cache_desc(k_cache)
    n = int(pairs.numel() // 2)
    st = lib().pa_copy_blocks(_dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"), _dev(pairs, "pairs"), n,
                              ctypes.byref(desc), _stream(k_cache, stream))
    _check(st, "pa_copy_blocks")


def _reachable(t, name):
    """Device tensor or pinned host tensor (both reachable from kernels)."""
    if not t.is_contiguous() or not (t.is_cuda or t.is_pinned()):
        raise ValueError(f"{name} must be a contiguous CUDA tensor or pinned host tensor")
    return ctypes.c_void_p(t.data_ptr())


def pa_swap_blocks(dst_k, dst_v, src_k, src_v, pairs, stream=None):
    """Copy whole blocks between pools of one block shape (device or pinned
    host memory); pairs: int32 [n, 2] of (source, destination) block ids on
    the device or in pinned host memory."""
    import torch
    if pairs.dtype != torch.int32:
        raise TypeError("pairs must be int32")
    n = int(pairs.numel() // 2)
    if n == 0:
        return
    dev = dst_k if dst_k.is_cuda else src_k
    desc = _native.CacheDesc(0, dst_k.shape[1], dst_k.shape[2], dst_k.shape[3], _dtype_code(dst_k))
    st = lib().pa_swap_blocks(_reachable(dst_k, "dst_k"), _reachable(dst_v, "dst_v"), int(dst_k.shape[0]),
                              _reachable(src_k, "src_k"), _reachable(src_v, "src_v"), int(src_k.shape[0]),
                              _reachable(pairs, "pairs"), n, ctypes.byref(desc), _stream(dev, stream))
    _check(st, "pa_swap_blocks")


def pa_decode_workspace_size(num_seqs, num_heads, head_dim, max_context_len, partition_size=0):
    return int(lib().pa_decode_workspace_size(num_seqs, num_heads, head_dim, max_context_len, partition_size))


def pa_decode(out, q, k_cache, v_cache, block_tables, context_lens, scale, block_size=None, num_kv_heads=None,
              max_context_len=None, partition_size=0, workspace=None, stream=None):
    """One paged decode-attention step.

    q, out: [S, Hq, D]; caches [NB, bs, Hkv, D]; block_tables int32 [S, max_blocks];
    context_lens int32 [S].  ``max_context_len`` bounds every context length
    (default: the table capacity).  ``workspace``: a uint8 CUDA tensor of at
    least pa_decode_workspace_size bytes, allocated here when omitted.
    """
    import torch
    nb, bs, hkv, d = k_cache.shape
    block_size = bs if block_size is None else block_size
    num_kv_heads = hkv if num_kv_heads is None else num_kv_heads
    S, Hq, D = q.shape
    maxb = block_tables.shape[1] if block_tables.dim() == 2 else 1
    if max_context_len is None:
        max_context_len = maxb * block_size
    # the library bounds contexts by the table's capacity as well
    need = pa_decode_workspace_size(S, Hq, D, min(int(max_context_len), maxb * int(block_size)), partition_size)
    ws_ptr, ws_bytes = ctypes.c_void_p(0), 0
    if need:
        if workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        if workspace.numel() < need:
            raise ValueError(f"workspace needs {need} bytes")
        ws_ptr, ws_bytes = ctypes.c_void_p(workspace.data_ptr()), int(workspace.numel())
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise TypeError("block_tables and context_lens must be int32")
    st = lib().pa_decode(_dev(out, "out"), _dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
                         _dev(block_tables, "block_tables"), _dev(context_lens, "context_lens"), float(scale),
                         int(block_size), int(num_kv_heads), S, Hq, D, maxb, int(max_context_len), nb,
                         _dtype_code(q), int(partition_size), ws_ptr, ws_bytes, _stream(q, stream))
    _check(st, "pa_decode")
    return out


def pa_write_decode(k, v, slot_mapping, out, q, k_cache, v_cache, block_tables, context_lens, scale,
                    block_size=None, num_kv_heads=None, max_context_len=None, partition_size=0, workspace=None,
                    stream=None):
    """pa_cache_write of the new rows k, v [T, Hkv, D] through int64 slots, then
    pa_decode, in one call (fewer launches).  Arguments as for those two."""
    import torch
    nb, bs, hkv, d = k_cache.shape
    block_size = bs if block_size is None else block_size
    num_kv_heads = hkv if num_kv_heads is None else num_kv_heads
    S, Hq, D = q.shape
    maxb = block_tables.shape[1] if block_tables.dim() == 2 else 1
    if max_context_len is None:
        max_context_len = maxb * block_size
    # the library bounds contexts by the table's capacity as well
    need = pa_decode_workspace_size(S, Hq, D, min(int(max_context_len), maxb * int(block_size)), partition_size)
    ws_ptr, ws_bytes = ctypes.c_void_p(0), 0
    if need:
        if workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        if workspace.numel() < need:
            raise ValueError(f"workspace needs {need} bytes")
        ws_ptr, ws_bytes = ctypes.c_void_p(workspace.data_ptr()), int(workspace.numel())
    if slot_mapping.dtype != torch.int64:
        raise TypeError("slot_mapping must be int64")
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise TypeError("block_tables and context_lens must be int32")
    T = int(slot_mapping.numel())
    st = lib().pa_write_decode(_dev(k, "k"), _dev(v, "v"), _dev(slot_mapping, "slot_mapping"), T, _dev(out, "out"),
                               _dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
                               _dev(block_tables, "block_tables"), _dev(context_lens, "context_lens"), float(scale),
                               int(block_size), int(num_kv_heads), S, Hq, D, maxb, int(max_context_len), nb,
                               _dtype_code(q), int(partition_size), ws_ptr, ws_bytes, _stream(q, stream))
    _check(st, "pa_write_decode")
    return out


def pa_verify_partition_size(num_seqs, num_queries, num_heads, num_kv_heads, max_context_len, block_size,
                             partition_size=0):
    """The partition (tokens) pa_verify uses for these shapes."""
    return int(lib().pa_verify_partition_size(num_seqs, num_queries, num_heads, num_kv_heads, int(max_context_len),
                                              int(block_size), partition_size))


def pa_verify_workspace_size(num_seqs, num_queries, num_heads, head_dim, max_context_len, partition_size=0):
    return int(lib().pa_verify_workspace_size(num_seqs, num_queries, num_heads, head_dim, max_context_len,
                                              partition_size))


def pa_verify(out, q, k_cache, v_cache, block_tables, context_lens, scale, block_size=None, num_kv_heads=None,
              max_context_len=None, partition_size=0, workspace=None, stream=None):
    """Multi-query paged attention (speculative verification pass).

    q, out: [S, Q, Hq, D]; the K/V of the Q query tokens are the last Q
    positions of each context.  Other arguments as for pa_decode.
    """
    import torch
    nb, bs, hkv, d = k_cache.shape
    block_size = bs if block_size is None else block_size
    num_kv_heads = hkv if num_kv_heads is None else num_kv_heads
    S, Q, Hq, D = q.shape
    maxb = block_tables.shape[1] if block_tables.dim() == 2 else 1
    if max_context_len is None:
        max_context_len = maxb * block_size
    need = pa_verify_workspace_size(S, Q, Hq, D, max_context_len, partition_size)
    ws_ptr, ws_bytes = ctypes.c_void_p(0), 0
    if need:
        if workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        if workspace.numel() < need:
            raise ValueError(f"workspace needs {need} bytes")
        ws_ptr, ws_bytes = ctypes.c_void_p(workspace.data_ptr()), int(workspace.numel())
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise TypeError("block_tables and context_lens must be int32")
    st = lib().pa_verify(_dev(out, "out"), _dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
                         _dev(block_tables, "block_tables"), _dev(context_lens, "context_lens"), float(scale),
                         int(block_size), int(num_kv_heads), S, Q, Hq, D, maxb, int(max_context_len), nb,
                         _dtype_code(q), int(partition_size), ws_ptr, ws_bytes, _stream(q, stream))
    _check(st, "pa_verify")
    return out


def pa_decode_noalloc(out, q, k_cache, v_cache, block_tables, context_lens, scale, block_size=None,
                      num_kv_heads=None, max_context_len=None, partition_size=0, stream=None):
    """pa_decode without a workspace: the library's fixed scratch array is used
    (for callers that cannot allocate device memory; see include/pa.h)."""
    import torch
    nb, bs, hkv, d = k_cache.shape
    block_size = bs if block_size is None else block_size
    num_kv_heads = hkv if num_kv_heads is None else num_kv_heads
    S, Hq, D = q.shape
    maxb = block_tables.shape[1] if block_tables.dim() == 2 else 1
    if max_context_len is None:
        max_context_len = maxb * block_size
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise TypeError("block_tables and context_lens must be int32")
    st = lib().pa_decode_noalloc(_dev(out, "out"), _dev(q, "q"), _dev(k_cache, "k_cache"),
                                 _dev(v_cache, "v_cache"), _dev(block_tables, "block_tables"),
                                 _dev(context_lens, "context_lens"), float(scale), int(block_size),
                                 int(num_kv_heads), S, Hq, D, maxb, int(max_context_len), nb, _dtype_code(q),
                                 int(partition_size), _stream(q, stream))
    _check(st, "pa_decode_noalloc")
    return out


def _step_structs(host, dev, k_cache, scale, max_context_len, partition_size):
    nb, bs, hkv, d = k_cache.shape
    S, Hq, D = host["q"].shape
    T = int(host["slot_mapping"].numel())
    cow = host.get("cow_pairs")
    ncow = 0 if cow is None else int(cow.numel() // 2)
    ptr = lambda t: ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)
    h = _native.StepHost(ptr(host["q"]), ptr(host["k"]), ptr(host["v"]), ptr(host["slot_mapping"]),
                         ptr(host["block_tables"]), ptr(host["context_lens"]), ptr(cow), ptr(host["out"]))
    ws = dev.get("workspace")
    dv = _native.StepDevice(ptr(dev["q"]), ptr(dev["k"]), ptr(dev["v"]), ptr(dev["slot_mapping"]),
                            ptr(dev["block_tables"]), ptr(dev["context_lens"]), ptr(dev.get("cow_pairs")),
                            ptr(dev["out"]), ptr(ws), 0 if ws is None else int(ws.numel()))
    shape = _native.StepShape(S, Hq, hkv, D, bs, nb, int(host["block_tables"].shape[1]), int(max_context_len), T,
                              ncow, _dtype_code(k_cache), float(scale), int(partition_size))
    return h, dv, shape


def pa_step(host, dev, k_cache, v_cache, scale, max_context_len, partition_size=0, stream=None):
    """One layer-step from host buffers (see include/pa.h, pa_step).

    host: dict of pinned CPU tensors q, k, v, slot_mapping, block_tables,
    context_lens, out (and optionally cow_pairs); dev: dict of CUDA tensors of
    the same shapes plus ``workspace``.
    """
    h, dv, shape = _step_structs(host, dev, k_cache, scale, max_context_len, partition_size)
    st = lib().pa_step(ctypes.byref(h), ctypes.byref(dv), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
                       ctypes.byref(shape), _stream(k_cache, stream))
    _check(st, "pa_step")


class Pipeline:
    """pa_step with overlapped host<->device copies (pa_pipeline_*): use
    staging set i % depth for step i; bracket a run of steps with begin/end."""

    def __init__(self, depth=2):
        self._h = ctypes.c_void_p()
        self._destroy = lib().pa_pipeline_destroy
        _check(lib().pa_pipeline_create(int(depth), ctypes.byref(self._h)), "pa_pipeline_create")
        self.depth = int(depth)

    def __del__(self):
        # the destroy call was bound at construction: module globals may already be
        # gone when this runs at interpreter exit
        h = getattr(self, "_h", None)
        destroy = getattr(self, "_destroy", None)
        if h and destroy is not None:
            destroy(h)
            self._h = None

    def begin(self, like, stream=None):
        _check(lib().pa_pipeline_begin(self._h, _stream(like, stream)), "pa_pipeline_begin")

    def step(self, set_index, host, dev, k_cache, v_cache, scale, max_context_len, partition_size=0, stream=None):
        h, dv, shape = _step_structs(host, dev, k_cache, scale, max_context_len, partition_size)
        st = lib().pa_pipeline_step(self._h, int(set_index), ctypes.byref(h), ctypes.byref(dv),
                                    _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"), ctypes.byref(shape),
                                    _stream(k_cache, stream))
        _check(st, "pa_pipeline_step")

    def end(self, like, stream=None):
        _check(lib().pa_pipeline_end(self._h, _stream(like, stream)), "pa_pipeline_end")


def pa_get_device_error(stream=None):
    """Read and clear the device error word; returns the PA_DEVERR_* bits."""
    import torch
    flags = ctypes.c_uint32(0)
    s = ctypes.c_void_p(stream.cuda_stream if stream is not None else torch.cuda.current_stream().cuda_stream)
    st = lib().pa_get_device_error(ctypes.byref(flags), s)
    if st not in (PA_OK, 5):
        _check(st, "pa_get_device_error")
    return int(flags.value)


MATH_AUTO, MATH_SIMT, MATH_TENSOR = 0, 1, 2


def pa_check_wait_expiry(stream=None):
    """Launch the bounded-wait diagnostic (one CTA whose wait must expire after
    about 2 s and set DEVERR_TIMEOUT); read the flag with pa_get_device_error."""
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    _check(lib().pa_check_wait_expiry(ctypes.c_void_p(s.cuda_stream)), "pa_check_wait_expiry")


def set_decode_math(mode):
    """Choose tensor-core (default for fp16/bf16) or CUDA-core decode arithmetic."""
    _check(lib().pa_set_decode_math(int(mode)), "pa_set_decode_math")


def get_decode_math():
    return int(lib().pa_get_decode_math())


MERGE_FUSED, MERGE_KERNEL = 0, 1


def set_split_merge(mode):
    """Merge split partitions with the separate log-sum-exp reduce kernel
    (default) or inside the decode kernel."""
    _check(lib().pa_set_split_merge(int(mode)), "pa_set_split_merge")


def get_split_merge():
    return int(lib().pa_get_split_merge())


VERIFY_MMA_SYNC, VERIFY_TCGEN05, VERIFY_AUTO = 0, 1, 2


def set_verify_kernel(kind):
    """pa_verify's tensor-core path: VERIFY_MMA_SYNC, VERIFY_TCGEN05 or VERIFY_AUTO (default)."""
    _check(lib().pa_set_verify_kernel(int(kind)), "pa_set_verify_kernel")


def get_verify_kernel():
    return int(lib().pa_get_verify_kernel())


def launch_count():
    return int(lib().pa_launch_count())


def profile_begin(kernels=None):
    """Start per-launch event timing, for all kernels or the named ones."""
    if kernels is None:
        _check(lib().pa_profile_begin(), "pa_profile_begin")
    else:
        mask = 0
        for k in kernels:
            mask |= 1 << KERNELS.index(k)
        _check(lib().pa_profile_begin_mask(mask), "pa_profile_begin_mask")


def profile_end():
    """Stop recording; returns {kernel name: (total_ms, launches)}."""
    ms = (ctypes.c_double * len(KERNELS))()
    n = (ctypes.c_int64 * len(KERNELS))()
    _check(lib().pa_profile_end(ms, n), "pa_profile_end")
    return {k: (float(ms[i]), int(n[i])) for i, k in enumerate(KERNELS)}


# ---------------------------------------------------------------------------
# host block manager and scheduler
# ---------------------------------------------------------------------------

def _i32(a):
    return np.ascontiguousarray(a, dtype=np.int32)


def _ptr(a):
    return ctypes.c_void_p(a.ctypes.data) if a is not None and a.size else ctypes.c_void_p(0)


class BlockManager:
    """Free list, reference counts and block tables (pa_bm_*)."""

    def __init__(self, num_blocks, block_size, initial_free_order=None):
        self._h = ctypes.c_void_p()
        self._destroy = lib().pa_bm_destroy
        order = None if initial_free_order is None else _i32(initial_free_order)
        _check(lib().pa_bm_create(num_blocks, block_size, _ptr(order), ctypes.byref(self._h)), "pa_bm_create")
        self.num_blocks, self.block_size = num_blocks, block_size

    def __del__(self):
        # the destroy call was bound at construction: module globals may already be
        # gone when this runs at interpreter exit
        h = getattr(self, "_h", None)
        destroy = getattr(self, "_destroy", None)
        if h and destroy is not None:
            destroy(h)
            self._h = None

    @property
    def handle(self):
        return self._h

    def allocate(self, seq, num_tokens):
        _check(lib().pa_bm_allocate(self._h, seq, num_tokens), "pa_bm_allocate")

    def fork(self, parent, child):
        _check(lib().pa_bm_fork(self._h, parent, child), "pa_bm_fork")

    def append_slot(self, seq):
        slot, src, dst = ctypes.c_int64(), ctypes.c_int32(), ctypes.c_int32()
        _check(lib().pa_bm_append_slot(self._h, seq, ctypes.byref(slot), ctypes.byref(src), ctypes.byref(dst)),
               "pa_bm_append_slot")
        return slot.value, src.value, dst.value

    def free(self, seq):
        _check(lib().pa_bm_free(self._h, seq), "pa_bm_free")

    def block_table(self, seq):
        n = ctypes.c_int()
        lib().pa_bm_block_table(self._h, seq, ctypes.c_void_p(0), 0, ctypes.byref(n))
        out = np.zeros(max(n.value, 1), dtype=np.int32)
        _check(lib().pa_bm_block_table(self._h, seq, _ptr(out), out.size, ctypes.byref(n)), "pa_bm_block_table")
        return out[:n.value].tolist()

    def slots(self, seq, start, count):
        out = np.zeros(max(count, 1), dtype=np.int64)
        _check(lib().pa_bm_slots(self._h, seq, start, count, _ptr(out)), "pa_bm_slots")
        return out[:count]

    def stats(self, seq=-1):
        f, u, c = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
        _check(lib().pa_bm_stats(self._h, seq, ctypes.byref(f), ctypes.byref(u), ctypes.byref(c)), "pa_bm_stats")
        return f.value, u.value, c.value

    @property
    def num_free(self):
        return self.stats()[0]

    def context_len(self, seq):
        c = self.stats(seq)[2]
        if c < 0:
            raise PagedAttentionError(1, "unknown sequence")
        return c

    def ref_count(self, block):
        c = ctypes.c_int()
        _check(lib().pa_bm_ref_count(self._h, block, ctypes.byref(c)), "pa_bm_ref_count")
        return c.value

    def free_list(self):
        out = np.zeros(self.num_blocks, dtype=np.int32)
        n = ctypes.c_int()
        _check(lib().pa_bm_free_list(self._h, _ptr(out), out.size, ctypes.byref(n)), "pa_bm_free_list")
        return out[:n.value].tolist()

    def pack(self, seq_ids, width):
        """Device-layout tables [n, width] (-1 padded) and context lengths [n]."""
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        tables = np.full((len(ids), max(width, 1)), -1, dtype=np.int32)
        lens = np.zeros(len(ids), dtype=np.int32)
        _check(lib().pa_bm_pack(self._h, _ptr(ids), len(ids), width, _ptr(tables), _ptr(lens)), "pa_bm_pack")
        return tables[:, :width], lens

    def usage(self):
        """(blocks held by live sequences, their slots holding a token)."""
        h, f = ctypes.c_int64(), ctypes.c_int64()
        _check(lib().pa_bm_usage(self._h, ctypes.byref(h), ctypes.byref(f)), "pa_bm_usage")
        return h.value, f.value

    # ---- host swap pool (pa_bm_set_cpu_blocks and friends) ----

    def set_cpu_blocks(self, n):
        _check(lib().pa_bm_set_cpu_blocks(self._h, int(n)), "pa_bm_set_cpu_blocks")

    def _swap(self, fn, seq, what):
        n = ctypes.c_int()
        st = fn(self._h, seq, ctypes.c_void_p(0), 0, ctypes.byref(n))
        if st == 0:                       # nothing to move
            return np.zeros((0, 2), dtype=np.int32)
        if n.value <= 0:
            _check(st, what)
        out = np.zeros((n.value, 2), dtype=np.int32)
        _check(fn(self._h, seq, _ptr(out), n.value, ctypes.byref(n)), what)
        return out[:n.value]                # a swap-in may copy fewer blocks than it takes back

    def swap_out(self, seq):
        """(gpu, cpu) block pairs [n, 2] to copy device -> host."""
        return self._swap(lib().pa_bm_swap_out, seq, "pa_bm_swap_out")

    def swap_in(self, seq):
        """(cpu, gpu) block pairs [n, 2] to copy host -> device."""
        return self._swap(lib().pa_bm_swap_in, seq, "pa_bm_swap_in")

    def swapped(self, seq):
        f = ctypes.c_int()
        _check(lib().pa_bm_swapped(self._h, seq, ctypes.byref(f)), "pa_bm_swapped")
        return bool(f.value)

    def cpu_free_list(self):
        n = ctypes.c_int()
        lib().pa_bm_cpu_free_list(self._h, ctypes.c_void_p(0), 0, ctypes.byref(n))
        out = np.zeros(max(n.value, 1), dtype=np.int32)
        _check(lib().pa_bm_cpu_free_list(self._h, _ptr(out), out.size, ctypes.byref(n)), "pa_bm_cpu_free_list")
        return out[:n.value].tolist()

    # ---- prefix cache (pa_bm_enable_prefix_cache and friends) ----

    def enable_prefix_cache(self, enable=True):
        _check(lib().pa_bm_enable_prefix_cache(self._h, int(bool(enable))), "pa_bm_enable_prefix_cache")

    def allocate_prefix(self, seq, tokens):
        """New sequence holding the prompt `tokens`; returns the number of leading
        tokens whose K/V is already cached (a multiple of block_size)."""
        toks = np.ascontiguousarray(tokens, dtype=np.int32)
        cached = ctypes.c_int()
        _check(lib().pa_bm_allocate_prefix(self._h, seq, _ptr(toks), toks.size, ctypes.byref(cached)),
               "pa_bm_allocate_prefix")
        return cached.value

    def append_token(self, seq, token):
        slot, src, dst = ctypes.c_int64(), ctypes.c_int32(), ctypes.c_int32()
        _check(lib().pa_bm_append_token(self._h, seq, int(token), ctypes.byref(slot), ctypes.byref(src),
                                        ctypes.byref(dst)), "pa_bm_append_token")
        return slot.value, src.value, dst.value

    def cache_stats(self):
        """(cached blocks, evictable blocks, block hits, block lookups)."""
        c, e, h, l = ctypes.c_int(), ctypes.c_int(), ctypes.c_int64(), ctypes.c_int64()
        _check(lib().pa_bm_cache_stats(self._h, ctypes.byref(c), ctypes.byref(e), ctypes.byref(h), ctypes.byref(l)),
               "pa_bm_cache_stats")
        return c.value, e.value, h.value, l.value

    def forget(self, block):
        """Drop the cache key of an unreferenced cached block and free it."""
        _check(lib().pa_bm_forget(self._h, int(block)), "pa_bm_forget")

    def evictable(self):
        """Evictable cached blocks, next victim first."""
        out = np.zeros(self.num_blocks, dtype=np.int32)
        n = ctypes.c_int()
        _check(lib().pa_bm_evictable(self._h, _ptr(out), out.size, ctypes.byref(n)), "pa_bm_evictable")
        return out[:n.value].tolist()


class Scheduler:
    """Iteration-level batching over a BlockManager (pa_sched_*)."""

    def __init__(self, bm, max_running, prefix_seq=-1, preempt="recompute", prefix_cache=False,
                 prefix_tokens=None, token_fn=None):
        """``prefix_cache=True`` admits through the block manager's prefix cache
        (pa_sched_enable_prefix_cache): ``prefix_tokens`` are the prefix
        holder's token ids, ``token_fn(seq_id, position)`` gives the token id a
        decode step writes at that position, and requests need their ``tokens``."""
        self.bm = bm           # keeps the block manager alive
        self._h = ctypes.c_void_p()
        self._destroy = lib().pa_sched_destroy
        self._token_cb = None
        _check(lib().pa_sched_create(bm.handle, max_running, prefix_seq, ctypes.byref(self._h)), "pa_sched_create")
        _check(lib().pa_sched_set_preemption(self._h, {"recompute": 0, "swap": 1}[preempt]),
               "pa_sched_set_preemption")
        if prefix_cache:
            if token_fn is None:
                raise ValueError("admission through the prefix cache needs token_fn")
            fn = token_fn
            # kept on self: the library calls it back from every step
            self._token_cb = _native.TokenFn(lambda _ctx, seq, pos: int(fn(seq, pos)))
            toks = np.ascontiguousarray(prefix_tokens if prefix_tokens is not None else [], dtype=np.int32)
            _check(lib().pa_sched_enable_prefix_cache(self._h, _ptr(toks), toks.size, self._token_cb, None),
                   "pa_sched_enable_prefix_cache")

    def __del__(self):
        # the destroy call was bound at construction: module globals may already be
        # gone when this runs at interpreter exit
        h = getattr(self, "_h", None)
        destroy = getattr(self, "_destroy", None)
        if h and destroy is not None:
            destroy(h)
            self._h = None

    def add_request(self, seq_id, prompt_len, output_len, shares_prefix=False, fork_child=-1, fork_output_len=0,
                    tokens=None):
        if tokens is None:
            _check(lib().pa_sched_add_request(self._h, seq_id, prompt_len, output_len, int(bool(shares_prefix)),
                                              fork_child, fork_output_len), "pa_sched_add_request")
            return
        toks = np.ascontiguousarray(tokens, dtype=np.int32)
        if toks.size != prompt_len:
            raise ValueError("prompt tokens and prompt length disagree")
        _check(lib().pa_sched_add_request_tokens(self._h, seq_id, _ptr(toks), prompt_len, output_len,
                                                 int(bool(shares_prefix)), fork_child, fork_output_len),
               "pa_sched_add_request_tokens")

    def step(self, raw=False):
        """Run one iteration; returns the step record as a dict of lists.

        ``raw=True`` leaves the ops as four numpy arrays (``op_kind``: 0 write,
        1 copy-on-write, 2 swap-out, 3 swap-in; ``op_a``, ``op_b``, ``op_c`` as in
        pa_sched_record) instead of a list of tuples, for callers that hand them
        to the device without looking at each one."""
        _check(lib().pa_sched_step(self._h), "pa_sched_step")
        c = _native.SchedCounts()
        _check(lib().pa_sched_counts_get(self._h, ctypes.byref(c)), "pa_sched_counts_get")
        fin = np.zeros(c.num_finished, np.int64)
        adm = np.zeros(c.num_admitted, np.int64)
        pre = np.zeros(c.num_preempted, np.int64)
        kind = np.zeros(c.num_ops, np.int32)
        oa, ob, oc = (np.zeros(c.num_ops, np.int64) for _ in range(3))
        run = np.zeros(c.num_running, np.int64)
        ctx = np.zeros(c.num_running, np.int32)
        _check(lib().pa_sched_record(self._h, _ptr(fin), _ptr(adm), _ptr(pre), _ptr(kind), _ptr(oa), _ptr(ob),
                                     _ptr(oc), _ptr(run), _ptr(ctx)), "pa_sched_record")
        if raw:
            ops = None
        else:
            names = {1: "c", 2: "so", 3: "si"}
            ops = [("w", a, b, cc) if k == 0 else (names[k], a, b)
                   for k, a, b, cc in zip(kind.tolist(), oa.tolist(), ob.tolist(), oc.tolist())]
        n_out, n_in, n_q = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
        _check(lib().pa_sched_swap_counts(self._h, ctypes.byref(n_out), ctypes.byref(n_in), ctypes.byref(n_q)),
               "pa_sched_swap_counts")
        so, si = np.zeros(n_out.value, np.int64), np.zeros(n_in.value, np.int64)
        _check(lib().pa_sched_swap_record(self._h, _ptr(so), _ptr(si)), "pa_sched_swap_record")
        rec = {"finished": fin.tolist(), "admitted": adm.tolist(), "preempted": pre.tolist(), "ops": ops,
               "running": run.tolist(), "context_lens": ctx.tolist(), "num_waiting": c.num_waiting,
               "swapped_out": so.tolist(), "swapped_in": si.tolist(), "num_swapped": n_q.value}
        if raw:
            rec.update(op_kind=kind, op_a=oa, op_b=ob, op_c=oc)
        return rec
