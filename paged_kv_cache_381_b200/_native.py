"""ctypes declarations of libpa.so (include/pa.h).  Loading fails loudly when
the library has not been built: there is no fallback implementation."""

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libpa.so")

c_int, c_int32, c_int64, c_size_t, c_float, c_double, c_void_p, c_uint32 = (
    ctypes.c_int, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float,
    ctypes.c_double, ctypes.c_void_p, ctypes.c_uint32)
P = ctypes.POINTER

# pa_token_fn: token id of (seq_id, position), called back from pa_sched_step
TokenFn = ctypes.CFUNCTYPE(c_int32, c_void_p, c_int64, c_int64)


class CacheDesc(ctypes.Structure):
    _fields_ = [("num_blocks", c_int), ("block_size", c_int), ("num_kv_heads", c_int),
                ("head_dim", c_int), ("dtype", c_int)]


class StepHost(ctypes.Structure):
    _fields_ = [("q", c_void_p), ("k", c_void_p), ("v", c_void_p), ("slot_mapping", c_void_p),
                ("block_tables", c_void_p), ("context_lens", c_void_p), ("cow_pairs", c_void_p),
                ("out", c_void_p)]


class StepDevice(ctypes.Structure):
    _fields_ = [("q", c_void_p), ("k", c_void_p), ("v", c_void_p), ("slot_mapping", c_void_p),
                ("block_tables", c_void_p), ("context_lens", c_void_p), ("cow_pairs", c_void_p),
                ("out", c_void_p), ("workspace", c_void_p), ("workspace_bytes", c_size_t)]


class StepShape(ctypes.Structure):
    _fields_ = [("num_seqs", c_int), ("num_heads", c_int), ("num_kv_heads", c_int), ("head_dim", c_int),
                ("block_size", c_int), ("num_blocks", c_int), ("max_blocks_per_seq", c_int),
                ("max_context_len", c_int), ("num_tokens", c_int), ("num_cow", c_int), ("dtype", c_int),
                ("scale", c_float), ("partition_size", c_int)]


class SchedCounts(ctypes.Structure):
    _fields_ = [("num_finished", c_int), ("num_admitted", c_int), ("num_preempted", c_int),
                ("num_ops", c_int), ("num_running", c_int), ("num_waiting", c_int)]


# name -> (restype, argtypes); must match include/pa.h
SIGNATURES = {
    "pa_cache_write": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int, P(CacheDesc), c_void_p]),
    "pa_decode_workspace_size": (c_size_t, [c_int, c_int, c_int, c_int, c_int]),
    "pa_decode": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_float, c_int, c_int,
                          c_int, c_int, c_int, c_int, c_int, c_int, c_int, c_int, c_void_p, c_size_t, c_void_p]),
    "pa_write_decode": (c_int, [c_void_p, c_void_p, c_void_p, c_int, c_void_p, c_void_p, c_void_p, c_void_p,
                                c_void_p, c_void_p, c_float, c_int, c_int, c_int, c_int, c_int, c_int, c_int,
                                c_int, c_int, c_int, c_void_p, c_size_t, c_void_p]),
    "pa_verify_workspace_size": (c_size_t, [c_int, c_int, c_int, c_int, c_int, c_int]),
    "pa_verify_partition_size": (c_int, [c_int, c_int, c_int, c_int, c_int, c_int, c_int]),
    "pa_verify": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_float, c_int, c_int,
                          c_int, c_int, c_int, c_int, c_int, c_int, c_int, c_int, c_int, c_void_p, c_size_t,
                          c_void_p]),
    "pa_decode_noalloc": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_float, c_int,
                                  c_int, c_int, c_int, c_int, c_int, c_int, c_int, c_int, c_int, c_void_p]),
    "pa_copy_blocks": (c_int, [c_void_p, c_void_p, c_void_p, c_int, P(CacheDesc), c_void_p]),
    "pa_step": (c_int, [P(StepHost), P(StepDevice), c_void_p, c_void_p, P(StepShape), c_void_p]),
    "pa_pipeline_create": (c_int, [c_int, P(c_void_p)]),
    "pa_pipeline_destroy": (None, [c_void_p]),
    "pa_pipeline_begin": (c_int, [c_void_p, c_void_p]),
    "pa_pipeline_step": (c_int, [c_void_p, c_int, P(StepHost), P(StepDevice), c_void_p, c_void_p, P(StepShape),
                                 c_void_p]),
    "pa_pipeline_end": (c_int, [c_void_p, c_void_p]),
    "pa_get_device_error": (c_int, [P(c_uint32), c_void_p]),
    "pa_check_wait_expiry": (c_int, [c_void_p]),
    "pa_status_string": (ctypes.c_char_p, [c_int]),
    "pa_launch_count": (c_int64, []),
    "pa_set_decode_math": (c_int, [c_int]),
    "pa_get_decode_math": (c_int, []),
    "pa_set_split_merge": (c_int, [c_int]),
    "pa_set_verify_kernel": (c_int, [c_int]),
    "pa_get_verify_kernel": (c_int, []),
    "pa_get_split_merge": (c_int, []),
    "pa_profile_begin": (c_int, []),
    "pa_profile_begin_mask": (c_int, [c_uint32]),
    "pa_profile_end": (c_int, [P(c_double), P(c_int64)]),
    "pa_bm_create": (c_int, [c_int, c_int, c_void_p, P(c_void_p)]),
    "pa_bm_destroy": (None, [c_void_p]),
    "pa_bm_allocate": (c_int, [c_void_p, c_int64, c_int]),
    "pa_bm_fork": (c_int, [c_void_p, c_int64, c_int64]),
    "pa_bm_append_slot": (c_int, [c_void_p, c_int64, P(c_int64), P(c_int32), P(c_int32)]),
    "pa_bm_free": (c_int, [c_void_p, c_int64]),
    "pa_bm_block_table": (c_int, [c_void_p, c_int64, c_void_p, c_int, P(c_int)]),
    "pa_bm_slots": (c_int, [c_void_p, c_int64, c_int, c_int, c_void_p]),
    "pa_bm_stats": (c_int, [c_void_p, c_int64, P(c_int), P(c_int), P(c_int)]),
    "pa_bm_ref_count": (c_int, [c_void_p, c_int32, P(c_int)]),
    "pa_bm_free_list": (c_int, [c_void_p, c_void_p, c_int, P(c_int)]),
    "pa_bm_pack": (c_int, [c_void_p, c_void_p, c_int, c_int, c_void_p, c_void_p]),
    "pa_bm_usage": (c_int, [c_void_p, P(c_int64), P(c_int64)]),
    "pa_bm_set_cpu_blocks": (c_int, [c_void_p, c_int]),
    "pa_bm_swap_out": (c_int, [c_void_p, c_int64, c_void_p, c_int, P(c_int)]),
    "pa_bm_swap_in": (c_int, [c_void_p, c_int64, c_void_p, c_int, P(c_int)]),
    "pa_bm_swapped": (c_int, [c_void_p, c_int64, P(c_int)]),
    "pa_bm_cpu_free_list": (c_int, [c_void_p, c_void_p, c_int, P(c_int)]),
    "pa_swap_blocks": (c_int, [c_void_p, c_void_p, c_int, c_void_p, c_void_p, c_int, c_void_p, c_int, P(CacheDesc),
                               c_void_p]),
    "pa_bm_enable_prefix_cache": (c_int, [c_void_p, c_int]),
    "pa_bm_allocate_prefix": (c_int, [c_void_p, c_int64, c_void_p, c_int, P(c_int)]),
    "pa_bm_append_token": (c_int, [c_void_p, c_int64, c_int32, P(c_int64), P(c_int32), P(c_int32)]),
    "pa_bm_cache_stats": (c_int, [c_void_p, P(c_int), P(c_int), P(c_int64), P(c_int64)]),
    "pa_bm_evictable": (c_int, [c_void_p, c_void_p, c_int, P(c_int)]),
    "pa_sched_create": (c_int, [c_void_p, c_int, c_int64, P(c_void_p)]),
    "pa_sched_destroy": (None, [c_void_p]),
    "pa_sched_add_request": (c_int, [c_void_p, c_int64, c_int, c_int, c_int, c_int64, c_int]),
    "pa_sched_step": (c_int, [c_void_p]),
    "pa_sched_set_preemption": (c_int, [c_void_p, c_int]),
    "pa_sched_swap_counts": (c_int, [c_void_p, P(c_int), P(c_int), P(c_int)]),
    "pa_sched_swap_record": (c_int, [c_void_p, c_void_p, c_void_p]),
    "pa_sched_counts_get": (c_int, [c_void_p, P(SchedCounts)]),
    "pa_sched_record": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                c_void_p, c_void_p, c_void_p]),
    "pa_bm_forget": (c_int, [c_void_p, c_int32]),
    "pa_sched_enable_prefix_cache": (c_int, [c_void_p, c_void_p, c_int, TokenFn, c_void_p]),
    "pa_sched_add_request_tokens": (c_int, [c_void_p, c_int64, c_void_p, c_int, c_int, c_int, c_int64, c_int]),
}

_lib = None


def load():
    """Load libpa.so once and declare every entry point."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m paged_kv_cache_381_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib
