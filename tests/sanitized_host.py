"""pytest plugin: serve the block manager and scheduler calls (pa_bm_*,
pa_sched_*) from a copy of the host sources built with AddressSanitizer and
UndefinedBehaviorSanitizer, named by PA_SANITIZED_HOST_LIB; every other call
goes to the regular library.  Loaded by test_host_sanitizers in a child
process that has the sanitizer runtimes preloaded."""

import ctypes
import os

from paged_kv_cache_381_b200 import _native

_san = ctypes.CDLL(os.environ["PA_SANITIZED_HOST_LIB"])
_reg = ctypes.CDLL(_native.LIB_PATH)


class _Mixed:
    def __getattr__(self, name):
        src = _san if name.startswith(("pa_bm_", "pa_sched_")) else _reg
        fn = getattr(src, name)
        if name in _native.SIGNATURES:
            fn.restype, fn.argtypes = _native.SIGNATURES[name]
        setattr(self, name, fn)
        return fn


_native._lib = _Mixed()
