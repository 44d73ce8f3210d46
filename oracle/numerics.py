"""Exact widening of stored KV / query values to float64 (oracle; test
infrastructure only).

Storage convention shared with the seeded input generators: ``"f32"`` arrays
are ``numpy.float32``; ``"f16"`` and ``"bf16"`` arrays hold the raw 16-bit
patterns as ``numpy.uint16``.  Widening is exact for all three formats, so the
oracle sees precisely the values the kernels read.

bfloat16 is, by definition, the upper half of an IEEE-754 binary32 word
(sign, 8 exponent bits, 7 mantissa bits); its value is recovered by shifting
the 16 stored bits into the top of a 32-bit word.  binary16 is widened by
numpy's own half-precision conversion.

The pages say the KV cache stays in 16-bit floating point even when weights are
quantised ([P3] "大模型推理显存优化实战：PagedAttention机制原理与vLLM连续批处理配置",
section "生产部署注意事项": KV Cache 仍以FP16存储), which is why the 16-bit
formats are the production ones; float32 is the exact-parity test format.
"""

import numpy as np

DTYPES = ("f32", "f16", "bf16")
ELEMENT_BYTES = {"f32": 4, "f16": 2, "bf16": 2}


def storage_dtype(dtype):
    """numpy dtype used to hold stored values of ``dtype``."""
    if dtype == "f32":
        return np.float32
    if dtype in ("f16", "bf16"):
        return np.uint16
    raise ValueError(f"unknown dtype {dtype!r}")


def widen(stored, dtype):
    """Return ``stored`` (values of ``dtype`` in storage form) as float64."""
    a = np.asarray(stored)
    if dtype == "f32":
        if a.dtype == np.uint32:
            a = a.view(np.float32)
        if a.dtype != np.float32:
            raise TypeError("f32 storage must be float32")
        return a.astype(np.float64)
    if a.dtype != np.uint16:
        raise TypeError(f"{dtype} storage must be uint16 bit patterns")
    if dtype == "f16":
        return a.view(np.float16).astype(np.float64)
    if dtype == "bf16":
        with np.errstate(invalid="ignore"):      # NaN patterns stay NaN
            return (a.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    raise ValueError(f"unknown dtype {dtype!r}")
