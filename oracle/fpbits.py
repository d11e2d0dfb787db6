"""Exact decode of 16-bit floating-point bit patterns to float64 (oracle side).

Both half (IEEE binary16) and bfloat16 values are exactly representable in
float64, so decoding loses nothing. NumPy's own float16 type decodes half;
bfloat16 is the upper 16 bits of a float32, so shifting the pattern into the
high half of a 32-bit word and reinterpreting it gives the value.
"""

import numpy as np


def bits_to_f64(bits, dtype: str) -> np.ndarray:
    bits = np.asarray(bits, dtype=np.uint16)
    if dtype == "f16":
        return bits.view(np.float16).astype(np.float64)
    if dtype == "bf16":
        return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    raise ValueError(f"unknown dtype {dtype!r}")
