"""Comparison helpers shared by the GPU parity tests.

Attention outputs are checked against the float64 oracle elementwise with
|y - ref| <= 2e-3 + 1e-2 * |ref| (max abs 2e-3, relative 1e-2, in allclose
form: at context 1 the output is a value row of size up to ~4, where one bf16
half-ulp is already 2^-7, so a pure absolute bound would reject a correctly
rounded answer), and per (sequence, head) row with relative L2 error <= 1e-2,
which keeps the check meaningful when long flat softmaxes shrink outputs
towards zero.
"""

import numpy as np

ATOL = 2e-3
RTOL = 1e-2
ROW_REL_L2 = 1e-2


def out_to_f64(t, dtype: str) -> np.ndarray:
    """GPU output tensor -> float64 via its 16-bit patterns (decoded exactly)."""
    import torch
    bits = t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
    if dtype == "f16":
        return bits.view(np.float16).astype(np.float64)
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def tensor_bits(t) -> np.ndarray:
    import torch
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def assert_close(got: np.ndarray, ref: np.ndarray, what: str = ""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = np.abs(got - ref)
    bound = ATOL + RTOL * np.abs(ref)
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(f"{what}: {bad.sum()} elements out of tolerance; worst at {i}: "
                             f"got {got[i]!r} ref {ref[i]!r} (max abs err {err.max():.3e})")
    d = ref.shape[-1]
    num = np.linalg.norm((got - ref).reshape(-1, d), axis=1)
    den = np.linalg.norm(ref.reshape(-1, d), axis=1)
    rel = num / np.maximum(den, 1e-30)
    assert (rel <= ROW_REL_L2).all(), f"{what}: row relative L2 error {rel.max():.3e}"
    return float(err.max()), float(rel.max())
