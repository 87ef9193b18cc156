"""Widening of stored 16-bit floats to float64 (exact), oracle-side."""
import numpy as np


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """bfloat16 storage bits (uint16) -> float64.  A bf16 value is the top half
    of the float32 with the same bits, so the widening is exact."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def f16_to_f64(bits: np.ndarray) -> np.ndarray:
    """IEEE half storage bits (uint16) -> float64 (exact)."""
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)
