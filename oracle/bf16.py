"""bf16 round-to-nearest-even on numpy arrays (oracle; test infrastructure only).

bf16 keeps the fp32 exponent and 8 significant bits.  Rounding is done on
the bit pattern: add half an ulp (minus one, plus the kept lsb, which is the
ties-to-even rule) and clear the dropped bits.  Values stay finite for the
magnitudes in this workload; NaN and overflow are not handled.
"""
from __future__ import annotations

import numpy as np


def f32_to_bf16_bits(x) -> np.ndarray:
    """fp32 -> bf16 bit pattern (uint16), round to nearest even."""
    b = np.ascontiguousarray(np.asarray(x, dtype=np.float32)).view(np.uint32).astype(np.uint64)
    lsb = (b >> np.uint64(16)) & np.uint64(1)
    b = (b + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    return b.astype(np.uint16)


def bf16_bits_to_f32(bits) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32)


def round_f32(x) -> np.ndarray:
    """fp32 values rounded to bf16, returned as fp32."""
    return bf16_bits_to_f32(f32_to_bf16_bits(x))


def round_f64(x) -> np.ndarray:
    """float64 values rounded directly (one rounding) to bf16, returned as float64."""
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    b = a.view(np.uint64)
    lsb = (b >> np.uint64(45)) & np.uint64(1)
    b = (b + np.uint64((1 << 44) - 1) + lsb) & ~np.uint64((1 << 45) - 1)
    return b.view(np.float64)


def ident(x):
    return np.asarray(x, dtype=np.float64)
