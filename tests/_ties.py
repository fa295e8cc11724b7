"""Inputs whose products s * g land on bf16 rounding midpoints.

grad_y = bf16(s * g) must be the exact product rounded once.  Rounding the
fp32 product first gives a different bf16 value only when that fp32 product
is exactly a midpoint between two bf16 values while the exact product is
not.  Random data reaches that case about once in 65536 products; these
inputs reach it in most of them.  g = +-3 * 2^j (exact in bf16), and
s = fp32(m / 3) for a bf16 midpoint m in [1, 2), so s * g = m * 2^j plus the
small error of s.  When that error is under half an fp32 ulp of m, the fp32
product is m * 2^j: a midpoint reached by rounding.
"""
import numpy as np


def midpoint_products(T: int, K: int, H: int, seed: int):
    """(scales fp32 [T, K], g as fp32 [T, H] holding exact bf16 values)."""
    rng = np.random.default_rng(seed)
    i = rng.integers(0, 128, size=(T, K))
    m = 1.0 + (2 * i + 1) * 2.0 ** -8                          # bf16 midpoints in [1, 2)
    s = (m / 3.0).astype(np.float32) * np.float32(2.0) ** rng.integers(-3, 1, size=(T, K))
    j = rng.integers(-6, 7, size=(T, H))
    sign = np.where(rng.random((T, H)) < 0.5, -1.0, 1.0)
    g = (sign * 3.0 * 2.0 ** j).astype(np.float32)
    return s.astype(np.float32), g


def fraction_on_midpoints(s: np.ndarray, g: np.ndarray) -> float:
    """Share of the products s[t, k] * g[t, h] whose fp32 rounding is a bf16
    midpoint while the exact product differs from it."""
    p = (s[:, :, None] * g[:, None, :]).astype(np.float32)     # fp32 products
    bits = p.view(np.uint32)
    exact = s.astype(np.float64)[:, :, None] * g.astype(np.float64)[:, None, :]
    return float(np.mean(((bits & 0xFFFF) == 0x8000) & (exact != p.astype(np.float64))))
