"""Helpers shared by the GPU parity tests: run a workload through the CUDA
library (via its Python binding) and through the CPU oracle on the same
seeded inputs, and the tolerances the comparisons use."""
import numpy as np
import torch

from combine_moe_dispatch_05_b200 import build as B
from combine_moe_dispatch_05_b200 import ops
from combine_moe_dispatch_05_b200 import workloads as W

U32 = 2.0 ** -24  # fp32 unit roundoff


def ensure_lib():
    B.build()
    return ops.lib()


def f64(u16: np.ndarray) -> np.ndarray:
    return W.from_u16(u16).to(torch.float64).numpy()


def dev_u16(t: torch.Tensor) -> np.ndarray:
    """bf16 CUDA tensor -> uint16 bits on the host."""
    return W.as_u16(t.cpu())


def gamma(n: int) -> float:
    return n * U32 / (1 - n * U32)


def assert_bf16_close(got: np.ndarray, ref: np.ndarray, mag: np.ndarray, n_terms: int,
                      what: str):
    """got, ref: uint16 bf16 bits; mag: float64 sum of |terms| per element.

    Bound: the oracle value is the exact sum rounded once to bf16; the kernel
    rounds an fp32 running sum of n_terms terms, whose error is at most
    gamma(n_terms) * mag.  Two roundings of values that far apart differ by at
    most that distance plus one bf16 ulp (<= 2^-7 |ref|)."""
    g, r = f64(got), f64(ref)
    tol = 2.0 ** -7 * np.abs(r) + gamma(n_terms) * mag + 2.0 ** -133
    err = np.abs(g - r)
    bad = err > tol
    assert not bad.any(), (f"{what}: {bad.sum()} elements out of tolerance; "
                           f"worst err {err.max():.3g} at ref {r.flat[err.argmax()]:.3g}")
    return float(np.mean(got == ref))


def exact_sum_and_mag(y_u16: np.ndarray, dst_row: np.ndarray, scales: np.ndarray,
                      shared_u16=None, chunk: int = 256):
    """fp64 exact sum_k s_k * y[dst_row[t, k]] (+ shared) and sum of |terms|,
    per output element, formed a few hundred tokens at a time."""
    T, K = scales.shape
    H = y_u16.shape[1]
    rows = np.asarray(dst_row)[:T * K].reshape(T, K)
    exact = np.empty((T, H), np.float64)
    mag = np.empty((T, H), np.float64)
    for a in range(0, T, chunk):
        b = min(T, a + chunk)
        yv = f64(y_u16[rows[a:b]])                                  # [c, K, H]
        sv = scales[a:b].astype(np.float64)
        exact[a:b] = np.einsum("tk,tkh->th", sv, yv)
        mag[a:b] = np.einsum("tk,tkh->th", np.abs(sv), np.abs(yv))
        if shared_u16 is not None:
            sh = f64(shared_u16[a:b])
            exact[a:b] += sh
            mag[a:b] += np.abs(sh)
    return exact, mag


def assert_one_ulp_except_cancellation(got: np.ndarray, exact: np.ndarray, mag: np.ndarray,
                                       n_terms: int, what: str) -> int:
    """The stated accuracy target, element by element: |got - exact| <=
    2^-7 |exact| (one bf16 ulp).  An fp32 running sum of n terms is within
    gamma_n * sum|terms| of the exact sum, and one rounding to bf16 adds at
    most 2^-8 of its magnitude, so an element can exceed one ulp only when
    |exact| < 257 * gamma_n * sum|terms| (cancellation).  Every element over
    one ulp must be such a case and stay within the accumulation bound.
    Returns how many elements are over one ulp."""
    g = f64(got)
    err = np.abs(g - exact)
    gam = gamma(n_terms)
    over = err > 2.0 ** -7 * np.abs(exact)
    cancel = np.abs(exact) < 257 * gam * mag + 2.0 ** -126
    bad = over & ~cancel
    assert not bad.any(), (f"{what}: {int(bad.sum())} elements over one ulp of the exact sum "
                           f"without cancellation; worst err {err[bad].max():.3g}")
    beyond = over & (err > 2.0 ** -7 * np.abs(exact) + gam * mag + 2.0 ** -133)
    assert not beyond.any(), f"{what}: {int(beyond.sum())} elements beyond the fp32 bound"
    return int(over.sum())
