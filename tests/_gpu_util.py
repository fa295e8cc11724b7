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
