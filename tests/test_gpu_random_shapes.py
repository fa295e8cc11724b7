"""GPU parity on seeded random shapes.

The other GPU tests use the workloads' sizes and hand-picked edge shapes.
Here every call of the path runs on shapes drawn at random from the whole
accepted range, so that no size class is covered by hand-picked cases alone:
T from 1 to a few thousand, K from 1 to 16 (powers of two or not), E up to
512 and a multiple of R, H any multiple of 8 (every other shape a multiple
of 128, so that the E4M3 calls run too), uniform or Zipf routing.  Each call
is held to the same bar as in its own tests: layout, permuted bytes,
counters, grad_y, E4M3 codes and scales bit-exact against the oracle;
combine and dispatch_bwd within one bf16 ulp of the exact sum except proven
cancellation cases; grad_scales within the fp32 dot-product bound.
"""
import numpy as np
import pytest
import torch

import oracle
from _gpu_util import dev_u16, ensure_lib
from combine_moe_dispatch_05_b200 import ops
from combine_moe_dispatch_05_b200 import workloads as W
from test_gpu_combine import check_combine, check_combine_bwd, check_dispatch_bwd
from test_gpu_dispatch import check_counters, check_layout, run_permute_bf16, run_permute_fp8
from test_gpu_dispatch_fused import _fused_and_separate_bf16
from test_gpu_quant_dispatch import run as run_fused_quant

pytestmark = pytest.mark.gpu
DEV = "cuda"
N_SHAPES = 32
MAX_ELEMS = 24_000_000  # bound on T*K*H, so each oracle call takes about a second


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_lib()


def draw_shape(i: int) -> W.Spec:
    rng = np.random.default_rng(20261203 + i)
    while True:
        K = int(rng.integers(1, 17))
        R = int(rng.choice([1, 2, 3, 4, 5, 8, 16]))
        E = R * int(rng.integers(1, 512 // R + 1))
        if E < K:
            continue
        T = int(rng.choice([1, 2, 7])) if rng.random() < 0.15 else int(rng.integers(1, 6001))
        H = 128 * int(rng.integers(1, 41)) if i % 2 == 0 else 8 * int(rng.integers(1, 701))
        if T * K * H > MAX_ELEMS:
            continue
        if rng.random() < 0.5:
            return W.Spec(f"rand{i}", T, H, E, K, R, "zipf", zipf_s=float(rng.uniform(0.3, 1.3)),
                          seed=31000 + i)
        return W.Spec(f"rand{i}", T, H, E, K, R, "uniform", seed=31000 + i)


def test_shapes_span_the_range():
    shapes = [draw_shape(i) for i in range(N_SHAPES)]
    assert len({s.K for s in shapes}) >= 6
    assert any(s.K & (s.K - 1) for s in shapes)           # K not a power of two
    assert any(s.H % 128 for s in shapes) and any(s.H % 128 == 0 for s in shapes)
    assert max(s.E for s in shapes) >= 256 and min(s.T for s in shapes) <= 7


@pytest.mark.parametrize("i", range(N_SHAPES))
def test_random_shape_every_call(i):
    s = draw_shape(i)
    check_layout(W.topk_ids(s), s.E, s.R)

    x = W.tokens(s)
    L, ref, xp, xp_ref = run_permute_bf16(s, x)
    assert np.array_equal(dev_u16(xp), xp_ref)
    check_counters(L, ref)
    _fused_and_separate_bf16(s, x.to(DEV))  # the one-call dispatch equals the two calls

    check_combine(s, shared=(i % 3 == 0))
    check_combine_bwd(s)
    check_dispatch_bwd(s)

    if s.H % 128 == 0:
        codes, xs = W.e4m3_codes(s), W.block_scales(s)
        _, _, xp8, xps8, xp8_ref, xps8_ref = run_permute_fp8(s, codes, xs)
        assert np.array_equal(xp8.cpu().numpy(), xp8_ref)
        assert np.array_equal(xps8.cpu().numpy().view(np.uint32), xps8_ref.view(np.uint32))
        q, qs = ops.moe_quantize_e4m3(x.to(DEV))
        q_ref, s_ref = oracle.quantize_e4m3(W.as_u16(x))
        assert np.array_equal(q.cpu().numpy(), q_ref)
        assert np.array_equal(qs.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
        run_fused_quant(s)
