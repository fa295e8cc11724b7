"""Pins for the oracle's combine, combine backward, dispatch backward and the
E4M3 per-128-channel quantiser.

Against: a hand-worked example (tests/golden), closed forms (one-hot scales
return the routed row; zero scales return the shared row; equal rows c give
c * sum(s)), numpy float64 reductions with torch's own bf16 rounding as an
independent library route, the adjoint identity of a linear map, the exact
identity dispatch_bwd(dispatch(x)) = K x for K a power of two, and the E4M3
error bound.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from combine_moe_dispatch_05_b200 import workloads as W

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def f64(u16):
    return W.from_u16(u16).to(torch.float64).numpy()


def bf16_bits(a64):
    """float64 -> float32 -> bf16 via torch (a second, double-rounding route)."""
    return W.as_u16(torch.from_numpy(np.ascontiguousarray(a64)).to(torch.float32).to(torch.bfloat16))


def bf16_ulp(v):
    a = np.abs(v)
    e = np.floor(np.log2(np.where(a > 0, a, 2.0**-126)))
    return 2.0 ** (np.maximum(e, -126) - 7)


def setup(T, K, E, H, seed, R=1, shared=False):
    s = W.Spec("t", T, H, E, K, R, "uniform", seed=seed)
    ids = W.topk_ids(s).numpy()
    L = oracle.layout(ids, E, R)
    y = W.as_u16(W.expert_out(s, L.P_cap))
    sc = W.topk_scales(s).numpy()
    sh = W.as_u16(W.shared_out(s)) if shared else None
    return s, ids, L, y, sc, sh


def test_golden_hand_worked_combine():
    g = json.load(open(os.path.join(GOLD, "combine_T2_K2_H4.json")))
    ids = np.array(g["ids"], np.int32)
    L = oracle.layout(ids, g["E"], g["R"])
    assert L.dst_row.tolist() == g["dst_row"]
    y = np.zeros((L.P_cap, g["H"]), np.uint16)
    for r, vals in g["y_rows"].items():
        y[int(r)] = [oracle.bf16_encode(v) for v in vals]
    sc = np.array(g["scales"], np.float32)
    sh = np.array([[oracle.bf16_encode(v) for v in row] for row in g["shared"]], np.uint16)
    out = oracle.combine(y, L.dst_row, sc, sh)
    assert np.array_equal(f64(out), np.array(g["out_with_shared"]))
    out = oracle.combine(y, L.dst_row, sc, None)
    assert np.array_equal(f64(out), np.array(g["out_without_shared"]))


@pytest.mark.parametrize("shared", [False, True])
def test_combine_matches_numpy_float64(shared):
    s, ids, L, y, sc, sh = setup(97, 3, 7, 136, 5, shared=shared)
    out = oracle.combine(y, L.dst_row, sc, sh)
    T, K = sc.shape
    gathered = f64(y)[L.dst_row.reshape(T, K)]                       # [T, K, H]
    exact = np.einsum("tk,tkh->th", sc.astype(np.float64), gathered)
    if shared:
        exact = exact + f64(sh)
    got = f64(out)
    assert np.all(np.abs(got - exact) <= 0.5 * bf16_ulp(exact) + 1e-300)  # correctly rounded
    alt = f64(bf16_bits(exact))                                      # torch rounding route
    assert np.all(np.abs(got - alt) <= bf16_ulp(exact))
    assert np.mean(got == alt) > 0.999


def test_combine_one_hot_returns_routed_row_exactly():
    s, ids, L, y, sc, _ = setup(64, 4, 9, 64, 6)
    T, K = sc.shape
    for kk in range(K):
        oh = np.zeros_like(sc)
        oh[:, kk] = 1.0
        out = oracle.combine(y, L.dst_row, oh, None)
        assert np.array_equal(out, y[L.dst_row.reshape(T, K)[:, kk]])


def test_combine_zero_scales_returns_shared_and_constant_rows():
    s, ids, L, y, sc, sh = setup(50, 2, 4, 32, 7, shared=True)
    out = oracle.combine(y, L.dst_row, np.zeros_like(sc), sh)
    assert np.array_equal(out, sh)
    c = oracle.bf16_encode(1.5)
    yc = np.full_like(y, c)
    out = oracle.combine(yc, L.dst_row, sc, None)
    expect = 1.5 * sc.astype(np.float64).sum(1)
    for t in range(50):
        assert np.all(out[t] == oracle.bf16_encode(expect[t]))


def test_combine_bwd_grad_scales_and_grad_y():
    s, ids, L, y, sc, _ = setup(61, 3, 5, 72, 8)
    T, K = sc.shape
    g = W.as_u16(W.grad_out(s))
    gy = np.full((L.P_cap, s.H), 0x7777, np.uint16)
    gs = oracle.combine_bwd(g, y, sc, L.dst_row, L.counts, L.offsets, gy)
    rows = L.dst_row.reshape(T, K)
    dots = np.einsum("th,tkh->tk", f64(g), f64(y)[rows])
    assert np.allclose(gs, dots.astype(np.float32), rtol=0, atol=1e-6 * np.abs(dots).max())
    exact = sc.astype(np.float64)[:, :, None] * f64(g)[:, None, :]   # [T, K, H]
    got = f64(gy)[rows]
    assert np.all(np.abs(got - exact) <= 0.5 * bf16_ulp(exact) + 1e-300)
    pad = [p for p in range(L.P) if L.row_src[p] < 0]
    assert np.all(gy[pad] == 0)
    assert np.all(gy[L.P:] == 0x7777)


def _bf16_nearest_rational(q):
    """bf16 bits of the value nearest the rational q, ties to the even code
    (normal range only): exact arithmetic, no floating point."""
    from fractions import Fraction
    sign = 0x8000 if q < 0 else 0
    a = abs(Fraction(q))
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    ulp = Fraction(2) ** (e - 7)
    n = a / ulp                                      # in [128, 256)
    fl = n.numerator // n.denominator
    rem = n - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    bits = int(np.float32(float(fl * ulp)).view(np.uint32)) >> 16
    return sign | bits


def test_combine_bwd_grad_y_single_rounding_on_midpoint_products():
    """grad_y = bf16(s * g) rounded once from the exact product.  On inputs
    whose fp32 products are bf16 midpoints (tests/_ties.py) the oracle must
    match an exact rational rounding, and rounding the fp32 product again (a
    plausible mistake) must differ from it on many elements."""
    from fractions import Fraction

    from _ties import fraction_on_midpoints, midpoint_products
    T, K, H, E = 6, 2, 40, 4
    sc, gf = midpoint_products(T, K, H, seed=12)
    assert fraction_on_midpoints(sc, gf) > 0.3
    g = (gf.view(np.uint32) >> 16).astype(np.uint16)          # exact: gf holds bf16 values
    ids = np.array([[t % E, (t + 1) % E] for t in range(T)], np.int32)
    L = oracle.layout(ids, E, 1)
    y = np.zeros((L.P_cap, H), np.uint16)
    gy = np.zeros((L.P_cap, H), np.uint16)
    oracle.combine_bwd(g, y, sc, L.dst_row, L.counts, L.offsets, gy)
    rows = L.dst_row.reshape(T, K)
    twice = W.as_u16(torch.from_numpy(sc[:, :, None] * gf[:, None, :]).to(torch.bfloat16))
    differ = 0
    for t in range(T):
        for k in range(K):
            for h in range(H):
                want = _bf16_nearest_rational(Fraction(float(sc[t, k])) * Fraction(float(gf[t, h])))
                assert gy[rows[t, k], h] == want, (t, k, h)
                differ += int(twice[t, k, h] != want)
    assert differ > 0.1 * T * K * H


def test_combine_bwd_adjoint_identity():
    """<combine(y), g> == <y, grad_y> and d<combine, g>/ds = grad_s (linearity)."""
    s, ids, L, y, sc, _ = setup(40, 4, 6, 48, 9)
    g = W.as_u16(W.grad_out(s))
    gy = np.zeros((L.P_cap, s.H), np.uint16)
    gs = oracle.combine_bwd(g, y, sc, L.dst_row, L.counts, L.offsets, gy)
    out = oracle.combine(y, L.dst_row, sc, None)
    lhs = (f64(out) * f64(g)).sum()
    rhs = (f64(y) * f64(gy)).sum()
    bound = 2 * 2.0**-8 * (np.abs(f64(out) * f64(g)).sum() + np.abs(f64(y) * f64(gy)).sum())
    assert abs(lhs - rhs) <= bound
    rhs_s = (gs.astype(np.float64) * sc).sum()
    assert abs(lhs - rhs_s) <= bound


@pytest.mark.parametrize("K", [1, 2, 4, 8])
def test_dispatch_bwd_of_dispatch_is_K_times_x(K):
    E, T, H = 9, 83, 40
    s = W.Spec("t", T, H, E, K, 1, "uniform", seed=100 + K)
    ids = W.topk_ids(s).numpy()
    L = oracle.layout(ids, E, 1)
    x = W.as_u16(W.tokens(s))
    xp = np.zeros((L.P_cap, H), np.uint16)
    oracle.permute_rows(x, L.dst_row, K, L.counts, L.offsets, xp)
    gx = oracle.dispatch_bwd(xp, L.dst_row, T, K)
    assert np.array_equal(f64(gx), K * f64(x))


def test_dispatch_bwd_matches_numpy():
    s, ids, L, y, sc, _ = setup(70, 3, 6, 56, 10)
    T, K = sc.shape
    gx = oracle.dispatch_bwd(y, L.dst_row, T, K)
    exact = f64(y)[L.dst_row.reshape(T, K)].sum(1)
    assert np.all(np.abs(f64(gx) - exact) <= 0.5 * bf16_ulp(exact) + 1e-300)


# ------------------------------------------------------------ quantiser ---
def test_quantize_matches_torch_fp32_route_and_bounds():
    s = W.config(3).with_(T=64, H=1024)
    x = W.tokens(s)
    q, sc = oracle.quantize_e4m3(W.as_u16(x))
    xf = x.to(torch.float32).view(64, 8, 128)
    amax = xf.abs().amax(-1, keepdim=True)
    st = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    qt = (xf / st).to(torch.float8_e4m3fn).view(torch.uint8).view(64, 1024).numpy()
    assert np.array_equal(sc, st.view(64, 8).numpy())
    assert np.array_equal(q, qt)
    # the block maximum maps to +-448 exactly
    idx = xf.abs().argmax(-1)
    codes = q.reshape(64, 8, 128)
    top = np.take_along_axis(codes, idx.numpy()[..., None], -1)[..., 0]
    assert np.all((top & 0x7F) == 0x7E)
    deq = oracle.dequantize_e4m3(q, sc).reshape(64, 8, 128)
    xv = xf.numpy()
    r = np.abs(xv) / st.numpy()
    normal = r >= 2.0**-6
    err = np.abs(deq - xv)
    assert np.all(err[normal] <= 2.0**-4 * np.abs(xv[normal]) * (1 + 1e-6))
    sub_bound = (2.0**-10 * st.numpy() * (1 + 1e-6)) * np.ones_like(xv)
    assert np.all(err[~normal] <= sub_bound[~normal])


def test_quantize_zero_block_and_saturation():
    x = np.zeros((2, 256), np.uint16)
    x[1, 128:] = oracle.bf16_encode(-3.0)
    q, s = oracle.quantize_e4m3(x)
    assert np.array_equal(s, np.array([[1.0, 1.0], [1.0, np.float32(3.0) / np.float32(448.0)]], np.float32))
    assert np.all(q[0] == 0) and np.all(q[1, :128] == 0)
    assert np.all(q[1, 128:] == 0xFE)                                # -448
