"""GPU parity: combine, combine backward and dispatch backward against the CPU
oracle, on the workloads' sizes and on ragged edge shapes.

Tolerance (bf16 outputs of combine and dispatch_bwd): the oracle rounds the
exact sum once; the kernel rounds an fp32 running sum, so
|gpu - ref| <= 2^-7 |ref| + gamma_n * sum|terms| (see
_gpu_util.assert_bf16_close), and against the exact sum every element is
within one bf16 ulp (2^-7 |exact|) unless it is a cancellation case, where
|exact| < 257 gamma_n sum|terms| (_gpu_util.assert_one_ulp_except_cancellation).
In practice nearly every element is bit-identical, which the tests also
report.  grad_y is the exact product rounded once on both sides, so it is
compared for equality.  grad_scales is an fp32 dot product over H terms in a
fixed but different order than the oracle's double sum:
|err| <= gamma_H * sum_h |g_h y_h| + 2^-24 |ref|.
"""
import os

import numpy as np
import pytest
import torch

import oracle
from _gpu_util import (assert_bf16_close, assert_one_ulp_except_cancellation, dev_u16,
                       ensure_lib, exact_sum_and_mag, f64, gamma)
from _ties import fraction_on_midpoints, midpoint_products
from combine_moe_dispatch_05_b200 import ops
from combine_moe_dispatch_05_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_lib()


def prepare(s, identity=False):
    ids = W.topk_ids(s)
    ref = oracle.layout(ids.numpy(), s.E, s.R)
    st = ops.new_status()
    L = ops.moe_dispatch_layout(ids.to(DEV), s.E, s.R, status=st)
    assert ops.read_status(st) == 0
    scales = W.topk_scales(s)
    if identity:  # y = the dispatched x (identity experts)
        x = W.tokens(s)
        y = np.zeros((ref.P_cap, s.H), np.uint16)
        oracle.permute_rows(W.as_u16(x), ref.dst_row, s.K, ref.counts, ref.offsets, y)
        y_cpu = W.from_u16(y)
    else:
        y_cpu = W.expert_out(s, ref.P_cap)
    return L, ref, scales, y_cpu


def check_combine(s, shared=False, identity=False):
    """Returns (gpu out, oracle out, elements over one ulp of the exact sum)."""
    L, ref, scales, y_cpu = prepare(s, identity)
    sh_cpu = W.shared_out(s) if shared else None
    st = ops.new_status()
    out = ops.moe_combine(y_cpu.to(DEV), L.dst_row, scales.to(DEV),
                          shared_x=None if sh_cpu is None else sh_cpu.to(DEV), status=st)
    assert ops.read_status(st) == 0
    y = W.as_u16(y_cpu)
    sh = None if sh_cpu is None else W.as_u16(sh_cpu)
    out_ref = oracle.combine(y, ref.dst_row, scales.numpy(), sh)
    exact_sum, mag = exact_sum_and_mag(y, ref.dst_row, scales.numpy(), sh)
    got = dev_u16(out)
    n = s.K + (1 if shared else 0)
    same = assert_bf16_close(got, out_ref, mag, n, "combine")
    assert same > 0.99, same
    over = assert_one_ulp_except_cancellation(got, exact_sum, mag, n, "combine")
    return out, out_ref, over


@pytest.mark.parametrize("cfg,shared,identity", [(1, False, True), (1, False, False),
                                                 (2, False, False), (4, True, False)])
def test_combine_parity_workloads(cfg, shared, identity):
    check_combine(W.config(cfg), shared, identity)


def test_combine_identity_experts_returns_x_within_an_ulp():
    """Tiny workload, identity experts: out = x * sum_k s_k with sum_k s_k = 1
    up to fp32 rounding, so out equals x to within one bf16 ulp."""
    s = W.config(1)
    out, _, _ = check_combine(s, identity=True)
    x = f64(W.as_u16(W.tokens(s)))
    assert np.all(np.abs(f64(dev_u16(out)) - x) <= 2.0 ** -7 * np.abs(x) + 1e-30)


@pytest.mark.parametrize("T,H,E,K,R,shared", [
    (1, 8, 1, 1, 1, False), (3, 16, 4, 2, 2, True), (129, 24, 9, 3, 3, False),
    (513, 520, 33, 5, 1, True), (40, 7176, 17, 16, 1, False), (1000, 64, 512, 16, 8, True),
    (77, 20480, 9, 1, 3, False), (300, 4096, 8, 2, 2, True), (200, 2048, 16, 3, 4, False)])
def test_combine_parity_edge_shapes(T, H, E, K, R, shared):
    check_combine(W.Spec("edge", T, H, E, K, R, "uniform", seed=3 + T * H), shared)


def test_combine_one_hot_is_bit_exact():
    s = W.config(4)
    L, ref, scales, y_cpu = prepare(s)
    oh = torch.zeros_like(scales)
    oh[:, 3] = 1.0
    out = ops.moe_combine(y_cpu.to(DEV), L.dst_row, oh.to(DEV))
    rows = ref.dst_row.reshape(s.T, s.K)[:, 3]
    assert np.array_equal(dev_u16(out), W.as_u16(y_cpu)[rows])


# ------------------------------------------------------------ backward ----
def check_combine_bwd(s):
    L, ref, scales, y_cpu = prepare(s)
    g_cpu = W.grad_out(s)
    SENT = 0x3C3C
    gy = torch.full((L.P_cap, s.H), 0, dtype=torch.bfloat16, device=DEV)
    gy.view(torch.int16).fill_(SENT)
    st = ops.new_status()
    gy, gs = ops.moe_combine_bwd(g_cpu.to(DEV), y_cpu.to(DEV), scales.to(DEV), L, grad_y=gy,
                                 status=st)
    assert ops.read_status(st) == 0
    g, y = W.as_u16(g_cpu), W.as_u16(y_cpu)
    gy_ref = np.full((ref.P_cap, s.H), SENT, np.uint16)
    gs_ref = oracle.combine_bwd(g, y, scales.numpy(), ref.dst_row, ref.counts, ref.offsets, gy_ref)
    got = dev_u16(gy)
    # every row, bit for bit: slots (the exact product rounded once on both
    # sides), zeroed padding and the untouched tail
    assert np.array_equal(got, gy_ref)
    T, K = s.T, s.K
    rows = ref.dst_row.reshape(T, K)
    dmag = np.einsum("th,tkh->tk", np.abs(f64(g)), np.abs(f64(y)[rows]))
    err = np.abs(gs.cpu().numpy().astype(np.float64) - gs_ref.astype(np.float64))
    assert np.all(err <= gamma(s.H) * dmag + 2.0 ** -24 * np.abs(gs_ref) + 1e-30)


def check_dispatch_bwd(s):
    L, ref, _, y_cpu = prepare(s)
    st = ops.new_status()
    gx = ops.moe_dispatch_bwd(y_cpu.to(DEV), L.dst_row, s.T, s.K, status=st)
    assert ops.read_status(st) == 0
    y = W.as_u16(y_cpu)
    ref_out = oracle.dispatch_bwd(y, ref.dst_row, s.T, s.K)
    ones = np.ones((s.T, s.K), np.float32)
    exact_sum, mag = exact_sum_and_mag(y, ref.dst_row, ones)
    got = dev_u16(gx)
    same = assert_bf16_close(got, ref_out, mag, s.K, "dispatch_bwd")
    assert same > 0.99
    assert_one_ulp_except_cancellation(got, exact_sum, mag, s.K, "dispatch_bwd")


@pytest.mark.parametrize("variant", ["p60", "p100"])
def test_backward_parity_skewed_workload(variant):
    s = W.config(5)
    if variant == "p100":
        s = s.with_(hot_p=1.0)
    check_combine_bwd(s)
    check_dispatch_bwd(s)


@pytest.mark.parametrize("cfg", [1, 2, 4])
def test_backward_parity_workloads(cfg):
    s = W.config(cfg)
    check_combine_bwd(s)
    check_dispatch_bwd(s)


@pytest.mark.parametrize("T,H,E,K,R", [(1, 8, 1, 1, 1), (77, 24, 6, 3, 2), (300, 1032, 40, 16, 4),
                                       (2, 7168, 256, 8, 8), (1000, 64, 512, 16, 8),
                                       (500, 40, 37, 3, 1), (129, 7176, 300, 2, 2),
                                       (60, 20480, 6, 1, 2), (400, 4096, 8, 2, 1)])
def test_backward_parity_edge_shapes(T, H, E, K, R):
    s = W.Spec("edge", T, H, E, K, R, "uniform", seed=11 + T + H)
    check_combine_bwd(s)
    check_dispatch_bwd(s)


@pytest.mark.parametrize("K", [2, 4, 8])
def test_dispatch_bwd_of_dispatch_is_exactly_K_x(K):
    s = W.Spec("k", 600, 264, 24, K, 4, "uniform", seed=900 + K)
    ids = W.topk_ids(s)
    L = ops.moe_dispatch_layout(ids.to(DEV), s.E, s.R)
    x = W.tokens(s).to(DEV)
    xp = ops.moe_dispatch_permute(x, L)
    gx = ops.moe_dispatch_bwd(xp, L.dst_row, s.T, s.K)
    assert torch.equal(gx.float(), x.float() * K)


@pytest.mark.parametrize("cfg,shared", [(2, False), (4, True)])
def test_combine_strict_one_ulp_on_workloads(cfg, shared):
    """The stated accuracy target, element by element on the decode and
    shared-expert workloads: within one bf16 ulp of the exact sum, with no
    allowance but the provable cancellation cases (check_combine)."""
    _, _, over = check_combine(W.config(cfg), shared=shared)
    print(f"config {cfg}: {over} elements over one ulp of the exact sum, all cancellation cases")


def test_grad_y_single_rounding_on_midpoint_products():
    """Scales and gradients whose fp32 products are bf16 midpoints
    (tests/_ties.py): grad_y must equal the oracle's single rounding of the
    exact product bit for bit, where rounding the fp32 product again would
    differ on many elements."""
    T, K, H, E = 256, 4, 1024, 8
    sc, gf = midpoint_products(T, K, H, seed=21)
    assert fraction_on_midpoints(sc, gf) > 0.3
    s = W.Spec("ties", T, H, E, K, 2, "uniform", seed=77)
    ids = W.topk_ids(s)
    ref = oracle.layout(ids.numpy(), E, 2)
    L = ops.moe_dispatch_layout(ids.to(DEV), E, 2)
    g = torch.from_numpy(gf).to(torch.bfloat16)                 # exact: gf holds bf16 values
    y_cpu = W.expert_out(s, ref.P_cap)
    st = ops.new_status()
    gy, _ = ops.moe_combine_bwd(g.to(DEV), y_cpu.to(DEV), torch.from_numpy(sc).to(DEV), L,
                                status=st)
    assert ops.read_status(st) == 0
    gy_ref = np.zeros((ref.P_cap, H), np.uint16)
    oracle.combine_bwd(W.as_u16(g), W.as_u16(y_cpu), sc, ref.dst_row, ref.counts, ref.offsets,
                       gy_ref)
    got = dev_u16(gy)[:ref.P]
    assert np.array_equal(got, gy_ref[:ref.P])
    twice = W.as_u16(torch.from_numpy(sc[:, :, None] * gf[:, None, :]).to(torch.bfloat16))
    rows = ref.dst_row.reshape(T, K)
    assert np.mean(twice != gy_ref[rows]) > 0.1


def test_combine_and_backward_full_prefill_every_token():
    """Full prefill size (T=32768, H=7168, K=8: 262144 slots over 2.2 M rows of
    bf16 expert outputs) in the launch configuration the benchmark uses; every
    token of combine, combine_bwd and dispatch_bwd is compared with the oracle
    element by element.  The oracle runs on 1024-token ranges in parallel
    host threads; each range sees its own tokens' rows gathered into a
    compact buffer (local row indices), so the range's arithmetic is the same
    as over the whole buffer.  grad_y is compared bit for bit (slots here,
    zeroed padding rows on the device)."""
    from concurrent.futures import ThreadPoolExecutor

    s = W.config(3)
    ids = W.topk_ids(s).to(DEV)
    st = ops.new_status()
    L = ops.moe_dispatch_layout(ids, s.E, s.R, status=st)
    y = W.expert_out(s, L.P_cap, device=DEV)
    g = W.grad_out(s, device=DEV)
    sc = W.topk_scales(s).to(DEV)
    out = ops.moe_combine(y, L.dst_row, sc, status=st)
    gy, gs = ops.moe_combine_bwd(g, y, sc, L, status=st)
    gx = ops.moe_dispatch_bwd(gy, L.dst_row, s.T, s.K, status=st)
    assert ops.read_status(st) == 0
    K, H = s.K, s.H
    # padding rows of grad_y (below P) are zero
    P = int(L.expert_offsets[s.E])
    pad = torch.nonzero(L.row_src[:P] < 0).flatten()
    assert pad.numel() == P - s.T * K
    assert not gy[pad].view(torch.int16).any().item()

    sc_h = sc.cpu().numpy()
    chunk = 1024
    ranges = [(a, min(s.T, a + chunk)) for a in range(0, s.T, chunk)]

    def check(i):
        a, b = ranges[i]
        rows = L.dst_row[a * K:b * K].long()              # this range's rows, device -> host
        y_s, gy_s = W.as_u16(y[rows].cpu()), W.as_u16(gy[rows].cpu())
        g_s, out_s, gx_s = (W.as_u16(t[a:b].cpu()) for t in (g, out, gx))
        gs_s = gs[a:b].cpu().numpy()
        n = b - a
        local = np.arange(n * K, dtype=np.int32)          # row j of y_s holds slot a*K + j
        sc_s = sc_h[a:b]
        ref = oracle.combine(y_s, local, sc_s, None)
        ex, mag = exact_sum_and_mag(y_s, local, sc_s)
        assert_bf16_close(out_s, ref, mag, K, "combine")
        over = assert_one_ulp_except_cancellation(out_s, ex, mag, K, "combine")
        counts = np.zeros(1, np.int32)
        offs = np.zeros(2, np.int32)                      # no padding rows in the compact buffer
        gy_ref = np.zeros((n * K, H), np.uint16)
        gs_ref = oracle.combine_bwd(g_s, y_s, sc_s, local, counts, offs, gy_ref)
        assert np.array_equal(gy_s, gy_ref)
        dmag = np.concatenate([np.einsum("th,tkh->tk", np.abs(f64(g_s[c:c + 128])),
                                         np.abs(f64(y_s[c * K:(c + 128) * K])).reshape(-1, K, H))
                               for c in range(0, n, 128)])
        err = np.abs(gs_s.astype(np.float64) - gs_ref.astype(np.float64))
        assert np.all(err <= gamma(H) * dmag + 2.0 ** -24 * np.abs(gs_ref) + 1e-30)
        gx_ref = oracle.dispatch_bwd(gy_ref, local, n, K)
        ones = np.ones((n, K), np.float32)
        ex, mag = exact_sum_and_mag(gy_ref, local, ones)
        assert_bf16_close(gx_s, gx_ref, mag, K, "dispatch_bwd")
        assert_one_ulp_except_cancellation(gx_s, ex, mag, K, "dispatch_bwd")
        return over

    with ThreadPoolExecutor(max_workers=min(4, os.cpu_count() or 1)) as pool:
        over = sum(pool.map(check, range(len(ranges))))
    print(f"full prefill: {over} combine elements over one ulp of the exact sum "
          f"(all cancellation cases)")
