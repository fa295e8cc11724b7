"""Host-side pieces of bench.py that need no GPU: the token-partitioned oracle
run reported beside the single-threaded one must compute exactly what one
unpartitioned oracle pass computes, and the algorithmic byte counts follow
their per-call formulas."""
import numpy as np
import pytest

import bench
import oracle
from combine_moe_dispatch_05_b200 import workloads as W


def _serial(s, ids, sc, x, g):
    L = oracle.layout(ids, s.E, s.R)
    xp = np.zeros((L.P_cap, s.H), np.uint16)
    oracle.permute_rows(x, L.dst_row, s.K, L.counts, L.offsets, xp)
    out = oracle.combine(xp, L.dst_row, sc, None)
    gy = np.zeros_like(xp)
    gs = oracle.combine_bwd(g, xp, sc, L.dst_row, L.counts, L.offsets, gy)
    gx = oracle.dispatch_bwd(gy, L.dst_row, s.T, s.K)
    return dict(xp=xp, out=out, grad_y=gy, grad_scales=gs, grad_x=gx)


@pytest.mark.parametrize("cfg,threads", [(1, 1), (1, 3), (1, 7), (4, 5)])
def test_partitioned_oracle_pass_equals_one_pass(cfg, threads):
    s = W.config(cfg)
    if cfg != 1:
        s = s.with_(T=200, H=256)
    ids, sc = W.topk_ids(s).numpy(), W.topk_scales(s).numpy()
    x, g = W.as_u16(W.tokens(s)), W.as_u16(W.grad_out(s))
    ref = _serial(s, ids, sc, x, g)
    _, res = bench.oracle_pass_partitioned(s, ids, sc, x, g, False, threads)
    for key in ("xp", "out", "grad_y", "grad_x"):
        assert np.array_equal(res[key], ref[key]), key
    assert np.array_equal(res["grad_scales"].view(np.uint32), ref["grad_scales"].view(np.uint32))


def test_partitioned_oracle_pass_more_threads_than_tokens():
    s = W.config(1).with_(T=5)
    ids, sc = W.topk_ids(s).numpy(), W.topk_scales(s).numpy()
    x, g = W.as_u16(W.tokens(s)), W.as_u16(W.grad_out(s))
    ref = _serial(s, ids, sc, x, g)
    _, res = bench.oracle_pass_partitioned(s, ids, sc, x, g, False, 16)
    assert np.array_equal(res["out"], ref["out"]) and np.array_equal(res["grad_x"], ref["grad_x"])


def test_step_bytes_formulas():
    T, K, H, E, P = 4096, 8, 7168, 256, 49152
    b = bench.step_bytes(T, K, H, E, P)
    assert b["permute"] == 2 * T * H + 2 * P * H
    assert b["combine"] == 2 * T * K * H + 8 * T * K + 2 * T * H
    assert b["combine_bwd"] == 2 * T * H + 2 * T * K * H + 2 * P * H + 12 * T * K
    assert b["dispatch_bwd"] == 2 * T * K * H + 2 * T * H + 4 * T * K
    assert set(bench.step_bytes(T, K, H, E, P, fwd_only=True)) == {"layout", "permute", "combine"}


def test_host_cpu_reports_threads_and_model():
    n, model = bench.host_cpu()
    assert n >= 1 and isinstance(model, str) and model


def _fake_gpu_outputs(s, res):
    L = res["layout"]
    return {"counts": L.counts.copy(), "offsets": L.offsets.copy(),
            "scales": W.topk_scales(s).numpy(),
            "rank_counts": L.rank_counts.copy(), "rank_offsets": L.rank_offsets.copy(),
            "dst_row": L.dst_row.copy(), "row_src": L.row_src.copy(),
            "xp": res["xp"][:L.P].view(np.int16).copy(), "out": res["out"].view(np.int16).copy(),
            "grad_y": res["grad_y"][:L.P].view(np.int16).copy(),
            "grad_scales": res["grad_scales"].copy(), "grad_x": res["grad_x"].view(np.int16).copy()}


def test_timed_run_check_accepts_identical_and_flags_changes():
    s = W.config(1)
    ids, sc = W.topk_ids(s).numpy(), W.topk_scales(s).numpy()
    x, g = W.as_u16(W.tokens(s)), W.as_u16(W.grad_out(s))
    _, res = bench.oracle_pass_partitioned(s, ids, sc, x, g, False, 2)
    ok = bench.check_timed_outputs(s, res, _fake_gpu_outputs(s, res), x, g, False)
    assert ok["layout_bit_exact"] and ok["permute_bytes_exact"]
    assert ok["combine_max_ulp"] == 0 and ok["dispatch_bwd_max_ulp"] == 0
    assert ok["combine_bwd_grad_y_max_ulp"] == 0 and ok["grad_scales_max_err_over_norms"] == 0
    assert ok["combine_bwd_grad_y_bit_exact"]
    assert ok["combine_vs_exact_sum"]["over_one_ulp_of_exact"] == 0
    assert ok["combine_vs_exact_sum"]["elements"] == s.T * s.H

    bad = _fake_gpu_outputs(s, res)
    bad["dst_row"][7] += 1
    bad["xp"][3, 5] ^= 1
    flat = bad["out"].reshape(-1)  # two bf16 ulps (same binade), away from cancellation
    j = int(np.flatnonzero(((flat.view(np.uint16) & 0x7F) < 0x70) &
                           ((flat.view(np.uint16) & 0x7F80) > 0x3C00))[0])
    flat[j] += 2
    bad["grad_y"][1, 2] ^= 1
    # three ulps, at an element whose mantissa leaves room inside its binade
    flat = bad["grad_x"].reshape(-1)
    i = int(np.flatnonzero((flat.view(np.uint16) & 0x7F) < 0x70)[0])
    flat[i] += 3
    chk = bench.check_timed_outputs(s, res, bad, x, g, False)
    assert not chk["layout_bit_exact"] and not chk["permute_bytes_exact"]
    assert chk["combine_max_ulp"] == 2 and chk["dispatch_bwd_max_ulp"] == 3
    assert chk["combine_vs_exact_sum"]["over_one_ulp_of_exact"] == 1
    assert chk["combine_vs_exact_sum"]["over_one_ulp_not_cancellation"] == 1
    assert not chk["combine_bwd_grad_y_bit_exact"]


def test_bf16_max_ulp_units():
    one, next_up = np.array([0x3F80], np.uint16), np.array([0x3F81], np.uint16)
    assert bench.bf16_max_ulp(next_up, one) == 1.0
    assert bench.bf16_max_ulp(one, one) == 0.0
    # 2.0 vs 1.0: one unit of 1.0's binade is 2^-7, so the gap is 128 ulps
    assert bench.bf16_max_ulp(np.array([0x4000], np.uint16), one) == 128.0


def test_groups_gbs_sums_bytes_and_times():
    nb = {"layout": 100, "permute": 900, "combine": 500, "combine_bwd": 1000, "dispatch_bwd": 400}
    us = {"layout": 1.0, "permute": 9.0, "combine": 5.0, "combine_bwd": 10.0, "dispatch_bwd": 4.0}
    g = bench.groups_gbs(nb, us)
    assert g["dispatch"] == {"GBps": 0.1, "us": 10.0, "bytes": 1000}
    assert g["dispatch_plus_combine"]["bytes"] == 1500 and g["dispatch_plus_combine"]["us"] == 15.0
    assert g["backward"]["bytes"] == 1400
    fwd = bench.groups_gbs({k: nb[k] for k in ("layout", "permute", "combine")},
                           {k: us[k] for k in ("layout", "permute", "combine")})
    assert "backward" not in fwd
