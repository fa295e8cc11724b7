"""GPU: chunk-completion counters and the reference consumer.

A consumer that acquires a tile's counter at 128 must see the whole tile
(content checksums equal the oracle's); a consumer with no producer must give
up within its time limit and report MOE_ERR_TIMEOUT, leaving the context
usable.  Device-side data errors are reported through the status word and
the offending writes are skipped.
"""
import numpy as np
import pytest
import torch

import oracle
from _gpu_util import assert_bf16_close, dev_u16, ensure_lib, f64
from combine_moe_dispatch_05_b200 import ops
from combine_moe_dispatch_05_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_lib()


@pytest.mark.parametrize("cfg", [1, 2, 4])
def test_consumer_sees_complete_tiles_bf16(cfg):
    s = W.config(cfg)
    ids = W.topk_ids(s)
    x = W.tokens(s)
    ref = oracle.layout(ids.numpy(), s.E, s.R)
    xp_ref = np.zeros((ref.P_cap, s.H), np.uint16)
    oracle.permute_rows(W.as_u16(x), ref.dst_row, s.K, ref.counts, ref.offsets, xp_ref)
    cs_ref = oracle.tile_checksums(xp_ref, ref.P // 128)

    st = ops.new_status()
    L = ops.moe_dispatch_layout(ids.to(DEV), s.E, s.R, status=st)
    xp = ops.moe_dispatch_permute(x.to(DEV), L, status=st)
    cs = ops.moe_wait_tiles_checksum(L, xp, status=st, timeout_ns=2 * 10**9)
    assert ops.read_status(st) == 0
    got = cs.cpu().numpy().view(np.uint32)[:ref.P // 128]
    assert np.array_equal(got, cs_ref)


def test_consumer_sees_complete_tiles_fp8_with_scales():
    s = W.config(3).with_(T=3000, H=1024, E=32, K=4, R=4)
    ids = W.topk_ids(s)
    codes, xs = W.e4m3_codes(s), W.block_scales(s)
    ref = oracle.layout(ids.numpy(), s.E, s.R)
    xp_ref = np.zeros((ref.P_cap, s.H), np.uint8)
    xps_ref = np.zeros((ref.P_cap, s.H // 128), np.float32)
    oracle.permute_rows(codes.numpy(), ref.dst_row, s.K, ref.counts, ref.offsets, xp_ref)
    oracle.permute_rows(xs.numpy(), ref.dst_row, s.K, ref.counts, ref.offsets, xps_ref)
    cs_ref = oracle.tile_checksums(xp_ref, ref.P // 128, xps_ref)
    st = ops.new_status()
    L = ops.moe_dispatch_layout(ids.to(DEV), s.E, s.R, status=st)
    xp, xps = ops.moe_dispatch_permute(codes.to(DEV), L, x_scales=xs.to(DEV), status=st)
    cs = ops.moe_wait_tiles_checksum(L, xp, xps, status=st)
    assert ops.read_status(st) == 0
    assert np.array_equal(cs.cpu().numpy().view(np.uint32)[:ref.P // 128], cs_ref)


def test_consumer_without_producer_times_out_and_context_survives():
    s = W.config(1)
    ids = W.topk_ids(s)
    st = ops.new_status()
    L = ops.moe_dispatch_layout(ids.to(DEV), s.E, s.R, status=st)   # counters reset to 0
    xp = torch.zeros((L.P_cap, s.H), dtype=torch.bfloat16, device=DEV)
    assert ops.read_status(st) == 0
    ops.moe_wait_tiles_checksum(L, xp, status=st, timeout_ns=20 * 10**6)   # 20 ms
    assert ops.read_status(st) == ops.ERR_TIMEOUT
    # the context is still usable: a normal dispatch succeeds afterwards
    st2 = ops.new_status()
    xp2 = ops.moe_dispatch_permute(W.tokens(s).to(DEV), L, status=st2)
    cs = ops.moe_wait_tiles_checksum(L, xp2, status=st2)
    assert ops.read_status(st2) == 0


def test_permute_without_counters_leaves_them_alone():
    s = W.config(1)
    ids = W.topk_ids(s)
    L = ops.moe_dispatch_layout(ids.to(DEV), s.E, s.R)
    ops.moe_dispatch_permute(W.tokens(s).to(DEV), L, use_counters=False)
    assert int(L.tile_ready.abs().sum()) == 0


def test_bounds_guard_skips_rows_outside_the_buffer():
    """A corrupted dst_row entry (host-made fault) is reported and its write is
    skipped; guard rows around the buffer stay intact."""
    s = W.config(1)
    ids = W.topk_ids(s)
    L = ops.moe_dispatch_layout(ids.to(DEV), s.E, s.R)
    torch.cuda.synchronize()
    L.dst_row[7] = L.P_cap + 5          # outside [0, P_cap)
    L.dst_row[9] = -12
    guard = torch.full((L.P_cap + 64, s.H), 0, dtype=torch.bfloat16, device=DEV)
    guard.view(torch.int16).fill_(0x1234)
    xp = guard[:L.P_cap]
    st = ops.new_status()
    ops.moe_dispatch_permute(W.tokens(s).to(DEV), L, xp=xp, status=st)
    assert ops.read_status(st) == ops.ERR_BOUNDS
    assert bool((guard[L.P_cap:].view(torch.int16) == 0x1234).all())
    st = ops.new_status()
    y = torch.zeros((L.P_cap, s.H), dtype=torch.bfloat16, device=DEV)
    ops.moe_combine(y, L.dst_row, W.topk_scales(s).to(DEV), status=st)
    assert ops.read_status(st) == ops.ERR_BOUNDS
    st = ops.new_status()
    ops.moe_dispatch_bwd(y, L.dst_row, s.T, s.K, status=st)
    assert ops.read_status(st) == ops.ERR_BOUNDS
    st = ops.new_status()
    gy = guard[:L.P_cap]
    ops.moe_combine_bwd(W.grad_out(s).to(DEV), y, W.topk_scales(s).to(DEV), L, grad_y=gy,
                        status=st)
    assert ops.read_status(st) == ops.ERR_BOUNDS
    assert bool((guard[L.P_cap:].view(torch.int16) == 0x1234).all())
    # E4M3 rows: the byte permute and the fused quantise-dispatch
    gq = torch.full((L.P_cap + 64, s.H), 0x77, dtype=torch.uint8, device=DEV)
    gqs = torch.full((L.P_cap + 64, s.H // 128), -5.0, dtype=torch.float32, device=DEV)
    st = ops.new_status()
    ops.moe_dispatch_permute(W.e4m3_codes(s).to(DEV), L, xp=gq[:L.P_cap],
                             x_scales=W.block_scales(s).to(DEV), xp_scales=gqs[:L.P_cap],
                             status=st)
    assert ops.read_status(st) == ops.ERR_BOUNDS
    st = ops.new_status()
    ops.moe_dispatch_permute_quant(W.tokens(s).to(DEV), L, xp=gq[:L.P_cap],
                                   xp_scales=gqs[:L.P_cap], status=st)
    assert ops.read_status(st) == ops.ERR_BOUNDS
    assert bool((gq[L.P_cap:] == 0x77).all()) and bool((gqs[L.P_cap:] == -5.0).all())


def test_out_of_range_ids_are_skipped_downstream():
    s = W.config(4)
    ids = W.topk_ids(s)
    ids[10, 1] = s.E + 3
    ref = oracle.layout(ids.numpy(), s.E, s.R)
    st = ops.new_status()
    L = ops.moe_dispatch_layout(ids.to(DEV), s.E, s.R, status=st)
    assert ops.read_status(st) == ops.ERR_EXPERT_RANGE
    x = W.tokens(s)
    st2 = ops.new_status()
    xp = ops.moe_dispatch_permute(x.to(DEV), L, status=st2)
    assert ops.read_status(st2) == 0          # -1 rows are skipped silently
    xp_ref = np.zeros((ref.P_cap, s.H), np.uint16)
    oracle.permute_rows(W.as_u16(x), ref.dst_row, s.K, ref.counts, ref.offsets, xp_ref)
    assert np.array_equal(dev_u16(xp)[:ref.P], xp_ref[:ref.P])
    sc = W.topk_scales(s)
    out = ops.moe_combine(xp, L.dst_row, sc.to(DEV), status=st2)
    assert ops.read_status(st2) == 0
    out_ref = oracle.combine(xp_ref, ref.dst_row, sc.numpy(), None)
    rows = np.where(ref.dst_row >= 0, ref.dst_row, ref.P_cap - 1).reshape(s.T, s.K)
    mag = np.einsum("tk,tkh->th", np.abs(sc.numpy().astype(np.float64)),
                    np.abs(f64(xp_ref)[rows]) * (ref.dst_row.reshape(s.T, s.K, 1) >= 0))
    assert_bf16_close(dev_u16(out), out_ref, mag, s.K + 1, "combine with an unplaced slot")


# ---------------------------------------------- concurrent consumer (fused) ----
def _oracle_tiles(s, ids, data, scales=None):
    ref = oracle.layout(ids.numpy(), s.E, s.R)
    xp_ref = np.zeros((ref.P_cap, data.shape[1]), data.dtype)
    oracle.permute_rows(data, ref.dst_row, s.K, ref.counts, ref.offsets, xp_ref)
    xs_ref = None
    if scales is not None:
        xs_ref = np.zeros((ref.P_cap, scales.shape[1]), np.float32)
        oracle.permute_rows(scales, ref.dst_row, s.K, ref.counts, ref.offsets, xs_ref)
    return ref, xp_ref, xs_ref, oracle.tile_checksums(xp_ref, ref.P // 128, xs_ref)


@pytest.mark.parametrize("cfg", [1, 2, 4])
def test_concurrent_consumer_sees_only_complete_tiles_bf16(cfg):
    """Producer warps and consumer warps run at the same time (one cooperative
    launch); every tile the consumers acquire must already be complete."""
    s = W.config(cfg)
    ids, x = W.topk_ids(s), W.tokens(s)
    ref, xp_ref, _, cs_ref = _oracle_tiles(s, ids, W.as_u16(x))
    for rep in range(3):
        st = ops.new_status()
        L = ops.moe_dispatch_layout(ids.to(DEV), s.E, s.R, status=st)
        xp, cs = ops.moe_dispatch_permute_consume(x.to(DEV), L, status=st, timeout_ns=2 * 10**9)
        assert ops.read_status(st) == 0
        assert np.array_equal(cs.cpu().numpy().view(np.uint32)[:ref.P // 128], cs_ref), rep
        assert np.array_equal(dev_u16(xp)[:ref.P], xp_ref[:ref.P])
        assert np.all(L.tile_ready.cpu().numpy()[:ref.P // 128] == 128)


def test_concurrent_consumer_fp8_with_scales():
    s = W.config(3).with_(T=4000, H=1024, E=48, K=6, R=4)
    ids, codes, xs = W.topk_ids(s), W.e4m3_codes(s), W.block_scales(s)
    ref, xp_ref, xs_ref, cs_ref = _oracle_tiles(s, ids, codes.numpy(), xs.numpy())
    st = ops.new_status()
    L = ops.moe_dispatch_layout(ids.to(DEV), s.E, s.R, status=st)
    xp, xps, cs = ops.moe_dispatch_permute_consume(codes.to(DEV), L, x_scales=xs.to(DEV),
                                                   status=st)
    assert ops.read_status(st) == 0
    assert np.array_equal(cs.cpu().numpy().view(np.uint32)[:ref.P // 128], cs_ref)
    assert np.array_equal(xp.cpu().numpy()[:ref.P], xp_ref[:ref.P])
    assert np.array_equal(xps.cpu().numpy()[:ref.P], xs_ref[:ref.P])


def test_vectorised_reference_consumer_matches_scalar_weights():
    """The stream-ordered consumer reads 16 bytes at a time when aligned and
    4 bytes otherwise; both give the oracle's checksums."""
    s = W.config(1)
    ids, x = W.topk_ids(s), W.tokens(s)
    ref, xp_ref, _, cs_ref = _oracle_tiles(s, ids, W.as_u16(x))
    L = ops.moe_dispatch_layout(ids.to(DEV), s.E, s.R)
    xp = ops.moe_dispatch_permute(x.to(DEV), L)
    cs16 = ops.moe_wait_tiles_checksum(L, xp)
    # a 4-byte-aligned but not 16-byte-aligned copy takes the scalar path
    buf = torch.zeros(xp.numel() * 2 + 8, dtype=torch.uint8, device=DEV)
    off = buf[4:4 + xp.numel() * 2]
    off.copy_(xp.view(torch.uint8).reshape(-1))
    row_bytes = s.H * 2
    cs4 = torch.zeros_like(cs16)
    st = ops.new_status()
    rc = ops.lib().moe_wait_tiles_checksum(
        ops._ptr(L.tile_ready), ops._ptr(L.expert_offsets), s.E, ops._ptr(off), row_bytes, None, 0,
        L.P_cap, ops._ptr(cs4), 10**9, ops._ptr(st), ops._stream())
    assert rc == 0
    assert ops.read_status(st) == 0
    n = ref.P // 128
    assert np.array_equal(cs16.cpu().numpy().view(np.uint32)[:n], cs_ref)
    assert np.array_equal(cs4.cpu().numpy().view(np.uint32)[:n], cs_ref)


@pytest.mark.parametrize("T,H,E,K,R,fp8", [(257, 20480, 12, 3, 3, False), (190, 20480, 10, 2, 5, True),
                                          (1500, 64, 512, 16, 8, False)])
def test_concurrent_consumer_chunked_rows_and_many_experts(T, H, E, K, R, fp8):
    """Rows over 16 KiB (several bulk chunks per row), scales past 64 columns,
    and a layout with many mostly-padding tiles."""
    s = W.config(3).with_(T=T, H=H, E=E, K=K, R=R)
    ids = W.topk_ids(s)
    st = ops.new_status()
    L = ops.moe_dispatch_layout(ids.to(DEV), s.E, s.R, status=st)
    if fp8:
        codes, xs = W.e4m3_codes(s), W.block_scales(s)
        ref, xp_ref, xs_ref, cs_ref = _oracle_tiles(s, ids, codes.numpy(), xs.numpy())
        xp, xps, cs = ops.moe_dispatch_permute_consume(codes.to(DEV), L, x_scales=xs.to(DEV),
                                                       status=st)
        assert np.array_equal(xps.cpu().numpy()[:ref.P], xs_ref[:ref.P])
        got = xp.cpu().numpy()[:ref.P]
    else:
        x = W.tokens(s)
        ref, xp_ref, _, cs_ref = _oracle_tiles(s, ids, W.as_u16(x))
        xp, cs = ops.moe_dispatch_permute_consume(x.to(DEV), L, status=st)
        got = dev_u16(xp)[:ref.P]
    assert ops.read_status(st) == 0
    assert np.array_equal(got, xp_ref[:ref.P])
    assert np.array_equal(cs.cpu().numpy().view(np.uint32)[:ref.P // 128], cs_ref)
