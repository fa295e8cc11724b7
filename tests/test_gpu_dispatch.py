"""GPU parity: dispatch layout and permute against the CPU oracle.

Integer outputs (counts, offsets, rank sums, dst_row, row_src) and permuted
bytes must match bit for bit; padding rows are zero, rows past P keep their
previous contents, and every counter of a finished tile reads 128.
"""
import numpy as np
import pytest
import torch

import oracle
from _gpu_util import ensure_lib, dev_u16
from combine_moe_dispatch_05_b200 import ops
from combine_moe_dispatch_05_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_lib()


def run_layout(ids_cpu: torch.Tensor, E: int, R: int):
    ids = ids_cpu.to(DEV)
    st = ops.new_status()
    L = ops.moe_dispatch_layout(ids, E, R, status=st)
    return L, ops.read_status(st)


def check_layout(ids_cpu, E, R, expect_status=0):
    T, K = ids_cpu.shape
    L, st = run_layout(ids_cpu, E, R)
    ref = oracle.layout(ids_cpu.numpy(), E, R)
    assert st == ref.status == expect_status
    assert L.P_cap == ref.P_cap
    assert np.array_equal(L.expert_counts.cpu().numpy(), ref.counts)
    assert np.array_equal(L.expert_offsets.cpu().numpy(), ref.offsets)
    assert np.array_equal(L.rank_counts.cpu().numpy(), ref.rank_counts)
    assert np.array_equal(L.rank_offsets.cpu().numpy(), ref.rank_offsets)
    if T:
        assert np.array_equal(L.dst_row.cpu().numpy()[:T * K], ref.dst_row)
    assert np.array_equal(L.row_src.cpu().numpy()[:ref.P_cap], ref.row_src)
    n_tiles = (ref.P_cap + 127) // 128
    assert np.all(L.tile_ready.cpu().numpy()[:n_tiles] == 0)
    return L, ref


@pytest.mark.parametrize("cfg", [1, 2, 3, 4, 5])
@pytest.mark.parametrize("seed_offset", [0, 1])
def test_layout_parity_workloads(cfg, seed_offset):
    s = W.config(cfg, seed_offset)
    check_layout(W.topk_ids(s), s.E, s.R)


def test_layout_parity_hot_expert_everywhere():
    s = W.config(5).with_(hot_p=1.0)
    check_layout(W.topk_ids(s), s.E, s.R)


@pytest.mark.parametrize("T,K,E,R", [
    (1, 1, 1, 1), (0, 4, 8, 2), (1, 16, 16, 4), (63, 3, 5, 5), (65, 8, 512, 8),
    (1000, 16, 512, 512), (3000, 1, 2, 2), (129, 2, 3, 1), (257, 7, 64, 16), (4097, 6, 64, 16),
    # runs of 2048 slots per block: exact multiples and one token past them
    (4096, 8, 256, 8), (4097, 8, 256, 8), (2048, 16, 512, 8), (2049, 16, 64, 4),
    (10912, 3, 9, 3), (10913, 3, 9, 3), (700, 5, 40, 8), (3000, 7, 100, 4),
    # runs of 1024 slots per block (batches of at most 65536 slots), and both
    # sides of that bound
    (128, 8, 256, 8), (129, 8, 256, 8), (1024, 1, 2, 2), (1025, 1, 2, 2), (341, 3, 9, 3),
    (342, 3, 9, 3), (8192, 8, 256, 8), (8193, 8, 256, 8), (21845, 3, 9, 3),
    (21846, 3, 9, 3), (65536, 1, 4, 2), (65537, 1, 4, 2)])
def test_layout_parity_edge_shapes(T, K, E, R):
    s = W.Spec("edge", T, 8, E, K, R, "uniform", seed=77 + T + K + E)
    ids = W.topk_ids(s) if T else torch.zeros((0, K), dtype=torch.int32)
    check_layout(ids, E, R)


@pytest.mark.parametrize("T,K,E", [(4096, 8, 256), (20000, 8, 256)])
def test_layout_reuses_buffers_holding_stale_values(T, K, E):
    """A second call on the same buffers, with garbage left in row_src and
    tile_ready and different routing, gives exactly the oracle's layout."""
    s1 = W.Spec("reuse1", T, 8, E, K, 8, "zipf", zipf_s=0.6, seed=901)
    s2 = W.Spec("reuse2", T, 8, E, K, 8, "zipf", zipf_s=1.2, seed=902)
    L = ops.moe_dispatch_layout(W.topk_ids(s1).to(DEV), E, 8)
    L.row_src.fill_(12345)
    L.tile_ready.fill_(77)
    L.dst_row.fill_(-9)
    ids2 = W.topk_ids(s2)
    st = ops.new_status()
    ops.moe_dispatch_layout(ids2.to(DEV), E, 8, layout=L, status=st)
    ref = oracle.layout(ids2.numpy(), E, 8)
    assert ops.read_status(st) == 0
    assert np.array_equal(L.expert_offsets.cpu().numpy(), ref.offsets)
    assert np.array_equal(L.dst_row.cpu().numpy()[:T * K], ref.dst_row)
    assert np.array_equal(L.row_src.cpu().numpy()[:ref.P_cap], ref.row_src)
    assert np.all(L.tile_ready.cpu().numpy()[:(ref.P_cap + 127) // 128] == 0)


def test_layout_all_tokens_one_expert_multi_tile():
    ids = torch.full((1000, 1), 3, dtype=torch.int32)
    L, ref = check_layout(ids, 4, 2)
    assert ref.offsets.tolist() == [0, 0, 0, 0, 1024]


def test_layout_reports_out_of_range_and_duplicates():
    s = W.config(4)
    ids = W.topk_ids(s)
    bad = ids.clone()
    bad[100, 2] = s.E            # out of range
    bad[2000, 0] = -3
    check_layout(bad, s.E, s.R, expect_status=oracle.ERR_EXPERT_RANGE)
    dup = ids.clone()
    dup[555, 1] = dup[555, 0]
    check_layout(dup, s.E, s.R, expect_status=oracle.ERR_DUPLICATE_EXPERT)


@pytest.mark.parametrize("T,K,E", [(300, 8, 64), (9000, 8, 64), (100, 16, 32), (5000, 2, 4),
                                   (2000, 4, 512), (4096, 8, 256), (700, 5, 40)])
def test_layout_duplicates_and_range_errors_every_k(T, K, E):
    """A repeated id inside one token, first at its last slot and then at its
    second, for K a power of two (found from the lane match) or not (found by
    comparison), in the first, a middle and the last block."""
    s = W.Spec("dup", T, 8, E, K, 1, "uniform", seed=5000 + T + K)
    ids = W.topk_ids(s)
    for t, j in ((T - 1, K - 1), (T // 2, 1)):
        dup = ids.clone()
        dup[t, j] = dup[t, 0]
        check_layout(dup, E, 1, expect_status=oracle.ERR_DUPLICATE_EXPERT)
    bad = ids.clone()
    bad[T // 3, K - 1] = E
    check_layout(bad, E, 1, expect_status=oracle.ERR_EXPERT_RANGE)


# ------------------------------------------------------------ permute ----
SENT = 0x5A


def run_permute_bf16(s, x_cpu, strided=False):
    ids = W.topk_ids(s)
    L, _ = run_layout(ids, s.E, s.R)
    ref = oracle.layout(ids.numpy(), s.E, s.R)
    if strided:  # rows of a wider buffer
        wide = torch.zeros((s.T, s.H + 24), dtype=torch.bfloat16)
        wide[:, 8:8 + s.H] = x_cpu
        xd = wide.to(DEV)[:, 8:8 + s.H]
    else:
        xd = x_cpu.to(DEV)
    xp = torch.full((L.P_cap, s.H), 0, dtype=torch.bfloat16, device=DEV)
    xp.view(torch.uint8).fill_(SENT)
    st = ops.new_status()
    ops.moe_dispatch_permute(xd, L, xp=xp, status=st)
    assert ops.read_status(st) == 0
    xp_ref = np.full((ref.P_cap, s.H), SENT * 0x0101, np.uint16)
    oracle.permute_rows(W.as_u16(x_cpu), ref.dst_row, s.K, ref.counts, ref.offsets, xp_ref)
    return L, ref, xp, xp_ref


def check_counters(L, ref):
    cnt = L.tile_ready.cpu().numpy().view(np.uint32)
    n_full = ref.P // 128
    assert np.all(cnt[:n_full] == 128)
    assert np.all(cnt[n_full:] == 0)


@pytest.mark.parametrize("cfg", [1, 2, 4])
def test_permute_bf16_parity(cfg):
    s = W.config(cfg)
    L, ref, xp, xp_ref = run_permute_bf16(s, W.tokens(s))
    assert np.array_equal(dev_u16(xp), xp_ref)
    check_counters(L, ref)


@pytest.mark.parametrize("T,H,E,K,R", [
    (1, 8, 1, 1, 1), (5, 16, 4, 2, 2), (300, 24, 7, 3, 7), (777, 520, 33, 5, 3),
    (64, 8200, 16, 4, 4), (2049, 40, 512, 16, 8), (100, 16384, 8, 2, 2)])
def test_permute_bf16_edge_shapes(T, H, E, K, R):
    s = W.Spec("edge", T, H, E, K, R, "uniform", seed=5 + T + H)
    L, ref, xp, xp_ref = run_permute_bf16(s, W.tokens(s))
    assert np.array_equal(dev_u16(xp), xp_ref)
    check_counters(L, ref)


def test_permute_bf16_strided_rows_and_skew():
    s = W.config(5).with_(T=3001, H=264)
    L, ref, xp, xp_ref = run_permute_bf16(s, W.tokens(s), strided=True)
    assert np.array_equal(dev_u16(xp), xp_ref)
    check_counters(L, ref)


def run_permute_fp8(s, codes_cpu, xs_cpu):
    ids = W.topk_ids(s)
    L, _ = run_layout(ids, s.E, s.R)
    ref = oracle.layout(ids.numpy(), s.E, s.R)
    xp = torch.full((L.P_cap, s.H), SENT, dtype=torch.uint8, device=DEV)
    xps = torch.full((L.P_cap, s.H // 128), -7.0, dtype=torch.float32, device=DEV)
    st = ops.new_status()
    ops.moe_dispatch_permute(codes_cpu.to(DEV), L, xp=xp, x_scales=xs_cpu.to(DEV), xp_scales=xps,
                             status=st)
    assert ops.read_status(st) == 0
    xp_ref = np.full((ref.P_cap, s.H), SENT, np.uint8)
    xps_ref = np.full((ref.P_cap, s.H // 128), -7.0, np.float32)
    oracle.permute_rows(codes_cpu.numpy(), ref.dst_row, s.K, ref.counts, ref.offsets, xp_ref)
    oracle.permute_rows(xs_cpu.numpy(), ref.dst_row, s.K, ref.counts, ref.offsets, xps_ref)
    return L, ref, xp, xps, xp_ref, xps_ref


@pytest.mark.parametrize("T,H,E,K,R", [(2048, 7168, 256, 8, 8), (333, 384, 12, 3, 4),
                                       (50, 128, 3, 2, 1),
                                       # 20 KiB rows: two bulk chunks, 160 scale columns
                                       (300, 20480, 24, 4, 4), (64, 8320, 8, 2, 2)])
def test_permute_fp8_parity(T, H, E, K, R):
    s = W.config(3).with_(T=T, H=H, E=E, K=K, R=R)
    L, ref, xp, xps, xp_ref, xps_ref = run_permute_fp8(s, W.e4m3_codes(s), W.block_scales(s))
    assert np.array_equal(xp.cpu().numpy(), xp_ref)
    assert np.array_equal(xps.cpu().numpy().view(np.uint32), xps_ref.view(np.uint32))
    check_counters(L, ref)


def test_permute_fp8_full_prefill_sampled_rows():
    """Full prefill size (T=32768): every row checked against x through the
    oracle's own map (row_src), padding rows zero, counters complete."""
    s = W.config(3)
    ids = W.topk_ids(s)
    ref = oracle.layout(ids.numpy(), s.E, s.R)
    codes = W.e4m3_codes(s, device=DEV)
    xs = W.block_scales(s, device=DEV)
    L, _ = run_layout(ids, s.E, s.R)
    st = ops.new_status()
    xp, xps = ops.moe_dispatch_permute(codes, L, x_scales=xs, status=st)
    assert ops.read_status(st) == 0
    rs = torch.from_numpy(ref.row_src[:ref.P]).to(DEV).long()
    real = rs >= 0
    tok = torch.where(real, rs // s.K, torch.zeros_like(rs))
    assert torch.equal(xp[:ref.P][real], codes[tok[real]])
    assert torch.equal(xps[:ref.P][real], xs[tok[real]])
    assert int(xp[:ref.P][~real].to(torch.int32).sum()) == 0
    assert float(xps[:ref.P][~real].abs().sum()) == 0.0
    check_counters(L, ref)


# ---------------------------------------------------------- quantiser ----
@pytest.mark.parametrize("T,H", [(64, 1024), (1000, 7168), (3, 128), (300, 384), (70, 8320),
                                 (5, 20480), (8192, 7168)])
def test_quantize_e4m3_parity(T, H):
    s = W.config(3).with_(T=T, H=H)
    x = W.tokens(s)
    q, qs = ops.moe_quantize_e4m3(x.to(DEV))
    q_ref, s_ref = oracle.quantize_e4m3(W.as_u16(x))
    assert np.array_equal(qs.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(q.cpu().numpy(), q_ref)


def test_quantize_e4m3_strided_rows_and_8_byte_aligned_codes():
    """x with a row stride wider than H, and a code buffer that is only
    8-byte aligned (each lane stores its own 8 codes)."""
    s = W.config(3).with_(T=257, H=640)
    x = W.tokens(s)
    wide = torch.zeros((s.T, s.H + 24), dtype=torch.bfloat16)
    wide[:, 16:16 + s.H] = x
    xd = wide.to(DEV)[:, 16:16 + s.H]
    flat = torch.full((s.T * s.H + 8,), 0xA5, dtype=torch.uint8, device=DEV)
    q = flat[8:].view(s.T, s.H)
    q, qs = ops.moe_quantize_e4m3(xd, q=q)
    q_ref, s_ref = oracle.quantize_e4m3(W.as_u16(x))
    assert np.array_equal(qs.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert int(flat[:8].to(torch.int32).sum()) == 8 * 0xA5


def test_quantize_then_dispatch_fp8_pipeline():
    """x -> E4M3 codes (+scales) on both sides independently, then the permute;
    the two pipelines agree byte for byte."""
    s = W.config(3).with_(T=1500, H=1024, E=40, K=4, R=4)
    x = W.tokens(s)
    q, qs = ops.moe_quantize_e4m3(x.to(DEV))
    q_ref, s_ref = oracle.quantize_e4m3(W.as_u16(x))
    ids = W.topk_ids(s)
    L, _ = run_layout(ids, s.E, s.R)
    ref = oracle.layout(ids.numpy(), s.E, s.R)
    xp, xps = ops.moe_dispatch_permute(q, L, x_scales=qs)
    xp_ref = np.zeros((ref.P_cap, s.H), np.uint8)
    xps_ref = np.zeros((ref.P_cap, s.H // 128), np.float32)
    oracle.permute_rows(q_ref, ref.dst_row, s.K, ref.counts, ref.offsets, xp_ref)
    oracle.permute_rows(s_ref, ref.dst_row, s.K, ref.counts, ref.offsets, xps_ref)
    P = ref.P
    assert np.array_equal(xp.cpu().numpy()[:P], xp_ref[:P])
    assert np.array_equal(xps.cpu().numpy()[:P], xps_ref[:P])


def _extreme_block_rows(T, H, seed):
    """bf16 rows whose 128-channel blocks span the whole bf16 range: each
    block gets a random magnitude 2^m (m from -133, the smallest subnormal,
    up to 127) times N(0,1) values, some blocks all zero, some single-value
    blocks, some with values pushed to exact bf16 extremes."""
    g = torch.Generator().manual_seed(seed)
    nb = H // 128
    mags = torch.randint(-133, 128, (T, nb, 1), generator=g).to(torch.float64)
    x = torch.randn((T, nb, 128), generator=g, dtype=torch.float64) * torch.exp2(mags)
    x = x.clamp(-3.0e38, 3.0e38)
    zero = torch.rand((T, nb, 1), generator=g) < 0.05
    x = torch.where(zero, torch.zeros_like(x), x)
    one = torch.rand((T, nb, 1), generator=g) < 0.05
    x = torch.where(one & (torch.arange(128) > 0), torch.zeros_like(x), x)
    return x.view(T, H).to(torch.float32).to(torch.bfloat16)


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_quantize_e4m3_extreme_block_scales(seed):
    """Block scales from bf16 subnormals (scale below 2^-100: the quotient
    path rescales by 2^64 first) to near the largest bf16 values: codes and
    scales bit for bit against the oracle, standalone and fused."""
    T, H = 1024, 1024
    x = _extreme_block_rows(T, H, seed)
    q_ref, s_ref = oracle.quantize_e4m3(W.as_u16(x))
    assert float(np.min(s_ref[s_ref > 0])) < 2.0 ** -100     # the tiny-scale path is used
    q, qs = ops.moe_quantize_e4m3(x.to(DEV))
    assert np.array_equal(qs.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(q.cpu().numpy(), q_ref)
    s = W.Spec("extreme", T, H, 16, 4, 4, "uniform", seed=seed)
    ids = W.topk_ids(s)
    ref = oracle.layout(ids.numpy(), s.E, s.R)
    L, _ = run_layout(ids, s.E, s.R)
    xp, xps = ops.moe_dispatch_permute_quant(x.to(DEV), L)
    xp_ref = np.zeros((ref.P_cap, H), np.uint8)
    xps_ref = np.zeros((ref.P_cap, H // 128), np.float32)
    oracle.permute_rows(q_ref, ref.dst_row, s.K, ref.counts, ref.offsets, xp_ref)
    oracle.permute_rows(s_ref, ref.dst_row, s.K, ref.counts, ref.offsets, xps_ref)
    assert np.array_equal(xp.cpu().numpy()[:ref.P], xp_ref[:ref.P])
    assert np.array_equal(xps.cpu().numpy()[:ref.P].view(np.uint32),
                          xps_ref[:ref.P].view(np.uint32))


def _every_bf16_under(amax_bits):
    """128-channel blocks led by the bf16 value amax_bits (which fixes the
    block's scale), followed by every bf16 value of either sign whose
    magnitude does not exceed it, 127 to a block (the last block padded with
    zeros)."""
    mags = np.arange(0, amax_bits + 1, dtype=np.uint16)
    vals = np.concatenate([mags, mags[1:] | np.uint16(0x8000)])
    n = (len(vals) + 126) // 127
    rows = np.zeros((n, 128), np.uint16)
    rows[:, 0] = amax_bits
    body = np.zeros(n * 127, np.uint16)
    body[:len(vals)] = vals
    rows[:, 1:] = body.reshape(n, 127)
    return rows


def test_quantize_e4m3_every_bf16_value_under_inexact_scales():
    """For block maxima whose scale amax/448 is inexact (and one whose scale
    is below 2^-100, and a subnormal one), every bf16 value up to the block
    maximum: the quotient x/s must round exactly as the IEEE division does,
    so codes agree bit for bit with the oracle's, standalone and fused."""
    amaxes = [0x3F80, 0x4040, 0x3DCD, 0x40B0, 0x43DF, 0x43E1, 0x7149, 0x1000, 0x0005]
    x = W.from_u16(np.concatenate([_every_bf16_under(a) for a in amaxes]))
    T, H = x.shape
    q_ref, s_ref = oracle.quantize_e4m3(W.as_u16(x))
    assert float(np.min(s_ref)) < 2.0 ** -100
    q, qs = ops.moe_quantize_e4m3(x.to(DEV))
    assert np.array_equal(qs.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(q.cpu().numpy(), q_ref)
    s = W.Spec("every_bf16", T, H, 16, 4, 4, "uniform", seed=7)
    ids = W.topk_ids(s)
    ref = oracle.layout(ids.numpy(), s.E, s.R)
    L, _ = run_layout(ids, s.E, s.R)
    xp, xps = ops.moe_dispatch_permute_quant(x.to(DEV), L)
    xp_ref = np.zeros((ref.P_cap, H), np.uint8)
    xps_ref = np.zeros((ref.P_cap, H // 128), np.float32)
    oracle.permute_rows(q_ref, ref.dst_row, s.K, ref.counts, ref.offsets, xp_ref)
    oracle.permute_rows(s_ref, ref.dst_row, s.K, ref.counts, ref.offsets, xps_ref)
    assert np.array_equal(xp.cpu().numpy()[:ref.P], xp_ref[:ref.P])
    assert np.array_equal(xps.cpu().numpy()[:ref.P].view(np.uint32),
                          xps_ref[:ref.P].view(np.uint32))


def test_quantize_e4m3_round_trip_bound_on_gpu_codes():
    """Codes and scales from the GPU quantiser, decoded by torch's own E4M3
    conversion: |x - q*s| <= 2^-4 |x| where x/s is a normal E4M3 number and
    <= 2^-10 s in the subnormal range (half a step of 3 mantissa bits)."""
    s = W.config(3).with_(T=2048, H=7168)
    x = W.tokens(s, device=DEV)
    q, qs = ops.moe_quantize_e4m3(x)
    deq = q.view(torch.float8_e4m3fn).float().view(s.T, s.H // 128, 128) * qs.unsqueeze(-1)
    xv = x.float().view(s.T, s.H // 128, 128)
    err = (deq - xv).abs()
    r = xv.abs() / qs.unsqueeze(-1)
    normal = r >= 2.0 ** -6
    assert bool((err[normal] <= 2.0 ** -4 * xv.abs()[normal] * (1 + 1e-6)).all())
    sub_bound = (2.0 ** -10 * qs.unsqueeze(-1) * (1 + 1e-6)).expand_as(xv)
    assert bool((err[~normal] <= sub_bound[~normal]).all())
    # every block's largest magnitude lands on +-448 exactly
    top = torch.gather(q.view(s.T, s.H // 128, 128), 2, xv.abs().argmax(-1, keepdim=True))
    assert bool(((top & 0x7F) == 0x7E).all())
