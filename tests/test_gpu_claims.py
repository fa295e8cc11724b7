"""The scheduling words of the dynamically claimed copy kernels (the permute
and the fused quantise-dispatch): every completed call returns them to zero,
so the same words serve call after call; repeated calls on the same inputs
give the same bytes and complete counters; shapes with far more CTAs than
tickets (one token, padding-heavy layouts) and with several tokens per
ticket (short rows) are covered against the oracle."""
import numpy as np
import pytest
import torch

import oracle
from _gpu_util import dev_u16, ensure_lib
from combine_moe_dispatch_05_b200 import ops
from combine_moe_dispatch_05_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_lib()


def _words_zero(L):
    torch.cuda.synchronize()
    return int(L.work.abs().sum().item()) == 0


def _counters_complete(L, P):
    cnt = L.tile_ready.cpu().numpy().view(np.uint32)
    return bool(np.all(cnt[:P // 128] == 128) and np.all(cnt[P // 128:] == 0))


@pytest.mark.parametrize("cfg", [2, 4])
def test_permute_repeated_calls_identical_and_words_zero(cfg):
    s = W.config(cfg)
    ids = W.topk_ids(s).to(DEV)
    x = W.tokens(s, device=DEV)
    st = ops.new_status()
    L = ops.moe_dispatch_layout(ids, s.E, s.R, status=st)
    first = ops.moe_dispatch_permute(x, L, status=st)
    assert _words_zero(L)
    P = int(L.expert_offsets[s.E])
    xp = torch.empty_like(first)
    for _ in range(20):
        ops.moe_dispatch_layout(ids, s.E, s.R, layout=L, status=st)  # resets the counters
        ops.moe_dispatch_permute(x, L, xp=xp, status=st)
        assert _words_zero(L)
        assert torch.equal(xp[:P], first[:P])
        assert _counters_complete(L, P)
    assert ops.read_status(st) == 0


@pytest.mark.parametrize("T,H,E,K", [(1, 7168, 256, 8), (1, 64, 1, 1), (3, 4096, 512, 16),
                                     (2, 128, 512, 2), (40000, 64, 4, 2), (9000, 128, 64, 1)])
def test_permute_claim_edge_shapes_match_oracle(T, H, E, K):
    """More CTAs than tickets (T = 1..3, padding far exceeding the slots) and
    several tokens per ticket (rows of 128-256 bytes)."""
    s = W.Spec("claims", T, H, E, K, 1, "uniform", seed=31 + T + H)
    ids = W.topk_ids(s)
    ref = oracle.layout(ids.numpy(), E, 1)
    st = ops.new_status()
    L = ops.moe_dispatch_layout(ids.to(DEV), E, 1, status=st)
    x = W.tokens(s)
    xp = torch.zeros((L.P_cap, H), dtype=torch.bfloat16, device=DEV)
    xp.view(torch.int16).fill_(0x5A5A)
    for _ in range(2):
        ops.moe_dispatch_permute(x.to(DEV), L, xp=xp, status=st)
        assert _words_zero(L)
    assert ops.read_status(st) == 0
    xp_ref = np.full((ref.P_cap, H), 0x5A5A, np.uint16)
    oracle.permute_rows(W.as_u16(x), ref.dst_row, K, ref.counts, ref.offsets, xp_ref)
    assert np.array_equal(dev_u16(xp), xp_ref)


def test_fused_quant_dispatch_repeated_calls_and_words_zero():
    s = W.config(3).with_(T=4096)
    ids = W.topk_ids(s).to(DEV)
    x = W.tokens(s, device=DEV)
    st = ops.new_status()
    L = ops.moe_dispatch_layout(ids, s.E, s.R, status=st)
    q1, s1 = ops.moe_dispatch_permute_quant(x, L, status=st)
    assert _words_zero(L)
    P = int(L.expert_offsets[s.E])
    for _ in range(5):
        ops.moe_dispatch_layout(ids, s.E, s.R, layout=L, status=st)
        q2, s2 = ops.moe_dispatch_permute_quant(x, L, status=st)
        assert _words_zero(L)
        assert torch.equal(q1[:P], q2[:P])
        assert torch.equal(s1[:P].view(torch.int32), s2[:P].view(torch.int32))
        assert _counters_complete(L, P)
    assert ops.read_status(st) == 0


def test_permute_kinds_share_one_pair_of_words_in_stream_order():
    """The bf16 permute, the E4M3 permute and the fused quantise-dispatch
    called back to back on one stream with the same words."""
    s = W.config(3).with_(T=2000)
    ids = W.topk_ids(s).to(DEV)
    x = W.tokens(s, device=DEV)
    st = ops.new_status()
    L = ops.moe_dispatch_layout(ids, s.E, s.R, status=st)
    q, qs = ops.moe_quantize_e4m3(x, status=st)
    a = ops.moe_dispatch_permute(x, L, status=st, use_counters=False)
    b, bs = ops.moe_dispatch_permute(q, L, x_scales=qs, status=st, use_counters=False)
    c, cs = ops.moe_dispatch_permute_quant(x, L, status=st, use_counters=False)
    assert _words_zero(L) and ops.read_status(st) == 0
    P = int(L.expert_offsets[s.E])
    assert torch.equal(b[:P], c[:P]) and torch.equal(bs[:P].view(torch.int32),
                                                      cs[:P].view(torch.int32))
    rs = L.row_src[:P].long()
    real = rs >= 0
    assert torch.equal(a[:P][real], x[(rs[real] // s.K)])


@pytest.mark.parametrize("H,fp8", [(8, False), (128, True)])
def test_permute_with_more_tiles_than_the_table_releases_in_batches(H, fp8):
    """T=131072, K=8, E=256: about 1.08 M padded rows, 8447 tiles, more than a
    CTA's tile table holds, so the counters are released in batches during
    the copy.  Bytes (and E4M3 scales) against the oracle, complete counters,
    scheduling words back at zero."""
    s = W.Spec("many_tiles", 131072, H, 256, 8, 8, "uniform", seed=404 + H)
    ids = W.topk_ids(s)
    ref = oracle.layout(ids.numpy(), s.E, s.R)
    assert (ref.P_cap + 127) // 128 > 8192
    st = ops.new_status()
    L = ops.moe_dispatch_layout(ids.to(DEV), s.E, s.R, status=st)
    if fp8:
        codes, xs = W.e4m3_codes(s), W.block_scales(s)
        xp, xps = ops.moe_dispatch_permute(codes.to(DEV), L, x_scales=xs.to(DEV), status=st)
        xp_ref = np.zeros((ref.P_cap, H), np.uint8)
        xps_ref = np.zeros((ref.P_cap, H // 128), np.float32)
        oracle.permute_rows(codes.numpy(), ref.dst_row, s.K, ref.counts, ref.offsets, xp_ref)
        oracle.permute_rows(xs.numpy(), ref.dst_row, s.K, ref.counts, ref.offsets, xps_ref)
    else:
        x = W.tokens(s)
        xp = ops.moe_dispatch_permute(x.to(DEV), L, status=st)
        xp_ref = np.zeros((ref.P_cap, H), np.uint16)
        oracle.permute_rows(W.as_u16(x), ref.dst_row, s.K, ref.counts, ref.offsets, xp_ref)
    assert _words_zero(L) and ops.read_status(st) == 0
    P = ref.P
    got = xp[:P].cpu().numpy() if fp8 else dev_u16(xp)[:P]
    assert np.array_equal(got, xp_ref[:P])
    if fp8:
        assert np.array_equal(xps[:P].cpu().numpy().view(np.uint32), xps_ref[:P].view(np.uint32))
    assert _counters_complete(L, P)
