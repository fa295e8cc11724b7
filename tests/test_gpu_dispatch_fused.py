"""GPU parity: moe_dispatch (layout + permute in one call, the permute's first
row loads overlapping the layout) gives exactly what moe_dispatch_layout
followed by moe_dispatch_permute gives, and what the oracle gives: every
layout output, every byte of the expert-major buffer (padding rows and the
untouched rows past P included), complete chunk counters, scheduling words
back at zero; also under CUDA-graph replay on new inputs."""
import numpy as np
import pytest
import torch

import oracle
from _gpu_util import dev_u16, ensure_lib
from combine_moe_dispatch_05_b200 import ops
from combine_moe_dispatch_05_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda"
SENT = 0x3A3A


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_lib()


LAYOUT_FIELDS = ("expert_counts", "expert_offsets", "rank_counts", "rank_offsets", "dst_row",
                 "row_src", "tile_ready")


def _fused_and_separate_bf16(s, x):
    ids = W.topk_ids(s).to(DEV)
    st = ops.new_status()
    L1 = ops.alloc_layout(s.T, s.K, s.E, s.R, DEV)
    xp1 = torch.zeros((L1.P_cap, s.H), dtype=torch.bfloat16, device=DEV)
    xp1.view(torch.int16).fill_(SENT)
    ops.moe_dispatch(ids, x, s.E, s.R, layout=L1, xp=xp1, status=st)
    L2 = ops.moe_dispatch_layout(ids, s.E, s.R, status=st)
    xp2 = torch.zeros_like(xp1)
    xp2.view(torch.int16).fill_(SENT)
    ops.moe_dispatch_permute(x, L2, xp=xp2, status=st)
    assert ops.read_status(st) == 0
    for f in LAYOUT_FIELDS:
        assert torch.equal(getattr(L1, f), getattr(L2, f)), f
    assert torch.equal(xp1, xp2)
    assert int(L1.work.abs().sum().item()) == 0
    return L1, xp1


@pytest.mark.parametrize("cfg", [1, 2, 4, 5])
def test_dispatch_in_one_call_equals_two_calls(cfg):
    s = W.config(cfg)
    _fused_and_separate_bf16(s, W.tokens(s, device=DEV))


@pytest.mark.parametrize("T,H,E,K,R", [(1, 8, 1, 1, 1), (3, 4096, 512, 16, 8),
                                       (777, 520, 33, 5, 3), (2049, 40, 512, 16, 8),
                                       (100, 16384, 8, 2, 2), (40000, 64, 4, 2, 2)])
def test_dispatch_in_one_call_matches_oracle(T, H, E, K, R):
    s = W.Spec("fused", T, H, E, K, R, "uniform", seed=17 + T + H)
    x = W.tokens(s)
    L, xp = _fused_and_separate_bf16(s, x.to(DEV))
    ref = oracle.layout(W.topk_ids(s).numpy(), E, R)
    assert np.array_equal(L.dst_row.cpu().numpy()[:T * K], ref.dst_row)
    assert np.array_equal(L.expert_offsets.cpu().numpy(), ref.offsets)
    xp_ref = np.full((ref.P_cap, H), SENT, np.uint16)
    oracle.permute_rows(W.as_u16(x), ref.dst_row, K, ref.counts, ref.offsets, xp_ref)
    assert np.array_equal(dev_u16(xp), xp_ref)
    cnt = L.tile_ready.cpu().numpy().view(np.uint32)
    assert np.all(cnt[:ref.P // 128] == 128) and np.all(cnt[ref.P // 128:] == 0)


def test_dispatch_in_one_call_strided_rows():
    s = W.config(5).with_(T=3001, H=264)
    x = W.tokens(s)
    wide = torch.zeros((s.T, s.H + 16), dtype=torch.bfloat16)
    wide[:, 8:8 + s.H] = x
    _fused_and_separate_bf16(s, wide.to(DEV)[:, 8:8 + s.H])


@pytest.mark.parametrize("T,H,E,K,R", [(2048, 7168, 256, 8, 8), (300, 20480, 24, 4, 4),
                                       (50, 128, 3, 2, 1)])
def test_dispatch_in_one_call_e4m3(T, H, E, K, R):
    s = W.config(3).with_(T=T, H=H, E=E, K=K, R=R)
    ids = W.topk_ids(s).to(DEV)
    codes = W.e4m3_codes(s, device=DEV)
    xs = W.block_scales(s, device=DEV)
    st = ops.new_status()
    L1, xp1, xps1 = ops.moe_dispatch(ids, codes, E, R, x_scales=xs, status=st)
    L2 = ops.moe_dispatch_layout(ids, E, R, status=st)
    xp2, xps2 = ops.moe_dispatch_permute(codes, L2, x_scales=xs, status=st)
    assert ops.read_status(st) == 0
    P = int(L1.expert_offsets[E])
    for f in LAYOUT_FIELDS:
        assert torch.equal(getattr(L1, f), getattr(L2, f)), f
    assert torch.equal(xp1[:P], xp2[:P])
    assert torch.equal(xps1[:P].view(torch.int32), xps2[:P].view(torch.int32))
    assert int(L1.work.abs().sum().item()) == 0


def test_dispatch_in_one_call_in_cuda_graph():
    s = W.config(4)
    ids = W.topk_ids(s).to(DEV)
    x = W.tokens(s, device=DEV)
    sc = W.topk_scales(s).to(DEV)
    L = ops.alloc_layout(s.T, s.K, s.E, s.R, DEV)
    xp = torch.empty((L.P_cap, s.H), dtype=torch.bfloat16, device=DEV)
    out = torch.empty((s.T, s.H), dtype=torch.bfloat16, device=DEV)
    st = ops.new_status()

    def step():
        ops.moe_dispatch(ids, x, s.E, s.R, layout=L, xp=xp, status=st)
        ops.moe_combine(xp, L.dst_row, sc, out=out, status=st)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for seed_offset in (1, 2):
        s2 = W.config(4, seed_offset)
        ids.copy_(W.topk_ids(s2).to(DEV))
        x.copy_(W.tokens(s2, device=DEV))
        graph.replay()
        torch.cuda.synchronize()
        got = [t.clone() for t in (L.dst_row, L.expert_offsets, out)]
        P = int(L.expert_offsets[s.E])
        got_xp = xp[:P].clone()
        step()
        torch.cuda.synchronize()
        for a, b in zip(got, (L.dst_row, L.expert_offsets, out)):
            assert torch.equal(a, b)
        assert torch.equal(got_xp, xp[:P])
        assert int(L.work.abs().sum().item()) == 0
    assert ops.read_status(st) == 0
    del graph


@pytest.mark.parametrize("kind", ["range", "duplicate"])
def test_dispatch_in_one_call_reports_bad_ids(kind):
    """Ids out of range or repeated inside a token: the status carries the
    oracle's error, the layout and the expert-major buffer equal the
    oracle's (an out-of-range slot takes no row; a repeated id is placed
    twice), and the scheduling words are back at zero."""
    s = W.config(4).with_(H=256)
    ids = W.topk_ids(s).clone()
    if kind == "range":
        ids[100, 2] = s.E
        ids[2000, 0] = -3
        expect = oracle.ERR_EXPERT_RANGE
    else:
        ids[555, 1] = ids[555, 0]
        expect = oracle.ERR_DUPLICATE_EXPERT
    ref = oracle.layout(ids.numpy(), s.E, s.R)
    assert ref.status == expect
    x = W.tokens(s)
    st = ops.new_status()
    L = ops.alloc_layout(s.T, s.K, s.E, s.R, DEV)
    xp = torch.zeros((L.P_cap, s.H), dtype=torch.bfloat16, device=DEV)
    xp.view(torch.int16).fill_(SENT)
    ops.moe_dispatch(ids.to(DEV), x.to(DEV), s.E, s.R, layout=L, xp=xp, status=st)
    assert ops.read_status(st) == expect
    assert np.array_equal(L.dst_row.cpu().numpy(), ref.dst_row)
    assert np.array_equal(L.row_src.cpu().numpy()[:ref.P_cap], ref.row_src)
    assert np.array_equal(L.expert_offsets.cpu().numpy(), ref.offsets)
    xp_ref = np.full((ref.P_cap, s.H), SENT, np.uint16)
    oracle.permute_rows(W.as_u16(x), ref.dst_row, s.K, ref.counts, ref.offsets, xp_ref)
    assert np.array_equal(dev_u16(xp), xp_ref)
    assert int(L.work.abs().sum().item()) == 0
