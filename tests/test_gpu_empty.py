"""An empty batch (T = 0) through every call: the layout reports zero
counts and offsets, every other call succeeds without writing anything, and
buffers without rows may be empty tensors (NULL pointers at the C ABI)."""
import pytest
import torch

from _gpu_util import ensure_lib
from combine_moe_dispatch_05_b200 import ops

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_lib()


@pytest.mark.parametrize("K,E,R,H", [(8, 256, 8, 7168), (2, 8, 2, 128), (16, 512, 4, 1024)])
def test_every_call_accepts_an_empty_batch(K, E, R, H):
    st = ops.new_status()
    ids = torch.zeros((0, K), dtype=torch.int32, device=DEV)
    L = ops.alloc_layout(0, K, E, R, DEV)
    assert L.P_cap == 0
    L.expert_counts.fill_(7)
    L.expert_offsets.fill_(7)
    L.rank_counts.fill_(7)
    L.rank_offsets.fill_(7)
    ops.moe_dispatch_layout(ids, E, R, layout=L, status=st)
    torch.cuda.synchronize()
    assert ops.read_status(st) == 0
    assert not L.expert_counts.any() and not L.expert_offsets.any()
    assert not L.rank_counts.any() and not L.rank_offsets.any()

    x = torch.empty((0, H), dtype=torch.bfloat16, device=DEV)
    xp = ops.moe_dispatch_permute(x, L, status=st)
    assert xp.shape == (0, H)
    q, qs = ops.moe_quantize_e4m3(x, status=st)
    assert q.shape == (0, H) and qs.shape == (0, H // 128)
    xq, xqs = ops.moe_dispatch_permute(q, L, x_scales=qs, status=st)
    assert xq.shape == (0, H) and xqs.shape == (0, H // 128)
    fq, fqs = ops.moe_dispatch_permute_quant(x, L, status=st)
    assert fq.shape == (0, H)
    sc = torch.empty((0, K), dtype=torch.float32, device=DEV)
    out = ops.moe_combine(xp, L.dst_row[:0], sc, P_cap=0, status=st)
    assert out.shape == (0, H)
    out = ops.moe_combine(xp, L.dst_row[:0], sc, shared_x=x, P_cap=0, status=st)
    assert out.shape == (0, H)
    gy, gs = ops.moe_combine_bwd(x, xp, sc, L, status=st)
    assert gy.shape == (0, H) and gs.shape == (0, K)
    gx = ops.moe_dispatch_bwd(xp, L.dst_row[:0], 0, K, P_cap=0, status=st)
    assert gx.shape == (0, H)
    res = ops.moe_dispatch_permute_consume(x, L, status=st)
    assert res[0].shape == (0, H)
    torch.cuda.synchronize()
    assert ops.read_status(st) == 0


def test_binding_rejects_inconsistent_shapes():
    """The binding refuses shapes that would make a kernel read or write past
    a buffer, before anything is launched."""
    st = ops.new_status()
    ids = torch.randint(0, 8, (64, 1), dtype=torch.int32, device=DEV)
    L = ops.moe_dispatch_layout(ids, 8, 2, status=st)
    x = torch.zeros((65, 128), dtype=torch.bfloat16, device=DEV)          # one row too many
    with pytest.raises(ValueError):
        ops.moe_dispatch_permute(x, L)
    with pytest.raises(ValueError):
        ops.moe_dispatch_permute_quant(x, L)
    y = torch.zeros((L.P_cap, 128), dtype=torch.bfloat16, device=DEV)
    sc = torch.ones((64, 2), dtype=torch.float32, device=DEV)              # K=2 > layout's 1
    with pytest.raises(ValueError):
        ops.moe_combine(y, L.dst_row, sc)                                  # dst_row too short
    with pytest.raises(ValueError):
        ops.moe_combine(y, L.dst_row, sc[:, :1], P_cap=L.P_cap + 1)        # P_cap past y
    with pytest.raises(ValueError):
        ops.moe_combine(y, L.dst_row, sc[:, :1], shared_x=x)               # shared_x rows
    with pytest.raises(ValueError):
        ops.moe_dispatch_bwd(y, L.dst_row, 64, 2)                          # dst_row too short
    g = torch.zeros((64, 128), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(ValueError):
        ops.moe_combine_bwd(g, y[:-1], sc[:, :1], L)                       # y shorter than P_cap
    with pytest.raises(ValueError):
        ops.moe_combine_bwd(g, y, sc, L)                                   # K differs from layout
    torch.cuda.synchronize()
    assert ops.read_status(st) == 0
