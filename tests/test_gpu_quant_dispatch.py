"""GPU parity: fused quantise-on-dispatch (moe_dispatch_permute_quant) against
the oracle's quantiser followed by its permute, byte for byte (codes and
scales), including padding rows (code 0, scale 0), untouched rows past P and
complete chunk counters."""
import numpy as np
import pytest
import torch

import oracle
from _gpu_util import ensure_lib
from combine_moe_dispatch_05_b200 import ops
from combine_moe_dispatch_05_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_lib()


def run(s, strided=False, scales_offset=0):
    ids = W.topk_ids(s)
    x = W.tokens(s)
    ref = oracle.layout(ids.numpy(), s.E, s.R)
    q_ref, s_ref = oracle.quantize_e4m3(W.as_u16(x))
    xp_ref = np.full((ref.P_cap, s.H), 0xA5, np.uint8)
    xs_ref = np.full((ref.P_cap, s.H // 128), -3.0, np.float32)
    oracle.permute_rows(q_ref, ref.dst_row, s.K, ref.counts, ref.offsets, xp_ref)
    oracle.permute_rows(s_ref, ref.dst_row, s.K, ref.counts, ref.offsets, xs_ref)

    st = ops.new_status()
    L = ops.moe_dispatch_layout(ids.to(DEV), s.E, s.R, status=st)
    if strided:
        wide = torch.zeros((s.T, s.H + 64), dtype=torch.bfloat16)
        wide[:, 32:32 + s.H] = x
        xd = wide.to(DEV)[:, 32:32 + s.H]
    else:
        xd = x.to(DEV)
    xp = torch.full((L.P_cap, s.H), 0xA5, dtype=torch.uint8, device=DEV)
    # scales_offset > 0 moves the scale buffer off 16-byte alignment
    flat = torch.full((L.P_cap * (s.H // 128) + scales_offset,), -3.0, dtype=torch.float32,
                      device=DEV)
    xs = flat[scales_offset:].view(L.P_cap, s.H // 128)
    ops.moe_dispatch_permute_quant(xd, L, xp=xp, xp_scales=xs, status=st)
    assert ops.read_status(st) == 0
    assert np.array_equal(xp.cpu().numpy(), xp_ref)
    assert np.array_equal(xs.cpu().numpy().view(np.uint32), xs_ref.view(np.uint32))
    cnt = L.tile_ready.cpu().numpy()
    assert np.all(cnt[:ref.P // 128] == 128) and np.all(cnt[ref.P // 128:] == 0)
    return L, xd, xp, xs


@pytest.mark.parametrize("T,H,E,K,R", [(2000, 7168, 256, 8, 8), (333, 384, 12, 3, 4),
                                       (50, 128, 3, 2, 1), (1, 128, 1, 1, 1),
                                       (700, 1152, 512, 16, 8), (129, 896, 7, 7, 7),
                                       (90, 20480, 16, 4, 4), (61, 8704, 9, 3, 3),
                                       (75, 8320, 6, 5, 2), (5000, 1024, 4, 2, 2),
                                       (8192, 7168, 256, 8, 8)])
def test_fused_quant_dispatch_matches_oracle(T, H, E, K, R):
    run(W.config(3).with_(T=T, H=H, E=E, K=K, R=R))


def test_fused_quant_dispatch_strided_rows():
    run(W.config(3).with_(T=517, H=640, E=20, K=4, R=5), strided=True)


@pytest.mark.parametrize("H", [1024, 8704])
def test_fused_quant_dispatch_unaligned_scale_buffer(H):
    """A scale buffer that is only 4-byte aligned takes the plain-store path
    for the scales; codes and scales are unchanged."""
    run(W.config(3).with_(T=300, H=H, E=10, K=3, R=2), scales_offset=1)


def test_fused_equals_unfused_gpu_path_full_prefill():
    """Full prefill size (T=32768): the fused call equals the GPU quantiser
    followed by the GPU permute, byte for byte."""
    s = W.config(3)
    ids = W.topk_ids(s).to(DEV)
    x = W.tokens(s, device=DEV)
    st = ops.new_status()
    L = ops.moe_dispatch_layout(ids, s.E, s.R, status=st)
    q, qs = ops.moe_quantize_e4m3(x, status=st)
    xp1, xs1 = ops.moe_dispatch_permute(q, L, x_scales=qs, use_counters=False, status=st)
    P = int(L.expert_offsets[s.E])
    xp2, xs2 = ops.moe_dispatch_permute_quant(x, L, status=st)
    assert ops.read_status(st) == 0
    cnt = L.tile_ready.cpu().numpy()
    assert np.all(cnt[:P // 128] == 128) and np.all(cnt[P // 128:] == 0)
    assert torch.equal(xp1[:P], xp2[:P])
    assert torch.equal(xs1[:P].view(torch.int32), xs2[:P].view(torch.int32))


def test_fused_quant_dispatch_full_prefill_matches_oracle():
    """Full prefill size (T=32768, H=7168, E=256, K=8, Zipf 1.2): every code
    and scale of the expert-major buffer, padding rows and the untouched rows
    past P included, against the oracle's quantiser followed by its permute."""
    run(W.config(3))
