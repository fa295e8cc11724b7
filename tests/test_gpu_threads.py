"""Several host threads calling the library at once, each on its own stream
and with its own row size (so each needs different launch settings): every
result still matches the oracle.  The library's per-device caches and
kernel attributes must be safe to share."""
import concurrent.futures

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


SHAPES = [(700, 7168, 64, 8, 8), (900, 2048, 32, 4, 4), (500, 20480, 16, 2, 2),
          (1200, 512, 128, 6, 8), (300, 8320, 24, 3, 3), (800, 4096, 8, 2, 1)]


def _one(i, T, H, E, K, R):
    s = W.Spec(f"thr{i}", T, H, E, K, R, "zipf", zipf_s=0.8, seed=700 + i)
    ids, x = W.topk_ids(s), W.tokens(s)
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        st = ops.new_status()
        L = ops.moe_dispatch_layout(ids.to(DEV), E, R, status=st, stream=stream)
        xp = ops.moe_dispatch_permute(x.to(DEV), L, status=st, stream=stream)
        q, qs = ops.moe_dispatch_permute_quant(x.to(DEV), L, use_counters=False, status=st,
                                               stream=stream)
    stream.synchronize()
    assert ops.read_status(st) == 0
    ref = oracle.layout(ids.numpy(), E, R)
    xp_ref = np.zeros((ref.P_cap, H), np.uint16)
    oracle.permute_rows(W.as_u16(x), ref.dst_row, K, ref.counts, ref.offsets, xp_ref)
    assert np.array_equal(W.as_u16(xp.cpu())[:ref.P], xp_ref[:ref.P])
    q_ref, s_ref = oracle.quantize_e4m3(W.as_u16(x))
    qp_ref = np.zeros((ref.P_cap, H), np.uint8)
    oracle.permute_rows(q_ref, ref.dst_row, K, ref.counts, ref.offsets, qp_ref)
    assert np.array_equal(q.cpu().numpy()[:ref.P], qp_ref[:ref.P])
    return True


def test_concurrent_host_threads_with_different_shapes():
    for rnd in range(3):
        with concurrent.futures.ThreadPoolExecutor(max_workers=len(SHAPES)) as ex:
            futs = [ex.submit(_one, i + 10 * rnd, *shape) for i, shape in enumerate(SHAPES)]
            assert all(f.result() for f in futs)
