"""The allocation-free layout entry point, moe_dispatch_layout_static.

It serves callers that cannot allocate device memory when they call (engines
whose device memory is planned once and may not grow, callers without a
device allocator, hot paths that must not pay for cudaMalloc's device-wide
synchronisation): its scratch is a static array inside the library.  These
tests call it through the C ABI and check that it gives exactly what the
workspace-based moe_dispatch_layout gives, on several calls in a row (the
shared scratch keeps the previous call's contents, which must not matter),
and that sizes beyond its fixed scratch are refused before any launch.

This file is collected last so a run that stops at the first failure has
already run every other test.
"""
import ctypes

import pytest
import torch

from _gpu_util import ensure_lib
from combine_moe_dispatch_05_b200 import ops
from combine_moe_dispatch_05_b200 import workloads as W

DEV = "cuda"
SCRATCH = 4 << 20  # MOE_LAYOUT_STATIC_SCRATCH_BYTES


def _outputs(T, K, E, R):
    P_cap = ops.padded_capacity(T, K, E)
    i32 = dict(dtype=torch.int32, device=DEV)
    return dict(counts=torch.full((E,), -7, **i32), offsets=torch.full((E + 1,), -7, **i32),
                rank_counts=torch.full((R,), -7, **i32),
                rank_offsets=torch.full((R + 1,), -7, **i32),
                dst_row=torch.full((max(T * K, 1),), -7, **i32),
                row_src=torch.full((P_cap,), -7, **i32),
                tile_ready=torch.full(((P_cap + 127) // 128,), 99, **i32),
                status=torch.zeros(1, **i32), P_cap=P_cap)


def _call_static(ids, E, R, o):
    T, K = ids.shape
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return ops.lib().moe_dispatch_layout_static(
        p(ids), T, K, E, R, p(o["counts"]), p(o["offsets"]), p(o["rank_counts"]),
        p(o["rank_offsets"]), p(o["dst_row"]), p(o["row_src"]), p(o["tile_ready"]), o["P_cap"],
        p(o["status"]), stream)


@pytest.mark.gpu
def test_static_layout_matches_workspace_layout_on_consecutive_calls():
    ensure_lib()
    runs = [W.config(2), W.config(4), W.config(2, seed_offset=1), W.config(1)]
    for s in runs:
        ids = W.topk_ids(s).to(DEV)
        ref_status = ops.new_status()
        ref = ops.moe_dispatch_layout(ids, s.E, s.R, status=ref_status)
        o = _outputs(s.T, s.K, s.E, s.R)
        assert _call_static(ids, s.E, s.R, o) == ops.OK
        torch.cuda.synchronize()
        assert ops.read_status(ref_status) == 0 and int(o["status"].item()) == 0
        _assert_same(o, ref, s.name)


def _assert_same(o, ref, what):
    for mine, theirs in [("counts", ref.expert_counts), ("offsets", ref.expert_offsets),
                         ("rank_counts", ref.rank_counts), ("rank_offsets", ref.rank_offsets),
                         ("dst_row", ref.dst_row), ("row_src", ref.row_src),
                         ("tile_ready", ref.tile_ready)]:
        assert torch.equal(o[mine], theirs), (what, mine)


@pytest.mark.gpu
def test_static_layout_at_the_largest_accepted_size():
    """T = 116480, K = 8, E = 256: the largest size whose scratch fits the
    4 MiB array (455 count blocks fill 4193280 of its 4194304 bytes), so the
    end of the array is written and read back; ids are distinct per row and
    drawn at random.  Two calls in a row, each equal to the workspace form."""
    ensure_lib()
    T, K, E, R = 116480, 8, 256, 8
    assert ops.layout_workspace_bytes(T, K, E) == 4193280
    for seed in (5, 6):
        s = W.Spec("max", T, 64, E, K, R, "uniform", seed=seed)
        ids = W.topk_ids(s).to(DEV)
        ref_status = ops.new_status()
        ref = ops.moe_dispatch_layout(ids, E, R, status=ref_status)
        o = _outputs(T, K, E, R)
        assert _call_static(ids, E, R, o) == ops.OK
        torch.cuda.synchronize()
        assert ops.read_status(ref_status) == 0 and int(o["status"].item()) == 0
        _assert_same(o, ref, f"T={T} seed={seed}")


@pytest.mark.gpu
def test_static_layout_through_the_binding_allocates_no_workspace():
    """ops.moe_dispatch_layout_static with outputs from
    alloc_layout(with_workspace=False): no workspace tensor exists, and the
    result equals the workspace form's."""
    ensure_lib()
    s = W.config(2)
    ids = W.topk_ids(s).to(DEV)
    ref = ops.moe_dispatch_layout(ids, s.E, s.R)
    L = ops.alloc_layout(s.T, s.K, s.E, s.R, DEV, with_workspace=False)
    assert L.workspace is None
    st = ops.new_status()
    got = ops.moe_dispatch_layout_static(ids, s.E, s.R, layout=L, status=st)
    assert got is L and ops.read_status(st) == 0
    o = dict(counts=L.expert_counts, offsets=L.expert_offsets, rank_counts=L.rank_counts,
             rank_offsets=L.rank_offsets, dst_row=L.dst_row, row_src=L.row_src,
             tile_ready=L.tile_ready)
    _assert_same(o, ref, "binding")
    assert ops.moe_dispatch_layout_static(ids, s.E, s.R).workspace is None


@pytest.mark.gpu
def test_static_layout_refuses_sizes_beyond_its_scratch():
    ensure_lib()
    T, K, E = 116481, 8, 256            # needs just over 4 MiB of scratch
    assert ops.layout_workspace_bytes(T, K, E) > SCRATCH
    assert ops.layout_workspace_bytes(T - 1, K, E) <= SCRATCH
    fake = ctypes.c_void_p(256)          # never dereferenced: refused on the host
    rc = ops.lib().moe_dispatch_layout_static(fake, T, K, E, 8, fake, fake, fake, fake, fake,
                                              fake, fake, ops.padded_capacity(T, K, E), fake,
                                              None)
    assert rc == ops.ERR_UNSUPPORTED
