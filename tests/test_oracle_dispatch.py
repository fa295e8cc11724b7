"""Pins for the oracle's dispatch layout and permute.

Against: a hand-worked example (tests/golden), an independent brute-force
placement written here with numpy primitives (sort / cumsum), and the
invariants the method must keep on every workload: counts sum to T*K, every
(token, k) slot gets exactly one row, offsets are 128-aligned, rows of an
expert are in ascending token order, padding rows are zero, rows past P are
untouched.
"""
import json
import os

import numpy as np
import pytest

import oracle
from combine_moe_dispatch_05_b200 import workloads as W

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def brute_layout(ids, E, R):
    """Independent restatement: group slots by expert with a stable sort."""
    T, K = ids.shape
    flat = ids.reshape(-1).astype(np.int64)
    counts = np.bincount(flat, minlength=E).astype(np.int64)
    padded = -(-counts // 128) * 128
    offsets = np.concatenate([[0], np.cumsum(padded)])
    order = np.argsort(flat, kind="stable")      # slots grouped by expert, slot order kept
    dst = np.empty(T * K, np.int64)
    start = np.concatenate([[0], np.cumsum(counts)])
    for e in range(E):
        sl = order[start[e]:start[e + 1]]
        dst[sl] = offsets[e] + np.arange(len(sl))
    El = E // R
    rank_counts = counts.reshape(R, El).sum(1)
    rank_offsets = np.concatenate([offsets[0:E:El], [offsets[E]]])
    return counts, offsets, rank_counts, rank_offsets, dst


def check_invariants(ids, L, E, R):
    T, K = ids.shape
    assert L.status == oracle.OK
    assert L.counts.sum() == T * K
    assert np.all(L.offsets % 128 == 0)
    assert np.all(np.diff(L.offsets) >= L.counts)
    assert np.all(np.diff(L.offsets) - L.counts < 128)
    assert np.all((L.counts == 0) == (np.diff(L.offsets) == 0))  # empty experts take no rows
    d = L.dst_row
    assert d.min() >= 0 and d.max() < L.P
    assert len(np.unique(d)) == T * K                              # injective
    assert np.array_equal(L.row_src[d], np.arange(T * K))           # row_src o dst_row = id
    assert (L.row_src >= 0).sum() == T * K                         # every other row is -1
    assert np.all(L.row_src[L.P:] == -1)
    flat = ids.reshape(-1)
    e_of_row = np.searchsorted(L.offsets, d, side="right") - 1
    assert np.array_equal(e_of_row, flat)                          # row lies in its expert
    for e in range(E):                                             # ascending tokens inside expert
        rows = L.row_src[L.offsets[e]:L.offsets[e] + L.counts[e]]
        assert np.all(rows >= 0)
        assert np.all(np.diff(rows // K) > 0)
    El = E // R
    assert np.array_equal(L.rank_offsets[:-1], L.offsets[0:E:El])
    assert np.array_equal(L.rank_counts, L.counts.reshape(R, El).sum(1))


def test_golden_hand_worked_layout():
    g = json.load(open(os.path.join(GOLD, "layout_T5_K2_E4_R2.json")))
    ids = np.array(g["ids"], np.int32)
    L = oracle.layout(ids, g["E"], g["R"])
    assert L.status == oracle.OK
    assert L.P_cap == g["P_cap"] == oracle.padded_capacity(g["T"], g["K"], g["E"])
    assert L.counts.tolist() == g["counts"]
    assert L.offsets.tolist() == g["offsets"]
    assert L.rank_counts.tolist() == g["rank_counts"]
    assert L.rank_offsets.tolist() == g["rank_offsets"]
    assert L.dst_row.tolist() == g["dst_row"]
    expect = np.full(g["P_cap"], -1)
    for k, v in g["row_src_nonneg"].items():
        expect[int(k)] = v
    assert np.array_equal(L.row_src, expect)
    assert L.P == g["P"]


@pytest.mark.parametrize("seed", range(40))
def test_layout_matches_brute_force_tiny(seed):
    rng = np.random.default_rng(seed)
    E = int(rng.choice([1, 2, 3, 4, 6, 8]))
    K = int(rng.integers(1, E + 1))
    T = int(rng.integers(0, 300))
    divisors = [r for r in range(1, E + 1) if E % r == 0]
    R = int(rng.choice(divisors))
    ids = np.stack([rng.permutation(E)[:K] for _ in range(T)]).astype(np.int32).reshape(T, K)
    L = oracle.layout(ids, E, R)
    counts, offsets, rc, ro, dst = brute_layout(ids, E, R)
    assert np.array_equal(L.counts, counts)
    assert np.array_equal(L.offsets, offsets)
    assert np.array_equal(L.rank_counts, rc)
    assert np.array_equal(L.rank_offsets, ro)
    assert np.array_equal(L.dst_row, dst)
    if T:
        check_invariants(ids, L, E, R)


@pytest.mark.parametrize("cfg", [1, 2, 4, 5])
def test_layout_invariants_on_workloads(cfg):
    s = W.config(cfg)
    ids = W.topk_ids(s).numpy()
    L = oracle.layout(ids, s.E, s.R)
    check_invariants(ids, L, s.E, s.R)
    counts, offsets, rc, ro, dst = brute_layout(ids, s.E, s.R)
    assert np.array_equal(L.dst_row, dst)
    assert np.array_equal(L.offsets, offsets)


def test_layout_capacity_bound_is_tight():
    # every expert gets exactly one token: P = 128 * E = T*K + 127*E
    E, K = 16, 4
    T = 4
    ids = np.arange(16, dtype=np.int32).reshape(T, K)
    L = oracle.layout(ids, E, 1)
    assert L.P == 128 * E == T * K + 127 * E
    assert L.P_cap == L.P


def test_layout_multi_tile_and_empty_expert():
    T = 300
    ids = np.full((T, 1), 1, np.int32)
    L = oracle.layout(ids, 3, 1)
    assert L.counts.tolist() == [0, 300, 0]
    assert L.offsets.tolist() == [0, 0, 384, 384]
    assert np.array_equal(L.dst_row, np.arange(T))
    assert np.all(L.row_src[300:] == -1)


def test_layout_validation():
    ids = np.array([[0, 1], [1, 5]], np.int32)     # 5 out of range for E=4
    L = oracle.layout(ids, 4, 1)
    assert L.status == oracle.ERR_EXPERT_RANGE
    assert L.dst_row[3] == -1 and L.counts.sum() == 3
    ids = np.array([[0, 0], [1, 2]], np.int32)     # repeated id in a row
    L = oracle.layout(ids, 4, 2)
    assert L.status == oracle.ERR_DUPLICATE_EXPERT
    ids = np.array([[-1, 0]], np.int32)
    assert oracle.layout(ids, 4, 1).status == oracle.ERR_EXPERT_RANGE
    assert oracle.layout(np.zeros((2, 1), np.int32), 6, 4).status == oracle.ERR_INVALID_ARG
    assert oracle.layout(np.zeros((2, 1), np.int32), 4, 1, P_cap=128).status == oracle.ERR_CAPACITY


@pytest.mark.parametrize("dtype,width", [(np.uint16, 40), (np.uint8, 256), (np.float32, 7)])
def test_permute_rows_bytewise(dtype, width):
    rng = np.random.default_rng(1)
    T, K, E = 77, 3, 5
    ids = np.stack([rng.permutation(E)[:K] for _ in range(T)]).astype(np.int32)
    L = oracle.layout(ids, E, 1)
    raw = rng.integers(0, 2**31, size=(T, width + 3)).astype(np.int64)
    x_full = raw.astype(dtype) if dtype != np.float32 else rng.standard_normal((T, width + 3)).astype(np.float32)
    x = x_full[:, 1:width + 1]                      # strided rows
    sentinel = np.array(0xAB, np.uint8)
    xp = np.full((L.P_cap, width), 0, dtype)
    xp.view(np.uint8)[...] = sentinel
    oracle.permute_rows(x, L.dst_row, K, L.counts, L.offsets, xp)
    for t in range(T):
        for k in range(K):
            assert np.array_equal(xp[L.dst_row[t * K + k]].view(np.uint8), x[t].copy().view(np.uint8))
    pad = [p for p in range(L.P) if L.row_src[p] < 0]
    assert len(pad) == L.P - T * K
    assert np.all(xp[pad].view(np.uint8) == 0)
    assert np.all(xp[L.P:].view(np.uint8) == 0xAB)   # untouched capacity rows


def test_tile_checksums_match_numpy_and_detect_swaps():
    rng = np.random.default_rng(2)
    xp = rng.integers(0, 2**16, size=(512, 24)).astype(np.uint16)
    xs = rng.standard_normal((512, 2)).astype(np.float32)
    got = oracle.tile_checksums(xp, 4, xs)
    for j in range(4):
        w = np.concatenate([xp[j * 128:(j + 1) * 128].reshape(-1).view(np.uint32),
                            xs[j * 128:(j + 1) * 128].reshape(-1).view(np.uint32)]).astype(np.uint64)
        i = np.arange(len(w), dtype=np.uint64)
        assert got[j] == int((w * (2 * i + 1)).sum() % 2**32)
    xp2 = xp.copy()
    xp2[[3, 4]] = xp2[[4, 3]]
    assert oracle.tile_checksums(xp2, 4, xs)[0] != got[0]
