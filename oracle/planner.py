"""CPU oracle for the host balance planner (test infrastructure only).

Sources: DeepEP pull request "Intra-node compute compensation + overlap
robustness (CUDA719 fix)", Python section: a water-filling chunk-migration
planner with expert-affinity batching, a makespan guard, a cost-aware no-op
and a 128-aligned fine-balance pass; TEMPO summary, section 2 (cost
modelling): the time of a GPU's expert work is max-affine,
t = max(a + b*G, c + beta*N) with G activated expert replicas and N tokens,
and the tile-aware form adds b2 * (tiles - G) inside the first term, where a
tile is a 128-token M-tile (section 1).

Plain loops over small lists, written to follow those steps.  The pages give
the steps only by name; the reading taken for each is stated at the function
that implements it.  The library's C++ planner must produce the same plan,
move for move (all costs in double, evaluated in the same order).

A plan is a list of moves (expert, src_rank, dst_rank, tokens).
"""
from __future__ import annotations

import dataclasses

TILE = 128


@dataclasses.dataclass(frozen=True)
class Cost:
    a: float = 0.0      # fixed cost of a GPU's expert work
    b: float = 1.0      # activation floor: cost per activated expert replica
    b2: float = 0.0     # tile-aware term: cost per 128-token tile beyond one per replica
    c: float = 0.0      # fixed cost of the token-linear regime
    beta: float = 0.01  # cost per token
    mig: float = 0.0    # cost per migrated token, charged to the receiving rank


def rank_cost(load, migrated_in, cost):
    """t_r = max(a + b*G + b2*(tiles - G), c + beta*N) + mig * migrated_in
    over the experts with tokens on the rank: G of them, N tokens, tiles =
    sum of ceil(n_e / 128)."""
    G = N = tiles = 0
    for e in sorted(load):
        n = load[e]
        if n > 0:
            G += 1
            N += n
            tiles += (n + TILE - 1) // TILE
    t1 = cost.a + cost.b * G + cost.b2 * (tiles - G)
    t2 = cost.c + cost.beta * N
    return (t1 if t1 > t2 else t2) + cost.mig * migrated_in


def initial_loads(counts, R):
    """Expert e starts on logical rank e // (E/R) (contiguous blocks)."""
    El = len(counts) // R
    loads = [dict() for _ in range(R)]
    for e, n in enumerate(counts):
        loads[e // El][e] = int(n)
    return loads


def makespan(loads, mig_in, cost):
    return max(rank_cost(loads[r], mig_in[r], cost) for r in range(len(loads)))


def _moved(loads, mig_in, src, dst, e, n):
    """Copies of the two ranks' loads after moving n tokens of e src -> dst."""
    ls, ld = dict(loads[src]), dict(loads[dst])
    ls[e] -= n
    ld[e] = ld.get(e, 0) + n
    return ls, ld


def _chunk_for(loads, mig_in, cost, src, dst, e, fine):
    """Tokens to move.  Fine pass: one 128-token chunk (or the remainder).
    Water-filling pass: the largest whole number of chunks (the last one may
    be the remainder) after which dst costs no more than src; one chunk if no
    number does."""
    have = loads[src][e]
    one = TILE if have > TILE else have
    if fine:
        return one
    k = (have + TILE - 1) // TILE
    while k >= 1:
        n = k * TILE if k * TILE < have else have
        ls, ld = _moved(loads, mig_in, src, dst, e, n)
        if rank_cost(ld, mig_in[dst] + n, cost) <= rank_cost(ls, mig_in[src], cost):
            return n
        k -= 1
    return one


def plan(counts, R, cost: Cost, max_moves=256, min_gain=0.0):
    """Water-filling migration, then a 128-token fine-balance pass.

    Each step pairs the most expensive rank (src; the lowest index on ties)
    with the cheapest (dst; the lowest index on ties).  Experts on src are
    tried in this order (expert-affinity batching): those that already have
    tokens on dst first (no new replica there), then the most tokens on src,
    then the lower id.  A move is kept only if it lowers the makespan by more
    than min_gain (makespan guard; min_gain > 0 is the cost-aware no-op);
    otherwise the next expert is tried, and the pass ends when none helps or
    max_moves moves have been made.
    """
    loads = initial_loads(counts, R)
    mig_in = [0] * R
    moves = []
    before = makespan(loads, mig_in, cost)
    for fine in (False, True):
        while len(moves) < max_moves:
            costs = [rank_cost(loads[r], mig_in[r], cost) for r in range(R)]
            src = dst = 0
            for r in range(1, R):
                if costs[r] > costs[src]:
                    src = r
                if costs[r] < costs[dst]:
                    dst = r
            if src == dst:
                break
            cands = [e for e in loads[src] if loads[src][e] > 0]
            cands.sort(key=lambda e: (0 if loads[dst].get(e, 0) > 0 else 1, -loads[src][e], e))
            kept = False
            for e in cands:
                n = _chunk_for(loads, mig_in, cost, src, dst, e, fine)
                ls, ld = _moved(loads, mig_in, src, dst, e, n)
                trial = list(loads)
                trial[src], trial[dst] = ls, ld
                trial_mig = list(mig_in)
                trial_mig[dst] += n
                if makespan(trial, trial_mig, cost) < costs[src] - min_gain:
                    loads, mig_in = trial, trial_mig
                    moves.append((e, src, dst, n))
                    kept = True
                    break
            if not kept:
                break
    return moves, before, makespan(loads, mig_in, cost), loads


def ideal_makespan(counts, R, cost: Cost):
    """A lower bound for every plan: some rank holds at least 1/R of the
    activated experts (each expert needs a replica) and at least 1/R of the
    tokens, and the tile and migration terms are never negative."""
    G = sum(1 for n in counts if n > 0)
    N = sum(int(n) for n in counts)
    t1 = cost.a + cost.b * G / R
    t2 = cost.c + cost.beta * N / R
    return t1 if t1 > t2 else t2
