"""The planner oracle's pins catch plausible mistakes.

Each case plants one mistake in the text of oracle/planner.py (a dropped
cost term, a wrong rounding, a flipped comparison, a lost ordering rule, a
missing guard), loads the mutated text as a module, and runs the oracle pins
of tests/test_planner.py against it in place of the oracle.  Every mutant
must fail at least one pin; the unmodified text, loaded the same way, must
pass them all.
"""
import os
import sys
import types

import pytest

import test_planner as TP

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle",
                   "planner.py")

MUTANTS = {
    "cost_drops_tile_term": ("t1 = cost.a + cost.b * G + cost.b2 * (tiles - G)",
                             "t1 = cost.a + cost.b * G"),
    "tiles_rounded_down": ("tiles += (n + TILE - 1) // TILE", "tiles += n // TILE"),
    "migration_not_charged": ("return (t1 if t1 > t2 else t2) + cost.mig * migrated_in",
                              "return (t1 if t1 > t2 else t2)"),
    "experts_dealt_round_robin": ("loads[e // El][e] = int(n)", "loads[e % R][e] = int(n)"),
    "fine_pass_moves_whole_expert": ("one = TILE if have > TILE else have", "one = have"),
    "water_filling_test_flipped": (
        "if rank_cost(ld, mig_in[dst] + n, cost) <= rank_cost(ls, mig_in[src], cost):",
        "if rank_cost(ld, mig_in[dst] + n, cost) >= rank_cost(ls, mig_in[src], cost):"),
    "no_expert_affinity": (
        "cands.sort(key=lambda e: (0 if loads[dst].get(e, 0) > 0 else 1, -loads[src][e], e))",
        "cands.sort(key=lambda e: (-loads[src][e], e))"),
    "no_makespan_guard": ("if makespan(trial, trial_mig, cost) < costs[src] - min_gain:",
                          "if True:"),
    "lower_bound_not_divided": ("t1 = cost.a + cost.b * G / R", "t1 = cost.a + cost.b * G"),
    "src_is_cheapest_rank": ("if costs[r] > costs[src]:", "if costs[r] < costs[src]:"),
}


def _load(text, name):
    mod = types.ModuleType(name)
    sys.modules[name] = mod  # dataclasses looks the defining module up by name
    try:
        exec(compile(text, name, "exec"), mod.__dict__)
    finally:
        del sys.modules[name]
    return mod


def _pins():
    yield TP.test_golden_hand_worked_plan, ()
    yield TP.test_golden_affinity_prefers_expert_already_on_dst, ()
    yield TP.test_golden_tile_term_and_rounded_up_tiles, ()
    yield TP.test_golden_affinity_decides_the_second_move, ()
    yield TP.test_golden_single_chunk_when_no_split_fits, ()
    yield TP.test_fine_chunk_is_one_tile_or_the_remainder, ()
    for seed in range(25):
        yield TP.test_oracle_invariants_and_independent_cost, (seed,)
    for counts, R in [([512, 0], 2), ([384, 128, 0, 0], 2), ([640, 0, 0], 3), ([300, 200], 2),
                      ([256, 256, 512, 0], 2)]:
        yield TP.test_oracle_against_exhaustive_search, (counts, R)


def _fails_a_pin(mod, monkeypatch):
    monkeypatch.setattr(TP, "OP", mod)
    for fn, args in _pins():
        try:
            fn(*args)
        except Exception:  # an assertion, or the mutant breaking outright
            return True
    return False


def test_original_text_passes_the_pins(monkeypatch):
    assert not _fails_a_pin(_load(open(SRC).read(), "planner_original"), monkeypatch)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_fails_a_pin(name, monkeypatch):
    old, new = MUTANTS[name]
    text = open(SRC).read()
    assert text.count(old) == 1, "the text to mutate must occur exactly once"
    assert _fails_a_pin(_load(text.replace(old, new), f"planner_{name}"), monkeypatch)
