"""Pins of the oracle's DVL allocation and packing (CPU only).

Expected values come from hand-worked cases, from brute force over every
verify-length vector that fits the budget (B <= 4, L <= 4), from math.prod
(left-to-right fp64 products) and itertools.accumulate (the scan)."""
import itertools
import json
import math
import os

import numpy as np
import pytest

import oracle


def _check_slot_map(res, B, L, budget):
    vl, off, sm = res["verify_len"], res["offsets"], res["slot_map"]
    assert list(off) == [0] + list(itertools.accumulate(int(v) + 1 for v in vl))
    assert len(sm) == budget
    for s in range(budget):
        if s < off[B]:
            b = int(np.searchsorted(off, s, side="right")) - 1
            assert sm[s] == b * (L + 1) + (s - off[b])
        else:
            assert sm[s] == -1


def test_golden_hand_cases(golden_dir):
    with open(os.path.join(golden_dir, "dvl_hand.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        s = np.array(c["scores"], np.float32)
        B, L = s.shape
        for budget, want in c["budgets"].items():
            r = oracle.dvl_allocate(s, int(budget))
            assert list(r["verify_len"]) == want, (c["name"], budget)
            _check_slot_map(r, B, L, int(budget))
        r = oracle.dvl_allocate(s, 5)
        assert list(r["offsets"]) == c["offsets_at_5"]
        assert list(r["slot_map"]) == c["slot_map_at_5"]
        if "slot_map_at_7" in c:
            assert list(oracle.dvl_allocate(s, 7)["slot_map"]) == c["slot_map_at_7"]


def test_prefix_products_left_to_right():
    rng = np.random.default_rng(0)
    s = rng.random((5, 9)).astype(np.float32)
    r = oracle.dvl_allocate(s, 5)
    for b in range(5):
        for i in range(9):
            assert r["prefix"][b, i] == math.prod(float(v) for v in s[b, :i + 1])


@pytest.mark.parametrize("B,L", [(1, 4), (2, 3), (3, 2), (4, 4), (3, 4)])
def test_greedy_matches_brute_force(B, L):
    rng = np.random.default_rng(100 * B + L)
    for trial in range(6):
        s = rng.beta(6.0, 2.0, size=(B, L)).astype(np.float32)
        if trial % 2:
            s = -np.sort(-s, axis=1)
        P = np.array([[math.prod(float(v) for v in s[b, :i + 1]) for i in range(L)] for b in range(B)])
        for budget in range(B, B * (L + 1) + 2):
            r = oracle.dvl_allocate(s, budget)
            assert r["flags"] == 0
            got = sum(P[b, :r["verify_len"][b]].sum() for b in range(B))
            best, arg = -1.0, []
            for ell in itertools.product(range(L + 1), repeat=B):
                if sum(e + 1 for e in ell) > budget:
                    continue
                val = sum(P[b, :ell[b]].sum() for b in range(B))
                if val > best + 1e-15:
                    best, arg = val, [ell]
                elif abs(val - best) <= 1e-15:
                    arg.append(ell)
            assert abs(got - best) <= 1e-14 * max(1.0, best), (s, budget)
            if len(arg) == 1:
                assert tuple(r["verify_len"]) == arg[0]
            assert int(r["offsets"][B]) == min(budget, B * (L + 1))
            _check_slot_map(r, B, L, budget)


def test_budget_edges_and_errors():
    s = np.full((3, 4), 0.7, np.float32)
    assert list(oracle.dvl_allocate(s, 3)["verify_len"]) == [0, 0, 0]
    assert list(oracle.dvl_allocate(s, 15)["verify_len"]) == [4, 4, 4]
    assert list(oracle.dvl_allocate(s, 100)["verify_len"]) == [4, 4, 4]
    with pytest.raises(ValueError):
        oracle.dvl_allocate(s, 2)
    bad = s.copy()
    bad[1, 2] = 1.5
    assert oracle.dvl_allocate(bad, 6)["flags"] & oracle.FLAG_SCORES
    bad[1, 2] = np.nan
    assert oracle.dvl_allocate(bad, 6)["flags"] & oracle.FLAG_SCORES


def test_half_capacity_rows_are_prefixes():
    rng = np.random.default_rng(5)
    B, L = 32, 16
    s = -np.sort(-rng.beta(6.0, 2.0, size=(B, L)), axis=1).astype(np.float32)
    budget = B * (L + 1) // 2
    r = oracle.dvl_allocate(s, budget)
    assert budget == 272 and int(r["offsets"][B]) == 272
    P = r["prefix"]
    # every selected product is >= every unselected one
    sel = np.zeros((B, L), bool)
    for b in range(B):
        sel[b, :r["verify_len"][b]] = True
    assert P[sel].min() >= P[~sel].max()


def test_pack_places_rows():
    rng = np.random.default_rng(6)
    B, L, V = 3, 4, 16
    dense = rng.integers(0, 65535, size=(B, L + 1, V), dtype=np.uint16)
    r = oracle.dvl_allocate(rng.random((B, L)).astype(np.float32), 8)
    packed = oracle.pack(dense, r["verify_len"], r["offsets"], 8)
    for b in range(B):
        for i in range(r["verify_len"][b] + 1):
            np.testing.assert_array_equal(packed[r["offsets"][b] + i], dense[b, i])
