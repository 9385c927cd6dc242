"""Pins for oracle.routing_alternatives (CPU only): the routings of a token
whose top logits are closer than the tie gap, which the full-size GPU tests
use to check y on near-tie tokens without taking any GPU value as an input.

Pinned by closed forms (the two-way softmax is the logistic function of the
logit difference), hand-built ties, and brute force over small perturbations
of the logits; then mistakes are planted in a copy of the function and each
must fail a pin.  The gate rule followed is the softmax over the Top-K logits
of the layer equation ("Mixtral of Experts" section 2.1; Part 3, Step 3 of
"Mixture of Experts: Why Mixtral Only Wakes Up Two Specialists")."""
import inspect
import itertools
import math
import textwrap

import numpy as np
import pytest

import oracle

GAP = 1e-4


def logistic(z):
    return 1.0 / (1.0 + math.exp(-z))


def as_set(alts):
    return {tuple(int(e) for e in i) for i, _ in alts}


def pin_no_tie_is_the_router(ra):
    rng = np.random.default_rng(7)
    x = rng.standard_normal((40, 16))
    Wg = rng.standard_normal((16, 8))
    idx, gate, logits = oracle.router(x, Wg, 2)
    for t in range(40):
        srt = np.sort(logits[t])[::-1]
        if (srt[:3][:-1] - srt[1:3]).min() < 10 * GAP:
            continue
        alts = ra(logits[t], 2, GAP)
        assert len(alts) == 1
        assert np.array_equal(alts[0][0], idx[t])
        a, b = logits[t][idx[t]]
        assert abs(alts[0][1][0] - logistic(a - b)) < 1e-14
        assert abs(alts[0][1][1] - logistic(b - a)) < 1e-14


def pin_tie_at_the_kth_place(ra):
    alts = ra([3.0, 2.0, 2.0 + 5e-5, 0.0], 2, GAP)
    assert [tuple(i) for i, _ in alts] == [(0, 2), (0, 1)]
    assert abs(alts[0][1][0] - logistic(3.0 - (2.0 + 5e-5))) < 1e-14
    assert abs(alts[1][1][0] - logistic(1.0)) < 1e-14
    assert abs(alts[1][1][1] - logistic(-1.0)) < 1e-14


def pin_exact_tie_lower_index_first(ra):
    alts = ra([1.0, 1.0, 0.0], 2, GAP)
    assert [tuple(i) for i, _ in alts] == [(0, 1), (1, 0)]
    for _, g in alts:
        assert np.allclose(g, [0.5, 0.5], rtol=0, atol=1e-15)


def pin_k1(ra):
    alts = ra([1.0, 1.0 + 5e-5, 0.5], 1, GAP)
    assert [tuple(i) for i, _ in alts] == [(1,), (0,)]
    assert all(g[0] == 1.0 for _, g in alts)


def pin_chain_past_k_plus_one(ra):
    alts = ra([5.0, 1.0, 1.0 + 3e-5, 1.0 + 6e-5], 2, GAP)
    assert [tuple(i) for i, _ in alts] == [(0, 3), (0, 2), (0, 1)]


def pin_gap_is_strict(ra):
    assert len(ra([3.0, 2.0, 2.0 - 2 * GAP, 0.0], 2, GAP)) == 1
    assert len(ra([3.0, 2.0, 1.5, 1.5], 2, GAP)) == 1       # a tie below the K+1-th place


def pin_brute_force_perturbations(ra):
    """Every routing that moving each logit by less than GAP/2 produces (so any
    two logits closer than GAP can trade places) is among the alternatives,
    and the unperturbed routing comes first."""
    rng = np.random.default_rng(3)
    base = [0.0, 0.3, 0.3 + 4e-5, 0.3 + 8e-5, -0.2]
    for trial in range(6):
        L = np.array(base)[rng.permutation(5)]
        K = 1 + trial % 3
        alts = ra(L, K, GAP)
        got = as_set(alts)
        d = 0.49 * GAP
        seen = set()
        for delta in itertools.product((-d, 0.0, d), repeat=5):
            Lp = L + np.array(delta)
            order = sorted(range(5), key=lambda e: (-Lp[e], e))
            seen.add(tuple(order[:K]))
        assert seen <= got, (L, K, seen - got)
        own = sorted(range(5), key=lambda e: (-L[e], e))[:K]
        assert tuple(alts[0][0]) == tuple(own)
        for i, g in alts:
            assert abs(g.sum() - 1.0) < 1e-14 and (np.diff(g) <= 1e-3).all()


PINS = [pin_no_tie_is_the_router, pin_tie_at_the_kth_place, pin_exact_tie_lower_index_first, pin_k1,
        pin_chain_past_k_plus_one, pin_gap_is_strict, pin_brute_force_perturbations]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_routing_alternatives_pin(pin):
    pin(oracle.routing_alternatives)


MUTANTS = {
    "ascending_rank": ("key=lambda e: (-L[e], e)", "key=lambda e: (L[e], e)"),
    "ties_high_index": ("key=lambda e: (-L[e], e)", "key=lambda e: (-L[e], -e)"),
    "gap_not_strict": ("L[order[p]] >= gap", "L[order[p]] > 2 * gap"),
    "run_misses_last": ("members = order[a:b + 1]", "members = order[a:b]"),
    "one_place_short": ("m = min(b, K - 1) - a + 1", "m = max(1, min(b, K - 1) - a)"),
    "gates_unnormalised": ("g / g.sum()", "g"),
    "gates_over_all_logits": ("z = L[sel]", "z = L"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_routing_alternatives_mutant_is_caught(name):
    src = textwrap.dedent(inspect.getsource(oracle.routing_alternatives))
    old, new = MUTANTS[name]
    assert old in src, "mutation anchor not found: %r" % old
    ns = {"np": np}
    exec(compile(src.replace(old, new), "<mutant %s>" % name, "exec"), ns)
    mutant = ns["routing_alternatives"]
    caught = []
    for pin in PINS:
        try:
            pin(mutant)
        except (AssertionError, ValueError, IndexError, TypeError):
            caught.append(pin.__name__)
    assert caught, "no pin caught mutant %s" % name
