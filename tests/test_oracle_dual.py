"""Pins for the Lagrangian allocator: exhaustive search on tiny inputs (CPU only)."""
import itertools

import numpy as np
import pytest

from oracle import jolt


def tiny_units(seed=0, groups=2):
    """Two groups of a 2-layer, H=2, T=8, D=8 K cache with a step-1 grid and b in 0..4."""
    rng = np.random.default_rng(seed)
    L, H, T, D = 2 * groups, 2, 8, 8
    X = rng.standard_normal((L, H, T, D)) * np.linspace(2.0, 0.05, D)
    p = jolt.Plan(L=L, H=H, T=T, D=D, has_v=False, budget=3 * H * T * D, num_groups=groups,
                  encoder="exact", rank_step=1, rt_cap=8, bits=(0, 1, 2, 3, 4))
    E = {l * 2: jolt.analyse_layer_tensor(p, X[l], seed, l * 2)["E"] for l in range(L)}
    return p, jolt.build_units(p, E, jolt.kappa(D))


def brute_choose(u, lam):
    best = None
    for i in range(len(u.err)):
        key = (u.err[i] + lam * float(u.nbytes[i]), int(u.nbytes[i]), int(u.b[i]), int(u.rt[i]), int(u.rd[i]))
        if best is None or key < best[0]:
            best = (key, i)
    return best[1]


@pytest.mark.parametrize("lam", [0.0, 1e-6, 1e-4, 3e-3, 0.1, 10.0])
def test_inner_argmin_is_exhaustive(lam):
    _, units = tiny_units()
    for u in units:
        assert jolt.choose(u, lam) == brute_choose(u, lam)


def test_no_joint_assignment_beats_the_dual():
    p, units = tiny_units(1)
    idx, lam = jolt.dual_allocate(units, p.budget)
    best = sum(u.err[i] + lam * u.nbytes[i] for u, i in zip(units, idx))
    u0, u1 = units
    tot = (u0.err[:, None] + u1.err[None, :]) + lam * (u0.nbytes[:, None] + u1.nbytes[None, :])
    assert tot.min() >= best - 1e-9 * abs(best)


@pytest.mark.parametrize("seed", range(4))
def test_dual_equals_constrained_brute_force_at_hull_budgets(seed):
    """At a budget equal to the bytes chosen at some lambda, the dual is the exact optimum."""
    p, units = tiny_units(seed)
    u0, u1 = units
    errs = u0.err[:, None] + u1.err[None, :]
    byts = u0.nbytes[:, None] + u1.nbytes[None, :]
    for lam in (1e-5, 1e-4, 1e-3, 1e-2):
        bud = sum(int(u.nbytes[jolt.choose(u, lam)]) for u in units)
        idx, _ = jolt.dual_allocate(units, bud)
        got = sum(u.err[i] for u, i in zip(units, idx))
        assert sum(int(u.nbytes[i]) for u, i in zip(units, idx)) <= bud
        opt = errs[byts <= bud].min()
        assert abs(got - opt) <= 1e-12 * max(1.0, opt)


@pytest.mark.parametrize("seed", range(3))
def test_budget_always_met_and_gap_small(seed):
    p, units = tiny_units(seed)
    u0, u1 = units
    errs = u0.err[:, None] + u1.err[None, :]
    byts = u0.nbytes[:, None] + u1.nbytes[None, :]
    rng = np.random.default_rng(seed)
    for bud in rng.integers(64, 2 * 2 * 2 * 8 * 8 * 2, 20):
        idx, lam = jolt.dual_allocate(units, int(bud))
        tb = sum(int(u.nbytes[i]) for u, i in zip(units, idx))
        assert tb <= bud
        got = sum(u.err[i] for u, i in zip(units, idx))
        assert got >= errs[byts <= bud].min() - 1e-12


def test_infeasible_budget_raises():
    p, units = tiny_units()
    units = [jolt.Unit(u.group, u.kind, u.err[u.b > 0], u.nbytes[u.b > 0], u.b[u.b > 0],
                       u.rt[u.b > 0], u.rd[u.b > 0], u.energy) for u in units]
    minb = sum(int(u.nbytes.min()) for u in units)
    with pytest.raises(jolt.BudgetInfeasible):
        jolt.dual_allocate(units, minb - 1)
    idx, _ = jolt.dual_allocate(units, minb)
    assert sum(int(u.nbytes[i]) for u, i in zip(units, idx)) == minb


def test_three_units_exhaustive():
    p, units = tiny_units(5, groups=3)
    sub = []
    for u in units:                                   # thin the tables so 3-way search is cheap
        keep = (u.rt % 2 == 0) & (u.rd % 2 == 0)
        sub.append(jolt.Unit(u.group, u.kind, u.err[keep], u.nbytes[keep], u.b[keep], u.rt[keep],
                             u.rd[keep], u.energy))
    for lam in (1e-4, 1e-3):
        bud = sum(int(u.nbytes[jolt.choose(u, lam)]) for u in sub)
        idx, _ = jolt.dual_allocate(sub, bud)
        got = sum(u.err[i] for u, i in zip(sub, idx))
        best = np.inf
        for i, j in itertools.product(range(len(sub[0].err)), range(len(sub[1].err))):
            rest = bud - sub[0].nbytes[i] - sub[1].nbytes[j]
            ok = sub[2].nbytes <= rest
            if ok.any():
                best = min(best, sub[0].err[i] + sub[1].err[j] + sub[2].err[ok].min())
        assert abs(got - best) <= 1e-12 * max(1.0, best)
