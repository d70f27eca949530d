"""Pins for the oracle's measured-b refinement (CPU only).

After the dual has chosen (r_t, r_d, b) per unit with the phi(b) quantiser model, the
refinement measures the exact squared quantisation error of every allowed width at the chosen
ranks and runs the same dual again over b alone. These tests pin the measurement (it equals the
decoded error), the structure of the second dual (ranks kept, budgets met, every unit's width
optimal for the returned lambda) and the optimality of its widths for the bytes they spend.
"""
import numpy as np
import pytest

import synth
from oracle import jolt


def _total_bytes(plan, alloc):
    tot = 0
    for g, lay in enumerate(jolt.group_ranges(plan.L, plan.num_groups)):
        for k in plan.kinds():
            tot += len(lay) * jolt.layer_bytes(plan.H, plan.T, plan.D, *(int(v) for v in alloc[g, k]))
    return tot


def _plan(L, H, T, D, budget, groups, **kw):
    return jolt.Plan(L=L, H=H, T=T, D=D, has_v=False, budget=budget, num_groups=groups, encoder="exact",
                     rank_step=16, **kw)


@pytest.fixture(scope="module")
def x4():
    """Four layers of the config-0 generator (H = 8, T = 256, D = 128), float64."""
    cfg = synth.config(0, layers=4, rho=None)
    K, _ = synth.gen_cache_numpy(cfg)
    return K.astype(np.float64)


def test_measured_errors_equal_the_decoded_error(x4):
    """The refinement's measured error of the chosen width is the decoded error itself:
    X - X_hat = (Y - Y_hat) Pi^T with Pi orthogonal, so the sum over units of the measured
    errors at the chosen widths equals ||X - X_hat||^2."""
    L, H, T, D = x4.shape
    p = _plan(L, H, T, D, x4.size * 2 // 3, 2, measured_b=True)
    st, dbg = jolt.encode(p, x4, None, seed=11, spec=True)
    Xh, _ = jolt.decode(st, rounded=False)
    lhs = float(np.sum((x4 - Xh) ** 2))
    rhs = sum(dbg["measured"][(g, 0)][int(st.alloc[g, 0][2])] for g in range(p.num_groups))
    assert abs(lhs - rhs) <= 1e-10 * float(np.sum(x4 ** 2))


def test_second_dual_keeps_ranks_and_is_optimal_at_its_lambda(x4):
    """Ranks come from the first dual; every unit's width minimises measured error + lambda *
    bytes over the allowed widths at those ranks (ties: fewer bytes); the pool stays in budget."""
    L, H, T, D = x4.shape
    budget = x4.size * 2 // 3
    p0 = _plan(L, H, T, D, budget, 4)
    p1 = _plan(L, H, T, D, budget, 4, measured_b=True)
    st0, _ = jolt.encode(p0, x4, None, seed=11, spec=True)
    st1, dbg = jolt.encode(p1, x4, None, seed=11, spec=True)
    assert np.array_equal(st0.alloc[:, 0, :2], st1.alloc[:, 0, :2])
    assert _total_bytes(p1, st1.alloc) <= budget
    lam = dbg["lambdas"][0]
    for g, lay in enumerate(jolt.group_ranges(L, 4)):
        rt, rd, b = (int(v) for v in st1.alloc[g, 0])
        m = dbg["measured"][(g, 0)]
        cost = {bb: m[bb] + lam * len(lay) * jolt.layer_bytes(H, T, D, rt, rd, bb) for bb in p1.bits}
        best = min(cost.values())
        assert cost[b] == best
        ties = [bb for bb in p1.bits if cost[bb] == best]
        assert b == min(ties, key=lambda bb: (jolt.layer_bytes(H, T, D, rt, rd, bb), bb))


def test_refined_widths_are_optimal_for_their_bytes(x4):
    """A Lagrangian solution is optimal for its own byte count: no assignment of widths (ranks
    fixed) that spends at most the refined allocation's bytes has a smaller total measured
    error. Checked by enumerating all 5^4 assignments of four units."""
    import itertools
    L, H, T, D = x4.shape
    bits = (0, 1, 2, 3, 4)
    p = _plan(L, H, T, D, x4.size * 2 // 5, 4, measured_b=True, bits=bits)
    st, dbg = jolt.encode(p, x4, None, seed=11, spec=True)
    lay = jolt.group_ranges(L, 4)
    ranks = [(int(st.alloc[g, 0][0]), int(st.alloc[g, 0][1])) for g in range(4)]
    meas = [dbg["measured"][(g, 0)] for g in range(4)]

    def cost(assign):
        e = sum(meas[g][b] for g, b in enumerate(assign))
        nb = sum(len(lay[g]) * jolt.layer_bytes(H, T, D, *ranks[g], b) for g, b in enumerate(assign))
        return e, nb

    e1, nb1 = cost([int(st.alloc[g, 0][2]) for g in range(4)])
    assert nb1 <= p.budget
    for assign in itertools.product(bits, repeat=4):
        e, nb = cost(assign)
        if nb <= nb1:
            assert e >= e1 * (1 - 1e-12), (assign, e, e1)
