"""The cell planner (loopkv_plan_cells, host code in the C library) against a
brute-force oracle that enumerates every admissible plan of small models:
same optimum (reads, then damage, then storage), budgets respected, the final
loop never reuses, infeasible budgets reported, and a full 4 x 24 model
planned quickly."""

import time

import numpy as np
import pytest

from oracle.planner_oracle import plan_brute_force, plan_cost

CODE = {"q4": 0, "q2": 1, "reuse": 2}


@pytest.fixture(scope="module")
def m():
    import mixed_precision_kv_loopkv_b200 as pkg  # built at session start (conftest)
    return pkg


def _damage(rng, L, N):
    # 4-bit hurts least, 2-bit more, reuse varies (later loops tolerate it better)
    d4 = rng.integers(0, 4, (L, N))
    d2 = d4 + rng.integers(1, 10, (L, N))
    dr = rng.integers(0, 25, (L, N)) * (L - np.arange(L))[:, None]
    return np.stack([d4, d2, dr], axis=2).astype(np.int32)


def _as_choices(plan, L, N):
    return [[CODE[plan[l * N + j]] for j in range(N)] for l in range(L)]


@pytest.mark.parametrize("L,N", [(1, 3), (2, 2), (2, 3), (3, 2)])
@pytest.mark.parametrize("seed", range(6))
def test_matches_brute_force(m, L, N, seed):
    rng = np.random.default_rng(seed * 10 + L * 3 + N)
    dmg = _damage(rng, L, N)
    full_storage = 5 * L * N
    for q4 in (128, 131, 160):
        for frac_d, frac_s in ((1.0, 1.0), (0.5, 0.7), (0.25, 0.5), (0.1, 0.3)):
            db = int(dmg.sum(axis=2).max() * L * N * frac_d) // 2
            sb = int(full_storage * frac_s)
            want = plan_brute_force(dmg.tolist(), db, sb, q4)
            if want is None:
                with pytest.raises(Exception) as e:
                    m.loopkv_plan_cells(dmg, db, sb, q4)
                assert getattr(e.value, "status", None) == 2
                continue
            plan, reads = m.loopkv_plan_cells(dmg, db, sb, q4)
            got = plan_cost(dmg.tolist(), _as_choices(plan, L, N), q4)
            assert got == want[0], (got, want)
            assert reads == got[0]
            assert all(plan[(L - 1) * N + j] != "reuse" for j in range(N))


def test_budgets_trade_reads(m):
    rng = np.random.default_rng(5)
    L, N = 4, 24
    dmg = _damage(rng, L, N)
    prev = None
    for sb in (5 * L * N, 300, 250, 200):
        plan, reads = m.loopkv_plan_cells(dmg, 10 ** 6 // 1000, sb, 130)
        got = plan_cost(dmg.tolist(), _as_choices(plan, L, N), 130)
        assert got[2] <= sb and got[1] <= 1000 and got[0] == reads
        assert all(plan[(L - 1) * N + j] != "reuse" for j in range(N))
        if prev is not None:
            assert reads >= prev       # a tighter storage budget cannot read less
        prev = reads


def test_full_model_is_fast(m):
    rng = np.random.default_rng(9)
    dmg = _damage(rng, 4, 24)
    t0 = time.perf_counter()
    plan, reads = m.loopkv_plan_cells(dmg, 800, 330, 130)
    assert time.perf_counter() - t0 < 5.0
    assert len(plan) == 96


def test_invalid_and_infeasible(m):
    from mixed_precision_kv_loopkv_b200 import LoopKVError
    dmg = np.zeros((2, 2, 3), dtype=np.int32)
    with pytest.raises(LoopKVError) as e:
        m.loopkv_plan_cells(dmg, 0, 0, 128)      # storage 0 needs every cell reused: not allowed
    assert e.value.status == 2
    with pytest.raises(LoopKVError) as e:
        m.loopkv_plan_cells(-np.ones((2, 2, 3), dtype=np.int32), 10, 10, 128)
    assert e.value.status == 1
    with pytest.raises(LoopKVError) as e:
        m.loopkv_plan_cells(np.zeros((7, 1, 3), dtype=np.int32), 10, 10, 128)
    assert e.value.status == 1


def test_oracle_pinned_on_hand_worked_case():
    """Two loops, one layer, worked by hand: cell (0,0) damages 1/5/2 for
    4-bit/2-bit/reuse, cell (1,0) 0/4.  Budgets damage 3, storage 8: only
    'reuse of a 4-bit final cell' fits: reads 128 + 128, damage 2, storage 5.
    Unlimited budgets: a 2-bit final cell with the first loop reusing it or
    storing 2-bit both read 192; the reuse has less damage (6 vs 9).  Damage
    budget 1: only both cells 4-bit fit; budget 0: nothing."""
    dmg = [[[1, 5, 2]], [[0, 4, 0]]]
    best = plan_brute_force(dmg, 3, 8, 128)
    assert best[0] == (256, 2, 5) and best[1] == [[2], [0]]
    best = plan_brute_force(dmg, 100, 100, 128)
    assert best[0] == (192, 6, 3) and best[1] == [[2], [1]]
    assert plan_brute_force(dmg, 1, 100, 128)[0] == (256, 1, 10)   # both 4-bit
    assert plan_brute_force(dmg, 0, 100, 128) is None                # every plan damages


def test_library_on_hand_worked_case(m):
    dmg = np.array([[[1, 5, 2]], [[0, 4, 0]]], dtype=np.int32)
    assert m.loopkv_plan_cells(dmg, 3, 8, 128) == (["reuse", "q4"], 256)
    assert m.loopkv_plan_cells(dmg, 100, 100, 128) == (["reuse", "q2"], 192)
