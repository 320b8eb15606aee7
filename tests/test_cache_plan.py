"""The expert cache's replacement rule (flint_cache_plan, a host-only C function) against a plain Python
model of least-recently-used replacement: every distinct selected expert gets a slot, hits keep theirs,
a miss takes a free slot or else the least recently used slot that the forward does not need; too many
distinct experts leave the state untouched."""

import numpy as np
import pytest

B = pytest.importorskip("bit_routed_expert_sigmoid_b200.binding")


def model_plan(E, S, slot_of, expert_of, last_use, tick, ids):
    uniq = list(dict.fromkeys(int(i) for i in ids))
    if len(uniq) > S or any(not 0 <= e < E for e in uniq):
        return -1, []
    for e in uniq:
        if slot_of[e] >= 0:
            last_use[slot_of[e]] = tick
    loads = []
    for e in uniq:
        if slot_of[e] >= 0:
            continue
        free = [s for s in range(S) if expert_of[s] < 0]
        if free:
            v = free[0]
        else:
            cand = [s for s in range(S) if last_use[s] != tick]
            v = min(cand, key=lambda s: (last_use[s], s))
        if expert_of[v] >= 0:
            slot_of[expert_of[v]] = -1
        expert_of[v], slot_of[e], last_use[v] = e, v, tick
        loads.append((e, v))
    return len(loads), loads


@pytest.mark.parametrize("E,S,P", [(32, 8, 6), (256, 64, 48), (64, 12, 12)])
def test_plan_matches_lru_model(E, S, P):
    rng = np.random.default_rng(E + S)
    st = [np.full(E, -1, np.int32), np.full(S, -1, np.int32), np.zeros(S, np.uint64)]
    ref = [[-1] * E, [-1] * S, [0] * S]
    hot = rng.choice(E, size=max(2, S // 2), replace=False)       # a few experts recur often
    for tick in range(1, 200):
        n_ids = int(rng.integers(1, P + 1))
        pool = np.concatenate([hot, rng.choice(E, size=8, replace=False)])
        ids = rng.choice(pool, size=n_ids).astype(np.int32)
        loads = np.zeros(2 * S, np.int32)
        n = B.flint_cache_plan(E, S, st[0], st[1], st[2], tick, ids, loads)
        n_ref, loads_ref = model_plan(E, S, ref[0], ref[1], ref[2], tick, ids)
        assert n == n_ref, tick
        assert [tuple(loads[2 * i:2 * i + 2]) for i in range(max(n, 0))] == loads_ref
        np.testing.assert_array_equal(st[0], ref[0])
        np.testing.assert_array_equal(st[1], ref[1])
        np.testing.assert_array_equal(st[2], np.array(ref[2], np.uint64))
        # every selected expert now has a slot, and slots and experts agree
        if n >= 0:
            assert all(st[0][e] >= 0 for e in ids)
        for s_ in range(S):
            if st[1][s_] >= 0:
                assert st[0][st[1][s_]] == s_


def test_plan_rejects_more_experts_than_slots_and_bad_ids():
    E, S = 16, 4
    slot_of, expert_of, last_use = np.full(E, -1, np.int32), np.full(S, -1, np.int32), np.zeros(S, np.uint64)
    loads = np.zeros(2 * S, np.int32)
    assert B.flint_cache_plan(E, S, slot_of, expert_of, last_use, 1, np.arange(5, dtype=np.int32), loads) == -1
    assert B.flint_cache_plan(E, S, slot_of, expert_of, last_use, 1, np.array([3, 16], np.int32), loads) == -1
    assert np.all(slot_of == -1) and np.all(expert_of == -1)        # state untouched
    assert B.flint_cache_plan(E, S, slot_of, expert_of, last_use, 1, np.array([3, 3, 7], np.int32), loads) == 2
    assert B.flint_cache_plan(E, S, slot_of, expert_of, last_use, 2, np.array([7, 3], np.int32), loads) == 0
