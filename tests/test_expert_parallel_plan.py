"""Host logic of expert parallelism (CPU): which requests each rank has
accepted, how many rows go to each rank, and the regrouping of received rows,
checked against a brute-force replay of group-wide token-order acceptance."""
import numpy as np
import pytest

from tests import ep_host_plan as ep


def _brute(counts_all, C):
    """Replay requests in group token order (rank 0's first) per expert."""
    R, E = counts_all.shape
    acc = np.zeros((R, E), np.int64)
    for e in range(E):
        taken = 0
        for s in range(R):
            for _ in range(int(counts_all[s, e])):
                if taken < C:
                    acc[s, e] += 1
                    taken += 1
    return acc


@pytest.mark.parametrize("R,E,C,seed", [(2, 8, 5, 0), (4, 8, 3, 1), (4, 16, 40, 2), (8, 64, 7, 3), (1, 4, 2, 4)])
def test_plan_matches_brute_force(R, E, C, seed):
    rng = np.random.default_rng(seed)
    counts = rng.integers(0, 12, size=(R, E))
    acc = ep.accepted_counts(counts, C)
    np.testing.assert_array_equal(acc, _brute(counts, C))
    rows = ep.send_rows(acc, R)
    El = E // R
    for s in range(R):
        for r in range(R):
            assert rows[s, r] == acc[s, r * El:(r + 1) * El].sum()
    for r in range(R):
        index, offsets = ep.regroup(acc, r, R)
        n = int(rows[:, r].sum())
        assert sorted(index.tolist()) == list(range(n))       # a permutation of the received rows
        assert offsets[-1] == n and len(offsets) == El + 1
        # received rows: source-major, each source's block in owned-expert order
        src = []
        for s in range(R):
            for j in range(El):
                src += [(s, j)] * int(acc[s, r * El + j])
        got = [src[i] for i in index]
        want = [(s, j) for j in range(El) for s in range(R) for _ in range(int(acc[s, r * El + j]))]
        assert got == want


@pytest.mark.parametrize("R,E,C,seed", [(2, 8, 5, 0), (4, 8, 3, 1), (4, 16, 40, 2), (8, 64, 7, 3)])
def test_fused_exchange_positions_are_the_owners_expert_major_order(R, E, C, seed):
    """Where the fused exchange writes each accepted row: source s's i-th row
    for expert e lands at dest_base[e] + i in the owner's buffer, which must be
    exactly that row's place in expert-major order (owned expert, then source,
    then token order), built here by brute force."""
    rng = np.random.default_rng(seed)
    counts = rng.integers(0, 12, size=(R, E))
    acc = _brute(counts, C)
    El = E // R
    for owner in range(R):
        order = [(s, e, i) for e in range(owner * El, (owner + 1) * El) for s in range(R) for i in range(acc[s, e])]
        place = {key: n for n, key in enumerate(order)}
        for s in range(R):
            base = ep.dest_base(acc, s, R)
            for e in range(owner * El, (owner + 1) * El):
                for i in range(acc[s, e]):
                    assert base[e] + i == place[(s, e, i)]
        # the owner's expert offsets are the starts of its experts in that order
        _, offsets = ep.regroup(acc, owner, R)
        for j in range(El):
            e = owner * El + j
            first = [n for n, key in enumerate(order) if key[1] == e]
            assert offsets[j] == (first[0] if first else offsets[j + 1] if j + 1 <= El else offsets[j])
