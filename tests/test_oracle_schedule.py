"""Pins of the schedule oracle: hand-worked work lists (one and two query
tiles per unit) and the closed-form total cost.  CPU only."""
import numpy as np
import pytest

from oracle.schedule import schedule_ref, unit_cost


def test_hand_worked_causal():
    # docs: [0,300) L=300, [300,300) empty, [300,700) L=400
    got = schedule_ref([0, 300, 300, 700], causal=True)
    want = [(300, 400, 3, 4), (0, 300, 2, 3), (300, 400, 2, 3), (0, 300, 1, 2),
            (300, 400, 1, 2), (0, 300, 0, 1), (300, 400, 0, 1)]
    np.testing.assert_array_equal(got, np.array(want, dtype=np.int32))


def test_hand_worked_noncausal():
    got = schedule_ref([0, 300, 300, 700], causal=False)
    want = [(300, 400, 0, 4), (300, 400, 1, 4), (300, 400, 2, 4), (300, 400, 3, 4),
            (0, 300, 0, 3), (0, 300, 1, 3), (0, 300, 2, 3)]
    np.testing.assert_array_equal(got, np.array(want, dtype=np.int32))


def test_hand_worked_pairs():
    # two query tiles per unit: L=300 has tiles 0,1 | 2; L=400 has 0,1 | 2,3
    got = schedule_ref([0, 300, 300, 700], causal=True, tiles_per_unit=2)
    want = [(300, 400, 1, 7), (0, 300, 0, 3), (0, 300, 1, 3), (300, 400, 0, 3)]
    np.testing.assert_array_equal(got, np.array(want, dtype=np.int32))
    got = schedule_ref([0, 300, 300, 700], causal=False, tiles_per_unit=2)
    want = [(300, 400, 0, 8), (300, 400, 1, 8), (0, 300, 0, 6), (0, 300, 1, 3)]
    np.testing.assert_array_equal(got, np.array(want, dtype=np.int32))


@pytest.mark.parametrize("tpu", [1, 2])
def test_total_cost_closed_form(tpu):
    rng = np.random.default_rng(0)
    lengths = rng.integers(1, 5000, size=40)
    cu = np.concatenate([[0], np.cumsum(lengths)])
    for causal in (False, True):
        lst = schedule_ref(cu, causal, tpu)
        n = -(-lengths // 128)
        want = (n * (n + 1) // 2).sum() if causal else (n * n).sum()
        assert int(lst[:, 3].sum()) == int(want)
        assert (np.diff(lst[:, 3]) <= 0).all()
        # every (doc, unit) appears once
        assert len(lst) == int((-(-lengths // (128 * tpu))).sum())


def test_unit_cost_edges():
    assert unit_cost(1, 0, True) == 1
    assert unit_cost(128, 0, True) == 1
    assert unit_cost(129, 0, True) == 1
    assert unit_cost(129, 1, True) == 2
    assert unit_cost(256, 0, False) == 2
    assert unit_cost(257, 2, True) == 3
    assert unit_cost(1000, 3, True) == 4
    # pairs
    assert unit_cost(1, 0, True, 2) == 1
    assert unit_cost(129, 0, True, 2) == 3
    assert unit_cost(256, 0, False, 2) == 4
    assert unit_cost(257, 1, True, 2) == 3


@pytest.mark.parametrize("causal", [False, True])
def test_backward_reads_the_list_as_key_tiles(causal):
    """The backward takes each entry (doc_start, doc_len, t, cost) of the
    one-tile list as key tile kb = n_tiles - 1 - t of that document.  Counted
    by brute force over (query tile, key tile) pairs of the mask: the key
    tiles so obtained are each document's key tiles exactly once, and an
    entry's cost is the number of query tiles that see its key tile, so the
    list stays heaviest first for the backward's units."""
    lengths = [1, 300, 0, 128, 129, 1000, 64]
    cu = np.concatenate([[0], np.cumsum(lengths)])
    lst = schedule_ref(cu, causal, 1)
    seen = set()
    for a, L, t, cost in lst:
        n = -(-int(L) // 128)
        kb = n - 1 - int(t)
        assert 0 <= kb < n
        assert (int(a), kb) not in seen
        seen.add((int(a), kb))
        # query tiles qb with some query i >= some key j of tile kb (causal),
        # or any query tile (not causal), inside the document
        sees = sum(1 for qb in range(n)
                   if not causal or min(128 * qb + 127, int(L) - 1) >= 128 * kb)
        assert sees == int(cost)
    assert len(seen) == sum(-(-L // 128) for L in lengths)
