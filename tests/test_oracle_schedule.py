"""Pins of the schedule oracle: hand-worked work lists and the closed-form
total cost.  CPU only."""
import numpy as np

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


def test_total_cost_closed_form():
    rng = np.random.default_rng(0)
    lengths = rng.integers(1, 5000, size=40)
    cu = np.concatenate([[0], np.cumsum(lengths)])
    for causal in (False, True):
        lst = schedule_ref(cu, causal)
        n = -(-lengths // 128)
        want = (n * (n + 1) // 2).sum() if causal else (n * n).sum()
        assert int(lst[:, 3].sum()) == int(want)
        assert (np.diff(lst[:, 3]) <= 0).all()
        # every (doc, query tile) appears once
        assert len(lst) == int((-(-lengths // 128)).sum())


def test_unit_cost_edges():
    assert unit_cost(1, 0, True) == 1
    assert unit_cost(128, 0, True) == 1
    assert unit_cost(129, 0, True) == 1
    assert unit_cost(129, 1, True) == 2
    assert unit_cost(256, 0, False) == 2
    assert unit_cost(257, 2, True) == 3
    assert unit_cost(1000, 3, True) == 4
