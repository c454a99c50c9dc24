"""Pins of the schedule oracle: hand-worked work lists and the closed-form
total cost.  CPU only."""
import numpy as np

from oracle.schedule import schedule_ref, unit_cost


def test_hand_worked_causal():
    # docs: [0,300) L=300, [300,300) empty, [300,700) L=400
    got = schedule_ref([0, 300, 300, 700], causal=True)
    want = [(300, 400, 1, 7), (0, 300, 0, 3), (0, 300, 1, 3), (300, 400, 0, 3)]
    np.testing.assert_array_equal(got, np.array(want, dtype=np.int32))


def test_hand_worked_noncausal():
    got = schedule_ref([0, 300, 300, 700], causal=False)
    want = [(300, 400, 0, 8), (300, 400, 1, 8), (0, 300, 0, 6), (0, 300, 1, 3)]
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
        # every (doc, pair) appears once
        assert len(lst) == int((-(-lengths // 256)).sum())


def test_unit_cost_edges():
    assert unit_cost(1, 0, True) == 1
    assert unit_cost(128, 0, True) == 1
    assert unit_cost(129, 0, True) == 3
    assert unit_cost(256, 0, False) == 4
    assert unit_cost(257, 1, True) == 3
