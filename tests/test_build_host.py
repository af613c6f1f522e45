"""Host logic of the offline build driver (CPU only): the starting assignment that turns the
chosen calibration rows into one-member clusters, and its argument checks."""
import numpy as np
import pytest

from memory_bounded_kv_b200.asm_build import _initial_assignment


def test_initial_assignment_places_each_chosen_row_in_its_cluster():
    init = np.array([[4, 0, 2], [1, 3, 5]])
    idx = _initial_assignment(init, 6, "cpu").numpy()
    assert idx.shape == (6, 2) and idx.dtype == np.int32
    for h in range(2):
        for k in range(3):
            assert idx[init[h, k], h] == k
        assert (idx[:, h] >= 0).sum() == 3
    assert idx[1, 0] == -1 and idx[0, 1] == -1


@pytest.mark.parametrize("init", [[[0, 0, 1]], [[0, 1, 6]], [[-1, 1, 2]]])
def test_initial_assignment_rejects_repeated_or_missing_rows(init):
    with pytest.raises(ValueError):
        _initial_assignment(np.array(init), 6, "cpu")
