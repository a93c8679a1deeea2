"""CPU checks of the near-tie rule that the GPU selection tests apply (tests/_util.py).

A GPU row may differ from the oracle's selection only when the oracle's k-th
and (k+1)-th scores are within 1e-5 relative of each other, and only in cubes
whose scores lie within that band of the k-th; the tests count such rows and
allow at most 2% of a comparison's rows to be excused.
"""
import numpy as np
import pytest

from tests import _util as U


@pytest.fixture(autouse=True)
def _keep_session_log_clean():
    """These hand rows are checks of the rule itself, not comparisons with a GPU: drop their log lines."""
    n = len(U.NEAR_TIE_LOG)
    yield
    del U.NEAR_TIE_LOG[n:]


def _rows():
    # row 0: a near-tie between cubes 1 and 2 (gap 1e-7, band 5e-6); row 1: a clear gap
    return np.array([[[1.0, 0.5, 0.5 - 1e-7, 0.2],
                      [1.0, 0.5, 0.4, 0.2]]])


def test_identical_selection_is_not_excused():
    s = _rows()
    ora = np.array([[[0, 1], [0, 1]]])
    r = U.near_tie_check(ora.copy(), ora, s, 2, "identical")
    assert r.ok.all() and r.differ == 0 and r.excused == 0 and r.rows == 2


def test_swap_inside_the_band_is_excused_and_counted():
    s = _rows()
    ora = np.array([[[0, 1], [0, 1]]])
    gpu = np.array([[[0, 2], [0, 1]]])
    r = U.near_tie_check(gpu, ora, s, 2, "swap in band")
    assert r.ok.tolist() == [[True, True]]
    assert r.differ == 1 and r.excused == 1
    assert U.NEAR_TIE_LOG[-1] == ("swap in band", 2, 1, 0)


@pytest.mark.parametrize("gpu_row0,gpu_row1", [
    ([0, 3], [0, 1]),        # near-tie row, but cube 3 lies outside the band
    ([0, 1], [0, 2]),        # clear-gap row: any swap fails
    ([1, 2], [0, 1]),        # near-tie row, but cube 0 (far above the band) dropped
])
def test_swap_outside_the_rule_fails(gpu_row0, gpu_row1):
    s = _rows()
    ora = np.array([[[0, 1], [0, 1]]])
    gpu = np.array([[gpu_row0, gpu_row1]])
    r = U.near_tie_check(gpu, ora, s, 2, "bad swap")
    assert not r.ok.all() and r.excused == 0 and r.differ == 1
    with pytest.raises(AssertionError):
        U.assert_selection(gpu, ora, s, 2, "bad swap")


def test_excused_share_is_bounded():
    # 10 rows, each a near-tie swap: the rule accepts every row, the 2% bound does not
    base = np.array([1.0, 0.5, 0.5 - 1e-7, 0.2])
    s = np.tile(base, (10, 1))
    ora = np.tile([0, 1], (10, 1))
    gpu = np.tile([0, 2], (10, 1))
    r = U.near_tie_check(gpu, ora, s, 2, "all near ties")
    assert r.ok.all() and r.excused == 10
    with pytest.raises(AssertionError, match="excused as near-ties"):
        U.assert_selection(gpu, ora, s, 2, "all near ties")
    # one excused row in 50 is within the bound
    s50 = np.tile(np.array([1.0, 0.5, 0.3, 0.2]), (50, 1))
    s50[0] = base
    ora50 = np.tile([0, 1], (50, 1))
    gpu50 = ora50.copy()
    gpu50[0] = [0, 2]
    assert U.assert_selection(gpu50, ora50, s50, 2, "one in fifty").excused == 1
