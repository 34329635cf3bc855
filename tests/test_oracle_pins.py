"""The float64 oracle against its pins (closed forms, brute force, invariants,
hand-derived examples).  CPU only."""
import pytest

import oracle
from _pins import ALL_PINS


@pytest.fixture(scope="module")
def orc():
    return oracle.get()


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__)
def test_pin(orc, pin):
    pin(orc)


def test_threads_match_single_thread(orc):
    """The thread pool only distributes rows: results are identical for 1 and many threads."""
    import numpy as np
    from _pins import rand_decode, run_decode

    rng = np.random.default_rng(5)
    arr = rand_decode(rng, 3, 8, 2, 16, 4, 40, 3)
    a = run_decode(orc, arr, 4, 6, False, n_threads=1)
    b = run_decode(orc, arr, 4, 6, False, n_threads=8)
    assert (a["out"] == b["out"]).all() and (a["sel"] == b["sel"]).all()


def test_row_subset_matches_full(orc):
    import numpy as np
    from _pins import rand_decode, run_decode

    rng = np.random.default_rng(6)
    arr = rand_decode(rng, 2, 4, 2, 8, 3, 10, 2)
    full = run_decode(orc, arr, 3, 3, False)
    rows = [7, 0, 3]
    part = run_decode(orc, arr, 3, 3, False, rows=rows)
    assert (part["out"] == full["out"][rows]).all()


def test_rejects_bad_arguments(orc):
    import numpy as np
    from _pins import rand_decode, run_decode

    rng = np.random.default_rng(7)
    arr = rand_decode(rng, 1, 2, 1, 4, 2, 5, 1)
    arr["n_gists"][0] = 99  # beyond n_max
    with pytest.raises(ValueError):
        run_decode(orc, arr, 2, 2, False)
    arr["n_gists"][0] = 5
    with pytest.raises(ValueError):  # forced selection names a chunk twice
        run_decode(orc, arr, 2, 2, False, sel_in=np.array([[1, 1], [0, 2]]))
