"""Host-side policy of the serving loop: the decode scheduling order."""

import numpy as np

from paged_kv_cache_451_b200.serving import schedule_order


def test_schedule_orders_are_permutations_with_the_stated_priority():
    rng = np.random.default_rng(3)
    lens = rng.integers(1, 5000, size=300).astype(np.int32)
    for policy in ("long_first", "longest", "batch"):
        o = schedule_order(lens, policy)
        assert o.dtype == np.int32 and sorted(o.tolist()) == list(range(len(lens)))
    assert schedule_order(lens, "batch").tolist() == list(range(len(lens)))
    lo = schedule_order(lens, "longest")
    assert np.all(np.diff(lens[lo]) <= 0)
    lf = schedule_order(lens, "long_first")
    n_long = int(np.sum(lens > lens.mean()))
    assert np.all(np.diff(lens[lf[:n_long]]) <= 0) and np.all(lens[lf[:n_long]] > lens.mean())
    assert np.all(np.diff(lf[n_long:]) > 0)  # the rest keeps batch order
    assert schedule_order(np.zeros(0, np.int32)).size == 0
