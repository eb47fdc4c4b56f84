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


def test_prefill_sizes_take_the_admitted_rows():
    """Admitted sequences are the last rows of the running set; their prompt
    is the context minus the step's appended token, less the cached part."""
    import types
    from paged_kv_cache_451_b200.serving import DecodeLoop
    info = types.SimpleNamespace(num_admitted=2)
    plan = {"info": info, "context_lens": np.array([40, 1601, 70], np.int32), "cached": np.array([1536, 0])}
    a, new, cached = DecodeLoop.prefill_sizes(plan)
    assert a == 2 and list(new) == [64, 69] and list(cached) == [1536, 0]
    info.num_admitted = 0
    assert DecodeLoop.prefill_sizes(plan)[0] == 0


def test_metadata_layout_is_16_byte_aligned_with_prefill_fields():
    from paged_kv_cache_451_b200.serving import DecodeLoop
    lay, total = DecodeLoop._layout(5, 77, 3, 9, 2)
    for name, (off, n) in lay.items():
        assert off % 16 == 0, name
    assert lay["cu"][1] == 3 and lay["pf_lens"][1] == 2
    assert total >= lay["pf_lens"][0] + 8


def test_find_shared_prefix_groups_the_largest_common_leading_run():
    from paged_kv_cache_451_b200.serving import find_shared_prefix
    bs = 16
    tables = np.array([
        [7, 8, 9, 30, -1],   # sharer: prefix 7 8 9
        [1, 2, -1, -1, -1],  # own blocks
        [7, 8, 9, 31, 32],   # sharer
        [7, 8, 9, 33, -1],   # sharer
        [7, 8, 5, -1, -1],   # shares only 7 8
    ], np.int32)
    lens = np.array([60, 20, 70, 49, 40], np.int32)
    rows, blocks = find_shared_prefix(tables, lens, bs, min_sharers=2)
    assert rows.tolist() == [0, 2, 3, 4] and blocks.tolist() == [7, 8]  # the fourth diverges at block 2
    rows, blocks = find_shared_prefix(tables[:4], lens[:4], bs, min_sharers=2)
    assert rows.tolist() == [0, 2, 3] and blocks.tolist() == [7, 8, 9]
    # cut to whole blocks inside every member's context: 33 tokens -> 2 blocks
    lens2 = np.array([60, 20, 70, 33], np.int32)
    rows, blocks = find_shared_prefix(tables[:4], lens2, bs, min_sharers=2)
    assert blocks.tolist() == [7, 8]
    # thresholds
    assert find_shared_prefix(tables[:4], lens[:4], bs, min_sharers=4) == (None, None)
    assert find_shared_prefix(tables[:4], lens[:4], bs, min_sharers=2, min_tokens=64) == (None, None)
    assert find_shared_prefix(tables[[1]], lens[[1]], bs) == (None, None)
