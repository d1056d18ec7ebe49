"""Host side of the bench's attention probe: the compacted key lists it builds from the
workload's ids are the per-user distinct (item id, time bucket) keys with their token
counts, the same number the roofline charges the attention with."""
import numpy as np

import bench
from workloads import make_stca, make_stca_history


def test_history_generator_draws_what_the_full_workload_draws():
    a = make_stca(3, users=3, L=400, n_items=5000, data_seed=bench.rank_data_seed(3, 0))
    b = make_stca_history(3, users=3, L=400, n_items=5000, data_seed=bench.rank_data_seed(3, 0))
    np.testing.assert_array_equal(a["lengths"], b["lengths"])
    np.testing.assert_array_equal(a["ids"], b["ids"])
    np.testing.assert_array_equal(a["dt"], b["dt"])


def test_compacted_keys_cover_every_token_once():
    h = make_stca_history(3, users=4, L=900, n_items=300, data_seed=11)
    rows, mult, lens, U = bench.compacted_keys(h["ids"], h["dt"], h["lengths"])
    assert lens.sum() == len(rows) == len(mult)
    assert int(lens.sum()) == bench.user_distinct_rows(h["ids"], h["dt"], h["lengths"])
    assert U == bench.distinct_rows(h["ids"], h["dt"])
    keys = bench._row_keys(h["ids"], h["dt"])
    uniq = np.unique(keys)
    off = t0 = 0
    for L, n in zip(h["lengths"], lens):
        r, c = rows[off:off + n], mult[off:off + n]
        assert len(np.unique(r)) == n and c.sum() == L and (c >= 1).all()
        # each row's key is one of the user's keys, counted as often as the user has it
        user_keys = keys[t0:t0 + L]
        for row, cnt in zip(r[:20], c[:20]):
            assert (user_keys == uniq[row]).sum() == cnt
        # first-token order
        firsts = [int(np.flatnonzero(user_keys == uniq[row])[0]) for row in r]
        assert firsts == sorted(firsts)
        off += n
        t0 += L
