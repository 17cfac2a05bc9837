"""The synthetic input recipe: seeded, deterministic, and fixed in its draw order (the MLA draws come
after the indexer's, so skipping them changes nothing else). No GPU."""
import numpy as np

import dsa_inputs as DI


def test_same_seed_same_inputs():
    a = DI.make_inputs("tiny_decode", seed=3)
    b = DI.make_inputs("tiny_decode", seed=3)
    for x, y in ((a.idx_q, b.idx_q), (a.idx_k, b.idx_k), (a.idx_w, b.idx_w), (a.mla_q, b.mla_q), (a.mla_kv, b.mla_kv)):
        assert np.array_equal(x, y)
    c = DI.make_inputs("tiny_decode", seed=4)
    assert not np.array_equal(a.idx_q, c.idx_q)


def test_skipping_the_mla_draws_changes_no_other_array():
    a = DI.make_inputs("decode_b8", seed=0, with_mla=True)
    b = DI.make_inputs("decode_b8", seed=0, with_mla=False)
    assert b.mla_q is None and b.mla_kv is None
    for x, y in ((a.idx_q, b.idx_q), (a.idx_k, b.idx_k), (a.idx_w, b.idx_w)):
        assert np.array_equal(x, y)


def test_decode_context_lengths_and_positions():
    inp = DI.make_inputs("decode_b8", seed=0)
    assert np.all((inp.kv_len >= 2048) & (inp.kv_len <= 4096))
    assert np.array_equal(inp.q_pos[:, 0], inp.kv_len - 1)


def test_hot_key_rows_are_scaled():
    wl = DI.Workload("hot", batch=1, queries=4, s_max=1000, topk=16, decode=False, hot_key_frac=0.01, with_mla=False)
    inp = DI.make_inputs(wl, seed=1)
    assert inp.hot_rows is not None and len(inp.hot_rows) == 10
    cold = DI.make_inputs(DI.Workload("cold", batch=1, queries=4, s_max=1000, topk=16, decode=False, with_mla=False),
                          seed=1)
    assert np.allclose(inp.idx_k[0, inp.hot_rows], 8 * cold.idx_k[0, inp.hot_rows])


def test_paged_layout_pages_are_distinct_with_spares():
    table, num_pages = DI.paged_layout(3, 5, 64, seed=2, spare_pages=4)
    assert num_pages == 3 * 5 + 4
    ids = table.ravel()
    assert len(set(ids.tolist())) == ids.size and ids.min() >= 0 and ids.max() < num_pages
