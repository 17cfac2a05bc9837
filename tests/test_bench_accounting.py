"""The benchmark's work accounting (the numerators of its throughput and roofline figures), checked
against hand counts of the workloads' definitions. No GPU."""
import numpy as np

import bench
import dsa_inputs as DI


def test_decode_pairs_are_the_visible_keys():
    inp = DI.make_inputs("tiny_decode", with_mla=False)          # one query at 1023, context 1024
    u = bench.work_units(inp)
    assert u["pairs"] == 1024 and u["queries"] == 1 and u["selected"] == 256
    assert u["index_scores_flops"] == 1024 * 64 * 128 * 2
    assert u["topk_bytes"] == 1024 * 4 + 256 * 4
    # the measurement unit: 1152 B gathered per (query, selected key); the query's q and output
    # rows and its indices are reported beside it
    assert u["sparse_mla_bytes"] == 256 * 1152
    assert u["sparse_mla_other_bytes"] == 128 * (576 + 512) * 2 + 256 * 4
    assert u["sparse_mla_flops"] == 256 * 128 * (576 + 512) * 2
    # index scores: 132 B of K-cache per (query, key) pair; the scores written and the query
    # codes, scales and weights read are beside it
    assert u["index_scores_bytes"] == 1024 * 132
    assert u["index_scores_other_bytes"] == 1024 * 4 + 64 * (128 + 4 + 4)


def test_decode_b8_pairs_sum_the_context_lengths():
    inp = DI.make_inputs("decode_b8", with_mla=False)
    u = bench.work_units(inp)
    assert u["pairs"] == int(inp.kv_len.sum())
    assert u["selected"] == int(np.minimum(inp.kv_len, 2048).sum()) == 8 * 2048
    assert 8 * 2048 <= u["pairs"] <= 8 * 4096


def test_prefill_pairs_are_the_causal_triangle():
    inp = DI.make_inputs(DI.Workload("p", batch=1, queries=300, s_max=300, topk=64, decode=False, with_mla=False))
    u = bench.work_units(inp)
    assert u["pairs"] == 300 * 301 // 2
    assert u["selected"] == sum(min(t + 1, 64) for t in range(300))


def test_producer_units():
    u = bench.producer_units(8)
    w = 128 * 128 * 512 * 2
    assert u["q_absorb"]["bytes"] == 8 * 128 * (128 + 64 + 576) * 2 + w + 8 * (4 + 256)
    assert u["q_absorb"]["flops"] == 8 * 128 * 128 * 512 * 2
    assert u["out_absorb"]["bytes"] == 8 * 128 * (512 + 128) * 2 + w
    assert u["out_absorb"]["flops"] == u["q_absorb"]["flops"]


def test_prefill_oracle_unit_counts_its_causal_pairs():
    from oracle import dsa_oracle as O
    wl = DI.Workload("p", batch=1, queries=64, s_max=64, topk=16, decode=False, with_mla=True)
    inp = DI.make_inputs(wl)
    table = O.rope_table(128)
    caches = O.index_keys(inp.idx_k, np.arange(64)[None, :], table)
    assert bench.oracle_prefill_rows(inp, 16, table, caches) == sum(t + 1 for t in range(16, 16 + bench.PREFILL_CHUNK))
    units = bench._oracle_units(inp)
    assert units[0] == ("rows", 0) and units[-1] == ("rows", 64 - bench.PREFILL_CHUNK)


def test_decode_b64_units_follow_the_measurement_rules():
    inp = DI.make_inputs(DI.Workload("d", batch=64, queries=1, s_max=64, topk=16, decode=True,
                                     kv_len_range=(64, 64), with_mla=False))
    u = bench.work_units(inp)
    assert u["pairs"] == 64 * 64 and u["selected"] == 64 * 16
    assert u["sparse_mla_bytes"] == 64 * 16 * 1152
    assert u["index_scores_bytes"] == 64 * 64 * 132
