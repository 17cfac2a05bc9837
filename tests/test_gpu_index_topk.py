"""The fused decode indexer + top-k (dsa_index_topk) against the two calls it replaces,
dsa_index_scores then dsa_topk, on the same device inputs: the selections must be identical
(the fused kernel forms the same fp32 scores and selects with the same tie rule). The cases reach
every cluster size (1 to 8 CTAs per row), rows with at most k visible keys, ragged and causal
rows, heavy exact ties (the third radix digit, resolved by position across the cluster) and the
decode_b64 shape; one small case is also checked against the oracle."""
import numpy as np
import pytest
import torch

import dsa_inputs as DI
from oracle import dsa_oracle as O
from tests import parity as P

pytestmark = pytest.mark.gpu

dsa = pytest.importorskip("sparse_attention_keys_b200")


@pytest.fixture(scope="module")
def gpu():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    assert dsa.dsa_device_supported(), "libdsa needs an sm_100 device"
    return torch.device("cuda")


def _inputs(B, T, S, seed, ties=False):
    rng = np.random.default_rng(seed)
    q8, _ = DI.filler_e4m3((B, T, 64, 128), seed=seed)
    k8, _ = DI.filler_e4m3((B, S, 128), seed=seed + 1)
    qs = rng.uniform(0.5, 2.0, (B, T, 64)).astype(np.float32)
    ks = rng.uniform(0.5, 2.0, (B, S)).astype(np.float32)
    w = rng.standard_normal((B, T, 64)).astype(np.float32)
    if ties:                                         # sixteen distinct keys, repeated: exact ties
        k8[:] = k8[:, np.arange(S) % 16]
        ks[:] = ks[:, np.arange(S) % 16]
    return q8, qs, w, k8, ks


def _both(q8, qs, w, k8, ks, q_pos, kv_len, k):
    d = [P.to_dev(a) for a in (q8, qs, w, k8, ks, q_pos, kv_len)]
    two = dsa.dsa_topk(dsa.dsa_index_scores(*d), d[5], d[6], k).cpu().numpy()
    fused = dsa.dsa_index_topk(*d, k).cpu().numpy()
    assert dsa.dsa_get_device_status() == 0
    return two, fused


@pytest.mark.parametrize("B,kv,k", [
    (5, [1, 127, 128, 129, 1000], 64),               # rows shorter and longer than k, ragged tails
    (5, [1, 127, 128, 129, 1000], 300),
    (5, [1, 127, 128, 129, 1000], 2048),             # every row selects everything: -1 padding
    (1, [1000], 1),
    (40, None, 200),                                 # fewer CTAs per row (larger batch)
    (300, None, 50),                                 # one CTA per row
])
def test_fused_equals_scores_then_topk(gpu, B, kv, k):
    S = 1000
    q8, qs, w, k8, ks = _inputs(B, 1, S, seed=7 + B + k)
    kv_len = np.array(kv if kv is not None else [S - (b * 37) % 400 for b in range(B)], np.int32)
    q_pos = (kv_len - 1).reshape(B, 1).astype(np.int32)
    two, fused = _both(q8, qs, w, k8, ks, q_pos, kv_len, k)
    assert np.array_equal(fused, two)


def test_fused_causal_multi_query(gpu):
    B, T, S, k = 2, 6, 700, 128
    q8, qs, w, k8, ks = _inputs(B, T, S, seed=21)
    q_pos = np.array([[0, 5, 127, 128, 400, 699], [-1, 64, 200, 300, 650, 699]], np.int32)
    kv_len = np.array([700, 680], np.int32)
    two, fused = _both(q8, qs, w, k8, ks, q_pos, kv_len, k)
    assert np.array_equal(fused, two)


@pytest.mark.parametrize("k", [7, 100, 1000])
def test_fused_exact_ties(gpu, k):
    """Every key repeats sixteen times over: the k-th key ties with keys in other CTAs of the
    cluster, which must give up their places by position."""
    B, S = 3, 4000
    q8, qs, w, k8, ks = _inputs(B, 1, S, seed=31 + k, ties=True)
    kv_len = np.array([4000, 3001, 2500], np.int32)
    q_pos = (kv_len - 1).reshape(B, 1)
    two, fused = _both(q8, qs, w, k8, ks, q_pos, kv_len, k)
    assert np.array_equal(fused, two)


@pytest.mark.parametrize("B,S", [(64, 16384), (8, 16384), (2, 32768)])
def test_fused_full_size(gpu, B, S):
    """decode_b64 and decode_b8 shapes (4 and 8 CTAs per row, 32 and 16 key tiles each) and the
    longest row accepted (8 CTAs of 32 tiles)."""
    k = 2048
    q8, qs, w, k8, ks = _inputs(B, 1, S, seed=41 + B)
    kv_len = np.array([S - (b * 131) % 3000 for b in range(B)], np.int32)
    q_pos = (kv_len - 1).reshape(B, 1)
    two, fused = _both(q8, qs, w, k8, ks, q_pos, kv_len, k)
    assert np.array_equal(fused, two)


def test_fused_against_oracle(gpu):
    """Against the oracle's scores and selection: equal except where scores tie within the
    score tolerance (the two sides' fp32 summation orders differ)."""
    B, S, k = 3, 600, 100
    q8, qs, w, k8, ks = _inputs(B, 1, S, seed=51)
    kv_len = np.array([600, 450, 90], np.int32)
    q_pos = (kv_len - 1).reshape(B, 1)
    d = [P.to_dev(a) for a in (q8, qs, w, k8, ks, q_pos, kv_len)]
    fused = dsa.dsa_index_topk(*d, k).cpu().numpy()
    assert dsa.dsa_get_device_status() == 0
    ref = O.index_scores(q8, qs, w, k8, ks, q_pos, kv_len)
    mag = O.index_score_magnitude(q8, qs, w, k8, ks, q_pos, kv_len)
    want = O.topk_indices(ref, q_pos, kv_len, k)
    for b in range(B):
        P.check_topk_near_ties(fused[b], want[b], ref[b], mag[b], k)


def test_fused_rejects_long_rows_and_flags(gpu):
    import ctypes
    S = 40000                                        # above the 32768 keys a row may hold
    q8, qs, w, k8, ks = _inputs(1, 1, S, seed=61)
    d = [P.to_dev(a) for a in (q8, qs, w, k8, ks, np.array([[S - 1]], np.int32), np.array([S], np.int32))]
    with pytest.raises(dsa.DsaError):
        dsa.dsa_index_topk(*d, 8)
    idx = torch.empty((1, 1, 8), dtype=torch.int32, device="cuda")
    args = [ctypes.c_void_p(t.data_ptr()) for t in d]
    rc = dsa.lib.dsa_index_topk(*args, 1, 1, 64, ctypes.c_float(0.1), 8, 1, ctypes.c_void_p(idx.data_ptr()), None)
    assert rc != 0                                   # flags are reserved
