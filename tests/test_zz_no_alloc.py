"""dsa_sparse_mla_noalloc: the sparse-MLA entry point for callers that cannot allocate device
memory (its split-KV scratch is a fixed array inside the library instead of a caller-allocated
workspace). Checked through the C ABI against dsa_sparse_mla on two calls in a row, plus the
rejection of a shape whose scratch would not fit. Kept in its own file so it runs last."""
import numpy as np
import pytest
import torch

import dsa_inputs as DI
from tests import parity as P

pytestmark = pytest.mark.gpu

dsa = pytest.importorskip("sparse_attention_keys_b200")


def _random_idx(rng, kv_len, k):
    B = len(kv_len)
    idx = np.full((B, 1, k), -1, np.int32)
    for b, n in enumerate(kv_len):
        m = min(int(n), k)
        idx[b, 0, :m] = np.sort(rng.choice(int(n), m, replace=False))
    return idx


def _ref_and_noalloc(q, kv, idx):
    ref_out, ref_lse = dsa.dsa_sparse_mla(q, kv, idx)          # caller-allocated workspace
    out = torch.empty_like(ref_out)
    lse = torch.empty_like(ref_lse)
    dsa.dsa_sparse_mla_noalloc(q, kv, idx, out, lse)          # fixed scratch inside the library
    assert dsa.dsa_get_device_status() == 0
    return ref_out.float().cpu().numpy(), ref_lse.cpu().numpy(), out.float().cpu().numpy(), lse.cpu().numpy()


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    inp = DI.make_inputs("decode_b8")
    B = inp.q_pos.shape[0]
    k = inp.workload.topk
    # the shape really uses split-KV scratch, and it fits the fixed array
    need = dsa.dsa_sparse_mla_workspace_size(B, 1, k)
    assert 0 < need <= dsa.dsa_sparse_mla_noalloc_scratch_bytes()
    rng = np.random.default_rng(77)
    kv = P.bf16_dev(inp.mla_kv)
    for call in range(2):                                     # the second call sees the first's scratch
        q_bits = inp.mla_q if call == 0 else DI.bf16_bits_from_f32(rng.standard_normal(inp.mla_q.shape, np.float32))
        idx = _random_idx(rng, inp.kv_len, k)
        if call == 1:
            idx[3, 0, 100:] = -1                              # a ragged row
        ro, rl, no, nl = _ref_and_noalloc(P.bf16_dev(q_bits), kv, P.to_dev(idx))
        assert np.all(np.abs(no - ro) <= P.MLA_ATOL), np.max(np.abs(no - ro))
        assert np.all(np.abs(nl - rl) <= P.LSE_ATOL)


def test_noalloc_matches_on_a_multi_query_shape():
    """Several queries per sequence (T = 4): the split-KV partials are laid out per (query, split),
    so this exercises a scratch layout the one-query decode shapes do not."""
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    B, T, S, k = 1, 4, 4096, 2048
    need = dsa.dsa_sparse_mla_workspace_size(B, T, k)
    assert 0 < need <= dsa.dsa_sparse_mla_noalloc_scratch_bytes()
    rng = np.random.default_rng(78)
    q = P.bf16_dev(DI.bf16_bits_from_f32(rng.standard_normal((B, T, 128, 576), np.float32)))
    kv = P.bf16_dev(DI.bf16_bits_from_f32(rng.standard_normal((B, S, 576), np.float32)))
    idx = np.full((B, T, k), -1, np.int32)
    for t, n in enumerate((S, 3000, 2048, 700)):              # full, partial and short rows
        m = min(n, k)
        idx[0, t, :m] = np.sort(rng.choice(n, m, replace=False))
    for call in range(2):
        ro, rl, no, nl = _ref_and_noalloc(q, kv, P.to_dev(idx))
        assert np.all(np.abs(no - ro) <= P.MLA_ATOL), np.max(np.abs(no - ro))
        assert np.all(np.abs(nl - rl) <= P.LSE_ATOL)
        idx[0, 1, 1500:] = -1                                  # the second call changes a row


def test_noalloc_rejects_shape_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    B, k = 73, 16384                                           # 8+ key splits of 73 queries
    assert dsa.dsa_sparse_mla_workspace_size(B, 1, k) > dsa.dsa_sparse_mla_noalloc_scratch_bytes()
    q = torch.zeros((B, 1, 128, 576), dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros((B, 64, 576), dtype=torch.bfloat16, device="cuda")
    idx = torch.full((B, 1, k), -1, dtype=torch.int32, device="cuda")
    out = torch.empty((B, 1, 128, 512), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(dsa.DsaError) as e:
        dsa.dsa_sparse_mla_noalloc(q, kv, idx, out)
    assert e.value.code == 6                                   # DSA_ERR_WORKSPACE, nothing launched
