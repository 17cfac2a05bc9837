"""GPU parity of the head-parallel sparse MLA shard (dsa_sparse_mla_heads with 64 heads): each half
of the 128 heads, run as its own shard, against the oracle restricted to those heads and against
the 128-head call on the same inputs. One GPU runs both shards in turn; nothing in a shard waits
on the other."""
import numpy as np
import pytest
import torch

import dsa_inputs as DI
from oracle import dsa_oracle as O
from tests import parity as P

pytestmark = pytest.mark.gpu

dsa = pytest.importorskip("sparse_attention_keys_b200")


def _random_idx(rng, B, T, k, q_pos, kv_len):
    idx = np.full((B, T, k), -1, np.int32)
    nv = O.valid_len(q_pos, kv_len)
    for b in range(B):
        for t in range(T):
            m = min(int(nv[b, t]), k)
            if m:
                idx[b, t, :m] = np.sort(rng.choice(int(nv[b, t]), m, replace=False))
    return idx


def _check(got, got_lse, ref, ref_lse):
    assert np.all(np.abs(got - ref) <= P.MLA_ATOL), np.max(np.abs(got - ref))
    fin = np.isfinite(ref_lse)
    assert np.array_equal(fin, np.isfinite(got_lse))
    assert np.all(np.abs(got_lse[fin] - ref_lse[fin]) <= P.LSE_ATOL)


@pytest.mark.parametrize("case", ["ragged", "decode_b8", "multi_query", "decode_b64_sampled"])
def test_64_head_shards_match_the_oracle_and_the_full_call(case):
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    rng = np.random.default_rng(90)
    if case == "ragged":                       # several tiles, a ragged tail, an empty row; no key split
        inp = DI.make_custom(2, 3, 300, 64, decode=False, seed=9)
        q_pos = np.array([[0, 40, 299], [63, 64, 250]], np.int32)
        idx = _random_idx(rng, 2, 3, 64, q_pos, inp.kv_len)
        idx[1, 2, 5:] = -1
        idx[1, 0, :] = -1
    elif case == "multi_query":                # several queries per sequence, split-KV partials
        inp = DI.make_custom(1, 4, 4096, 2048, decode=False, seed=10)
        q_pos = np.array([[4095, 3000, 2047, 700]], np.int32)
        idx = _random_idx(rng, 1, 4, 2048, q_pos, inp.kv_len)
    else:
        inp = DI.make_inputs("decode_b64" if case == "decode_b64_sampled" else "decode_b8")
        q_pos = inp.q_pos
        idx = _random_idx(rng, q_pos.shape[0], 1, inp.workload.topk, q_pos, inp.kv_len)
    B, T = q_pos.shape
    k = idx.shape[-1]
    q_dev = P.bf16_dev(inp.mla_q)
    kv_dev = P.bf16_dev(inp.mla_kv)
    idx_dev = P.to_dev(idx)
    full, full_lse = dsa.dsa_sparse_mla(q_dev, kv_dev, idx_dev)
    shards = []
    for h0 in (0, 64):
        q_shard = q_dev[:, :, h0:h0 + 64].contiguous()
        out, lse = dsa.dsa_sparse_mla_heads(q_shard, kv_dev, idx_dev)
        shards.append((out.float().cpu().numpy(), lse.cpu().numpy()))
    assert dsa.dsa_get_device_status() == 0
    if case in ("decode_b8", "multi_query"):   # these shapes split the keys: the merge path runs
        assert dsa.dsa_sparse_mla_heads_workspace_size(B, T, k, 64) > 0
    full_np, full_lse_np = full.float().cpu().numpy(), full_lse.cpu().numpy()
    rows = [(b, t) for b in range(B) for t in range(T)]
    if case == "decode_b64_sampled":
        rows = [(b, 0) for b in (0, 21, 63)]
    for i, h0 in enumerate((0, 64)):
        out, lse = shards[i]
        hs = slice(h0, h0 + 64)
        # against the 128-head call: each head's result does not depend on the shard it runs in
        _check(out, lse, full_np[:, :, hs], full_lse_np[:, :, hs])
        for b, t in rows:
            sl = (slice(b, b + 1), slice(t, t + 1))
            ref, ref_lse = O.sparse_mla(inp.mla_q[sl][:, :, hs], inp.mla_kv[b:b + 1], idx[sl])
            _check(out[sl], lse[sl], ref, ref_lse)


def test_head_count_is_checked():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    q = torch.zeros((1, 1, 32, 576), dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros((1, 64, 576), dtype=torch.bfloat16, device="cuda")
    idx = torch.zeros((1, 1, 8), dtype=torch.int32, device="cuda")
    with pytest.raises(ValueError):
        dsa.dsa_sparse_mla_heads(q, kv, idx)
    out = torch.empty((1, 1, 32, 512), dtype=torch.bfloat16, device="cuda")
    rc = dsa.lib.dsa_sparse_mla_heads(dsa._ptr(q), dsa._ptr(kv), dsa._ptr(idx), 1, 1, 64, 8, 32, 0.1,
                                      dsa._ptr(out), None, None, 0, dsa._stream(None))
    assert rc == 1                                             # DSA_ERR_INVALID_ARG, nothing launched
