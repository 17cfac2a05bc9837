"""GPU parity of the paged-cache calls: dsa_index_scores_paged and dsa_sparse_mla_paged against the
dense calls (bit-exact: the arithmetic is the same, only the rows' addresses differ) and against the
oracle on the dense view the block table defines. Pool pages that no sequence uses, and the table
entries of pages past a sequence's end, hold NaN codes or bad page ids, so a stray read shows."""
import numpy as np
import pytest
import torch

import dsa_inputs as DI
from oracle import dsa_oracle as O
from tests import parity as P

pytestmark = pytest.mark.gpu

dsa = pytest.importorskip("sparse_attention_keys_b200")

TABLE = O.rope_table(16384)
E4M3_NAN = 0x7F
BF16_NAN = 0x7FC0
DSA_ERR_DEVICE_BOUNDS = 5


@pytest.fixture(scope="module")
def table_dev():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    assert dsa.dsa_device_supported(), "libdsa needs an sm_100 device"
    return torch.from_numpy(TABLE).cuda()


def _status():
    return dsa.dsa_get_device_status()


def _paged_k(k8, ks, kv_len, page_size, seed, past_end):
    B, S = k8.shape[:2]
    table, num_pages = DI.paged_layout(B, S // page_size, page_size, seed, kv_len=kv_len, past_end=past_end)
    k8_pool = DI.to_paged(k8, table, page_size, num_pages, fill=E4M3_NAN)
    ks_pool = DI.to_paged(ks, table, page_size, num_pages, fill=np.float32(np.nan))
    return table, k8_pool, ks_pool


def _scores_both(q8, qs, w, k8, ks, q_pos, kv_len, table, k8_pool, ks_pool, page_size):
    S = k8.shape[1]
    dense = dsa.dsa_index_scores(P.to_dev(q8), P.to_dev(qs), P.to_dev(w), P.to_dev(k8), P.to_dev(ks),
                                 P.to_dev(q_pos), P.to_dev(kv_len), ld=S, flags=dsa.DSA_FILL_MASKED)
    paged = dsa.dsa_index_scores_paged(P.to_dev(q8), P.to_dev(qs), P.to_dev(w), P.to_dev(k8_pool), P.to_dev(ks_pool),
                                       P.to_dev(table), page_size, P.to_dev(q_pos), P.to_dev(kv_len), ld=S,
                                       flags=dsa.DSA_FILL_MASKED)
    return dense.cpu().numpy(), paged.cpu().numpy()


# ---------------------------------------------------------------------------------- index scores
@pytest.mark.parametrize("page_size,past_end,decode", [(64, -1, False), (128, 1_000_000, False),
                                                        (64, 1_000_000, True), (256, -1, True)])
def test_index_scores_paged_matches_dense_and_oracle(table_dev, page_size, past_end, decode):
    max_pages = (700 + page_size - 1) // page_size
    S = max_pages * page_size
    if decode:
        kv_len = [1, 64, 65, 300, S]
        B, T = len(kv_len), 1
        q_pos = np.array(kv_len, np.int32).reshape(B, 1) - 1
    else:
        kv_len = [S, 450, 129]
        B, T = len(kv_len), 70
        q_pos = np.stack([np.arange(T) * (n // T) + (n - 1 - (T - 1) * (n // T)) for n in kv_len]).astype(np.int32)
    inp = DI.make_custom(B, T, S, 64, decode=decode, seed=11, kv_len=kv_len, q_pos=q_pos, with_mla=False)
    q8, qs = O.index_keys(inp.idx_q, inp.q_pos[..., None], TABLE)
    k8, ks = O.index_keys(inp.idx_k, np.arange(S)[None, :], TABLE)
    table, k8_pool, ks_pool = _paged_k(k8, ks, inp.kv_len, page_size, seed=12, past_end=past_end)
    dense, paged = _scores_both(q8, qs, inp.idx_w, k8, ks, inp.q_pos, inp.kv_len, table, k8_pool, ks_pool, page_size)
    assert _status() == 0
    assert np.array_equal(paged, dense, equal_nan=False)
    view = O.paged_gather(k8_pool, table, page_size, inp.kv_len)
    sview = O.paged_gather(ks_pool, table, page_size, inp.kv_len)
    ref = O.index_scores(q8, qs, inp.idx_w, view, sview, inp.q_pos, inp.kv_len)
    mag = O.index_score_magnitude(q8, qs, inp.idx_w, view, sview, inp.q_pos, inp.kv_len)
    nv = O.valid_len(inp.q_pos, inp.kv_len)
    for b in range(B):
        P.check_scores(paged[b], ref[b], mag[b], nv[b])


def test_index_scores_paged_bad_page_sets_status(table_dev):
    P_ = 64
    inp = DI.make_custom(1, 1, 256, 64, decode=True, seed=13, kv_len=[256], with_mla=False)
    q8, qs = DI.filler_e4m3(inp.idx_q.shape, seed=14)
    k8, ks = DI.filler_e4m3(inp.idx_k.shape, seed=15)
    table, k8_pool, ks_pool = _paged_k(k8, ks, inp.kv_len, P_, seed=16, past_end=-1)
    table[0, 2] = -1                            # a visible page with no pool page
    _scores_both(q8, qs, inp.idx_w, k8, ks, inp.q_pos, inp.kv_len, table, k8_pool, ks_pool, P_)
    assert _status() == DSA_ERR_DEVICE_BOUNDS


# ------------------------------------------------------------------------------------ sparse MLA
def _random_idx(rng, B, T, k, q_pos, kv_len):
    idx = np.full((B, T, k), -1, np.int32)
    nv = O.valid_len(q_pos, kv_len)
    for b in range(B):
        for t in range(T):
            m = min(int(nv[b, t]), k)
            idx[b, t, :m] = rng.choice(int(nv[b, t]), m, replace=False) if m else []
    return idx


def _mla_both(q_bits, kv_bits, idx, table, pool, page_size):
    q = P.bf16_dev(q_bits)
    dense, dlse = dsa.dsa_sparse_mla(q, P.bf16_dev(kv_bits), P.to_dev(idx))
    paged, plse = dsa.dsa_sparse_mla_paged(q, P.bf16_dev(pool), P.to_dev(table), page_size, P.to_dev(idx))
    return dense, dlse, paged, plse


@pytest.mark.parametrize("page_size,B,T,S,k", [(64, 2, 3, 320, 128), (128, 2, 3, 640, 96),
                                               (64, 2, 1, 4096, 2048), (256, 3, 1, 2048, 2048)])
def test_sparse_mla_paged_matches_dense_and_oracle(table_dev, page_size, B, T, S, k):
    rng = np.random.default_rng(50 + page_size + S)
    kv_len = [S] + [S // 2 + 17 * b for b in range(1, B)]
    q_pos = np.stack([np.linspace(0, n - 1, T).astype(np.int32) if T > 1 else np.array([n - 1]) for n in kv_len])
    inp = DI.make_custom(B, T, S, k, decode=T == 1, seed=17, kv_len=kv_len, q_pos=q_pos)
    idx = _random_idx(rng, B, T, k, inp.q_pos, inp.kv_len)
    table, num_pages = DI.paged_layout(B, S // page_size, page_size, seed=18, kv_len=inp.kv_len, past_end=-1)
    pool = DI.to_paged(inp.mla_kv, table, page_size, num_pages, fill=BF16_NAN)
    dense, dlse, paged, plse = _mla_both(inp.mla_q, inp.mla_kv, idx, table, pool, page_size)
    assert _status() == 0
    assert torch.equal(paged, dense) and torch.equal(plse, dlse)
    view = O.paged_gather(pool, table, page_size, inp.kv_len)
    ref, ref_lse = O.sparse_mla(inp.mla_q, view, idx)
    got = paged.float().cpu().numpy()
    assert np.all(np.abs(got - ref) <= P.MLA_ATOL), np.max(np.abs(got - ref))
    assert np.all(np.abs(plse.cpu().numpy() - ref_lse) <= P.LSE_ATOL)


def test_sparse_mla_paged_bad_page_sets_status(table_dev):
    page_size, S, k = 64, 256, 64
    inp = DI.make_custom(1, 1, S, k, decode=True, seed=19, kv_len=[S])
    idx = np.arange(k, dtype=np.int32).reshape(1, 1, k) * 4          # touches every page
    table, num_pages = DI.paged_layout(1, S // page_size, page_size, seed=20)
    pool = DI.to_paged(inp.mla_kv, table, page_size, num_pages, fill=BF16_NAN)
    table[0, 1] = num_pages                                           # one past the pool
    _mla_both(inp.mla_q, inp.mla_kv, idx, table, pool, page_size)
    assert _status() == DSA_ERR_DEVICE_BOUNDS


# ------------------------------------------------------------------------------------ whole path
def test_pipeline_paged_equals_dense(table_dev):
    """index_keys writes a paged K-cache through dst_row; paged scores, top-k and paged sparse MLA
    then give bit for bit what the dense path gives on the decode_b8 workload."""
    inp = DI.make_inputs("decode_b8")
    B, S = inp.idx_k.shape[:2]
    k = inp.workload.topk
    page_size = 64
    table, num_pages = DI.paged_layout(B, S // page_size, page_size, seed=21, kv_len=inp.kv_len, past_end=-1)
    q_pos, kv_len = P.to_dev(inp.q_pos), P.to_dev(inp.kv_len)
    # dense K-cache, and the paged one through the block table (only rows below kv_len are written)
    kx = P.to_dev(inp.idx_k.reshape(B * S, 128))
    kpos = P.to_dev(np.tile(np.arange(S, dtype=np.int32), B))
    cache = torch.zeros((B, S, 128), dtype=torch.uint8, device="cuda")
    cscale = torch.zeros((B, S), dtype=torch.float32, device="cuda")
    dsa.dsa_index_keys(kx, kpos, table_dev, out_fp8=cache, out_scale=cscale,
                       dst_row=P.to_dev(np.arange(B * S, dtype=np.int64)))
    rows = np.concatenate([table[b, np.arange(n) // page_size].astype(np.int64) * page_size + np.arange(n) % page_size
                           for b, n in enumerate(inp.kv_len)])
    src = np.concatenate([b * S + np.arange(n) for b, n in enumerate(inp.kv_len)])
    pool8 = torch.full((num_pages * page_size, 128), E4M3_NAN, dtype=torch.uint8, device="cuda")
    pools = torch.full((num_pages * page_size,), float("nan"), dtype=torch.float32, device="cuda")
    dsa.dsa_index_keys(kx[torch.from_numpy(src).cuda()].contiguous(), kpos[torch.from_numpy(src).cuda()].contiguous(),
                       table_dev, out_fp8=pool8, out_scale=pools, dst_row=P.to_dev(rows))
    q8, qs = dsa.dsa_index_keys(P.to_dev(inp.idx_q.reshape(B, 64, 128)), P.to_dev(inp.q_pos.reshape(-1)), table_dev)
    q8, qs = q8.view(B, 1, 64, 128), qs.view(B, 1, 64)
    w = P.to_dev(inp.idx_w)
    sd = dsa.dsa_index_scores(q8, qs, w, cache, cscale, q_pos, kv_len, ld=S)
    sp = dsa.dsa_index_scores_paged(q8, qs, w, pool8, pools, P.to_dev(table), page_size, q_pos, kv_len, ld=S)
    idd = dsa.dsa_topk(sd, q_pos, kv_len, k)
    idp = dsa.dsa_topk(sp, q_pos, kv_len, k)
    kv_pool = DI.to_paged(inp.mla_kv, table, page_size, num_pages, fill=BF16_NAN)
    od, ld_ = dsa.dsa_sparse_mla(P.bf16_dev(inp.mla_q), P.bf16_dev(inp.mla_kv), idd)
    op, lp = dsa.dsa_sparse_mla_paged(P.bf16_dev(inp.mla_q), P.bf16_dev(kv_pool), P.to_dev(table), page_size, idp)
    assert _status() == 0
    assert torch.equal(idp, idd)
    assert torch.equal(op, od) and torch.equal(lp, ld_)
    nv = O.valid_len(inp.q_pos, inp.kv_len)
    a, c = sd.cpu().numpy(), sp.cpu().numpy()
    for b in range(B):
        assert np.array_equal(a[b, 0, :nv[b, 0]], c[b, 0, :nv[b, 0]])
