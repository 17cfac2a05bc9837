"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle, element by element on
small shapes that span several tiles and a ragged tail, and on sampled outputs at the full
workload sizes in the launch configuration the benchmark times."""
import numpy as np
import pytest
import torch

import dsa_inputs as DI
from oracle import dsa_oracle as O
from tests import parity as P

pytestmark = pytest.mark.gpu

dsa = pytest.importorskip("sparse_attention_keys_b200")

TABLE = O.rope_table(16384)


@pytest.fixture(scope="module")
def table_dev():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    assert dsa.dsa_device_supported(), "libdsa needs an sm_100 device"
    return torch.from_numpy(TABLE).cuda()


def _status():
    return dsa.dsa_get_device_status()


# ----------------------------------------------------------------------------------- index_keys
@pytest.mark.parametrize("hadamard", [True, False])
def test_index_keys_queries(table_dev, hadamard):
    rng = np.random.default_rng(20)
    x = rng.standard_normal((37, 64, 128)).astype(np.float32)
    x[3] *= 1e-3
    x[5, 7] = 0.0                                      # amax guard block
    pos = rng.integers(0, 16384, 37).astype(np.int32)
    pos[0] = 0
    codes, scales = dsa.dsa_index_keys(P.to_dev(x), P.to_dev(pos), table_dev,
                                       flags=dsa.DSA_HADAMARD if hadamard else 0)
    torch.cuda.synchronize()
    assert _status() == 0
    P.check_codes(codes.cpu().numpy(), scales.cpu().numpy(), x, pos[:, None], TABLE, hadamard)


def test_index_keys_bf16_input(table_dev):
    """bf16 rows: the kernel widens them exactly, so the oracle runs on the widened fp32 values."""
    rng = np.random.default_rng(21)
    xf = rng.standard_normal((29, 64, 128)).astype(np.float32) * 3.0
    bits = DI.bf16_bits_from_f32(xf)
    x_wide = (bits.astype(np.uint32) << 16).view(np.float32)
    pos = rng.integers(0, 16384, 29).astype(np.int32)
    xb = torch.from_numpy(bits).cuda().view(torch.bfloat16)
    codes, scales = dsa.dsa_index_keys(xb, P.to_dev(pos), table_dev)
    torch.cuda.synchronize()
    assert _status() == 0
    P.check_codes(codes.cpu().numpy(), scales.cpu().numpy(), x_wide, pos[:, None], TABLE, True)


def test_index_keys_cache_write(table_dev):
    """Keys scattered into a [B, S_max, 128] cache through dst_row; untouched rows keep their bytes."""
    B, S = 2, 300
    rng = np.random.default_rng(21)
    x = rng.standard_normal((450, 128)).astype(np.float32)
    x[::37] *= 8.0                                      # hot rows stress the block scales
    b = rng.integers(0, B, 450)
    pos = rng.permutation(B * S)[:450]
    sel_b, sel_p = pos // S, (pos % S).astype(np.int32)
    dst = (sel_b * S + sel_p).astype(np.int64)
    cache = torch.full((B, S, 128), 0xAB, dtype=torch.uint8, device="cuda")
    cscale = torch.full((B, S), -1.0, dtype=torch.float32, device="cuda")
    dsa.dsa_index_keys(P.to_dev(x), P.to_dev(sel_p), table_dev, out_fp8=cache, out_scale=cscale,
                       dst_row=P.to_dev(dst))
    torch.cuda.synchronize()
    assert _status() == 0
    c = cache.cpu().numpy().reshape(B * S, 128)
    s = cscale.cpu().numpy().reshape(B * S)
    P.check_codes(c[dst], s[dst], x, sel_p, TABLE, True)
    untouched = np.setdiff1d(np.arange(B * S), dst)
    assert np.all(c[untouched] == 0xAB) and np.all(s[untouched] == -1.0)


def test_index_keys_full_prefill_16384_launch(table_dev):
    """The benchmark's 16384-token prefill launches: all 16384 keys (1% of them scaled x8 before
    RoPE and quantisation) written into the K-cache, and all 16384 x 64 query blocks. Every key row
    is checked; query blocks on sampled rows: the first, the hot-key positions, the middle and the
    last positions up to 16383."""
    inp = DI.make_inputs("prefill_16384")
    S = inp.idx_k.shape[1]
    cache = torch.zeros((1, S, 128), dtype=torch.uint8, device="cuda")
    cscale = torch.zeros((1, S), dtype=torch.float32, device="cuda")
    dsa.dsa_index_keys(P.to_dev(inp.idx_k.reshape(S, 128)), P.to_dev(np.arange(S, dtype=np.int32)), table_dev,
                       out_fp8=cache, out_scale=cscale, dst_row=P.to_dev(np.arange(S, dtype=np.int64)))
    q8, qs = dsa.dsa_index_keys(P.to_dev(inp.idx_q.reshape(S, 64, 128)), P.to_dev(inp.q_pos.reshape(-1)), table_dev)
    assert _status() == 0
    hot = inp.hot_rows
    assert hot is not None and len(hot) == 164
    g_cache, g_scale = cache.cpu().numpy()[0], cscale.cpu().numpy()[0]
    P.check_codes(g_cache, g_scale, inp.idx_k[0], np.arange(S), TABLE)
    # the hot rows' scales are ~8x the others' (amax grows with the row)
    cold = np.setdiff1d(np.arange(S), hot)
    assert np.median(g_scale[hot]) > 6 * np.median(g_scale[cold])
    rows = sorted(set([0, 1, 127, 128, 8191, 16381, 16382, 16383] + [int(r) for r in hot[:4]]))
    g_q8, g_qs = q8.cpu().numpy(), qs.cpu().numpy()
    P.check_codes(g_q8[rows], g_qs[rows], inp.idx_q[0, rows], np.array(rows)[:, None], TABLE)


def test_index_keys_position_out_of_range_sets_status(table_dev):
    x = torch.zeros((4, 128), dtype=torch.float32, device="cuda")
    pos = torch.tensor([0, 1, 20000, 3], dtype=torch.int32, device="cuda")
    small = table_dev[:16384]
    dsa.dsa_index_keys(x, pos, small)
    assert _status() == 5          # DSA_ERR_DEVICE_BOUNDS


def _qk_inputs(k_rows, q_rows, dtype, seed):
    rng = np.random.default_rng(seed)
    kx = rng.standard_normal((k_rows, 128)).astype(np.float32) * 2.0
    qx = rng.standard_normal((q_rows, 64, 128)).astype(np.float32)
    k_pos = rng.integers(0, 16384, k_rows).astype(np.int32)
    q_pos = rng.integers(0, 16384, q_rows).astype(np.int32)
    if dtype == "bf16":
        to = lambda a: torch.from_numpy(DI.bf16_bits_from_f32(a)).cuda().view(torch.bfloat16)
    else:
        to = P.to_dev
    return to(kx), to(qx), P.to_dev(k_pos), P.to_dev(q_pos)


@pytest.mark.parametrize("k_rows,q_rows,dtype", [
    (8, 8, "f32"),          # a decode step of 8 sequences: one key CTA, 64 query CTAs
    (13, 7, "bf16"),        # ragged: the key CTAs' last one partly empty, the query range 448 blocks
    (0, 5, "f32"),          # no new keys
    (9, 0, "f32"),          # no queries
    (2048, 64, "f32"),      # many key CTAs ahead of the queries
])
@pytest.mark.parametrize("scatter", [True, False])
def test_index_qk_equals_two_index_keys_calls(table_dev, k_rows, q_rows, dtype, scatter):
    """dsa_index_qk against dsa_index_keys on the keys then on the queries: bit for bit, including
    the bytes of the cache rows it must not touch."""
    kx, qx, k_pos, q_pos = _qk_inputs(k_rows, q_rows, dtype, seed=100 + k_rows + q_rows)
    B, S = 3, 1000
    dst = (torch.randperm(B * S, device="cuda")[:k_rows].to(torch.int64).contiguous() if scatter else None)
    shape_k = (B, S, 128) if scatter else (max(k_rows, 1), 128)
    shape_ks = (B, S) if scatter else (max(k_rows, 1),)
    want_c = torch.full(shape_k, 0xAB, dtype=torch.uint8, device="cuda")
    want_s = torch.full(shape_ks, -1.0, dtype=torch.float32, device="cuda")
    got_c, got_s = want_c.clone(), want_s.clone()
    if k_rows:
        dsa.dsa_index_keys(kx, k_pos, table_dev, out_fp8=want_c, out_scale=want_s, dst_row=dst)
    want_q8, want_qs = (dsa.dsa_index_keys(qx, q_pos, table_dev) if q_rows else
                        (torch.empty((0, 64, 128), dtype=torch.uint8, device="cuda"),
                         torch.empty((0, 64), dtype=torch.float32, device="cuda")))
    got_q8, got_qs = dsa.dsa_index_qk(kx, k_pos, qx, q_pos, table_dev, got_c, got_s, k_dst_row=dst)
    torch.cuda.synchronize()
    assert _status() == 0
    assert torch.equal(got_c, want_c) and torch.equal(got_s, want_s)
    assert torch.equal(got_q8, want_q8) and torch.equal(got_qs, want_qs)


def test_index_qk_against_the_oracle(table_dev):
    """One decode-shaped call against the oracle's codes for both sides."""
    rng = np.random.default_rng(7)
    kx = rng.standard_normal((6, 128)).astype(np.float32)
    qx = rng.standard_normal((6, 64, 128)).astype(np.float32)
    pos = rng.integers(0, 16384, 6).astype(np.int32)
    k8 = torch.empty((6, 128), dtype=torch.uint8, device="cuda")
    ks = torch.empty((6,), dtype=torch.float32, device="cuda")
    q8, qs = dsa.dsa_index_qk(P.to_dev(kx), P.to_dev(pos), P.to_dev(qx), P.to_dev(pos), table_dev, k8, ks)
    torch.cuda.synchronize()
    assert _status() == 0
    P.check_codes(k8.cpu().numpy(), ks.cpu().numpy(), kx, pos, TABLE)
    P.check_codes(q8.cpu().numpy(), qs.cpu().numpy(), qx, pos[:, None], TABLE)


def test_index_qk_key_position_out_of_range_sets_status(table_dev):
    kx = torch.zeros((3, 128), dtype=torch.float32, device="cuda")
    qx = torch.zeros((2, 64, 128), dtype=torch.float32, device="cuda")
    k_pos = torch.tensor([0, 20000, 2], dtype=torch.int32, device="cuda")
    q_pos = torch.tensor([4, 5], dtype=torch.int32, device="cuda")
    k8 = torch.empty((3, 128), dtype=torch.uint8, device="cuda")
    ks = torch.empty((3,), dtype=torch.float32, device="cuda")
    dsa.dsa_index_qk(kx, k_pos, qx, q_pos, table_dev, k8, ks)
    assert _status() == 5          # DSA_ERR_DEVICE_BOUNDS


# ----------------------------------------------------------------------------------- scores
def _quantised(inp, q_rows=None, k_seqs=None):
    """Oracle-quantised q/k for a workload (the same bytes are fed to the GPU). With q_rows
    [(b, t)] / k_seqs [b], only those rows come from the oracle and the rest are seeded filler
    codes (the oracle's plain encoder is too slow for every row of the largest workloads)."""
    B, T = inp.q_pos.shape
    S = inp.idx_k.shape[1]
    if q_rows is None:
        q8, qs = O.index_keys(inp.idx_q, inp.q_pos[..., None], TABLE)
    else:
        q8, qs = DI.filler_e4m3(inp.idx_q.shape, seed=101)
        for b, t in q_rows:
            q8[b, t], qs[b, t] = O.index_keys(inp.idx_q[b, t], inp.q_pos[b, t], TABLE)
    if k_seqs is None:
        k8, ks = O.index_keys(inp.idx_k, np.arange(S)[None, :], TABLE)
    else:
        k8, ks = DI.filler_e4m3(inp.idx_k.shape, seed=102)
        for b in k_seqs:
            k8[b], ks[b] = O.index_keys(inp.idx_k[b], np.arange(S), TABLE)
    return q8, qs, k8, ks


def _gpu_scores(q8, qs, w, k8, ks, q_pos, kv_len, flags=0, ld=None):
    return dsa.dsa_index_scores(P.to_dev(q8), P.to_dev(qs), P.to_dev(w), P.to_dev(k8), P.to_dev(ks),
                                P.to_dev(q_pos), P.to_dev(kv_len), flags=flags, ld=ld)


@pytest.mark.parametrize("case", ["prefill_ragged", "decode_ragged", "tiny"])
def test_index_scores_small(table_dev, case):
    if case == "prefill_ragged":
        inp = DI.make_custom(2, 133, 300, 64, decode=False, seed=3, kv_len=[300, 250], with_mla=False)
        inp.q_pos = np.stack([np.arange(133), np.minimum(np.arange(133) + 150, 299)]).astype(np.int32)
    elif case == "decode_ragged":
        inp = DI.make_custom(5, 1, 1000, 64, decode=True, seed=4, kv_len=[1, 127, 128, 129, 1000], with_mla=False)
    else:
        inp = DI.make_inputs("tiny_decode", with_mla=False)
    q8, qs, k8, ks = _quantised(inp)
    got = _gpu_scores(q8, qs, inp.idx_w, k8, ks, inp.q_pos, inp.kv_len).cpu().numpy()
    assert _status() == 0
    ref = O.index_scores(q8, qs, inp.idx_w, k8, ks, inp.q_pos, inp.kv_len)
    mag = O.index_score_magnitude(q8, qs, inp.idx_w, k8, ks, inp.q_pos, inp.kv_len)
    nv = O.valid_len(inp.q_pos, inp.kv_len)
    for b in range(inp.idx_q.shape[0]):
        P.check_scores(got[b], ref[b], mag[b], nv[b])


def test_index_scores_fill_masked(table_dev):
    inp = DI.make_custom(1, 9, 260, 8, decode=False, seed=5, with_mla=False)
    inp.q_pos = np.array([[0, 1, 5, 127, 128, 129, 200, 258, 259]], np.int32)
    q8, qs, k8, ks = _quantised(inp)
    ld = 264
    out = torch.full((1, 9, ld), 7.0, dtype=torch.float32, device="cuda")
    dsa.dsa_index_scores(P.to_dev(q8), P.to_dev(qs), P.to_dev(inp.idx_w), P.to_dev(k8), P.to_dev(ks),
                         P.to_dev(inp.q_pos), P.to_dev(inp.kv_len), scores=out, ld=ld, flags=dsa.DSA_FILL_MASKED)
    got = out.cpu().numpy()[0]
    for t, p in enumerate(inp.q_pos[0]):
        assert np.all(np.isneginf(got[t, p + 1:260]))
        assert np.all(np.isfinite(got[t, :p + 1]))
        assert np.all(got[t, 260:] == 7.0)                # padding past S_max untouched


@pytest.mark.parametrize("name", ["decode_b8", "prefill_4096", "prefill_16384", "decode_b64"])
def test_index_scores_full_size_sampled(table_dev, name):
    inp = DI.make_inputs(name, with_mla=False)
    B, T = inp.idx_q.shape[:2]
    if name == "decode_b8":
        rows = [(b, 0) for b in range(B)]
    elif name == "decode_b64":
        rows = [(b, 0) for b in (0, 17, 40, 63)]
    else:
        cand = [0, 1, 2, 3, 127, 128, 129, 2047, 2048, 2049, T // 2 + 3, T - 2, T - 1]
        if inp.hot_rows is not None:
            cand += [int(r) for r in inp.hot_rows[:3]]
        rows = [(0, t) for t in sorted(set(cand)) if t < T]
    q8, qs, k8, ks = _quantised(inp, q_rows=rows, k_seqs=sorted(set(b for b, _ in rows)))
    got_t = _gpu_scores(q8, qs, inp.idx_w, k8, ks, inp.q_pos, inp.kv_len)
    assert _status() == 0
    for (b, t) in rows:
        got = got_t[b, t].cpu().numpy()
        q_sl = (slice(b, b + 1), slice(t, t + 1))
        ref = O.index_scores(q8[q_sl], qs[q_sl], inp.idx_w[q_sl], k8[b:b + 1], ks[b:b + 1], inp.q_pos[q_sl],
                             inp.kv_len[b:b + 1])
        mag = O.index_score_magnitude(q8[q_sl], qs[q_sl], inp.idx_w[q_sl], k8[b:b + 1], ks[b:b + 1],
                                      inp.q_pos[q_sl], inp.kv_len[b:b + 1])
        nv = O.valid_len(inp.q_pos[q_sl], inp.kv_len[b:b + 1])
        P.check_scores(got[None], ref[0], mag[0], nv[0])


# ----------------------------------------------------------------------------------- top-k
def _gpu_topk(scores, q_pos, kv_len, k):
    return dsa.dsa_topk(P.to_dev(scores), P.to_dev(q_pos), P.to_dev(kv_len), k).cpu().numpy()


@pytest.mark.parametrize("k", [1, 7, 64, 300, 2048])
def test_topk_exact_on_synthetic_scores(table_dev, k):
    rng = np.random.default_rng(30 + k)
    B, T, S = 3, 5, 3000
    sc = rng.standard_normal((B, T, S)).astype(np.float32)
    sc[0] = np.round(sc[0] * 4) / 4                     # heavy ties
    sc[1, 0, :100] = 0.0
    sc[1, 0, 100:200] = -0.0                            # signed zeros compare equal
    sc[1, 1, ::3] = -np.inf
    sc[2, 2] = 1.0                                      # a fully tied row
    q_pos = np.array([[2999, 10, 1999, 2047, 2048], [2999, 2999, 500, 0, 64], [2999, 2999, 2999, 299, 7]], np.int32)
    kv_len = np.array([3000, 3000, 2500], np.int32)
    got = _gpu_topk(sc, q_pos, kv_len, k)
    assert _status() == 0
    want = O.topk_indices(sc.astype(np.float64), q_pos, kv_len, k)
    assert np.array_equal(got, want)


@pytest.mark.parametrize("k", [1, 7, 300, 2048, 4096])
def test_topk_sorted_on_synthetic_scores(table_dev, k):
    """DSA_SORTED: the selection in descending-score order (ties by position), exactly the oracle's
    stable sort, including rows with fewer visible keys than k."""
    rng = np.random.default_rng(40 + k)
    B, T, S = 2, 4, 5000
    sc = rng.standard_normal((B, T, S)).astype(np.float32)
    sc[0] = np.round(sc[0] * 4) / 4                     # heavy ties
    sc[1, 0, :100] = 0.0
    sc[1, 0, 100:200] = -0.0
    q_pos = np.array([[4999, 10, 1999, 4095], [4999, 0, 2047, 3000]], np.int32)
    kv_len = np.array([5000, 4500], np.int32)
    got = dsa.dsa_topk(P.to_dev(sc), P.to_dev(q_pos), P.to_dev(kv_len), k, flags=dsa.DSA_SORTED).cpu().numpy()
    assert _status() == 0
    want = O.topk_indices(sc.astype(np.float64), q_pos, kv_len, k, sorted_by_score=True)
    assert np.array_equal(got, want)


@pytest.mark.parametrize("in_band", [1024, 1025, 2500])
def test_topk_first_digit_crowded(table_dev, in_band):
    """Rows whose k-th largest score sits in a band of `in_band` keys sharing the top 12 key bits
    ([1.0, 1.125): sign, exponent and 3 mantissa bits). Rows of 4096 hold up to 1024 such candidate
    positions for the last two radix digits; past that the kernel runs those digits over every key.
    Both paths must give the oracle's selection, in both output orders."""
    rng = np.random.default_rng(50 + in_band)
    S, k = 4096, 2048
    above = 1500                                         # larger than the band: always selected
    rows = []
    for _ in range(3):
        v = np.empty(S, np.float32)
        v[:above] = rng.uniform(2.0, 3.0, above)
        v[above:above + in_band] = 1.0 + rng.uniform(0.0, 0.124, in_band)
        v[above + in_band:] = rng.uniform(-3.0, 0.9, S - above - in_band)
        v[above + 5:above + 40] = v[above + 5]           # ties inside the band
        rows.append(rng.permutation(v))
    sc = np.stack(rows)[None]                            # [1, 3, S]
    q_pos = np.full((1, 3), S - 1, np.int32)
    kv_len = np.array([S], np.int32)
    got = _gpu_topk(sc, q_pos, kv_len, k)
    gs = dsa.dsa_topk(P.to_dev(sc), P.to_dev(q_pos), P.to_dev(kv_len), k, flags=dsa.DSA_SORTED).cpu().numpy()
    assert _status() == 0
    assert np.array_equal(got, O.topk_indices(sc.astype(np.float64), q_pos, kv_len, k))
    assert np.array_equal(gs, O.topk_indices(sc.astype(np.float64), q_pos, kv_len, k, sorted_by_score=True))


def test_topk_longest_row_and_overlong_row(table_dev):
    rng = np.random.default_rng(31)
    S = 32768
    sc = rng.standard_normal((1, 2, S)).astype(np.float32)
    q_pos = np.array([[S - 1, S - 1]], np.int32)
    got = _gpu_topk(sc, q_pos, np.array([S], np.int32), 2048)
    assert _status() == 0
    assert np.array_equal(got, O.topk_indices(sc.astype(np.float64), q_pos, [S], 2048))
    sc2 = rng.standard_normal((1, 1, S + 4)).astype(np.float32)
    dsa.dsa_topk(P.to_dev(sc2), P.to_dev(np.array([[S + 3]], np.int32)), P.to_dev(np.array([S + 4], np.int32)), 16)
    assert _status() == 5


@pytest.mark.parametrize("name", ["prefill_4096", "prefill_16384", "decode_b64"])
def test_topk_full_size_on_oracle_scores(table_dev, name):
    """Full launch on fp32 scores made by the oracle; sampled rows checked bit-exact. The 16384-token
    prefill rows are up to 16384 wide and include the rows of the x8 hot keys."""
    inp = DI.make_inputs(name, with_mla=False)
    B, T = inp.idx_q.shape[:2]
    if name.startswith("prefill"):
        cand = [0, 5, 2046, 2047, 2048, 3000, T // 2 + 1, T - 2, T - 1]
        if inp.hot_rows is not None:
            cand += [int(r) for r in inp.hot_rows[-2:]]
        rows = [(0, t) for t in sorted(set(cand)) if t < T]
    else:
        rows = [(b, 0) for b in (0, 31, 63)]
    q8, qs, k8, ks = _quantised(inp, q_rows=rows, k_seqs=sorted(set(b for b, _ in rows)))
    ld = inp.idx_k.shape[1]
    gen = torch.Generator(device="cuda").manual_seed(1)
    sc_dev = torch.randn((B, T, ld), generator=gen, device="cuda", dtype=torch.float32)   # background rows
    sc = {}
    for b, t in rows:
        sl = (slice(b, b + 1), slice(t, t + 1))
        r = O.index_scores(q8[sl], qs[sl], inp.idx_w[sl], k8[b:b + 1], ks[b:b + 1], inp.q_pos[sl], inp.kv_len[b:b + 1])
        sc[b, t] = r[0, 0].astype(np.float32)
        sc_dev[b, t] = torch.from_numpy(sc[b, t]).cuda()
    got = dsa.dsa_topk(sc_dev, P.to_dev(inp.q_pos), P.to_dev(inp.kv_len), inp.workload.topk).cpu().numpy()
    assert _status() == 0
    for b, t in rows:
        want = O.topk_indices(sc[b, t][None, None].astype(np.float64), inp.q_pos[b:b + 1, t:t + 1],
                              inp.kv_len[b:b + 1], inp.workload.topk)
        assert np.array_equal(got[b, t], want[0, 0]), (b, t)


# ----------------------------------------------------------------------------------- sparse MLA
def _gpu_mla(q_bits, kv_bits, idx):
    out, lse = dsa.dsa_sparse_mla(P.bf16_dev(q_bits), P.bf16_dev(kv_bits), P.to_dev(idx))
    return out.float().cpu().numpy(), lse.cpu().numpy()


def _check_mla(got, got_lse, q_bits, kv_bits, idx, rows=None):
    ref, ref_lse = O.sparse_mla(q_bits, kv_bits, idx)
    if rows is not None:
        got, got_lse = got[rows], got_lse[rows]
    assert np.all(np.abs(got - ref) <= P.MLA_ATOL), np.max(np.abs(got - ref))
    fin = np.isfinite(ref_lse)
    assert np.array_equal(fin, np.isfinite(got_lse))
    assert np.all(np.abs(got_lse[fin] - ref_lse[fin]) <= P.LSE_ATOL)


def _random_idx(rng, B, T, k, q_pos, kv_len):
    idx = np.full((B, T, k), -1, np.int32)
    nv = O.valid_len(q_pos, kv_len)
    for b in range(B):
        for t in range(T):
            n = int(nv[b, t])
            m = min(n, k)
            idx[b, t, :m] = np.sort(rng.choice(n, m, replace=False)) if m else []
    return idx


def test_sparse_mla_small_ragged(table_dev):
    rng = np.random.default_rng(40)
    B, T, S, k = 2, 3, 300, 64
    inp = DI.make_custom(B, T, S, k, decode=False, seed=6)
    q_pos = np.array([[0, 40, 299], [63, 64, 250]], np.int32)
    idx = _random_idx(rng, B, T, k, q_pos, inp.kv_len)
    idx[1, 2, 5:] = -1                       # a ragged row
    idx[1, 0, :] = -1                        # an empty row
    idx[0, 1] = rng.permutation(idx[0, 1])   # order must not matter
    got, lse = _gpu_mla(inp.mla_q, inp.mla_kv, idx)
    assert _status() == 0
    _check_mla(got, lse, inp.mla_q, inp.mla_kv, idx)
    assert np.all(got[1, 0] == 0) and np.all(np.isneginf(lse[1, 0]))


def test_sparse_mla_q_ready_flag(table_dev):
    """DSA_Q_READY only moves when the kernel loads q (before it waits for the preceding kernel):
    the outputs are bitwise those of the plain call, on a split-KV shape and a single-split one,
    with the indices written by a kernel right before. Other flag bits are rejected."""
    rng = np.random.default_rng(41)
    for B, T, S, k in ((2, 3, 300, 64), (4, 1, 3000, 2048)):
        inp = DI.make_custom(B, T, S, k, decode=(T == 1), seed=8 + B)
        q_pos = np.minimum(np.tile(np.arange(T, dtype=np.int32) * 37 + S - T * 37, (B, 1)), S - 1)
        idx = _random_idx(rng, B, T, k, q_pos, inp.kv_len)
        q, kv = P.bf16_dev(inp.mla_q), P.bf16_dev(inp.mla_kv)
        idx_src = P.to_dev(idx)
        idx_dev = torch.empty_like(idx_src)
        idx_dev.copy_(idx_src)                            # a kernel on the stream writes the indices
        o0, l0 = dsa.dsa_sparse_mla(q, kv, idx_dev)
        idx_dev.zero_()
        idx_dev.copy_(idx_src)
        o1, l1 = dsa.dsa_sparse_mla(q, kv, idx_dev, flags=dsa.DSA_Q_READY)
        assert _status() == 0
        assert torch.equal(o0, o1) and torch.equal(l0, l1)
    with pytest.raises(dsa.DsaError):
        dsa.dsa_sparse_mla(q, kv, idx_dev, flags=0x10)


def test_sparse_mla_full_context_equals_dense(table_dev):
    inp = DI.make_custom(1, 4, 200, 256, decode=False, seed=7)
    q_pos = np.array([[10, 99, 150, 199]], np.int32)
    idx = _random_idx(np.random.default_rng(41), 1, 4, 256, q_pos, inp.kv_len)
    got, lse = _gpu_mla(inp.mla_q, inp.mla_kv, idx)
    dense, dlse = O.dense_mla(inp.mla_q, inp.mla_kv, q_pos, inp.kv_len)
    assert np.all(np.abs(got - dense) <= P.MLA_ATOL)
    assert np.all(np.abs(lse - dlse) <= P.LSE_ATOL)


def test_sparse_mla_bad_index_sets_status(table_dev):
    inp = DI.make_custom(1, 1, 64, 32, decode=True, seed=8)
    idx = np.arange(32, dtype=np.int32).reshape(1, 1, 32)
    idx[0, 0, 3] = 64                        # == S_max: out of range
    _gpu_mla(inp.mla_q, inp.mla_kv, idx)
    assert _status() == 5


@pytest.mark.parametrize("name", ["decode_b8", "prefill_4096", "decode_b64"])
def test_sparse_mla_full_size_sampled(table_dev, name):
    inp = DI.make_inputs(name)
    rng = np.random.default_rng(42)
    B, T = inp.q_pos.shape
    idx = _random_idx(rng, B, T, inp.workload.topk, inp.q_pos, inp.kv_len)
    got, lse = _gpu_mla(inp.mla_q, inp.mla_kv, idx)
    assert _status() == 0
    if name == "decode_b8":
        _check_mla(got, lse, inp.mla_q, inp.mla_kv, idx)
        return
    rows = [(0, t) for t in (0, 1, 2047, 2048, T - 1)] if T > 1 else [(b, 0) for b in (0, 21, 63)]
    for b, t in rows:
        sl = (slice(b, b + 1), slice(t, t + 1))
        _check_mla(got[sl], lse[sl], inp.mla_q[sl], inp.mla_kv[b:b + 1], idx[sl])


# ----------------------------------------------------------------------------------- whole path
E2E_ROWS = {
    "prefill_4096": [(0, t) for t in (0, 1, 127, 2047, 2048, 2049, 3001, 4095)],
    "decode_b64": [(b, 0) for b in (0, 17, 40, 63)],
}


@pytest.mark.parametrize("name", ["tiny_decode", "decode_b8", "prefill_4096", "decode_b64"])
def test_pipeline_end_to_end(table_dev, name):
    """index_keys (cache + queries) -> scores -> top-k -> sparse MLA, all through the C ABI in the
    order and launch configuration the benchmark's step uses, at the workload's full size.

    Checked link by link against the oracle, on every row of the small workloads and on sampled
    rows of the large ones: the GPU's codes and scales against the oracle's quantiser; the GPU's
    scores against the oracle's scores on those same codes (identical quantised inputs); the
    selection against the GPU's own score buffer (bit-exact, both output orders) and against the
    oracle's selection on the oracle's scores (equal except at near-ties); the attention output of
    the GPU's selection against the oracle's."""
    inp = DI.make_inputs(name)
    B, S = inp.idx_k.shape[:2]
    T = inp.q_pos.shape[1]
    k = inp.workload.topk
    rows = E2E_ROWS.get(name, [(b, t) for b in range(B) for t in range(T)])
    seqs = sorted(set(b for b, _ in rows))
    cache = torch.zeros((B, S, 128), dtype=torch.uint8, device="cuda")
    cscale = torch.zeros((B, S), dtype=torch.float32, device="cuda")
    kx = P.to_dev(inp.idx_k.reshape(B * S, 128))
    kpos = P.to_dev(np.tile(np.arange(S, dtype=np.int32), B))
    dst = P.to_dev(np.arange(B * S, dtype=np.int64))
    dsa.dsa_index_keys(kx, kpos, table_dev, out_fp8=cache, out_scale=cscale, dst_row=dst)
    del kx, kpos, dst
    q8, qs = dsa.dsa_index_keys(P.to_dev(inp.idx_q.reshape(B * T, 64, 128)), P.to_dev(inp.q_pos.reshape(-1)),
                                table_dev)
    q8 = q8.view(B, T, 64, 128)
    qs = qs.view(B, T, 64)
    ld = (S + 3) // 4 * 4
    sc = dsa.dsa_index_scores(q8, qs, P.to_dev(inp.idx_w), cache, cscale, P.to_dev(inp.q_pos), P.to_dev(inp.kv_len),
                              ld=ld)
    idx = dsa.dsa_topk(sc, P.to_dev(inp.q_pos), P.to_dev(inp.kv_len), k)
    out, lse = dsa.dsa_sparse_mla(P.bf16_dev(inp.mla_q), P.bf16_dev(inp.mla_kv), idx)
    gs = dsa.dsa_topk(sc, P.to_dev(inp.q_pos), P.to_dev(inp.kv_len), k, flags=dsa.DSA_SORTED)
    assert _status() == 0
    # 1. the GPU's codes against the oracle's quantiser
    g_cache = cache.cpu().numpy()
    g_cscale = cscale.cpu().numpy()
    for b in seqs:
        n = int(inp.kv_len[b])
        P.check_codes(g_cache[b, :n], g_cscale[b, :n], inp.idx_k[b, :n], np.arange(n), TABLE)
    g_q8 = np.stack([q8[b, t].cpu().numpy() for b, t in rows])
    g_qs = np.stack([qs[b, t].cpu().numpy() for b, t in rows])
    P.check_codes(g_q8, g_qs, np.stack([inp.idx_q[b, t] for b, t in rows]),
                  np.array([inp.q_pos[b, t] for b, t in rows])[:, None], TABLE)
    g_idx = idx.cpu().numpy()
    g_sorted = gs.cpu().numpy()
    g_out = out.float().cpu().numpy()
    g_lse = lse.cpu().numpy()
    for j, (b, t) in enumerate(rows):
        qsl = (slice(b, b + 1), slice(t, t + 1))
        args = (g_q8[j][None, None], g_qs[j][None, None], inp.idx_w[qsl], g_cache[b:b + 1], g_cscale[b:b + 1],
                inp.q_pos[qsl], inp.kv_len[b:b + 1])
        # 2. scores on identical quantised inputs
        ref = O.index_scores(*args)
        mag = O.index_score_magnitude(*args)
        nv = O.valid_len(inp.q_pos[qsl], inp.kv_len[b:b + 1])
        own = sc[b, t].cpu().numpy()[None]
        P.check_scores(own, ref[0], mag[0], nv[0])
        # 3. the selection: bit-exact on the GPU's own scores, near-ties only against the oracle's
        own64 = own[None].astype(np.float64)
        assert np.array_equal(g_idx[b, t], O.topk_indices(own64, inp.q_pos[qsl], inp.kv_len[b:b + 1], k)[0, 0])
        assert np.array_equal(g_sorted[b, t],
                              O.topk_indices(own64, inp.q_pos[qsl], inp.kv_len[b:b + 1], k, sorted_by_score=True)[0, 0])
        ref_idx = O.topk_indices(ref, inp.q_pos[qsl], inp.kv_len[b:b + 1], k)
        P.check_topk_near_ties(g_idx[b, t][None], ref_idx[0], ref[0], mag[0], k)
        # 4. attention over the GPU's selection
        _check_mla(g_out[qsl], g_lse[qsl], inp.mla_q[qsl], inp.mla_kv[b:b + 1], g_idx[qsl])


def test_pipeline_degenerate_sequences(table_dev):
    """Decode over sequences with nothing visible (kv_len 0), one visible key, and a ragged normal
    context: masked scores are -inf, an empty selection is all -1 and gives zero output with
    lse -inf, a single key gets all the weight (the output is that latent row), and the normal
    sequence matches the oracle."""
    kv_len = [0, 1, 300]
    B, S, k = 3, 320, 64
    inp = DI.make_custom(B, 1, S, k, decode=True, seed=60, kv_len=kv_len)
    q8, qs, k8, ks = _quantised(inp)
    ld = S
    sc = torch.full((B, 1, ld), 5.0, dtype=torch.float32, device="cuda")
    dsa.dsa_index_scores(P.to_dev(q8), P.to_dev(qs), P.to_dev(inp.idx_w), P.to_dev(k8), P.to_dev(ks),
                         P.to_dev(inp.q_pos), P.to_dev(inp.kv_len), scores=sc, ld=ld, flags=dsa.DSA_FILL_MASKED)
    idx = dsa.dsa_topk(sc, P.to_dev(inp.q_pos), P.to_dev(inp.kv_len), k)
    out, lse = dsa.dsa_sparse_mla(P.bf16_dev(inp.mla_q), P.bf16_dev(inp.mla_kv), idx)
    assert _status() == 0
    s, i, o, l = sc.cpu().numpy(), idx.cpu().numpy(), out.float().cpu().numpy(), lse.cpu().numpy()
    assert np.all(np.isneginf(s[0, 0])) and np.all(i[0, 0] == -1)
    assert np.all(o[0] == 0) and np.all(np.isneginf(l[0]))
    assert np.all(np.isneginf(s[1, 0, 1:])) and np.isfinite(s[1, 0, 0])
    assert i[1, 0, 0] == 0 and np.all(i[1, 0, 1:] == -1)
    assert np.array_equal(o[1, 0], np.broadcast_to(O.bf16_to_f64(inp.mla_kv[1, 0, :512]), (128, 512)))
    ref = O.index_scores(q8, qs, inp.idx_w, k8, ks, inp.q_pos, inp.kv_len)
    mag = O.index_score_magnitude(q8, qs, inp.idx_w, k8, ks, inp.q_pos, inp.kv_len)
    P.check_scores(s[2], ref[2], mag[2], O.valid_len(inp.q_pos, inp.kv_len)[2])
    assert np.array_equal(i[2], O.topk_indices(s[2:3].astype(np.float64), inp.q_pos[2:3], inp.kv_len[2:3], k)[0])
    _check_mla(o[2:3], l[2:3], inp.mla_q[2:3], inp.mla_kv[2:3], i[2:3])
