"""Pins for the CPU oracle: each oracle function checked against something other than itself
(closed forms, hand-derived examples in tests/golden, library routines, brute-force loops,
invariants). These run without a GPU.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import scipy.linalg
import torch

from oracle import dsa_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ------------------------------------------------------------------------------------- e4m3 codec
def test_e4m3_decode_closed_form_and_torch():
    codes = np.arange(256, dtype=np.uint8)
    mine = O.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(mine), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(mine[ok], ref[ok])
    # closed-form spot values of the format definition
    assert O.e4m3_decode(0x7E) == 448.0
    assert O.e4m3_decode(0xFE) == -448.0
    assert O.e4m3_decode(0x01) == 2.0 ** -9
    assert O.e4m3_decode(0x07) == 7 * 2.0 ** -9
    assert O.e4m3_decode(0x08) == 2.0 ** -6
    assert O.e4m3_decode(0x76) == 224.0
    assert O.e4m3_decode(0x38) == 1.0
    assert np.isnan(O.e4m3_decode(0x7F)) and np.isnan(O.e4m3_decode(0xFF))


def _torch_e4m3(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_e4m3_encode_matches_torch_on_values_midpoints_and_random():
    vals = O.e4m3_decode(np.arange(127, dtype=np.uint8))
    mids = (vals[1:] + vals[:-1]) / 2          # exact in fp32: every tie point
    nudged = np.concatenate([np.nextafter(mids.astype(np.float32), np.float32(0)),
                             np.nextafter(mids.astype(np.float32), np.float32(1e9))])
    rng = np.random.default_rng(1)
    rand = np.concatenate([rng.uniform(-464, 464, 200000),
                           rng.standard_normal(200000) * 0.01,
                           np.ldexp(rng.uniform(1, 2, 20000), rng.integers(-14, 9, 20000))])
    x = np.concatenate([vals, -vals, mids, -mids, nudged, -nudged, rand]).astype(np.float32)
    x = x[np.abs(x) <= 464]                    # torch's cast does not saturate beyond the 448/480 tie
    assert np.array_equal(O.e4m3_encode(x), _torch_e4m3(x))


def test_e4m3_encode_ties_to_even_and_saturation():
    # 1.0625 lies halfway between 1.0 (code 0x38, even) and 1.125 (0x39): goes to 1.0
    assert O.e4m3_encode(np.float32(1.0625)) == 0x38
    # 1.1875 halfway between 1.125 (0x39) and 1.25 (0x3A, even): goes to 1.25
    assert O.e4m3_encode(np.float32(1.1875)) == 0x3A
    # half the smallest subnormal ties to zero; 3/4 of it rounds up
    assert O.e4m3_encode(np.float32(2.0 ** -10)) == 0x00
    assert O.e4m3_encode(np.float32(0.75 * 2.0 ** -9)) == 0x01
    for big in (448.0, 464.0, 465.0, 480.0, 1e6, 3.0e38):
        assert O.e4m3_encode(np.float32(big)) == 0x7E
        assert O.e4m3_encode(np.float32(-big)) == 0xFE
    assert O.e4m3_encode(np.float32(-1e-9)) == 0x80
    assert O.e4m3_encode(np.float32(np.nan)) == 0x7F


# ------------------------------------------------------------------------------------- YaRN / RoPE
def test_yarn_frequencies_closed_form():
    g = _golden("rope_yarn_values.json")
    assert O.yarn_correction_range() == (g["low"], g["high"])
    f = O.yarn_inv_freq()
    base = 1e4 ** (-np.arange(32) / 32.0)
    assert f[0] == g["inv_freq_0"]
    assert math.isclose(f[31], g["inv_freq_31"], rel_tol=1e-12)
    for i in range(32):
        if i <= 10:
            want = base[i]
        elif i >= 23:
            want = base[i] / 40
        else:
            r = (i - 10) / 13
            want = base[i] / 40 * r + base[i] * (1 - r)
        assert math.isclose(f[i], want, rel_tol=1e-12), i


def test_rope_table_and_pairing():
    g = _golden("rope_yarn_values.json")
    tab = O.rope_table(64)
    assert tab.shape == (64, 32, 2) and tab.dtype == np.float32
    assert np.all(tab[0, :, 0] == 1.0) and np.all(tab[0, :, 1] == 0.0)
    assert tab[1, 0, 0] == np.float32(g["pos1_pair0_cos"])
    assert tab[1, 0, 1] == np.float32(g["pos1_pair0_sin"])
    e0 = np.zeros(128); e0[0] = 1
    y = O.rope_noninterleaved(e0, 1, tab)
    # pair 0 is features (0, 32), not (0, 1)
    assert y[0] == np.float64(tab[1, 0, 0]) and y[32] == np.float64(tab[1, 0, 1])
    assert np.count_nonzero(y) == 2
    e32 = np.zeros(128); e32[32] = 1
    y = O.rope_noninterleaved(e32, 1, tab)
    assert y[0] == -np.float64(tab[1, 0, 1]) and y[32] == np.float64(tab[1, 0, 0])


def test_rope_invariants():
    tab = O.rope_table(4096)
    rng = np.random.default_rng(2)
    x = rng.standard_normal((50, 128)).astype(np.float32)
    pos = rng.integers(0, 4096, 50)
    y = O.rope_noninterleaved(x, pos, tab)
    assert np.array_equal(y[:, 64:], x[:, 64:].astype(np.float64))          # tail unchanged
    assert np.array_equal(O.rope_noninterleaved(x, 0, tab), x.astype(np.float64))  # pos 0 identity
    n_in = x[:, :32].astype(np.float64) ** 2 + x[:, 32:64].astype(np.float64) ** 2
    n_out = y[:, :32] ** 2 + y[:, 32:64] ** 2
    assert np.allclose(n_in, n_out, rtol=1e-6, atol=1e-9)                      # rotation per pair
    # relative-position property of the rotated part: q(t).k(s) depends only on t-s
    q = rng.standard_normal(128); k = rng.standard_normal(128)
    d1 = O.rope_noninterleaved(q, 700, tab)[:64] @ O.rope_noninterleaved(k, 500, tab)[:64]
    d2 = O.rope_noninterleaved(q, 1200, tab)[:64] @ O.rope_noninterleaved(k, 1000, tab)[:64]
    assert math.isclose(d1, d2, rel_tol=1e-4, abs_tol=1e-4)


# ------------------------------------------------------------------------------------- Hadamard
def test_hadamard_against_scipy_and_orthonormal():
    H = O.hadamard_matrix(128)
    assert np.array_equal(H, scipy.linalg.hadamard(128).astype(np.float64))
    assert np.array_equal(H @ H.T, 128 * np.eye(128))
    rng = np.random.default_rng(3)
    x = rng.standard_normal((7, 128))
    y = O.hadamard_rotate(x)
    assert np.allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-12)
    assert np.allclose(O.hadamard_rotate(y), x, atol=1e-12)
    e0 = np.zeros(128); e0[0] = 1
    assert np.allclose(O.hadamard_rotate(e0), np.full(128, 128 ** -0.5), atol=0)


# ------------------------------------------------------------------------------------- act_quant
def test_act_quant_scale_and_error_bound():
    rng = np.random.default_rng(4)
    x = (rng.standard_normal((300, 128)) * np.exp(rng.uniform(-8, 8, (300, 1)))).astype(np.float32)
    codes, scale = O.act_quant(x)
    amax = np.abs(x).max(axis=1)
    assert np.array_equal(scale, (amax / np.float32(448)).astype(np.float32))
    # the largest-magnitude element lands on +-448
    j = np.abs(x).argmax(axis=1)
    top = codes[np.arange(300), j]
    assert np.all((top == 0x7E) | (top == 0xFE))
    deq = O.e4m3_decode(codes) * scale[:, None].astype(np.float64)
    # round-to-nearest: error at most half a step; e4m3 steps are 2^-3 relative for normals
    # and 2^-9 absolute (times the scale) in the subnormal range
    err = np.abs(deq - x)
    bound = np.maximum(np.abs(x) * 2.0 ** -4, 2.0 ** -10 * scale[:, None]) * (1 + 1e-6)
    assert np.all(err <= bound)


def test_act_quant_zero_block():
    codes, scale = O.act_quant(np.zeros((2, 128), np.float32))
    assert np.all(codes == 0) and np.all(scale == np.float32(np.float32(1e-4) / np.float32(448)))


def test_index_keys_composition():
    tab = O.rope_table(100)
    rng = np.random.default_rng(5)
    x = rng.standard_normal((3, 4, 128)).astype(np.float32)
    c0, s0 = O.index_keys(x, 0, tab, hadamard=False)                # pos 0, no Hadamard -> plain quant
    c1, s1 = O.act_quant(x)
    assert np.array_equal(c0, c1) and np.array_equal(s0, s1)
    c, s = O.index_keys(x, 57, tab, hadamard=True)
    deq = O.e4m3_decode(c) * s[..., None]
    want = O.hadamard_rotate(O.rope_noninterleaved(x, 57, tab))
    assert np.all(np.abs(deq - want) <= np.abs(want) * 2.0 ** -4 + 2.0 ** -9 * s[..., None] + 1e-7)


# ------------------------------------------------------------------------------------- scores
def _two_head_case(w_pair):
    g = _golden("indexer_two_head_example.json")
    enc = {int(k): v for k, v in g["codes"].items()}
    q8 = np.zeros((1, 1, 64, 128), np.uint8)
    q8[0, 0, 0, 64] = enc[448]
    q8[0, 0, 1, 65] = enc[448]
    k8 = np.zeros((1, 4, 128), np.uint8)
    for s, (a, b) in enumerate(g["k_features"]):
        k8[0, s, 64] = enc[a]
        k8[0, s, 65] = enc[b]
    w = np.zeros((1, 1, 64), np.float32)
    w[0, 0, :2] = w_pair
    return q8, np.ones((1, 1, 64), np.float32), w, k8, np.ones((1, 4), np.float32)


def test_scores_two_head_golden_example():
    g = _golden("indexer_two_head_example.json")
    unit = 1568 * math.sqrt(2)
    for case in g["cases"]:
        q8, qs, w, k8, ks = _two_head_case(case["w"])
        sc = O.index_scores(q8, qs, w, k8, ks, q_pos=[[3]], kv_len=[4])
        assert np.allclose(sc[0, 0], np.array(case["scores_over_1568_sqrt2"]) * unit, rtol=1e-12)
        top = O.topk_indices(sc, [[3]], [4], 2)
        assert top[0, 0].tolist() == case["top2"]


def _brute_scores(q8, qs, w, k8, ks, q_pos, kv_len, sm, magnitude=False):
    """Triple loop over (query, key, head) of the score; with magnitude=True the same sum with
    every folded head weight replaced by its absolute value (the error scale of an accumulation
    of mixed-sign terms)."""
    B, T, H, D = q8.shape
    S = k8.shape[1]
    out = np.full((B, T, S), -np.inf) if not magnitude else np.zeros((B, T, S))
    dec = {c: float(O.e4m3_decode(c)) for c in range(256)}
    for b in range(B):
        for t in range(T):
            n = min(q_pos[b][t] + 1, kv_len[b]) if not magnitude else S
            for s in range(n):
                tot = 0.0
                for j in range(H):
                    dot = 0.0
                    for i in range(D):
                        dot += dec[int(q8[b, t, j, i])] * dec[int(k8[b, s, i])]
                    wj = float(w[b, t, j]) * H ** -0.5 * float(qs[b, t, j]) * sm
                    tot += (abs(wj) if magnitude else wj) * max(dot, 0.0)
                out[b, t, s] = tot * float(ks[b, s])
    return out


def test_scores_bruteforce_small():
    rng = np.random.default_rng(6)
    B, T, H, S, D = 2, 3, 4, 6, 128
    q8 = rng.integers(0, 256, (B, T, H, D)).astype(np.uint8)
    k8 = rng.integers(0, 256, (B, S, D)).astype(np.uint8)
    q8[(q8 & 0x7F) == 0x7F] = 0x10       # no NaN codes
    k8[(k8 & 0x7F) == 0x7F] = 0x10
    qs = rng.uniform(0.01, 1, (B, T, H)).astype(np.float32)
    ks = rng.uniform(0.01, 1, (B, S)).astype(np.float32)
    w = rng.standard_normal((B, T, H)).astype(np.float32)
    q_pos = [[2, 4, 5], [0, 1, 5]]
    kv_len = [6, 4]
    got = O.index_scores(q8, qs, w, k8, ks, q_pos, kv_len, softmax_scale=0.3)
    want = _brute_scores(q8, qs, w, k8, ks, q_pos, kv_len, 0.3)
    assert np.array_equal(np.isinf(got), np.isinf(want))
    fin = np.isfinite(want)
    assert np.allclose(got[fin], want[fin], rtol=1e-12, atol=1e-12)


def test_score_magnitude_bruteforce_mixed_sign_weights():
    """index_score_magnitude (the denominator of the score parity bar) against the triple loop with
    |w'_j|: a dropped abs, a wrong factor of the weight fold or a missing k_scale fails here."""
    rng = np.random.default_rng(16)
    B, T, H, S, D = 2, 2, 5, 7, 128
    q8 = rng.integers(0, 256, (B, T, H, D)).astype(np.uint8)
    k8 = rng.integers(0, 256, (B, S, D)).astype(np.uint8)
    q8[(q8 & 0x7F) == 0x7F] = 0x21
    k8[(k8 & 0x7F) == 0x7F] = 0x21
    qs = rng.uniform(0.01, 1, (B, T, H)).astype(np.float32)
    ks = rng.uniform(0.01, 1, (B, S)).astype(np.float32)
    w = rng.standard_normal((B, T, H)).astype(np.float32)
    w[0, 0, :3] = [-2.0, 1.5, -0.25]                     # mixed signs on purpose
    q_pos, kv_len = [[3, 6], [6, 2]], [7, 5]
    got = O.index_score_magnitude(q8, qs, w, k8, ks, q_pos, kv_len, softmax_scale=0.3)
    want = _brute_scores(q8, qs, w, k8, ks, q_pos, kv_len, 0.3, magnitude=True)
    assert np.allclose(got, want, rtol=1e-12, atol=1e-12)
    # it bounds the score, and equals it where every weight is positive
    sc = O.index_scores(q8, qs, w, k8, ks, q_pos, kv_len, softmax_scale=0.3)
    fin = np.isfinite(sc)
    assert np.all(np.abs(sc[fin]) <= got[fin] * (1 + 1e-12))
    pos_w = np.abs(w)
    sc_pos = O.index_scores(q8, qs, pos_w, k8, ks, q_pos, kv_len, softmax_scale=0.3)
    fin = np.isfinite(sc_pos)
    assert np.allclose(sc_pos[fin], got[fin], rtol=1e-12, atol=0)
    # with some weight negative somewhere the magnitude is strictly larger for some entry
    assert np.any(got[fin] > np.abs(sc[fin]) * (1 + 1e-9))


def test_gemm_abs_terms_explicit_loops():
    """gemm_abs_terms (the error scale of the absorption parity bars) against explicit loops on
    the two contractions the producers use, with mixed-sign operands."""
    rng = np.random.default_rng(17)
    T, H, D, C = 2, 3, 4, 5
    a = rng.standard_normal((T, H, D))
    w = rng.standard_normal((H, D, C))
    got = O.gemm_abs_terms(a, w, "thd,hdc->thc")
    for t in range(T):
        for h in range(H):
            for c in range(C):
                want = sum(abs(a[t, h, d]) * abs(w[h, d, c]) for d in range(D))
                assert math.isclose(got[t, h, c], want, rel_tol=1e-13)
    o = rng.standard_normal((T, H, C))
    got = O.gemm_abs_terms(o, w, "thc,hdc->thd")
    for t in range(T):
        for h in range(H):
            for d in range(D):
                want = sum(abs(o[t, h, c]) * abs(w[h, d, c]) for c in range(C))
                assert math.isclose(got[t, h, d], want, rel_tol=1e-13)
    # it is never below the magnitude of the contraction itself
    assert np.all(got >= np.abs(np.einsum("thc,hdc->thd", o, w)) - 1e-12)


def test_bf16_decode_every_bit_pattern_against_torch():
    """bf16_to_f64 (which decodes every bf16 input of the MLA oracle) against torch's bf16 -> fp64
    conversion over all 65,536 bit patterns, and on closed-form values of the format."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    with np.errstate(invalid="ignore"):              # signalling-NaN patterns widen to quiet NaNs
        mine = O.bf16_to_f64(bits)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(mine), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(mine[ok], ref[ok])
    assert np.array_equal(np.signbit(mine[ok]), np.signbit(ref[ok]))
    # closed forms: 1 sign, 8 exponent bits (bias 127), 7 mantissa bits
    assert O.bf16_to_f64(np.uint16(0x3F80)) == 1.0
    assert O.bf16_to_f64(np.uint16(0xC000)) == -2.0
    assert O.bf16_to_f64(np.uint16(0x3FC0)) == 1.5
    assert O.bf16_to_f64(np.uint16(0x0001)) == 2.0 ** -133          # smallest subnormal
    assert O.bf16_to_f64(np.uint16(0x7F7F)) == (2 - 2.0 ** -7) * 2.0 ** 127
    assert np.isinf(O.bf16_to_f64(np.uint16(0x7F80))) and np.isnan(O.bf16_to_f64(np.uint16(0x7FC0)))


def test_scores_single_head_is_relu_matmul():
    rng = np.random.default_rng(7)
    q = rng.standard_normal((5, 128)).astype(np.float32)
    k = rng.standard_normal((9, 128)).astype(np.float32)
    q8, _ = O.act_quant(q)
    k8, _ = O.act_quant(k)
    qd, kd = O.e4m3_decode(q8), O.e4m3_decode(k8)
    got = O.index_scores(q8[None, :, None, :], np.ones((1, 5, 1), np.float32), np.ones((1, 5, 1), np.float32),
                         k8[None], np.ones((1, 9), np.float32), [[8] * 5], [9], softmax_scale=1.0)
    want = torch.clamp(torch.from_numpy(qd) @ torch.from_numpy(kd).T, min=0).numpy()
    assert np.array_equal(got[0], want)


def test_relu_zeroes_negative_dots_and_causal_mask():
    q8 = np.zeros((1, 2, 64, 128), np.uint8)
    q8[:, :, :, 0] = 0x38                 # +1 in feature 0 for every head
    k8 = np.zeros((1, 3, 128), np.uint8)
    k8[0, 0, 0] = 0xB8                    # -1: every head's dot is negative
    k8[0, 1, 0] = 0x38
    k8[0, 2, 0] = 0x38
    w = np.ones((1, 2, 64), np.float32)
    sc = O.index_scores(q8, np.ones((1, 2, 64), np.float32), w, k8, np.ones((1, 3), np.float32),
                        q_pos=[[1, 2]], kv_len=[3])
    assert sc[0, 0, 0] == 0.0 and sc[0, 1, 0] == 0.0
    assert sc[0, 0, 1] > 0 and np.isneginf(sc[0, 0, 2])     # s > pos is masked
    g = _golden("rope_yarn_values.json")
    assert O.valid_len([[1000]], [1001])[0, 0] == g["visible_keys_at_p1000"]


# ------------------------------------------------------------------------------------- top-k
def test_topk_against_sorted_bruteforce_with_ties():
    rng = np.random.default_rng(8)
    for S in range(1, 9):
        for trial in range(30):
            vals = rng.integers(-3, 4, S).astype(np.float64)     # many exact ties
            for k in range(1, S + 2):
                got = O.topk_indices(vals[None, None, :], [[S - 1]], [S], k)[0, 0]
                order = sorted(range(S), key=lambda s: (-vals[s], s))[:min(k, S)]
                want = sorted(order) + [-1] * (k - min(k, S))
                assert got.tolist() == want


def test_topk_respects_visibility_and_pads():
    rng = np.random.default_rng(9)
    sc = rng.standard_normal((1, 3, 40))
    out = O.topk_indices(sc, [[0, 9, 39]], [30], 16)
    assert out[0, 0].tolist() == [0] + [-1] * 15
    assert out[0, 1].tolist() == list(range(10)) + [-1] * 6
    assert max(out[0, 2]) < 30 and -1 not in out[0, 2]
    want = sorted(sorted(range(30), key=lambda s: (-sc[0, 2, s], s))[:16])
    assert out[0, 2].tolist() == want


# ------------------------------------------------------------------------------------- sparse MLA
def test_mla_softmax_scale_closed_form():
    assert math.isclose(O.MLA_SOFTMAX_SCALE, 192 ** -0.5 * (1 + 0.1 * math.log(40)) ** 2, rel_tol=1e-15)
    assert abs(O.MLA_SOFTMAX_SCALE - 0.13523378) < 1e-8
    assert math.isclose(O.INDEXER_SOFTMAX_SCALE * O.INDEXER_HEAD_SCALE, 1 / (8 * math.sqrt(128)), rel_tol=1e-15)


def _bf16(rng, shape):
    return torch.from_numpy(rng.standard_normal(shape).astype(np.float32)).to(torch.bfloat16).view(torch.uint16).numpy()


def test_sparse_mla_single_key_returns_latent():
    rng = np.random.default_rng(10)
    q = _bf16(rng, (1, 2, 4, 576))
    kv = _bf16(rng, (1, 10, 576))
    idx = np.array([[[7, -1, -1], [-1, 3, -1]]], np.int32)
    out, lse = O.sparse_mla(q, kv, idx)
    kvf = O.bf16_to_f64(kv)
    assert np.array_equal(out[0, 0], np.broadcast_to(kvf[0, 7, :512], (4, 512)))
    assert np.array_equal(out[0, 1], np.broadcast_to(kvf[0, 3, :512], (4, 512)))
    z = O.bf16_to_f64(q)[0, 0] @ kvf[0, 7] * O.MLA_SOFTMAX_SCALE
    assert np.allclose(lse[0, 0], z, rtol=1e-14)


def test_sparse_mla_full_selection_equals_torch_sdpa():
    rng = np.random.default_rng(11)
    B, T, H, S = 2, 5, 3, 7
    q = _bf16(rng, (B, T, H, 576))
    kv = _bf16(rng, (B, S, 576))
    q_pos = np.array([[2, 3, 4, 5, 6]] * B)
    kv_len = np.array([S, S])
    idx = np.full((B, T, S), -1, np.int32)
    for b in range(B):
        for t in range(T):
            idx[b, t, :q_pos[b, t] + 1] = rng.permutation(q_pos[b, t] + 1)   # order must not matter
    out, _ = O.sparse_mla(q, kv, idx)
    qt = torch.from_numpy(O.bf16_to_f64(q)).permute(0, 2, 1, 3)               # [B,H,T,576]
    kt = torch.from_numpy(O.bf16_to_f64(kv))[:, None].expand(B, H, S, 576)
    vt = kt[..., :512]
    mask = torch.from_numpy(np.arange(S)[None, :] <= q_pos[0][:, None])        # [T,S]
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask,
                                                           scale=O.MLA_SOFTMAX_SCALE)
    assert np.allclose(out, ref.permute(0, 2, 1, 3).numpy(), rtol=1e-10, atol=1e-12)
    dense, _ = O.dense_mla(q, kv, q_pos, kv_len)
    assert np.allclose(out, dense, rtol=1e-12, atol=1e-14)


def test_sparse_mla_bruteforce_tiny_dims():
    rng = np.random.default_rng(12)
    q = _bf16(rng, (1, 1, 2, 6))
    kv = _bf16(rng, (1, 5, 6))
    idx = np.array([[[4, -1, 0, 2]]], np.int32)
    out, lse = O.sparse_mla(q, kv, idx, softmax_scale=0.7, d_v=4)
    qf, kf = O.bf16_to_f64(q), O.bf16_to_f64(kv)
    for h in range(2):
        zs = [0.7 * sum(qf[0, 0, h, d] * kf[0, u, d] for d in range(6)) for u in (4, 0, 2)]
        den = sum(math.exp(z) for z in zs)
        for d in range(4):
            want = sum(math.exp(z) / den * kf[0, u, d] for z, u in zip(zs, (4, 0, 2)))
            assert math.isclose(out[0, 0, h, d], want, rel_tol=1e-12, abs_tol=1e-14)
        assert math.isclose(lse[0, 0, h], math.log(den), rel_tol=1e-12)


def test_sparse_mla_empty_row():
    rng = np.random.default_rng(13)
    out, lse = O.sparse_mla(_bf16(rng, (1, 1, 2, 576)), _bf16(rng, (1, 4, 576)), np.full((1, 1, 3), -1, np.int32))
    assert np.all(out == 0) and np.all(np.isneginf(lse))


def test_topk_sorted_order_against_python_sort():
    """sorted_by_score is the order of Python's stable sort by (-score, position) (tiny rows with
    forced ties and negative zero), truncated to k and padded with -1."""
    rng = np.random.default_rng(11)
    for trial in range(200):
        n = int(rng.integers(1, 12))
        row = rng.choice([-1.5, -0.0, 0.0, 0.25, 2.0, 3.0], size=n).astype(np.float32)
        k = int(rng.integers(1, 14))
        got = O.topk_indices(row[None, None, :], np.array([[n - 1]], np.int32), np.array([n], np.int32), k,
                             sorted_by_score=True)[0, 0]
        want = sorted(range(n), key=lambda s: (-float(row[s]), s))[:k]
        want = want + [-1] * (k - len(want))
        assert got.tolist() == want, (row, k)


# ------------------------------------------------------------------------------------ paged caches
def test_paged_gather_worked_example():
    # page_size 2, pool rows labelled by their own row number: sequence 0 uses pages (2, 0), so its
    # positions 0..3 are pool rows 4, 5, 0, 1; sequence 1 uses pages (1, 3): rows 2, 3, 6, 7
    pool = np.arange(8, dtype=np.int64)[:, None] * np.ones((1, 3), np.int64)
    got = O.paged_gather(pool, np.array([[2, 0], [1, 3]]), 2, [4, 4])
    assert got[:, :, 0].tolist() == [[4, 5, 0, 1], [2, 3, 6, 7]]
    assert np.all(got == got[:, :, :1])


def test_paged_gather_identity_table_is_a_reshape():
    rng = np.random.default_rng(0)
    B, max_pages, P = 3, 4, 8
    pool = rng.standard_normal((B * max_pages * P, 5))
    table = np.arange(B * max_pages).reshape(B, max_pages)
    got = O.paged_gather(pool, table, P, [max_pages * P] * B)
    assert np.array_equal(got, pool.reshape(B, max_pages * P, 5))


def test_paged_gather_inverts_a_shuffled_layout():
    import dsa_inputs as DI
    rng = np.random.default_rng(1)
    B, max_pages, P = 2, 5, 64
    dense = rng.integers(0, 256, (B, max_pages * P, 7), dtype=np.uint8)
    kv_len = np.array([max_pages * P, 130])
    table, num_pages = DI.paged_layout(B, max_pages, P, seed=2, kv_len=kv_len, past_end=-7)
    pool = DI.to_paged(dense, table, P, num_pages, fill=255)
    got = O.paged_gather(pool, table, P, kv_len)
    for b in range(B):
        assert np.array_equal(got[b, :kv_len[b]], dense[b, :kv_len[b]])
        assert np.all(got[b, kv_len[b]:] == 0)
    assert np.all(table[1, 3:] == -7)                       # pages past the end are never read


def test_paged_gather_rejects_a_visible_bad_page():
    pool = np.zeros((8, 2))
    with pytest.raises(IndexError):
        O.paged_gather(pool, np.array([[0, 4]]), 2, [3])      # position 2 lives on page 4 of 4
    O.paged_gather(pool, np.array([[0, 4]]), 2, [2])          # ... unless it is past the end


# ---------------------------------------------------------------------------- MLA producers
def _bf16_bits(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_rope_interleaved_is_the_regrouped_noninterleaved_rotation():
    # the excerpt's interleaved=False path regroups the halves into pairs, rotates, and restores
    # the halves: so rotating the de-interleaved vector the non-interleaved way and interleaving
    # the result back must give the interleaved rotation
    rng = np.random.default_rng(3)
    table = O.rope_table(5000)
    x = rng.standard_normal((6, 64))
    pos = np.array([0, 1, 17, 1000, 4095, 4999])
    halves = np.concatenate([x[:, 0::2], x[:, 1::2]], axis=1)
    y = O.rope_noninterleaved(halves, pos, table)
    back = np.empty_like(x)
    back[:, 0::2], back[:, 1::2] = y[:, :32], y[:, 32:]
    assert np.allclose(O.rope_interleaved(x, pos, table), back, rtol=0, atol=1e-12)


def test_rope_interleaved_complex_product_and_norms():
    rng = np.random.default_rng(4)
    table = O.rope_table(3000)
    x = rng.standard_normal((5, 64))
    pos = np.array([0, 3, 100, 2047, 2999])
    got = O.rope_interleaved(x, pos, table)
    z = (x[:, 0::2] + 1j * x[:, 1::2]) * (table[pos, :, 0] + 1j * table[pos, :, 1]).astype(np.complex128)
    assert np.allclose(got[:, 0::2], z.real, atol=1e-12) and np.allclose(got[:, 1::2], z.imag, atol=1e-12)
    pair_norm = lambda v: np.hypot(v[:, 0::2], v[:, 1::2])
    assert np.allclose(pair_norm(got), pair_norm(x), rtol=1e-6)
    assert np.array_equal(got[0], x[0])                          # position 0: cos 1, sin 0


def test_q_absorb_gives_the_unabsorbed_scores():
    # MHA prefill path: k_nope[s,h,d] = sum_c w[h,d,c] kv[s,c] (wkv_b up-projection), score =
    # q_nope . k_nope; the absorbed query must give the same latent score q_abs . kv
    rng = np.random.default_rng(5)
    H, D, C, T, S = 2, 3, 5, 2, 4
    qn = _bf16_bits(rng.standard_normal((T, H, D)))
    qp = _bf16_bits(rng.standard_normal((T, H, 64)))
    w = _bf16_bits(rng.standard_normal((H, D, C)))
    kv = O.bf16_to_f64(_bf16_bits(rng.standard_normal((S, C))))
    table = O.rope_table(16)
    q = O.mla_q_absorb(qn, qp, np.array([3, 9]), table, w)
    qn64, w64 = O.bf16_to_f64(qn), O.bf16_to_f64(w)
    for t in range(T):
        for h in range(H):
            for s in range(S):
                k_nope = [sum(w64[h, d, c] * kv[s, c] for c in range(C)) for d in range(D)]
                want = sum(qn64[t, h, d] * k_nope[d] for d in range(D))
                assert math.isclose(sum(q[t, h, c] * kv[s, c] for c in range(C)), want, rel_tol=1e-12, abs_tol=1e-12)
    assert np.allclose(q[..., C:], O.rope_interleaved(O.bf16_to_f64(qp), np.array([[3], [9]]), table), atol=0)


def test_out_absorb_gives_the_unabsorbed_values():
    # MHA prefill path: v[s,h,d] = sum_c w_uv[h,d,c] kv[s,c]; out = sum_s p_s v[s]. The absorbed
    # form up-projects the latent mix o = sum_s p_s kv[s] instead
    rng = np.random.default_rng(6)
    H, D, C, S = 2, 3, 4, 5
    kv = rng.standard_normal((S, C))
    p = rng.random((H, S))
    p /= p.sum(axis=1, keepdims=True)
    w = _bf16_bits(rng.standard_normal((H, D, C)))
    o = np.einsum("hs,sc->hc", p, kv)
    ob = _bf16_bits(o)[None]                                    # [1, H, C]
    got = O.mla_out_absorb(ob, w)[0]
    o64, w64 = O.bf16_to_f64(ob)[0], O.bf16_to_f64(w)
    for h in range(H):
        for d in range(D):
            assert math.isclose(got[h, d], sum(o64[h, c] * w64[h, d, c] for c in range(C)), rel_tol=1e-12)
            v = [sum(w64[h, d, c] * kv[s, c] for c in range(C)) for s in range(S)]
            exact = sum(p[h, s] * v[s] for s in range(S))
            assert abs(got[h, d] - exact) <= 2 ** -7 * sum(abs(o[h, c] * w64[h, d, c]) for c in range(C))


def test_kv_entry_keeps_the_latent_and_rotates_the_rope_key():
    rng = np.random.default_rng(7)
    kv = _bf16_bits(rng.standard_normal((3, 512)))
    kp = _bf16_bits(rng.standard_normal((3, 64)))
    table = O.rope_table(64)
    row = O.mla_kv_entry(kv, kp, np.array([0, 5, 63]), table)
    assert np.array_equal(row[:, :512], O.bf16_to_f64(kv))
    assert np.array_equal(row[0, 512:], O.bf16_to_f64(kp)[0])
    assert np.allclose(row[1:, 512:], O.rope_interleaved(O.bf16_to_f64(kp)[1:], np.array([5, 63]), table), atol=0)
