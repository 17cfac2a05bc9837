"""CPU oracle for the DeepSeek Sparse Attention hot path (TEST INFRASTRUCTURE ONLY).

This module is the plain, slow, obviously-correct definition of what the CUDA
path computes. Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may import it; the product package never does, and the two
share no code (only the seeded input generators in ``dsa_inputs``).

Arithmetic is numpy float64 unless a page fixes a precision (the FP8 codes and
the fp32 block scales). Every function cites the page passage it restates:

* "DeepSeek fixes RoPE mismatch in the V3.2-Exp inference demo" (aipricedb.com news
  page): the index-score formula I[t,s] = sum_j w[t,j] * ReLU(q[t,j] . k[s]) with
  64 heads, ReLU instead of softmax, block-wise FP8 quantisation with 128-element
  blocks, and the non-interleaved indexer RoPE notice.
* "DeepSeek-V3.2-Exp - RoPE coefficients" (atlas page, block-rotations): the YaRN
  frequency code (precompute excerpt) and the ModelArgs defaults.
* "DeepSeek-V3.2-Exp - Dense transformer block / Sparse latent attention" (atlas
  page, dense-blocks): the lightning-indexer steps (RoPE_64, (1/sqrt 128) H_128,
  S^I = 1/(sqrt64 sqrt128) sum_h w ReLU(.), top-2048 with the causal mask) and the
  sparse-attention steps (S' = S m^2/sqrt(192), m = 1 + 0.1 ln 40, softmax, O = AV);
  the MLA prefill excerpt.
* "DeepSeek-V3.2-Exp - Rotate first features" (atlas page, index-keys/rotate):
  Indexer.forward excerpt and apply_rotary_emb excerpt.
* "DeepSeek-V3.2-Exp - Similarities" (atlas page, attend/weights/similarities):
  the absorbed MQA decode excerpt and the p+1 visible keys at p=1000.

Readings where the pages are silent or garbled are marked READING.
Pins for every function live in tests/test_oracle_pins.py.
"""
from __future__ import annotations

import math

import numpy as np

H_I = 64
D_I = 128
BLOCK = 128                 # FP8 quantisation block (one indexer head row)
E4M3_MAX = 448.0
ROPE_DIM = 64               # qk_rope_head_dim; also the rotated prefix of the indexer head
ROPE_PAIRS = ROPE_DIM // 2

# ModelArgs defaults (RoPE coefficients page, model-args excerpt)
MAX_SEQ_LEN = 4096 * 4
ORIGINAL_SEQ_LEN = 4096
ROPE_THETA = 10000.0
ROPE_FACTOR = 40.0
BETA_FAST = 32
BETA_SLOW = 1
MSCALE = 1.0

# Indexer score scale: 1/(sqrt(64) sqrt(128)) (dense-block page, lightning indexer step);
# in Indexer.forward it is n_heads**-0.5 times softmax_scale = head_dim**-0.5.
INDEXER_SOFTMAX_SCALE = D_I ** -0.5
INDEXER_HEAD_SCALE = H_I ** -0.5

# MLA softmax scale: qk_head_dim**-0.5 * mscale**2 with mscale = 0.1*ln(factor)+1
# (MLA init excerpt; dense-block page "S' = S m^2/sqrt(192)").
MLA_QK_HEAD_DIM = 128 + 64
MLA_MSCALE = 0.1 * MSCALE * math.log(ROPE_FACTOR) + 1.0
MLA_SOFTMAX_SCALE = MLA_QK_HEAD_DIM ** -0.5 * MLA_MSCALE * MLA_MSCALE


# ----------------------------------------------------------------------------------------------
# e4m3fn codec, written from the format definition (1 sign, 4 exponent bits with bias 7,
# 3 mantissa bits; no infinities; S.1111.111 is NaN; largest finite 448; smallest subnormal 2^-9)
# ----------------------------------------------------------------------------------------------
def e4m3_decode(codes) -> np.ndarray:
    """Value of each e4m3fn byte, float64 (NaN for the two NaN codes)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    normal = np.ldexp(1.0 + m / 8.0, (e - 7).astype(np.int64))
    subnormal = m * 2.0 ** -9
    mag = np.where(e == 0, subnormal, normal)
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return sign * mag


_E4M3_POS = e4m3_decode(np.arange(127, dtype=np.uint8))   # codes 0..126, strictly increasing


def e4m3_encode(x) -> np.ndarray:
    """Round each value to the nearest e4m3fn code, ties to the even code, saturating at 448.

    Input is fp32 (the quotient x/scale of act_quant); the sign of zero-rounded values is kept
    (negative values that round to zero give 0x80). NaN maps to 0x7F.
    """
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    hi = np.searchsorted(_E4M3_POS, a, side="left")          # first code with value >= a
    hi = np.clip(hi, 0, 126)
    lo = np.clip(hi - 1, 0, 126)
    d_lo = a - _E4M3_POS[lo]
    d_hi = _E4M3_POS[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo)
    code = np.where(a >= E4M3_MAX, 126, code)                 # satfinite
    code = np.where(a == 0.0, 0, code)
    out = code.astype(np.uint8) | np.where(np.signbit(x), 0x80, 0).astype(np.uint8)
    return np.where(np.isnan(x), np.uint8(0x7F), out).astype(np.uint8)


# ----------------------------------------------------------------------------------------------
# YaRN RoPE table (RoPE coefficients page, precompute excerpt; helper bodies omitted there)
# ----------------------------------------------------------------------------------------------
def yarn_correction_dim(num_rotations: float, dim: int = ROPE_DIM, base: float = ROPE_THETA,
                        max_pos: int = ORIGINAL_SEQ_LEN) -> float:
    """READING: dimension index whose wavelength makes ``num_rotations`` turns over the original
    context (the YaRN paper's correction dimension), dim*ln(L/(2*pi*r)) / (2*ln(base))."""
    return dim * math.log(max_pos / (num_rotations * 2 * math.pi)) / (2 * math.log(base))


def yarn_correction_range(beta_fast=BETA_FAST, beta_slow=BETA_SLOW, dim=ROPE_DIM, base=ROPE_THETA,
                          max_pos=ORIGINAL_SEQ_LEN):
    low = math.floor(yarn_correction_dim(beta_fast, dim, base, max_pos))
    high = math.ceil(yarn_correction_dim(beta_slow, dim, base, max_pos))
    return max(low, 0), min(high, dim - 1)


def yarn_linear_ramp(low: float, high: float, n: int) -> np.ndarray:
    """READING: 0 below ``low``, 1 above ``high``, linear in between (high==low nudged by 1e-3)."""
    if low == high:
        high += 0.001
    return np.clip((np.arange(n, dtype=np.float64) - low) / (high - low), 0.0, 1.0)


def yarn_inv_freq() -> np.ndarray:
    """The 32 rotary frequencies after the YaRN blend, float64.

    base frequencies theta^(-2i/64); because max_seq_len (16384) exceeds the original 4096 the
    blend freqs/factor*(1-smooth) + freqs*smooth with smooth = 1 - ramp(low, high) is always on.
    """
    i = np.arange(0, ROPE_DIM, 2, dtype=np.float64)
    freqs = 1.0 / (ROPE_THETA ** (i / ROPE_DIM))
    if MAX_SEQ_LEN > ORIGINAL_SEQ_LEN:
        low, high = yarn_correction_range()
        smooth = 1.0 - yarn_linear_ramp(low, high, ROPE_PAIRS)
        freqs = freqs / ROPE_FACTOR * (1.0 - smooth) + freqs * smooth
    return freqs


def rope_table(max_pos: int = MAX_SEQ_LEN) -> np.ndarray:
    """(cos, sin) per position and pair, fp32 [max_pos, 32, 2].

    The page builds freqs in float32 and the angle as a float32 outer product t*freq; the
    angle is rounded to fp32 here the same way, cos/sin are evaluated in float64 and rounded.
    """
    f32 = yarn_inv_freq().astype(np.float32)
    ang = (np.arange(max_pos, dtype=np.float32)[:, None] * f32[None, :]).astype(np.float32)
    a64 = ang.astype(np.float64)
    return np.stack([np.cos(a64), np.sin(a64)], axis=-1).astype(np.float32)


def rope_noninterleaved(x, pos, table) -> np.ndarray:
    """Rotate the first 64 features, pairing feature j with j+32 (apply_rotary_emb with
    interleaved=False, as Indexer.forward calls it); features 64.. are returned unchanged.

    x [..., D] (D >= 64), pos broadcastable to x.shape[:-1]; float64 out.
    """
    x = np.asarray(x, dtype=np.float64)
    cs = np.asarray(table, dtype=np.float64)[np.asarray(pos)]     # [..., 32, 2]
    c, s = cs[..., 0], cs[..., 1]
    a = x[..., :ROPE_PAIRS]                  # real parts: features 0..31
    b = x[..., ROPE_PAIRS:ROPE_DIM]          # imaginary parts: features 32..63
    y = x.copy()
    y[..., :ROPE_PAIRS] = a * c - b * s
    y[..., ROPE_PAIRS:ROPE_DIM] = a * s + b * c
    return y


def hadamard_matrix(n: int = D_I) -> np.ndarray:
    """Sylvester Hadamard matrix in natural order, H[i,j] = (-1)^popcount(i & j)."""
    idx = np.arange(n)
    bits = np.bitwise_and(idx[:, None], idx[None, :])
    pop = np.zeros_like(bits)
    while np.any(bits):
        pop += bits & 1
        bits >>= 1
    return np.where(pop % 2 == 0, 1.0, -1.0)


def hadamard_rotate(x) -> np.ndarray:
    """x (1/sqrt 128) H_128 along the last axis (dense-block page, indexer steps), float64."""
    x = np.asarray(x, dtype=np.float64)
    n = x.shape[-1]
    return x @ hadamard_matrix(n) / math.sqrt(n)


def act_quant(x):
    """Block FP8 quantisation with one scale per 128-element block (news page: 128-element
    blocks; Indexer.forward act_quant calls).

    READING: scale = fp32(amax / 448) with amax guarded below by 1e-4; code = RNE-satfinite
    e4m3 of the IEEE fp32 quotient x/scale. x is fp32 [..., 128]; returns (uint8 codes,
    fp32 scales [...]).
    """
    x = np.asarray(x, dtype=np.float32)
    amax = np.max(np.abs(x), axis=-1)
    amax = np.maximum(amax, np.float32(1e-4)).astype(np.float32)
    scale = (amax / np.float32(E4M3_MAX)).astype(np.float32)
    q = (x / scale[..., None]).astype(np.float32)
    return e4m3_encode(q), scale


def index_keys_prequant(x, pos, table, hadamard: bool = True) -> np.ndarray:
    """The fp32 rows act_quant receives in index_keys (RoPE_64, optional Hadamard, rounded to fp32)."""
    y = rope_noninterleaved(x, pos, table)
    if hadamard:
        y = hadamard_rotate(y)
    return y.astype(np.float32)


def index_keys(x, pos, table, hadamard: bool = True):
    """Indexer q or k transform of Indexer.forward up to act_quant.

    x fp32 [..., 128] (one head row per block), pos broadcastable to x.shape[:-1].
    RoPE_64 (non-interleaved) then, if ``hadamard``, (1/sqrt 128) H_128, both in float64;
    READING: the rotated row is rounded to fp32 (the activation dtype) before act_quant.
    """
    return act_quant(index_keys_prequant(x, pos, table, hadamard))


# ----------------------------------------------------------------------------------------------
# Indexer scores (fp8_index) and top-k
# ----------------------------------------------------------------------------------------------
def valid_len(q_pos, kv_len) -> np.ndarray:
    """Keys visible to each query: s <= q_pos (causal mask) and s < kv_len; [B, T]."""
    q_pos = np.asarray(q_pos, dtype=np.int64)
    kv_len = np.asarray(kv_len, dtype=np.int64)
    return np.clip(np.minimum(q_pos + 1, kv_len[:, None]), 0, None)


def index_scores(q8, q_scale, w, k8, k_scale, q_pos, kv_len,
                 softmax_scale: float = INDEXER_SOFTMAX_SCALE) -> np.ndarray:
    """I[b,t,s] = k_scale[b,s] * sum_j w'[b,t,j] * ReLU(sum_i q8[b,t,j,i] k8[b,s,i]) for visible s,
    -inf elsewhere, with w' = w * H_I^-0.5 * q_scale * softmax_scale.

    The fold follows Indexer.forward (weights * n_heads**-0.5, then * q_scale * softmax_scale);
    READING: k_scale multiplies outside the ReLU (exact, since k_scale > 0). The code-domain dot
    products are exact in float64 (each product of two e4m3 values is a multiple of 2^-18 below
    2^18, so a 128-term sum needs < 53 bits) and so may come from a matmul.
    q8 [B,T,H,128] u8, q_scale [B,T,H], w [B,T,H], k8 [B,S,128] u8, k_scale [B,S].
    """
    q = e4m3_decode(q8)
    k = e4m3_decode(k8)
    B, T, H, _ = q.shape
    S = k.shape[1]
    wf = (np.asarray(w, np.float64) * (H ** -0.5) * np.asarray(q_scale, np.float64)
          * float(softmax_scale))                                   # [B,T,H]
    out = np.full((B, T, S), -np.inf)
    nv = valid_len(q_pos, kv_len)
    ks = np.asarray(k_scale, np.float64)
    for b in range(B):
        for t0 in range(0, T, 64):        # query rows in groups, only to bound memory
            t1 = min(T, t0 + 64)
            n = t1 - t0
            dots = (q[b, t0:t1].reshape(n * H, -1) @ k[b].T).reshape(n, H, S)   # exact
            relu = np.maximum(dots, 0.0)
            score = np.einsum("th,ths->ts", wf[b, t0:t1], relu) * ks[b][None, :]
            for t in range(t0, t1):
                out[b, t, :nv[b, t]] = score[t - t0, :nv[b, t]]
    return out


def index_score_magnitude(q8, q_scale, w, k8, k_scale, q_pos, kv_len,
                          softmax_scale: float = INDEXER_SOFTMAX_SCALE) -> np.ndarray:
    """M[b,t,s] = k_scale * sum_j |w'_j| * ReLU(dot_j): the scale against which an fp32
    accumulation's error is measured (sums of mixed-sign w' can cancel to near 0)."""
    q = e4m3_decode(q8)
    k = e4m3_decode(k8)
    B, T, H, _ = q.shape
    wf = np.abs(np.asarray(w, np.float64) * (H ** -0.5) * np.asarray(q_scale, np.float64)
                * float(softmax_scale))
    out = np.zeros((B, T, k.shape[1]))
    ks = np.asarray(k_scale, np.float64)
    for b in range(B):
        for t0 in range(0, T, 64):
            t1 = min(T, t0 + 64)
            n = t1 - t0
            relu = np.maximum((q[b, t0:t1].reshape(n * H, -1) @ k[b].T).reshape(n, H, -1), 0.0)
            out[b, t0:t1] = np.einsum("th,ths->ts", wf[b, t0:t1], relu) * ks[b][None, :]
    return out


def topk_indices(scores, q_pos, kv_len, k: int, sorted_by_score: bool = False) -> np.ndarray:
    """Per query, the min(k, n_valid) visible positions with the largest scores
    (index_score.topk(min(index_topk, end_pos)) after the causal mask).

    READING: equal scores go to the smaller position; the selected positions are written in
    ascending order (or, with sorted_by_score, in the order of the stable sort by descending
    score), followed by -1 padding. int32 [B, T, k].
    """
    scores = np.asarray(scores)
    B, T, _ = scores.shape
    nv = valid_len(q_pos, kv_len)
    out = np.full((B, T, k), -1, dtype=np.int32)
    for b in range(B):
        for t in range(T):
            n = int(nv[b, t])
            if n == 0:
                continue
            row = scores[b, t, :n]
            order = np.lexsort((np.arange(n), -row))     # by score desc, then position asc
            sel = order[:min(k, n)] if sorted_by_score else np.sort(order[:min(k, n)])
            out[b, t, :sel.size] = sel
    return out


# ----------------------------------------------------------------------------------------------
# Sparse MLA in the absorbed (MQA) form
# ----------------------------------------------------------------------------------------------
def bf16_to_f64(bits) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def sparse_mla(q_bits, kv_bits, idx, softmax_scale: float = MLA_SOFTMAX_SCALE, d_v: int = 512):
    """For each (b, t, head): z_u = scale * q . kv[idx_u] over all 576 features, softmax over the
    selected u (entries -1 are not selected), o = sum_u p_u kv[idx_u][:512] (similarities page, MQA
    decode: latent and rotary score terms, index mask, softmax, latent-weighted sum).

    q_bits bf16 [B,T,H,Dqk], kv_bits bf16 [B,S,Dqk], idx int32 [B,T,K].
    Returns (out float64 [B,T,H,d_v], lse float64 [B,T,H]); a row with no selection gives 0, -inf.
    """
    q = bf16_to_f64(q_bits)
    kv = bf16_to_f64(kv_bits)
    B, T, H, _ = q.shape
    out = np.zeros((B, T, H, d_v))
    lse = np.full((B, T, H), -np.inf)
    idx = np.asarray(idx)
    for b in range(B):
        for t in range(T):
            sel = idx[b, t][idx[b, t] >= 0]
            if sel.size == 0:
                continue
            rows = kv[b, sel]                                  # [K, Dqk]
            z = (q[b, t] @ rows.T) * softmax_scale             # [H, K]
            m = z.max(axis=1, keepdims=True)
            e = np.exp(z - m)
            l = e.sum(axis=1, keepdims=True)
            out[b, t] = (e / l) @ rows[:, :d_v]
            lse[b, t] = (m + np.log(l))[:, 0]
    return out, lse


def dense_mla(q_bits, kv_bits, q_pos, kv_len, softmax_scale: float = MLA_SOFTMAX_SCALE, d_v: int = 512):
    """Masked dense softmax attention over every visible key (the MLA prefill excerpt with the
    index mask removed, written in the absorbed form): the k >= context limit of sparse_mla."""
    B, T = np.asarray(q_pos).shape
    nv = valid_len(q_pos, kv_len)
    K = int(nv.max()) if nv.size else 0
    idx = np.full((B, T, max(K, 1)), -1, dtype=np.int32)
    for b in range(B):
        for t in range(T):
            idx[b, t, :nv[b, t]] = np.arange(nv[b, t])
    return sparse_mla(q_bits, kv_bits, idx, softmax_scale, d_v)


# ----------------------------------------------------------------------------------------------
# Producers of the sparse-MLA inputs and the output absorption (absorbed MQA form)
# ----------------------------------------------------------------------------------------------
def rope_interleaved(x, pos, table) -> np.ndarray:
    """Rotate feature pairs (2i, 2i+1) by pair i's angle: apply_rotary_emb with interleaved=True,
    the layout the MLA uses for q_pe and k_pe (Rotate first features page: attention pairs 2j with
    2j+1, the indexer j with j+32). x [..., 64], pos broadcastable to x.shape[:-1]; float64 out.

    READING: the excerpt widens the bf16 input to fp32 and multiplies complex64 numbers; the
    oracle rotates in float64 (the difference is far below the bf16 rounding of the result).
    """
    x = np.asarray(x, dtype=np.float64)
    cs = np.asarray(table, dtype=np.float64)[np.asarray(pos)]     # [..., 32, 2]
    c, s = cs[..., 0], cs[..., 1]
    re, im = x[..., 0::2], x[..., 1::2]
    y = np.empty_like(x)
    y[..., 0::2] = re * c - im * s
    y[..., 1::2] = re * s + im * c
    return y


def mla_q_absorb(q_nope_bits, q_pe_bits, pos, table, w_uk_bits) -> np.ndarray:
    """The sparse-MLA query [rows, H, 576]: features 0..511 are q_nope absorbed into the latent
    space, q[t,h,c] = sum_d q_nope[t,h,d] w_uk[h,d,c] (the MQA-decode excerpt's einsum of q_nope
    with wkv_b[:, :qk_nope_head_dim]); features 512..575 are q_pe rotated at pos[t] (interleaved).

    q_nope_bits bf16 [rows, H, 128], q_pe_bits bf16 [rows, H, 64], pos [rows],
    w_uk_bits bf16 [H, 128, 512]. float64 out (the CUDA path rounds it to bf16).
    """
    qn = bf16_to_f64(q_nope_bits)
    w = bf16_to_f64(w_uk_bits)
    lat = np.einsum("thd,hdc->thc", qn, w)
    rot = rope_interleaved(bf16_to_f64(q_pe_bits), np.asarray(pos)[:, None], table)
    return np.concatenate([lat, rot], axis=-1)


def mla_kv_entry(kv_bits, k_pe_bits, pos, table) -> np.ndarray:
    """One latent-cache row per token [rows, 576]: the (normalised) latent kv unchanged, then k_pe
    rotated at pos (interleaved) -- the rows the MQA-decode excerpt reads from kv_cache and
    pe_cache, kept side by side. float64 out."""
    return np.concatenate([bf16_to_f64(kv_bits),
                           rope_interleaved(bf16_to_f64(k_pe_bits), np.asarray(pos), table)], axis=-1)


def mla_out_absorb(o_bits, w_uv_bits) -> np.ndarray:
    """Per-head value up-projection of the attention output, x[t,h,d] = sum_c o[t,h,c] w_uv[h,d,c]
    (the excerpt's final einsum with wkv_b[:, -v_head_dim:]). o_bits bf16 [rows, H, 512],
    w_uv_bits bf16 [H, 128, 512]; float64 [rows, H, 128] out."""
    return np.einsum("thc,hdc->thd", bf16_to_f64(o_bits), bf16_to_f64(w_uv_bits))


def gemm_abs_terms(a, b, spec: str) -> np.ndarray:
    """sum over the contracted index of |a * b| for an einsum spec: the scale an fp32
    accumulation's rounding error is measured against."""
    return np.einsum(spec, np.abs(np.asarray(a, np.float64)), np.abs(np.asarray(b, np.float64)))


def paged_gather(pool, block_table, page_size: int, seq_len) -> np.ndarray:
    """Dense per-sequence view [B, max_pages * page_size, ...] of a paged cache.

    The pages say nothing of paging. READING: the block-table layout of paged KV caches in
    serving systems -- sequence b's position s is pool row
    block_table[b, s // page_size] * page_size + s % page_size. Positions at or past seq_len[b]
    are not read (their table entries may be anything) and come out zero; a position below it
    whose page id is outside the pool is an error.
    """
    pool = np.asarray(pool)
    block_table = np.asarray(block_table)
    B, max_pages = block_table.shape
    num_pages = pool.shape[0] // page_size
    out = np.zeros((B, max_pages * page_size) + pool.shape[1:], dtype=pool.dtype)
    for b in range(B):
        for s in range(int(np.asarray(seq_len).reshape(B)[b])):
            page = int(block_table[b, s // page_size])
            if not 0 <= page < num_pages:
                raise IndexError(f"sequence {b} position {s}: page id {page} outside the pool")
            out[b, s] = pool[page * page_size + s % page_size]
    return out
