"""Comparison rules shared by the GPU parity tests (CUDA path vs the CPU oracle).

Tolerances (written here once, used by every test):
* e4m3 codes: bit-exact, except an element whose oracle quotient y/scale lies within
  CODE_TOL of an e4m3 rounding midpoint (relative to the block's 2-norm / scale); those may land
  one code step away. The kernel's fp32 RoPE + 7-stage fp32 butterfly differs from the oracle's
  float64 rotation by at most ~8 ulp of the row norm, far inside 2^-15.
* block scales: within 2^-15 relative (amax may differ by a few fp32 ulp for the same reason).
* index scores: |I_gpu - I_ref| <= 1e-3 * max(|I_ref|, M) with M = k_scale * sum_j |w'_j| ReLU(dot_j)
  (the relative 1e-3 bar, measured against the magnitude of the terms that were summed, since
  mixed-sign head weights can cancel a score to near 0).
* top-k: bit-exact on identical fp32 inputs; against oracle scores (on identical quantised inputs)
  only positions whose score lies within twice the score tolerance of the k-th largest may differ
  (the derivation is in check_topk_near_ties).
* sparse MLA: 2e-2 absolute on the bf16 outputs; lse 1e-3 absolute.
"""
import numpy as np
import torch

from oracle import dsa_oracle as O

CODE_TOL = 2.0 ** -15
SCALE_RTOL = 2.0 ** -15
SCORE_RTOL = 1e-3
MLA_ATOL = 2e-2
LSE_ATOL = 1e-3

_VALS = O.e4m3_decode(np.arange(127, dtype=np.uint8))
_MIDS = (_VALS[1:] + _VALS[:-1]) / 2


def to_dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype) if t.element_size() == torch.empty((), dtype=dtype).element_size() else t.to(dtype)
    return t.cuda()


def bf16_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits)).view(torch.bfloat16).cuda()


def check_codes(codes_gpu, scales_gpu, x, pos, table, hadamard=True):
    """Returns the number of tolerated boundary mismatches; asserts everything else."""
    y = O.index_keys_prequant(x, pos, table, hadamard)
    codes, scales = O.act_quant(y)
    sg = np.asarray(scales_gpu, np.float64)
    so = scales.astype(np.float64)
    assert np.all(np.abs(sg - so) <= SCALE_RTOL * so), np.max(np.abs(sg - so) / so)
    cg = np.asarray(codes_gpu, np.uint8)
    diff = cg != codes
    # +0 and -0 codes are the same value
    diff &= ~(((cg & 0x7F) == 0) & ((codes & 0x7F) == 0))
    if not diff.any():
        return 0
    v = np.abs(y.astype(np.float64) / so[..., None])
    norm = np.linalg.norm(y.astype(np.float64), axis=-1) / so
    tol = CODE_TOL * np.broadcast_to(norm[..., None], v.shape) + v * SCALE_RTOL
    j = np.clip(np.searchsorted(_MIDS, v), 1, len(_MIDS) - 1)
    dist = np.minimum(np.abs(v - _MIDS[j - 1]), np.abs(_MIDS[j] - v))
    near = dist <= tol
    step = np.abs((cg & 0x7F).astype(int) - (codes & 0x7F).astype(int))
    same_sign = ((cg ^ codes) & 0x80) == 0
    ok = near & (step <= 1) & (same_sign | ((cg & 0x7F) == 0) | ((codes & 0x7F) == 0))
    bad = diff & ~ok
    assert not bad.any(), f"{bad.sum()} code mismatches away from a rounding boundary"
    assert diff.mean() < 1e-3
    return int(diff.sum())


def check_scores(gpu, ref, mag, nvalid):
    """gpu/ref/mag: [T, S] rows of one sequence; nvalid: [T] visible counts."""
    for t in range(ref.shape[0]):
        n = int(nvalid[t])
        g = np.asarray(gpu[t, :n], np.float64)
        r = ref[t, :n]
        m = mag[t, :n]
        err = np.abs(g - r)
        lim = SCORE_RTOL * np.maximum(np.abs(r), m) + 1e-30
        assert np.all(err <= lim), f"row {t}: worst {np.max(err / lim):.3g} x tolerance"


def check_topk_near_ties(idx_gpu, idx_ref, scores_ref, mag_ref, k):
    """Selected sets may differ only at near-ties.

    Both selections come from scores that agree within the score tolerance tol_x =
    SCORE_RTOL * max(|I_x|, M_x) (check_scores). If the GPU keeps x and drops y where the oracle
    keeps y and drops x, then I_ref(x) + tol_x >= I_gpu(x) >= I_gpu(y) >= I_ref(y) - tol_y, and the
    oracle's k-th score theta lies between I_ref(x) and I_ref(y). The two sets have equal sizes,
    so every element of their symmetric difference D pairs with one on the other side, and
    |I_ref(x) - theta| <= 2 * max_{j in D} tol_j for every x in D. That bound, and nothing looser,
    is what is checked: the sets are equal except at scores that tie within the tolerance."""
    for r in range(idx_ref.shape[0]):
        a = set(int(i) for i in idx_gpu[r] if i >= 0)
        b = set(int(i) for i in idx_ref[r] if i >= 0)
        assert len(a) == len(b), (r, len(a), len(b))
        if a == b:
            continue
        row, mag = scores_ref[r], mag_ref[r]
        theta = min(row[i] for i in b)
        d = a ^ b
        tol_d = max(SCORE_RTOL * max(abs(row[i]), mag[i]) for i in d)
        for i in d:
            assert abs(row[i] - theta) <= 2.0 * tol_d, (r, i, row[i], theta, tol_d)
