"""Seeded synthetic inputs for the DeepSeek Sparse Attention hot path.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic (no RoPE, no Hadamard, no quantisation, no scores). Both the
CPU oracle (tests only) and the CUDA path read the arrays it returns, so the
two sides always start from identical bytes.

Workload shapes follow the pages' model configuration
(DeepSeek-V3.2-Exp, "Lightning indexer" and "Sparse attention" steps on the
dense-block page; Indexer.forward on the index-keys page; the MQA decode
excerpt on the similarities page): 64 indexer heads of 128 features, 128 MLA
heads over a 512-d latent plus a 64-d rotary key, top-2048 selection.

Draw order is fixed: indexer q, indexer k, indexer weights, MLA q, MLA kv,
then per-workload extras. Everything comes from numpy's PCG64
(``numpy.random.default_rng(seed)``).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

H_I = 64          # indexer heads
D_I = 128         # indexer head dim (one FP8 block)
H_MLA = 128       # MLA heads
D_LATENT = 512    # kv_lora_rank
D_ROPE = 64       # qk_rope_head_dim
D_QK = D_LATENT + D_ROPE
MAX_SEQ_LEN = 16384


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    queries: int          # T: queries per sequence in this step
    s_max: int            # cache length per sequence
    topk: int
    decode: bool          # one query per sequence at the end of its context
    kv_len_range: tuple | None = None   # decode: context length drawn per sequence (inclusive)
    hot_key_frac: float = 0.0           # fraction of key rows scaled by hot_key_gain
    hot_key_gain: float = 8.0
    with_mla: bool = True
    note: str = ""


WORKLOADS = {
    "tiny_decode": Workload("tiny_decode", batch=1, queries=1, s_max=1024, topk=256, decode=True,
                            kv_len_range=(1024, 1024),
                            note="1 query at position 1023, context 1024, top-256"),
    "decode_b8": Workload("decode_b8", batch=8, queries=1, s_max=4096, topk=2048, decode=True,
                          kv_len_range=(2048, 4096),
                          note="8 sequences, 1 query each, context ~U[2048,4096], top-2048"),
    "prefill_4096": Workload("prefill_4096", batch=1, queries=4096, s_max=4096, topk=2048, decode=False,
                             note="4096 causal queries x 4096 keys, top-2048"),
    "prefill_16384": Workload("prefill_16384", batch=1, queries=16384, s_max=16384, topk=2048, decode=False,
                              hot_key_frac=0.01, with_mla=False,
                              note="16384 causal queries, 1% of key rows x8, no MLA"),
    "decode_b64": Workload("decode_b64", batch=64, queries=1, s_max=16384, topk=2048, decode=True,
                           kv_len_range=(16384, 16384),
                           note="64 sequences, 1 query each at context 16384, top-2048"),
}


def bf16_bits_from_f32(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bfloat16 (nearest, ties to even) and return the raw uint16 bits.

    This is storage-format conversion of the synthetic draw, not method arithmetic.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    rounding_bias = ((u >> 16) & np.uint32(1)) + np.uint32(0x7FFF)   # finite inputs: no overflow
    return ((u + rounding_bias) >> 16).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


@dataclass
class Inputs:
    workload: Workload
    idx_q: np.ndarray                # fp32 [B, T, 64, 128]   raw indexer queries (before RoPE)
    idx_k: np.ndarray                # fp32 [B, S_max, 128]   raw indexer keys for every cache row
    idx_w: np.ndarray                # fp32 [B, T, 64]        raw per-head weights
    q_pos: np.ndarray                # int32 [B, T]           absolute position of each query
    kv_len: np.ndarray               # int32 [B]              keys present per sequence
    mla_q: np.ndarray | None = None  # bf16 bits [B, T, 128, 576]
    mla_kv: np.ndarray | None = None # bf16 bits [B, S_max, 576]
    hot_rows: np.ndarray | None = None
    extra: dict = field(default_factory=dict)


def _normal_f32(rng: np.random.Generator, shape) -> np.ndarray:
    return rng.standard_normal(size=shape, dtype=np.float32)


def make_inputs(name_or_wl, seed: int = 0, with_mla: bool | None = None) -> Inputs:
    """Draw one workload's inputs.

    ``with_mla`` (default: the workload's own choice) skips the sparse-MLA draws;
    skipping them changes no other array because they come after q, k and w.
    """
    wl = WORKLOADS[name_or_wl] if isinstance(name_or_wl, str) else name_or_wl
    if with_mla is None:
        with_mla = wl.with_mla
    rng = np.random.default_rng(seed)
    B, T, S = wl.batch, wl.queries, wl.s_max
    q = _normal_f32(rng, (B, T, H_I, D_I))
    k = _normal_f32(rng, (B, S, D_I))
    w = _normal_f32(rng, (B, T, H_I))
    mla_q = mla_kv = None
    if with_mla:
        mla_q = bf16_bits_from_f32(_normal_f32(rng, (B, T, H_MLA, D_QK)))
        kv = np.empty((B, S, D_QK), dtype=np.uint16)
        for b in range(B):  # per sequence keeps the fp32 temporary small at 64 x 16384 x 576
            kv[b] = bf16_bits_from_f32(_normal_f32(rng, (S, D_QK)))
        mla_kv = kv
    # extras, drawn after the tensors above
    hot_rows = None
    if wl.decode:
        lo, hi = wl.kv_len_range
        if lo == hi:
            kv_len = np.full(B, lo, dtype=np.int32)
        else:
            kv_len = rng.integers(lo, hi, endpoint=True, size=B).astype(np.int32)
        q_pos = (kv_len - 1).astype(np.int32).reshape(B, 1)
    else:
        kv_len = np.full(B, S, dtype=np.int32)
        q_pos = np.broadcast_to(np.arange(T, dtype=np.int32), (B, T)).copy()
    if wl.hot_key_frac > 0:
        n_hot = int(round(wl.hot_key_frac * S))
        hot_rows = np.sort(rng.choice(S, n_hot, replace=False))
        k[:, hot_rows, :] *= np.float32(wl.hot_key_gain)
    return Inputs(wl, q, k, w, q_pos, kv_len, mla_q, mla_kv, hot_rows)


def filler_e4m3(shape, seed: int):
    """Seeded e4m3 codes and fp32 block scales for rows no test checks (full-size launches where
    only sampled rows are compared). Uses torch's fp32 -> float8_e4m3fn cast as a data source."""
    import torch
    g = torch.Generator().manual_seed(seed)
    v = (torch.randn(shape, generator=g) * 100.0).clamp_(-448.0, 448.0)
    codes = v.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    scales = (0.005 + 0.015 * torch.rand(shape[:-1], generator=g)).numpy().astype(np.float32)
    return codes, scales


def make_custom(batch: int, queries: int, s_max: int, topk: int, *, decode: bool, seed: int = 0,
                kv_len=None, q_pos=None, with_mla: bool = True, scale_rows=None) -> Inputs:
    """Small ad-hoc shapes for parity tests (ragged tails, empty rows, tiny contexts).

    ``kv_len``/``q_pos`` override the positions; ``scale_rows`` maps key row -> gain.
    """
    wl = Workload(f"custom_{batch}x{queries}x{s_max}", batch, queries, s_max, topk, decode,
                  kv_len_range=(s_max, s_max) if decode else None, with_mla=with_mla)
    inp = make_inputs(wl, seed=seed)
    if kv_len is not None:
        inp.kv_len = np.asarray(kv_len, dtype=np.int32).reshape(batch)
        if decode and q_pos is None:
            inp.q_pos = (inp.kv_len - 1).astype(np.int32).reshape(batch, 1)
    if q_pos is not None:
        inp.q_pos = np.asarray(q_pos, dtype=np.int32).reshape(batch, queries)
    if scale_rows:
        for r, g in scale_rows.items():
            inp.idx_k[:, r, :] *= np.float32(g)
    return inp


def paged_layout(batch: int, max_pages: int, page_size: int, seed: int, spare_pages: int = 3,
                 kv_len=None, past_end=-1):
    """A seeded block table for a paged cache: each (sequence, page) gets its own pool page, in
    shuffled order, with ``spare_pages`` pool pages that no sequence uses. With ``kv_len``, the
    entries of pages wholly past a sequence's length are set to ``past_end`` (they must not be
    read). Returns (block_table int32 [batch, max_pages], num_pages)."""
    rng = np.random.default_rng(seed)
    num_pages = batch * max_pages + spare_pages
    table = rng.permutation(num_pages)[:batch * max_pages].astype(np.int32).reshape(batch, max_pages)
    if kv_len is not None:
        for b, n in enumerate(np.asarray(kv_len).reshape(batch)):
            table[b, (int(n) + page_size - 1) // page_size:] = past_end
    return table, num_pages


def to_paged(dense: np.ndarray, block_table: np.ndarray, page_size: int, num_pages: int, fill) -> np.ndarray:
    """Lay a per-sequence cache dense [B, S, ...] (S = max_pages * page_size) out in a pool
    [num_pages * page_size, ...] through block_table; rows of pages no entry names hold ``fill``."""
    B, S = dense.shape[:2]
    pool = np.full((num_pages * page_size,) + dense.shape[2:], fill, dtype=dense.dtype)
    for b in range(B):
        for pg in range(S // page_size):
            dst = int(block_table[b, pg])
            if 0 <= dst < num_pages:
                pool[dst * page_size:(dst + 1) * page_size] = dense[b, pg * page_size:(pg + 1) * page_size]
    return pool


@dataclass
class MlaProducerInputs:
    """Inputs of the MLA producers and output absorption for ``rows`` tokens (bf16 bit patterns)."""
    q_nope: np.ndarray    # [rows, 128, 128]
    q_pe: np.ndarray      # [rows, 128, 64]
    kv: np.ndarray        # [rows, 512]  (the normalised latent)
    k_pe: np.ndarray      # [rows, 64]
    o: np.ndarray         # [rows, 128, 512]  (a sparse-MLA output)
    wkv_b: np.ndarray     # [128, 256, 512]: rows 0..127 of each head are w_uk, 128..255 w_uv
    pos: np.ndarray       # int32 [rows]


def make_mla_producer_inputs(rows: int, seed: int = 0, max_pos: int = MAX_SEQ_LEN) -> MlaProducerInputs:
    """N(0,1) activations, wkv_b ~ N(0, 1/512) (unit-scale outputs), positions uniform in [0, max_pos).
    Draw order: q_nope, q_pe, kv, k_pe, o, wkv_b, pos."""
    rng = np.random.default_rng(seed)
    q_nope = bf16_bits_from_f32(_normal_f32(rng, (rows, H_MLA, 128)))
    q_pe = bf16_bits_from_f32(_normal_f32(rng, (rows, H_MLA, D_ROPE)))
    kv = bf16_bits_from_f32(_normal_f32(rng, (rows, D_LATENT)))
    k_pe = bf16_bits_from_f32(_normal_f32(rng, (rows, D_ROPE)))
    o = bf16_bits_from_f32(_normal_f32(rng, (rows, H_MLA, D_LATENT)))
    wkv_b = bf16_bits_from_f32(_normal_f32(rng, (H_MLA, 256, D_LATENT)) * np.float32(D_LATENT ** -0.5))
    pos = rng.integers(0, max_pos, size=rows).astype(np.int32)
    return MlaProducerInputs(q_nope, q_pe, kv, k_pe, o, wkv_b, pos)
