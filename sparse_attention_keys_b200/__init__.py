"""Python binding of libdsa, the sm_100a hot path of DeepSeek Sparse Attention.

Thin ctypes marshalling over the C ABI declared in include/dsa.h: every function takes torch
tensors (device memory owned by the caller, or allocated here with torch.empty as plumbing),
passes raw pointers and sizes, and raises DsaError on a non-zero status. All arithmetic runs in
the library's CUDA kernels; there is no fallback path. Names follow the C entry points.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "DsaError", "lib", "lib_path", "DSA_HADAMARD", "DSA_FILL_MASKED", "DSA_SORTED", "DSA_Q_READY", "DSA_F32", "DSA_BF16", "INDEXER_SOFTMAX_SCALE",
    "MLA_SOFTMAX_SCALE", "dsa_rope_table", "dsa_index_keys", "dsa_index_qk", "dsa_index_scores", "dsa_topk",
    "dsa_index_topk", "dsa_sparse_mla", "dsa_sparse_mla_workspace_size", "dsa_sparse_mla_noalloc", "dsa_sparse_mla_heads",
    "dsa_sparse_mla_heads_workspace_size",
    "dsa_index_scores_paged", "dsa_sparse_mla_paged", "dsa_mla_q_absorb", "dsa_mla_kv_entry",
    "dsa_mla_out_absorb",
    "dsa_sparse_mla_noalloc_scratch_bytes", "dsa_get_device_status", "dsa_get_error_detail",
    "dsa_selftest_wait_timeout", "dsa_status_string", "dsa_device_supported", "dsa_version",
    "SITE_NAMES",
]

DSA_OK = 0
DSA_HADAMARD = 0x1
DSA_FILL_MASKED = 0x2
DSA_SORTED = 0x4
DSA_Q_READY = 0x8
DSA_F32 = 0
DSA_BF16 = 1
MAX_POS = 16384                 # max_seq_len of the model (ModelArgs)
INDEXER_SOFTMAX_SCALE = 128 ** -0.5
MLA_SOFTMAX_SCALE = 192 ** -0.5 * (1.0 + 0.1 * __import__("math").log(40.0)) ** 2

# wait-site codes recorded with DSA_ERR_TIMEOUT (DSA_SITE_* in include/dsa.h)
SITE_NAMES = {
    0x11: "scores:q", 0x12: "scores:k_full", 0x13: "scores:k_empty", 0x14: "scores:acc_full",
    0x15: "scores:acc_empty", 0x21: "mla:q", 0x22: "mla:kv_full", 0x23: "mla:kv_empty",
    0x24: "mla:s_full", 0x25: "mla:p_full", 0x26: "mla:p_empty", 0x27: "mla:o_full",
    0x31: "selftest", 0x41: "absorb:w", 0x42: "absorb:a_full", 0x43: "absorb:a_empty",
    0x44: "absorb:acc_full", 0x45: "absorb:acc_empty",
}

_HERE = os.path.dirname(os.path.abspath(__file__))
lib_path = os.path.join(_HERE, "libdsa.so")


class DsaError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {dsa_status_string(code) if _lib is not None else code}")


def _load():
    if not os.path.exists(lib_path):
        raise ImportError(f"libdsa.so not built at {lib_path}; run `python -m sparse_attention_keys_b200.build`")
    L = ctypes.CDLL(lib_path)
    vp, i32, i64, u32, f32, sz = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_uint32,
                                  ctypes.c_float, ctypes.c_size_t)
    L.dsa_rope_table.argtypes = [vp, i32]
    L.dsa_index_keys.argtypes = [vp, i32, i64, i32, vp, vp, i32, u32, vp, vp, vp, vp]
    L.dsa_index_qk.argtypes = [vp, i64, vp, vp, vp, vp, vp, i64, i32, vp, vp, vp, i32, vp, i32, u32, vp]
    L.dsa_index_scores.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, f32, vp, i64, u32, vp]
    L.dsa_topk.argtypes = [vp, i64, vp, vp, i32, i32, i32, u32, vp, vp]
    L.dsa_index_topk.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, f32, i32, u32, vp, vp]
    L.dsa_sparse_mla.argtypes = [vp, vp, vp, i32, i32, i32, i32, f32, vp, vp, vp, sz, vp]
    L.dsa_sparse_mla_ex.argtypes = [vp, vp, vp, i32, i32, i32, i32, f32, vp, vp, vp, sz, u32, vp]
    L.dsa_sparse_mla_workspace_size.argtypes = [i32, i32, i32]
    L.dsa_sparse_mla_heads.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, f32, vp, vp, vp, sz, vp]
    L.dsa_sparse_mla_heads_workspace_size.argtypes = [i32, i32, i32, i32]
    L.dsa_sparse_mla_heads_workspace_size.restype = sz
    L.dsa_index_scores_paged.argtypes = [vp, vp, vp, vp, vp, i64, vp, i32, i32, vp, vp, i32, i32, f32, vp, i64, u32,
                                         vp]
    L.dsa_sparse_mla_paged.argtypes = [vp, vp, i64, vp, i32, i32, vp, i32, i32, i32, f32, vp, vp, vp, sz, vp]
    L.dsa_mla_q_absorb.argtypes = [vp, vp, vp, vp, i32, vp, i64, i64, vp, vp]
    L.dsa_mla_kv_entry.argtypes = [vp, vp, vp, vp, i32, i64, vp, vp, i64, vp]
    L.dsa_mla_out_absorb.argtypes = [vp, vp, i64, i64, vp, vp]
    L.dsa_sparse_mla_workspace_size.restype = sz
    L.dsa_sparse_mla_noalloc.argtypes = [vp, vp, vp, i32, i32, i32, i32, f32, vp, vp, vp]
    L.dsa_sparse_mla_noalloc_scratch_bytes.argtypes = []
    L.dsa_sparse_mla_noalloc_scratch_bytes.restype = sz
    L.dsa_get_device_status.argtypes = [vp]
    L.dsa_get_error_detail.argtypes = [vp, vp, vp]
    L.dsa_selftest_wait_timeout.argtypes = [vp]
    L.dsa_status_string.argtypes = [i32]
    L.dsa_status_string.restype = ctypes.c_char_p
    L.dsa_device_supported.argtypes = []
    L.dsa_version.restype = ctypes.c_char_p
    for f in ("dsa_rope_table", "dsa_index_keys", "dsa_index_qk", "dsa_index_scores", "dsa_topk", "dsa_index_topk", "dsa_sparse_mla",
              "dsa_sparse_mla_ex",
              "dsa_sparse_mla_heads",
              "dsa_sparse_mla_noalloc", "dsa_get_device_status", "dsa_get_error_detail",
              "dsa_selftest_wait_timeout", "dsa_device_supported"):
        getattr(L, f).restype = ctypes.c_int
    return L


_lib = _load()
lib = _lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(rc: int, what: str):
    if rc != DSA_OK:
        raise DsaError(rc, what)


def _need(t, dtype, name, device=True):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if device and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")


def dsa_status_string(code: int) -> str:
    return _lib.dsa_status_string(int(code)).decode()


def dsa_version() -> str:
    return _lib.dsa_version().decode()


def dsa_device_supported() -> bool:
    return bool(_lib.dsa_device_supported())


def dsa_rope_table(max_pos: int = MAX_POS) -> torch.Tensor:
    """(cos, sin) YaRN table, fp32 [max_pos, 32, 2], in HOST memory (computed by the library)."""
    out = torch.empty((max_pos, 32, 2), dtype=torch.float32)
    _check(_lib.dsa_rope_table(_ptr(out), int(max_pos)), "dsa_rope_table")
    return out


def dsa_index_keys(x, pos, rope_cs, flags: int = DSA_HADAMARD, out_fp8=None, out_scale=None,
                   dst_row=None, stream=None):
    """x fp32 or bf16 [rows, heads, 128] (or [rows, 128] for keys) -> (codes uint8, scales fp32).

    With dst_row (int64 [rows]) the outputs are written into the given cache tensors at those rows.
    """
    if x.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("x must be float32 or bfloat16")
    _need(x, x.dtype, "x")
    _need(pos, torch.int32, "pos")
    _need(rope_cs, torch.float32, "rope_cs")
    if x.shape[-1] != 128:
        raise ValueError("last dim of x must be 128")
    rows = x.shape[0]
    heads = 1 if x.dim() == 2 else int(x[0].numel() // 128)
    if pos.numel() != rows:
        raise ValueError("pos must have one entry per row of x")
    if dst_row is None:
        if out_fp8 is None:
            out_fp8 = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
        if out_scale is None:
            out_scale = torch.empty(x.shape[:-1], dtype=torch.float32, device=x.device)
    else:
        _need(dst_row, torch.int64, "dst_row")
        if out_fp8 is None or out_scale is None:
            raise ValueError("dst_row needs the destination out_fp8 and out_scale tensors")
    _need(out_fp8, torch.uint8, "out_fp8")
    _need(out_scale, torch.float32, "out_scale")
    x_dtype = DSA_BF16 if x.dtype == torch.bfloat16 else DSA_F32
    rc = _lib.dsa_index_keys(_ptr(x), x_dtype, rows, heads, _ptr(pos), _ptr(rope_cs), rope_cs.shape[0], int(flags),
                             _ptr(out_fp8), _ptr(out_scale), _ptr(dst_row), _stream(stream))
    _check(rc, "dsa_index_keys")
    return out_fp8, out_scale


def dsa_index_qk(kx, k_pos, qx, q_pos, rope_cs, k_out_fp8, k_out_scale, k_dst_row=None, q_out_fp8=None,
                 q_out_scale=None, flags: int = DSA_HADAMARD, stream=None):
    """The new keys kx [k_rows, 128] and the queries qx [q_rows, heads, 128] (one dtype, fp32 or
    bf16) through dsa_index_keys in one launch. The key codes and scales go to k_out_fp8 /
    k_out_scale (at the rows k_dst_row names, or densely when it is None); returns the query
    (codes, scales)."""
    if kx.dtype not in (torch.float32, torch.bfloat16) or qx.dtype != kx.dtype:
        raise TypeError("kx and qx must be both float32 or both bfloat16")
    for t, dt, n in ((kx, kx.dtype, "kx"), (qx, qx.dtype, "qx"), (k_pos, torch.int32, "k_pos"),
                     (q_pos, torch.int32, "q_pos"), (rope_cs, torch.float32, "rope_cs"),
                     (k_out_fp8, torch.uint8, "k_out_fp8"), (k_out_scale, torch.float32, "k_out_scale")):
        _need(t, dt, n)
    if kx.dim() != 2 or kx.shape[-1] != 128 or qx.dim() != 3 or qx.shape[-1] != 128:
        raise ValueError("kx must be [rows, 128] and qx [rows, heads, 128]")
    if k_pos.numel() != kx.shape[0] or q_pos.numel() != qx.shape[0]:
        raise ValueError("k_pos and q_pos must have one entry per row")
    if k_dst_row is not None:
        _need(k_dst_row, torch.int64, "k_dst_row")
        if k_dst_row.numel() != kx.shape[0]:
            raise ValueError("k_dst_row must have one entry per key row")
    elif k_out_fp8.numel() < kx.numel() or k_out_scale.numel() < kx.shape[0]:
        raise ValueError("dense key outputs are smaller than kx")
    if q_out_fp8 is None:
        q_out_fp8 = torch.empty(qx.shape, dtype=torch.uint8, device=qx.device)
    if q_out_scale is None:
        q_out_scale = torch.empty(qx.shape[:-1], dtype=torch.float32, device=qx.device)
    _need(q_out_fp8, torch.uint8, "q_out_fp8")
    _need(q_out_scale, torch.float32, "q_out_scale")
    if q_out_fp8.numel() < qx.numel() or q_out_scale.numel() < qx.numel() // 128:
        raise ValueError("query outputs are smaller than qx")
    devs = {t.device for t in (kx, qx, k_pos, q_pos, rope_cs, k_out_fp8, k_out_scale, q_out_fp8, q_out_scale)}
    if len(devs) != 1:
        raise ValueError("all tensors must be on one device")
    x_dtype = DSA_BF16 if kx.dtype == torch.bfloat16 else DSA_F32
    rc = _lib.dsa_index_qk(_ptr(kx), kx.shape[0], _ptr(k_pos), _ptr(k_dst_row), _ptr(k_out_fp8), _ptr(k_out_scale),
                           _ptr(qx), qx.shape[0], qx.shape[1], _ptr(q_pos), _ptr(q_out_fp8), _ptr(q_out_scale),
                           x_dtype, _ptr(rope_cs), rope_cs.shape[0], int(flags), _stream(stream))
    _check(rc, "dsa_index_qk")
    return q_out_fp8, q_out_scale


def dsa_index_scores(q8, q_scale, w, k8, k_scale, q_pos, kv_len, softmax_scale: float = INDEXER_SOFTMAX_SCALE,
                     scores=None, ld=None, flags: int = 0, stream=None):
    """q8 [B,T,64,128] u8, q_scale/w [B,T,64] f32, k8 [B,S,128] u8, k_scale [B,S] f32,
    q_pos [B,T] i32, kv_len [B] i32 -> scores fp32 [B,T,ld]."""
    for t, dt, n in ((q8, torch.uint8, "q8"), (q_scale, torch.float32, "q_scale"), (w, torch.float32, "w"),
                     (k8, torch.uint8, "k8"), (k_scale, torch.float32, "k_scale"), (q_pos, torch.int32, "q_pos"),
                     (kv_len, torch.int32, "kv_len")):
        _need(t, dt, n)
    B, T = q8.shape[0], q8.shape[1]
    S = k8.shape[1]
    if ld is None:
        ld = (S + 3) // 4 * 4
    if scores is None:
        scores = torch.empty((B, T, ld), dtype=torch.float32, device=q8.device)
    _need(scores, torch.float32, "scores")
    rc = _lib.dsa_index_scores(_ptr(q8), _ptr(q_scale), _ptr(w), _ptr(k8), _ptr(k_scale), _ptr(q_pos),
                               _ptr(kv_len), B, T, S, float(softmax_scale), _ptr(scores), int(ld), int(flags),
                               _stream(stream))
    _check(rc, "dsa_index_scores")
    return scores


def dsa_index_topk(q8, q_scale, w, k8, k_scale, q_pos, kv_len, k: int,
                   softmax_scale: float = INDEXER_SOFTMAX_SCALE, idx=None, stream=None):
    """The decode indexer fused with its top-k: the same idx int32 [B,T,k] as
    dsa_topk(dsa_index_scores(...), q_pos, kv_len, k), in one launch and with no scores buffer.
    Inputs as dsa_index_scores (dense K-cache, S <= 32768)."""
    for t, dt, n in ((q8, torch.uint8, "q8"), (q_scale, torch.float32, "q_scale"), (w, torch.float32, "w"),
                     (k8, torch.uint8, "k8"), (k_scale, torch.float32, "k_scale"), (q_pos, torch.int32, "q_pos"),
                     (kv_len, torch.int32, "kv_len")):
        _need(t, dt, n)
    B, T = q8.shape[0], q8.shape[1]
    S = k8.shape[1]
    if tuple(q8.shape[2:]) != (64, 128) or tuple(q_scale.shape) != (B, T, 64) or tuple(w.shape) != (B, T, 64):
        raise ValueError("q8 must be [B, T, 64, 128] with q_scale and w [B, T, 64]")
    if k8.dim() != 3 or k8.shape[0] != B or k8.shape[2] != 128 or tuple(k_scale.shape) != (B, S):
        raise ValueError("k8 must be [B, S, 128] with k_scale [B, S]")
    if tuple(q_pos.shape) != (B, T) or tuple(kv_len.shape) != (B,):
        raise ValueError("q_pos must be [B, T] and kv_len [B]")
    if idx is None:
        idx = torch.empty((B, T, int(k)), dtype=torch.int32, device=q8.device)
    _need(idx, torch.int32, "idx")
    if tuple(idx.shape) != (B, T, int(k)):
        raise ValueError(f"idx must be [{B}, {T}, {int(k)}]")
    for t, n in ((q_scale, "q_scale"), (w, "w"), (k8, "k8"), (k_scale, "k_scale"), (q_pos, "q_pos"),
                 (kv_len, "kv_len"), (idx, "idx")):
        if t.device != q8.device:
            raise ValueError(f"{n} is on {t.device}, q8 on {q8.device}: all tensors must be on one device")
    rc = _lib.dsa_index_topk(_ptr(q8), _ptr(q_scale), _ptr(w), _ptr(k8), _ptr(k_scale), _ptr(q_pos), _ptr(kv_len),
                             B, T, S, float(softmax_scale), int(k), 0, _ptr(idx), _stream(stream))
    _check(rc, "dsa_index_topk")
    return idx


def dsa_index_scores_paged(q8, q_scale, w, k8_pool, k_scale_pool, block_table, page_size: int, q_pos, kv_len,
                           softmax_scale: float = INDEXER_SOFTMAX_SCALE, scores=None, ld=None, flags: int = 0,
                           stream=None):
    """dsa_index_scores over a paged K-cache: k8_pool u8 [num_pages*page_size,128], k_scale_pool f32
    [num_pages*page_size], block_table i32 [B,max_pages] -> scores fp32 [B,T,ld], ld >= max_pages*page_size."""
    for t, dt, n in ((q8, torch.uint8, "q8"), (q_scale, torch.float32, "q_scale"), (w, torch.float32, "w"),
                     (k8_pool, torch.uint8, "k8_pool"), (k_scale_pool, torch.float32, "k_scale_pool"),
                     (block_table, torch.int32, "block_table"), (q_pos, torch.int32, "q_pos"),
                     (kv_len, torch.int32, "kv_len")):
        _need(t, dt, n)
    B, T = q8.shape[0], q8.shape[1]
    max_pages = block_table.shape[1]
    num_pages = k8_pool.shape[0] // int(page_size)
    S = max_pages * int(page_size)
    if ld is None:
        ld = S
    if scores is None:
        scores = torch.empty((B, T, ld), dtype=torch.float32, device=q8.device)
    _need(scores, torch.float32, "scores")
    rc = _lib.dsa_index_scores_paged(_ptr(q8), _ptr(q_scale), _ptr(w), _ptr(k8_pool), _ptr(k_scale_pool), num_pages,
                                     _ptr(block_table), max_pages, int(page_size), _ptr(q_pos), _ptr(kv_len), B, T,
                                     float(softmax_scale), _ptr(scores), int(ld), int(flags), _stream(stream))
    _check(rc, "dsa_index_scores_paged")
    return scores


def dsa_topk(scores, q_pos, kv_len, k: int, idx=None, flags: int = 0, stream=None):
    """scores fp32 [B,T,ld] -> idx int32 [B,T,k] (ascending positions, or by descending score with
    flags=DSA_SORTED; -1 padded)."""
    _need(scores, torch.float32, "scores")
    _need(q_pos, torch.int32, "q_pos")
    _need(kv_len, torch.int32, "kv_len")
    B, T, ld = scores.shape
    if idx is None:
        idx = torch.empty((B, T, k), dtype=torch.int32, device=scores.device)
    _need(idx, torch.int32, "idx")
    rc = _lib.dsa_topk(_ptr(scores), int(ld), _ptr(q_pos), _ptr(kv_len), B, T, int(k), int(flags), _ptr(idx),
                       _stream(stream))
    _check(rc, "dsa_topk")
    return idx


def _mla_shapes(q, kv, idx, out, lse, kv_name="kv", heads=128):
    """Shape and device checks of the sparse-MLA arguments (before any pointer reaches the library,
    so a mismatched buffer raises here instead of being written out of bounds):
    q [B,T,H,576], kv [...,576], idx [B,T,k], out [B,T,H,512], lse [B,T,H] or None (H = heads)."""
    if q.dim() != 4 or tuple(q.shape[2:]) != (heads, 576):
        raise ValueError(f"q must be [B, T, {heads}, 576], got {tuple(q.shape)}")
    B, T = int(q.shape[0]), int(q.shape[1])
    if kv.shape[-1] != 576:
        raise ValueError(f"{kv_name} rows must have 576 features, got {tuple(kv.shape)}")
    if idx.dim() != 3 or tuple(idx.shape[:2]) != (B, T) or idx.shape[2] < 1:
        raise ValueError(f"idx must be [B={B}, T={T}, k>=1], got {tuple(idx.shape)}")
    if out is not None and tuple(out.shape) != (B, T, heads, 512):
        raise ValueError(f"out must be [{B}, {T}, {heads}, 512], got {tuple(out.shape)}")
    if lse is not None and tuple(lse.shape) != (B, T, heads):
        raise ValueError(f"lse must be [{B}, {T}, {heads}], got {tuple(lse.shape)}")
    for t, n in ((kv, kv_name), (idx, "idx"), (out, "out"), (lse, "lse")):
        if t is not None and t.device != q.device:
            raise ValueError(f"{n} is on {t.device}, q on {q.device}: all tensors must be on one device")
    return B, T, int(idx.shape[2])


def dsa_sparse_mla_workspace_size(B: int, T: int, k: int) -> int:
    return int(_lib.dsa_sparse_mla_workspace_size(int(B), int(T), int(k)))


def dsa_sparse_mla(q, kv, idx, softmax_scale: float = MLA_SOFTMAX_SCALE, out=None, lse=None, workspace=None,
                   want_lse: bool = True, flags: int = 0, stream=None):
    """q bf16 [B,T,128,576], kv bf16 [B,S,576], idx int32 [B,T,k] -> (out bf16 [B,T,128,512], lse fp32).
    flags = DSA_Q_READY when q is complete before the call (not written by the kernel right before)."""
    _need(q, torch.bfloat16, "q")
    _need(kv, torch.bfloat16, "kv")
    _need(idx, torch.int32, "idx")
    if out is not None:
        _need(out, torch.bfloat16, "out")
    if lse is not None:
        _need(lse, torch.float32, "lse")
    if kv.dim() != 3 or kv.shape[0] != q.shape[0]:
        raise ValueError(f"kv must be [B, S_max, 576], got {tuple(kv.shape)}")
    B, T, k = _mla_shapes(q, kv, idx, out, lse)
    S = kv.shape[1]
    if out is None:
        out = torch.empty((B, T, 128, 512), dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, T, 128), dtype=torch.float32, device=q.device)
    ws_bytes = dsa_sparse_mla_workspace_size(B, T, k)
    if workspace is not None:
        _need(workspace, workspace.dtype, "workspace")
        if workspace.device != q.device:
            raise ValueError("workspace must be on q's device")
    if workspace is None and ws_bytes > 0:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    ws_len = 0 if workspace is None else workspace.numel() * workspace.element_size()
    if flags:
        rc = _lib.dsa_sparse_mla_ex(_ptr(q), _ptr(kv), _ptr(idx), B, T, S, int(k), float(softmax_scale), _ptr(out),
                                    _ptr(lse), _ptr(workspace), ws_len, int(flags), _stream(stream))
    else:
        rc = _lib.dsa_sparse_mla(_ptr(q), _ptr(kv), _ptr(idx), B, T, S, int(k), float(softmax_scale), _ptr(out),
                                 _ptr(lse), _ptr(workspace), ws_len, _stream(stream))
    _check(rc, "dsa_sparse_mla")
    return out, lse


def dsa_sparse_mla_heads_workspace_size(B: int, T: int, k: int, heads: int) -> int:
    return int(_lib.dsa_sparse_mla_heads_workspace_size(int(B), int(T), int(k), int(heads)))


def dsa_sparse_mla_heads(q, kv, idx, softmax_scale: float = MLA_SOFTMAX_SCALE, out=None, lse=None, workspace=None,
                         want_lse: bool = True, stream=None):
    """dsa_sparse_mla over a head shard: q bf16 [B,T,H,576] with H = 64 (half of the heads, as one
    rank of a two-way head split holds) or 128 -> (out bf16 [B,T,H,512], lse fp32 [B,T,H])."""
    _need(q, torch.bfloat16, "q")
    _need(kv, torch.bfloat16, "kv")
    _need(idx, torch.int32, "idx")
    if out is not None:
        _need(out, torch.bfloat16, "out")
    if lse is not None:
        _need(lse, torch.float32, "lse")
    heads = int(q.shape[2]) if q.dim() == 4 else -1
    if heads not in (64, 128):
        raise ValueError(f"q must hold 64 or 128 heads, got {tuple(q.shape)}")
    if kv.dim() != 3 or kv.shape[0] != q.shape[0]:
        raise ValueError(f"kv must be [B, S_max, 576], got {tuple(kv.shape)}")
    B, T, k = _mla_shapes(q, kv, idx, out, lse, heads=heads)
    if out is None:
        out = torch.empty((B, T, heads, 512), dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, T, heads), dtype=torch.float32, device=q.device)
    ws_bytes = dsa_sparse_mla_heads_workspace_size(B, T, k, heads)
    if workspace is None and ws_bytes > 0:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    rc = _lib.dsa_sparse_mla_heads(_ptr(q), _ptr(kv), _ptr(idx), B, T, kv.shape[1], int(k), heads,
                                   float(softmax_scale), _ptr(out), _ptr(lse), _ptr(workspace),
                                   0 if workspace is None else workspace.numel() * workspace.element_size(),
                                   _stream(stream))
    _check(rc, "dsa_sparse_mla_heads")
    return out, lse


def dsa_sparse_mla_paged(q, kv_pool, block_table, page_size: int, idx, softmax_scale: float = MLA_SOFTMAX_SCALE,
                         out=None, lse=None, workspace=None, want_lse: bool = True, stream=None):
    """dsa_sparse_mla over a paged latent cache: kv_pool bf16 [num_pages*page_size,576], block_table
    i32 [B,max_pages]; idx holds logical positions -> (out bf16 [B,T,128,512], lse fp32)."""
    _need(q, torch.bfloat16, "q")
    _need(kv_pool, torch.bfloat16, "kv_pool")
    _need(block_table, torch.int32, "block_table")
    _need(idx, torch.int32, "idx")
    if out is not None:
        _need(out, torch.bfloat16, "out")
    if lse is not None:
        _need(lse, torch.float32, "lse")
    B, T, k = _mla_shapes(q, kv_pool, idx, out, lse, kv_name="kv_pool")
    if block_table.dim() != 2 or block_table.shape[0] != B or block_table.device != q.device:
        raise ValueError(f"block_table must be [B={B}, max_pages] on q's device, got {tuple(block_table.shape)}")
    max_pages = block_table.shape[1]
    num_pages = kv_pool.shape[0] // int(page_size)
    if out is None:
        out = torch.empty((B, T, 128, 512), dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, T, 128), dtype=torch.float32, device=q.device)
    ws_bytes = dsa_sparse_mla_workspace_size(B, T, k)
    if workspace is None and ws_bytes > 0:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    rc = _lib.dsa_sparse_mla_paged(_ptr(q), _ptr(kv_pool), num_pages, _ptr(block_table), max_pages, int(page_size),
                                   _ptr(idx), B, T, int(k), float(softmax_scale), _ptr(out), _ptr(lse),
                                   _ptr(workspace), 0 if workspace is None else workspace.numel() * workspace.element_size(),
                                   _stream(stream))
    _check(rc, "dsa_sparse_mla_paged")
    return out, lse


def _head_weights(w, name):
    """A [128 heads][128][512] bf16 view whose rows of 512 are contiguous (e.g. a slice of wkv_b
    viewed as [128][256][512]) -> (tensor, elements between heads)."""
    if not isinstance(w, torch.Tensor) or w.dtype != torch.bfloat16 or not w.is_cuda:
        raise TypeError(f"{name} must be a bfloat16 CUDA tensor")
    if tuple(w.shape) != (128, 128, 512) or w.stride(2) != 1 or w.stride(1) != 512:
        raise ValueError(f"{name} must be [128, 128, 512] with contiguous rows of 512")
    return w, int(w.stride(0))


def dsa_mla_q_absorb(q_nope, q_pe, pos, rope_cs, w_uk, q_out=None, stream=None):
    """q_nope bf16 [rows,128,128], q_pe bf16 [rows,128,64], pos i32 [rows], w_uk bf16 [128,128,512]
    (head, d, c) -> the sparse-MLA query bf16 [rows,128,576] (absorbed latent part | rotated q_pe)."""
    _need(q_nope, torch.bfloat16, "q_nope")
    _need(q_pe, torch.bfloat16, "q_pe")
    _need(pos, torch.int32, "pos")
    _need(rope_cs, torch.float32, "rope_cs")
    w, ws = _head_weights(w_uk, "w_uk")
    rows = q_nope.shape[0]
    if q_out is None:
        q_out = torch.empty((rows, 128, 576), dtype=torch.bfloat16, device=q_nope.device)
    _need(q_out, torch.bfloat16, "q_out")
    rc = _lib.dsa_mla_q_absorb(_ptr(q_nope), _ptr(q_pe), _ptr(pos), _ptr(rope_cs), rope_cs.shape[0], _ptr(w), ws,
                               rows, _ptr(q_out), _stream(stream))
    _check(rc, "dsa_mla_q_absorb")
    return q_out


def dsa_mla_kv_entry(kv, k_pe, pos, rope_cs, dst_row, kv_cache, stream=None):
    """Write latent-cache rows: kv_cache[dst_row[t]] = [kv[t] | interleaved RoPE of k_pe[t] at pos[t]].
    kv bf16 [rows,512], k_pe bf16 [rows,64], dst_row i64 [rows], kv_cache bf16 [..., 576]."""
    _need(kv, torch.bfloat16, "kv")
    _need(k_pe, torch.bfloat16, "k_pe")
    _need(pos, torch.int32, "pos")
    _need(rope_cs, torch.float32, "rope_cs")
    _need(dst_row, torch.int64, "dst_row")
    _need(kv_cache, torch.bfloat16, "kv_cache")
    rc = _lib.dsa_mla_kv_entry(_ptr(kv), _ptr(k_pe), _ptr(pos), _ptr(rope_cs), rope_cs.shape[0], kv.shape[0],
                               _ptr(dst_row), _ptr(kv_cache), kv_cache.numel() // 576, _stream(stream))
    _check(rc, "dsa_mla_kv_entry")
    return kv_cache


def dsa_mla_out_absorb(o, w_uv, out=None, stream=None):
    """o bf16 [rows,128,512] (sparse-MLA output), w_uv bf16 [128,128,512] (head, d, c) -> bf16 [rows,128,128]."""
    _need(o, torch.bfloat16, "o")
    w, ws = _head_weights(w_uv, "w_uv")
    rows = o.shape[0]
    if out is None:
        out = torch.empty((rows, 128, 128), dtype=torch.bfloat16, device=o.device)
    _need(out, torch.bfloat16, "out")
    rc = _lib.dsa_mla_out_absorb(_ptr(o), _ptr(w), ws, rows, _ptr(out), _stream(stream))
    _check(rc, "dsa_mla_out_absorb")
    return out


def dsa_sparse_mla_noalloc_scratch_bytes() -> int:
    return int(_lib.dsa_sparse_mla_noalloc_scratch_bytes())


def dsa_sparse_mla_noalloc(q, kv, idx, out, lse=None, softmax_scale: float = MLA_SOFTMAX_SCALE, stream=None):
    """dsa_sparse_mla for callers that cannot allocate device memory: the caller passes the
    output buffers (out bf16 [B,T,128,512], optional lse fp32 [B,T,128]) and the library takes
    its scratch from a fixed array of dsa_sparse_mla_noalloc_scratch_bytes(). Nothing is
    allocated here either. Calls that overlap on the GPU share that array: serialise them."""
    _need(q, torch.bfloat16, "q")
    _need(kv, torch.bfloat16, "kv")
    _need(idx, torch.int32, "idx")
    _need(out, torch.bfloat16, "out")
    if lse is not None:
        _need(lse, torch.float32, "lse")
    if kv.dim() != 3 or kv.shape[0] != q.shape[0]:
        raise ValueError(f"kv must be [B, S_max, 576], got {tuple(kv.shape)}")
    B, T, _ = _mla_shapes(q, kv, idx, out, lse)
    rc = _lib.dsa_sparse_mla_noalloc(_ptr(q), _ptr(kv), _ptr(idx), B, T, kv.shape[1], int(idx.shape[-1]),
                                     float(softmax_scale), _ptr(out), _ptr(lse), _stream(stream))
    _check(rc, "dsa_sparse_mla_noalloc")
    return out, lse


def dsa_get_device_status(stream=None) -> int:
    return int(_lib.dsa_get_device_status(_stream(stream)))


def dsa_get_error_detail() -> dict:
    """Detail of the last non-OK status read back: wait site, CTA index, wait length (us)."""
    site, block, wait_us = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int(0)
    _check(_lib.dsa_get_error_detail(ctypes.byref(site), ctypes.byref(block), ctypes.byref(wait_us)),
           "dsa_get_error_detail")
    return {"site": site.value, "site_name": SITE_NAMES.get(site.value, "none"), "block": block.value,
            "wait_us": wait_us.value}


def dsa_selftest_wait_timeout(stream=None) -> None:
    """Launch the bounded-wait self-test; the next dsa_get_device_status() reports the timeout."""
    _check(_lib.dsa_selftest_wait_timeout(_stream(stream)), "dsa_selftest_wait_timeout")
