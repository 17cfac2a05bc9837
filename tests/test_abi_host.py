"""Host-side checks of the C-ABI library that need no GPU: every symbol the header declares is
exported, arguments are rejected before any launch, and the library's own RoPE table agrees with
the oracle's (the two are written independently)."""
import ctypes
import os
import re
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dsa.h")


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"DSA_API\s+[\w\s\*]+?\b(dsa_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def L():
    import __graft_entry__
    __graft_entry__._build_module().build()
    import sparse_attention_keys_b200 as m
    return m.lib


def test_header_declares_the_path():
    names = _declared()
    for n in ("dsa_index_keys", "dsa_index_scores", "dsa_topk", "dsa_sparse_mla", "dsa_rope_table",
              "dsa_get_device_status", "dsa_status_string", "dsa_sparse_mla_workspace_size"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    nm = subprocess.run(["nm", "-D", "--defined-only", L._name], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(dsa_\w+)", nm))
    missing = [n for n in _declared() if n not in exported]
    assert not missing, missing
    for n in _declared():
        assert hasattr(L, n)


def test_status_strings(L):
    import sparse_attention_keys_b200 as m
    assert m.dsa_status_string(0) == "DSA_OK"
    assert m.dsa_status_string(1) == "DSA_ERR_INVALID_ARG"
    assert m.dsa_status_string(5) == "DSA_ERR_DEVICE_BOUNDS"
    assert m.dsa_status_string(99) == "DSA_ERR_UNKNOWN"
    assert m.dsa_version().startswith("dsa-b200")


def test_invalid_arguments_rejected_before_launch(L):
    """These calls fail validation on the host; no device is touched (none exists here)."""
    p = ctypes.c_void_p(16)          # non-null, aligned dummy; never dereferenced
    bad = ctypes.c_void_p(17)        # misaligned
    n = None
    assert L.dsa_index_keys(p, 0, 4, 0, p, p, 10, 1, p, p, n, n) == 1           # heads < 1
    assert L.dsa_index_keys(p, 0, 4, 1, p, p, 10, 8, p, p, n, n) == 1           # unknown flag
    assert L.dsa_index_keys(p, 2, 4, 1, p, p, 10, 1, p, p, n, n) == 1           # unknown input type
    assert L.dsa_index_keys(bad, 0, 4, 1, p, p, 10, 1, p, p, n, n) == 1         # misaligned x
    assert L.dsa_index_keys(n, 1, 4, 1, p, p, 10, 1, p, p, n, n) == 1           # null x
    assert L.dsa_index_keys(p, 0, 0, 1, p, p, 10, 1, p, p, n, n) == 0           # empty: nothing to do
    # dsa_index_qk: (kx, k_rows, k_pos, k_dst_row, k_fp8, k_scale, qx, q_rows, q_heads, q_pos, q_fp8, q_scale,
    #                x_dtype, rope_cs, max_pos, flags, stream), the checks of dsa_index_keys on each side
    qk = [p, 4, p, n, p, p, p, 2, 64, p, p, p, 0, p, 10, 1, n]
    a = list(qk); a[8] = 0; assert L.dsa_index_qk(*a) == 1                    # query heads < 1
    a = list(qk); a[15] = 8; assert L.dsa_index_qk(*a) == 1                   # unknown flag
    a = list(qk); a[12] = 2; assert L.dsa_index_qk(*a) == 1                   # unknown input type
    a = list(qk); a[3] = bad; assert L.dsa_index_qk(*a) == 1                  # misaligned k_dst_row
    a = list(qk); a[6] = n; assert L.dsa_index_qk(*a) == 1                    # null qx with query rows
    a = list(qk); a[1] = -1; assert L.dsa_index_qk(*a) == 1                   # negative key rows
    a = list(qk); a[14] = 0; assert L.dsa_index_qk(*a) == 1                   # max_pos < 1
    a = list(qk); a[1] = 0; a[7] = 0; assert L.dsa_index_qk(*a) == 0          # both sides empty
    f = ctypes.c_float
    args = [p, p, p, p, p, p, p, 1, 1, 128, f(0.088), p, 128, 0, n]
    a = list(args); a[12] = 126; assert L.dsa_index_scores(*a) == 1          # ld not a multiple of 4
    a = list(args); a[12] = 64; assert L.dsa_index_scores(*a) == 1           # ld < S_max
    a = list(args); a[10] = f(0.0); assert L.dsa_index_scores(*a) == 1       # scale <= 0
    a = list(args); a[13] = 4; assert L.dsa_index_scores(*a) == 1            # unknown flag
    a = list(args); a[3] = bad; assert L.dsa_index_scores(*a) == 1          # misaligned k8
    assert L.dsa_topk(p, 130, p, p, 1, 1, 8, 0, p, n) == 1                   # ld % 4
    assert L.dsa_topk(p, 128, p, p, 1, 1, 0, 0, p, n) == 1                   # k < 1
    assert L.dsa_topk(p, 128, p, p, 0, 1, 8, 0, p, n) == 1                   # B < 1
    assert L.dsa_topk(p, 128, p, p, 1, 1, 8, 8, p, n) == 1                   # unknown flag
    assert L.dsa_topk(p, 128, p, p, 1, 1, 4097, 4, p, n) == 1                # DSA_SORTED with k > 4096
    assert L.dsa_sparse_mla(p, p, p, 1, 1, 16, 0, f(0.1), p, n, n, 0, n) == 1  # k < 1
    assert L.dsa_sparse_mla(p, p, p, 1, 1, 16, 4, f(-1.0), p, n, n, 0, n) == 1
    assert L.dsa_sparse_mla(p, bad, p, 1, 1, 16, 4, f(0.1), p, n, n, 0, n) == 1
    # paged calls: (..., num_pages, block_table, max_pages, page_size, ...)
    sargs = [p, p, p, p, p, 8, p, 4, 64, p, p, 1, 1, f(0.088), p, 256, 0, n]
    a = list(sargs); a[8] = 32; assert L.dsa_index_scores_paged(*a) == 1    # page_size < 64
    a = list(sargs); a[8] = 96; assert L.dsa_index_scores_paged(*a) == 1    # page_size not a power of two
    a = list(sargs); a[8] = 192; assert L.dsa_index_scores_paged(*a) == 1   # page_size not a power of two
    a = list(sargs); a[5] = 0; assert L.dsa_index_scores_paged(*a) == 1     # empty pool
    a = list(sargs); a[7] = 0; assert L.dsa_index_scores_paged(*a) == 1     # max_pages < 1
    a = list(sargs); a[6] = n; assert L.dsa_index_scores_paged(*a) == 1     # null block table
    a = list(sargs); a[6] = ctypes.c_void_p(18); assert L.dsa_index_scores_paged(*a) == 1   # table not int32-aligned
    a = list(sargs); a[15] = 128; assert L.dsa_index_scores_paged(*a) == 1  # ld < max_pages * page_size
    a = list(sargs); a[5] = 1 << 26; assert L.dsa_index_scores_paged(*a) == 1   # pool rows past int32
    a = list(sargs); a[3] = bad; assert L.dsa_index_scores_paged(*a) == 1   # misaligned pool
    margs = [p, p, 8, p, 4, 64, p, 1, 1, 16, f(0.1), p, n, n, 0, n]
    a = list(margs); a[5] = 100; assert L.dsa_sparse_mla_paged(*a) == 1     # page_size
    a = list(margs); a[3] = n; assert L.dsa_sparse_mla_paged(*a) == 1       # null block table
    a = list(margs); a[9] = 0; assert L.dsa_sparse_mla_paged(*a) == 1       # k < 1
    a = list(margs); a[1] = bad; assert L.dsa_sparse_mla_paged(*a) == 1     # misaligned pool
    # MLA producers: (q_nope, q_pe, pos, rope_cs, max_pos, w, w_head_stride, rows, q_out, stream)
    ws = 256 * 512
    assert L.dsa_mla_q_absorb(p, p, p, p, 16, p, ws, 0, p, n) == 0            # no rows: nothing to do
    assert L.dsa_mla_q_absorb(p, p, p, p, 16, p, 1000, 4, p, n) == 1         # head stride < 128*512
    assert L.dsa_mla_q_absorb(p, p, p, p, 16, p, ws + 4, 4, p, n) == 1       # head stride not 16-byte
    assert L.dsa_mla_q_absorb(p, p, p, p, 0, p, ws, 4, p, n) == 1            # empty table
    assert L.dsa_mla_q_absorb(p, p, p, p, 16, bad, ws, 4, p, n) == 1         # misaligned weights
    assert L.dsa_mla_q_absorb(p, p, p, p, 16, p, ws, -1, p, n) == 1          # negative rows
    assert L.dsa_mla_out_absorb(p, p, ws, 1 << 31, p, n) == 1                # rows past int32
    assert L.dsa_mla_out_absorb(p, n, ws, 4, p, n) == 1                      # null weights
    assert L.dsa_mla_kv_entry(p, p, p, p, 16, 4, p, p, 0, n) == 1            # empty cache
    assert L.dsa_mla_kv_entry(p, p, p, p, 16, 4, bad, p, 8, n) == 1          # misaligned dst_row
    assert L.dsa_rope_table(n, 10) == 1
    assert L.dsa_rope_table(p, 0) == 1


def test_library_rope_table_matches_oracle(L):
    from oracle import dsa_oracle as O
    import sparse_attention_keys_b200 as m
    mine = m.dsa_rope_table(16384).numpy()
    ref = O.rope_table(16384)
    assert mine.shape == ref.shape
    diff = np.abs(mine.view(np.int32).astype(np.int64) - ref.view(np.int32).astype(np.int64))
    # both round cos/sin of the same fp32 angle from double; libm and numpy may differ by an ulp
    assert diff.max() <= 1
    assert (diff > 0).mean() < 1e-3


def test_binding_fails_loudly_without_library(tmp_path):
    """Importing the binding with no built library raises; there is no fallback path."""
    pkg = tmp_path / "sparse_attention_keys_b200"
    pkg.mkdir()
    src = open(os.path.join(ROOT, "sparse_attention_keys_b200", "__init__.py")).read()
    (pkg / "__init__.py").write_text(src)
    r = subprocess.run([sys.executable, "-c", "import sparse_attention_keys_b200"], cwd=tmp_path,
                       capture_output=True, text=True)
    assert r.returncode != 0 and "libdsa.so not built" in r.stderr


def test_site_names_match_header(L):
    """The binding's wait-site table carries exactly the DSA_SITE_* codes the header defines."""
    import sparse_attention_keys_b200 as m
    codes = {int(v, 16) for v in re.findall(r"#define DSA_SITE_\w+ (0x[0-9a-fA-F]+)", open(HEADER).read())}
    assert codes == set(m.SITE_NAMES)
