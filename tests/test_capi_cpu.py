"""The C-ABI library on a machine without a GPU: it loads, exports every symbol the header declares,
its structs match the binding, and host-side validation rejects bad arguments before any launch."""
import ctypes
import os
import re
import subprocess

import pytest

import compressed_sparse_kv_overlapped_b200 as csa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "csa.h")


def header_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*([a-z_0-9]+)\s*\(", src, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(csa.LIB_PATH):
        csa.build()
    return csa.lib()


def test_exports_every_declared_function(lib):
    names = header_functions()
    assert set(names) >= {"csa_compress", "csa_index_topk", "csa_sparse_attn", "hca_dense_attn",
                          "hybrid_attn_decode", "hybrid_attn_prefill", "csa_workspace_size", "csa_last_error",
                          "csa_sync_status", "csa_version"}
    out = subprocess.run(["nm", "-D", "--defined-only", csa.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (\w+)$", out, flags=re.M))
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    assert set(csa.EXPORTS) <= exported


def test_struct_layouts_match_header(tmp_path):
    prog = tmp_path / "sizes.c"
    prog.write_text(
        '#include <stdio.h>\n#include <stddef.h>\n#include "csa.h"\n'
        "int main(void){printf(\"%zu %zu %zu %zu %zu %zu %zu %zu %zu %zu %zu %zu %zu %zu\\n\", sizeof(csa_dims), sizeof(csa_seq),"
        " sizeof(csa_query), sizeof(csa_ws_query), sizeof(csa_decode_args), sizeof(csa_prefill_args),"
        " offsetof(csa_decode_args, out), offsetof(csa_prefill_args, idx_out),"
        " offsetof(csa_decode_args, new_rows), offsetof(csa_decode_args, norms), offsetof(csa_prefill_args, norms),"
        " sizeof(csa_norms), offsetof(csa_decode_args, entries_q), offsetof(csa_decode_args, hca_scales));return 0;}\n")
    exe = tmp_path / "sizes"
    subprocess.run(["gcc", "-std=c11", "-I", os.path.join(ROOT, "include"), str(prog), "-o", str(exe)], check=True)
    got = [int(v) for v in subprocess.run([str(exe)], capture_output=True, text=True).stdout.split()]
    assert got == [ctypes.sizeof(csa.csa_dims), 32, 16, ctypes.sizeof(csa.csa_ws_query),
                   ctypes.sizeof(csa.csa_decode_args), ctypes.sizeof(csa.csa_prefill_args),
                   csa.csa_decode_args.out.offset, csa.csa_prefill_args.idx_out.offset,
                   csa.csa_decode_args.new_rows.offset, csa.csa_decode_args.norms.offset,
                   csa.csa_prefill_args.norms.offset, ctypes.sizeof(csa.csa_norms),
                   csa.csa_decode_args.entries_q.offset, csa.csa_decode_args.hca_scales.offset]


def test_version_and_error_string(lib):
    assert csa.csa_version() == 200
    assert isinstance(csa.csa_last_error(), str)


def test_host_validation_rejects_bad_arguments(lib):
    P = ctypes.POINTER
    dims = csa.make_dims()
    # NULL pointers
    rc = lib.csa_compress(ctypes.byref(dims), 0, None, None, 1, 10, None, None, None, None, None, None, None)
    assert rc == csa.CSA_ERR_ARG and "NULL" in csa.csa_last_error()
    # unsupported widths
    bad = csa.make_dims(d=256)
    rc = lib.csa_compress(ctypes.byref(bad), 0, 16, 16, 1, 10, 16, 16, 16, None, 16, None, None)
    assert rc == csa.CSA_ERR_UNSUPPORTED and "d = 256" in csa.csa_last_error()
    for kw in ({"k": 0}, {"k": 4096}, {"H": 65}, {"d_I": 48}, {"m": 3}, {"W": -1}):
        rc = lib.csa_compress(ctypes.byref(csa.make_dims(**kw)), 0, 16, 16, 1, 1, 16, 16, 16, None, 16, None, None)
        assert rc == csa.CSA_ERR_UNSUPPORTED, kw
    # misaligned tensor
    rc = lib.csa_compress(ctypes.byref(dims), 0, 16, 16, 1, 10, 18, 16, 16, None, 16, None, None)
    assert rc == csa.CSA_ERR_ARG and "aligned" in csa.csa_last_error()
    # HCA with indexer keys
    rc = lib.csa_compress(ctypes.byref(dims), 1, 16, 16, 1, 10, 16, 16, 16, 16, 16, 16, None)
    assert rc == csa.CSA_ERR_ARG
    # decode: too-small workspace
    a = csa.csa_decode_args()
    a.dims = dims
    a.B, a.max_len = 1, 4096
    for f in ("seqs", "x", "logit_c", "logit_h", "idx_key", "bias_c", "bias_h", "entries", "entry_keys",
              "hca_entries", "q", "q_idx", "w", "out"):
        setattr(a, f, 256)
    rc = lib.hybrid_attn_decode(ctypes.byref(a), 256, 16, None)
    assert rc == csa.CSA_ERR_ARG and "workspace" in csa.csa_last_error()
    # decode: appended rows handed over without an append, or misaligned
    a.append, a.new_rows = 0, 256
    rc = lib.hybrid_attn_decode(ctypes.byref(a), 256, 1 << 30, None)
    assert rc == csa.CSA_ERR_ARG and "new_rows without append" in csa.csa_last_error()
    a.append, a.new_rows = 1, 264
    rc = lib.hybrid_attn_decode(ctypes.byref(a), 256, 1 << 30, None)
    assert rc == csa.CSA_ERR_ARG and "aligned" in csa.csa_last_error()
    a.new_rows = None
    # decode: the FP4 entry caches come as a set of four, 16-byte aligned, for the block shapes
    a.entries_q = 256
    rc = lib.hybrid_attn_decode(ctypes.byref(a), 256, 1 << 30, None)
    assert rc == csa.CSA_ERR_ARG and "go together" in csa.csa_last_error()
    a.entry_scales, a.hca_q, a.hca_scales = 256, 264, 256
    rc = lib.hybrid_attn_decode(ctypes.byref(a), 256, 1 << 30, None)
    assert rc == csa.CSA_ERR_ARG and "aligned" in csa.csa_last_error()
    a.hca_q = 256
    a.dims = csa.make_dims(m=2)
    rc = lib.hybrid_attn_decode(ctypes.byref(a), 256, 1 << 30, None)
    assert rc == csa.CSA_ERR_UNSUPPORTED and "FP4" in csa.csa_last_error()
    a.dims = dims
    a.entries_q = a.entry_scales = a.hca_q = a.hca_scales = None
    # FP4 quantization and attention calls
    rc = lib.csa_quantize_entries(ctypes.byref(dims), 16, 16, 1, 10, 2, 16, 16, 16, None)
    assert rc == csa.CSA_ERR_ARG and "which" in csa.csa_last_error()
    rc = lib.csa_quantize_entries(ctypes.byref(dims), 16, 16, 1, 10, 0, 16, 24, 16, None)
    assert rc == csa.CSA_ERR_ARG and "aligned" in csa.csa_last_error()
    rc = lib.csa_quantize_entries(ctypes.byref(dims), 16, None, 1, 10, 0, 16, 16, 16, None)
    assert rc == csa.CSA_ERR_ARG and "NULL" in csa.csa_last_error()
    rc = lib.csa_sparse_attn_fp4(ctypes.byref(dims), 16, 16, 1, 16, 16, None, 16, 16, 0.1, 16, None, None, 0, None)
    assert rc == csa.CSA_ERR_ARG and "NULL" in csa.csa_last_error()
    rc = lib.hca_dense_attn_fp4(ctypes.byref(dims), 16, 16, 1, 100, 16, 24, 16, 16, 0, 0.1, 16, None, None, 0, None)
    assert rc == csa.CSA_ERR_ARG and "aligned" in csa.csa_last_error()
    # prefill: bad query range
    pa = csa.csa_prefill_args()
    pa.dims = dims
    pa.len, pa.q_begin, pa.q_end = 10, 5, 20
    rc = lib.hybrid_attn_prefill(ctypes.byref(pa), 256, 1 << 20, None)
    assert rc == csa.CSA_ERR_ARG and "query range" in csa.csa_last_error()


def test_compress_all_and_fault_injection_validation(lib):
    dims = csa.make_dims()
    P = [16] * 11
    rc = lib.csa_compress_all(ctypes.byref(dims), 16, None, 1, 10, *P[:9], None, None)
    assert rc == csa.CSA_ERR_ARG and "NULL" in csa.csa_last_error()
    rc = lib.csa_compress_all(ctypes.byref(dims), 16, 16, 1, 10, 16, 16, 16, 16, 24, 16, 16, 16, 16, None, None)
    assert rc == csa.CSA_ERR_ARG and "aligned" in csa.csa_last_error()
    rc = lib.csa_compress_all(ctypes.byref(dims), 16, 16, 0, 10, *P[:9], None, None)
    assert rc == csa.CSA_ERR_ARG
    assert lib.csa_compress_all(ctypes.byref(dims), 16, 16, 1, 0, *P[:9], None, None) == csa.CSA_OK  # nothing to do
    # normalization parameters
    n = csa.make_norms()
    n.reserved = 1
    rc = lib.csa_compress_all(ctypes.byref(dims), 16, 16, 1, 10, *P[:9], ctypes.byref(n), None)
    assert rc == csa.CSA_ERR_ARG and "reserved" in csa.csa_last_error()
    n.reserved, n.q_norm = 0, 24
    rc = lib.csa_compress_all(ctypes.byref(dims), 16, 16, 1, 10, *P[:9], ctypes.byref(n), None)
    assert rc == csa.CSA_ERR_ARG and "aligned" in csa.csa_last_error()
    n.q_norm, n.entry_norm_c = None, 16
    rc = lib.csa_compress_all(ctypes.byref(csa.make_dims(m=2)), 16, 16, 1, 10, *P[:9], ctypes.byref(n), None)
    assert rc == csa.CSA_ERR_UNSUPPORTED and "m = 4" in csa.csa_last_error()
    n.entry_norm_c, n.entry_norm_h = None, 16
    rc = lib.csa_compress_all(ctypes.byref(csa.make_dims(m_hca=256)), 16, 16, 1, 10, *P[:9], ctypes.byref(n), None)
    assert rc == csa.CSA_ERR_UNSUPPORTED
    assert lib.csa_debug_inject(3, 0) == csa.CSA_ERR_ARG
    assert lib.csa_debug_inject(2, 0) == csa.CSA_OK
    assert lib.csa_debug_inject(1, -5) == csa.CSA_ERR_ARG
    assert lib.csa_debug_inject(0, 0) == csa.CSA_OK


def test_workspace_sizes(lib):
    dims = csa.make_dims()
    a = csa.csa_decode_args()
    a.dims = dims
    a.B, a.max_len = 4, (1 << 20) + 128
    n = csa.csa_workspace_size(csa.CSA_OP_DECODE, a)
    # scores (4 B) + candidates (8 B) per CSA entry dominate
    assert n >= 4 * ((1 << 20) // 4) * 12
    assert n < 200 << 20
    w = csa.csa_ws_query()
    w.dims, w.Q, w.max_len = dims, 8, 65536
    assert csa.csa_workspace_size(csa.CSA_OP_INDEX_TOPK, w) > 8 * 16384 * 12
    assert csa.csa_workspace_size(99, w) == 0
    bad = csa.csa_ws_query()
    bad.dims, bad.Q, bad.max_len = csa.make_dims(d=100), 1, 10
    assert csa.csa_workspace_size(csa.CSA_OP_INDEX_TOPK, bad) == 0
