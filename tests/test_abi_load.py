"""The C-ABI library loads on a machine without a GPU, exports every entry
point include/v4a.h declares, and rejects bad arguments on the host before
any launch (these calls never reach CUDA)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "v4a.h")


def declared_symbols():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"V4A_API\s+[\w\s\*]+?\b(v4a_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def v4a():
    import compressed_sparse_long_v4a_b200 as v
    return v


def test_header_declares_the_five_operations():
    syms = declared_symbols()
    for name in ["v4a_compress", "v4a_index_scores", "v4a_topk", "v4a_csa_attend", "v4a_hca_attend",
                 "v4a_workspace_size", "v4a_status_string", "v4a_last_error", "v4a_version"]:
        assert name in syms


def test_library_exports_every_declared_symbol(v4a):
    out = subprocess.run(["nm", "-D", "--defined-only", v4a.library_path()], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\sT\s(v4a_\w+)", out))
    missing = [s for s in declared_symbols() if s not in exported]
    assert not missing, missing
    lib = ctypes.CDLL(v4a.library_path())
    for s in declared_symbols():
        assert hasattr(lib, s)
    # nothing but the declared API leaks out of the library
    assert exported == set(declared_symbols())


def test_status_strings_and_version(v4a):
    assert v4a.v4a_status_string(0) == "ok"
    assert "device fault" in v4a.v4a_status_string(4)
    assert v4a.v4a_version() >= 100


def test_host_side_argument_errors(v4a):
    L = v4a.lib
    # NULL kv stream
    assert L.v4a_compress(None, None, 1, 4, 4, None) == 1
    assert b"kv" in L.v4a_last_error()
    # channels not a multiple of 8
    io = v4a.CompressIO(16, 16, 16, None, 12, 0, 0, 48, 48, 12, 0)
    assert L.v4a_compress(ctypes.byref(io), None, 1, 4, 4, None) == 1
    # unsupported output dtype for the input
    io = v4a.CompressIO(16, 16, 16, None, 16, 2, 0, 64, 64, 16, 0)
    assert L.v4a_compress(ctypes.byref(io), None, 1, 4, 4, None) == 2
    shape = v4a.Shape(1, 1, 64, 512, 4, 0, 128, 1024)
    # csa without idx / k
    assert L.v4a_csa_attend(16, 16, None, 16, 896, 128, 16, 1, 256, 1 << 20, None, ctypes.byref(shape), None) == 1
    # window not covered by token_kv
    shape = v4a.Shape(1, 1, 64, 512, 128, 0, 128, 1024)
    assert L.v4a_hca_attend(16, 16, 16, 900, 124, 16, 1, 256, 1 << 20, ctypes.byref(shape), None) == 1
    assert b"cover" in L.v4a_last_error()
    # unsupported d
    shape = v4a.Shape(1, 1, 64, 96, 128, 0, 128, 1024)
    assert L.v4a_hca_attend(16, 16, 16, 896, 128, 16, 1, 256, 1 << 20, ctypes.byref(shape), None) == 2
    # n_q > ctx_len
    shape = v4a.Shape(1, 9, 4, 64, 4, 4, 0, 8)
    assert L.v4a_index_scores(16, 16, 16, None, 16, 4, 64, 0, 0, ctypes.byref(shape), None) == 1
    # fp8 keys without scales
    shape = v4a.Shape(1, 1, 4, 64, 4, 4, 0, 64)
    assert L.v4a_index_scores(16, 16, 16, None, 16, 4, 64, 1, 2, ctypes.byref(shape), None) == 1
    # top-k: k out of range, then a workspace that is too small
    shape = v4a.Shape(1, 1, 4, 64, 4, 0, 0, 64)
    assert L.v4a_topk(16, 16, 16, None, 16, None, 4, 64, 0, 0, 256, 1 << 20, ctypes.byref(shape), None) == 1
    shape = v4a.Shape(1, 1, 4, 64, 4, 8, 0, 1 << 20)
    assert L.v4a_topk(16, 16, 16, None, 16, None, 4, 64, 0, 0, 256, 16, ctypes.byref(shape), None) == 1
    assert b"workspace" in L.v4a_last_error()


def test_mxfp4_host_side_argument_errors(v4a):
    L = v4a.lib
    # quantiser: cols not a multiple of 32, then an unsupported dtype
    assert L.v4a_quantize_mxfp4(16, 0, 4, 48, 16, 16, None) == 1
    assert L.v4a_quantize_mxfp4(16, 2, 4, 64, 16, 16, None) == 2
    assert L.v4a_quantize_mxfp4(None, 0, 0, 64, None, None, None) == 0  # nothing to do
    shape = v4a.Shape(1, 1, 4, 64, 4, 8, 0, 64)
    # MXFP4 keys go through the _mxfp4 calls only
    assert L.v4a_index_scores(16, 16, 16, None, 16, 4, 64, 1, 3, ctypes.byref(shape), None) == 2
    assert b"mxfp4" in L.v4a_last_error()
    assert L.v4a_topk(16, 16, 16, None, 16, None, 4, 64, 1, 3, 256, 1 << 20, ctypes.byref(shape), None) == 2
    # d_i not a multiple of 32; block exponents missing
    assert L.v4a_index_scores_mxfp4(16, 16, 16, 16, 16, 4, 48, 1, ctypes.byref(shape), None) == 1
    assert L.v4a_index_scores_mxfp4(16, 16, 16, None, 16, 4, 64, 1, ctypes.byref(shape), None) == 1
    assert b"k_exp" in L.v4a_last_error()
    assert L.v4a_topk_mxfp4(16, 16, 16, None, 16, None, 4, 64, 1, 256, 1 << 20, ctypes.byref(shape), None) == 1
    # compress with MXFP4 output: channels must be a multiple of 32 and out_exp is required
    io = v4a.CompressIO(16, 16, 16, None, 16, 1, 3, 64, 64, 16, 0, 16, 1)
    assert L.v4a_compress(ctypes.byref(io), None, 1, 4, 4, None) == 1
    io = v4a.CompressIO(16, 16, 16, None, 64, 1, 3, 256, 256, 64, 0, None, 2)
    assert L.v4a_compress(ctypes.byref(io), None, 1, 4, 4, None) == 1
    assert b"out_exp" in L.v4a_last_error()


def test_paged_host_side_argument_errors(v4a):
    L = v4a.lib
    shape = v4a.Shape(1, 1, 64, 512, 4, 8, 128, 1024)
    bt = ctypes.c_int32 * 8
    tab = bt()
    # no block table
    pg = v4a.Paged(None, 8, 128, 4, 256)
    assert L.v4a_topk_paged(16, 16, 16, None, 16, None, 4, 64, 1, 1, 256, 1 << 20, None, ctypes.byref(pg),
                            ctypes.byref(shape), None) == 1
    assert b"block table" in L.v4a_last_error()
    # block_tokens not a multiple of m, then a table too short for the context (1024/4 = 256 entries)
    fake = 1 << 20  # a device-looking pointer that is never dereferenced on the host
    pg = v4a.Paged(fake, 8, 130, 4, 256)
    assert L.v4a_topk_paged(16, 16, 16, None, 16, None, 4, 64, 1, 1, 256, 1 << 20, None, ctypes.byref(pg),
                            ctypes.byref(shape), None) == 1
    pg = v4a.Paged(fake, 4, 128, 4, 256)
    assert L.v4a_topk_paged(16, 16, 16, None, 16, None, 4, 64, 1, 1, 256, 1 << 20, None, ctypes.byref(pg),
                            ctypes.byref(shape), None) == 1
    assert b"block table" in L.v4a_last_error()
    # a ring that cannot hold the window
    pg = v4a.Paged(fake, 8, 128, 4, 100)
    assert L.v4a_csa_attend_paged(16, 16, 16, 16, 16, 1, 256, 1 << 20, None, None, ctypes.byref(pg),
                                  ctypes.byref(shape), None) == 1
    assert b"ring" in L.v4a_last_error()
    # ring append: too many streams, misaligned rows
    ios = (v4a.RingIO * 9)()
    assert L.v4a_ring_append(ios, 9, 1, 0, None) == 1
    ios[0] = v4a.RingIO(16, 16, 12, 256, 1, 12)  # 24-byte rows
    assert L.v4a_ring_append(ios, 1, 1, 0, None) == 1
    del tab


def test_workspace_sizes(v4a):
    assert v4a.v4a_workspace_size("nonsense", batch=1) == 0
    ws = v4a.v4a_workspace_size("topk", batch=4, m=4, k=1024, ctx_len=1 << 20, heads_i=16, d_i=128)
    assert ws >= 4 * (1 << 18) * 4  # at least one fp32 score per entry
    assert v4a.v4a_workspace_size("hca_attend", batch=32, heads=64, d=512, m=128, window=128, ctx_len=1 << 20) > 0
