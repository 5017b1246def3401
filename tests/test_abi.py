"""The C ABI on the host: libcsa.so loads without a GPU, exports every
function include/csa.h declares, and rejects bad arguments before any CUDA
call (every case below returns before touching the device)."""
import ctypes
import re
from pathlib import Path

import pytest

import compressed_sparse_attention_17_b200 as csa
from compressed_sparse_attention_17_b200 import build as csa_build

HEADER = Path(__file__).resolve().parents[1] / "include" / "csa.h"


@pytest.fixture(scope="module")
def lib():
    csa_build.build()
    return csa.load()


def declared_functions():
    text = re.sub(r"/\*.*?\*/", "", HEADER.read_text(), flags=re.S)
    return re.findall(r"^\s*(?:const\s+char\s*\*|csa_status|size_t|u?int64_t|int|void)\s+\**\s*"
                      r"(csa_\w+|hca_\w+)\s*\(", text, flags=re.M)


def test_header_declares_the_entry_points():
    names = set(declared_functions())
    for n in ("csa_compress", "csa_index_topk", "csa_attend", "hca_attend", "csa_rmsnorm_rope",
              "csa_compress_decode", "csa_sync_status"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_status_strings(lib):
    assert lib.csa_status_string(0) == b"CSA_OK"
    assert lib.csa_status_string(4) == b"CSA_ERR_TIMEOUT"
    assert lib.csa_version().startswith(b"libcsa")


def test_workspace_queries(lib):
    g = csa.geom()
    assert lib.csa_compress_workspace_size(ctypes.byref(g), 0, 8192, 4096) >= 8192 * 4 * 512 * 4
    assert lib.csa_compress_workspace_size(ctypes.byref(g), 1, 8192, 4096) >= 2048 * 512 * 4
    assert lib.csa_index_topk_workspace_size(32, 32768, 1024) >= 0
    assert lib.csa_compress_decode_state_floats(ctypes.byref(g)) == 2 * 4 * 4 * 512
    gh = csa.geom(m=128, overlap=0)
    assert lib.csa_compress_decode_state_floats(ctypes.byref(gh)) == 128 * 2 * 512


P = ctypes.c_void_p
BAD = P(0x1001)   # misaligned, never dereferenced
OK = P(0x10000)   # aligned fake device address, never dereferenced


@pytest.mark.parametrize("field,value", [("c", 24), ("c", 2048), ("rope_dims", 3),
                                         ("rope_dims", 1024), ("m", 0), ("overlap", 2),
                                         ("vis_offset", 5), ("n_win", -1), ("rope_base", 0.0)])
def test_bad_geometry_rejected(lib, field, value):
    g = csa.geom()
    setattr(g, field, value)
    st = lib.csa_rmsnorm_rope(ctypes.byref(g), 1, 1, OK, 4, None, 0, 1, None, OK, None, None)
    assert st == 1


def test_null_and_misaligned_pointers_rejected(lib):
    g = csa.geom()
    assert lib.csa_rmsnorm_rope(None, 1, 1, OK, 4, None, 0, 1, None, OK, None, None) == 1
    assert lib.csa_rmsnorm_rope(ctypes.byref(g), 1, 1, BAD, 4, None, 0, 1, None, OK, None, None) == 1
    assert lib.csa_rmsnorm_rope(ctypes.byref(g), 1, 1, None, 4, None, 0, 1, None, OK, None, None) == 1
    # mixed output needs c = 512 and 64 RoPE dims
    g2 = csa.geom(c=256)
    assert lib.csa_rmsnorm_rope(ctypes.byref(g2), 1, 2, OK, 4, None, 0, 1, None, OK, None, None) == 1


def test_index_topk_argument_checks(lib):
    g = csa.geom()
    args = lambda k, HI, cI, ws, wsb: (ctypes.byref(g), 1, OK, OK, OK, 100, 1, OK, OK, OK, 4, HI,
                                       cI, k, OK, None, ws, wsb, None)
    assert lib.csa_index_topk(*args(0, 64, 128, OK, 1 << 20)) == 1      # k = 0
    assert lib.csa_index_topk(*args(4096, 64, 128, OK, 1 << 20)) == 1   # k > max
    assert lib.csa_index_topk(*args(16, 64, 100, OK, 1 << 20)) == 1     # c_I % 16
    assert lib.csa_index_topk(*args(16, 300, 128, OK, 1 << 20)) == 1    # H_I > 128
    assert lib.csa_index_topk(*args(16, 64, 128, None, 0)) == 1         # no workspace


def test_index_scores_argument_checks(lib):
    g = csa.geom()
    args = lambda HI, cI, sc, ld, w=OK: (ctypes.byref(g), 1, OK, w, OK, 100, 1, OK, OK, OK, 4, HI,
                                         cI, sc, ld, None)
    assert lib.csa_index_scores(*args(64, 100, OK, 100)) == 1      # c_I % 16
    assert lib.csa_index_scores(*args(300, 128, OK, 100)) == 1     # H_I > 128
    assert lib.csa_index_scores(*args(64, 128, OK, 99)) == 1       # ld_scores < ldK
    assert lib.csa_index_scores(*args(64, 128, None, 100)) == 1    # no output
    assert lib.csa_index_scores(*args(64, 128, BAD, 100)) == 1     # misaligned output
    assert lib.csa_index_scores(*args(64, 128, OK, 100, w=None)) == 1  # no weights


def test_compress_argument_checks(lib):
    g = csa.geom()
    # CSA without the b-series weights
    assert lib.csa_compress(ctypes.byref(g), 1, OK, 64, 128, OK, None, OK, None, OK, None, 1, OK,
                            OK, 1 << 30, None) == 1
    gh = csa.geom(m=128, overlap=0)
    # HCA with b-series weights
    assert lib.csa_compress(ctypes.byref(gh), 1, OK, 256, 128, OK, OK, OK, OK, OK, None, 1, OK,
                            OK, 1 << 30, None) == 1
    # too small a workspace
    assert lib.csa_compress(ctypes.byref(g), 1, OK, 64, 128, OK, OK, OK, OK, OK, None, 1, OK,
                            OK, 16, None) == 1


def test_attend_argument_checks(lib):
    g = csa.geom(win_ring=1)
    # ring window with fewer rows than n_win
    assert lib.csa_attend(ctypes.byref(g), 1, 1, OK, None, OK, OK, 10, 1, OK, OK, 8, OK, 64, OK,
                          OK, 2, 64, OK, None, 0, None) == 1
    # bad q dtype
    g0 = csa.geom()
    assert lib.csa_attend(ctypes.byref(g0), 2, 1, OK, None, OK, OK, 10, 1, OK, OK, 8, OK, 500, OK,
                          OK, 2, 64, OK, None, 0, None) == 1
