"""FP64 CPU oracle for the CSA / HCA layer (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The product path (the CUDA library and
its Python binding) never does, and the two share no code.

The arithmetic lives in ``csa_oracle.c`` (plain C, IEEE double, OpenMP over
independent queries/blocks). This module only compiles it, marshals numpy
arrays into it, and converts stored formats (BF16 bits, FP8 mixed rows) to
exact FP64 values.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "csa_oracle.c"
_LIB_PATH = _HERE / "liboracle.so"
_lib = None


def build(force: bool = False) -> Path:
    """Compile csa_oracle.c into liboracle.so (gcc, -O2, OpenMP, IEEE)."""
    if force or not _LIB_PATH.exists() or _LIB_PATH.stat().st_mtime < _SRC.stat().st_mtime:
        tmp = _LIB_PATH.with_suffix(f".so.tmp{os.getpid()}")
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
               "-shared", "-fPIC", str(_SRC), "-o", str(tmp), "-lm"]
        subprocess.check_call(cmd)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(str(_LIB_PATH))
        P = ctypes.c_void_p
        I64, I32, D = ctypes.c_int64, ctypes.c_int, ctypes.c_double
        lib.orc_compress_blocks.argtypes = [I64, I32, I32, I32, I32, P, P, P, P, P, P, P, D, I32,
                                            D, P, I64, P, P]
        lib.orc_index_topk.argtypes = [I64, I32, I32, I32, I32, I32, P, P, P, I64, P, P, P, P, P,
                                       P, P]
        lib.orc_attend.argtypes = [I64, I32, I32, I32, D, D, I32, I32, P, P, P, P, I64, P, P, I32,
                                   I32, I32, I32, P, I64, P, P, P, P]
        lib.orc_rmsnorm_rows.argtypes = [P, I64, I32, P, D, P]
        lib.orc_rope_rows.argtypes = [P, I64, I32, I32, D, P]
        lib.orc_rmsnorm_rope_rows.argtypes = [P, I64, I32, I32, D, D, P, P, P]
        lib.orc_visible_entries.argtypes = [I64, I32, I32, I64]
        lib.orc_visible_entries.restype = I64
        lib.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
        lib.orc_e4m3_decode.restype = D
        lib.orc_e4m3_encode.argtypes = [D]
        lib.orc_e4m3_encode.restype = ctypes.c_uint8
        lib.orc_pack_mixed_row.argtypes = [P, P]
        lib.orc_unpack_mixed_row.argtypes = [P, P]
        for f in ("orc_compress_blocks", "orc_index_topk", "orc_attend"):
            getattr(lib, f).restype = I32
        _lib = lib
    return _lib


def _f64(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a):
    return None if a is None else a.ctypes.data


def to_f64(a) -> np.ndarray:
    """Exact FP64 values of a stored tensor: float32/float64 arrays as they
    are, uint16 arrays as BF16 bit patterns."""
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


# --------------------------------------------------------------------------
# building blocks
# --------------------------------------------------------------------------
def rmsnorm(x, eps=1e-6, gain=None):
    lib = _load()
    x = _f64(x)
    c = x.shape[-1]
    y = np.empty_like(x)
    g = _f64(gain)  # kept referenced until the call returns
    lib.orc_rmsnorm_rows(_ptr(x), x.size // c, c, _ptr(g), eps, _ptr(y))
    return y


def rope(x, pos, rope_dims, base=10000.0):
    lib = _load()
    y = _f64(x).copy()
    c = y.shape[-1]
    rows = y.size // c
    p = np.ascontiguousarray(np.broadcast_to(np.asarray(pos, dtype=np.float64), y.shape[:-1]))
    lib.orc_rope_rows(_ptr(y), rows, c, rope_dims, base, _ptr(p))
    return y


def rmsnorm_rope(x, pos, rope_dims, base=10000.0, eps=1e-6, gain=None):
    lib = _load()
    x = _f64(x)
    c = x.shape[-1]
    rows = x.size // c
    p = np.ascontiguousarray(np.broadcast_to(np.asarray(pos, dtype=np.float64), x.shape[:-1]))
    y = np.empty_like(x)
    g = _f64(gain)
    lib.orc_rmsnorm_rope_rows(_ptr(x), rows, c, rope_dims, base, eps, _ptr(g), _ptr(p), _ptr(y))
    return y


def visible_entries(p, m, vis_offset, n_entries):
    return int(_load().orc_visible_entries(int(p), m, vis_offset, int(n_entries)))


# --------------------------------------------------------------------------
# the three stages
# --------------------------------------------------------------------------
def compress(H, W_aKV, W_aZ, bias, m, W_bKV=None, W_bZ=None, gain=None, eps=1e-6,
             rope_dims=0, base=10000.0, blocks=None, return_pooled=False):
    """Compressed entries [len(blocks), c] (all floor(T/m) blocks by default).
    CSA when W_bKV/W_bZ are given (overlap), HCA otherwise."""
    lib = _load()
    H = _f64(H)
    T, d = H.shape
    c = np.asarray(W_aKV).shape[1]
    overlap = 1 if W_bKV is not None else 0
    if blocks is None:
        blocks = np.arange(T // m, dtype=np.int64)
    blocks = np.ascontiguousarray(blocks, dtype=np.int64)
    E = np.empty((blocks.size, c), np.float64)
    pooled = np.empty((blocks.size, c), np.float64) if return_pooled else None
    arrs = [_f64(a) for a in (W_aKV, W_bKV, W_aZ, W_bZ, bias, gain)]
    rc = lib.orc_compress_blocks(T, d, c, m, overlap, _ptr(H), *[_ptr(a) for a in arrs[:5]],
                                 _ptr(arrs[5]), eps, rope_dims, base, _ptr(blocks), blocks.size,
                                 _ptr(E), _ptr(pooled))
    if rc != 0:
        raise ValueError("oracle compress: invalid arguments")
    return (E, pooled) if return_pooled else E


def index_topk(qI, w, KI, seq_of_q, pos, n_entries, m, k, vis_offset=1, want_scores=False):
    """Returns dict(idx [Q,k] int32, tau [Q], amag [Q], scores [Q,ldK] or None)."""
    lib = _load()
    qI = _f64(qI)
    Q, HI, cI = qI.shape
    KI = _f64(KI)
    ldK = KI.shape[1]
    seq = np.ascontiguousarray(seq_of_q, dtype=np.int32)
    pos = np.ascontiguousarray(pos, dtype=np.int64)
    ne = np.ascontiguousarray(n_entries, dtype=np.int64)
    idx = np.empty((Q, k), np.int32)
    tau = np.empty(Q, np.float64)
    amag = np.empty(Q, np.float64)
    scores = np.full((Q, ldK), np.nan) if want_scores else None
    w = _f64(w)
    rc = lib.orc_index_topk(Q, HI, cI, k, m, vis_offset, _ptr(qI), _ptr(w), _ptr(KI), ldK,
                            _ptr(seq), _ptr(pos), _ptr(ne), _ptr(idx), _ptr(tau), _ptr(amag),
                            _ptr(scores))
    if rc != 0:
        raise ValueError("oracle index_topk: invalid arguments")
    return dict(idx=idx, tau=tau, amag=amag, scores=scores)


def attend(q, sink, E, win, seq_of_q, pos, n_entries, *, rope_dims, idx=None, m=4,
           vis_offset=1, n_win=128, win_ring=0, q_gain=None, eps=1e-6, base=10000.0,
           return_nkeys=False):
    """O [Q, H_q, c]. Sparse (CSA) when idx is given, dense over visible
    entries (HCA) when idx is None. E [nseq, ldE, c], win [nseq, ldW, c]."""
    lib = _load()
    q = _f64(q)
    Q, Hq, c = q.shape
    E = _f64(E)
    win = _f64(win)
    seq = np.ascontiguousarray(seq_of_q, dtype=np.int32)
    pos = np.ascontiguousarray(pos, dtype=np.int64)
    ne = np.ascontiguousarray(n_entries, dtype=np.int64)
    dense = 1 if idx is None else 0
    idxa = None if idx is None else np.ascontiguousarray(idx, dtype=np.int32)
    k = 0 if idx is None else idxa.shape[1]
    O = np.empty_like(q)
    nk = np.empty(Q, np.int32)
    qg, sk = _f64(q_gain), _f64(sink)
    rc = lib.orc_attend(Q, Hq, c, rope_dims, base, eps, n_win, win_ring, _ptr(q),
                        _ptr(qg), _ptr(sk), _ptr(E), E.shape[1], _ptr(ne),
                        _ptr(idxa), k, dense, m, vis_offset, _ptr(win), win.shape[1], _ptr(seq),
                        _ptr(pos), _ptr(O), _ptr(nk))
    if rc != 0:
        raise ValueError("oracle attend: invalid arguments")
    return (O, nk) if return_nkeys else O


# --------------------------------------------------------------------------
# FP8 mixed entry rows
# --------------------------------------------------------------------------
MIXED_ROW_BYTES = 592


def e4m3_decode(codes) -> np.ndarray:
    lib = _load()
    table = np.array([lib.orc_e4m3_decode(i) for i in range(256)], np.float64)
    return table[np.asarray(codes, dtype=np.uint8)]


def e4m3_encode(x) -> np.ndarray:
    lib = _load()
    x = np.asarray(x, np.float64)
    return np.array([lib.orc_e4m3_encode(float(v)) for v in x.ravel()], np.uint8).reshape(x.shape)


def pack_mixed(x) -> np.ndarray:
    """Rows [n, 512] (FP32 values) -> mixed rows [n, 592] uint8."""
    lib = _load()
    x = np.ascontiguousarray(x, dtype=np.float32).reshape(-1, 512)
    out = np.zeros((x.shape[0], MIXED_ROW_BYTES), np.uint8)
    for i in range(x.shape[0]):
        lib.orc_pack_mixed_row(x[i].ctypes.data, out[i].ctypes.data)
    return out


def unpack_mixed(rows) -> np.ndarray:
    """Mixed rows [..., 592] uint8 -> exact FP64 values [..., 512]."""
    lib = _load()
    rows = np.ascontiguousarray(rows, dtype=np.uint8)
    flat = rows.reshape(-1, MIXED_ROW_BYTES)
    out = np.empty((flat.shape[0], 512), np.float64)
    for i in range(flat.shape[0]):
        lib.orc_unpack_mixed_row(flat[i].ctypes.data, out[i].ctypes.data)
    return out.reshape(rows.shape[:-1] + (512,))
