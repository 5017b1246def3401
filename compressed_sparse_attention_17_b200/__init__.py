"""B200-native compressed sparse attention (CSA) and heavily compressed
attention (HCA) layer of DeepSeek-V4.

The work runs in ``libcsa.so`` (hand-written CUDA for sm_100a behind a C
ABI, declared in ``include/csa.h``). This module is the thin Python binding:
it allocates outputs and workspaces with PyTorch, marshals pointers and the
current CUDA stream, and raises on a non-OK status. There is no fallback:
if the library is missing or fails to load, every call raises.
"""
from __future__ import annotations

import ctypes
from pathlib import Path

import torch

__all__ = [
    "Geom", "CsaError", "load", "geom", "rmsnorm_rope", "quantize_mixed", "compress",
    "compress_decode", "decode_state", "index_topk", "attend", "hca_attend", "sync_status",
    "kernel_launches", "MIXED_ROW_BYTES", "CSA_F32", "CSA_BF16", "CSA_FP8_MIXED",
]

LIB_PATH = Path(__file__).resolve().parent / "libcsa.so"
MIXED_ROW_BYTES = 592
CSA_F32, CSA_BF16, CSA_FP8_MIXED = 0, 1, 2
_STATUS = {0: "CSA_OK", 1: "CSA_ERR_INVALID_ARG", 2: "CSA_ERR_UNSUPPORTED", 3: "CSA_ERR_CUDA",
           4: "CSA_ERR_TIMEOUT", 5: "CSA_ERR_TOO_LARGE"}


class CsaError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__(f"{fn} returned {_STATUS.get(status, status)}")


class Geom(ctypes.Structure):
    """Mirror of csa_geom (include/csa.h)."""
    _fields_ = [("m", ctypes.c_int), ("overlap", ctypes.c_int), ("c", ctypes.c_int),
                ("rope_dims", ctypes.c_int), ("rope_base", ctypes.c_double),
                ("eps", ctypes.c_float), ("vis_offset", ctypes.c_int), ("n_win", ctypes.c_int),
                ("win_ring", ctypes.c_int)]


def geom(m=4, overlap=1, c=512, rope_dims=64, rope_base=10000.0, eps=1e-6, vis_offset=1,
         n_win=128, win_ring=0) -> Geom:
    return Geom(m, overlap, c, rope_dims, rope_base, eps, vis_offset, n_win, win_ring)


_lib = None
_P, _I64, _I32, _SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
_GP = ctypes.POINTER(Geom)

_SIGS = {
    "csa_status_string": ([_I32], ctypes.c_char_p),
    "csa_version": ([], ctypes.c_char_p),
    "csa_sync_status": ([_P], _I32),
    "csa_kernel_launches": ([], ctypes.c_uint64),
    "csa_rmsnorm_rope": ([_GP, _I32, _I32, _P, _I64, _P, _I64, _I64, _P, _P, _P, _P], _I32),
    "csa_quantize_mixed": ([_I32, _P, _I64, _P, _P], _I32),
    "csa_compress_workspace_size": ([_GP, _I32, _I64, _I32], _SZ),
    "csa_compress": ([_GP, _I32, _P, _I64, _I32, _P, _P, _P, _P, _P, _P, _I32, _P, _P, _SZ, _P],
                     _I32),
    "csa_compress_decode_state_floats": ([_GP], _I64),
    "csa_compress_decode_workspace_size": ([_GP, _I32, _I32, _I32], _SZ),
    "csa_compress_decode": ([_GP, _I32, _P, _P, _I32, _I32, _P, _P, _P, _P, _P, _P, _P, _I32, _P,
                             _I64, _P, _SZ, _P], _I32),
    "csa_index_topk_workspace_size": ([_I32, _I64, _I32], _SZ),
    "csa_index_topk": ([_GP, _I32, _P, _P, _P, _I64, _I32, _P, _P, _P, _I32, _I32, _I32, _I32,
                        _P, _P, _P, _SZ, _P], _I32),
    "csa_index_scores": ([_GP, _I32, _P, _P, _P, _I64, _I32, _P, _P, _P, _I32, _I32, _I32, _P,
                          _I64, _P], _I32),
    "csa_index_topk_noalloc": ([_GP, _I32, _P, _P, _P, _I64, _I32, _P, _P, _P, _I32, _I32, _I32,
                                _I32, _P, _P, _P], _I32),
    "csa_attend_workspace_size": ([_I32, _I32, _I32, _I32, _I32], _SZ),
    "csa_attend": ([_GP, _I32, _I32, _P, _P, _P, _P, _I64, _I32, _P, _P, _I32, _P, _I64, _P, _P,
                    _I32, _I32, _P, _P, _SZ, _P], _I32),
    "hca_attend_workspace_size": ([_I32, _I32, _I32, _I64, _I32], _SZ),
    "hca_attend": ([_GP, _I32, _I32, _P, _P, _P, _P, _I64, _I32, _P, _P, _I64, _P, _P, _I32, _I32,
                    _P, _P, _SZ, _P], _I32),
}


def load():
    """Load libcsa.so (raises if it is missing: there is no fallback)."""
    global _lib
    if _lib is None:
        if not LIB_PATH.exists():
            raise RuntimeError(f"{LIB_PATH} is missing; build it with "
                               "compressed_sparse_attention_17_b200.build.build()")
        lib = ctypes.CDLL(str(LIB_PATH))
        for name, (args, res) in _SIGS.items():
            f = getattr(lib, name)
            f.argtypes = args
            f.restype = res
        _lib = lib
    return _lib


def _call(name, *args):
    st = getattr(load(), name)(*args)
    if st != 0:
        raise CsaError(name, st)


def _stream(t: torch.Tensor):
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return CSA_F32
    if t.dtype == torch.bfloat16:
        return CSA_BF16
    if t.dtype == torch.uint8 and t.shape[-1] == MIXED_ROW_BYTES:
        return CSA_FP8_MIXED
    raise TypeError(f"unsupported tensor dtype {t.dtype} / shape {tuple(t.shape)}")


def _torch_dtype(dt: int):
    return {CSA_F32: torch.float32, CSA_BF16: torch.bfloat16}[dt]


def _check(*ts):
    for t in ts:
        if t is not None:
            if not t.is_cuda or not t.is_contiguous():
                raise ValueError("tensors must be contiguous CUDA tensors")


def _rows_out(shape_rows, c, out_dtype, device):
    if out_dtype == CSA_FP8_MIXED:
        return torch.empty(*shape_rows, MIXED_ROW_BYTES, dtype=torch.uint8, device=device)
    return torch.empty(*shape_rows, c, dtype=_torch_dtype(out_dtype), device=device)


def sync_status(device=None) -> None:
    """Synchronise the current stream and raise if a device wait gave up."""
    s = torch.cuda.current_stream(device)
    st = load().csa_sync_status(ctypes.c_void_p(s.cuda_stream))
    if st != 0:
        raise CsaError("csa_sync_status", st)


def rmsnorm_rope(x, g: Geom, pos=None, pos0=0, pos_step=1, gain=None, out_dtype=None,
                 out=None, out_row=None):
    """RoPE_pos(RMSNorm(x) * gain) per row of x [..., c]. With `out` and
    `out_row` given, row r is written to row out_row[r] of `out`."""
    _check(x, pos, gain, out, out_row)
    odt = (_dt(x) if out_dtype is None else out_dtype) if out is None else _dt(out)
    rows = x.numel() // x.shape[-1]
    if out is None:
        out = _rows_out(tuple(x.shape[:-1]), x.shape[-1], odt, x.device)
    _call("csa_rmsnorm_rope", ctypes.byref(g), _dt(x), odt, _ptr(x), rows, _ptr(pos), pos0,
          pos_step, _ptr(gain), _ptr(out), _ptr(out_row), _stream(x))
    return out


def kernel_launches() -> int:
    """Kernels libcsa has launched in this process."""
    return int(load().csa_kernel_launches())


def quantize_mixed(x):
    """Rows [..., 512] -> mixed FP8/BF16 rows [..., 592] uint8."""
    _check(x)
    out = torch.empty(*x.shape[:-1], MIXED_ROW_BYTES, dtype=torch.uint8, device=x.device)
    _call("csa_quantize_mixed", _dt(x), _ptr(x), x.numel() // 512, _ptr(out), _stream(x))
    return out


def compress(H, W_aKV, W_aZ, bias, g: Geom, W_bKV=None, W_bZ=None, gain=None, out_dtype=None,
             workspace=None):
    """Compressed entries [T // m, c] of one sequence H [T, d]."""
    _check(H, W_aKV, W_aZ, bias, W_bKV, W_bZ, gain)
    T, d = H.shape
    odt = _dt(H) if out_dtype is None else out_dtype
    E = _rows_out((T // g.m,), g.c, odt, H.device)
    ws_bytes = load().csa_compress_workspace_size(ctypes.byref(g), _dt(H), T, d)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=H.device)
    _call("csa_compress", ctypes.byref(g), _dt(H), _ptr(H), T, d, _ptr(W_aKV), _ptr(W_bKV),
          _ptr(W_aZ), _ptr(W_bZ), _ptr(bias), _ptr(gain), odt, _ptr(E), _ptr(workspace),
          workspace.numel() * workspace.element_size(), _stream(H))
    return E


def decode_state(B, g: Geom, device="cuda"):
    """Zeroed compressor state for B sequences."""
    n = load().csa_compress_decode_state_floats(ctypes.byref(g))
    return torch.zeros(B, n, dtype=torch.float32, device=device)


def compress_decode(h, pos, W_aKV, W_aZ, bias, state, E_cache, g: Geom, W_bKV=None, W_bZ=None,
                    gain=None, workspace=None):
    """One decode step of the compressor: h [B, d] at positions pos [B]."""
    _check(h, pos, W_aKV, W_aZ, bias, state, E_cache, W_bKV, W_bZ, gain)
    B, d = h.shape
    ws_bytes = load().csa_compress_decode_workspace_size(ctypes.byref(g), _dt(h), B, d)
    if workspace is None and ws_bytes > 0:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=h.device)
    _call("csa_compress_decode", ctypes.byref(g), _dt(h), _ptr(h), _ptr(pos), B, d, _ptr(W_aKV),
          _ptr(W_bKV), _ptr(W_aZ), _ptr(W_bZ), _ptr(bias), _ptr(gain), _ptr(state),
          _dt(E_cache), _ptr(E_cache), E_cache.shape[1], _ptr(workspace),
          0 if workspace is None else workspace.numel() * workspace.element_size(), _stream(h))


def index_topk(qI, w, KI, seq_of_q, pos, n_entries, k, g: Geom, want_scores=False,
               workspace=None, out=None):
    """Top-k entry indices [Q, k] (int32, ascending, -1 padded)."""
    _check(qI, w, KI, seq_of_q, pos, n_entries)
    Q, HI, cI = qI.shape
    ldK = KI.shape[1]
    idx = out if out is not None else torch.empty(Q, k, dtype=torch.int32, device=qI.device)
    scores = torch.full((Q, ldK), float("nan"), device=qI.device) if want_scores else None
    ws_bytes = load().csa_index_topk_workspace_size(Q, ldK, k)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=qI.device)
    _call("csa_index_topk", ctypes.byref(g), _dt(qI), _ptr(qI), _ptr(w), _ptr(KI), ldK,
          KI.shape[0], _ptr(seq_of_q), _ptr(pos), _ptr(n_entries), Q, HI, cI, k, _ptr(idx), _ptr(scores),
          _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(qI))
    return (idx, scores) if want_scores else idx


def index_scores(qI, w, KI, seq_of_q, pos, n_entries, g: Geom, out=None):
    """Indexer scores I [Q, ldK] (FP32) for the visible entries of each query;
    the other slots of a new buffer hold NaN."""
    _check(qI, w, KI, seq_of_q, pos, n_entries)
    Q, HI, cI = qI.shape
    ldK = KI.shape[1]
    sc = out if out is not None else torch.full((Q, ldK), float("nan"), device=qI.device)
    _call("csa_index_scores", ctypes.byref(g), _dt(qI), _ptr(qI), _ptr(w), _ptr(KI), ldK,
          KI.shape[0], _ptr(seq_of_q), _ptr(pos), _ptr(n_entries), Q, HI, cI, _ptr(sc),
          sc.shape[1], _stream(qI))
    return sc


def attend(q, sink, E, idx, win, seq_of_q, pos, n_entries, g: Geom, q_gain=None, out=None,
           workspace=None):
    """Sparse shared-KV attention, O [Q, H_q, c] in q's dtype."""
    _check(q, sink, E, idx, win, seq_of_q, pos, n_entries, q_gain)
    Q, Hq, c = q.shape
    k = idx.shape[1]
    O = out if out is not None else torch.empty_like(q)
    ws_bytes = load().csa_attend_workspace_size(Q, Hq, c, k, g.n_win)
    if workspace is None and ws_bytes > 0:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    _call("csa_attend", ctypes.byref(g), _dt(q), _dt(E), _ptr(q), _ptr(q_gain), _ptr(sink),
          _ptr(E), E.shape[1], E.shape[0], _ptr(n_entries), _ptr(idx), k, _ptr(win), win.shape[1],
          _ptr(seq_of_q), _ptr(pos), Q, Hq, _ptr(O), _ptr(workspace),
          0 if workspace is None else workspace.numel() * workspace.element_size(), _stream(q))
    return O


def hca_attend(q, sink, E, win, seq_of_q, pos, n_entries, g: Geom, q_gain=None, out=None,
               workspace=None):
    """Dense shared-KV attention over every visible entry plus the window."""
    _check(q, sink, E, win, seq_of_q, pos, n_entries, q_gain)
    Q, Hq, c = q.shape
    O = out if out is not None else torch.empty_like(q)
    ws_bytes = load().hca_attend_workspace_size(Q, Hq, c, E.shape[1], g.n_win)
    if workspace is None and ws_bytes > 0:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    _call("hca_attend", ctypes.byref(g), _dt(q), _dt(E), _ptr(q), _ptr(q_gain), _ptr(sink),
          _ptr(E), E.shape[1], E.shape[0], _ptr(n_entries), _ptr(win), win.shape[1], _ptr(seq_of_q),
          _ptr(pos), Q, Hq, _ptr(O), _ptr(workspace),
          0 if workspace is None else workspace.numel() * workspace.element_size(), _stream(q))
    return O
