"""csa_index_topk_noalloc: the index/top-k entry point for callers that
cannot allocate device memory around a call (a memory arena that forbids
outside allocations, a serving loop that must not allocate). Its scratch is
one fixed device buffer inside libcsa.so. Two calls in a row, on different
inputs, must give the same indices as csa_index_topk with a workspace."""
import ctypes

import numpy as np
import pytest
import torch

import compressed_sparse_attention_17_b200 as csa
from compressed_sparse_attention_17_b200 import synth

pytestmark = pytest.mark.gpu


def _inputs(seed, Q, HI, cI, nseq, N):
    rg = np.random.default_rng(seed)
    spec = lambda n, shape, dt: synth.Spec(n, shape, 1.0, dt, seed).values()
    qI = torch.from_numpy(spec("qI", (Q, HI, cI), "bf16")).to(torch.bfloat16).cuda()
    KI = torch.from_numpy(spec("KI", (nseq, N, cI), "bf16")).to(torch.bfloat16).cuda()
    w = torch.from_numpy(spec("w", (Q, HI), "f32")).cuda()
    seq = torch.from_numpy(rg.integers(0, nseq, Q).astype(np.int32)).cuda()
    pos = torch.from_numpy(rg.integers(0, 4 * N + 8, Q).astype(np.int64)).cuda()
    ne = torch.tensor([N - 11 * b for b in range(nseq)], dtype=torch.int64).cuda()
    return qI, w, KI, seq, pos, ne


def _noalloc(lib, g, qI, w, KI, seq, pos, ne, k):
    Q, HI, cI = qI.shape
    idx = torch.full((Q, k), -7, dtype=torch.int32, device="cuda")
    st = lib.csa_index_topk_noalloc(
        ctypes.byref(g), csa.CSA_BF16, ctypes.c_void_p(qI.data_ptr()), ctypes.c_void_p(w.data_ptr()),
        ctypes.c_void_p(KI.data_ptr()), KI.shape[1], KI.shape[0], ctypes.c_void_p(seq.data_ptr()),
        ctypes.c_void_p(pos.data_ptr()), ctypes.c_void_p(ne.data_ptr()), Q, HI, cI, k,
        ctypes.c_void_p(idx.data_ptr()), None,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, lib.csa_status_string(st)
    return idx


def test_index_topk_noalloc_matches_workspace_entry_point():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = csa.load()
    g = csa.geom()
    # two calls in a row on different inputs: the shared buffer keeps the
    # first call's contents when the second one runs
    cases = [(5, 24, 64, 128, 3, 30000, 1024), (6, 40, 64, 128, 2, 9000, 256)]
    for seed, Q, HI, cI, nseq, N, k in cases:
        args = _inputs(seed, Q, HI, cI, nseq, N)
        got = _noalloc(lib, g, *args, k)
        want = csa.index_topk(*args, k, g)
        torch.cuda.synchronize()
        assert torch.equal(got, want)


def test_index_topk_noalloc_rejects_oversized_calls():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = csa.load()
    g = csa.geom()
    Q, N = 64, 40000  # 64 x 40000 FP32 scores alone exceed the fixed buffer
    assert lib.csa_index_topk_workspace_size(Q, N, 1024) > (8 << 20)
    idx = torch.zeros(Q, 1024, dtype=torch.int32, device="cuda")
    dummy = torch.zeros(16, dtype=torch.uint8, device="cuda")
    p = ctypes.c_void_p(dummy.data_ptr())
    st = lib.csa_index_topk_noalloc(ctypes.byref(g), csa.CSA_BF16, p, p, p, N, 1, p, p, p, Q, 64,
                                    128, 1024, ctypes.c_void_p(idx.data_ptr()), None, None)
    assert st == 5 and lib.csa_status_string(st) == b"CSA_ERR_TOO_LARGE"
