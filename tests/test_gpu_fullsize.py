"""Parity at the workloads' full sizes, in the launch configurations the
benchmark times, on outputs the FP64 oracle can compute one by one.

Each stage gets its own seeded inputs of the workload's shape (stage inputs
are never taken from another GPU stage): sampled compressed entries, sampled
index/top-k queries (margin rule, and the kernel's own scores select exactly
its set), sampled attention queries with synthetic top-k index sets."""
import math

import numpy as np
import pytest
import torch

import compressed_sparse_attention_17_b200 as csa
from compressed_sparse_attention_17_b200 import synth
from gpu_helpers import TOL, dev, dev_i, exact_topk_of, host, max_abs, topk_margin_check

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    csa.load()
    yield
    csa.sync_status()


def _bf16_dev(spec: synth.Spec):
    t = torch.from_numpy(spec.storage())
    return (t.view(torch.int16).view(torch.bfloat16) if spec.dtype == "bf16" else t).cuda()


def _sample(rg, n, count, must=()):
    s = set(int(x) for x in must if 0 <= x < n)
    s |= set(int(x) for x in rg.choice(n, size=min(count, n), replace=False))
    return np.array(sorted(s), dtype=np.int64)


@pytest.mark.parametrize("wl", ["csa_prefill_bf16", "hca_prefill_bf16"])
def test_compress_full_size(orc, wl):
    """Entries of the full prefill compressor, sampled blocks vs the oracle."""
    w = synth.WORKLOADS[wl]()
    s = w.specs()
    rg = np.random.default_rng(1)
    if w.kind == "csa_prefill":
        names = ("W_aKV", "W_aZ", "W_bKV", "W_bZ")
        g = csa.geom(m=w.m, overlap=1, c=w.c, rope_dims=w.rope_dims)
    else:
        names = ("W_KV", "W_Z")
        g = csa.geom(m=w.m, overlap=0, c=w.c, rope_dims=w.rope_dims)
    H = _bf16_dev(s["H"])
    Wd = {n: _bf16_dev(s[n]) for n in names}
    bias = _bf16_dev(s["bias"])
    if w.kind == "csa_prefill":
        E = csa.compress(H, Wd["W_aKV"], Wd["W_aZ"], bias, g, W_bKV=Wd["W_bKV"], W_bZ=Wd["W_bZ"])
    else:
        E = csa.compress(H, Wd["W_KV"], Wd["W_Z"], bias, g)
    nb = w.T // w.m
    blocks = _sample(rg, nb, 24, must=(0, 1, 30, 31, 32, nb - 1))
    # compact sequence for the oracle: each sampled block (after its
    # predecessor, for CSA) becomes one block of a short sequence; the pooled
    # rows are then normalised and rotated at the true positions b*m
    Wh = {n: s[n].values() for n in names}
    order, pick = [], []
    for b in blocks:
        if w.kind == "csa_prefill" and b >= 1:
            order += [b - 1, b]
        else:
            order += [b]
        pick.append(len(order) - 1)
    rows = np.concatenate([np.arange(b * w.m, (b + 1) * w.m) for b in order])
    Hc = s["H"].rows(rows)
    if w.kind == "csa_prefill":
        _, pooled = orc.compress(Hc, Wh["W_aKV"], Wh["W_aZ"], s["bias"].values(), w.m,
                                 W_bKV=Wh["W_bKV"], W_bZ=Wh["W_bZ"], return_pooled=True)
        # a compact block whose true predecessor is absent (true block 0) has
        # no b-series: it sits at compact index 0 when sampled
    else:
        _, pooled = orc.compress(Hc, Wh["W_KV"], Wh["W_Z"], s["bias"].values(), w.m,
                                 return_pooled=True)
    want = orc.rmsnorm_rope(pooled[pick], blocks * w.m, w.rope_dims)
    assert E.shape[0] == nb
    assert max_abs(host(E[torch.from_numpy(blocks).cuda()]), want) <= TOL["bf16"]


def test_index_topk_prefill_full_size(orc):
    """Index + top-k over T=8192 queries x 2048 entries (k=1024)."""
    w = synth.csa_prefill_bf16()
    s = w.specs()
    nb = w.T // w.m
    KIs = synth.Spec("KI_full", (1, nb, w.c_I), 1.0, "bf16", w.seed)
    qI, wv, KI = _bf16_dev(s["qI"]), _bf16_dev(s["w"]), _bf16_dev(KIs)
    pos = torch.arange(w.T, dtype=torch.int64, device="cuda")
    seq = torch.zeros(w.T, dtype=torch.int32, device="cuda")
    ne = torch.tensor([nb], dtype=torch.int64, device="cuda")
    idx, sc = csa.index_topk(qI, wv, KI, seq, pos, ne, w.k, csa.geom(), want_scores=True)
    rg = np.random.default_rng(2)
    qs = _sample(rg, w.T, 40, must=(0, 3, 4, 4095, 4096, 4099, w.T - 1))
    ref = orc.index_topk(s["qI"].rows(np.concatenate([np.arange(q * 64, q * 64 + 64) for q in qs]))
                         .reshape(len(qs), 64, w.c_I), s["w"].rows(qs), KIs.values(),
                         np.zeros(len(qs)), qs, [nb], m=w.m, k=w.k, want_scores=True)
    idx_h, sc_h = idx.cpu().numpy()[qs], sc.cpu().numpy()[qs]
    for i, q in enumerate(qs):
        nv = orc.visible_entries(q, w.m, 1, nb)
        topk_margin_check(idx_h[i], ref["scores"][i], nv, w.k, ref["tau"][i], ref["amag"][i])
        np.testing.assert_array_equal(idx_h[i], exact_topk_of(sc_h[i], nv, w.k))


@pytest.mark.parametrize("wl", ["csa_decode_bf16", "csa_decode_long_mixed"])
def test_index_topk_decode_full_size(orc, wl):
    """Decode indexer over every visible entry of every sequence."""
    w = synth.WORKLOADS[wl]()
    s = w.specs()
    N = w.n_entries
    KI = torch.zeros(w.B, N + 8, w.c_I, dtype=torch.bfloat16, device="cuda")
    KI[:, :N] = _bf16_dev(s["KI"])
    qI, wv = _bf16_dev(s["qI"]), _bf16_dev(s["w"])
    pos = torch.full((w.B,), w.L, dtype=torch.int64, device="cuda")
    seq = torch.arange(w.B, dtype=torch.int32, device="cuda")
    ne = torch.full((w.B,), N, dtype=torch.int64, device="cuda")
    idx, sc = csa.index_topk(qI, wv, KI, seq, pos, ne, w.k, csa.geom(), want_scores=True)
    idx_h, sc_h = idx.cpu().numpy(), sc.cpu().numpy()
    qsel = list(range(w.B)) if w.B <= 4 else [0, 1, 17, w.B - 1]
    KIsel = np.stack([s["KI"].rows(np.arange(b * N, (b + 1) * N)) for b in qsel])
    ref = orc.index_topk(s["qI"].values()[qsel], s["w"].values()[qsel], KIsel,
                         np.arange(len(qsel)), np.full(len(qsel), w.L), np.full(len(qsel), N),
                         m=w.m, k=w.k, want_scores=True)
    for i, b in enumerate(qsel):
        topk_margin_check(idx_h[b], ref["scores"][i], N, w.k, ref["tau"][i], ref["amag"][i])
        np.testing.assert_array_equal(idx_h[b], exact_topk_of(sc_h[b], N, w.k))


def _prepared(orc, raw_rows, positions, r):
    return orc.rmsnorm_rope(raw_rows, positions, r)


@pytest.mark.parametrize("wl", ["csa_decode_bf16", "csa_decode_long_mixed"])
def test_attend_decode_full_size(orc, wl):
    """Decode attention over 1024 selected entries + the 128-row ring for
    every sequence of the workload (synthetic index sets)."""
    w = synth.WORKLOADS[wl]()
    s = w.specs()
    N, c, r = w.n_entries, w.c, w.rope_dims
    rg = np.random.default_rng(3)
    idx = np.stack([np.sort(rg.choice(N, w.k, replace=False)) for _ in range(w.B)]).astype(np.int32)
    raw = _bf16_dev(s["E_raw"])  # stored rows, used as they are (an attention input)
    if w.kv_mixed:
        E = torch.zeros(w.B, N + 8, csa.MIXED_ROW_BYTES, dtype=torch.uint8, device="cuda")
        for b in range(w.B):
            E[b, :N] = csa.quantize_mixed(raw[b])
    else:
        E = torch.zeros(w.B, N + 8, c, dtype=torch.bfloat16, device="cuda")
        E[:, :N] = raw
    del raw
    ring = _bf16_dev(s["win_raw"])
    q, sink = _bf16_dev(s["q"]), _bf16_dev(s["sink"])
    pos = torch.full((w.B,), w.L, dtype=torch.int64, device="cuda")
    seq = torch.arange(w.B, dtype=torch.int32, device="cuda")
    ne = torch.full((w.B,), N, dtype=torch.int64, device="cuda")
    g = csa.geom(win_ring=1)
    O = host(csa.attend(q, sink, E, torch.from_numpy(idx).cuda(), ring, seq, pos, ne, g))
    qsel = list(range(w.B)) if w.B <= 4 else [0, 5, 17, w.B - 1]
    for b in qsel:
        rows = s["E_raw"].rows(b * N + idx[b].astype(np.int64))
        if w.kv_mixed:
            rows = orc.unpack_mixed(orc.pack_mixed(rows))
        # only the selected rows, renumbered 0..k-1 in the same order
        want = orc.attend(s["q"].values()[b:b + 1], s["sink"].values(), rows[None],
                          s["win_raw"].values()[b:b + 1], [0], [w.L], [w.k], rope_dims=r,
                          idx=np.arange(w.k, dtype=np.int32)[None], win_ring=1)
        assert max_abs(O[b:b + 1], want) <= TOL["bf16"]


def test_attend_prefill_full_size(orc):
    """CSA prefill attention, T=8192 queries x (<=1024 selected + window)."""
    w = synth.csa_prefill_bf16()
    s = w.specs()
    nb, c, r = w.T // w.m, w.c, w.rope_dims
    Es = synth.Spec("E_full", (1, nb, c), 1.0, "bf16", w.seed)
    rg = np.random.default_rng(4)
    pos = np.arange(w.T)
    nv = np.array([orc.visible_entries(p, w.m, 1, nb) for p in pos])
    idx = synth.random_topk_indices(rg, nv, w.k)
    q, sink, win, E = _bf16_dev(s["q"]), _bf16_dev(s["sink"]), _bf16_dev(s["kv_win"]), _bf16_dev(Es)
    O = csa.attend(q, sink, E, torch.from_numpy(idx).cuda(), win[None].contiguous(),
                   torch.zeros(w.T, dtype=torch.int32, device="cuda"),
                   torch.arange(w.T, dtype=torch.int64, device="cuda"),
                   torch.tensor([nb], dtype=torch.int64, device="cuda"), csa.geom())
    qs = _sample(rg, w.T, 12, must=(0, 1, 127, 128, 4096, w.T - 1))
    Oh = host(O[torch.from_numpy(qs).cuda()])
    want = orc.attend(s["q"].rows(np.concatenate([np.arange(p * 64, p * 64 + 64) for p in qs]))
                      .reshape(len(qs), 64, c), s["sink"].values(), Es.values(),
                      s["kv_win"].values()[None], np.zeros(len(qs)), qs, [nb], rope_dims=r,
                      idx=idx[qs])
    assert max_abs(Oh, want) <= TOL["bf16"]


def test_hca_attend_full_size(orc):
    """HCA prefill attention, T=65536 queries over <=512 entries + window."""
    w = synth.hca_prefill_bf16()
    s = w.specs()
    nb, c, r = w.T // w.m, w.c, w.rope_dims
    Es = synth.Spec("E_hca_full", (1, nb, c), 1.0, "bf16", w.seed)
    q, sink, win, E = _bf16_dev(s["q"]), _bf16_dev(s["sink"]), _bf16_dev(s["kv_win"]), _bf16_dev(Es)
    g = csa.geom(m=w.m, overlap=0)
    O = csa.hca_attend(q, sink, E, win[None].contiguous(),
                       torch.zeros(w.T, dtype=torch.int32, device="cuda"),
                       torch.arange(w.T, dtype=torch.int64, device="cuda"),
                       torch.tensor([nb], dtype=torch.int64, device="cuda"), g)
    rg = np.random.default_rng(5)
    qs = _sample(rg, w.T, 10, must=(0, 126, 127, 128, 255, 32768, w.T - 1))
    Oh = host(O[torch.from_numpy(qs).cuda()])
    want = orc.attend(s["q"].rows(np.concatenate([np.arange(p * 64, p * 64 + 64) for p in qs]))
                      .reshape(len(qs), 64, c), s["sink"].values(), Es.values(),
                      s["kv_win"].values()[None], np.zeros(len(qs)), qs, [nb], rope_dims=r, m=w.m)
    assert max_abs(Oh, want) <= TOL["bf16"]
