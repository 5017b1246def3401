"""GPU parity: every C-ABI entry point against the FP64 oracle on the same
seeded inputs, at sizes that span several tiles and a ragged tail.

Bars: integer / index work bit-exact (top-k sets on integer inputs, FP8
codes); FP32 paths max-abs <= 1e-4; BF16 paths max-abs <= 2e-2; top-k on
real-valued inputs by the margin rule (tests/gpu_helpers.py)."""
import math

import numpy as np
import pytest
import torch

import compressed_sparse_attention_17_b200 as csa
from compressed_sparse_attention_17_b200 import synth
from gpu_helpers import (TOL, dev, dev_i, exact_topk_of, host, max_abs, topk_margin_check)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    csa.load()
    yield
    csa.sync_status()


def _spec(name, shape, std=1.0, dtype="bf16", seed=11):
    return synth.Spec(name, shape, std, dtype, seed)


# ------------------------------------------------------------------ rows
@pytest.mark.parametrize("dt,c,r", [("f32", 128, 32), ("bf16", 512, 64), ("bf16", 32, 0),
                                    ("f32", 512, 64)])
def test_rmsnorm_rope(orc, dt, c, r):
    rows = 301
    x = _spec("x", (rows, c), 2.0, dt).values()
    # a gain near one keeps outputs in the range where BF16 rounding is below the tolerance
    gain = 1.0 + 0.1 * _spec("g", (c,), 1.0, "f32").values()
    pos = np.random.default_rng(1).integers(0, 1 << 20, rows)
    g = csa.geom(c=c, rope_dims=r)
    out = csa.rmsnorm_rope(dev(x, dt), g, pos=dev_i(pos), gain=dev(gain, "f32"))
    want = orc.rmsnorm_rope(x, pos, r, gain=gain)
    assert max_abs(host(out), want) <= TOL[dt]
    # affine positions: entry i at position 4 i
    out2 = csa.rmsnorm_rope(dev(x, dt), g, pos0=0, pos_step=4)
    assert max_abs(host(out2), orc.rmsnorm_rope(x, np.arange(rows) * 4, r)) <= TOL[dt]


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_quantize_mixed_codes_bit_exact(orc, dt):
    x = _spec("xm", (257, 512), 3.0, dt).values()
    x[5, :448] = 0.0  # all-zero FP8 part: scale 0, zero codes
    x[7, 10] = 1e-3   # subnormal codes
    got = csa.quantize_mixed(dev(x, dt)).cpu().numpy()
    want = orc.pack_mixed(x)
    np.testing.assert_array_equal(got, want)


def test_rmsnorm_rope_to_mixed_rows(orc):
    x = _spec("xr", (130, 512), 1.0, "bf16").values()
    g = csa.geom()
    rows = csa.rmsnorm_rope(dev(x, "bf16"), g, pos0=0, pos_step=4,
                            out_dtype=csa.CSA_FP8_MIXED).cpu().numpy()
    got = orc.unpack_mixed(rows)
    want = orc.rmsnorm_rope(x, np.arange(130) * 4, 64)
    scale = np.abs(want[:, :448]).max(1, keepdims=True) / 448
    # E4M3 keeps 3 mantissa bits: half-ulp <= 2^-4 relative (2^-10 scale below normals)
    bound = np.abs(want[:, :448]) * 2.0 ** -4 + scale * 2.0 ** -9 + 1e-5
    assert (np.abs(got[:, :448] - want[:, :448]) <= bound).all()
    assert max_abs(got[:, 448:], want[:, 448:]) <= TOL["bf16"]


# ------------------------------------------------------------------ compressor
def _compress_case(w: synth.Workload, index_keys=False):
    s = w.specs()
    pre = "WI_" if index_keys else "W_"
    names = [pre + n for n in ("aKV", "bKV", "aZ", "bZ")]
    W = {n[len(pre):]: s[n].values() for n in names}
    bias = s["biasI" if index_keys else "bias"].values()
    return s["H"].values(), W, bias


@pytest.mark.parametrize("which", ["tiny_main", "tiny_index", "bf16_main", "bf16_index"])
def test_compress_csa(orc, which):
    if which.startswith("tiny"):
        w = synth.tiny_csa_fp32()
    else:
        w = synth.csa_prefill_bf16(T=1102, d=512)  # ragged: 275 entries, 2 tokens left over
    index_keys = which.endswith("index")
    H, W, bias = _compress_case(w, index_keys)
    c = w.c_I if index_keys else w.c
    r = 0 if index_keys else w.rope_dims
    g = csa.geom(m=w.m, overlap=1, c=c, rope_dims=r)
    d = lambda a: dev(a, w.dtype)
    E = csa.compress(d(H), d(W["aKV"]), d(W["aZ"]), dev(bias, "f32"), g, W_bKV=d(W["bKV"]),
                     W_bZ=d(W["bZ"]))
    want = orc.compress(H, W["aKV"], W["aZ"], bias, w.m, W_bKV=W["bKV"], W_bZ=W["bZ"],
                        rope_dims=r)
    assert E.shape[0] == w.T // w.m
    assert max_abs(host(E), want) <= TOL[w.dtype]


def test_compress_hca(orc):
    w = synth.hca_prefill_bf16(T=1000, d=256)
    s = w.specs()
    H, Wkv, Wz, bias = (s[n].values() for n in ("H", "W_KV", "W_Z", "bias"))
    g = csa.geom(m=128, overlap=0)
    E = csa.compress(dev(H, "bf16"), dev(Wkv, "bf16"), dev(Wz, "bf16"), dev(bias, "f32"), g)
    want = orc.compress(H, Wkv, Wz, bias, 128, rope_dims=64)
    assert E.shape[0] == 7
    assert max_abs(host(E), want) <= TOL["bf16"]


def test_compress_mixed_output(orc):
    w = synth.csa_prefill_bf16(T=260, d=256)
    H, W, bias = _compress_case(w)
    g = csa.geom()
    d = lambda a: dev(a, "bf16")
    rows = csa.compress(d(H), d(W["aKV"]), d(W["aZ"]), dev(bias, "f32"), g, W_bKV=d(W["bKV"]),
                        W_bZ=d(W["bZ"]), out_dtype=csa.CSA_FP8_MIXED).cpu().numpy()
    got = orc.unpack_mixed(rows)
    want = orc.compress(H, W["aKV"], W["aZ"], bias, 4, W_bKV=W["bKV"], W_bZ=W["bZ"],
                        rope_dims=64)
    scale = np.abs(want[:, :448]).max(1, keepdims=True) / 448
    bound = np.abs(want[:, :448]) * 2.0 ** -4 + scale * 2.0 ** -9 + 1e-4
    assert (np.abs(got[:, :448] - want[:, :448]) <= bound).all()
    assert max_abs(got[:, 448:], want[:, 448:]) <= TOL["bf16"]


@pytest.mark.parametrize("kind", ["csa_f32", "csa_bf16", "hca_bf16"])
def test_compress_decode_matches_prefill_oracle(orc, kind):
    """Feeding tokens one at a time through the decode compressor yields the
    entries the oracle computes from the whole sequence."""
    B = 3
    if kind == "hca_bf16":
        m, overlap, c, r, d, T, dt = 128, 0, 512, 64, 128, 384, "bf16"
    elif kind == "csa_bf16":
        m, overlap, c, r, d, T, dt = 4, 1, 512, 64, 256, 48, "bf16"
    else:
        m, overlap, c, r, d, T, dt = 4, 1, 128, 32, 64, 40, "f32"
    nW = 4 if overlap else 2
    H = _spec("Hd", (B, T, d), 1.0, dt).values()
    Ws = [_spec(f"Wd{i}", (d, c), 1 / math.sqrt(d), dt).values() for i in range(nW)]
    bias = _spec("bd", ((1 + overlap) * m, c), 0.3, "f32").values()
    g = csa.geom(m=m, overlap=overlap, c=c, rope_dims=r)
    state = csa.decode_state(B, g)
    E = torch.zeros(B, T // m + 2, c, dtype=torch.float32 if dt == "f32" else torch.bfloat16,
                    device="cuda")
    Wd = [dev(x, dt) for x in Ws]
    Hd = dev(H, dt)
    for t in range(T):
        pos = torch.full((B,), t, dtype=torch.int64, device="cuda")
        h = Hd[:, t].contiguous()
        if overlap:
            csa.compress_decode(h, pos, Wd[0], Wd[2], dev(bias, "f32"), state, E, g, W_bKV=Wd[1],
                                W_bZ=Wd[3])
        else:
            csa.compress_decode(h, pos, Wd[0], Wd[1], dev(bias, "f32"), state, E, g)
    got = host(E)
    for b in range(B):
        if overlap:
            want = orc.compress(H[b], Ws[0], Ws[2], bias, m, W_bKV=Ws[1], W_bZ=Ws[3], rope_dims=r)
        else:
            want = orc.compress(H[b], Ws[0], Ws[1], bias, m, rope_dims=r)
        assert max_abs(got[b, :T // m], want) <= TOL[dt]
        assert np.abs(got[b, T // m:]).max() == 0.0  # no entry past the last complete block


# ------------------------------------------------------------------ indexer
def _index_inputs(Q, HI, cI, nseq, N, dt, integer=False, seed=0):
    rg = np.random.default_rng(seed)
    if integer:
        qI = rg.integers(-2, 3, (Q, HI, cI)).astype(np.float32)
        KI = rg.integers(-2, 3, (nseq, N, cI)).astype(np.float32)
        w = rg.integers(-3, 4, (Q, HI)).astype(np.float32)
    else:
        qI = _spec("qI", (Q, HI, cI), 1.0, dt, seed).values()
        KI = _spec("KI", (nseq, N, cI), 1.0, dt, seed).values()
        w = _spec("w", (Q, HI), 1.0, "f32", seed).values()
    seq = rg.integers(0, nseq, Q).astype(np.int32)
    ne = np.array([N - 37 * b for b in range(nseq)], np.int64)
    pos = rg.integers(0, 4 * N + 16, Q).astype(np.int64)
    pos[:4] = [0, 2, 3, 4 * N + 3][:4]
    return qI, w, KI, seq, pos, ne


def _run_index(qI, w, KI, seq, pos, ne, k, dt, m=4, want_scores=False, vis_offset=1):
    g = csa.geom(m=m, vis_offset=vis_offset)
    return csa.index_topk(dev(qI, dt), dev(w, "f32"), dev(KI, dt), dev_i(seq, torch.int32),
                          dev_i(pos), dev_i(ne), k, g, want_scores=want_scores)


@pytest.mark.parametrize("dt,HI,cI", [("f32", 4, 32), ("bf16", 64, 128), ("bf16", 8, 64)])
def test_index_topk_integer_inputs_bit_exact(orc, dt, HI, cI):
    qI, w, KI, seq, pos, ne = _index_inputs(40, HI, cI, 3, 700, dt, integer=True, seed=3)
    for vo in (1, 0):
        idx = _run_index(qI, w, KI, seq, pos, ne, 64, dt, vis_offset=vo).cpu().numpy()
        want = orc.index_topk(qI, w, KI, seq, pos, ne, m=4, k=64, vis_offset=vo)["idx"]
        np.testing.assert_array_equal(idx, want)


@pytest.mark.parametrize("dt,HI,cI,k", [("f32", 4, 32, 32), ("bf16", 64, 128, 256),
                                        ("bf16", 64, 128, 2048)])
def test_index_topk_margin_rule(orc, dt, HI, cI, k):
    qI, w, KI, seq, pos, ne = _index_inputs(24, HI, cI, 2, 1000, dt, seed=4)
    idx, sc = _run_index(qI, w, KI, seq, pos, ne, k, dt, want_scores=True)
    idx, sc = idx.cpu().numpy(), sc.cpu().numpy()
    ref = orc.index_topk(qI, w, KI, seq, pos, ne, m=4, k=k, want_scores=True)
    in_band = 0
    for q in range(len(pos)):
        nv = orc.visible_entries(pos[q], 4, 1, ne[seq[q]])
        in_band += topk_margin_check(idx[q], ref["scores"][q], nv, k, ref["tau"][q],
                                     ref["amag"][q])
        # the kernel's own FP32 scores select exactly the kernel's set
        np.testing.assert_array_equal(idx[q], exact_topk_of(sc[q], nv, k))
        assert max_abs(sc[q, :nv], ref["scores"][q, :nv]) <= 2.0 ** -14 * ref["amag"][q] + 1e-6
    print("entries inside the rounding band:", in_band)


@pytest.mark.parametrize("HI,cI", [(64, 128), (16, 64)])
def test_index_topk_grouped_queries(orc, HI, cI):
    """Many queries per call: queries are processed in groups that share an
    entry tile; groups that straddle two sequences are split into passes."""
    Q, N, k = 1100, 520, 128  # more queries than the persistent decode kernel takes
    rg = np.random.default_rng(12)
    qI = _spec("qIg", (Q, HI, cI), 1.0, "bf16").values()
    KI = _spec("KIg", (2, N, cI), 1.0, "bf16").values()
    w = _spec("wg", (Q, HI), 1.0, "f32").values()
    seq = np.zeros(Q, np.int32)
    seq[600:] = rg.integers(0, 2, Q - 600)
    pos = np.sort(rg.integers(0, 4 * N, Q)).astype(np.int64)
    ne = np.array([N, N - 100])
    idx, sc = _run_index(qI, w, KI, seq, pos, ne, k, "bf16", want_scores=True)
    idx, sc = idx.cpu().numpy(), sc.cpu().numpy()
    ref = orc.index_topk(qI, w, KI, seq, pos, ne, m=4, k=k, want_scores=True)
    for q in range(Q):
        nv = orc.visible_entries(pos[q], 4, 1, ne[seq[q]])
        topk_margin_check(idx[q], ref["scores"][q], nv, k, ref["tau"][q], ref["amag"][q])
        np.testing.assert_array_equal(idx[q], exact_topk_of(sc[q], nv, k))
        assert max_abs(sc[q, :nv], ref["scores"][q, :nv]) <= 2.0 ** -14 * ref["amag"][q] + 1e-6


@pytest.mark.parametrize("dt,HI,cI,Q,nseq", [("bf16", 64, 128, 300, 1), ("bf16", 64, 128, 40, 3),
                                           ("f32", 4, 32, 40, 3)])
def test_index_scores_integer_inputs_bit_exact(orc, dt, HI, cI, Q, nseq):
    """csa_index_scores alone: integer inputs make every score exact, so the
    visible slots equal the oracle's scores; grouped queries (one sequence),
    single queries and the CUDA-core path."""
    qI, w, KI, seq, pos, ne = _index_inputs(Q, HI, cI, nseq, 700, dt, integer=True, seed=31)
    g = csa.geom(m=4, vis_offset=1)
    sc = csa.index_scores(dev(qI, dt), dev(w, "f32"), dev(KI, dt), dev_i(seq, torch.int32),
                          dev_i(pos), dev_i(ne), g).cpu().numpy()
    ref = orc.index_topk(qI, w, KI, seq, pos, ne, m=4, k=8, want_scores=True)["scores"]
    for q in range(Q):
        nv = orc.visible_entries(pos[q], 4, 1, ne[seq[q]])
        np.testing.assert_array_equal(sc[q, :nv], ref[q, :nv])
        assert np.isnan(sc[q, nv:]).all()


@pytest.mark.parametrize("Q", [257, 2501])
def test_index_topk_single_sequence_groups_bit_exact(orc, Q):
    """One sequence, many queries (the prefill shape): queries are scored in
    groups of four that share each entry tile. Unsorted positions give the
    members of a group different visible counts (some none); Q is not a
    multiple of four; 257 queries split the units into contiguous ranges,
    2501 deal whole groups to CTAs in turn. Integer inputs make every score
    exact, so the selected sets must equal the oracle's."""
    N, k = 300, 64
    qI, w, KI, seq, pos, ne = _index_inputs(Q, 64, 128, 1, N, "bf16", integer=True, seed=21)
    rg = np.random.default_rng(22)
    pos[:] = rg.integers(0, 4 * N + 16, Q)
    pos[:6] = [0, 3, 4, 4 * N + 3, 2, 1]
    idx = _run_index(qI, w, KI, seq, pos, ne, k, "bf16").cpu().numpy()
    want = orc.index_topk(qI, w, KI, seq, pos, ne, m=4, k=k)["idx"]
    np.testing.assert_array_equal(idx, want)


@pytest.mark.parametrize("k", [1024, 300])
def test_index_topk_many_entries_bit_exact(orc, k):
    """More visible entries than one selection block holds: chunk top-k
    candidates are merged; integer inputs make the result exact."""
    qI, w, KI, seq, pos, ne = _index_inputs(6, 16, 64, 2, 21000, "bf16", integer=True, seed=8)
    pos[:] = [4 * 21000, 4 * 21000 + 7, 4 * 9000, 4 * 16384 - 1, 4 * 16384, 5]
    idx = _run_index(qI, w, KI, seq, pos, ne, k, "bf16").cpu().numpy()
    want = orc.index_topk(qI, w, KI, seq, pos, ne, m=4, k=k)["idx"]
    np.testing.assert_array_equal(idx, want)


@pytest.mark.parametrize("N,k", [(1500, 700), (40000, 1024), (70000, 512)])
def test_index_topk_equal_scores(orc, N, k):
    """Zero indexer queries make every score 0: all visible entries tie and
    the lowest k_eff indices are kept. One bin then holds every key, so the
    exact ranking of that bin (1,500 entries), the radix selection over a
    whole multi-CTA row (40,000) and chunked rows (70,000) all run."""
    qI, w, KI, seq, pos, ne = _index_inputs(6, 4, 32, 2, N, "f32", integer=True, seed=11)
    qI[:] = 0.0
    pos[:] = [4 * N + 3, 4 * k - 1, 4 * k + 3, 4 * (N // 2), 7, 4 * N - 9]
    idx = _run_index(qI, w, KI, seq, pos, ne, k, "f32").cpu().numpy()
    want = orc.index_topk(qI, w, KI, seq, pos, ne, m=4, k=k)["idx"]
    np.testing.assert_array_equal(idx, want)
    for q in range(len(pos)):
        nv = orc.visible_entries(pos[q], 4, 1, ne[seq[q]])
        ke = min(k, nv)
        np.testing.assert_array_equal(idx[q, :ke], np.arange(ke))
        assert (idx[q, ke:] == -1).all()


def test_index_topk_no_visible_entries(orc):
    qI, w, KI, seq, pos, ne = _index_inputs(8, 4, 32, 1, 50, "f32", seed=5)
    pos[:] = [0, 1, 2, 3, 4, 5, 6, 7]
    idx = _run_index(qI, w, KI, seq, pos, ne, 8, "f32").cpu().numpy()
    want = orc.index_topk(qI, w, KI, seq, pos, ne, m=4, k=8)["idx"]
    np.testing.assert_array_equal(idx, want)
    assert (idx[:3] == -1).all()


# ------------------------------------------------------------------ attention
def _attend_case(orc, Q, Hq, c, r, nseq, N, k, dt, kv="same", ring=False, seed=7, hole=0.1):
    rg = np.random.default_rng(seed)
    q = _spec("q", (Q, Hq, c), 1.0, dt, seed).values()
    E = _spec("E", (nseq, N, c), 1.0, "bf16" if kv == "mixed" else dt, seed).values()
    ldW = 128 if ring else 4 * N + 200
    win = _spec("win", (nseq, ldW, c), 1.0, "bf16" if kv == "mixed" else dt, seed).values()
    sink = _spec("sink", (Hq,), 1.0, "f32", seed).values()
    gain = 1.0 + 0.1 * _spec("qg", (c,), 1.0, "f32", seed).values()
    seq = rg.integers(0, nseq, Q).astype(np.int32)
    ne = np.array([N - 5 * b for b in range(nseq)], np.int64)
    pos = rg.integers(0, 4 * N + 100, Q).astype(np.int64)
    pos[:3] = [0, 1, 130][:Q if Q < 3 else 3]
    nv = np.array([orc.visible_entries(p, 4, 1, ne[s]) for p, s in zip(pos, seq)])
    idx = synth.random_topk_indices(rg, nv, k, hole_frac=hole)
    return q, E, win, sink, gain, seq, ne, pos, idx


@pytest.mark.parametrize("dt,Hq,c,r,k,ring", [("f32", 8, 128, 32, 32, False),
                                               ("bf16", 64, 512, 64, 96, True),
                                               ("bf16", 16, 256, 64, 40, False)])
def test_csa_attend(orc, dt, Hq, c, r, k, ring):
    q, E, win, sink, gain, seq, ne, pos, idx = _attend_case(orc, 13, Hq, c, r, 3, 300, k, dt, ring=ring)
    g = csa.geom(c=c, rope_dims=r, win_ring=int(ring))
    O = csa.attend(dev(q, dt), dev(sink, "f32"), dev(E, dt), dev_i(idx, torch.int32), dev(win, dt),
                   dev_i(seq, torch.int32), dev_i(pos), dev_i(ne), g, q_gain=dev(gain, "f32"))
    want = orc.attend(q, sink, E, win, seq, pos, ne, rope_dims=r, idx=idx, win_ring=int(ring),
                      q_gain=gain)
    assert max_abs(host(O), want) <= TOL[dt]


@pytest.mark.parametrize("dt,m", [("bf16", 128), ("f32", 4)])
def test_hca_attend(orc, dt, m):
    Q, Hq, c, r, N = 11, 8, 256, 64, 40
    q, E, win, sink, gain, seq, ne, pos, _ = _attend_case(orc, Q, Hq, c, r, 2, N, 8, dt)
    pos = np.random.default_rng(9).integers(0, m * N + 50, Q).astype(np.int64)
    pos[0] = 0
    ldW = win.shape[1]
    win = _spec("win2", (2, max(ldW, int(pos.max()) + 1), c), 1.0, dt).values()
    g = csa.geom(m=m, overlap=0, c=c, rope_dims=r)
    O = csa.hca_attend(dev(q, dt), dev(sink, "f32"), dev(E, dt), dev(win, dt),
                       dev_i(seq, torch.int32), dev_i(pos), dev_i(ne), g)
    want = orc.attend(q, sink, E, win, seq, pos, ne, rope_dims=r, m=m)
    assert max_abs(host(O), want) <= TOL[dt]


@pytest.mark.parametrize("Q,k,hole", [(80, 1024, 0.05), (20, 300, 0.3)])
def test_csa_attend_tensor_core_paths(orc, Q, k, hole):
    """64 heads x 512 in BF16 run on the tensor-core kernel: many queries use
    one CTA per query, few queries split the keys over CTAs and merge."""
    Hq, c, r, N = 64, 512, 64, 1500
    q, E, win, sink, gain, seq, ne, pos, idx = _attend_case(orc, Q, Hq, c, r, 2, N, k, "bf16",
                                                            ring=False, seed=21, hole=hole)
    g = csa.geom(c=c, rope_dims=r)
    O = csa.attend(dev(q, "bf16"), dev(sink, "f32"), dev(E, "bf16"), dev_i(idx, torch.int32),
                   dev(win, "bf16"), dev_i(seq, torch.int32), dev_i(pos), dev_i(ne), g,
                   q_gain=dev(gain, "f32"))
    want = orc.attend(q, sink, E, win, seq, pos, ne, rope_dims=r, idx=idx, q_gain=gain)
    assert max_abs(host(O), want) <= TOL["bf16"]


def test_csa_attend_batch_invariance(orc):
    """A query's output does not depend on the batch it is in: alone, inside
    a batch of 32 and inside a permuted batch it gives the same bits."""
    Q, Hq, c, r, N, k = 32, 64, 512, 64, 1500, 1024
    q, E, win, sink, gain, seq, ne, pos, idx = _attend_case(orc, Q, Hq, c, r, 4, N, k, "bf16",
                                                            seed=41, hole=0.02)
    g = csa.geom(c=c, rope_dims=r)
    dE, dwin, dsink, dgain, dne = dev(E, "bf16"), dev(win, "bf16"), dev(sink, "f32"), dev(gain, "f32"), dev_i(ne)

    def run(sel):
        return host(csa.attend(dev(q[sel], "bf16"), dsink, dE, dev_i(idx[sel], torch.int32), dwin,
                               dev_i(seq[sel], torch.int32), dev_i(pos[sel]), dne, g, q_gain=dgain))

    full = run(np.arange(Q))
    perm = np.random.default_rng(3).permutation(Q)
    np.testing.assert_array_equal(run(perm), full[perm])
    for i in (0, 5, 31):
        np.testing.assert_array_equal(run(np.array([i]))[0], full[i])
    want = orc.attend(q, sink, E, win, seq, pos, ne, rope_dims=r, idx=idx, q_gain=gain)
    assert max_abs(full, want) <= TOL["bf16"]


def test_csa_attend_rescale_across_tiles(orc):
    """Window rows four times larger than the selected entries: the logits of
    the last key tiles exceed the running reference by far, so the output
    accumulated over the earlier tiles is rescaled part-way.

    Outputs here reach about 9, where one BF16 output ulp is already 0.06 and
    logits of standard deviation 4 magnify the BF16 rounding of Qhat and of
    the weights in proportion. The bar is the BF16 bar scaled to the output
    magnitude; a missed or wrong rescale errs by the size of the output."""
    Q, Hq, c, r, N, k = 6, 64, 512, 64, 1500, 512
    q, E, win, sink, gain, seq, ne, pos, idx = _attend_case(orc, Q, Hq, c, r, 2, N, k, "bf16",
                                                            seed=43, hole=0.0)
    pos[:] = 4 * N - 1  # every query sees a full selection and a full window
    nv = np.array([orc.visible_entries(p, 4, 1, ne[s]) for p, s in zip(pos, seq)])
    idx = synth.random_topk_indices(np.random.default_rng(44), nv, k, hole_frac=0.0)
    win = win * 4.0  # exact in BF16
    g = csa.geom(c=c, rope_dims=r)
    O = csa.attend(dev(q, "bf16"), dev(sink, "f32"), dev(E, "bf16"), dev_i(idx, torch.int32),
                   dev(win, "bf16"), dev_i(seq, torch.int32), dev_i(pos), dev_i(ne), g,
                   q_gain=dev(gain, "f32"))
    want = orc.attend(q, sink, E, win, seq, pos, ne, rope_dims=r, idx=idx, q_gain=gain)
    assert max_abs(host(O), want) <= TOL["bf16"] * max(1.0, float(np.abs(want).max()))


@pytest.mark.parametrize("Q", [24, 300])
def test_hca_attend_tensor_core_paths(orc, Q):
    Hq, c, r, N, m = 64, 512, 64, 40, 128
    rg = np.random.default_rng(31)
    q = _spec("qh", (Q, Hq, c), 1.0, "bf16", 31).values()
    E = _spec("Eh", (2, N, c), 1.0, "bf16", 31).values()
    sink = _spec("sh", (Hq,), 1.0, "f32", 31).values()
    seq = rg.integers(0, 2, Q).astype(np.int32)
    pos = rg.integers(0, m * N + 300, Q).astype(np.int64)
    pos[:3] = [0, 126, 127]
    ne = np.array([N, N - 3])
    win = _spec("wh", (2, int(pos.max()) + 1, c), 1.0, "bf16", 31).values()
    g = csa.geom(m=m, overlap=0, c=c, rope_dims=r)
    O = csa.hca_attend(dev(q, "bf16"), dev(sink, "f32"), dev(E, "bf16"), dev(win, "bf16"),
                       dev_i(seq, torch.int32), dev_i(pos), dev_i(ne), g)
    want = orc.attend(q, sink, E, win, seq, pos, ne, rope_dims=r, m=m)
    assert max_abs(host(O), want) <= TOL["bf16"]


def test_csa_attend_mixed_entries(orc):
    Q, Hq, c, r, N, k = 9, 64, 512, 64, 200, 64
    q, E, win, sink, gain, seq, ne, pos, idx = _attend_case(orc, Q, Hq, c, r, 2, N, k, "bf16",
                                                            kv="mixed", ring=True)
    rows_gpu = csa.quantize_mixed(dev(E.reshape(-1, 512), "bf16")).reshape(2, N, -1)
    rows_orc = orc.pack_mixed(E.reshape(-1, 512)).reshape(2, N, -1)
    np.testing.assert_array_equal(rows_gpu.cpu().numpy(), rows_orc)
    g = csa.geom(win_ring=1)
    O = csa.attend(dev(q, "bf16"), dev(sink, "f32"), rows_gpu, dev_i(idx, torch.int32),
                   dev(win, "bf16"), dev_i(seq, torch.int32), dev_i(pos), dev_i(ne), g)
    want = orc.attend(q, sink, orc.unpack_mixed(rows_orc), win, seq, pos, ne, rope_dims=r, idx=idx,
                      win_ring=1)
    assert max_abs(host(O), want) <= TOL["bf16"]


# ------------------------------------------------------------------ whole layer, FP32 tiny
def test_tiny_csa_layer_end_to_end(orc):
    """The tiny FP32 workload through compress -> index -> attend, against
    the oracle's own chain. Index sets follow the margin rule; attention
    outputs are compared on every query whose selected set matches the
    oracle's exactly."""
    w = synth.tiny_csa_fp32()
    s = w.specs()
    v = {n: s[n].values() for n in s}
    T, m, k = w.T, w.m, w.k
    d = lambda a: dev(a, "f32")
    gE = csa.geom(c=w.c, rope_dims=w.rope_dims)
    gI = csa.geom(c=w.c_I, rope_dims=0)
    E = csa.compress(d(v["H"]), d(v["W_aKV"]), d(v["W_aZ"]), d(v["bias"]), gE, W_bKV=d(v["W_bKV"]),
                     W_bZ=d(v["W_bZ"]))
    KI = csa.compress(d(v["H"]), d(v["WI_aKV"]), d(v["WI_aZ"]), d(v["biasI"]), gI,
                      W_bKV=d(v["WI_bKV"]), W_bZ=d(v["WI_bZ"]))
    win = csa.rmsnorm_rope(d(v["kv_win"]), gE, pos0=0, pos_step=1)
    pos = np.arange(T)
    seq = np.zeros(T, np.int32)
    ne = np.array([T // m])
    idx = csa.index_topk(d(v["qI"]), d(v["w"]), KI[None].contiguous(), dev_i(seq, torch.int32),
                         dev_i(pos), dev_i(ne), k, gE)
    O = csa.attend(d(v["q"]), d(v["sink"]), E[None].contiguous(), idx, win[None].contiguous(),
                   dev_i(seq, torch.int32), dev_i(pos), dev_i(ne), gE)
    # oracle chain
    Eo = orc.compress(v["H"], v["W_aKV"], v["W_aZ"], v["bias"], m, W_bKV=v["W_bKV"],
                      W_bZ=v["W_bZ"], rope_dims=w.rope_dims)
    KIo = orc.compress(v["H"], v["WI_aKV"], v["WI_aZ"], v["biasI"], m, W_bKV=v["WI_bKV"],
                       W_bZ=v["WI_bZ"])
    wino = orc.rmsnorm_rope(v["kv_win"], pos, w.rope_dims)
    ref = orc.index_topk(v["qI"], v["w"], KIo[None], seq, pos, ne, m=m, k=k, want_scores=True)
    Oo = orc.attend(v["q"], v["sink"], Eo[None], wino[None], seq, pos, ne, rope_dims=w.rope_dims,
                    idx=ref["idx"])
    assert max_abs(host(E), Eo) <= TOL["f32"]
    assert max_abs(host(KI), KIo) <= TOL["f32"]
    assert max_abs(host(win), wino) <= TOL["f32"]
    idx_h = idx.cpu().numpy()
    same = np.all(idx_h == ref["idx"], axis=1)
    for q in np.nonzero(~same)[0]:
        nv = orc.visible_entries(q, m, 1, T // m)
        # the compressed keys differ by rounding too: widen the band by the key error
        topk_margin_check(idx_h[q], ref["scores"][q], nv, k, ref["tau"][q], ref["amag"][q],
                          eps_rel=2.0 ** -10)
    assert same.mean() > 0.95
    assert max_abs(host(O)[same], Oo[same]) <= TOL["f32"]
