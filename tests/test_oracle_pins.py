"""Pins of the FP64 oracle to facts outside itself: library routines
(numpy matmul, torch rms_norm / scaled_dot_product_attention, torch's FP8
cast), closed forms, invariants, and the counts the pages print.

No test here retypes an oracle formula; each one checks a special case or a
property that a dropped term, a wrong sign or index, or a transposed operand
in the oracle would break.
"""
import math
from pathlib import Path

import numpy as np
import pytest
import torch

GOLDEN = Path(__file__).parent / "golden"


def _rng(seed=0):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------- helpers
def rope_complex(x, pos, r, base=10000.0):
    """RoPE as complex multiplication: pair (x0, x1) is z = x0 + i x1,
    rotated as z * exp(i * pos * base^(-2j/r)) - a different formulation
    from the oracle's cos/sin pair update."""
    x = np.array(x, dtype=np.float64, copy=True)
    c = x.shape[-1]
    z = x[..., c - r::2] + 1j * x[..., c - r + 1::2]
    j = np.arange(r // 2)
    ang = np.asarray(pos, np.float64)[..., None] * np.exp(-np.log(base) * 2.0 * j / r)
    z = z * np.exp(1j * ang)
    x[..., c - r::2] = z.real
    x[..., c - r + 1::2] = z.imag
    return x


def rms_torch(x, eps=1e-6, gain=None):
    t = torch.from_numpy(np.asarray(x, np.float64))
    g = None if gain is None else torch.from_numpy(np.asarray(gain, np.float64))
    return torch.nn.functional.rms_norm(t, (t.shape[-1],), g, eps).numpy()


# ---------------------------------------------------------------- RMSNorm / RoPE
def test_rmsnorm_matches_torch(orc):
    x = _rng(1).standard_normal((7, 96)) * 3
    g = _rng(2).standard_normal(96)
    np.testing.assert_allclose(orc.rmsnorm(x, 1e-6, g), rms_torch(x, 1e-6, g), rtol=1e-13,
                               atol=1e-13)


def test_rope_matches_complex_rotation(orc):
    x = _rng(3).standard_normal((5, 64))
    pos = np.array([0, 1, 7, 1000, 1048576], np.float64)
    np.testing.assert_allclose(orc.rope(x, pos, 32), rope_complex(x, pos, 32), rtol=1e-9,
                               atol=1e-9)
    # only the last r dims move
    np.testing.assert_array_equal(orc.rope(x, pos, 32)[:, :32], x[:, :32])


def test_rope_group_properties(orc):
    x = _rng(4).standard_normal((3, 32))
    a, b = 123.0, -45.5
    ra = orc.rope(x, a, 16)
    np.testing.assert_allclose(np.linalg.norm(ra, axis=-1), np.linalg.norm(x, axis=-1),
                               rtol=1e-13)
    np.testing.assert_allclose(orc.rope(ra, b, 16), orc.rope(x, a + b, 16), atol=1e-12)
    np.testing.assert_allclose(orc.rope(ra, -a, 16), x, atol=1e-12)
    # relative position: <R(a)u, R(b)v> depends on a-b only
    u, v = x[0], x[1]
    d1 = orc.rope(u, 10.0, 16) @ orc.rope(v, 3.0, 16)
    d2 = orc.rope(u, 1007.0, 16) @ orc.rope(v, 1000.0, 16)
    assert abs(d1 - d2) < 1e-10


def test_rmsnorm_rope_unit_rms(orc):
    x = _rng(5).standard_normal((4, 128)) * 5
    y = orc.rmsnorm_rope(x, [0, 4, 8, 12], 32, eps=0.0)
    np.testing.assert_allclose(np.sqrt((y ** 2).mean(-1)), 1.0, rtol=1e-12)


# ---------------------------------------------------------------- compressor
def _compress_inputs(T=40, d=24, c=16, cI=None, seed=6):
    r = _rng(seed)
    H = r.standard_normal((T, d))
    W = {k: r.standard_normal((d, c)) / math.sqrt(d) for k in ("aKV", "bKV", "aZ", "bZ")}
    return H, W


def test_pool_zero_logits_is_mean(orc):
    """With zero gate logits and zero bias the softmax pool is the plain mean
    of the candidates (the mean-pooling special case the cooking-agi page
    contrasts V4 with, Sec 3)."""
    m, T = 4, 40
    H, W = _compress_inputs(T)
    Z0 = np.zeros_like(W["aZ"])
    bias = np.zeros((2 * m, W["aKV"].shape[1]))
    _, pooled = orc.compress(H, W["aKV"], Z0, bias, m, W_bKV=W["bKV"], W_bZ=Z0,
                             return_pooled=True)
    Ca, Cb = H @ W["aKV"], H @ W["bKV"]
    for i in range(T // m):
        cands = [Ca[i * m:(i + 1) * m]]
        if i >= 1:
            cands.append(Cb[(i - 1) * m:i * m])
        np.testing.assert_allclose(pooled[i], np.concatenate(cands).mean(0), rtol=1e-12,
                                   atol=1e-13)


def test_pool_two_candidates_logistic(orc):
    """m = 1 with overlap: entry i pools token i (a-series) and token i-1
    (b-series); softmax of two logits is the logistic function."""
    T, d, c = 9, 12, 8
    H, W = _compress_inputs(T, d, c, seed=7)
    bias = _rng(8).standard_normal((2, c))
    _, pooled = orc.compress(H, W["aKV"], W["aZ"], bias, 1, W_bKV=W["bKV"], W_bZ=W["bZ"],
                             return_pooled=True)
    Ca, Cb, Za, Zb = (H @ W[k] for k in ("aKV", "bKV", "aZ", "bZ"))
    np.testing.assert_allclose(pooled[0], Ca[0], rtol=1e-12)  # block 0: own token only
    for i in range(1, T):
        za, zb = Za[i] + bias[1], Zb[i - 1] + bias[0]
        sa = 1.0 / (1.0 + np.exp(zb - za))
        np.testing.assert_allclose(pooled[i], sa * Ca[i] + (1 - sa) * Cb[i - 1], rtol=1e-11,
                                   atol=1e-12)


def test_pool_large_bias_selects_candidate(orc):
    m, T = 4, 32
    H, W = _compress_inputs(T, seed=9)
    c = W["aKV"].shape[1]
    Z0 = np.zeros_like(W["aZ"])
    Ca, Cb = H @ W["aKV"], H @ W["bKV"]
    for r in range(2 * m):
        bias = np.zeros((2 * m, c))
        bias[r] = 80.0
        _, pooled = orc.compress(H, W["aKV"], Z0, bias, m, W_bKV=W["bKV"], W_bZ=Z0,
                                 return_pooled=True)
        for i in range(1, T // m):
            want = Cb[(i - 1) * m + r] if r < m else Ca[i * m + r - m]
            np.testing.assert_allclose(pooled[i], want, atol=1e-30 + 1e-12 * np.abs(want).max())


def test_pool_logit_shift_and_equal_values_invariance(orc):
    m, T = 4, 24
    H, W = _compress_inputs(T, seed=10)
    c = W["aKV"].shape[1]
    bias = _rng(11).standard_normal((2 * m, c))
    _, p1 = orc.compress(H, W["aKV"], W["aZ"], bias, m, W_bKV=W["bKV"], W_bZ=W["bZ"],
                         return_pooled=True)
    shift = _rng(12).standard_normal(c) * 5
    _, p2 = orc.compress(H, W["aKV"], W["aZ"], bias + shift, m, W_bKV=W["bKV"], W_bZ=W["bZ"],
                         return_pooled=True)
    np.testing.assert_allclose(p1, p2, rtol=1e-10, atol=1e-12)
    # identical values in every candidate: any gate gives that value
    Hc = np.tile(H[:1], (T, 1))
    _, p3 = orc.compress(Hc, W["aKV"], W["aZ"], bias, m, W_bKV=W["aKV"], W_bZ=W["bZ"],
                         return_pooled=True)
    np.testing.assert_allclose(p3, np.tile((Hc @ W["aKV"])[0], (T // m, 1)), rtol=1e-11)


def test_csa_with_masked_b_series_is_hca(orc):
    """CSA whose preceding-block candidates carry -inf logits equals the
    non-overlapping HCA pool with the same a-series and m' = m."""
    m, T = 4, 36
    H, W = _compress_inputs(T, seed=13)
    c = W["aKV"].shape[1]
    bias = _rng(14).standard_normal((2 * m, c))
    bias_csa = bias.copy()
    bias_csa[:m] = -np.inf
    e_csa = orc.compress(H, W["aKV"], W["aZ"], bias_csa, m, W_bKV=W["bKV"], W_bZ=W["bZ"],
                         rope_dims=8)
    e_hca = orc.compress(H, W["aKV"], W["aZ"], bias[m:], m, rope_dims=8)
    np.testing.assert_allclose(e_csa, e_hca, rtol=1e-13, atol=1e-14)


def test_hca_m1_is_normalised_projection(orc):
    T, d, c = 10, 16, 32
    H, W = _compress_inputs(T, d, c, seed=15)
    g = _rng(16).standard_normal(c)
    E, pooled = orc.compress(H, W["aKV"], W["aZ"], np.zeros((1, c)), 1, gain=g, rope_dims=16,
                             return_pooled=True)
    C = H @ W["aKV"]
    np.testing.assert_allclose(pooled, C, rtol=1e-12, atol=1e-13)
    want = rope_complex(rms_torch(C, 1e-6, g), np.arange(T), 16)
    np.testing.assert_allclose(E, want, rtol=1e-9, atol=1e-10)


@pytest.mark.parametrize("T,m,overlap,want", [(1024, 4, 1, 256), (1027, 4, 1, 256),
                                               (1000, 128, 0, 7), (127, 128, 0, 0)])
def test_one_entry_per_m_tokens(orc, T, m, overlap, want):
    H = _rng(17).standard_normal((T, 8))
    W = _rng(18).standard_normal((8, 8))
    E = orc.compress(H, W, W, np.zeros(((1 + overlap) * m, 8)), m,
                     W_bKV=W if overlap else None, W_bZ=W if overlap else None)
    assert E.shape == (want, 8)


def test_compressed_entry_depends_only_on_its_blocks(orc):
    """Entry i reads tokens (i-1)m .. im+m-1 and nothing later."""
    m, T = 4, 32
    H, W = _compress_inputs(T, seed=19)
    c = W["aKV"].shape[1]
    bias = _rng(20).standard_normal((2 * m, c))
    args = (W["aKV"], W["aZ"], bias, m)
    kw = dict(W_bKV=W["bKV"], W_bZ=W["bZ"])
    E0 = orc.compress(H, *args, **kw)
    H2 = H.copy()
    H2[13] += 1.0  # token 13 lies in block 3 (own) and feeds block 4 (preceding)
    E1 = orc.compress(H2, *args, **kw)
    changed = np.nonzero(np.abs(E1 - E0).max(1) > 0)[0]
    assert list(changed) == [3, 4]


# ---------------------------------------------------------------- visibility / counts
def _golden_rows(name):
    rows = []
    for line in (GOLDEN / name).read_text().splitlines():
        line = line.strip()
        if line and not line.startswith("#"):
            rows.append(line.split())
    return rows


def test_visible_entry_counts_printed_on_pages(orc):
    for pos, m, want in _golden_rows("causality_m4.txt"):
        assert orc.visible_entries(int(pos), int(m), 1, 1 << 40) == int(want)
    # literal 0-based reading differs exactly at block ends
    assert orc.visible_entries(7, 4, 0, 100) == 1
    assert orc.visible_entries(8, 4, 0, 100) == 2
    # clipping to the stored entries
    assert orc.visible_entries(1000, 4, 1, 10) == 10


# ---------------------------------------------------------------- indexer / top-k
def test_index_scores_reduce_to_matmul(orc):
    """One head with w = 1 and non-negative inputs: I = q . K^T (numpy)."""
    r = _rng(21)
    Q, N, cI = 6, 40, 16
    qI = np.abs(r.standard_normal((Q, 1, cI)))
    K = np.abs(r.standard_normal((1, N, cI)))
    out = orc.index_topk(qI, np.ones((Q, 1)), K, np.zeros(Q), np.full(Q, 4 * N), [N], m=4,
                         k=8, want_scores=True)
    np.testing.assert_allclose(out["scores"], qI[:, 0] @ K[0].T, rtol=1e-13)


def test_index_scores_one_hot_weight_is_relu_of_head(orc):
    r = _rng(22)
    Q, HI, N, cI = 5, 3, 30, 8
    qI = r.standard_normal((Q, HI, cI))
    K = r.standard_normal((1, N, cI))
    for h in range(HI):
        w = np.zeros((Q, HI))
        w[:, h] = -2.5
        out = orc.index_topk(qI, w, K, np.zeros(Q), np.full(Q, 4 * N), [N], m=4, k=4,
                             want_scores=True)
        np.testing.assert_allclose(out["scores"], -2.5 * np.maximum(qI[:, h] @ K[0].T, 0),
                                   rtol=1e-13, atol=1e-14)


def _check_topk_property(idx_row, scores, n_vis, k):
    """Brute-force check of a top-k answer: size, order, dominance, ties."""
    ke = min(k, n_vis)
    kept = idx_row[:ke]
    assert (idx_row[ke:] == -1).all()
    assert (np.diff(kept) > 0).all() and (kept >= 0).all() and (kept < n_vis).all()
    S = set(kept.tolist())
    for s in S:
        for t in range(n_vis):
            if t in S:
                continue
            assert scores[s] > scores[t] or (scores[s] == scores[t] and s < t)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_topk_integer_inputs_brute_force(orc, seed):
    """Integer inputs make every score exact and produce many ties; the
    selected sets must dominate and break ties by the lower index."""
    r = _rng(100 + seed)
    Q, HI, cI, N, m, k = 24, 4, 8, 60, 4, 10
    qI = r.integers(-2, 3, (Q, HI, cI)).astype(np.float64)
    K = r.integers(-2, 3, (2, N, cI)).astype(np.float64)
    w = r.integers(-3, 4, (Q, HI)).astype(np.float64)
    seq = r.integers(0, 2, Q)
    pos = r.integers(0, 4 * N + 8, Q)
    ne = np.array([N, N - 7])
    out = orc.index_topk(qI, w, K, seq, pos, ne, m=m, k=k, want_scores=True)
    for q in range(Q):
        nv = min((pos[q] + 1) // m, ne[seq[q]])
        # scores from numpy: exact for these integers
        dots = np.einsum("hj,sj->hs", qI[q], K[seq[q], :nv])
        sc = (w[q][:, None] * np.maximum(dots, 0)).sum(0)
        np.testing.assert_array_equal(out["scores"][q, :nv], sc)
        _check_topk_property(out["idx"][q], sc, nv, k)


def test_topk_fewer_visible_than_k(orc):
    r = _rng(23)
    qI = r.standard_normal((3, 2, 4))
    K = r.standard_normal((1, 50, 4))
    out = orc.index_topk(qI, np.ones((3, 2)), K, [0, 0, 0], [2, 10, 30], [50], m=4, k=16)
    assert (out["idx"][0] == -1).all()  # p=2: no complete block
    assert list(out["idx"][1][:2]) == [0, 1] and (out["idx"][1][2:] == -1).all()
    assert (out["idx"][2][:7] == np.arange(7)).all() and (out["idx"][2][7:] == -1).all()


# ---------------------------------------------------------------- attention
def _attn_setup(seed=30, Q=4, Hq=3, c=32, r=8, N=20, nw=6, T=40):
    rg = _rng(seed)
    q = rg.standard_normal((Q, Hq, c))
    E = rg.standard_normal((1, N, c))
    win = rg.standard_normal((1, T, c))
    sink = rg.standard_normal(Hq)
    pos = np.array([0, 5, 17, 39])[:Q]
    return q, E, win, sink, pos


def _keys_for(E, win, idx_row, p, n_win):
    ks = [E[0, s] for s in idx_row if s >= 0]
    ks += [win[0, j] for j in range(max(0, p - n_win + 1), p + 1)]
    return np.array(ks)


def _qhat(q, p, r, gain=None):
    return rope_complex(rms_torch(q, 1e-6, gain), np.full(q.shape[:-1], p), r)


@pytest.mark.parametrize("finite_sink", [False, True])
def test_attention_matches_torch_sdpa(orc, finite_sink):
    """sink -> -inf is plain softmax attention (torch SDPA, float64); a
    finite sink equals SDPA with one extra zero key/value whose logit is
    forced to the sink value through an additive mask."""
    q, E, win, sink, pos = _attn_setup()
    if not finite_sink:
        sink = np.full_like(sink, -1e300)
    Q, Hq, c = q.shape
    r, n_win = 8, 6
    rg = _rng(31)
    idx = np.stack([np.sort(rg.choice(20, 5, replace=False)) for _ in range(Q)]).astype(np.int32)
    idx[0] = -1
    O = orc.attend(q, sink, E, win, np.zeros(Q), pos, [20], rope_dims=r, idx=idx, n_win=n_win)
    for i in range(Q):
        K = _keys_for(E, win, idx[i], pos[i], n_win)
        qh = _qhat(q[i], pos[i], r)
        kt = torch.from_numpy(K)[None, None].expand(1, Hq, -1, -1)
        qt = torch.from_numpy(qh)[None, :, None, :]
        if finite_sink:
            kt = torch.cat([kt, torch.zeros(1, Hq, 1, c, dtype=torch.float64)], 2)
            mask = torch.zeros(1, Hq, 1, kt.shape[2], dtype=torch.float64)
            mask[..., -1] = torch.from_numpy(sink)[None, :, None]
            o = torch.nn.functional.scaled_dot_product_attention(qt, kt, kt, attn_mask=mask)
        else:
            o = torch.nn.functional.scaled_dot_product_attention(qt, kt, kt)
        o = rope_complex(o[0, :, 0].numpy(), np.full(Hq, -pos[i]), r)
        np.testing.assert_allclose(O[i], o, rtol=1e-10, atol=1e-12)


def test_attention_sink_large_gives_zero(orc):
    q, E, win, sink, pos = _attn_setup()
    idx = np.tile(np.arange(5, dtype=np.int32), (4, 1))
    O = orc.attend(q, np.full(3, 700.0), E, win, np.zeros(4), pos, [20], rope_dims=8, idx=idx,
                   n_win=6)
    assert np.abs(O).max() < 1e-250


def test_attention_equal_keys_closed_form(orc):
    """All keys equal to v: o = n e^l / (e^z' + n e^l) * v, so the weights
    sum to less than one by exactly the sink's share."""
    c, r, Hq = 16, 4, 2
    rg = _rng(32)
    v = rg.standard_normal(c)
    E = np.tile(v, (1, 10, 1))
    win = np.tile(v, (1, 50, 1))
    q = rg.standard_normal((1, Hq, c))
    sink = np.array([0.3, -1.2])
    p, n_win = 0, 4  # p = 0: window holds one row; 3 selected entries
    idx = np.array([[1, 4, 7, -1]], np.int32)
    O = orc.attend(q, sink, E, win, [0], [p], [10], rope_dims=r, idx=idx, n_win=n_win)
    n = 4
    for h in range(Hq):
        qh = _qhat(q[0, h], p, r)
        l = qh @ v / math.sqrt(c)
        frac = n * math.exp(l) / (math.exp(sink[h]) + n * math.exp(l))
        np.testing.assert_allclose(O[0, h], frac * v, rtol=1e-12)
        assert frac < 1.0


def test_attention_first_token_closed_form(orc):
    """p = 0 with no compressed entry: the only key is the window row of
    position 0 and inverse RoPE at 0 is the identity: o = sigmoid(l - z') k."""
    c, r = 32, 8
    rg = _rng(33)
    q = rg.standard_normal((1, 2, c))
    win = rg.standard_normal((1, 5, c))
    sink = np.array([0.7, -0.4])
    O = orc.attend(q, sink, np.zeros((1, 1, c)), win, [0], [0], [0], rope_dims=r,
                   idx=np.full((1, 4), -1, np.int32))
    k0 = win[0, 0]
    for h in range(2):
        l = _qhat(q[0, h], 0, r) @ k0 / math.sqrt(c)
        np.testing.assert_allclose(O[0, h], k0 / (1 + math.exp(sink[h] - l)), rtol=1e-12)


def test_hca_equals_csa_with_all_entries_selected(orc):
    q, E, win, sink, pos = _attn_setup(seed=34)
    m = 2
    nv = np.array([orc.visible_entries(p, m, 1, 20) for p in pos])
    idx = np.full((4, 32), -1, np.int32)
    for i, n in enumerate(nv):
        idx[i, :n] = np.arange(n)
    Od = orc.attend(q, sink, E, win, np.zeros(4), pos, [20], rope_dims=8, m=m, n_win=6)
    Os = orc.attend(q, sink, E, win, np.zeros(4), pos, [20], rope_dims=8, idx=idx, n_win=6)
    np.testing.assert_allclose(Od, Os, rtol=1e-13, atol=1e-15)


def test_one_softmax_differs_from_two_branches(orc):
    """The pages insist on one normalisation over window, compressed and sink
    terms; separately normalised branches added together differ."""
    q, E, win, sink, pos = _attn_setup(seed=35)
    idx = np.tile(np.arange(6, dtype=np.int32), (4, 1))
    joint = orc.attend(q, sink, E, win, np.zeros(4), pos, [20], rope_dims=8, idx=idx, n_win=6)
    only_cmp = orc.attend(q, sink, E, win, np.zeros(4), pos, [20], rope_dims=8, idx=idx, n_win=0)
    only_win = orc.attend(q, sink, E, win, np.zeros(4), pos, [20], rope_dims=8,
                          idx=np.full((4, 6), -1, np.int32), n_win=6)
    assert np.abs(joint - (only_cmp + only_win)).max() > 1e-2


def test_attention_relative_position_invariance(orc):
    """Shifting the query and every key position by D leaves O unchanged:
    logits depend on position differences and O is rotated back by -(p+D)."""
    c, r, Hq, n_win = 32, 8, 2, 8
    rg = _rng(36)
    raw_e = rg.standard_normal((12, c))
    raw_w = rg.standard_normal((60, c))
    q = rg.standard_normal((1, Hq, c))
    sink = rg.standard_normal(Hq)
    p, D = 40, 1000
    idx = np.array([[0, 3, 5, 9]], np.int32)
    outs = []
    for shift in (0, D):
        E = orc.rmsnorm_rope(raw_e, np.arange(12) * 4 + shift, r)[None]
        win = np.zeros((1, 60 + D, c))
        win[0, shift:shift + 60] = orc.rmsnorm_rope(raw_w, np.arange(60) + shift, r)
        outs.append(orc.attend(q, sink, E, win, [0], [p + shift], [12], rope_dims=r, idx=idx,
                               n_win=n_win))
    np.testing.assert_allclose(outs[0], outs[1], rtol=1e-9, atol=1e-11)


# ---------------------------------------------------------------- whole layer
def _layer(orc, H, qI, w, q, kvw, sink, Wm, Wi, bm, bi, m=4, k=6, n_win=8, r=8):
    E = orc.compress(H, Wm["aKV"], Wm["aZ"], bm, m, W_bKV=Wm["bKV"], W_bZ=Wm["bZ"], rope_dims=r)
    KI = orc.compress(H, Wi["aKV"], Wi["aZ"], bi, m, W_bKV=Wi["bKV"], W_bZ=Wi["bZ"])
    T = H.shape[0]
    pos = np.arange(T)
    ne = [E.shape[0]]
    sel = orc.index_topk(qI, w, KI[None], np.zeros(T), pos, ne, m=m, k=k)["idx"]
    win = orc.rmsnorm_rope(kvw, pos, r)
    O, nk = orc.attend(q, sink, E[None], win[None], np.zeros(T), pos, ne, rope_dims=r, idx=sel,
                       m=m, n_win=n_win, return_nkeys=True)
    return O, nk


def _layer_inputs(seed=40, T=24, d=12, c=16, cI=8, HI=2, Hq=2, m=4):
    rg = _rng(seed)
    H = rg.standard_normal((T, d))
    Wm = {kk: rg.standard_normal((d, c)) / math.sqrt(d) for kk in ("aKV", "bKV", "aZ", "bZ")}
    Wi = {kk: rg.standard_normal((d, cI)) / math.sqrt(d) for kk in ("aKV", "bKV", "aZ", "bZ")}
    bm = rg.standard_normal((2 * m, c)) * 0.1
    bi = rg.standard_normal((2 * m, cI)) * 0.1
    qI = rg.standard_normal((T, HI, cI))
    w = rg.standard_normal((T, HI))
    q = rg.standard_normal((T, Hq, c))
    kvw = rg.standard_normal((T, c))
    sink = rg.standard_normal(Hq)
    return H, qI, w, q, kvw, sink, Wm, Wi, bm, bi


def test_layer_future_tokens_do_not_leak(orc):
    """Positions 3, 4, 7, 8 (the cooking-agi page, Sec 3): perturbing any
    input of a later token leaves the output at p unchanged, bit for bit."""
    base = _layer_inputs()
    O0, _ = _layer(orc, *base)
    T = base[0].shape[0]
    for p in (3, 4, 7, 8):
        pert = [a.copy() if isinstance(a, np.ndarray) else a for a in base]
        for j in (0, 1, 2, 3, 4):  # H, qI, w, q, kv_win of later tokens
            pert[j][p + 1:] += 3.0
        O1, _ = _layer(orc, *pert)
        np.testing.assert_array_equal(O1[p], O0[p])
        assert np.abs(O1[p + 1:] - O0[p + 1:]).max() > 0


def test_layer_block_becomes_visible_at_its_last_token(orc):
    """Entry 1 (tokens 4..7) is read at p = 7 and not at p = 6."""
    base = list(_layer_inputs(seed=41))
    O0, _ = _layer(orc, *base)
    H2 = base[0].copy()
    H2[5] += 2.0  # token 5 feeds entry 1 (own block) and entry 2 (preceding block)
    base[0] = H2
    O1, _ = _layer(orc, *base)
    np.testing.assert_array_equal(O1[6], O0[6])
    assert np.abs(O1[7] - O0[7]).max() > 1e-6


def test_ledger_read_counts(orc):
    """Main-KV reads of the page's accounting example (golden file):
    history 1024 -> CSA reads min(32, 256) + 128 = 160, HCA 8 + 128 = 136;
    history 9 -> one token waits in the unfinished CSA block."""
    rows = {(int(a[0]), a[5]): int(a[6]) for a in _golden_rows("attention_ledger.txt")}
    rg = _rng(42)
    c, p = 16, 1023
    q = rg.standard_normal((1, 1, c))
    win = rg.standard_normal((1, 1024, c))
    E4 = rg.standard_normal((1, 256, c))
    qI = rg.standard_normal((1, 2, 8))
    KI = rg.standard_normal((1, 256, 8))
    idx = orc.index_topk(qI, np.ones((1, 2)), KI, [0], [p], [256], m=4, k=32)["idx"]
    _, nk = orc.attend(q, [0.0], E4, win, [0], [p], [256], rope_dims=4, idx=idx, m=4,
                       n_win=128, return_nkeys=True)
    assert nk[0] == rows[(1024, "light_main_reads")]
    E128 = rg.standard_normal((1, 8, c))
    _, nk = orc.attend(q, [0.0], E128, win, [0], [p], [8], rope_dims=4, m=128, n_win=128,
                       return_nkeys=True)
    assert nk[0] == rows[(1024, "heavy_main_reads")]
    p9 = 8  # history 9
    assert (p9 + 1) - 4 * orc.visible_entries(p9, 4, 1, 10 ** 9) == rows[(9, "light_tail")]


# ---------------------------------------------------------------- FP8 mixed rows
def test_e4m3_decode_matches_torch(orc):
    codes = np.arange(256, dtype=np.uint8)
    ours = orc.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    finite = ~np.isnan(ref)
    np.testing.assert_array_equal(ours[finite], ref[finite])
    assert np.isnan(ours[~finite]).all()


def test_e4m3_encode_matches_torch_rounding(orc):
    rg = _rng(43)
    x = np.concatenate([rg.standard_normal(3000) * 30, rg.standard_normal(500) * 0.01,
                        [0.0, -0.0, 448.0, -448.0, 0.0009765625, 0.0029296875, 17.0, 19.0]])
    x = x[np.abs(x) <= 448]
    ours = orc.e4m3_encode(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(orc.e4m3_decode(ours), orc.e4m3_decode(ref))


def test_mixed_row_roundtrip(orc):
    rg = _rng(44)
    x = rg.standard_normal((6, 512)).astype(np.float32)
    x[1, :448] = 0.0
    rows = orc.pack_mixed(x)
    back = orc.unpack_mixed(rows)
    scale = np.abs(x[:, :448]).max(1) / 448.0
    err = np.abs(back[:, :448] - x[:, :448])
    # E4M3 keeps 3 mantissa bits: relative rounding error <= 2^-4
    assert (err <= np.abs(x[:, :448]) * 2.0 ** -4 + scale[:, None] * 2.0 ** -9 + 1e-12).all()
    assert (back[1, :448] == 0).all()
    np.testing.assert_allclose(back[:, 448:], x[:, 448:], rtol=2 ** -8)
