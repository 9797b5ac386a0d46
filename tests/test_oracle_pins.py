"""Pins of the float64 oracle against things other than itself (CPU only).

Each test checks the oracle against a closed form, a second independent
spelling (pure-Python loops), finite differences, an exact invariant of the
method, or a value printed in ``tests/golden/`` with its source.  The last
group plants plausible mistakes in the oracle (on the CPU) and checks that the
pins catch them.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import attention as A
from oracle import brute, tiles
from padded_variable_length_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
EPIS = (A.SIGMOID, A.SOFTMAX, A.SOFTMAX1)


def _golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            rows.append([c.strip() for c in line.split("|")])
    return rows


def _num(tok):
    if tok == "ln2":
        return math.log(2)
    if tok == "ln3":
        return math.log(3)
    return float(tok)


# ----------------------------------------------------------------------------------------
# golden values from the pages' formulas
# ----------------------------------------------------------------------------------------

def test_golden_softmax1_points():
    for name, logits, expected in _golden("softmax1_points.txt"):
        x = np.array([[_num(t) for t in logits.split()]])
        want = np.array([float(Fraction(t)) for t in expected.split()])
        epi = A.SOFTMAX1 if name.endswith("softmax1") else A.SOFTMAX
        p, _ = A.weights(x, np.ones_like(x, dtype=bool), epi)
        np.testing.assert_allclose(p[0], want, rtol=1e-11, atol=1e-300, err_msg=name)


def test_golden_sigmoid_bias_points():
    for n, expected in _golden("sigmoid_bias_points.txt"):
        b = A.bias_from_counts(np.array([int(n)]))
        p, _ = A.weights(b[:, None], np.ones((1, 1), dtype=bool), A.SIGMOID)
        assert p[0, 0] == pytest.approx(float(Fraction(expected)), rel=1e-14)


def test_golden_tile_counts():
    for name, npad, lens, nonempty, full, partial in _golden("tile_counts.txt"):
        t = tiles.tile_list_from_lengths([int(x) for x in lens.split()], int(npad))
        assert len(t["col_idx"]) == int(nonempty), name
        assert int((t["kind"] == 1).sum()) == int(full), name
        assert int((t["kind"] == 2).sum()) == int(partial), name
        assert t["bits"].shape[0] == int(partial), name


# ----------------------------------------------------------------------------------------
# closed forms at Q = 0
# ----------------------------------------------------------------------------------------

def _rand(rng, *shape):
    return rng.standard_normal(shape)


@pytest.mark.parametrize("n,npad", [(1, 5), (7, 7), (37, 50), (130, 200)])
def test_q_zero_sigmoid_closed_form(n, npad):
    rng = np.random.default_rng(n)
    d = 8
    q = np.zeros((1, npad, 1, d))
    k, v, do = (_rand(rng, 1, npad, 1, d) for _ in range(3))
    bias = A.bias_from_counts(W.lengths_counts(np.array([n]), npad))
    scale = 1 / math.sqrt(d)
    o, _ = A.forward(q, k, v, bias, scale, A.SIGMOID, lengths=[n])
    want = v[0, :n, 0].sum(0) / (n + 1)
    np.testing.assert_allclose(o[0, :n, 0], np.broadcast_to(want, (n, d)), rtol=1e-12, atol=1e-14)
    assert np.all(o[0, n:] == 0)
    dq, dk, dv = A.backward(q, k, v, do, bias, scale, A.SIGMOID, lengths=[n])
    # dv_j = sum_i do_i / (n+1);  ds_ij = (do_i . v_j) n/(n+1)^2;  dq_i = scale sum_j ds_ij k_j; dk = 0
    np.testing.assert_allclose(dv[0, :n, 0], np.broadcast_to(do[0, :n, 0].sum(0) / (n + 1), (n, d)),
                               rtol=1e-12, atol=1e-14)
    c = n / (n + 1) ** 2
    dq_want = scale * c * (do[0, :n, 0] @ v[0, :n, 0].T) @ k[0, :n, 0]
    np.testing.assert_allclose(dq[0, :n, 0], dq_want, rtol=1e-11, atol=1e-13)
    assert np.all(dk == 0)
    assert np.all(dq[0, n:] == 0) and np.all(dv[0, n:] == 0)


@pytest.mark.parametrize("n", [1, 9, 128])
def test_q_zero_softmax_and_softmax1(n):
    rng = np.random.default_rng(7)
    d = 4
    q = np.zeros((1, n, 1, d))
    k, v = _rand(rng, 1, n, 1, d), _rand(rng, 1, n, 1, d)
    zero_bias = np.zeros((1, n))
    o, _ = A.forward(q, k, v, zero_bias, 0.5, A.SOFTMAX, lengths=[n])
    np.testing.assert_allclose(o[0, :, 0], np.broadcast_to(v[0, :, 0].mean(0), (n, d)), rtol=1e-12)
    o1, _ = A.forward(q, k, v, zero_bias, 0.5, A.SOFTMAX1, lengths=[n])
    np.testing.assert_allclose(o1[0, :, 0], np.broadcast_to(v[0, :, 0].sum(0) / (n + 1), (n, d)),
                               rtol=1e-12)
    # sigmoid with b = -log n coincides with softmax_1 with b = 0 at Q = 0
    sb = A.bias_from_counts(np.full((1, n), n))
    os_, _ = A.forward(q, k, v, sb, 0.5, A.SIGMOID, lengths=[n])
    np.testing.assert_allclose(os_, o1, rtol=1e-12)


# ----------------------------------------------------------------------------------------
# brute force loops vs the vectorised oracle
# ----------------------------------------------------------------------------------------

def _tiny_case(seed, Nq=9, Nk=11, d=5, density=0.6, empty_row=True):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((Nq, d)) * 1.5
    k = rng.standard_normal((Nk, d)) * 1.5
    v = rng.standard_normal((Nk, d))
    do = rng.standard_normal((Nq, d))
    m = rng.random((Nq, Nk)) < density
    if empty_row:
        m[Nq // 2] = False
    bias = rng.standard_normal(Nq) - 1.0
    return q, k, v, do, m, bias


@pytest.mark.parametrize("epi", EPIS)
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_brute_force_matches(epi, seed):
    q, k, v, do, m, bias = _tiny_case(seed)
    scale = 0.37
    mr = lambda i0, i1: m[i0:i1]
    o, _ = A.head_forward(q, k, v, mr, bias, scale, epi)
    ob, _ = brute.forward_head(q.tolist(), k.tolist(), v.tolist(), m.tolist(), bias.tolist(), scale, epi)
    np.testing.assert_allclose(o, np.array(ob), rtol=1e-12, atol=1e-14)
    dq, dk, dv = A.head_backward(q, k, v, do, mr, bias, scale, epi)
    bq, bk, bv = brute.backward_head(q.tolist(), k.tolist(), v.tolist(), do.tolist(), m.tolist(),
                                     bias.tolist(), scale, epi)
    np.testing.assert_allclose(dq, np.array(bq), rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(dk, np.array(bk), rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(dv, np.array(bv), rtol=1e-11, atol=1e-13)
    # the empty row gives exactly zero output and zero dq
    i = q.shape[0] // 2
    assert np.all(o[i] == 0) and np.all(dq[i] == 0)


# ----------------------------------------------------------------------------------------
# finite differences pin the three backward formulas
# ----------------------------------------------------------------------------------------

def _fd_check(epi, seed, fwd=None, bwd=None):
    fwd = fwd or A.head_forward
    bwd = bwd or A.head_backward
    q, k, v, do, m, bias = _tiny_case(seed, Nq=6, Nk=7, d=3)
    scale = 0.61
    mr = lambda i0, i1: m[i0:i1]

    def L(q_, k_, v_):
        o, _ = fwd(q_, k_, v_, mr, bias, scale, epi)
        return float(np.sum(o * do))

    dq, dk, dv = bwd(q, k, v, do, mr, bias, scale, epi)
    h = 1e-6
    worst = 0.0
    for name, X, G in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(X)
        for idx in np.ndindex(X.shape):
            Xp, Xm = X.copy(), X.copy()
            Xp[idx] += h
            Xm[idx] -= h
            args_p = {"q": (Xp, k, v), "k": (q, Xp, v), "v": (q, k, Xp)}[name]
            args_m = {"q": (Xm, k, v), "k": (q, Xm, v), "v": (q, k, Xm)}[name]
            num[idx] = (L(*args_p) - L(*args_m)) / (2 * h)
        err = np.max(np.abs(num - G)) / max(1e-12, np.max(np.abs(num)))
        worst = max(worst, err)
    return worst


@pytest.mark.parametrize("epi", EPIS)
@pytest.mark.parametrize("seed", [3, 4])
def test_finite_differences(epi, seed):
    assert _fd_check(epi, seed) < 1e-6


# ----------------------------------------------------------------------------------------
# invariants
# ----------------------------------------------------------------------------------------

@pytest.mark.parametrize("epi", EPIS)
def test_padding_invariance(epi):
    rng = np.random.default_rng(11)
    lengths = np.array([5, 13, 1, 0])
    npad = 13
    H, d = 2, 4
    q, k, v, do = (rng.standard_normal((4, npad, H, d)) for _ in range(4))
    bias = A.bias_from_counts(W.lengths_counts(lengths, npad)) if epi == A.SIGMOID else np.zeros((4, npad))
    o, _ = A.forward(q, k, v, bias, 0.5, epi, lengths=lengths)
    g = A.backward(q, k, v, do, bias, 0.5, epi, lengths=lengths)
    # append 7 pad tokens of fresh random content
    extra = 7
    cat = lambda x: np.concatenate([x, rng.standard_normal((4, extra, H, d)) * 3], axis=1)
    q2, k2, v2, do2 = cat(q), cat(k), cat(v), cat(do)
    bias2 = np.concatenate([bias, np.zeros((4, extra))], axis=1)
    o2, _ = A.forward(q2, k2, v2, bias2, 0.5, epi, lengths=lengths)
    g2 = A.backward(q2, k2, v2, do2, bias2, 0.5, epi, lengths=lengths)
    for b, n in enumerate(lengths):
        np.testing.assert_allclose(o2[b, :n], o[b, :n], rtol=1e-13, atol=1e-15)
        for x, x2 in zip(g, g2):
            np.testing.assert_allclose(x2[b, :n], x[b, :n], rtol=1e-12, atol=1e-15)
        assert np.all(o2[b, n:] == 0)
        for x2 in g2:
            assert np.all(x2[b, n:] == 0)


@pytest.mark.parametrize("epi", EPIS)
def test_permutation_equivariance(epi):
    q, k, v, do, m, bias = _tiny_case(21, Nq=8, Nk=10, d=4, density=1.0, empty_row=False)
    mr = lambda i0, i1: m[i0:i1]
    o, _ = A.head_forward(q, k, v, mr, bias, 0.4, epi)
    dq, dk, dv = A.head_backward(q, k, v, do, mr, bias, 0.4, epi)
    pk = np.random.default_rng(5).permutation(k.shape[0])
    o2, _ = A.head_forward(q, k[pk], v[pk], mr, bias, 0.4, epi)
    np.testing.assert_allclose(o2, o, rtol=1e-12)
    dq2, dk2, dv2 = A.head_backward(q, k[pk], v[pk], do, mr, bias, 0.4, epi)
    np.testing.assert_allclose(dq2, dq, rtol=1e-11, atol=1e-14)
    np.testing.assert_allclose(dk2, dk[pk], rtol=1e-11, atol=1e-14)
    np.testing.assert_allclose(dv2, dv[pk], rtol=1e-11, atol=1e-14)
    pq = np.random.default_rng(6).permutation(q.shape[0])
    o3, _ = A.head_forward(q[pq], k, v, mr, bias[pq], 0.4, epi)
    np.testing.assert_allclose(o3, o[pq], rtol=1e-12)


def test_softmax1_is_softmax_with_a_zero_logit_and_zero_value():
    q, k, v, do, m, _ = _tiny_case(31, Nq=7, Nk=9, d=4)
    zb = np.zeros(q.shape[0])
    mr = lambda i0, i1: m[i0:i1]
    o1, _ = A.head_forward(q, k, v, mr, zb, 0.5, A.SOFTMAX1)
    k0 = np.vstack([k, np.zeros((1, 4))])
    v0 = np.vstack([v, np.zeros((1, 4))])
    m0 = np.hstack([m, np.ones((m.shape[0], 1), dtype=bool)])
    o0, _ = A.head_forward(q, k0, v0, lambda i0, i1: m0[i0:i1], zb, 0.5, A.SOFTMAX)
    np.testing.assert_allclose(o1, o0, rtol=1e-12, atol=1e-15)
    g1 = A.head_backward(q, k, v, do, mr, zb, 0.5, A.SOFTMAX1)
    g0 = A.head_backward(q, k0, v0, do, lambda i0, i1: m0[i0:i1], zb, 0.5, A.SOFTMAX)
    np.testing.assert_allclose(g1[0], g0[0], rtol=1e-11, atol=1e-14)
    np.testing.assert_allclose(g1[1], g0[1][:-1], rtol=1e-11, atol=1e-14)
    np.testing.assert_allclose(g1[2], g0[2][:-1], rtol=1e-11, atol=1e-14)


def test_softmax1_row_sums_and_ratios():
    rng = np.random.default_rng(2)
    s = rng.standard_normal((50, 30)) * 4
    m = rng.random((50, 30)) < 0.7
    m[:, 0] = True
    p1, _ = A.weights(s, m, A.SOFTMAX1)
    p, _ = A.weights(s, m, A.SOFTMAX)
    sums = p1.sum(1)
    assert np.all(sums > 0) and np.all(sums < 1)
    np.testing.assert_allclose(p.sum(1), 1.0, rtol=1e-13)
    ratio1 = p1[:, 1:][m[:, 1:]] / np.repeat(p1[:, :1], 29, axis=1)[m[:, 1:]]
    ratio = p[:, 1:][m[:, 1:]] / np.repeat(p[:, :1], 29, axis=1)[m[:, 1:]]
    np.testing.assert_allclose(ratio1, ratio, rtol=1e-12)


@pytest.mark.parametrize("epi", [A.SOFTMAX, A.SOFTMAX1])
def test_online_blockwise_softmax_equals_oracle(epi):
    """Running max / running sum over 128-key blocks, with the partial sums and the
    output rescaled by exp(m_old - m_new) ("Flash Attention: révolutionner...",
    section on the mathematics: softmax decomposition and blockwise fusion, read
    with the sums, not the normalised softmax, rescaled).  softmax_1 starts from
    m = 0, l = 1: the zero logit with a zero value row."""
    rng = np.random.default_rng(9)
    Nq, Nk, d = 40, 700, 16
    q, k, v = (rng.standard_normal((n, d)) for n in (Nq, Nk, Nk))
    m = rng.random((Nq, Nk)) < 0.3
    m[3] = False
    s_all = 0.25 * q @ k.T
    o_ref, lse_ref = A.head_forward(q, k, v, lambda i0, i1: m[i0:i1], np.zeros(Nq), 0.25, epi)
    mx = np.full(Nq, 0.0 if epi == A.SOFTMAX1 else -np.inf)
    l = np.full(Nq, 1.0 if epi == A.SOFTMAX1 else 0.0)
    acc = np.zeros((Nq, d))
    np.seterr(invalid="ignore", divide="ignore")
    for j0 in range(0, Nk, 128):
        s = np.where(m[:, j0:j0 + 128], s_all[:, j0:j0 + 128], -np.inf)
        mnew = np.maximum(mx, s.max(1))
        fin = np.isfinite(mnew)
        alpha = np.where(fin, np.exp(np.where(fin, mx - mnew, 0.0)), 1.0)
        p = np.where(fin[:, None], np.exp(s - np.where(fin, mnew, 0.0)[:, None]), 0.0)
        l = alpha * l + p.sum(1)
        acc = alpha[:, None] * acc + p @ v[j0:j0 + 128]
        mx = mnew
    out = np.where(l[:, None] > 0, acc / np.where(l > 0, l, 1.0)[:, None], 0.0)
    np.testing.assert_allclose(out, o_ref, rtol=1e-12, atol=1e-14)
    ok = np.isfinite(lse_ref)
    np.testing.assert_allclose((mx + np.log(l))[ok], lse_ref[ok], rtol=1e-13)
    np.seterr(invalid="warn", divide="warn")


def test_sigmoid_derivative_bound():
    q, k, v, do, m, bias = _tiny_case(41, Nq=20, Nk=30, d=6)
    s = 0.5 * q @ k.T + bias[:, None]
    p, _ = A.weights(s, m, A.SIGMOID)
    dp = do @ v.T
    ds = dp * p * (1 - p)
    assert np.all(np.abs(ds) <= np.abs(dp) / 4 + 1e-15)


def test_sampled_row_and_column_helpers_match_full():
    for epi in EPIS:
        q, k, v, do, m, bias = _tiny_case(51, Nq=300, Nk=280, d=4, density=0.5)
        mr = lambda i0, i1: m[i0:i1]
        o, lse = A.head_forward(q, k, v, mr, bias, 0.3, epi)
        dq, dk, dv = A.head_backward(q, k, v, do, mr, bias, 0.3, epi)
        rows = np.array([0, 7, 150, 299])
        cols = np.array([1, 100, 279])
        o_s, _ = A.head_forward(q, k, v, mr, bias, 0.3, epi, rows=rows)
        np.testing.assert_allclose(o_s, o[rows], rtol=1e-12, atol=1e-15)
        dq_s = A.query_rows_backward(q, k, v, do, mr, bias, 0.3, epi, rows)
        np.testing.assert_allclose(dq_s, dq[rows], rtol=1e-11, atol=1e-14)
        dk_s, dv_s = A.key_columns_backward(q, k, v, do, mr, bias, 0.3, epi, cols)
        np.testing.assert_allclose(dk_s, dk[cols], rtol=1e-11, atol=1e-14)
        np.testing.assert_allclose(dv_s, dv[cols], rtol=1e-11, atol=1e-14)


def test_column_helper_with_narrow_key_ranges():
    """Causal documents: each row chunk sees a narrow key range, so sampled key columns lie
    outside it for most chunks (weight 0 there).  The column helper still equals the full
    backward, for every epilogue (the softmax forms read the chunk's range of keys)."""
    docs = [300, 250, 150, 320]
    n = sum(docs)
    m = np.zeros((n, n), dtype=bool)
    o0 = 0
    for ln in docs:
        m[o0:o0 + ln, o0:o0 + ln] = np.tril(np.ones((ln, ln), dtype=bool))
        o0 += ln
    rng = np.random.default_rng(61)
    q, k, v, do = (rng.standard_normal((n, 5)) for _ in range(4))
    bias = -np.log(np.repeat(np.array(docs, dtype=np.float64), docs))
    mr = lambda i0, i1: m[i0:i1]
    cols = np.array([0, 5, 299, 300, 420, 549, 550, 640, 700, 1019])
    for epi in EPIS:
        dq, dk, dv = A.head_backward(q, k, v, do, mr, bias, 0.3, epi)
        dk_s, dv_s = A.key_columns_backward(q, k, v, do, mr, bias, 0.3, epi, cols)
        np.testing.assert_allclose(dk_s, dk[cols], rtol=1e-11, atol=1e-14)
        np.testing.assert_allclose(dv_s, dv[cols], rtol=1e-11, atol=1e-14)


# ----------------------------------------------------------------------------------------
# tile list
# ----------------------------------------------------------------------------------------

def _check_tile_invariants(mask, t):
    mask = np.asarray(mask) != 0
    B, Nq, Nk = mask.shape
    QT, KT = t["QT"], t["KT"]
    nfull = int((t["kind"] == 1).sum())
    pop = int(np.unpackbits(t["bits"].view(np.uint8)).sum()) if t["bits"].size else 0
    assert pop + 128 * 128 * nfull == int(mask.sum())
    # each listed entry agrees with the mask block; bit order is word q*4 + k/32, bit k%32
    e = 0
    for r in range(B * QT):
        b, qt = divmod(r, QT)
        for e in range(t["row_ptr"][r], t["row_ptr"][r + 1]):
            kt = t["col_idx"][e]
            blk = np.zeros((128, 128), dtype=bool)
            sub = mask[b, qt * 128:(qt + 1) * 128, kt * 128:(kt + 1) * 128]
            blk[:sub.shape[0], :sub.shape[1]] = sub
            if t["kind"][e] == 1:
                assert blk.all()
            else:
                assert blk.any() and not blk.all()
                w = t["bits"][t["pidx"][e]].reshape(128, 4)
                qq, kk = np.nonzero(np.ones((128, 128), dtype=bool))
                got = (w[qq, kk // 32] >> (kk % 32).astype(np.uint32)) & 1
                assert np.array_equal(got.reshape(128, 128).astype(bool), blk)
    # CSC is the transpose of CSR
    pairs_csr = set()
    for r in range(B * QT):
        for e in range(t["row_ptr"][r], t["row_ptr"][r + 1]):
            pairs_csr.add((r // QT, r % QT, int(t["col_idx"][e]), e))
    pairs_csc = set()
    for c in range(B * KT):
        for e in range(t["colT_ptr"][c], t["colT_ptr"][c + 1]):
            pairs_csc.add((c // KT, int(t["rowT_idx"][e]), c % KT, int(t["csc_map"][e])))
    assert pairs_csr == pairs_csc


def test_tile_list_random_masks():
    rng = np.random.default_rng(3)
    for (Nq, Nk) in [(300, 300), (128, 256), (257, 129)]:
        m = W.random_mask(rng, 2, Nq, Nk, density=0.3, empty_rows=3)
        t = tiles.tile_list(m)
        _check_tile_invariants(m, t)
        assert set(np.unique(t["kind"])) <= {1, 2}


def test_tile_list_packed_documents_count():
    rng = np.random.default_rng(5)
    docs = W.packed_documents(rng, 1000, 100)
    m, c = W.causal_document_mask(docs, 1000)
    assert int(m.sum()) == sum(l * (l + 1) // 2 for l in docs)
    t = tiles.tile_list(m[None])
    _check_tile_invariants(m[None], t)
    # diagonal blocks are never FULL (causal), and every diagonal block is present
    QT = t["QT"]
    diag = [e for r in range(QT) for e in range(t["row_ptr"][r], t["row_ptr"][r + 1])
            if t["col_idx"][e] == r]
    assert len(diag) == QT and all(t["kind"][e] == 2 for e in diag)


def test_tile_list_lengths_closed_form():
    rng = np.random.default_rng(8)
    for _ in range(5):
        npad = int(rng.integers(1, 700))
        lengths = rng.integers(0, npad + 1, int(rng.integers(1, 6)))
        t = tiles.tile_list_from_lengths(lengths, npad)
        assert len(t["col_idx"]) == int(sum((-(-int(n) // 128)) ** 2 for n in lengths))
        assert int((t["kind"] == 1).sum()) == int(sum((int(n) // 128) ** 2 for n in lengths))
        _check_tile_invariants(tiles.mask_from_lengths(lengths, npad), t)


# ----------------------------------------------------------------------------------------
# workloads
# ----------------------------------------------------------------------------------------

def test_workload_shapes():
    w1 = W.config(1)
    assert (w1.B, w1.Nq, w1.H, w1.d) == (4, 128, 2, 64) and list(w1.lengths) == [37, 64, 100, 128]
    assert w1.pairs() == 37 ** 2 + 64 ** 2 + 100 ** 2 + 128 ** 2 == 31849
    w2 = W.config(2)
    assert w2.B == 32 and w2.H == 8 and w2.d == 64
    assert w2.lengths.min() >= 200 and w2.lengths.max() <= 2048 and w2.Nq == w2.lengths.max()
    w5 = W.config(5)
    assert np.array_equal(w5.lengths, w2.lengths) and w5.seed == w2.seed
    w4 = W.config(4)
    assert w4.mask.shape == (4, 8192, 8192)
    for b in range(4):
        assert sum(w4.doc_lengths[b]) == 8192
        assert int(w4.mask[b].sum()) == sum(l * (l + 1) // 2 for l in w4.doc_lengths[b])
    t = W.tensors(w1)
    assert t["q"].dtype.itemsize == 2 and tuple(t["q"].shape) == (4, 128, 2, 64)


# ----------------------------------------------------------------------------------------
# planted mistakes: the pins above must catch each of them
# ----------------------------------------------------------------------------------------

def test_planted_sign_error_in_sigmoid_is_caught(monkeypatch):
    monkeypatch.setattr(A, "sigmoid", lambda x: np.exp(-np.logaddexp(0.0, x)))  # sigma(-x)
    with pytest.raises(AssertionError):
        test_golden_sigmoid_bias_points()


def test_planted_dropped_term_in_backward_is_caught():
    def bad_bwd(q, k, v, do, mr, bias, scale, epi, o=None):
        # drops the (1 - p) factor of sigma'
        m = mr(0, q.shape[0])
        s = scale * q @ k.T + bias[:, None]
        p, _ = A.weights(s, m, epi)
        ds = (do @ v.T) * p
        return scale * ds @ k, scale * ds.T @ q, p.T @ do
    assert _fd_check(A.SIGMOID, 3, bwd=bad_bwd) > 1e-3


def test_planted_transposed_operand_is_caught():
    def bad_bwd(q, k, v, do, mr, bias, scale, epi, o=None):
        dq, dk, dv = A.head_backward(q, k, v, do, mr, bias, scale, epi, o)
        m = mr(0, q.shape[0])
        s = scale * q @ k.T + bias[:, None]
        p, _ = A.weights(s, m, epi)
        return dq, dk, p.T @ do[::-1]            # wrong query index in dv
    assert _fd_check(A.SIGMOID, 4, bwd=bad_bwd) > 1e-3


def test_planted_missing_D_term_in_softmax_backward_is_caught():
    def bad_bwd(q, k, v, do, mr, bias, scale, epi, o=None):
        m = mr(0, q.shape[0])
        s = scale * q @ k.T + bias[:, None]
        p, _ = A.weights(s, m, epi)
        ds = p * (do @ v.T)                      # forgot - D_i
        return scale * ds @ k, scale * ds.T @ q, p.T @ do
    assert _fd_check(A.SOFTMAX, 3, bwd=bad_bwd) > 1e-3


# ----------------------------------------------------------------------------------------
# the other mask families (Longformer, token trees)
# ----------------------------------------------------------------------------------------

def test_longformer_mask_counts():
    n, r, g = 300, 17, 5
    m = W.longformer_mask(n, r, g)
    i = np.arange(n)
    # a non-global row sees its window (clipped at the ends) plus the g global tokens
    # that lie outside the window
    for row in (g, 100, n - 1):
        lo, hi = max(0, row - r), min(n - 1, row + r)
        outside = sum(1 for j in range(g) if j < lo or j > hi)
        assert m[row].sum() == (hi - lo + 1) + outside
    assert np.all(m[:g] == 1) and np.all(m[:, :g] == 1)
    assert np.array_equal(m, m.T)
    assert m[50, 50 + r] == 1 and m[50, 50 + r + 1] == 0


def test_tree_mask_is_ancestor_closure():
    rng = np.random.default_rng(3)
    parent = W.tree_parents(rng, 40, max_children=3)
    assert parent[0] == -1 and np.all(parent[1:] < np.arange(1, 40)) and np.all(parent[1:] >= 0)
    assert np.bincount(parent[1:], minlength=40).max() <= 3
    P = 25
    m = W.tree_mask(P, parent)
    assert np.array_equal(m[:P, :P], np.tril(np.ones((P, P), dtype=np.uint8)))
    assert np.all(m[:P, P:] == 0) and np.all(m[P:, :P] == 1)
    for k in range(40):
        anc, a = set(), k
        while a >= 0:
            anc.add(a)
            a = parent[a]
        assert set(np.flatnonzero(m[P + k, P:]).tolist()) == anc


def test_row_runs_rebuild_the_tile_list_and_are_maximal():
    rng = np.random.default_rng(4)
    m = W.random_mask(rng, 2, 600, 700, density=0.3, empty_rows=2)
    t = tiles.tile_list(m)
    run_ptr, runs = tiles.row_runs(t)
    col, kind = [], []
    for r in range(len(run_ptr) - 1):
        prev = None
        for kt0, n, kd, e0 in runs[run_ptr[r]:run_ptr[r + 1]]:
            assert n >= 1 and e0 == len(col)
            if prev is not None:  # maximal: the next run is not a continuation
                assert not (kt0 == prev[0] + prev[1] and kd == prev[2])
            col.extend(range(kt0, kt0 + n))
            kind.extend([kd] * n)
            prev = (kt0, n, kd)
        assert len(col) == t["row_ptr"][r + 1]
    assert np.array_equal(np.array(col), t["col_idx"]) and np.array_equal(np.array(kind), t["kind"])
    # a padded batch: full rows are one FULL run and at most one PARTIAL tail
    tl = tiles.tile_list_from_lengths([300], 300)
    rp, rr = tiles.row_runs(tl)
    assert rr.tolist()[:2] == [[0, 2, 1, 0], [2, 1, 2, 2]]
