"""Pins of the oracle's batched entry points (CPU only).

``oracle.attention.forward`` / ``backward`` walk the [B, N, H, d] layout and pick each
(batch entry, head) slice, its bias row and its mask (from the lengths or from an element
mask).  Every GPU parity test goes through them, so they are checked here against the
pure-Python loops of ``oracle.brute`` called once per (b, h) on slices cut out by the
test itself, on non-square shapes with B != H and a different bias per batch entry, so
that a b <-> h slip, a bias taken from the wrong row or a transposed / mis-sliced mask
fails.  The method is the definition of "Better Models, Faster Training", section 2A
(s = scale q.k + b, sigma weights, b per sequence) and the softmax / softmax_1 forms of
the QuietAttention page; the padded batch is query i sees key j iff i, j < n_b (section 1
of the same page, cells padded to the longest one).

The last tests plant the mistakes named above into a copy of the oracle's own source
(on the CPU) and check that these pins catch each of them.
"""
import inspect
import math

import numpy as np
import pytest

from oracle import attention as A
from oracle import brute, tiles

EPIS = (A.SIGMOID, A.SOFTMAX, A.SOFTMAX1)


def _case(seed, B=3, Nq=9, Nk=11, H=2, d=4, density=0.55):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, Nq, H, d)) * 1.3
    k = rng.standard_normal((B, Nk, H, d)) * 1.3
    v = rng.standard_normal((B, Nk, H, d))
    do = rng.standard_normal((B, Nq, H, d))
    mask = (rng.random((B, Nq, Nk)) < density).astype(np.uint8)
    mask[0, 2] = 0                      # a query with no key
    mask[1, :, 3] = 0                   # a key no query sees
    mask[2, 5, :] = 1                   # a full row
    # a different bias in every batch entry and row, so that bias[b] vs bias[h] differs
    bias = rng.standard_normal((B, Nq)) - 1.0 + np.arange(B)[:, None]
    return q, k, v, do, mask, bias


def _brute_batched(q, k, v, do, mask_of_b, bias, scale, epi):
    """Per-(b, h) brute force on slices cut here, reassembled into [B, N, H, d]."""
    B, Nq, H, d = q.shape
    Nk = k.shape[1]
    o = np.zeros((B, Nq, H, v.shape[3]))
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    for b in range(B):
        m = mask_of_b(b).tolist()
        for h in range(H):
            qs, ks, vs, dos = (x[b, :, h].tolist() for x in (q, k, v, do))
            ob, _ = brute.forward_head(qs, ks, vs, m, list(bias[b]), scale, epi)
            gq, gk, gv = brute.backward_head(qs, ks, vs, dos, m, list(bias[b]), scale, epi)
            o[b, :, h] = ob
            dq[b, :, h], dk[b, :, h], dv[b, :, h] = gq, gk, gv
    return o, dq, dk, dv


def _batched_error(fwd, bwd, epi, seed, square=False):
    """max |oracle - brute| over O, dQ, dK, dV of the batched calls with an element mask."""
    q, k, v, do, mask, bias = _case(seed, Nk=9 if square else 11)
    scale = 0.43
    o, _ = fwd(q, k, v, bias, scale, epi, mask=mask)
    g = bwd(q, k, v, do, bias, scale, epi, mask=mask)
    ref = _brute_batched(q, k, v, do, lambda b: mask[b].astype(bool), bias, scale, epi)
    return max(float(np.max(np.abs(x - r))) for x, r in zip((o,) + tuple(g), ref))


@pytest.mark.parametrize("epi", EPIS)
@pytest.mark.parametrize("seed", [0, 1])
def test_batched_mask_forward_backward_match_brute_force(epi, seed):
    assert _batched_error(A.forward, A.backward, epi, seed) <= 1e-11
    assert _batched_error(A.forward, A.backward, epi, seed, square=True) <= 1e-11


@pytest.mark.parametrize("epi", EPIS)
def test_batched_lengths_match_brute_force(epi):
    """The lengths branch: B = 4 entries with n = 0, 3, Npad, 7 and H = 3."""
    rng = np.random.default_rng(7 + epi)
    B, N, H, d = 4, 10, 3, 4
    lengths = np.array([0, 3, N, 7])
    q, k, v, do = (rng.standard_normal((B, N, H, d)) for _ in range(4))
    bias = rng.standard_normal((B, N)) - np.arange(B)[:, None]
    o, _ = A.forward(q, k, v, bias, 0.5, epi, lengths=lengths)
    g = A.backward(q, k, v, do, bias, 0.5, epi, lengths=lengths)
    idx = np.arange(N)

    def mask_of_b(b):
        valid = idx < lengths[b]
        return valid[:, None] & valid[None, :]

    ref = _brute_batched(q, k, v, do, mask_of_b, bias, 0.5, epi)
    for x, r in zip((o,) + tuple(g), ref):
        np.testing.assert_allclose(x, r, rtol=1e-11, atol=1e-13)
    assert np.all(o[0] == 0) and all(np.all(x[0] == 0) for x in g)


@pytest.mark.parametrize("epi", EPIS)
def test_mask_of_lengths_equals_lengths(epi):
    """forward / backward given the element mask of a padded batch agree exactly with the
    same calls given the lengths."""
    rng = np.random.default_rng(3)
    B, N, H, d = 3, 140, 2, 8
    lengths = np.array([140, 1, 77])
    q, k, v, do = (rng.standard_normal((B, N, H, d)) for _ in range(4))
    bias = rng.standard_normal((B, N))
    m = tiles.mask_from_lengths(lengths, N)
    o1, l1 = A.forward(q, k, v, bias, 0.3, epi, lengths=lengths)
    o2, l2 = A.forward(q, k, v, bias, 0.3, epi, mask=m)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)
    for x, y in zip(A.backward(q, k, v, do, bias, 0.3, epi, lengths=lengths),
                    A.backward(q, k, v, do, bias, 0.3, epi, mask=m)):
        np.testing.assert_array_equal(x, y)


def test_random_mask_forward_at_tile_sizes_matches_brute_force_rows():
    """A mask wider than the oracle's 256-row chunk, checked on sampled rows by brute force."""
    rng = np.random.default_rng(12)
    B, Nq, Nk, H, d = 2, 300, 260, 2, 4
    q, k, v = rng.standard_normal((B, Nq, H, d)), rng.standard_normal((B, Nk, H, d)), \
        rng.standard_normal((B, Nk, H, d))
    mask = (rng.random((B, Nq, Nk)) < 0.05).astype(np.uint8)
    mask[1, 299] = 0
    bias = rng.standard_normal((B, Nq)) - 2.0 * np.arange(B)[:, None]
    for epi in EPIS:
        o, _ = A.forward(q, k, v, bias, 0.5, epi, mask=mask)
        for b in range(B):
            for h in range(H):
                for i in (0, 1, 255, 256, 257, 299):
                    ob, _ = brute.forward_head(q[b, i:i + 1, h].tolist(), k[b, :, h].tolist(),
                                               v[b, :, h].tolist(), mask[b, i:i + 1].astype(bool).tolist(),
                                               [bias[b, i]], 0.5, epi)
                    np.testing.assert_allclose(o[b, i, h], ob[0], rtol=1e-12, atol=1e-14)


# ----------------------------------------------------------------------------------------
# planted mistakes in a copy of the oracle's own source
# ----------------------------------------------------------------------------------------

def _mutant(func, old, new):
    """A copy of ``func`` (an oracle.attention function) with ``old`` replaced by ``new``
    in its source, compiled in a copy of the module's namespace."""
    src = inspect.getsource(func)
    assert old in src, old
    ns = dict(vars(A))
    exec(compile(src.replace(old, new), "<mutant>", "exec"), ns)
    return ns[func.__name__], ns


def _caught(fwd, bwd, square=False):
    try:
        return _batched_error(fwd, bwd, A.SIGMOID, 0, square=square) > 1e-6
    except (IndexError, ValueError):
        return True                      # a shape error is a catch too


def test_planted_bias_of_head_instead_of_batch_is_caught():
    fwd, _ = _mutant(A.forward, "bias[b], scale", "bias[h], scale")
    assert _caught(fwd, A.backward)
    bwd, _ = _mutant(A.backward, "mr, bias[b], scale", "mr, bias[h], scale")
    assert _caught(A.forward, bwd)


def test_planted_batch_head_swap_is_caught():
    fwd, _ = _mutant(A.forward, "k[b, :, h], v[b, :, h]", "k[h, :, b], v[h, :, b]")
    assert _caught(fwd, A.backward, square=True)


def _wrappers_with_mask_provider(old, new):
    """forward / backward compiled against a mask_provider whose source has ``old``
    replaced by ``new``."""
    mp, ns = _mutant(A.mask_provider, old, new)
    ns["mask_provider"] = mp
    exec(compile(inspect.getsource(A.forward), "<mutant>", "exec"), ns)
    exec(compile(inspect.getsource(A.backward), "<mutant>", "exec"), ns)
    return ns["forward"], ns["backward"]


def test_planted_transposed_mask_is_caught():
    fwd, bwd = _wrappers_with_mask_provider("return mask[b, i0:i1]", "return mask[b].T[i0:i1]")
    assert _caught(fwd, bwd, square=True)


def test_planted_mask_of_wrong_batch_entry_is_caught():
    fwd, bwd = _wrappers_with_mask_provider("return mask[b, i0:i1]", "return mask[0, i0:i1]")
    assert _caught(fwd, bwd)


def test_planted_length_off_by_one_is_caught():
    fwd, _ = _wrappers_with_mask_provider("jv = np.arange(Nk) < n", "jv = np.arange(Nk) <= n")
    with pytest.raises(AssertionError):
        rng = np.random.default_rng(1)
        B, N, H, d = 2, 6, 2, 3
        lengths = np.array([3, 5])
        q, k, v = (rng.standard_normal((B, N, H, d)) for _ in range(3))
        bias = np.zeros((B, N))
        o, _ = fwd(q, k, v, bias, 0.5, A.SIGMOID, lengths=lengths)
        idx = np.arange(N)
        ref = _brute_batched(q, k, v, np.zeros_like(q),
                             lambda b: (idx < lengths[b])[:, None] & (idx < lengths[b])[None, :],
                             bias, 0.5, A.SIGMOID)[0]
        np.testing.assert_allclose(o, ref, rtol=1e-11, atol=1e-13)


def test_scale_is_used_not_rederived():
    """The wrappers pass the caller's scale through (1/sqrt(d) is the caller's choice)."""
    q, k, v, do, mask, bias = _case(5)
    o1, _ = A.forward(q, k, v, bias, 0.43, A.SIGMOID, mask=mask)
    o2, _ = A.forward(q, k, v, bias, 1 / math.sqrt(q.shape[3]), A.SIGMOID, mask=mask)
    assert np.max(np.abs(o1 - o2)) > 1e-3
