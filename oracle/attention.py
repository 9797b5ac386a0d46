"""Float64 definition of attention over a padded ragged batch (test infrastructure).

Forward, for one (batch b, head h) and a query row i whose key set
J(i) = {j : mask(i, j) = 1} is not empty:

    s_ij = scale * (q_i . k_j) + bias_i                       (j in J(i))
    SIGMOID   p_ij = sigma(s_ij) = 1 / (1 + exp(-s_ij))
    SOFTMAX   p_ij = exp(s_ij) / sum_{j' in J(i)} exp(s_ij')
    SOFTMAX1  p_ij = exp(s_ij) / (1 + sum_{j' in J(i)} exp(s_ij'))
    o_i  = sum_{j in J(i)} p_ij v_j

Rows with an empty key set, and pad rows, give o_i = 0.

Sources:
  * sigmoid attention sigma(QK^T / sqrt(d) + b) V with b = -log(n): "Better
    Models, Faster Training: Sigmoid Attention for single-cell Foundation
    Models", section 2A (sigmoid attention mechanism, bias term).
  * sigma' = sigma (1 - sigma) and the diagonal Jacobian: same page, section 2B.
  * softmax attention softmax(QK^T / sqrt(d)) V and softmax_1 with
    exp(x_i) / (1 + sum_j exp(x_j)): the softmax_1 / QuietAttention page,
    sections "Les limites du softmax dans l'attention interne" and
    "Proposition : softmax_1 et QuietAttention".

Backward (analytic, float64), with L = sum(dO * O):

    dv_j = sum_i p_ij do_i
    dp_ij = do_i . v_j
    SIGMOID            ds_ij = dp_ij p_ij (1 - p_ij)
    SOFTMAX/SOFTMAX1   ds_ij = p_ij (dp_ij - D_i),  D_i = do_i . o_i
    dq_i = scale sum_j ds_ij k_j ;   dk_j = scale sum_i ds_ij q_i

softmax_1 has the same ds as softmax because it equals softmax with one more
logit fixed at 0 whose value row is the zero vector (softmax_1 page, Hacker News
comments on add_zero_attention and the "virtual logit"); that extra column adds
nothing to dv, dq or dk.  The bias is an input constant: no gradient.

Implementation: per (b, h), query rows in chunks; each chunk's score block
[rows, keys] is formed with np.matmul and the masked-out keys contribute exactly
zero.  Keys outside the smallest column range that holds every unmasked entry of
the chunk are skipped (they would only add zeros); nothing else is reordered.
"""
from __future__ import annotations

import numpy as np

SIGMOID, SOFTMAX, SOFTMAX1 = 0, 1, 2

_CHUNK = 256


def bias_from_counts(counts: np.ndarray) -> np.ndarray:
    """b = -log(n) per query row (section 2A of the sigmoid-attention page);
    rows with n = 0 (padding) get 0, a value that is never used."""
    c = np.asarray(counts, dtype=np.float64)
    out = np.zeros_like(c)
    nz = c > 0
    out[nz] = -np.log(c[nz])
    return out


def sigmoid(x: np.ndarray) -> np.ndarray:
    """1 / (1 + exp(-x)) evaluated without overflow: exp(-log(1 + exp(-x)))."""
    return np.exp(-np.logaddexp(0.0, -x))


def _logsumexp_rows(s: np.ndarray, m: np.ndarray) -> np.ndarray:
    """log sum_{j: m_ij} exp(s_ij) per row; -inf on rows with no unmasked entry."""
    sm = np.where(m, s, -np.inf)
    mx = sm.max(axis=1) if sm.shape[1] else np.full(sm.shape[0], -np.inf)
    fin = np.isfinite(mx)
    out = np.full(s.shape[0], -np.inf)
    if fin.any():
        sh = np.exp(sm[fin] - mx[fin, None])
        out[fin] = mx[fin] + np.log(sh.sum(axis=1))
    return out


def weights(s: np.ndarray, m: np.ndarray, epilogue: int):
    """Attention weights p [rows, keys] for scores s and boolean mask m.

    Returns (p, lse) where lse is the per-row log-normaliser used by the softmax
    modes (log sum exp for SOFTMAX, log(1 + sum exp) for SOFTMAX1); for SIGMOID
    lse is all-NaN (no normalisation exists)."""
    if epilogue == SIGMOID:
        p = np.where(m, sigmoid(s), 0.0)
        return p, np.full(s.shape[0], np.nan)
    lse = _logsumexp_rows(s, m)
    if epilogue == SOFTMAX1:
        lse = np.logaddexp(0.0, lse)       # log(1 + sum exp): the extra "+1"
    elif epilogue != SOFTMAX:
        raise ValueError(epilogue)
    with np.errstate(invalid="ignore"):
        p = np.where(m, np.exp(s - lse[:, None]), 0.0)
    p[~np.isfinite(lse)] = 0.0             # softmax row with no key: o = 0
    return p, lse


def _key_range(m: np.ndarray):
    cols = np.flatnonzero(m.any(axis=0))
    if cols.size == 0:
        return 0, 0
    return int(cols[0]), int(cols[-1]) + 1


def head_forward(q, k, v, mask_rows, bias, scale, epilogue, rows=None):
    """One (b, h): q [Nq, d], k/v [Nk, d] float64; mask_rows(i0, i1) -> bool
    [i1 - i0, Nk]; bias [Nq].  Returns o [Nq, d] and lse [Nq] (for ``rows`` only,
    when given: o [len(rows), d])."""
    Nq, d = q.shape
    if rows is not None:
        rows = np.asarray(rows)
        o = np.zeros((rows.size, v.shape[1]))
        lse = np.full(rows.size, np.nan)
        for t, i in enumerate(rows):
            m = mask_rows(int(i), int(i) + 1)
            a, e = _key_range(m)
            if a == e:
                lse[t] = -np.inf if epilogue == SOFTMAX else (0.0 if epilogue == SOFTMAX1 else np.nan)
                continue
            s = scale * (q[i:i + 1] @ k[a:e].T) + bias[i]
            p, l = weights(s, m[:, a:e], epilogue)
            o[t] = (p @ v[a:e])[0]
            lse[t] = l[0]
        return o, lse
    o = np.zeros((Nq, v.shape[1]))
    lse = np.full(Nq, np.nan)
    for i0 in range(0, Nq, _CHUNK):
        i1 = min(Nq, i0 + _CHUNK)
        m = mask_rows(i0, i1)
        a, e = _key_range(m)
        if a == e:
            lse[i0:i1] = -np.inf if epilogue == SOFTMAX else (0.0 if epilogue == SOFTMAX1 else np.nan)
            continue
        s = scale * (q[i0:i1] @ k[a:e].T) + bias[i0:i1, None]
        p, l = weights(s, m[:, a:e], epilogue)
        o[i0:i1] = p @ v[a:e]
        lse[i0:i1] = l
    return o, lse


def head_backward(q, k, v, do, mask_rows, bias, scale, epilogue, o=None):
    """One (b, h): returns (dq, dk, dv), all float64, for L = sum(do * o)."""
    Nq, d = q.shape
    Nk = k.shape[0]
    if epilogue != SIGMOID and o is None:
        o, _ = head_forward(q, k, v, mask_rows, bias, scale, epilogue)
    dq = np.zeros_like(q)
    dk = np.zeros((Nk, d))
    dv = np.zeros((Nk, v.shape[1]))
    for i0 in range(0, Nq, _CHUNK):
        i1 = min(Nq, i0 + _CHUNK)
        m = mask_rows(i0, i1)
        a, e = _key_range(m)
        if a == e:
            continue
        s = scale * (q[i0:i1] @ k[a:e].T) + bias[i0:i1, None]
        p, _ = weights(s, m[:, a:e], epilogue)
        dp = do[i0:i1] @ v[a:e].T
        if epilogue == SIGMOID:
            ds = dp * p * (1.0 - p)
        else:
            D = np.sum(do[i0:i1] * o[i0:i1], axis=1)
            ds = p * (dp - D[:, None])
        dq[i0:i1] = scale * (ds @ k[a:e])
        dk[a:e] += scale * (ds.T @ q[i0:i1])
        dv[a:e] += p.T @ do[i0:i1]
    return dq, dk, dv


def key_columns_backward(q, k, v, do, mask_rows, bias, scale, epilogue, cols, o=None):
    """dk, dv for the key rows ``cols`` only (one (b, h)): each needs every query."""
    Nq, d = q.shape
    cols = np.asarray(cols)
    if epilogue != SIGMOID and o is None:
        o, _ = head_forward(q, k, v, mask_rows, bias, scale, epilogue)
    dk = np.zeros((cols.size, d))
    dv = np.zeros((cols.size, v.shape[1]))
    # softmax weights need the full row normaliser
    for i0 in range(0, Nq, _CHUNK):
        i1 = min(Nq, i0 + _CHUNK)
        m = mask_rows(i0, i1)
        if not m[:, cols].any():
            continue
        if epilogue == SIGMOID:
            s = scale * (q[i0:i1] @ k[cols].T) + bias[i0:i1, None]
            p, _ = weights(s, m[:, cols], epilogue)
        else:
            a, e = _key_range(m)
            s = scale * (q[i0:i1] @ k[a:e].T) + bias[i0:i1, None]
            pf, _ = weights(s, m[:, a:e], epilogue)
            # a key outside the chunk's key range is masked for every row of the chunk:
            # its weight is 0
            p = np.zeros((i1 - i0, cols.size))
            inside = (cols >= a) & (cols < e)
            p[:, inside] = pf[:, cols[inside] - a]
        dp = do[i0:i1] @ v[cols].T
        if epilogue == SIGMOID:
            ds = dp * p * (1.0 - p)
        else:
            D = np.sum(do[i0:i1] * o[i0:i1], axis=1)
            ds = p * (dp - D[:, None])
        dk += scale * (ds.T @ q[i0:i1])
        dv += p.T @ do[i0:i1]
    return dk, dv


def query_rows_backward(q, k, v, do, mask_rows, bias, scale, epilogue, rows):
    """dq for the query rows ``rows`` only (one (b, h))."""
    rows = np.asarray(rows)
    dq = np.zeros((rows.size, q.shape[1]))
    for t, i in enumerate(rows):
        m = mask_rows(int(i), int(i) + 1)
        a, e = _key_range(m)
        if a == e:
            continue
        s = scale * (q[i:i + 1] @ k[a:e].T) + bias[i]
        p, _ = weights(s, m[:, a:e], epilogue)
        dp = do[i:i + 1] @ v[a:e].T
        if epilogue == SIGMOID:
            ds = dp * p * (1.0 - p)
        else:
            oi = p @ v[a:e]
            D = np.sum(do[i] * oi[0])
            ds = p * (dp - D)
        dq[t] = scale * (ds @ k[a:e])[0]
    return dq


# --------------------------------------------------------------------------------------
# Batched helpers over [B, N, H, d] arrays
# --------------------------------------------------------------------------------------

def mask_provider(lengths=None, mask=None, Nq=None, Nk=None):
    """Returns f(b) -> mask_rows(i0, i1) for a padded batch (lengths) or an
    element mask [B, Nq, Nk]."""
    if lengths is not None:
        lengths = np.asarray(lengths)

        def per_b(b):
            n = int(lengths[b])
            jv = np.arange(Nk) < n

            def rows(i0, i1):
                iv = np.arange(i0, i1) < n
                return iv[:, None] & jv[None, :]
            return rows
        return per_b
    mask = np.asarray(mask).astype(bool)

    def per_b(b):
        def rows(i0, i1):
            return mask[b, i0:i1]
        return rows
    return per_b


def forward(q, k, v, bias, scale, epilogue, lengths=None, mask=None):
    """q [B, Nq, H, d], k/v [B, Nk, H, d] (any float dtype), bias [B, Nq].
    Returns o [B, Nq, H, d] float64 and lse [B, H, Nq]."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, Nq, H, d = q.shape
    Nk = k.shape[1]
    mp = mask_provider(lengths, mask, Nq, Nk)
    o = np.zeros((B, Nq, H, v.shape[3]))
    lse = np.zeros((B, H, Nq))
    for b in range(B):
        mr = mp(b)
        for h in range(H):
            o[b, :, h], lse[b, h] = head_forward(q[b, :, h], k[b, :, h], v[b, :, h], mr,
                                                 bias[b], scale, epilogue)
    return o, lse


def backward(q, k, v, do, bias, scale, epilogue, lengths=None, mask=None):
    """Returns (dq, dk, dv) float64 with the layouts of q, k, v."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    do = np.asarray(do, dtype=np.float64)
    B, Nq, H, d = q.shape
    Nk = k.shape[1]
    mp = mask_provider(lengths, mask, Nq, Nk)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(B):
        mr = mp(b)
        for h in range(H):
            dq[b, :, h], dk[b, :, h], dv[b, :, h] = head_backward(
                q[b, :, h], k[b, :, h], v[b, :, h], do[b, :, h], mr, bias[b], scale, epilogue)
    return dq, dk, dv
