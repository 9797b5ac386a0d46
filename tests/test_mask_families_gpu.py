"""The other block-mask families of "Binary Block Masking for FlashAttention" (section on
applications: tree attention masks for parallel decoding, Longformer masks) through the
element-mask planner and the attention kernels (GPU).

* the plan of each full-size workload (B=4 rows; Longformer N=8192, radius 256, 32 global
  tokens; tree N=4096: causal prefix of 3840 and a 256-node token tree) is bit-exact with
  the oracle's brute-force tile list;
* forward and backward match the float64 oracle element by element on smaller instances of
  the same families (several tiles, ragged tails, every epilogue);
* at full size (H=16, d=128, sigmoid), sampled rows of O, dQ and key rows of dK, dV match
  the oracle computed one by one.
"""
import math

import numpy as np
import pytest
import torch

from oracle import attention as A
from oracle import tiles as OT
from padded_variable_length_b200 import workloads as W
from tests import harness as Hn
from tests.test_plan_gpu import _compare

pytestmark = pytest.mark.gpu

EPIS = (W.SIGMOID, W.SOFTMAX, W.SOFTMAX1)


@pytest.mark.parametrize("kind", ["longformer", "tree"])
def test_plan_of_full_size_family_is_bit_exact(kind):
    from padded_variable_length_b200 import binding as Bd
    w = W.mask_family(kind)
    plan = Bd.Plan.from_mask(torch.from_numpy(w.mask).cuda())
    _compare(plan, OT.tile_list(w.mask))


def _small(kind, epi, d, seed):
    rng = np.random.default_rng(seed)
    if kind == "longformer":
        m = np.stack([W.longformer_mask(700, 100, 9), W.longformer_mask(700, 37, 1)])
    else:
        m = np.stack([W.tree_mask(300, W.tree_parents(rng, 90)),
                      W.tree_mask(257, W.tree_parents(rng, 133, max_children=2))])
    counts = m.sum(axis=2, dtype=np.int64).astype(np.int32)
    return W.masked_workload(kind, m, counts, H=2, d=d, epilogue=epi, backward=True, seed=seed)


@pytest.mark.parametrize("kind", ["longformer", "tree"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("epi", EPIS)
def test_family_forward_backward_parity(kind, d, epi):
    from padded_variable_length_b200 import binding as Bd
    w = _small(kind, epi, d, seed=31 + d + epi)
    t = W.tensors(w, with_grad=True)
    d_, plan, bias = Hn.device_setup(w, t)
    b_arg = bias if epi == W.SIGMOID else None
    o, lse = Bd.fwd(plan, d_["q"], d_["k"], d_["v"], b_arg, epi)
    grads = [Bd.bwd(plan, d_["q"], d_["k"], d_["v"], o, d_["do"], b_arg, epi, lse=lse)]
    if d == 64:
        grads.append(Bd.bwd_fused(plan, d_["q"], d_["k"], d_["v"], o, d_["do"], b_arg, epi, lse=lse))
    assert Bd.get_status() == 0
    f64 = {k: Hn.to_f64(v) for k, v in t.items()}
    scale = 1.0 / math.sqrt(w.d)
    bias_ref = Hn.oracle_bias(w, epi)
    ref_o, _ = A.forward(f64["q"], f64["k"], f64["v"], bias_ref, scale, epi, mask=w.mask)
    Hn.check_close(Hn.to_f64(o), ref_o, f"{kind} O")
    ref = A.backward(f64["q"], f64["k"], f64["v"], f64["do"], bias_ref, scale, epi, mask=w.mask)
    for g in grads:
        for name, x, r in zip(("dQ", "dK", "dV"), g, ref):
            Hn.check_close(Hn.to_f64(x), r, f"{kind} {name}")


def _sample_rows(rng, n, count=20):
    base = [0, 1, 127, 128, 129, n // 2, n - 2, n - 1]
    extra = rng.choice(n, size=min(count, n), replace=False).tolist()
    return np.array(sorted(set(base + extra)))


@pytest.mark.slow
@pytest.mark.parametrize("kind", ["longformer", "tree"])
def test_full_size_family_sampled(kind):
    from padded_variable_length_b200 import binding as Bd
    w = W.mask_family(kind)
    t = W.tensors(w)
    d_, plan, bias = Hn.device_setup(w, t)
    o, _ = Bd.fwd(plan, d_["q"], d_["k"], d_["v"], bias)
    dq, dk, dv = Bd.bwd(plan, d_["q"], d_["k"], d_["v"], o, d_["do"], bias)
    assert Bd.get_status() == 0
    rng = np.random.default_rng(5)
    scale = 1.0 / math.sqrt(w.d)
    bias_ref = A.bias_from_counts(w.counts)
    mp = A.mask_provider(None, w.mask, w.Nq, w.Nk)
    got = {"o": [], "dq": [], "dk": [], "dv": []}
    ref = {"o": [], "dq": [], "dk": [], "dv": []}
    for (b, h) in [(0, 0), (w.B - 1, w.H - 1)]:
        rows = _sample_rows(rng, w.Nq)
        q, k, v, do = (Hn.to_f64(t[x][b, :, h]) for x in ("q", "k", "v", "do"))
        mr = mp(b)
        o_ref, _ = A.head_forward(q, k, v, mr, bias_ref[b], scale, A.SIGMOID, rows=rows)
        dq_ref = A.query_rows_backward(q, k, v, do, mr, bias_ref[b], scale, A.SIGMOID, rows)
        dk_ref, dv_ref = A.key_columns_backward(q, k, v, do, mr, bias_ref[b], scale, A.SIGMOID, rows)
        for name, x, r in (("o", o, o_ref), ("dq", dq, dq_ref), ("dk", dk, dk_ref), ("dv", dv, dv_ref)):
            got[name].append(Hn.to_f64(x[b, rows, h]))
            ref[name].append(r)
    for name in got:
        Hn.check_close(np.concatenate(got[name]), np.concatenate(ref[name]), f"{kind} {name} (sampled)")
