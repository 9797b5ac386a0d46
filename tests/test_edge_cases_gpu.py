"""Degenerate plans through the CUDA path: a batch in which every sequence is empty, an
element mask that keeps nothing, and one that keeps everything on whole tiles.  Outputs
are preset to a sentinel, so every row the kernels must write (as values or as zeros) is
checked, and compared with the float64 oracle."""
import math

import numpy as np
import pytest
import torch

from oracle import attention as A
from padded_variable_length_b200 import workloads as W
from tests import harness as Hn

pytestmark = pytest.mark.gpu

EPIS = (W.SIGMOID, W.SOFTMAX, W.SOFTMAX1)
SENTINEL = 3.0


def _run(w: W.Workload, epi: int, fused: bool):
    from padded_variable_length_b200 import binding as Bd
    t = W.tensors(w, with_grad=True)
    d, plan, bias = Hn.device_setup(w, t)
    b_arg = bias if epi == W.SIGMOID else None
    o = torch.full_like(d["q"], SENTINEL)
    lse = torch.full((w.B, w.H, w.Nq), SENTINEL, dtype=torch.float32, device="cuda")
    Bd.fwd(plan, d["q"], d["k"], d["v"], b_arg, epi, out=o, lse=lse)
    dq, dk, dv = (torch.full_like(d[x], SENTINEL) for x in ("q", "k", "v"))
    run = Bd.bwd_fused if fused else Bd.bwd
    run(plan, d["q"], d["k"], d["v"], o, d["do"], b_arg, epi, lse=lse, dq=dq, dk=dk, dv=dv)
    assert Bd.get_status() == 0
    scale = 1.0 / math.sqrt(w.d)
    ref_o, ref_lse = A.forward(Hn.to_f64(t["q"]), Hn.to_f64(t["k"]), Hn.to_f64(t["v"]),
                               Hn.oracle_bias(w, epi), scale, epi, lengths=w.lengths, mask=w.mask)
    ref = dict(zip(("dq", "dk", "dv"), A.backward(
        Hn.to_f64(t["q"]), Hn.to_f64(t["k"]), Hn.to_f64(t["v"]), Hn.to_f64(t["do"]),
        Hn.oracle_bias(w, epi), scale, epi, lengths=w.lengths, mask=w.mask)))
    all_q = np.ones((w.B, w.Nq), bool)
    all_k = np.ones((w.B, w.Nk), bool)
    Hn.check_close(Hn.to_f64(o), ref_o, "O", all_q)
    for name, x, rows in (("dq", dq, all_q), ("dk", dk, all_k), ("dv", dv, all_k)):
        Hn.check_close(Hn.to_f64(x), ref[name], name, rows)
    if epi != W.SIGMOID:
        g = lse.cpu().numpy().astype(np.float64)
        fin = np.isfinite(ref_lse)
        assert np.all(np.abs(g[fin] - ref_lse[fin]) <= 2e-3 * np.maximum(1, np.abs(ref_lse[fin])))
        if epi == W.SOFTMAX:
            assert np.all(np.isneginf(g[np.isneginf(ref_lse)]))
    return {"o": o, "dq": dq, "dk": dk, "dv": dv}


@pytest.mark.parametrize("fused", [False, True])
@pytest.mark.parametrize("epi", EPIS)
def test_every_sequence_empty(epi, fused):
    """Lengths all 0: the plan lists no tile; O, dQ, dK, dV are written as zeros."""
    w = W.padded_workload("all_empty", [0, 0, 0], H=2, d=64, epilogue=epi, seed=61, npad=300)
    out = _run(w, epi, fused)
    for name, x in out.items():
        assert torch.all(x == 0), f"{name}: not all zero"


@pytest.mark.parametrize("fused", [False, True])
@pytest.mark.parametrize("epi", EPIS)
def test_mask_that_keeps_nothing(epi, fused):
    """An all-zero element mask: every row sees no key."""
    m = np.zeros((2, 300, 260), np.uint8)
    w = W.masked_workload("keep_none", m, np.ones((2, 300), np.int32), H=2, d=64, epilogue=epi,
                          seed=62)
    out = _run(w, epi, fused)
    for name, x in out.items():
        assert torch.all(x == 0), f"{name}: not all zero"


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("epi", EPIS)
def test_mask_of_whole_full_tiles(d, epi):
    """An all-one mask on a whole number of tiles: every tile FULL, none PARTIAL."""
    from padded_variable_length_b200 import binding as Bd
    m = np.ones((2, 256, 384), np.uint8)
    w = W.masked_workload("keep_all", m, np.full((2, 256), 384, np.int32), H=2, d=d, epilogue=epi,
                          seed=63)
    t = W.tensors(w, with_grad=True)
    _, plan, _ = Hn.device_setup(w, t)
    z = plan.sizes()
    assert z["partial"] == 0 and z["full"] == 2 * 2 * 3
    _run(w, epi, fused=False)
    if d == 64:
        _run(w, epi, fused=True)
