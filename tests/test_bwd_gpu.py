"""Backward parity: dQ, dK, dV from the CUDA path (dK/dV kernel + dQ kernel, through the
C ABI) vs the float64 oracle's analytic backward, element by element; pad rows exactly 0."""
import math

import numpy as np
import pytest
import torch

from oracle import attention as A
from padded_variable_length_b200 import workloads as W
from tests import harness as Hn

pytestmark = pytest.mark.gpu

EPIS = (W.SIGMOID, W.SOFTMAX, W.SOFTMAX1)


def _bwd_parity(w: W.Workload, epi: int, t=None, fused=False):
    from padded_variable_length_b200 import binding as Bd
    t = t or W.tensors(w, with_grad=True)
    d, plan, bias = Hn.device_setup(w, t)
    b_arg = bias if epi == W.SIGMOID else None
    o, lse = Bd.fwd(plan, d["q"], d["k"], d["v"], b_arg, epi)
    run = Bd.bwd_fused if fused else Bd.bwd
    dq, dk, dv = run(plan, d["q"], d["k"], d["v"], o, d["do"], b_arg, epi, lse=lse)
    assert Bd.get_status() == 0
    got = {n: Hn.to_f64(x) for n, x in (("dq", dq), ("dk", dk), ("dv", dv))}
    ref = dict(zip(("dq", "dk", "dv"), A.backward(
        Hn.to_f64(t["q"]), Hn.to_f64(t["k"]), Hn.to_f64(t["v"]), Hn.to_f64(t["do"]),
        Hn.oracle_bias(w, epi), 1.0 / math.sqrt(w.d), epi, lengths=w.lengths, mask=w.mask)))
    name = W.EPILOGUE_NAMES[epi]
    Hn.check_close(got["dq"], ref["dq"], f"dQ[{name}]", Hn.valid_rows_q(w))
    Hn.check_close(got["dk"], ref["dk"], f"dK[{name}]", Hn.valid_rows_k(w))
    Hn.check_close(got["dv"], ref["dv"], f"dV[{name}]", Hn.valid_rows_k(w))
    Hn.check_pad_zero(got["dq"], w, "dQ", "q")
    Hn.check_pad_zero(got["dk"], w, "dK", "k")
    Hn.check_pad_zero(got["dv"], w, "dV", "k")
    return got, ref


@pytest.mark.parametrize("epi", EPIS)
def test_tiny_workload_backward(epi):
    w = W.config(1, epilogue=epi)
    w.backward = True
    _bwd_parity(w, epi)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("epi", EPIS)
def test_ragged_lengths_backward(d, epi):
    w = W.padded_workload("ragged", [0, 1, 127, 128, 129, 300, 385], H=2, d=d, epilogue=epi,
                          backward=True, seed=6, npad=385)
    _bwd_parity(w, epi)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("epi", EPIS)
def test_element_mask_backward(d, epi):
    rng = np.random.default_rng(100 + d + epi)
    m = W.random_mask(rng, 2, 300, 300, density=0.4, empty_rows=3)
    counts = np.maximum(m.sum(axis=2), 1).astype(np.int32)
    w = W.masked_workload("mask", m, counts, H=2, d=d, epilogue=epi, backward=True, seed=10)
    _bwd_parity(w, epi)


def test_element_mask_rectangular_backward():
    rng = np.random.default_rng(4)
    m = W.random_mask(rng, 2, 200, 333, density=0.5, empty_rows=2)
    counts = np.maximum(m.sum(axis=2), 1).astype(np.int32)
    for epi in EPIS:
        w = W.masked_workload("rect", m, counts, H=2, d=64, epilogue=epi, backward=True, seed=5)
        _bwd_parity(w, epi)


def test_q_zero_gives_zero_dk():
    """With Q = 0: dK = scale sum_i ds_ij q_i = 0 exactly; dV_j = sum_i dO_i / (n + 1)."""
    from padded_variable_length_b200 import binding as Bd
    w = W.padded_workload("qzero", [130, 256], H=2, d=64, backward=True, seed=2, npad=256)
    t = W.tensors(w)
    t["q"].zero_()
    d, plan, bias = Hn.device_setup(w, t)
    o, _ = Bd.fwd(plan, d["q"], d["k"], d["v"], bias)
    dq, dk, dv = Bd.bwd(plan, d["q"], d["k"], d["v"], o, d["do"], bias)
    assert torch.all(dk == 0)
    dvf = Hn.to_f64(dv)
    do = Hn.to_f64(t["do"])
    for b, n in enumerate(w.lengths):
        want = do[b, :n].sum(0) / (n + 1)
        assert np.max(np.abs(dvf[b, :n] - want[None])) <= 1e-2 * np.max(np.abs(want)) + 1e-3


@pytest.mark.parametrize("epi", EPIS)
def test_single_cell_full_backward(epi):
    """The single-cell batch (B=32, log-uniform lengths in [200, 2048], H=8, d=64), whole."""
    _bwd_parity(W.config(2 if epi == W.SIGMOID else 5, epilogue=epi), epi)


# ----------------------------------------------------------------------------------------
# the fused backward (one walk over the k-tile columns; dQ through TMA reduce-adds), d = 64
# ----------------------------------------------------------------------------------------

@pytest.mark.parametrize("epi", EPIS)
def test_fused_tiny_workload(epi):
    w = W.config(1, epilogue=epi)
    w.backward = True
    _bwd_parity(w, epi, fused=True)


@pytest.mark.parametrize("epi", EPIS)
def test_fused_ragged_lengths(epi):
    w = W.padded_workload("ragged", [0, 1, 127, 128, 129, 300, 385], H=2, d=64, epilogue=epi,
                          backward=True, seed=16, npad=385)
    _bwd_parity(w, epi, fused=True)


@pytest.mark.parametrize("epi", EPIS)
def test_fused_element_mask(epi):
    rng = np.random.default_rng(200 + epi)
    m = W.random_mask(rng, 2, 300, 300, density=0.4, empty_rows=3)
    counts = np.maximum(m.sum(axis=2), 1).astype(np.int32)
    w = W.masked_workload("mask", m, counts, H=3, d=64, epilogue=epi, backward=True, seed=20)
    _bwd_parity(w, epi, fused=True)


def test_fused_element_mask_rectangular():
    rng = np.random.default_rng(14)
    m = W.random_mask(rng, 2, 200, 333, density=0.5, empty_rows=2)
    counts = np.maximum(m.sum(axis=2), 1).astype(np.int32)
    for epi in EPIS:
        w = W.masked_workload("rect", m, counts, H=2, d=64, epilogue=epi, backward=True, seed=15)
        _bwd_parity(w, epi, fused=True)


@pytest.mark.parametrize("epi", EPIS)
def test_fused_single_cell_full(epi):
    """The single-cell batch (B=32, log-uniform lengths in [200, 2048], H=8, d=64), whole."""
    _bwd_parity(W.config(2 if epi == W.SIGMOID else 5, epilogue=epi), epi, fused=True)


def test_fused_matches_split_and_reuses_a_dirty_workspace():
    """Fused and split backward agree to within rounding; a workspace full of NaNs (or of
    an earlier call's values) gives the same result: every accumulator row that is read is
    zeroed first."""
    from padded_variable_length_b200 import binding as Bd
    w = W.padded_workload("fs", [700, 129, 1, 0, 256], H=4, d=64, backward=True, seed=41, npad=700)
    t = W.tensors(w, with_grad=True)
    d, plan, bias = Hn.device_setup(w, t)
    o, _ = Bd.fwd(plan, d["q"], d["k"], d["v"], bias)
    ref = Bd.bwd(plan, d["q"], d["k"], d["v"], o, d["do"], bias)
    need = Bd.bwd_fused_workspace_bytes(plan, w.H, w.d)
    ws = torch.full(((need + 3) // 4,), float("nan"), dtype=torch.float32, device="cuda")
    for _ in range(2):
        got = Bd.bwd_fused(plan, d["q"], d["k"], d["v"], o, d["do"], bias, workspace=ws)
        assert Bd.get_status() == 0
        dq_err = (got[0].float() - ref[0].float()).abs().max().item()
        assert dq_err <= 1e-2 * ref[0].float().abs().max().item() + 1e-4
        Hn.check_pad_zero(Hn.to_f64(got[0]), w, "dQ fused", "q")
        for name, x, y in (("dK", got[1], ref[1]), ("dV", got[2], ref[2])):
            rows = torch.from_numpy(Hn.valid_rows_k(w)).cuda()
            diff = (x.float() - y.float()).abs()[rows].max().item()
            assert diff <= 1e-2 * y.float().abs().max().item(), f"{name} fused vs split {diff}"


def test_fused_rejects_bad_workspace_and_head_dim():
    from padded_variable_length_b200 import binding as Bd
    w = W.config(1)
    t = W.tensors(w, with_grad=True)
    d, plan, bias = Hn.device_setup(w, t)
    o, _ = Bd.fwd(plan, d["q"], d["k"], d["v"], bias)
    small = torch.empty(16, dtype=torch.float32, device="cuda")
    with pytest.raises(Bd.SigattnError) as e:
        Bd.bwd_fused(plan, d["q"], d["k"], d["v"], o, d["do"], bias, workspace=small)
    assert e.value.code == -1
    x = torch.zeros((4, 128, 2, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(Bd.SigattnError) as e:
        Bd.bwd_fused(plan, x, x, x, x, x, bias)
    assert e.value.code == -2
    assert Bd.get_status() == 0
