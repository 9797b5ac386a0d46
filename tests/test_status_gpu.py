"""Failure path without a GPU fault: a device wait on a barrier that nothing arrives at
gives up after its limit, records SIGATTN_ERR_TIMEOUT in the status word, and the
context stays usable."""
import numpy as np
import pytest
import torch

from padded_variable_length_b200 import workloads as W
from tests import harness as Hn

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    from padded_variable_length_b200 import binding as Bd
    assert Bd.get_status() == 0
    Bd.selftest_wait_timeout(20_000_000)  # 20 ms
    assert Bd.get_status() == -6           # TIMEOUT recorded
    assert Bd.get_status() == 0            # and cleared by the read
    # the context still runs kernels correctly
    w = W.config(1)
    t = W.tensors(w, with_grad=False)
    d, plan, bias = Hn.device_setup(w, t)
    o, _ = Bd.fwd(plan, d["q"], d["k"], d["v"], bias)
    assert Bd.get_status() == 0
    assert torch.isfinite(o).all()


def test_argument_errors_on_device():
    from padded_variable_length_b200 import binding as Bd
    w = W.config(1)
    t = W.tensors(w, with_grad=False)
    d, plan, bias = Hn.device_setup(w, t)
    bad = torch.empty((4, 128, 2, 32), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(Bd.SigattnError) as e:
        Bd.fwd(plan, bad, bad, bad, bias)
    assert e.value.code == -2  # d = 32 unsupported
    odd = torch.empty(4 * 128 * 2 * 64 + 8, dtype=torch.bfloat16, device="cuda")[1:]
    q_mis = odd[: 4 * 128 * 2 * 64].view(4, 128, 2, 64)
    with pytest.raises(Bd.SigattnError) as e:
        Bd.fwd(plan, q_mis, d["k"], d["v"], bias)
    assert e.value.code == -3  # misaligned
    # softmax modes need an lse buffer: the raw ABI call is rejected with INVALID
    rc = Bd.lib.sigattn_fwd(plan.handle, 1, 2, 64, 0.125, d["q"].data_ptr(), Bd._strides(d["q"]),
                            d["k"].data_ptr(), Bd._strides(d["k"]), d["v"].data_ptr(),
                            Bd._strides(d["v"]), None, 0, d["q"].data_ptr(), Bd._strides(d["q"]),
                            None, None)
    assert rc == -1
    assert Bd.get_status() == 0


def test_attention_kernels_give_up_on_a_short_wait_limit_and_the_context_survives():
    """With a wait limit far shorter than any copy, the attention kernels' waits expire: each
    call records SIGATTN_ERR_TIMEOUT and returns (its CTAs let their copies land and their
    MMAs finish before they release shared memory and TMEM).  Calls after the limit is
    restored match the oracle."""
    import math

    from oracle import attention as A
    from padded_variable_length_b200 import binding as Bd
    w = W.padded_workload("abort", [37, 200, 129, 0], H=2, d=64, backward=True, seed=12, npad=200)
    t = W.tensors(w, with_grad=True)
    d, plan, bias = Hn.device_setup(w, t)
    o, _ = Bd.fwd(plan, d["q"], d["k"], d["v"], bias)
    assert Bd.get_status() == 0
    try:
        Bd.set_wait_limit_ns(1)
        runs = [
            lambda: Bd.fwd(plan, d["q"], d["k"], d["v"], bias),
            lambda: Bd.fwd(plan, d["q"], d["k"], d["v"], None, W.SOFTMAX),
            lambda: Bd.bwd(plan, d["q"], d["k"], d["v"], o, d["do"], bias),
            lambda: Bd.bwd_fused(plan, d["q"], d["k"], d["v"], o, d["do"], bias),
        ]
        for run in runs:
            run()
            assert Bd.get_status() == -6  # TIMEOUT recorded, kernel returned
    finally:
        Bd.set_wait_limit_ns(500_000_000)
    assert Bd.get_status() == 0
    o, _ = Bd.fwd(plan, d["q"], d["k"], d["v"], bias)
    dq, dk, dv = Bd.bwd_fused(plan, d["q"], d["k"], d["v"], o, d["do"], bias)
    assert Bd.get_status() == 0
    f64 = {k: Hn.to_f64(v) for k, v in t.items()}
    scale = 1.0 / math.sqrt(w.d)
    ob = A.bias_from_counts(w.counts)
    ref_o, _ = A.forward(f64["q"], f64["k"], f64["v"], ob, scale, A.SIGMOID, lengths=w.lengths)
    Hn.check_close(Hn.to_f64(o), ref_o, "O after aborts", Hn.valid_rows_q(w))
    ref = A.backward(f64["q"], f64["k"], f64["v"], f64["do"], ob, scale, A.SIGMOID, lengths=w.lengths)
    for name, x, r, rows in (("dQ", dq, ref[0], Hn.valid_rows_q(w)), ("dK", dk, ref[1], Hn.valid_rows_k(w)),
                             ("dV", dv, ref[2], Hn.valid_rows_k(w))):
        Hn.check_close(Hn.to_f64(x), r, f"{name} after aborts", rows)
