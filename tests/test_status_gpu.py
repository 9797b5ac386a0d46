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
    # big enough that some wait of every kernel has to suspend (a tiny case can find every
    # barrier complete on its first try)
    w = W.padded_workload("abort", [2000, 1500, 1999, 700, 0, 1024, 1800, 1300], H=8, d=64,
                          backward=True, seed=12, npad=2000)
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
            status = []
            for _ in range(3):  # a timeout needs one wait that is not complete on its first try
                run()
                status.append(Bd.get_status())
                if status[-1] == -6:
                    break
            assert status[-1] == -6, status  # TIMEOUT recorded, kernel returned
            assert all(x in (0, -6) for x in status)
    finally:
        Bd.set_wait_limit_ns(500_000_000)
    assert Bd.get_status() == 0
    o, _ = Bd.fwd(plan, d["q"], d["k"], d["v"], bias)
    dq, dk, dv = Bd.bwd_fused(plan, d["q"], d["k"], d["v"], o, d["do"], bias)
    assert Bd.get_status() == 0
    # the oracle on two of the batch entries (n = 700 and n = 0; entries are independent)
    sel = slice(3, 5)
    f64 = {k: Hn.to_f64(v[sel]) for k, v in t.items()}
    scale = 1.0 / math.sqrt(w.d)
    lengths = w.lengths[sel]
    ob = A.bias_from_counts(w.counts[sel])
    rows = np.arange(w.Nq)[None, :] < lengths[:, None]
    ref_o, _ = A.forward(f64["q"], f64["k"], f64["v"], ob, scale, A.SIGMOID, lengths=lengths)
    Hn.check_close(Hn.to_f64(o[sel]), ref_o, "O after aborts", rows)
    ref = A.backward(f64["q"], f64["k"], f64["v"], f64["do"], ob, scale, A.SIGMOID, lengths=lengths)
    for name, x, r in (("dQ", dq, ref[0]), ("dK", dk, ref[1]), ("dV", dv, ref[2])):
        Hn.check_close(Hn.to_f64(x[sel]), r, f"{name} after aborts", rows)
