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
