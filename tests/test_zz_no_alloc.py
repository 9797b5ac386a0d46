"""The allocation-free backward entry point, sigattn_bwd_noalloc.

It serves callers that cannot call cudaMalloc -- code whose device memory is owned by
another memory manager (a framework's caching allocator, a host application's fixed budget)
and step loops that cannot take cudaMalloc's device-wide synchronisation.  Instead of a
caller-provided workspace it uses a scratch array that lives in the library's device image.

Checked here through the C ABI: two calls in a row (different shapes, so the second call
runs over what the first one left in the shared array) give bit-identical dQ, dK, dV to the
existing sigattn_bwd with a caller workspace -- both run the same kernels on the same
values, so anything but equality would mean a wrong scratch address or a stale value --
for the two softmax modes (which use the scratch) and for sigmoid (which passes no
workspace); one case is also checked against the float64 oracle within the parity
tolerance of the other GPU tests; sizes past the array's limit are rejected.  This file is
collected last, and sets up everything it uses, so it passes alone in a fresh process and
after the other tests.
"""
import numpy as np
import pytest
import torch

from oracle import attention as A
from padded_variable_length_b200 import workloads as W
from tests import harness as Hn

pytestmark = pytest.mark.gpu


def _noalloc(Bd, plan, epi, d, bias, o, lse, scale):
    q, k, v, do = d["q"], d["k"], d["v"], d["do"]
    B, Nq, H, hd = q.shape
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    bp, bs = (bias.data_ptr(), bias.stride(0)) if bias is not None else (None, 0)
    rc = Bd.lib.sigattn_bwd_noalloc(
        plan.handle, epi, H, hd, scale, q.data_ptr(), Bd._strides(q), k.data_ptr(), Bd._strides(k),
        v.data_ptr(), Bd._strides(v), o.data_ptr(), Bd._strides(o), do.data_ptr(), Bd._strides(do),
        bp, bs, lse.data_ptr() if lse is not None else None, dq.data_ptr(), Bd._strides(dq),
        dk.data_ptr(), Bd._strides(dk), dv.data_ptr(), Bd._strides(dv),
        torch.cuda.current_stream().cuda_stream)
    return rc, dq, dk, dv


def test_noalloc_backward_matches_workspace_backward_twice():
    from padded_variable_length_b200 import binding as Bd
    cases = [
        (W.padded_workload("call1", [0, 129, 300, 385], H=3, d=64, epilogue=W.SOFTMAX, seed=31,
                           npad=385), W.SOFTMAX),
        (W.padded_workload("call2", [200, 77], H=2, d=128, epilogue=W.SOFTMAX1, seed=32,
                           npad=200), W.SOFTMAX1),
        (W.padded_workload("call3", [5, 256, 131], H=2, d=64, epilogue=W.SIGMOID, seed=33,
                           npad=256), W.SIGMOID),
    ]
    for w, epi in cases:
        t = W.tensors(w, with_grad=True)
        d, plan, bias = Hn.device_setup(w, t)
        b_arg = bias if epi == W.SIGMOID else None
        scale = 1.0 / np.sqrt(w.d)
        o, lse = Bd.fwd(plan, d["q"], d["k"], d["v"], b_arg, epi)
        ref = Bd.bwd(plan, d["q"], d["k"], d["v"], o, d["do"], b_arg, epi, lse=lse)
        rc, dq, dk, dv = _noalloc(Bd, plan, epi, d, b_arg, o, lse, scale)
        assert rc == 0, Bd.lib.sigattn_error_string(rc)
        assert Bd.get_status() == 0
        for name, got, want in (("dQ", dq, ref[0]), ("dK", dk, ref[1]), ("dV", dv, ref[2])):
            assert torch.equal(got, want), f"noalloc {w.name} {name} differs from sigattn_bwd"
        if epi == W.SOFTMAX:
            # and against the float64 oracle, within the parity tolerance
            want = A.backward(Hn.to_f64(t["q"]), Hn.to_f64(t["k"]), Hn.to_f64(t["v"]),
                              Hn.to_f64(t["do"]), Hn.oracle_bias(w, epi), scale, epi,
                              lengths=w.lengths)
            for name, got, r, rows in (("dQ", dq, want[0], Hn.valid_rows_q(w)),
                                       ("dK", dk, want[1], Hn.valid_rows_k(w)),
                                       ("dV", dv, want[2], Hn.valid_rows_k(w))):
                Hn.check_close(Hn.to_f64(got), r, f"noalloc {w.name} {name} vs oracle", rows)
                Hn.check_pad_zero(Hn.to_f64(got), w, name, "q" if name == "dQ" else "k")


def test_noalloc_rejects_sizes_past_the_scratch_limit():
    from padded_variable_length_b200 import binding as Bd
    limit = 1 << 21
    npad = limit // 8 + 128  # B * H * Nq > limit with B = 1, H = 8
    plan = Bd.Plan.from_lengths(torch.tensor([5], dtype=torch.int32, device="cuda"), npad)
    x = torch.zeros((1, 128, 8, 64), dtype=torch.bfloat16, device="cuda")
    d = {"q": x, "k": x, "v": x, "do": x}
    lse = torch.zeros((1, 8, 128), dtype=torch.float32, device="cuda")
    rc, *_ = _noalloc(Bd, plan, W.SOFTMAX, d, None, x, lse, 0.125)
    assert rc == -2  # SIGATTN_ERR_UNSUPPORTED, nothing launched
    assert Bd.get_status() == 0
