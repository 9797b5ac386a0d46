"""Packed (unpadded) batches: sequence b is rows cu[b] .. cu[b+1] of [T, H, d] tensors
("Better Models, Faster Training", section 1: ragged cells -- here without padding them to
the longest).  A plan from the cumulative offsets lists the tiles of the padded batch with
the same lengths, so the packed path must give exactly the padded path's values on every
valid row (masked pairs contribute exact zeros whatever the rows around a sequence hold),
must write no row outside its sequences, and matches the float64 oracle."""
import math

import numpy as np
import pytest
import torch

from oracle import attention as A
from padded_variable_length_b200 import workloads as W
from tests import harness as Hn

pytestmark = pytest.mark.gpu

EPIS = (W.SIGMOID, W.SOFTMAX, W.SOFTMAX1)


def _pack(x, lengths):
    return torch.cat([x[b, :int(n)] for b, n in enumerate(lengths)], dim=0).contiguous()


def _setup(lengths, H, d, seed):
    from padded_variable_length_b200 import binding as Bd
    lengths = np.asarray(lengths, dtype=np.int32)
    w = W.padded_workload("packed", lengths, H=H, d=d, backward=True, seed=seed)
    t = W.tensors(w, with_grad=True)
    d_pad, plan_pad, bias_pad = Hn.device_setup(w, t)
    cu = torch.from_numpy(np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)).cuda()
    plan = Bd.Plan.from_cu_seqlens(cu, int(lengths.max()))
    assert plan.validate() == -1  # the library's structural check of the tile list
    packed = {k: _pack(v, lengths) for k, v in d_pad.items()}
    bias = _pack(bias_pad, lengths)
    return w, t, d_pad, plan_pad, bias_pad, packed, plan, bias


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("epi", EPIS)
def test_packed_equals_padded(d, epi):
    from padded_variable_length_b200 import binding as Bd
    lengths = [129, 1, 0, 300, 256, 77]
    w, t, dp, plan_pad, bias_pad, pk, plan, bias = _setup(lengths, H=2, d=d, seed=50 + d + epi)
    bp = bias_pad if epi == W.SIGMOID else None
    bk = bias if epi == W.SIGMOID else None
    o_pad, lse_pad = Bd.fwd(plan_pad, dp["q"], dp["k"], dp["v"], bp, epi)
    # outputs start as NaN: rows the packed path does not own must stay untouched
    T = pk["q"].shape[0]
    o = torch.full_like(pk["q"], float("nan"))
    o, lse = Bd.fwd(plan, pk["q"], pk["k"], pk["v"], bk, epi, out=o)
    assert Bd.get_status() == 0
    assert torch.equal(o, _pack(o_pad, lengths))
    if epi != W.SIGMOID:
        for b, n in enumerate(lengths):
            assert torch.equal(lse[b, :, :n], lse_pad[b, :, :n])
    g_pad = Bd.bwd(plan_pad, dp["q"], dp["k"], dp["v"], o_pad, dp["do"], bp, epi, lse=lse_pad)
    g = Bd.bwd(plan, pk["q"], pk["k"], pk["v"], o, pk["do"], bk, epi, lse=lse)
    assert Bd.get_status() == 0
    for name, x, y in zip(("dQ", "dK", "dV"), g, g_pad):
        assert x.shape[0] == T
        assert torch.equal(x, _pack(y, lengths)), f"packed {name} differs from padded"
    if d == 64:
        gf = Bd.bwd_fused(plan, pk["q"], pk["k"], pk["v"], o, pk["do"], bk, epi, lse=lse)
        assert Bd.get_status() == 0
        assert torch.equal(gf[1], g[1]) and torch.equal(gf[2], g[2])
        err = (gf[0].float() - g[0].float()).abs().max().item()
        assert err <= 1e-2 * g[0].float().abs().max().item() + 1e-4


def test_packed_matches_oracle_and_writes_only_its_rows():
    """Packed Q/K/V/O/dO as views into wider buffers (head stride 3d): the guard columns
    stay untouched; O, dQ, dK, dV match the oracle."""
    from padded_variable_length_b200 import binding as Bd
    lengths = [200, 129, 5]
    w, t, dp, _, _, pk, plan, bias = _setup(lengths, H=2, d=64, seed=7)
    T = pk["q"].shape[0]

    def wide(x):
        buf = torch.full((T, 2, 3, 64), 5.0, dtype=torch.bfloat16, device="cuda")
        buf[:, :, 1] = x
        return buf, buf[:, :, 1]

    bufs = {k: wide(v) for k, v in pk.items()}
    outs = {k: wide(torch.zeros_like(pk["q"])) for k in ("o", "dq", "dk", "dv")}
    Bd.fwd(plan, bufs["q"][1], bufs["k"][1], bufs["v"][1], bias, out=outs["o"][1])
    Bd.bwd(plan, bufs["q"][1], bufs["k"][1], bufs["v"][1], outs["o"][1], bufs["do"][1], bias,
           dq=outs["dq"][1], dk=outs["dk"][1], dv=outs["dv"][1])
    assert Bd.get_status() == 0
    for buf, _ in outs.values():
        assert torch.all(buf[:, :, 0] == 5.0) and torch.all(buf[:, :, 2] == 5.0)
    f64 = {k: Hn.to_f64(v) for k, v in t.items()}
    scale = 1.0 / math.sqrt(64)
    ob = A.bias_from_counts(w.counts)
    ref_o, _ = A.forward(f64["q"], f64["k"], f64["v"], ob, scale, A.SIGMOID, lengths=w.lengths)
    ref = A.backward(f64["q"], f64["k"], f64["v"], f64["do"], ob, scale, A.SIGMOID, lengths=w.lengths)
    pack_np = lambda x: np.concatenate([x[b, :n] for b, n in enumerate(lengths)], axis=0)
    Hn.check_close(Hn.to_f64(outs["o"][1]), pack_np(ref_o), "packed O")
    for name, r in zip(("dq", "dk", "dv"), ref):
        Hn.check_close(Hn.to_f64(outs[name][1]), pack_np(r), f"packed {name}")


def test_packed_plan_rejects_bad_offsets():
    from padded_variable_length_b200 import binding as Bd
    bad = torch.tensor([0, 100, 90], dtype=torch.int32, device="cuda")  # negative length
    with pytest.raises(Bd.SigattnError) as e:
        Bd.Plan.from_cu_seqlens(bad, 128)
    assert e.value.code == -1
    long = torch.tensor([0, 300], dtype=torch.int32, device="cuda")     # above max_seqlen
    with pytest.raises(Bd.SigattnError) as e:
        Bd.Plan.from_cu_seqlens(long, 256)
    assert e.value.code == -1
    assert Bd.get_status() == 0
