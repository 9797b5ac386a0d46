"""Plan builds that return before the device has run them.  A bounded spin keeps the build's
stream busy: the build call must come back while the stream is still busy, the forward
launched right after on ANOTHER stream must wait for the build (it matches the float64
oracle), and sizes() waits for the build on the host (its counts equal the oracle's)."""
import math

import numpy as np
import pytest
import torch

from oracle import attention as A
from oracle import tiles as OT
from padded_variable_length_b200 import workloads as W
from tests import harness as Hn

pytestmark = pytest.mark.gpu

SPIN_CYCLES = 200_000_000  # about 0.1 s at 2 GHz: ends by itself


def _workload(kind):
    if kind == "lengths":
        return W.padded_workload("async_lengths", [300, 0, 129, 640], H=2, d=64, seed=71,
                                 backward=False)
    rng = np.random.default_rng(72)
    m = W.random_mask(rng, 2, 400, 520, density=0.3, empty_rows=3)
    counts = np.maximum(m.sum(axis=2), 1)
    return W.masked_workload("async_mask", m, counts, H=2, d=64, backward=False, seed=73)


@pytest.mark.parametrize("kind", ["lengths", "mask"])
def test_plan_build_does_not_wait_and_is_waited_for(kind):
    from padded_variable_length_b200 import binding as Bd
    w = _workload(kind)
    t = W.tensors(w, with_grad=False)
    d = {k: v.cuda() for k, v in t.items()}
    counts = torch.from_numpy(np.ascontiguousarray(w.counts, dtype=np.int32)).cuda()
    bias = Bd.bias_from_counts(counts)
    src = (torch.from_numpy(w.lengths.astype(np.int32)) if kind == "lengths"
           else torch.from_numpy(w.mask)).cuda()
    # one build beforehand: the first use of the planner's kernels loads their module, which
    # the CUDA runtime may do with a device-wide wait
    (Bd.Plan.from_lengths(src, w.Nq) if kind == "lengths" else Bd.Plan.from_mask(src)).close()
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        torch.cuda._sleep(SPIN_CYCLES)
        plan = (Bd.Plan.from_lengths(src, w.Nq, stream=side) if kind == "lengths"
                else Bd.Plan.from_mask(src, stream=side))
        still_busy = not side.query()
    assert still_busy, "the build waited for its stream"
    # the forward on the default stream, queued while the build has not run yet
    o, _ = Bd.fwd(plan, d["q"], d["k"], d["v"], bias, W.SIGMOID)
    torch.cuda.synchronize()
    assert Bd.get_status() == 0
    ref, _ = A.forward(Hn.to_f64(t["q"]), Hn.to_f64(t["k"]), Hn.to_f64(t["v"]),
                       Hn.oracle_bias(w, W.SIGMOID), 1.0 / math.sqrt(w.d), W.SIGMOID,
                       lengths=w.lengths, mask=w.mask)
    got = Hn.to_f64(o)
    Hn.check_close(got, ref, "O", Hn.valid_rows_q(w))
    Hn.check_pad_zero(got, w, "O")
    tl = OT.tile_list_from_lengths(w.lengths, w.Nq) if kind == "lengths" else OT.tile_list(w.mask)
    z = plan.sizes()
    assert z["nonempty"] == len(tl["col_idx"])
    assert z["partial"] == int((tl["kind"] == 2).sum())
    assert z["rows_nonempty"] == int((np.diff(tl["row_ptr"]) > 0).sum())
    assert z["cols_nonempty"] == int((np.diff(tl["colT_ptr"]) > 0).sum())
    plan.close()


def test_destroy_before_the_build_has_run():
    """A plan destroyed while its build still waits behind a spin on a non-blocking stream:
    its memory goes back to the pool only after the build, so a plan built next (which may
    take the same memory) is not overwritten by the late build.  The first plan comes from
    a different mask, so that a late write would change the second plan's lists."""
    from padded_variable_length_b200 import binding as Bd
    rng = np.random.default_rng(74)
    m_old = W.random_mask(rng, 2, 400, 520, density=0.6, empty_rows=0)
    w = _workload("mask")
    old_src = torch.from_numpy(m_old).cuda()
    new_src = torch.from_numpy(w.mask).cuda()
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        torch.cuda._sleep(SPIN_CYCLES)
        old = Bd.Plan.from_mask(old_src, stream=side)
    old.close()
    plan = Bd.Plan.from_mask(new_src)
    torch.cuda.synchronize()
    got = plan.export()
    ref = OT.tile_list(w.mask)
    for k in ("row_ptr", "col_idx", "kind", "pidx", "colT_ptr", "rowT_idx", "csc_map", "bits"):
        assert np.array_equal(got[k], ref[k]), f"{k} differs"
    plan.close()


def test_graph_captured_with_a_plan_not_yet_waited_for():
    """A forward captured into a CUDA graph right after an asynchronous build (no sizes()
    call, so the attention call still has to wait for the build's event): capture succeeds
    and every replay equals the eager forward."""
    from padded_variable_length_b200 import binding as Bd
    w = _workload("lengths")
    t = W.tensors(w, with_grad=False)
    d = {k: v.cuda() for k, v in t.items()}
    counts = torch.from_numpy(np.ascontiguousarray(w.counts, dtype=np.int32)).cuda()
    bias = Bd.bias_from_counts(counts)
    src = torch.from_numpy(w.lengths.astype(np.int32)).cuda()
    torch.cuda.synchronize()
    plan = Bd.Plan.from_lengths(src, w.Nq)
    o = torch.empty_like(d["q"])
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        Bd.fwd(plan, d["q"], d["k"], d["v"], bias, W.SIGMOID, out=o)
    torch.cuda.synchronize()
    eager, _ = Bd.fwd(plan, d["q"], d["k"], d["v"], bias, W.SIGMOID)
    for _ in range(2):
        o.fill_(7.0)
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(o, eager)
    assert Bd.get_status() == 0
    del g
    plan.close()
