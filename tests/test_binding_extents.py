"""Host-side extent checks of the Python binding (no GPU: shape-only tensors on the meta
device and a Plan that carries its dimensions but no device handle).

The C ABI sees pointers and strides only and addresses the plan's B x N rows of each
tensor, so the binding rejects a tensor that is smaller than that before any launch."""
import pytest
import torch

from padded_variable_length_b200 import binding as Bd


def _t(*shape, dtype=torch.bfloat16):
    return torch.empty(shape, dtype=dtype, device="meta")


def _plan(B, Nq, Nk, packed=False):
    return Bd.Plan(0, dims=(B, Nq, Nk, packed))  # null handle: never destroyed


def test_padded_extents_accept_exact_and_larger_tensors():
    p = _plan(2, 200, 300)
    q, k = _t(2, 200, 4, 64), _t(2, 300, 4, 64)
    Bd._check_extents(p, (q, q), (k, k), _t(2, 200, dtype=torch.float32),
                      _t(2, 4, 200, dtype=torch.float32), _t(2 * 4 * 200, dtype=torch.float32))
    big_q, big_k = _t(3, 256, 4, 64), _t(2, 384, 4, 64)  # rows past the plan are untouched
    Bd._check_extents(p, (big_q,), (big_k,), _t(3, 256, dtype=torch.float32))


@pytest.mark.parametrize("which,shape", [
    ("q", (1, 200, 4, 64)),   # fewer batch entries than the plan
    ("q", (2, 199, 4, 64)),   # fewer query rows
    ("k", (2, 200, 4, 64)),   # K side sized for Nq, plan has Nk = 300
    ("k", (2, 300, 3, 64)),   # head count differs from Q
    ("k", (2, 300, 4, 128)),  # head dim differs from Q
])
def test_padded_extents_reject_short_or_mismatched_tensors(which, shape):
    p = _plan(2, 200, 300)
    q, k = _t(2, 200, 4, 64), _t(2, 300, 4, 64)
    if which == "q":
        q_side, k_side = (q, _t(*shape)), (k,)
    else:
        q_side, k_side = (q,), (k, _t(*shape))
    with pytest.raises(ValueError):
        Bd._check_extents(p, q_side, k_side)


def test_padded_extents_reject_short_bias_lse_and_workspace():
    p = _plan(2, 200, 200)
    q = _t(2, 200, 4, 64)
    f32 = torch.float32
    with pytest.raises(ValueError):
        Bd._check_extents(p, (q,), (q,), bias=_t(2, 128, dtype=f32))
    with pytest.raises(ValueError):
        Bd._check_extents(p, (q,), (q,), bias=_t(200, dtype=f32))  # packed-style bias
    with pytest.raises(ValueError):
        Bd._check_extents(p, (q,), (q,), lse=_t(2, 4, 199, dtype=f32))
    with pytest.raises(ValueError):
        Bd._check_extents(p, (q,), (q,), lse=_t(2, 4, 200, dtype=torch.bfloat16))
    with pytest.raises(ValueError):
        Bd._check_extents(p, (q,), (q,), workspace=_t(2 * 4 * 200 - 1, dtype=f32))


def test_packed_extents():
    p = _plan(3, 300, 300, packed=True)
    x = _t(629, 2, 64)
    Bd._check_extents(p, (x, x), (x, x), _t(629, dtype=torch.float32),
                      _t(3, 2, 300, dtype=torch.float32))
    for bad in (_t(628, 2, 64), _t(629, 1, 64), _t(1, 629, 2, 64)):
        with pytest.raises(ValueError):
            Bd._check_extents(p, (x,), (x, bad))
    with pytest.raises(ValueError):
        Bd._check_extents(p, (x,), (x,), bias=_t(628, dtype=torch.float32))
    with pytest.raises(ValueError):
        Bd._check_extents(_plan(3, 300, 300), (x,), (x,))  # packed tensors, padded plan


def test_plan_dims_come_from_construction_arguments():
    assert _plan(4, 128, 96).dims() == (4, 128, 96, False)
    assert Bd._shape(_plan(3, 300, 300, packed=True), _t(629, 2, 64)) == (3, 300, 2, 64)
