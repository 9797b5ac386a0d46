"""Thin ctypes binding of libsigattn.so (declared in include/sigattn.h).

Argument marshalling only: every step of the attention path runs in the library's
CUDA kernels.  PyTorch provides device memory and streams.  There is no fallback: if
the library is missing, importing this module raises.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsigattn.so")

SIGMOID, SOFTMAX, SOFTMAX1 = 0, 1, 2
OK = 0
ERR_PLAN = -9  # SIGATTN_ERR_PLAN: a tile list failed a structural check
ERR = {-1: "INVALID", -2: "UNSUPPORTED", -3: "ALIGNMENT", -4: "SHAPE", -5: "CUDA",
       -6: "TIMEOUT", -7: "NO_DEVICE", -8: "NOMEM", -9: "PLAN"}


class SigattnError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        detail = _lib.sigattn_error_string(code).decode()
        if code in (-5, -8):
            detail += f" [{_lib.sigattn_last_cuda_error().decode()}]"
        super().__init__(f"{what}: sigattn error {code} ({ERR.get(code, '?')}): {detail}")


if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is not built; run `python -m padded_variable_length_b200.build`")

_lib = ctypes.CDLL(LIB_PATH)

_p = ctypes.c_void_p
_i32 = ctypes.c_int32
_i64 = ctypes.c_int64
_u64 = ctypes.c_uint64
_I64x3 = ctypes.c_int64 * 3


class PlanSizes(ctypes.Structure):
    _fields_ = [("B", _i32), ("Nq", _i32), ("Nk", _i32), ("QT", _i32), ("KT", _i32),
                ("nonempty", _i64), ("full", _i64), ("partial", _i64), ("grid_total", _i64),
                ("rows_nonempty", _i32), ("cols_nonempty", _i32)]


def _sig(name, res, *args):
    f = getattr(_lib, name)
    f.restype = res
    f.argtypes = list(args)
    return f


_sig("sigattn_plan_from_lengths", ctypes.c_int, _p, ctypes.c_int, ctypes.c_int, _p, ctypes.POINTER(_p))
_sig("sigattn_plan_from_mask", ctypes.c_int, _p, ctypes.c_int, ctypes.c_int, ctypes.c_int, _i64, _i64,
     _p, ctypes.POINTER(_p))
_sig("sigattn_plan_from_cu_seqlens", ctypes.c_int, _p, ctypes.c_int, ctypes.c_int, _p, ctypes.POINTER(_p))
_sig("sigattn_plan_get_sizes", ctypes.c_int, _p, ctypes.POINTER(PlanSizes))
_sig("sigattn_plan_export", ctypes.c_int, _p, _p, _p, _p, _p, _p, _p, _p, _p)
_sig("sigattn_plan_export_work", ctypes.c_int, _p, _p, _p)
_sig("sigattn_plan_export_runs", ctypes.c_int, _p, _p, _p, ctypes.POINTER(_i64))
_sig("sigattn_plan_destroy", None, _p)
_sig("sigattn_plan_validate", ctypes.c_int, _p, _p, ctypes.POINTER(_i64))
_sig("sigattn_tile_list_check_host", ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, _i64, _i64,
     _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _i64, ctypes.POINTER(_i64))
_sig("sigattn_bias_from_counts", ctypes.c_int, _p, _i64, _p, _p)
_sig("sigattn_fwd", ctypes.c_int, _p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float,
     _p, _I64x3, _p, _I64x3, _p, _I64x3, _p, _i64, _p, _I64x3, _p, _p)
_sig("sigattn_bwd", ctypes.c_int, _p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float,
     _p, _I64x3, _p, _I64x3, _p, _I64x3, _p, _I64x3, _p, _I64x3, _p, _i64, _p, _p,
     _p, _I64x3, _p, _I64x3, _p, _I64x3, _p)
_sig("sigattn_bwd_ex", ctypes.c_int, _p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float,
     _p, _I64x3, _p, _I64x3, _p, _I64x3, _p, _I64x3, _p, _I64x3, _p, _i64, _p, _p,
     _p, _I64x3, _p, _I64x3, _p, _I64x3, ctypes.c_int, _p)
_sig("sigattn_bwd_noalloc", ctypes.c_int, _p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float,
     _p, _I64x3, _p, _I64x3, _p, _I64x3, _p, _I64x3, _p, _I64x3, _p, _i64, _p,
     _p, _I64x3, _p, _I64x3, _p, _I64x3, _p)
_sig("sigattn_bwd_fused_workspace_size", ctypes.c_int, _p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
     ctypes.POINTER(ctypes.c_size_t))
_sig("sigattn_bwd_fused", ctypes.c_int, _p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float,
     _p, _I64x3, _p, _I64x3, _p, _I64x3, _p, _I64x3, _p, _I64x3, _p, _i64, _p, _p, ctypes.c_size_t,
     _p, _I64x3, _p, _I64x3, _p, _I64x3, _p)
_sig("sigattn_get_status", ctypes.c_int, _p)
_sig("sigattn_set_wait_limit_ns", ctypes.c_int, _u64)
_sig("sigattn_selftest_wait_timeout", ctypes.c_int, _u64, _p)
_sig("sigattn_error_string", ctypes.c_char_p, ctypes.c_int)
_sig("sigattn_version", ctypes.c_int)
_sig("sigattn_last_cuda_error", ctypes.c_char_p)

lib = _lib


def _check(rc: int, what: str):
    if rc != OK:
        raise SigattnError(rc, what)


# torch's current stream of the current device as a raw handle, without building a Stream
# object on every call (the public route below is the fallback)
_raw_current_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)
_current_device = getattr(torch._C, "_cuda_getDevice", None)


def _stream(stream) -> Optional[int]:
    if stream is None:
        if _raw_current_stream is not None and _current_device is not None:
            return _raw_current_stream(_current_device())
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _strides(t: torch.Tensor) -> ctypes.Array:
    """(batch, token, head) element strides of a padded [B, N, H, d] tensor, or of a packed
    [T, H, d] tensor (batch stride 0: ignored by the library for packed plans)."""
    if t.dtype != torch.bfloat16 or t.stride(-1) != 1 or t.dim() not in (3, 4):
        raise ValueError("expected a bf16 [B, N, H, d] or packed [T, H, d] tensor, d contiguous")
    if t.dim() == 3:
        return _I64x3(0, t.stride(0), t.stride(1))
    return _I64x3(t.stride(0), t.stride(1), t.stride(2))


def _keep_until_run(t: torch.Tensor, stream):
    """The plan builds return before the device has read their input: when the build runs
    on another torch stream than the current one, the caching allocator is told that the
    input is in use there (on the current stream, stream order already covers it)."""
    if isinstance(stream, torch.cuda.Stream):
        t.record_stream(stream)


class Plan:
    """A tile plan (owns device buffers; destroyed with the object).  Lengths and mask
    plans are built asynchronously on the stream: the attention calls wait for the build,
    and sizes() / the exports wait for it on the host."""

    def __init__(self, handle: int, dims=None):
        self._h = ctypes.c_void_p(handle)
        self._dims = dims  # (B, Nq, Nk, packed) when known on the host at construction

    @classmethod
    def from_lengths(cls, lengths: torch.Tensor, npad: int, stream=None) -> "Plan":
        if lengths.dtype != torch.int32 or not lengths.is_cuda or not lengths.is_contiguous():
            raise ValueError("lengths must be a contiguous int32 CUDA tensor")
        h = ctypes.c_void_p()
        _keep_until_run(lengths, stream)
        _check(_lib.sigattn_plan_from_lengths(lengths.data_ptr(), lengths.numel(), int(npad),
                                              _stream(stream), ctypes.byref(h)), "plan_from_lengths")
        return cls(h.value, (lengths.numel(), int(npad), int(npad), False))

    @classmethod
    def from_cu_seqlens(cls, cu: torch.Tensor, max_seqlen: int, stream=None) -> "Plan":
        """Plan of a packed batch: sequence b is rows cu[b] .. cu[b+1] of [T, H, d] tensors."""
        if cu.dtype != torch.int32 or not cu.is_cuda or not cu.is_contiguous() or cu.dim() != 1:
            raise ValueError("cu must be a contiguous int32 CUDA tensor [B + 1]")
        h = ctypes.c_void_p()
        _check(_lib.sigattn_plan_from_cu_seqlens(cu.data_ptr(), cu.numel() - 1, int(max_seqlen),
                                                 _stream(stream), ctypes.byref(h)), "plan_from_cu_seqlens")
        return cls(h.value, (cu.numel() - 1, int(max_seqlen), int(max_seqlen), True))

    @classmethod
    def from_mask(cls, mask: torch.Tensor, stream=None) -> "Plan":
        if mask.dtype != torch.uint8 or not mask.is_cuda or mask.dim() != 3 or mask.stride(2) != 1:
            raise ValueError("mask must be a uint8 CUDA tensor [B, Nq, Nk] with Nk contiguous")
        h = ctypes.c_void_p()
        _keep_until_run(mask, stream)
        B, Nq, Nk = mask.shape
        _check(_lib.sigattn_plan_from_mask(mask.data_ptr(), B, Nq, Nk, mask.stride(0), mask.stride(1),
                                           _stream(stream), ctypes.byref(h)), "plan_from_mask")
        return cls(h.value, (B, Nq, Nk, False))

    @property
    def handle(self):
        return self._h

    def dims(self):
        """(B, Nq, Nk, packed): the batch and row extents the plan addresses.  Known on the
        host from the construction arguments, so this never waits for the build (a Plan
        wrapped around a raw handle asks sigattn_plan_get_sizes, which may).  For a packed
        plan Nq = Nk = the longest sequence."""
        if self._dims is None:
            z = self.sizes()
            self._dims = (z["B"], z["Nq"], z["Nk"], False)
        return self._dims

    def sizes(self) -> dict:
        s = PlanSizes()
        _check(_lib.sigattn_plan_get_sizes(self._h, ctypes.byref(s)), "plan_get_sizes")
        return {f: getattr(s, f) for f, _ in PlanSizes._fields_}

    def export(self) -> dict:
        z = self.sizes()
        rows, cols, nz, npart = z["B"] * z["QT"], z["B"] * z["KT"], z["nonempty"], z["partial"]
        out = {
            "row_ptr": np.zeros(rows + 1, np.int32), "col_idx": np.zeros(nz, np.int32),
            "kind": np.zeros(nz, np.uint8), "pidx": np.zeros(nz, np.int32),
            "colT_ptr": np.zeros(cols + 1, np.int32), "rowT_idx": np.zeros(nz, np.int32),
            "csc_map": np.zeros(nz, np.int32), "bits": np.zeros((npart, 512), np.uint32),
        }
        ptr = lambda a: a.ctypes.data if a.size else None
        _check(_lib.sigattn_plan_export(self._h, *(ptr(out[k]) for k in
                                                   ("row_ptr", "col_idx", "kind", "pidx", "colT_ptr",
                                                    "rowT_idx", "csc_map", "bits"))), "plan_export")
        return out

    def export_work(self):
        z = self.sizes()
        rw = np.zeros(z["B"] * z["QT"], np.int32)
        cw = np.zeros(z["B"] * z["KT"], np.int32)
        _check(_lib.sigattn_plan_export_work(self._h, rw.ctypes.data, cw.ctypes.data), "plan_export_work")
        return rw, cw

    def export_runs(self):
        """(run_ptr int32 [B*QT + 1], runs int32 [nruns, 4]): each q-tile row's maximal
        ranges of consecutive k-tiles of one kind, {first k-tile, count, kind, first entry}."""
        z = self.sizes()
        n = _i64()
        _check(_lib.sigattn_plan_export_runs(self._h, None, None, ctypes.byref(n)), "plan_export_runs")
        run_ptr = np.zeros(z["B"] * z["QT"] + 1, np.int32)
        runs = np.zeros((n.value, 4), np.int32)
        _check(_lib.sigattn_plan_export_runs(self._h, run_ptr.ctypes.data,
                                             runs.ctypes.data if runs.size else None,
                                             ctypes.byref(n)), "plan_export_runs")
        return run_ptr, runs

    def validate(self, stream=None) -> int:
        """Debug check of the plan's device arrays (sigattn_plan_validate): -1 when every
        structural property holds, else (check number << 40) | index of the first failure."""
        where = _i64()
        rc = _lib.sigattn_plan_validate(self._h, _stream(stream), ctypes.byref(where))
        if rc not in (OK, ERR_PLAN):
            _check(rc, "plan_validate")
        return where.value

    def close(self):
        if self._h is not None and self._h.value:
            _lib.sigattn_plan_destroy(self._h)
        self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def tile_list_check_host(t: dict, run_ptr=None, runs=None) -> int:
    """sigattn_tile_list_check_host on host arrays in the export layout (a dict with B, QT,
    KT, row_ptr, col_idx, kind, pidx, colT_ptr, rowT_idx, csc_map, bits): -1 when the list
    passes, else (check number << 40) | index of the first failure.  Needs no GPU."""
    a = {k: np.ascontiguousarray(t[k], dtype=dt) for k, dt in (
        ("row_ptr", np.int32), ("col_idx", np.int32), ("kind", np.uint8), ("pidx", np.int32),
        ("colT_ptr", np.int32), ("rowT_idx", np.int32), ("csc_map", np.int32), ("bits", np.uint32))}
    ptr = lambda x: x.ctypes.data if x is not None and x.size else None
    rp = None if run_ptr is None else np.ascontiguousarray(run_ptr, dtype=np.int32)
    ru = None if runs is None else np.ascontiguousarray(runs, dtype=np.int32).reshape(-1, 4)
    where = _i64()
    rc = _lib.sigattn_tile_list_check_host(
        int(t["B"]), int(t["QT"]), int(t["KT"]), a["col_idx"].size, a["bits"].size // 512,
        *(ptr(a[k]) for k in ("row_ptr", "col_idx", "kind", "pidx", "colT_ptr", "rowT_idx",
                              "csc_map", "bits")),
        ptr(rp), ptr(ru), 0 if ru is None else ru.shape[0], ctypes.byref(where))
    if rc not in (OK, ERR_PLAN):
        _check(rc, "tile_list_check_host")
    return where.value


def bias_from_counts(counts: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """b = -log(n) per query row from the int32 counts n (0 where n = 0)."""
    if counts.dtype != torch.int32 or not counts.is_cuda or not counts.is_contiguous():
        raise ValueError("counts must be a contiguous int32 CUDA tensor")
    if out is None:
        out = torch.empty(counts.shape, dtype=torch.float32, device=counts.device)
    _check(_lib.sigattn_bias_from_counts(counts.data_ptr(), counts.numel(), out.data_ptr(),
                                         _stream(stream)), "bias_from_counts")
    return out


def _bias_args(bias):
    if bias is None:
        return None, 0
    if bias.dtype != torch.float32 or bias.stride(-1) != 1 or bias.dim() not in (1, 2):
        raise ValueError("bias must be fp32 [B, Nq] (or [T] for a packed plan) with unit row stride")
    return bias.data_ptr(), (bias.stride(0) if bias.dim() == 2 else 0)


def _shape(plan: "Plan", q: torch.Tensor):
    """(B, Nq, H, d): from a padded Q, or from the plan for a packed [T, H, d] Q."""
    if q.dim() == 4:
        return tuple(q.shape)
    B, Nq, _, _ = plan.dims()
    return B, Nq, q.shape[1], q.shape[2]


def _check_extents(plan: "Plan", q_side, k_side, bias=None, lse=None, workspace=None):
    """The library sees pointers and strides only: it addresses B x Nq (Q side) and B x Nk
    (K side) rows of every tensor, B x Nq bias values and B x H x Nq fp32 row statistics,
    with the plan's B and N.  Raise ValueError, before anything is launched, when a tensor
    is smaller than that or disagrees with Q in H or d (a larger tensor is fine: rows past
    the plan's extents are not touched).  Packed [T, H, d] tensors must all have Q's shape."""
    B, Nq, Nk, packed = plan.dims()
    q = q_side[0]
    if packed:
        if q.dim() != 3:
            raise ValueError("a packed plan takes [T, H, d] tensors")
        for t in list(q_side) + list(k_side):
            if t.dim() != 3 or tuple(t.shape) != tuple(q.shape):
                raise ValueError(f"packed tensors must all be {tuple(q.shape)}, got {tuple(t.shape)}")
        H = q.shape[1]
        if bias is not None and (bias.dim() != 1 or bias.shape[0] < q.shape[0]):
            raise ValueError(f"bias of a packed plan must be [T] with T >= {q.shape[0]}")
    else:
        if q.dim() != 4:
            raise ValueError("a padded plan takes [B, N, H, d] tensors")
        H, d = q.shape[2], q.shape[3]
        for side, n in ((q_side, Nq), (k_side, Nk)):
            for t in side:
                if (t.dim() != 4 or t.shape[0] < B or t.shape[1] < n or t.shape[2] != H
                        or t.shape[3] != d):
                    raise ValueError(f"tensor {tuple(t.shape)} does not cover the plan's "
                                     f"[{B}, {n}, {H}, {d}]")
        if bias is not None and (bias.dim() != 2 or bias.shape[0] < B or bias.shape[1] < Nq):
            raise ValueError(f"bias {tuple(bias.shape)} does not cover the plan's [{B}, {Nq}]")
    rows = B * H * Nq
    if lse is not None and (lse.dtype != torch.float32 or not lse.is_contiguous()
                            or lse.numel() < rows):
        raise ValueError(f"lse must be a contiguous fp32 [B, H, Nq] buffer of >= {rows} values")
    if workspace is not None and workspace.numel() * workspace.element_size() < 4 * rows:
        raise ValueError(f"workspace must hold >= {rows} fp32 values")


def fwd(plan: Plan, q, k, v, bias=None, epilogue: int = SIGMOID, scale: Optional[float] = None,
        out=None, lse=None, stream=None):
    """O (and the row log-normaliser for the softmax modes) of the planned attention."""
    B, Nq, H, d = _shape(plan, q)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if epilogue != SIGMOID and lse is None:
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    _check_extents(plan, (q, out), (k, v), bias, lse)
    bp, bs = _bias_args(bias)
    _check(_lib.sigattn_fwd(plan.handle, epilogue, H, d, float(scale),
                            q.data_ptr(), _strides(q), k.data_ptr(), _strides(k),
                            v.data_ptr(), _strides(v), bp, bs, out.data_ptr(), _strides(out),
                            lse.data_ptr() if lse is not None else None, _stream(stream)), "fwd")
    return out, lse


BWD_PREP, BWD_DKDV, BWD_DQ, BWD_ALL = 1, 2, 4, 7


def bwd(plan: Plan, q, k, v, o, do, bias=None, epilogue: int = SIGMOID, lse=None,
        scale: Optional[float] = None, workspace=None, dq=None, dk=None, dv=None, stream=None,
        parts: int = BWD_ALL):
    """dQ, dK, dV of L = sum(dO * O) (``parts`` selects PREP / DKDV / DQ)."""
    B, Nq, H, d = _shape(plan, q)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if epilogue != SIGMOID and workspace is None:
        workspace = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    _check_extents(plan, [x for x in (q, o, do, dq) if x is not None], (k, v, dk, dv), bias, lse,
                   workspace)
    bp, bs = _bias_args(bias)
    o_ptr = o.data_ptr() if o is not None else None
    o_str = _strides(o) if o is not None else _I64x3(0, 0, 0)
    _check(_lib.sigattn_bwd_ex(plan.handle, epilogue, H, d, float(scale),
                               q.data_ptr(), _strides(q), k.data_ptr(), _strides(k),
                               v.data_ptr(), _strides(v), o_ptr, o_str, do.data_ptr(), _strides(do),
                               bp, bs, lse.data_ptr() if lse is not None else None,
                               workspace.data_ptr() if workspace is not None else None,
                               dq.data_ptr(), _strides(dq), dk.data_ptr(), _strides(dk),
                               dv.data_ptr(), _strides(dv), int(parts), _stream(stream)), "bwd")
    return dq, dk, dv


def bwd_fused_workspace_bytes(plan: Plan, H: int, d: int, epilogue: int = SIGMOID) -> int:
    n = ctypes.c_size_t()
    _check(_lib.sigattn_bwd_fused_workspace_size(plan.handle, epilogue, H, d, ctypes.byref(n)),
           "bwd_fused_workspace_size")
    return n.value


def bwd_fused(plan: Plan, q, k, v, o, do, bias=None, epilogue: int = SIGMOID, lse=None,
              scale: Optional[float] = None, workspace=None, dq=None, dk=None, dv=None, stream=None):
    """dQ, dK, dV of L = sum(dO * O) in one walk over the k-tile columns (d = 64): dQ is
    accumulated in fp32 in ``workspace`` (a 16-byte aligned CUDA buffer of at least
    bwd_fused_workspace_bytes bytes; allocated here if None) and converted at the end."""
    B, Nq, H, d = _shape(plan, q)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    need = bwd_fused_workspace_bytes(plan, H, d, epilogue)
    if workspace is None:
        workspace = torch.empty((need + 3) // 4, dtype=torch.float32, device=q.device)
    nbytes = workspace.numel() * workspace.element_size()
    _check_extents(plan, [x for x in (q, o, do, dq) if x is not None], (k, v, dk, dv), bias, lse)
    bp, bs = _bias_args(bias)
    o_ptr = o.data_ptr() if o is not None else None
    o_str = _strides(o) if o is not None else _I64x3(0, 0, 0)
    _check(_lib.sigattn_bwd_fused(plan.handle, epilogue, H, d, float(scale),
                                  q.data_ptr(), _strides(q), k.data_ptr(), _strides(k),
                                  v.data_ptr(), _strides(v), o_ptr, o_str, do.data_ptr(), _strides(do),
                                  bp, bs, lse.data_ptr() if lse is not None else None,
                                  workspace.data_ptr(), nbytes,
                                  dq.data_ptr(), _strides(dq), dk.data_ptr(), _strides(dk),
                                  dv.data_ptr(), _strides(dv), _stream(stream)), "bwd_fused")
    return dq, dk, dv


def get_status(stream=None) -> int:
    """Synchronises the stream; returns and clears the device status word (0 or TIMEOUT)."""
    return _lib.sigattn_get_status(_stream(stream))


def set_wait_limit_ns(ns: int):
    _check(_lib.sigattn_set_wait_limit_ns(int(ns)), "set_wait_limit_ns")


def selftest_wait_timeout(ns: int, stream=None):
    _check(_lib.sigattn_selftest_wait_timeout(int(ns), _stream(stream)), "selftest_wait_timeout")
