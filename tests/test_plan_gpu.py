"""GPU tile planner vs the brute-force oracle tile list: bit-exact (CSR, CSC, kinds,
PARTIAL bitmasks), plus validity of the longest-first work lists."""
import numpy as np
import pytest
import torch

from oracle import tiles as OT
from padded_variable_length_b200 import workloads as W

pytestmark = pytest.mark.gpu

KEYS = ("row_ptr", "col_idx", "kind", "pidx", "colT_ptr", "rowT_idx", "csc_map", "bits")


def _compare(plan, ref):
    from padded_variable_length_b200 import binding as Bd
    got = plan.export()
    for k in KEYS:
        assert got[k].shape == ref[k].shape, (k, got[k].shape, ref[k].shape)
        assert np.array_equal(got[k], ref[k]), f"{k} differs"
    z = plan.sizes()
    assert z["nonempty"] == len(ref["col_idx"])
    assert z["full"] == int((ref["kind"] == 1).sum())
    assert z["partial"] == ref["bits"].shape[0]
    rows_cnt = np.diff(ref["row_ptr"])
    cols_cnt = np.diff(ref["colT_ptr"])
    assert z["rows_nonempty"] == int((rows_cnt > 0).sum())
    assert z["cols_nonempty"] == int((cols_cnt > 0).sum())
    # the library's own structural check passes on the device arrays (bitmask transposes,
    # work lists and runs included) and, on the exported copy, with its host twin
    assert plan.validate() == -1
    assert Bd.tile_list_check_host({**got, "B": z["B"], "QT": z["QT"], "KT": z["KT"]},
                                   *plan.export_runs()) == -1
    rw, cw = plan.export_work()
    for work, cnt in ((rw, rows_cnt), (cw, cols_cnt)):
        assert sorted(work.tolist()) == list(range(len(cnt)))
        c = np.minimum(cnt[work], 4095)
        assert np.all(np.diff(c) <= 0), "work list not longest-first"
        for v in np.unique(c):  # ties keep ascending index (stable)
            idx = work[c == v]
            assert np.all(np.diff(idx) > 0)


LENGTH_CASES = [
    ([37, 64, 100, 128], 128),
    ([0, 1, 128, 129, 256], 300),
    ([640], 640),
    ([383, 129], 384),
    ([0, 0, 0], 5),
    ([1], 1),
]


@pytest.mark.parametrize("lengths,npad", LENGTH_CASES)
def test_plan_from_lengths(lengths, npad):
    from padded_variable_length_b200 import binding as Bd
    plan = Bd.Plan.from_lengths(torch.tensor(lengths, dtype=torch.int32, device="cuda"), npad)
    _compare(plan, OT.tile_list_from_lengths(lengths, npad))


def test_plan_from_lengths_random():
    from padded_variable_length_b200 import binding as Bd
    rng = np.random.default_rng(12)
    for _ in range(6):
        npad = int(rng.integers(1, 1500))
        lengths = rng.integers(0, npad + 1, int(rng.integers(1, 9))).astype(np.int32)
        plan = Bd.Plan.from_lengths(torch.from_numpy(lengths).cuda(), npad)
        _compare(plan, OT.tile_list_from_lengths(lengths, npad))


@pytest.mark.parametrize("cfg", [1, 2, 3])
def test_plan_workload_lengths(cfg):
    from padded_variable_length_b200 import binding as Bd
    w = W.config(cfg)
    plan = Bd.Plan.from_lengths(torch.from_numpy(w.lengths.astype(np.int32)).cuda(), w.Nq)
    _compare(plan, OT.tile_list_from_lengths(w.lengths, w.Nq))


@pytest.mark.parametrize("shape", [(2, 300, 300), (1, 128, 256), (3, 257, 129), (1, 1, 1)])
def test_plan_from_random_mask(shape):
    from padded_variable_length_b200 import binding as Bd
    rng = np.random.default_rng(sum(shape))
    m = W.random_mask(rng, *shape, density=0.3, empty_rows=2)
    plan = Bd.Plan.from_mask(torch.from_numpy(m).cuda())
    _compare(plan, OT.tile_list(m))


def test_plan_from_strided_mask():
    """A mask that is a view with a padded row stride (not 16-byte aligned rows)."""
    from padded_variable_length_b200 import binding as Bd
    rng = np.random.default_rng(77)
    big = W.random_mask(rng, 2, 260, 301, density=0.5, empty_rows=1)
    view = torch.from_numpy(big).cuda()[:, :, :290]
    plan = Bd.Plan.from_mask(view)
    _compare(plan, OT.tile_list(big[:, :, :290]))


def test_plan_packed_documents():
    from padded_variable_length_b200 import binding as Bd
    w = W.config(4)
    plan = Bd.Plan.from_mask(torch.from_numpy(w.mask).cuda())
    ref = OT.tile_list(w.mask)
    _compare(plan, ref)
    z = plan.sizes()
    pop = int(np.unpackbits(ref["bits"].view(np.uint8)).sum())
    assert pop + 16384 * z["full"] == w.pairs()


def test_plan_with_more_rows_than_one_sort_chunk():
    """More than 1024 q-tile rows and k-tile columns (the work lists are sorted in chunks
    of 1024): still bit-exact, longest-first and stable."""
    from padded_variable_length_b200 import binding as Bd
    rng = np.random.default_rng(77)
    npad = 7000
    lengths = rng.integers(0, npad + 1, 24).astype(np.int32)
    lengths[0] = npad
    plan = Bd.Plan.from_lengths(torch.from_numpy(lengths).cuda(), npad)
    assert plan.sizes()["B"] * plan.sizes()["QT"] > 1024
    _compare(plan, OT.tile_list_from_lengths(lengths, npad))


RUN_CASES = ["lengths", "mask", "packed", "tree", "longformer"]


@pytest.mark.parametrize("case", RUN_CASES)
def test_plan_runs_bit_exact(case):
    """The run-length rows of the plan equal the oracle's, walked entry by entry."""
    from padded_variable_length_b200 import binding as Bd
    rng = np.random.default_rng(9)
    if case == "lengths":
        lengths = np.array([0, 1, 640, 129, 1000], dtype=np.int32)
        plan = Bd.Plan.from_lengths(torch.from_numpy(lengths).cuda(), 1000)
        ref = OT.tile_list_from_lengths(lengths, 1000)
    else:
        if case == "mask":
            m = W.random_mask(rng, 3, 700, 900, density=0.3, empty_rows=4)
        elif case == "packed":
            m = W.config(4).mask[:2]
        else:
            m = W.mask_family(case).mask[:2]
        plan = Bd.Plan.from_mask(torch.from_numpy(m).cuda())
        ref = OT.tile_list(m)
    run_ptr, runs = plan.export_runs()
    ref_ptr, ref_runs = OT.row_runs(ref)
    assert np.array_equal(run_ptr, ref_ptr)
    assert np.array_equal(runs, ref_runs)


def _lengths_plan_closed_form(lengths, npad):
    """The tile list of a lengths plan written out directly (no oracle pass over the grid):
    sequence b with n valid rows lists the T x T tiles of its first T = ceil(n / 128)
    q-tiles and k-tiles; a tile is FULL iff both of its 128-row ranges lie inside n."""
    QT = (npad + 127) // 128
    n = np.clip(np.asarray(lengths, dtype=np.int64), 0, npad)
    T, F = (n + 127) // 128, n // 128
    row_cnt = np.zeros((len(n), QT), dtype=np.int64)
    for b in range(len(n)):
        row_cnt[b, :T[b]] = T[b]
    row_ptr = np.concatenate([[0], np.cumsum(row_cnt.ravel())]).astype(np.int32)
    col_idx, kind, csc_map = [], [], []
    for b in range(len(n)):
        t, f = int(T[b]), int(F[b])
        if t == 0:
            continue
        qt, kt = np.meshgrid(np.arange(t), np.arange(t), indexing="ij")
        col_idx.append(kt.ravel())
        kind.append(np.where((qt < f) & (kt < f), 1, 2).ravel())
        base = row_ptr[b * QT: b * QT + t].astype(np.int64)
        csc_map.append((base[None, :] + np.arange(t)[:, None]).ravel())  # column kt, row qt
    col_idx = np.concatenate(col_idx).astype(np.int32)
    kind = np.concatenate(kind).astype(np.uint8)
    pidx = np.full(len(kind), -1, dtype=np.int32)
    pidx[kind == 2] = np.arange(int((kind == 2).sum()), dtype=np.int32)
    return {"row_ptr": row_ptr, "col_idx": col_idx, "kind": kind, "pidx": pidx,
            "colT_ptr": row_ptr, "rowT_idx": col_idx,
            "csc_map": np.concatenate(csc_map).astype(np.int32)}


def test_plan_large_grid_sizes_after_counting():
    """A grid large enough (4.2 M blocks) that the planner reads the counts back before it
    sizes the tile arrays, instead of sizing them for the worst case: the lists equal the
    closed form, and sampled PARTIAL bitmasks equal the rows and columns inside n."""
    from padded_variable_length_b200 import binding as Bd
    rng = np.random.default_rng(31)
    npad = 16384
    lengths = rng.integers(0, npad + 1, 256).astype(np.int32)
    lengths[:3] = [npad, 0, 128 * 7]
    plan = Bd.Plan.from_lengths(torch.from_numpy(lengths).cuda(), npad)
    got = plan.export()
    ref = _lengths_plan_closed_form(lengths, npad)
    for k in ("row_ptr", "col_idx", "kind", "pidx", "colT_ptr", "rowT_idx", "csc_map"):
        assert np.array_equal(got[k], ref[k]), f"{k} differs"
    z = plan.sizes()
    assert z["nonempty"] == len(ref["col_idx"]) and z["partial"] == got["bits"].shape[0]
    # PARTIAL bitmasks, sampled: row q keeps column k iff both lie inside the sequence
    QT = (npad + 127) // 128
    ends = np.repeat(np.arange(len(lengths)), QT)  # batch entry of each q-tile row
    part = np.flatnonzero(ref["kind"] == 2)
    rows_of = np.searchsorted(ref["row_ptr"], np.arange(len(ref["kind"])), side="right") - 1
    for e in rng.choice(part, 64, replace=False):
        r = rows_of[e]
        b, qt, kt = ends[r], r % QT, ref["col_idx"][e]
        nv = int(min(max(lengths[b], 0), npad))
        q_ok = qt * 128 + np.arange(128) < nv
        k_ok = kt * 128 + np.arange(128) < nv
        dense = q_ok[:, None] & k_ok[None, :]
        words = np.packbits(dense.reshape(128, 4, 32)[:, :, ::-1], axis=-1, bitorder="big")
        want = words.view(">u4").reshape(128, 4).astype(np.uint32).ravel()
        assert np.array_equal(got["bits"][ref["pidx"][e]], want), f"bits of tile {e}"
    # every bitmask, its transpose, the runs and the work lists, by the library's own check
    assert plan.validate() == -1
