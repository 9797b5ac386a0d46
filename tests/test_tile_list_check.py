"""The library's structural tile-list check (sigattn_tile_list_check_host, the host twin of
sigattn_plan_validate), run on the CPU: correct lists from the oracle's tile builder pass,
and one planted mistake per property is reported with that property's check number."""
import numpy as np
import pytest

from oracle import tiles as OT
from padded_variable_length_b200 import binding as Bd


def _lists():
    rng = np.random.default_rng(7)
    out = [OT.tile_list_from_lengths([0, 1, 128, 129, 300, 385], 385)]
    m = np.zeros((2, 300, 520), dtype=np.uint8)
    m[0, :, :] = rng.random((300, 520)) < 0.02
    m[0, :128, 128:256] = 1                  # a FULL block
    m[1, 5:260, 10:400] = 1                  # FULL and PARTIAL blocks, runs of both kinds
    m[1, 200:, 450:] = rng.random((100, 70)) < 0.5
    out.append(OT.tile_list(m))
    return out


def _code(v):
    return v >> 40 if v >= 0 else 0


def _check(t, runs=True):
    rp, ru = OT.row_runs(t) if runs else (None, None)
    return Bd.tile_list_check_host(t, rp, ru)


@pytest.mark.parametrize("i", [0, 1])
def test_correct_lists_pass(i):
    t = _lists()[i]
    assert _check(t) == -1
    assert _check(t, runs=False) == -1


def _copy(t):
    return {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in t.items()}


def _first(t, kind_val):
    return int(np.nonzero(t["kind"] == kind_val)[0][0])


def test_planted_mistakes_are_reported_with_their_check():
    base = _lists()[1]
    assert base["kind"].tolist().count(2) >= 2 and base["kind"].tolist().count(1) >= 1
    rows = base["B"] * base["QT"]
    cases = []

    t = _copy(base); r = int(np.argmax(np.diff(t["row_ptr"]) > 0))
    t["row_ptr"][r + 1] = t["row_ptr"][r] - 1                     # offsets go backwards
    cases.append((t, 1))
    t = _copy(base); t["col_idx"][0] = base["KT"]                 # k-tile out of range
    cases.append((t, 2))
    t = _copy(base); r = int(np.argmax(np.diff(t["row_ptr"]) >= 2)); e = t["row_ptr"][r]
    t["col_idx"][e], t["col_idx"][e + 1] = t["col_idx"][e + 1], t["col_idx"][e]  # not ascending
    cases.append((t, 2))
    t = _copy(base); t["kind"][0] = 3                              # bad kind byte
    cases.append((t, 3))
    t = _copy(base); e = _first(t, 1); t["pidx"][e] = 0            # FULL entry with a bitmask
    cases.append((t, 4))
    t = _copy(base); p = np.nonzero(t["kind"] == 2)[0]
    t["pidx"][p[0]], t["pidx"][p[-1]] = t["pidx"][p[-1]], t["pidx"][p[0]]  # numbering out of order
    cases.append((t, 4))
    t = _copy(base); t["colT_ptr"][-1] += 1                        # CSC total disagrees
    cases.append((t, 5))
    t = _copy(base); c = int(np.argmax(np.diff(t["colT_ptr"]) >= 2)); e = t["colT_ptr"][c]
    t["rowT_idx"][e + 1] = t["rowT_idx"][e]                        # repeated q-tile
    cases.append((t, 6))
    t = _copy(base); c = int(np.argmax(np.diff(t["colT_ptr"]) >= 2)); e = t["colT_ptr"][c]
    t["csc_map"][e], t["csc_map"][e + 1] = t["csc_map"][e + 1], t["csc_map"][e]  # transposed map
    cases.append((t, 7))
    t = _copy(base); t["bits"][0, :] = 0                           # PARTIAL block with no pair
    cases.append((t, 8))
    t = _copy(base); t["bits"][-1, :] = 0xFFFFFFFF                 # PARTIAL block that is FULL
    cases.append((t, 8))
    for t, want in cases:
        got = _check(t)
        assert _code(got) == want, (want, got)

    rp, ru = OT.row_runs(base)
    j = int(np.argmax(ru[:, 1] >= 2))
    bad = ru.copy(); bad[j, 1] -= 1                                # run shorter than its range
    assert _code(Bd.tile_list_check_host(base, rp, bad)) == 9
    # two runs where one maximal run belongs: split run j after its first tile
    split = np.insert(ru.copy(), j + 1, [ru[j, 0] + 1, ru[j, 1] - 1, ru[j, 2], ru[j, 3] + 1], axis=0)
    split[j, 1] = 1
    rp2 = rp.copy(); rp2[np.searchsorted(rp, j, side="right"):] += 1
    assert _code(Bd.tile_list_check_host(base, rp2, split)) == 9
    assert rows == len(base["row_ptr"]) - 1


def test_bad_sizes_are_rejected_without_reading():
    t = _lists()[0]
    with pytest.raises(Bd.SigattnError):
        Bd.tile_list_check_host({**t, "B": 0})
