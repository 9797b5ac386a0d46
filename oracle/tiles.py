"""Brute-force tile list of an element mask (test infrastructure).

"Binary Block Masking for FlashAttention", section "Comment ça marche ?": the
element mask is turned into a binary matrix of blocks, a block being kept iff it
holds at least one non-zero entry, and only kept blocks are computed.  The
sigmoid-attention page (section 2C, native padding support) applies the same
idea to padding: blocks that are padding on the query side or on the key side
are skipped.

Conventions fixed here (the pages leave them open):
  * T = 128 on both axes; block (qt, kt) of batch b covers query rows
    [qt T, qt T + T) and key columns [kt T, kt T + T); positions past Nq / Nk
    count as masked.
  * kind 0 = empty (not listed), 1 = FULL (every one of the T x T entries is 1),
    2 = PARTIAL.
  * CSR by query-tile row r = b * QT + qt, entries in ascending kt.
  * CSC by key-tile column c = b * KT + kt, entries in ascending qt; csc_map
    gives the CSR index of each CSC entry.
  * PARTIAL blocks own a 128 x 128 bitmask of 512 uint32 words, numbered in CSR
    order of the PARTIAL entries: bit (k mod 32) of word (q * 4 + k div 32) is
    mask(qt T + q, kt T + k).  pidx[e] is that number, -1 for FULL entries.
"""
from __future__ import annotations

import numpy as np

T = 128


def _mask_blocks(mask: np.ndarray):
    mask = np.asarray(mask) != 0
    B, Nq, Nk = mask.shape

    def block(b, qt, kt):
        blk = np.zeros((T, T), dtype=bool)
        sub = mask[b, qt * T:(qt + 1) * T, kt * T:(kt + 1) * T]
        blk[:sub.shape[0], :sub.shape[1]] = sub
        return blk
    return B, Nq, Nk, block


def _length_blocks(lengths, npad: int):
    """Blocks of the padded-batch mask (query i sees key j iff i, j < n_b),
    produced one at a time so that no Npad x Npad array is held."""
    lengths = np.asarray(lengths)
    B = lengths.shape[0]

    def block(b, qt, kt):
        n = int(lengths[b])
        i = np.arange(qt * T, qt * T + T)
        j = np.arange(kt * T, kt * T + T)
        iv = (i < n) & (i < npad)
        jv = (j < n) & (j < npad)
        return iv[:, None] & jv[None, :]
    return B, npad, npad, block


def block_kinds_from(B, Nq, Nk, block) -> np.ndarray:
    QT, KT = -(-Nq // T), -(-Nk // T)
    kinds = np.zeros((B, QT, KT), dtype=np.uint8)
    for b in range(B):
        for qt in range(QT):
            for kt in range(KT):
                blk = block(b, qt, kt)
                if blk.all():
                    kinds[b, qt, kt] = 1
                elif blk.any():
                    kinds[b, qt, kt] = 2
    return kinds


def block_kinds(mask: np.ndarray) -> np.ndarray:
    """mask [B, Nq, Nk] (nonzero = attend) -> kinds uint8 [B, QT, KT] by any/all."""
    return block_kinds_from(*_mask_blocks(mask))


def mask_from_lengths(lengths, npad: int) -> np.ndarray:
    """Element mask of a padded batch: query i sees key j iff both are < n_b."""
    lengths = np.asarray(lengths)
    idx = np.arange(npad)
    valid = idx[None, :] < lengths[:, None]
    return (valid[:, :, None] & valid[:, None, :]).astype(np.uint8)


def _tile_list(B, Nq, Nk, block) -> dict:
    QT, KT = -(-Nq // T), -(-Nk // T)
    kinds = block_kinds_from(B, Nq, Nk, block)
    row_ptr = [0]
    col_idx, kind, pidx, bits = [], [], [], []
    for b in range(B):
        for qt in range(QT):
            for kt in range(KT):
                kd = int(kinds[b, qt, kt])
                if kd == 0:
                    continue
                col_idx.append(kt)
                kind.append(kd)
                if kd == 2:
                    pidx.append(len(bits))
                    blk = block(b, qt, kt)
                    words = np.zeros((T, 4), dtype=np.uint64)
                    for k in range(T):
                        words[:, k // 32] |= blk[:, k].astype(np.uint64) << np.uint64(k % 32)
                    bits.append(words.astype(np.uint32).reshape(-1))
                else:
                    pidx.append(-1)
            row_ptr.append(len(col_idx))
    # CSC with the CSR index of each entry
    entry_of = {}
    e = 0
    for r in range(B * QT):
        for _ in range(row_ptr[r], row_ptr[r + 1]):
            entry_of[(r // QT, r % QT, col_idx[e])] = e
            e += 1
    colT_ptr = [0]
    rowT_idx, csc_map = [], []
    for b in range(B):
        for kt in range(KT):
            for qt in range(QT):
                if kinds[b, qt, kt]:
                    rowT_idx.append(qt)
                    csc_map.append(entry_of[(b, qt, kt)])
            colT_ptr.append(len(rowT_idx))
    return {
        "B": B, "QT": QT, "KT": KT, "kinds": kinds,
        "row_ptr": np.asarray(row_ptr, dtype=np.int32),
        "col_idx": np.asarray(col_idx, dtype=np.int32),
        "kind": np.asarray(kind, dtype=np.uint8),
        "pidx": np.asarray(pidx, dtype=np.int32),
        "colT_ptr": np.asarray(colT_ptr, dtype=np.int32),
        "rowT_idx": np.asarray(rowT_idx, dtype=np.int32),
        "csc_map": np.asarray(csc_map, dtype=np.int32),
        "bits": (np.stack(bits) if bits else np.zeros((0, 512), dtype=np.uint32)),
    }


def tile_list(mask: np.ndarray) -> dict:
    """The full tile list of an element mask [B, Nq, Nk], as numpy arrays."""
    return _tile_list(*_mask_blocks(mask))


def tile_list_from_lengths(lengths, npad: int) -> dict:
    """The tile list of a padded batch, block by block from the lengths."""
    return _tile_list(*_length_blocks(lengths, npad))


def row_runs(t: dict):
    """Runs of a tile list (the dict of tile_list / tile_list_from_lengths): for each q-tile
    row, the maximal ranges of consecutive k-tiles of one kind ("Binary Block Masking",
    section "Comment ça marche ?", consecutive non-zero blocks).  Returns run_ptr int32
    [B*QT + 1] and runs int32 [nruns, 4] = {first k-tile, number of tiles, kind, first CSR
    entry}, rows in order, runs in ascending k-tile order; found by walking each row's
    entries one by one."""
    run_ptr = [0]
    runs = []
    for r in range(len(t["row_ptr"]) - 1):
        e0, e1 = int(t["row_ptr"][r]), int(t["row_ptr"][r + 1])
        e = e0
        while e < e1:
            start = e
            while (e + 1 < e1 and t["col_idx"][e + 1] == t["col_idx"][e] + 1
                   and t["kind"][e + 1] == t["kind"][start]):
                e += 1
            runs.append([int(t["col_idx"][start]), e - start + 1, int(t["kind"][start]), start])
            e += 1
        run_ptr.append(len(runs))
    return (np.asarray(run_ptr, dtype=np.int32),
            np.asarray(runs, dtype=np.int32).reshape(-1, 4))
