// Structural checks of a tile list: the debug aid behind sigattn_plan_validate (the plan's
// own device arrays, checked by one kernel) and sigattn_tile_list_check_host (the same
// checks on host arrays in the export layout).  Nothing on the attention path calls them.
//
// What a tile list must satisfy ("Binary Block Masking for FlashAttention", section
// "Comment ça marche ?": the non-empty blocks of each row, FULL or PARTIAL with a block
// mask): CSR offsets non-decreasing from 0 to the entry count; k-tiles in range and strictly
// ascending within a row; kinds 1 (FULL) or 2 (PARTIAL); a FULL entry has no bitmask number,
// PARTIAL entries are numbered 0, 1, ... in CSR order; CSC offsets likewise, q-tiles in range
// and strictly ascending within a column, and each CSC entry maps to the CSR entry of the
// same (batch entry, q-tile, k-tile) -- with both lists sorted and of equal length that makes
// the map a bijection; a PARTIAL bitmask has at least one set and one clear bit (else the
// block would be empty or FULL); each row's runs cover its entries exactly, in maximal
// ranges of consecutive k-tiles of one kind.  The device check adds what only the plan
// holds: the transposed bitmasks and the longest-first work lists with their records.
#include <cuda_runtime.h>

#include <cstdint>

#include "internal.h"

namespace sigattn {
namespace {

// Codes of the failing check (the high bits of the reported position).
enum CheckCode : int64_t {
  kChkRowPtr = 1, kChkColIdx, kChkKind, kChkPidx, kChkColPtr, kChkRowT, kChkCscMap,
  kChkBits, kChkRuns, kChkBitsT, kChkWork
};

__host__ __device__ inline int64_t bad(CheckCode c, int64_t i) { return (static_cast<int64_t>(c) << 40) | i; }

struct TileListView {
  int B, QT, KT;
  int64_t nonempty, partial, nruns;
  const int32_t* row_ptr;
  const int32_t* col_idx;
  const uint8_t* kind;
  const int32_t* pidx;
  const int32_t* colT_ptr;
  const int32_t* rowT_idx;
  const int32_t* csc_map;
  const uint32_t* bits;
  const int32_t* run_ptr;  // may be null (runs not checked)
  const int4* run;
};

// Row r = b * QT + qt of the CSR list, its kinds and bitmask numbers, and its runs.
// Returns 0 or the first failure found.
__host__ __device__ int64_t check_row(const TileListView& t, int64_t r) {
  const int64_t rows = static_cast<int64_t>(t.B) * t.QT;
  const int64_t lo = t.row_ptr[r], hi = t.row_ptr[r + 1];
  if (lo < 0 || hi < lo || hi > t.nonempty || (r == 0 && lo != 0) ||
      (r == rows - 1 && hi != t.nonempty))
    return bad(kChkRowPtr, r);
  int32_t last_p = -1;
  for (int64_t e = lo; e < hi; ++e) {
    const int32_t k = t.col_idx[e];
    if (k < 0 || k >= t.KT || (e > lo && k <= t.col_idx[e - 1])) return bad(kChkColIdx, e);
    const int kd = t.kind[e];
    if (kd != 1 && kd != 2) return bad(kChkKind, e);
    const int32_t p = t.pidx[e];
    if (kd == 1 ? p != -1 : (p < 0 || p >= t.partial || (last_p >= 0 && p != last_p + 1)))
      return bad(kChkPidx, e);
    if (kd == 2) last_p = p;
  }
  if (!t.run_ptr) return 0;
  const int64_t r0 = t.run_ptr[r], r1 = t.run_ptr[r + 1];
  if (r0 < 0 || r1 < r0 || r1 > t.nruns || (r == 0 && r0 != 0) || (r == rows - 1 && r1 != t.nruns))
    return bad(kChkRuns, r);
  int64_t e = lo;
  for (int64_t j = r0; j < r1; ++j) {
    const int4 u = t.run[j];  // {first k-tile, tiles, kind, first entry}
    if (u.w != e || u.y < 1 || e + u.y > hi) return bad(kChkRuns, r);
    for (int i = 0; i < u.y; ++i)
      if (t.col_idx[e + i] != u.x + i || t.kind[e + i] != u.z) return bad(kChkRuns, r);
    e += u.y;
    // maximal: the next entry of the row must not extend this run
    if (e < hi && t.col_idx[e] == u.x + u.y && t.kind[e] == u.z) return bad(kChkRuns, r);
  }
  return e == hi ? 0 : bad(kChkRuns, r);
}

// Column c = b * KT + kt of the CSC list and its map to the CSR entries.
__host__ __device__ int64_t check_col(const TileListView& t, int64_t c) {
  const int64_t cols = static_cast<int64_t>(t.B) * t.KT;
  const int64_t lo = t.colT_ptr[c], hi = t.colT_ptr[c + 1];
  if (lo < 0 || hi < lo || hi > t.nonempty || (c == 0 && lo != 0) ||
      (c == cols - 1 && hi != t.nonempty))
    return bad(kChkColPtr, c);
  const int64_t b = c / t.KT, kt = c % t.KT;
  for (int64_t e = lo; e < hi; ++e) {
    const int32_t q = t.rowT_idx[e];
    if (q < 0 || q >= t.QT || (e > lo && q <= t.rowT_idx[e - 1])) return bad(kChkRowT, e);
    const int64_t m = t.csc_map[e], r = b * t.QT + q;
    if (m < 0 || m >= t.nonempty || t.col_idx[m] != kt || m < t.row_ptr[r] || m >= t.row_ptr[r + 1])
      return bad(kChkCscMap, e);
  }
  return 0;
}

// Bitmask p: neither all clear nor all set.
__host__ __device__ int64_t check_bits(const TileListView& t, int64_t p) {
  uint32_t any = 0, all = 0xFFFFFFFFu;
  for (int w = 0; w < 512; ++w) {
    const uint32_t x = t.bits[p * 512 + w];
    any |= x;
    all &= x;
  }
  return (any != 0 && all != 0xFFFFFFFFu) ? 0 : bad(kChkBits, p);
}

__device__ void record(int64_t* first_bad, int64_t v) {
  if (v) atomicMin(reinterpret_cast<unsigned long long*>(first_bad), static_cast<unsigned long long>(v));
}

// One thread per row, column, bitmask word and work-list slot (grid-stride).
__global__ void k_plan_check(TileListView t, const uint32_t* __restrict__ bitsT,
                             const int32_t* __restrict__ row_work, const int4* __restrict__ row_desc,
                             const int32_t* __restrict__ col_work, const int4* __restrict__ col_desc,
                             int64_t* first_bad) {
  const int64_t rows = static_cast<int64_t>(t.B) * t.QT, cols = static_cast<int64_t>(t.B) * t.KT;
  const int64_t words = t.partial * 512;
  const int64_t n = rows + cols + t.partial + words + rows + cols;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    int64_t j = i;
    if (j < rows) { record(first_bad, check_row(t, j)); continue; }
    j -= rows;
    if (j < cols) { record(first_bad, check_col(t, j)); continue; }
    j -= cols;
    if (j < t.partial) { record(first_bad, check_bits(t, j)); continue; }
    j -= t.partial;
    if (j < words) {
      // word w = q * 4 + k / 32 of bitmask p against the transposed copy: bit (q % 32) of
      // word (k * 4 + q / 32)
      const int64_t p = j / 512;
      const int w = static_cast<int>(j % 512), q = w >> 2, kb = (w & 3) * 32;
      const uint32_t x = t.bits[j];
      for (int s = 0; s < 32; ++s) {
        const uint32_t y = bitsT[p * 512 + (kb + s) * 4 + (q >> 5)];
        if (((x >> s) & 1u) != ((y >> (q & 31)) & 1u)) {
          record(first_bad, bad(kChkBitsT, p));
          break;
        }
      }
      continue;
    }
    j -= words;
    // work lists: every slot names a row (column) in range, lengths never grow along the
    // list, and the slot's record is {item, first entry, entries, first run (rows) or 0}
    const bool is_row = j < rows;
    if (!is_row) j -= rows;
    const int64_t m = is_row ? rows : cols;
    const int32_t* work = is_row ? row_work : col_work;
    const int32_t* ptr = is_row ? t.row_ptr : t.colT_ptr;
    const int32_t it = work[j];
    bool ok = it >= 0 && it < m;
    if (ok) {
      const int4 d = (is_row ? row_desc : col_desc)[j];
      const int32_t len = ptr[it + 1] - ptr[it];
      ok = d.x == it && d.y == ptr[it] && d.z == len && d.w == (is_row && t.run_ptr ? t.run_ptr[it] : 0);
      if (ok && j + 1 < m) {
        const int32_t nx = work[j + 1];
        ok = nx >= 0 && nx < m && ptr[nx + 1] - ptr[nx] <= len;
      }
    }
    if (!ok) record(first_bad, bad(kChkWork, j));
  }
}

}  // namespace
}  // namespace sigattn

using namespace sigattn;

extern "C" int sigattn_plan_validate(const sigattn_plan* plan, sigattn_stream stream_,
                                     int64_t* first_bad) {
  if (!plan) return SIGATTN_ERR_INVALID;
  if (first_bad) *first_bad = -1;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != plan->device) {
    cudaGetLastError();
    return SIGATTN_ERR_SHAPE;
  }
  if (const int rc = plan_counts(const_cast<sigattn_plan*>(plan)); rc != SIGATTN_OK) return rc;
  const cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  const int64_t rows = static_cast<int64_t>(plan->B) * plan->QT;
  int32_t nruns = 0;
  int64_t* d_bad = nullptr;
  int64_t h_bad = 0;
  int rc = SIGATTN_OK;
  // the run count bounds the run array: read it first (a count above the entry count fails
  // the check without a read past the array)
  if (cudaMemcpy(&nruns, plan->run_ptr + rows, sizeof(int32_t), cudaMemcpyDeviceToHost) != cudaSuccess ||
      cudaMalloc(&d_bad, sizeof(int64_t)) != cudaSuccess) {
    cudaGetLastError();
    cudaFree(d_bad);
    return SIGATTN_ERR_CUDA;
  }
  if (nruns < 0 || nruns > plan->nonempty) {
    h_bad = bad(kChkRuns, rows);
  } else {
    TileListView t{plan->B, plan->QT, plan->KT, plan->nonempty, plan->partial, nruns,
                   plan->row_ptr, plan->col_idx, plan->kind, plan->pidx, plan->colT_ptr,
                   plan->rowT_idx, plan->csc_map, plan->bits, plan->run_ptr, plan->run};
    const int64_t all = 0x7FFFFFFFFFFFFFFFll;
    cudaMemcpyAsync(d_bad, &all, sizeof(int64_t), cudaMemcpyHostToDevice, stream);
    k_plan_check<<<4 * 148, 256, 0, stream>>>(t, plan->bitsT, plan->row_work, plan->row_desc,
                                              plan->col_work, plan->col_desc, d_bad);
    if (cudaMemcpyAsync(&h_bad, d_bad, sizeof(int64_t), cudaMemcpyDeviceToHost, stream) != cudaSuccess ||
        cudaStreamSynchronize(stream) != cudaSuccess) {
      cudaGetLastError();
      rc = SIGATTN_ERR_CUDA;
    }
    if (h_bad == all) h_bad = 0;
  }
  cudaFree(d_bad);
  if (rc != SIGATTN_OK) return rc;
  if (first_bad && h_bad) *first_bad = h_bad;
  return h_bad ? SIGATTN_ERR_PLAN : SIGATTN_OK;
}

extern "C" int sigattn_tile_list_check_host(int B, int QT, int KT, int64_t nonempty, int64_t partial,
                                            const int32_t* row_ptr, const int32_t* col_idx,
                                            const uint8_t* kind, const int32_t* pidx,
                                            const int32_t* colT_ptr, const int32_t* rowT_idx,
                                            const int32_t* csc_map, const uint32_t* bits,
                                            const int32_t* run_ptr, const int32_t* runs,
                                            int64_t nruns, int64_t* first_bad) {
  if (first_bad) *first_bad = -1;
  if (B < 1 || QT < 1 || KT < 1 || nonempty < 0 || partial < 0 || nruns < 0 || !row_ptr ||
      !colT_ptr || (nonempty > 0 && (!col_idx || !kind || !pidx || !rowT_idx || !csc_map)) ||
      (partial > 0 && !bits) || (run_ptr && nruns > 0 && !runs))
    return SIGATTN_ERR_INVALID;
  TileListView t{B, QT, KT, nonempty, partial, nruns, row_ptr, col_idx, kind, pidx, colT_ptr,
                 rowT_idx, csc_map, bits, run_ptr, reinterpret_cast<const int4*>(runs)};
  int64_t v = 0;
  const int64_t rows = static_cast<int64_t>(B) * QT, cols = static_cast<int64_t>(B) * KT;
  for (int64_t r = 0; r < rows && !v; ++r) v = check_row(t, r);
  if (!v) {
    // PARTIAL entries numbered 0, 1, ... in CSR order, one bitmask each
    int64_t next = 0;
    for (int64_t e = 0; e < nonempty && !v; ++e)
      if (kind[e] == 2 && pidx[e] != next++) v = bad(kChkPidx, e);
    if (!v && next != partial) v = bad(kChkPidx, nonempty);
  }
  for (int64_t c = 0; c < cols && !v; ++c) v = check_col(t, c);
  for (int64_t p = 0; p < partial && !v; ++p) v = check_bits(t, p);
  if (first_bad && v) *first_bad = v;
  return v ? SIGATTN_ERR_PLAN : SIGATTN_OK;
}
