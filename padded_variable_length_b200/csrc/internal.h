// Host-side internals shared by the translation units of libsigattn.so.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "sigattn.h"

// Device buffers of a tile plan.  Layouts are those of sigattn_plan_export; in addition
// the plan keeps the transposed PARTIAL bitmasks (for kernels that own a key per thread)
// and two work lists ordered longest-first (count descending, then index):
//   row_work[B*QT]  every (b, q-tile) row, rows with no tile last
//   col_work[B*KT]  every (b, k-tile) column, columns with no tile last
struct sigattn_plan {
  int device;
  // packed batches only (else nullptr / 0): device copy of the cumulative offsets [B + 1]
  // and the total number of rows T = cu[B]
  int32_t* cu;
  int64_t T;
  // the device allocations every buffer below is carved from: one for a plan whose tile
  // arrays are sized for the worst case (it also holds the build's scratch), else two
  void* arena[2];
  int B, Nq, Nk, QT, KT;
  // the counts below are written by the build's kernels into dcount (device, indexed by
  // sigattn::PlanCount) and copied into these host fields on first use (plan_counts), so
  // that a build queues its work and returns without waiting for the device
  int64_t nonempty, full, partial;
  int64_t run_cap;  // entries allocated in the per-tile arrays (>= nonempty)
  int32_t rows_nonempty, cols_nonempty;
  int64_t* dcount;
  bool counts_known;
  cudaEvent_t ready;  // recorded after the build's last kernel (nullptr: the build waited)
  int32_t* row_ptr;
  int32_t* col_idx;
  uint8_t* kind;
  int32_t* pidx;
  int32_t* colT_ptr;
  int32_t* rowT_idx;
  int32_t* csc_map;
  uint32_t* bits;
  uint32_t* bitsT;  // [partial * 512] the same bitmasks transposed: bit (q % 32) of word (k*4 + q/32)
  int32_t* row_work;
  int32_t* col_work;
  // the work lists again, one 16-byte record per entry: {row or column, first list entry,
  // number of entries, first run (rows) or 0 (columns)}, so that a kernel decodes a work
  // item with one independent load
  int4* row_desc;
  int4* col_desc;
  // runs of each q-tile row: maximal ranges of consecutive k-tiles of one kind, one 16-byte
  // record each {first k-tile, number of tiles, kind, first CSR entry}; row r's runs are
  // run[run_ptr[r] .. run_ptr[r+1])
  int32_t* run_ptr;
  int4* run;
};

namespace sigattn {

constexpr int kTile = 128;

// Slots of a plan's device counts (int64 each): listed tiles, PARTIAL tiles, q-tile rows
// with tiles, k-tile columns with tiles, the build's barrier-timeout flag, and the arrival
// counters of the build's grid barriers (two 32-bit counters in one slot).
enum PlanCount : int {
  kCountListed = 0,
  kCountPartial,
  kCountRows,
  kCountCols,
  kCountTimeout,
  kCountArrive,
  kCountSlots
};

// Host copies of the plan's counts: waits for the build (if it has not been waited for),
// reads the device counts once.  Errors: TIMEOUT (a grid barrier of the build gave up),
// CUDA.
int plan_counts(sigattn_plan* plan);

// Makes work queued on `stream` from now on wait for the plan's build.
int plan_wait(const sigattn_plan* plan, cudaStream_t stream);

// Where the rows of sequence b live.  Padded batches index tensors by (b, row) with a batch
// stride; a packed batch (a plan built from cumulative offsets cu[0..B]) keeps sequence b in
// rows cu[b] .. cu[b+1] of one [T, H, d] tensor, so it has no batch coordinate, its rows
// start at cu[b], and only its own n_b = cu[b+1] - cu[b] rows may be written.
struct SeqRows {
  int tma_b;  // batch coordinate for the TMA maps (0 when packed)
  int row0;   // first row of the sequence in the token dimension (0 when padded)
  int limit;  // rows of the sequence present in the tensors (N when padded, n_b when packed)
};

__host__ __device__ __forceinline__ SeqRows seq_rows(const int32_t* cu, int b, int N) {
  if (cu == nullptr) return SeqRows{b, 0, N};
  const int a = cu[b];
  return SeqRows{0, a, cu[b + 1] - a};
}

// Element offset of row r of a sequence in a tensor with batch / token strides sb, sn.
__host__ __device__ __forceinline__ int64_t seq_row_offset(const SeqRows& s, int64_t sb, int64_t sn,
                                                          int r) {
  return static_cast<int64_t>(s.tma_b) * sb + static_cast<int64_t>(s.row0 + r) * sn;
}

// Per-tensor description handed to the launchers (element strides).
struct TensorDesc {
  const void* ptr;
  int64_t sb, sn, sh;  // batch, token, head strides in elements; d is contiguous
  int N;               // rows (Nq or Nk)
};

// Builds a 4-D TMA descriptor over a [B, N, H, d] bf16 tensor with a box of
// 64 (d) x 128 (tokens) x 1 x 1 and 128-byte swizzle.
int make_tmap_bf16(CUtensorMap* map, const TensorDesc& t, int B, int H, int d);

// 4-D TMA descriptor over a contiguous fp32 [B, N, H, d] tensor with a box of 32 (d) x 16
// (tokens) x 1 x 1 and 128-byte swizzle (the fused backward's dQ accumulator).
int make_tmap_f32_acc(CUtensorMap* map, float* base, int B, int N, int H, int d);

int cuda_status(cudaError_t e);

// Device address of this device's status word (the record of bounded waits that gave up).
int status_ptr(int** out);

// Per-device cache of the device address of one file-scope __device__ variable.  In host
// code such a variable's name is only a host-side stand-in, so its address is looked up with
// cudaGetSymbolAddress once per device, with that device current, and reused.  The cache
// lives as long as the process: a cudaDeviceReset invalidates the addresses it holds (this
// library does not support resetting a device it has been used on).
constexpr int kMaxDevices = 64;

struct SymbolAddressCache {
  std::mutex mu;
  void* addr[kMaxDevices] = {nullptr};

  // *out = the symbol's address on the current device.  Errors: NO_DEVICE, UNSUPPORTED
  // (device ordinal past kMaxDevices), CUDA.
  template <class T>
  int get(const T& symbol, void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
      cudaGetLastError();
      return SIGATTN_ERR_NO_DEVICE;
    }
    if (dev < 0 || dev >= kMaxDevices) return SIGATTN_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
      void* p = nullptr;
      const cudaError_t e = cudaGetSymbolAddress(&p, symbol);
      if (e != cudaSuccess) return cuda_status(e);
      addr[dev] = p;
    }
    *out = addr[dev];
    return SIGATTN_OK;
  }
};

}  // namespace sigattn
