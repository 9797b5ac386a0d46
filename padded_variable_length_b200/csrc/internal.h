// Host-side internals shared by the translation units of libsigattn.so.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "sigattn.h"

// Device buffers of a tile plan.  Layouts are those of sigattn_plan_export; in addition
// the plan keeps the transposed PARTIAL bitmasks (for kernels that own a key per thread)
// and two work lists ordered longest-first (count descending, then index):
//   row_work[B*QT]  every (b, q-tile) row, rows with no tile last
//   col_work[B*KT]  every (b, k-tile) column, columns with no tile last
struct sigattn_plan {
  int device;
  int B, Nq, Nk, QT, KT;
  int64_t nonempty, full, partial;
  int32_t rows_nonempty, cols_nonempty;
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
  // number of entries, 0}, so that a kernel decodes a work item with one independent load
  int4* row_desc;
  int4* col_desc;
};

namespace sigattn {

constexpr int kTile = 128;

// Per-tensor description handed to the launchers (element strides).
struct TensorDesc {
  const void* ptr;
  int64_t sb, sn, sh;  // batch, token, head strides in elements; d is contiguous
  int N;               // rows (Nq or Nk)
};

// Builds a 4-D TMA descriptor over a [B, N, H, d] bf16 tensor with a box of
// 64 (d) x 128 (tokens) x 1 x 1 and 128-byte swizzle.
int make_tmap_bf16(CUtensorMap* map, const TensorDesc& t, int B, int H, int d);

int cuda_status(cudaError_t e);

}  // namespace sigattn
