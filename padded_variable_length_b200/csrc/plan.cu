// Tile planner: element mask or per-sequence lengths -> list of non-empty 128 x 128 tiles.
//
// "Binary Block Masking for FlashAttention", section "Comment ça marche ?": the element
// mask becomes a binary matrix of blocks (a block is kept iff it holds a non-zero entry)
// and only kept blocks are computed; the block matrix is built in parallel once and
// shared by every head (section "Présentation de Binary Block Masking").  "Better
// Models, Faster Training: Sigmoid Attention for single-cell Foundation Models", section
// 2C: blocks that are padding on the query side or the key side are skipped.
//
// Pipeline (all on the device, one plan per batch, broadcast over heads):
//   1 classify every block of the padded grid: 0 empty, 1 FULL, 2 PARTIAL
//   2 count listed blocks per q-tile row (and PARTIAL ones), per k-tile column
//   3 exclusive scans -> CSR / CSC offsets and the PARTIAL numbering
//   4 work lists: rows and columns ordered by tile count, longest first (stable)
//   5 fill CSR, CSC and the PARTIAL bitmasks
// Steps 2-5 are one cooperative launch with grid-wide barriers between them.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "internal.h"
#include "sm100.cuh"

namespace sigattn {
namespace {

constexpr int kSortBuckets = 4096;  // tile counts >= 4095 share the longest bucket

// Per-byte "is nonzero" flags of a 32-bit word: bit 7 of each byte set iff that byte != 0.
__device__ __forceinline__ uint32_t nonzero_bytes(uint32_t w) {
  return (((w & 0x7F7F7F7Fu) + 0x7F7F7F7Fu) | w) & 0x80808080u;
}

// Compresses the flags of nonzero_bytes() into 4 bits (byte 0 -> bit 0).
__device__ __forceinline__ uint32_t flags4(uint32_t f) {
  return ((f >> 7) & 1u) | ((f >> 14) & 2u) | ((f >> 21) & 4u) | ((f >> 28) & 8u);
}

__device__ __forceinline__ uint32_t low_bits(int m) {
  return m >= 32 ? 0xFFFFFFFFu : (m <= 0 ? 0u : ((1u << m) - 1u));
}

__global__ void k_kinds_from_lengths(const int32_t* __restrict__ lengths, int B, int Npad, int QT,
                                     int KT, uint8_t* __restrict__ kinds, int64_t* __restrict__ zero2) {
  if (blockIdx.x == 0 && threadIdx.x < 2) zero2[threadIdx.x] = 0;
  const int64_t total = static_cast<int64_t>(B) * QT * KT;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int kt = static_cast<int>(i % KT);
    const int qt = static_cast<int>((i / KT) % QT);
    const int b = static_cast<int>(i / (static_cast<int64_t>(KT) * QT));
    const int n = min(max(lengths[b], 0), Npad);
    const bool any = qt * kTile < n && kt * kTile < n;
    const bool all = (qt + 1) * kTile <= n && (kt + 1) * kTile <= n;
    kinds[i] = all ? 1 : (any ? 2 : 0);
  }
}

// Reads the 128 mask bytes of row `row` of a block from column col0 on: bit i of w[c] is
// column col0 + 32c + i.  Columns past Nk and rows past Nq read as zero.
__device__ __forceinline__ void row_bits(const uint8_t* __restrict__ mask, int Nq, int Nk,
                                         int64_t sb, int64_t sq, int b, int row, int col0,
                                         uint32_t (&w)[4]) {
  w[0] = w[1] = w[2] = w[3] = 0u;
  if (row >= Nq || col0 >= Nk) return;
  const uint8_t* p = mask + b * sb + row * sq + col0;
  const int nv = min(kTile, Nk - col0);
  if (nv == kTile && (reinterpret_cast<uintptr_t>(p) & 15u) == 0) {
    const uint4* p4 = reinterpret_cast<const uint4*>(p);
    uint4 v[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) v[c] = __ldg(p4 + c);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const uint32_t f = flags4(nonzero_bytes(v[c].x)) | (flags4(nonzero_bytes(v[c].y)) << 4) |
                         (flags4(nonzero_bytes(v[c].z)) << 8) | (flags4(nonzero_bytes(v[c].w)) << 12);
      w[c >> 1] |= f << ((c & 1) * 16);
    }
  } else {
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4) {
      uint32_t x = 0u;
      for (int i = 0; i < 32; ++i) {
        const int c = c4 * 32 + i;
        if (c < nv && p[c] != 0) x |= 1u << i;
      }
      w[c4] = x;
    }
  }
}

// One CTA of 256 threads per block of the grid (grid-stride over blocks): warp w reads rows
// 16w .. 16w + 15 of the block, lane l the 16 bytes at column 16 (l % 8) of rows
// 16w + l/8 + 4i (i < 4) -- every load instruction of a warp covers four whole 128-byte rows,
// and all four loads of a thread are in flight at once -- and the CTA votes on "any element
// kept" and "all kept".  Rows past Nq and columns past Nk count as not kept.  Masks whose
// rows are not 16-byte aligned take a byte-wise path.  zero2: two words zeroed for the
// steps that follow.
__global__ void __launch_bounds__(256) k_kinds_from_mask(const uint8_t* __restrict__ mask, int B,
                                                         int Nq, int Nk, int64_t sb, int64_t sq,
                                                         int QT, int KT,
                                                         uint8_t* __restrict__ kinds,
                                                         int64_t* __restrict__ zero2) {
  if (blockIdx.x == 0 && threadIdx.x < 2) zero2[threadIdx.x] = 0;
  const int64_t total = static_cast<int64_t>(B) * QT * KT;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const bool vec = ((reinterpret_cast<uintptr_t>(mask) | static_cast<uintptr_t>(sb) |
                     static_cast<uintptr_t>(sq)) & 15u) == 0;
  for (int64_t blk = blockIdx.x; blk < total; blk += gridDim.x) {
    const int kt = static_cast<int>(blk % KT);
    const int qt = static_cast<int>((blk / KT) % QT);
    const int b = static_cast<int>(blk / (static_cast<int64_t>(KT) * QT));
    const int col = kt * kTile + (lane & 7) * 16;
    const uint8_t* base = mask + b * sb + col;
    const int row0 = qt * kTile + warp * 16 + (lane >> 3);
    bool any = false, all = true;
    if (vec && kt * kTile + kTile <= Nk) {
      uint4 v[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int row = row0 + 4 * i;
        v[i] = row < Nq ? __ldg(reinterpret_cast<const uint4*>(base + row * sq)) : make_uint4(0u, 0u, 0u, 0u);
        if (row >= Nq) all = false;
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        any |= (v[i].x | v[i].y | v[i].z | v[i].w) != 0u;
        all &= (nonzero_bytes(v[i].x) & nonzero_bytes(v[i].y) & nonzero_bytes(v[i].z) &
                nonzero_bytes(v[i].w)) == 0x80808080u;
      }
    } else {
      for (int i = 0; i < 4; ++i) {
        const int row = row0 + 4 * i;
        for (int j = 0; j < 16; ++j) {
          const bool in = row < Nq && col + j < Nk;
          const bool kept = in && base[row * sq + j] != 0;
          any |= kept;
          all &= kept;
        }
      }
    }
    any = __syncthreads_or(any);
    all = __syncthreads_and(all);
    if (threadIdx.x == 0) kinds[blk] = all ? 1 : (any ? 2 : 0);
  }
}

// A listed block starts a run iff the block before it in the row is not listed or is of
// the other kind (runs: maximal ranges of consecutive k-tiles of one kind).
__device__ __forceinline__ bool starts_run(const uint8_t* __restrict__ k, int kt, uint8_t v) {
  return v != 0 && (kt == 0 || k[kt - 1] != v);
}

// The steps after the classification run as one cooperative launch of one 1024-thread CTA
// per SM, in four phases separated by grid-wide barriers:
//   0 counts: listed / PARTIAL blocks and runs per q-tile row, listed blocks per column
//   1 the four exclusive scans (CSR, PARTIAL numbering, CSC, runs) and the two
//     longest-first sorts, one CTA each
//   2 the work descriptors (from the first thread of the grid on), and CSR + PARTIAL
//     numbering + runs (one warp per row, from the last warp of the grid down)
//   3 the PARTIAL blocks' bitmasks with their transposes (from the first CTA on), and CSC
//     (one warp per column, from the last warp down): the two parts of a phase run side by
//     side on different CTAs
// A launch may run a range of the phases (a plan too large to size for the worst case
// runs 0..2, lets the host read the counts, then runs the fill part of 2 and 3).

// Row r < rows: number of listed blocks, of PARTIAL blocks and of runs; then column
// c = b*KT + kt: number of listed blocks.  One warp per row or column; gw / nw: this warp's
// index in the grid and the number of warps.
__device__ void count_step(const uint8_t* __restrict__ kinds, int B, int QT, int KT,
                           int32_t* __restrict__ row_cnt, int32_t* __restrict__ row_pcnt,
                           int32_t* __restrict__ run_cnt, int32_t* __restrict__ col_cnt, int gw,
                           int nw) {
  const int lane = threadIdx.x & 31;
  const int rows = B * QT, total = rows + B * KT;
  for (int w = gw; w < total; w += nw) {
    if (w < rows) {
      const uint8_t* k = kinds + static_cast<int64_t>(w) * KT;
      int c = 0, p = 0, n = 0;
      for (int kt = lane; kt < KT; kt += 32) {
        const uint8_t v = k[kt];
        c += v != 0;
        p += v == 2;
        n += starts_run(k, kt, v);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        c += __shfl_xor_sync(0xFFFFFFFFu, c, o);
        p += __shfl_xor_sync(0xFFFFFFFFu, p, o);
        n += __shfl_xor_sync(0xFFFFFFFFu, n, o);
      }
      if (lane == 0) {
        row_cnt[w] = c;
        row_pcnt[w] = p;
        run_cnt[w] = n;
      }
    } else {
      const int col = w - rows;
      const int b = col / KT, kt = col % KT;
      int c = 0;
      for (int qt = lane; qt < QT; qt += 32)
        c += kinds[(static_cast<int64_t>(b) * QT + qt) * KT + kt] != 0;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xFFFFFFFFu, c, o);
      if (lane == 0) col_cnt[col] = c;
    }
  }
}

// Inclusive scan over the 1024 threads of a CTA (every thread must call it).
__device__ __forceinline__ int block_inclusive_scan(int x, int32_t* warp_sums) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int s = warp_sums[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xFFFFFFFFu, s, o);
      if (lane >= o) s += y;
    }
    warp_sums[lane] = s;  // inclusive over warps
  }
  __syncthreads();
  const int r = incl + (warp > 0 ? warp_sums[warp - 1] : 0);
  __syncthreads();  // warp_sums is reused by the next call
  return r;
}

// Exclusive scan of in[0..n) into out[0..n]; out[n] is the total, also stored to *total.
struct ScanJob {
  const int32_t* in;
  int n;
  int32_t* out;
  int64_t* total;
};

// One CTA of 1024 threads walks the input in chunks of 1024.
__device__ void scan_job(const ScanJob& j, int32_t* warp_sums, int32_t* chunk_total) {
  int carry = 0;
  for (int base = 0; base < j.n; base += 1024) {
    const int i = base + threadIdx.x;
    const int x = i < j.n ? j.in[i] : 0;
    const int incl = block_inclusive_scan(x, warp_sums);
    if (i < j.n) j.out[i] = carry + incl - x;
    if (threadIdx.x == 1023) *chunk_total = incl;
    __syncthreads();
    carry += *chunk_total;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    j.out[j.n] = carry;
    if (j.total) *j.total = carry;
  }
}

// Stable counting sort of indices 0..n-1 by cnt[i] descending (counts past 4094 share a
// bucket); also stores the number of nonzero counts to *nonzero.
struct SortJob {
  const int32_t* cnt;
  int n;
  int32_t* out;
  int64_t* nonzero;
};

__device__ __forceinline__ int sort_key(int c) {
  return kSortBuckets - 1 - min(c, kSortBuckets - 1);  // ascending key = descending count
}

// One CTA of 1024 threads.  Histogram and bucket offsets in shared memory (start: 4096
// words); then the indices are placed in chunks of 1024 in index order: equal keys within
// a warp are ranked by lane (match), and the 32 warps of a chunk claim their slots one
// after another, so that the order of equal keys is the index order.
__device__ void sort_job(const SortJob& j, int32_t* start, int32_t* warp_sums, int32_t* nz_total) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int i = tid; i < kSortBuckets; i += 1024) start[i] = 0;
  if (tid == 0) *nz_total = 0;
  __syncthreads();
  int nz = 0;
  for (int i = tid; i < j.n; i += 1024) {
    const int c = j.cnt[i];
    nz += c > 0;
    atomicAdd(&start[sort_key(c)], 1);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) nz += __shfl_xor_sync(0xFFFFFFFFu, nz, o);
  if (lane == 0) atomicAdd(nz_total, nz);
  __syncthreads();
  // exclusive scan over the buckets: thread t owns buckets [4t, 4t + 4)
  static_assert(kSortBuckets == 4 * 1024, "four buckets per thread");
  int v[4], sum = 0;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    v[k] = start[4 * tid + k];
    sum += v[k];
  }
  int run = block_inclusive_scan(sum, warp_sums) - sum;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    start[4 * tid + k] = run;
    run += v[k];
  }
  __syncthreads();
  for (int base = 0; base < j.n; base += 1024) {
    const int i = base + tid;
    const bool act = i < j.n;
    const int key = act ? sort_key(j.cnt[i]) : -1 - lane;
    const unsigned peers = __match_any_sync(0xFFFFFFFFu, key);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    const int leader = __ffs(peers) - 1;
    int first = 0;
    const int warps_used = min(32, (j.n - base + 31) >> 5);  // the chunk's warps with indices
    for (int w = 0; w < warps_used; ++w) {
      if (warp == w && act && rank == 0) {
        first = start[key];
        start[key] = first + __popc(peers);
      }
      __syncthreads();
    }
    const int pos = __shfl_sync(0xFFFFFFFFu, first, leader) + rank;
    if (act) j.out[pos] = i;
  }
  if (tid == 0 && j.nonzero) *j.nonzero = *nz_total;
}

// desc[k] = {work[k], ptr[work[k]], ptr[work[k] + 1] - ptr[work[k]], w} for the row list
// (k < rows, w = the row's first run) and then the column list (w = 0); gt / nt: this
// thread's index in the grid and the number of threads.
__device__ void desc_step(const int32_t* __restrict__ row_work, const int32_t* __restrict__ row_ptr,
                          const int32_t* __restrict__ run_ptr, int rows, int4* __restrict__ row_desc,
                          const int32_t* __restrict__ col_work, const int32_t* __restrict__ col_ptr,
                          int cols, int4* __restrict__ col_desc, int gt, int nt) {
  for (int k = gt; k < rows + cols; k += nt) {
    const bool is_row = k < rows;
    const int kk = is_row ? k : k - rows;
    const int r = (is_row ? row_work : col_work)[kk];
    const int32_t* ptr = is_row ? row_ptr : col_ptr;
    const int a = ptr[r];
    (is_row ? row_desc : col_desc)[kk] = make_int4(r, a, ptr[r + 1] - a, is_row ? run_ptr[r] : 0);
  }
}

// One warp per q-tile row: CSR entries in ascending kt, the PARTIAL numbering, the dense
// entry index of every listed block, the block of every PARTIAL number, and the row's runs
// {first k-tile, number of tiles, kind, first CSR entry} at run[run_ptr[r] ..).
__device__ void fill_csr_step(const uint8_t* __restrict__ kinds, int rows, int KT,
                              const int32_t* __restrict__ row_ptr,
                              const int32_t* __restrict__ row_poff, int32_t* __restrict__ col_idx,
                              uint8_t* __restrict__ kind, int32_t* __restrict__ pidx,
                              int32_t* __restrict__ eidx, int64_t* __restrict__ ptile,
                              const int32_t* __restrict__ run_ptr, int4* __restrict__ run, int gw,
                              int nw) {
  const int lane = threadIdx.x & 31;
  const unsigned lt = (1u << lane) - 1u;
  for (int r = gw; r < rows; r += nw) {
    int e = row_ptr[r];
    int p = row_poff[r];
    int rpos = run_ptr[r];
    const uint8_t* k = kinds + static_cast<int64_t>(r) * KT;
    for (int base = 0; base < KT; base += 32) {
      const int kt = base + lane;
      const uint8_t v = kt < KT ? k[kt] : 0;
      const bool start = kt < KT && starts_run(k, kt, v);
      const unsigned sm = __ballot_sync(0xFFFFFFFFu, start);
      const unsigned nzm = __ballot_sync(0xFFFFFFFFu, v != 0);
      const unsigned pm = __ballot_sync(0xFFFFFFFFu, v == 2);
      if (start) run[rpos + __popc(sm & lt)] = make_int4(kt, 0, v, e + __popc(nzm & lt));
      rpos += __popc(sm);
      if (v != 0) {
        const int my = e + __popc(nzm & lt);
        col_idx[my] = kt;
        kind[my] = v;
        eidx[static_cast<int64_t>(r) * KT + kt] = my;
        if (v == 2) {
          const int mp = p + __popc(pm & lt);
          pidx[my] = mp;
          ptile[mp] = static_cast<int64_t>(r) * KT + kt;
        } else {
          pidx[my] = -1;
        }
      }
      e += __popc(nzm);
      p += __popc(pm);
    }
    __syncwarp();
    // length = first entry of the next run (or the row's end) minus the run's first entry
    const int a = run_ptr[r], b = run_ptr[r + 1], end = row_ptr[r + 1];
    for (int j = a + lane; j < b; j += 32) {
      const int next = j + 1 < b ? run[j + 1].w : end;
      run[j].y = next - run[j].w;
    }
    __syncwarp();
  }
}

// One warp per k-tile column: CSC entries in ascending qt with their CSR index.
__device__ void fill_csc_step(const uint8_t* __restrict__ kinds, const int32_t* __restrict__ eidx,
                              int B, int QT, int KT, const int32_t* __restrict__ colT_ptr,
                              int32_t* __restrict__ rowT_idx, int32_t* __restrict__ csc_map, int gw,
                              int nw) {
  const int lane = threadIdx.x & 31;
  for (int c = gw; c < B * KT; c += nw) {
    const int b = c / KT, kt = c % KT;
    int e = colT_ptr[c];
    for (int base = 0; base < QT; base += 32) {
      const int qt = base + lane;
      const int64_t g = (static_cast<int64_t>(b) * QT + qt) * KT + kt;
      const uint8_t v = qt < QT ? kinds[g] : 0;
      const unsigned nzm = __ballot_sync(0xFFFFFFFFu, v != 0);
      if (v != 0) {
        const int my = e + __popc(nzm & ((1u << lane) - 1u));
        rowT_idx[my] = qt;
        csc_map[my] = eidx[g];
      }
      e += __popc(nzm);
    }
  }
}

// The element mask a plan is built from.
struct MaskSrc {
  const uint8_t* mask;
  int Nq, Nk;
  int64_t sb, sq;
};

// The per-sequence lengths a plan is built from (padded rows of Npad).
struct LengthSrc {
  const int32_t* lengths;
  int Npad;
};

// Transpose of a 32 x 32 bit matrix held one row per lane (bit c of lane r's word = entry
// (r, c)): returns column `lane` (bit r = entry (r, lane)).  Five steps, each exchanging the
// off-diagonal halves of ever smaller blocks between lanes lane and lane ^ j.
__device__ __forceinline__ uint32_t transpose32(uint32_t x, int lane) {
  constexpr uint32_t kLow[5] = {0x0000FFFFu, 0x00FF00FFu, 0x0F0F0F0Fu, 0x33333333u, 0x55555555u};
#pragma unroll
  for (int r = 0; r < 5; ++r) {
    const int j = 16 >> r;
    const uint32_t m = kLow[r];  // bits c with (c & j) == 0
    const uint32_t y = __shfl_xor_sync(0xFFFFFFFFu, x, j);
    x = (lane & j) ? ((x & ~m) | ((y & ~m) >> j)) : ((x & m) | ((y & m) << j));
  }
  return x;
}

// The bitmasks of the n PARTIAL blocks (ptile: block of each PARTIAL number) from the mask:
// groups of 128 threads, one block each, thread q reading row q (128 bytes, eight loads in
// flight).  The transposed copy (bit (q % 32) of word (k*4 + q/32) = column k of row q)
// comes from 32 x 32 transposes in registers: warp j of a group holds rows 32j .. 32j + 31,
// and the transpose of its words c gives word (32c + lane)*4 + j.
__device__ void bits_step(const MaskSrc& s, int QT, int KT, const int64_t* __restrict__ ptile,
                          int64_t n, uint32_t* __restrict__ bits, uint32_t* __restrict__ bitsT,
                          uint32_t*) {
  const int groups = blockDim.x / kTile, grp = threadIdx.x / kTile, q = threadIdx.x % kTile;
  const int lane = threadIdx.x & 31, j = q >> 5;
  for (int64_t pb = static_cast<int64_t>(blockIdx.x) * groups + grp; pb < n;
       pb += static_cast<int64_t>(gridDim.x) * groups) {
    const int64_t g = ptile[pb];
    const int kt = static_cast<int>(g % KT);
    const int qt = static_cast<int>((g / KT) % QT);
    const int b = static_cast<int>(g / (static_cast<int64_t>(KT) * QT));
    uint32_t w[4];
    row_bits(s.mask, s.Nq, s.Nk, s.sb, s.sq, b, qt * kTile + q, kt * kTile, w);
    reinterpret_cast<uint4*>(bits + pb * 512)[q] = make_uint4(w[0], w[1], w[2], w[3]);
    uint32_t* dt = bitsT + pb * 512 + j;
#pragma unroll
    for (int c = 0; c < 4; ++c) dt[(32 * c + lane) * 4] = transpose32(w[c], lane);
  }
}

// The same from the lengths: row q of a PARTIAL block is valid iff qt*128 + q < n, column
// k iff kt*128 + k < n.  One thread per (block, q): row q of the bitmask and (the same rule
// with the roles swapped) column q of the transposed copy.
__device__ void bits_step(const LengthSrc& s, int QT, int KT, const int64_t* __restrict__ ptile,
                          int64_t n, uint32_t* __restrict__ bits, uint32_t* __restrict__ bitsT,
                          uint32_t*) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n * 128;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t pb = i >> 7;
    const int q = static_cast<int>(i & 127);
    const int64_t g = ptile[pb];
    const int kt = static_cast<int>(g % KT);
    const int qt = static_cast<int>((g / KT) % QT);
    const int b = static_cast<int>(g / (static_cast<int64_t>(KT) * QT));
    const int len = min(max(s.lengths[b], 0), s.Npad);
    const bool row_ok = qt * kTile + q < len;
    uint4 w;
    w.x = row_ok ? low_bits(len - (kt * kTile + 0)) : 0u;
    w.y = row_ok ? low_bits(len - (kt * kTile + 32)) : 0u;
    w.z = row_ok ? low_bits(len - (kt * kTile + 64)) : 0u;
    w.w = row_ok ? low_bits(len - (kt * kTile + 96)) : 0u;
    reinterpret_cast<uint4*>(bits + pb * 512)[q] = w;
    const bool col_ok = kt * kTile + q < len;
    uint4 wt;
    wt.x = col_ok ? low_bits(len - (qt * kTile + 0)) : 0u;
    wt.y = col_ok ? low_bits(len - (qt * kTile + 32)) : 0u;
    wt.z = col_ok ? low_bits(len - (qt * kTile + 64)) : 0u;
    wt.w = col_ok ? low_bits(len - (qt * kTile + 96)) : 0u;
    reinterpret_cast<uint4*>(bitsT + pb * 512)[q] = wt;
  }
}

// Limit of one grid-barrier wait.  Every CTA of a cooperative launch is resident, so the
// wait ends unless the device is gone; past the limit the plan's timeout flag and the
// device status word record it and the CTA goes on (the plan's counts then report
// SIGATTN_ERR_TIMEOUT, and so does sigattn_get_status).
constexpr unsigned long long kPlanBarrierNs = 2000000000ull;

__device__ __forceinline__ unsigned long long plan_clock_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Grid-wide barrier on a monotonic arrival counter: the k-th barrier of a launch ends when
// k * gridDim.x arrivals are counted.  Thread 0 of each CTA arrives (after a fence that
// publishes the CTA's writes) and waits; the CTA barriers around it order the other threads.
__device__ void grid_barrier(unsigned* arrive, unsigned target, int64_t* timeout, int* status) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(arrive, 1u);
    const unsigned long long t0 = plan_clock_ns();
    while (ld_acquire(arrive) < target) {
      if (plan_clock_ns() - t0 > kPlanBarrierNs) {
        atomicOr(reinterpret_cast<unsigned long long*>(timeout), 1ull);
        atomicOr(status, kStatusTimeout);
        break;
      }
      __nanosleep(32);
    }
    __threadfence();
  }
  __syncthreads();
}

// Everything the steps after the classification read and write.
struct StepArgs {
  const uint8_t* kinds;
  int B, QT, KT;
  int32_t *row_cnt, *row_pcnt, *run_cnt, *col_cnt, *row_poff, *eidx;
  int64_t* totals;  // the plan's device counts (kCountSlots entries)
  int* status;      // the device status word
  int64_t* ptile;
  int32_t *row_ptr, *colT_ptr, *run_ptr, *row_work, *col_work;
  int4 *row_desc, *col_desc;
  int32_t *col_idx, *pidx, *rowT_idx, *csc_map;
  uint8_t* kind;
  int4* run;
  uint32_t *bits, *bitsT;
  int first, last;  // the phases this launch runs (0..3)
  int desc, fill;   // phase 2: write the work descriptors / fill CSR
  int launch;       // 0 or 1: which arrival counter the barriers use
};

constexpr int kStepThreads = 1024;

template <class Src>
__global__ void __launch_bounds__(kStepThreads, 1) k_plan_steps(StepArgs a, Src src) {
  __shared__ int32_t sh[kSortBuckets + 64];
  int32_t* warp_sums = sh + kSortBuckets;
  int32_t* scalar = sh + kSortBuckets + 32;
  const int gt = blockIdx.x * blockDim.x + threadIdx.x, nt = gridDim.x * blockDim.x;
  const int gw = gt >> 5, nw = nt >> 5;
  const int rows = a.B * a.QT, cols = a.B * a.KT;
  unsigned* arrive = reinterpret_cast<unsigned*>(a.totals + kCountArrive) + a.launch;
  unsigned passed = 0;
  for (int ph = a.first; ph <= a.last; ++ph) {
    if (ph > a.first) grid_barrier(arrive, ++passed * gridDim.x, a.totals + kCountTimeout, a.status);
    if (ph == 0) {
      count_step(a.kinds, a.B, a.QT, a.KT, a.row_cnt, a.row_pcnt, a.run_cnt, a.col_cnt, gw, nw);
    } else if (ph == 1) {
      for (int job = blockIdx.x; job < 6; job += gridDim.x) {
        __syncthreads();
        switch (job) {
          case 0: scan_job(ScanJob{a.row_cnt, rows, a.row_ptr, a.totals + kCountListed}, warp_sums, scalar); break;
          case 1: scan_job(ScanJob{a.row_pcnt, rows, a.row_poff, a.totals + kCountPartial}, warp_sums, scalar); break;
          case 2: scan_job(ScanJob{a.col_cnt, cols, a.colT_ptr, nullptr}, warp_sums, scalar); break;
          case 3: scan_job(ScanJob{a.run_cnt, rows, a.run_ptr, nullptr}, warp_sums, scalar); break;
          case 4: sort_job(SortJob{a.row_cnt, rows, a.row_work, a.totals + kCountRows}, sh, warp_sums, scalar); break;
          default: sort_job(SortJob{a.col_cnt, cols, a.col_work, a.totals + kCountCols}, sh, warp_sums, scalar); break;
        }
      }
    } else if (ph == 2) {
      if (a.desc)
        desc_step(a.row_work, a.row_ptr, a.run_ptr, rows, a.row_desc, a.col_work, a.colT_ptr, cols,
                  a.col_desc, gt, nt);
      if (a.fill)
        fill_csr_step(a.kinds, rows, a.KT, a.row_ptr, a.row_poff, a.col_idx, a.kind, a.pidx, a.eidx,
                      a.ptile, a.run_ptr, a.run, nw - 1 - gw, nw);
    } else {
      fill_csc_step(a.kinds, a.eidx, a.B, a.QT, a.KT, a.colT_ptr, a.rowT_idx, a.csc_map,
                    nw - 1 - gw, nw);
      const int64_t np = *reinterpret_cast<volatile int64_t*>(a.totals + kCountPartial);
      bits_step(src, a.QT, a.KT, a.ptile, np, a.bits, a.bitsT, reinterpret_cast<uint32_t*>(sh));
    }
  }
}

// Buffers are carved out of a few large allocations: a byte count laid out first (every
// buffer 256-byte aligned), then one allocation, then the pointers.
struct Carve {
  size_t bytes = 0;
  template <class T>
  size_t add(size_t count) {
    bytes = (bytes + 255) & ~size_t(255);
    const size_t at = bytes;
    bytes += count * sizeof(T);
    return at;
  }
  template <class T>
  static T* at(void* base, size_t off) {
    return reinterpret_cast<T*>(static_cast<uint8_t*>(base) + off);
  }
};

int alloc_status(cudaError_t e) {
  if (e == cudaSuccess) return SIGATTN_OK;
  cudaGetLastError();
  return e == cudaErrorMemoryAllocation ? SIGATTN_ERR_NOMEM : SIGATTN_ERR_CUDA;
}

// All plan memory (the plan's arenas and the scratch of a build) comes from one memory pool
// per device that keeps what it has reserved (release threshold: never), so that building a
// plan after the first allocates nothing from the driver, and no allocation or free stalls
// the device: allocations and frees are ordered on streams.
std::mutex g_pool_mu;
cudaMemPool_t g_pool[kMaxDevices] = {};

int plan_pool(int dev, cudaMemPool_t* out) {
  if (dev < 0 || dev >= kMaxDevices) return SIGATTN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_pool_mu);
  if (!g_pool[dev]) {
    cudaMemPoolProps props = {};
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaMemPool_t pool = nullptr;
    cudaError_t e = cudaMemPoolCreate(&pool, &props);
    if (e != cudaSuccess) return alloc_status(e);
    uint64_t keep = UINT64_MAX;
    e = cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
    if (e != cudaSuccess) {
      cudaMemPoolDestroy(pool);
      return alloc_status(e);
    }
    g_pool[dev] = pool;
  }
  *out = g_pool[dev];
  return SIGATTN_OK;
}

int pool_alloc(void** p, size_t bytes, cudaStream_t s) {
  *p = nullptr;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return SIGATTN_ERR_NO_DEVICE;
  }
  cudaMemPool_t pool = nullptr;
  const int rc = plan_pool(dev, &pool);
  if (rc != SIGATTN_OK) return rc;
  return alloc_status(cudaMallocFromPoolAsync(p, bytes > 0 ? bytes : 256, pool, s));
}

// Plan memory (owned by the plan until sigattn_plan_destroy).
int plan_alloc(void** p, size_t bytes, cudaStream_t s) { return pool_alloc(p, bytes, s); }

// Scratch of one plan build, released on the stream at the end.
int scratch_alloc(void** p, size_t bytes, cudaStream_t s) { return pool_alloc(p, bytes, s); }

struct Scratch {
  void* block[2] = {nullptr, nullptr};
  uint8_t* kinds = nullptr;
  int32_t* eidx = nullptr;
  int32_t* row_cnt = nullptr;
  int32_t* row_pcnt = nullptr;
  int32_t* row_poff = nullptr;
  int32_t* col_cnt = nullptr;
  int32_t* run_cnt = nullptr;
  int64_t* ptile = nullptr;
  void release(cudaStream_t s) {
    for (void*& p : block) {
      if (p) cudaFreeAsync(p, s);
      p = nullptr;
    }
  }
};

// The arenas go back to the pool in the order of the legacy default stream, after the
// plan's build (the caller has made sure that no other kernel still uses the plan).
void plan_free_buffers(sigattn_plan* p) {
  if (p->ready && !p->counts_known) cudaStreamWaitEvent(cudaStreamLegacy, p->ready, 0);
  for (void*& a : p->arena) {
    if (a) cudaFreeAsync(a, cudaStreamLegacy);
    a = nullptr;
  }
  if (p->ready) cudaEventDestroy(p->ready);
  p->ready = nullptr;
}

// On failure: kernels of the build may already be queued on `stream` (which need not be
// ordered with the legacy stream the plan's memory is freed on), so wait for it first.
#define SIGATTN_TRY(x)                 \
  do {                                 \
    const int rc_ = (x);               \
    if (rc_ != SIGATTN_OK) {           \
      cudaStreamSynchronize(stream);   \
      cudaGetLastError();              \
      sc.release(stream);              \
      plan_free_buffers(plan);         \
      delete plan;                     \
      return rc_;                      \
    }                                  \
  } while (0)

#define SIGATTN_TRY_CUDA(x) SIGATTN_TRY(cuda_status(x))

int grid_for(int64_t work, int per_block) {
  const int64_t g = (work + per_block - 1) / per_block;
  return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(g, 1 << 30)));
}

// Plan memory for the tile lists: nz listed tiles, np of them PARTIAL.
struct TileArena {
  size_t ci, k, pi, ri, cm, b, bt, run, bytes;
  TileArena(size_t nz, size_t np) {
    Carve c;
    ci = c.add<int32_t>(nz);
    k = c.add<uint8_t>(nz);
    pi = c.add<int32_t>(nz);
    ri = c.add<int32_t>(nz);
    cm = c.add<int32_t>(nz);
    b = c.add<uint32_t>(np * 512);
    bt = c.add<uint32_t>(np * 512);
    run = c.add<int4>(nz);  // at most one run per listed tile
    bytes = c.bytes;
  }
  void place(sigattn_plan* plan, void* m) const {
    plan->col_idx = Carve::at<int32_t>(m, ci);
    plan->kind = Carve::at<uint8_t>(m, k);
    plan->pidx = Carve::at<int32_t>(m, pi);
    plan->rowT_idx = Carve::at<int32_t>(m, ri);
    plan->csc_map = Carve::at<int32_t>(m, cm);
    plan->bits = Carve::at<uint32_t>(m, b);
    plan->bitsT = Carve::at<uint32_t>(m, bt);
    plan->run = Carve::at<int4>(m, run);
  }
};

// Tile arrays sized for the worst case up to this many bytes, so that the whole plan is
// queued before the one synchronisation; above it the counts are read back first.
constexpr size_t kOnePassBytes = size_t(256) << 20;

// CTAs of the cooperative launch per device: one per SM when the steps kernel fits one per
// SM (checked once per device), else 0 (the build reports SIGATTN_ERR_UNSUPPORTED).
std::mutex g_steps_mu;
int g_steps_grid[kMaxDevices] = {};
bool g_steps_known[kMaxDevices] = {};

int steps_grid(int dev, int* grid) {
  if (dev < 0 || dev >= kMaxDevices) return SIGATTN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_steps_mu);
  if (!g_steps_known[dev]) {
    int sms = 0, coop = 0, per_sm = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_plan_steps<MaskSrc>, kStepThreads,
                                                      0) != cudaSuccess) {
      cudaGetLastError();
      return SIGATTN_ERR_CUDA;
    }
    int per_sm2 = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm2, k_plan_steps<LengthSrc>,
                                                      kStepThreads, 0) != cudaSuccess) {
      cudaGetLastError();
      return SIGATTN_ERR_CUDA;
    }
    g_steps_grid[dev] = (coop && per_sm >= 1 && per_sm2 >= 1) ? sms : 0;
    g_steps_known[dev] = true;
  }
  *grid = g_steps_grid[dev];
  return *grid > 0 ? SIGATTN_OK : SIGATTN_ERR_UNSUPPORTED;
}

template <class Src>
int launch_steps(const StepArgs& a, const Src& src, int grid, cudaStream_t stream) {
  StepArgs a_ = a;
  Src s_ = src;
  void* args[] = {&a_, &s_};
  return cuda_status(cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(k_plan_steps<Src>),
                                                 dim3(grid), dim3(kStepThreads), args, 0, stream));
}

// Both planners: `classify` writes every block's kind into sc.kinds (and zeroes the two
// barrier words it is given); `src` is the mask or the lengths the PARTIAL blocks' bitmasks
// come from.  np_bound: most PARTIAL blocks the classification can yield (the grid for a
// mask; two tile strips per sequence for lengths).  When the tile arrays sized for the grid
// and np_bound fit kOnePassBytes, the classification and one cooperative launch of every
// later step are queued, and the call returns without waiting (the counts stay on the
// device until plan_counts) unless there is a host check to make: packed batches then
// synchronise once at the end.  Otherwise the launch stops after the counts and the work
// lists, the host reads the counts, sizes the arrays exactly, and a second launch fills
// them.  cu_src (packed batches only): the cumulative offsets, copied into the plan;
// check_dev / check_host: one device int read back at the synchronisation (an argument
// check).
template <class ClassifyFn, class Src>
int build_plan(sigattn_plan* plan, cudaStream_t stream, ClassifyFn classify, const Src& src,
               sigattn_plan** out, int64_t np_bound, const int32_t* cu_src = nullptr,
               const int32_t* check_dev = nullptr, int32_t* check_host = nullptr) {
  Scratch sc;
  const int B = plan->B, QT = plan->QT, KT = plan->KT;
  const int rows = B * QT, cols = B * KT;
  const int64_t grid_total = static_cast<int64_t>(rows) * KT;
  int grid = 0;
  SIGATTN_TRY(steps_grid(plan->device, &grid));
  int* status = nullptr;
  SIGATTN_TRY(status_ptr(&status));
  const int64_t np_max = std::min<int64_t>(grid_total, np_bound);
  const TileArena worst(static_cast<size_t>(grid_total), static_cast<size_t>(np_max));
  const bool one_pass = worst.bytes <= kOnePassBytes;
  // Layouts: the build's scratch (cs), the plan's lists and counts (ca), the tile arrays.
  // One-pass plans take all three from one allocation (the scratch then stays with the plan:
  // 5 bytes per block of the grid, 8 per possible PARTIAL block), so that the
  // classification is launched after a single allocation; two-pass ones free the scratch.
  Carve cs;
  const size_t o_kinds = cs.add<uint8_t>(grid_total), o_eidx = cs.add<int32_t>(grid_total),
               o_rc = cs.add<int32_t>(rows), o_rpc = cs.add<int32_t>(rows),
               o_ro = cs.add<int32_t>(rows + 1), o_cc = cs.add<int32_t>(cols),
               o_run = cs.add<int32_t>(rows),
               o_pt = cs.add<int64_t>(one_pass ? std::max<int64_t>(np_max, 1) : 0);
  Carve ca;
  const size_t o_rptr = ca.add<int32_t>(rows + 1), o_cptr = ca.add<int32_t>(cols + 1),
               o_rw = ca.add<int32_t>(rows), o_cw = ca.add<int32_t>(cols),
               o_rd = ca.add<int4>(rows), o_cd = ca.add<int4>(cols),
               o_rp = ca.add<int32_t>(rows + 1), o_cu = ca.add<int32_t>(cu_src ? B + 1 : 0),
               o_cnt = ca.add<int64_t>(kCountSlots);
  const size_t a_bytes = (ca.bytes + 255) & ~size_t(255);
  const size_t t_bytes = (worst.bytes + 255) & ~size_t(255);
  void* ms = nullptr;  // scratch base
  void* m = nullptr;   // lists and counts base
  if (one_pass) {
    SIGATTN_TRY(plan_alloc(&plan->arena[0], a_bytes + t_bytes + cs.bytes, stream));
    m = plan->arena[0];
    worst.place(plan, static_cast<uint8_t*>(m) + a_bytes);
    ms = static_cast<uint8_t*>(m) + a_bytes + t_bytes;
  } else {
    SIGATTN_TRY(scratch_alloc(&sc.block[0], cs.bytes, stream));
    SIGATTN_TRY(plan_alloc(&plan->arena[0], ca.bytes, stream));
    ms = sc.block[0];
    m = plan->arena[0];
  }
  sc.kinds = Carve::at<uint8_t>(ms, o_kinds);
  sc.eidx = Carve::at<int32_t>(ms, o_eidx);
  sc.row_cnt = Carve::at<int32_t>(ms, o_rc);
  sc.row_pcnt = Carve::at<int32_t>(ms, o_rpc);
  sc.row_poff = Carve::at<int32_t>(ms, o_ro);
  sc.col_cnt = Carve::at<int32_t>(ms, o_cc);
  sc.run_cnt = Carve::at<int32_t>(ms, o_run);
  sc.ptile = one_pass ? Carve::at<int64_t>(ms, o_pt) : nullptr;
  plan->dcount = Carve::at<int64_t>(m, o_cnt);
  plan->row_ptr = Carve::at<int32_t>(m, o_rptr);
  plan->colT_ptr = Carve::at<int32_t>(m, o_cptr);
  plan->row_work = Carve::at<int32_t>(m, o_rw);
  plan->col_work = Carve::at<int32_t>(m, o_cw);
  plan->row_desc = Carve::at<int4>(m, o_rd);
  plan->col_desc = Carve::at<int4>(m, o_cd);
  plan->run_ptr = Carve::at<int32_t>(m, o_rp);
  classify(sc.kinds, plan->dcount + kCountTimeout);
  SIGATTN_TRY_CUDA(cudaGetLastError());
  if (cu_src) {
    plan->cu = Carve::at<int32_t>(m, o_cu);
    SIGATTN_TRY_CUDA(cudaMemcpyAsync(plan->cu, cu_src, (B + 1) * sizeof(int32_t),
                                     cudaMemcpyDeviceToDevice, stream));
  }
  auto args = [&]() {
    StepArgs a;
    a.kinds = sc.kinds;
    a.B = B;
    a.QT = QT;
    a.KT = KT;
    a.row_cnt = sc.row_cnt;
    a.row_pcnt = sc.row_pcnt;
    a.run_cnt = sc.run_cnt;
    a.col_cnt = sc.col_cnt;
    a.row_poff = sc.row_poff;
    a.eidx = sc.eidx;
    a.totals = plan->dcount;
    a.status = status;
    a.ptile = sc.ptile;
    a.row_ptr = plan->row_ptr;
    a.colT_ptr = plan->colT_ptr;
    a.run_ptr = plan->run_ptr;
    a.row_work = plan->row_work;
    a.col_work = plan->col_work;
    a.row_desc = plan->row_desc;
    a.col_desc = plan->col_desc;
    a.col_idx = plan->col_idx;
    a.pidx = plan->pidx;
    a.rowT_idx = plan->rowT_idx;
    a.csc_map = plan->csc_map;
    a.kind = plan->kind;
    a.run = plan->run;
    a.bits = plan->bits;
    a.bitsT = plan->bitsT;
    a.first = 0;
    a.last = 3;
    a.desc = 1;
    a.fill = 1;
    a.launch = 0;
    return a;
  };
  {
    StepArgs a = args();
    if (!one_pass) a.last = 2, a.fill = 0;
    SIGATTN_TRY(launch_steps(a, src, grid, stream));
  }
  // one entry past the listed tiles stays readable: kernels bound their reads by it
  plan->run_cap = one_pass ? grid_total : 0;
  if (one_pass && !cu_src && !check_dev) {
    // nothing to check on the host: the counts stay on the device until first asked for
    SIGATTN_TRY_CUDA(cudaEventCreateWithFlags(&plan->ready, cudaEventDisableTiming));
    SIGATTN_TRY_CUDA(cudaEventRecord(plan->ready, stream));
    sc.release(stream);
    *out = plan;
    return SIGATTN_OK;
  }
  int64_t totals[kCountSlots] = {};
  int32_t last_row = 0;
  auto read_back = [&]() -> int {
    int rc = cuda_status(cudaMemcpyAsync(totals, plan->dcount, sizeof(totals),
                                         cudaMemcpyDeviceToHost, stream));
    if (rc == SIGATTN_OK) rc = cuda_status(cudaStreamSynchronize(stream));
    if (rc == SIGATTN_OK && totals[kCountTimeout] != 0) rc = SIGATTN_ERR_TIMEOUT;
    return rc;
  };
  if (cu_src)
    SIGATTN_TRY_CUDA(cudaMemcpyAsync(&last_row, cu_src + B, sizeof(int32_t), cudaMemcpyDeviceToHost,
                                     stream));
  if (check_dev)
    SIGATTN_TRY_CUDA(cudaMemcpyAsync(check_host, check_dev, sizeof(int32_t), cudaMemcpyDeviceToHost,
                                     stream));
  SIGATTN_TRY(read_back());
  if (check_host && *check_host != 0) SIGATTN_TRY(SIGATTN_ERR_INVALID);
  if (cu_src && last_row < 1) SIGATTN_TRY(SIGATTN_ERR_INVALID);  // a packed batch needs rows
  plan->T = last_row;
  plan->nonempty = totals[kCountListed];
  plan->partial = totals[kCountPartial];
  plan->full = totals[kCountListed] - totals[kCountPartial];
  plan->rows_nonempty = static_cast<int32_t>(totals[kCountRows]);
  plan->cols_nonempty = static_cast<int32_t>(totals[kCountCols]);
  plan->counts_known = true;
  if (!one_pass) {
    const TileArena exact(static_cast<size_t>(plan->nonempty), static_cast<size_t>(plan->partial));
    SIGATTN_TRY(plan_alloc(&plan->arena[1], exact.bytes, stream));
    exact.place(plan, plan->arena[1]);
    SIGATTN_TRY(scratch_alloc(&sc.block[1],
                              std::max<int64_t>(plan->partial, 1) * sizeof(int64_t), stream));
    sc.ptile = static_cast<int64_t*>(sc.block[1]);
    StepArgs a = args();
    a.first = 2;
    a.desc = 0;
    a.launch = 1;
    SIGATTN_TRY(launch_steps(a, src, grid, stream));
    SIGATTN_TRY(read_back());
    plan->run_cap = plan->nonempty;
  }
  sc.release(stream);
  *out = plan;
  return SIGATTN_OK;
}

}  // namespace

namespace {
// Serialises the first read of a plan's counts between host threads that share the plan.
std::mutex g_counts_mu;
}  // namespace

int plan_counts(sigattn_plan* plan) {
  std::lock_guard<std::mutex> lock(g_counts_mu);
  if (plan->counts_known) return SIGATTN_OK;
  int64_t c[kCountSlots] = {};
  int rc = cuda_status(cudaEventSynchronize(plan->ready));
  if (rc == SIGATTN_OK)
    rc = cuda_status(cudaMemcpy(c, plan->dcount, sizeof(c), cudaMemcpyDeviceToHost));
  if (rc != SIGATTN_OK) return rc;
  if (c[kCountTimeout] != 0) return SIGATTN_ERR_TIMEOUT;
  plan->nonempty = c[kCountListed];
  plan->partial = c[kCountPartial];
  plan->full = c[kCountListed] - c[kCountPartial];
  plan->rows_nonempty = static_cast<int32_t>(c[kCountRows]);
  plan->cols_nonempty = static_cast<int32_t>(c[kCountCols]);
  plan->counts_known = true;
  return SIGATTN_OK;
}

int plan_wait(const sigattn_plan* plan, cudaStream_t stream) {
  if (!plan->ready || plan->counts_known) return SIGATTN_OK;
  // inside a stream capture the wait becomes an external-event node of the graph (the
  // build's event was recorded outside the capture)
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  int rc = cuda_status(cudaStreamIsCapturing(stream, &cs));
  if (rc != SIGATTN_OK) return rc;
  return cuda_status(cudaStreamWaitEvent(
      stream, plan->ready,
      cs == cudaStreamCaptureStatusActive ? cudaEventWaitExternal : cudaEventWaitDefault));
}

namespace {

int current_device(int* dev) {
  if (cudaGetDevice(dev) != cudaSuccess) {
    cudaGetLastError();
    return SIGATTN_ERR_NO_DEVICE;
  }
  return SIGATTN_OK;
}

constexpr int64_t kMaxGrid = int64_t(1) << 28;

}  // namespace
}  // namespace sigattn

using namespace sigattn;

extern "C" int sigattn_plan_from_lengths(const int32_t* d_lengths, int B, int Npad,
                                         sigattn_stream s, sigattn_plan** out) {
  if (!out) return SIGATTN_ERR_INVALID;
  *out = nullptr;
  if (!d_lengths || B < 1 || Npad < 1) return SIGATTN_ERR_INVALID;
  const int QT = (Npad + kTile - 1) / kTile;
  if (static_cast<int64_t>(B) * QT * QT > kMaxGrid) return SIGATTN_ERR_UNSUPPORTED;
  cudaStream_t stream = static_cast<cudaStream_t>(s);
  sigattn_plan* plan = new sigattn_plan();
  std::memset(plan, 0, sizeof(*plan));
  Scratch sc;
  SIGATTN_TRY(current_device(&plan->device));
  plan->B = B;
  plan->Nq = plan->Nk = Npad;
  plan->QT = plan->KT = QT;
  const int64_t grid_total = static_cast<int64_t>(B) * QT * QT;
  auto classify = [&](uint8_t* kinds, int64_t* zero2) {
    k_kinds_from_lengths<<<grid_for(grid_total, 256), 256, 0, stream>>>(d_lengths, B, Npad, QT,
                                                                          QT, kinds, zero2);
  };
  // PARTIAL blocks of a length: the last q-tile row and k-tile column of the sequence
  return build_plan(plan, stream, classify, LengthSrc{d_lengths, Npad}, out,
                    2 * static_cast<int64_t>(B) * QT);
}

namespace sigattn {
namespace {

// lengths[b] = cu[b+1] - cu[b]; *bad = 1 if a length is negative or above maxlen.
__global__ void k_lengths_from_cu(const int32_t* __restrict__ cu, int B, int maxlen,
                                  int32_t* __restrict__ lengths, int32_t* __restrict__ bad) {
  for (int b = blockIdx.x * blockDim.x + threadIdx.x; b < B; b += gridDim.x * blockDim.x) {
    const int n = cu[b + 1] - cu[b];
    lengths[b] = n;
    if (n < 0 || n > maxlen) atomicOr(bad, 1);
  }
}

}  // namespace
}  // namespace sigattn

extern "C" int sigattn_plan_from_cu_seqlens(const int32_t* d_cu, int B, int max_seqlen,
                                            sigattn_stream s, sigattn_plan** out) {
  if (!out) return SIGATTN_ERR_INVALID;
  *out = nullptr;
  if (!d_cu || B < 1 || max_seqlen < 1) return SIGATTN_ERR_INVALID;
  const int QT = (max_seqlen + kTile - 1) / kTile;
  if (static_cast<int64_t>(B) * QT * QT > kMaxGrid) return SIGATTN_ERR_UNSUPPORTED;
  cudaStream_t stream = static_cast<cudaStream_t>(s);
  // lengths and the argument check live in a scratch block of their own, released at the end
  void* tmp = nullptr;
  int rc = scratch_alloc(&tmp, static_cast<size_t>(B + 1) * sizeof(int32_t) + 256, stream);
  if (rc != SIGATTN_OK) return rc;
  int32_t* lengths = static_cast<int32_t*>(tmp);
  int32_t* bad = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(tmp) +
                                            ((static_cast<size_t>(B) * 4 + 255) & ~size_t(255)));
  cudaMemsetAsync(bad, 0, sizeof(int32_t), stream);
  k_lengths_from_cu<<<grid_for(B, 256), 256, 0, stream>>>(d_cu, B, max_seqlen, lengths, bad);
  sigattn_plan* plan = new sigattn_plan();
  std::memset(plan, 0, sizeof(*plan));
  rc = current_device(&plan->device);
  if (rc != SIGATTN_OK) {
    delete plan;
    cudaFreeAsync(tmp, stream);
    return rc;
  }
  plan->B = B;
  plan->Nq = plan->Nk = max_seqlen;
  plan->QT = plan->KT = QT;
  const int64_t grid_total = static_cast<int64_t>(B) * QT * QT;
  auto classify = [&](uint8_t* kinds, int64_t* zero2) {
    k_kinds_from_lengths<<<grid_for(grid_total, 256), 256, 0, stream>>>(lengths, B, max_seqlen, QT,
                                                                          QT, kinds, zero2);
  };
  int32_t bad_host = 0;
  rc = build_plan(plan, stream, classify, LengthSrc{lengths, max_seqlen}, out,
                  2 * static_cast<int64_t>(B) * QT, d_cu, bad, &bad_host);
  cudaFreeAsync(tmp, stream);
  return rc;
}

extern "C" int sigattn_plan_from_mask(const uint8_t* d_mask, int B, int Nq, int Nk,
                                      int64_t stride_b, int64_t stride_q, sigattn_stream s,
                                      sigattn_plan** out) {
  if (!out) return SIGATTN_ERR_INVALID;
  *out = nullptr;
  if (!d_mask || B < 1 || Nq < 1 || Nk < 1 || stride_b < 0 || stride_q < 0)
    return SIGATTN_ERR_INVALID;
  const int QT = (Nq + kTile - 1) / kTile, KT = (Nk + kTile - 1) / kTile;
  if (static_cast<int64_t>(B) * QT * KT > kMaxGrid) return SIGATTN_ERR_UNSUPPORTED;
  cudaStream_t stream = static_cast<cudaStream_t>(s);
  sigattn_plan* plan = new sigattn_plan();
  std::memset(plan, 0, sizeof(*plan));
  Scratch sc;
  SIGATTN_TRY(current_device(&plan->device));
  plan->B = B;
  plan->Nq = Nq;
  plan->Nk = Nk;
  plan->QT = QT;
  plan->KT = KT;
  const int64_t grid_total = static_cast<int64_t>(B) * QT * KT;
  auto classify = [&](uint8_t* kinds, int64_t* zero2) {
    // one CTA per block
    const int64_t ctas = std::min<int64_t>(grid_total, int64_t(1) << 20);
    k_kinds_from_mask<<<static_cast<unsigned>(ctas), 256, 0, stream>>>(
        d_mask, B, Nq, Nk, stride_b, stride_q, QT, KT, kinds, zero2);
  };
  return build_plan(plan, stream, classify, MaskSrc{d_mask, Nq, Nk, stride_b, stride_q}, out,
                    grid_total);
}

extern "C" int sigattn_plan_get_sizes(const sigattn_plan* plan, sigattn_plan_sizes* sz) {
  if (!plan || !sz) return SIGATTN_ERR_INVALID;
  const int rc = plan_counts(const_cast<sigattn_plan*>(plan));
  if (rc != SIGATTN_OK) return rc;
  sz->B = plan->B;
  sz->Nq = plan->Nq;
  sz->Nk = plan->Nk;
  sz->QT = plan->QT;
  sz->KT = plan->KT;
  sz->nonempty = plan->nonempty;
  sz->full = plan->full;
  sz->partial = plan->partial;
  sz->grid_total = static_cast<int64_t>(plan->B) * plan->QT * plan->KT;
  sz->rows_nonempty = plan->rows_nonempty;
  sz->cols_nonempty = plan->cols_nonempty;
  return SIGATTN_OK;
}

extern "C" int sigattn_plan_export(const sigattn_plan* plan, int32_t* row_ptr, int32_t* col_idx,
                                   uint8_t* kind, int32_t* pidx, int32_t* colT_ptr,
                                   int32_t* rowT_idx, int32_t* csc_map, uint32_t* bits) {
  if (!plan) return SIGATTN_ERR_INVALID;
  if (cudaDeviceSynchronize() != cudaSuccess) {
    cudaGetLastError();
    return SIGATTN_ERR_CUDA;
  }
  if (const int rc = plan_counts(const_cast<sigattn_plan*>(plan)); rc != SIGATTN_OK) return rc;
  const size_t rows = static_cast<size_t>(plan->B) * plan->QT;
  const size_t cols = static_cast<size_t>(plan->B) * plan->KT;
  const size_t nz = static_cast<size_t>(plan->nonempty);
  struct Item {
    void* dst;
    const void* src;
    size_t bytes;
  } items[] = {
      {row_ptr, plan->row_ptr, (rows + 1) * 4},
      {col_idx, plan->col_idx, nz * 4},
      {kind, plan->kind, nz},
      {pidx, plan->pidx, nz * 4},
      {colT_ptr, plan->colT_ptr, (cols + 1) * 4},
      {rowT_idx, plan->rowT_idx, nz * 4},
      {csc_map, plan->csc_map, nz * 4},
      {bits, plan->bits, static_cast<size_t>(plan->partial) * 512 * 4},
  };
  for (const Item& it : items) {
    if (!it.dst || it.bytes == 0) continue;
    if (cudaMemcpy(it.dst, it.src, it.bytes, cudaMemcpyDeviceToHost) != cudaSuccess) {
      cudaGetLastError();
      return SIGATTN_ERR_CUDA;
    }
  }
  return SIGATTN_OK;
}

extern "C" int sigattn_plan_export_work(const sigattn_plan* plan, int32_t* row_work,
                                        int32_t* col_work) {
  if (!plan) return SIGATTN_ERR_INVALID;
  if (cudaDeviceSynchronize() != cudaSuccess) {
    cudaGetLastError();
    return SIGATTN_ERR_CUDA;
  }
  if (const int rc = plan_counts(const_cast<sigattn_plan*>(plan)); rc != SIGATTN_OK) return rc;
  const size_t rows = static_cast<size_t>(plan->B) * plan->QT;
  const size_t cols = static_cast<size_t>(plan->B) * plan->KT;
  if (row_work && cudaMemcpy(row_work, plan->row_work, rows * 4, cudaMemcpyDeviceToHost) != cudaSuccess) {
    cudaGetLastError();
    return SIGATTN_ERR_CUDA;
  }
  if (col_work && cudaMemcpy(col_work, plan->col_work, cols * 4, cudaMemcpyDeviceToHost) != cudaSuccess) {
    cudaGetLastError();
    return SIGATTN_ERR_CUDA;
  }
  return SIGATTN_OK;
}

extern "C" int sigattn_plan_export_runs(const sigattn_plan* plan, int32_t* run_ptr, int32_t* runs,
                                        int64_t* nruns) {
  if (!plan) return SIGATTN_ERR_INVALID;
  if (cudaDeviceSynchronize() != cudaSuccess) {
    cudaGetLastError();
    return SIGATTN_ERR_CUDA;
  }
  if (const int rc = plan_counts(const_cast<sigattn_plan*>(plan)); rc != SIGATTN_OK) return rc;
  const size_t rows = static_cast<size_t>(plan->B) * plan->QT;
  int32_t total = 0;
  if (cudaMemcpy(&total, plan->run_ptr + rows, sizeof(int32_t), cudaMemcpyDeviceToHost) !=
      cudaSuccess) {
    cudaGetLastError();
    return SIGATTN_ERR_CUDA;
  }
  if (nruns) *nruns = total;
  if (run_ptr && cudaMemcpy(run_ptr, plan->run_ptr, (rows + 1) * 4, cudaMemcpyDeviceToHost) != cudaSuccess) {
    cudaGetLastError();
    return SIGATTN_ERR_CUDA;
  }
  if (runs && total > 0 &&
      cudaMemcpy(runs, plan->run, static_cast<size_t>(total) * 16, cudaMemcpyDeviceToHost) != cudaSuccess) {
    cudaGetLastError();
    return SIGATTN_ERR_CUDA;
  }
  return SIGATTN_OK;
}

extern "C" void sigattn_plan_destroy(sigattn_plan* plan) {
  if (!plan) return;
  plan_free_buffers(plan);
  delete plan;
}
