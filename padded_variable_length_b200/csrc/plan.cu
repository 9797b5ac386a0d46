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
//   5 (after the host has sized the buffers) fill CSR, CSC and the PARTIAL bitmasks
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "internal.h"

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
                                     int KT, uint8_t* __restrict__ kinds) {
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

// Reads the 64 mask bytes of one thread's half row of a block; returns the 64 nonzero
// flags as two 32-bit words (bit c = column c of the half row).  Columns past Nk and
// rows past Nq read as zero.
__device__ __forceinline__ void half_row_bits(const uint8_t* __restrict__ mask, int Nq, int Nk,
                                              int64_t sb, int64_t sq, int b, int row, int col0,
                                              uint32_t& w0, uint32_t& w1, bool& all) {
  w0 = 0u;
  w1 = 0u;
  all = false;
  if (row >= Nq || col0 >= Nk) return;
  const uint8_t* p = mask + b * sb + row * sq + col0;
  const int nv = min(64, Nk - col0);
  if (nv == 64 && (reinterpret_cast<uintptr_t>(p) & 15u) == 0) {
    const uint4* p4 = reinterpret_cast<const uint4*>(p);
    uint32_t bits[2] = {0u, 0u};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint4 v = __ldg(p4 + c);
      const uint32_t f = flags4(nonzero_bytes(v.x)) | (flags4(nonzero_bytes(v.y)) << 4) |
                         (flags4(nonzero_bytes(v.z)) << 8) | (flags4(nonzero_bytes(v.w)) << 12);
      bits[c >> 1] |= f << ((c & 1) * 16);
    }
    w0 = bits[0];
    w1 = bits[1];
  } else {
    for (int c = 0; c < nv; ++c) {
      if (p[c] != 0) {
        if (c < 32)
          w0 |= 1u << c;
        else
          w1 |= 1u << (c - 32);
      }
    }
  }
  all = (nv == 64) && w0 == 0xFFFFFFFFu && w1 == 0xFFFFFFFFu;
}

// One CTA of 256 threads per block (b, qt, kt): thread t covers row t/2, columns
// (t%2)*64 .. +64 of the block.
// One warp per block of the grid (grid-stride): lane l reads 16 bytes at column
// 16 (l % 8) of rows l / 8, l / 8 + 4, ... -- every load instruction of the warp covers four
// whole 128-byte rows -- and the warp votes on "any element kept" and "all kept".  Rows
// past Nq and columns past Nk count as not kept.  Masks whose rows are not 16-byte aligned
// take a byte-wise path.
__global__ void __launch_bounds__(256) k_kinds_from_mask(const uint8_t* __restrict__ mask, int B,
                                                         int Nq, int Nk, int64_t sb, int64_t sq,
                                                         int QT, int KT,
                                                         uint8_t* __restrict__ kinds) {
  const int64_t total = static_cast<int64_t>(B) * QT * KT;
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const bool vec = ((reinterpret_cast<uintptr_t>(mask) | static_cast<uintptr_t>(sb) |
                     static_cast<uintptr_t>(sq)) & 15u) == 0;
  for (int64_t blk = ((static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5);
       blk < total; blk += nwarps) {
    const int kt = static_cast<int>(blk % KT);
    const int qt = static_cast<int>((blk / KT) % QT);
    const int b = static_cast<int>(blk / (static_cast<int64_t>(KT) * QT));
    const int col = kt * kTile + (lane & 7) * 16;
    const uint8_t* base = mask + b * sb + col;
    bool any = false, all = true;
    if (vec && kt * kTile + kTile <= Nk) {
#pragma unroll 8
      for (int i = 0; i < 32; ++i) {
        const int row = qt * kTile + (lane >> 3) + 4 * i;
        if (row < Nq) {
          const uint4 v = __ldg(reinterpret_cast<const uint4*>(base + row * sq));
          any |= (v.x | v.y | v.z | v.w) != 0u;
          all &= (nonzero_bytes(v.x) & nonzero_bytes(v.y) & nonzero_bytes(v.z) &
                  nonzero_bytes(v.w)) == 0x80808080u;
        } else {
          all = false;
        }
      }
    } else {
      for (int i = 0; i < 32; ++i) {
        const int row = qt * kTile + (lane >> 3) + 4 * i;
        for (int j = 0; j < 16; ++j) {
          const bool in = row < Nq && col + j < Nk;
          const bool kept = in && base[row * sq + j] != 0;
          any |= kept;
          all &= kept;
        }
      }
    }
    any = __any_sync(0xFFFFFFFFu, any);
    all = __all_sync(0xFFFFFFFFu, all);
    if (lane == 0) kinds[blk] = all ? 1 : (any ? 2 : 0);
  }
}

// One warp per q-tile row r < rows (number of listed blocks and of PARTIAL blocks), then
// one warp per k-tile column c = b*KT + kt (number of listed blocks).
// A listed block starts a run iff the block before it in the row is not listed or is of
// the other kind (runs: maximal ranges of consecutive k-tiles of one kind).
__device__ __forceinline__ bool starts_run(const uint8_t* __restrict__ k, int kt, uint8_t v) {
  return v != 0 && (kt == 0 || k[kt - 1] != v);
}

// Row r < rows: number of listed blocks, of PARTIAL blocks and of runs; then one warp per
// k-tile column c = b*KT + kt: number of listed blocks.
__global__ void k_count(const uint8_t* __restrict__ kinds, int B, int QT, int KT,
                        int32_t* __restrict__ row_cnt, int32_t* __restrict__ row_pcnt,
                        int32_t* __restrict__ run_cnt, int32_t* __restrict__ col_cnt) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int rows = B * QT;
  if (warp < rows) {
    const uint8_t* k = kinds + static_cast<int64_t>(warp) * KT;
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
      row_cnt[warp] = c;
      row_pcnt[warp] = p;
      run_cnt[warp] = n;
    }
    return;
  }
  const int col = warp - rows;
  if (col >= B * KT) return;
  const int b = col / KT, kt = col % KT;
  int c = 0;
  for (int qt = lane; qt < QT; qt += 32) c += kinds[(static_cast<int64_t>(b) * QT + qt) * KT + kt] != 0;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xFFFFFFFFu, c, o);
  if (lane == 0) col_cnt[col] = c;
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

// One CTA of 1024 threads per job (blockIdx.x picks one of four), walking its input in
// chunks of 1024.
__global__ void __launch_bounds__(1024) k_scan4(ScanJob j0, ScanJob j1, ScanJob j2, ScanJob j3) {
  __shared__ int32_t warp_sums[32];
  __shared__ int32_t chunk_total;
  const ScanJob j = blockIdx.x == 0 ? j0 : (blockIdx.x == 1 ? j1 : (blockIdx.x == 2 ? j2 : j3));
  int carry = 0;
  for (int base = 0; base < j.n; base += 1024) {
    const int i = base + threadIdx.x;
    const int x = i < j.n ? j.in[i] : 0;
    const int incl = block_inclusive_scan(x, warp_sums);
    if (i < j.n) j.out[i] = carry + incl - x;
    if (threadIdx.x == 1023) chunk_total = incl;
    __syncthreads();
    carry += chunk_total;
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

// One CTA of 1024 threads per job (blockIdx.x picks one of two).  Histogram and bucket
// offsets in shared memory; then the indices are placed in chunks of 1024 in index order:
// equal keys within a warp are ranked by lane (match), and the 32 warps of a chunk claim
// their slots one after another, so that the order of equal keys is the index order.
__global__ void __launch_bounds__(1024) k_sort_longest_first(SortJob j0, SortJob j1) {
  __shared__ int32_t start[kSortBuckets];
  __shared__ int32_t warp_sums[32];
  __shared__ int32_t nz_total;
  const SortJob j = blockIdx.x == 0 ? j0 : j1;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int i = tid; i < kSortBuckets; i += 1024) start[i] = 0;
  if (tid == 0) nz_total = 0;
  __syncthreads();
  int nz = 0;
  for (int i = tid; i < j.n; i += 1024) {
    const int c = j.cnt[i];
    nz += c > 0;
    atomicAdd(&start[sort_key(c)], 1);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) nz += __shfl_xor_sync(0xFFFFFFFFu, nz, o);
  if (lane == 0) atomicAdd(&nz_total, nz);
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
    for (int w = 0; w < 32; ++w) {
      if (warp == w && act && rank == 0) {
        first = start[key];
        start[key] = first + __popc(peers);
      }
      __syncthreads();
    }
    const int pos = __shfl_sync(0xFFFFFFFFu, first, leader) + rank;
    if (act) j.out[pos] = i;
  }
  if (tid == 0 && j.nonzero) *j.nonzero = nz_total;
}

// One warp per q-tile row: CSR entries in ascending kt, the PARTIAL numbering, the dense
// entry index of every listed block and the block of every PARTIAL number.
// One warp per q-tile row: CSR entries in ascending kt, the PARTIAL numbering, the dense
// entry index of every listed block, the block of every PARTIAL number, and the row's runs
// {first k-tile, number of tiles, kind, first CSR entry} at run[run_ptr[r] ..).
__global__ void k_fill_csr(const uint8_t* __restrict__ kinds, int rows, int KT,
                           const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ row_poff,
                           int32_t* __restrict__ col_idx, uint8_t* __restrict__ kind,
                           int32_t* __restrict__ pidx, int32_t* __restrict__ eidx,
                           int64_t* __restrict__ ptile, const int32_t* __restrict__ run_ptr,
                           int4* __restrict__ run) {
  const int r = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
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
    if (start)
      run[rpos + __popc(sm & ((1u << lane) - 1u))] =
          make_int4(kt, 0, v, e + __popc(nzm & ((1u << lane) - 1u)));
    rpos += __popc(sm);
    const unsigned lt = (1u << lane) - 1u;
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
}

// One warp per k-tile column: CSC entries in ascending qt with their CSR index.
__global__ void k_fill_csc(const uint8_t* __restrict__ kinds, const int32_t* __restrict__ eidx,
                           int B, int QT, int KT, const int32_t* __restrict__ colT_ptr,
                           int32_t* __restrict__ rowT_idx, int32_t* __restrict__ csc_map) {
  const int c = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (c >= B * KT) return;
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

// Thread k < 128 of a CTA: column k of the 128 x 128 bitmask w (512 words in shared memory,
// bit (k % 32) of word (q*4 + k/32)), i.e. bit (q % 32) of word (k*4 + q/32) of the transpose.
__device__ __forceinline__ void store_transposed(const uint32_t* w, uint32_t* __restrict__ dstT) {
  const int k = threadIdx.x;
  uint32_t out[4] = {0u, 0u, 0u, 0u};
  for (int q = 0; q < 128; ++q) out[q >> 5] |= ((w[q * 4 + (k >> 5)] >> (k & 31)) & 1u) << (q & 31);
  reinterpret_cast<uint4*>(dstT)[k] = make_uint4(out[0], out[1], out[2], out[3]);
}

// One CTA of 256 threads per PARTIAL block: its 128 x 128 bitmask from the mask, and the
// transposed copy.
__global__ void __launch_bounds__(256) k_bits_from_mask(const uint8_t* __restrict__ mask, int Nq,
                                                        int Nk, int64_t sb, int64_t sq, int QT,
                                                        int KT, const int64_t* __restrict__ ptile,
                                                        const int64_t* __restrict__ np,
                                                        uint32_t* __restrict__ bits,
                                                        uint32_t* __restrict__ bitsT) {
  __shared__ uint32_t w[512];
  const int64_t n = *np;  // PARTIAL blocks, from the counting step
  for (int64_t pb = blockIdx.x; pb < n; pb += gridDim.x) {
  const int64_t g = ptile[pb];
  const int kt = static_cast<int>(g % KT);
  const int qt = static_cast<int>((g / KT) % QT);
  const int b = static_cast<int>(g / (static_cast<int64_t>(KT) * QT));
  const int q = threadIdx.x >> 1, half = threadIdx.x & 1;
  uint32_t w0, w1;
  bool all;
  half_row_bits(mask, Nq, Nk, sb, sq, b, qt * kTile + q, kt * kTile + half * 64, w0, w1, all);
  uint32_t* dst = bits + pb * 512 + q * 4 + half * 2;
  dst[0] = w0;
  dst[1] = w1;
  w[q * 4 + half * 2] = w0;
  w[q * 4 + half * 2 + 1] = w1;
  __syncthreads();
  if (threadIdx.x < 128) store_transposed(w, bitsT + pb * 512);
  __syncthreads();
  }
}

// One CTA of 128 threads per PARTIAL block of a padded batch: row q is valid iff
// qt*128 + q < n, column k iff kt*128 + k < n.  Thread q writes row q of the bitmask and
// (the same rule with the roles swapped) column q of the transposed copy.
__global__ void __launch_bounds__(128) k_bits_from_lengths(const int32_t* __restrict__ lengths,
                                                           int Npad, int QT, int KT,
                                                           const int64_t* __restrict__ ptile,
                                                           const int64_t* __restrict__ np,
                                                           uint32_t* __restrict__ bits,
                                                           uint32_t* __restrict__ bitsT) {
  const int64_t npart = *np;  // PARTIAL blocks, from the counting step
  for (int64_t pb = blockIdx.x; pb < npart; pb += gridDim.x) {
  const int64_t g = ptile[pb];
  const int kt = static_cast<int>(g % KT);
  const int qt = static_cast<int>((g / KT) % QT);
  const int b = static_cast<int>(g / (static_cast<int64_t>(KT) * QT));
  const int n = min(max(lengths[b], 0), Npad);
  const int q = threadIdx.x;
  const bool row_ok = qt * kTile + q < n;
  uint4 w;
  w.x = row_ok ? low_bits(n - (kt * kTile + 0)) : 0u;
  w.y = row_ok ? low_bits(n - (kt * kTile + 32)) : 0u;
  w.z = row_ok ? low_bits(n - (kt * kTile + 64)) : 0u;
  w.w = row_ok ? low_bits(n - (kt * kTile + 96)) : 0u;
  reinterpret_cast<uint4*>(bits + pb * 512)[q] = w;
  const bool col_ok = kt * kTile + q < n;
  uint4 wt;
  wt.x = col_ok ? low_bits(n - (qt * kTile + 0)) : 0u;
  wt.y = col_ok ? low_bits(n - (qt * kTile + 32)) : 0u;
  wt.z = col_ok ? low_bits(n - (qt * kTile + 64)) : 0u;
  wt.w = col_ok ? low_bits(n - (qt * kTile + 96)) : 0u;
  reinterpret_cast<uint4*>(bitsT + pb * 512)[q] = wt;
  }
}

// desc[k] = {work[k], ptr[work[k]], ptr[work[k] + 1] - ptr[work[k]], w} for the row list
// (k < rows, w = the row's first run) and then the column list (w = 0).
__global__ void k_work_desc(const int32_t* __restrict__ row_work, const int32_t* __restrict__ row_ptr,
                            const int32_t* __restrict__ run_ptr, int rows,
                            int4* __restrict__ row_desc, const int32_t* __restrict__ col_work,
                            const int32_t* __restrict__ col_ptr, int cols,
                            int4* __restrict__ col_desc) {
  for (int k = blockIdx.x * blockDim.x + threadIdx.x; k < rows + cols; k += gridDim.x * blockDim.x) {
    const bool is_row = k < rows;
    const int kk = is_row ? k : k - rows;
    const int r = (is_row ? row_work : col_work)[kk];
    const int32_t* ptr = is_row ? row_ptr : col_ptr;
    const int a = ptr[r];
    (is_row ? row_desc : col_desc)[kk] = make_int4(r, a, ptr[r + 1] - a, is_row ? run_ptr[r] : 0);
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
  int64_t* totals = nullptr;
  int32_t* run_cnt = nullptr;
  int64_t* ptile = nullptr;
  void release(cudaStream_t s) {
    for (void*& p : block) {
      if (p) cudaFreeAsync(p, s);
      p = nullptr;
    }
  }
};

// The arenas go back to the pool in the order of the legacy default stream (the caller has
// made sure that no kernel still uses the plan).
void plan_free_buffers(sigattn_plan* p) {
  for (void*& a : p->arena) {
    if (a) cudaFreeAsync(a, cudaStreamLegacy);
    a = nullptr;
  }
}

#define SIGATTN_TRY(x)            \
  do {                            \
    const int rc_ = (x);          \
    if (rc_ != SIGATTN_OK) {      \
      sc.release(stream);         \
      plan_free_buffers(plan);    \
      delete plan;                \
      return rc_;                 \
    }                             \
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

// Both planners: `classify` writes every block's kind into sc.kinds, `bits_kernel` the
// bitmasks of the PARTIAL blocks (their number read on the device).  np_bound: most
// PARTIAL blocks the classification can yield (the grid for a mask; two tile strips per
// sequence for lengths).  When the tile arrays sized for the grid and np_bound fit
// kOnePassBytes, every step is queued and the host synchronises once at the end, for the
// counts and the argument checks; otherwise it synchronises after the counting step and
// sizes the arrays exactly.  cu_src (packed batches only): the cumulative offsets, copied
// into the plan; check_dev / check_host: one device int read back at the synchronisation
// (an argument check).
template <class ClassifyFn, class BitsFn>
int build_plan(sigattn_plan* plan, cudaStream_t stream, ClassifyFn classify, BitsFn bits_kernel,
               sigattn_plan** out, int64_t np_bound, const int32_t* cu_src = nullptr,
               const int32_t* check_dev = nullptr, int32_t* check_host = nullptr) {
  Scratch sc;
  const int B = plan->B, QT = plan->QT, KT = plan->KT;
  const int rows = B * QT, cols = B * KT;
  const int64_t grid_total = static_cast<int64_t>(rows) * KT;
  {
    Carve c;
    const size_t o_kinds = c.add<uint8_t>(grid_total), o_eidx = c.add<int32_t>(grid_total),
                 o_rc = c.add<int32_t>(rows), o_rp = c.add<int32_t>(rows),
                 o_ro = c.add<int32_t>(rows + 1), o_cc = c.add<int32_t>(cols),
                 o_tot = c.add<int64_t>(8), o_run = c.add<int32_t>(rows);
    SIGATTN_TRY(scratch_alloc(&sc.block[0], c.bytes, stream));
    void* m = sc.block[0];
    sc.kinds = Carve::at<uint8_t>(m, o_kinds);
    sc.eidx = Carve::at<int32_t>(m, o_eidx);
    sc.row_cnt = Carve::at<int32_t>(m, o_rc);
    sc.row_pcnt = Carve::at<int32_t>(m, o_rp);
    sc.row_poff = Carve::at<int32_t>(m, o_ro);
    sc.col_cnt = Carve::at<int32_t>(m, o_cc);
    sc.totals = Carve::at<int64_t>(m, o_tot);
    sc.run_cnt = Carve::at<int32_t>(m, o_run);
  }
  {
    Carve c;
    const size_t o_rptr = c.add<int32_t>(rows + 1), o_cptr = c.add<int32_t>(cols + 1),
                 o_rw = c.add<int32_t>(rows), o_cw = c.add<int32_t>(cols),
                 o_rd = c.add<int4>(rows), o_cd = c.add<int4>(cols),
                 o_rp = c.add<int32_t>(rows + 1), o_cu = c.add<int32_t>(cu_src ? B + 1 : 0);
    SIGATTN_TRY(plan_alloc(&plan->arena[0], c.bytes, stream));
    void* m = plan->arena[0];
    plan->row_ptr = Carve::at<int32_t>(m, o_rptr);
    plan->colT_ptr = Carve::at<int32_t>(m, o_cptr);
    plan->row_work = Carve::at<int32_t>(m, o_rw);
    plan->col_work = Carve::at<int32_t>(m, o_cw);
    plan->row_desc = Carve::at<int4>(m, o_rd);
    plan->col_desc = Carve::at<int4>(m, o_cd);
    plan->run_ptr = Carve::at<int32_t>(m, o_rp);
    if (cu_src) {
      plan->cu = Carve::at<int32_t>(m, o_cu);
      SIGATTN_TRY_CUDA(cudaMemcpyAsync(plan->cu, cu_src, (B + 1) * sizeof(int32_t),
                                       cudaMemcpyDeviceToDevice, stream));
    }
  }
  classify(sc.kinds);
  k_count<<<grid_for(static_cast<int64_t>(rows + cols) * 32, 256), 256, 0, stream>>>(
      sc.kinds, B, QT, KT, sc.row_cnt, sc.row_pcnt, sc.run_cnt, sc.col_cnt);
  k_scan4<<<4, 1024, 0, stream>>>(ScanJob{sc.row_cnt, rows, plan->row_ptr, sc.totals + 0},
                                  ScanJob{sc.row_pcnt, rows, sc.row_poff, sc.totals + 1},
                                  ScanJob{sc.col_cnt, cols, plan->colT_ptr, nullptr},
                                  ScanJob{sc.run_cnt, rows, plan->run_ptr, nullptr});
  k_sort_longest_first<<<2, 1024, 0, stream>>>(SortJob{sc.row_cnt, rows, plan->row_work, sc.totals + 2},
                                               SortJob{sc.col_cnt, cols, plan->col_work, sc.totals + 3});
  k_work_desc<<<grid_for(rows + cols, 256), 256, 0, stream>>>(
      plan->row_work, plan->row_ptr, plan->run_ptr, rows, plan->row_desc, plan->col_work,
      plan->colT_ptr, cols, plan->col_desc);
  SIGATTN_TRY_CUDA(cudaGetLastError());
  const int64_t np_max = std::min<int64_t>(grid_total, np_bound);
  const TileArena worst(static_cast<size_t>(grid_total), static_cast<size_t>(np_max));
  const bool one_pass = worst.bytes <= kOnePassBytes;
  // the fill steps, on arrays of capacity for (nz_cap, np_cap) tiles
  auto fill = [&](int64_t np_cap) -> int {
    SIGATTN_TRY(scratch_alloc(&sc.block[1], std::max<int64_t>(np_cap, 1) * sizeof(int64_t),
                              stream));
    sc.ptile = static_cast<int64_t*>(sc.block[1]);
    k_fill_csr<<<grid_for(static_cast<int64_t>(rows) * 32, 256), 256, 0, stream>>>(
        sc.kinds, rows, KT, plan->row_ptr, sc.row_poff, plan->col_idx, plan->kind, plan->pidx,
        sc.eidx, sc.ptile, plan->run_ptr, plan->run);
    k_fill_csc<<<grid_for(static_cast<int64_t>(cols) * 32, 256), 256, 0, stream>>>(
        sc.kinds, sc.eidx, B, QT, KT, plan->colT_ptr, plan->rowT_idx, plan->csc_map);
    if (np_cap > 0)
      bits_kernel(sc.ptile, sc.totals + 1, plan->bits, plan->bitsT,
                  static_cast<int>(std::min<int64_t>(np_cap, 2048)));
    return cuda_status(cudaGetLastError());
  };
  if (one_pass) {
    SIGATTN_TRY(plan_alloc(&plan->arena[1], worst.bytes, stream));
    worst.place(plan, plan->arena[1]);
    SIGATTN_TRY(fill(np_max));
  }
  int64_t totals[4] = {0, 0, 0, 0};
  int32_t last_row = 0;
  SIGATTN_TRY_CUDA(cudaMemcpyAsync(totals, sc.totals, sizeof(totals), cudaMemcpyDeviceToHost,
                                   stream));
  if (cu_src)
    SIGATTN_TRY_CUDA(cudaMemcpyAsync(&last_row, cu_src + B, sizeof(int32_t), cudaMemcpyDeviceToHost,
                                     stream));
  if (check_dev)
    SIGATTN_TRY_CUDA(cudaMemcpyAsync(check_host, check_dev, sizeof(int32_t), cudaMemcpyDeviceToHost,
                                     stream));
  SIGATTN_TRY_CUDA(cudaStreamSynchronize(stream));
  if (check_host && *check_host != 0) SIGATTN_TRY(SIGATTN_ERR_INVALID);
  if (cu_src && last_row < 1) SIGATTN_TRY(SIGATTN_ERR_INVALID);  // a packed batch needs rows
  plan->T = last_row;
  plan->nonempty = totals[0];
  plan->partial = totals[1];
  plan->full = totals[0] - totals[1];
  plan->rows_nonempty = static_cast<int32_t>(totals[2]);
  plan->cols_nonempty = static_cast<int32_t>(totals[3]);
  if (!one_pass) {
    const TileArena exact(static_cast<size_t>(plan->nonempty), static_cast<size_t>(plan->partial));
    SIGATTN_TRY(plan_alloc(&plan->arena[1], exact.bytes, stream));
    exact.place(plan, plan->arena[1]);
    SIGATTN_TRY(fill(plan->partial));
  }
  // one entry past the listed tiles stays readable: kernels bound their reads by it
  plan->run_cap = one_pass ? grid_total : plan->nonempty;
  sc.release(stream);
  *out = plan;
  return SIGATTN_OK;
}

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
  auto classify = [&](uint8_t* kinds) {
    k_kinds_from_lengths<<<grid_for(grid_total, 256), 256, 0, stream>>>(d_lengths, B, Npad, QT,
                                                                          QT, kinds);
  };
  auto bits = [&](const int64_t* ptile, const int64_t* np, uint32_t* dst, uint32_t* dstT,
                  int grid) {
    k_bits_from_lengths<<<grid, 128, 0, stream>>>(d_lengths, Npad, QT, QT, ptile, np, dst, dstT);
  };
  // PARTIAL blocks of a length: the last q-tile row and k-tile column of the sequence
  return build_plan(plan, stream, classify, bits, out, 2 * static_cast<int64_t>(B) * QT);
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
  auto classify = [&](uint8_t* kinds) {
    k_kinds_from_lengths<<<grid_for(grid_total, 256), 256, 0, stream>>>(lengths, B, max_seqlen, QT,
                                                                          QT, kinds);
  };
  auto bits = [&](const int64_t* ptile, const int64_t* np, uint32_t* dst, uint32_t* dstT,
                  int grid) {
    k_bits_from_lengths<<<grid, 128, 0, stream>>>(lengths, max_seqlen, QT, QT, ptile, np, dst,
                                                  dstT);
  };
  int32_t bad_host = 0;
  rc = build_plan(plan, stream, classify, bits, out, 2 * static_cast<int64_t>(B) * QT, d_cu, bad,
                  &bad_host);
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
  auto classify = [&](uint8_t* kinds) {
    // one warp per block, eight per CTA, at most 16 CTAs per SM's worth of work at once
    const int64_t ctas = std::min<int64_t>((grid_total + 7) / 8, 148 * 16);
    k_kinds_from_mask<<<static_cast<unsigned>(ctas), 256, 0, stream>>>(
        d_mask, B, Nq, Nk, stride_b, stride_q, QT, KT, kinds);
  };
  auto bits = [&](const int64_t* ptile, const int64_t* np, uint32_t* dst, uint32_t* dstT,
                  int grid) {
    k_bits_from_mask<<<grid, 256, 0, stream>>>(d_mask, Nq, Nk, stride_b, stride_q, QT, KT, ptile,
                                               np, dst, dstT);
  };
  return build_plan(plan, stream, classify, bits, out, grid_total);
}

extern "C" int sigattn_plan_get_sizes(const sigattn_plan* plan, sigattn_plan_sizes* sz) {
  if (!plan || !sz) return SIGATTN_ERR_INVALID;
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
