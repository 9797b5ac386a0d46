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
__global__ void __launch_bounds__(256) k_kinds_from_mask(const uint8_t* __restrict__ mask, int B,
                                                         int Nq, int Nk, int64_t sb, int64_t sq,
                                                         int QT, int KT,
                                                         uint8_t* __restrict__ kinds) {
  const int64_t blk = blockIdx.x;
  const int kt = static_cast<int>(blk % KT);
  const int qt = static_cast<int>((blk / KT) % QT);
  const int b = static_cast<int>(blk / (static_cast<int64_t>(KT) * QT));
  const int row = qt * kTile + (threadIdx.x >> 1);
  const int col0 = kt * kTile + (threadIdx.x & 1) * 64;
  uint32_t w0, w1;
  bool all;
  half_row_bits(mask, Nq, Nk, sb, sq, b, row, col0, w0, w1, all);
  const int any_b = __syncthreads_or((w0 | w1) != 0u);
  const int all_b = __syncthreads_and(all);
  if (threadIdx.x == 0) kinds[blk] = all_b ? 1 : (any_b ? 2 : 0);
}

// One warp per q-tile row: number of listed blocks and of PARTIAL blocks.
__global__ void k_count_rows(const uint8_t* __restrict__ kinds, int rows, int KT,
                             int32_t* __restrict__ cnt, int32_t* __restrict__ pcnt) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= rows) return;
  const uint8_t* k = kinds + static_cast<int64_t>(warp) * KT;
  int c = 0, p = 0;
  for (int kt = lane; kt < KT; kt += 32) {
    const uint8_t v = k[kt];
    c += v != 0;
    p += v == 2;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    c += __shfl_xor_sync(0xFFFFFFFFu, c, o);
    p += __shfl_xor_sync(0xFFFFFFFFu, p, o);
  }
  if (lane == 0) {
    cnt[warp] = c;
    pcnt[warp] = p;
  }
}

// One warp per k-tile column c = b*KT + kt.
__global__ void k_count_cols(const uint8_t* __restrict__ kinds, int B, int QT, int KT,
                             int32_t* __restrict__ cnt) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= B * KT) return;
  const int b = warp / KT, kt = warp % KT;
  int c = 0;
  for (int qt = lane; qt < QT; qt += 32) c += kinds[(static_cast<int64_t>(b) * QT + qt) * KT + kt] != 0;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xFFFFFFFFu, c, o);
  if (lane == 0) cnt[warp] = c;
}

// Exclusive scan of in[0..n) into out[0..n]; out[n] is the total, also stored to *total.
// One CTA of 1024 threads walking the input in chunks.
__global__ void __launch_bounds__(1024) k_scan(const int32_t* __restrict__ in, int n,
                                               int32_t* __restrict__ out, int64_t* total) {
  __shared__ int32_t warp_sums[32];
  __shared__ int32_t carry;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int base = 0; base < n; base += 1024) {
    const int i = base + threadIdx.x;
    const int x = i < n ? in[i] : 0;
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
    const int before = carry + (warp > 0 ? warp_sums[warp - 1] : 0) + incl - x;
    if (i < n) out[i] = before;
    __syncthreads();
    if (threadIdx.x == 0) carry += warp_sums[31];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    out[n] = carry;
    if (total) *total = carry;
  }
}

// Stable counting sort of indices 0..n-1 by cnt[i] descending (counts past 4094 share a
// bucket).  One warp.  Also stores the number of nonzero counts to *nonzero.
__global__ void __launch_bounds__(32) k_sort_longest_first(const int32_t* __restrict__ cnt, int n,
                                                           int32_t* __restrict__ out,
                                                           int64_t* nonzero) {
  __shared__ int32_t start[kSortBuckets];
  const int lane = threadIdx.x;
  for (int i = lane; i < kSortBuckets; i += 32) start[i] = 0;
  __syncwarp();
  int nz = 0;
  // key = kSortBuckets - 1 - min(cnt, kSortBuckets - 1): ascending key = descending count
  for (int i = lane; i < n; i += 32) {
    const int c = cnt[i];
    nz += c > 0;
    atomicAdd(&start[kSortBuckets - 1 - min(c, kSortBuckets - 1)], 1);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) nz += __shfl_xor_sync(0xFFFFFFFFu, nz, o);
  __syncwarp();
  // exclusive scan over the buckets: lane l owns buckets [l*128, l*128+128)
  constexpr int per = kSortBuckets / 32;
  int sum = 0;
  for (int j = 0; j < per; ++j) sum += start[lane * per + j];
  int incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += y;
  }
  int run = incl - sum;
  __syncwarp();
  for (int j = 0; j < per; ++j) {
    const int c = start[lane * per + j];
    start[lane * per + j] = run;
    run += c;
  }
  __syncwarp();
  for (int base = 0; base < n; base += 32) {
    const int i = base + lane;
    const bool act = i < n;
    const int key = act ? kSortBuckets - 1 - min(cnt[i], kSortBuckets - 1) : -1 - lane;
    const unsigned peers = __match_any_sync(0xFFFFFFFFu, key);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    int pos = 0;
    if (act) pos = start[key] + rank;
    __syncwarp();
    if (act) {
      out[pos] = i;
      if (rank == 0) start[key] += __popc(peers);
    }
    __syncwarp();
  }
  if (lane == 0 && nonzero) *nonzero = nz;
}

// One warp per q-tile row: CSR entries in ascending kt, the PARTIAL numbering, the dense
// entry index of every listed block and the block of every PARTIAL number.
__global__ void k_fill_csr(const uint8_t* __restrict__ kinds, int rows, int KT,
                           const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ row_poff,
                           int32_t* __restrict__ col_idx, uint8_t* __restrict__ kind,
                           int32_t* __restrict__ pidx, int32_t* __restrict__ eidx,
                           int64_t* __restrict__ ptile) {
  const int r = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  int e = row_ptr[r];
  int p = row_poff[r];
  const uint8_t* k = kinds + static_cast<int64_t>(r) * KT;
  for (int base = 0; base < KT; base += 32) {
    const int kt = base + lane;
    const uint8_t v = kt < KT ? k[kt] : 0;
    const unsigned nzm = __ballot_sync(0xFFFFFFFFu, v != 0);
    const unsigned pm = __ballot_sync(0xFFFFFFFFu, v == 2);
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

// One CTA of 256 threads per PARTIAL block: its 128 x 128 bitmask from the mask.
__global__ void __launch_bounds__(256) k_bits_from_mask(const uint8_t* __restrict__ mask, int Nq,
                                                        int Nk, int64_t sb, int64_t sq, int QT,
                                                        int KT, const int64_t* __restrict__ ptile,
                                                        uint32_t* __restrict__ bits) {
  const int64_t g = ptile[blockIdx.x];
  const int kt = static_cast<int>(g % KT);
  const int qt = static_cast<int>((g / KT) % QT);
  const int b = static_cast<int>(g / (static_cast<int64_t>(KT) * QT));
  const int q = threadIdx.x >> 1, half = threadIdx.x & 1;
  uint32_t w0, w1;
  bool all;
  half_row_bits(mask, Nq, Nk, sb, sq, b, qt * kTile + q, kt * kTile + half * 64, w0, w1, all);
  uint32_t* dst = bits + static_cast<int64_t>(blockIdx.x) * 512 + q * 4 + half * 2;
  dst[0] = w0;
  dst[1] = w1;
}

// One CTA of 128 threads per PARTIAL block of a padded batch: row q is valid iff
// qt*128 + q < n, column k iff kt*128 + k < n.
__global__ void __launch_bounds__(128) k_bits_from_lengths(const int32_t* __restrict__ lengths,
                                                           int Npad, int QT, int KT,
                                                           const int64_t* __restrict__ ptile,
                                                           uint32_t* __restrict__ bits) {
  const int64_t g = ptile[blockIdx.x];
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
  reinterpret_cast<uint4*>(bits + static_cast<int64_t>(blockIdx.x) * 512)[q] = w;
}

// desc[k] = {work[k], ptr[work[k]], ptr[work[k] + 1] - ptr[work[k]], 0}
__global__ void k_work_desc(const int32_t* __restrict__ work, const int32_t* __restrict__ ptr, int n,
                            int4* __restrict__ desc) {
  for (int k = blockIdx.x * blockDim.x + threadIdx.x; k < n; k += gridDim.x * blockDim.x) {
    const int r = work[k];
    const int a = ptr[r];
    desc[k] = make_int4(r, a, ptr[r + 1] - a, 0);
  }
}

// One CTA of 128 threads per PARTIAL block: thread k gathers column k of the bitmask.
__global__ void __launch_bounds__(128) k_transpose_bits(const uint32_t* __restrict__ bits,
                                                        uint32_t* __restrict__ bitsT) {
  __shared__ uint32_t w[512];
  const uint32_t* src = bits + static_cast<int64_t>(blockIdx.x) * 512;
  for (int i = threadIdx.x; i < 512; i += 128) w[i] = src[i];
  __syncthreads();
  const int k = threadIdx.x;
  uint32_t out[4] = {0u, 0u, 0u, 0u};
  for (int q = 0; q < 128; ++q) out[q >> 5] |= ((w[q * 4 + (k >> 5)] >> (k & 31)) & 1u) << (q & 31);
  reinterpret_cast<uint4*>(bitsT + static_cast<int64_t>(blockIdx.x) * 512)[k] =
      make_uint4(out[0], out[1], out[2], out[3]);
}

template <class T>
int dev_alloc(T** p, size_t count) {
  *p = nullptr;
  if (count == 0) return SIGATTN_OK;
  const cudaError_t e = cudaMalloc(reinterpret_cast<void**>(p), count * sizeof(T));
  if (e != cudaSuccess) {
    *p = nullptr;
    cudaGetLastError();
    return e == cudaErrorMemoryAllocation ? SIGATTN_ERR_NOMEM : SIGATTN_ERR_CUDA;
  }
  return SIGATTN_OK;
}

template <class T>
int scratch_alloc(T** p, size_t count, cudaStream_t s) {
  *p = nullptr;
  if (count == 0) count = 1;
  const cudaError_t e = cudaMallocAsync(reinterpret_cast<void**>(p), count * sizeof(T), s);
  if (e != cudaSuccess) {
    *p = nullptr;
    cudaGetLastError();
    return e == cudaErrorMemoryAllocation ? SIGATTN_ERR_NOMEM : SIGATTN_ERR_CUDA;
  }
  return SIGATTN_OK;
}

struct Scratch {
  uint8_t* kinds = nullptr;
  int32_t* eidx = nullptr;
  int32_t* row_cnt = nullptr;
  int32_t* row_pcnt = nullptr;
  int32_t* row_poff = nullptr;
  int32_t* col_cnt = nullptr;
  int64_t* totals = nullptr;
  int64_t* ptile = nullptr;
  void release(cudaStream_t s) {
    void* ps[] = {kinds, eidx, row_cnt, row_pcnt, row_poff, col_cnt, totals, ptile};
    for (void* p : ps)
      if (p) cudaFreeAsync(p, s);
  }
};

void plan_free_buffers(sigattn_plan* p) {
  void* ps[] = {p->row_ptr, p->col_idx, p->kind,     p->pidx,     p->colT_ptr, p->rowT_idx,
                p->csc_map, p->bits,    p->bitsT,    p->row_work, p->col_work, p->row_desc,
                p->col_desc};
  for (void* q : ps)
    if (q) cudaFree(q);
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

// Shared tail of both planners: kinds are in sc.kinds; `bits_kernel` fills bitmasks.
template <class BitsFn>
int finish_plan(sigattn_plan* plan, Scratch& sc, cudaStream_t stream, BitsFn bits_kernel,
                sigattn_plan** out) {
  const int B = plan->B, QT = plan->QT, KT = plan->KT;
  const int rows = B * QT, cols = B * KT;
  SIGATTN_TRY(dev_alloc(&plan->row_ptr, rows + 1));
  SIGATTN_TRY(dev_alloc(&plan->colT_ptr, cols + 1));
  SIGATTN_TRY(dev_alloc(&plan->row_work, rows));
  SIGATTN_TRY(dev_alloc(&plan->col_work, cols));
  SIGATTN_TRY(dev_alloc(&plan->row_desc, rows));
  SIGATTN_TRY(dev_alloc(&plan->col_desc, cols));
  SIGATTN_TRY(scratch_alloc(&sc.row_cnt, rows, stream));
  SIGATTN_TRY(scratch_alloc(&sc.row_pcnt, rows, stream));
  SIGATTN_TRY(scratch_alloc(&sc.row_poff, rows + 1, stream));
  SIGATTN_TRY(scratch_alloc(&sc.col_cnt, cols, stream));
  SIGATTN_TRY(scratch_alloc(&sc.totals, 8, stream));
  k_count_rows<<<grid_for(static_cast<int64_t>(rows) * 32, 256), 256, 0, stream>>>(
      sc.kinds, rows, KT, sc.row_cnt, sc.row_pcnt);
  k_count_cols<<<grid_for(static_cast<int64_t>(cols) * 32, 256), 256, 0, stream>>>(
      sc.kinds, B, QT, KT, sc.col_cnt);
  k_scan<<<1, 1024, 0, stream>>>(sc.row_cnt, rows, plan->row_ptr, sc.totals + 0);
  k_scan<<<1, 1024, 0, stream>>>(sc.row_pcnt, rows, sc.row_poff, sc.totals + 1);
  k_scan<<<1, 1024, 0, stream>>>(sc.col_cnt, cols, plan->colT_ptr, nullptr);
  k_sort_longest_first<<<1, 32, 0, stream>>>(sc.row_cnt, rows, plan->row_work, sc.totals + 2);
  k_sort_longest_first<<<1, 32, 0, stream>>>(sc.col_cnt, cols, plan->col_work, sc.totals + 3);
  k_work_desc<<<grid_for(rows, 256), 256, 0, stream>>>(plan->row_work, plan->row_ptr, rows,
                                                        plan->row_desc);
  k_work_desc<<<grid_for(cols, 256), 256, 0, stream>>>(plan->col_work, plan->colT_ptr, cols,
                                                        plan->col_desc);
  SIGATTN_TRY_CUDA(cudaGetLastError());
  int64_t totals[8] = {0};
  SIGATTN_TRY_CUDA(cudaMemcpyAsync(totals, sc.totals, 4 * sizeof(int64_t), cudaMemcpyDeviceToHost,
                                   stream));
  SIGATTN_TRY_CUDA(cudaStreamSynchronize(stream));
  plan->nonempty = totals[0];
  plan->partial = totals[1];
  plan->full = totals[0] - totals[1];
  plan->rows_nonempty = static_cast<int32_t>(totals[2]);
  plan->cols_nonempty = static_cast<int32_t>(totals[3]);
  SIGATTN_TRY(dev_alloc(&plan->col_idx, plan->nonempty));
  SIGATTN_TRY(dev_alloc(&plan->kind, plan->nonempty));
  SIGATTN_TRY(dev_alloc(&plan->pidx, plan->nonempty));
  SIGATTN_TRY(dev_alloc(&plan->rowT_idx, plan->nonempty));
  SIGATTN_TRY(dev_alloc(&plan->csc_map, plan->nonempty));
  SIGATTN_TRY(dev_alloc(&plan->bits, static_cast<size_t>(plan->partial) * 512));
  SIGATTN_TRY(dev_alloc(&plan->bitsT, static_cast<size_t>(plan->partial) * 512));
  SIGATTN_TRY(scratch_alloc(&sc.eidx, static_cast<size_t>(rows) * KT, stream));
  SIGATTN_TRY(scratch_alloc(&sc.ptile, static_cast<size_t>(plan->partial), stream));
  if (plan->nonempty > 0) {
    k_fill_csr<<<grid_for(static_cast<int64_t>(rows) * 32, 256), 256, 0, stream>>>(
        sc.kinds, rows, KT, plan->row_ptr, sc.row_poff, plan->col_idx, plan->kind, plan->pidx,
        sc.eidx, sc.ptile);
    k_fill_csc<<<grid_for(static_cast<int64_t>(cols) * 32, 256), 256, 0, stream>>>(
        sc.kinds, sc.eidx, B, QT, KT, plan->colT_ptr, plan->rowT_idx, plan->csc_map);
  }
  if (plan->partial > 0) {
    bits_kernel(sc.ptile, plan->bits, static_cast<int>(plan->partial));
    k_transpose_bits<<<static_cast<unsigned>(plan->partial), 128, 0, stream>>>(plan->bits,
                                                                               plan->bitsT);
  }
  SIGATTN_TRY_CUDA(cudaGetLastError());
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
  SIGATTN_TRY(scratch_alloc(&sc.kinds, static_cast<size_t>(grid_total), stream));
  k_kinds_from_lengths<<<grid_for(grid_total, 256), 256, 0, stream>>>(d_lengths, B, Npad, QT, QT,
                                                                        sc.kinds);
  auto bits = [&](const int64_t* ptile, uint32_t* dst, int np) {
    k_bits_from_lengths<<<np, 128, 0, stream>>>(d_lengths, Npad, QT, QT, ptile, dst);
  };
  return finish_plan(plan, sc, stream, bits, out);
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
  SIGATTN_TRY(scratch_alloc(&sc.kinds, static_cast<size_t>(grid_total), stream));
  k_kinds_from_mask<<<static_cast<unsigned>(grid_total), 256, 0, stream>>>(
      d_mask, B, Nq, Nk, stride_b, stride_q, QT, KT, sc.kinds);
  auto bits = [&](const int64_t* ptile, uint32_t* dst, int np) {
    k_bits_from_mask<<<np, 256, 0, stream>>>(d_mask, Nq, Nk, stride_b, stride_q, QT, KT, ptile,
                                             dst);
  };
  return finish_plan(plan, sc, stream, bits, out);
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

extern "C" void sigattn_plan_destroy(sigattn_plan* plan) {
  if (!plan) return;
  plan_free_buffers(plan);
  delete plan;
}
