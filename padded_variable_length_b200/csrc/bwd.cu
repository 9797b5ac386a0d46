// Backward kernels, sm_100a: a dK/dV kernel that walks each k-tile column of the plan and
// a dQ kernel that walks each q-tile row, both recomputing the attention weights tile by
// tile, so that neither needs atomics ("Better Models, Faster Training: Sigmoid Attention
// for single-cell Foundation Models", section 2C, backward split into a Q-gradient kernel
// and a K/V-gradient kernel that recompute activations on the fly).
//
// Per tile, with s = scale * q.k + bias:
//   SIGMOID            p = sigma(s)                   ds = dp * p * (1 - p)   (section 2B:
//                      sigma' = sigma (1 - sigma); the Jacobian is diagonal, no row term)
//   SOFTMAX/SOFTMAX1   p = exp(s - lse)               ds = p * (dp - D),  D = dO . O
//   dV += P^T dO      dK += scale dS^T Q      dQ += scale dS K
//
// Thread layout as in the forward: warp 0 TMA producer, warp 1 TMEM allocator and MMA
// issuer, warps 4-11 two epilogue warpgroups (thread = TMEM lane; warpgroup h owns column
// half h of every tile and accumulator columns [h d/2, (h+1) d/2)).
// TMEM: [0,128) S (or S^T), [128,256) dP (or dP^T), then the fp32 accumulators.  The bf16
// P / dS values overwrite the columns of S / dP that the same warpgroup already read, and
// are the TMEM A operand of the accumulating MMAs.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>
#include <type_traits>

#include "internal.h"
#include "sm100.cuh"

namespace sigattn {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kThreads = 384;
constexpr int kEpiWarp0 = 4;

struct BwdParams {
  const int32_t* row_ptr;
  const int32_t* col_idx;
  const uint8_t* kind;
  const int32_t* pidx;
  const uint32_t* bits;
  const uint32_t* bitsT;
  const int32_t* colT_ptr;
  const int32_t* rowT_idx;
  const int32_t* csc_map;
  const int4* row_desc;
  const int4* col_desc;
  const int32_t* cu;  // packed batches: cumulative row offsets [B + 1]; nullptr when padded
  int B, QT, KT, Nq, Nk, H;
  // items with tiles: the first counts[kCountCols] * H (k-tile column, head) items of the
  // column list and the first counts[kCountRows] * H (q-tile row, head) items of the row
  // list; the rest are empty (the plan's device counts: its build need not have been waited
  // for on the host)
  const int64_t* counts;
  float scale;
  const float* bias;
  int64_t bias_sb;
  const float* lse;   // [B, H, Nq] softmax modes
  const float* Dws;   // [B, H, Nq] softmax modes
  __nv_bfloat16* dq;
  int64_t dq_sb, dq_sn, dq_sh;
  __nv_bfloat16* dk;
  int64_t dk_sb, dk_sn, dk_sh;
  __nv_bfloat16* dv;
  int64_t dv_sb, dv_sn, dv_sh;
  int* status;
  unsigned long long wait_ns;
};

// Offset of one query row in the weight's argument t = c1 s + off, c1 = scale log2 e:
// SIGMOID  p = sigma(t ln 2),  off = bias log2 e  (sigmoid_grad2);
// softmax  p = 2^t,            off = (bias - lse) log2 e.
template <int EPI>
__device__ __forceinline__ float row_offset(const BwdParams& p, const SeqRows& sq, int b, int h,
                                           int qg) {
  if (qg >= p.Nq) return 0.0f;
  const float bias =
      (p.bias && qg < sq.limit) ? p.bias[static_cast<int64_t>(sq.tma_b) * p.bias_sb + sq.row0 + qg]
                                : 0.0f;
  if (EPI == 0) return bias * kLog2e;
  return (bias - p.lse[(static_cast<int64_t>(b) * p.H + h) * p.Nq + qg]) * kLog2e;
}

template <int EPI>
__device__ __forceinline__ float row_D(const BwdParams& p, int b, int h, int qg) {
  if (EPI == 0 || qg >= p.Nq) return 0.0f;
  return p.Dws[(static_cast<int64_t>(b) * p.H + h) * p.Nq + qg];
}

// p and ds of two neighbouring elements (packed fp32 pairs); k0 / k1 are the mask bits.
// SIGMOID: p = sigma(x), ds = dp sigma'(x) with sigma' = sigma (1 - sigma) from the same
//   exp2 (sigmoid_grad2); a masked element takes t = -inf, which gives p = ds = 0.
// softmax: p = 2^t, ds = p (dp - D); a masked element takes p = 0.
template <int EPI>
__device__ __forceinline__ void weight_grad2(float2 s, float2 dp, float2 c1, float2 off, float2 Dv,
                                             bool k0, bool k1, float2& pw, float2& ds) {
  float2 x = fma2(s, c1, off);
  if (EPI == 0) {
    x.x = k0 ? x.x : -INFINITY;
    x.y = k1 ? x.y : -INFINITY;
    float2 w;
    sigmoid_grad2(x, pw, w);
    ds = mul2(w, dp);
  } else {
    pw = make_float2(k0 ? ex2_approx(x.x) : 0.0f, k1 ? ex2_approx(x.y) : 0.0f);
    ds = mul2(pw, fma2(Dv, make_float2(-1.0f, -1.0f), dp));
  }
}

template <int D>
__device__ __forceinline__ void zero_rows(__nv_bfloat16* base, int64_t sn, int rows, int tid,
                                          int nthreads) {
  constexpr int kChunks = D / 8;
  for (int i = tid; i < rows * kChunks; i += nthreads) {
    const int row = i / kChunks, c = i % kChunks;
    *reinterpret_cast<uint4*>(base + static_cast<int64_t>(row) * sn + c * 8) =
        make_uint4(0u, 0u, 0u, 0u);
  }
}

// ---------------------------------------------------------------------------------------
// D_i = dO_i . O_i for the softmax modes.  One thread per 16-byte chunk; d/8 lanes per row.
// ---------------------------------------------------------------------------------------
template <int D>
__global__ void d_preprocess_kernel(const __nv_bfloat16* __restrict__ o, int64_t o_sb, int64_t o_sn,
                                    int64_t o_sh, const __nv_bfloat16* __restrict__ dout,
                                    int64_t do_sb, int64_t do_sn, int64_t do_sh, int B, int Nq,
                                    int H, const int32_t* __restrict__ cu, float* __restrict__ Dws) {
  constexpr int kLanes = D / 8;
  const int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  const int64_t row = t / kLanes;
  const int chunk = static_cast<int>(t % kLanes);
  const bool act = row < static_cast<int64_t>(B) * Nq * H;
  float acc = 0.0f;
  int b = 0, i = 0, h = 0;
  if (act) {
    h = static_cast<int>(row % H);
    i = static_cast<int>((row / H) % Nq);
    b = static_cast<int>(row / (static_cast<int64_t>(H) * Nq));
  }
  const SeqRows sq = seq_rows(cu, b, Nq);
  if (act && i < sq.limit) {
    const uint4 ov = *reinterpret_cast<const uint4*>(o + seq_row_offset(sq, o_sb, o_sn, i) + h * o_sh + chunk * 8);
    const uint4 dv = *reinterpret_cast<const uint4*>(dout + seq_row_offset(sq, do_sb, do_sn, i) + h * do_sh + chunk * 8);
    const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&ov);
    const __nv_bfloat162* d2 = reinterpret_cast<const __nv_bfloat162*>(&dv);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const float2 a = __bfloat1622float2(o2[c]);
      const float2 g = __bfloat1622float2(d2[c]);
      acc = fmaf(a.x, g.x, acc);
      acc = fmaf(a.y, g.y, acc);
    }
  }
#pragma unroll
  for (int off = kLanes / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, off);
  if (act && chunk == 0) Dws[(static_cast<int64_t>(b) * H + h) * Nq + i] = acc;
}

// ---------------------------------------------------------------------------------------
// Shared pieces of the two gradient kernels.
//
// Both are persistent (one CTA per SM, snake order over the plan's longest-first work
// list) and split every 128 x 128 tile into two halves along the walked axis: epilogue
// warpgroup h owns half h.  d = 64 runs the "unit" schedule (three rotating TMEM buffers,
// the MMAs of a half-tile issued three halves ahead, see the dK / dV layout); d = 128 keeps
// one buffer per half and interleaves the halves.  The MMA issuer is a whole warp issuing
// from warp-uniform values.
// ---------------------------------------------------------------------------------------
struct WorkRef {
  int b, t, h, e0, n;  // batch, tile index on the item's own axis, head, list range
  SeqRows sq;          // where the rows of sequence b live (padded or packed)
};

// dK/dV: item w -> (k-tile column, head); dQ: item w -> (q-tile row, head).
__device__ __forceinline__ WorkRef decode_col(const BwdParams& p, int w) {
  WorkRef r;
  const int4 d = p.col_desc[w / p.H];
  r.h = w % p.H;
  r.b = d.x / p.KT;
  r.t = d.x % p.KT;
  r.e0 = d.y;
  r.n = d.z;
  r.sq = seq_rows(p.cu, r.b, p.Nk);
  return r;
}

__device__ __forceinline__ WorkRef decode_row(const BwdParams& p, int w) {
  WorkRef r;
  const int4 d = p.row_desc[w / p.H];
  r.h = w % p.H;
  r.b = d.x / p.QT;
  r.t = d.x % p.QT;
  r.e0 = d.y;
  r.n = d.z;
  r.sq = seq_rows(p.cu, r.b, p.Nq);
  return r;
}

// Zero gradient rows for the items without tiles, [nwork, nitems) of a longest-first list
// (k-tiles that no query attends to, for dK / dV; q-tiles past their sequence's length or
// seeing no key, for dQ).  The items are dealt round-robin to every epilogue warp of the
// grid, one item per warp at a time, with no dependent loads between them; run before the
// first tile, while the epilogue would otherwise wait for its first S.  x1 may be null.
template <int D, bool kCols>
__device__ void zero_empty_items(const BwdParams& p, int nwork, int nitems, int ew, int lane,
                                 __nv_bfloat16* x0, int64_t sb0, int64_t sn0, int64_t sh0,
                                 __nv_bfloat16* x1, int64_t sb1, int64_t sn1, int64_t sh1) {
  constexpr int kChunks = D / 8;
  const int stride = static_cast<int>(gridDim.x) * 8;
  for (int w = nwork + static_cast<int>(blockIdx.x) * 8 + ew; w < nitems; w += stride) {
    const WorkRef x = kCols ? decode_col(p, w) : decode_row(p, w);
    const int rows = min(kTile, x.sq.limit - x.t * kTile);
    for (int c = lane; c < rows * kChunks; c += 32) {
      const int r = x.t * kTile + c / kChunks, ch = (c % kChunks) * 8;
      *reinterpret_cast<uint4*>(x0 + seq_row_offset(x.sq, sb0, sn0, r) + x.h * sh0 + ch) =
          make_uint4(0u, 0u, 0u, 0u);
      if (x1 != nullptr)
        *reinterpret_cast<uint4*>(x1 + seq_row_offset(x.sq, sb1, sn1, r) + x.h * sh1 + ch) =
            make_uint4(0u, 0u, 0u, 0u);
    }
  }
}

// Walks this CTA's work items (snake order, see snake_item) with the next item's decode
// issued one item ahead, so that its global loads overlap the current item.
template <bool kCols>
struct WorkIter {
  const BwdParams& p;
  int k, w, wn, nitems;  // round, this item, next item, list length
  WorkRef cur, nxt;
  __device__ WorkRef dec(int ww) const { return kCols ? decode_col(p, ww) : decode_row(p, ww); }
  __device__ WorkIter(const BwdParams& pp, int n)
      : p(pp), k(0), w(snake_item(0)), wn(snake_item(1)), nitems(n) {
    if (w < nitems) cur = dec(w);
    if (wn < nitems) nxt = dec(wn);
  }
  __device__ bool valid() const { return w < nitems; }
  __device__ void advance() {
    ++k;
    w = wn;
    wn = snake_item(k + 1);
    cur = nxt;
    if (wn < nitems) nxt = dec(wn);
  }
};

// ---------------------------------------------------------------------------------------
// dK / dV: one item = one k-tile column of the plan for one head; thread = key row.
// d = 128 TMEM: S^T half h [64h, 64h+64), dP^T half h [128+64h, ...), dV [256, 384),
// dK [384, 512).
// d = 64 ("unit" schedule): a unit is one query half of one tile, u = 2 (tile) + half, and
// warpgroup h takes the units of half h.  Three unit buffers rotate: S^T of unit u in
// [128 (u % 3), +64), dP^T in [128 (u % 3) + 64, +64); P^T and dS^T overwrite the first 32
// columns of each.  The MMA issuer computes S^T / dP^T of unit u right after the dV / dK
// MMAs of unit u - 3, the last user of that buffer, so they are ready a tile and a half
// before the epilogue needs them.  dV [384, 448), dK [448, 512) (one accumulator: the
// epilogue reads an item's dV / dK after its first unit of the next item).
// ---------------------------------------------------------------------------------------
template <int D>
struct DkvLayout {
  static constexpr bool kUnits = D == 64;
  static constexpr int kStages = kUnits ? 4 : 2;  // Q / dO ring
  static constexpr int kKVBufs = D == 64 ? 2 : 1;   // K / V of consecutive items
  static constexpr int kAccBufs = 1;                // dV / dK accumulators in TMEM
  static constexpr int kBoxes = D / 64;
  static constexpr int kBoxBytes = 128 * 128;
  static constexpr int kTileBytes = kBoxes * kBoxBytes;
  static constexpr int kK = 0;
  static constexpr int kV = kK + kKVBufs * kTileBytes;
  static constexpr int kQ = kV + kKVBufs * kTileBytes;
  static constexpr int kDO = kQ + kStages * kTileBytes;
  static constexpr int kVec = kDO + kStages * kTileBytes;  // float [S][2][128]
  // per Q/dO stage: the tile's transposed PARTIAL bitmask and its kind, staged by the producer
  static constexpr int kMetaBits = kVec + kStages * 2 * 128 * 4;
  static constexpr int kMetaKind = kMetaBits + kStages * 2048;
  static constexpr int kBar = kMetaKind + 16 * ((kStages * 4 + 15) / 16);
  // kv_full[KV] kv_empty[KV] q_full[S] q_empty[S] s_full[NR] p_full[NR] acc_full[A] acc_empty[A]
  // (NR = 4 unit slots for d = 64, one per half for d = 128)
  static constexpr int kRing = kUnits ? 4 : 2;
  static constexpr int kNumBars = 2 * kKVBufs + 2 * kStages + 2 * kRing + 2 * kAccBufs + 1;
  static constexpr int kMisc = kBar + 8 * kNumBars;
  static constexpr int kBytes = kMisc + 16;
  static constexpr int kAlloc = kBytes + 1024;
};

template <int D, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    dkdv_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tdo,
                const BwdParams p) {
  using L = DkvLayout<D>;
  constexpr int S = L::kStages, KVB = L::kKVBufs, ACB = L::kAccBufs;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int warp = warp_id(), lane = lane_id();
  const int nitems = p.B * p.KT * p.H, nwork = static_cast<int>(__ldg(p.counts + kCountCols)) * p.H;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = kv_full + KVB;
  uint64_t* q_full = kv_empty + KVB;
  uint64_t* q_empty = q_full + S;
  constexpr int NR = L::kRing;
  uint64_t* s_full = q_empty + S;    // [NR] per unit slot (d = 64) or per half
  uint64_t* p_full = s_full + NR;    // [NR]
  uint64_t* acc_full = p_full + NR;  // [ACB]
  uint64_t* acc_empty = acc_full + ACB;
  uint64_t* done = acc_empty + ACB;  // all MMAs complete (end of the kernel)
  float* vec = reinterpret_cast<float*>(smem + L::kVec);
  uint32_t* meta_bits = reinterpret_cast<uint32_t*>(smem + L::kMetaBits);
  int* meta_kind = reinterpret_cast<int*>(smem + L::kMetaKind);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  volatile int* drain_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 8);
  const WaitCtx wctx{p.status, p.wait_ns, abort_flag};

  if (threadIdx.x == 0) {
    for (int i = 0; i < KVB; ++i) {
      mbar_init(kv_full + i, 1);
      mbar_init(kv_empty + i, 1);
    }
    for (int i = 0; i < S; ++i) {
      mbar_init(q_full + i, 2);  // TMA bytes + the producer warp's column vectors
      mbar_init(q_empty + i, 1);
    }
    for (int i = 0; i < NR; ++i) {
      mbar_init(s_full + i, 1);
      mbar_init(p_full + i, 4);  // the four warps of one epilogue warpgroup
    }
    for (int i = 0; i < ACB; ++i) {
      mbar_init(acc_full + i, 1);
      mbar_init(acc_empty + i, 8);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    *drain_flag = 0;
    fence_barrier_init();
  }
  __syncwarp();
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    // Lane 0 waits and issues the copies.  All 32 lanes fetch the list entries of the next
    // 32 q-tiles in one round trip and the column vectors (bias / LSE / D of the tile's 128
    // queries) one tile ahead, so no global load sits between two copies.
    int qc = 0, ii = 0;
    bool ok = true;
    for (WorkIter<true> iter(p, nwork); ok && iter.valid(); iter.advance()) {
      const WorkRef it = iter.cur;
      if (it.n == 0) continue;
      const int kb = ii % KVB;
      if (lane == 0 && ii >= KVB) ok = mbar_wait(kv_empty + kb, ((ii / KVB) - 1) & 1, wctx);
      ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(kv_full + kb, 2 * L::kTileBytes);
        for (int x = 0; x < L::kBoxes; ++x) {
          tma_load_4d(smem + L::kK + kb * L::kTileBytes + x * L::kBoxBytes, &tk, kv_full + kb,
                      x * 64, it.sq.row0 + it.t * kTile, it.h, it.sq.tma_b);
          tma_load_4d(smem + L::kV + kb * L::kTileBytes + x * L::kBoxBytes, &tv, kv_full + kb,
                      x * 64, it.sq.row0 + it.t * kTile, it.h, it.sq.tma_b);
        }
      }
      ++ii;
      // column vectors of one q-tile: lane l holds queries l, l+32, l+64, l+96
      auto fetch_vec = [&](int qt, float (&v0)[4], float (&v1)[4]) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int qg = qt * kTile + lane + 32 * k;
          v0[k] = row_offset<EPI>(p, it.sq, it.b, it.h, qg);
          v1[k] = row_D<EPI>(p, it.b, it.h, qg);
        }
      };
      float cur0[4], cur1[4], nx0[4], nx1[4];
      fetch_vec(p.rowT_idx[it.e0], cur0, cur1);
      for (int i0 = 0; ok && i0 < it.n; i0 += 32) {
        const int il = i0 + lane;
        int qt_l = 0, kd_l = 0, pi_l = 0;
        if (il < it.n) {
          qt_l = p.rowT_idx[it.e0 + il];
          const int e = p.csc_map[it.e0 + il];
          kd_l = p.kind[e];
          if (kd_l == 2) pi_l = p.pidx[e];
        }
        const int jn = min(32, it.n - i0);
        for (int u = 0; u < jn; ++u, ++qc) {
          const int qt = __shfl_sync(0xFFFFFFFFu, qt_l, u);
          const int kd = __shfl_sync(0xFFFFFFFFu, kd_l, u);
          const int pi = __shfl_sync(0xFFFFFFFFu, pi_l, u);
          const int i = i0 + u;
          if (i + 1 < it.n) {  // next tile's column vectors, in flight during this tile's wait
            const int qn = (u + 1 < jn) ? __shfl_sync(0xFFFFFFFFu, qt_l, u + 1)
                                        : p.rowT_idx[it.e0 + i + 1];
            fetch_vec(qn, nx0, nx1);
          }
          const int s = qc % S;
          if (lane == 0 && qc >= S) ok = mbar_wait(q_empty + s, ((qc / S) - 1) & 1, wctx);
          ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
          if (!ok) break;
          if (lane == 0) {
            meta_kind[s] = kd;
            mbar_arrive_expect_tx(q_full + s, 2 * L::kTileBytes + (kd == 2 ? 2048 : 0));
            for (int x = 0; x < L::kBoxes; ++x) {
              tma_load_4d(smem + L::kQ + s * L::kTileBytes + x * L::kBoxBytes, &tq, q_full + s,
                          x * 64, it.sq.row0 + qt * kTile, it.h, it.sq.tma_b);
              tma_load_4d(smem + L::kDO + s * L::kTileBytes + x * L::kBoxBytes, &tdo, q_full + s,
                          x * 64, it.sq.row0 + qt * kTile, it.h, it.sq.tma_b);
            }
            if (kd == 2)
              bulk_load(meta_bits + s * 512, p.bitsT + static_cast<int64_t>(pi) * 512, 2048,
                        q_full + s);
          }
          float* vs = vec + s * 256;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            vs[lane + 32 * k] = cur0[k];
            vs[128 + lane + 32 * k] = cur1[k];
            cur0[k] = nx0[k];
            cur1[k] = nx1[k];
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(q_full + s);
        }
      }
    }
    if (lane == 0 && *abort_flag) {
      const WaitCtx drain{p.status, kDrainWaitNs, drain_flag};
      for (int u = max(0, ii - KVB); u < ii; ++u) mbar_wait(kv_full + u % KVB, (u / KVB) & 1, drain);
      for (int u = max(0, qc - S); u < qc; ++u) mbar_wait(q_full + u % S, (u / S) & 1, drain);
    }
  } else if (warp == 1 && L::kUnits) {
    // ---------------------------------------------------------------- MMA issuer (units)
    // The whole warp runs the issue loop on warp-uniform values; lane 0 waits on barriers
    // (the result is broadcast) and an elected lane issues.  Unit u: S^T / dP^T of query
    // half u % 2 of tile u / 2; issue order dV / dK of unit u - 3, then S^T / dP^T of u.
    constexpr uint32_t kHi = sw128_desc_hi(1024);
    constexpr uint32_t idesc_half = idesc_bf16_f32(128, 64, false);  // S^T / dP^T halves
    constexpr uint32_t idesc_acc = idesc_bf16_f32(128, D, true);     // dV / dK
    constexpr uint32_t kT = L::kTileBytes >> 4;
    const uint32_t k_lo0 = sw128_desc_lo(smem_u32(smem + L::kK), 16);
    const uint32_t v_lo0 = sw128_desc_lo(smem_u32(smem + L::kV), 16);
    const uint32_t q_lo0 = sw128_desc_lo(smem_u32(smem + L::kQ), 16);
    const uint32_t do_lo0 = sw128_desc_lo(smem_u32(smem + L::kDO), 16);
    const uint32_t q_mn0 = sw128_desc_lo(smem_u32(smem + L::kQ), L::kBoxBytes);
    const uint32_t do_mn0 = sw128_desc_lo(smem_u32(smem + L::kDO), L::kBoxBytes);
    static_assert(!L::kUnits || (S == 4 && KVB == 2 && ACB == 1 && NR == 4), "unit rings");
    // FIFO of the (up to three) units whose dV / dK MMAs are still to issue, oldest first:
    // stage | half << 2 | first of item << 3 | last of item << 4 | item << 5
    int f0 = 0, f1 = 0, f2 = 0;
    bool ok = true;
    // dV += P^T dO, dK += dS^T Q for unit x (buffer b = x % 3), once its warpgroup is done
    auto acc = [&](int x, uint32_t b) -> bool {
      const int info = f0;
      f0 = f1;
      f1 = f2;
      const int s = info & 3, hh = (info >> 2) & 1, item = info >> 5;
      const bool first = ((info >> 3) & 1) != 0, last = ((info >> 4) & 1) != 0;
      if (!mbar_wait_w(p_full + (x & 3), (x >> 2) & 1, wctx)) return false;
      if (first && item >= 1 && !mbar_wait_w(acc_empty, (item - 1) & 1, wctx)) return false;
      tc_fence_after();
      const uint32_t pt = tmem + b * 128;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint32_t a = (first && kk == 0) ? 0u : 1u;
        const uint32_t rows = (4 * hh + kk) * 128;  // query rows 64 hh + 16 kk (2 KB each)
        mma_ts_lh_w(tmem + 384, pt + kk * 8, do_mn0 + s * kT + rows, kHi, idesc_acc, a);
        mma_ts_lh_w(tmem + 448, pt + 64 + kk * 8, q_mn0 + s * kT + rows, kHi, idesc_acc, a);
      }
      if (hh == 1) mma_commit_w(q_empty + s);
      if (last) mma_commit_w(acc_full);
      return true;
    };
    int qc = 0, ii = 0, u = 0;
    uint32_t b3 = 0;  // u % 3
    for (WorkIter<true> iter(p, nwork); ok && iter.valid(); iter.advance()) {
      const WorkRef it = iter.cur;
      if (it.n == 0) continue;
      const int kb = ii & 1;
      if (!(ok = mbar_wait_w(kv_full + kb, (ii >> 1) & 1, wctx))) break;
      const uint32_t k_lo = k_lo0 + kb * kT, v_lo = v_lo0 + kb * kT;
      for (int i = 0; ok && i < it.n; ++i, ++qc) {
        const int s = qc & 3;
        if (!(ok = mbar_wait_w(q_full + s, (qc >> 2) & 1, wctx))) break;
        for (int hh = 0; hh < 2; ++hh, ++u) {
          // S^T / dP^T of unit u go to the buffer of unit u - 3: its dV / dK MMAs first
          if (u >= 3 && !(ok = acc(u - 3, b3))) break;
          tc_fence_after();
          const uint32_t st = tmem + b3 * 128;
          const uint32_t qh = q_lo0 + s * kT + hh * 512, dh = do_lo0 + s * kT + hh * 512;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_ss_lh_w(st, k_lo + kk * 2, qh + kk * 2, kHi, idesc_half, kk > 0 ? 1u : 0u);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_ss_lh_w(st + 64, v_lo + kk * 2, dh + kk * 2, kHi, idesc_half, kk > 0 ? 1u : 0u);
          mma_commit_w(s_full + (u & 3));
          const int info = s | (hh << 2) | ((i == 0 && hh == 0) ? 8 : 0) |
                           ((i == it.n - 1 && hh == 1) ? 16 : 0) | (ii << 5);
          if (u == 0) f0 = info;
          else if (u == 1) f1 = info;
          else f2 = info;
          b3 = b3 == 2 ? 0 : b3 + 1;
        }
      }
      if (!ok) break;
      mma_commit_w(kv_empty + kb);  // K / V feed only S^T / dP^T
      ++ii;
    }
    for (int x = max(0, u - 3); ok && x < u; ++x)
      ok = acc(x, static_cast<uint32_t>((static_cast<int>(b3) + 3 + x - u) % 3));
    // every MMA complete before the TMEM is released (also after an abort)
    mma_commit_w(done);
    {
      const WaitCtx drain{p.status, kDrainWaitNs, drain_flag};
      mbar_wait_w(done, 0, drain);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer (d = 128)
    // Whole-warp issue (see the unit schedule).  Per q-tile: S^T / dP^T of both halves, then
    // the dV / dK MMAs of half 0 and half 1 once the matching epilogue warpgroup is done,
    // which frees the tile's Q / dO stage one tile earlier and keeps the next loads ahead
    // of the MMAs.
    {
      constexpr uint32_t kHi = sw128_desc_hi(1024);
      constexpr uint32_t idesc_half = idesc_bf16_f32(128, 64, false);  // S^T / dP^T halves
      constexpr uint32_t idesc_acc = idesc_bf16_f32(128, D, true);     // dV / dK
      bool ok = true;
      // accumulating MMAs of half h of the q-tile with global index qt_, stage s, buffer ab
      auto acc_half = [&](int h, int qt_, int s, int ab, bool first, int item) -> bool {
        if (!mbar_wait_w(p_full + h, qt_ & 1, wctx)) return false;
        if (h == 0 && first && item >= ACB &&
            !mbar_wait_w(acc_empty + ab, ((item / ACB) - 1) & 1, wctx))
          return false;
        tc_fence_after();
        const uint32_t q_s = smem_u32(smem + L::kQ + s * L::kTileBytes);
        const uint32_t do_s = smem_u32(smem + L::kDO + s * L::kTileBytes);
        const uint32_t t_dv = tmem + 256 + ab * 2 * D, t_dk = t_dv + D;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint32_t acc = (first && h == 0 && kk == 0) ? 0u : 1u;
          const uint32_t boff = (4 * h + kk) * 2048;  // query rows 64h + 16kk
          mma_ts_lh_w(t_dv, tmem + 64 * h + kk * 8, sw128_desc_lo(do_s + boff, L::kBoxBytes),
                      kHi, idesc_acc, acc);
          mma_ts_lh_w(t_dk, tmem + 128 + 64 * h + kk * 8, sw128_desc_lo(q_s + boff, L::kBoxBytes),
                      kHi, idesc_acc, acc);
        }
        return true;
      };
      auto sdp_half = [&](int h, uint32_t k_base, uint32_t v_base, uint32_t q_s, uint32_t do_s) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * L::kBoxBytes + (kk & 3) * 32;
          mma_ss_lh_w(tmem + 64 * h, sw128_desc_lo(k_base + off, 16),
                      sw128_desc_lo(q_s + off + h * 8192, 16), kHi, idesc_half, kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * L::kBoxBytes + (kk & 3) * 32;
          mma_ss_lh_w(tmem + 128 + 64 * h, sw128_desc_lo(v_base + off, 16),
                      sw128_desc_lo(do_s + off + h * 8192, 16), kHi, idesc_half, kk > 0);
        }
        mma_commit_w(s_full + h);
      };
      int qc = 0, ii = 0;
      for (WorkIter<true> iter(p, nwork); ok && iter.valid(); iter.advance()) {
        const WorkRef it = iter.cur;
        if (it.n == 0) continue;
        const int kb = ii % KVB, ab = ii % ACB;
        if (!(ok = mbar_wait_w(kv_full + kb, (ii / KVB) & 1, wctx))) break;
        tc_fence_after();
        const uint32_t k_base = smem_u32(smem + L::kK + kb * L::kTileBytes);
        const uint32_t v_base = smem_u32(smem + L::kV + kb * L::kTileBytes);
        for (int i = 0; i < it.n; ++i, ++qc) {
          const int s = qc % S;
          if (!(ok = mbar_wait_w(q_full + s, (qc / S) & 1, wctx))) break;
          tc_fence_after();
          const uint32_t q_s = smem_u32(smem + L::kQ + s * L::kTileBytes);
          const uint32_t do_s = smem_u32(smem + L::kDO + s * L::kTileBytes);
          sdp_half(0, k_base, v_base, q_s, do_s);
          sdp_half(1, k_base, v_base, q_s, do_s);
          if (!(ok = acc_half(0, qc, s, ab, i == 0, ii) && acc_half(1, qc, s, ab, i == 0, ii)))
            break;
          mma_commit_w(q_empty + s);
          if (i == it.n - 1) {
            mma_commit_w(acc_full + ab);
            mma_commit_w(kv_empty + kb);
          }
        }
        ++ii;
      }
    }
    // every MMA complete before the TMEM is released (also after an abort)
    mma_commit_w(done);
    {
      const WaitCtx drain{p.status, kDrainWaitNs, drain_flag};
      mbar_wait_w(done, 0, drain);
    }
  } else if (warp >= kEpiWarp0 && L::kUnits) {
    // ---------------------------------------------------------------- epilogue (units)
    const int h = (warp - kEpiWarp0) >> 2;  // query half of every tile
    const int wq = warp & 3;
    const int row = wq * 32 + lane;  // key row of the tile
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const float c1s = p.scale * kLog2e;
    const float2 c1 = make_float2(c1s, c1s);
    constexpr int kOc = D / 2;  // dV / dK columns written by this warpgroup
    bool ok = true;
    // dV / dK of the last item with tiles, written out after the first unit of the next
    bool pend = false;
    WorkRef pit{};
    int pi = 0;
    auto flush = [&]() {
      pend = false;
      ok = ok && mbar_wait(acc_full, pi & 1, wctx);
      ok = __all_sync(0xFFFFFFFFu, ok);
      if (!ok) return;
      tc_fence_after();
      uint32_t pv[kOc / 2], pkk[kOc / 2];
      {
        uint32_t acc[32];
        tmem_ld32(t_lane + 384 + h * kOc, acc);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 16; ++c)
          pv[c] = pack_bf16x2(__uint_as_float(acc[2 * c]), __uint_as_float(acc[2 * c + 1]));
        tmem_ld32(t_lane + 448 + h * kOc, acc);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 16; ++c)
          pkk[c] = pack_bf16x2(__uint_as_float(acc[2 * c]) * p.scale,
                               __uint_as_float(acc[2 * c + 1]) * p.scale);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);
      const int kg = pit.t * kTile + row;
      if (kg < pit.sq.limit) {
        uint4* dvp = reinterpret_cast<uint4*>(p.dv + seq_row_offset(pit.sq, p.dv_sb, p.dv_sn, kg) +
                                              pit.h * p.dv_sh + h * kOc);
        uint4* dkp = reinterpret_cast<uint4*>(p.dk + seq_row_offset(pit.sq, p.dk_sb, p.dk_sn, kg) +
                                              pit.h * p.dk_sh + h * kOc);
#pragma unroll
        for (int c = 0; c < kOc / 8; ++c) {
          dvp[c] = make_uint4(pv[4 * c], pv[4 * c + 1], pv[4 * c + 2], pv[4 * c + 3]);
          dkp[c] = make_uint4(pkk[4 * c], pkk[4 * c + 1], pkk[4 * c + 2], pkk[4 * c + 3]);
        }
      }
    };
    int qc = 0, ii = 0;
    zero_empty_items<D, true>(p, nwork, nitems, warp - kEpiWarp0, lane, p.dk, p.dk_sb, p.dk_sn, p.dk_sh,
                              p.dv, p.dv_sb, p.dv_sn, p.dv_sh);
    for (WorkIter<true> iter(p, nwork); ok && iter.valid(); iter.advance()) {
      const WorkRef it = iter.cur;
      if (it.n == 0) continue;  // not in [0, nwork)
      for (int i = 0; i < it.n; ++i, ++qc) {
        const int s = qc & 3, u = 2 * qc + h;
        // q_full of the stage also publishes the kind, bitmask and column vectors
        if (ok) ok = mbar_wait(q_full + s, (qc >> 2) & 1, wctx);
        if (ok) ok = mbar_wait(s_full + (u & 3), (u >> 2) & 1, wctx);
        ok = __all_sync(0xFFFFFFFFu, ok);
        if (!ok) break;
        tc_fence_after();
        uint2 mb = make_uint2(0xFFFFFFFFu, 0xFFFFFFFFu);
        if (meta_kind[s] == 2)
          mb = *reinterpret_cast<const uint2*>(meta_bits + s * 512 + row * 4 + 2 * h);
        const float* vs = vec + s * 256 + 64 * h;
        const uint32_t base = t_lane + (u % 3) * 128;
        uint32_t sr[2][32], dpr[2][32];
        tmem_ld32(base, sr[0]);
        tmem_ld32(base + 64, dpr[0]);
        tmem_wait_ld();
        tmem_ld32(base + 32, sr[1]);
        tmem_ld32(base + 96, dpr[1]);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          if (c == 1) tmem_wait_ld();
          const uint32_t mw = c ? mb.y : mb.x;
          uint32_t pk[16], dk[16];
#pragma unroll
          for (int cc = 0; cc < 32; cc += 2) {
            float2 pw, ds;
            const float2 off2 = *reinterpret_cast<const float2*>(vs + 32 * c + cc);
            const float2 D2 = EPI == 0 ? make_float2(0.0f, 0.0f)
                                       : *reinterpret_cast<const float2*>(vs + 128 + 32 * c + cc);
            weight_grad2<EPI>(
                make_float2(__uint_as_float(sr[c][cc]), __uint_as_float(sr[c][cc + 1])),
                make_float2(__uint_as_float(dpr[c][cc]), __uint_as_float(dpr[c][cc + 1])), c1, off2,
                D2, (mw >> cc) & 1u, (mw >> (cc + 1)) & 1u, pw, ds);
            pk[cc >> 1] = pack_bf16x2(pw.x, pw.y);
            dk[cc >> 1] = pack_bf16x2(ds.x, ds.y);
          }
          tmem_st16(base + 16 * c, pk);
          tmem_st16(base + 64 + 16 * c, dk);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full + (u & 3));
        if (pend) flush();
      }
      if (!ok) break;
      pend = true;
      pit = it;
      pi = ii;
      ++ii;
    }
    if (ok && pend) flush();
  } else if (warp >= kEpiWarp0) {
    // ---------------------------------------------------------------- epilogue
    const int h = (warp - kEpiWarp0) >> 2;  // query half of every tile
    const int wq = warp & 3;
    const int row = wq * 32 + lane;  // key row of the tile
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const float c1s = p.scale * kLog2e;
    const float2 c1 = make_float2(c1s, c1s);
    bool ok = true;
    int qc = 0, ii = 0;
    zero_empty_items<D, true>(p, nwork, nitems, warp - kEpiWarp0, lane, p.dk, p.dk_sb, p.dk_sn, p.dk_sh,
                              p.dv, p.dv_sb, p.dv_sn, p.dv_sh);
    for (WorkIter<true> iter(p, nwork); iter.valid(); iter.advance()) {
      const WorkRef it = iter.cur;
      if (it.n == 0) continue;  // not in [0, nwork)
      if (!ok) break;
      const int ab = ii % ACB;
      for (int i = 0; i < it.n; ++i, ++qc) {
        const int s = qc % S;
        // q_full of the stage also publishes the kind and bitmask the producer staged
        if (ok) ok = mbar_wait(q_full + s, (qc / S) & 1, wctx);
        if (ok) ok = mbar_wait(s_full + h, qc & 1, wctx);
        ok = __all_sync(0xFFFFFFFFu, ok);
        if (!ok) break;
        tc_fence_after();
        uint2 mb = make_uint2(0xFFFFFFFFu, 0xFFFFFFFFu);
        if (meta_kind[s] == 2)
          mb = *reinterpret_cast<const uint2*>(meta_bits + s * 512 + row * 4 + 2 * h);
        const float* vs = vec + s * 256 + 64 * h;
        uint32_t sr[2][32], dpr[2][32];
        tmem_ld32(t_lane + 64 * h, sr[0]);
        tmem_ld32(t_lane + 128 + 64 * h, dpr[0]);
        tmem_wait_ld();
        tmem_ld32(t_lane + 64 * h + 32, sr[1]);
        tmem_ld32(t_lane + 128 + 64 * h + 32, dpr[1]);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          if (c == 1) tmem_wait_ld();
          const uint32_t mw = c ? mb.y : mb.x;
          uint32_t pk[16], dk[16];
#pragma unroll
          for (int cc = 0; cc < 32; cc += 2) {
            float2 pw, ds;
            const float2 off2 = *reinterpret_cast<const float2*>(vs + 32 * c + cc);
            const float2 D2 = EPI == 0 ? make_float2(0.0f, 0.0f)
                                       : *reinterpret_cast<const float2*>(vs + 128 + 32 * c + cc);
            weight_grad2<EPI>(make_float2(__uint_as_float(sr[c][cc]), __uint_as_float(sr[c][cc + 1])),
                              make_float2(__uint_as_float(dpr[c][cc]), __uint_as_float(dpr[c][cc + 1])),
                              c1, off2, D2, (mw >> cc) & 1u, (mw >> (cc + 1)) & 1u, pw, ds);
            pk[cc >> 1] = pack_bf16x2(pw.x, pw.y);
            dk[cc >> 1] = pack_bf16x2(ds.x, ds.y);
          }
          tmem_st16(t_lane + 64 * h + 16 * c, pk);
          tmem_st16(t_lane + 128 + 64 * h + 16 * c, dk);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full + h);
      }
      if (!ok) break;
      // ---- output of this item: dV, dK (this warpgroup's half of the columns)
      ok = mbar_wait(acc_full + ab, (ii / ACB) & 1, wctx);
      ok = __all_sync(0xFFFFFFFFu, ok);
      if (!ok) break;
      tc_fence_after();
      constexpr int kOc = D / 2;
      uint32_t pv[kOc / 2], pkk[kOc / 2];
#pragma unroll
      for (int c0 = 0; c0 < kOc; c0 += 32) {
        uint32_t acc[32];
        tmem_ld32(t_lane + 256 + ab * 2 * D + h * kOc + c0, acc);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 16; ++c)
          pv[c0 / 2 + c] = pack_bf16x2(__uint_as_float(acc[2 * c]), __uint_as_float(acc[2 * c + 1]));
        tmem_ld32(t_lane + 256 + ab * 2 * D + D + h * kOc + c0, acc);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 16; ++c)
          pkk[c0 / 2 + c] = pack_bf16x2(__uint_as_float(acc[2 * c]) * p.scale,
                                        __uint_as_float(acc[2 * c + 1]) * p.scale);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty + ab);
      const int kg = it.t * kTile + row;
      if (kg < it.sq.limit) {
        uint4* dvp = reinterpret_cast<uint4*>(p.dv + seq_row_offset(it.sq, p.dv_sb, p.dv_sn, kg) +
                                              it.h * p.dv_sh + h * kOc);
        uint4* dkp = reinterpret_cast<uint4*>(p.dk + seq_row_offset(it.sq, p.dk_sb, p.dk_sn, kg) +
                                              it.h * p.dk_sh + h * kOc);
#pragma unroll
        for (int c = 0; c < kOc / 8; ++c) {
          dvp[c] = make_uint4(pv[4 * c], pv[4 * c + 1], pv[4 * c + 2], pv[4 * c + 3]);
          dkp[c] = make_uint4(pkk[4 * c], pkk[4 * c + 1], pkk[4 * c + 2], pkk[4 * c + 3]);
        }
      }
      ++ii;
    }
  }
  // Single-lane roles (MMA issue, copy issue) end at different times than the rest of
  // their warp: reconverge every warp before the CTA-wide barrier, which counts warps.
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------------------
// dQ: one item = one q-tile row of the plan for one head; thread = query row.
// d = 128 TMEM: S half h [64h, 64h+64), dP half h [128+64h, ...), dQ [256, 384).
// d = 64: the unit schedule of the dK / dV kernel, with units = key halves of a tile:
// S of unit u in [128 (u % 3), +64), dP in [128 (u % 3) + 64, +64) (dS overwrites its
// first 32 columns); dQ buffer a in [384 + 64a, +64).
// ---------------------------------------------------------------------------------------
template <int D>
struct DqLayout {
  static constexpr bool kUnits = D == 64;
  static constexpr int kStages = kUnits ? 4 : 2;    // K / V ring
  static constexpr int kQBufs = D == 64 ? 2 : 1;    // Q / dO of consecutive items
  static constexpr int kAccBufs = D == 64 ? 2 : 1;  // dQ accumulators in TMEM
  static constexpr int kBoxes = D / 64;
  static constexpr int kBoxBytes = 128 * 128;
  static constexpr int kTileBytes = kBoxes * kBoxBytes;
  static constexpr int kQ = 0;
  static constexpr int kDO = kQ + kQBufs * kTileBytes;
  static constexpr int kK = kDO + kQBufs * kTileBytes;
  static constexpr int kV = kK + kStages * kTileBytes;
  // per K/V stage: the tile's PARTIAL bitmask and its kind, staged by the producer
  static constexpr int kMetaBits = kV + kStages * kTileBytes;
  static constexpr int kMetaKind = kMetaBits + kStages * 2048;
  static constexpr int kBar = kMetaKind + 16 * ((kStages * 4 + 15) / 16);
  // qd_full[QB] qd_empty[QB] kv_full[S] kv_empty[S] s_full[NR] ds_full[NR] acc_full[A]
  // acc_empty[A] (NR = 4 unit slots for d = 64, one per half for d = 128)
  static constexpr int kRing = kUnits ? 4 : 2;
  static constexpr int kNumBars = 2 * kQBufs + 2 * kStages + 2 * kRing + 2 * kAccBufs + 1;
  static constexpr int kMisc = kBar + 8 * kNumBars;
  static constexpr int kBytes = kMisc + 16;
  static constexpr int kAlloc = kBytes + 1024;
};

template <int D, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    dq_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
              const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tdo,
              const BwdParams p) {
  using L = DqLayout<D>;
  constexpr int S = L::kStages, QB = L::kQBufs, ACB = L::kAccBufs;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int warp = warp_id(), lane = lane_id();
  const int nitems = p.B * p.QT * p.H, nwork = static_cast<int>(__ldg(p.counts + kCountRows)) * p.H;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* qd_full = bars;
  uint64_t* qd_empty = qd_full + QB;
  uint64_t* kv_full = qd_empty + QB;
  uint64_t* kv_empty = kv_full + S;
  constexpr int NR = L::kRing;
  uint64_t* s_full = kv_empty + S;    // [NR] per unit slot (d = 64) or per half
  uint64_t* ds_full = s_full + NR;    // [NR]
  uint64_t* acc_full = ds_full + NR;  // [ACB]
  uint64_t* acc_empty = acc_full + ACB;
  uint64_t* done = acc_empty + ACB;  // all MMAs complete (end of the kernel)
  uint32_t* meta_bits = reinterpret_cast<uint32_t*>(smem + L::kMetaBits);
  int* meta_kind = reinterpret_cast<int*>(smem + L::kMetaKind);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  volatile int* drain_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 8);
  const WaitCtx wctx{p.status, p.wait_ns, abort_flag};

  if (threadIdx.x == 0) {
    for (int i = 0; i < QB; ++i) {
      mbar_init(qd_full + i, 1);
      mbar_init(qd_empty + i, 1);
    }
    for (int i = 0; i < S; ++i) {
      mbar_init(kv_full + i, 1);
      mbar_init(kv_empty + i, 1);
    }
    for (int i = 0; i < NR; ++i) {
      mbar_init(s_full + i, 1);
      mbar_init(ds_full + i, 4);
    }
    for (int i = 0; i < ACB; ++i) {
      mbar_init(acc_full + i, 1);
      mbar_init(acc_empty + i, 8);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    *drain_flag = 0;
    fence_barrier_init();
  }
  __syncwarp();
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    // Lane 0 waits and issues the copies; all 32 lanes fetch the list entries of the next
    // 32 k-tiles in one round trip.
    int tk_ = 0, ii = 0;
    bool ok = true;
    for (WorkIter<false> iter(p, nwork); ok && iter.valid(); iter.advance()) {
      const WorkRef it = iter.cur;
      if (it.n == 0) continue;
      const int qb = ii % QB;
      if (lane == 0) {
        if (ii >= QB) ok = mbar_wait(qd_empty + qb, ((ii / QB) - 1) & 1, wctx);
        if (ok) {
          mbar_arrive_expect_tx(qd_full + qb, 2 * L::kTileBytes);
          for (int x = 0; x < L::kBoxes; ++x) {
            tma_load_4d(smem + L::kQ + qb * L::kTileBytes + x * L::kBoxBytes, &tq, qd_full + qb,
                        x * 64, it.sq.row0 + it.t * kTile, it.h, it.sq.tma_b);
            tma_load_4d(smem + L::kDO + qb * L::kTileBytes + x * L::kBoxBytes, &tdo, qd_full + qb,
                        x * 64, it.sq.row0 + it.t * kTile, it.h, it.sq.tma_b);
          }
        }
      }
      ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      ++ii;
      for (int j0 = 0; ok && j0 < it.n; j0 += 32) {
        const int jj = j0 + lane;
        int kt_l = 0, kd_l = 0, pi_l = 0;
        if (jj < it.n) {
          kt_l = p.col_idx[it.e0 + jj];
          kd_l = p.kind[it.e0 + jj];
        }
        if (kd_l == 2) pi_l = p.pidx[it.e0 + jj];
        const int jn = min(32, it.n - j0);
        for (int u = 0; u < jn; ++u, ++tk_) {
          const int kt = __shfl_sync(0xFFFFFFFFu, kt_l, u);
          const int kd = __shfl_sync(0xFFFFFFFFu, kd_l, u);
          const int pi = __shfl_sync(0xFFFFFFFFu, pi_l, u);
          const int s = tk_ % S;
          if (lane == 0) {
            if (tk_ >= S) ok = mbar_wait(kv_empty + s, ((tk_ / S) - 1) & 1, wctx);
            if (ok) {
              meta_kind[s] = kd;
              mbar_arrive_expect_tx(kv_full + s, 2 * L::kTileBytes + (kd == 2 ? 2048 : 0));
              for (int x = 0; x < L::kBoxes; ++x) {
                tma_load_4d(smem + L::kK + s * L::kTileBytes + x * L::kBoxBytes, &tk, kv_full + s,
                            x * 64, it.sq.row0 + kt * kTile, it.h, it.sq.tma_b);
                tma_load_4d(smem + L::kV + s * L::kTileBytes + x * L::kBoxBytes, &tv, kv_full + s,
                            x * 64, it.sq.row0 + kt * kTile, it.h, it.sq.tma_b);
              }
              if (kd == 2)
                bulk_load(meta_bits + s * 512, p.bits + static_cast<int64_t>(pi) * 512, 2048,
                          kv_full + s);
            }
          }
          ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
          if (!ok) break;
        }
      }
    }
    if (lane == 0 && *abort_flag) {
      const WaitCtx drain{p.status, kDrainWaitNs, drain_flag};
      for (int u = max(0, ii - QB); u < ii; ++u) mbar_wait(qd_full + u % QB, (u / QB) & 1, drain);
      for (int u = max(0, tk_ - S); u < tk_; ++u) mbar_wait(kv_full + u % S, (u / S) & 1, drain);
    }
  } else if (warp == 1 && L::kUnits) {
    // ---------------------------------------------------------------- MMA issuer (units)
    // As in the dK / dV kernel: whole-warp issue; unit u = key half u % 2 of k-tile u / 2;
    // dQ MMAs of unit u - 3, then S / dP of unit u.
    constexpr uint32_t kHi = sw128_desc_hi(1024);
    constexpr uint32_t idesc_half = idesc_bf16_f32(128, 64, false);  // S / dP halves
    constexpr uint32_t idesc_acc = idesc_bf16_f32(128, D, true);     // dQ
    constexpr uint32_t kT = L::kTileBytes >> 4;
    const uint32_t q_lo0 = sw128_desc_lo(smem_u32(smem + L::kQ), 16);
    const uint32_t do_lo0 = sw128_desc_lo(smem_u32(smem + L::kDO), 16);
    const uint32_t k_lo0 = sw128_desc_lo(smem_u32(smem + L::kK), 16);
    const uint32_t v_lo0 = sw128_desc_lo(smem_u32(smem + L::kV), 16);
    const uint32_t k_mn0 = sw128_desc_lo(smem_u32(smem + L::kK), L::kBoxBytes);
    static_assert(!L::kUnits || (S == 4 && QB == 2 && ACB == 2 && NR == 4), "unit rings");
    // FIFO of the (up to three) units whose dQ MMAs are still to issue, oldest first:
    // stage | half << 2 | first of item << 3 | last of item << 4 | item << 5
    int f0 = 0, f1 = 0, f2 = 0;
    bool ok = true;
    // dQ += dS K for unit x (buffer b = x % 3), once its warpgroup is done
    auto acc = [&](int x, uint32_t b) -> bool {
      const int info = f0;
      f0 = f1;
      f1 = f2;
      const int s = info & 3, hh = (info >> 2) & 1, item = info >> 5, ab = item & 1;
      const bool first = ((info >> 3) & 1) != 0, last = ((info >> 4) & 1) != 0;
      if (!mbar_wait_w(ds_full + (x & 3), (x >> 2) & 1, wctx)) return false;
      if (first && item >= 2 && !mbar_wait_w(acc_empty + ab, ((item >> 1) - 1) & 1, wctx))
        return false;
      tc_fence_after();
      const uint32_t pt = tmem + b * 128 + 64;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_ts_lh_w(tmem + 384 + ab * D, pt + kk * 8, k_mn0 + s * kT + (4 * hh + kk) * 128, kHi,
                    idesc_acc, (first && kk == 0) ? 0u : 1u);
      if (hh == 1) mma_commit_w(kv_empty + s);
      if (last) mma_commit_w(acc_full + ab);
      return true;
    };
    int tc = 0, ii = 0, u = 0;
    uint32_t b3 = 0;  // u % 3
    for (WorkIter<false> iter(p, nwork); ok && iter.valid(); iter.advance()) {
      const WorkRef it = iter.cur;
      if (it.n == 0) continue;
      const int qb = ii & 1;
      if (!(ok = mbar_wait_w(qd_full + qb, (ii >> 1) & 1, wctx))) break;
      const uint32_t q_lo = q_lo0 + qb * kT, do_lo = do_lo0 + qb * kT;
      for (int j = 0; ok && j < it.n; ++j, ++tc) {
        const int s = tc & 3;
        if (!(ok = mbar_wait_w(kv_full + s, (tc >> 2) & 1, wctx))) break;
        for (int hh = 0; hh < 2; ++hh, ++u) {
          // S / dP of unit u go to the buffer of unit u - 3: its dQ MMAs first
          if (u >= 3 && !(ok = acc(u - 3, b3))) break;
          tc_fence_after();
          const uint32_t st = tmem + b3 * 128;
          const uint32_t kh = k_lo0 + s * kT + hh * 512, vh = v_lo0 + s * kT + hh * 512;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_ss_lh_w(st, q_lo + kk * 2, kh + kk * 2, kHi, idesc_half, kk > 0 ? 1u : 0u);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_ss_lh_w(st + 64, do_lo + kk * 2, vh + kk * 2, kHi, idesc_half, kk > 0 ? 1u : 0u);
          mma_commit_w(s_full + (u & 3));
          const int info = s | (hh << 2) | ((j == 0 && hh == 0) ? 8 : 0) |
                           ((j == it.n - 1 && hh == 1) ? 16 : 0) | (ii << 5);
          if (u == 0) f0 = info;
          else if (u == 1) f1 = info;
          else f2 = info;
          b3 = b3 == 2 ? 0 : b3 + 1;
        }
      }
      if (!ok) break;
      mma_commit_w(qd_empty + qb);  // Q / dO feed only S / dP
      ++ii;
    }
    for (int x = max(0, u - 3); ok && x < u; ++x)
      ok = acc(x, static_cast<uint32_t>((static_cast<int>(b3) + 3 + x - u) % 3));
    // every MMA complete before the TMEM is released (also after an abort)
    mma_commit_w(done);
    {
      const WaitCtx drain{p.status, kDrainWaitNs, drain_flag};
      mbar_wait_w(done, 0, drain);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer (d = 128)
    // Whole-warp issue; per k-tile: S / dP of both halves, then the dQ MMAs of each half
    // once the matching epilogue warpgroup is done.
    {
      constexpr uint32_t kHi = sw128_desc_hi(1024);
      constexpr uint32_t idesc_half = idesc_bf16_f32(128, 64, false);  // S / dP halves
      constexpr uint32_t idesc_acc = idesc_bf16_f32(128, D, true);     // dQ
      bool ok = true;
      auto acc_half = [&](int h, int t_, int s, int ab, bool first, int item) -> bool {
        if (!mbar_wait_w(ds_full + h, t_ & 1, wctx)) return false;
        if (h == 0 && first && item >= ACB &&
            !mbar_wait_w(acc_empty + ab, ((item / ACB) - 1) & 1, wctx))
          return false;
        tc_fence_after();
        const uint32_t k_s = smem_u32(smem + L::kK + s * L::kTileBytes);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ts_lh_w(tmem + 256 + ab * D, tmem + 128 + 64 * h + kk * 8,
                      sw128_desc_lo(k_s + (4 * h + kk) * 2048, L::kBoxBytes), kHi, idesc_acc,
                      (first && h == 0 && kk == 0) ? 0u : 1u);
        return true;
      };
      auto sdp_half = [&](int h, uint32_t q_base, uint32_t do_base, uint32_t k_s, uint32_t v_s) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * L::kBoxBytes + (kk & 3) * 32;
          mma_ss_lh_w(tmem + 64 * h, sw128_desc_lo(q_base + off, 16),
                      sw128_desc_lo(k_s + off + h * 8192, 16), kHi, idesc_half, kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * L::kBoxBytes + (kk & 3) * 32;
          mma_ss_lh_w(tmem + 128 + 64 * h, sw128_desc_lo(do_base + off, 16),
                      sw128_desc_lo(v_s + off + h * 8192, 16), kHi, idesc_half, kk > 0);
        }
        mma_commit_w(s_full + h);
      };
      int tk_ = 0, ii = 0;
      for (WorkIter<false> iter(p, nwork); ok && iter.valid(); iter.advance()) {
        const WorkRef it = iter.cur;
        if (it.n == 0) continue;
        const int qb = ii % QB, ab = ii % ACB;
        if (!(ok = mbar_wait_w(qd_full + qb, (ii / QB) & 1, wctx))) break;
        tc_fence_after();
        const uint32_t q_base = smem_u32(smem + L::kQ + qb * L::kTileBytes);
        const uint32_t do_base = smem_u32(smem + L::kDO + qb * L::kTileBytes);
        for (int j = 0; j < it.n; ++j, ++tk_) {
          const int s = tk_ % S;
          if (!(ok = mbar_wait_w(kv_full + s, (tk_ / S) & 1, wctx))) break;
          tc_fence_after();
          const uint32_t k_s = smem_u32(smem + L::kK + s * L::kTileBytes);
          const uint32_t v_s = smem_u32(smem + L::kV + s * L::kTileBytes);
          sdp_half(0, q_base, do_base, k_s, v_s);
          sdp_half(1, q_base, do_base, k_s, v_s);
          if (!(ok = acc_half(0, tk_, s, ab, j == 0, ii) && acc_half(1, tk_, s, ab, j == 0, ii)))
            break;
          mma_commit_w(kv_empty + s);
          if (j == it.n - 1) {
            mma_commit_w(acc_full + ab);
            mma_commit_w(qd_empty + qb);
          }
        }
        ++ii;
      }
    }
    // every MMA complete before the TMEM is released (also after an abort)
    mma_commit_w(done);
    {
      const WaitCtx drain{p.status, kDrainWaitNs, drain_flag};
      mbar_wait_w(done, 0, drain);
    }
  } else if (warp >= kEpiWarp0 && L::kUnits) {
    // ---------------------------------------------------------------- epilogue (units)
    const int h = (warp - kEpiWarp0) >> 2;  // key half of every tile
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const float c1s = p.scale * kLog2e;
    const float2 c1 = make_float2(c1s, c1s);
    constexpr int kOc = D / 2;  // dQ columns written by this warpgroup
    bool ok = true;
    // dQ of the last item with tiles, written out after the first unit of the next item
    bool pend = false;
    WorkRef pit{};
    int pi = 0;
    auto flush = [&]() {
      pend = false;
      const int ab = pi & 1;
      ok = ok && mbar_wait(acc_full + ab, (pi >> 1) & 1, wctx);
      ok = __all_sync(0xFFFFFFFFu, ok);
      if (!ok) return;
      tc_fence_after();
      uint32_t pk[kOc / 2];
      {
        uint32_t acc[32];
        tmem_ld32(t_lane + 384 + ab * D + h * kOc, acc);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 16; ++c)
          pk[c] = pack_bf16x2(__uint_as_float(acc[2 * c]) * p.scale,
                              __uint_as_float(acc[2 * c + 1]) * p.scale);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty + ab);
      const int qg = pit.t * kTile + row;
      if (qg < pit.sq.limit) {
        uint4* dqp = reinterpret_cast<uint4*>(p.dq + seq_row_offset(pit.sq, p.dq_sb, p.dq_sn, qg) +
                                              pit.h * p.dq_sh + h * kOc);
#pragma unroll
        for (int c = 0; c < kOc / 8; ++c)
          dqp[c] = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      }
    };
    int tc = 0, ii = 0;
    zero_empty_items<D, false>(p, nwork, nitems, warp - kEpiWarp0, lane, p.dq, p.dq_sb, p.dq_sn, p.dq_sh,
                               nullptr, 0, 0, 0);
    WorkIter<false> iter(p, nwork);
    float off_cur = 0.0f, D_cur = 0.0f;
    if (iter.valid()) {
      off_cur = row_offset<EPI>(p, iter.cur.sq, iter.cur.b, iter.cur.h, iter.cur.t * kTile + row);
      D_cur = row_D<EPI>(p, iter.cur.b, iter.cur.h, iter.cur.t * kTile + row);
    }
    for (; ok && iter.valid(); iter.advance()) {
      const WorkRef it = iter.cur;
      // the next item's row values, in flight while this one is processed
      float off_nxt = 0.0f, D_nxt = 0.0f;
      if (iter.wn < nwork && iter.nxt.n > 0) {
        off_nxt = row_offset<EPI>(p, iter.nxt.sq, iter.nxt.b, iter.nxt.h, iter.nxt.t * kTile + row);
        D_nxt = row_D<EPI>(p, iter.nxt.b, iter.nxt.h, iter.nxt.t * kTile + row);
      }
      const float off = off_cur, Drow = D_cur;
      off_cur = off_nxt;
      D_cur = D_nxt;
      if (it.n == 0) continue;  // not in [0, nwork)
      const float2 off2 = make_float2(off, off), D2 = make_float2(Drow, Drow);
      for (int j = 0; j < it.n; ++j, ++tc) {
        const int s = tc & 3, u = 2 * tc + h;
        // kv_full of the stage also publishes the kind and bitmask the producer staged
        if (ok) ok = mbar_wait(kv_full + s, (tc >> 2) & 1, wctx);
        if (ok) ok = mbar_wait(s_full + (u & 3), (u >> 2) & 1, wctx);
        ok = __all_sync(0xFFFFFFFFu, ok);
        if (!ok) break;
        tc_fence_after();
        uint2 mb = make_uint2(0xFFFFFFFFu, 0xFFFFFFFFu);
        if (meta_kind[s] == 2)
          mb = *reinterpret_cast<const uint2*>(meta_bits + s * 512 + row * 4 + 2 * h);
        const uint32_t base = t_lane + (u % 3) * 128;
        uint32_t sr[2][32], dpr[2][32];
        tmem_ld32(base, sr[0]);
        tmem_ld32(base + 64, dpr[0]);
        tmem_wait_ld();
        tmem_ld32(base + 32, sr[1]);
        tmem_ld32(base + 96, dpr[1]);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          if (c == 1) tmem_wait_ld();
          const uint32_t mw = c ? mb.y : mb.x;
          uint32_t dk[16];
#pragma unroll
          for (int cc = 0; cc < 32; cc += 2) {
            float2 pw, ds;
            weight_grad2<EPI>(
                make_float2(__uint_as_float(sr[c][cc]), __uint_as_float(sr[c][cc + 1])),
                make_float2(__uint_as_float(dpr[c][cc]), __uint_as_float(dpr[c][cc + 1])), c1, off2,
                D2, (mw >> cc) & 1u, (mw >> (cc + 1)) & 1u, pw, ds);
            dk[cc >> 1] = pack_bf16x2(ds.x, ds.y);
          }
          tmem_st16(base + 64 + 16 * c, dk);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(ds_full + (u & 3));
        if (pend) flush();
      }
      if (!ok) break;
      pend = true;
      pit = it;
      pi = ii;
      ++ii;
    }
    if (ok && pend) flush();
  } else if (warp >= kEpiWarp0) {
    // ---------------------------------------------------------------- epilogue
    const int h = (warp - kEpiWarp0) >> 2;  // key half of every tile
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const float c1s = p.scale * kLog2e;
    const float2 c1 = make_float2(c1s, c1s);
    bool ok = true;
    int tk_ = 0, ii = 0;
    zero_empty_items<D, false>(p, nwork, nitems, warp - kEpiWarp0, lane, p.dq, p.dq_sb, p.dq_sn, p.dq_sh,
                               nullptr, 0, 0, 0);
    WorkIter<false> iter(p, nwork);
    float off_cur = 0.0f, D_cur = 0.0f;
    if (iter.valid()) {
      off_cur = row_offset<EPI>(p, iter.cur.sq, iter.cur.b, iter.cur.h, iter.cur.t * kTile + row);
      D_cur = row_D<EPI>(p, iter.cur.b, iter.cur.h, iter.cur.t * kTile + row);
    }
    for (; iter.valid(); iter.advance()) {
      const WorkRef it = iter.cur;
      // the next item's row values, in flight while this one is processed
      float off_nxt = 0.0f, D_nxt = 0.0f;
      if (iter.wn < nwork && iter.nxt.n > 0) {
        off_nxt = row_offset<EPI>(p, iter.nxt.sq, iter.nxt.b, iter.nxt.h, iter.nxt.t * kTile + row);
        D_nxt = row_D<EPI>(p, iter.nxt.b, iter.nxt.h, iter.nxt.t * kTile + row);
      }
      const float off = off_cur, Drow = D_cur;
      off_cur = off_nxt;
      D_cur = D_nxt;
      if (it.n == 0) continue;  // not in [0, nwork)
      if (!ok) break;
      const int ab = ii % ACB;
      const int qg = it.t * kTile + row;
      const float2 off2 = make_float2(off, off), D2 = make_float2(Drow, Drow);
      for (int j = 0; j < it.n; ++j, ++tk_) {
        const int s = tk_ % S;
        // kv_full of the stage also publishes the kind and bitmask the producer staged
        if (ok) ok = mbar_wait(kv_full + s, (tk_ / S) & 1, wctx);
        if (ok) ok = mbar_wait(s_full + h, tk_ & 1, wctx);
        ok = __all_sync(0xFFFFFFFFu, ok);
        if (!ok) break;
        tc_fence_after();
        uint2 mb = make_uint2(0xFFFFFFFFu, 0xFFFFFFFFu);
        if (meta_kind[s] == 2)
          mb = *reinterpret_cast<const uint2*>(meta_bits + s * 512 + row * 4 + 2 * h);
        uint32_t sr[2][32], dpr[2][32];
        tmem_ld32(t_lane + 64 * h, sr[0]);
        tmem_ld32(t_lane + 128 + 64 * h, dpr[0]);
        tmem_wait_ld();
        tmem_ld32(t_lane + 64 * h + 32, sr[1]);
        tmem_ld32(t_lane + 128 + 64 * h + 32, dpr[1]);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          if (c == 1) tmem_wait_ld();
          const uint32_t mw = c ? mb.y : mb.x;
          uint32_t dk[16];
#pragma unroll
          for (int cc = 0; cc < 32; cc += 2) {
            float2 pw, ds;
            weight_grad2<EPI>(make_float2(__uint_as_float(sr[c][cc]), __uint_as_float(sr[c][cc + 1])),
                              make_float2(__uint_as_float(dpr[c][cc]), __uint_as_float(dpr[c][cc + 1])),
                              c1, off2, D2, (mw >> cc) & 1u, (mw >> (cc + 1)) & 1u, pw, ds);
            dk[cc >> 1] = pack_bf16x2(ds.x, ds.y);
          }
          tmem_st16(t_lane + 128 + 64 * h + 16 * c, dk);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(ds_full + h);
      }
      if (!ok) break;
      ok = mbar_wait(acc_full + ab, (ii / ACB) & 1, wctx);
      ok = __all_sync(0xFFFFFFFFu, ok);
      if (!ok) break;
      tc_fence_after();
      constexpr int kOc = D / 2;
      uint32_t pk[kOc / 2];
#pragma unroll
      for (int c0 = 0; c0 < kOc; c0 += 32) {
        uint32_t acc[32];
        tmem_ld32(t_lane + 256 + ab * D + h * kOc + c0, acc);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 16; ++c)
          pk[c0 / 2 + c] = pack_bf16x2(__uint_as_float(acc[2 * c]) * p.scale,
                                       __uint_as_float(acc[2 * c + 1]) * p.scale);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty + ab);
      if (qg < it.sq.limit) {
        uint4* dqp = reinterpret_cast<uint4*>(p.dq + seq_row_offset(it.sq, p.dq_sb, p.dq_sn, qg) +
                                              it.h * p.dq_sh + h * kOc);
#pragma unroll
        for (int c = 0; c < kOc / 8; ++c)
          dqp[c] = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      }
      ++ii;
    }
  }
  // Single-lane roles (MMA issue, copy issue) end at different times than the rest of
  // their warp: reconverge every warp before the CTA-wide barrier, which counts warps.
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}
// ---------------------------------------------------------------------------------------
// Fused backward (d = 64): dK, dV and dQ in one walk over the k-tile columns of the plan.
//
// Per q-tile t of a column (thread = key row in the epilogue, as in the dK / dV kernel):
//   S^T = K Q^T,  dP^T = V dO^T                  (full-width N = 128 MMAs)
//   P^T, dS^T from the epilogue                  (TMEM, bf16, A operands of the next two)
//   dV += P^T dO,  dK += dS^T Q                   (accumulated over the column in TMEM)
//   dQ_t = dS K                                   (dS from shared memory, M = queries)
// and dQ_t is added into an fp32 accumulator in global memory with TMA bulk reduce-adds, so
// S and dP are computed once per tile instead of once per kernel of the two-kernel split
// ("Better Models, Faster Training", section 2C, names that split; this is the variant it
// avoids, with the reductions done by the TMA unit instead of atomics).  A zeroing kernel
// before and a conversion kernel after (dQ = bf16(scale dQacc), pad rows 0) complete it.
//
// TMEM columns: X0 [0,128), X1 [128,256): S^T of tile t in X[t % 2]; the epilogue overwrites
// it with P^T and dS^T (bf16, interleaved per 16 queries: P at 16j + [0,8), dS at
// 16j + [8,16)); after the dV / dK MMAs have read them, dQ_t (fp32, 64 columns) is
// accumulated in X[t % 2] [0,64) and drained by the epilogue.  Y [256,384): dP^T of tile t.
// dV [384,448), dK [448,512).  The tensor pipe runs MMAs in issue order, so an MMA that
// writes columns an earlier one reads needs no barrier between them.
//
// MMA issue order: S^T / dP^T of tile t, then dV / dK / dQ of tile t - 1 -- so the next
// tile's scores are computed while the epilogue still works on the current one.
// Barriers: sdp_full (S^T, dP^T of t ready), y_free (epilogue read dP^T of t), p_full (P /
// dS of t in TMEM and dS in shared memory), dq_full (dQ_t done: its TMEM columns hold the
// result and the shared dS buffer is free), x_free (dQ_t drained, X[t % 2] free).
// ---------------------------------------------------------------------------------------
struct FusedLayout {
  static constexpr int kStages = 3;  // Q / dO ring
  static constexpr int kKVBufs = 2;  // K / V of consecutive items
  static constexpr int kTileBytes = 128 * 128;  // 128 rows x 64 bf16
  static constexpr int kK = 0;
  static constexpr int kV = kK + kKVBufs * kTileBytes;
  static constexpr int kQ = kV + kKVBufs * kTileBytes;
  static constexpr int kDO = kQ + kStages * kTileBytes;
  static constexpr int kDS = kDO + kStages * kTileBytes;       // dS, two 64-query boxes
  static constexpr int kStg = kDS + 2 * kTileBytes;            // dQ staging, 2 x 2 KB per drain warp
  static constexpr int kVec = kStg + 8 * 2048;                 // float [S][2][128]
  static constexpr int kMetaBits = kVec + kStages * 2 * 128 * 4;
  static constexpr int kMetaKind = kMetaBits + kStages * 2048;
  static constexpr int kBar = kMetaKind + 16;
  // kv_full[2] kv_empty[2] q_full[S] q_empty[S] sdp_full[2] p_full[2] dq_full[2] x_free[2]
  // y_free acc_full acc_empty done
  static constexpr int kNumBars = 4 + 2 * kStages + 8 + 4;
  static constexpr int kMisc = kBar + 8 * kNumBars;
  static constexpr int kBytes = kMisc + 16;
  static constexpr int kAlloc = kBytes + 1024;
  static_assert(kStages * 4 <= 16, "meta kinds");
};

// 14 warps: 0 producer, 1 MMA issuer, 4-11 epilogue, and 2, 3, 12, 13 the dQ drain (one
// warp per TMEM lane quarter: warp w reaches lanes [32 (w % 4), +32)).
constexpr int kFusedThreads = 448;

template <int EPI>
__global__ void __launch_bounds__(kFusedThreads, 1)
    fused_bwd_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                     const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tdo,
                     const __grid_constant__ CUtensorMap tdq, const BwdParams p) {
  using L = FusedLayout;
  constexpr int D = 64;
  constexpr int S = L::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int warp = warp_id(), lane = lane_id();
  const int nitems = p.B * p.KT * p.H, nwork = static_cast<int>(__ldg(p.counts + kCountCols)) * p.H;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = bars + 2;
  uint64_t* q_full = bars + 4;
  uint64_t* q_empty = q_full + S;
  uint64_t* sdp_full = q_empty + S;  // [2]
  uint64_t* p_full = sdp_full + 2;   // [2]
  uint64_t* dq_full = p_full + 2;    // [2]
  uint64_t* x_free = dq_full + 2;    // [2]
  uint64_t* y_free = x_free + 2;
  uint64_t* acc_full = y_free + 1;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* done = acc_empty + 1;
  float* vec = reinterpret_cast<float*>(smem + L::kVec);
  uint32_t* meta_bits = reinterpret_cast<uint32_t*>(smem + L::kMetaBits);
  int* meta_kind = reinterpret_cast<int*>(smem + L::kMetaKind);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  volatile int* drain_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 8);
  const WaitCtx wctx{p.status, p.wait_ns, abort_flag};

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(kv_full + i, 1);
      mbar_init(kv_empty + i, 1);
      mbar_init(sdp_full + i, 1);
      mbar_init(p_full + i, 8);
      mbar_init(dq_full + i, 1);
      mbar_init(x_free + i, 4);  // the four drain warps
    }
    for (int i = 0; i < S; ++i) {
      mbar_init(q_full + i, 2);  // TMA bytes + the producer's column vectors
      mbar_init(q_empty + i, 1);
    }
    mbar_init(y_free, 8);
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 8);
    mbar_init(done, 1);
    *abort_flag = 0;
    *drain_flag = 0;
    fence_barrier_init();
  }
  __syncwarp();
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  constexpr uint32_t kY = 256, kDV = 384, kDK = 448;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    // As in the dK / dV kernel: lane 0 waits and issues the copies; all lanes fetch the
    // list entries of the next 32 q-tiles at once and the column vectors one tile ahead.
    if (lane == 0) {
      tma_prefetch_desc(&tq);
      tma_prefetch_desc(&tk);
      tma_prefetch_desc(&tv);
      tma_prefetch_desc(&tdo);
    }
    int qc = 0, ii = 0;
    bool ok = true;
    for (WorkIter<true> iter(p, nwork); ok && iter.valid(); iter.advance()) {
      const WorkRef it = iter.cur;
      if (it.n == 0) continue;
      const int kb = ii & 1;
      if (lane == 0 && ii >= 2) ok = mbar_wait(kv_empty + kb, ((ii >> 1) - 1) & 1, wctx);
      ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(kv_full + kb, 2 * L::kTileBytes);
        tma_load_4d(smem + L::kK + kb * L::kTileBytes, &tk, kv_full + kb, 0, it.sq.row0 + it.t * kTile, it.h, it.sq.tma_b);
        tma_load_4d(smem + L::kV + kb * L::kTileBytes, &tv, kv_full + kb, 0, it.sq.row0 + it.t * kTile, it.h, it.sq.tma_b);
      }
      ++ii;
      auto fetch_vec = [&](int qt, float (&v0)[4], float (&v1)[4]) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int qg = qt * kTile + lane + 32 * k;
          v0[k] = row_offset<EPI>(p, it.sq, it.b, it.h, qg);
          v1[k] = row_D<EPI>(p, it.b, it.h, qg);
        }
      };
      float cur0[4], cur1[4], nx0[4], nx1[4];
      fetch_vec(p.rowT_idx[it.e0], cur0, cur1);
      for (int i0 = 0; ok && i0 < it.n; i0 += 32) {
        const int il = i0 + lane;
        int qt_l = 0, kd_l = 0, pi_l = 0;
        if (il < it.n) {
          qt_l = p.rowT_idx[it.e0 + il];
          const int e = p.csc_map[it.e0 + il];
          kd_l = p.kind[e];
          if (kd_l == 2) pi_l = p.pidx[e];
        }
        const int jn = min(32, it.n - i0);
        for (int u = 0; u < jn; ++u, ++qc) {
          const int qt = __shfl_sync(0xFFFFFFFFu, qt_l, u);
          const int kd = __shfl_sync(0xFFFFFFFFu, kd_l, u);
          const int pi = __shfl_sync(0xFFFFFFFFu, pi_l, u);
          const int i = i0 + u;
          if (i + 1 < it.n) {
            const int qn = (u + 1 < jn) ? __shfl_sync(0xFFFFFFFFu, qt_l, u + 1)
                                        : p.rowT_idx[it.e0 + i + 1];
            fetch_vec(qn, nx0, nx1);
          }
          const int s = qc % S;
          if (lane == 0 && qc >= S) ok = mbar_wait(q_empty + s, ((qc / S) - 1) & 1, wctx);
          ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
          if (!ok) break;
          if (lane == 0) {
            meta_kind[s] = kd;
            mbar_arrive_expect_tx(q_full + s, 2 * L::kTileBytes + (kd == 2 ? 2048 : 0));
            tma_load_4d(smem + L::kQ + s * L::kTileBytes, &tq, q_full + s, 0, it.sq.row0 + qt * kTile, it.h,
                        it.sq.tma_b);
            tma_load_4d(smem + L::kDO + s * L::kTileBytes, &tdo, q_full + s, 0,
                        it.sq.row0 + qt * kTile, it.h, it.sq.tma_b);
            if (kd == 2)
              bulk_load(meta_bits + s * 512, p.bitsT + static_cast<int64_t>(pi) * 512, 2048,
                        q_full + s);
          }
          float* vs = vec + s * 256;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            vs[lane + 32 * k] = cur0[k];
            vs[128 + lane + 32 * k] = cur1[k];
            cur0[k] = nx0[k];
            cur1[k] = nx1[k];
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(q_full + s);
        }
      }
    }
    if (lane == 0 && *abort_flag) {
      // Let the copies still in flight land before the CTA's shared memory goes away.
      const WaitCtx drain{p.status, kDrainWaitNs, drain_flag};
      for (int u = max(0, ii - 2); u < ii; ++u) mbar_wait(kv_full + (u & 1), (u >> 1) & 1, drain);
      for (int u = max(0, qc - S); u < qc; ++u) mbar_wait(q_full + u % S, (u / S) & 1, drain);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    constexpr uint32_t kHi = sw128_desc_hi(1024);
    constexpr uint32_t idesc_sdp = idesc_bf16_f32(128, 128, false);       // S^T, dP^T
    constexpr uint32_t idesc_acc = idesc_bf16_f32(128, D, true);          // dV, dK
    constexpr uint32_t idesc_dq = idesc_bf16_f32(128, D, true, true);     // dQ (A = dS, MN-major)
    constexpr uint32_t kT = L::kTileBytes >> 4;
    const uint32_t k_lo0 = sw128_desc_lo(smem_u32(smem + L::kK), 16);
    const uint32_t v_lo0 = sw128_desc_lo(smem_u32(smem + L::kV), 16);
    const uint32_t q_lo0 = sw128_desc_lo(smem_u32(smem + L::kQ), 16);
    const uint32_t do_lo0 = sw128_desc_lo(smem_u32(smem + L::kDO), 16);
    const uint32_t q_mn0 = sw128_desc_lo(smem_u32(smem + L::kQ), L::kTileBytes);
    const uint32_t do_mn0 = sw128_desc_lo(smem_u32(smem + L::kDO), L::kTileBytes);
    const uint32_t k_mn0 = sw128_desc_lo(smem_u32(smem + L::kK), L::kTileBytes);
    const uint32_t ds_mn = sw128_desc_lo(smem_u32(smem + L::kDS), L::kTileBytes);
    bool ok = true;
    // the tile whose dV / dK / dQ are still to issue: stage | kv buffer << 2 |
    // first of item << 3 | last of item << 4 | item << 5
    int pend = -1;
    // dV += P^T dO, dK += dS^T Q, dQ_x = dS K for tile x, once its epilogue is done
    auto acc = [&](int x, int info) -> bool {
      const int s = info & 3, kb = (info >> 2) & 1, item = info >> 5;
      const bool first = ((info >> 3) & 1) != 0, last = ((info >> 4) & 1) != 0;
      if (!mbar_wait_w(p_full + (x & 1), (x >> 1) & 1, wctx)) return false;
      if (first && item >= 1 && !mbar_wait_w(acc_empty, (item - 1) & 1, wctx)) return false;
      tc_fence_after();
      const uint32_t xb = tmem + (x & 1) * 128;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        // P^T of queries 16kk.. at columns [16kk, 16kk+8), dS^T at [16kk+8, 16kk+16)
        const uint32_t a = (first && kk == 0) ? 0u : 1u;
        mma_ts_lh_w(tmem + kDV, xb + 16 * kk, do_mn0 + s * kT + kk * 128, kHi, idesc_acc, a);
        mma_ts_lh_w(tmem + kDK, xb + 16 * kk + 8, q_mn0 + s * kT + kk * 128, kHi, idesc_acc, a);
      }
      // dQ_x = dS K: keys 16kk.. are rows 16kk.. of the dS boxes and of the K tile
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_ss_lh_w(xb, ds_mn + kk * 128, k_mn0 + kb * kT + kk * 128, kHi, idesc_dq,
                    kk > 0 ? 1u : 0u);
      mma_commit_w(q_empty + s);
      mma_commit_w(dq_full + (x & 1));
      if (last) {
        mma_commit_w(acc_full);
        mma_commit_w(kv_empty + kb);
      }
      return true;
    };
    int t = 0, ii = 0;
    for (WorkIter<true> iter(p, nwork); ok && iter.valid(); iter.advance()) {
      const WorkRef it = iter.cur;
      if (it.n == 0) continue;
      const int kb = ii & 1;
      if (!(ok = mbar_wait_w(kv_full + kb, (ii >> 1) & 1, wctx))) break;
      const uint32_t k_lo = k_lo0 + kb * kT, v_lo = v_lo0 + kb * kT;
      for (int i = 0; i < it.n; ++i, ++t) {
        const int s = t % S;
        if (!(ok = mbar_wait_w(q_full + s, (t / S) & 1, wctx))) break;
        if (t >= 2 && !(ok = mbar_wait_w(x_free + (t & 1), ((t - 2) >> 1) & 1, wctx))) break;
        if (t >= 1 && !(ok = mbar_wait_w(y_free, (t - 1) & 1, wctx))) break;
        tc_fence_after();
        const uint32_t xb = tmem + (t & 1) * 128;
        const uint32_t q_lo = q_lo0 + s * kT, do_lo = do_lo0 + s * kT;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss_lh_w(xb, k_lo + kk * 2, q_lo + kk * 2, kHi, idesc_sdp, kk > 0 ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss_lh_w(tmem + kY, v_lo + kk * 2, do_lo + kk * 2, kHi, idesc_sdp, kk > 0 ? 1u : 0u);
        mma_commit_w(sdp_full + (t & 1));
        if (pend >= 0 && !(ok = acc(t - 1, pend))) break;
        pend = s | (kb << 2) | (i == 0 ? 8 : 0) | (i == it.n - 1 ? 16 : 0) | (ii << 5);
      }
      if (!ok) break;
      ++ii;
    }
    if (ok && pend >= 0) ok = acc(t - 1, pend);
    // every MMA complete before the TMEM is released (also after an abort)
    mma_commit_w(done);
    {
      const WaitCtx drain{p.status, kDrainWaitNs, drain_flag};
      mbar_wait_w(done, 0, drain);
    }
  } else if (warp >= kEpiWarp0 && warp < kEpiWarp0 + 8) {
    // ---------------------------------------------------------------- epilogue
    // Warpgroup g owns queries [64g, 64g+64) of every tile; thread = key row (TMEM lane).
    const int g = (warp - kEpiWarp0) >> 2;
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const float c1s = p.scale * kLog2e;
    const float2 c1 = make_float2(c1s, c1s);
    uint8_t* ds_box = smem + L::kDS + g * L::kTileBytes;          // this warpgroup's queries
    bool ok = true;
    // previous item (its dV / dK are read out at the first tile of the next item)
    WorkRef pit{};
    bool have_item = false;
    int t = 0, ii = 0;
    // dV / dK of item `x` (number ix) from TMEM to global memory, bf16
    auto read_acc = [&](const WorkRef& x, int ix) {
      ok = ok && mbar_wait(acc_full, ix & 1, wctx);
      ok = __all_sync(0xFFFFFFFFu, ok);
      if (!ok) return;
      tc_fence_after();
      uint32_t av[32], ak[32];
      tmem_ld32(t_lane + kDV + 32 * g, av);
      tmem_ld32(t_lane + kDK + 32 * g, ak);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);
      const int kg = x.t * kTile + row;
      if (kg < x.sq.limit) {
        uint4* dvp = reinterpret_cast<uint4*>(p.dv + seq_row_offset(x.sq, p.dv_sb, p.dv_sn, kg) +
                                              x.h * p.dv_sh + 32 * g);
        uint4* dkp = reinterpret_cast<uint4*>(p.dk + seq_row_offset(x.sq, p.dk_sb, p.dk_sn, kg) +
                                              x.h * p.dk_sh + 32 * g);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t w0[4], w1[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int k = 8 * c + 2 * e;
            w0[e] = pack_bf16x2(__uint_as_float(av[k]), __uint_as_float(av[k + 1]));
            w1[e] = pack_bf16x2(__uint_as_float(ak[k]) * p.scale, __uint_as_float(ak[k + 1]) * p.scale);
          }
          dvp[c] = make_uint4(w0[0], w0[1], w0[2], w0[3]);
          dkp[c] = make_uint4(w1[0], w1[1], w1[2], w1[3]);
        }
      }
    };
    zero_empty_items<D, true>(p, nwork, nitems, warp - kEpiWarp0, lane, p.dk, p.dk_sb, p.dk_sn, p.dk_sh,
                              p.dv, p.dv_sb, p.dv_sn, p.dv_sh);
    for (WorkIter<true> iter(p, nwork); ok && iter.valid(); iter.advance()) {
      const WorkRef it = iter.cur;
      if (it.n == 0) continue;  // not in [0, nwork)
      for (int i = 0; i < it.n; ++i, ++t) {
        const int s = t % S;
        // q_full of the stage also publishes the kind, bitmask and column vectors
        if (ok) ok = mbar_wait(q_full + s, (t / S) & 1, wctx);
        if (ok) ok = mbar_wait(sdp_full + (t & 1), (t >> 1) & 1, wctx);
        ok = __all_sync(0xFFFFFFFFu, ok);
        if (!ok) break;
        tc_fence_after();
        uint2 mb = make_uint2(0xFFFFFFFFu, 0xFFFFFFFFu);
        if (meta_kind[s] == 2)
          mb = *reinterpret_cast<const uint2*>(meta_bits + s * 512 + row * 4 + 2 * g);
        const float* vs = vec + s * 256 + 64 * g;
        const uint32_t xb = t_lane + (t & 1) * 128 + 64 * g;
        const uint32_t yb = t_lane + kY + 64 * g;
        // four chunks of 16 queries; the TMEM loads of chunk c + 1 overlap the math of
        // chunk c.  P and dS of chunk c overwrite its own S^T columns [16c, 16c+16): P in
        // the first 8, dS in the last 8.
        uint32_t sr[2][16], dpr[2][16];
        uint32_t dsr[4][8];  // dS of the four chunks, kept for the shared-memory copy
        tmem_ld16(xb, sr[0]);
        tmem_ld16(yb, dpr[0]);
        tmem_wait_ld();
        // the chunk loop, in two versions: with the PARTIAL bitmask, and without
        auto chunks = [&](auto masked_tag) {
          constexpr bool kMasked = decltype(masked_tag)::value;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            if (c < 3) {
              tmem_ld16(xb + 16 * (c + 1), sr[(c + 1) & 1]);
              tmem_ld16(yb + 16 * (c + 1), dpr[(c + 1) & 1]);
            }
            const uint32_t mw = (c < 2 ? mb.x : mb.y) >> (16 * (c & 1));
            uint32_t pk[8];
            uint32_t (&dk)[8] = dsr[c];
#pragma unroll
            for (int cc = 0; cc < 16; cc += 2) {
              float2 pw, ds;
              const float2 off2 = *reinterpret_cast<const float2*>(vs + 16 * c + cc);
              const float2 D2 = EPI == 0 ? make_float2(0.0f, 0.0f)
                                         : *reinterpret_cast<const float2*>(vs + 128 + 16 * c + cc);
              weight_grad2<EPI>(
                  make_float2(__uint_as_float(sr[c & 1][cc]), __uint_as_float(sr[c & 1][cc + 1])),
                  make_float2(__uint_as_float(dpr[c & 1][cc]), __uint_as_float(dpr[c & 1][cc + 1])),
                  c1, off2, D2, !kMasked || ((mw >> cc) & 1u) != 0,
                  !kMasked || ((mw >> (cc + 1)) & 1u) != 0, pw, ds);
              pk[cc >> 1] = pack_bf16x2(pw.x, pw.y);
              dk[cc >> 1] = pack_bf16x2(ds.x, ds.y);
            }
            tmem_st8(xb + 16 * c, pk);
            tmem_st8(xb + 16 * c + 8, dk);
            if (c < 3) tmem_wait_ld();
            if (c == 2) {
              // every dP^T column read: the next tile's dP^T may go into Y
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(y_free);
            }
          }
        };
        if (meta_kind[s] == 2) chunks(std::true_type{});
        else chunks(std::false_type{});
        // dS into shared memory for the dQ MMA, once dQ of the previous tile has read it:
        // row = key, 64 queries of this warpgroup, 128-byte swizzled (16-byte chunk j of row
        // k at position j ^ (k % 8)), from the registers that also went to TMEM.
        if (t >= 1) ok = mbar_wait(dq_full + ((t - 1) & 1), ((t - 1) >> 1) & 1, wctx);
        ok = __all_sync(0xFFFFFFFFu, ok);
        if (!ok) break;
        {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const uint32_t* w = &dsr[j >> 1][4 * (j & 1)];
            *reinterpret_cast<uint4*>(ds_box + row * 128 + ((j ^ (row & 7)) << 4)) =
                make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
        // dV / dK of the previous item leave TMEM before this tile's dV / dK MMAs may
        // start a new accumulation
        if (i == 0 && have_item) read_acc(pit, ii - 1);
        if (!ok) break;
        fence_proxy_async_smem();
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full + (t & 1));
      }
      if (!ok) break;
      pit = it;
      have_item = true;
      ++ii;
    }
    if (ok && have_item) read_acc(pit, ii - 1);
  } else {
    // ---------------------------------------------------------------- dQ drain
    // Warps 2, 3, 12, 13: thread = query row of the dQ tile (TMEM lane).  Per tile: wait for
    // dQ_t, load its 64 fp32 columns, release X[t % 2] to the MMA warp, and add the tile into
    // the fp32 accumulator with TMA bulk reduce-adds from two 2 KB staging boxes per warp
    // (16 rows x 32 fp32, 128-byte swizzle) used alternately, so that writing one box
    // overlaps the TMA unit reading the other.
    const int wq = warp & 3;
    const int di = warp < 4 ? warp - 2 : warp - 10;  // 0..3
    uint8_t* stg = smem + L::kStg + di * 4096;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    bool ok = true;
    int t = 0;
    for (WorkIter<true> iter(p, nwork); ok && iter.valid(); iter.advance()) {
      const WorkRef it = iter.cur;
      for (int i = 0; i < it.n; ++i, ++t) {
        const int qt = p.rowT_idx[it.e0 + i];
        if (ok) ok = mbar_wait(dq_full + (t & 1), (t >> 1) & 1, wctx);
        ok = __all_sync(0xFFFFFFFFu, ok);
        if (!ok) break;
        tc_fence_after();
        uint32_t r0[32], r1[32];
        tmem_ld32(t_lane + (t & 1) * 128, r0);
        tmem_ld32(t_lane + (t & 1) * 128 + 32, r1);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(x_free + (t & 1));
#pragma unroll
        for (int part = 0; part < 4; ++part) {
          const int half = part >> 1, cg = part & 1;  // rows 16 half.., columns 32 cg..
          uint8_t* box = stg + (part & 1) * 2048;
          if (lane == 0) bulk_wait_read_1();  // the box's previous reduce has read it
          __syncwarp();
          if ((lane >> 4) == half) {
            const int rr = lane & 15;
            const uint32_t* r = cg ? r1 : r0;
#pragma unroll
            for (int j = 0; j < 8; ++j)
              *reinterpret_cast<uint4*>(box + rr * 128 + ((j ^ (rr & 7)) << 4)) =
                  make_uint4(r[4 * j], r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_reduce_add_4d(&tdq, box, 32 * cg, qt * kTile + 32 * wq + 16 * half, it.h, it.b);
            bulk_commit_group();
          }
        }
      }
    }
    if (lane == 0) bulk_wait_all();
  }
  // Single-lane roles (MMA issue, copy issue) end at different times than the rest of
  // their warp: reconverge every warp before the CTA-wide barrier, which counts warps.
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Zeroes the fp32 dQ accumulator rows of every q-tile that has tiles (the others are never
// read): rows qt*128 .. of batch entry b for each listed row r = b*QT + qt.  Block
// (k, part) takes part `part` of listed row k's span (one contiguous range of the
// [B, Nq, H, 64] accumulator), four 16-byte stores per thread in flight.
constexpr int kZeroParts = 8;
__global__ void dq_zero_kernel(const int4* __restrict__ row_desc, const int64_t* __restrict__ counts,
                               int QT, int Nq, int H, float* __restrict__ dqacc) {
  if (blockIdx.x >= counts[kCountRows]) return;  // the grid may cover every row
  const int r = row_desc[blockIdx.x].x;
  const int b = r / QT, qt = r % QT;
  const int rows = min(kTile, Nq - qt * kTile);
  float4* base = reinterpret_cast<float4*>(
      dqacc + (static_cast<int64_t>(b) * Nq + static_cast<int64_t>(qt) * kTile) * H * 64);
  const int n = rows * H * 16;  // float4 per row: 64 H / 4
  const int per = (n + kZeroParts - 1) / kZeroParts;
  const int i0 = blockIdx.y * per, i1 = min(n, i0 + per);
  for (int i = i0 + threadIdx.x; i < i1; i += blockDim.x) base[i] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
}

// dQ = bf16(scale acc) on the rows of the listed q-tiles, 0 on the others.  Block
// (qt * kConvParts + part, b) takes part `part` of the q-tile's 8-column pieces, so that the
// listed q-tiles (which read the accumulator) spread over the whole GPU instead of a few of
// them landing twice on one SM; each thread converts four pieces at a time, all loads issued
// before the stores.
constexpr int kConvParts = 8;
__global__ void dq_convert_kernel(const int32_t* __restrict__ row_ptr, const float* __restrict__ dqacc,
                                  int QT, int Nq, int H, const int32_t* __restrict__ cu,
                                  float scale, __nv_bfloat16* __restrict__ dq, int64_t sb, int64_t sn,
                                  int64_t sh) {
  const int qt = blockIdx.x / kConvParts, part = blockIdx.x % kConvParts, b = blockIdx.y;
  const SeqRows sq = seq_rows(cu, b, Nq);
  const int rows = min(kTile, sq.limit - qt * kTile);  // a packed sequence owns only its rows
  if (rows <= 0) return;
  const int r = b * QT + qt;
  const bool listed = row_ptr[r + 1] > row_ptr[r];
  const int per_row = H * 8;
  const int n_all = rows * per_row;
  const int per = (n_all + kConvParts - 1) / kConvParts;
  const int i_begin = part * per, n = min(n_all, i_begin + per);
  constexpr int kU = 4;
  for (int i0 = i_begin + threadIdx.x; i0 < n; i0 += kU * blockDim.x) {
    float4 a[kU], e[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int i = i0 + u * blockDim.x;
      a[u] = e[u] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      if (listed && i < n) {
        const int rr = i / per_row, hc = i - rr * per_row;
        const float4* src = reinterpret_cast<const float4*>(
            dqacc + ((static_cast<int64_t>(b) * Nq + qt * kTile + rr) * H + (hc >> 3)) * 64 +
            (hc & 7) * 8);
        a[u] = src[0];
        e[u] = src[1];
      }
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int i = i0 + u * blockDim.x;
      if (i < n) {
        const int rr = i / per_row, hc = i - rr * per_row;
        *reinterpret_cast<uint4*>(dq + seq_row_offset(sq, sb, sn, qt * kTile + rr) + (hc >> 3) * sh +
                                  (hc & 7) * 8) =
            make_uint4(pack_bf16x2(a[u].x * scale, a[u].y * scale),
                       pack_bf16x2(a[u].z * scale, a[u].w * scale),
                       pack_bf16x2(e[u].x * scale, e[u].y * scale),
                       pack_bf16x2(e[u].z * scale, e[u].w * scale));
      }
    }
  }
}

int num_sms() {
  static int sms = 0;
  static std::once_flag once;
  std::call_once(once, [] {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      sms = 148;
    }
  });
  return sms;
}

template <int D, int EPI>
int launch_bwd_t(const sigattn_plan* plan, int H, float scale, const CUtensorMap& tq,
                 const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tdo,
                 const TensorDesc& o, const TensorDesc& dout, const float* bias, int64_t bias_sb,
                 const float* lse, float* workspace, const TensorDesc& dq, const TensorDesc& dk,
                 const TensorDesc& dv, int parts, int* status, unsigned long long wait_ns,
                 cudaStream_t stream) {
  BwdParams p;
  p.row_ptr = plan->row_ptr;
  p.col_idx = plan->col_idx;
  p.kind = plan->kind;
  p.pidx = plan->pidx;
  p.bits = plan->bits;
  p.bitsT = plan->bitsT;
  p.colT_ptr = plan->colT_ptr;
  p.rowT_idx = plan->rowT_idx;
  p.csc_map = plan->csc_map;
  p.row_desc = plan->row_desc;
  p.col_desc = plan->col_desc;
  p.cu = plan->cu;
  p.B = plan->B;
  p.QT = plan->QT;
  p.KT = plan->KT;
  p.counts = plan->dcount;
  p.Nq = plan->Nq;
  p.Nk = plan->Nk;
  p.H = H;
  p.scale = scale;
  p.bias = bias;
  p.bias_sb = bias_sb;
  p.lse = lse;
  p.Dws = workspace;
  p.dq = static_cast<__nv_bfloat16*>(const_cast<void*>(dq.ptr));
  p.dq_sb = dq.sb;
  p.dq_sn = dq.sn;
  p.dq_sh = dq.sh;
  p.dk = static_cast<__nv_bfloat16*>(const_cast<void*>(dk.ptr));
  p.dk_sb = dk.sb;
  p.dk_sn = dk.sn;
  p.dk_sh = dk.sh;
  p.dv = static_cast<__nv_bfloat16*>(const_cast<void*>(dv.ptr));
  p.dv_sb = dv.sb;
  p.dv_sn = dv.sn;
  p.dv_sh = dv.sh;
  p.status = status;
  p.wait_ns = wait_ns;
  cudaError_t e;
  if (EPI != 0 && (parts & SIGATTN_BWD_PREP)) {
    const int64_t threads = static_cast<int64_t>(plan->B) * plan->Nq * H * (D / 8);
    d_preprocess_kernel<D><<<static_cast<unsigned>((threads + 255) / 256), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(o.ptr), o.sb, o.sn, o.sh,
        static_cast<const __nv_bfloat16*>(dout.ptr), dout.sb, dout.sn, dout.sh, plan->B, plan->Nq,
        H, plan->cu, workspace);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_status(e);
  }
  if (parts & SIGATTN_BWD_DKDV) {
    auto kdkv = dkdv_kernel<D, EPI>;
    if ((e = cudaFuncSetAttribute(kdkv, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  DkvLayout<D>::kAlloc)) != cudaSuccess)
      return cuda_status(e);
    const int items = plan->B * plan->KT * H;
    kdkv<<<std::min(items, num_sms()), kThreads, DkvLayout<D>::kAlloc, stream>>>(tq, tk, tv, tdo, p);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_status(e);
  }
  if (parts & SIGATTN_BWD_DQ) {
    auto kdq = dq_kernel<D, EPI>;
    if ((e = cudaFuncSetAttribute(kdq, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  DqLayout<D>::kAlloc)) != cudaSuccess)
      return cuda_status(e);
    const int items = plan->B * plan->QT * H;
    kdq<<<std::min(items, num_sms()), kThreads, DqLayout<D>::kAlloc, stream>>>(tq, tk, tv, tdo, p);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_status(e);
  }
  return SIGATTN_OK;
}

}  // namespace

int launch_bwd_fused_impl(const sigattn_plan* plan, int epilogue, int H, float scale,
                          const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                          const CUtensorMap& tdo, const CUtensorMap& tdq, const TensorDesc& o,
                          const TensorDesc& dout, const float* bias, int64_t bias_sb,
                          const float* lse, float* Dws, float* dqacc, const TensorDesc& dq,
                          const TensorDesc& dk, const TensorDesc& dv, int* status,
                          unsigned long long wait_ns, cudaStream_t stream) {
  constexpr int D = 64;
  BwdParams p{};
  p.rowT_idx = plan->rowT_idx;
  p.csc_map = plan->csc_map;
  p.kind = plan->kind;
  p.pidx = plan->pidx;
  p.bitsT = plan->bitsT;
  p.col_desc = plan->col_desc;
  p.row_desc = plan->row_desc;
  p.cu = plan->cu;
  p.B = plan->B;
  p.QT = plan->QT;
  p.KT = plan->KT;
  p.counts = plan->dcount;
  p.Nq = plan->Nq;
  p.Nk = plan->Nk;
  p.H = H;
  p.scale = scale;
  p.bias = bias;
  p.bias_sb = bias_sb;
  p.lse = lse;
  p.Dws = Dws;
  p.dk = static_cast<__nv_bfloat16*>(const_cast<void*>(dk.ptr));
  p.dk_sb = dk.sb;
  p.dk_sn = dk.sn;
  p.dk_sh = dk.sh;
  p.dv = static_cast<__nv_bfloat16*>(const_cast<void*>(dv.ptr));
  p.dv_sb = dv.sb;
  p.dv_sn = dv.sn;
  p.dv_sh = dv.sh;
  p.status = status;
  p.wait_ns = wait_ns;
  cudaError_t e;
  if (epilogue != 0) {
    const int64_t threads = static_cast<int64_t>(plan->B) * plan->Nq * H * (D / 8);
    d_preprocess_kernel<D><<<static_cast<unsigned>((threads + 255) / 256), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(o.ptr), o.sb, o.sn, o.sh,
        static_cast<const __nv_bfloat16*>(dout.ptr), dout.sb, dout.sn, dout.sh, plan->B, plan->Nq,
        H, plan->cu, Dws);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_status(e);
  }
  const int sms = num_sms();
  // one block per listed row: the count is on the device when the host has not read it
  const int zero_rows = plan->counts_known ? plan->rows_nonempty : plan->B * plan->QT;
  if (zero_rows > 0) {
    dq_zero_kernel<<<dim3(zero_rows, kZeroParts), 256, 0, stream>>>(
        plan->row_desc, plan->dcount, plan->QT, plan->Nq, H, dqacc);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_status(e);
  }
  static_assert(FusedLayout::kAlloc <= 227 * 1024, "shared memory");
  {
    auto kern = epilogue == 0 ? fused_bwd_kernel<0>
                              : (epilogue == 1 ? fused_bwd_kernel<1> : fused_bwd_kernel<2>);
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  FusedLayout::kAlloc)) != cudaSuccess)
      return cuda_status(e);
    const int items = plan->B * plan->KT * H;
    kern<<<std::min(items, sms), kFusedThreads, FusedLayout::kAlloc, stream>>>(tq, tk, tv, tdo, tdq, p);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_status(e);
  }
  {
    dq_convert_kernel<<<dim3(plan->QT * kConvParts, plan->B), 256, 0, stream>>>(plan->row_ptr, dqacc, plan->QT,
                                                                     plan->Nq, H, plan->cu, scale,
                                                   static_cast<__nv_bfloat16*>(const_cast<void*>(dq.ptr)),
                                                   dq.sb, dq.sn, dq.sh);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_status(e);
  }
  return SIGATTN_OK;
}

int launch_bwd_impl(const sigattn_plan* plan, int epilogue, int H, int d, float scale,
                    const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                    const CUtensorMap& tdo, const TensorDesc& o, const TensorDesc& dout,
                    const float* bias, int64_t bias_sb, const float* lse, float* workspace,
                    const TensorDesc& dq, const TensorDesc& dk, const TensorDesc& dv, int parts,
                    int* status, unsigned long long wait_ns, cudaStream_t stream) {
#define SIGATTN_BWD_CASE(DD, EE)                                                              \
  if (d == DD && epilogue == EE)                                                              \
    return launch_bwd_t<DD, EE>(plan, H, scale, tq, tk, tv, tdo, o, dout, bias, bias_sb, lse, \
                                workspace, dq, dk, dv, parts, status, wait_ns, stream);
  SIGATTN_BWD_CASE(64, 0)
  SIGATTN_BWD_CASE(64, 1)
  SIGATTN_BWD_CASE(64, 2)
  SIGATTN_BWD_CASE(128, 0)
  SIGATTN_BWD_CASE(128, 1)
  SIGATTN_BWD_CASE(128, 2)
#undef SIGATTN_BWD_CASE
  return SIGATTN_ERR_UNSUPPORTED;
}

}  // namespace sigattn

// ---------------------------------------------------------------------------------------
// Allocation-free backward.  Callers that cannot call cudaMalloc (see sigattn.h) get the
// softmax modes' D workspace from this array instead of passing one in.  It is part of the
// library's device image, so every GPU that loads the library holds it until exit.
// ---------------------------------------------------------------------------------------
static __device__ __align__(256) float g_noalloc_scratch[SIGATTN_NOALLOC_MAX_ROWS];

namespace {

sigattn::SymbolAddressCache g_noalloc_addr;

// Device address of g_noalloc_scratch on the current device (looked up once per device,
// with that device current; see SymbolAddressCache).
int noalloc_scratch(float** out) {
  void* p = nullptr;
  const int rc = g_noalloc_addr.get(g_noalloc_scratch, &p);
  *out = static_cast<float*>(p);
  return rc;
}

}  // namespace

extern "C" int sigattn_bwd_noalloc(const sigattn_plan* plan, int epilogue, int H, int d,
                                   float scale, const void* q, const int64_t q_strides[3],
                                   const void* k, const int64_t k_strides[3], const void* v,
                                   const int64_t v_strides[3], const void* o,
                                   const int64_t o_strides[3], const void* dout,
                                   const int64_t do_strides[3], const float* bias,
                                   int64_t bias_stride_b, const float* lse, void* dq,
                                   const int64_t dq_strides[3], void* dk,
                                   const int64_t dk_strides[3], void* dv,
                                   const int64_t dv_strides[3], sigattn_stream stream) {
  if (!plan || H < 1) return SIGATTN_ERR_INVALID;
  float* workspace = nullptr;
  if (epilogue == SIGATTN_SOFTMAX || epilogue == SIGATTN_SOFTMAX1) {
    // The D preprocess writes every one of the B * H * Nq values before the two gradient
    // kernels read them, so the array needs no clearing between calls.
    if (static_cast<int64_t>(plan->B) * H * plan->Nq > SIGATTN_NOALLOC_MAX_ROWS)
      return SIGATTN_ERR_UNSUPPORTED;
    const int rc = noalloc_scratch(&workspace);
    if (rc != SIGATTN_OK) return rc;
  }
  return sigattn_bwd_ex(plan, epilogue, H, d, scale, q, q_strides, k, k_strides, v, v_strides, o,
                        o_strides, dout, do_strides, bias, bias_stride_b, lse, workspace, dq,
                        dq_strides, dk, dk_strides, dv, dv_strides, SIGATTN_BWD_ALL, stream);
}
