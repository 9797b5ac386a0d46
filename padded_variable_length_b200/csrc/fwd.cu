// Forward kernels: fused tiled sigmoid (fwd_sigmoid_kernel, below) and softmax / softmax_1
// (fwd_kernel) attention over the tile list of a plan, sm_100a.
//
// Method: "Better Models, Faster Training: Sigmoid Attention for single-cell Foundation
// Models", section 2A: O = sigma(Q K^T / sqrt(d) + b) V, each weight computed on its own
// with no row normalisation; section 2C: one fused kernel that skips every tile that is
// padding on the query or the key side.  The sigmoid is evaluated as in sm100.cuh
// (sigmoid2: hardware exp2 plus a polynomial reciprocal, accurate in relative terms for
// the tiny weights that b = -log n gives long sequences) instead of the page's hardware
// tanh, which loses them.  softmax and softmax_1 (the QuietAttention page, section
// "Proposition : softmax_1 et QuietAttention") run through the same kernel with the online
// max / sum recombination of the FlashAttention article (section on the mathematics of
// blockwise softmax); softmax_1 starts from a zero logit whose value row is zero (m = 0,
// l = 1).
//
// Persistent: one CTA per SM walks the plan's longest-first list of (q-tile row, head)
// work items in snake order (even rounds forward, odd rounds backward over the grid).
// All tiles of all of a CTA's items form one stream.  fwd_kernel (softmax modes): the
// S = Q K^T of tile t is issued before the O += P V of tile t - 1, also across item
// boundaries, so the tensor pipe works on the next item while the epilogue finishes the
// last one.  384 threads:
//   warp 0      TMA producer: Q of each item (two buffers), K and V tiles into a ring
//   warp 1      TMEM allocator and MMA issuer (whole warp, one elected lane issues)
//   warps 4-11  two epilogue warpgroups; thread = query row (TMEM lane); warpgroup g
//               owns S columns [64g, 64g+64) and O columns [g d/2, (g+1) d/2)
// TMEM columns: S0 [0,128), S1 [128,256), O0 [256, 256+d), O1 [256+d, 256+2d).  P (bf16)
// overwrites the first half of the S columns each warpgroup read and is the TMEM A
// operand of the PV MMA.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>
#include <mutex>

#include "internal.h"
#include "sm100.cuh"

namespace sigattn {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kNegBig = -1.0e30f;
constexpr int kThreads = 384;
constexpr int kEpiWarp0 = 4;

struct FwdParams {
  const int32_t* row_ptr;
  const int32_t* col_idx;
  const uint8_t* kind;
  const int32_t* pidx;
  const uint32_t* bits;
  const int4* row_desc;
  const int32_t* cu;  // packed batches: cumulative row offsets [B + 1]; nullptr when padded
  const int4* run;  // runs of consecutive k-tiles of one kind (see sigattn_plan)
  int run_cap;      // entries allocated in run (reads stay below it)
  int QT, Nq, H;
  int nitems;  // B QT H items: (q-tile row, head), in the order of the longest-first list
  // the first counts[kCountRows] * H items have tiles; the rest are empty (the plan's
  // device counts: its build need not have been waited for on the host)
  const int64_t* counts;
  int zero_tma;  // sigmoid kernel: zero rows of the empty items by tensor-map stores of O
  float scale;
  const float* bias;
  int64_t bias_sb;
  __nv_bfloat16* o;
  int64_t o_sb, o_sn, o_sh;
  float* lse;
  int* status;
  unsigned long long wait_ns;
};

template <int D>
struct FwdLayout {
  static constexpr int kStages = D == 64 ? 4 : 2;
  static constexpr int kBoxes = D / 64;
  static constexpr int kBoxBytes = 128 * 128;  // 128 rows x 64 bf16
  static constexpr int kTileBytes = kBoxes * kBoxBytes;
  static constexpr int kQ = 0;                  // two Q buffers
  static constexpr int kK = 2 * kTileBytes;
  static constexpr int kV = kK + kStages * kTileBytes;
  // per K/V stage: the tile's PARTIAL bitmask (2 KB) and its kind, staged by the producer
  static constexpr int kMetaBits = kV + kStages * kTileBytes;
  static constexpr int kMetaKind = kMetaBits + kStages * 2048;
  static constexpr int kBar = kMetaKind + 16 * ((kStages * 4 + 15) / 16);
  // q_full[2] q_empty[2] o_full[2] o_empty[2] s_full[2] p_full[2] pv_done
  // k_full[S] v_full[S] kv_empty[S] done
  static constexpr int kNumBars = 14 + 3 * kStages;
  static constexpr int kRed = kBar + 8 * kNumBars;      // float [2][2][128] row maxima
  static constexpr int kRedL = kRed + 2 * 2 * 128 * 4;  // float [2][128] row sums
  static constexpr int kMisc = kRedL + 2 * 128 * 4;      // tmem base, abort, drain flags
  static constexpr int kBytes = kMisc + 16;
  static constexpr int kAlloc = kBytes + 1024;           // slack for 1024-byte alignment
};

struct Item {
  int b, qt, h, e0, n, run0;  // run0: the row's first run
  SeqRows sq;                 // where the rows of sequence b live (padded or packed)
};

__device__ __forceinline__ Item decode_item(const FwdParams& p, int w) {
  Item it;
  const int4 d = p.row_desc[w / p.H];
  it.h = w % p.H;
  it.b = d.x / p.QT;
  it.qt = d.x % p.QT;
  it.e0 = d.y;
  it.n = d.z;
  it.run0 = d.w;
  it.sq = seq_rows(p.cu, it.b, p.Nq);
  return it;
}

// Walks this CTA's items with tiles (snake order over [0, nwork), see snake_item) with the
// next item's decode issued one item ahead, so that its global loads overlap the current
// item.
struct ItemIter {
  const FwdParams& p;
  int nw;        // items with tiles
  int k, w, wn;  // round, this item, next item
  Item cur, nxt;
  __device__ ItemIter(const FwdParams& pp, int nwork)
      : p(pp), nw(nwork), k(0), w(snake_item(0)), wn(snake_item(1)) {
    if (w < nw) cur = decode_item(p, w);
    if (wn < nw) nxt = decode_item(p, wn);
  }
  __device__ bool valid() const { return w < nw; }
  __device__ void advance() {
    ++k;
    w = wn;
    wn = snake_item(k + 1);
    cur = nxt;
    if (wn < nw) nxt = decode_item(p, wn);
  }
};

// O = 0 on the rows of the items without tiles, [nwork, nitems) of the longest-first list:
// q-tiles past their sequence's length, or whose rows see no key (and, for the softmax
// modes, LSE = -inf resp. 0 there).  The items are dealt round-robin to every epilogue warp
// of the grid, one item per warp at a time, with no dependent loads between them; run
// before the first tile, while the epilogue would otherwise wait for its first S.  The
// sigmoid kernel uses this for packed layouts only: on padded ones its tile-kind producer
// writes these rows with tensor-map stores in the background.
template <int D, int EPI>
__device__ void zero_empty_items(const FwdParams& p, int nwork, int ew, int lane) {
  constexpr int kChunks = D / 8;
  const int stride = static_cast<int>(gridDim.x) * 8;
  for (int w = nwork + static_cast<int>(blockIdx.x) * 8 + ew; w < p.nitems; w += stride) {
    const Item x = decode_item(p, w);
    const int rows = min(kTile, x.sq.limit - x.qt * kTile);
    for (int c = lane; c < rows * kChunks; c += 32)
      *reinterpret_cast<uint4*>(p.o + seq_row_offset(x.sq, p.o_sb, p.o_sn, x.qt * kTile + c / kChunks) +
                                x.h * p.o_sh + (c % kChunks) * 8) = make_uint4(0u, 0u, 0u, 0u);
    if constexpr (EPI != 0) {
      for (int c = lane; c < min(kTile, p.Nq - x.qt * kTile); c += 32)
        p.lse[(static_cast<int64_t>(x.b) * p.H + x.h) * p.Nq + x.qt * kTile + c] =
            EPI == 1 ? -INFINITY : 0.0f;
    }
  }
}

template <int D, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
               const __grid_constant__ CUtensorMap tv, const FwdParams p) {
  using L = FwdLayout<D>;
  constexpr int S = L::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int warp = warp_id(), lane = lane_id();
  const int nwork = static_cast<int>(__ldg(p.counts + kCountRows)) * p.H;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* q_full = bars + 0;    // [2]
  uint64_t* q_empty = bars + 2;   // [2]
  uint64_t* o_full = bars + 4;    // [2]
  uint64_t* o_empty = bars + 6;   // [2]
  uint64_t* s_full = bars + 8;    // [2]
  uint64_t* p_full = bars + 10;   // [2]
  uint64_t* pv_done = bars + 12;
  uint64_t* k_full = bars + 13;   // [S]
  uint64_t* v_full = bars + 13 + S;
  uint64_t* kv_empty = bars + 13 + 2 * S;
  uint64_t* done = bars + 13 + 3 * S;  // every MMA complete (end of the kernel)
  uint32_t* meta_bits = reinterpret_cast<uint32_t*>(smem + L::kMetaBits);
  int* meta_kind = reinterpret_cast<int*>(smem + L::kMetaKind);
  float* red_max = reinterpret_cast<float*>(smem + L::kRed);
  float* red_l = reinterpret_cast<float*>(smem + L::kRedL);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  volatile int* drain_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 8);
  const WaitCtx wctx{p.status, p.wait_ns, abort_flag};

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(q_full + i, 1);
      mbar_init(q_empty + i, 1);
      mbar_init(o_full + i, 1);
      mbar_init(o_empty + i, 8);
      mbar_init(s_full + i, 1);
      mbar_init(p_full + i, 8);
    }
    mbar_init(pv_done, 1);
    for (int i = 0; i < S; ++i) {
      mbar_init(k_full + i, 1);
      mbar_init(v_full + i, 1);
      mbar_init(kv_empty + i, 1);
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
    // ---------------------------------------------------------------- TMA producer
    // Lane 0 waits and issues the copies; all 32 lanes fetch the list entries of the next
    // 32 tiles in one round trip, so index loads never sit between two copies.
    if (lane == 0) {
      tma_prefetch_desc(&tq);
      tma_prefetch_desc(&tk);
      tma_prefetch_desc(&tv);
    }
    int t = 0, i = 0;
    bool ok = true;
    for (ItemIter iter(p, nwork); ok && iter.valid(); iter.advance()) {
      const Item it = iter.cur;
      if (it.n == 0) continue;
      const int qb = i & 1;
      if (lane == 0) {
        if (i >= 2) ok = mbar_wait(q_empty + qb, ((i >> 1) - 1) & 1, wctx);
        if (ok) {
          mbar_arrive_expect_tx(q_full + qb, L::kTileBytes);
          for (int x = 0; x < L::kBoxes; ++x)
            tma_load_4d(smem + L::kQ + qb * L::kTileBytes + x * L::kBoxBytes, &tq, q_full + qb,
                        x * 64, it.sq.row0 + it.qt * kTile, it.h, it.sq.tma_b);
        }
      }
      ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      ++i;
      for (int j0 = 0; ok && j0 < it.n; j0 += 32) {
        const int jj = j0 + lane;
        int kt_l = 0, kd_l = 0, pi_l = 0;
        if (jj < it.n) {
          kt_l = p.col_idx[it.e0 + jj];
          kd_l = p.kind[it.e0 + jj];
        }
        if (kd_l == 2) pi_l = p.pidx[it.e0 + jj];
        const int jn = min(32, it.n - j0);
        for (int u = 0; u < jn; ++u, ++t) {
          const int kt = __shfl_sync(0xFFFFFFFFu, kt_l, u);
          const int kd = __shfl_sync(0xFFFFFFFFu, kd_l, u);
          const int pi = __shfl_sync(0xFFFFFFFFu, pi_l, u);
          const int s = t % S;
          if (lane == 0) {
            if (t >= S) ok = mbar_wait(kv_empty + s, ((t / S) - 1) & 1, wctx);
            if (ok) {
              meta_kind[s] = kd;
              mbar_arrive_expect_tx(k_full + s, L::kTileBytes + (kd == 2 ? 2048 : 0));
              for (int x = 0; x < L::kBoxes; ++x)
                tma_load_4d(smem + L::kK + s * L::kTileBytes + x * L::kBoxBytes, &tk, k_full + s,
                            x * 64, it.sq.row0 + kt * kTile, it.h, it.sq.tma_b);
              if (kd == 2)
                bulk_load(meta_bits + s * 512, p.bits + static_cast<int64_t>(pi) * 512, 2048,
                          k_full + s);
              mbar_arrive_expect_tx(v_full + s, L::kTileBytes);
              for (int x = 0; x < L::kBoxes; ++x)
                tma_load_4d(smem + L::kV + s * L::kTileBytes + x * L::kBoxBytes, &tv, v_full + s,
                            x * 64, it.sq.row0 + kt * kTile, it.h, it.sq.tma_b);
            }
          }
          ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
          if (!ok) break;
        }
      }
    }
    if (lane == 0 && *abort_flag) {
      // Let the copies still in flight land before the CTA's shared memory goes away.
      const WaitCtx drain{p.status, kDrainWaitNs, drain_flag};
      for (int u = max(0, i - 2); u < i; ++u) mbar_wait(q_full + (u & 1), (u >> 1) & 1, drain);
      for (int u = max(0, t - S); u < t; ++u) {
        mbar_wait(k_full + u % S, (u / S) & 1, drain);
        mbar_wait(v_full + u % S, (u / S) & 1, drain);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    // Whole-warp issue from warp-uniform values (see mma_ss_lh_w).
    {
      constexpr uint32_t kHi = sw128_desc_hi(1024);
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, true);
      // the PV still to issue: its global tile, item number and place in the item
      int pv_t = -1, pv_item = 0;
      bool pv_first = false, pv_last = false;
      bool ok = true;
      auto issue_pv = [&]() -> bool {
        const int pb = pv_t & 1, s2 = pv_t % S, ob = pv_item & 1;
        if (!mbar_wait_w(p_full + pb, (pv_t >> 1) & 1, wctx)) return false;
        if (!mbar_wait_w(v_full + s2, (pv_t / S) & 1, wctx)) return false;
        if (pv_first && pv_item >= 2 && !mbar_wait_w(o_empty + ob, ((pv_item >> 1) - 1) & 1, wctx))
          return false;
        tc_fence_after();
        const uint32_t v_base = smem_u32(smem + L::kV + s2 * L::kTileBytes);
        const uint32_t o_tmem = tmem + 256 + ob * D;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          // warpgroup g wrote the P of keys [64g, 64g+64) at columns [64g, 64g+32)
          const uint32_t a_tmem = tmem + pb * 128 + (kk >> 2) * 64 + (kk & 3) * 8;
          mma_ts_lh_w(o_tmem, a_tmem, sw128_desc_lo(v_base + kk * 2048, L::kBoxBytes), kHi,
                      idesc_pv, (pv_first && kk == 0) ? 0u : 1u);
        }
        mma_commit_w(kv_empty + s2);
        if (EPI != 0) mma_commit_w(pv_done);
        if (pv_last) mma_commit_w(o_full + ob);
        return true;
      };
      int t = 0, i = 0;
      for (ItemIter iter(p, nwork); ok && iter.valid(); iter.advance()) {
        const Item it = iter.cur;
        if (it.n == 0) continue;
        const int qb = i & 1;
        if (!(ok = mbar_wait_w(q_full + qb, (i >> 1) & 1, wctx))) break;
        tc_fence_after();
        const uint32_t q_base = smem_u32(smem + L::kQ + qb * L::kTileBytes);
        for (int j = 0; j < it.n; ++j, ++t) {
          const int s = t % S;
          if (!(ok = mbar_wait_w(k_full + s, (t / S) & 1, wctx))) break;
          tc_fence_after();
          const uint32_t k_base = smem_u32(smem + L::kK + s * L::kTileBytes);
          const uint32_t d_tmem = tmem + (t & 1) * 128;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * L::kBoxBytes + (kk & 3) * 32;
            mma_ss_lh_w(d_tmem, sw128_desc_lo(q_base + off, 16), sw128_desc_lo(k_base + off, 16),
                        kHi, idesc_qk, kk > 0);
          }
          mma_commit_w(s_full + (t & 1));
          if (j == it.n - 1) mma_commit_w(q_empty + qb);
          if (pv_t >= 0 && !(ok = issue_pv())) break;
          pv_t = t;
          pv_item = i;
          pv_first = j == 0;
          pv_last = j == it.n - 1;
        }
        ++i;
      }
      if (ok && pv_t >= 0) issue_pv();
      // every MMA complete before the TMEM is released (also after an abort)
      mma_commit_w(done);
      const WaitCtx drain{p.status, kDrainWaitNs, drain_flag};
      mbar_wait_w(done, 0, drain);
    }
  } else if (warp >= kEpiWarp0) {
    // ---------------------------------------------------------------- softmax epilogue
    // Column split: warpgroup g owns S columns [64g, 64g+64) of every tile and O columns
    // [g d/2, (g+1) d/2); the row maximum is exchanged through shared memory.
    const int g = (warp - kEpiWarp0) >> 2;
    const int wq = warp & 3;                // TMEM lanes [32 wq, 32 wq + 32)
    const int row = wq * 32 + lane;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    constexpr int kOc = D / 2;  // O columns of this warpgroup
    // `ok` stays warp-uniform (tcgen05.ld/st are warp-collective).  After an abort the
    // loops keep running without touching TMEM so that every epilogue thread executes the
    // same sequence of named barriers and nobody waits forever.
    bool ok = true;
    int t = 0, i = 0;
    auto row_bias = [&](const Item& x) {
      const int r = x.qt * kTile + row;
      return (p.bias != nullptr && x.n > 0 && r < x.sq.limit)
                 ? p.bias[static_cast<int64_t>(x.sq.tma_b) * p.bias_sb + x.sq.row0 + r]
                 : 0.0f;
    };
    zero_empty_items<D, EPI>(p, nwork, warp - kEpiWarp0, lane);
    ItemIter iter(p, nwork);
    float bias_cur = iter.valid() ? row_bias(iter.cur) : 0.0f;
    for (; iter.valid(); iter.advance()) {
      const Item it = iter.cur;
      const float bias_nxt =
          iter.wn < nwork ? row_bias(iter.nxt) : 0.0f;
      const float bias_r = bias_cur;
      bias_cur = bias_nxt;
      if (it.n == 0) continue;  // not in [0, nwork)
      const int ob = i & 1;
      const int rg = it.qt * kTile + row;
      const float c1 = p.scale * kLog2e;  // t = (scale s + bias) log2 e
      const float c0 = bias_r * kLog2e;
      float m_run = EPI == 2 ? 0.0f : kNegBig;  // base-2 running max
      float l_run = (EPI == 2 && g == 0) ? 1.0f : 0.0f;
      for (int j = 0; j < it.n; ++j, ++t) {
        const int sb = t & 1, s = t % S;
        if (ok) ok = mbar_wait(k_full + s, (t / S) & 1, wctx);
        if (ok) ok = mbar_wait(s_full + sb, (t >> 1) & 1, wctx);
        ok = __all_sync(0xFFFFFFFFu, ok);
        if (ok) tc_fence_after();
        uint32_t mw0 = 0xFFFFFFFFu, mw1 = 0xFFFFFFFFu;
        if (ok && meta_kind[s] == 2) {
          const uint2 mb = *reinterpret_cast<const uint2*>(meta_bits + s * 512 + row * 4 + g * 2);
          mw0 = mb.x;
          mw1 = mb.y;
        }
        uint32_t sr[64];
        if (ok) {
          tmem_ld32(t_lane + sb * 128 + g * 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
          tmem_ld32(t_lane + sb * 128 + g * 64 + 32,
                    *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int c = 0; c < 64; ++c) sr[c] = 0u;
        }
        float pv[64];
        float tmax = kNegBig;
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const float tt = fmaf(__uint_as_float(sr[c]), c1, c0);
          const uint32_t bit = ((c < 32 ? mw0 : mw1) >> (c & 31)) & 1u;
          pv[c] = bit ? tt : kNegBig;
          tmax = fmaxf(tmax, pv[c]);
        }
        red_max[(sb * 2 + g) * 128 + row] = tmax;
        named_barrier_sync(1, 256);
        tmax = fmaxf(tmax, red_max[(sb * 2 + (g ^ 1)) * 128 + row]);
        // Lazy rescaling: keep the running max unless the tile's max exceeds it by more
        // than 8 (base 2), so that exp2(t - m) stays <= 256; the result is exact either
        // way because numerator and denominator share m.
        const bool need = tmax > m_run + 8.0f;
        const float m_new = need ? tmax : m_run;
        const float alpha = ex2_approx(m_run - m_new);
        if (ok && __any_sync(0xFFFFFFFFu, need) && j > 0) {
          // O must not be read while PV of the previous tile may still accumulate into it.
          ok = mbar_wait(pv_done, (t - 1) & 1, wctx);
          ok = __all_sync(0xFFFFFFFFu, ok);
          if (ok) {
            tc_fence_after();
#pragma unroll
            for (int c0o = 0; c0o < kOc; c0o += 32) {
              uint32_t orr[32];
              tmem_ld32(t_lane + 256 + ob * D + g * kOc + c0o, orr);
              tmem_wait_ld();
#pragma unroll
              for (int c = 0; c < 32; ++c)
                orr[c] = __float_as_uint(__uint_as_float(orr[c]) * alpha);
              tmem_st32(t_lane + 256 + ob * D + g * kOc + c0o, orr);
            }
          }
        }
        l_run *= alpha;
        m_run = m_new;
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const float e2 = pv[c] > 0.5f * kNegBig ? ex2_approx(pv[c] - m_run) : 0.0f;
          pv[c] = e2;
          l_run += e2;
        }
        if (ok) {
          uint32_t pk[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) pk[c] = pack_bf16x2(pv[2 * c], pv[2 * c + 1]);
          tmem_st32(t_lane + sb * 128 + g * 64, pk);
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(p_full + sb);
        }
      }
      // ---- output of this item: O and LSE from TMEM buffer ob
      if (ok) ok = mbar_wait(o_full + ob, (i >> 1) & 1, wctx);
      ok = __all_sync(0xFFFFFFFFu, ok);
      red_l[g * 128 + row] = l_run;
      named_barrier_sync(1, 256);
      const float l_tot = l_run + red_l[(g ^ 1) * 128 + row];
      named_barrier_sync(1, 256);  // red_l is rewritten by the next item
      const float inv_l = l_tot > 0.0f ? 1.0f / l_tot : 0.0f;
      if (ok && g == 0 && rg < p.Nq) {
        const float lse = l_tot > 0.0f ? (m_run + __log2f(l_tot)) * kLn2 : -INFINITY;
        p.lse[(static_cast<int64_t>(it.b) * p.H + it.h) * p.Nq + rg] = lse;
      }
      if (ok) {
        tc_fence_after();
        uint32_t pk[kOc / 2];
#pragma unroll
        for (int c0o = 0; c0o < kOc; c0o += 32) {
          uint32_t orr[32];
          tmem_ld32(t_lane + 256 + ob * D + g * kOc + c0o, orr);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 16; ++c)
            pk[c0o / 2 + c] = pack_bf16x2(__uint_as_float(orr[2 * c]) * inv_l,
                                          __uint_as_float(orr[2 * c + 1]) * inv_l);
        }
        // O buffer ob may be overwritten by item i + 2 from here on
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(o_empty + ob);
        if (rg < it.sq.limit) {
          uint4* d4 = reinterpret_cast<uint4*>(p.o + seq_row_offset(it.sq, p.o_sb, p.o_sn, rg) +
                                               it.h * p.o_sh + g * kOc);
#pragma unroll
          for (int c = 0; c < kOc / 8; ++c)
            d4[c] = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        }
      }
      ++i;
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

// ------------------------------------------------------------------------------------
// Sigmoid forward.
//
// The weights of sigmoid attention need no row statistics, so nothing but buffers ties
// one key tile to the next.  S and P of a tile share a TMEM buffer (P overwrites columns
// of S already read), and there are three such buffers: the MMA issuer computes S_t as
// soon as O += P_{t-3} V_{t-3}, the last user of that buffer, is issued, i.e. once the
// epilogue has finished tile t - 3.  One commit per MMA group: s_ready (S_t ready, K_t
// consumed) and step (V_t consumed).
// Warps: 0 Q/K producer, 1 TMEM allocator + MMA issuer, 2 V producer, 3 kind / bitmask
// producer (and writer of the empty items' zero rows), 4-11 two epilogue warpgroups that
// take alternate tiles (thread = query row = TMEM lane).  The O of an item is written out after the first tile of the next item,
// when the last PV of the item has long completed; warpgroup g writes O columns
// [g d/2, (g+1) d/2).
// TMEM columns: S/P buffers [0,128), [128,256), [256,384); O in [384,512) (two buffers
// of 64 columns for d = 64, one of 128 for d = 128).  P of keys 16kk.. (the A operand of
// the kk-th K-step of the PV MMA) sits at column 64 (kk / 4) + 8 (kk % 4) of its buffer.
template <int D>
struct SigLayout {
  static constexpr int kBoxes = D / 64;
  static constexpr int kBoxBytes = 128 * 128;
  static constexpr int kTileBytes = kBoxes * kBoxBytes;
  static constexpr int kKStages = D == 64 ? 4 : 2;
  static constexpr int kVStages = D == 64 ? 4 : 2;
  static constexpr int kMStages = 4;
  static constexpr int kSteps = 4;  // ring of step barriers, >= both stage counts
  static constexpr int kOBufs = D == 64 ? 2 : 1;
  static constexpr int kOCol = 384;
  static constexpr int kQ = 0;
  static constexpr int kK = 2 * kTileBytes;
  static constexpr int kV = kK + kKStages * kTileBytes;
  static constexpr int kZero = kV + kVStages * kTileBytes;  // a 64-column box of zeros
  static constexpr int kMetaBits = kZero + kBoxBytes;
  static constexpr int kMetaKind = kMetaBits + kMStages * 2048;
  static constexpr int kBar = kMetaKind + 16 * ((kMStages * 4 + 15) / 16);
  // q_full[2] q_empty[2] o_full[2] o_empty[2] e_done[4] done, s_ready[kSteps],
  // step[kSteps], k_full[SK] v_full[SV] m_full[SM] m_empty[SM]
  static constexpr int kNumBars = 13 + 2 * kSteps + kKStages + kVStages + 2 * kMStages;
  static constexpr int kMisc = kBar + 8 * kNumBars;
  static constexpr int kBytes = kMisc + 16;
  static constexpr int kAlloc = kBytes + 1024;
  static_assert(kSteps >= kKStages && kSteps >= kVStages && kSteps >= 3, "step ring");
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_sigmoid_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                       const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap to,
                       const FwdParams p) {
  using L = SigLayout<D>;
  constexpr int SK = L::kKStages, SV = L::kVStages, SM = L::kMStages, NS = L::kSteps;
  constexpr int OB = L::kOBufs;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int warp = warp_id(), lane = lane_id();
  const int nwork = static_cast<int>(__ldg(p.counts + kCountRows)) * p.H;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 2;
  uint64_t* o_full = bars + 4;
  uint64_t* o_empty = bars + 6;
  uint64_t* e_done = bars + 8;
  uint64_t* done = bars + 12;
  uint64_t* s_ready = bars + 13;
  uint64_t* step = s_ready + NS;
  uint64_t* k_full = step + NS;
  uint64_t* v_full = k_full + SK;
  uint64_t* m_full = v_full + SV;
  uint64_t* m_empty = m_full + SM;
  uint32_t* meta_bits = reinterpret_cast<uint32_t*>(smem + L::kMetaBits);
  int* meta_kind = reinterpret_cast<int*>(smem + L::kMetaKind);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  volatile int* drain_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 8);
  const WaitCtx wctx{p.status, p.wait_ns, abort_flag};

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(q_full + i, 1);
      mbar_init(q_empty + i, 1);
      mbar_init(o_full + i, 1);
      mbar_init(o_empty + i, 8);
    }
    for (int i = 0; i < 4; ++i) mbar_init(e_done + i, 4);
    mbar_init(done, 1);
    for (int i = 0; i < NS; ++i) {
      mbar_init(s_ready + i, 1);
      mbar_init(step + i, 1);
    }
    for (int i = 0; i < SK; ++i) mbar_init(k_full + i, 1);
    for (int i = 0; i < SV; ++i) mbar_init(v_full + i, 1);
    for (int i = 0; i < SM; ++i) {
      mbar_init(m_full + i, 1);
      mbar_init(m_empty + i, 4);
    }
    *abort_flag = 0;
    *drain_flag = 0;
    fence_barrier_init();
  }
  if (p.zero_tma) {
    uint4* z = reinterpret_cast<uint4*>(smem + L::kZero);
    for (int i = threadIdx.x; i < L::kBoxBytes / 16; i += kThreads) z[i] = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
  }
  __syncwarp();
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 || warp == 2 || warp == 3) {
    // ---------------------------------------------------------------- producers
    // warp 0: Q of each item and the K ring (a slot is free again once the S of the tile
    // that used it has completed: s_ready); warp 2: the V ring (free once that tile's PV has
    // completed: step); warp 3: each tile's kind and PARTIAL bitmask (slot released by the
    // epilogue) and, on padded layouts, the zero rows of this CTA's empty items.  A row is walked by its runs (ranges
    // of consecutive k-tiles of one kind): all 32 lanes fetch the next 32 runs in one round
    // trip, and within a run the k-tile and bitmask number just count up, with no per-tile
    // list lookup.  Lane 0 waits and issues the copies.
    const int role = warp == 0 ? 0 : (warp == 2 ? 1 : 2);
    if (lane == 0 && role < 2) {
      tma_prefetch_desc(role == 0 ? &tk : &tv);
      if (role == 0) tma_prefetch_desc(&tq);
    }
    const int NR = role == 0 ? SK : (role == 1 ? SV : SM);
    uint64_t* full = role == 0 ? k_full : (role == 1 ? v_full : m_full);
    const int ring = role == 0 ? L::kK : L::kV;
    const CUtensorMap* map = role == 0 ? &tk : &tv;
    int t = 0, i = 0;
    bool ok = true;
    // meta producer, lane 0: the zero rows of this CTA's empty items (items nwork +
    // blockIdx.x + k gridDim.x), one item after each tile it produces, as tensor-map stores
    // of a box of zeros; the next item's descriptor is loaded one store ahead.
    int zw = nwork + static_cast<int>(blockIdx.x);
    const bool zeroing = p.zero_tma && role == 2 && lane == 0;
    int4 zd = make_int4(0, 0, 0, 0);
    if (zeroing && zw < p.nitems) zd = p.row_desc[zw / p.H];
    auto zero_one = [&]() {
      if (!zeroing || zw >= p.nitems) return;
      const int b = zd.x / p.QT, qt = zd.x % p.QT, h = zw % p.H;
#pragma unroll
      for (int x = 0; x < L::kBoxes; ++x) tma_store_4d(&to, smem + L::kZero, x * 64, qt * kTile, h, b);
      bulk_commit_group();
      zw += static_cast<int>(gridDim.x);
      if (zw < p.nitems) zd = p.row_desc[zw / p.H];
    };
    for (ItemIter iter(p, nwork); ok && iter.valid(); iter.advance()) {
      const Item it = iter.cur;
      if (it.n == 0) continue;
      if (role == 0) {
        const int qb = i & 1;
        if (lane == 0) {
          if (i >= 2) ok = mbar_wait(q_empty + qb, ((i >> 1) - 1) & 1, wctx);
          if (ok) {
            mbar_arrive_expect_tx(q_full + qb, L::kTileBytes);
            for (int x = 0; x < L::kBoxes; ++x)
              tma_load_4d(smem + L::kQ + qb * L::kTileBytes + x * L::kBoxBytes, &tq, q_full + qb,
                          x * 64, it.sq.row0 + it.qt * kTile, it.h, it.sq.tma_b);
          }
        }
        ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
      }
      ++i;
      for (int rb = it.run0, left = it.n; ok && left > 0;) {
        // lanes past the row's last run read other rows' runs, or unwritten entries below
        // run_cap: their values are never used, and the pidx index is kept in bounds
        int4 run_l = make_int4(0, 0, 0, 0);
        if (rb + lane < p.run_cap) run_l = p.run[rb + lane];
        int pi0_l = 0;
        if (role == 2 && run_l.z == 2 && run_l.w >= 0 && run_l.w < p.run_cap)
          pi0_l = p.pidx[run_l.w];  // first bitmask number of a PARTIAL run
        int used = 0;
        for (int v = 0; ok && v < 32 && left > 0; ++v, ++used) {
          const int kt0 = __shfl_sync(0xFFFFFFFFu, run_l.x, v);
          const int len = __shfl_sync(0xFFFFFFFFu, run_l.y, v);
          const int kd = __shfl_sync(0xFFFFFFFFu, run_l.z, v);
          const int pi0 = __shfl_sync(0xFFFFFFFFu, pi0_l, v);
          left -= len;
        for (int u = 0; u < len; ++u, ++t) {
          const int kt = kt0 + u;
          const int pi = pi0 + u;
          const int s = t % NR;
          if (lane == 0) {
            if (t >= NR) {
              if (role == 2) {
                ok = mbar_wait(m_empty + s, ((t / NR) - 1) & 1, wctx);
              } else {
                // K of tile x is consumed by S_x (s_ready), V of tile x by its PV (step)
                const int x = t - NR;
                ok = mbar_wait((role == 0 ? s_ready : step) + x % NS, (x / NS) & 1, wctx);
              }
            }
            if (ok) {
              if (role < 2) {
                mbar_arrive_expect_tx(full + s, L::kTileBytes);
                for (int x = 0; x < L::kBoxes; ++x)
                  tma_load_4d(smem + ring + s * L::kTileBytes + x * L::kBoxBytes, map, full + s,
                              x * 64, it.sq.row0 + kt * kTile, it.h, it.sq.tma_b);
              } else {
                meta_kind[s] = kd;
                if (kd == 2) {
                  mbar_arrive_expect_tx(full + s, 2048);
                  bulk_load(meta_bits + s * 512, p.bits + static_cast<int64_t>(pi) * 512, 2048,
                            full + s);
                } else {
                  mbar_arrive(full + s);
                }
                zero_one();
              }
            }
          }
          ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
          if (!ok) break;
        }
        }
        rb += used;
      }
    }
    if (ok)
      while (zeroing && zw < p.nitems) zero_one();
    if (zeroing) bulk_wait_all();  // the stores have read the box before shared memory goes
    if (lane == 0 && *abort_flag) {
      // Let the copies still in flight land before the CTA's shared memory goes away.
      const WaitCtx drain{p.status, kDrainWaitNs, drain_flag};
      if (role == 0)
        for (int u = max(0, i - 2); u < i; ++u) mbar_wait(q_full + (u & 1), (u >> 1) & 1, drain);
      for (int u = max(0, t - NR); u < t; ++u) mbar_wait(full + u % NR, (u / NR) & 1, drain);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    // The whole warp runs the issue loop on warp-uniform values: every lane tests or waits
    // on the barriers and a vote combines them, and an elected lane issues the MMAs (a
    // tile's S, or its PV, with the commit after them, under one elect.sync).
    {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, true);
      // FIFO of the (up to three) tiles whose PV is still to issue, oldest first:
      // item number << 2 | first of item << 1 | last of item
      int pq0 = 0, pq1 = 0, pq2 = 0;
      bool ok = true;
      // The issue path is kept short: descriptors are (lo, hi) halves stepped by constant
      // offsets, ring positions are masks of power-of-two stage counts, buffer t % 3 a
      // running counter.
      constexpr uint32_t kHiKm = sw128_desc_hi(1024);       // Q, K: K-major, SBO 1024
      constexpr uint32_t kHiMn = sw128_desc_hi(1024);       // V: MN-major, SBO 1024
      const uint32_t q_lo0 = sw128_desc_lo(smem_u32(smem + L::kQ), 16);
      const uint32_t k_lo0 = sw128_desc_lo(smem_u32(smem + L::kK), 16);
      const uint32_t v_lo0 = sw128_desc_lo(smem_u32(smem + L::kV), L::kBoxBytes);
      constexpr uint32_t kTileLo = L::kTileBytes >> 4;
      static_assert((SK & (SK - 1)) == 0 && (SV & (SV - 1)) == 0 && NS == 4, "ring sizes");
      // O += P_x V_x for the oldest tile x of the FIFO (buffer b3 = x % 3) once the
      // epilogue has finished it, then commit step(x); `ready` says its P and V are
      // already known to be in place (tested together with the next K)
      auto pv = [&](int x, uint32_t b3, bool ready) -> bool {
        const int i = pq0 >> 2;
        const bool first = (pq0 & 2) != 0, last = (pq0 & 1) != 0;
        pq0 = pq1;
        pq1 = pq2;
        const int sv = x & (SV - 1);
        if (!ready) {
          if (!mbar_wait_w(e_done + (x & 3), (x >> 2) & 1, wctx)) return false;
          if (!mbar_wait_w(v_full + sv, (x / SV) & 1, wctx)) return false;
        }
        const int ob = OB == 1 ? 0 : (i & 1);
        if (first && i >= OB && !mbar_wait_w(o_empty + ob, ((i / OB) - 1) & 1, wctx))
          return false;
        tc_fence_after();
        mma_pv8_commit_w(tmem + L::kOCol + ob * D, tmem + b3 * 128, v_lo0 + sv * kTileLo,
                         kHiMn, idesc_pv, first ? 0u : 1u, step + (x & 3));
        if (last) mma_commit_w(o_full + ob);
        return true;
      };
      int t = 0, i = 0;
      uint32_t b3 = 0;  // t % 3
      for (ItemIter iter(p, nwork); ok && iter.valid(); iter.advance()) {
        const Item it = iter.cur;
        if (it.n == 0) continue;
        const int qb = i & 1;
        if (!(ok = mbar_wait_w(q_full + qb, (i >> 1) & 1, wctx))) break;
        const uint32_t q_lo = q_lo0 + qb * kTileLo;
        for (int j = 0; j < it.n; ++j, ++t) {
          const int s = t & (SK - 1);
          // The usual case: P and V of tile t - 3 and K of tile t are all in place.  One
          // non-blocking test of the three barriers; the bounded waits only when it fails.
          bool ready = mbar_test_wait(k_full + s, (t / SK) & 1);
          if (t >= 3)
            ready = ready & mbar_test_wait(e_done + ((t - 3) & 3), ((t - 3) >> 2) & 1) &
                    mbar_test_wait(v_full + ((t - 3) & (SV - 1)), ((t - 3) / SV) & 1);
          ready = __all_sync(0xFFFFFFFFu, ready);
          // S_t goes to the buffer of tile t - 3: its PV first (the pipe runs in order)
          if (t >= 3 && !(ok = pv(t - 3, b3, ready))) break;
          if (!ready && !(ok = mbar_wait_w(k_full + s, (t / SK) & 1, wctx))) break;
          tc_fence_after();
          static_assert(L::kBoxBytes >> 4 == 1024, "box offset in the S issue");
          mma_s_commit_w<D / 16>(tmem + b3 * 128, q_lo, k_lo0 + s * kTileLo, kHiKm, idesc_qk,
                                 s_ready + (t & 3));
          if (j == it.n - 1) mma_commit_w(q_empty + qb);
          const int info = (i << 2) | (j == 0 ? 2 : 0) | (j == it.n - 1 ? 1 : 0);
          if (t == 0) pq0 = info;
          else if (t == 1) pq1 = info;
          else pq2 = info;
          b3 = b3 == 2 ? 0 : b3 + 1;
        }
        ++i;
      }
      // the last PVs: tile x uses buffer x % 3; b3 is t % 3 here
      for (int x = max(0, t - 3); ok && x < t; ++x) {
        const uint32_t bx = static_cast<uint32_t>((x - t + 3) % 3 + static_cast<int>(b3)) % 3;
        ok = pv(x, bx, false);
      }
      // every MMA complete before the TMEM is released
      mma_commit_w(done);
      const WaitCtx drain{p.status, kDrainWaitNs, drain_flag};
      mbar_wait_w(done, 0, drain);
    }
  } else if (warp >= kEpiWarp0) {
    // ---------------------------------------------------------------- epilogue
    // Ping-pong: warpgroup g takes the tiles t with t % 2 == g, all 128 keys, in four
    // chunks of 32 columns whose TMEM loads overlap the previous chunk's math; while one
    // warpgroup waits, loads or stores, the other keeps the MUFU busy.  Thread = query row.
    // P of chunk c (keys [32c, 32c+32)) overwrites columns 64 (c / 2) + 16 (c % 2) + [0, 16)
    // of the tile's buffer, which belong to chunk 0 or 2, already read.
    const int g = (warp - kEpiWarp0) >> 2;
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    constexpr int kOc = D / 2;  // O columns written by this warpgroup
    // t = x log2(e) = (scale s + bias) log2(e), the argument of sigmoid2
    const float2 c1 = make_float2(p.scale * kLog2e, p.scale * kLog2e);
    bool ok = true;
    auto row_bias = [&](const Item& x) {
      const int r = x.qt * kTile + row;
      return (p.bias != nullptr && x.n > 0 && r < x.sq.limit)
                 ? p.bias[static_cast<int64_t>(x.sq.tma_b) * p.bias_sb + x.sq.row0 + r]
                 : 0.0f;
    };
    // O of the last item with tiles, written out late (see above)
    bool pend = false;
    Item pit{};
    int pi = 0;
    auto flush_o = [&]() {
      pend = false;
      const int ob = pi % OB;
      ok = ok && mbar_wait(o_full + ob, (pi / OB) & 1, wctx);
      ok = __all_sync(0xFFFFFFFFu, ok);
      if (!ok) return;
      tc_fence_after();
      uint32_t pk[kOc / 2];
#pragma unroll
      for (int c0o = 0; c0o < kOc; c0o += 32) {
        uint32_t orr[32];
        tmem_ld32(t_lane + L::kOCol + ob * D + g * kOc + c0o, orr);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 16; ++c)
          pk[c0o / 2 + c] = pack_bf16x2(__uint_as_float(orr[2 * c]), __uint_as_float(orr[2 * c + 1]));
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(o_empty + ob);
      const int rg = pit.qt * kTile + row;
      if (rg < pit.sq.limit) {
        uint4* d4 = reinterpret_cast<uint4*>(p.o + seq_row_offset(pit.sq, p.o_sb, p.o_sn, rg) +
                                             pit.h * p.o_sh + g * kOc);
#pragma unroll
        for (int c = 0; c < kOc / 8; ++c)
          d4[c] = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      }
    };
    if (!p.zero_tma) zero_empty_items<D, 0>(p, nwork, warp - kEpiWarp0, lane);
    int t = 0, i = 0;
    ItemIter iter(p, nwork);
    float bias_cur = iter.valid() ? row_bias(iter.cur) : 0.0f;
    for (; ok && iter.valid(); iter.advance()) {
      const Item it = iter.cur;
      // the next item's bias, in flight while this one is processed
      const float bias_nxt =
          iter.wn < nwork ? row_bias(iter.nxt) : 0.0f;
      const float bias_r = bias_cur;
      bias_cur = bias_nxt;
      if (it.n == 0) continue;  // not in [0, nwork)
      const float2 c0 = make_float2(bias_r * kLog2e, bias_r * kLog2e);
      const int t_end = t + it.n;
      for (int tt = t + ((t & 1) != g ? 1 : 0); tt < t_end; tt += 2) {
        const int ms = tt % SM;
        if (ok) ok = mbar_wait(s_ready + tt % NS, (tt / NS) & 1, wctx);
        if (ok) ok = mbar_wait(m_full + ms, (tt / SM) & 1, wctx);
        ok = __all_sync(0xFFFFFFFFu, ok);
        if (!ok) break;
        tc_fence_after();
        const bool masked = meta_kind[ms] == 2;
        uint4 mb = make_uint4(0xFFFFFFFFu, 0xFFFFFFFFu, 0xFFFFFFFFu, 0xFFFFFFFFu);
        if (masked) mb = *reinterpret_cast<const uint4*>(meta_bits + ms * 512 + row * 4);
        const uint32_t sp = t_lane + (tt % 3) * 128;
        uint32_t buf[2][32];
        tmem_ld32(sp, buf[0]);
        __syncwarp();
        if (lane == 0) mbar_arrive(m_empty + ms);
        tmem_wait_ld();
        // one chunk: sigma of 32 columns from b, P into 16 columns at `dst`
        auto chunk = [&](const uint32_t (&b)[32], uint32_t mw, uint32_t dst) {
          uint32_t pk[16];
#pragma unroll
          for (int cc = 0; cc < 32; cc += 2) {
            float2 x = fma2(make_float2(__uint_as_float(b[cc]), __uint_as_float(b[cc + 1])), c1, c0);
            if (masked) {
              x.x = ((mw >> cc) & 1u) ? x.x : -INFINITY;
              x.y = ((mw >> (cc + 1)) & 1u) ? x.y : -INFINITY;
            }
            const float2 pw = sigmoid2(x);
            pk[cc >> 1] = pack_bf16x2(pw.x, pw.y);
          }
          tmem_st16(dst, pk);
        };
        // chunks c2 and c2 + 1 per pass (buffers 0 and 1); a loop, not unrolled, keeps the
        // epilogue's code small
#pragma unroll 1
        for (int c2 = 0; c2 < 4; c2 += 2) {
          tmem_ld32(sp + 32 * (c2 + 1), buf[1]);
          chunk(buf[0], c2 == 0 ? mb.x : mb.z, sp + (c2 >> 1) * 64);
          tmem_wait_ld();
          if (c2 == 0) tmem_ld32(sp + 64, buf[0]);
          chunk(buf[1], c2 == 0 ? mb.y : mb.w, sp + (c2 >> 1) * 64 + 16);
          if (c2 == 0) tmem_wait_ld();
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(e_done + (tt & 3));
        if (pend) flush_o();
      }
      if (!ok) break;
      if (pend) flush_o();
      pend = true;
      pit = it;
      pi = i;
      t = t_end;
      ++i;
    }
    if (ok && pend) flush_o();
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

template <int D>
int launch_fwd_sigmoid_t(const FwdParams& p, const CUtensorMap& tq, const CUtensorMap& tk,
                         const CUtensorMap& tv, const CUtensorMap& to, cudaStream_t stream) {
  using L = SigLayout<D>;
  static_assert(L::kAlloc <= 227 * 1024, "shared memory");
  auto kern = fwd_sigmoid_kernel<D>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
  if (e != cudaSuccess) return cuda_status(e);
  const int grid = std::min(p.nitems, num_sms());
  kern<<<grid, kThreads, L::kAlloc, stream>>>(tq, tk, tv, to, p);
  return cuda_status(cudaGetLastError());
}

template <int D, int EPI>
int launch_fwd_t(const sigattn_plan* plan, int H, float scale, const CUtensorMap& tq,
                 const CUtensorMap& tk, const CUtensorMap& tv, const float* bias, int64_t bias_sb,
                 const TensorDesc& o, float* lse, int* status, unsigned long long wait_ns,
                 cudaStream_t stream) {
  using L = FwdLayout<D>;
  FwdParams p;
  p.row_ptr = plan->row_ptr;
  p.col_idx = plan->col_idx;
  p.kind = plan->kind;
  p.pidx = plan->pidx;
  p.bits = plan->bits;
  p.row_desc = plan->row_desc;
  p.cu = plan->cu;
  p.run = plan->run;
  p.run_cap = static_cast<int>(plan->run_cap);
  p.QT = plan->QT;
  p.Nq = plan->Nq;
  p.H = H;
  p.nitems = plan->B * plan->QT * H;
  p.counts = plan->dcount;
  p.zero_tma = 0;
  p.scale = scale;
  p.bias = bias;
  p.bias_sb = bias_sb;
  p.o = static_cast<__nv_bfloat16*>(const_cast<void*>(o.ptr));
  p.o_sb = o.sb;
  p.o_sn = o.sn;
  p.o_sh = o.sh;
  p.lse = lse;
  p.status = status;
  p.wait_ns = wait_ns;
  if constexpr (EPI == 0) {
    // padded layouts: the zero rows of the empty items go out as tensor-map stores (rows
    // past the tensor's extent are clipped); packed ones keep the per-row stores, which
    // stop at each sequence's end
    CUtensorMap to;
    std::memset(&to, 0, sizeof(to));
    p.zero_tma = (plan->cu == nullptr && make_tmap_bf16(&to, o, plan->B, H, D) == SIGATTN_OK) ? 1 : 0;
    return launch_fwd_sigmoid_t<D>(p, tq, tk, tv, to, stream);
  } else {
    auto kern = fwd_kernel<D, EPI>;
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
    if (e != cudaSuccess) return cuda_status(e);
    const int grid = std::min(p.nitems, num_sms());
    kern<<<grid, kThreads, L::kAlloc, stream>>>(tq, tk, tv, p);
    return cuda_status(cudaGetLastError());
  }
}

}  // namespace

int launch_fwd_impl(const sigattn_plan* plan, int epilogue, int H, int d, float scale,
                    const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                    const float* bias, int64_t bias_sb, const TensorDesc& o, float* lse,
                    int* status, unsigned long long wait_ns, cudaStream_t stream) {
#define SIGATTN_FWD_CASE(DD, EE)                                                          \
  if (d == DD && epilogue == EE)                                                          \
    return launch_fwd_t<DD, EE>(plan, H, scale, tq, tk, tv, bias, bias_sb, o, lse, status, \
                                wait_ns, stream);
  SIGATTN_FWD_CASE(64, 0)
  SIGATTN_FWD_CASE(64, 1)
  SIGATTN_FWD_CASE(64, 2)
  SIGATTN_FWD_CASE(128, 0)
  SIGATTN_FWD_CASE(128, 1)
  SIGATTN_FWD_CASE(128, 2)
#undef SIGATTN_FWD_CASE
  return SIGATTN_ERR_UNSUPPORTED;
}

}  // namespace sigattn
