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
// issuer, warps 4-11 two epilogue warpgroups (thread = TMEM lane; warpgroup g owns tile
// columns [64g, 64g+64) and accumulator columns [g d/2, (g+1) d/2)).
// TMEM: [0,128) S (or S^T), [128,256) dP (or dP^T), then the fp32 accumulators.  The bf16
// P / dS values overwrite the columns of S / dP that the same warpgroup already read, and
// are the TMEM A operand of the accumulating MMAs.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <mutex>

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
  const int32_t* row_work;
  const int32_t* col_work;
  int QT, KT, Nq, Nk, H;
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

// Offset of one query row in the weight's argument, with c1 the matching slope:
// SIGMOID  p = 0.5 + 0.5 tanh(c1 s + off),  c1 = scale / 2,  off = bias / 2;
// softmax  p = 2^(c1 s + off),               c1 = scale log2 e,  off = (bias - lse) log2 e.
template <int EPI>
__device__ __forceinline__ float row_offset(const BwdParams& p, int b, int h, int qg) {
  if (qg >= p.Nq) return 0.0f;
  const float bias = p.bias ? p.bias[b * p.bias_sb + qg] : 0.0f;
  if (EPI == 0) return 0.5f * bias;
  return (bias - p.lse[(static_cast<int64_t>(b) * p.H + h) * p.Nq + qg]) * kLog2e;
}

template <int EPI>
__device__ __forceinline__ float row_D(const BwdParams& p, int b, int h, int qg) {
  if (EPI == 0 || qg >= p.Nq) return 0.0f;
  return p.Dws[(static_cast<int64_t>(b) * p.H + h) * p.Nq + qg];
}

// p and ds of one element; `keep` is the mask bit.
template <int EPI>
__device__ __forceinline__ void weight_grad(float s, float dp, float c1, float off, float Drow,
                                            bool keep, float& pw, float& ds) {
  if (EPI == 0) {
    const float sg = sigmoid_tanh(s, c1, off);
    pw = keep ? sg : 0.0f;
    ds = dp * pw * (1.0f - pw);
  } else {
    pw = keep ? ex2_approx(fmaf(s, c1, off)) : 0.0f;
    ds = pw * (dp - Drow);
  }
}

__device__ __forceinline__ void store_row_bf16(__nv_bfloat16* dst, const uint32_t (&acc)[32],
                                               float mul) {
  uint32_t pk[16];
#pragma unroll
  for (int c = 0; c < 16; ++c)
    pk[c] = pack_bf16x2(__uint_as_float(acc[2 * c]) * mul, __uint_as_float(acc[2 * c + 1]) * mul);
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int c = 0; c < 4; ++c) d4[c] = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
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
                                    int H, float* __restrict__ Dws) {
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
    const uint4 ov = *reinterpret_cast<const uint4*>(o + b * o_sb + i * o_sn + h * o_sh + chunk * 8);
    const uint4 dv = *reinterpret_cast<const uint4*>(dout + b * do_sb + i * do_sn + h * do_sh + chunk * 8);
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
// dK / dV
// ---------------------------------------------------------------------------------------
template <int D>
struct DkvLayout {
  static constexpr int kStages = D == 64 ? 4 : 2;
  static constexpr int kBoxes = D / 64;
  static constexpr int kBoxBytes = 128 * 128;
  static constexpr int kTileBytes = kBoxes * kBoxBytes;
  static constexpr int kK = 0;
  static constexpr int kV = kTileBytes;
  static constexpr int kQ = 2 * kTileBytes;
  static constexpr int kDO = kQ + kStages * kTileBytes;
  static constexpr int kVec = kDO + kStages * kTileBytes;      // float [S][2][128]
  static constexpr int kBar = kVec + kStages * 2 * 128 * 4;
  // kv_full, acc_full, s_full, p_full, q_full[S], q_empty[S]
  static constexpr int kNumBars = 4 + 2 * kStages;
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
  constexpr int S = L::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int warp = warp_id(), lane = lane_id();
  const int wi = blockIdx.x / p.H, h = blockIdx.x % p.H;
  const int c = p.col_work[wi];
  const int b = c / p.KT, kt = c % p.KT;
  const int e0 = p.colT_ptr[c];
  const int n = p.colT_ptr[c + 1] - e0;

  if (n == 0) {
    // No query attends to this k-tile: dK = dV = 0 on its rows.
    const int rows = min(kTile, p.Nk - kt * kTile);
    zero_rows<D>(p.dk + b * p.dk_sb + static_cast<int64_t>(kt * kTile) * p.dk_sn + h * p.dk_sh,
                 p.dk_sn, rows, threadIdx.x, kThreads);
    zero_rows<D>(p.dv + b * p.dv_sb + static_cast<int64_t>(kt * kTile) * p.dv_sn + h * p.dv_sh,
                 p.dv_sn, rows, threadIdx.x, kThreads);
    return;
  }

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* kv_full = bars + 0;
  uint64_t* acc_full = bars + 1;
  uint64_t* s_full = bars + 2;
  uint64_t* p_full = bars + 3;
  uint64_t* q_full = bars + 4;
  uint64_t* q_empty = bars + 4 + S;
  float* vec = reinterpret_cast<float*>(smem + L::kVec);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  volatile int* drain_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 8);
  const WaitCtx wctx{p.status, p.wait_ns, abort_flag};

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    mbar_init(acc_full, 1);
    mbar_init(s_full, 1);
    mbar_init(p_full, 8);
    for (int i = 0; i < S; ++i) {
      mbar_init(q_full + i, 2);  // TMA bytes + the producer warp's column vectors
      mbar_init(q_empty + i, 1);
    }
    *abort_flag = 0;
    *drain_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      tma_prefetch_desc(&tq);
      tma_prefetch_desc(&tk);
      tma_prefetch_desc(&tv);
      tma_prefetch_desc(&tdo);
      mbar_arrive_expect_tx(kv_full, 2 * L::kTileBytes);
      for (int x = 0; x < L::kBoxes; ++x) {
        tma_load_4d(smem + L::kK + x * L::kBoxBytes, &tk, kv_full, x * 64, kt * kTile, h, b);
        tma_load_4d(smem + L::kV + x * L::kBoxBytes, &tv, kv_full, x * 64, kt * kTile, h, b);
      }
    }
    int issued = 0;
    for (int i = 0; i < n; ++i) {
      const int s = i % S;
      bool ok = true;
      if (lane == 0 && i >= S) ok = mbar_wait(q_empty + s, ((i / S) - 1) & 1, wctx);
      ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      const int qt = p.rowT_idx[e0 + i];
      if (lane == 0) {
        mbar_arrive_expect_tx(q_full + s, 2 * L::kTileBytes);
        for (int x = 0; x < L::kBoxes; ++x) {
          tma_load_4d(smem + L::kQ + s * L::kTileBytes + x * L::kBoxBytes, &tq, q_full + s, x * 64,
                      qt * kTile, h, b);
          tma_load_4d(smem + L::kDO + s * L::kTileBytes + x * L::kBoxBytes, &tdo, q_full + s,
                      x * 64, qt * kTile, h, b);
        }
      }
      float* vs = vec + s * 256;
      for (int cc = lane; cc < 128; cc += 32) {
        const int qg = qt * kTile + cc;
        vs[cc] = row_offset<EPI>(p, b, h, qg);
        vs[128 + cc] = row_D<EPI>(p, b, h, qg);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(q_full + s);
      issued = i + 1;
    }
    if (lane == 0 && *abort_flag) {
      const WaitCtx drain{p.status, p.wait_ns, drain_flag};
      mbar_wait(kv_full, 0, drain);
      for (int i = max(0, issued - S); i < issued; ++i) mbar_wait(q_full + i % S, (i / S) & 1, drain);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_ss = idesc_bf16_f32(128, 128, false);
      constexpr uint32_t idesc_acc = idesc_bf16_f32(128, D, true);
      const uint32_t k_base = smem_u32(smem + L::kK);
      const uint32_t v_base = smem_u32(smem + L::kV);
      const uint32_t t_dv = tmem + 256, t_dk = tmem + 256 + D;
      bool ok = mbar_wait(kv_full, 0, wctx);
      tc_fence_after();
      for (int i = 0; ok && i <= n; ++i) {
        if (i >= 1) {
          const int ii = i - 1, s2 = ii % S;
          if (!(ok = mbar_wait(p_full, ii & 1, wctx))) break;
          tc_fence_after();
          const uint32_t q_s = smem_u32(smem + L::kQ + s2 * L::kTileBytes);
          const uint32_t do_s = smem_u32(smem + L::kDO + s2 * L::kTileBytes);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t a_col = (kk >> 2) * 64 + (kk & 3) * 8;
            const uint32_t acc = (ii > 0 || kk > 0) ? 1u : 0u;
            mma_ts(t_dv, tmem + a_col, smem_desc_sw128(do_s + kk * 2048, L::kBoxBytes, 1024),
                   idesc_acc, acc);
            mma_ts(t_dk, tmem + 128 + a_col, smem_desc_sw128(q_s + kk * 2048, L::kBoxBytes, 1024),
                   idesc_acc, acc);
          }
          mma_commit(q_empty + s2);
        }
        if (i < n) {
          const int s = i % S;
          if (!(ok = mbar_wait(q_full + s, (i / S) & 1, wctx))) break;
          tc_fence_after();
          const uint32_t q_s = smem_u32(smem + L::kQ + s * L::kTileBytes);
          const uint32_t do_s = smem_u32(smem + L::kDO + s * L::kTileBytes);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * L::kBoxBytes + (kk & 3) * 32;
            mma_ss(tmem, smem_desc_sw128(k_base + off, 16, 1024),
                   smem_desc_sw128(q_s + off, 16, 1024), idesc_ss, kk > 0);
          }
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * L::kBoxBytes + (kk & 3) * 32;
            mma_ss(tmem + 128, smem_desc_sw128(v_base + off, 16, 1024),
                   smem_desc_sw128(do_s + off, 16, 1024), idesc_ss, kk > 0);
          }
          mma_commit(s_full);
        }
      }
      mma_commit(acc_full);
    }
  } else if (warp >= kEpiWarp0) {
    // ---------------------------------------------------------------- epilogue
    const int g = (warp - kEpiWarp0) >> 2;
    const int wq = warp & 3;
    const int row = wq * 32 + lane;  // key row of the tile
    const int kg = kt * kTile + row;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const float c1 = EPI == 0 ? 0.5f * p.scale : p.scale * kLog2e;
    bool ok = true;
    for (int i = 0; i < n; ++i) {
      const int s = i % S;
      if (ok) ok = mbar_wait(q_full + s, (i / S) & 1, wctx);
      if (ok) ok = mbar_wait(s_full, i & 1, wctx);
      ok = __all_sync(0xFFFFFFFFu, ok);
      if (!ok) break;
      tc_fence_after();
      const int e = p.csc_map[e0 + i];
      const int kd = p.kind[e];
      uint32_t mw0 = 0xFFFFFFFFu, mw1 = 0xFFFFFFFFu;
      if (kd == 2) {
        const uint2 mb = *reinterpret_cast<const uint2*>(
            p.bitsT + static_cast<int64_t>(p.pidx[e]) * 512 + row * 4 + g * 2);
        mw0 = mb.x;
        mw1 = mb.y;
      }
      const float* vs = vec + s * 256 + g * 64;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int col = g * 64 + half * 32;
        uint32_t sr[32], dpr[32];
        tmem_ld32(t_lane + col, sr);
        tmem_ld32(t_lane + 128 + col, dpr);
        tmem_wait_ld();
        const uint32_t mw = half ? mw1 : mw0;
        uint32_t pk[16], dk[16];
#pragma unroll
        for (int cc = 0; cc < 32; cc += 2) {
          float p0, p1, d0, d1;
          weight_grad<EPI>(__uint_as_float(sr[cc]), __uint_as_float(dpr[cc]), c1,
                           vs[half * 32 + cc], vs[128 + half * 32 + cc], (mw >> cc) & 1u, p0, d0);
          weight_grad<EPI>(__uint_as_float(sr[cc + 1]), __uint_as_float(dpr[cc + 1]), c1,
                           vs[half * 32 + cc + 1], vs[128 + half * 32 + cc + 1],
                           (mw >> (cc + 1)) & 1u, p1, d1);
          pk[cc >> 1] = pack_bf16x2(p0, p1);
          dk[cc >> 1] = pack_bf16x2(d0, d1);
        }
        tmem_st16(t_lane + g * 64 + half * 16, pk);
        tmem_st16(t_lane + 128 + g * 64 + half * 16, dk);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    if (ok) ok = mbar_wait(acc_full, 0, wctx);
    ok = __all_sync(0xFFFFFFFFu, ok);
    if (ok) {
      tc_fence_after();
      constexpr int kOc = D / 2;
      __nv_bfloat16* dvp = p.dv + b * p.dv_sb + static_cast<int64_t>(kg) * p.dv_sn + h * p.dv_sh + g * kOc;
      __nv_bfloat16* dkp = p.dk + b * p.dk_sb + static_cast<int64_t>(kg) * p.dk_sn + h * p.dk_sh + g * kOc;
#pragma unroll
      for (int c0 = 0; c0 < kOc; c0 += 32) {
        uint32_t acc[32];
        tmem_ld32(t_lane + 256 + g * kOc + c0, acc);
        tmem_wait_ld();
        if (kg < p.Nk) store_row_bf16(dvp + c0, acc, 1.0f);
        tmem_ld32(t_lane + 256 + D + g * kOc + c0, acc);
        tmem_wait_ld();
        if (kg < p.Nk) store_row_bf16(dkp + c0, acc, p.scale);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------------------
// dQ
// ---------------------------------------------------------------------------------------
template <int D>
struct DqLayout {
  static constexpr int kStages = D == 64 ? 4 : 2;
  static constexpr int kBoxes = D / 64;
  static constexpr int kBoxBytes = 128 * 128;
  static constexpr int kTileBytes = kBoxes * kBoxBytes;
  static constexpr int kQ = 0;
  static constexpr int kDO = kTileBytes;
  static constexpr int kK = 2 * kTileBytes;
  static constexpr int kV = kK + kStages * kTileBytes;
  static constexpr int kBar = kV + kStages * kTileBytes;
  // qd_full, acc_full, s_full, ds_full, kv_full[S], kv_empty[S]
  static constexpr int kNumBars = 4 + 2 * kStages;
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
  constexpr int S = L::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int warp = warp_id(), lane = lane_id();
  const int wi = blockIdx.x / p.H, h = blockIdx.x % p.H;
  const int r = p.row_work[wi];
  const int b = r / p.QT, qt = r % p.QT;
  const int e0 = p.row_ptr[r];
  const int n = p.row_ptr[r + 1] - e0;

  if (n == 0) {
    const int rows = min(kTile, p.Nq - qt * kTile);
    zero_rows<D>(p.dq + b * p.dq_sb + static_cast<int64_t>(qt * kTile) * p.dq_sn + h * p.dq_sh,
                 p.dq_sn, rows, threadIdx.x, kThreads);
    return;
  }

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* qd_full = bars + 0;
  uint64_t* acc_full = bars + 1;
  uint64_t* s_full = bars + 2;
  uint64_t* ds_full = bars + 3;
  uint64_t* kv_full = bars + 4;
  uint64_t* kv_empty = bars + 4 + S;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  volatile int* drain_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 8);
  const WaitCtx wctx{p.status, p.wait_ns, abort_flag};

  if (threadIdx.x == 0) {
    mbar_init(qd_full, 1);
    mbar_init(acc_full, 1);
    mbar_init(s_full, 1);
    mbar_init(ds_full, 8);
    for (int i = 0; i < S; ++i) {
      mbar_init(kv_full + i, 1);
      mbar_init(kv_empty + i, 1);
    }
    *abort_flag = 0;
    *drain_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tq);
      tma_prefetch_desc(&tk);
      tma_prefetch_desc(&tv);
      tma_prefetch_desc(&tdo);
      mbar_arrive_expect_tx(qd_full, 2 * L::kTileBytes);
      for (int x = 0; x < L::kBoxes; ++x) {
        tma_load_4d(smem + L::kQ + x * L::kBoxBytes, &tq, qd_full, x * 64, qt * kTile, h, b);
        tma_load_4d(smem + L::kDO + x * L::kBoxBytes, &tdo, qd_full, x * 64, qt * kTile, h, b);
      }
      int issued = 0;
      for (int j = 0; j < n; ++j) {
        const int s = j % S;
        if (j >= S && !mbar_wait(kv_empty + s, ((j / S) - 1) & 1, wctx)) break;
        const int kt = p.col_idx[e0 + j];
        mbar_arrive_expect_tx(kv_full + s, 2 * L::kTileBytes);
        for (int x = 0; x < L::kBoxes; ++x) {
          tma_load_4d(smem + L::kK + s * L::kTileBytes + x * L::kBoxBytes, &tk, kv_full + s,
                      x * 64, kt * kTile, h, b);
          tma_load_4d(smem + L::kV + s * L::kTileBytes + x * L::kBoxBytes, &tv, kv_full + s,
                      x * 64, kt * kTile, h, b);
        }
        issued = j + 1;
      }
      if (*abort_flag) {
        const WaitCtx drain{p.status, p.wait_ns, drain_flag};
        mbar_wait(qd_full, 0, drain);
        for (int j = max(0, issued - S); j < issued; ++j) mbar_wait(kv_full + j % S, (j / S) & 1, drain);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc_ss = idesc_bf16_f32(128, 128, false);
      constexpr uint32_t idesc_acc = idesc_bf16_f32(128, D, true);
      const uint32_t q_base = smem_u32(smem + L::kQ);
      const uint32_t do_base = smem_u32(smem + L::kDO);
      const uint32_t t_dq = tmem + 256;
      bool ok = mbar_wait(qd_full, 0, wctx);
      tc_fence_after();
      for (int j = 0; ok && j <= n; ++j) {
        if (j >= 1) {
          const int jj = j - 1, s2 = jj % S;
          if (!(ok = mbar_wait(ds_full, jj & 1, wctx))) break;
          tc_fence_after();
          const uint32_t k_s = smem_u32(smem + L::kK + s2 * L::kTileBytes);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t a_col = 128 + (kk >> 2) * 64 + (kk & 3) * 8;
            mma_ts(t_dq, tmem + a_col, smem_desc_sw128(k_s + kk * 2048, L::kBoxBytes, 1024),
                   idesc_acc, (jj > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(kv_empty + s2);
        }
        if (j < n) {
          const int s = j % S;
          if (!(ok = mbar_wait(kv_full + s, (j / S) & 1, wctx))) break;
          tc_fence_after();
          const uint32_t k_s = smem_u32(smem + L::kK + s * L::kTileBytes);
          const uint32_t v_s = smem_u32(smem + L::kV + s * L::kTileBytes);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * L::kBoxBytes + (kk & 3) * 32;
            mma_ss(tmem, smem_desc_sw128(q_base + off, 16, 1024),
                   smem_desc_sw128(k_s + off, 16, 1024), idesc_ss, kk > 0);
          }
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * L::kBoxBytes + (kk & 3) * 32;
            mma_ss(tmem + 128, smem_desc_sw128(do_base + off, 16, 1024),
                   smem_desc_sw128(v_s + off, 16, 1024), idesc_ss, kk > 0);
          }
          mma_commit(s_full);
        }
      }
      mma_commit(acc_full);
    }
  } else if (warp >= kEpiWarp0) {
    const int g = (warp - kEpiWarp0) >> 2;
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const int qg = qt * kTile + row;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const float c1 = EPI == 0 ? 0.5f * p.scale : p.scale * kLog2e;
    const float off = row_offset<EPI>(p, b, h, qg);
    const float Drow = row_D<EPI>(p, b, h, qg);
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      if (ok) ok = mbar_wait(s_full, j & 1, wctx);
      ok = __all_sync(0xFFFFFFFFu, ok);
      if (!ok) break;
      tc_fence_after();
      const int e = e0 + j;
      const int kd = p.kind[e];
      uint32_t mw0 = 0xFFFFFFFFu, mw1 = 0xFFFFFFFFu;
      if (kd == 2) {
        const uint2 mb = *reinterpret_cast<const uint2*>(
            p.bits + static_cast<int64_t>(p.pidx[e]) * 512 + row * 4 + g * 2);
        mw0 = mb.x;
        mw1 = mb.y;
      }
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int col = g * 64 + half * 32;
        uint32_t sr[32], dpr[32];
        tmem_ld32(t_lane + col, sr);
        tmem_ld32(t_lane + 128 + col, dpr);
        tmem_wait_ld();
        const uint32_t mw = half ? mw1 : mw0;
        uint32_t dk[16];
#pragma unroll
        for (int cc = 0; cc < 32; cc += 2) {
          float p0, p1, d0, d1;
          weight_grad<EPI>(__uint_as_float(sr[cc]), __uint_as_float(dpr[cc]), c1, off, Drow,
                           (mw >> cc) & 1u, p0, d0);
          weight_grad<EPI>(__uint_as_float(sr[cc + 1]), __uint_as_float(dpr[cc + 1]), c1, off,
                           Drow, (mw >> (cc + 1)) & 1u, p1, d1);
          dk[cc >> 1] = pack_bf16x2(d0, d1);
        }
        tmem_st16(t_lane + 128 + g * 64 + half * 16, dk);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(ds_full);
    }
    if (ok) ok = mbar_wait(acc_full, 0, wctx);
    ok = __all_sync(0xFFFFFFFFu, ok);
    if (ok) {
      tc_fence_after();
      constexpr int kOc = D / 2;
      __nv_bfloat16* dqp = p.dq + b * p.dq_sb + static_cast<int64_t>(qg) * p.dq_sn + h * p.dq_sh + g * kOc;
#pragma unroll
      for (int c0 = 0; c0 < kOc; c0 += 32) {
        uint32_t acc[32];
        tmem_ld32(t_lane + 256 + g * kOc + c0, acc);
        tmem_wait_ld();
        if (qg < p.Nq) store_row_bf16(dqp + c0, acc, p.scale);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
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
  p.row_work = plan->row_work;
  p.col_work = plan->col_work;
  p.QT = plan->QT;
  p.KT = plan->KT;
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
        H, workspace);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_status(e);
  }
  if (parts & SIGATTN_BWD_DKDV) {
    auto kdkv = dkdv_kernel<D, EPI>;
    if ((e = cudaFuncSetAttribute(kdkv, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  DkvLayout<D>::kAlloc)) != cudaSuccess)
      return cuda_status(e);
    kdkv<<<static_cast<unsigned>(static_cast<int64_t>(plan->B) * plan->KT * H), kThreads,
           DkvLayout<D>::kAlloc, stream>>>(tq, tk, tv, tdo, p);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_status(e);
  }
  if (parts & SIGATTN_BWD_DQ) {
    auto kdq = dq_kernel<D, EPI>;
    if ((e = cudaFuncSetAttribute(kdq, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  DqLayout<D>::kAlloc)) != cudaSuccess)
      return cuda_status(e);
    kdq<<<static_cast<unsigned>(static_cast<int64_t>(plan->B) * plan->QT * H), kThreads,
          DqLayout<D>::kAlloc, stream>>>(tq, tk, tv, tdo, p);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_status(e);
  }
  return SIGATTN_OK;
}

}  // namespace

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

constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mu;
float* g_noalloc_ptr[kNoAllocMaxDevices] = {nullptr};

// Device address of g_noalloc_scratch on the current device.  In host code the array's
// name is only a host-side stand-in, so the address is looked up once per device, with that
// device current, and reused.
int noalloc_scratch(float** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return SIGATTN_ERR_NO_DEVICE;
  }
  if (dev < 0 || dev >= kNoAllocMaxDevices) return SIGATTN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    float* ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void**>(&ptr), g_noalloc_scratch);
    if (e != cudaSuccess) return sigattn::cuda_status(e);
    g_noalloc_ptr[dev] = ptr;
  }
  *out = g_noalloc_ptr[dev];
  return SIGATTN_OK;
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
