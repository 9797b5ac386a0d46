// Forward kernel: fused tiled sigmoid (or softmax / softmax_1) attention over the tile
// list of a plan, sm_100a.
//
// Method: "Better Models, Faster Training: Sigmoid Attention for single-cell Foundation
// Models", section 2A: O = sigma(Q K^T / sqrt(d) + b) V, each weight computed on its own
// with no row normalisation; section 2C: one fused kernel that skips every tile that is
// padding on the query or the key side.  softmax and softmax_1 (the QuietAttention page,
// section "Proposition : softmax_1 et QuietAttention") run through the same kernel with
// the online max / sum recombination of the FlashAttention article (section on the
// mathematics of blockwise softmax); softmax_1 starts from a zero logit whose value row is
// zero (m = 0, l = 1).
//
// One CTA per (q-tile row of the plan, head), 384 threads:
//   warp 0      TMA producer: Q once, then K and V tiles of each listed k-tile into a ring
//   warp 1      TMEM allocator and MMA issuer (one thread): S = Q K^T into one of two
//               TMEM S buffers, then O += P V with P read from TMEM
//   warps 4-11  two epilogue warpgroups; thread = query row (TMEM lane); warpgroup g
//               owns S columns [64g, 64g+64) and O columns [g d/2, (g+1) d/2)
// TMEM columns: S0 [0,128), S1 [128,256), O [256, 256+d).  P (bf16) overwrites the first
// half of the columns each warpgroup read, so the two warpgroups never touch each
// other's S values.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

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
  const int32_t* row_work;
  int QT, Nq, H;
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
  static constexpr int kQ = 0;
  static constexpr int kK = kTileBytes;
  static constexpr int kV = kK + kStages * kTileBytes;
  static constexpr int kBar = kV + kStages * kTileBytes;
  // barriers: q_full, o_full, pv_done, s_full[2], p_full[2], k_full[S], v_full[S], kv_empty[S]
  static constexpr int kNumBars = 7 + 3 * kStages;
  static constexpr int kRed = kBar + 8 * kNumBars;          // float [2][2][128] row maxima
  static constexpr int kRedL = kRed + 2 * 2 * 128 * 4;      // float [2][128] row sums
  static constexpr int kMisc = kRedL + 2 * 128 * 4;          // tmem base, abort flag
  static constexpr int kBytes = kMisc + 16;
  static constexpr int kAlloc = kBytes + 1024;               // slack for 1024-byte alignment
};

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
  const int w = blockIdx.x / p.H, h = blockIdx.x % p.H;
  const int r = p.row_work[w];
  const int b = r / p.QT, qt = r % p.QT;
  const int e0 = p.row_ptr[r];
  const int n = p.row_ptr[r + 1] - e0;

  if (n == 0) {
    // No tile in this row: the whole q-tile is padding or sees no key.  O = 0.
    const int rows = min(kTile, p.Nq - qt * kTile);
    constexpr int kChunks = D / 8;  // 16-byte chunks per row
    for (int i = threadIdx.x; i < rows * kChunks; i += kThreads) {
      const int row = i / kChunks, c = i % kChunks;
      __nv_bfloat16* dst = p.o + b * p.o_sb + static_cast<int64_t>(qt * kTile + row) * p.o_sn +
                           h * p.o_sh + c * 8;
      *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
    }
    if (EPI != 0) {
      const float v = EPI == 1 ? -INFINITY : 0.0f;
      for (int i = threadIdx.x; i < rows; i += kThreads)
        p.lse[(static_cast<int64_t>(b) * p.H + h) * p.Nq + qt * kTile + i] = v;
    }
    return;
  }

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* q_full = bars + 0;
  uint64_t* o_full = bars + 1;
  uint64_t* pv_done = bars + 2;
  uint64_t* s_full = bars + 3;   // [2]
  uint64_t* p_full = bars + 5;   // [2]
  uint64_t* k_full = bars + 7;   // [S]
  uint64_t* v_full = bars + 7 + S;
  uint64_t* kv_empty = bars + 7 + 2 * S;
  float* red_max = reinterpret_cast<float*>(smem + L::kRed);
  float* red_l = reinterpret_cast<float*>(smem + L::kRedL);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  const WaitCtx wctx{p.status, p.wait_ns, abort_flag};

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(o_full, 1);
    mbar_init(pv_done, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full + i, 1);
      mbar_init(p_full + i, 8);
    }
    for (int i = 0; i < S; ++i) {
      mbar_init(k_full + i, 1);
      mbar_init(v_full + i, 1);
      mbar_init(kv_empty + i, 1);
    }
    *abort_flag = 0;
    *reinterpret_cast<volatile int*>(smem + L::kMisc + 8) = 0;  // drain flag
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tq);
      tma_prefetch_desc(&tk);
      tma_prefetch_desc(&tv);
      mbar_arrive_expect_tx(q_full, L::kTileBytes);
      for (int x = 0; x < L::kBoxes; ++x)
        tma_load_4d(smem + L::kQ + x * L::kBoxBytes, &tq, q_full, x * 64, qt * kTile, h, b);
      int issued = 0;
      for (int j = 0; j < n; ++j) {
        const int s = j % S;
        if (j >= S && !mbar_wait(kv_empty + s, ((j / S) - 1) & 1, wctx)) break;
        const int kt = p.col_idx[e0 + j];
        mbar_arrive_expect_tx(k_full + s, L::kTileBytes);
        for (int x = 0; x < L::kBoxes; ++x)
          tma_load_4d(smem + L::kK + s * L::kTileBytes + x * L::kBoxBytes, &tk, k_full + s,
                      x * 64, kt * kTile, h, b);
        mbar_arrive_expect_tx(v_full + s, L::kTileBytes);
        for (int x = 0; x < L::kBoxes; ++x)
          tma_load_4d(smem + L::kV + s * L::kTileBytes + x * L::kBoxBytes, &tv, v_full + s,
                      x * 64, kt * kTile, h, b);
        issued = j + 1;
      }
      if (*abort_flag) {
        // Let the copies still in flight land before the CTA's shared memory goes away.
        mbar_wait(q_full, 0, WaitCtx{p.status, p.wait_ns, reinterpret_cast<volatile int*>(
                                                               smem + L::kMisc + 8)});
        for (int j = max(0, issued - S); j < issued; ++j) {
          const WaitCtx drain{p.status, p.wait_ns,
                              reinterpret_cast<volatile int*>(smem + L::kMisc + 8)};
          mbar_wait(k_full + j % S, (j / S) & 1, drain);
          mbar_wait(v_full + j % S, (j / S) & 1, drain);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, true);
      const uint32_t q_base = smem_u32(smem + L::kQ);
      bool ok = mbar_wait(q_full, 0, wctx);
      tc_fence_after();
      for (int j = 0; ok && j <= n; ++j) {
        if (j < n) {
          const int s = j % S;
          if (!(ok = mbar_wait(k_full + s, (j / S) & 1, wctx))) break;
          tc_fence_after();
          const uint32_t k_base = smem_u32(smem + L::kK + s * L::kTileBytes);
          const uint32_t d_tmem = tmem + (j & 1) * 128;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * L::kBoxBytes + (kk & 3) * 32;
            mma_ss(d_tmem, smem_desc_sw128(q_base + off, 16, 1024),
                   smem_desc_sw128(k_base + off, 16, 1024), idesc_qk, kk > 0);
          }
          mma_commit(s_full + (j & 1));
        }
        if (j >= 1) {
          const int jj = j - 1, s2 = jj % S, pb = jj & 1;
          if (!(ok = mbar_wait(p_full + pb, (jj >> 1) & 1, wctx))) break;
          if (!(ok = mbar_wait(v_full + s2, (jj / S) & 1, wctx))) break;
          tc_fence_after();
          const uint32_t v_base = smem_u32(smem + L::kV + s2 * L::kTileBytes);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t a_tmem = tmem + pb * 128 + (kk >> 2) * 64 + (kk & 3) * 8;
            mma_ts(tmem + 256, a_tmem, smem_desc_sw128(v_base + kk * 2048, L::kBoxBytes, 1024),
                   idesc_pv, (jj > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(kv_empty + s2);
          if (EPI != 0) mma_commit(pv_done);
        }
      }
      mma_commit(o_full);
    }
  } else if (warp >= kEpiWarp0) {
    // ---------------------------------------------------------------- epilogue
    const int g = (warp - kEpiWarp0) >> 2;  // warpgroup: S columns [64g, 64g+64)
    const int wq = warp & 3;                // TMEM lanes [32 wq, 32 wq + 32)
    const int row = wq * 32 + lane;
    const int rg = qt * kTile + row;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const float bias_r = (p.bias != nullptr && rg < p.Nq) ? p.bias[b * p.bias_sb + rg] : 0.0f;
    // sigmoid: sigma(x) = 0.5 + 0.5 tanh(x/2), x = scale s + bias -> (c1, c0) = halves;
    // softmax: t = (scale s + bias) log2 e
    const float c1 = EPI == 0 ? 0.5f * p.scale : p.scale * kLog2e;
    const float c0 = EPI == 0 ? 0.5f * bias_r : bias_r * kLog2e;
    float m_run = EPI == 2 ? 0.0f : kNegBig;  // base-2 running max (softmax modes)
    float l_run = (EPI == 2 && g == 0) ? 1.0f : 0.0f;
    // `ok` stays warp-uniform (tcgen05.ld/st are warp-collective).  After an abort the
    // loop keeps running without touching TMEM so that every epilogue thread executes the
    // same sequence of named barriers (softmax modes) and nobody waits forever.
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      const int sb = j & 1;
      if (ok) ok = mbar_wait(s_full + sb, (j >> 1) & 1, wctx);
      ok = __all_sync(0xFFFFFFFFu, ok);
      if (ok) tc_fence_after();
      const int e = e0 + j;
      const int kd = p.kind[e];
      uint32_t mw0 = 0xFFFFFFFFu, mw1 = 0xFFFFFFFFu;
      if (kd == 2) {
        const uint2 mb = *reinterpret_cast<const uint2*>(
            p.bits + static_cast<int64_t>(p.pidx[e]) * 512 + row * 4 + g * 2);
        mw0 = mb.x;
        mw1 = mb.y;
      }
      uint32_t sr[64];
      if (ok) {
        tmem_ld32(t_lane + sb * 128 + g * 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        tmem_ld32(t_lane + sb * 128 + g * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int c = 0; c < 64; ++c) sr[c] = 0u;
      }
      float pv[64];
      if (EPI == 0) {
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const float sg = sigmoid_tanh(__uint_as_float(sr[c]), c1, c0);
          const uint32_t bit = ((c < 32 ? mw0 : mw1) >> (c & 31)) & 1u;
          pv[c] = bit ? sg : 0.0f;
        }
      } else {
        float tmax = kNegBig;
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const float t = fmaf(__uint_as_float(sr[c]), c1, c0);
          const uint32_t bit = ((c < 32 ? mw0 : mw1) >> (c & 31)) & 1u;
          pv[c] = bit ? t : kNegBig;
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
          // O must not be read while PV_{j-1} may still accumulate into it.
          ok = mbar_wait(pv_done, (j - 1) & 1, wctx);
          ok = __all_sync(0xFFFFFFFFu, ok);
          if (ok) {
            tc_fence_after();
            constexpr int kOc = D / 2;  // O columns of this warpgroup
#pragma unroll
            for (int c0o = 0; c0o < kOc; c0o += 32) {
              uint32_t orr[32];
              tmem_ld32(t_lane + 256 + g * kOc + c0o, orr);
              tmem_wait_ld();
#pragma unroll
              for (int c = 0; c < 32; ++c)
                orr[c] = __float_as_uint(__uint_as_float(orr[c]) * alpha);
              tmem_st32(t_lane + 256 + g * kOc + c0o, orr);
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
    if (ok) ok = mbar_wait(o_full, 0, wctx);
    ok = __all_sync(0xFFFFFFFFu, ok);
    float inv_l = 1.0f;
    if (EPI != 0) {
      red_l[g * 128 + row] = l_run;
      named_barrier_sync(1, 256);
      const float l_tot = l_run + red_l[(g ^ 1) * 128 + row];
      inv_l = l_tot > 0.0f ? 1.0f / l_tot : 0.0f;
      if (ok && g == 0 && rg < p.Nq) {
        const float lse = l_tot > 0.0f ? (m_run + __log2f(l_tot)) * kLn2 : -INFINITY;
        p.lse[(static_cast<int64_t>(b) * p.H + h) * p.Nq + rg] = lse;
      }
    }
    if (ok) {
      tc_fence_after();
      constexpr int kOc = D / 2;
      __nv_bfloat16* dst = p.o + b * p.o_sb + static_cast<int64_t>(rg) * p.o_sn + h * p.o_sh +
                           g * kOc;
#pragma unroll
      for (int c0o = 0; c0o < kOc; c0o += 32) {
        uint32_t orr[32];
        tmem_ld32(t_lane + 256 + g * kOc + c0o, orr);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 16; ++c)
          pk[c] = pack_bf16x2(__uint_as_float(orr[2 * c]) * inv_l,
                              __uint_as_float(orr[2 * c + 1]) * inv_l);
        if (rg < p.Nq) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + c0o);
#pragma unroll
          for (int c = 0; c < 4; ++c)
            d4[c] = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        }
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
  p.row_work = plan->row_work;
  p.QT = plan->QT;
  p.Nq = plan->Nq;
  p.H = H;
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
  auto kern = fwd_kernel<D, EPI>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
  if (e != cudaSuccess) return cuda_status(e);
  const int64_t blocks = static_cast<int64_t>(plan->B) * plan->QT * H;
  kern<<<static_cast<unsigned>(blocks), kThreads, L::kAlloc, stream>>>(tq, tk, tv, p);
  return cuda_status(cudaGetLastError());
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
