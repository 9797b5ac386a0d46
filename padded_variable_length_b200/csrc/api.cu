// C ABI of libsigattn.so: argument checks, TMA descriptors, the device status word, and
// the small helper kernels (bias, bounded-wait self-test).  The attention kernels live in
// fwd.cu and bwd.cu, the planner in plan.cu.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <mutex>

#include "internal.h"
#include "sm100.cuh"

namespace sigattn {

__device__ int g_status_word;

int launch_fwd_impl(const sigattn_plan* plan, int epilogue, int H, int d, float scale,
                    const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                    const float* bias, int64_t bias_sb, const TensorDesc& o, float* lse,
                    int* status, unsigned long long wait_ns, cudaStream_t stream);

int launch_bwd_impl(const sigattn_plan* plan, int epilogue, int H, int d, float scale,
                    const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                    const CUtensorMap& tdo, const TensorDesc& o, const TensorDesc& dout,
                    const float* bias, int64_t bias_sb, const float* lse, float* workspace,
                    const TensorDesc& dq, const TensorDesc& dk, const TensorDesc& dv,
                    int parts, int* status, unsigned long long wait_ns, cudaStream_t stream);

int launch_bwd_fused_impl(const sigattn_plan* plan, int epilogue, int H, float scale,
                          const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                          const CUtensorMap& tdo, const CUtensorMap& tdq, const TensorDesc& o,
                          const TensorDesc& dout, const float* bias, int64_t bias_sb,
                          const float* lse, float* Dws, float* dqacc, const TensorDesc& dq,
                          const TensorDesc& dk, const TensorDesc& dv, int* status,
                          unsigned long long wait_ns, cudaStream_t stream);

std::atomic<int> g_last_cuda_error{0};

SymbolAddressCache g_status_addr;

int status_ptr(int** out) {
  void* p = nullptr;
  const int rc = g_status_addr.get(g_status_word, &p);
  *out = static_cast<int*>(p);
  return rc;
}

int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return SIGATTN_OK;
  g_last_cuda_error.store(static_cast<int>(e));
  cudaGetLastError();
  return e == cudaErrorMemoryAllocation ? SIGATTN_ERR_NOMEM : SIGATTN_ERR_CUDA;
}

namespace {

std::atomic<unsigned long long> g_wait_limit_ns{2000000000ull};

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    cudaGetLastError();
  });
  return fn;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_tensor(const void* ptr, const int64_t* strides, int64_t N, TensorDesc* t) {
  if (N < 1 || N > 0x7FFFFFFF) return SIGATTN_ERR_UNSUPPORTED;
  if (!ptr || !strides) return SIGATTN_ERR_INVALID;
  for (int i = 0; i < 3; ++i)
    if (strides[i] < 0) return SIGATTN_ERR_INVALID;
  if (!aligned16(ptr)) return SIGATTN_ERR_ALIGNMENT;
  for (int i = 0; i < 3; ++i)
    if (strides[i] % 8 != 0) return SIGATTN_ERR_ALIGNMENT;
  t->ptr = ptr;
  t->sb = strides[0];
  t->sn = strides[1];
  t->sh = strides[2];
  t->N = static_cast<int>(N);
  return SIGATTN_OK;
}

// Rows of the Q-side / K-side tensors and the batch extent of their TMA maps: padded batches
// are [B, N, H, d]; a packed batch is one [T, H, d] tensor (T = the plan's last offset).
int64_t rows_q(const sigattn_plan* plan) { return plan->cu ? plan->T : plan->Nq; }
int64_t rows_k(const sigattn_plan* plan) { return plan->cu ? plan->T : plan->Nk; }
int tma_batches(const sigattn_plan* plan) { return plan->cu ? 1 : plan->B; }

int check_plan_device(const sigattn_plan* plan) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return SIGATTN_ERR_NO_DEVICE;
  }
  return dev == plan->device ? SIGATTN_OK : SIGATTN_ERR_SHAPE;
}

__global__ void k_bias_from_counts(const int32_t* __restrict__ counts, int64_t n,
                                   float* __restrict__ bias) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int c = counts[i];
    bias[i] = c > 0 ? -logf(static_cast<float>(c)) : 0.0f;
  }
}

// Waits on a barrier that nothing ever arrives at; the bounded wait gives up after
// `limit_ns`, records the timeout and the kernel returns.
__global__ void k_wait_selftest(int* status, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncwarp();
  __syncthreads();
  if (threadIdx.x == 0) {
    const WaitCtx w{status, limit_ns, &abort_flag};
    mbar_wait(&bar, 0, w);
  }
  __syncwarp();
  __syncthreads();
}

}  // namespace

int make_tmap_bf16(CUtensorMap* map, const TensorDesc& t, int B, int H, int d) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
  if (!fn) return SIGATTN_ERR_CUDA;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(t.N),
                              static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(B)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(t.sn) * 2,
                                 static_cast<cuuint64_t>(t.sh) * 2,
                                 static_cast<cuuint64_t>(t.sb) * 2};
  const cuuint32_t box[4] = {64, 128, 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(t.ptr), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SIGATTN_OK : SIGATTN_ERR_ALIGNMENT;
}

int make_tmap_f32_acc(CUtensorMap* map, float* base, int B, int N, int H, int d) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
  if (!fn) return SIGATTN_ERR_CUDA;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                              static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(B)};
  const cuuint64_t row = static_cast<cuuint64_t>(d) * 4;  // bytes of one (token, head) row
  const cuuint64_t st[3] = {row * H, row, row * H * N};   // token, head, batch strides
  const cuuint32_t box[4] = {32, 16, 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, base, dims, st, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SIGATTN_OK : SIGATTN_ERR_ALIGNMENT;
}

}  // namespace sigattn

using namespace sigattn;

extern "C" int sigattn_fwd(const sigattn_plan* plan, int epilogue, int H, int d, float scale,
                           const void* q, const int64_t q_strides[3], const void* k,
                           const int64_t k_strides[3], const void* v, const int64_t v_strides[3],
                           const float* bias, int64_t bias_stride_b, void* o,
                           const int64_t o_strides[3], float* lse, sigattn_stream s) {
  if (!plan || H < 1 || !std::isfinite(scale)) return SIGATTN_ERR_INVALID;
  if (epilogue < 0 || epilogue > 2) return SIGATTN_ERR_INVALID;
  if (d != 64 && d != 128) return SIGATTN_ERR_UNSUPPORTED;
  if (epilogue != SIGATTN_SIGMOID && !lse) return SIGATTN_ERR_INVALID;
  if (bias && bias_stride_b < 0) return SIGATTN_ERR_INVALID;
  if (static_cast<int64_t>(plan->B) * plan->QT * H > 0x7FFFFFFF) return SIGATTN_ERR_UNSUPPORTED;
  TensorDesc tq, tk, tv, to;
  int rc;
  if ((rc = check_tensor(q, q_strides, rows_q(plan), &tq)) != SIGATTN_OK) return rc;
  if ((rc = check_tensor(k, k_strides, rows_k(plan), &tk)) != SIGATTN_OK) return rc;
  if ((rc = check_tensor(v, v_strides, rows_k(plan), &tv)) != SIGATTN_OK) return rc;
  if ((rc = check_tensor(o, o_strides, rows_q(plan), &to)) != SIGATTN_OK) return rc;
  if ((rc = check_plan_device(plan)) != SIGATTN_OK) return rc;
  if ((rc = plan_wait(plan, static_cast<cudaStream_t>(s))) != SIGATTN_OK) return rc;
  int* status = nullptr;
  if ((rc = status_ptr(&status)) != SIGATTN_OK) return rc;
  CUtensorMap mq, mk, mv;
  if ((rc = make_tmap_bf16(&mq, tq, tma_batches(plan), H, d)) != SIGATTN_OK) return rc;
  if ((rc = make_tmap_bf16(&mk, tk, tma_batches(plan), H, d)) != SIGATTN_OK) return rc;
  if ((rc = make_tmap_bf16(&mv, tv, tma_batches(plan), H, d)) != SIGATTN_OK) return rc;
  return launch_fwd_impl(plan, epilogue, H, d, scale, mq, mk, mv, bias, bias_stride_b, to, lse,
                         status, g_wait_limit_ns.load(), static_cast<cudaStream_t>(s));
}

extern "C" int sigattn_bwd_ex(const sigattn_plan* plan, int epilogue, int H, int d, float scale,
                              const void* q, const int64_t q_strides[3], const void* k,
                              const int64_t k_strides[3], const void* v,
                              const int64_t v_strides[3], const void* o,
                              const int64_t o_strides[3], const void* dout,
                              const int64_t do_strides[3], const float* bias,
                              int64_t bias_stride_b, const float* lse, float* workspace, void* dq,
                              const int64_t dq_strides[3], void* dk, const int64_t dk_strides[3],
                              void* dv, const int64_t dv_strides[3], int parts,
                              sigattn_stream s) {
  if (!plan || H < 1 || !std::isfinite(scale)) return SIGATTN_ERR_INVALID;
  if (parts <= 0 || (parts & ~SIGATTN_BWD_ALL) != 0) return SIGATTN_ERR_INVALID;
  if (epilogue < 0 || epilogue > 2) return SIGATTN_ERR_INVALID;
  if (d != 64 && d != 128) return SIGATTN_ERR_UNSUPPORTED;
  if (epilogue != SIGATTN_SIGMOID && (!lse || !workspace || !o)) return SIGATTN_ERR_INVALID;
  if (bias && bias_stride_b < 0) return SIGATTN_ERR_INVALID;
  if (static_cast<int64_t>(plan->B) * (plan->QT > plan->KT ? plan->QT : plan->KT) * H >
      0x7FFFFFFF)
    return SIGATTN_ERR_UNSUPPORTED;
  TensorDesc tq, tk, tv, to{}, tdo, tdq, tdk, tdv;
  int rc;
  if ((rc = check_tensor(q, q_strides, rows_q(plan), &tq)) != SIGATTN_OK) return rc;
  if ((rc = check_tensor(k, k_strides, rows_k(plan), &tk)) != SIGATTN_OK) return rc;
  if ((rc = check_tensor(v, v_strides, rows_k(plan), &tv)) != SIGATTN_OK) return rc;
  if (epilogue != SIGATTN_SIGMOID &&
      (rc = check_tensor(o, o_strides, rows_q(plan), &to)) != SIGATTN_OK)
    return rc;
  if ((rc = check_tensor(dout, do_strides, rows_q(plan), &tdo)) != SIGATTN_OK) return rc;
  if ((rc = check_tensor(dq, dq_strides, rows_q(plan), &tdq)) != SIGATTN_OK) return rc;
  if ((rc = check_tensor(dk, dk_strides, rows_k(plan), &tdk)) != SIGATTN_OK) return rc;
  if ((rc = check_tensor(dv, dv_strides, rows_k(plan), &tdv)) != SIGATTN_OK) return rc;
  if ((rc = check_plan_device(plan)) != SIGATTN_OK) return rc;
  if ((rc = plan_wait(plan, static_cast<cudaStream_t>(s))) != SIGATTN_OK) return rc;
  int* status = nullptr;
  if ((rc = status_ptr(&status)) != SIGATTN_OK) return rc;
  CUtensorMap mq, mk, mv, mdo;
  if ((rc = make_tmap_bf16(&mq, tq, tma_batches(plan), H, d)) != SIGATTN_OK) return rc;
  if ((rc = make_tmap_bf16(&mk, tk, tma_batches(plan), H, d)) != SIGATTN_OK) return rc;
  if ((rc = make_tmap_bf16(&mv, tv, tma_batches(plan), H, d)) != SIGATTN_OK) return rc;
  if ((rc = make_tmap_bf16(&mdo, tdo, tma_batches(plan), H, d)) != SIGATTN_OK) return rc;
  return launch_bwd_impl(plan, epilogue, H, d, scale, mq, mk, mv, mdo, to, tdo, bias,
                         bias_stride_b, lse, workspace, tdq, tdk, tdv, parts, status,
                         g_wait_limit_ns.load(), static_cast<cudaStream_t>(s));
}

extern "C" int sigattn_bwd_fused_workspace_size(const sigattn_plan* plan, int epilogue, int H,
                                                int d, size_t* bytes) {
  if (!plan || !bytes || H < 1 || epilogue < 0 || epilogue > 2) return SIGATTN_ERR_INVALID;
  if (d != 64) return SIGATTN_ERR_UNSUPPORTED;
  const size_t rows = static_cast<size_t>(plan->B) * plan->Nq * H;
  *bytes = rows * d * sizeof(float) + (epilogue != SIGATTN_SIGMOID ? rows * sizeof(float) : 0);
  return SIGATTN_OK;
}

extern "C" int sigattn_bwd_fused(const sigattn_plan* plan, int epilogue, int H, int d, float scale,
                                 const void* q, const int64_t q_strides[3], const void* k,
                                 const int64_t k_strides[3], const void* v,
                                 const int64_t v_strides[3], const void* o,
                                 const int64_t o_strides[3], const void* dout,
                                 const int64_t do_strides[3], const float* bias,
                                 int64_t bias_stride_b, const float* lse, void* workspace,
                                 size_t workspace_bytes, void* dq, const int64_t dq_strides[3],
                                 void* dk, const int64_t dk_strides[3], void* dv,
                                 const int64_t dv_strides[3], sigattn_stream s) {
  if (!plan || H < 1 || !std::isfinite(scale)) return SIGATTN_ERR_INVALID;
  if (epilogue < 0 || epilogue > 2) return SIGATTN_ERR_INVALID;
  if (d != 64) return SIGATTN_ERR_UNSUPPORTED;
  if (epilogue != SIGATTN_SIGMOID && (!lse || !o)) return SIGATTN_ERR_INVALID;
  if (bias && bias_stride_b < 0) return SIGATTN_ERR_INVALID;
  size_t need = 0;
  int rc = sigattn_bwd_fused_workspace_size(plan, epilogue, H, d, &need);
  if (rc != SIGATTN_OK) return rc;
  if (!workspace || workspace_bytes < need) return SIGATTN_ERR_INVALID;
  if (!aligned16(workspace)) return SIGATTN_ERR_ALIGNMENT;
  if (static_cast<int64_t>(plan->B) * (plan->QT > plan->KT ? plan->QT : plan->KT) * H >
      0x7FFFFFFF)
    return SIGATTN_ERR_UNSUPPORTED;
  TensorDesc tq, tk, tv, to{}, tdo, tdq, tdk, tdv;
  if ((rc = check_tensor(q, q_strides, rows_q(plan), &tq)) != SIGATTN_OK) return rc;
  if ((rc = check_tensor(k, k_strides, rows_k(plan), &tk)) != SIGATTN_OK) return rc;
  if ((rc = check_tensor(v, v_strides, rows_k(plan), &tv)) != SIGATTN_OK) return rc;
  if (epilogue != SIGATTN_SIGMOID &&
      (rc = check_tensor(o, o_strides, rows_q(plan), &to)) != SIGATTN_OK)
    return rc;
  if ((rc = check_tensor(dout, do_strides, rows_q(plan), &tdo)) != SIGATTN_OK) return rc;
  if ((rc = check_tensor(dq, dq_strides, rows_q(plan), &tdq)) != SIGATTN_OK) return rc;
  if ((rc = check_tensor(dk, dk_strides, rows_k(plan), &tdk)) != SIGATTN_OK) return rc;
  if ((rc = check_tensor(dv, dv_strides, rows_k(plan), &tdv)) != SIGATTN_OK) return rc;
  if ((rc = check_plan_device(plan)) != SIGATTN_OK) return rc;
  if ((rc = plan_wait(plan, static_cast<cudaStream_t>(s))) != SIGATTN_OK) return rc;
  int* status = nullptr;
  if ((rc = status_ptr(&status)) != SIGATTN_OK) return rc;
  float* dqacc = static_cast<float*>(workspace);
  float* Dws = epilogue != SIGATTN_SIGMOID
                   ? dqacc + static_cast<size_t>(plan->B) * plan->Nq * H * d
                   : nullptr;
  CUtensorMap mq, mk, mv, mdo, macc;
  if ((rc = make_tmap_bf16(&mq, tq, tma_batches(plan), H, d)) != SIGATTN_OK) return rc;
  if ((rc = make_tmap_bf16(&mk, tk, tma_batches(plan), H, d)) != SIGATTN_OK) return rc;
  if ((rc = make_tmap_bf16(&mv, tv, tma_batches(plan), H, d)) != SIGATTN_OK) return rc;
  if ((rc = make_tmap_bf16(&mdo, tdo, tma_batches(plan), H, d)) != SIGATTN_OK) return rc;
  if ((rc = make_tmap_f32_acc(&macc, dqacc, plan->B, plan->Nq, H, d)) != SIGATTN_OK) return rc;
  return launch_bwd_fused_impl(plan, epilogue, H, scale, mq, mk, mv, mdo, macc, to, tdo, bias,
                               bias_stride_b, lse, Dws, dqacc, tdq, tdk, tdv, status,
                               g_wait_limit_ns.load(), static_cast<cudaStream_t>(s));
}

extern "C" int sigattn_bwd(const sigattn_plan* plan, int epilogue, int H, int d, float scale,
                           const void* q, const int64_t q_strides[3], const void* k,
                           const int64_t k_strides[3], const void* v, const int64_t v_strides[3],
                           const void* o, const int64_t o_strides[3], const void* dout,
                           const int64_t do_strides[3], const float* bias, int64_t bias_stride_b,
                           const float* lse, float* workspace, void* dq,
                           const int64_t dq_strides[3], void* dk, const int64_t dk_strides[3],
                           void* dv, const int64_t dv_strides[3], sigattn_stream s) {
  return sigattn_bwd_ex(plan, epilogue, H, d, scale, q, q_strides, k, k_strides, v, v_strides, o,
                        o_strides, dout, do_strides, bias, bias_stride_b, lse, workspace, dq,
                        dq_strides, dk, dk_strides, dv, dv_strides, SIGATTN_BWD_ALL, s);
}

extern "C" int sigattn_bias_from_counts(const int32_t* d_counts, int64_t n, float* d_bias,
                                        sigattn_stream s) {
  if (n < 0 || (n > 0 && (!d_counts || !d_bias))) return SIGATTN_ERR_INVALID;
  if (n == 0) return SIGATTN_OK;
  const int64_t blocks = std::min<int64_t>((n + 255) / 256, 148 * 16);
  k_bias_from_counts<<<static_cast<unsigned>(blocks), 256, 0, static_cast<cudaStream_t>(s)>>>(
      d_counts, n, d_bias);
  return cuda_status(cudaGetLastError());
}

extern "C" int sigattn_get_status(sigattn_stream s) {
  int* status = nullptr;
  int rc = status_ptr(&status);
  if (rc != SIGATTN_OK) return rc;
  if ((rc = cuda_status(cudaStreamSynchronize(static_cast<cudaStream_t>(s)))) != SIGATTN_OK)
    return rc;
  int word = 0;
  if ((rc = cuda_status(cudaMemcpy(&word, status, sizeof(int), cudaMemcpyDeviceToHost))) !=
      SIGATTN_OK)
    return rc;
  const int zero = 0;
  if ((rc = cuda_status(cudaMemcpy(status, &zero, sizeof(int), cudaMemcpyHostToDevice))) !=
      SIGATTN_OK)
    return rc;
  return (word & kStatusTimeout) ? SIGATTN_ERR_TIMEOUT : SIGATTN_OK;
}

extern "C" int sigattn_set_wait_limit_ns(uint64_t ns) {
  if (ns == 0) return SIGATTN_ERR_INVALID;
  g_wait_limit_ns.store(ns);
  return SIGATTN_OK;
}

extern "C" int sigattn_selftest_wait_timeout(uint64_t ns, sigattn_stream s) {
  if (ns == 0 || ns > 10000000000ull) return SIGATTN_ERR_INVALID;
  int* status = nullptr;
  const int rc = status_ptr(&status);
  if (rc != SIGATTN_OK) return rc;
  k_wait_selftest<<<1, 32, 0, static_cast<cudaStream_t>(s)>>>(status, ns);
  return cuda_status(cudaGetLastError());
}

extern "C" const char* sigattn_error_string(int code) {
  switch (code) {
    case SIGATTN_OK: return "ok";
    case SIGATTN_ERR_INVALID: return "invalid argument";
    case SIGATTN_ERR_UNSUPPORTED: return "unsupported head dim or size";
    case SIGATTN_ERR_ALIGNMENT: return "pointer not 16-byte aligned or stride not a multiple of 8 elements";
    case SIGATTN_ERR_SHAPE: return "the plan belongs to another device";
    case SIGATTN_ERR_CUDA: return "CUDA runtime or driver error";
    case SIGATTN_ERR_TIMEOUT: return "a device-side bounded wait expired";
    case SIGATTN_ERR_NO_DEVICE: return "no CUDA device is current";
    case SIGATTN_ERR_NOMEM: return "device allocation failed";
    case SIGATTN_ERR_PLAN: return "the tile list failed a structural check";
    default: return "unknown error code";
  }
}

extern "C" const char* sigattn_last_cuda_error(void) {
  const int e = g_last_cuda_error.load();
  return e == 0 ? "no CUDA error" : cudaGetErrorName(static_cast<cudaError_t>(e));
}

extern "C" int sigattn_version(void) { return 100; }
