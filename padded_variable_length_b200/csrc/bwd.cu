// Backward kernels (dK/dV and dQ); filled in below the forward.
#include "internal.h"

namespace sigattn {

int launch_bwd_impl(const sigattn_plan*, int, int, int, float, const CUtensorMap&,
                    const CUtensorMap&, const CUtensorMap&, const CUtensorMap&, const TensorDesc&,
                    const TensorDesc&, const float*, int64_t, const float*, float*,
                    const TensorDesc&, const TensorDesc&, const TensorDesc&, int*,
                    unsigned long long, cudaStream_t) {
  return SIGATTN_ERR_UNSUPPORTED;
}

}  // namespace sigattn
