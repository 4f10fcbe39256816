// fa_fwd_sparse.cu — block-sparse instantiations of the forward kernel (the
// roles walk the plan rows built by fa_plan.cu).
#include "fa_fwd_launch.cuh"

namespace fa {

cudaError_t launch_fwd_sparse(int d, int elem, const FwdLaunch& l) {
  if (elem == kElemE4M3) return d == 128 ? launch_fwd_t<128, kElemE4M3, true>(l) : cudaErrorInvalidValue;
  const bool f16 = elem == kElemF16;
  switch (d) {
    case 32: return f16 ? launch_fwd_t<32, kElemF16, true>(l) : launch_fwd_t<32, kElemBF16, true>(l);
    case 64: return f16 ? launch_fwd_t<64, kElemF16, true>(l) : launch_fwd_t<64, kElemBF16, true>(l);
    case 128: return f16 ? launch_fwd_t<128, kElemF16, true>(l) : launch_fwd_t<128, kElemBF16, true>(l);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace fa
