// fa_fwd_fp8.cu — e4m3 Q/K instantiation of the forward kernel (V, O bf16).
#include "fa_fwd_launch.cuh"

namespace fa {

cudaError_t launch_fwd_e4m3(int d, const FwdLaunch& l) {
  if (d != 128) return cudaErrorInvalidValue;
  if (l.args->plan != nullptr) return launch_fwd_sparse(d, kElemE4M3, l);
  return launch_fwd_t<128, kElemE4M3, false>(l);
}

}  // namespace fa
