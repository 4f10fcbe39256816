// fa_fwd_fp8.cu — e4m3 instantiations of the forward kernel: Q, K in e4m3
// with V, P, O bf16; and Q, K, V, P all in e4m3 (O bf16).
#include "fa_fwd_launch.cuh"

namespace fa {

cudaError_t launch_fwd_e4m3(int d, const FwdLaunch& l) {
  if (d != 128) return cudaErrorInvalidValue;
  if (l.args->plan != nullptr) return launch_fwd_sparse(d, kElemE4M3, l);
  return launch_fwd_t<128, kElemE4M3, false>(l);
}

cudaError_t launch_fwd_e4m3_all(int d, const FwdLaunch& l) {
  if (d != 128 || l.args->plan != nullptr) return cudaErrorInvalidValue;
  return launch_fwd_t<128, kElemE4M3All, false>(l);
}

}  // namespace fa
