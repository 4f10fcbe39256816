// fa_fwd_16bit.cu — bf16 and fp16 instantiations of the forward kernel.
#include "fa_fwd_launch.cuh"

namespace fa {

cudaError_t launch_fwd_bf16(int d, const FwdLaunch& l) {
  if (l.args->plan != nullptr) return launch_fwd_sparse(d, kElemBF16, l);
  switch (d) {
    case 32: return launch_fwd_t<32, kElemBF16, false>(l);
    case 64: return launch_fwd_t<64, kElemBF16, false>(l);
    case 128: return launch_fwd_t<128, kElemBF16, false>(l);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_fwd_f16(int d, const FwdLaunch& l) {
  if (l.args->plan != nullptr) return launch_fwd_sparse(d, kElemF16, l);
  switch (d) {
    case 32: return launch_fwd_t<32, kElemF16, false>(l);
    case 64: return launch_fwd_t<64, kElemF16, false>(l);
    case 128: return launch_fwd_t<128, kElemF16, false>(l);
    default: return cudaErrorInvalidValue;
  }
}

int fwd_smem_bytes(int d, int elem) {
  if (elem == kElemE4M3) return FwdCfg<128, kElemE4M3>::SMEM_BYTES;
  switch (d) {
    case 32: return FwdCfg<32, kElemBF16>::SMEM_BYTES;
    case 64: return FwdCfg<64, kElemBF16>::SMEM_BYTES;
    default: return FwdCfg<128, kElemBF16>::SMEM_BYTES;
  }
}

}  // namespace fa

#ifdef FA_TRACE
// Trace-enabled builds only: copies the trace array (8 slices of
// FA_TRACE_CAP / 8 records; unused records are 0) out and clears it.
extern "C" int fa_trace_read(unsigned long long* host, int cap) {
  if (cap < FA_TRACE_CAP) return -1;
  if (cudaMemcpyFromSymbol(host, fa::g_fa_trace, FA_TRACE_CAP * sizeof(unsigned long long)) != cudaSuccess)
    return -1;
  static unsigned long long zeros[FA_TRACE_CAP];
  if (cudaMemcpyToSymbol(fa::g_fa_trace, zeros, sizeof(zeros)) != cudaSuccess) return -1;
  return FA_TRACE_CAP;
}
#endif
