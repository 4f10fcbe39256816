// fa_fwd_launch.cuh — launches one instantiation of the forward kernel.
#pragma once

#include "fa_fwd_kernel.cuh"
#include "fa_launch.h"

namespace fa {

// BS: the block-sparse instantiation (walks l.args->plan); the dense one
// compiles without any of the plan logic.
template <int D, int ELEM, bool BS>
cudaError_t launch_fwd_t(const FwdLaunch& l) {
  using C = FwdCfg<D, ELEM>;
  auto kernel = fa_fwd_kernel<D, ELEM, BS>;
  // The attribute is per device; setting it again is harmless.
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  kernel<<<l.grid, C::THREADS, C::SMEM_BYTES, l.stream>>>(l.map_q, l.map_k, l.map_v, *l.args);
  return cudaGetLastError();
}

}  // namespace fa
