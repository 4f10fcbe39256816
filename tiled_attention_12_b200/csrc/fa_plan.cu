// fa_plan.cu — block-sparse plan builder: turns a per-head 128 x 128 block
// mask into the per-work-tile K/V lists the forward kernel walks
// ("深度解析注意力机制的变体与演进", Block Sparse Attention: only the chosen
// blocks of the attention matrix are computed).
//
// One warp per work tile (two consecutive 128-row Q tiles of one head).  For
// each 32 K/V tiles the warp ballots which tiles Q tile 0, Q tile 1 and
// either of them use, and compacts the indices with prefix popcounts, so the
// lists come out in ascending tile order.  Causal additionally drops tiles
// above each Q tile's diagonal.
#include <cuda_runtime.h>

#include <cstdint>

#include "fa_fwd_kernel.cuh"
#include "fa_launch.h"

namespace fa {
namespace {

__global__ void __launch_bounds__(256) block_sparse_plan_kernel(const uint8_t* __restrict__ mask,
                                                                uint16_t* __restrict__ plan, int BH, int n_qtiles,
                                                                int n_qpairs, int stride, int causal) {
  const int pair = static_cast<int>((blockIdx.x * static_cast<unsigned>(blockDim.x) + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (pair >= BH * n_qpairs) return;  // whole warps leave together
  const int bh = pair / n_qpairs;
  const int qt0 = 2 * (pair - bh * n_qpairs), qt1 = qt0 + 1;
  const bool has1 = qt1 < n_qtiles;
  const uint8_t* r0 = mask + (static_cast<size_t>(bh) * n_qtiles + qt0) * n_qtiles;
  const uint8_t* r1 = r0 + n_qtiles;
  uint16_t* row = plan + static_cast<size_t>(pair) * (kPlanHeader + 3 * stride);
  uint16_t* uni = row + kPlanHeader;
  uint16_t* l0 = uni + stride;
  uint16_t* l1 = l0 + stride;
  const unsigned below = (1u << lane) - 1u;
  int cu = 0, c0 = 0, c1 = 0;
  for (int base = 0; base < n_qtiles; base += 32) {
    const int j = base + lane;
    const bool in = j < n_qtiles;
    const bool a0 = in && r0[j] != 0 && (!causal || j <= qt0);
    const bool a1 = in && has1 && r1[j] != 0 && (!causal || j <= qt1);
    const unsigned bu = __ballot_sync(0xffffffffu, a0 || a1);
    const unsigned b0 = __ballot_sync(0xffffffffu, a0);
    const unsigned b1 = __ballot_sync(0xffffffffu, a1);
    if (a0 || a1) uni[cu + __popc(bu & below)] = static_cast<uint16_t>((j << 2) | (a0 ? 1 : 0) | (a1 ? 2 : 0));
    if (a0) l0[c0 + __popc(b0 & below)] = static_cast<uint16_t>(j);
    if (a1) l1[c1 + __popc(b1 & below)] = static_cast<uint16_t>(j);
    cu += __popc(bu);
    c0 += __popc(b0);
    c1 += __popc(b1);
  }
  if (lane < kPlanHeader) row[lane] = static_cast<uint16_t>(lane == 0 ? cu : lane == 1 ? c0 : lane == 2 ? c1 : 0);
}

}  // namespace

int block_sparse_plan_stride(int N) { return (((N + 127) / 128) + 7) / 8 * 8; }

size_t block_sparse_plan_bytes(int BH, int N) {
  const size_t pairs = static_cast<size_t>(BH) * ((N + 255) / 256);
  return pairs * 2 * (kPlanHeader + 3 * static_cast<size_t>(block_sparse_plan_stride(N)));
}

cudaError_t launch_block_sparse_plan(const uint8_t* mask, uint16_t* plan, int BH, int N, int causal,
                                     cudaStream_t stream) {
  const int n_qtiles = (N + 127) / 128;
  const int n_qpairs = (N + 255) / 256;
  const long long warps = static_cast<long long>(BH) * n_qpairs;
  const int blocks = static_cast<int>((warps + 7) / 8);
  block_sparse_plan_kernel<<<blocks, 256, 0, stream>>>(mask, plan, BH, n_qtiles, n_qpairs,
                                                       block_sparse_plan_stride(N), causal);
  return cudaGetLastError();
}

}  // namespace fa
