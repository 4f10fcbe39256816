// fa_merge.cu — folds one partial attention result into fp32 accumulators.
//
// Ring attention ("深度解析注意力机制的变体与演进", Ring Attention) attends each
// device's query block to one key/value block per step and combines the
// partial results.  The combination is the online-softmax renormalisation
// ("从理论到实现：基于Triton剖析FlashAttention三代的演进与优化" §2.1) applied to
// whole blocks, with the log-sum-exp in place of the running max:
//     LSE = log(exp(LSE_acc) + exp(LSE_part))
//     O   = exp(LSE_acc - LSE) * O_acc + exp(LSE_part - LSE) * O_part
// An empty side (LSE = -inf) contributes nothing.
//
// HBM-bound: one pass over the partial (16-bit) and the accumulator (fp32).
// A warp covers 32 / (d / 8) rows; each lane owns 8 consecutive elements of
// one row (16-byte loads of the partial, 32-byte of the accumulator).  The
// row's LSE is read by all its lanes before lane 0 of the row rewrites it.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "fa_launch.h"

namespace fa {
namespace {

template <bool F16>
__device__ __forceinline__ void unpack8(const uint4 u, float (&x)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if constexpr (F16) {
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
      x[2 * i] = f.x;
      x[2 * i + 1] = f.y;
    } else {
      x[2 * i] = __uint_as_float(w[i] << 16);
      x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
}

template <bool F16>
__device__ __forceinline__ uint4 pack8(const float (&x)[8]) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if constexpr (F16) {
      const __half2 h = __floats2half2_rn(x[2 * i], x[2 * i + 1]);
      w[i] = *reinterpret_cast<const uint32_t*>(&h);
    } else {
      const __nv_bfloat162 h = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
      w[i] = *reinterpret_cast<const uint32_t*>(&h);
    }
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

template <int D, bool F16>
__global__ void __launch_bounds__(256) merge_kernel(const uint4* __restrict__ o_part, const float* __restrict__ lse_part,
                                                    float* __restrict__ o_acc, float* __restrict__ lse_acc,
                                                    uint4* __restrict__ o_out, long long rows, int first) {
  constexpr int VPR = D / 8;  // 8-element vectors per row
  constexpr int RPW = 32 / VPR;
  const int lane = threadIdx.x & 31;
  const long long warp = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long long row = warp * RPW + lane / VPR;
  const int vec = lane % VPR;
  const bool valid = row < rows;
  const long long v = row * VPR + vec;  // vector index within the [rows, D] tensor

  float part[8], acc[8];
  float lse = -INFINITY;
  if (valid) {
    unpack8<F16>(o_part[v], part);
    const float lp = lse_part[row];
    if (first) {
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = part[i];
      lse = lp;
    } else {
      const float la = lse_acc[row];
      const float4 a0 = reinterpret_cast<const float4*>(o_acc)[2 * v];
      const float4 a1 = reinterpret_cast<const float4*>(o_acc)[2 * v + 1];
      const float old[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float hi = fmaxf(la, lp);
      if (hi == -INFINITY) {  // both sides empty
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.f;
      } else {
        const float w_old = expf(la - hi), w_new = expf(lp - hi);
        const float tot = w_old + w_new;
        const float a = w_old / tot, b = w_new / tot;
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = a * old[i] + b * part[i];
        lse = hi + logf(tot);
      }
    }
  }
  __syncwarp();  // every lane has read the row's old LSE before it is rewritten
  if (!valid) return;
  if (o_out != nullptr) {
    o_out[v] = pack8<F16>(acc);
  } else {
    reinterpret_cast<float4*>(o_acc)[2 * v] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    reinterpret_cast<float4*>(o_acc)[2 * v + 1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
  }
  if (vec == 0) lse_acc[row] = lse;
}

template <int D>
cudaError_t launch_merge_d(const void* o_part, const float* lse_part, float* o_acc, float* lse_acc, void* o_out,
                           long long rows, bool f16, int first, cudaStream_t stream) {
  constexpr int RPW = 32 / (D / 8);
  const long long warps = (rows + RPW - 1) / RPW;
  const long long blocks = (warps + 7) / 8;
  if (blocks > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  const auto* p = static_cast<const uint4*>(o_part);
  auto* out = static_cast<uint4*>(o_out);
  if (f16)
    merge_kernel<D, true><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(p, lse_part, o_acc, lse_acc, out, rows,
                                                                               first);
  else
    merge_kernel<D, false><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(p, lse_part, o_acc, lse_acc, out, rows,
                                                                                first);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_merge_partial(const void* o_part, const float* lse_part, float* o_acc, float* lse_acc, void* o_out,
                                 long long rows, int d, bool f16, int first, cudaStream_t stream) {
  switch (d) {
    case 32: return launch_merge_d<32>(o_part, lse_part, o_acc, lse_acc, o_out, rows, f16, first, stream);
    case 64: return launch_merge_d<64>(o_part, lse_part, o_acc, lse_acc, o_out, rows, f16, first, stream);
    case 128: return launch_merge_d<128>(o_part, lse_part, o_acc, lse_acc, o_out, rows, f16, first, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace fa
