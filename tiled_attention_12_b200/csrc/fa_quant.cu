// fa_quant.cu — per-(batch, head, 128-row tile) dynamic-scale e4m3 quantiser.
//
// "从理论到实现：基于Triton剖析FlashAttention三代的演进与优化" §4.1 derives a
// dynamic scale from the operand's absolute maximum and undoes it on the
// product; with the e4m3 format the scale maps the tile's amax onto 448, the
// largest finite e4m3 value:
//     scale = 448 / amax   (1 for an all-zero tile)
//     code  = e4m3_rne_satfinite(x * scale)
// Both the division and the multiply are single IEEE fp32 operations with
// round-to-nearest-even, so the codes are reproducible bit for bit.
//
// One CTA of 256 threads per tile: a vectorised amax pass, a block reduction,
// then a second pass over the same 16-byte vectors (served from L1/L2) that
// scales, converts pairs and stores 8 codes per vector.  HBM-bound: reads the
// tile once from DRAM and writes half as many bytes.
#include <cuda_runtime.h>

#include <cstdint>

#include "fa_launch.h"

namespace fa {

namespace {

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Two fp32 -> two e4m3 codes; `lo` lands in the low byte.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// x is read at element strides (batch, head, row); its rows are contiguous.
// TR = false: the codes are written contiguously as [B*H, N, d].
// TR = true: each head's codes are written transposed, [B*H, d, np] (np a
// multiple of 128, keys past N zero), so that a tile of them is a K-major
// operand for the P V product (keys along the K dimension).
template <bool TR>
__global__ void __launch_bounds__(256) quantize_e4m3_kernel(const uint16_t* __restrict__ x, uint2* __restrict__ x8,
                                                            float* __restrict__ scales, int H, int N, int d,
                                                            int n_tiles, int vec_shift, long long sb, long long sh,
                                                            long long sn, long long np) {
  const int t = blockIdx.x % n_tiles;
  const int bh = blockIdx.x / n_tiles;
  const int b = bh / H, h = bh - b * H;
  const int r0 = t * 128;
  const int rows = (N - r0) < 128 ? (N - r0) : 128;
  const size_t vec0 = ((static_cast<size_t>(bh) * N + r0) * d) / 8;  // 8 elements per vector
  const int n_vec = rows * d / 8;
  const uint16_t* tile = x + b * sb + h * sh + r0 * sn;
  const int vec_mask = (1 << vec_shift) - 1;  // vectors per row - 1
  // the 16-byte vector v of the tile: row v >> vec_shift, column vector v & vec_mask
  auto load = [&](int v) {
    return *reinterpret_cast<const uint4*>(tile + (v >> vec_shift) * sn + (v & vec_mask) * 8);
  };
  float amax = 0.f;
  for (int v = threadIdx.x; v < n_vec; v += 256) {
    const uint4 u = load(v);
    amax = fmaxf(amax, fmaxf(fmaxf(fabsf(bf16_lo(u.x)), fabsf(bf16_hi(u.x))),
                             fmaxf(fabsf(bf16_lo(u.y)), fabsf(bf16_hi(u.y)))));
    amax = fmaxf(amax, fmaxf(fmaxf(fabsf(bf16_lo(u.z)), fabsf(bf16_hi(u.z))),
                             fmaxf(fabsf(bf16_lo(u.w)), fabsf(bf16_hi(u.w)))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  __shared__ float warp_max[8];
  if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = warp_max[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) amax = fmaxf(amax, warp_max[i]);
  const float sc = amax > 0.f ? __fdiv_rn(448.0f, amax) : 1.0f;

  __shared__ __align__(16) uint8_t staged[TR ? 128 * 128 : 16];  // TR: [row][col] codes of the tile
  for (int v = threadIdx.x; v < n_vec; v += 256) {
    const uint4 u = load(v);
    const uint32_t c0 = cvt_e4m3x2(__fmul_rn(bf16_lo(u.x), sc), __fmul_rn(bf16_hi(u.x), sc));
    const uint32_t c1 = cvt_e4m3x2(__fmul_rn(bf16_lo(u.y), sc), __fmul_rn(bf16_hi(u.y), sc));
    const uint32_t c2 = cvt_e4m3x2(__fmul_rn(bf16_lo(u.z), sc), __fmul_rn(bf16_hi(u.z), sc));
    const uint32_t c3 = cvt_e4m3x2(__fmul_rn(bf16_lo(u.w), sc), __fmul_rn(bf16_hi(u.w), sc));
    const uint2 codes = make_uint2(c0 | (c1 << 16), c2 | (c3 << 16));
    if constexpr (TR)
      *reinterpret_cast<uint2*>(staged + v * 8) = codes;  // row v >> vec_shift, column (v & vec_mask) * 8
    else
      x8[vec0 + v] = codes;
  }
  if constexpr (TR) {
    for (int i = n_vec * 8 + threadIdx.x; i < 128 * d; i += 256) staged[i] = 0;  // rows past the sequence end
    __syncthreads();
    // row `col` of the transposed tile: 128 keys in 8 chunks of 16 bytes
    uint8_t* out = reinterpret_cast<uint8_t*>(x8) + static_cast<size_t>(bh) * d * np + r0;
    for (int w = threadIdx.x; w < d * 8; w += 256) {
      const int col = w >> 3, kc = w & 7;
      uint32_t word[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int r = kc * 16 + q * 4;
        word[q] = static_cast<uint32_t>(staged[r * d + col]) |
                  (static_cast<uint32_t>(staged[(r + 1) * d + col]) << 8) |
                  (static_cast<uint32_t>(staged[(r + 2) * d + col]) << 16) |
                  (static_cast<uint32_t>(staged[(r + 3) * d + col]) << 24);
      }
      *reinterpret_cast<uint4*>(out + static_cast<size_t>(col) * np + kc * 16) =
          make_uint4(word[0], word[1], word[2], word[3]);
    }
  }
  if (threadIdx.x == 0) scales[static_cast<size_t>(bh) * n_tiles + t] = sc;
}

// Smallest scale of each head's tiles (one warp per head).
__global__ void __launch_bounds__(256) min_scale_kernel(const float* __restrict__ scales, float* __restrict__ out,
                                                        int BH, int n_tiles) {
  const int head = static_cast<int>((blockIdx.x * static_cast<unsigned>(blockDim.x) + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (head >= BH) return;  // whole warps leave together
  float m = INFINITY;
  for (int t = lane; t < n_tiles; t += 32) m = fminf(m, scales[static_cast<size_t>(head) * n_tiles + t]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fminf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) out[head] = m;
}

}  // namespace

cudaError_t launch_quantize_e4m3(const void* x, void* x8, float* scales, int B, int H, int N, int d,
                                 const Strides& st, cudaStream_t stream) {
  const int n_tiles = (N + 127) / 128;
  const long long blocks = static_cast<long long>(n_tiles) * B * H;
  if (blocks > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  const int vec_shift = d == 32 ? 2 : (d == 64 ? 3 : 4);  // log2(d / 8) vectors per row
  if ((8 << vec_shift) != d) return cudaErrorInvalidValue;
  quantize_e4m3_kernel<false><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
      static_cast<const uint16_t*>(x), static_cast<uint2*>(x8), scales, H, N, d, n_tiles, vec_shift, st.b, st.h, st.n,
      0);
  return cudaGetLastError();
}

long long transposed_row(int N) { return (static_cast<long long>(N) + 127) / 128 * 128; }

cudaError_t launch_quantize_e4m3_t(const void* x, void* x8t, float* scales, int B, int H, int N, int d,
                                   const Strides& st, cudaStream_t stream) {
  const int n_tiles = (N + 127) / 128;
  const long long blocks = static_cast<long long>(n_tiles) * B * H;
  if (blocks > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  const int vec_shift = d == 32 ? 2 : (d == 64 ? 3 : 4);
  if ((8 << vec_shift) != d) return cudaErrorInvalidValue;
  quantize_e4m3_kernel<true><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
      static_cast<const uint16_t*>(x), static_cast<uint2*>(x8t), scales, H, N, d, n_tiles, vec_shift, st.b, st.h,
      st.n, transposed_row(N));
  return cudaGetLastError();
}

cudaError_t launch_min_scale(const float* scales, float* out, int BH, int N, cudaStream_t stream) {
  const int n_tiles = (N + 127) / 128;
  const long long blocks = (static_cast<long long>(BH) + 7) / 8;
  if (blocks > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  min_scale_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(scales, out, BH, n_tiles);
  return cudaGetLastError();
}

}  // namespace fa
