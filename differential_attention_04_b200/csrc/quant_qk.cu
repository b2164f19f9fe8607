// Low-bit codes of the queries or keys, with one absmax scale per (batch,
// head, map) -- the low-bit reading of the peer review "Differential
// Transformer" (Strengths, the activation-outlier bullet, which cites 4-bit
// attention-logit quantisation; Questions, the quantisation bullet: absmax
// quantisation per logit map and per head).
//
//   pass 1  absmax of each group, as the bits of a non-negative float
//           (integer atomicMax on those bits orders like the values)
//   pass 2  scale = absmax / fmax in place (1 for an all-zero group), fmax the
//           format's largest value: 448 for e4m3, 6 for e2m1
//   pass 3  code = fmt(x / scale): float32 division, round to nearest even,
//           saturating at +-fmax
//
// x is [B, N, H, 2, d]; group g = (b * H + h) * 2 + i owns the d contiguous
// elements of (b, n, h, i) for every n.  e4m3 codes take one byte each (rows
// of d bytes); e2m1 codes two per byte, channel 2j in the low nibble (rows of
// d / 2 bytes).  Each CTA takes one group and up to kTokPerCta tokens; every
// row is d / 8 loads of 16 bytes.  HBM-bound: reads x twice (the second time
// mostly from L2) and writes one byte (e4m3) or half a byte (e2m1) per
// element.
#include <cuda_bf16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "internal.h"

namespace diffattn {

namespace {

constexpr int kTokPerCta = 256;
constexpr int kThreadsQ = 256;
constexpr int kUnroll = 4;  // independent 16-byte loads in flight per thread
constexpr float kE4m3Max = 448.0f;
constexpr float kE2m1Max = 6.0f;

__device__ __forceinline__ void bf16x8_to_float(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

__device__ __forceinline__ const uint4* row_ptr(const __nv_bfloat16* x, int b, int n, int hi, int N, int H, int d) {
  return reinterpret_cast<const uint4*>(x + ((static_cast<size_t>(b) * N + n) * (2 * H) + hi) * d);
}

__global__ void __launch_bounds__(kThreadsQ) qk_absmax_kernel(const __nv_bfloat16* __restrict__ x, int N, int H,
                                                              int d, unsigned int* __restrict__ amax_bits) {
  const int g = blockIdx.y;
  const int b = g / (2 * H), hi = g % (2 * H);
  const int n0 = blockIdx.x * kTokPerCta;
  const int rows = min(N - n0, kTokPerCta);
  const int vec = d / 8;
  const int total = rows * vec;
  float m = 0.f;
  for (int base = threadIdx.x; base < total; base += kUnroll * kThreadsQ) {
    uint4 u[kUnroll];
#pragma unroll
    for (int k = 0; k < kUnroll; ++k) {
      const int idx = base + k * kThreadsQ;
      u[k] = idx < total ? __ldg(row_ptr(x, b, n0 + idx / vec, hi, N, H, d) + idx % vec) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int k = 0; k < kUnroll; ++k) {
      float f[8];
      bf16x8_to_float(u[k], f);
#pragma unroll
      for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(f[i]));
    }
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ float wmax[kThreadsQ / 32];
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = wmax[0];
    for (int w = 1; w < kThreadsQ / 32; ++w) t = fmaxf(t, wmax[w]);
    atomicMax(amax_bits + g, __float_as_uint(t));
  }
}

__global__ void qk_scale_kernel(float* __restrict__ scales, int G, float fmax) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < G) {
    const float a = scales[i];  // the absmax, written as its bit pattern by pass 1
    scales[i] = a > 0.f ? a / fmax : 1.0f;
  }
}

// 8 consecutive elements (already divided by the scale) -> 8 e4m3 codes
__device__ __forceinline__ uint2 encode8_e4m3(const float (&r)[8]) {
  uint32_t w[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const __nv_fp8x2_storage_t lo =
        __nv_cvt_float2_to_fp8x2(make_float2(r[4 * i], r[4 * i + 1]), __NV_SATFINITE, __NV_E4M3);
    const __nv_fp8x2_storage_t up =
        __nv_cvt_float2_to_fp8x2(make_float2(r[4 * i + 2], r[4 * i + 3]), __NV_SATFINITE, __NV_E4M3);
    w[i] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(up) << 16);
  }
  return make_uint2(w[0], w[1]);
}

// 8 consecutive elements -> 8 e2m1 codes in 4 bytes, element j in nibble j
// (the conversion saturates at +-6 and rounds to nearest even)
__device__ __forceinline__ uint32_t encode8_e2m1(const float (&r)[8]) {
  uint32_t w = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j)
    w |= (static_cast<uint32_t>(__nv_cvt_float_to_fp4(r[j], __NV_E2M1, cudaRoundNearest)) & 0xFu) << (4 * j);
  return w;
}

template <int BITS>
__global__ void __launch_bounds__(kThreadsQ) qk_quant_kernel(const __nv_bfloat16* __restrict__ x, int N, int H,
                                                             int d, const float* __restrict__ scales,
                                                             uint8_t* __restrict__ codes) {
  const int g = blockIdx.y;
  const int b = g / (2 * H), hi = g % (2 * H);
  const int n0 = blockIdx.x * kTokPerCta;
  const int rows = min(N - n0, kTokPerCta);
  const int vec = d / 8;
  const float s = __ldg(scales + g);
  const int total = rows * vec;
  for (int base = threadIdx.x; base < total; base += kUnroll * kThreadsQ) {
    uint4 u[kUnroll];
#pragma unroll
    for (int k = 0; k < kUnroll; ++k) {
      const int idx = base + k * kThreadsQ;
      u[k] = idx < total ? __ldg(row_ptr(x, b, n0 + idx / vec, hi, N, H, d) + idx % vec) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int k = 0; k < kUnroll; ++k) {
      const int idx = base + k * kThreadsQ;
      if (idx >= total) break;
      const int n = n0 + idx / vec, c = idx % vec;
      float f[8];
      bf16x8_to_float(u[k], f);
#pragma unroll
      for (int i = 0; i < 8; ++i) f[i] = f[i] / s;
      const size_t row = (static_cast<size_t>(b) * N + n) * (2 * H) + hi;
      if constexpr (BITS == 8)
        *reinterpret_cast<uint2*>(codes + row * d + 8 * c) = encode8_e4m3(f);
      else
        *reinterpret_cast<uint32_t*>(codes + row * (d / 2) + 4 * c) = encode8_e2m1(f);
    }
  }
}

}  // namespace

cudaError_t launch_quantize_qk(const void* x, int B, int N, int H, int d, int bits, void* codes, float* scales,
                               cudaStream_t stream) {
  if (bits != 8 && bits != 4) return cudaErrorInvalidValue;
  const int G = B * H * 2;
  cudaError_t e = cudaMemsetAsync(scales, 0, sizeof(float) * G, stream);
  if (e != cudaSuccess) return e;
  const dim3 grid((N + kTokPerCta - 1) / kTokPerCta, G);
  const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
  qk_absmax_kernel<<<grid, kThreadsQ, 0, stream>>>(xb, N, H, d, reinterpret_cast<unsigned int*>(scales));
  qk_scale_kernel<<<(G + 255) / 256, 256, 0, stream>>>(scales, G, bits == 8 ? kE4m3Max : kE2m1Max);
  if (bits == 8)
    qk_quant_kernel<8><<<grid, kThreadsQ, 0, stream>>>(xb, N, H, d, scales, static_cast<uint8_t*>(codes));
  else
    qk_quant_kernel<4><<<grid, kThreadsQ, 0, stream>>>(xb, N, H, d, scales, static_cast<uint8_t*>(codes));
  return cudaGetLastError();
}

}  // namespace diffattn
