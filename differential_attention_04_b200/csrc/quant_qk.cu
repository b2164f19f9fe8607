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
// d / 2 bytes).  HBM-bound: reads x twice (the second time mostly from L2)
// and writes one byte (e4m3) or half a byte (e2m1) per element.
//
// Each CTA takes one group and up to kTokPerCta tokens; the grid runs the
// token chunks of a group next to each other, so the CTAs resident at once
// read whole token rows of neighbouring groups.  A row is d / 8 vectors of 16
// bytes.  Every thread keeps one vector column and walks the rows with a
// fixed stride (kThreadsQ / (d / 8) rows per pass), so the loop carries no
// integer division; the e2m1 pass converts its values in pairs.
#include <cuda_bf16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "common.cuh"
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

// Thread layout over a chunk of `rows` rows of `vec` vectors: this thread's
// first row and column, the row stride, and whether it takes part (all of
// kThreadsQ do when vec divides it; for vec > kThreadsQ each thread walks
// several columns of every row).
struct Walk {
  int r0, c0, r_step, c_step;
  bool active;
};
__device__ __forceinline__ Walk walk_of(int vec) {
  if (vec <= kThreadsQ) {
    const int rpp = kThreadsQ / vec;
    return {static_cast<int>(threadIdx.x) / vec, static_cast<int>(threadIdx.x) % vec, rpp, vec,
            static_cast<int>(threadIdx.x) < rpp * vec};
  }
  return {0, static_cast<int>(threadIdx.x), 1, kThreadsQ, true};
}

__global__ void __launch_bounds__(kThreadsQ) qk_absmax_kernel(const __nv_bfloat16* __restrict__ x, int N, int H,
                                                              int d, unsigned int* __restrict__ amax_bits,
                                                              int* dbg) {
  // debug builds: the elements read below lie in x [B, N, H, 2, d] (rows n0 .. n0 + rows - 1 of group g)
  const int g = blockIdx.y;
  const int b = g / (2 * H), hi = g % (2 * H);
  const int n0 = blockIdx.x * kTokPerCta;
  const int rows = min(N - n0, kTokPerCta);
  const int vec = d / 8;
  const Walk w = walk_of(vec);
  const size_t row_vecs = static_cast<size_t>(2 * H) * vec;  // vectors from one token row to the next
  float m = 0.f;
  if (w.active && DA_CHECK(dbg, n0 >= 0 && rows >= 1 && n0 + rows <= N && b < static_cast<int>(gridDim.y) / (2 * H) &&
                                    d % 8 == 0)) {
    for (int c = w.c0; c < vec; c += w.c_step) {
      const uint4* p = row_ptr(x, b, n0, hi, N, H, d) + c;
      for (int r = w.r0; r < rows; r += kUnroll * w.r_step) {
        uint4 v[kUnroll];
#pragma unroll
        for (int k = 0; k < kUnroll; ++k) {
          const int rr = r + k * w.r_step;
          v[k] = rr < rows ? __ldg(p + rr * row_vecs) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int k = 0; k < kUnroll; ++k) {
          float f[8];
          bf16x8_to_float(v[k], f);
#pragma unroll
          for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(f[i]));
        }
      }
    }
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ float wmax[kThreadsQ / 32];
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = wmax[0];
    for (int i = 1; i < kThreadsQ / 32; ++i) t = fmaxf(t, wmax[i]);
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
// (the conversion saturates at +-6 and rounds to nearest even; a pair's
// first element lands in the low nibble of its byte)
__device__ __forceinline__ uint32_t encode8_e2m1(const float (&r)[8]) {
  uint32_t w = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j)
    w |= static_cast<uint32_t>(__nv_cvt_float2_to_fp4x2(make_float2(r[2 * j], r[2 * j + 1]), __NV_E2M1,
                                                        cudaRoundNearest))
         << (8 * j);
  return w;
}

template <int BITS>
__global__ void __launch_bounds__(kThreadsQ) qk_quant_kernel(const __nv_bfloat16* __restrict__ x, int N, int H,
                                                             int d, const float* __restrict__ scales,
                                                             uint8_t* __restrict__ codes, int* dbg) {
  const int g = blockIdx.y;
  const int b = g / (2 * H), hi = g % (2 * H);
  const int n0 = blockIdx.x * kTokPerCta;
  const int rows = min(N - n0, kTokPerCta);
  const int vec = d / 8;
  const Walk w = walk_of(vec);
  if (!w.active) return;
  // debug builds: rows n0 .. n0 + rows - 1 of group g lie in x and in the codes
  if (!DA_CHECK(dbg, n0 >= 0 && rows >= 1 && n0 + rows <= N && b < static_cast<int>(gridDim.y) / (2 * H) &&
                         d % 8 == 0))
    return;
  const float s = __ldg(scales + g);
  const size_t row_vecs = static_cast<size_t>(2 * H) * vec;
  constexpr int kOutBytes = BITS == 8 ? 8 : 4;  // code bytes per vector
  for (int c = w.c0; c < vec; c += w.c_step) {
    const uint4* p = row_ptr(x, b, n0, hi, N, H, d) + c;
    uint8_t* q = codes + ((static_cast<size_t>(b) * N + n0) * (2 * H) + hi) * (vec * kOutBytes) + c * kOutBytes;
    for (int r = w.r0; r < rows; r += kUnroll * w.r_step) {
      uint4 v[kUnroll];
#pragma unroll
      for (int k = 0; k < kUnroll; ++k) {
        const int rr = r + k * w.r_step;
        v[k] = rr < rows ? __ldg(p + rr * row_vecs) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int k = 0; k < kUnroll; ++k) {
        const int rr = r + k * w.r_step;
        if (rr >= rows) break;
        float f[8];
        bf16x8_to_float(v[k], f);
#pragma unroll
        for (int i = 0; i < 8; ++i) f[i] = f[i] / s;
        uint8_t* dst = q + rr * row_vecs * kOutBytes;
        if constexpr (BITS == 8)
          *reinterpret_cast<uint2*>(dst) = encode8_e4m3(f);
        else
          *reinterpret_cast<uint32_t*>(dst) = encode8_e2m1(f);
      }
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
  int* dbg = debug_status();
  qk_absmax_kernel<<<grid, kThreadsQ, 0, stream>>>(xb, N, H, d, reinterpret_cast<unsigned int*>(scales), dbg);
  qk_scale_kernel<<<(G + 255) / 256, 256, 0, stream>>>(scales, G, bits == 8 ? kE4m3Max : kE2m1Max);
  if (bits == 8)
    qk_quant_kernel<8><<<grid, kThreadsQ, 0, stream>>>(xb, N, H, d, scales, static_cast<uint8_t*>(codes), dbg);
  else
    qk_quant_kernel<4><<<grid, kThreadsQ, 0, stream>>>(xb, N, H, d, scales, static_cast<uint8_t*>(codes), dbg);
  return cudaGetLastError();
}

}  // namespace diffattn
