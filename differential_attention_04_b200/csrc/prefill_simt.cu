// CUDA-core (FFMA) prefill for float32 tensors with any per-map width
// 1 <= d <= 128.  Tensor cores are not used here: their tf32 path cannot meet
// a 1e-5 tolerance, and this path exists for exact fp32 work.
//
// Per head it computes the DiffAttn equation (page "Differential Transformer:
// Canceling Context Noise with Differential Attention", "Cancelling Context
// Noise Through Attention Map Subtraction"; peer review "Differential
// Transformer", Summary, Eq. 1), keeping one online-softmax state (running
// max, running sum) per map and query row, then the headwise RMSNorm over the
// 2d channels and the (1 - lambda_init) scale (peer review, Summary, Eq. 3).
//
// CTA = 8 warps over 32 query rows of one (batch, head); each warp owns 4
// rows.  Keys stream through shared memory 32 at a time; lane j scores key j,
// then every lane accumulates the output channels c = lane + 32u.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace diffattn {

namespace {
constexpr int kRowsPerCta = 32;
constexpr int kRowsPerWarp = 4;
constexpr int kKeysPerTile = 32;
constexpr int kMaxU = 8;  // ceil(2 * 128 / 32)
}  // namespace

__global__ void __launch_bounds__(256) prefill_simt_f32_kernel(
    const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v, float* __restrict__ o,
    int N, int H, int d, int causal, const float* __restrict__ lambda_ptr, float lambda_init,
    const float* __restrict__ rms_w, float eps, int mode, int* dbg) {
  extern __shared__ float smem[];
  const int kstride = (d % 2 == 0) ? d + 1 : d;  // odd row pitch: conflict-free column reads
  const int dv = 2 * d;
  float* q1s = smem;                          // [32][d]
  float* q2s = q1s + kRowsPerCta * d;         // [32][d]
  float* k1s = q2s + kRowsPerCta * d;         // [32][kstride]
  float* k2s = k1s + kKeysPerTile * kstride;  // [32][kstride]
  float* vs = k2s + kKeysPerTile * kstride;   // [32][2d]

  const int b = blockIdx.z, h = blockIdx.y;
  const int q0 = blockIdx.x * kRowsPerCta;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t tok_qk = static_cast<size_t>(H) * 2 * d;  // elements per token in q / k
  const size_t tok_v = static_cast<size_t>(H) * dv;      // elements per token in v / o
  const float* qb = q + static_cast<size_t>(b) * N * tok_qk + static_cast<size_t>(h) * 2 * d;
  const float* kb = k + static_cast<size_t>(b) * N * tok_qk + static_cast<size_t>(h) * 2 * d;
  const float* vb = v + static_cast<size_t>(b) * N * tok_v + static_cast<size_t>(h) * dv;
  float* ob = o + static_cast<size_t>(b) * N * tok_v + static_cast<size_t>(h) * dv;

  for (int i = threadIdx.x; i < kRowsPerCta * d; i += blockDim.x) {
    const int r = i / d, c = i % d;
    const int n = q0 + r;
    q1s[i] = n < N ? qb[n * tok_qk + c] : 0.f;
    q2s[i] = n < N ? qb[n * tok_qk + d + c] : 0.f;
  }

  const float scale = 1.0f / sqrtf(static_cast<float>(d));
  float m1[kRowsPerWarp], l1[kRowsPerWarp], m2[kRowsPerWarp], l2[kRowsPerWarp];
  float o1[kRowsPerWarp][kMaxU], o2[kRowsPerWarp][kMaxU];
#pragma unroll
  for (int rr = 0; rr < kRowsPerWarp; ++rr) {
    m1[rr] = m2[rr] = -INFINITY;
    l1[rr] = l2[rr] = 0.f;
#pragma unroll
    for (int u = 0; u < kMaxU; ++u) o1[rr][u] = o2[rr][u] = 0.f;
  }

  const int key_end = causal ? min(N, q0 + kRowsPerCta) : N;
  for (int kt = 0; kt < key_end; kt += kKeysPerTile) {
    __syncthreads();
    for (int i = threadIdx.x; i < kKeysPerTile * d; i += blockDim.x) {
      const int j = i / d, c = i % d;
      const int n = kt + j;
      k1s[j * kstride + c] = n < N ? kb[n * tok_qk + c] : 0.f;
      k2s[j * kstride + c] = n < N ? kb[n * tok_qk + d + c] : 0.f;
    }
    for (int i = threadIdx.x; i < kKeysPerTile * dv; i += blockDim.x) {
      const int j = i / dv, c = i % dv;
      const int n = kt + j;
      vs[i] = n < N ? vb[n * tok_v + c] : 0.f;
    }
    __syncthreads();

#pragma unroll
    for (int rr = 0; rr < kRowsPerWarp; ++rr) {
      const int r = warp * kRowsPerWarp + rr;
      const int qi = q0 + r;
      if (qi >= N) continue;
      const int j = kt + lane;
      const bool valid = j < N && (!causal || j <= qi);
      float s1 = -INFINITY, s2 = -INFINITY;
      if (valid) {
        float a1 = 0.f, a2 = 0.f;
        for (int c = 0; c < d; ++c) {
          a1 = fmaf(q1s[r * d + c], k1s[lane * kstride + c], a1);
          a2 = fmaf(q2s[r * d + c], k2s[lane * kstride + c], a2);
        }
        s1 = a1 * scale;
        s2 = a2 * scale;
      }
      float t1 = s1, t2 = s2;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        t1 = fmaxf(t1, __shfl_xor_sync(0xffffffffu, t1, off));
        t2 = fmaxf(t2, __shfl_xor_sync(0xffffffffu, t2, off));
      }
      if (t1 == -INFINITY) continue;  // no visible key in this tile (both maps share the mask)
      const float mn1 = fmaxf(m1[rr], t1), mn2 = fmaxf(m2[rr], t2);
      const float al1 = expf(m1[rr] - mn1), al2 = expf(m2[rr] - mn2);
      const float p1 = valid ? expf(s1 - mn1) : 0.f;
      const float p2 = valid ? expf(s2 - mn2) : 0.f;
      float sp1 = p1, sp2 = p2;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        sp1 += __shfl_xor_sync(0xffffffffu, sp1, off);
        sp2 += __shfl_xor_sync(0xffffffffu, sp2, off);
      }
      l1[rr] = l1[rr] * al1 + sp1;
      l2[rr] = l2[rr] * al2 + sp2;
      m1[rr] = mn1;
      m2[rr] = mn2;
#pragma unroll
      for (int u = 0; u < kMaxU; ++u) {
        o1[rr][u] *= al1;
        o2[rr][u] *= al2;
      }
      const int jn = min(kKeysPerTile, N - kt);
      for (int jj = 0; jj < jn; ++jj) {
        const float pj1 = __shfl_sync(0xffffffffu, p1, jj);
        const float pj2 = __shfl_sync(0xffffffffu, p2, jj);
#pragma unroll
        for (int u = 0; u < kMaxU; ++u) {
          const int c = lane + 32 * u;
          if (c < dv) {
            const float vv = vs[jj * dv + c];
            o1[rr][u] = fmaf(pj1, vv, o1[rr][u]);
            o2[rr][u] = fmaf(pj2, vv, o2[rr][u]);
          }
        }
      }
    }
  }

  const float coef2 = map2_coefficient(mode, *lambda_ptr);  // c in softmax(S1) + c softmax(S2)
  const float out_scale = 1.0f - lambda_init;
#pragma unroll
  for (int rr = 0; rr < kRowsPerWarp; ++rr) {
    const int qi = q0 + warp * kRowsPerWarp + rr;
    if (qi >= N) continue;
    const float inv1 = 1.0f / l1[rr], inv2 = coef2 / l2[rr];
    float ov[kMaxU];
    float ss = 0.f;
#pragma unroll
    for (int u = 0; u < kMaxU; ++u) {
      const int c = lane + 32 * u;
      ov[u] = (c < dv) ? o1[rr][u] * inv1 + o2[rr][u] * inv2 : 0.f;
      ss = fmaf(ov[u], ov[u], ss);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    const float rs = 1.0f / sqrtf(ss / static_cast<float>(dv) + eps);
#pragma unroll
    for (int u = 0; u < kMaxU; ++u) {
      const int c = lane + 32 * u;
      // debug builds: the element lies in o [B, N, H, 2d]
      if (c < dv && DA_CHECK(dbg, (ob - o) + static_cast<size_t>(qi) * tok_v + c <
                                      static_cast<size_t>(gridDim.z) * N * tok_v))
        ob[static_cast<size_t>(qi) * tok_v + c] = out_scale * rms_w[c] * ov[u] * rs;
    }
  }
}

cudaError_t launch_prefill_simt_f32(const float* q, const float* k, const float* v, float* o, int B, int N, int H,
                                    int d, int causal, const float* lambda, float lambda_init, const float* rms_w,
                                    float eps, int mode, cudaStream_t stream) {
  const int kstride = (d % 2 == 0) ? d + 1 : d;
  const size_t smem =
      sizeof(float) * (2 * kRowsPerCta * d + 2 * kKeysPerTile * kstride + kKeysPerTile * 2 * d);
  cudaError_t e = cudaFuncSetAttribute(prefill_simt_f32_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid((N + kRowsPerCta - 1) / kRowsPerCta, H, B);
  prefill_simt_f32_kernel<<<grid, 256, smem, stream>>>(q, k, v, o, N, H, d, causal, lambda, lambda_init, rms_w,
                                                       eps, mode, debug_status());
  return cudaGetLastError();
}

}  // namespace diffattn
