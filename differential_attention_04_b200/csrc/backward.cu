// Backward pass of the prefill, on CUDA cores (fp32 arithmetic; bf16 or fp32
// inputs).  It differentiates the DiffAttn equation (page "Differential
// Transformer: Canceling Context Noise with Differential Attention",
// "Cancelling Context Noise Through Attention Map Subtraction"; peer review
// "Differential Transformer", Summary, Eq. 1), the headwise RMSNorm and the
// (1 - lambda_init) scale (Eq. 3), for any combination mode
// O = A_1 V + c A_2 V (c = -lambda, 0, +lambda):
//
//   G = dO  = g r (w dy) - O g r^3 / (2d) * sum_c (w dy O),  r = 1/sqrt(mean O^2 + eps)
//   dw      = sum over rows of g r O dy
//   dV      = A_1^T G + c A_2^T G
//   dS_i    = A_i * (c_i G V^T - D_i),  c_1 = 1, c_2 = c,  D_i = c_i rowsum(G * (A_i V))
//   dQ_i    = dS_i K_i / sqrt(d),  dK_i = dS_i^T Q_i / sqrt(d)
//   dlambda = (dc/dlambda) <G, A_2 V>
//
// Three kernels, each CTA = 8 warps over 32 rows of one (batch, head), tiles
// of 32 streamed through shared memory.  Lane j takes element j of the
// streamed tile against the warp's own 4 rows (or keys), which sit transposed
// in shared memory so that one broadcast float4 load feeds 4 FMAs; the
// gradient sums likewise update 4 rows per loaded operand:
//   rows:    recompute both maps' online softmax per query row, keeping A_1 V
//            and A_2 V apart; write G, the two log-sum-exps and D_1, D_2 to
//            the workspace; reduce dw and dlambda per CTA, then add them.
//   keys:    per 32-key tile, stream the query tiles: recompute P_i, form
//            dS_i, accumulate dK_1, dK_2 and dV in registers; plain stores.
//   queries: per 32-query tile, stream the key tiles: accumulate dQ_1, dQ_2.
// The lambda re-parameterisation (Eq. 2) has its own one-warp kernel.
#include <cuda_bf16.h>
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace diffattn {

namespace {

constexpr int kRows = 32;      // query rows (or keys) per CTA
constexpr int kTile = 32;      // keys (or queries) per streamed tile
constexpr int kPerWarp = 4;    // rows (or keys) per warp
constexpr int kMaxU = 8;       // channels per lane for 2d <= 256
constexpr int kMaxD = 4;       // channels per lane for d <= 128

__device__ __forceinline__ float ldf(const float* p) { return *p; }
__device__ __forceinline__ float ldf(const __nv_bfloat16* p) { return __bfloat162float(*p); }

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}
__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}

struct BwdArgs {
  int B, N, H, d, causal;
  int* dbg;           // debug builds: where the bounds checks record DIFFATTN_ERR_BOUNDS
  float dcoef;        // dc/dlambda of map 2's coefficient c (c itself is formed on the device from lambda)
  float lambda_init, eps;
  const float* rms_w;
  float* G;           // workspace [B, N, H, 2d]
  float4* stats;      // workspace [B, N, H]: lse_1, lse_2, D_1, D_2
  float* dq;          // [B, N, H, 2, d]
  float* dk;
  float* dv;          // [B, N, H, 2d]
  float* dlambda;
  float* drms_w;      // [2d]
};

// ------------------------------------------------------------------ rows --
template <typename T>
__global__ void __launch_bounds__(256) bwd_rows_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                       const T* __restrict__ v, const T* __restrict__ dy,
                                                       const float* __restrict__ lambda_ptr, int mode, BwdArgs a) {
  extern __shared__ float sm[];
  const int d = a.d, dv = 2 * d, N = a.N, H = a.H;
  const int kstride = (d % 2 == 0) ? d + 1 : d;
  float* q1T = sm;                        // [d][32] this CTA's queries, transposed
  float* q2T = q1T + d * kRows;
  float* k1s = q2T + d * kRows;           // [32][kstride] the streamed keys
  float* k2s = k1s + kTile * kstride;
  float* vs = k2s + kTile * kstride;      // [32][2d]
  const float4* q1T4 = reinterpret_cast<const float4*>(q1T);
  const float4* q2T4 = reinterpret_cast<const float4*>(q2T);
  const int b = blockIdx.z, h = blockIdx.y, q0 = blockIdx.x * kRows;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t tok_qk = static_cast<size_t>(H) * 2 * d, tok_v = static_cast<size_t>(H) * dv;
  const T* qb = q + static_cast<size_t>(b) * N * tok_qk + static_cast<size_t>(h) * 2 * d;
  const T* kb = k + static_cast<size_t>(b) * N * tok_qk + static_cast<size_t>(h) * 2 * d;
  const T* vb = v + static_cast<size_t>(b) * N * tok_v + static_cast<size_t>(h) * dv;
  const T* dyb = dy + static_cast<size_t>(b) * N * tok_v + static_cast<size_t>(h) * dv;
  const float coef = map2_coefficient(mode, *lambda_ptr);

  for (int i = threadIdx.x; i < kRows * d; i += blockDim.x) {
    const int r = i % kRows, c = i / kRows, n = q0 + r;
    q1T[i] = n < N ? ldf(qb + n * tok_qk + c) : 0.f;
    q2T[i] = n < N ? ldf(qb + n * tok_qk + d + c) : 0.f;
  }
  const float scale = 1.0f / sqrtf(static_cast<float>(d));
  float m1[kPerWarp], l1[kPerWarp], m2[kPerWarp], l2[kPerWarp];
  float o1[kPerWarp][kMaxU], o2[kPerWarp][kMaxU];
#pragma unroll
  for (int rr = 0; rr < kPerWarp; ++rr) {
    m1[rr] = m2[rr] = -INFINITY;
    l1[rr] = l2[rr] = 0.f;
#pragma unroll
    for (int u = 0; u < kMaxU; ++u) o1[rr][u] = o2[rr][u] = 0.f;
  }
  const int key_end = a.causal ? min(N, q0 + kRows) : N;
  for (int kt = 0; kt < key_end; kt += kTile) {
    __syncthreads();
    for (int i = threadIdx.x; i < kTile * d; i += blockDim.x) {
      const int j = i / d, c = i % d, n = kt + j;
      k1s[j * kstride + c] = n < N ? ldf(kb + n * tok_qk + c) : 0.f;
      k2s[j * kstride + c] = n < N ? ldf(kb + n * tok_qk + d + c) : 0.f;
    }
    for (int i = threadIdx.x; i < kTile * dv; i += blockDim.x) {
      const int j = i / dv, c = i % dv, n = kt + j;
      vs[i] = n < N ? ldf(vb + n * tok_v + c) : 0.f;
    }
    __syncthreads();
    // scores of key kt + lane against the warp's 4 rows, both maps
    float s1[kPerWarp], s2[kPerWarp];
#pragma unroll
    for (int rr = 0; rr < kPerWarp; ++rr) s1[rr] = s2[rr] = 0.f;
    for (int c = 0; c < d; ++c) {
      const float ka = k1s[lane * kstride + c], kb2 = k2s[lane * kstride + c];
      const float4 qa = q1T4[c * (kRows / 4) + warp], qb4 = q2T4[c * (kRows / 4) + warp];
      s1[0] = fmaf(qa.x, ka, s1[0]); s1[1] = fmaf(qa.y, ka, s1[1]);
      s1[2] = fmaf(qa.z, ka, s1[2]); s1[3] = fmaf(qa.w, ka, s1[3]);
      s2[0] = fmaf(qb4.x, kb2, s2[0]); s2[1] = fmaf(qb4.y, kb2, s2[1]);
      s2[2] = fmaf(qb4.z, kb2, s2[2]); s2[3] = fmaf(qb4.w, kb2, s2[3]);
    }
    const int j = kt + lane;
    float p1[kPerWarp], p2[kPerWarp];
#pragma unroll
    for (int rr = 0; rr < kPerWarp; ++rr) {
      const int qi = q0 + warp * kPerWarp + rr;
      const bool valid = qi < N && j < N && (!a.causal || j <= qi);
      const float v1 = valid ? s1[rr] * scale : -INFINITY, v2 = valid ? s2[rr] * scale : -INFINITY;
      const float t1 = warp_max(v1), t2 = warp_max(v2);
      p1[rr] = p2[rr] = 0.f;
      if (t1 == -INFINITY) continue;  // this row sees no key of the tile (both maps share the mask)
      const float mn1 = fmaxf(m1[rr], t1), mn2 = fmaxf(m2[rr], t2);
      const float al1 = expf(m1[rr] - mn1), al2 = expf(m2[rr] - mn2);
      p1[rr] = valid ? expf(v1 - mn1) : 0.f;
      p2[rr] = valid ? expf(v2 - mn2) : 0.f;
      l1[rr] = l1[rr] * al1 + warp_sum(p1[rr]);
      l2[rr] = l2[rr] * al2 + warp_sum(p2[rr]);
      m1[rr] = mn1;
      m2[rr] = mn2;
#pragma unroll
      for (int u = 0; u < kMaxU; ++u) {
        o1[rr][u] *= al1;
        o2[rr][u] *= al2;
      }
    }
    const int jn = min(kTile, N - kt);
    for (int jj = 0; jj < jn; ++jj) {
      float pj1[kPerWarp], pj2[kPerWarp];
#pragma unroll
      for (int rr = 0; rr < kPerWarp; ++rr) {
        pj1[rr] = __shfl_sync(0xffffffffu, p1[rr], jj);
        pj2[rr] = __shfl_sync(0xffffffffu, p2[rr], jj);
      }
#pragma unroll
      for (int u = 0; u < kMaxU; ++u) {
        const int c = lane + 32 * u;
        if (c < dv) {
          const float vv = vs[jj * dv + c];
#pragma unroll
          for (int rr = 0; rr < kPerWarp; ++rr) {
            o1[rr][u] = fmaf(pj1[rr], vv, o1[rr][u]);
            o2[rr][u] = fmaf(pj2[rr], vv, o2[rr][u]);
          }
        }
      }
    }
  }

  // per row: G, log-sum-exps, D_1, D_2; partial dw and dlambda
  const float g = 1.0f - a.lambda_init;
  float dw_acc[kMaxU];
#pragma unroll
  for (int u = 0; u < kMaxU; ++u) dw_acc[u] = 0.f;
  float dlam_acc = 0.f;
#pragma unroll
  for (int rr = 0; rr < kPerWarp; ++rr) {
    const int qi = q0 + warp * kPerWarp + rr;
    if (qi >= N) continue;
    const float i1 = 1.0f / l1[rr], i2 = 1.0f / l2[rr];
    float on1[kMaxU], on2[kMaxU], O[kMaxU], dyv[kMaxU], wv[kMaxU];
    float ss = 0.f, t = 0.f;
    const size_t row = (static_cast<size_t>(b) * N + qi) * H + h;
#pragma unroll
    for (int u = 0; u < kMaxU; ++u) {
      const int c = lane + 32 * u;
      const bool in = c < dv;
      on1[u] = in ? o1[rr][u] * i1 : 0.f;
      on2[u] = in ? o2[rr][u] * i2 : 0.f;
      O[u] = on1[u] + coef * on2[u];
      dyv[u] = in ? ldf(dyb + static_cast<size_t>(qi) * tok_v + c) : 0.f;
      wv[u] = in ? a.rms_w[c] : 0.f;
      ss = fmaf(O[u], O[u], ss);
      t = fmaf(wv[u] * dyv[u], O[u], t);
    }
    ss = warp_sum(ss);
    t = warp_sum(t);
    const float r = 1.0f / sqrtf(ss / static_cast<float>(dv) + a.eps);
    const float corr = g * r * r * r / static_cast<float>(dv) * t;
    float d1 = 0.f, d2 = 0.f;
#pragma unroll
    for (int u = 0; u < kMaxU; ++u) {
      const int c = lane + 32 * u;
      const float Gc = g * r * wv[u] * dyv[u] - O[u] * corr;
      if (c < dv && DA_CHECK(a.dbg, row < static_cast<size_t>(a.B) * a.N * a.H)) a.G[row * dv + c] = Gc;
      d1 = fmaf(Gc, on1[u], d1);
      d2 = fmaf(Gc, on2[u], d2);
      dw_acc[u] = fmaf(g * r * O[u], dyv[u], dw_acc[u]);
    }
    d1 = warp_sum(d1);
    d2 = warp_sum(d2);
    dlam_acc += a.dcoef * d2;
    if (lane == 0)
      a.stats[row] = make_float4(m1[rr] + logf(l1[rr]), m2[rr] + logf(l2[rr]), d1, coef * d2);
  }
  // CTA reduction of dw and dlambda, then one atomic per channel and one for dlambda
  __syncthreads();  // the tiles are no longer read
  float* red = sm;  // [8 warps][dv]
#pragma unroll
  for (int u = 0; u < kMaxU; ++u) {
    const int c = lane + 32 * u;
    if (c < dv) red[warp * dv + c] = dw_acc[u];
  }
  float* lred = sm + 8 * dv;  // [8]
  if (lane == 0) lred[warp] = dlam_acc;
  __syncthreads();
  for (int c = threadIdx.x; c < dv; c += blockDim.x) {
    float s = 0.f;
    for (int w = 0; w < 8; ++w) s += red[w * dv + c];
    atomicAdd(a.drms_w + c, s);
  }
  if (threadIdx.x == 0) {
    float s = 0.f;
    for (int w = 0; w < 8; ++w) s += lred[w];
    atomicAdd(a.dlambda, s);
  }
}

// ------------------------------------------------------------------ keys --
template <typename T>
__global__ void __launch_bounds__(256) bwd_keys_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                       const T* __restrict__ v, const float* __restrict__ lambda_ptr,
                                                       int mode, BwdArgs a) {
  extern __shared__ float sm[];
  const int d = a.d, dv = 2 * d, N = a.N, H = a.H;
  const int qstride = (d % 2 == 0) ? d + 1 : d;
  const int gstride = dv + 1;
  float* k1T = sm;                        // [d][32]  this CTA's keys, transposed
  float* k2T = k1T + d * kRows;
  float* vT = k2T + d * kRows;            // [2d][32]
  float* q1s = vT + dv * kRows;           // [32][qstride] the streamed queries
  float* q2s = q1s + kTile * qstride;
  float* gs = q2s + kTile * qstride;      // [32][gstride]
  float4* st = reinterpret_cast<float4*>(gs + kTile * gstride);  // [32]
  const float4* k1T4 = reinterpret_cast<const float4*>(k1T);
  const float4* k2T4 = reinterpret_cast<const float4*>(k2T);
  const float4* vT4 = reinterpret_cast<const float4*>(vT);
  const int b = blockIdx.z, h = blockIdx.y, k0 = blockIdx.x * kRows;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t tok_qk = static_cast<size_t>(H) * 2 * d, tok_v = static_cast<size_t>(H) * dv;
  const T* qb = q + static_cast<size_t>(b) * N * tok_qk + static_cast<size_t>(h) * 2 * d;
  const T* kb = k + static_cast<size_t>(b) * N * tok_qk + static_cast<size_t>(h) * 2 * d;
  const T* vb = v + static_cast<size_t>(b) * N * tok_v + static_cast<size_t>(h) * dv;
  const float coef = map2_coefficient(mode, *lambda_ptr);
  const float scale = 1.0f / sqrtf(static_cast<float>(d));

  for (int i = threadIdx.x; i < kRows * d; i += blockDim.x) {
    const int r = i % kRows, c = i / kRows, n = k0 + r;
    k1T[i] = n < N ? ldf(kb + n * tok_qk + c) : 0.f;
    k2T[i] = n < N ? ldf(kb + n * tok_qk + d + c) : 0.f;
  }
  for (int i = threadIdx.x; i < kRows * dv; i += blockDim.x) {
    const int r = i % kRows, c = i / kRows, n = k0 + r;
    vT[i] = n < N ? ldf(vb + n * tok_v + c) : 0.f;
  }
  float dk1[kPerWarp][kMaxD], dk2[kPerWarp][kMaxD], dvacc[kPerWarp][kMaxU];
#pragma unroll
  for (int kk = 0; kk < kPerWarp; ++kk) {
#pragma unroll
    for (int u = 0; u < kMaxD; ++u) dk1[kk][u] = dk2[kk][u] = 0.f;
#pragma unroll
    for (int u = 0; u < kMaxU; ++u) dvacc[kk][u] = 0.f;
  }
  const int kw = k0 + warp * kPerWarp;   // the warp's first key
  // causal: queries before this key tile see none of its keys (k0 is a multiple of the tile)
  for (int qt = a.causal ? k0 : 0; qt < N; qt += kTile) {
    __syncthreads();
    for (int i = threadIdx.x; i < kTile * d; i += blockDim.x) {
      const int j = i / d, c = i % d, n = qt + j;
      q1s[j * qstride + c] = n < N ? ldf(qb + n * tok_qk + c) : 0.f;
      q2s[j * qstride + c] = n < N ? ldf(qb + n * tok_qk + d + c) : 0.f;
    }
    for (int i = threadIdx.x; i < kTile * dv; i += blockDim.x) {
      const int j = i / dv, c = i % dv, n = qt + j;
      gs[j * gstride + c] = n < N ? a.G[((static_cast<size_t>(b) * N + n) * H + h) * dv + c] : 0.f;
    }
    for (int j = threadIdx.x; j < kTile; j += blockDim.x) {
      const int n = qt + j;
      st[j] = n < N ? a.stats[(static_cast<size_t>(b) * N + n) * H + h] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    __syncthreads();
    // query qt + lane against the warp's 4 keys: scores of both maps and G . V
    float s1[kPerWarp], s2[kPerWarp], vg[kPerWarp];
#pragma unroll
    for (int kk = 0; kk < kPerWarp; ++kk) s1[kk] = s2[kk] = vg[kk] = 0.f;
    for (int c = 0; c < d; ++c) {
      const float qa = q1s[lane * qstride + c], qb2 = q2s[lane * qstride + c];
      const float4 ka = k1T4[c * (kRows / 4) + warp], kb4 = k2T4[c * (kRows / 4) + warp];
      s1[0] = fmaf(ka.x, qa, s1[0]); s1[1] = fmaf(ka.y, qa, s1[1]);
      s1[2] = fmaf(ka.z, qa, s1[2]); s1[3] = fmaf(ka.w, qa, s1[3]);
      s2[0] = fmaf(kb4.x, qb2, s2[0]); s2[1] = fmaf(kb4.y, qb2, s2[1]);
      s2[2] = fmaf(kb4.z, qb2, s2[2]); s2[3] = fmaf(kb4.w, qb2, s2[3]);
    }
    for (int c = 0; c < dv; ++c) {
      const float gv = gs[lane * gstride + c];
      const float4 v4 = vT4[c * (kRows / 4) + warp];
      vg[0] = fmaf(v4.x, gv, vg[0]); vg[1] = fmaf(v4.y, gv, vg[1]);
      vg[2] = fmaf(v4.z, gv, vg[2]); vg[3] = fmaf(v4.w, gv, vg[3]);
    }
    const int qi = qt + lane;
    const float4 s4 = st[lane];
    float ds1[kPerWarp], ds2[kPerWarp], pv[kPerWarp];
#pragma unroll
    for (int kk = 0; kk < kPerWarp; ++kk) {
      const int kj = kw + kk;
      const bool valid = qi < N && kj < N && (!a.causal || qi >= kj);
      const float p1 = valid ? expf(s1[kk] * scale - s4.x) : 0.f;
      const float p2 = valid ? expf(s2[kk] * scale - s4.y) : 0.f;
      ds1[kk] = p1 * (vg[kk] - s4.z);
      ds2[kk] = p2 * (coef * vg[kk] - s4.w);
      pv[kk] = p1 + coef * p2;  // dV gets (A_1 + c A_2)^T G
    }
    const int jn = min(kTile, N - qt);
    for (int jj = 0; jj < jn; ++jj) {
      float d1[kPerWarp], d2[kPerWarp], pj[kPerWarp];
#pragma unroll
      for (int kk = 0; kk < kPerWarp; ++kk) {
        d1[kk] = __shfl_sync(0xffffffffu, ds1[kk], jj);
        d2[kk] = __shfl_sync(0xffffffffu, ds2[kk], jj);
        pj[kk] = __shfl_sync(0xffffffffu, pv[kk], jj);
      }
#pragma unroll
      for (int u = 0; u < kMaxD; ++u) {
        const int c = lane + 32 * u;
        if (c < d) {
          const float qa = q1s[jj * qstride + c], qb2 = q2s[jj * qstride + c];
#pragma unroll
          for (int kk = 0; kk < kPerWarp; ++kk) {
            dk1[kk][u] = fmaf(d1[kk], qa, dk1[kk][u]);
            dk2[kk][u] = fmaf(d2[kk], qb2, dk2[kk][u]);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < kMaxU; ++u) {
        const int c = lane + 32 * u;
        if (c < dv) {
          const float gv = gs[jj * gstride + c];
#pragma unroll
          for (int kk = 0; kk < kPerWarp; ++kk) dvacc[kk][u] = fmaf(pj[kk], gv, dvacc[kk][u]);
        }
      }
    }
  }
#pragma unroll
  for (int kk = 0; kk < kPerWarp; ++kk) {
    const int kj = kw + kk;
    if (kj >= N) continue;
    const size_t row = (static_cast<size_t>(b) * N + kj) * H + h;
    if (!DA_CHECK(a.dbg, row < static_cast<size_t>(a.B) * N * H)) continue;  // debug builds
#pragma unroll
    for (int u = 0; u < kMaxD; ++u) {
      const int c = lane + 32 * u;
      if (c < d) {
        a.dk[row * 2 * d + c] = dk1[kk][u] * scale;
        a.dk[row * 2 * d + d + c] = dk2[kk][u] * scale;
      }
    }
#pragma unroll
    for (int u = 0; u < kMaxU; ++u) {
      const int c = lane + 32 * u;
      if (c < dv) a.dv[row * dv + c] = dvacc[kk][u];
    }
  }
}

// --------------------------------------------------------------- queries --
template <typename T>
__global__ void __launch_bounds__(256) bwd_queries_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                          const T* __restrict__ v,
                                                          const float* __restrict__ lambda_ptr, int mode,
                                                          BwdArgs a) {
  extern __shared__ float sm[];
  const int d = a.d, dv = 2 * d, N = a.N, H = a.H;
  const int kstride = (d % 2 == 0) ? d + 1 : d;
  const int vstride = dv + 1;
  float* q1T = sm;                       // [d][32]  this CTA's queries, transposed
  float* q2T = q1T + d * kRows;
  float* gT = q2T + d * kRows;           // [2d][32]
  float* k1s = gT + dv * kRows;          // [32][kstride] the streamed keys
  float* k2s = k1s + kTile * kstride;
  float* vs = k2s + kTile * kstride;     // [32][vstride]
  const float4* q1T4 = reinterpret_cast<const float4*>(q1T);
  const float4* q2T4 = reinterpret_cast<const float4*>(q2T);
  const float4* gT4 = reinterpret_cast<const float4*>(gT);
  const int b = blockIdx.z, h = blockIdx.y, q0 = blockIdx.x * kRows;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t tok_qk = static_cast<size_t>(H) * 2 * d, tok_v = static_cast<size_t>(H) * dv;
  const T* qb = q + static_cast<size_t>(b) * N * tok_qk + static_cast<size_t>(h) * 2 * d;
  const T* kb = k + static_cast<size_t>(b) * N * tok_qk + static_cast<size_t>(h) * 2 * d;
  const T* vb = v + static_cast<size_t>(b) * N * tok_v + static_cast<size_t>(h) * dv;
  const float coef = map2_coefficient(mode, *lambda_ptr);
  const float scale = 1.0f / sqrtf(static_cast<float>(d));

  for (int i = threadIdx.x; i < kRows * d; i += blockDim.x) {
    const int r = i % kRows, c = i / kRows, n = q0 + r;
    q1T[i] = n < N ? ldf(qb + n * tok_qk + c) : 0.f;
    q2T[i] = n < N ? ldf(qb + n * tok_qk + d + c) : 0.f;
  }
  for (int i = threadIdx.x; i < kRows * dv; i += blockDim.x) {
    const int r = i % kRows, c = i / kRows, n = q0 + r;
    gT[i] = n < N ? a.G[((static_cast<size_t>(b) * N + n) * H + h) * dv + c] : 0.f;
  }
  const int qw = q0 + warp * kPerWarp;   // the warp's first query row
  float4 srow[kPerWarp];
#pragma unroll
  for (int rr = 0; rr < kPerWarp; ++rr) {
    const int n = qw + rr;
    srow[rr] = n < N ? a.stats[(static_cast<size_t>(b) * N + n) * H + h] : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  float dq1[kPerWarp][kMaxD], dq2[kPerWarp][kMaxD];
#pragma unroll
  for (int rr = 0; rr < kPerWarp; ++rr)
#pragma unroll
    for (int u = 0; u < kMaxD; ++u) dq1[rr][u] = dq2[rr][u] = 0.f;
  const int key_end = a.causal ? min(N, q0 + kRows) : N;
  for (int kt = 0; kt < key_end; kt += kTile) {
    __syncthreads();
    for (int i = threadIdx.x; i < kTile * d; i += blockDim.x) {
      const int j = i / d, c = i % d, n = kt + j;
      k1s[j * kstride + c] = n < N ? ldf(kb + n * tok_qk + c) : 0.f;
      k2s[j * kstride + c] = n < N ? ldf(kb + n * tok_qk + d + c) : 0.f;
    }
    for (int i = threadIdx.x; i < kTile * dv; i += blockDim.x) {
      const int j = i / dv, c = i % dv, n = kt + j;
      vs[j * vstride + c] = n < N ? ldf(vb + n * tok_v + c) : 0.f;
    }
    __syncthreads();
    // key kt + lane against the warp's 4 rows: scores of both maps and G . V
    float s1[kPerWarp], s2[kPerWarp], vg[kPerWarp];
#pragma unroll
    for (int rr = 0; rr < kPerWarp; ++rr) s1[rr] = s2[rr] = vg[rr] = 0.f;
    for (int c = 0; c < d; ++c) {
      const float ka = k1s[lane * kstride + c], kb2 = k2s[lane * kstride + c];
      const float4 qa = q1T4[c * (kRows / 4) + warp], qb4 = q2T4[c * (kRows / 4) + warp];
      s1[0] = fmaf(qa.x, ka, s1[0]); s1[1] = fmaf(qa.y, ka, s1[1]);
      s1[2] = fmaf(qa.z, ka, s1[2]); s1[3] = fmaf(qa.w, ka, s1[3]);
      s2[0] = fmaf(qb4.x, kb2, s2[0]); s2[1] = fmaf(qb4.y, kb2, s2[1]);
      s2[2] = fmaf(qb4.z, kb2, s2[2]); s2[3] = fmaf(qb4.w, kb2, s2[3]);
    }
    for (int c = 0; c < dv; ++c) {
      const float vv = vs[lane * vstride + c];
      const float4 g4 = gT4[c * (kRows / 4) + warp];
      vg[0] = fmaf(g4.x, vv, vg[0]); vg[1] = fmaf(g4.y, vv, vg[1]);
      vg[2] = fmaf(g4.z, vv, vg[2]); vg[3] = fmaf(g4.w, vv, vg[3]);
    }
    const int kj = kt + lane;
    float ds1[kPerWarp], ds2[kPerWarp];
#pragma unroll
    for (int rr = 0; rr < kPerWarp; ++rr) {
      const int qi = qw + rr;
      const bool valid = qi < N && kj < N && (!a.causal || kj <= qi);
      const float p1 = valid ? expf(s1[rr] * scale - srow[rr].x) : 0.f;
      const float p2 = valid ? expf(s2[rr] * scale - srow[rr].y) : 0.f;
      ds1[rr] = p1 * (vg[rr] - srow[rr].z);
      ds2[rr] = p2 * (coef * vg[rr] - srow[rr].w);
    }
    const int jn = min(kTile, N - kt);
    for (int jj = 0; jj < jn; ++jj) {
      float d1[kPerWarp], d2[kPerWarp];
#pragma unroll
      for (int rr = 0; rr < kPerWarp; ++rr) {
        d1[rr] = __shfl_sync(0xffffffffu, ds1[rr], jj);
        d2[rr] = __shfl_sync(0xffffffffu, ds2[rr], jj);
      }
#pragma unroll
      for (int u = 0; u < kMaxD; ++u) {
        const int c = lane + 32 * u;
        if (c < d) {
          const float ka = k1s[jj * kstride + c], kb2 = k2s[jj * kstride + c];
#pragma unroll
          for (int rr = 0; rr < kPerWarp; ++rr) {
            dq1[rr][u] = fmaf(d1[rr], ka, dq1[rr][u]);
            dq2[rr][u] = fmaf(d2[rr], kb2, dq2[rr][u]);
          }
        }
      }
    }
  }
#pragma unroll
  for (int rr = 0; rr < kPerWarp; ++rr) {
    const int qi = qw + rr;
    if (qi >= N) continue;
    const size_t row = (static_cast<size_t>(b) * N + qi) * H + h;
    if (!DA_CHECK(a.dbg, row < static_cast<size_t>(a.B) * N * H)) continue;  // debug builds
#pragma unroll
    for (int u = 0; u < kMaxD; ++u) {
      const int c = lane + 32 * u;
      if (c < d) {
        a.dq[row * 2 * d + c] = dq1[rr][u] * scale;
        a.dq[row * 2 * d + d + c] = dq2[rr][u] * scale;
      }
    }
  }
}

// ------------------------------------------------------------- lambda --
// dlq1 = dlambda e1 lk1, dlk1 = dlambda e1 lq1, dlq2 = -dlambda e2 lk2,
// dlk2 = -dlambda e2 lq2, e1 = exp(lq1 . lk1), e2 = exp(lq2 . lk2).
__global__ void lambda_bwd_kernel(const float* __restrict__ lq1, const float* __restrict__ lk1,
                                  const float* __restrict__ lq2, const float* __restrict__ lk2, int d,
                                  const float* __restrict__ dlambda, float* dlq1, float* dlk1, float* dlq2,
                                  float* dlk2) {
  const int lane = threadIdx.x;
  float s1 = 0.f, s2 = 0.f;
  for (int i = lane; i < d; i += 32) {
    s1 = fmaf(lq1[i], lk1[i], s1);
    s2 = fmaf(lq2[i], lk2[i], s2);
  }
  s1 = warp_sum(s1);
  s2 = warp_sum(s2);
  const float g = *dlambda, e1 = expf(s1), e2 = expf(s2);
  for (int i = lane; i < d; i += 32) {
    const float a1 = lq1[i], b1 = lk1[i], a2 = lq2[i], b2 = lk2[i];
    dlq1[i] = g * e1 * b1;
    dlk1[i] = g * e1 * a1;
    dlq2[i] = -g * e2 * b2;
    dlk2[i] = -g * e2 * a2;
  }
}

template <typename T>
cudaError_t launch_bwd_t(const void* q, const void* k, const void* v, const void* dy, int B, int N, int H, int d,
                         int causal, const float* lambda, float lambda_init, const float* rms_w, float eps, int mode,
                         float* dq, float* dk, float* dv, float* dlambda, float* drms_w, void* workspace,
                         cudaStream_t stream) {
  const int dvw = 2 * d;
  BwdArgs a;
  a.B = B;
  a.dbg = debug_status();
  a.N = N;
  a.H = H;
  a.d = d;
  a.causal = causal ? 1 : 0;
  a.dcoef = mode == 0 ? -1.0f : (mode == 2 ? 1.0f : 0.0f);
  a.lambda_init = lambda_init;
  a.eps = eps;
  a.rms_w = rms_w;
  a.G = static_cast<float*>(workspace);
  const size_t g_bytes = ((sizeof(float) * B * N * H * dvw) + 255) / 256 * 256;
  a.stats = reinterpret_cast<float4*>(static_cast<char*>(workspace) + g_bytes);
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.dlambda = dlambda;
  a.drms_w = drms_w;
  cudaError_t e = cudaMemsetAsync(drms_w, 0, sizeof(float) * dvw, stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(dlambda, 0, sizeof(float), stream);
  if (e != cudaSuccess) return e;
  const int kstride = (d % 2 == 0) ? d + 1 : d;
  const size_t sm_rows = sizeof(float) * (2 * kRows * d + 2 * kTile * kstride + kTile * dvw);
  const size_t sm_keys = sizeof(float) * (2 * kRows * d + kRows * dvw + 2 * kTile * kstride + kTile * (dvw + 1)) +
                         sizeof(float4) * kTile;
  const size_t sm_qs = sizeof(float) * (2 * kRows * d + kRows * dvw + 2 * kTile * kstride + kTile * (dvw + 1));
  e = cudaFuncSetAttribute(bwd_rows_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(sm_rows));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(bwd_keys_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(sm_keys));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(bwd_queries_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(sm_qs));
  if (e != cudaSuccess) return e;
  const dim3 grid((N + kRows - 1) / kRows, H, B);
  const T* qt = static_cast<const T*>(q);
  const T* kt = static_cast<const T*>(k);
  const T* vt = static_cast<const T*>(v);
  bwd_rows_kernel<T><<<grid, 256, sm_rows, stream>>>(qt, kt, vt, static_cast<const T*>(dy), lambda, mode, a);
  bwd_keys_kernel<T><<<grid, 256, sm_keys, stream>>>(qt, kt, vt, lambda, mode, a);
  bwd_queries_kernel<T><<<grid, 256, sm_qs, stream>>>(qt, kt, vt, lambda, mode, a);
  return cudaGetLastError();
}

}  // namespace

size_t bwd_workspace_bytes(int B, int N, int H, int d) {
  const size_t g = ((sizeof(float) * static_cast<size_t>(B) * N * H * 2 * d) + 255) / 256 * 256;
  return g + sizeof(float4) * static_cast<size_t>(B) * N * H;
}

cudaError_t launch_bwd(const void* q, const void* k, const void* v, const void* dy, int bf16, int B, int N, int H,
                       int d, int causal, const float* lambda, float lambda_init, const float* rms_w, float eps,
                       int mode, float* dq, float* dk, float* dv, float* dlambda, float* drms_w, void* workspace,
                       cudaStream_t stream) {
  if (bf16)
    return launch_bwd_t<__nv_bfloat16>(q, k, v, dy, B, N, H, d, causal, lambda, lambda_init, rms_w, eps, mode, dq,
                                       dk, dv, dlambda, drms_w, workspace, stream);
  return launch_bwd_t<float>(q, k, v, dy, B, N, H, d, causal, lambda, lambda_init, rms_w, eps, mode, dq, dk, dv,
                             dlambda, drms_w, workspace, stream);
}

cudaError_t launch_lambda_bwd(const float* lq1, const float* lk1, const float* lq2, const float* lk2, int d,
                              const float* dlambda, float* dlq1, float* dlk1, float* dlq2, float* dlk2,
                              cudaStream_t stream) {
  lambda_bwd_kernel<<<1, 32, 0, stream>>>(lq1, lk1, lq2, lk2, d, dlambda, dlq1, dlk1, dlq2, dlk2);
  return cudaGetLastError();
}

}  // namespace diffattn
