// Split-KV decode (query length 1) over a packed bf16 KV cache, d = 128.
//
// Per (sequence, head) it computes the DiffAttn equation for one query (page
// "Differential Transformer: Canceling Context Noise with Differential
// Attention", "Cancelling Context Noise Through Attention Map Subtraction";
// peer review "Differential Transformer", Summary, Eq. 1) against every cached
// key of the sequence, then the headwise RMSNorm and the (1 - lambda_init)
// scale (Eq. 3).
//
// The work is bandwidth-bound (1 KiB of K and V per key and head, about 1.5
// flop per byte), so it runs on CUDA cores:
//   * decode_plan_kernel: one CTA turns cu_seqlens into the chunk offsets of
//     each sequence (ceil(L / 512) chunks of up to 512 keys, at least one),
//     so that the next kernel visits only chunks that exist.
//   * decode_partial_kernel: a persistent grid (as many CTAs as fit on the
//     GPU at once) takes (chunk, head) units from a counter one at a time,
//     so that every CTA keeps working until the units run out whatever the
//     mix of full and partial chunks.  Each warp streams its keys with
//     16-byte non-allocating loads,
//     8 keys in flight per lane group; lane l holds elements [8l, 8l+8) of
//     the 256-wide K row (lanes 0-15: map 1, lanes 16-31: map 2) and of the V
//     row.  The 8 partial dot products are reduced across 16 lanes with a
//     transposing shuffle tree (8 shuffles for 8 keys), and each map keeps its
//     own online softmax state in the log2 domain.  The 4 warps merge, and
//     the CTA writes (m1, l1, m2, l2, o1[256], o2[256]) for its chunk.
//   * decode_combine_kernel: one CTA per (head, sequence) merges the
//     sequence's chunks with the log-sum-exp rescale per map (four groups of
//     256 threads, one thread per channel, each group a quarter of the
//     chunks, then the groups' sums in a fixed order), forms
//     o1/l1 - lambda o2/l2, and applies the RMSNorm and scale.
// Workspace: the chunk records (room for S * ceil(max_seqlen / 512) chunks
// per head), then the S + 1 chunk offsets and the work counter.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace diffattn {

namespace {
constexpr int kD = 128;                 // per-map width
constexpr int kDV = 2 * kD;             // value / output width
constexpr int kWarps = 4;
constexpr int kGroup = 8;               // keys in flight per warp
constexpr int kKeysPerWarp = 128;
constexpr int kChunk = kWarps * kKeysPerWarp;  // keys per CTA
constexpr int kRecFloats = 4 + 2 * kDV;        // m1, l1, m2, l2, o1[256], o2[256]
constexpr int kCombGroups = 4;                  // chunk groups the combine merges side by side
constexpr int kCombThreads = kCombGroups * kDV;  // combine CTA: one thread per (group, channel)
constexpr float kLog2e = 1.4426950408889634f;
}  // namespace

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float (&f)[8]) {
  f[0] = bf16lo_to_f32(u.x); f[1] = bf16hi_to_f32(u.x);
  f[2] = bf16lo_to_f32(u.y); f[3] = bf16hi_to_f32(u.y);
  f[4] = bf16lo_to_f32(u.z); f[5] = bf16hi_to_f32(u.z);
  f[6] = bf16lo_to_f32(u.w); f[7] = bf16hi_to_f32(u.w);
}

// Keys of sequence s (its first key in *lo).  Debug builds check that the
// keys lie in the packed cache (offsets non-decreasing and ending at
// cu_seqlens[S]), where a sequence outside it is skipped, and that there are
// at most max_seqlen of them: a longer sequence is cut to its first
// max_seqlen keys, as release builds always do, and flagged.
__device__ __forceinline__ int seq_keys(const int* __restrict__ cu, int s, int S, int max_seqlen, int* dbg,
                                        int* lo) {
  *lo = cu[s];
  const int hi = cu[s + 1];
  if (!DA_CHECK(dbg, *lo >= 0 && hi >= *lo && hi <= cu[S])) return 0;
  (void)DA_CHECK(dbg, hi - *lo <= max_seqlen);
  return min(hi - *lo, max_seqlen);
}

// chunk_start[s] = chunks of the sequences before s; chunk_start[S] = all chunks.
// chunk_start[S + 1] is the partial kernel's work counter: set to 0 here.
__global__ void __launch_bounds__(1024) decode_plan_kernel(const int* __restrict__ cu_seqlens, int S,
                                                           int max_seqlen, int* __restrict__ chunk_start,
                                                           int* dbg) {
  __shared__ int warp_sum[32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int carry = 0;
  for (int base = 0; base < S; base += 1024) {
    const int s = base + static_cast<int>(threadIdx.x);
    int n = 0;
    if (s < S) {
      int lo;
      const int L = seq_keys(cu_seqlens, s, S, max_seqlen, dbg, &lo);
      n = max(1, (L + kChunk - 1) / kChunk);
    }
    // inclusive scan of n over the block: within each warp, then over the warps
    int x = n;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, off);
      if (lane >= off) x += y;
    }
    if (lane == 31) warp_sum[warp] = x;
    __syncthreads();
    if (warp == 0) {
      int w = warp_sum[lane];
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, w, off);
        if (lane >= off) w += y;
      }
      warp_sum[lane] = w;  // inclusive over warps
    }
    __syncthreads();
    const int before = (warp > 0 ? warp_sum[warp - 1] : 0) + x - n;
    if (s < S) chunk_start[s] = carry + before;
    carry += warp_sum[31];
    __syncthreads();  // warp_sum is rewritten by the next pass
  }
  if (threadIdx.x == 0) {
    chunk_start[S] = carry;
    chunk_start[S + 1] = 0;
  }
}

__global__ void __launch_bounds__(kWarps * 32) decode_partial_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ kc, const __nv_bfloat16* __restrict__ vc,
    const int* __restrict__ cu_seqlens, int S, int max_seqlen, int H, const int* __restrict__ chunk_start,
    float* __restrict__ ws, int* dbg) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int half = lane >> 4;  // 0: map 1, 1: map 2
  const int hl = lane & 15;
  const int total = chunk_start[S];
  int* next = const_cast<int*>(chunk_start) + S + 1;  // work counter: (chunk, head) units handed out
  __shared__ float sm_m[kWarps][2], sm_l[kWarps][2];
  __shared__ float sm_o[kWarps][2][kDV];
  __shared__ int s_unit[2];  // this CTA's current and next unit

  // Units are taken from the counter one at a time (the next one while the
  // current is processed), so a CTA that drew short chunks takes more of
  // them and all finish together.  Unit u is chunk u / H of head u % H.
  const int units = total * H;
  if (threadIdx.x == 0) s_unit[0] = atomicAdd(next, 1);
  __syncthreads();
  for (int it = 0;; ++it) {
    const int u = s_unit[it & 1];
    if (u >= units) break;
    if (threadIdx.x == 0) s_unit[(it + 1) & 1] = atomicAdd(next, 1);
    const int c = u / H, h = u % H;
    // the sequence of chunk c: the last s with chunk_start[s] <= c
    int s = 0;
    {
      int hi = S - 1;
      while (s < hi) {
        const int m = (s + hi + 1) >> 1;
        if (chunk_start[m] <= c) s = m;
        else hi = m - 1;
      }
    }
    const int chunk = c - chunk_start[s];
    int lo;
    const int L = seq_keys(cu_seqlens, s, S, max_seqlen, dbg, &lo);
    const int c0 = chunk * kChunk;

    // This lane's slice of q (map `half`, elements [8*hl, 8*hl + 8)), pre-scaled
    // so that scores come out in log2 units: s * log2(e) / sqrt(d).
    float qf[8];
    {
      const uint4 qu = *reinterpret_cast<const uint4*>(q + (static_cast<size_t>(s) * H + h) * kDV + 8 * lane);
      bf16x8_to_f32(qu, qf);
      const float sc = kLog2e * rsqrtf(static_cast<float>(kD));
#pragma unroll
      for (int i = 0; i < 8; ++i) qf[i] *= sc;
    }

    float m1 = -INFINITY, m2 = -INFINITY;  // running max per map (same in all lanes)
    float lsum = 0.f;                      // this lane's share of its map's running sum
    float o1[8], o2[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) o1[i] = o2[i] = 0.f;

    const size_t row_stride = static_cast<size_t>(H) * kDV;  // elements between consecutive keys
    const int kbeg = c0 + warp * kKeysPerWarp;
    const int kend = min(L, kbeg + kKeysPerWarp);
    const __nv_bfloat16* kbase = kc + static_cast<size_t>(lo) * row_stride + static_cast<size_t>(h) * kDV + 8 * lane;
    const __nv_bfloat16* vbase = vc + static_cast<size_t>(lo) * row_stride + static_cast<size_t>(h) * kDV + 8 * lane;

    for (int k0 = kbeg; k0 < kend; k0 += kGroup) {
      uint4 kr[kGroup], vr[kGroup];
#pragma unroll
      for (int g = 0; g < kGroup; ++g) {
        const int key = k0 + g;
        if (key < kend) {
          kr[g] = ldg_stream_v4(kbase + static_cast<size_t>(key) * row_stride);
          vr[g] = ldg_stream_v4(vbase + static_cast<size_t>(key) * row_stride);
        } else {
          kr[g] = make_uint4(0, 0, 0, 0);
          vr[g] = make_uint4(0, 0, 0, 0);
        }
      }
      // partial dot products of this lane's 8 elements, one per key
      float part[kGroup];
#pragma unroll
      for (int g = 0; g < kGroup; ++g) {
        float kf[8];
        bf16x8_to_f32(kr[g], kf);
        float a = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) a = fmaf(qf[i], kf[i], a);
        part[g] = a;
      }
      // Transposing reduction over the 16 lanes of each half-warp: after the
      // xor-8, xor-4 and xor-2 steps lane hl holds key g = 4*b3 + 2*b2 + b1
      // (bits of hl) summed over 8 lanes; the xor-1 step completes the sum.
      const bool b3 = (hl >> 3) & 1, b2 = (hl >> 2) & 1, b1 = (hl >> 1) & 1;
      float r4[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float keep = b3 ? part[4 + i] : part[i];
        const float give = b3 ? part[i] : part[4 + i];
        r4[i] = keep + __shfl_xor_sync(0xffffffffu, give, 8);
      }
      float r2[2];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const float keep = b2 ? r4[2 + i] : r4[i];
        const float give = b2 ? r4[i] : r4[2 + i];
        r2[i] = keep + __shfl_xor_sync(0xffffffffu, give, 4);
      }
      float sc;
      {
        const float keep = b1 ? r2[1] : r2[0];
        const float give = b1 ? r2[0] : r2[1];
        sc = keep + __shfl_xor_sync(0xffffffffu, give, 2);
      }
      sc += __shfl_xor_sync(0xffffffffu, sc, 1);
      const int my_key = 4 * b3 + 2 * b2 + b1;  // lanes 2g and 2g+1 of each half hold key g
      if (k0 + my_key >= kend) sc = -INFINITY;

      // group max per map, shared with the other half
      float mx = sc;
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float mx_other = __shfl_xor_sync(0xffffffffu, mx, 16);
      const float gm1 = half ? mx_other : mx;
      const float gm2 = half ? mx : mx_other;
      const float mn1 = fmaxf(m1, gm1), mn2 = fmaxf(m2, gm2);
      const float al1 = fast_exp2(m1 - mn1), al2 = fast_exp2(m2 - mn2);  // exp2(-inf) = 0
      m1 = mn1;
      m2 = mn2;
      const float p = fast_exp2(sc - (half ? mn2 : mn1));  // 0 for masked keys
      lsum = lsum * (half ? al2 : al1) + ((lane & 1) ? 0.f : p);

#pragma unroll
      for (int i = 0; i < 8; ++i) {
        o1[i] *= al1;
        o2[i] *= al2;
      }
#pragma unroll
      for (int g = 0; g < kGroup; ++g) {
        const float p1 = __shfl_sync(0xffffffffu, p, 2 * g);
        const float p2 = __shfl_sync(0xffffffffu, p, 16 + 2 * g);
        float vf[8];
        bf16x8_to_f32(vr[g], vf);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          o1[i] = fmaf(p1, vf[i], o1[i]);
          o2[i] = fmaf(p2, vf[i], o2[i]);
        }
      }
    }

    // running sums per map: sum the lanes of each half
    float l = lsum;
    l += __shfl_xor_sync(0xffffffffu, l, 8);
    l += __shfl_xor_sync(0xffffffffu, l, 4);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    const float l_other = __shfl_xor_sync(0xffffffffu, l, 16);
    const float l1 = half ? l_other : l, l2 = half ? l : l_other;

    // merge the warps of the CTA
    if (lane == 0) {
      sm_m[warp][0] = m1; sm_m[warp][1] = m2;
      sm_l[warp][0] = l1; sm_l[warp][1] = l2;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      sm_o[warp][0][8 * lane + i] = o1[i];
      sm_o[warp][1][8 * lane + i] = o2[i];
    }
    __syncthreads();
    float* rec = ws + (static_cast<size_t>(c) * H + h) * kRecFloats;
    for (int mp = 0; mp < 2; ++mp) {
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) M = fmaxf(M, sm_m[w][mp]);
      float f[kWarps];
#pragma unroll
      for (int w = 0; w < kWarps; ++w) f[w] = (M == -INFINITY) ? 0.f : fast_exp2(sm_m[w][mp] - M);
      for (int cc = threadIdx.x; cc < kDV; cc += blockDim.x) {
        float acc = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) acc = fmaf(f[w], sm_o[w][mp][cc], acc);
        rec[4 + mp * kDV + cc] = acc;
      }
      if (threadIdx.x == 0) {
        float Ls = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) Ls = fmaf(f[w], sm_l[w][mp], Ls);
        rec[2 * mp] = M;
        rec[2 * mp + 1] = Ls;
      }
    }
    __syncthreads();  // the merge buffers are refilled by the next chunk; the next unit is visible
  }
}

__global__ void __launch_bounds__(kCombThreads) decode_combine_kernel(const float* __restrict__ ws,
                                                                      const int* __restrict__ chunk_start, int H,
                                                                      __nv_bfloat16* __restrict__ o,
                                                                      const float* __restrict__ lambda_ptr, int mode,
                                                                      float lambda_init,
                                                                      const float* __restrict__ rms_w, float eps,
                                                                      int* dbg) {
  const int h = blockIdx.x, s = blockIdx.y;
  const int tid = threadIdx.x;
  const int c = tid % kDV;     // output channel
  const int grp = tid / kDV;   // chunk group: chunks grp, grp + kCombGroups, ...
  const int first = chunk_start[s];
  int nch = chunk_start[s + 1] - first;
  if (!DA_CHECK(dbg, nch >= 1 && first >= 0 && first + nch <= chunk_start[gridDim.y])) nch = 0;
  // The maxima over the chunks: each thread takes every kCombThreads-th
  // chunk, then a reduction over the block (one round of loads instead of
  // one per chunk).
  __shared__ float mx[2][kCombThreads / 32];
  float M1 = -INFINITY, M2 = -INFINITY;
  for (int i = tid; i < nch; i += kCombThreads) {
    const float* r = ws + (static_cast<size_t>(first + i) * H + h) * kRecFloats;
    M1 = fmaxf(M1, r[0]);
    M2 = fmaxf(M2, r[2]);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    M1 = fmaxf(M1, __shfl_xor_sync(0xffffffffu, M1, off));
    M2 = fmaxf(M2, __shfl_xor_sync(0xffffffffu, M2, off));
  }
  if ((tid & 31) == 0) {
    mx[0][tid >> 5] = M1;
    mx[1][tid >> 5] = M2;
  }
  __syncthreads();
#pragma unroll
  for (int w = 0; w < kCombThreads / 32; ++w) {
    M1 = fmaxf(M1, mx[0][w]);
    M2 = fmaxf(M2, mx[1][w]);
  }
  // Each group's weighted sums over its chunks (the groups run side by side,
  // so a long sequence's chain of loads is kCombGroups times shorter).
  float L1 = 0.f, L2 = 0.f, O1 = 0.f, O2 = 0.f;
#pragma unroll 4
  for (int i = grp; i < nch; i += kCombGroups) {
    const float* r = ws + (static_cast<size_t>(first + i) * H + h) * kRecFloats;
    const float f1 = fast_exp2(r[0] - M1), f2 = fast_exp2(r[2] - M2);
    L1 = fmaf(f1, r[1], L1);
    L2 = fmaf(f2, r[3], L2);
    O1 = fmaf(f1, r[4 + c], O1);
    O2 = fmaf(f2, r[4 + kDV + c], O2);
  }
  __shared__ float po[2][kCombGroups][kDV];
  __shared__ float pl[2][kCombGroups];
  po[0][grp][c] = O1;
  po[1][grp][c] = O2;
  if (c == 0) {
    pl[0][grp] = L1;
    pl[1][grp] = L2;
  }
  __syncthreads();
  // the groups' sums in a fixed order, by the first 256 threads
  float ov = 0.f;
  if (grp == 0) {
    float o1 = 0.f, o2 = 0.f, l1 = 0.f, l2 = 0.f;
#pragma unroll
    for (int g = 0; g < kCombGroups; ++g) {
      o1 += po[0][g][c];
      o2 += po[1][g][c];
      l1 += pl[0][g];
      l2 += pl[1][g];
    }
    ov = o1 / l1 + map2_coefficient(mode, *lambda_ptr) * (o2 / l2);  // c = -lambda, 0 or +lambda
  }
  // sum of squares over the 256 channels
  __shared__ float red[kDV / 32];
  float ss = ov * ov;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
  if (grp == 0 && (c & 31) == 0) red[c >> 5] = ss;
  __syncthreads();
  if (grp == 0) {
    float tot = 0.f;
#pragma unroll
    for (int i = 0; i < kDV / 32; ++i) tot += red[i];
    const float rs = rsqrtf(tot / static_cast<float>(kDV) + eps);
    o[(static_cast<size_t>(s) * H + h) * kDV + c] = __float2bfloat16_rn((1.0f - lambda_init) * rms_w[c] * ov * rs);
  }
}

namespace {
// Byte offset of the chunk offsets in the workspace (after the records).
size_t plan_offset(int S, int H, int max_seqlen) {
  const size_t chunks = (static_cast<size_t>(max_seqlen) + kChunk - 1) / kChunk;
  const size_t rec = static_cast<size_t>(S) * chunks * H * kRecFloats * sizeof(float);
  return (rec + 15) & ~static_cast<size_t>(15);
}
}  // namespace

size_t decode_workspace_bytes(int S, int H, int d, int max_seqlen) {
  if (S <= 0 || H <= 0 || d != kD || max_seqlen <= 0) return 0;
  return plan_offset(S, H, max_seqlen) + ((static_cast<size_t>(S + 2) * sizeof(int) + 15) & ~static_cast<size_t>(15));
}

cudaError_t launch_decode(const void* q, const void* k_cache, const void* v_cache, const int* cu_seqlens,
                          int max_seqlen, void* o, int S, int H, int d, const float* lambda, float lambda_init,
                          const float* rms_w, float eps, int mode, void* workspace, cudaStream_t stream) {
  (void)d;
  int* dbg = debug_status();
  // persistent partial grid: the CTAs that fit on the GPU at once (looked up
  // once per device)
  static int resident[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (resident[dev] == 0) {
    int sms = 0, per_sm = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess)
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_partial_kernel, kWarps * 32, 0);
    if (e != cudaSuccess) return e;
    resident[dev] = sms * (per_sm > 0 ? per_sm : 1);
  }
  const long long max_chunks = (static_cast<long long>(max_seqlen) + kChunk - 1) / kChunk;
  const long long upper = static_cast<long long>(S) * max_chunks;  // chunks there can be
  long long gx = resident[dev];
  if (gx > upper * H) gx = upper * H;
  if (gx < 1) gx = 1;
  float* recs = static_cast<float*>(workspace);
  int* chunk_start = reinterpret_cast<int*>(static_cast<char*>(workspace) + plan_offset(S, H, max_seqlen));
  decode_plan_kernel<<<1, 1024, 0, stream>>>(cu_seqlens, S, max_seqlen, chunk_start, dbg);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  decode_partial_kernel<<<static_cast<unsigned>(gx), kWarps * 32, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k_cache),
      static_cast<const __nv_bfloat16*>(v_cache), cu_seqlens, S, max_seqlen, H, chunk_start, recs, dbg);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  decode_combine_kernel<<<dim3(H, S), kCombThreads, 0, stream>>>(recs, chunk_start, H, static_cast<__nv_bfloat16*>(o), lambda,
                                                        mode, lambda_init, rms_w, eps, dbg);
  return cudaGetLastError();
}

}  // namespace diffattn
