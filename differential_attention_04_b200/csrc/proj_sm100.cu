// The dense steps either side of the attention path, on the tensor cores:
// the query/key/value projection with the rotary position embedding fused
// into its epilogue, and the output projection (page "Differential
// attention", "How it's wired (and why it's nearly free)": each head's query
// and key projections split into halves Q1, K1 and Q2, K2; the layer sits in
// a standard transformer block).  RoPE follows RoFormer (cited on page
// "Differential Transformer", "Builds on"): consecutive channel pairs of each
// d-wide Q1, Q2, K1, K2 rotated by n * base^(-2j/d) at token position n.
//
// One persistent GEMM kernel, C[M, N] = A[M, K] B[N, K]^T (bf16 operands,
// fp32 accumulation in tensor memory, bf16 output):
//   warp 0       TMA producer: A [128 x 64] and B [256 x 64] tiles, 4 stages
//   warp 1       MMA issuer: tcgen05.mma M=128 N=256 K=16, two accumulator
//                buffers of 256 columns so that a tile's epilogue overlaps
//                the next tile's products
//   warps 4-7    epilogue: one output row per thread, 32 columns at a time:
//                rotate pairs (columns below rope_end) with the cos/sin
//                table, round to bf16, store into the destination that owns
//                the columns (q | k | v for the projection)
// Tiles are visited in groups of 16 row blocks so that the CTAs working at
// the same time share their B (weight) columns and A rows in L2.
#include <cuda_bf16.h>
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace diffattn {

namespace {

constexpr int kPThreads = 256;
constexpr int kPBM = 128, kPBN = 256, kPBK = 64;
constexpr int kPStages = 4;
constexpr int kPGroupM = 16;
constexpr int kPABytes = kPBM * kPBK * 2;  // 16 KB
constexpr int kPBBytes = kPBN * kPBK * 2;  // 32 KB
constexpr int kPStageBytes = kPABytes + kPBBytes;
constexpr int kPOffBar = kPStages * kPStageBytes;
constexpr int kPSmem = kPOffBar + 256 + 1024;
static_assert(kPSmem <= 232448, "shared memory per CTA");

struct ProjBars {
  uint64_t full[kPStages], empty[kPStages];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t mma_done;  // every product this CTA issued has completed
  uint32_t tmem_base;
  int abort;
};

__global__ void __launch_bounds__(kPThreads, 1)
    proj_gemm_sm100_kernel(const __grid_constant__ CUtensorMap ta, const __grid_constant__ CUtensorMap tb,
                           const ProjParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  ProjBars* bars = reinterpret_cast<ProjBars*>(smem + kPOffBar);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tiles_m = (p.M + kPBM - 1) / kPBM, tiles_n = (p.N + kPBN - 1) / kPBN;
  const int n_tiles = tiles_m * tiles_n;
  const int k_steps = p.K / kPBK;
  auto tile_coords = [&](int t, int& tm, int& tn) {
    const int per_group = kPGroupM * tiles_n;
    const int g = t / per_group, first = g * kPGroupM;
    const int gm = min(kPGroupM, tiles_m - first);
    const int r = t % per_group;
    tm = first + r % gm;
    tn = r / gm;
  };

  if (tid == 0) {
    for (int i = 0; i < kPStages; ++i) {
      mbar_init(&bars->full[i], 1);
      mbar_init(&bars->empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->acc_full[i], 1);
      mbar_init(&bars->acc_empty[i], 4);  // one arrival per epilogue warp
    }
    mbar_init(&bars->mma_done, 1);
    bars->abort = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&ta);
    tma_prefetch_desc(&tb);
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const WaitCtl wc{p.status, &bars->abort, p.limit_ns};
  int drain_abort = 0;
  const WaitCtl wdrain{p.status, &drain_abort, 1000000000ull};

  if (warp == 0) {
    // ------------------------------------------------------------ producer --
    if (lane == 0) {
      int it = 0;  // k steps issued (all tiles)
      bool ok = true;
      for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x) {
        int tm, tn;
        tile_coords(t, tm, tn);
        for (int ks = 0; ks < k_steps; ++ks, ++it) {
          const int s = it % kPStages;
          if (!(ok = mbar_wait(&bars->empty[s], ((it / kPStages) & 1) ^ 1, wc))) break;
          mbar_arrive_expect_tx(&bars->full[s], kPStageBytes);
          uint8_t* st = smem + s * kPStageBytes;
          tma_load_4d(st, &ta, &bars->full[s], ks * kPBK, 0, tm * kPBM, 0);
          tma_load_4d(st + kPABytes, &tb, &bars->full[s], ks * kPBK, 0, tn * kPBN, 0);
        }
      }
      for (int j = max(0, it - kPStages); j < it; ++j) mbar_wait(&bars->full[j % kPStages], (j / kPStages) & 1, wdrain);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kPBM, kPBN, false, false);
      const uint32_t s0 = smem_u32(smem);
      int it = 0, lt = 0;  // k steps consumed, tiles done (this CTA)
      bool ok = true;
      for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x, ++lt) {
        const int ab = lt & 1;
        // the epilogue has drained this accumulator buffer (tile lt - 2)
        if (lt >= 2 && !(ok = mbar_wait(&bars->acc_empty[ab], ((lt - 2) >> 1) & 1, wc))) break;
        tc_fence_after();
        for (int ks = 0; ks < k_steps; ++ks, ++it) {
          const int s = it % kPStages;
          if (!(ok = mbar_wait(&bars->full[s], (it / kPStages) & 1, wc))) break;
          tc_fence_after();
          const uint32_t sa = s0 + s * kPStageBytes, sb = sa + kPABytes;
#pragma unroll
          for (int kk = 0; kk < kPBK / 16; ++kk)
            umma_ss(tmem + 256u * ab, smem_desc_sw128(sa + kk * 32, 16, 1024), smem_desc_sw128(sb + kk * 32, 16, 1024),
                    idesc, (ks > 0 || kk > 0) ? 1u : 0u);
          umma_commit(&bars->empty[s]);  // the stage is free once these products have read it
        }
        if (ok) umma_commit(&bars->acc_full[ab]);
      }
      // drain: no product may still be writing tensor memory when it is freed
      umma_commit(&bars->mma_done);
      mbar_wait(&bars->mma_done, 0, wdrain);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue --
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t tl = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    int lt = 0;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++lt) {
      const int ab = lt & 1;
      int tm, tn;
      tile_coords(t, tm, tn);
      if (!mbar_wait(&bars->acc_full[ab], (lt >> 1) & 1, wc)) break;
      tc_fence_after();
      const int m = tm * kPBM + r;
      const bool live = m < p.M;
      const int pos = live ? m % p.seq_len : 0;
#pragma unroll 1
      for (int c = 0; c < kPBN / 32; ++c) {
        uint32_t v[32];
        tmem_ld32_sync(tl + 256u * ab + 32 * c, v);
        const int col = tn * kPBN + 32 * c;
        if (!live || col >= p.N) continue;
        // destination: the output owning these 32 columns (selects, no indexed parameter reads)
        const bool in0 = col < p.col_end[0], in1 = !in0 && col < p.col_end[1];
        const int start = in0 ? 0 : (in1 ? p.col_end[0] : p.col_end[1]);
        const int width = (in0 ? p.col_end[0] : (in1 ? p.col_end[1] : p.col_end[2])) - start;
        __nv_bfloat16* obase = in0 ? p.out[0] : (in1 ? p.out[1] : p.out[2]);
        const int c_in = col - start;
        if (p.rope && col < p.rope_end) {
          // rotate 16 consecutive pairs: channel (c_in mod d), position pos
          const float2* cs = p.rope + static_cast<size_t>(pos) * (p.d / 2) + (c_in % p.d) / 2;
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float2 t2 = __ldg(cs + j);
            const float x0 = __uint_as_float(v[2 * j]), x1 = __uint_as_float(v[2 * j + 1]);
            v[2 * j] = __float_as_uint(fmaf(x0, t2.x, -x1 * t2.y));
            v[2 * j + 1] = __float_as_uint(fmaf(x0, t2.y, x1 * t2.x));
          }
        }
        uint4* dst = reinterpret_cast<uint4*>(obase + static_cast<size_t>(m) * width + c_in);
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4)
          dst[q4] = make_uint4(pack_bf16x2(__uint_as_float(v[8 * q4 + 0]), __uint_as_float(v[8 * q4 + 1])),
                               pack_bf16x2(__uint_as_float(v[8 * q4 + 2]), __uint_as_float(v[8 * q4 + 3])),
                               pack_bf16x2(__uint_as_float(v[8 * q4 + 4]), __uint_as_float(v[8 * q4 + 5])),
                               pack_bf16x2(__uint_as_float(v[8 * q4 + 6]), __uint_as_float(v[8 * q4 + 7])));
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->acc_empty[ab]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

__global__ void rope_table_kernel(int seq_len, int d, double base, float2* table) {
  const int half = d / 2;
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= static_cast<long long>(seq_len) * half) return;
  const int n = static_cast<int>(i / half), j = static_cast<int>(i % half);
  const double ang = static_cast<double>(n) * pow(base, -2.0 * j / d);
  double s, c;
  sincos(ang, &s, &c);
  table[i] = make_float2(static_cast<float>(c), static_cast<float>(s));
}

}  // namespace

cudaError_t launch_proj_gemm(const CUtensorMap& ta, const CUtensorMap& tb, const ProjParams& prm,
                             cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(proj_gemm_sm100_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kPSmem);
  if (e != cudaSuccess) return e;
  static int sms[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
  if (sms[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) n = 1;
    sms[dev] = n;
  }
  const int tiles = ((prm.M + kPBM - 1) / kPBM) * ((prm.N + kPBN - 1) / kPBN);
  const int grid = tiles < sms[dev] ? tiles : sms[dev];
  proj_gemm_sm100_kernel<<<grid, kPThreads, kPSmem, stream>>>(ta, tb, prm);
  return cudaGetLastError();
}

cudaError_t launch_rope_table(int seq_len, int d, double base, float* table, cudaStream_t stream) {
  const long long n = static_cast<long long>(seq_len) * (d / 2);
  const unsigned grid = static_cast<unsigned>((n + 255) / 256);
  rope_table_kernel<<<grid, 256, 0, stream>>>(seq_len, d, base, reinterpret_cast<float2*>(table));
  return cudaGetLastError();
}

}  // namespace diffattn
