// The dense steps either side of the attention path, on the tensor cores:
// the query/key/value projection with the rotary position embedding fused
// into its epilogue, and the output projection (page "Differential
// attention", "How it's wired (and why it's nearly free)": each head's query
// and key projections split into halves Q1, K1 and Q2, K2; the layer sits in
// a standard transformer block).  RoPE follows RoFormer (cited on page
// "Differential Transformer", "Builds on"): consecutive channel pairs of each
// d-wide Q1, Q2, K1, K2 rotated by n * base^(-2j/d) at token position n.
//
// One persistent GEMM kernel on CTA pairs, C[M, N] = A[M, K] B[N, K]^T (bf16
// operands, fp32 accumulation in tensor memory, bf16 output):
//   warp 0       TMA producer (each CTA): its 128 rows of A and 128 rows of B
//                per 64-wide K step, 6 stages
//   warp 1       MMA issuer (the pair's leader): tcgen05.mma cta_group::2,
//                M=256 N=256 K=16; two accumulator buffers of 256 columns in
//                each CTA so that a tile's epilogue overlaps the next tile's
//                products
//   warps 4-7    epilogue (each CTA): one output row per thread, 32 columns at
//                a time: rotate pairs (columns below rope_end) with the cos/sin
//                table, round to bf16, store into the destination that owns
//                the columns (q | k | v for the projection)
// Tiles are visited in groups of 8 row blocks (2048 rows) so that the pairs
// working at the same time share their B (weight) columns and A rows in L2.
#include <cuda_bf16.h>
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace diffattn {

namespace {

constexpr int kPThreads = 256;
constexpr int kPBK = 64;  // K per stage: one 128-byte swizzle row of bf16

// A 256 x 256 tile per CTA pair, tcgen05.mma with cta_group::2 (M = 256)
// issued by the pair's leader.  Each CTA loads its own 128 rows of A and its
// own 128 rows of B (half the tile's N) per stage, so each SM's shared memory
// carries half the B traffic of a one-CTA 128 x 256 tile; each CTA's tensor
// memory receives its 128 rows of D.  Stage barriers live in the leader
// (armed with both CTAs' bytes); the leader's commits arrive on both CTAs'
// barriers; the peer's epilogue hands accumulators back to the leader with
// remote arrivals.
constexpr int k2BM = 256, k2BN = 256;
constexpr int k2Stages = 6;
constexpr int k2ABytes = 128 * kPBK * 2;  // this CTA's 128 rows of A
constexpr int k2BBytes = 128 * kPBK * 2;  // this CTA's 128 rows of B
constexpr int k2StageBytes = k2ABytes + k2BBytes;
constexpr int k2OffBar = k2Stages * k2StageBytes;
constexpr int k2Smem = k2OffBar + 256 + 1024;
constexpr int k2GroupM = 8;
static_assert(k2Smem <= 232448, "shared memory per CTA");

struct Proj2Bars {
  uint64_t full[k2Stages], empty[k2Stages];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
};

__global__ void __launch_bounds__(kPThreads, 1)
    proj_gemm_sm100_kernel(const __grid_constant__ CUtensorMap ta, const __grid_constant__ CUtensorMap tb,
                         const ProjParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Proj2Bars* bars = reinterpret_cast<Proj2Bars*>(smem + k2OffBar);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();  // 0: the pair's leader (issues the MMAs)
  const bool leader = rank == 0;
  const int cid = static_cast<int>(blockIdx.x >> 1), n_cl = static_cast<int>(gridDim.x >> 1);
  const int tiles_m = (p.M + k2BM - 1) / k2BM, tiles_n = (p.N + k2BN - 1) / k2BN;
  const int n_tiles = tiles_m * tiles_n;
  const int k_steps = p.K / kPBK;
  auto tile_coords = [&](int t, int& tm, int& tn) {
    const int per_group = k2GroupM * tiles_n;
    const int g = t / per_group, first = g * k2GroupM;
    const int gm = min(k2GroupM, tiles_m - first);
    const int r = t % per_group;
    tm = first + r % gm;
    tn = r / gm;
  };
  auto lead = [&](uint64_t* bar) { return map_to_cta(smem_u32(bar), 0); };

  if (tid == 0) {
    for (int i = 0; i < k2Stages; ++i) {
      mbar_init(&bars->full[i], 1);
      mbar_init(&bars->empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->acc_full[i], 1);
      mbar_init(&bars->acc_empty[i], 8);  // every epilogue warp of both CTAs
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
    tmem_alloc_pair(&bars->tmem_base, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers exist before any cross-CTA arrival
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const WaitCtl wc{p.status, &bars->abort, p.limit_ns};
  int drain_abort = 0;
  const WaitCtl wdrain{p.status, &drain_abort, 1000000000ull};

  if (warp == 0) {
    // ------------------------------------------------------------ producer --
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int t = cid; ok && t < n_tiles; t += n_cl) {
        int tm, tn;
        tile_coords(t, tm, tn);
        for (int ks = 0; ks < k_steps; ++ks, ++it) {
          const int s = it % k2Stages;
          if (!(ok = mbar_wait(&bars->empty[s], ((it / k2Stages) & 1) ^ 1, wc))) break;
          if (leader) mbar_arrive_expect_tx(&bars->full[s], 2 * k2StageBytes);
          uint8_t* st = smem + s * k2StageBytes;
          const uint32_t fb = lead(&bars->full[s]);
          // debug builds: the tiles start inside A [M, K] and B [N, K] (TMA fills the rest with zeros)
          (void)DA_CHECK(p.status, ks * kPBK < p.K && tm * k2BM < p.M && tn * k2BN < p.N);
          tma_load_4d_pair(st, &ta, fb, ks * kPBK, 0, tm * k2BM + 128 * static_cast<int>(rank), 0);
          tma_load_4d_pair(st + k2ABytes, &tb, fb, ks * kPBK, 0, tn * k2BN + 128 * static_cast<int>(rank), 0);
        }
      }
      // the leader's barriers count both CTAs' bytes: wait until nothing is still landing
      if (leader)
        for (int j = max(0, it - k2Stages); j < it; ++j)
          mbar_wait(&bars->full[j % k2Stages], (j / k2Stages) & 1, wdrain);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer (leader) --
    if (lane == 0 && leader) {
      constexpr uint32_t idesc = idesc_bf16_f32(k2BM, k2BN, false, false);
      const uint64_t s_desc = smem_desc_sw128(smem_u32(smem), 16, 1024);
      auto adv = [](uint64_t desc, uint32_t bytes) { return desc + static_cast<uint64_t>(bytes >> 4); };
      int it = 0, lt = 0;
      bool ok = true;
      for (int t = cid; ok && t < n_tiles; t += n_cl, ++lt) {
        const int ab = lt & 1;
        // both CTAs' epilogues have drained this accumulator buffer (tile lt - 2)
        if (lt >= 2 && !(ok = mbar_wait_acq_cluster(&bars->acc_empty[ab], ((lt - 2) >> 1) & 1, wc))) break;
        tc_fence_after();
        for (int ks = 0; ks < k_steps; ++ks, ++it) {
          const int s = it % k2Stages;
          if (!(ok = mbar_wait(&bars->full[s], (it / k2Stages) & 1, wc))) break;
          tc_fence_after();
          const uint32_t so = s * k2StageBytes;
#pragma unroll
          for (int kk = 0; kk < kPBK / 16; ++kk)
            umma_ss_pair(tmem + 256u * ab, adv(s_desc, so + kk * 32), adv(s_desc, so + k2ABytes + kk * 32), idesc,
                         (ks > 0 || kk > 0) ? 1u : 0u);
          umma_commit_pair_mc(&bars->empty[s], 0x3);  // both CTAs' stage s is free once these have read it
        }
        if (ok) umma_commit_pair_mc(&bars->acc_full[ab], 0x3);
      }
      umma_commit_pair_mc(&bars->mma_done, 0x3);  // drain: both CTAs learn when every product has completed
    }
    if (lane == 0) mbar_wait(&bars->mma_done, 0, wdrain);
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue --
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t tl = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    int lt = 0;
    for (int t = cid; t < n_tiles; t += n_cl, ++lt) {
      const int ab = lt & 1;
      int tm, tn;
      tile_coords(t, tm, tn);
      if (!mbar_wait(&bars->acc_full[ab], (lt >> 1) & 1, wc)) break;
      tc_fence_after();
      const int m = tm * k2BM + 128 * static_cast<int>(rank) + r;
      const bool live = m < p.M;
      const int pos = live ? m % p.seq_len : 0;
#pragma unroll 1
      for (int c = 0; c < k2BN / 32; ++c) {
        uint32_t v[32];
        tmem_ld32_sync(tl + 256u * ab + 32 * c, v);
        const int col = tn * k2BN + 32 * c;
        if (!live || col >= p.N) continue;
        const bool in0 = col < p.col_end[0], in1 = !in0 && col < p.col_end[1];
        const int start = in0 ? 0 : (in1 ? p.col_end[0] : p.col_end[1]);
        const int width = (in0 ? p.col_end[0] : (in1 ? p.col_end[1] : p.col_end[2])) - start;
        __nv_bfloat16* obase = in0 ? p.out[0] : (in1 ? p.out[1] : p.out[2]);
        const int c_in = col - start;
        if (p.rope && col < p.rope_end) {
          const float2* cs = p.rope + static_cast<size_t>(pos) * (p.d / 2) + (c_in % p.d) / 2;
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float2 t2 = __ldg(cs + j);
            const float x0 = __uint_as_float(v[2 * j]), x1 = __uint_as_float(v[2 * j + 1]);
            v[2 * j] = __float_as_uint(fmaf(x0, t2.x, -x1 * t2.y));
            v[2 * j + 1] = __float_as_uint(fmaf(x0, t2.y, x1 * t2.x));
          }
        }
        // debug builds: the 32 columns lie in their output, and their rotary entries in the table
        if (!DA_CHECK(p.status, c_in >= 0 && c_in + 32 <= width && (!p.rope || col >= p.rope_end ||
                                                                    pos < p.seq_len)))
          continue;
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
      if (lane == 0) mbar_arrive_remote(lead(&bars->acc_empty[ab]));  // this CTA's rows of the buffer are read
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // no remote access to either CTA remains
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

__global__ void rope_table_kernel(int seq_len, int d, double base, float2* table, int* dbg) {
  const int half = d / 2;
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= static_cast<long long>(seq_len) * half) return;
  const int n = static_cast<int>(i / half), j = static_cast<int>(i % half);
  if (!DA_CHECK(dbg, n < seq_len && j < half)) return;
  const double ang = static_cast<double>(n) * pow(base, -2.0 * j / d);
  double s, c;
  sincos(ang, &s, &c);
  table[i] = make_float2(static_cast<float>(c), static_cast<float>(s));
}

}  // namespace

cudaError_t launch_proj_gemm(const CUtensorMap& ta, const CUtensorMap& tb, const ProjParams& prm,
                                 cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(proj_gemm_sm100_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, k2Smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kPThreads, 1, 1);
  cfg.dynamicSmemBytes = k2Smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  static int max_clusters[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
  int& mc = max_clusters[dev];
  if (mc == 0) {
    cfg.gridDim = dim3(2 * 128, 1, 1);
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, proj_gemm_sm100_kernel, &cfg) != cudaSuccess || n < 1) n = 1;
    mc = n;
  }
  const int tiles = ((prm.M + k2BM - 1) / k2BM) * ((prm.N + k2BN - 1) / k2BN);
  const int clusters = tiles < mc ? tiles : mc;
  cfg.gridDim = dim3(2 * clusters, 1, 1);
  return cudaLaunchKernelEx(&cfg, proj_gemm_sm100_kernel, ta, tb, prm);
}

cudaError_t launch_rope_table(int seq_len, int d, double base, float* table, cudaStream_t stream) {
  const long long n = static_cast<long long>(seq_len) * (d / 2);
  const unsigned grid = static_cast<unsigned>((n + 255) / 256);
  rope_table_kernel<<<grid, 256, 0, stream>>>(seq_len, d, base, reinterpret_cast<float2*>(table), debug_status());
  return cudaGetLastError();
}

}  // namespace diffattn
