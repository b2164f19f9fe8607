// Tensor-core backward pass of the prefill (bf16 inputs, d in {64, 128},
// float32 gradients).  It differentiates the DiffAttn equation (page
// "Differential Transformer: Canceling Context Noise with Differential
// Attention", "Cancelling Context Noise Through Attention Map Subtraction";
// peer review "Differential Transformer", Summary, Eq. 1), the headwise
// RMSNorm and the (1 - lambda_init) scale (Eq. 3), for any combination mode
// O = A_1 V + c A_2 V (c = -lambda, 0, +lambda):
//
//   G = dO  = g r (w dy) - O g r^3 / (2d) * sum_c (w dy O),  r = 1/sqrt(mean O^2 + eps)
//   dV      = A_1^T G + c A_2^T G
//   dS_i    = A_i * (c_i G V^T - D_i),  c_1 = 1, c_2 = c,  D_i = c_i G . (A_i V)
//   dQ_i    = dS_i K_i / sqrt(d),  dK_i = dS_i^T Q_i / sqrt(d)
//   dlambda = (dc/dlambda) <G, A_2 V>,  dw = sum over rows of g r O dy
//
// Five launches:
//   1. the tcgen05 prefill in its statistics mode: per map, A_i V (float32)
//      and the log-sum-exp of every query row;
//   2. prep (CUDA cores, one warp per row): G (rounded to bf16 for the tensor
//      cores), D_1, D_2, and the dw / dlambda sums;
//   3-5. three tcgen05 gradient kernels, one 128-row block per CTA:
//        dV  rows = keys:    S_i^T = K_i Q_i^T,  dV += (P_1 + c P_2)^T G
//        dK  rows = keys:    S_i^T, dP^T = V G^T, dK_i += dS_i^T Q_i
//        dQ  rows = queries: S_i, dP = G V^T,     dQ_i += dS_i K_i
//      The row operands stay in shared memory; column tiles of the other side
//      (32 columns for dK and dQ, 64 for dV) stream through a TMA ring.  S (and dP) land in tensor memory;
//      four softmax warps turn them into P or dS, store them back into
//      tensor memory as bf16, and the gradient product reads them from
//      there as its A operand (tcgen05.mma with A in tensor memory).  The
//      gradient accumulates in tensor memory across all column tiles and
//      is written once, as float32.
// Compared with one fused kernel per key block (dK, dV) plus atomics for dQ,
// this recomputes the scores three times (20d algorithmic flops per visible
// pair become 32d executed), but every accumulator fits in the 512 columns
// of tensor memory and every gradient is written once, without atomics.
#include <cuda_bf16.h>
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace diffattn {

namespace {

constexpr int kGradThreads = 256;
constexpr int kRowTile = 128;  // rows of a gradient block (keys for dK and dV, queries for dQ)
constexpr float kLog2eBwd = 1.4426950408889634f;

enum : int { kGradV = 0, kGradK = 1, kGradQ = 2 };

template <int D, int KIND>
struct GCfg {
  static constexpr int DV = 2 * D;
  static constexpr bool HAS_DP = KIND != kGradV;   // dK and dQ need dP = G V^T
  static constexpr bool COL_STATS = KIND != kGradQ;  // statistics belong to the columns (queries)
  static constexpr int QKB = D / 64;               // 128-byte boxes per Q / K row
  static constexpr int VGB = DV / 64;              // 128-byte boxes per V / G row
  static constexpr int RBOX = kRowTile * 128;      // [128 rows][128 bytes]
  // Streamed columns per tile: 64 for dV (one S buffer; its S products are N = 64
  // instructions, half as many as at N = 32 for the same columns), 32 for dK and
  // dQ (two S buffers: S, dP and dS of two tiles share the 256 free columns).
  static constexpr int NC = HAS_DP ? 32 : 64;
  static constexpr int NSB = HAS_DP ? 2 : 1;  // S buffers in tensor memory
  static constexpr int CBOX = NC * 128;       // [NC rows][128 bytes]
  // resident rows: both maps' K (dV, dK) or Q (dQ), then V (dK) or G (dQ)
  static constexpr int R_QK = 2 * QKB * RBOX;
  static constexpr int R_BYTES = R_QK + (HAS_DP ? VGB * RBOX : 0);
  // one column stage: both maps' Q (dV, dK) or K (dQ), then G (dV, dK) or V (dQ)
  static constexpr int C_QK = 2 * QKB * CBOX;
  static constexpr int C_BYTES = C_QK + VGB * CBOX;
  static constexpr int ST_BYTES = NC * 16;  // one float4 of statistics per column
  static constexpr int STAGES = HAS_DP ? 3 : 2;
  static constexpr int OFF_R = 0;
  static constexpr int OFF_C = R_BYTES;
  static constexpr int OFF_ST = OFF_C + STAGES * C_BYTES;
  static constexpr int OFF_BAR = OFF_ST + STAGES * ST_BYTES;
  static constexpr int SMEM_USED = OFF_BAR + 256;
  // slack for 1024-byte alignment, and at least 116 KB: one CTA per SM, so
  // that no CTA waits in its allocation of all 512 tensor-memory columns
  static constexpr int SMEM_ALLOC = (SMEM_USED + 1024 > 116 * 1024) ? SMEM_USED + 1024 : 116 * 1024;
  // tensor memory: the accumulator, then two tile buffers of 128 columns
  static constexpr uint32_t TM_ACC = 0;  // dV (2d columns) or both maps' dK / dQ (d columns each)
  // dK, dQ: two buffers of 128 columns at TM_BUF + 128 b: S_1 | S_2 | dP (float32,
  // 32 columns each) | dS_1 | dS_2 (bf16 pairs, 16 columns each).
  // dV: one S buffer at TM_BUF: S_1 | S_2 (64 columns each); two P buffers of 32
  // columns (bf16 pairs) at TM_BUF + 128 + 32 b.
  static constexpr uint32_t TM_BUF = 256;
  static constexpr uint32_t B_S1 = 0, B_S2 = NC, B_DP = 64;
  static constexpr uint32_t B_A1 = 96, B_A2 = 112;
  __device__ static uint32_t s_buf(int t) { return TM_BUF + (NSB == 2 ? 128u * (t & 1) : 0u); }
  __device__ static uint32_t a_buf(int t) { return NSB == 2 ? s_buf(t) + B_A1 : TM_BUF + 2 * NC + (NC / 2) * (t & 1); }
  static constexpr uint32_t TM_COLS = 512;
  static_assert(R_BYTES % 1024 == 0 && C_BYTES % 1024 == 0, "operand tiles keep 1024-byte alignment");
  static_assert(HAS_DP || TM_BUF + 2 * NC + NC <= 512, "dV's tensor memory: dV, one S buffer, two P buffers");
  static_assert(SMEM_ALLOC <= 232448, "shared memory per CTA");
};

struct GradBars {
  uint64_t r_full;  // the resident rows have landed
  uint64_t c_full[4], c_empty[4];
  uint64_t s_full[2];  // S (and dP) of the tile in S buffer b are in tensor memory
  uint64_t s_free[2];  // the softmax warps have read them (dV: buffer 0 only)
  uint64_t a_full[2];  // P or dS of the tile is in tensor memory (bf16)
  uint64_t acc_done;   // the last gradient product has completed
  uint32_t tmem_base;
  int abort;
};

struct GradParams {
  int B, N, H, causal;
  int n_rtiles, n_pad;
  const float* lambda;
  int mode;
  const float4* stats;  // [B][H][n_pad]: lse_1, lse_2 (scaled log2 units), D_1, D_2
  float* out;           // dV [B, N, H, 2d], or dK / dQ [B, N, H, 2, d]
  int* status;
  unsigned long long limit_ns;
};

template <int D, int KIND>
__global__ void __launch_bounds__(kGradThreads, 1)
    bwd_grad_sm100_kernel(const __grid_constant__ CUtensorMap t_rqk, const __grid_constant__ CUtensorMap t_rvg,
                          const __grid_constant__ CUtensorMap t_cqk, const __grid_constant__ CUtensorMap t_cvg,
                          const GradParams p) {
  using C = GCfg<D, KIND>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sR = smem + C::OFF_R;
  uint8_t* sC = smem + C::OFF_C;
  uint8_t* sST = smem + C::OFF_ST;
  GradBars* bars = reinterpret_cast<GradBars*>(smem + C::OFF_BAR);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int N = p.N;
  // block -> (batch, head, row tile): heads in order, and within a head the
  // row tiles with the most columns first
  const int bh = static_cast<int>(blockIdx.x) / p.n_rtiles;
  const int li = static_cast<int>(blockIdx.x) % p.n_rtiles;
  const int rt = (KIND == kGradQ) ? p.n_rtiles - 1 - li : li;
  const int b = bh / p.H, h = bh % p.H;
  const int row0 = rt * kRowTile;
  constexpr int NC = C::NC;
  const int n_ctiles = (N + NC - 1) / NC;
  int c_begin = 0, c_end = n_ctiles;
  if (p.causal) {
    if (KIND == kGradQ)
      c_end = min(n_ctiles, (row0 + kRowTile) / NC);  // keys <= the block's last query
    else
      c_begin = row0 / NC;  // queries >= the block's first key
  }
  const int T = c_end - c_begin;  // >= 1: row0 < N

  if (tid == 0) {
    mbar_init(&bars->r_full, 1);
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(&bars->c_full[i], 1);
      mbar_init(&bars->c_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->s_free[i], 4);  // one arrival per softmax warp
      mbar_init(&bars->a_full[i], 4);
    }
    mbar_init(&bars->acc_done, 1);
    bars->abort = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&t_rqk);
    tma_prefetch_desc(&t_cqk);
    tma_prefetch_desc(&t_cvg);
    if (C::HAS_DP) tma_prefetch_desc(&t_rvg);
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, C::TM_COLS);
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
      // debug builds: the block's rows lie in the tensors
      (void)DA_CHECK(p.status, b < p.B && h < p.H && row0 < N);
      mbar_arrive_expect_tx(&bars->r_full, C::R_BYTES);
#pragma unroll
      for (int m = 0; m < 2; ++m)
#pragma unroll
        for (int blk = 0; blk < C::QKB; ++blk)
          tma_load_4d(sR + (m * C::QKB + blk) * C::RBOX, &t_rqk, &bars->r_full, blk * 64, 2 * h + m, row0, b);
      if constexpr (C::HAS_DP) {
#pragma unroll
        for (int blk = 0; blk < C::VGB; ++blk)
          tma_load_4d(sR + C::R_QK + blk * C::RBOX, &t_rvg, &bars->r_full, blk * 64, h, row0, b);
      }
      int t = 0;
      for (; t < T; ++t) {
        const int st = t % C::STAGES;
        if (!mbar_wait(&bars->c_empty[st], ((t / C::STAGES) & 1) ^ 1, wc)) break;
        const int c0 = (c_begin + t) * NC;
        // debug builds: the column tile starts inside the tensors, and its
        // statistics (an untiled copy, which nothing else bounds) lie in the
        // [B][H][n_pad] array; when they do not, they are not copied
        (void)DA_CHECK(p.status, c0 < N);
        const bool st_ok = !C::COL_STATS || DA_CHECK(p.status, c0 + NC <= p.n_pad && bh < p.B * p.H);
        mbar_arrive_expect_tx(&bars->c_full[st], C::C_BYTES + (C::COL_STATS && st_ok ? C::ST_BYTES : 0));
        uint8_t* base = sC + st * C::C_BYTES;
#pragma unroll
        for (int m = 0; m < 2; ++m)
#pragma unroll
          for (int blk = 0; blk < C::QKB; ++blk)
            tma_load_4d(base + (m * C::QKB + blk) * C::CBOX, &t_cqk, &bars->c_full[st], blk * 64, 2 * h + m, c0, b);
#pragma unroll
        for (int blk = 0; blk < C::VGB; ++blk)
          tma_load_4d(base + C::C_QK + blk * C::CBOX, &t_cvg, &bars->c_full[st], blk * 64, h, c0, b);
        if (C::COL_STATS && st_ok)
          bulk_load_g2s(sST + st * C::ST_BYTES, p.stats + static_cast<size_t>(bh) * p.n_pad + c0, C::ST_BYTES,
                        &bars->c_full[st]);
      }
      // nothing may still be landing in shared memory when the CTA exits
      mbar_wait(&bars->r_full, 0, wdrain);
      for (int j = max(0, t - C::STAGES); j < t; ++j)
        mbar_wait(&bars->c_full[j % C::STAGES], (j / C::STAGES) & 1, wdrain);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, NC, false, false);
      constexpr uint32_t idesc_g = idesc_bf16_f32(128, KIND == kGradV ? C::DV : D, false, true);
      const uint32_t sRa = smem_u32(sR), sCa = smem_u32(sC);
      // Descriptors are built once and advanced by adding (offset >> 4) to
      // their address field: the issue queue holds about one instruction, so
      // address arithmetic between two products would delay the second.
      const uint64_t a_desc = smem_desc_sw128(sRa, 16, 1024);
      const uint64_t c_desc = smem_desc_sw128(sCa, 16, 1024);             // K-major column tiles
      const uint64_t c_desc_mn = smem_desc_sw128(sCa, C::CBOX, 1024);     // the same tiles read MN-major
      auto adv = [](uint64_t desc, uint32_t bytes) { return desc + static_cast<uint64_t>(bytes >> 4); };
      bool ok = mbar_wait(&bars->r_full, 0, wc);
      // S of tile i is issued before the gradient product of tile i - 1, so
      // that the tensor core works on tile i while the softmax warps turn
      // tile i - 1's scores into P or dS.
      for (int i = 0; ok && i <= T; ++i) {
        if (i < T) {
          const int bb = (C::NSB == 2) ? (i & 1) : 0, st = i % C::STAGES;
          // S_i overwrites the scores of tile i - NSB: the softmax warps must have read them
          if (i >= C::NSB) {
            const int jj = i - C::NSB;
            const uint32_t ph = (C::NSB == 2) ? ((jj >> 1) & 1) : (jj & 1);
            if (!(ok = mbar_wait(&bars->s_free[bb], ph, wc))) break;
          }
          if (!(ok = mbar_wait(&bars->c_full[st], (i / C::STAGES) & 1, wc))) break;
          tc_fence_after();
          const uint32_t tb = tmem + C::s_buf(i);
          const uint64_t cd = adv(c_desc, st * C::C_BYTES);
#pragma unroll
          for (int m = 0; m < 2; ++m) {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t blk = kk >> 2, koff = (kk & 3) * 32;
              umma_ss(tb + (m ? C::B_S2 : C::B_S1), adv(a_desc, (m * C::QKB + blk) * C::RBOX + koff),
                      adv(cd, (m * C::QKB + blk) * C::CBOX + koff), idesc_s, kk > 0 ? 1u : 0u);
            }
          }
          if constexpr (C::HAS_DP) {
#pragma unroll
            for (int kk = 0; kk < C::DV / 16; ++kk) {
              const uint32_t blk = kk >> 2, koff = (kk & 3) * 32;
              umma_ss(tb + C::B_DP, adv(a_desc, C::R_QK + blk * C::RBOX + koff), adv(cd, C::C_QK + blk * C::CBOX + koff),
                      idesc_s, kk > 0 ? 1u : 0u);
            }
          }
          umma_commit(&bars->s_full[bb]);
        }
        if (i >= 1) {
          const int j = i - 1, bj = j & 1, stj = j % C::STAGES;
          if (!(ok = mbar_wait(&bars->a_full[bj], (j >> 1) & 1, wc))) break;
          tc_fence_after();
          const uint32_t ta = tmem + C::a_buf(j);
          const uint64_t cd = adv(c_desc_mn, stj * C::C_BYTES);
          // B operands: the stage's rows [NC][width] read MN-major (K = the NC columns)
          if constexpr (KIND == kGradV) {
#pragma unroll
            for (int kk = 0; kk < NC / 16; ++kk)
              umma_ts(tmem + C::TM_ACC, ta + 8 * kk, adv(cd, C::C_QK + kk * 2048), idesc_g, (j > 0 || kk > 0) ? 1u : 0u);
          } else {
#pragma unroll
            for (int m = 0; m < 2; ++m) {
#pragma unroll
              for (int kk = 0; kk < NC / 16; ++kk)
                umma_ts(tmem + C::TM_ACC + m * D, ta + (m ? C::B_A2 - C::B_A1 : 0u) + 8 * kk,
                        adv(cd, m * C::QKB * C::CBOX + kk * 2048), idesc_g, (j > 0 || kk > 0) ? 1u : 0u);
            }
          }
          umma_commit(&bars->c_empty[stj]);  // S_j and the gradient product of tile j have read the stage
        }
      }
      umma_commit(&bars->acc_done);  // arrives once every MMA issued above has completed
      mbar_wait(&bars->acc_done, 0, wdrain);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // --------------------------------------------------- softmax + store --
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // row within the block (= TMEM lane)
    const int grow = row0 + r;
    const uint32_t tl = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const float sc = kLog2eBwd * rsqrtf(static_cast<float>(D));
    const float coef = map2_coefficient(p.mode, *p.lambda);
    float4 rs = make_float4(0.f, 0.f, 0.f, 0.f);  // dQ: this query row's statistics
    if (KIND == kGradQ && grow < N) rs = p.stats[static_cast<size_t>(bh) * p.n_pad + grow];
    const float4* stv = reinterpret_cast<const float4*>(sST);
    bool ok = true;
    for (int t = 0; t < T; ++t) {
      const int st = t % C::STAGES;
      const int sb = (C::NSB == 2) ? (t & 1) : 0;
      const uint32_t sph = (C::NSB == 2) ? ((t >> 1) & 1) : (t & 1);
      if (!(ok = mbar_wait(&bars->s_full[sb], sph, wc))) break;
      if constexpr (C::COL_STATS) {  // the stage's statistics (bulk copy) are visible after this wait
        if (!(ok = mbar_wait(&bars->c_full[st], (t / C::STAGES) & 1, wc))) break;
      }
      tc_fence_after();
      const uint32_t tb = tl + C::s_buf(t);
      uint32_t s1[NC], s2[NC], dp[C::HAS_DP ? NC : 1];
      auto chunk = [](uint32_t* a, int h) -> uint32_t(&)[32] { return *reinterpret_cast<uint32_t(*)[32]>(a + 32 * h); };
#pragma unroll
      for (int h = 0; h < NC / 32; ++h) {
        tmem_ld32(tb + C::B_S1 + 32 * h, chunk(s1, h));
        tmem_ld32(tb + C::B_S2 + 32 * h, chunk(s2, h));
        if constexpr (C::HAS_DP) tmem_ld32(tb + C::B_DP + 32 * h, chunk(dp, h));
      }
#pragma unroll
      for (int h = 0; h < NC / 32; ++h) {  // one wait; these only order the registers behind it
        tmem_ld_wait(chunk(s1, h));
        tmem_ld_wait(chunk(s2, h));
        if constexpr (C::HAS_DP) tmem_ld_wait(chunk(dp, h));
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->s_free[sb]);

      const int c0 = (c_begin + t) * NC;
      bool masked = c0 + NC > N;
      if (p.causal) masked = masked || (KIND == kGradQ ? (c0 + NC - 1 > row0) : (c0 < row0 + kRowTile - 1));
      uint32_t a1[NC / 2], a2[NC / 2];
#pragma unroll
      for (int c2 = 0; c2 < NC / 2; ++c2) {
        float v1[2], v2[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int c = 2 * c2 + e;
          const float4 sv = C::COL_STATS ? stv[st * NC + c] : rs;
          const float p1 = fast_exp2(fmaf(__uint_as_float(s1[c]), sc, -sv.x));
          const float p2 = fast_exp2(fmaf(__uint_as_float(s2[c]), sc, -sv.y));
          if constexpr (KIND == kGradV) {
            v1[e] = fmaf(coef, p2, p1);
          } else {
            const float g = __uint_as_float(dp[c]);
            v1[e] = p1 * (g - sv.z);
            v2[e] = p2 * fmaf(coef, g, -sv.w);
          }
          if (masked) {  // selects, not products: statistics past the last row are not initialised
            const int col = c0 + c;
            const bool vis = col < N && (!p.causal || (KIND == kGradQ ? col <= grow : grow <= col));
            v1[e] = vis ? v1[e] : 0.f;
            if constexpr (KIND != kGradV) v2[e] = vis ? v2[e] : 0.f;
          }
        }
        a1[c2] = pack_bf16x2(v1[0], v1[1]);
        if constexpr (KIND != kGradV) a2[c2] = pack_bf16x2(v2[0], v2[1]);
      }
      // P / dS buffer t & 1 was last read by the gradient product of tile t - 2,
      // issued before S_t: the s_full wait above covers its completion
      const uint32_t ta = tl + C::a_buf(t);
      if constexpr (NC == 64) {
        tmem_st32(ta, a1);
      } else {
        tmem_st16(ta, a1);
        if constexpr (KIND != kGradV) tmem_st16(ta + (C::B_A2 - C::B_A1), a2);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->a_full[t & 1]);
    }

    // ------------------------------------------------------- epilogue --
    mbar_wait(&bars->acc_done, 0, wdrain);
    tc_fence_after();
    const bool live = grow < N && DA_CHECK(p.status, b < p.B && h < p.H);
    const float scale = (KIND == kGradV) ? 1.0f : rsqrtf(static_cast<float>(D));
    // dV row [2d], or both maps' rows [2][d]: 2d contiguous floats either way
    float* orow = p.out + ((static_cast<size_t>(b) * N + (live ? grow : 0)) * p.H + h) * C::DV;
#pragma unroll 1
    for (int c = 0; c < C::DV / 32; ++c) {
      uint32_t ov[32];
      tmem_ld32_sync(tl + C::TM_ACC + 32 * c, ov);
      if (live) {
#pragma unroll
        for (int f = 0; f < 8; ++f)
          *reinterpret_cast<float4*>(orow + 32 * c + 4 * f) =
              make_float4(__uint_as_float(ov[4 * f + 0]) * scale, __uint_as_float(ov[4 * f + 1]) * scale,
                          __uint_as_float(ov[4 * f + 2]) * scale, __uint_as_float(ov[4 * f + 3]) * scale);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TM_COLS);
  }
}

// ---------------------------------------------------------------- prep --
// One warp per (batch, token, head) row: O = O_1 + c O_2 from the
// statistics pass, the RMSNorm backward G, D_1 = G . O_1 and D_2 = c G . O_2
// (with G rounded to bf16, as the tensor cores see it), and per-CTA sums of
// dw and dlambda added to the outputs at the end.
template <int D>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const float* __restrict__ o_maps,
                                                       const __nv_bfloat16* __restrict__ dy,
                                                       const float* __restrict__ rms_w,
                                                       const float* __restrict__ lambda_ptr, int mode, float dcoef,
                                                       float lambda_init, float eps, int B, int N, int H, int n_pad,
                                                       __nv_bfloat16* __restrict__ G, float4* __restrict__ stats,
                                                       float* __restrict__ dlambda, float* __restrict__ drms_w,
                                                       int* dbg) {
  constexpr int DV = 2 * D;
  constexpr int E = DV / 32;  // columns per lane, contiguous
  __shared__ float s_dw[8][DV];
  __shared__ float s_dl[8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float coef = map2_coefficient(mode, *lambda_ptr);
  const float g = 1.0f - lambda_init;
  float w[E], dw[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    w[e] = __ldg(rms_w + lane * E + e);
    dw[e] = 0.f;
  }
  float dl = 0.f;
  const long long rows = static_cast<long long>(B) * N * H;
  for (long long row = static_cast<long long>(blockIdx.x) * 8 + warp; row < rows;
       row += static_cast<long long>(gridDim.x) * 8) {
    const float* o1p = o_maps + row * 2 * DV + lane * E;
    const float* o2p = o1p + DV;
    float o1[E], o2[E], y[E], o[E];
#pragma unroll
    for (int e = 0; e < E; e += 4) {
      const float4 a = *reinterpret_cast<const float4*>(o1p + e);
      const float4 c = *reinterpret_cast<const float4*>(o2p + e);
      o1[e] = a.x, o1[e + 1] = a.y, o1[e + 2] = a.z, o1[e + 3] = a.w;
      o2[e] = c.x, o2[e + 1] = c.y, o2[e + 2] = c.z, o2[e + 3] = c.w;
    }
    const __nv_bfloat16* dyp = dy + row * DV + lane * E;
#pragma unroll
    for (int e = 0; e < E; e += 4) {
      const uint2 u = *reinterpret_cast<const uint2*>(dyp + e);
      y[e] = bf16lo_to_f32(u.x), y[e + 1] = bf16hi_to_f32(u.x);
      y[e + 2] = bf16lo_to_f32(u.y), y[e + 3] = bf16hi_to_f32(u.y);
    }
    float ss = 0.f, t = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      o[e] = fmaf(coef, o2[e], o1[e]);
      ss = fmaf(o[e], o[e], ss);
      t = fmaf(w[e] * y[e], o[e], t);
    }
#pragma unroll
    for (int s = 16; s >= 1; s >>= 1) {
      ss += __shfl_xor_sync(0xffffffffu, ss, s);
      t += __shfl_xor_sync(0xffffffffu, t, s);
    }
    const float r = rsqrtf(ss / DV + eps);
    const float gr = g * r;
    const float k3 = gr * r * r * t / DV;
    float d1 = 0.f, d2 = 0.f;
    uint32_t pk[E / 2];
#pragma unroll
    for (int e = 0; e < E; e += 2) {
      const float ga = fmaf(gr * w[e], y[e], -o[e] * k3);
      const float gb = fmaf(gr * w[e + 1], y[e + 1], -o[e + 1] * k3);
      dw[e] = fmaf(gr * o[e], y[e], dw[e]);
      dw[e + 1] = fmaf(gr * o[e + 1], y[e + 1], dw[e + 1]);
      dl = fmaf(ga, o2[e], fmaf(gb, o2[e + 1], dl));
      pk[e / 2] = pack_bf16x2(ga, gb);
      const float ra = bf16lo_to_f32(pk[e / 2]), rb = bf16hi_to_f32(pk[e / 2]);
      d1 = fmaf(ra, o1[e], fmaf(rb, o1[e + 1], d1));
      d2 = fmaf(ra, o2[e], fmaf(rb, o2[e + 1], d2));
    }
    uint32_t* gp = reinterpret_cast<uint32_t*>(G + row * DV + lane * E);
#pragma unroll
    for (int e = 0; e < E / 2; e += 2) *reinterpret_cast<uint2*>(gp + e) = make_uint2(pk[e], pk[e + 1]);
#pragma unroll
    for (int s = 16; s >= 1; s >>= 1) {
      d1 += __shfl_xor_sync(0xffffffffu, d1, s);
      d2 += __shfl_xor_sync(0xffffffffu, d2, s);
    }
    if (lane == 0 && DA_CHECK(dbg, row / H / N < B)) {
      const long long hh = row % H, bn = row / H;
      const long long n = bn % N, bb = bn / N;
      float* sp = reinterpret_cast<float*>(stats + (bb * H + hh) * n_pad + n);
      *reinterpret_cast<float2*>(sp + 2) = make_float2(d1, coef * d2);
    }
  }
#pragma unroll
  for (int e = 0; e < E; ++e) s_dw[warp][lane * E + e] = dw[e];
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) dl += __shfl_xor_sync(0xffffffffu, dl, s);
  if (lane == 0) s_dl[warp] = dl;
  __syncthreads();
  for (int c = threadIdx.x; c < DV; c += 256) {
    float a = 0.f;
#pragma unroll
    for (int w8 = 0; w8 < 8; ++w8) a += s_dw[w8][c];
    atomicAdd(drms_w + c, a);
  }
  if (threadIdx.x == 0) {
    float a = 0.f;
#pragma unroll
    for (int w8 = 0; w8 < 8; ++w8) a += s_dl[w8];
    atomicAdd(dlambda, dcoef * a);
  }
}

template <int D, int KIND>
cudaError_t launch_grad(const CUtensorMap& t_rqk, const CUtensorMap& t_rvg, const CUtensorMap& t_cqk,
                        const CUtensorMap& t_cvg, const GradParams& prm, cudaStream_t stream) {
  using C = GCfg<D, KIND>;
  cudaError_t e = cudaFuncSetAttribute(bwd_grad_sm100_kernel<D, KIND>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::SMEM_ALLOC);
  if (e != cudaSuccess) return e;
  const unsigned grid = static_cast<unsigned>(prm.B * prm.H * prm.n_rtiles);
  bwd_grad_sm100_kernel<D, KIND><<<grid, kGradThreads, C::SMEM_ALLOC, stream>>>(t_rqk, t_rvg, t_cqk, t_cvg, prm);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_bwd_sm100_d(const BwdTcMaps& m, const void* dy, int B, int N, int H, int causal,
                               const float* lambda, float lambda_init, const float* rms_w, float eps, int mode,
                               float* dq, float* dk, float* dv, float* dlambda, float* drms_w, void* workspace,
                               bool stats_ready, DevCtl ctl, cudaStream_t stream) {
  const BwdTcLayout L = bwd_tc_layout(B, N, H, D);
  char* ws = static_cast<char*>(workspace);
  float* o_maps = reinterpret_cast<float*>(ws + L.off_omaps);
  __nv_bfloat16* G = reinterpret_cast<__nv_bfloat16*>(ws + L.off_g);
  float4* stats = reinterpret_cast<float4*>(ws + L.off_stats);
  cudaError_t e = cudaMemsetAsync(drms_w, 0, sizeof(float) * 2 * D, stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(dlambda, 0, sizeof(float), stream);
  if (e != cudaSuccess) return e;
  if (!stats_ready) {
    e = launch_prefill_sm100_stats(m.q128, m.k128, m.v128, nullptr, nullptr, B, N, H, D, causal, lambda, lambda_init,
                                   rms_w, eps, mode, o_maps, reinterpret_cast<float*>(stats), L.n_pad, ctl, stream);
    if (e != cudaSuccess) return e;
  }
  const long long rows = static_cast<long long>(B) * N * H;
  const long long want = (rows + 7) / 8;
  const int grid = static_cast<int>(want < 148 * 16 ? want : 148 * 16);
  const float dcoef = mode == 0 ? -1.0f : (mode == 2 ? 1.0f : 0.0f);
  bwd_prep_kernel<D><<<grid, 256, 0, stream>>>(o_maps, static_cast<const __nv_bfloat16*>(dy), rms_w, lambda, mode,
                                               dcoef, lambda_init, eps, B, N, H, L.n_pad, G, stats, dlambda,
                                               drms_w, debug_status());
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  GradParams prm = {};
  prm.B = B;
  prm.N = N;
  prm.H = H;
  prm.causal = causal ? 1 : 0;
  prm.n_rtiles = (N + kRowTile - 1) / kRowTile;
  prm.n_pad = L.n_pad;
  prm.lambda = lambda;
  prm.mode = mode;
  prm.stats = stats;
  prm.status = ctl.status;
  prm.limit_ns = ctl.limit_ns;
  prm.out = dv;
  e = launch_grad<D, kGradV>(m.k128, m.k128, m.q64, m.g64, prm, stream);
  if (e != cudaSuccess) return e;
  prm.out = dk;
  e = launch_grad<D, kGradK>(m.k128, m.v128, m.q32, m.g32, prm, stream);
  if (e != cudaSuccess) return e;
  prm.out = dq;
  return launch_grad<D, kGradQ>(m.q128, m.g128, m.k32, m.v32, prm, stream);
}

}  // namespace

BwdTcLayout bwd_tc_layout(int B, int N, int H, int d) {
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  BwdTcLayout L;
  const size_t rows = static_cast<size_t>(B) * N * H;
  L.n_pad = (N + kRowTile - 1) / kRowTile * kRowTile;
  L.off_omaps = 0;
  L.off_g = up(sizeof(float) * rows * 2 * 2 * d);
  L.off_stats = L.off_g + up(2 * rows * 2 * d);
  L.bytes = L.off_stats + up(16 * static_cast<size_t>(B) * H * L.n_pad);
  return L;
}

cudaError_t launch_bwd_sm100(const BwdTcMaps& m, const void* dy, int B, int N, int H, int d, int causal,
                             const float* lambda, float lambda_init, const float* rms_w, float eps, int mode,
                             float* dq, float* dk, float* dv, float* dlambda, float* drms_w, void* workspace,
                             bool stats_ready, DevCtl ctl, cudaStream_t stream) {
  if (d == 128)
    return launch_bwd_sm100_d<128>(m, dy, B, N, H, causal, lambda, lambda_init, rms_w, eps, mode, dq, dk, dv,
                                   dlambda, drms_w, workspace, stats_ready, ctl, stream);
  if (d == 64)
    return launch_bwd_sm100_d<64>(m, dy, B, N, H, causal, lambda, lambda_init, rms_w, eps, mode, dq, dk, dv,
                                  dlambda, drms_w, workspace, stats_ready, ctl, stream);
  return cudaErrorInvalidValue;
}

}  // namespace diffattn
