// Fused dual-map differential-attention prefill for sm_100a (bf16 in, fp32
// accumulate, bf16 out), d in {64, 128}.
//
// Computes, per head, the DiffAttn equation (page "Differential Transformer:
// Canceling Context Noise with Differential Attention", "Cancelling Context
// Noise Through Attention Map Subtraction"; peer review "Differential
// Transformer", Summary, Eq. 1), then the headwise RMSNorm over the 2d value
// channels and the fixed (1 - lambda_init) scale (Eq. 3).  No N x N map is
// ever written to memory.
//
// Work decomposition
//   Persistent clusters of two CTAs.  An item is one 128-row query tile of one
//   (batch, head).  The (batch, head) pairs are taken in groups whose K and V
//   fit in about 48 MB of L2 together; within a group the items are ordered
//   longest first (causal: the last query tiles); the whole list is dealt to
//   the clusters in a snake.  Per item, CTA rank i
//   computes map i+1 only: S_i = Q_i K_i^T on the tensor cores,
//   its own online softmax (running max m_i and sum l_i per row), and
//   O_i += P_i V.  Both CTAs stream the same V tiles.  Tensor memory per CTA
//   (512 columns): S (fp32, one buffer) in columns [0, 128), P (bf16, two
//   buffers of 64 columns) in [128, 256), O_i in [256, 256 + 2d).  P feeds
//   the PV product straight from tensor memory.  Keeping P apart from S lets
//   S_{j+1} be computed as soon as the softmax has read S_j into registers.
//   The epilogue exchanges half of the columns through distributed shared
//   memory: rank 0 keeps output columns [0, d), rank 1 keeps [d, 2d); each
//   bulk-copies the other half of its O_i/l_i (scaled by -lambda on rank 1)
//   into the partner's shared memory, the partial sums of squares of each
//   row are swapped, and each CTA stages its columns of
//   (1 - lambda_init) * w * O / rms as bf16 and writes them with TMA stores.
//   The two CTAs meet through mbarriers only (each side says when its
//   receive buffer is free, the copies complete on the receiver's barrier,
//   and so do the sums of squares, sent with st.async), so the producer and
//   MMA threads run on into the next item: its Q and K tiles load and its
//   first S product runs while the epilogue finishes.  Warp 3 stores each
//   output tile, so the softmax warps start the next item as soon as the tile
//   is staged.
//
// Warp roles (256 threads)
//   warp 0: TMA producer for Q_i and K_i      warp 2: TMA producer for V
//   warp 1: tensor-memory allocator + the single MMA-issuing thread
//   warp 3: TMA store of each output tile     warps 4-7: softmax + epilogue,
//                                             one query row per thread
//
// Pipeline per key tile j (P buffer and K/V stage b = j % 2).  A
// tcgen05.mma issue returns only when the instruction is nearly done, so the
// issue order decides what overlaps:
//   MMA:     wait s_free (the softmax has read S_{j-1}) -> S_j -> commit
//            s_full, k_empty; then wait p_full[b'] of tile j-1 ->
//            O += P_{j-1} V_{j-1} -> commit v_empty, p_empty[b'].  PV_{j-1}
//            thus runs while the softmax works on tile j, and S_{j+1} is
//            ready when the softmax finishes it.
//   softmax: wait s_full (S_j done, and so every MMA issued before it:
//            PV_{j-2}, the last reader of P[b]); read the 128 scores of its
//            row; arrive s_free; mask; P = exp2(s*c - m) as bf16 into P[b],
//            relative to the reference maximum m, while forming the tile's
//            own maximum; arrive p_full[b].  Lazy rescale: only when the
//            running maximum exceeds m by more than 2^8 are O and l rescaled
//            to it, once PV_j has completed; a jump beyond 2^64, which could
//            overflow P, rescales first and recomputes P.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace diffattn {

namespace {

constexpr int kThreads = 256;
constexpr int kBM = 128;  // query rows per CTA
constexpr int kBN = 128;  // keys per tile
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr float kOverflowGuard = 64.0f;    // log2 units

// QK8: queries and keys arrive as low-bit codes with a float32 scale per
// (batch, head, map) and S is a kind::f8f6f4 product: e4m3 codes take one
// byte each; e2m1 codes come packed two per byte and the tensor map
// (16U4_ALIGN16B) widens every 8 bytes of them to 16 in shared memory, so both
// formats leave one byte of shared memory per element.  Otherwise they are
// bf16 and S is a kind::f16 product.
template <int D, bool QK8>
struct Cfg {
  static constexpr int DV = 2 * D;
  static constexpr int HALF = D;                 // output columns owned by each CTA
  static constexpr int QE = QK8 ? 1 : 2;         // bytes per Q/K element
  static constexpr int QBOX = 128 / QE;          // Q/K elements per 128-byte swizzle row
  static constexpr int QBLK = D / QBOX;          // 128-byte swizzle blocks per Q/K row
  static constexpr int KSTEP = QK8 ? 32 : 16;    // K of one S instruction
  static constexpr int VBLK = DV / 64;           // 64-column blocks per V row
  static constexpr int BLK_BYTES = 128 * 128;    // one [128 rows][128 bytes] block
  static constexpr int Q_BYTES = kBM * D * QE;
  static constexpr int K_BYTES = kBN * D * QE;
  static constexpr int V_BYTES = kBN * DV * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + 2 * K_BYTES;
  static constexpr int OFF_BAR = OFF_V + 2 * V_BYTES;
  static constexpr int OFF_SSX = OFF_BAR + 256;  // float[128]: the partner's sums of squares
  static constexpr int SMEM_USED = OFF_SSX + 512;
  static constexpr int EXCH_BYTES = kBM * HALF * 4;
  static constexpr int SMEM_ALLOC = SMEM_USED + 1024;  // slack for 1024-byte alignment
  static constexpr uint32_t TM_S = 0;            // S (fp32, 128 columns)
  static constexpr uint32_t TM_P = 128;          // P buffer b (bf16 pairs) at column TM_P + 64 * b
  static constexpr uint32_t TM_O = 256;
  static constexpr uint32_t TM_COLS = 512;
  static_assert(EXCH_BYTES <= V_BYTES, "exchange buffers must fit in one V stage each");
  static_assert(kBM * HALF * 2 <= V_BYTES, "output staging must fit in one V stage");
  static_assert(SMEM_USED + 1024 <= 232448, "shared memory per CTA");

};

struct Bars {
  uint64_t q_full, q_empty;  // per item; q_empty: the item's last S product has read Q
  uint64_t k_full[2], k_empty[2];
  uint64_t v_full[2], v_empty[2];
  uint64_t s_full, s_free;
  uint64_t p_full[2], p_empty[2];
  uint64_t mma_done;
  uint64_t exch_full;   // per item: the partner's half of the output has landed here
  uint64_t peer_ready;  // per item: the partner's receive buffer is free (remote arrive)
  uint64_t ss_full;     // per item: the partner's sums of squares are here (remote arrive)
  uint64_t epi_free;    // per item: the epilogue is done with the V stages
  uint32_t tmem_base;
  int abort;
};

}  // namespace

struct PrefillParams {
  __nv_bfloat16* o;
  int N, H, B, causal, n_qtiles;
  int n_items;     // B * H * n_qtiles
  int head_group;  // (batch, head) pairs per item group (K and V of a group stay in L2)
  const float* lambda;
  const float* q_scale;  // QK8 only: float32 [B][H][2], one scale per (batch, head, map)
  const float* k_scale;
  int mode;  // diffattn_mode: how map 2 enters the combination
  float lambda_init;
  const float* rms_w;
  float eps;
  int* status;
  unsigned long long limit_ns;
  // statistics mode (the backward pass's forward): per map, O_i / l_i and the log-sum-exp
  float* o_maps;  // float32 [B, N, H, 2, 2d]
  float* lse;     // float32 view of float4 [B][H][n_pad]: component i = map i's log2-sum-exp
  int n_pad;
};

// Wait for every tcgen05.ld issued so far and pin 128 registers behind the wait.
__device__ __forceinline__ void tmem_ld_wait4(uint32_t (&a)[32], uint32_t (&b)[32], uint32_t (&c)[32],
                                              uint32_t (&d)[32]) {
  tmem_ld_wait(a);
  tmem_ld_wait(b);  // no outstanding loads remain: these only order the registers
  tmem_ld_wait(c);
  tmem_ld_wait(d);
}

// OUT selects what the epilogue writes: kOutNorm the normalised output;
// kOutStats instead of it, each CTA's own map's O_i / l_i (float32) and
// log-sum-exp (what the backward pass needs); kOutBoth both (a training
// forward that saves the backward's statistics).
enum : int { kOutNorm = 0, kOutStats = 1, kOutBoth = 2 };
// QKF: the format of the queries and keys
enum : int { kQkBf16 = 0, kQkE4m3 = 1, kQkE2m1 = 2 };
template <int D, int QKF, int OUT>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_sm100_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                         const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap to,
                         const PrefillParams p) {
  constexpr bool QK8 = QKF != kQkBf16;
  using C = Cfg<D, QK8>;
  // bytes a Q / K tile brings in from global memory (packed e2m1: half its shared-memory size)
  constexpr uint32_t kQTx = QKF == kQkE2m1 ? C::Q_BYTES / 2 : C::Q_BYTES;
  constexpr uint32_t kKTx = QKF == kQkE2m1 ? C::K_BYTES / 2 : C::K_BYTES;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sK = smem + C::OFF_K;
  uint8_t* sV = smem + C::OFF_V;
  Bars* bars = reinterpret_cast<Bars*>(smem + C::OFF_BAR);
  float* ssx = reinterpret_cast<float*>(smem + C::OFF_SSX);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();  // 0: map 1, 1: map 2
  const uint32_t partner = rank ^ 1u;
  const int cid = static_cast<int>(blockIdx.x >> 1), n_clusters = static_cast<int>(gridDim.x >> 1);
  const int N = p.N;
  const int n_kvtiles = (N + kBN - 1) / kBN;
  const int BH = p.B * p.H;

  // This cluster's k-th item (-1 past the end): longest first, dealt in a snake.
  auto item_of = [&](int k) -> int {
    const int pos = (k & 1) ? (n_clusters - 1 - cid) : cid;
    const long long i = static_cast<long long>(k) * n_clusters + pos;
    return i < p.n_items ? static_cast<int>(i) : -1;
  };
  struct Item {
    int qtile, h, b, n_kv;
  };
  auto decode = [&](int i) -> Item {
    Item it;
    const int per_group = p.head_group * p.n_qtiles;
    const int grp = i / per_group, li = i % per_group;
    const int gsize = min(p.head_group, BH - grp * p.head_group);  // the last group may be smaller
    it.qtile = p.n_qtiles - 1 - li / gsize;
    const int bh = grp * p.head_group + li % gsize;
    it.b = bh / p.H;
    it.h = bh % p.H;
    it.n_kv = p.causal ? min(it.qtile + 1, n_kvtiles) : n_kvtiles;
    return it;
  };

  if (tid == 0) {
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->k_full[i], 1);
      mbar_init(&bars->k_empty[i], 1);
      mbar_init(&bars->v_full[i], 1);
      mbar_init(&bars->v_empty[i], 1);
      mbar_init(&bars->p_full[i], 4);  // one arrival per softmax warp
      mbar_init(&bars->p_empty[i], 1);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->s_free, 4);
    mbar_init(&bars->mma_done, 1);
    mbar_init(&bars->exch_full, 1);
    mbar_init(&bars->peer_ready, 1);
    mbar_init(&bars->ss_full, 1);
    mbar_init(&bars->epi_free, 1);
    bars->abort = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tq);
    tma_prefetch_desc(&tk);
    tma_prefetch_desc(&tv);
    tma_prefetch_desc(&to);
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, C::TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers exist before any remote arrival
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  const WaitCtl wc{p.status, &bars->abort, p.limit_ns};
  // Drains (after a normal run these return at once) ignore the abort flag.
  int drain_abort = 0;
  const WaitCtl wdrain{p.status, &drain_abort, 1000000000ull};

  if (warp == 0) {
    // ---------------------------------------------------- Q / K producer --
    if (lane == 0) {
      int gk = 0;  // K tiles issued (all items)
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int idx = item_of(k);
        if (idx < 0) break;
        const Item it = decode(idx);
        const int c1 = 2 * it.h + static_cast<int>(rank);
        // Q of this item replaces the last one's once that item's S products have read it
        if (k > 0 && !(ok = mbar_wait(&bars->q_empty, (k - 1) & 1, wc))) break;
        // debug builds: the tile lies in the tensor (else the load is skipped
        // and the phase completed without data)
        if (DA_CHECK(p.status, it.b >= 0 && it.b < p.B && it.h >= 0 && c1 < 2 * p.H && it.qtile >= 0 &&
                                   it.qtile * kBM < N)) {
          mbar_arrive_expect_tx(&bars->q_full, kQTx);
#pragma unroll
          for (int blk = 0; blk < C::QBLK; ++blk)
            tma_load_4d(sQ + blk * C::BLK_BYTES, &tq, &bars->q_full, blk * C::QBOX, c1, it.qtile * kBM, it.b);
        } else {
          mbar_arrive(&bars->q_full);
        }
        for (int j = 0; j < it.n_kv; ++j, ++gk) {
          const int st = gk & 1;
          if (!(ok = mbar_wait(&bars->k_empty[st], ((gk >> 1) & 1) ^ 1, wc))) break;
          if (DA_CHECK(p.status, j * kBN < N)) {
            mbar_arrive_expect_tx(&bars->k_full[st], kKTx);
#pragma unroll
            for (int blk = 0; blk < C::QBLK; ++blk)
              tma_load_4d(sK + st * C::K_BYTES + blk * C::BLK_BYTES, &tk, &bars->k_full[st], blk * C::QBOX, c1,
                          j * kBN, it.b);
          } else {
            mbar_arrive(&bars->k_full[st]);
          }
        }
      }
      // nothing may still be landing in shared memory when the CTA exits
      for (int j = max(0, gk - 2); j < gk; ++j) mbar_wait(&bars->k_full[j & 1], (j >> 1) & 1, wdrain);
    }
    __syncwarp();
  } else if (warp == 2) {
    // -------------------------------------------------------- V producer --
    if (lane == 0) {
      int gv = 0;  // V tiles issued (all items)
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int idx = item_of(k);
        if (idx < 0) break;
        const Item it = decode(idx);
        // the previous item's epilogue uses both V stages for its exchange
        if (k > 0 && !(ok = mbar_wait(&bars->epi_free, (k - 1) & 1, wc))) break;
        for (int j = 0; j < it.n_kv; ++j, ++gv) {
          const int st = gv & 1;
          if (!(ok = mbar_wait(&bars->v_empty[st], ((gv >> 1) & 1) ^ 1, wc))) break;
          if (DA_CHECK(p.status, it.b >= 0 && it.b < p.B && it.h >= 0 && it.h < p.H && j * kBN < N)) {
            mbar_arrive_expect_tx(&bars->v_full[st], C::V_BYTES);
#pragma unroll
            for (int blk = 0; blk < C::VBLK; ++blk)
              tma_load_4d(sV + st * C::V_BYTES + blk * C::BLK_BYTES, &tv, &bars->v_full[st], blk * 64, it.h,
                          j * kBN, it.b);
          } else {
            mbar_arrive(&bars->v_full[st]);
          }
        }
      }
      for (int j = max(0, gv - 2); j < gv; ++j) mbar_wait(&bars->v_full[j & 1], (j >> 1) & 1, wdrain);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      constexpr uint32_t idesc_s = QKF == kQkE2m1   ? idesc_f8f6f4_f32(128, 128, kF8f6f4E2m1)
                                   : QKF == kQkE4m3 ? idesc_f8f6f4_f32(128, 128, kF8f6f4E4m3)
                                                    : idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, C::DV, false, true);
      const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK), sVa = smem_u32(sV);
      int gs = 0;  // S products issued (all items)
      int gp = 0;  // PV products issued (all items)
      // O (+)= P V for the next tile, with P from buffer gp % 2 and V from stage gp % 2;
      // `first` starts a new item's O
      auto issue_pv = [&](bool first) -> bool {
        const int bb = gp & 1;
        const uint32_t ph = (gp >> 1) & 1;
        if (!mbar_wait(&bars->v_full[bb], ph, wc)) return false;
        if (!mbar_wait(&bars->p_full[bb], ph, wc)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          const uint32_t a_tmem = tmem + C::TM_P + 64 * bb + 8 * kk;
          const uint64_t bd = smem_desc_sw128(sVa + bb * C::V_BYTES + kk * 2048, C::BLK_BYTES, 1024);
          umma_ts(tmem + C::TM_O, a_tmem, bd, idesc_pv, (!first || kk > 0) ? 1u : 0u);
        }
        umma_commit(&bars->v_empty[bb]);
        umma_commit(&bars->p_empty[bb]);
        ++gp;
        return true;
      };
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int idx = item_of(k);
        if (idx < 0) break;
        const Item it = decode(idx);
        if (!(ok = mbar_wait(&bars->q_full, k & 1, wc))) break;
        for (int j = 0; ok && j < it.n_kv; ++j, ++gs) {
          const int st = gs & 1;
          // S overwrites the previous S tile: every softmax warp must have read it
          if (gs > 0 && !(ok = mbar_wait(&bars->s_free, (gs - 1) & 1, wc))) break;
          if (!(ok = mbar_wait(&bars->k_full[st], (gs >> 1) & 1, wc))) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / C::KSTEP; ++kk) {  // each instruction takes 32 bytes of every row
            const int blk = kk >> 2;
            const uint32_t koff = (kk & 3) * 32;
            const uint64_t ad = smem_desc_sw128(sQa + blk * C::BLK_BYTES + koff, 16, 1024);
            const uint64_t bd = smem_desc_sw128(sKa + st * C::K_BYTES + blk * C::BLK_BYTES + koff, 16, 1024);
            if constexpr (QK8)
              umma_ss_f8(tmem + C::TM_S, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
            else
              umma_ss(tmem + C::TM_S, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
          }
          umma_commit(&bars->k_empty[st]);
          umma_commit(&bars->s_full);
          if (j == it.n_kv - 1) umma_commit(&bars->q_empty);  // the item's S products are all issued
          if (j > 0) ok = issue_pv(j == 1);
        }
        if (ok) ok = issue_pv(it.n_kv == 1);
      }
      // drain: every issued MMA has completed before tensor memory is read or freed
      umma_commit(&bars->mma_done);
      mbar_wait(&bars->mma_done, 0, wdrain);
    }
    __syncwarp();
  } else if (warp == 3) {
    // --------------------------------------------------- output store --
    // Per item: once the softmax warps have staged the bf16 tile (V stage 1),
    // store it with TMA, wait until the store has read it, and free both V
    // stages for the next item.  The softmax warps do not wait for any of it.
    if constexpr (OUT != kOutStats) {
      const uint8_t* out_tile = sV + C::V_BYTES;
      const int own0 = (rank == 0) ? 0 : C::HALF;
      for (int k = 0;; ++k) {
        const int idx = item_of(k);
        if (idx < 0) break;
        const Item it = decode(idx);
        named_bar_sync(2, 160);  // with the softmax warps' arrivals
        if (lane == 0) {
#pragma unroll
          for (int blk = 0; blk < C::HALF / 64; ++blk)  // rows >= N are clipped by the store
            tma_store_4d(&to, out_tile + blk * C::BLK_BYTES, own0 + 64 * blk, it.h, it.qtile * kBM, it.b);
          bulk_commit_group();
          bulk_wait_group_read0();  // the stage must stay valid until the store has read it
          mbar_arrive(&bars->epi_free);
        }
        __syncwarp();
      }
    }
  }

  if (warp >= 4) {
    // ------------------------------------------------ softmax + epilogue --
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // query row within the tile (= TMEM lane)
    const uint32_t tl = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const float coef2 = map2_coefficient(p.mode, *p.lambda);  // c in softmax(S1) + c softmax(S2)
    constexpr int HALF = C::HALF;
    constexpr int NC = HALF / 4;  // float4 chunks per exchanged row
    float* recv = reinterpret_cast<float*>(sV);              // V stage 0: the partner's half
    float* stage = reinterpret_cast<float*>(sV + C::V_BYTES);  // V stage 1: the half sent, then the output
    const uint32_t own0 = (rank == 0) ? 0 : HALF;   // columns this CTA finishes
    const uint32_t send0 = (rank == 0) ? HALF : 0;  // columns it hands to the partner
    int g = 0;  // S / P tiles consumed (all items)
    bool sm_ok = true;
    for (int k = 0;; ++k) {
      const int idx = item_of(k);
      if (idx < 0) break;
      const Item it = decode(idx);
      const int N_kv = it.n_kv;
      const int qtile = it.qtile;
      const int qrow = qtile * kBM + r;
      float sc = kLog2e * rsqrtf(static_cast<float>(D));
      if constexpr (QK8) {  // scores of the codes times the two groups' scales
        const int gi = (it.b * p.H + it.h) * 2 + static_cast<int>(rank);
        sc *= __ldg(p.q_scale + gi) * __ldg(p.k_scale + gi);
      }
      float m_run = -INFINITY, l_run = 0.f;
      // O and l *= alpha (the whole warp takes part; alpha = 1 leaves a row as it is)
      auto rescale_o = [&](float alpha) {
#pragma unroll
        for (int c = 0; c < C::DV / 32; ++c) {
          uint32_t ov[32];
          tmem_ld32_sync(tl + C::TM_O + 32 * c, ov);
#pragma unroll
          for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
          tmem_st32(tl + C::TM_O + 32 * c, ov);
        }
        tmem_st_wait();
        l_run *= alpha;
      };
      for (int j = 0; sm_ok && j < N_kv; ++j, ++g) {
        const int bb = g & 1;
        // every exit is taken by the whole warp (a wait may end differently in its lanes)
        if (!(sm_ok = __all_sync(0xffffffffu, mbar_wait(&bars->s_full, g & 1, wc)))) break;
        // S_g has completed, and with it every MMA issued before it, PV_{g-2}
        // included: P buffer b is free.
        tc_fence_after();
        uint32_t s0[32], s1[32], s2[32], s3[32];
        tmem_ld32(tl + C::TM_S + 0, s0);
        tmem_ld32(tl + C::TM_S + 32, s1);
        tmem_ld32(tl + C::TM_S + 64, s2);
        tmem_ld32(tl + C::TM_S + 96, s3);
        tmem_ld_wait4(s0, s1, s2, s3);
        // S is in registers: the next S tile may overwrite the buffer
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->s_free);
        float x[128];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          x[i] = __uint_as_float(s0[i]);
          x[32 + i] = __uint_as_float(s1[i]);
          x[64 + i] = __uint_as_float(s2[i]);
          x[96 + i] = __uint_as_float(s3[i]);
        }
        const int key0 = j * kBN;
        if (key0 + kBN > N || (p.causal && j == qtile)) {
          const int lim = (p.causal ? min(N - 1, qrow) : N - 1) - key0;  // last visible key of the tile
#pragma unroll
          for (int i = 0; i < 128; ++i)
            if (i > lim) x[i] = -INFINITY;
        }
        if (j == 0) {  // the first tile sets the reference maximum
          float mk[8];
#pragma unroll
          for (int c = 0; c < 8; ++c) mk[c] = x[c];
#pragma unroll
          for (int i = 8; i < 128; i += 8) {
#pragma unroll
            for (int c = 0; c < 8; ++c) mk[c] = fmaxf(mk[c], x[i + c]);
          }
          m_run = fmaxf(fmaxf(fmaxf(mk[0], mk[1]), fmaxf(mk[2], mk[3])), fmaxf(fmaxf(mk[4], mk[5]), fmaxf(mk[6], mk[7]))) * sc;
        }
        // P = exp2(s*c - m_run) into P[b], taken relative to the reference
        // maximum m_run as it stands; the tile's own maximum is formed alongside.
        float lsum = 0.f, t_mx = -INFINITY;
        auto make_p = [&](bool with_max) {
          const float mneg = -m_run;
          float acc[4] = {0.f, 0.f, 0.f, 0.f};
          float mk[8];
#pragma unroll
          for (int c = 0; c < 8; ++c) mk[c] = -INFINITY;
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            uint32_t pk[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const float a0 = x[64 * half + 2 * i], a1 = x[64 * half + 2 * i + 1];
              if (with_max) mk[i & 7] = fmaxf(mk[i & 7], fmaxf(a0, a1));
              const float p0 = fast_exp2(fmaf(a0, sc, mneg));
              const float p1 = fast_exp2(fmaf(a1, sc, mneg));
              acc[i & 3] += p0 + p1;
              pk[i] = pack_bf16x2(p0, p1);
            }
            tmem_st32(tl + C::TM_P + 64 * bb + 32 * half, pk);
          }
          lsum = (acc[0] + acc[1]) + (acc[2] + acc[3]);
          if (with_max)
            t_mx = fmaxf(fmaxf(fmaxf(mk[0], mk[1]), fmaxf(mk[2], mk[3])), fmaxf(fmaxf(mk[4], mk[5]), fmaxf(mk[6], mk[7]))) * sc;
        };
        make_p(true);
        // A jump of the maximum by more than 2^64 would overflow P: rescale O
        // to the new maximum (after the previous tile's PV has completed) and redo P.
        const bool hard = t_mx > m_run + kOverflowGuard;
        if (__any_sync(0xffffffffu, hard)) {
          tmem_st_wait();
          if (!(sm_ok = __all_sync(0xffffffffu, mbar_wait(&bars->p_empty[(g - 1) & 1], ((g - 1) >> 1) & 1, wc))))
            break;
          tc_fence_after();
          rescale_o(hard ? fast_exp2(m_run - t_mx) : 1.0f);
          if (hard) m_run = t_mx;
          make_p(false);
        }
        tmem_st_wait();
        l_run += lsum;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->p_full[bb]);
        // Lazy rescale: keep the reference within 2^8 of the running maximum.
        // O is rescaled once this tile's PV (which used the old reference) has completed.
        const bool need = t_mx > m_run + kRescaleThreshold;
        if (__any_sync(0xffffffffu, need)) {
          if (!(sm_ok = __all_sync(0xffffffffu, mbar_wait(&bars->p_empty[bb], (g >> 1) & 1, wc)))) break;
          tc_fence_after();
          rescale_o(need ? fast_exp2(m_run - t_mx) : 1.0f);
          if (need) m_run = t_mx;
        }
      }
      // the loop above may stop early after an abort: keep the tile count in step
      g = 0;
      for (int kk = 0; kk <= k; ++kk) g += decode(item_of(kk)).n_kv;

      // ------------------------------------------------------ epilogue --
      // O is complete once the item's last PV (and with it every earlier MMA) has.
      if (sm_ok) sm_ok = mbar_wait(&bars->p_empty[(g - 1) & 1], ((g - 1) >> 1) & 1, wc);
      tc_fence_after();
      if constexpr (OUT != kOutNorm) {
        // This map's O_i / l_i for the row, and lse_i = m + log2(l) in the
        // scaled log2 units of P = exp2(s * sc - m): P / l = exp2(s * sc - lse_i).
        const bool live = qrow < N && DA_CHECK(p.status, qrow < p.n_pad && it.b < p.B && it.h < p.H);
        const float inv = 1.0f / l_run;
        float* orow = p.o_maps + ((static_cast<size_t>(it.b) * N + (live ? qrow : 0)) * p.H + it.h) * (2 * C::DV) +
                      rank * C::DV;
#pragma unroll 1
        for (int c = 0; c < C::DV / 32; ++c) {
          uint32_t ov[32];
          tmem_ld32_sync(tl + C::TM_O + 32 * c, ov);
          if (live) {
#pragma unroll
            for (int f = 0; f < 8; ++f)
              *reinterpret_cast<float4*>(orow + 32 * c + 4 * f) =
                  make_float4(__uint_as_float(ov[4 * f + 0]) * inv, __uint_as_float(ov[4 * f + 1]) * inv,
                              __uint_as_float(ov[4 * f + 2]) * inv, __uint_as_float(ov[4 * f + 3]) * inv);
          }
        }
        if (live) p.lse[((static_cast<size_t>(it.b) * p.H + it.h) * p.n_pad + qrow) * 4 + rank] = m_run + log2f(l_run);
        if constexpr (OUT == kOutStats) {
          tc_fence_before();
          named_bar_sync(1, 128);  // every row's tensor-memory reads are done
          if (tid == 128) mbar_arrive(&bars->epi_free);  // the next item's first PV may overwrite O
          __syncwarp();
          continue;
        }
        // kOutBoth: O is still in tensor memory (the next item's first PV waits for epi_free)
      }
      // Both V stages are free of this item's PV products: announce that this
      // CTA's receive buffer is ready, with the exchange barrier armed first.
      named_bar_sync(1, 128);
      if (tid == 128) {
        mbar_arrive_expect_tx(&bars->exch_full, C::EXCH_BYTES);
        mbar_arrive_expect_tx(&bars->ss_full, kBM * 4);  // the partner's sums of squares, by st.async
        mbar_arrive_remote(map_to_cta(smem_u32(&bars->peer_ready), partner));
      }
      const float inv = (rank == 0) ? 1.0f / l_run : coef2 / l_run;
      float* srow = stage + r * HALF;
#pragma unroll
      for (int c = 0; c < HALF / 32; ++c) {
        uint32_t ov[32];
        tmem_ld32_sync(tl + C::TM_O + send0 + 32 * c, ov);
#pragma unroll
        for (int f = 0; f < 8; ++f) {
          const int chunk = (c * 8 + f) ^ (r % NC);
          *reinterpret_cast<float4*>(srow + chunk * 4) =
              make_float4(__uint_as_float(ov[4 * f + 0]) * inv, __uint_as_float(ov[4 * f + 1]) * inv,
                          __uint_as_float(ov[4 * f + 2]) * inv, __uint_as_float(ov[4 * f + 3]) * inv);
        }
      }
      fence_proxy_async_smem();  // the staged rows are read by the bulk copy (async proxy)
      __syncwarp();
      // the partner's receive buffer must be free before this CTA writes into it
      const bool peer_ok = mbar_wait_acq_cluster(&bars->peer_ready, k & 1, wc);
      if (lane == 0 && peer_ok) {
        const int off = quarter * 32 * HALF;  // this warp's 32 rows, contiguous
        bulk_copy_s2cluster(map_to_cta(smem_u32(recv + off), partner), stage + off, 32 * HALF * 4,
                            map_to_cta(smem_u32(&bars->exch_full), partner));
        bulk_commit_group();
      }
      mbar_wait(&bars->exch_full, k & 1, wdrain);  // the partner's half has landed (even after an abort)
      float y[HALF];
      float ss = 0.f;
      const float* rrow = recv + r * HALF;
#pragma unroll
      for (int c = 0; c < HALF / 32; ++c) {
        uint32_t ov[32];
        tmem_ld32_sync(tl + C::TM_O + own0 + 32 * c, ov);
#pragma unroll
        for (int f = 0; f < 8; ++f) {
          const int chunk = (c * 8 + f) ^ (r % NC);
          const float4 xr = *reinterpret_cast<const float4*>(rrow + chunk * 4);
          const float xs[4] = {xr.x, xr.y, xr.z, xr.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float val = fmaf(__uint_as_float(ov[4 * f + e]), inv, xs[e]);
            y[32 * c + 4 * f + e] = val;
            ss = fmaf(val, val, ss);
          }
        }
      }
      // this row's half of the sum of squares to the partner: an asynchronous
      // store that completes on the partner's barrier (armed before its
      // receive buffer was announced)
      if (peer_ok)
        st_async_f32(map_to_cta(smem_u32(ssx + r), partner), ss, map_to_cta(smem_u32(&bars->ss_full), partner));
      if (lane == 0 && peer_ok) bulk_wait_group_read0();  // the outgoing copy has left the staging rows
      __syncwarp();
      named_bar_sync(1, 128);  // every warp's outgoing copy is done with the rows the output tile reuses
      mbar_wait_acq_cluster(&bars->ss_full, k & 1, wdrain);
      const float rs = rsqrtf((ss + ssx[r]) / static_cast<float>(C::DV) + p.eps);
      const float gsc = (1.0f - p.lambda_init) * rs;
      // bf16 tile [64-column block][128 rows][64 columns], 128-byte swizzle, in the staging stage
      const uint32_t sout = smem_u32(stage);
#pragma unroll
      for (int c8 = 0; c8 < HALF / 8; ++c8) {
        uint32_t w4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int c = 8 * c8 + 2 * e;
          w4[e] = pack_bf16x2(y[c] * gsc * __ldg(p.rms_w + own0 + c), y[c + 1] * gsc * __ldg(p.rms_w + own0 + c + 1));
        }
        const uint32_t a = sout + (c8 / 8) * C::BLK_BYTES + r * 128 + (((c8 % 8) ^ (r & 7)) << 4);
        st_shared_v4(a, w4[0], w4[1], w4[2], w4[3]);
      }
      fence_proxy_async_smem();  // the tile is read by the TMA store (async proxy)
      // hand the staged tile to warp 3, which stores it and frees the V stages,
      // and go on with the next item
      named_bar_arrive(2, 160);
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // no remote access to either CTA remains
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TM_COLS);
  }
}

template <int D, int QKF, int OUT = kOutNorm>
static cudaError_t launch_d(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& to, const PrefillParams& prm, cudaStream_t stream, int ctl_dev = -1,
                            unsigned long long ctl_ctx = 0) {
  using C = Cfg<D, QKF != kQkBf16>;
  // per device and context: the shared-memory size and the cluster shape (a
  // pair along x) are set as function attributes and the resident cluster
  // count looked up on the first launch only (again after a cudaDeviceReset,
  // which creates a new context).  A launch that carries no attributes costs
  // the host about 0.6 us less than one that passes the cluster shape.
  static int max_clusters[64] = {};
  static unsigned long long set_ctx[64] = {};
  int dev = ctl_dev;
  cudaError_t e = cudaSuccess;
  if (dev < 0 && (e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  const unsigned long long ctx = ctl_ctx != 0 ? ctl_ctx : current_context_id();
  int& mc = max_clusters[dev];
  if (ctx == 0 || set_ctx[dev] != ctx) mc = 0;
  if (mc == 0) {
    const auto fn = prefill_sm100_kernel<D, QKF, OUT>;
    if ((e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_ALLOC)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(fn, cudaFuncAttributeRequiredClusterWidth, 2)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(fn, cudaFuncAttributeRequiredClusterHeight, 1)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(fn, cudaFuncAttributeRequiredClusterDepth, 1)) != cudaSuccess)
      return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM_ALLOC;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // persistent grid: as many clusters as can be resident at once
  if (mc == 0) {
    cfg.gridDim = dim3(2 * 128, 1, 1);
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, prefill_sm100_kernel<D, QKF, OUT>, &cfg) != cudaSuccess || n < 1) n = 1;
    mc = n;
    set_ctx[dev] = ctx;
  }
  const int clusters = prm.n_items < mc ? prm.n_items : mc;
  cfg.gridDim = dim3(2 * clusters, 1, 1);
  cfg.attrs = nullptr;  // the required cluster shape is the function's own
  cfg.numAttrs = 0;
  return cudaLaunchKernelEx(&cfg, prefill_sm100_kernel<D, QKF, OUT>, tq, tk, tv, to, prm);
}

cudaError_t launch_prefill_sm100(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                 const CUtensorMap& to, void* o,
                                 int B, int N, int H, int d, int causal, const float* lambda, float lambda_init,
                                 const float* rms_w, float eps, int mode, const float* q_scale,
                                 const float* k_scale, int qk_bits, DevCtl ctl, cudaStream_t stream) {
  PrefillParams prm = {};
  prm.o = static_cast<__nv_bfloat16*>(o);
  prm.N = N;
  prm.H = H;
  prm.B = B;
  prm.causal = causal ? 1 : 0;
  prm.n_qtiles = (N + kBM - 1) / kBM;
  prm.n_items = B * H * prm.n_qtiles;
  {  // pairs per group: their K (both maps) and V, 8d bytes per token, in about 48 MB
    const long long per_head = static_cast<long long>(N) * 8 * d;
    const long long grp = (48ll << 20) / (per_head > 0 ? per_head : 1);
    prm.head_group = static_cast<int>(grp < 1 ? 1 : (grp > B * H ? B * H : grp));
  }
  prm.lambda = lambda;
  prm.q_scale = q_scale;
  prm.k_scale = k_scale;
  prm.mode = mode;
  prm.lambda_init = lambda_init;
  prm.rms_w = rms_w;
  prm.eps = eps;
  prm.status = ctl.status;
  prm.limit_ns = ctl.limit_ns;
  if (q_scale != nullptr) {
    if (d != 128) return cudaErrorInvalidValue;
    if (qk_bits == 8) return launch_d<128, kQkE4m3>(tq, tk, tv, to, prm, stream, ctl.dev, ctl.ctx);
    if (qk_bits == 4) return launch_d<128, kQkE2m1>(tq, tk, tv, to, prm, stream, ctl.dev, ctl.ctx);
    return cudaErrorInvalidValue;
  }
  if (d == 128) return launch_d<128, kQkBf16>(tq, tk, tv, to, prm, stream, ctl.dev, ctl.ctx);
  if (d == 64) return launch_d<64, kQkBf16>(tq, tk, tv, to, prm, stream, ctl.dev, ctl.ctx);
  return cudaErrorInvalidValue;
}

cudaError_t launch_prefill_sm100_stats(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                       const CUtensorMap* to, void* o, int B, int N, int H, int d, int causal,
                                       const float* lambda, float lambda_init, const float* rms_w, float eps, int mode,
                                       float* o_maps, float* lse, int n_pad, DevCtl ctl, cudaStream_t stream) {
  PrefillParams prm = {};
  prm.o = static_cast<__nv_bfloat16*>(o);
  prm.N = N;
  prm.H = H;
  prm.B = B;
  prm.causal = causal ? 1 : 0;
  prm.n_qtiles = (N + kBM - 1) / kBM;
  prm.n_items = B * H * prm.n_qtiles;
  {
    const long long per_head = static_cast<long long>(N) * 8 * d;
    const long long grp = (48ll << 20) / (per_head > 0 ? per_head : 1);
    prm.head_group = static_cast<int>(grp < 1 ? 1 : (grp > B * H ? B * H : grp));
  }
  prm.lambda = lambda;
  prm.mode = mode;
  prm.lambda_init = lambda_init;
  prm.rms_w = rms_w;
  prm.eps = eps;
  prm.status = ctl.status;
  prm.limit_ns = ctl.limit_ns;
  prm.o_maps = o_maps;
  prm.lse = lse;
  prm.n_pad = n_pad;
  if (to) {  // the normalised output as well
    if (d == 128) return launch_d<128, kQkBf16, kOutBoth>(tq, tk, tv, *to, prm, stream, ctl.dev, ctl.ctx);
    if (d == 64) return launch_d<64, kQkBf16, kOutBoth>(tq, tk, tv, *to, prm, stream, ctl.dev, ctl.ctx);
    return cudaErrorInvalidValue;
  }
  // statistics only: the output map is never used, tv stands in for it
  if (d == 128) return launch_d<128, kQkBf16, kOutStats>(tq, tk, tv, tv, prm, stream, ctl.dev, ctl.ctx);
  if (d == 64) return launch_d<64, kQkBf16, kOutStats>(tq, tk, tv, tv, prm, stream, ctl.dev, ctl.ctx);
  return cudaErrorInvalidValue;
}

}  // namespace diffattn
