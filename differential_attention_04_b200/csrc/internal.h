// Launchers shared between the C-ABI layer (api.cu) and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>

namespace diffattn {

// Unique id of the calling thread's current CUDA context (cuCtxGetId), or 0
// when it cannot be read.  A context that cudaDeviceReset tore down and the
// runtime re-created gets a new id, so per-device caches of device addresses
// key on it and look the address up again.
unsigned long long current_context_id();

// Device address of the status word on the current device (nullptr when it
// cannot be looked up).
int* status_word();
// What a kernel's debug bounds checks (DA_CHECK) record into: the status word
// in a debug build, nullptr in a release build (where the checks compile away).
inline int* debug_status() {
#ifdef DIFFATTN_DEBUG
  return status_word();
#else
  return nullptr;
#endif
}

// Where kernels record a failed bounded wait, and how long a wait may spin.
struct DevCtl {
  int* status;
  unsigned long long limit_ns;
  int dev = -1;                  // the current device, when the caller looked it up
  unsigned long long ctx = 0;    // its context's id (current_context_id), when looked up
};

cudaError_t launch_lambda(const float* lq1, const float* lk1, const float* lq2, const float* lk2, int d,
                          float lambda_init, float* out, cudaStream_t stream);

// CUDA-core prefill for float32 tensors, any 1 <= d <= 128.
cudaError_t launch_prefill_simt_f32(const float* q, const float* k, const float* v, float* o, int B, int N, int H,
                                    int d, int causal, const float* lambda, float lambda_init, const float* rms_w,
                                    float eps, int mode, cudaStream_t stream);

// Coefficient c of map 2 in D = softmax(S1) + c softmax(S2) for a diffattn_mode.
__host__ __device__ inline float map2_coefficient(int mode, float lam) {
  return mode == 0 ? -lam : (mode == 2 ? lam : 0.0f);
}

// Tensor-core (tcgen05) prefill, d in {64, 128} for bf16 queries and keys,
// d = 128 for low-bit ones (q_scale, k_scale non-null; qk_bits 8: e4m3 codes,
// 4: packed e2m1 codes).  tq/tk map [B, N, H*2, d]; tv and to map
// [B, N, H, 2d]; boxes are 128 bytes (bf16, e4m3) or 128 elements (e2m1) x
// 128 rows with 128-byte swizzle.
cudaError_t launch_prefill_sm100(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                 const CUtensorMap& to, void* o,
                                 int B, int N, int H, int d, int causal, const float* lambda, float lambda_init,
                                 const float* rms_w, float eps, int mode, const float* q_scale,
                                 const float* k_scale, int qk_bits, DevCtl ctl, cudaStream_t stream);

// Low-bit codes of a bf16 [B, N, H, 2, d] tensor with one float32 scale per
// (batch, head, map) (scales: [B][H][2], also the absmax accumulator).
// bits 8: e4m3 codes, one byte each; bits 4: e2m1 codes, two per byte
// (channel 2j in the low nibble).
cudaError_t launch_quantize_qk(const void* x, int B, int N, int H, int d, int bits, void* codes, float* scales,
                               cudaStream_t stream);

// Backward pass of the prefill (CUDA cores; bf16 or fp32 inputs, fp32 gradients).
size_t bwd_workspace_bytes(int B, int N, int H, int d);
cudaError_t launch_bwd(const void* q, const void* k, const void* v, const void* dy, int bf16, int B, int N, int H,
                       int d, int causal, const float* lambda, float lambda_init, const float* rms_w, float eps,
                       int mode, float* dq, float* dk, float* dv, float* dlambda, float* drms_w, void* workspace,
                       cudaStream_t stream);
// Tensor-core backward (bf16 inputs, d in {64, 128}).  Maps over q, k
// [B, N, H*2, d] and v, G [B, N, H, 2d] with boxes of 128 bytes x 128 rows
// (q128 ...), x 64 rows (q64, g64) or x 32 rows (q32 ...); G is the
// workspace's bf16 dO.
struct BwdTcMaps {
  CUtensorMap q128, q32, k128, k32, v128, v32, g128, g32;
  CUtensorMap q64, g64;  // the dV kernel's 64-row column tiles
};
// Workspace: per map A_i V as float32 [B, N, H, 2, 2d]; G bf16 [B, N, H, 2d];
// statistics float4 [B][H][n_pad] (n_pad = N rounded up to 128).
struct BwdTcLayout {
  size_t off_omaps, off_g, off_stats, bytes;
  int n_pad;
};
BwdTcLayout bwd_tc_layout(int B, int N, int H, int d);
// stats_ready: the workspace already holds the statistics (from the training
// forward with the same q, k, v, lambda and mask): the statistics pass is skipped.
cudaError_t launch_bwd_sm100(const BwdTcMaps& m, const void* dy, int B, int N, int H, int d, int causal,
                             const float* lambda, float lambda_init, const float* rms_w, float eps, int mode,
                             float* dq, float* dk, float* dv, float* dlambda, float* drms_w, void* workspace,
                             bool stats_ready, DevCtl ctl, cudaStream_t stream);
// The tcgen05 prefill in its statistics mode: per map, O_i / l_i into
// o_maps and the log2-sum-exp into component i of the float4 rows of lse;
// with `to` (the output map over o) non-null, the normalised output too.
cudaError_t launch_prefill_sm100_stats(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                       const CUtensorMap* to, void* o, int B, int N, int H, int d, int causal,
                                       const float* lambda, float lambda_init, const float* rms_w, float eps, int mode,
                                       float* o_maps, float* lse, int n_pad, DevCtl ctl, cudaStream_t stream);
cudaError_t launch_lambda_bwd(const float* lq1, const float* lk1, const float* lq2, const float* lk2, int d,
                              const float* dlambda, float* dlq1, float* dlk1, float* dlq2, float* dlk2,
                              cudaStream_t stream);

// Projection GEMM C[M, N] = A[M, K] B[N, K]^T on CTA pairs (tcgen05
// cta_group::2; bf16, fp32 accumulation, bf16 out; K a multiple of 64, N and
// the column boundaries multiples of 32).  Columns [col_end[o-1], col_end[o])
// go to out[o] (row stride = that width); columns below rope_end get RoPE from
// `rope` (float2 cos/sin [seq_len][d/2]) at position (row mod seq_len) when
// rope is non-null.  ta maps A as (K, 1, M, 1), tb maps B as (K, 1, N, 1),
// both with boxes of 64 x 128 rows.
struct ProjParams {
  int M, N, K, seq_len, d, rope_end;
  int col_end[3];
  __nv_bfloat16* out[3];
  const float2* rope;
  int* status;
  unsigned long long limit_ns;
};
cudaError_t launch_proj_gemm(const CUtensorMap& ta, const CUtensorMap& tb, const ProjParams& prm,
                             cudaStream_t stream);
// cos/sin of n * base^(-2j/d) in double precision, rounded to float: [seq_len][d/2] float2.
cudaError_t launch_rope_table(int seq_len, int d, double base, float* table, cudaStream_t stream);

// Split-KV decode (bf16, d = 128).
size_t decode_workspace_bytes(int S, int H, int d, int max_seqlen);
// Whether S * ceil(max_seqlen / 512) * H (chunk, head) units stay within the
// kernels' 32-bit counters.
inline bool decode_units_fit(int S, int H, int max_seqlen) {
  const long long chunks = (static_cast<long long>(max_seqlen) + 511) / 512;
  return static_cast<long long>(S) * chunks * H <= 0x3fffffffll;
}
cudaError_t launch_decode(const void* q, const void* k_cache, const void* v_cache, const int* cu_seqlens,
                          int max_seqlen, void* o, int S, int H, int d, const float* lambda, float lambda_init,
                          const float* rms_w, float eps, int mode, void* workspace, cudaStream_t stream);

}  // namespace diffattn
