/*
 * diffattn.h -- C ABI of the differential-attention forward library for
 * NVIDIA B200 (sm_100a).
 *
 * The operation (page "Differential Transformer: Canceling Context Noise with
 * Differential Attention", section "Cancelling Context Noise Through Attention
 * Map Subtraction"; page "Differential attention", section "The
 * noise-canceling idea"; peer review "Differential Transformer", Summary,
 * Eqs. 1-3):
 *
 *   lambda   = exp(lq1 . lk1) - exp(lq2 . lk2) + lambda_init            (Eq. 2)
 *   O        = (softmax(Q1 K1^T / sqrt(d)) - lambda softmax(Q2 K2^T / sqrt(d))) V
 *                                                                      (Eq. 1)
 *   Y        = (1 - lambda_init) * w * O / sqrt(mean_c(O^2) + eps)     (Eq. 3)
 *
 * per head, where each head's query and key are split into two halves of
 * width d (Q1|Q2, K1|K2) and V has width 2d (peer review, Strengths: heads are
 * halved, h = d_model / 2d; Weaknesses: query/key width d, value width 2d).
 * The headwise norm is RMSNorm over the 2d channels of each (token, head),
 * eps inside the square root, with one weight vector w[2d] shared by all
 * heads.
 *
 * Conventions shared by every entry point
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library
 *    never frees or keeps them.  The library allocates no device memory: the
 *    decode path takes a caller-provided workspace.
 *  - Every pointer of a call must belong to the CURRENT device (the one
 *    cudaSetDevice last selected on the calling thread), and `stream` must be
 *    a stream of that device: the library launches on the current device.
 *  - Every call is asynchronous and ordered on `stream` (0 = legacy default
 *    stream).  The return value reports argument validation and launch
 *    errors only; nothing is synchronised.  A kernel-side failure (a bounded
 *    wait that ran out) is recorded in a device status word that
 *    diffattn_device_status() reads.
 *  - Calls may be captured in a CUDA graph (stream capture) and replayed:
 *    each one enqueues only kernel launches and memsets on `stream`.  The
 *    first call of an entry point on a device and context sets kernel
 *    attributes and looks up occupancy, so make it once before capturing.
 *    A replay reads the buffers the captured call was given, at their
 *    current contents.
 *  - Tensors are dense and row-major in the layouts given below; every
 *    tensor pointer must be 16-byte aligned.
 *  - Return values are diffattn_status codes; 0 is success.
 *  - Debug build (libdiffattn_debug.so, compiled with -DDIFFATTN_DEBUG): the
 *    same entry points, whose kernels also check every global index and
 *    tensor-map coordinate before use.  An index out of range is skipped
 *    (never trapped) and DIFFATTN_ERR_BOUNDS is recorded in the device status
 *    word.  The release library compiles these checks away.
 */
#ifndef DIFFATTN_H_
#define DIFFATTN_H_

#include <stddef.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DIFFATTN_OK = 0,
  DIFFATTN_ERR_INVALID_ARG = 1,  /* null pointer, bad size, misalignment      */
  DIFFATTN_ERR_UNSUPPORTED = 2,  /* valid but not implemented (dtype, d)      */
  DIFFATTN_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed         */
  DIFFATTN_ERR_TIMEOUT = 4,      /* a kernel's bounded wait ran out           */
  DIFFATTN_ERR_WORKSPACE = 5,    /* workspace missing or too small            */
  DIFFATTN_ERR_BOUNDS = 6        /* debug build only: a kernel found an index
                                    out of range and skipped the access       */
} diffattn_status;

typedef enum {
  DIFFATTN_F32 = 0,   /* float32 storage and arithmetic                         */
  DIFFATTN_BF16 = 1   /* bfloat16 storage, float32 accumulation                 */
} diffattn_dtype;

/*
 * diffattn_lambda -- the lambda re-parameterisation (Eq. 2).
 *
 *   *lambda_out = exp(lq1 . lk1) - exp(lq2 . lk2) + lambda_init
 *
 * lq1, lk1, lq2, lk2 : device float32[d], 1 <= d <= 4096.
 * lambda_out         : device float32 scalar, written by the kernel.  The
 *                      prefill and decode calls read lambda from this pointer,
 *                      so no host round trip is needed.
 * Errors: DIFFATTN_ERR_INVALID_ARG for a null pointer or d out of range.
 */
int diffattn_lambda(const float* lq1, const float* lk1, const float* lq2,
                    const float* lk2, int d, float lambda_init,
                    float* lambda_out, cudaStream_t stream);

/*
 * diffattn_fwd -- prefill: differential attention for B sequences of N tokens
 * followed by the headwise RMSNorm and the (1 - lambda_init) scale.
 *
 * q, k   : [B, N, H, 2, d]  (per head: Q1 then Q2, K1 then K2 -- the paper's
 *                            2H heads of width d, in the same memory)
 * v      : [B, N, H, 2d]
 * o      : [B, N, H, 2d]    output, same dtype as the inputs
 * dtype  : DIFFATTN_BF16 (tensor-core path; d must be 64 or 128) or
 *          DIFFATTN_F32 (CUDA-core path; 1 <= d <= 128)
 * causal : nonzero -> key j is visible to query i iff j <= i
 * lambda : device float32 scalar (e.g. written by diffattn_lambda)
 * rms_w  : device float32[2d], shared by all heads
 * eps    : RMSNorm epsilon, >= 0, added to mean(O^2) inside the square root
 *
 * Sizes: B, H >= 1; N >= 0 (N = 0 is a no-op).  Shapes must satisfy
 * B*N*H*2d < 2^31 elements per tensor and N < 2^31.
 * Errors: DIFFATTN_ERR_INVALID_ARG (null/misaligned pointer, bad size),
 * DIFFATTN_ERR_UNSUPPORTED (dtype/d combination), DIFFATTN_ERR_CUDA.
 */
int diffattn_fwd(const void* q, const void* k, const void* v, void* o,
                 int dtype, int B, int N, int H, int d, int causal,
                 const float* lambda, float lambda_init, const float* rms_w,
                 float eps, cudaStream_t stream);

/* How the two maps are combined (peer review "Differential Transformer",
 * Weaknesses, second bullet, and Questions, first bullet: the controls it
 * asks for).  D = softmax(S1) + c * softmax(S2), then O = D V:
 *   DIFFATTN_MODE_DIFF        c = -lambda  (the method; diffattn_fwd)
 *   DIFFATTN_MODE_LAMBDA_ZERO c = 0        (lambda fixed to 0: one softmax map,
 *                                           same widths, norm and scale)
 *   DIFFATTN_MODE_SUM         c = +lambda  (the two maps added)          */
typedef enum {
  DIFFATTN_MODE_DIFF = 0,
  DIFFATTN_MODE_LAMBDA_ZERO = 1,
  DIFFATTN_MODE_SUM = 2
} diffattn_mode;

/*
 * diffattn_fwd_mode -- diffattn_fwd with the combination of the two maps
 * chosen by `mode` (a diffattn_mode).  All other arguments, layouts and
 * errors are those of diffattn_fwd; an unknown mode gives
 * DIFFATTN_ERR_INVALID_ARG.  In DIFFATTN_MODE_LAMBDA_ZERO the lambda pointer
 * must still be valid (it is read, then multiplied by zero).
 */
int diffattn_fwd_mode(const void* q, const void* k, const void* v, void* o,
                      int dtype, int B, int N, int H, int d, int causal,
                      const float* lambda, float lambda_init, const float* rms_w,
                      float eps, int mode, cudaStream_t stream);

/*
 * Backward pass (training).  Gradients of diffattn_fwd_mode's output with
 * respect to q, k, v, lambda and the RMSNorm weight, for an upstream gradient
 * dy: the derivative of the DiffAttn equation (first page, the section with
 * the DiffAttn equation; peer review "Differential Transformer", Summary,
 * Eq. 1) and of the headwise RMSNorm and (1 - lambda_init) scale (Eq. 3).
 *
 * diffattn_bwd_workspace_size -- bytes of workspace for diffattn_bwd (0 for
 *   sizes below 1): fp32 [B, N, H, 2d] plus 16 bytes per (b, n, h).
 * diffattn_bwd
 *   q, k, v, dy : as in diffattn_fwd (dy has v's shape), dtype BF16 or F32
 *   lambda, lambda_init, rms_w, eps, causal, mode : as in diffattn_fwd_mode
 *   dq, dk      : device float32 [B, N, H, 2, d], written
 *   dv          : device float32 [B, N, H, 2d], written
 *   dlambda     : device float32 scalar, written (0 in DIFFATTN_MODE_LAMBDA_ZERO)
 *   drms_w      : device float32 [2d], written
 *   workspace   : device, >= diffattn_bwd_workspace_size bytes, 16-byte aligned
 * CUDA cores (fp32 arithmetic), 1 <= d <= 128.  Stream-ordered; dlambda and
 * drms_w are summed with atomics, so their last bits may vary from run to run.
 * Errors: DIFFATTN_ERR_INVALID_ARG, DIFFATTN_ERR_UNSUPPORTED (d > 128),
 * DIFFATTN_ERR_WORKSPACE, DIFFATTN_ERR_CUDA.
 */
size_t diffattn_bwd_workspace_size(int B, int N, int H, int d);
int diffattn_bwd(const void* q, const void* k, const void* v, const void* dy,
                 int dtype, int B, int N, int H, int d, int causal,
                 const float* lambda, float lambda_init, const float* rms_w,
                 float eps, int mode, float* dq, float* dk, float* dv,
                 float* dlambda, float* drms_w, void* workspace, size_t ws_bytes,
                 cudaStream_t stream);

/*
 * Tensor-core backward pass: the gradients diffattn_bwd defines, computed
 * with tcgen05 products from bf16 operands, as a training step would.
 * P, G = dO and dS are rounded to bf16 before each product (fp32
 * accumulation), so the gradients carry bf16-level errors (normwise about
 * 1e-3 relative) where diffattn_bwd carries fp32-level ones.
 *
 * diffattn_bwd_tc_workspace_size -- bytes of workspace for diffattn_bwd_tc
 *   (0 for sizes below 1): fp32 [B, N, H, 2, 2d] (each map's A_i V), bf16
 *   [B, N, H, 2d] (dO) and 16 bytes per (b, h, n) with n rounded up to 128.
 * diffattn_bwd_tc
 *   q, k        : device bf16 [B, N, H, 2, d], d = 64 or 128
 *   v, dy       : device bf16 [B, N, H, 2d]
 *   other arguments, outputs and layouts as in diffattn_bwd
 *   workspace   : device, >= diffattn_bwd_tc_workspace_size bytes, 16-byte aligned
 * Five stream-ordered launches: the prefill in a statistics mode (per map
 * A_i V and the log-sum-exp per row), a per-row pass for dO, dw and dlambda,
 * and one kernel each for dV, dK and dQ.  No allocation.  dlambda and drms_w
 * are summed with atomics (last bits may vary from run to run); dq, dk, dv
 * are deterministic.
 * Errors: DIFFATTN_ERR_INVALID_ARG (null or unaligned pointers, bad mode or
 * sizes), DIFFATTN_ERR_UNSUPPORTED (d other than 64 or 128),
 * DIFFATTN_ERR_WORKSPACE, DIFFATTN_ERR_CUDA; DIFFATTN_ERR_TIMEOUT through
 * diffattn_device_status if a kernel wait ran out.
 */
size_t diffattn_bwd_tc_workspace_size(int B, int N, int H, int d);

/*
 * Training pair: a forward that also saves what the tensor-core backward
 * needs, and the backward that uses it instead of recomputing it.
 *
 * diffattn_fwd_train -- diffattn_fwd_mode's output o (bf16, d = 64 or 128),
 *   and into `workspace` (>= diffattn_bwd_tc_workspace_size bytes) each map's
 *   A_i V (float32) and the log-sum-exp of every query row.  Other arguments
 *   and errors as in diffattn_fwd_mode; DIFFATTN_ERR_WORKSPACE as below.
 * diffattn_bwd_tc_saved -- diffattn_bwd_tc without its statistics pass: the
 *   workspace must hold what diffattn_fwd_train wrote for the same q, k, v,
 *   lambda and mask (the mode may differ: the statistics do not depend on it).
 *   Arguments, outputs and errors as in diffattn_bwd_tc.
 */
int diffattn_fwd_train(const void* q, const void* k, const void* v, void* o,
                       int B, int N, int H, int d, int causal,
                       const float* lambda, float lambda_init, const float* rms_w,
                       float eps, int mode, void* workspace, size_t ws_bytes,
                       cudaStream_t stream);
int diffattn_bwd_tc_saved(const void* q, const void* k, const void* v, const void* dy,
                          int B, int N, int H, int d, int causal,
                          const float* lambda, float lambda_init, const float* rms_w,
                          float eps, int mode, float* dq, float* dk, float* dv,
                          float* dlambda, float* drms_w, void* workspace, size_t ws_bytes,
                          cudaStream_t stream);
int diffattn_bwd_tc(const void* q, const void* k, const void* v, const void* dy,
                    int B, int N, int H, int d, int causal,
                    const float* lambda, float lambda_init, const float* rms_w,
                    float eps, int mode, float* dq, float* dk, float* dv,
                    float* dlambda, float* drms_w, void* workspace, size_t ws_bytes,
                    cudaStream_t stream);

/*
 * diffattn_lambda_bwd -- gradients of the lambda re-parameterisation (Eq. 2)
 * for a device dlambda: dlq1 = dlambda e1 lk1, dlk1 = dlambda e1 lq1,
 * dlq2 = -dlambda e2 lk2, dlk2 = -dlambda e2 lq2, with e1 = exp(lq1 . lk1),
 * e2 = exp(lq2 . lk2).  All device float32; vectors of length d (1..4096).
 */
int diffattn_lambda_bwd(const float* lq1, const float* lk1, const float* lq2,
                        const float* lk2, int d, const float* dlambda,
                        float* dlq1, float* dlk1, float* dlq2, float* dlk2,
                        cudaStream_t stream);

/*
 * The steps either side of the path (page "Differential attention", "How it's
 * wired (and why it's nearly free)": each head's query and key projections
 * split into halves Q1, K1 and Q2, K2; the layer sits in a standard
 * transformer block).  Rotary position embedding as in RoFormer (cited on
 * page "Differential Transformer", "Builds on"): consecutive channel pairs
 * (2j, 2j+1) of every d-wide Q1, Q2, K1, K2 rotated by the angle
 * n * base^(-2j/d) at the token's position n within its sequence.
 *
 * diffattn_rope_table -- table[n][j] = (cos, sin) of n * base^(-2j/d),
 *   computed in double precision and rounded to float32.
 *   table : device float32 [seq_len][d/2][2], written.  d even, seq_len >= 1.
 * diffattn_qkv_proj -- [Q | K | V] = X W_qkv^T on the tensor cores (fp32
 *   accumulation), RoPE applied to Q and K in the same kernel's epilogue,
 *   rounded to bf16 and written in the layouts diffattn_fwd reads:
 *   x      : device bf16 [B * N, d_model] (rows: batch-major tokens)
 *   w_qkv  : device bf16 [H*2*d + H*2*d + H*2d, d_model], a linear layer's
 *            weight (one row per output feature): W_q, then W_k, then W_v;
 *            W_q's rows ordered (head, map, channel), W_v's (head, channel)
 *   rope_table : from diffattn_rope_table for at least N positions, or NULL
 *            for no rotation
 *   q, k   : device bf16 [B, N, H, 2, d], written;  v : [B, N, H, 2d], written
 *   d_model a multiple of 64; d a multiple of 32.
 * diffattn_out_proj -- y[M, n_out] = o[M, K] w_o[n_out, K]^T (bf16 in and out,
 *   fp32 accumulation): the output projection of the heads' concatenated
 *   outputs (o = diffattn_fwd's output viewed as [B * N, H * 2d]).
 *   K a multiple of 64, n_out a multiple of 32.
 * All pointers 16-byte aligned; stream-ordered; no allocation.
 * Errors: DIFFATTN_ERR_INVALID_ARG (null or unaligned pointers, sizes),
 * DIFFATTN_ERR_UNSUPPORTED (sizes outside the multiples above),
 * DIFFATTN_ERR_CUDA; DIFFATTN_ERR_TIMEOUT through diffattn_device_status.
 */
int diffattn_rope_table(int seq_len, int d, double base, float* table, cudaStream_t stream);
int diffattn_qkv_proj(const void* x, const void* w_qkv, int B, int N, int d_model, int H, int d,
                      const float* rope_table, void* q, void* k, void* v, cudaStream_t stream);
int diffattn_out_proj(const void* o, const void* w_o, int M, int K, int n_out, void* y,
                      cudaStream_t stream);

/*
 * Low-bit queries and keys (peer review "Differential Transformer",
 * Strengths, the activation-outlier bullet, and Questions, the quantisation
 * bullet: absmax quantisation per logit map and per head).
 *
 * diffattn_quantize_qk -- e4m3 codes of a bf16 query or key tensor, with one
 * absmax scale per (batch, head, map):
 *
 *   scales[b][h][i] = max |x[b, :, h, i, :]| / 448   (float32; 1 if that max is 0)
 *   codes[b, n, h, i, c] = e4m3(x[b, n, h, i, c] / scales[b][h][i])
 *
 * where e4m3 is the OCP FP8 E4M3 encoding, round to nearest even, saturating
 * at +-448 (the largest finite value, where each group's absmax lands).
 * x      : bf16 [B, N, H, 2, d] (the q or k of diffattn_fwd)
 * codes  : device uint8 [B, N, H, 2, d], written
 * scales : device float32 [B][H][2], written (also used as scratch)
 * d must be a multiple of 8; B * H * 2 <= 65535.  Three stream-ordered
 * kernels and one memset; no allocation.
 * Errors: DIFFATTN_ERR_INVALID_ARG, DIFFATTN_ERR_UNSUPPORTED, DIFFATTN_ERR_CUDA.
 */
int diffattn_quantize_qk(const void* x, int B, int N, int H, int d, void* codes,
                         float* scales, cudaStream_t stream);

/*
 * diffattn_fwd_qk8 -- the prefill of diffattn_fwd_mode with the scores taken
 * from e4m3 queries and keys (codes and scales as diffattn_quantize_qk writes
 * them): S_i = (Qcodes_i Kcodes_i^T) * q_scale * k_scale / sqrt(d), on the
 * tensor cores' 8-bit path (fp32 accumulation).  P, V and the output stay
 * bf16; everything after the scores is as in diffattn_fwd_mode.
 * v, o : bf16 [B, N, H, 2d].  d must be 128 (DIFFATTN_ERR_UNSUPPORTED
 * otherwise).  Other arguments and errors as in diffattn_fwd_mode.
 */
int diffattn_fwd_qk8(const void* q_codes, const float* q_scales,
                     const void* k_codes, const float* k_scales,
                     const void* v, void* o, int B, int N, int H, int d, int causal,
                     const float* lambda, float lambda_init, const float* rms_w,
                     float eps, int mode, cudaStream_t stream);

/*
 * diffattn_quantize_qk4 -- 4-bit codes (the peer review's 4-bit
 * attention-logit quantisation, Fig. 8 of the paper): e2m1 codes of a bf16
 * query or key tensor, with one absmax scale per (batch, head, map):
 *
 *   scales[b][h][i] = max |x[b, :, h, i, :]| / 6   (float32; 1 if that max is 0)
 *   code(b, n, h, i, c) = e2m1(x[b, n, h, i, c] / scales[b][h][i])
 *
 * where e2m1 is the OCP Microscaling FP4 E2M1 encoding (bit 3 sign, 2
 * exponent bits with bias 1, 1 mantissa bit: magnitudes 0, 0.5, 1, 1.5, 2,
 * 3, 4, 6), round to nearest even, saturating at +-6.  Two codes per byte:
 * codes[b, n, h, i, j] = code(.., 2j) | code(.., 2j + 1) << 4.
 * x      : bf16 [B, N, H, 2, d]
 * codes  : device uint8 [B, N, H, 2, d / 2], written
 * scales : device float32 [B][H][2], written (also used as scratch)
 * d must be a multiple of 8; B * H * 2 <= 65535.  Three stream-ordered
 * kernels and one memset; no allocation.
 * Errors: DIFFATTN_ERR_INVALID_ARG, DIFFATTN_ERR_UNSUPPORTED, DIFFATTN_ERR_CUDA.
 */
int diffattn_quantize_qk4(const void* x, int B, int N, int H, int d, void* codes,
                          float* scales, cudaStream_t stream);

/*
 * diffattn_fwd_qk4 -- diffattn_fwd_qk8 with e2m1 query and key codes (as
 * diffattn_quantize_qk4 writes them, two per byte): the scores are a
 * tensor-core product of the 4-bit codes (fp32 accumulation, exact) times
 * q_scale * k_scale / sqrt(d).  q_codes and k_codes must be 32-byte aligned
 * (DIFFATTN_ERR_INVALID_ARG otherwise); d must be 128.  Other arguments and
 * errors as in diffattn_fwd_qk8.
 */
int diffattn_fwd_qk4(const void* q_codes, const float* q_scales,
                     const void* k_codes, const float* k_scales,
                     const void* v, void* o, int B, int N, int H, int d, int causal,
                     const float* lambda, float lambda_init, const float* rms_w,
                     float eps, int mode, cudaStream_t stream);

/*
 * diffattn_decode_workspace_size -- bytes of device workspace that
 * diffattn_decode needs for S sequences of at most max_seqlen cached keys.
 * Returns 0 for invalid sizes.
 */
size_t diffattn_decode_workspace_size(int S, int H, int d, int max_seqlen);

/*
 * diffattn_decode -- one decode step (query length 1) for S sequences over a
 * packed KV cache, with the same DiffAttn + RMSNorm + scale as diffattn_fwd.
 *
 * q          : [S, H, 2, d] bf16 (Q1 then Q2 per head)
 * k_cache    : [T, H, 2, d] bf16, sequences packed back to back
 * v_cache    : [T, H, 2d]   bf16
 * cu_seqlens : device int32[S + 1], cu_seqlens[0] = 0, non-decreasing;
 *              sequence s owns cache rows cu_seqlens[s] .. cu_seqlens[s+1]-1
 *              (its current token included) and its query sees all of them.
 *              Every length must be in [1, max_seqlen].
 * max_seqlen : host int, an upper bound on every sequence length
 * o          : [S, H, 2d] bf16 output
 * lambda, lambda_init, rms_w, eps : as in diffattn_fwd
 * workspace  : device buffer of >= diffattn_decode_workspace_size() bytes,
 *              16-byte aligned; its contents need no initialisation and
 *              are scratch after the call.  Two calls that overlap on the
 *              GPU must not share a workspace.
 * Supported: d = 128, bf16 only (DIFFATTN_ERR_UNSUPPORTED otherwise).
 * Errors: DIFFATTN_ERR_INVALID_ARG, DIFFATTN_ERR_WORKSPACE,
 * DIFFATTN_ERR_CUDA.  A length outside [1, max_seqlen] is not detected on
 * the host (cu_seqlens lives on the device): the kernel skips keys beyond
 * max_seqlen and writes NaN for an empty sequence; the debug build also
 * records DIFFATTN_ERR_BOUNDS for a length above max_seqlen, and skips a
 * sequence whose offsets fall outside [0, cu_seqlens[S]].
 * Work layout: a planning kernel turns cu_seqlens into each sequence's
 * ceil(L / 512) key chunks, so the kernels visit only chunks that exist
 * (a long sequence among short ones costs its own keys, not S times them).
 */
int diffattn_decode(const void* q, const void* k_cache, const void* v_cache,
                    const int* cu_seqlens, int max_seqlen, void* o, int S,
                    int H, int d, const float* lambda, float lambda_init,
                    const float* rms_w, float eps, void* workspace,
                    size_t ws_bytes, cudaStream_t stream);

/*
 * diffattn_decode_mode -- diffattn_decode with the combination of the two
 * maps chosen by `mode` (a diffattn_mode, as in diffattn_fwd_mode).  Other
 * arguments, layouts and errors are those of diffattn_decode; an unknown mode
 * gives DIFFATTN_ERR_INVALID_ARG.
 */
int diffattn_decode_mode(const void* q, const void* k_cache, const void* v_cache,
                         const int* cu_seqlens, int max_seqlen, void* o, int S,
                         int H, int d, const float* lambda, float lambda_init,
                         const float* rms_w, float eps, int mode, void* workspace,
                         size_t ws_bytes, cudaStream_t stream);

/*
 * diffattn_decode_noalloc -- diffattn_decode for callers that cannot
 * allocate device memory.  The paper has no counterpart: this is a
 * deployment variant of the same computation, with the same arguments as
 * diffattn_decode except the workspace.
 *
 * Who needs it: callers that are not allowed to call cudaMalloc, for example
 * a plugin inside an inference engine that owns all device memory through
 * its own pool, or a serving loop that must never enter the driver's
 * allocator.  They cannot hand diffattn_decode a workspace, so this call
 * uses a scratch array that the library defines in device memory
 * (DIFFATTN_DECODE_NOALLOC_SCRATCH_BYTES = 16 MiB).  The call itself
 * allocates nothing.  Every GPU that loads the library holds that array
 * until the process exits.
 *
 *  - Limit: problems with diffattn_decode_workspace_size(S, H, d,
 *    max_seqlen) > DIFFATTN_DECODE_NOALLOC_SCRATCH_BYTES are rejected with
 *    DIFFATTN_ERR_WORKSPACE before anything is launched (at d = 128 the size
 *    is 2064 * S * H * ceil(max_seqlen / 512) bytes plus the S + 1 chunk
 *    offsets, so S * H * ceil(max_seqlen / 512) must stay a little under
 *    8128).
 *  - Set-up: the first call on each device looks up the array's device
 *    address (cudaGetSymbolAddress, with that device current).  Make that
 *    first call before any stream capture.  The address is kept per device
 *    and context: after cudaDeviceReset the next call (again before any
 *    capture) looks it up in the new context.
 *  - Sharing: every call on a device uses the same array, which keeps the
 *    last call's contents.  Two calls that overlap on the GPU (on different
 *    streams, or from different host threads) race on it; the caller must
 *    order them.  Nothing needs clearing between calls: the kernels write
 *    every scratch entry before they read it.
 * Other errors as diffattn_decode.
 */
#define DIFFATTN_DECODE_NOALLOC_SCRATCH_BYTES (16u << 20)
int diffattn_decode_noalloc(const void* q, const void* k_cache,
                            const void* v_cache, const int* cu_seqlens,
                            int max_seqlen, void* o, int S, int H, int d,
                            const float* lambda, float lambda_init,
                            const float* rms_w, float eps,
                            cudaStream_t stream);

/*
 * diffattn_device_status -- synchronises the current device, then returns
 * the device-side status word (DIFFATTN_OK, DIFFATTN_ERR_TIMEOUT, or in the
 * debug build DIFFATTN_ERR_BOUNDS) in *status_out and clears it.  Returns DIFFATTN_ERR_CUDA if the device could
 * not be queried.
 */
int diffattn_device_status(int* status_out);

/*
 * diffattn_set_wait_limit_ns -- upper bound, in nanoseconds, on every
 * pipeline wait inside the library's kernels (default 2e9, i.e. 2 s; 0
 * restores the default).  When a wait runs out, the kernel records
 * DIFFATTN_ERR_TIMEOUT in the device status word, stops its pipeline,
 * releases its tensor memory and returns, leaving the context usable.
 * Applies to launches made after the call.
 */
int diffattn_set_wait_limit_ns(long long limit_ns);

/* Human-readable name of a diffattn_status code. */
const char* diffattn_status_string(int status);

/* Library ABI version (major * 100 + minor); 101 adds the 4-bit pair
 * diffattn_quantize_qk4 / diffattn_fwd_qk4 to 100. */
int diffattn_version(void);

#ifdef __cplusplus
}
#endif
#endif /* DIFFATTN_H_ */
