// C-ABI entry points declared in include/diffattn.h: argument validation,
// TMA descriptor encoding, the device status word, and dispatch to the
// kernels.  No device memory is allocated here.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "diffattn.h"
#include "internal.h"

namespace diffattn {
namespace {

// Device-side status word: kernels record DIFFATTN_ERR_TIMEOUT here.
__device__ int g_status_word = 0;

constexpr int kMaxDevices = 64;
struct StatusSlot {
  int* ptr;
  unsigned long long ctx;  // context the address belongs to
};
StatusSlot g_status_slot[kMaxDevices] = {};
std::mutex g_mu;
std::atomic<unsigned long long> g_wait_limit_ns{2000000000ull};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int cuda_status(cudaError_t e) { return e == cudaSuccess ? DIFFATTN_OK : DIFFATTN_ERR_CUDA; }

// Address of this device's status word: looked up on the first call in each
// context of the device (again after a cudaDeviceReset), or on every call when
// the context id cannot be read.  The device and context id are reported too
// (dev, ctx may be null), so that a launcher need not look them up again.
cudaError_t status_ptr(int** out, int* dev_out = nullptr, unsigned long long* ctx_out = nullptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  const unsigned long long ctx = current_context_id();
  StatusSlot& slot = g_status_slot[dev];
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!slot.ptr || ctx == 0 || slot.ctx != ctx) {
      void* p = nullptr;
      e = cudaGetSymbolAddress(&p, g_status_word);
      if (e != cudaSuccess) return e;
      slot.ptr = static_cast<int*>(p);
      slot.ctx = ctx;
    }
    *out = slot.ptr;
  }
  if (dev_out) *dev_out = dev;
  if (ctx_out) *ctx_out = ctx;
  return cudaSuccess;
}

// The status word, wait limit, device and context of a launch.
cudaError_t dev_ctl(DevCtl* c) {
  c->limit_ns = g_wait_limit_ns.load();
  return status_ptr(&c->status, &c->dev, &c->ctx);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Encoded tensor maps, kept per (base address, dims, element type, box): a
// map is a pure function of those, so a cached one is valid whenever they
// match (even for a new allocation that reuses the address).  A small table
// with least-recently-used replacement keeps the host cost of a repeated call
// to a lookup instead of a driver call per map.
struct MapKey {
  const void* base;
  uint64_t d[4];
  int kind;      // 1: uint8, 2: bf16, 4: packed e2m1
  int box_rows;
  bool operator==(const MapKey& o) const {
    return base == o.base && d[0] == o.d[0] && d[1] == o.d[1] && d[2] == o.d[2] && d[3] == o.d[3] &&
           kind == o.kind && box_rows == o.box_rows;
  }
};
struct MapSlot {
  MapKey key;
  CUtensorMap map;
  unsigned long long used;  // 0: empty
};
constexpr int kMapSlots = 64;
MapSlot g_map_slots[kMapSlots];
unsigned long long g_map_clock = 0;
std::mutex g_map_mu;

bool encode_uncached(CUtensorMap* m, const MapKey& k) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[4] = {k.d[0], k.d[1], k.d[2], k.d[3]};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  if (k.kind == 4) {
    // packed e2m1 codes: d0 codes (two per byte; d0 a multiple of 128); box =
    // 128 codes x 1 x 128 rows x 1, widened to 128 bytes a row in shared
    // memory (8 bytes of codes, then 8 bytes of gap, per 16 codes)
    const cuuint64_t strides[3] = {k.d[0] / 2, k.d[0] / 2 * k.d[1], k.d[0] / 2 * k.d[1] * k.d[2]};
    const cuuint32_t box[4] = {128, 1, 128, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 4, const_cast<void*>(k.base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  }
  const uint64_t e = static_cast<uint64_t>(k.kind);
  const cuuint64_t strides[3] = {k.d[0] * e, k.d[0] * k.d[1] * e, k.d[0] * k.d[1] * k.d[2] * e};
  const cuuint32_t box[4] = {static_cast<cuuint32_t>(128 / e), 1, static_cast<cuuint32_t>(k.box_rows), 1};
  return fn(m, e == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 4,
            const_cast<void*>(k.base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Slot of a key: a hash of its fields picks one of two neighbouring slots
// (the other one on a miss when the first is taken), so a lookup compares at
// most two keys.
size_t map_slot(const MapKey& k) {
  uint64_t h = reinterpret_cast<uintptr_t>(k.base) * 0x9E3779B97F4A7C15ull;
  for (int i = 0; i < 4; ++i) h = (h ^ k.d[i]) * 0x100000001B3ull;
  h ^= static_cast<uint64_t>(k.kind) * 31 + static_cast<uint64_t>(k.box_rows);
  return static_cast<size_t>((h >> 29) % (kMapSlots / 2)) * 2;
}

bool encode_cached(CUtensorMap* m, const MapKey& k) {
  const size_t i = map_slot(k);
  std::lock_guard<std::mutex> lk(g_map_mu);
  for (size_t j = i; j < i + 2; ++j) {
    MapSlot& s = g_map_slots[j];
    if (s.used && s.key == k) {
      s.used = ++g_map_clock;
      *m = s.map;
      return true;
    }
  }
  if (!encode_uncached(m, k)) return false;
  // replace the less recently used of the two
  MapSlot& v = g_map_slots[g_map_slots[i].used <= g_map_slots[i + 1].used ? i : i + 1];
  v.key = k;
  v.map = *m;
  v.used = ++g_map_clock;
  return true;
}

// 4-D map over a row-major tensor with dims (innermost first) d0..d3 of bf16
// (esize 2) or byte (esize 1) elements; box = 128 bytes x 1 x box_rows x 1,
// 128-byte swizzle, zero fill out of bounds.
bool encode_4d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t d3,
               int esize = 2, int box_rows = 128) {
  return encode_cached(m, MapKey{base, {d0, d1, d2, d3}, esize, box_rows});
}

// 4-D map over packed e2m1 codes, dims (innermost first) d0 codes (two per
// byte; d0 a multiple of 128), d1..d3; box = 128 codes x 1 x 128 rows x 1,
// widened to 128 bytes a row in shared memory.  The base must be 32-byte
// aligned and every stride a multiple of 32 bytes.
bool encode_4d_e2m1(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t d3) {
  return encode_cached(m, MapKey{base, {d0, d1, d2, d3}, 4, 128});
}

bool fits_i32(long long x) { return x >= 0 && x < (1ll << 31); }

bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

int quantize_impl(const void* x, int B, int N, int H, int d, int bits, void* codes, float* scales,
                  cudaStream_t stream) {
  if (B < 1 || H < 1 || N < 1 || d < 8 || d % 8 != 0) return DIFFATTN_ERR_INVALID_ARG;
  if (!fits_i32(static_cast<long long>(B) * N * H * 2 * d)) return DIFFATTN_ERR_INVALID_ARG;
  if (!x || !codes || !scales) return DIFFATTN_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(codes) || !aligned16(scales)) return DIFFATTN_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * H * 2 > 65535) return DIFFATTN_ERR_UNSUPPORTED;
  return cuda_status(launch_quantize_qk(x, B, N, H, d, bits, codes, scales, stream));
}

// The prefill on low-bit query and key codes: bits 8 (e4m3) or 4 (packed e2m1).
int fwd_lowbit_impl(int bits, const void* q_codes, const float* q_scales, const void* k_codes,
                    const float* k_scales, const void* v, void* o, int B, int N, int H, int d, int causal,
                    const float* lambda, float lambda_init, const float* rms_w, float eps, int mode,
                    cudaStream_t stream) {
  if (B < 1 || H < 1 || N < 0 || d < 1 || !(eps >= 0.f)) return DIFFATTN_ERR_INVALID_ARG;
  if (mode != DIFFATTN_MODE_DIFF && mode != DIFFATTN_MODE_LAMBDA_ZERO && mode != DIFFATTN_MODE_SUM)
    return DIFFATTN_ERR_INVALID_ARG;
  if (!fits_i32(static_cast<long long>(B) * N * H * 2 * d)) return DIFFATTN_ERR_INVALID_ARG;
  if (N == 0) return DIFFATTN_OK;
  if (!q_codes || !q_scales || !k_codes || !k_scales || !v || !o || !lambda || !rms_w)
    return DIFFATTN_ERR_INVALID_ARG;
  if (!aligned16(q_codes) || !aligned16(k_codes) || !aligned16(v) || !aligned16(o)) return DIFFATTN_ERR_INVALID_ARG;
  if (bits == 4 && (!aligned32(q_codes) || !aligned32(k_codes))) return DIFFATTN_ERR_INVALID_ARG;
  if (d != 128) return DIFFATTN_ERR_UNSUPPORTED;
  if (B > 65535 || H > 65535) return DIFFATTN_ERR_UNSUPPORTED;
  CUtensorMap tq, tk, tv, to;
  const bool codes_ok = bits == 4 ? encode_4d_e2m1(&tq, q_codes, d, 2ull * H, N, B) &&
                                        encode_4d_e2m1(&tk, k_codes, d, 2ull * H, N, B)
                                  : encode_4d(&tq, q_codes, d, 2ull * H, N, B, 1) &&
                                        encode_4d(&tk, k_codes, d, 2ull * H, N, B, 1);
  if (!codes_ok || !encode_4d(&tv, v, 2ull * d, H, N, B) || !encode_4d(&to, o, 2ull * d, H, N, B))
    return DIFFATTN_ERR_CUDA;
  DevCtl ctl;
  if (dev_ctl(&ctl) != cudaSuccess) return DIFFATTN_ERR_CUDA;
  return cuda_status(launch_prefill_sm100(tq, tk, tv, to, o, B, N, H, d, causal, lambda, lambda_init, rms_w, eps,
                                          mode, q_scales, k_scales, bits, ctl, stream));
}

// A projection GEMM through launch_proj_gemm, with the maps over A [M, K] and B [n_total, K].
int proj_launch(const void* a, const void* b, int M, int K, int n_total, ProjParams& prm, cudaStream_t stream) {
  CUtensorMap ta, tb;  // 2-SM tiles: each CTA of a pair loads 128 rows of A and 128 rows of B
  if (!encode_4d(&ta, a, K, 1, M, 1, 2, 128) || !encode_4d(&tb, b, K, 1, n_total, 1, 2, 128)) return DIFFATTN_ERR_CUDA;
  DevCtl ctl;
  if (status_ptr(&ctl.status) != cudaSuccess) return DIFFATTN_ERR_CUDA;
  prm.M = M;
  prm.N = n_total;
  prm.K = K;
  prm.status = ctl.status;
  prm.limit_ns = g_wait_limit_ns.load();
  return cuda_status(launch_proj_gemm(ta, tb, prm, stream));
}

// diffattn_bwd_tc and diffattn_bwd_tc_saved: the same checks and maps; `saved`
// skips the statistics pass (the workspace already holds them).
int bwd_tc_impl(const void* q, const void* k, const void* v, const void* dy, int B, int N, int H, int d, int causal,
                const float* lambda, float lambda_init, const float* rms_w, float eps, int mode, float* dq, float* dk,
                float* dv, float* dlambda, float* drms_w, void* workspace, size_t ws_bytes, bool saved,
                cudaStream_t stream) {
  if (B < 1 || H < 1 || N < 1 || d < 1 || !(eps >= 0.f)) return DIFFATTN_ERR_INVALID_ARG;
  if (mode != DIFFATTN_MODE_DIFF && mode != DIFFATTN_MODE_LAMBDA_ZERO && mode != DIFFATTN_MODE_SUM)
    return DIFFATTN_ERR_INVALID_ARG;
  if (!fits_i32(static_cast<long long>(B) * N * H * 2 * d)) return DIFFATTN_ERR_INVALID_ARG;
  if (!q || !k || !v || !dy || !lambda || !rms_w || !dq || !dk || !dv || !dlambda || !drms_w)
    return DIFFATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dy) || !aligned16(dq) || !aligned16(dk) ||
      !aligned16(dv))
    return DIFFATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return DIFFATTN_ERR_UNSUPPORTED;
  if (B > 65535 || H > 65535) return DIFFATTN_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * H * ((N + 127) / 128) > 0x7fffffffll) return DIFFATTN_ERR_UNSUPPORTED;
  const BwdTcLayout L = bwd_tc_layout(B, N, H, d);
  if (!workspace || ws_bytes < L.bytes || !aligned16(workspace)) return DIFFATTN_ERR_WORKSPACE;
  const void* g = static_cast<const char*>(workspace) + L.off_g;
  BwdTcMaps m;
  if (!encode_4d(&m.q128, q, d, 2ull * H, N, B) || !encode_4d(&m.q32, q, d, 2ull * H, N, B, 2, 32) ||
      !encode_4d(&m.k128, k, d, 2ull * H, N, B) || !encode_4d(&m.k32, k, d, 2ull * H, N, B, 2, 32) ||
      !encode_4d(&m.v128, v, 2ull * d, H, N, B) || !encode_4d(&m.v32, v, 2ull * d, H, N, B, 2, 32) ||
      !encode_4d(&m.g128, g, 2ull * d, H, N, B) || !encode_4d(&m.g32, g, 2ull * d, H, N, B, 2, 32) ||
      !encode_4d(&m.q64, q, d, 2ull * H, N, B, 2, 64) || !encode_4d(&m.g64, g, 2ull * d, H, N, B, 2, 64))
    return DIFFATTN_ERR_CUDA;
  DevCtl ctl;
  if (status_ptr(&ctl.status) != cudaSuccess) return DIFFATTN_ERR_CUDA;
  ctl.limit_ns = g_wait_limit_ns.load();
  return cuda_status(launch_bwd_sm100(m, dy, B, N, H, d, causal, lambda, lambda_init, rms_w, eps, mode, dq, dk, dv,
                                      dlambda, drms_w, workspace, saved, ctl, stream));
}
}  // namespace

int* status_word() {
  int* p = nullptr;
  return status_ptr(&p) == cudaSuccess ? p : nullptr;
}

unsigned long long current_context_id() {
  typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
  typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  if (!get_current || !get_id) return 0;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  unsigned long long id = 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

}  // namespace diffattn

using namespace diffattn;

extern "C" {

int diffattn_version(void) { return 101; }  // 1.01: adds diffattn_quantize_qk4 and diffattn_fwd_qk4

const char* diffattn_status_string(int s) {
  switch (s) {
    case DIFFATTN_OK: return "ok";
    case DIFFATTN_ERR_INVALID_ARG: return "invalid argument";
    case DIFFATTN_ERR_UNSUPPORTED: return "unsupported dtype or size";
    case DIFFATTN_ERR_CUDA: return "CUDA error";
    case DIFFATTN_ERR_TIMEOUT: return "a kernel wait timed out";
    case DIFFATTN_ERR_WORKSPACE: return "workspace missing or too small";
    case DIFFATTN_ERR_BOUNDS: return "an index was out of range (debug build; the access was skipped)";
    default: return "unknown status";
  }
}

int diffattn_set_wait_limit_ns(long long limit_ns) {
  if (limit_ns < 0) return DIFFATTN_ERR_INVALID_ARG;
  g_wait_limit_ns.store(limit_ns == 0 ? 2000000000ull : static_cast<unsigned long long>(limit_ns));
  return DIFFATTN_OK;
}

int diffattn_device_status(int* status_out) {
  if (!status_out) return DIFFATTN_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return DIFFATTN_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_status_word, sizeof(int)) != cudaSuccess) return DIFFATTN_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_status_word, &zero, sizeof(int)) != cudaSuccess) return DIFFATTN_ERR_CUDA;
  *status_out = v;
  return DIFFATTN_OK;
}

int diffattn_lambda(const float* lq1, const float* lk1, const float* lq2, const float* lk2, int d,
                    float lambda_init, float* lambda_out, cudaStream_t stream) {
  if (!lq1 || !lk1 || !lq2 || !lk2 || !lambda_out) return DIFFATTN_ERR_INVALID_ARG;
  if (d < 1 || d > 4096) return DIFFATTN_ERR_INVALID_ARG;
  return cuda_status(launch_lambda(lq1, lk1, lq2, lk2, d, lambda_init, lambda_out, stream));
}

int diffattn_fwd(const void* q, const void* k, const void* v, void* o, int dtype, int B, int N, int H, int d,
                 int causal, const float* lambda, float lambda_init, const float* rms_w, float eps,
                 cudaStream_t stream) {
  return diffattn_fwd_mode(q, k, v, o, dtype, B, N, H, d, causal, lambda, lambda_init, rms_w, eps,
                           DIFFATTN_MODE_DIFF, stream);
}

int diffattn_fwd_mode(const void* q, const void* k, const void* v, void* o, int dtype, int B, int N, int H,
                      int d, int causal, const float* lambda, float lambda_init, const float* rms_w, float eps,
                      int mode, cudaStream_t stream) {
  if (B < 1 || H < 1 || N < 0 || d < 1 || !(eps >= 0.f)) return DIFFATTN_ERR_INVALID_ARG;
  if (mode != DIFFATTN_MODE_DIFF && mode != DIFFATTN_MODE_LAMBDA_ZERO && mode != DIFFATTN_MODE_SUM)
    return DIFFATTN_ERR_INVALID_ARG;
  if (dtype != DIFFATTN_F32 && dtype != DIFFATTN_BF16) return DIFFATTN_ERR_INVALID_ARG;
  if (!fits_i32(static_cast<long long>(B) * N * H * 2 * d)) return DIFFATTN_ERR_INVALID_ARG;
  if (N == 0) return DIFFATTN_OK;
  if (!q || !k || !v || !o || !lambda || !rms_w) return DIFFATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return DIFFATTN_ERR_INVALID_ARG;
  if (B > 65535 || H > 65535) return DIFFATTN_ERR_UNSUPPORTED;
  if (dtype == DIFFATTN_F32) {
    if (d > 128) return DIFFATTN_ERR_UNSUPPORTED;
    return cuda_status(launch_prefill_simt_f32(static_cast<const float*>(q), static_cast<const float*>(k),
                                               static_cast<const float*>(v), static_cast<float*>(o), B, N, H, d,
                                               causal, lambda, lambda_init, rms_w, eps, mode, stream));
  }
  if (d != 64 && d != 128) return DIFFATTN_ERR_UNSUPPORTED;
  CUtensorMap tq, tk, tv, to;
  if (!encode_4d(&tq, q, d, 2ull * H, N, B) || !encode_4d(&tk, k, d, 2ull * H, N, B) ||
      !encode_4d(&tv, v, 2ull * d, H, N, B) || !encode_4d(&to, o, 2ull * d, H, N, B))
    return DIFFATTN_ERR_CUDA;
  DevCtl ctl;
  if (dev_ctl(&ctl) != cudaSuccess) return DIFFATTN_ERR_CUDA;
  return cuda_status(
      launch_prefill_sm100(tq, tk, tv, to, o, B, N, H, d, causal, lambda, lambda_init, rms_w, eps, mode, nullptr,
                           nullptr, 16, ctl, stream));
}

int diffattn_quantize_qk(const void* x, int B, int N, int H, int d, void* codes, float* scales,
                         cudaStream_t stream) {
  return quantize_impl(x, B, N, H, d, 8, codes, scales, stream);
}

int diffattn_quantize_qk4(const void* x, int B, int N, int H, int d, void* codes, float* scales,
                          cudaStream_t stream) {
  return quantize_impl(x, B, N, H, d, 4, codes, scales, stream);
}

int diffattn_fwd_qk8(const void* q_codes, const float* q_scales, const void* k_codes, const float* k_scales,
                     const void* v, void* o, int B, int N, int H, int d, int causal, const float* lambda,
                     float lambda_init, const float* rms_w, float eps, int mode, cudaStream_t stream) {
  return fwd_lowbit_impl(8, q_codes, q_scales, k_codes, k_scales, v, o, B, N, H, d, causal, lambda, lambda_init,
                         rms_w, eps, mode, stream);
}

int diffattn_fwd_qk4(const void* q_codes, const float* q_scales, const void* k_codes, const float* k_scales,
                     const void* v, void* o, int B, int N, int H, int d, int causal, const float* lambda,
                     float lambda_init, const float* rms_w, float eps, int mode, cudaStream_t stream) {
  return fwd_lowbit_impl(4, q_codes, q_scales, k_codes, k_scales, v, o, B, N, H, d, causal, lambda, lambda_init,
                         rms_w, eps, mode, stream);
}

size_t diffattn_bwd_workspace_size(int B, int N, int H, int d) {
  if (B < 1 || N < 1 || H < 1 || d < 1) return 0;
  return bwd_workspace_bytes(B, N, H, d);
}

int diffattn_bwd(const void* q, const void* k, const void* v, const void* dy, int dtype, int B, int N, int H, int d,
                 int causal, const float* lambda, float lambda_init, const float* rms_w, float eps, int mode,
                 float* dq, float* dk, float* dv, float* dlambda, float* drms_w, void* workspace, size_t ws_bytes,
                 cudaStream_t stream) {
  if (B < 1 || H < 1 || N < 1 || d < 1 || !(eps >= 0.f)) return DIFFATTN_ERR_INVALID_ARG;
  if (dtype != DIFFATTN_F32 && dtype != DIFFATTN_BF16) return DIFFATTN_ERR_INVALID_ARG;
  if (mode != DIFFATTN_MODE_DIFF && mode != DIFFATTN_MODE_LAMBDA_ZERO && mode != DIFFATTN_MODE_SUM)
    return DIFFATTN_ERR_INVALID_ARG;
  if (!fits_i32(static_cast<long long>(B) * N * H * 2 * d)) return DIFFATTN_ERR_INVALID_ARG;
  if (!q || !k || !v || !dy || !lambda || !rms_w || !dq || !dk || !dv || !dlambda || !drms_w)
    return DIFFATTN_ERR_INVALID_ARG;
  if (d > 128) return DIFFATTN_ERR_UNSUPPORTED;
  if (B > 65535 || H > 65535) return DIFFATTN_ERR_UNSUPPORTED;
  if (!workspace || ws_bytes < bwd_workspace_bytes(B, N, H, d) || !aligned16(workspace))
    return DIFFATTN_ERR_WORKSPACE;
  return cuda_status(launch_bwd(q, k, v, dy, dtype == DIFFATTN_BF16, B, N, H, d, causal, lambda, lambda_init,
                                rms_w, eps, mode, dq, dk, dv, dlambda, drms_w, workspace, stream));
}

size_t diffattn_bwd_tc_workspace_size(int B, int N, int H, int d) {
  if (B < 1 || N < 1 || H < 1 || d < 1) return 0;
  return bwd_tc_layout(B, N, H, d).bytes;
}


int diffattn_bwd_tc(const void* q, const void* k, const void* v, const void* dy, int B, int N, int H, int d,
                    int causal, const float* lambda, float lambda_init, const float* rms_w, float eps, int mode,
                    float* dq, float* dk, float* dv, float* dlambda, float* drms_w, void* workspace,
                    size_t ws_bytes, cudaStream_t stream) {
  return bwd_tc_impl(q, k, v, dy, B, N, H, d, causal, lambda, lambda_init, rms_w, eps, mode, dq, dk, dv, dlambda,
                     drms_w, workspace, ws_bytes, false, stream);
}

int diffattn_bwd_tc_saved(const void* q, const void* k, const void* v, const void* dy, int B, int N, int H, int d,
                          int causal, const float* lambda, float lambda_init, const float* rms_w, float eps, int mode,
                          float* dq, float* dk, float* dv, float* dlambda, float* drms_w, void* workspace,
                          size_t ws_bytes, cudaStream_t stream) {
  return bwd_tc_impl(q, k, v, dy, B, N, H, d, causal, lambda, lambda_init, rms_w, eps, mode, dq, dk, dv, dlambda,
                     drms_w, workspace, ws_bytes, true, stream);
}

int diffattn_fwd_train(const void* q, const void* k, const void* v, void* o, int B, int N, int H, int d, int causal,
                       const float* lambda, float lambda_init, const float* rms_w, float eps, int mode, void* workspace,
                       size_t ws_bytes, cudaStream_t stream) {
  if (B < 1 || H < 1 || N < 1 || d < 1 || !(eps >= 0.f)) return DIFFATTN_ERR_INVALID_ARG;
  if (mode != DIFFATTN_MODE_DIFF && mode != DIFFATTN_MODE_LAMBDA_ZERO && mode != DIFFATTN_MODE_SUM)
    return DIFFATTN_ERR_INVALID_ARG;
  if (!fits_i32(static_cast<long long>(B) * N * H * 2 * d)) return DIFFATTN_ERR_INVALID_ARG;
  if (!q || !k || !v || !o || !lambda || !rms_w) return DIFFATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return DIFFATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return DIFFATTN_ERR_UNSUPPORTED;
  if (B > 65535 || H > 65535) return DIFFATTN_ERR_UNSUPPORTED;
  const BwdTcLayout L = bwd_tc_layout(B, N, H, d);
  if (!workspace || ws_bytes < L.bytes || !aligned16(workspace)) return DIFFATTN_ERR_WORKSPACE;
  CUtensorMap tq, tk, tv, to;
  if (!encode_4d(&tq, q, d, 2ull * H, N, B) || !encode_4d(&tk, k, d, 2ull * H, N, B) ||
      !encode_4d(&tv, v, 2ull * d, H, N, B) || !encode_4d(&to, o, 2ull * d, H, N, B))
    return DIFFATTN_ERR_CUDA;
  DevCtl ctl;
  if (status_ptr(&ctl.status) != cudaSuccess) return DIFFATTN_ERR_CUDA;
  ctl.limit_ns = g_wait_limit_ns.load();
  char* ws = static_cast<char*>(workspace);
  return cuda_status(launch_prefill_sm100_stats(tq, tk, tv, &to, o, B, N, H, d, causal, lambda, lambda_init, rms_w,
                                                eps, mode, reinterpret_cast<float*>(ws + L.off_omaps),
                                                reinterpret_cast<float*>(ws + L.off_stats), L.n_pad, ctl, stream));
}

int diffattn_rope_table(int seq_len, int d, double base, float* table, cudaStream_t stream) {
  if (seq_len < 1 || d < 2 || d % 2 || !(base > 0.0) || !table) return DIFFATTN_ERR_INVALID_ARG;
  if (!fits_i32(static_cast<long long>(seq_len) * d)) return DIFFATTN_ERR_INVALID_ARG;
  return cuda_status(launch_rope_table(seq_len, d, base, table, stream));
}


int diffattn_qkv_proj(const void* x, const void* w_qkv, int B, int N, int d_model, int H, int d,
                      const float* rope_table, void* q, void* k, void* v, cudaStream_t stream) {
  if (B < 1 || N < 1 || d_model < 1 || H < 1 || d < 1) return DIFFATTN_ERR_INVALID_ARG;
  if (!x || !w_qkv || !q || !k || !v) return DIFFATTN_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_qkv) || !aligned16(q) || !aligned16(k) || !aligned16(v) ||
      (rope_table && !aligned16(rope_table)))
    return DIFFATTN_ERR_INVALID_ARG;
  const long long hq = 2ll * H * d;
  if (!fits_i32(static_cast<long long>(B) * N * d_model) || !fits_i32(3 * hq * d_model) ||
      !fits_i32(static_cast<long long>(B) * N * 3 * hq))
    return DIFFATTN_ERR_INVALID_ARG;
  if (d_model % 64 || d % 32) return DIFFATTN_ERR_UNSUPPORTED;
  ProjParams prm = {};
  prm.seq_len = N;
  prm.d = d;
  prm.rope = reinterpret_cast<const float2*>(rope_table);
  prm.rope_end = static_cast<int>(2 * hq);
  prm.col_end[0] = static_cast<int>(hq);
  prm.col_end[1] = static_cast<int>(2 * hq);
  prm.col_end[2] = static_cast<int>(3 * hq);
  prm.out[0] = static_cast<__nv_bfloat16*>(q);
  prm.out[1] = static_cast<__nv_bfloat16*>(k);
  prm.out[2] = static_cast<__nv_bfloat16*>(v);
  return proj_launch(x, w_qkv, B * N, d_model, static_cast<int>(3 * hq), prm, stream);
}

int diffattn_out_proj(const void* o, const void* w_o, int M, int K, int n_out, void* y, cudaStream_t stream) {
  if (M < 1 || K < 1 || n_out < 1) return DIFFATTN_ERR_INVALID_ARG;
  if (!o || !w_o || !y) return DIFFATTN_ERR_INVALID_ARG;
  if (!aligned16(o) || !aligned16(w_o) || !aligned16(y)) return DIFFATTN_ERR_INVALID_ARG;
  if (!fits_i32(static_cast<long long>(M) * K) || !fits_i32(static_cast<long long>(n_out) * K) ||
      !fits_i32(static_cast<long long>(M) * n_out))
    return DIFFATTN_ERR_INVALID_ARG;
  if (K % 64 || n_out % 32) return DIFFATTN_ERR_UNSUPPORTED;
  ProjParams prm = {};
  prm.seq_len = 1;
  prm.d = 32;
  prm.rope = nullptr;
  prm.rope_end = 0;
  prm.col_end[0] = prm.col_end[1] = prm.col_end[2] = n_out;
  prm.out[0] = prm.out[1] = prm.out[2] = static_cast<__nv_bfloat16*>(y);
  return proj_launch(o, w_o, M, K, n_out, prm, stream);
}

int diffattn_lambda_bwd(const float* lq1, const float* lk1, const float* lq2, const float* lk2, int d,
                        const float* dlambda, float* dlq1, float* dlk1, float* dlq2, float* dlk2,
                        cudaStream_t stream) {
  if (!lq1 || !lk1 || !lq2 || !lk2 || !dlambda || !dlq1 || !dlk1 || !dlq2 || !dlk2) return DIFFATTN_ERR_INVALID_ARG;
  if (d < 1 || d > 4096) return DIFFATTN_ERR_INVALID_ARG;
  return cuda_status(launch_lambda_bwd(lq1, lk1, lq2, lk2, d, dlambda, dlq1, dlk1, dlq2, dlk2, stream));
}

size_t diffattn_decode_workspace_size(int S, int H, int d, int max_seqlen) {
  return decode_workspace_bytes(S, H, d, max_seqlen);
}

int diffattn_decode(const void* q, const void* k_cache, const void* v_cache, const int* cu_seqlens, int max_seqlen,
                    void* o, int S, int H, int d, const float* lambda, float lambda_init, const float* rms_w,
                    float eps, void* workspace, size_t ws_bytes, cudaStream_t stream) {
  return diffattn_decode_mode(q, k_cache, v_cache, cu_seqlens, max_seqlen, o, S, H, d, lambda, lambda_init, rms_w,
                              eps, DIFFATTN_MODE_DIFF, workspace, ws_bytes, stream);
}

int diffattn_decode_mode(const void* q, const void* k_cache, const void* v_cache, const int* cu_seqlens,
                         int max_seqlen, void* o, int S, int H, int d, const float* lambda, float lambda_init,
                         const float* rms_w, float eps, int mode, void* workspace, size_t ws_bytes,
                         cudaStream_t stream) {
  if (S < 1 || H < 1 || d < 1 || max_seqlen < 1 || !(eps >= 0.f)) return DIFFATTN_ERR_INVALID_ARG;
  if (mode != DIFFATTN_MODE_DIFF && mode != DIFFATTN_MODE_LAMBDA_ZERO && mode != DIFFATTN_MODE_SUM)
    return DIFFATTN_ERR_INVALID_ARG;
  if (!q || !k_cache || !v_cache || !cu_seqlens || !o || !lambda || !rms_w) return DIFFATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o))
    return DIFFATTN_ERR_INVALID_ARG;
  if (d != 128) return DIFFATTN_ERR_UNSUPPORTED;
  if (S > 65535 || H > 65535) return DIFFATTN_ERR_UNSUPPORTED;
  if (!decode_units_fit(S, H, max_seqlen)) return DIFFATTN_ERR_UNSUPPORTED;
  const size_t need = decode_workspace_bytes(S, H, d, max_seqlen);
  if (!workspace || ws_bytes < need || !aligned16(workspace)) return DIFFATTN_ERR_WORKSPACE;
  return cuda_status(launch_decode(q, k_cache, v_cache, cu_seqlens, max_seqlen, o, S, H, d, lambda, lambda_init,
                                   rms_w, eps, mode, workspace, stream));
}

}  // extern "C"
