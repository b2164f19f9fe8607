// diffattn_decode_noalloc: the decode step for callers that cannot allocate
// device memory.
//
// Some callers are not allowed to call cudaMalloc: for example a plugin
// inside an inference engine that owns every byte of device memory through
// its own pool, or code that runs where an allocation could block or fail
// (a latency-critical serving loop that must not touch the driver's
// allocator).  They cannot provide diffattn_decode's workspace.  This entry
// point instead uses a fixed scratch array that the library defines at file
// scope in device memory, so it allocates nothing; the caller still passes
// the inputs and the output.
//
// The array is a `static __device__` symbol.  In host code its name is only a
// host-side stand-in, not a device address, so the host looks up the real
// address once per device with cudaGetSymbolAddress (with that device
// current) and passes it to the kernels.  The cached address is tied to the
// device's context: after a cudaDeviceReset the runtime creates a new context
// (with a new id), and the next call looks the address up again instead of
// handing the kernels an address of the old one.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "diffattn.h"
#include "internal.h"

namespace {

constexpr size_t kScratchBytes = DIFFATTN_DECODE_NOALLOC_SCRATCH_BYTES;

// The scratch every diffattn_decode_noalloc call on a device shares.  Every
// GPU that loads the library holds it until the process exits.
static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
struct ScratchSlot {
  void* ptr;
  unsigned long long ctx;  // id of the context the address belongs to
};
ScratchSlot g_scratch_slot[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of g_decode_scratch on the current device: looked up on the
// first call per device (and again once the device's context has changed, or
// on every call when the context id cannot be read).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  const unsigned long long ctx = diffattn::current_context_id();
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  ScratchSlot& slot = g_scratch_slot[dev];
  if (!slot.ptr || ctx == 0 || slot.ctx != ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return e;
    slot.ptr = p;
    slot.ctx = ctx;
  }
  *out = slot.ptr;
  return cudaSuccess;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" int diffattn_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                       const int* cu_seqlens, int max_seqlen, void* o, int S, int H, int d,
                                       const float* lambda, float lambda_init, const float* rms_w, float eps,
                                       cudaStream_t stream) {
  if (S < 1 || H < 1 || d < 1 || max_seqlen < 1 || !(eps >= 0.f)) return DIFFATTN_ERR_INVALID_ARG;
  if (!q || !k_cache || !v_cache || !cu_seqlens || !o || !lambda || !rms_w) return DIFFATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o))
    return DIFFATTN_ERR_INVALID_ARG;
  if (d != 128) return DIFFATTN_ERR_UNSUPPORTED;
  if (S > 65535 || H > 65535) return DIFFATTN_ERR_UNSUPPORTED;
  if (!diffattn::decode_units_fit(S, H, max_seqlen)) return DIFFATTN_ERR_UNSUPPORTED;
  const size_t need = diffattn::decode_workspace_bytes(S, H, d, max_seqlen);
  if (need == 0 || need > kScratchBytes) return DIFFATTN_ERR_WORKSPACE;  // beyond the built-in scratch
  void* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return DIFFATTN_ERR_CUDA;
  // The decode kernels write every scratch entry they later read, so the
  // array needs no clearing between calls.
  return diffattn::launch_decode(q, k_cache, v_cache, cu_seqlens, max_seqlen, o, S, H, d, lambda, lambda_init,
                                 rms_w, eps, DIFFATTN_MODE_DIFF, scratch, stream) == cudaSuccess
             ? DIFFATTN_OK
             : DIFFATTN_ERR_CUDA;
}
