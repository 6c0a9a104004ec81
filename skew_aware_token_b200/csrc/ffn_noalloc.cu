// moe_expert_ffn_noalloc: the grouped SwiGLU expert FFN for callers that cannot allocate
// device memory.
//
// moe_expert_ffn needs a caller-allocated scratch buffer for the FC1 output A (bf16,
// R_max x f).  Some callers have no way to provide one: a plugin or custom operator that
// a host framework hands only its inputs and outputs (the framework's pool owns the
// device memory and offers no workspace), or a deployment that reserves all device
// memory at start-up and forbids cudaMalloc afterwards.  This entry point keeps A in a
// fixed-size array inside the library instead, and allocates nothing.
//
// The array is a file-scope __device__ variable of MOE_NOALLOC_SCRATCH_BYTES (64 MiB).
// Every GPU on which the library's device code is loaded reserves it until the process
// exits.  Host code cannot use the variable's name as a device address, so the first
// call on each device (with that device current) looks the address up with
// cudaGetSymbolAddress and caches it together with the CUDA context it belongs to; that
// first call should therefore come before any stream capture.  A later call under another
// context of the same device (after cudaDeviceReset, the module is loaded anew and the
// array may move) looks the address up again instead of using a stale one.  All calls
// share the one array: its contents are whatever the last call left, and calls whose
// kernels overlap on the GPU (for example on two streams) race on it.  Every call zeroes
// the parts that must start at zero: the tile-scheduler counters and, for the one-launch
// FFN, its per-tile-half readiness counters; FC1 writes every row of A that FC2 reads for
// an output row.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "moe_common.cuh"

namespace moe {
namespace {

static __device__ __align__(256) uint8_t g_ffn_scratch[MOE_NOALLOC_SCRATCH_BYTES];

std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};
CUcontext g_scratch_ctx[kMaxDevices] = {};

// The driver's cuCtxGetCurrent, found once through the runtime (no link-time dependency on
// the driver library).
PFN_cuCtxGetCurrent_v4000 ctx_get_current() {
  static PFN_cuCtxGetCurrent_v4000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
  });
  return fn;
}

// Device address of the array on the current device, looked up once per device and
// context (again after the context changed, e.g. after cudaDeviceReset).
int scratch_on_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
  auto get_ctx = ctx_get_current();
  if (!get_ctx) return MOE_ERR_CUDA;
  CUcontext ctx = nullptr;
  if (get_ctx(&ctx) != CUDA_SUCCESS) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!ctx || !g_scratch_ptr[dev] || g_scratch_ctx[dev] != ctx) {
    // the lookup also brings up the device's primary context when none is current yet
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_ffn_scratch) != cudaSuccess || !p) return MOE_ERR_CUDA;
    if (!ctx && (get_ctx(&ctx) != CUDA_SUCCESS || !ctx)) return MOE_ERR_CUDA;
    g_scratch_ptr[dev] = p;
    g_scratch_ctx[dev] = ctx;
  }
  *out = g_scratch_ptr[dev];
  return MOE_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" MOE_API int moe_expert_ffn_noalloc(const moe_cfg* cfg, const uint16_t* xp,
                                              const uint16_t* w1, const uint16_t* w2,
                                              const int32_t* tiles, const int32_t* plan_info,
                                              const int32_t* row_token, const float* row_gate,
                                              int mode, void* out, int32_t* status,
                                              moe_stream_t stream) {
  if (!cfg) return MOE_ERR_INVALID_ARG;
  const moe_cfg& c = *cfg;
  if (c.T < 0 || c.E < 1 || c.k < 1 || c.k > c.E || c.k > kMaxK || c.P < 1 || c.P > kMaxP ||
      c.s < 0 || (c.beta != 64 && c.beta != 128) || c.d < 1 || c.f < 1)
    return MOE_ERR_INVALID_ARG;
  if (c.E > kMaxE || (long long)c.T * c.k > kMaxN) return MOE_ERR_UNSUPPORTED;
  // the fixed array holds A and counters only: Z for a backward pass needs the caller's
  // scratch, and a slot record there could not be read back by the caller
  if (mode & ~kFfnModes || mode & (MOE_FFN_SAVE_Z | MOE_FFN_RECORD_SLOTS))
    return MOE_ERR_INVALID_ARG;
  if ((mode & (MOE_FFN_ONE_LAUNCH | MOE_FFN_TEST_WAIT_TIMEOUT)) && (mode & kOneLaunchExcludes))
    return MOE_ERR_INVALID_ARG;
  if (c.d % 256 || c.f % 128) return MOE_ERR_UNSUPPORTED;
  if ((mode & MOE_FFN_STRICT_SLOTS) && ffn_units(mode) < c.P) return MOE_ERR_UNSUPPORTED;
  for (const void* p : {(const void*)xp, (const void*)w1, (const void*)w2, (const void*)tiles,
                        (const void*)plan_info, (const void*)row_token, (const void*)row_gate,
                        (const void*)out, (const void*)status}) {
    if (!p) return MOE_ERR_INVALID_ARG;
    if (!aligned16(p)) return MOE_ERR_UNSUPPORTED;
  }
  // A (bf16 [R_max, f]) and the scheduler counters must fit the fixed array
  if ((unsigned long long)ffn_scratch_bytes(c) > (unsigned long long)MOE_NOALLOC_SCRATCH_BYTES)
    return MOE_ERR_TOO_LARGE;
  void* scratch = nullptr;
  const int rc = scratch_on_current_device(&scratch);
  if (rc != MOE_OK) return rc;
  const cudaError_t err = launch_ffn(c, xp, w1, w2, tiles, plan_info, row_token, row_gate, mode,
                                     static_cast<uint16_t*>(scratch), out, status,
                                     (cudaStream_t)stream);
  return err == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
