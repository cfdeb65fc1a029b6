// gla_noalloc.cu -- gla_fwd_f32_noalloc: the fp32 GLA forward for callers that
// must not allocate device memory.
//
// Some callers cannot call cudaMalloc (or cudaMallocAsync) when they run the
// GLA: a host framework that owns every device allocation through its own pool
// and forbids foreign ones, a real-time or embedded program that allocates
// everything at start-up because allocation may block or synchronise the
// device, or code recorded into a CUDA graph that must not contain memory
// nodes.  This entry point gives them the fp32 GLA forward with its scratch in a
// fixed device array that the library itself holds: the caller passes only the
// inputs and the output, and nothing is allocated or freed per call.
//
// The scratch is a file-scope static __device__ array of
// DIG_GLA_NOALLOC_SCRATCH_BYTES.  Every GPU that loads the library keeps it
// until the process exits.  In host code the array's name is only a host-side
// stand-in for the device symbol, so the first call on each device looks up the
// real device address with cudaGetSymbolAddress, with that device current, and
// caches it.
#include <mutex>

#include "dev_common.cuh"
#include "dig_gla.h"
#include "internal.h"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[DIG_GLA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices];  // device address of the scratch array, per device

// The current device's scratch address, looked up on first use (the caller has
// checked that the device is an sm_100 part).
int scratch_for_current_device(void** ptr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return GLA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return GLA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return GLA_ERR_CUDA;
    }
    g_noalloc_ptr[dev] = p;
  }
  *ptr = g_noalloc_ptr[dev];
  return GLA_OK;
}

}  // namespace

namespace dig {
// A context that is torn down and created again (cudaDeviceReset) places the array at
// a new address: dig_gla_release() forgets the cached ones.
void noalloc_forget() {
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  for (void*& p : g_noalloc_ptr) p = nullptr;
}
}  // namespace dig

extern "C" int gla_fwd_f32_noalloc(const float* q, const float* k, const float* v, const float* log_alpha, int B,
                                   int H, int Hgrid, int Wgrid, int dk, int dv, int dir, float* out,
                                   cudaStream_t stream) {
  int rc = dig::validate_gla(q, k, v, log_alpha, out, B, H, Hgrid, Wgrid, dk, dv, dir, 4);
  if (rc != GLA_OK) return rc;
  if (dir > 3) return GLA_ERR_UNSUPPORTED;  // zigzag orders need arranged copies beyond the fixed scratch
  if ((rc = dig::check_device()) != GLA_OK) return rc;
  const dig::GlaShape s{B, H, Hgrid, Wgrid, dk, dv, dir};
  if (dig::gla_f32_workspace_bytes(s) > (size_t)DIG_GLA_NOALLOC_SCRATCH_BYTES) return GLA_ERR_UNSUPPORTED;

  void* scratch = nullptr;
  if ((rc = scratch_for_current_device(&scratch)) != GLA_OK) return rc;
  // Every scratch word the passes read is written earlier in the same call, so
  // nothing needs clearing between calls.
  return dig::gla_f32_forward(q, k, v, log_alpha, out, s, scratch, stream) == cudaSuccess ? GLA_OK : GLA_ERR_CUDA;
}
