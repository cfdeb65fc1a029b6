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

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + nb && b0 < a0 + na;
}

// The current device's scratch address, looked up on first use.
int scratch_for_current_device(void** ptr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return GLA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return GLA_ERR_UNSUPPORTED;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return GLA_ERR_CUDA;
  if (major != 10 || minor != 0) return GLA_ERR_UNSUPPORTED;
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

extern "C" int gla_fwd_f32_noalloc(const float* q, const float* k, const float* v, const float* log_alpha, int B,
                                   int H, int Hgrid, int Wgrid, int dk, int dv, int dir, float* out,
                                   cudaStream_t stream) {
  if (!q || !k || !v || !log_alpha || !out) return GLA_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || Hgrid <= 0 || Wgrid <= 0 || dk <= 0 || dv <= 0) return GLA_ERR_INVALID_ARG;
  if (dir < 0 || dir > 3) return GLA_ERR_INVALID_ARG;
  if (dk % 8 || dv % 8 || dk > 128 || dv > 128) return GLA_ERR_UNSUPPORTED;
  const int64_t T = (int64_t)Hgrid * Wgrid;
  if (T > ((int64_t)1 << 30) || (int64_t)B * H > 65535) return GLA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(log_alpha) || !aligned16(out))
    return GLA_ERR_ALIGNMENT;
  const size_t rows = (size_t)B * (size_t)T * (size_t)H;
  const size_t nk = rows * dk * 4, nv = rows * dv * 4;
  if (overlaps(out, nv, q, nk) || overlaps(out, nv, k, nk) || overlaps(out, nv, v, nv) ||
      overlaps(out, nv, log_alpha, nk))
    return GLA_ERR_INVALID_ARG;

  const dig::GlaShape s{B, H, Hgrid, Wgrid, dk, dv, dir};
  if (dig::gla_f32_workspace_bytes(s) > (size_t)DIG_GLA_NOALLOC_SCRATCH_BYTES) return GLA_ERR_UNSUPPORTED;

  void* scratch = nullptr;
  const int rc = scratch_for_current_device(&scratch);
  if (rc != GLA_OK) return rc;
  // Every scratch word the passes read is written earlier in the same call, so
  // nothing needs clearing between calls.
  return dig::gla_f32_forward(q, k, v, log_alpha, out, s, scratch, stream) == cudaSuccess ? GLA_OK : GLA_ERR_CUDA;
}
