// internal.h -- launchers behind the C ABI (host side, C++).  Every launcher
// assumes its arguments were validated by api.cu and only enqueues work.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace dig {

// Geometry of one GLA call, shared by the launchers.
struct GlaShape {
  int B, H, Hg, Wg, dk, dv, dir;
  int T() const { return Hg * Wg; }
};

// ---- bf16 tensor-core path (chunks of 128 scan positions) ----
constexpr int kChunkTC = 128;

// ---- bf16 warp-specialised single-kernel path ----
size_t gla_ws_workspace_bytes(const GlaShape& s);
cudaError_t gla_ws_forward(const void* q, const void* k, const void* v, const float* la, void* out, const GlaShape& s,
                           void* workspace, cudaStream_t st);

// The same kernel with bf16 gate logits g in place of log_alpha:
// log_alpha = logsigmoid(g) / gate_norm, computed in the kernel (dk <= 120).
cudaError_t gla_ws_forward_glogit(const void* q, const void* k, const void* v, const void* g, float gate_norm, void* out,
                                  const GlaShape& s, void* workspace, cudaStream_t st);

// ---- fp32 SIMT path (chunks of 64 scan positions) ----
constexpr int kChunkF32 = 64;
size_t gla_f32_workspace_bytes(const GlaShape& s);
cudaError_t gla_f32_forward(const float* q, const float* k, const float* v, const float* la, float* out,
                            const GlaShape& s, void* workspace, cudaStream_t st);

// ---- GLA backward: tensor cores for bf16 with dk, dv <= 80 (chunks of 128 scan
// positions), else CUDA cores (chunks of 32) ----
size_t gla_bwd_workspace_bytes(const GlaShape& s, int bf16);
cudaError_t gla_bwd_launch(const void* q, const void* k, const void* v, const float* la, const void* dout, void* dq,
                           void* dk, void* dv, float* dla, const GlaShape& s, int bf16, void* workspace,
                           cudaStream_t st);

// ---- normalised variant: element-wise prep / post around the fp32 forward ----
cudaError_t gla_norm_prep_launch(const void* q, const void* k, const void* v, float* fq, float* fk, float* la,
                                 float* va, int64_t rows, int dk, int dv, int dva, int bf16, cudaStream_t s);
cudaError_t gla_norm_post_launch(const float* oa, void* out, int64_t rows, int dv, int dva, float eps, int bf16,
                                 cudaStream_t s);

// cuTensorMapEncodeTiled, reached through the runtime's driver entry point
// (nullptr when the driver does not provide it).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn tensor_map_encoder();

// ---- SREM ----
cudaError_t srem_reorient_launch(const void* x, void* y, int dir, int inverse, int B, int Hg, int Wg,
                                 size_t row_bytes, cudaStream_t st);
cudaError_t dwconv3x3_launch(const void* x, const float* w, void* y, int B, int Hg, int Wg, int C, int dtype,
                             cudaStream_t st);

// ---- test hook: work items the next bf16 GLA call leaves out (0 normally) ----
int take_test_skip_items();

// ---- host checks shared by the entry points (api.cu) ----
// GLA_OK when the current device is an sm_100 part (cached per device).
int check_device();
// Argument validation of a GLA call with q/k/v/out elements of `elt` bytes.
int validate_gla(const void* q, const void* k, const void* v, const void* la, const void* out, int B, int H, int Hg,
                 int Wg, int dk, int dv, int dir, size_t elt);
// Forgets the cached device address of the no-allocation scratch array (gla_noalloc.cu).
void noalloc_forget();

// ---- status word ----
cudaError_t read_and_clear_device_status(int* status, cudaStream_t st);

}  // namespace dig
