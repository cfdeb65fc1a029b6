// gla_norm.cu -- the element-wise kernels of the normalised GLA variant (the
// diffusers draft, page 4, `gated_linear_attention`): elu+1 features of q and k,
// the forget gate sigmoid(q * k) on the raw q and k, and a denominator that is
// gated like the state.
//
// The denominator is one more value column: with v extended by a column of ones,
// the state's last column is z_t = g_t * z_{t-1} + phi(k_t), and phi(q_t) S_t holds
// both the numerator and phi(q_t) . z_t.  So the variant runs as
//   prep:  phi(q), phi(k), log sigmoid(q * k), [v | 1 | 0...]   (fp32)
//   the fp32 chunk-wise GLA forward (64-row chunks: the draft's gates decay by
//   about 0.7 nats per token on its inputs, 45 nats over a chunk, inside the
//   fp32-safe range that 128-row chunks would leave)
//   post:  out = numerator / max(denominator, eps)
// All arithmetic fp32, as the draft's loop.
#include <math.h>

#include "dev_common.cuh"
#include "internal.h"

namespace dig {

namespace {

__device__ __forceinline__ float ld(const float* p) { return *p; }
__device__ __forceinline__ float ld(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ void st(float* p, float x) { *p = x; }
__device__ __forceinline__ void st(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

// elu(x) + 1: x + 1 above zero, e^x at or below.
__device__ __forceinline__ float feature(float x) { return x > 0.f ? x + 1.f : expf(x); }

// log sigmoid(x) = -log(1 + e^-x), written so that the exponential never overflows.
__device__ __forceinline__ float log_sigmoid(float x) {
  return x >= 0.f ? -log1pf(expf(-x)) : x - log1pf(expf(x));
}

template <typename TI>
__global__ void __launch_bounds__(256) gla_norm_prep(const TI* __restrict__ q, const TI* __restrict__ k,
                                                     const TI* __restrict__ v, float* __restrict__ fq,
                                                     float* __restrict__ fk, float* __restrict__ la,
                                                     float* __restrict__ va, int64_t rows, int dk, int dv, int dva) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < rows * dk; e += stride) {
    const float x = ld(q + e), y = ld(k + e);
    fq[e] = feature(x);
    fk[e] = feature(y);
    la[e] = log_sigmoid(x * y);
  }
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < rows * dva; e += stride) {
    const int64_t r = e / dva;
    const int j = (int)(e - r * dva);
    va[e] = j < dv ? ld(v + r * dv + j) : (j == dv ? 1.f : 0.f);
  }
}

template <typename TI>
__global__ void __launch_bounds__(256) gla_norm_post(const float* __restrict__ oa, TI* __restrict__ out,
                                                     int64_t rows, int dv, int dva, float eps) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < rows * dv; e += stride) {
    const int64_t r = e / dv;
    const int j = (int)(e - r * dv);
    st(out + e, oa[r * dva + j] / fmaxf(oa[r * dva + dv], eps));
  }
}

int grid_for(int64_t n) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t want = (n + 255) / 256;
  return (int)(want < (int64_t)sms * 8 ? want : (int64_t)sms * 8);
}

}  // namespace

cudaError_t gla_norm_prep_launch(const void* q, const void* k, const void* v, float* fq, float* fk, float* la,
                                 float* va, int64_t rows, int dk, int dv, int dva, int bf16, cudaStream_t s) {
  const int grid = grid_for(rows * (dk > dva ? dk : dva));
  if (bf16)
    gla_norm_prep<__nv_bfloat16><<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(q),
                                                       static_cast<const __nv_bfloat16*>(k),
                                                       static_cast<const __nv_bfloat16*>(v), fq, fk, la, va, rows, dk,
                                                       dv, dva);
  else
    gla_norm_prep<float><<<grid, 256, 0, s>>>(static_cast<const float*>(q), static_cast<const float*>(k),
                                               static_cast<const float*>(v), fq, fk, la, va, rows, dk, dv, dva);
  return cudaGetLastError();
}

cudaError_t gla_norm_post_launch(const float* oa, void* out, int64_t rows, int dv, int dva, float eps, int bf16,
                                 cudaStream_t s) {
  const int grid = grid_for(rows * dv);
  if (bf16)
    gla_norm_post<__nv_bfloat16><<<grid, 256, 0, s>>>(oa, static_cast<__nv_bfloat16*>(out), rows, dv, dva, eps);
  else
    gla_norm_post<float><<<grid, 256, 0, s>>>(oa, static_cast<float*>(out), rows, dv, dva, eps);
  return cudaGetLastError();
}

}  // namespace dig
