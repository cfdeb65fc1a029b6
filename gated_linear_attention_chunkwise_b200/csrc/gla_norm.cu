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

// elu(x) + 1: x + 1 above zero, e^x at or below.
__device__ __forceinline__ float feature(float x) { return x > 0.f ? x + 1.f : expf(x); }

// log sigmoid(x) = -log(1 + e^-x), written so that the exponential never overflows.
__device__ __forceinline__ float log_sigmoid(float x) {
  return x >= 0.f ? -log1pf(expf(-x)) : x - log1pf(expf(x));
}

// Four consecutive elements (dk, dv and the extended width are multiples of 8, so a
// group of four never crosses a row and is 16-byte aligned in fp32).
__device__ __forceinline__ void ld4(const float* p, float (&x)[4]) {
  const float4 t = *reinterpret_cast<const float4*>(p);
  x[0] = t.x;
  x[1] = t.y;
  x[2] = t.z;
  x[3] = t.w;
}
__device__ __forceinline__ void ld4(const __nv_bfloat16* p, float (&x)[4]) {
  const uint2 t = *reinterpret_cast<const uint2*>(p);
  const float2 a = unpack_bf16x2(t.x), b = unpack_bf16x2(t.y);
  x[0] = a.x;
  x[1] = a.y;
  x[2] = b.x;
  x[3] = b.y;
}
__device__ __forceinline__ void st4(float* p, const float (&x)[4]) {
  *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
}
__device__ __forceinline__ void st4(__nv_bfloat16* p, const float (&x)[4]) {
  *reinterpret_cast<uint2*>(p) = make_uint2(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]));
}

// One warp per (token, head) row, four columns per lane.
template <typename TI>
__global__ void __launch_bounds__(256) gla_norm_prep(const TI* __restrict__ q, const TI* __restrict__ k,
                                                     const TI* __restrict__ v, float* __restrict__ fq,
                                                     float* __restrict__ fk, float* __restrict__ la,
                                                     float* __restrict__ va, int64_t rows, int dk, int dv, int dva) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t r = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < rows; r += warps) {
    for (int c = 4 * lane; c < dk; c += 128) {
      const int64_t e = r * dk + c;
      float x[4], y[4], a[4], b[4], l[4];
      ld4(q + e, x);
      ld4(k + e, y);
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        a[m] = feature(x[m]);
        b[m] = feature(y[m]);
        l[m] = log_sigmoid(x[m] * y[m]);
      }
      st4(fq + e, a);
      st4(fk + e, b);
      st4(la + e, l);
    }
    for (int c = 4 * lane; c < dva; c += 128) {
      float x[4] = {0.f, 0.f, 0.f, 0.f};
      if (c < dv)
        ld4(v + r * dv + c, x);
      else if (c == dv)
        x[0] = 1.f;
      st4(va + r * dva + c, x);
    }
  }
}

// One warp per row: out = numerator / max(denominator, eps), four columns per lane.
template <typename TI>
__global__ void __launch_bounds__(256) gla_norm_post(const float* __restrict__ oa, TI* __restrict__ out,
                                                     int64_t rows, int dv, int dva, float eps) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t r = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < rows; r += warps) {
    const float den = fmaxf(oa[r * dva + dv], eps);
    for (int c = 4 * lane; c < dv; c += 128) {
      float x[4];
      ld4(oa + r * dva + c, x);
#pragma unroll
      for (int m = 0; m < 4; ++m) x[m] = x[m] / den;
      st4(out + r * dv + c, x);
    }
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
  const int grid = grid_for(rows * 32);
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
  const int grid = grid_for(rows * 32);
  if (bf16)
    gla_norm_post<__nv_bfloat16><<<grid, 256, 0, s>>>(oa, static_cast<__nv_bfloat16*>(out), rows, dv, dva, eps);
  else
    gla_norm_post<float><<<grid, 256, 0, s>>>(oa, static_cast<float*>(out), rows, dv, dva, eps);
  return cudaGetLastError();
}

}  // namespace dig
