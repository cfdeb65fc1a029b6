// srem.cu -- SREM kernels (DiG paper notes, "空间重定向与增强模块 (SREM)"):
//   srem_reorient_k : the scan-direction change as a gather of whole token rows
//                     (transpose of the 2D token matrix and/or flip of the
//                     sequence), bit-exact.
//   dwconv3x3_k     : 3x3 depthwise convolution on the channels-last token grid,
//                     zero padding, fp32 accumulation.
// Both are pure HBM streams: 128-bit loads and stores, no tensor cores.
#include "dev_common.cuh"
#include "internal.h"

namespace dig {

namespace {

// One warp per output row; rows are `vpr` 16-byte vectors long.
__global__ void __launch_bounds__(256) srem_reorient_k(const uint4* __restrict__ x, uint4* __restrict__ y,
                                                       ScanGeom g, int inverse, int64_t nrows, int vpr) {
  const int lane = threadIdx.x & 31;
  const int64_t wpb = blockDim.x >> 5;
  for (int64_t row = blockIdx.x * wpb + (threadIdx.x >> 5); row < nrows; row += (int64_t)gridDim.x * wpb) {
    const int64_t b = row / g.T;
    const int p = (int)(row - b * g.T);
    const int t = scan_pos_to_token(g, p);
    const int64_t src = b * g.T + (inverse ? p : t);
    const int64_t dst = b * g.T + (inverse ? t : p);
    const uint4* s = x + src * vpr;
    uint4* d = y + dst * vpr;
    for (int v = lane; v < vpr; v += 32) d[v] = __ldg(s + v);
  }
}

template <typename T>
struct VecTraits;
template <>
struct VecTraits<__nv_bfloat16> {
  static constexpr int kVec = 8;
  __device__ static void unpack(const uint4& u, float (&f)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 p = unpack_bf16x2(w[j]);
      f[2 * j] = p.x;
      f[2 * j + 1] = p.y;
    }
  }
  __device__ static uint4 pack(const float (&f)[8]) {
    return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                      pack_bf16x2(f[6], f[7]));
  }
};
template <>
struct VecTraits<float> {
  static constexpr int kVec = 4;
  __device__ static void unpack(const uint4& u, float (&f)[4]) {
    f[0] = __uint_as_float(u.x);
    f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z);
    f[3] = __uint_as_float(u.w);
  }
  __device__ static uint4 pack(const float (&f)[4]) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]), __float_as_uint(f[3]));
  }
};

constexpr int kConvCols = 4;   // pixel columns per block (threadIdx.y)
constexpr int kConvRows = 16;  // output rows per block, walked with a rolling 3-row window

// Thread (cv, col): channel vector cv (16 bytes) of pixel column `col`, rows
// y0 .. y0+kConvRows-1 of one image.  The 3x3 window of input vectors is kept in
// registers and shifted down one row per output row.
template <typename T>
__global__ void __launch_bounds__(32 * kConvCols) dwconv3x3_k(const uint4* __restrict__ x, const float* __restrict__ w,
                                                              uint4* __restrict__ y, int Hg, int Wg, int nvec,
                                                              int nbands) {
  constexpr int V = VecTraits<T>::kVec;
  const int cv = blockIdx.x * 32 + threadIdx.x;
  const int col = blockIdx.y * kConvCols + threadIdx.y;
  const int b = blockIdx.z / nbands;
  const int y0 = (blockIdx.z - b * nbands) * kConvRows;
  if (cv >= nvec || col >= Wg) return;

  float wr[9][V];
#pragma unroll
  for (int c = 0; c < V; ++c)
#pragma unroll
    for (int t = 0; t < 9; ++t) wr[t][c] = __ldg(w + (int64_t)(cv * V + c) * 9 + t);

  const int64_t img = (int64_t)b * Hg * Wg;
  auto load = [&](int yy, int xx) -> uint4 {
    if (yy < 0 || yy >= Hg || xx < 0 || xx >= Wg) return make_uint4(0u, 0u, 0u, 0u);
    return __ldg(x + ((img + (int64_t)yy * Wg + xx) * nvec + cv));
  };
  uint4 win[3][3];
#pragma unroll
  for (int dj = 0; dj < 3; ++dj) {
    win[0][dj] = load(y0 - 1, col + dj - 1);
    win[1][dj] = load(y0, col + dj - 1);
  }
  const int yend = min(y0 + kConvRows, Hg);
  for (int yy = y0; yy < yend; ++yy) {
#pragma unroll
    for (int dj = 0; dj < 3; ++dj) win[2][dj] = load(yy + 1, col + dj - 1);
    float acc[V];
#pragma unroll
    for (int c = 0; c < V; ++c) acc[c] = 0.f;
#pragma unroll
    for (int di = 0; di < 3; ++di)
#pragma unroll
      for (int dj = 0; dj < 3; ++dj) {
        float f[V];
        VecTraits<T>::unpack(win[di][dj], f);
#pragma unroll
        for (int c = 0; c < V; ++c) acc[c] = fmaf(wr[di * 3 + dj][c], f[c], acc[c]);
      }
    y[(img + (int64_t)yy * Wg + col) * nvec + cv] = VecTraits<T>::pack(acc);
#pragma unroll
    for (int dj = 0; dj < 3; ++dj) {
      win[0][dj] = win[1][dj];
      win[1][dj] = win[2][dj];
    }
  }
}

}  // namespace

cudaError_t srem_reorient_launch(const void* x, void* y, int dir, int inverse, int B, int Hg, int Wg,
                                 size_t row_bytes, cudaStream_t st) {
  const ScanGeom g = make_geom(Hg, Wg, dir);
  const int64_t nrows = (int64_t)B * g.T;
  const int vpr = (int)(row_bytes / 16);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t want = (nrows + 7) / 8;
  const int grid = (int)(want < (int64_t)sms * 16 ? want : (int64_t)sms * 16);
  srem_reorient_k<<<grid, 256, 0, st>>>(static_cast<const uint4*>(x), static_cast<uint4*>(y), g, inverse, nrows, vpr);
  return cudaGetLastError();
}

cudaError_t dwconv3x3_launch(const void* x, const float* w, void* y, int B, int Hg, int Wg, int C, int dtype,
                             cudaStream_t st) {
  const int V = (dtype == GLA_BF16) ? 8 : 4;
  const int nvec = C / V;
  const int nbands = (Hg + kConvRows - 1) / kConvRows;
  const dim3 block(32, kConvCols);
  const dim3 grid((nvec + 31) / 32, (Wg + kConvCols - 1) / kConvCols, B * nbands);
  if (dtype == GLA_BF16)
    dwconv3x3_k<__nv_bfloat16><<<grid, block, 0, st>>>(static_cast<const uint4*>(x), w, static_cast<uint4*>(y), Hg, Wg,
                                                       nvec, nbands);
  else
    dwconv3x3_k<float><<<grid, block, 0, st>>>(static_cast<const uint4*>(x), w, static_cast<uint4*>(y), Hg, Wg, nvec,
                                               nbands);
  return cudaGetLastError();
}

}  // namespace dig
