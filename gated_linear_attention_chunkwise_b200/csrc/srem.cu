// srem.cu -- SREM kernels (DiG paper notes, "空间重定向与增强模块 (SREM)"):
//   srem_reorient_k : the scan-direction change as a gather of whole token rows
//                     (transpose of the 2D token matrix and/or flip of the
//                     sequence), bit-exact.
//   dwconv3x3_k     : 3x3 depthwise convolution on the channels-last token grid,
//                     zero padding, fp32 accumulation.
// Both are pure HBM streams, no tensor cores.  The conv streams haloed tiles
// through shared memory with TMA; the reorientation copies 16-byte vectors.
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

// ---------------------------------------------------------------------------
// dwconv3x3_k: persistent blocks walk tiles of 16 x 16 pixels (rows x columns) x one
// 128-byte channel slice.  Each tile arrives with a one-pixel halo (18 x 18 pixels)
// by one TMA load into a 2-deep shared-memory ring, so the next tile loads while
// one is computed; pixels outside the image read as zero (the TMA fills
// out-of-bounds elements), which is the zero padding.  Lane = 4 bytes of channels
// (two bf16 or one fp32 channel), warp = two output columns; each thread walks the
// tile's rows with a 3-row x 4-column register window.  Each output sums its three
// kernel rows separately and then adds them, so three short FMA chains run side by
// side instead of one chain of nine.  Taller tiles than 8 rows halve the block
// barriers and the halo per output; two blocks per SM keep 16 warps resident.
// ---------------------------------------------------------------------------
constexpr int kTileR = 16, kTileC = 16;           // output rows, columns per tile
constexpr int kHaloR = kTileR + 2, kHaloC = kTileC + 2;
constexpr int kConvBufs = 2;                       // TMA ring depth per block
constexpr uint32_t kTileBytes = kHaloR * kHaloC * 128u;               // one haloed tile
constexpr uint32_t kBufBytes = (kTileBytes + 1023u) / 1024u * 1024u;  // buffer stride (1024-aligned)
constexpr size_t kConvSmem = 1024 + kConvBufs * (size_t)kBufBytes + 64;  // + alignment slack and barriers
constexpr int kConvThreads = 32 * (kTileC / 2);

template <typename T>
struct Lane4;  // the 4 bytes of channels a lane owns
template <>
struct Lane4<__nv_bfloat16> {
  static constexpr int kCh = 2;
  __device__ static float2 get(uint32_t v) { return unpack_bf16x2(v); }
  __device__ static uint32_t put(float2 f) { return pack_bf16x2(f.x, f.y); }
};
template <>
struct Lane4<float> {
  static constexpr int kCh = 1;
  __device__ static float2 get(uint32_t v) { return make_float2(__uint_as_float(v), 0.f); }
  __device__ static uint32_t put(float2 f) { return __float_as_uint(f.x); }
};

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, int c0, int c1, int c2, int c3,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar)
      : "memory");
}

template <typename T>
__global__ void __launch_bounds__(kConvThreads, 2) dwconv3x3_k(const __grid_constant__ CUtensorMap xmap,
                                                            const float* __restrict__ w, T* __restrict__ y, int Hg,
                                                            int Wg, int C, int ntx, int nty, int nct, int nsp) {
  constexpr int kCh = Lane4<T>::kCh;
  constexpr int kTC = 32 * kCh;  // channels per tile slice
  extern __shared__ uint8_t sm_raw[];
  // Tile buffers start on a 1024-byte boundary (TMA destinations); the two mbarriers
  // follow them.
  const uint32_t raw = smem_u32(sm_raw);
  const uint32_t sbuf = (raw + 1023u) & ~1023u;
  uint8_t* sm = sm_raw + (sbuf - raw);
  const uint32_t bar0 = sbuf + (uint32_t)kConvBufs * kBufBytes;
  const int lane = threadIdx.x & 31, wp = threadIdx.x >> 5;
  // Every block keeps one channel slice (its weights stay in registers) and walks the
  // spatial tiles sp = blockIdx.x / nct + k * (gridDim.x / nct).
  const int ct = blockIdx.x % nct, bpc = gridDim.x / nct, sp0 = blockIdx.x / nct;
  auto spatial = [&](int sp, int& b, int& ty, int& tx) {
    tx = sp % ntx;
    const int r = sp / ntx;
    ty = r % nty;
    b = r / nty;
  };
  auto issue = [&](int k, int buf) {
    int b, ty, tx;
    spatial(sp0 + k * bpc, b, ty, tx);
    mbar_expect_tx(bar0 + 8u * buf, kTileBytes);
    tma_load_4d(sbuf + (uint32_t)buf * kBufBytes, &xmap, ct * kTC, tx * kTileC - 1, ty * kTileR - 1, b, bar0 + 8u * buf);
  };
  if (threadIdx.x == 0) {
    for (int q = 0; q < kConvBufs; ++q) mbar_init(bar0 + 8u * q, 1);
    fence_mbar_init();
    for (int q = 0; q < kConvBufs; ++q)
      if (sp0 + q * bpc < nsp) issue(q, q);
  }
  __syncthreads();
  const int c = ct * kTC + kCh * lane;  // first channel of this lane
  float2 wt[9];  // weights of this lane's channels (zero past C)
#pragma unroll
  for (int t = 0; t < 9; ++t) {
    wt[t].x = c < C ? __ldg(w + (int64_t)c * 9 + t) : 0.f;
    wt[t].y = (kCh == 2 && c + 1 < C) ? __ldg(w + (int64_t)(c + 1) * 9 + t) : 0.f;
  }
  for (int k = 0;; ++k) {
    const int sp = sp0 + k * bpc;
    if (sp >= nsp) break;
    const int buf = k % kConvBufs;
    const uint32_t par = (uint32_t)((k / kConvBufs) & 1);
    int b, ty, tx;
    spatial(sp, b, ty, tx);
    // Bounded wait for the tile; the block leaves together if it expires.
    bool late = false;
    if (!mbar_try_wait(bar0 + 8u * buf, par)) {
      const long long t0 = clock64();
      while (!mbar_try_wait(bar0 + 8u * buf, par))
        if (clock64() - t0 > kWaitCycles) {
          late = true;
          break;
        }
    }
    if (__syncthreads_or(late)) {
      if (threadIdx.x == 0) {
        report_status(GLA_ERR_TIMEOUT);
        // Let the loads already issued into the ring land before leaving (bounded).
        for (int kk = k; kk < k + kConvBufs && sp0 + kk * bpc < nsp; ++kk) {
          const long long t0 = clock64();
          while (!mbar_try_wait(bar0 + 8u * (kk % kConvBufs), (uint32_t)((kk / kConvBufs) & 1)) &&
                 clock64() - t0 < kWaitCycles) {
          }
        }
      }
      return;
    }
    const uint32_t* tl = reinterpret_cast<const uint32_t*>(sm + (uint32_t)buf * kBufBytes);
    auto at = [&](int r, int cc) -> uint32_t { return tl[(r * kHaloC + cc) * 32 + lane]; };
    const int x0 = tx * kTileC + 2 * wp, y0 = ty * kTileR;
    // Window of input values as fp32 (converted once, when a row enters it).
    float2 win[3][4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      win[0][j] = Lane4<T>::get(at(0, 2 * wp + j));
      win[1][j] = Lane4<T>::get(at(1, 2 * wp + j));
    }
    // Output pointer of (row y0, column x0) for this lane; rows advance by Wg * C.
    T* out = y + (((int64_t)b * Hg + y0) * Wg + x0) * C + c;
    const int64_t rstride = (int64_t)Wg * C;
    const bool ok0 = c < C && x0 < Wg, ok1 = c < C && x0 + 1 < Wg;
    const int rows = min(kTileR, Hg - y0);
#pragma unroll
    for (int r = 0; r < kTileR; ++r) {
#pragma unroll
      for (int j = 0; j < 4; ++j) win[2][j] = Lane4<T>::get(at(r + 2, 2 * wp + j));
      float2 acc[2];
#pragma unroll
      for (int oc = 0; oc < 2; ++oc) {
        float2 part[3];  // one partial sum per kernel row
#pragma unroll
        for (int di = 0; di < 3; ++di) {
          part[di] = make_float2(0.f, 0.f);
#pragma unroll
          for (int dj = 0; dj < 3; ++dj) {
            if (kCh == 2) {  // both channels in one packed fp32 FMA (each rounded as fmaf)
              part[di] = __ffma2_rn(wt[di * 3 + dj], win[di][oc + dj], part[di]);
            } else {
              part[di].x = fmaf(wt[di * 3 + dj].x, win[di][oc + dj].x, part[di].x);
            }
          }
        }
        if (kCh == 2) {
          acc[oc] = __fadd2_rn(__fadd2_rn(part[0], part[1]), part[2]);
        } else {
          acc[oc] = make_float2((part[0].x + part[1].x) + part[2].x, 0.f);
        }
      }
      if (r < rows) {
        if (ok0) *reinterpret_cast<uint32_t*>(out) = Lane4<T>::put(acc[0]);
        if (ok1) *reinterpret_cast<uint32_t*>(out + C) = Lane4<T>::put(acc[1]);
      }
      out += rstride;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        win[0][j] = win[1][j];
        win[1][j] = win[2][j];
      }
    }
    __syncthreads();  // the buffer is read out before it is refilled
    if (threadIdx.x == 0 && sp + kConvBufs * bpc < nsp) issue(k + kConvBufs, buf);
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
  const bool bf = dtype == GLA_BF16;
  const int esz = bf ? 2 : 4;
  const int tc = 128 / esz;  // channels per tile slice
  EncodeTiledFn fn = tensor_map_encoder();
  if (!fn) return cudaErrorNotSupported;
  // 4-D view (channel, column, row, image); the box is one haloed tile.
  CUtensorMap map;
  const cuuint64_t dims[4] = {(cuuint64_t)C, (cuuint64_t)Wg, (cuuint64_t)Hg, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)C * esz, (cuuint64_t)Wg * C * esz, (cuuint64_t)Hg * Wg * C * esz};
  const cuuint32_t box[4] = {(cuuint32_t)tc, (cuuint32_t)kHaloC, (cuuint32_t)kHaloR, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  if (fn(&map, bf ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<void*>(x), dims,
         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
         CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const int ntx = (Wg + kTileC - 1) / kTileC, nty = (Hg + kTileR - 1) / kTileR, nct = (C + tc - 1) / tc;
  const int nsp = B * nty * ntx;  // spatial tiles
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // Two blocks per SM, a whole number of blocks per channel slice.
  int bpc = (2 * sms) / nct;
  bpc = bpc < 1 ? 1 : (bpc > nsp ? nsp : bpc);
  const int grid = bpc * nct;
  const size_t smem = kConvSmem;
  cudaError_t e;
  if (bf) {
    e = cudaFuncSetAttribute(dwconv3x3_k<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dwconv3x3_k<__nv_bfloat16><<<grid, kConvThreads, smem, st>>>(map, w, static_cast<__nv_bfloat16*>(y), Hg, Wg, C,
                                                                   ntx, nty, nct, nsp);
  } else {
    e = cudaFuncSetAttribute(dwconv3x3_k<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dwconv3x3_k<float><<<grid, kConvThreads, smem, st>>>(map, w, static_cast<float*>(y), Hg, Wg, C, ntx, nty, nct,
                                                         nsp);
  }
  return cudaGetLastError();
}

}  // namespace dig
