// gla_simt.cu -- chunk-wise GLA forward with fp32 q/k/v/out on CUDA cores.
//
// Chunk-wise decomposition in three kernels, with chunks of 64 scan
// positions and every product in fp32 FMA, so the result carries no bf16/tf32
// operand rounding:
//   pass 1  S_loc = K^T V with K^_s = k_s exp(u_s),  gamma = exp(g)
//   pass 2  G_c = Diag(gamma_c) S_in(c),  S_in(c+1) = G_c + S_loc(c)
//   pass 3  O = mask(Q~ K^T) V + Q~ G_c with Q~_r = q_r exp(-u_r)
// (u_r = sum of the log-gates scanned after row r inside the chunk, g the chunk
// total.)  Chunks whose gates decay by more than e^80 inside the chunk are
// flagged by pass 1 and evaluated token by token in pass 3 from the exact fp32
// incoming state, so every log_alpha <= 0 (including -inf) is handled.
#include <math.h>

#include "dev_common.cuh"
#include "internal.h"

namespace dig {

namespace {

constexpr int MC = kChunkF32;
constexpr int NT = 256;
constexpr float kMaxGateRange = 80.0f;

struct F32Args {
  const float* q;
  const float* k;
  const float* v;
  const float* la;
  float* out;
  float* s_locT;  // [BH][NC][dv][dk]
  float* gamma;   // [BH][NC][dk]
  float* GT;      // [BH][NC][dv][dk]  (Diag(gamma) S_in)^T
  int* flags;     // [BH][NC]  1: evaluate this chunk token by token
  int H, dk, dv, NC;
  ScanGeom g;
};

// Shared-memory tiles have an odd row pitch (d + 1 floats): a warp reading one column
// of many rows then touches as many banks as rows.
__host__ __device__ __forceinline__ int pitch_of(int d) { return d + 1; }

// Rows f0..f0+MC-1 of head h, batch b of a [B][T][H][d] fp32 tensor into a
// plain tile of pitch pitch_of(d); rows outside the sequence are zero.
__device__ __forceinline__ void stage_rows(float* dst, const float* src, int d, const ScanGeom& g, int f0, int b,
                                           int h, int H) {
  const int cpr = d / 4;
  const int pitch = pitch_of(d);
  for (int idx = threadIdx.x; idx < MC * cpr; idx += NT) {
    const int r = idx / cpr;
    const int cc = idx - r * cpr;
    const int f = f0 + r;
    float4 val = make_float4(0.f, 0.f, 0.f, 0.f);
    if (f >= 0 && f < g.T)
      val = *reinterpret_cast<const float4*>(src + (((int64_t)b * g.T + base_pos_to_token(g, f)) * H + h) * d +
                                             cc * 4);
    float* o = dst + r * pitch + cc * 4;
    o[0] = val.x;
    o[1] = val.y;
    o[2] = val.z;
    o[3] = val.w;
  }
}

// A 4 x 8 block of a matrix product in registers:
//   acc[i][j] += sum_{k < K} A[i*ar + k*ak] * B[k*bk + j*bc]
// (A and B point at the block's first row / column; the strides pick the layout of
// each operand).  Twelve shared-memory loads feed 32 multiply-adds.
__device__ __forceinline__ void mt48(float (&acc)[4][8], const float* A, int ar, int ak, const float* B, int bk,
                                     int bc, int K) {
#pragma unroll 2
  for (int k = 0; k < K; ++k) {
    float x[4], y[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) x[i] = A[i * ar];
#pragma unroll
    for (int j = 0; j < 8; ++j) y[j] = B[j * bc];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(x[i], y[j], acc[i][j]);
    A += ak;
    B += bk;
  }
}

__device__ __forceinline__ void zero48(float (&acc)[4][8]) {
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
}

// Threads i < dk: exclusive suffix sums of the log-gate along the scan order, in
// place; chunk total in sBL[i].  Returns bit 1 if the factorised form would leave
// fp32 range (use the serial path), bit 2 if the gates grow the state beyond it.
__device__ __forceinline__ int suffix64(float* sLA, float* sBL, int dk, int reverse) {
  const int i = threadIdx.x;
  int code = 0;
  if (i < dk) {
    const int pw = pitch_of(dk);
    float acc = 0.f, lo = 0.f, hi = 0.f;
    for (int s = 0; s < MC; ++s) {
      const int r = reverse ? s : (MC - 1 - s);
      const float la = sLA[r * pw + i];
      sLA[r * pw + i] = acc;
      lo = fminf(lo, acc);
      hi = fmaxf(hi, acc);
      acc += la;
    }
    sBL[i] = acc;
    hi = fmaxf(hi, acc);
    if (!(lo >= -kMaxGateRange) || !(hi <= kMaxGateRange)) code |= 1;
    if (!(hi <= kMaxGateRange)) code |= 2;
  }
  return code;
}

__global__ void __launch_bounds__(NT) gla_f32_chunk_state(const F32Args a) {
  extern __shared__ float4 smem_f4[];
  float* smem = reinterpret_cast<float*>(smem_f4);
  const int c = blockIdx.x, bh = blockIdx.y;
  const int b = bh / a.H, h = bh % a.H;
  const int pk = pitch_of(a.dk), pv = pitch_of(a.dv);
  float* sK = smem;
  float* sV = sK + MC * pk;
  float* sLA = sV + MC * pv;
  float* sBL = sLA + MC * pk;

  const int f0 = chunk_first_base_pos(a.g, c, MC);
  stage_rows(sK, a.k, a.dk, a.g, f0, b, h, a.H);
  stage_rows(sV, a.v, a.dv, a.g, f0, b, h, a.H);
  stage_rows(sLA, a.la, a.dk, a.g, f0, b, h, a.H);
  __syncthreads();
  const int code = suffix64(sLA, sBL, a.dk, a.g.reverse);
  if (code & 2) report_status(GLA_ERR_RANGE);
  const int wide = __syncthreads_or(code != 0);
  for (int e = threadIdx.x; e < MC * a.dk; e += NT) {
    const int r = e / a.dk, i = e - r * a.dk;
    sK[r * pk + i] *= expf(sLA[r * pk + i]);
  }
  __syncthreads();
  const int64_t cid = (int64_t)bh * a.NC + c;
  // 4 x 8 blocks of K^T V (dk x dv), stored transposed ([dv][dk])
  {
    const int ncg = a.dv / 8, nb = (a.dk / 4) * ncg;
    float* dst = a.s_locT + cid * a.dv * a.dk;
    for (int t = threadIdx.x; t < nb; t += NT) {
      const int i0 = 4 * (t / ncg), j0 = 8 * (t % ncg);
      float acc[4][8];
      zero48(acc);
      mt48(acc, sK + i0, 1, pk, sV + j0, pv, 1, MC);
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) dst[(int64_t)(j0 + j) * a.dk + i0 + i] = acc[i][j];
    }
  }
  if (threadIdx.x < a.dk) a.gamma[cid * a.dk + threadIdx.x] = expf(sBL[threadIdx.x]);
  if (threadIdx.x == 0) a.flags[cid] = wide;
}

// Each thread takes four consecutive state elements (i, ..., i+3) of one value column
// j (dk is a multiple of 8) as float4.  Chunks go in batches of kPrefixBatch held in
// two register sets: the next batch's loads are in flight while the current one is
// folded, so the walk is not one memory latency per chunk.
constexpr int kPrefixBatch = 4;
__global__ void __launch_bounds__(256) gla_f32_prefix(const F32Args a) {
  const int bh = blockIdx.y;
  const int e4 = blockIdx.x * blockDim.x + threadIdx.x;
  if (4 * e4 >= a.dk * a.dv) return;
  const int j = 4 * e4 / a.dk, i = 4 * e4 - j * a.dk;
  const int NC = a.NC;
  const int64_t c0id = (int64_t)bh * NC;
  // element (j, i) of chunk c in the [dv][dk] slots, and the chunk's gates at i
  auto slot = [&](int c) { return ((c0id + c) * a.dv + j) * a.dk + i; };
  float4 xa[kPrefixBatch], xb[kPrefixBatch], ga[kPrefixBatch], gb[kPrefixBatch];
  int fa[kPrefixBatch], fb[kPrefixBatch];
  auto load = [&](int c0, float4 (&x)[kPrefixBatch], float4 (&g)[kPrefixBatch], int (&fl)[kPrefixBatch]) {
#pragma unroll
    for (int u = 0; u < kPrefixBatch; ++u) {
      const int c = c0 + u;
      const bool in = c < NC;
      x[u] = in ? *reinterpret_cast<const float4*>(a.s_locT + slot(c)) : make_float4(0.f, 0.f, 0.f, 0.f);
      g[u] = in ? *reinterpret_cast<const float4*>(a.gamma + (c0id + c) * a.dk + i) : make_float4(0.f, 0.f, 0.f, 0.f);
      fl[u] = in ? a.flags[c0id + c] : 0;
    }
  };
  // G = Diag(gamma) S_in is written for every chunk, S_in itself for chunks that pass
  // 3 evaluates token by token; then S = G + S_loc.
  auto fold = [&](int c0, const float4 (&x)[kPrefixBatch], const float4 (&g)[kPrefixBatch],
                  const int (&fl)[kPrefixBatch], float4& S) {
#pragma unroll
    for (int u = 0; u < kPrefixBatch; ++u) {
      const int c = c0 + u;
      if (c < NC) {
        const float4 G = make_float4(g[u].x * S.x, g[u].y * S.y, g[u].z * S.z, g[u].w * S.w);
        *reinterpret_cast<float4*>(a.GT + slot(c)) = G;
        if (fl[u]) *reinterpret_cast<float4*>(a.s_locT + slot(c)) = S;
        S = make_float4(G.x + x[u].x, G.y + x[u].y, G.z + x[u].z, G.w + x[u].w);
      }
    }
  };
  float4 S = make_float4(0.f, 0.f, 0.f, 0.f);
  load(0, xa, ga, fa);
  for (int c0 = 0; c0 < NC; c0 += 2 * kPrefixBatch) {
    load(c0 + kPrefixBatch, xb, gb, fb);
    fold(c0, xa, ga, fa, S);
    load(c0 + 2 * kPrefixBatch, xa, ga, fa);
    fold(c0 + kPrefixBatch, xb, gb, fb, S);
  }
}

__global__ void __launch_bounds__(NT) gla_f32_output(const F32Args a) {
  extern __shared__ float4 smem_f4[];
  float* smem = reinterpret_cast<float*>(smem_f4);
  const int c = blockIdx.x, bh = blockIdx.y;
  const int b = bh / a.H, h = bh % a.H;
  const int pk = pitch_of(a.dk), pv = pitch_of(a.dv), pa = MC + 1;
  float* sQ = smem;
  float* sK = sQ + MC * pk;
  float* sLA = sK + MC * pk;
  float* sV = sLA + MC * pk;
  float* sG = sV + MC * pv;          // [dv][pitch_of(dk)]: G^T
  // The score tile [MC][MC+1] reuses the log-gate tile when it fits (dk >= MC): the
  // gates are dead once Q~ and K^ are formed, which frees a second block per SM.
  const bool a_in_la = pk >= pa;
  float* sA = a_in_la ? sLA : sG + a.dv * pk;
  float* sBL = a_in_la ? sG + a.dv * pk : sA + MC * pa;

  const int f0 = chunk_first_base_pos(a.g, c, MC);
  stage_rows(sQ, a.q, a.dk, a.g, f0, b, h, a.H);
  stage_rows(sK, a.k, a.dk, a.g, f0, b, h, a.H);
  stage_rows(sV, a.v, a.dv, a.g, f0, b, h, a.H);
  stage_rows(sLA, a.la, a.dk, a.g, f0, b, h, a.H);
  const int64_t cid = (int64_t)bh * a.NC + c;
  {
    const float* src = a.GT + cid * a.dv * a.dk;
    for (int e = threadIdx.x; e < a.dv * a.dk; e += NT) {
      const int j = e / a.dk, i = e - j * a.dk;
      sG[j * pk + i] = src[e];
    }
  }
  __syncthreads();
  if (a.flags[cid]) {
    // Exact token-by-token recurrence from S_in (left in the S_loc slot by pass 2):
    // thread j owns value column j of the state sS[dk][dv] (reuses sG and sA).
    float* sS = sG;
    const float* src = a.s_locT + cid * a.dv * a.dk;
    for (int e = threadIdx.x; e < a.dk * a.dv; e += NT) {
      const int j = e / a.dk, i = e - j * a.dk;
      sS[i * a.dv + j] = src[e];
    }
    for (int e = threadIdx.x; e < MC * a.dk; e += NT) {
      const int r = e / a.dk, i = e - r * a.dk;
      sLA[r * pk + i] = expf(sLA[r * pk + i]);
    }
    __syncthreads();
    for (int s = 0; s < MC; ++s) {
      const int r = a.g.reverse ? (MC - 1 - s) : s;
      const int f = f0 + r;
      if (f < 0 || f >= a.g.T) continue;
      for (int j = threadIdx.x; j < a.dv; j += NT) {
        const float vj = sV[r * pv + j];
        float acc = 0.f;
        for (int i = 0; i < a.dk; ++i) {
          const float st = fmaf(sLA[r * pk + i], sS[i * a.dv + j], sK[r * pk + i] * vj);
          sS[i * a.dv + j] = st;
          acc = fmaf(sQ[r * pk + i], st, acc);
        }
        a.out[(((int64_t)b * a.g.T + base_pos_to_token(a.g, f)) * a.H + h) * a.dv + j] = acc;
      }
    }
    return;
  }
  suffix64(sLA, sBL, a.dk, a.g.reverse);
  __syncthreads();
  for (int e = threadIdx.x; e < MC * a.dk; e += NT) {
    const int r = e / a.dk, i = e - r * a.dk;
    const float u = sLA[r * pk + i];
    sQ[r * pk + i] *= expf(-u);
    sK[r * pk + i] *= expf(u);
  }
  __syncthreads();
  const bool rev = a.g.reverse;
  // A = mask(Q~ K^T): position s <= t in scan order is tile row s <= t (s >= t reversed)
  {
    const int ncg = MC / 8, nm = (MC / 4) * ncg;
    for (int e = threadIdx.x; e < nm; e += NT) {
      const int t0 = 4 * (e / ncg), s0 = 8 * (e % ncg);
      float acc[4][8];
      zero48(acc);
      if (!(rev ? (s0 + 7 < t0) : (s0 > t0 + 3))) mt48(acc, sQ + t0 * pk, pk, 1, sK + s0 * pk, 1, pk, a.dk);
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int t = t0 + i, s2 = s0 + j;
          sA[t * pa + s2] = (rev ? (s2 >= t) : (s2 <= t)) ? acc[i][j] : 0.f;
        }
    }
  }
  __syncthreads();
  // O = A V + Q~ G (G held transposed: sG[j][i])
  {
    const int ncg = a.dv / 8, nb = (MC / 4) * ncg;
    for (int e = threadIdx.x; e < nb; e += NT) {
      const int t0 = 4 * (e / ncg), j0 = 8 * (e % ncg);
      const int lo = rev ? t0 : 0, hi = rev ? MC : t0 + 4;
      float acc[4][8];
      zero48(acc);
      mt48(acc, sA + t0 * pa + lo, pa, 1, sV + lo * pv + j0, pv, 1, hi - lo);
      mt48(acc, sQ + t0 * pk, pk, 1, sG + j0 * pk, 1, pk, a.dk);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int f = f0 + t0 + i;
        if (f < 0 || f >= a.g.T) continue;
        float* orow = a.out + (((int64_t)b * a.g.T + base_pos_to_token(a.g, f)) * a.H + h) * a.dv + j0;
#pragma unroll
        for (int j = 0; j < 8; ++j) orow[j] = acc[i][j];
      }
    }
  }
}

size_t rup(size_t x, size_t m) { return (x + m - 1) / m * m; }

}  // namespace

size_t gla_f32_workspace_bytes(const GlaShape& s) {
  const size_t NC = (size_t)(s.T() + MC - 1) / MC;
  const size_t BH = (size_t)s.B * s.H;
  return rup(BH * NC * s.dv * s.dk * 4, 256) * 2 + rup(BH * NC * s.dk * 4, 256) + rup(BH * NC * 4, 256);
}

cudaError_t gla_f32_forward(const float* q, const float* k, const float* v, const float* la, float* out,
                            const GlaShape& s, void* workspace, cudaStream_t st) {
  F32Args a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.la = la;
  a.out = out;
  a.H = s.H;
  a.dk = s.dk;
  a.dv = s.dv;
  a.NC = (s.T() + MC - 1) / MC;
  a.g = make_geom(s.Hg, s.Wg, s.dir);
  const size_t BH = (size_t)s.B * s.H;
  const size_t sl = rup(BH * a.NC * s.dv * s.dk * 4, 256);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  a.s_locT = reinterpret_cast<float*>(ws);
  a.GT = reinterpret_cast<float*>(ws + sl);
  a.gamma = reinterpret_cast<float*>(ws + 2 * sl);
  a.flags = reinterpret_cast<int*>(ws + 2 * sl + rup(BH * a.NC * s.dk * 4, 256));

  const size_t pk = pitch_of(s.dk), pv = pitch_of(s.dv);
  const size_t smem_state = (MC * pk * 2 + MC * pv + s.dk) * sizeof(float);
  const size_t score = pk >= (size_t)MC + 1 ? 0 : (size_t)MC * (MC + 1);  // else in the log-gate tile
  const size_t smem_out = (MC * pk * 3 + MC * pv + s.dv * pk + score + s.dk) * sizeof(float);
  cudaError_t e;
  e = cudaFuncSetAttribute(gla_f32_chunk_state, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_state);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(gla_f32_output, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_out);
  if (e != cudaSuccess) return e;
  const dim3 grid(a.NC, s.B * s.H);
  gla_f32_chunk_state<<<grid, NT, smem_state, st>>>(a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  gla_f32_prefix<<<dim3((s.dk * s.dv / 4 + 255) / 256, s.B * s.H), 256, 0, st>>>(a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  gla_f32_output<<<grid, NT, smem_out, st>>>(a);
  return cudaGetLastError();
}

}  // namespace dig
