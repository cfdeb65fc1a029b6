// gla_bwd.cu -- chunk-wise GLA backward: bf16 q/k/v/dout/dq/dk/dv with dk, dv <= 80
// on tensor cores (tcgen05, bf16 operands, fp32 accumulation), everything else on
// CUDA cores in fp32; fp32 log-gates and their gradient.
//
// The gradient of the recurrence S_t = Diag(alpha_t) S_{t-1} + k_t^T v_t,
// o_t = q_t S_t (DiG trains like DiT, so the GLA layers are differentiated) is
// taken chunk by chunk.  Inside a chunk of MC scan positions, with u_r the sum of
// the log-gates scanned after row r, g the chunk total, S_in the state entering
// the chunk and D the gradient of the loss with respect to the state leaving it:
//   Q~ = q e^{-u},  K^ = k e^{u},  G = Diag(e^g) S_in
//   A  = mask(dO V^T),  P = mask(Q~ K^T)             (s <= r in scan order)
//   dQ~ = dO G^T + A K^,    dq = e^{-u} dQ~
//   dK^ = A^T Q~ + V D^T,   dk = e^{u} dK^
//   dV  = P^T dO + K^ D
// Across chunks the forward state and its gradient run in opposite directions:
//   S_in(c+1) = Diag(gamma_c) S_in(c) + K^_c^T V_c
//   D(c-1)    = Diag(gamma_c) D(c) + Qbar_c^T dO_c,   Qbar = q e^{g-u} = q e^{b}
// (b the inclusive prefix sum of the log-gates inside the chunk).
// The log-gates enter only through their prefix sums b, and o depends on b through
// q e^{b} and k e^{-b}; so dlog_alpha_r = sum over t >= r (scan order) of
// q_t dq_t - k_t dk_t = Q~_t dQ~_t - K^_t dK^_t.  The part of that sum beyond the
// chunk is the gradient of a scalar gate placed at the chunk's end,
// carry_c[i] = sum_j D(c)[i][j] S_in(c+1)[i][j], so every chunk finishes on its own.
//
// Three kernels: per-chunk local terms (K^T V and Qbar^T dO), the two scans over
// chunks (four state elements per thread), and the per-chunk gradients.  Chunks of
// 128 scan positions on the tensor-core path, 32 on the CUDA-core one.  Chunks whose
// gates leave the fp32-safe range (|u| > 80, e.g. a full reset) take an exact
// token-by-token reverse sweep from S_in and D instead of the factorised form.
#include <math.h>

#include "dev_common.cuh"
#include "internal.h"

namespace dig {

namespace {

constexpr int NT = 256;
constexpr float kRange = 80.0f;

template <typename TI>
struct BwdArgs {
  const TI* q;
  const TI* k;
  const TI* v;
  const float* la;
  const TI* dout;
  TI* dq;
  TI* dk_out;
  TI* dv_out;
  float* dla;
  float* sx;     // [BH][NC][dk][dv]: K^T V of chunk c, then S_in(c+1)
  float* dd;     // [BH][NC][dk][dv]: Qbar^T dO of chunk c, then D(c)
  float* gamma;  // [BH][NC][dk]
  int* flags;    // [BH][NC]: 1 = evaluate this chunk token by token
  int H, dk, dv, NC;
  ScanGeom g;
};

__device__ __forceinline__ void load8(const float* p, float* d) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  const float4 b = *reinterpret_cast<const float4*>(p + 4);
  d[0] = a.x, d[1] = a.y, d[2] = a.z, d[3] = a.w, d[4] = b.x, d[5] = b.y, d[6] = b.z, d[7] = b.w;
}
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float* d) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int x = 0; x < 4; ++x) {
    const float2 f = __bfloat1622float2(h[x]);
    d[2 * x] = f.x;
    d[2 * x + 1] = f.y;
  }
}
__device__ __forceinline__ void store1(float* p, float x) { *p = x; }
__device__ __forceinline__ void store1(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

// Shared-memory tiles have an odd row pitch (d + 1 floats): a warp reading one column
// of many rows then touches as many banks as rows.
__host__ __device__ __forceinline__ int pitch_of(int d) { return d + 1; }

// Rows f0 .. f0+MC-1 (base positions) of head h, batch b of a [B][T][H][d] tensor
// into an fp32 tile of pitch pitch_of(d); rows outside the sequence are zero.
template <int MC, typename TE>
__device__ __forceinline__ void stage(float* dst, const TE* src, int d, const ScanGeom& g, int f0, int b, int h,
                                      int H) {
  const int cpr = d / 8;
  const int pitch = pitch_of(d);
  for (int idx = threadIdx.x; idx < MC * cpr; idx += blockDim.x) {
    const int r = idx / cpr;
    const int cc = idx - r * cpr;
    const int f = f0 + r;
    float x[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (f >= 0 && f < g.T) load8(src + (((int64_t)b * g.T + base_pos_to_token(g, f)) * H + h) * d + cc * 8, x);
    float* o = dst + r * pitch + cc * 8;
#pragma unroll
    for (int e = 0; e < 8; ++e) o[e] = x[e];
  }
}

// A 4 x 8 block of a matrix product in registers:
//   acc[i][j] += sum_{k < K} A[i*ar + k*ak] * B[k*bk + j*bc]
// (A and B point at the block's first row / column; the strides pick the layout of
// each operand).  Twelve shared-memory loads feed 32 multiply-adds.
template <int R>
__device__ __forceinline__ void mt48(float (&acc)[R][8], const float* A, int ar, int ak, const float* B, int bk,
                                     int bc, int K) {
#pragma unroll 2
  for (int k = 0; k < K; ++k) {
    float x[R], y[8];
#pragma unroll
    for (int i = 0; i < R; ++i) x[i] = A[i * ar];
#pragma unroll
    for (int j = 0; j < 8; ++j) y[j] = B[j * bc];
#pragma unroll
    for (int i = 0; i < R; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(x[i], y[j], acc[i][j]);
    A += ak;
    B += bk;
  }
}

template <int R>
__device__ __forceinline__ void zero48(float (&acc)[R][8]) {
#pragma unroll
  for (int i = 0; i < R; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
}



// carry[i] = sum_j D[i][j] S_out[i][j] for i < dk (both [dk][dv] fp32 rows in global
// memory): one warp per row i, lanes over j (coalesced), a fixed shuffle-tree sum.
__device__ __forceinline__ void chunk_carry(const float* D, const float* Sout, int dk, int dv, float* carry) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  // Rows i = warp, warp + nw, ... four at a time, all their loads issued first.
  for (int i0 = warp; i0 < dk; i0 += 4 * nw) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int j = lane; j < dv; j += 32) {
      float x[4], y[4];
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int i = i0 + m * nw;
        x[m] = i < dk ? D[(size_t)i * dv + j] : 0.f;
        y[m] = i < dk ? Sout[(size_t)i * dv + j] : 0.f;
      }
#pragma unroll
      for (int m = 0; m < 4; ++m) acc[m] = fmaf(x[m], y[m], acc[m]);
    }
#pragma unroll
    for (int m = 0; m < 4; ++m) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc[m] += __shfl_xor_sync(0xffffffffu, acc[m], o);
      const int i = i0 + m * nw;
      if (lane == 0 && i < dk) carry[i] = acc[m];
    }
  }
}

// Threads i < dk: the log-gate tile becomes, in place, the exclusive suffix sums u
// along the scan order; the chunk total goes to sTot[i].  Returns bit 1 if |u| or
// the total leave the fp32-safe range (evaluate token by token), bit 2 if growth
// gates exceed it (not representable).
template <int MC>
__device__ __forceinline__ int suffix_sums(float* sU, float* sTot, int dk, int reverse) {
  const int i = threadIdx.x;
  int code = 0;
  if (i < dk) {
    const int pw = pitch_of(dk);
    float acc = 0.f, lo = 0.f, hi = 0.f;
    for (int s = 0; s < MC; ++s) {
      const int r = reverse ? s : (MC - 1 - s);
      const float l = sU[r * pw + i];
      sU[r * pw + i] = acc;
      lo = fminf(lo, acc);
      hi = fmaxf(hi, acc);
      acc += l;
    }
    sTot[i] = acc;
    lo = fminf(lo, acc);
    hi = fmaxf(hi, acc);
    if (!(lo >= -kRange) || !(hi <= kRange)) code |= 1;
    if (!(hi <= kRange)) code |= 2;
  }
  return code;
}

// ---------------------------------------------------------------------------
// Kernel 1: per-chunk K^T V (forward state) and Qbar^T dO (backward state).
// ---------------------------------------------------------------------------
template <typename TI, int MC>
__global__ void __launch_bounds__(NT) gla_bwd_local(const BwdArgs<TI> a) {
  extern __shared__ float4 smem_f4[];
  float* smem = reinterpret_cast<float*>(smem_f4);
  const int c = blockIdx.x, bh = blockIdx.y;
  const int b = bh / a.H, h = bh % a.H;
  const int pk = pitch_of(a.dk), pv = pitch_of(a.dv);
  float* sK = smem;
  float* sQ = sK + MC * pk;
  float* sU = sQ + MC * pk;
  float* sV = sU + MC * pk;
  float* sO = sV + MC * pv;
  float* sTot = sO + MC * pv;

  const int f0 = chunk_first_base_pos(a.g, c, MC);
  stage<MC>(sK, a.k, a.dk, a.g, f0, b, h, a.H);
  stage<MC>(sQ, a.q, a.dk, a.g, f0, b, h, a.H);
  stage<MC>(sU, a.la, a.dk, a.g, f0, b, h, a.H);
  stage<MC>(sV, a.v, a.dv, a.g, f0, b, h, a.H);
  stage<MC>(sO, a.dout, a.dv, a.g, f0, b, h, a.H);
  __syncthreads();
  // Qbar = q e^{b}, b the inclusive prefix sum of the log-gates in scan order (formed
  // directly, not as g - u, so that a -inf gate gives 0 rather than inf - inf).
  for (int i = threadIdx.x; i < a.dk; i += NT) {
    float acc = 0.f;
    for (int s = 0; s < MC; ++s) {
      const int r = a.g.reverse ? (MC - 1 - s) : s;
      acc += sU[r * pk + i];
      sQ[r * pk + i] *= expf(acc);
    }
  }
  __syncthreads();
  const int code = suffix_sums<MC>(sU, sTot, a.dk, a.g.reverse);
  if (code & 2) report_status(GLA_ERR_RANGE);
  const int wide = __syncthreads_or(code != 0);
  // K^ = k e^{u}: the exponent is a sum of log-gates, so decays only shrink it.
  for (int e = threadIdx.x; e < MC * a.dk; e += NT) {
    const int r = e / a.dk, i = e - r * a.dk;
    sK[r * pk + i] *= expf(sU[r * pk + i]);
  }
  __syncthreads();
  const int64_t cid = (int64_t)bh * a.NC + c;
  float* sx = a.sx + cid * a.dk * a.dv;
  float* dd = a.dd + cid * a.dk * a.dv;
  // 4 x 8 blocks of K^T V (blocks 0 .. nb-1) and of Qbar^T dO (nb .. 2nb-1), dk x dv.
  const int ncg = a.dv / 8, nb = (a.dk / 4) * ncg;
  for (int t = threadIdx.x; t < 2 * nb; t += NT) {
    const int which = t >= nb, tt = which ? t - nb : t;
    const int i0 = 4 * (tt / ncg), j0 = 8 * (tt % ncg);
    float acc[4][8];
    zero48<4>(acc);
    mt48<4>(acc, (which ? sQ : sK) + i0, 1, pk, (which ? sO : sV) + j0, pv, 1, MC);
    float* dst = which ? dd : sx;
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) dst[(i0 + i) * a.dv + j0 + j] = acc[i][j];
  }
  if (threadIdx.x < a.dk) a.gamma[cid * a.dk + threadIdx.x] = expf(sTot[threadIdx.x]);
  if (threadIdx.x == 0) a.flags[cid] = wide;
}

// ---------------------------------------------------------------------------
// Kernel 2: per state element (i, j) of each head, the forward scan
// S_in(c+1) = gamma_c S_in(c) + (K^T V)_c and the reverse scan
// D(c-1) = gamma_c D(c) + (Qbar^T dO)_c, each written over its local term.
// ---------------------------------------------------------------------------
// Each thread takes four consecutive state elements of one row i (dv is a multiple of
// 8, so a group never crosses a row) as float4.  Chunks go in batches of kScanBatch
// held in two register sets: the next batch's loads are in flight while the current
// one is folded, so the scan is not one memory latency per chunk.
constexpr int kScanBatch = 8;
template <typename TI>
__global__ void __launch_bounds__(256) gla_bwd_scan(const BwdArgs<TI> a) {
  const int bh = blockIdx.y;
  const int e4 = blockIdx.x * blockDim.x + threadIdx.x;
  if (4 * e4 >= a.dk * a.dv) return;
  const int i = 4 * e4 / a.dv;
  const size_t st4 = (size_t)a.dk * a.dv / 4;
  float4* sx = reinterpret_cast<float4*>(a.sx) + (size_t)bh * a.NC * st4 + e4;
  float4* dd = reinterpret_cast<float4*>(a.dd) + (size_t)bh * a.NC * st4 + e4;
  const float* gam = a.gamma + (size_t)bh * a.NC * a.dk + i;
  const int NC = a.NC;
  float4 xa[kScanBatch], xb[kScanBatch];
  float ga[kScanBatch], gb[kScanBatch];
  // chunks c0, c0 + dir, ... (kScanBatch of them, those inside [0, NC))
  auto load = [&](const float4* src, int c0, int dir, float4 (&x)[kScanBatch], float (&g)[kScanBatch]) {
#pragma unroll
    for (int u = 0; u < kScanBatch; ++u) {
      const int c = c0 + dir * u;
      const bool in = c >= 0 && c < NC;
      x[u] = in ? src[(size_t)c * st4] : make_float4(0.f, 0.f, 0.f, 0.f);
      g[u] = in ? gam[(size_t)c * a.dk] : 0.f;
    }
  };
  // forward: S_in(c+1) = gamma_c S_in(c) + (K^T V)_c, written over the local term
  auto fwd = [&](int c0, const float4 (&x)[kScanBatch], const float (&g)[kScanBatch], float4& S) {
#pragma unroll
    for (int u = 0; u < kScanBatch; ++u) {
      const int c = c0 + u;
      if (c < NC) {
        S.x = fmaf(g[u], S.x, x[u].x);
        S.y = fmaf(g[u], S.y, x[u].y);
        S.z = fmaf(g[u], S.z, x[u].z);
        S.w = fmaf(g[u], S.w, x[u].w);
        sx[(size_t)c * st4] = S;
      }
    }
  };
  // reverse: D(c) is written over the local term, then D(c-1) = gamma_c D(c) + (Qbar^T dO)_c
  auto rev = [&](int c0, const float4 (&x)[kScanBatch], const float (&g)[kScanBatch], float4& D) {
#pragma unroll
    for (int u = 0; u < kScanBatch; ++u) {
      const int c = c0 - u;
      if (c >= 0) {
        dd[(size_t)c * st4] = D;
        D.x = fmaf(g[u], D.x, x[u].x);
        D.y = fmaf(g[u], D.y, x[u].y);
        D.z = fmaf(g[u], D.z, x[u].z);
        D.w = fmaf(g[u], D.w, x[u].w);
      }
    }
  };
  float4 S = make_float4(0.f, 0.f, 0.f, 0.f);
  load(sx, 0, 1, xa, ga);
  for (int c0 = 0; c0 < NC; c0 += 2 * kScanBatch) {
    load(sx, c0 + kScanBatch, 1, xb, gb);
    fwd(c0, xa, ga, S);
    load(sx, c0 + 2 * kScanBatch, 1, xa, ga);
    fwd(c0 + kScanBatch, xb, gb, S);
  }
  float4 D = make_float4(0.f, 0.f, 0.f, 0.f);
  load(dd, NC - 1, -1, xa, ga);
  for (int c0 = NC - 1; c0 >= 0; c0 -= 2 * kScanBatch) {
    load(dd, c0 - kScanBatch, -1, xb, gb);
    rev(c0, xa, ga, D);
    load(dd, c0 - 2 * kScanBatch, -1, xa, ga);
    rev(c0 - kScanBatch, xb, gb, D);
  }
}

// ---------------------------------------------------------------------------
// Kernel 3: per-chunk gradients.
// ---------------------------------------------------------------------------
template <typename TI>
__device__ __forceinline__ int64_t row_off(const BwdArgs<TI>& a, int b, int h, int f, int d) {
  return (((int64_t)b * a.g.T + base_pos_to_token(a.g, f)) * a.H + h) * d;
}

// Exact token-by-token reverse sweep through one chunk, from the state entering it
// (S_in(c) = the scan's S_in written for chunk c-1, zero for the first chunk) and the
// gradient D(c) leaving it.  Thread-private recomputation of S_{r-1} for every
// position keeps every state element's recurrence in one thread.
template <typename TI, int MC>
__device__ void chunk_serial_bwd(const BwdArgs<TI>& a, float* sQ, float* sK, float* sU, float* sV, float* sO,
                                 float* sGg, float* sW, int c, int b, int h, int f0) {
  const int pk = pitch_of(a.dk), pv = pitch_of(a.dv);
  const int64_t cid = (int64_t)blockIdx.y * a.NC + c;
  const size_t st = (size_t)a.dk * a.dv;
  const float* sin = c > 0 ? a.sx + (cid - 1) * st : nullptr;
  const float* dd = a.dd + cid * st;
  for (int e = threadIdx.x; e < a.dk * a.dv; e += NT) {
    const int i = e / a.dv, j = e - i * a.dv;
    sGg[i * pv + j] = dd[e];
  }
  for (int e = threadIdx.x; e < MC * a.dk; e += NT) {
    const int r = e / a.dk, i = e - r * a.dk;
    sU[r * pk + i] = expf(sU[r * pk + i]);  // alpha
  }
  __syncthreads();
  for (int step = MC - 1; step >= 0; --step) {
    const int r = a.g.reverse ? (MC - 1 - step) : step;
    const int f = f0 + r;
    // S_{r-1}: the state before this position, recomputed from S_in; and the
    // gradient of S_r picks up q_r^T dO_r.
    for (int e = threadIdx.x; e < a.dk * a.dv; e += NT) {
      const int i = e / a.dv, j = e - i * a.dv;
      float w = sin ? sin[e] : 0.f;
      for (int s2 = 0; s2 < step; ++s2) {
        const int r2 = a.g.reverse ? (MC - 1 - s2) : s2;
        w = fmaf(sU[r2 * pk + i], w, sK[r2 * pk + i] * sV[r2 * pv + j]);
      }
      sW[i * pv + j] = w;
      sGg[i * pv + j] = fmaf(sQ[r * pk + i], sO[r * pv + j], sGg[i * pv + j]);
    }
    __syncthreads();
    const bool real = f >= 0 && f < a.g.T;
    for (int i = threadIdx.x; i < a.dk; i += NT) {
      const float al = sU[r * pk + i], ki = sK[r * pk + i];
      float gq = 0.f, gk = 0.f, gl = 0.f;
      for (int j = 0; j < a.dv; ++j) {
        const float sr = fmaf(al, sW[i * pv + j], ki * sV[r * pv + j]);  // S_r
        gq = fmaf(sO[r * pv + j], sr, gq);
        gk = fmaf(sGg[i * pv + j], sV[r * pv + j], gk);
        gl = fmaf(sGg[i * pv + j], sW[i * pv + j], gl);
      }
      if (real) {
        const int64_t o = row_off(a, b, h, f, a.dk);
        store1(a.dq + o + i, gq);
        store1(a.dk_out + o + i, gk);
        a.dla[o + i] = al * gl;
      }
    }
    for (int j = threadIdx.x; j < a.dv; j += NT) {
      float gv = 0.f;
      for (int i = 0; i < a.dk; ++i) gv = fmaf(sK[r * pk + i], sGg[i * pv + j], gv);
      if (real) store1(a.dv_out + row_off(a, b, h, f, a.dv) + j, gv);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < a.dk * a.dv; e += NT) {
      const int i = e / a.dv, j = e - i * a.dv;
      sGg[i * pv + j] *= sU[r * pk + i];
    }
    __syncthreads();
  }
}

// kTR: rows per register block of the product phases -- 2 when the largest phase
// (dK^ and dV together) still has at most one block per thread, else 4.
template <typename TI, int MC, int kTR>
__global__ void __launch_bounds__(NT) gla_bwd_chunk(const BwdArgs<TI> a) {
  extern __shared__ float4 smem_f4[];
  float* smem = reinterpret_cast<float*>(smem_f4);
  const int c = blockIdx.x, bh = blockIdx.y;
  const int b = bh / a.H, h = bh % a.H;
  const int pk = pitch_of(a.dk), pv = pitch_of(a.dv), pa = MC + 1;
  float* sQ = smem;
  float* sK = sQ + MC * pk;
  float* sU = sK + MC * pk;
  float* sV = sU + MC * pk;
  float* sO = sV + MC * pv;
  float* sTot = sO + MC * pv;
  float* sCarry = sTot + 128;
  float* rest = sCarry + 128;
  // factorised form
  float* sDB = rest;                 // [MC][pk]   Q~ dQ~ - K^ dK^
  float* sS = sDB + MC * pk;         // [dk][pv]   G, then D
  float* sA = sS + a.dk * pv;        // [MC][MC+1] mask(dO V^T)
  float* sP = sA + MC * pa;          // [MC][MC+1] mask(Q~ K^T)
  // token-by-token form
  float* sGg = rest;                 // [dk][pv]
  float* sW = sGg + a.dk * pv;       // [dk][pv]

  const int f0 = chunk_first_base_pos(a.g, c, MC);
  stage<MC>(sQ, a.q, a.dk, a.g, f0, b, h, a.H);
  stage<MC>(sK, a.k, a.dk, a.g, f0, b, h, a.H);
  stage<MC>(sU, a.la, a.dk, a.g, f0, b, h, a.H);
  stage<MC>(sV, a.v, a.dv, a.g, f0, b, h, a.H);
  stage<MC>(sO, a.dout, a.dv, a.g, f0, b, h, a.H);
  const int64_t cid = (int64_t)bh * a.NC + c;
  __syncthreads();
  if (a.flags[cid]) {
    chunk_serial_bwd<TI, MC>(a, sQ, sK, sU, sV, sO, sGg, sW, c, b, h, f0);
    return;
  }
  suffix_sums<MC>(sU, sTot, a.dk, a.g.reverse);
  __syncthreads();
  const size_t st = (size_t)a.dk * a.dv;
  const float* sin = c > 0 ? a.sx + (cid - 1) * st : nullptr;
  for (int e = threadIdx.x; e < MC * a.dk; e += NT) {
    const int r = e / a.dk, i = e - r * a.dk;
    const float u = sU[r * pk + i];
    sQ[r * pk + i] *= expf(-u);
    sK[r * pk + i] *= expf(u);
  }
  for (int e = threadIdx.x; e < a.dk * a.dv; e += NT) {
    const int i = e / a.dv, j = e - i * a.dv;
    sS[i * pv + j] = sin ? expf(sTot[i]) * sin[e] : 0.f;
  }
  __syncthreads();
  const bool rev = a.g.reverse;
  // Positions s <= r in scan order are tile rows s <= r, or s >= r for reversed
  // directions: the nonzero range of a row block of A or P, and of a column block.
  auto lo_of_rows = [&](int r0) { return rev ? r0 : 0; };
  auto hi_of_rows = [&](int r0) { return rev ? MC : r0 + kTR; };
  auto lo_of_cols = [&](int s0) { return rev ? 0 : s0; };
  auto hi_of_cols = [&](int s0) { return rev ? s0 + kTR : MC; };
  // A = mask(dO V^T) (blocks 0 .. nm-1) and P = mask(Q~ K^T) (nm .. 2nm-1), MC x MC.
  {
    const int ncg = MC / 8, nm = (MC / kTR) * ncg;
    for (int t = threadIdx.x; t < 2 * nm; t += NT) {
      const int which = t >= nm, tt = which ? t - nm : t;
      const int r0 = kTR * (tt / ncg), s0 = 8 * (tt % ncg);
      float acc[kTR][8];
      zero48<kTR>(acc);
      const bool empty = rev ? (s0 + 7 < r0) : (s0 > r0 + kTR - 1);
      if (!empty) {
        if (which)
          mt48<kTR>(acc, sQ + r0 * pk, pk, 1, sK + s0 * pk, 1, pk, a.dk);
        else
          mt48<kTR>(acc, sO + r0 * pv, pv, 1, sV + s0 * pv, 1, pv, a.dv);
      }
      float* dst = which ? sP : sA;
#pragma unroll
      for (int i = 0; i < kTR; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int r = r0 + i, s2 = s0 + j;
          const bool keep = rev ? (s2 >= r) : (s2 <= r);
          dst[r * pa + s2] = keep ? acc[i][j] : 0.f;
        }
    }
  }
  __syncthreads();
  // dQ~ = dO G^T + A K^ (MC x dk)
  {
    const int ncg = a.dk / 8, nb = (MC / kTR) * ncg;
    for (int t = threadIdx.x; t < nb; t += NT) {
      const int r0 = kTR * (t / ncg), i0 = 8 * (t % ncg);
      float acc[kTR][8];
      zero48<kTR>(acc);
      mt48<kTR>(acc, sO + r0 * pv, pv, 1, sS + i0 * pv, 1, pv, a.dv);
      const int lo = lo_of_rows(r0), hi = hi_of_rows(r0);
      mt48<kTR>(acc, sA + r0 * pa + lo, pa, 1, sK + lo * pk + i0, pk, 1, hi - lo);
#pragma unroll
      for (int i = 0; i < kTR; ++i) {
        const int r = r0 + i, f = f0 + r;
        const bool real = f >= 0 && f < a.g.T;
        const int64_t o = real ? row_off(a, b, h, f, a.dk) : 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int ii = i0 + j;
          sDB[r * pk + ii] = sQ[r * pk + ii] * acc[i][j];
          if (real) store1(a.dq + o + ii, expf(-sU[r * pk + ii]) * acc[i][j]);
        }
      }
    }
  }
  __syncthreads();
  const float* dd = a.dd + cid * st;
  for (int e = threadIdx.x; e < a.dk * a.dv; e += NT) {
    const int i = e / a.dv, j = e - i * a.dv;
    sS[i * pv + j] = dd[e];
  }
  __syncthreads();
  // dK^ = A^T Q~ + V D^T (MC x dk, blocks 0 .. nk-1) and dV = P^T dO + K^ D (MC x dv,
  // blocks nk .. nk+nv-1)
  {
    const int nck = a.dk / 8, ncv = a.dv / 8, nk = (MC / kTR) * nck, nv = (MC / kTR) * ncv;
    for (int t = threadIdx.x; t < nk + nv; t += NT) {
      const bool isv = t >= nk;
      const int tt = isv ? t - nk : t;
      const int nc = isv ? ncv : nck;
      const int s0 = kTR * (tt / nc), c0 = 8 * (tt % nc);
      const int lo = lo_of_cols(s0), hi = hi_of_cols(s0);
      float acc[kTR][8];
      zero48<kTR>(acc);
      if (!isv) {
        mt48<kTR>(acc, sA + lo * pa + s0, 1, pa, sQ + lo * pk + c0, pk, 1, hi - lo);
        mt48<kTR>(acc, sV + s0 * pv, pv, 1, sS + c0 * pv, 1, pv, a.dv);
      } else {
        mt48<kTR>(acc, sP + lo * pa + s0, 1, pa, sO + lo * pv + c0, pv, 1, hi - lo);
        mt48<kTR>(acc, sK + s0 * pk, pk, 1, sS + c0, pv, 1, a.dk);
      }
#pragma unroll
      for (int i = 0; i < kTR; ++i) {
        const int s2 = s0 + i, f = f0 + s2;
        const bool real = f >= 0 && f < a.g.T;
        if (!isv) {
          const int64_t o = real ? row_off(a, b, h, f, a.dk) : 0;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int ii = c0 + j;
            sDB[s2 * pk + ii] = fmaf(-sK[s2 * pk + ii], acc[i][j], sDB[s2 * pk + ii]);
            if (real) store1(a.dk_out + o + ii, expf(sU[s2 * pk + ii]) * acc[i][j]);
          }
        } else if (real) {
          const int64_t o = row_off(a, b, h, f, a.dv);
#pragma unroll
          for (int j = 0; j < 8; ++j) store1(a.dv_out + o + c0 + j, acc[i][j]);
        }
      }
    }
  }
  // gradient of a gate at the chunk's end: sum_j D[i][j] S_in(c+1)[i][j]
  chunk_carry(a.dd + cid * st, a.sx + cid * st, a.dk, a.dv, sCarry);
  __syncthreads();
  // dlog_alpha_r = carry + sum of db over the chunk's positions at or after r
  for (int i = threadIdx.x; i < a.dk; i += NT) {
    float acc = sCarry[i];
    for (int step = MC - 1; step >= 0; --step) {
      const int r = rev ? (MC - 1 - step) : step;
      acc += sDB[r * pk + i];
      const int f = f0 + r;
      if (f >= 0 && f < a.g.T) a.dla[row_off(a, b, h, f, a.dk) + i] = acc;
    }
  }
}

// ---------------------------------------------------------------------------
// Kernel 3 on tensor cores (bf16 inputs, dk and dv at most 80): chunks of 128 rows,
// one CTA per chunk, every product a tcgen05 MMA (M = 128) from bf16 tiles in shared
// memory into fp32 TMEM accumulators:
//   A = dO V^T, P = Q~ K^^T                     (then masked and rounded to bf16)
//   dQ~ = dO G^T + A K^,  dK^ = A^T Q~ + V D^T,  dV = P^T dO + K^ D
// Tiles use the 32-byte swizzle in 16-channel blocks of `rows` rows; one tile serves as
// a K-major operand (rows = M or N, K = channels) and, transposed, as an MN-major one
// (K = rows).  The masked A and P are written back to shared memory once and read both
// ways.  Chunks flagged by kernel 1 take an exact token-by-token sweep instead.
// ---------------------------------------------------------------------------
constexpr int kTcRows = 128;
constexpr int kTcChunkNT = 512;  // threads of the gradient kernel (16 warps, one CTA per SM)
constexpr uint32_t kLayoutSW32b = 6;  // UMMA layout type of the 32-byte swizzle

__device__ __forceinline__ uint32_t sw32_at(uint32_t rows, uint32_t r, uint32_t ch) {
  return (ch >> 4) * (rows * 32u) + r * 32u + (((((ch >> 3) & 1u) ^ (r >> 2)) & 1u) << 4) + (ch & 7u) * 2u;
}
// Operand descriptors of a tile with `rows` rows: K-major (rows = M or N, K step kk =
// channels 16kk..16kk+15, one 32-byte-swizzled block of rows * 32 bytes each) or
// MN-major (MN = channels, K step kk = rows 16kk..16kk+15, 512 bytes further).
// The K steps of one operand: step kk's descriptor is the first one with its start
// address field (the byte address / 16) advanced by kk * inc.  Tiles lie below 256 KB
// of shared memory, so the field never carries into the next one; an MMA then costs
// its issuing thread one add per operand instead of a descriptor build.
struct OpSteps {
  uint64_t d0, inc;
  __device__ __forceinline__ uint64_t at(int kk) const { return d0 + (uint64_t)kk * inc; }
};
__device__ __forceinline__ OpSteps km_steps(uint32_t tile, uint32_t rows) {
  return OpSteps{umma_desc(tile, 16u, 256u, kLayoutSW32b), (uint64_t)(rows * 32u >> 4)};
}
__device__ __forceinline__ OpSteps mn_steps(uint32_t tile, uint32_t rows) {
  return OpSteps{umma_desc(tile, rows * 32u, 256u, kLayoutSW32b), (uint64_t)(512u >> 4)};
}

__device__ __forceinline__ void tc_ld16(uint32_t taddr, float (&v)[16]) { tmem_ld16(taddr, v); }
// 16-column TMEM load without its wait (several loads share one tcgen05.wait::ld),
// and the tie that orders every later use of the registers after that wait.
__device__ __forceinline__ void tc_ld16_issue(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tc_tie16(uint32_t (&r)[16]) {
  asm volatile(""
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                 "+r"(r[15]));
}
// Waits until at most N of this thread's cp.async groups are still in flight.
template <int N>
__device__ __forceinline__ void cp_async_wait_group() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Token index of each of the chunk's rows (base positions f0 .. f0+127), -1 for rows
// outside the sequence; the staging and the d log alpha stores index through it.
__device__ __forceinline__ void tc_row_tokens(int* sRow, const ScanGeom& g, int f0) {
  for (int r = threadIdx.x; r < kTcRows; r += blockDim.x) {
    const int f = f0 + r;
    sRow[r] = (f >= 0 && f < g.T) ? base_pos_to_token(g, f) : -1;
  }
}
template <typename TI>
__device__ __forceinline__ int64_t tok_off(const BwdArgs<TI>& a, int b, int h, int tok, int d) {
  return (((int64_t)b * a.g.T + tok) * a.H + h) * d;
}

// Asynchronous staging of the chunk's rows (zero outside the sequence and past d):
// bf16 operand tiles in the 32-byte-swizzled layout (`nch` channels, a multiple of 8)
// and the fp32 log-gate tile with a pitch of dk + 4 floats.  Every 16-byte copy of the
// CTA is in flight at once; the caller waits with cp_async_wait_all and a barrier.
template <typename TI>
__device__ __forceinline__ void tc_stage_bf16(uint8_t* sm, uint32_t tile, const __nv_bfloat16* src, int d, int nch,
                                              const BwdArgs<TI>& a, const int* sRow, int b, int h) {
  const int cc_n = nch / 8;
  for (int idx = threadIdx.x; idx < kTcRows * cc_n; idx += blockDim.x) {
    const int r = idx % kTcRows, cc = idx / kTcRows;
    const int tok = sRow[r];
    const bool valid = tok >= 0 && cc * 8 < d;
    const __nv_bfloat16* p = valid ? src + tok_off(a, b, h, tok, d) + cc * 8 : src;
    cp_async16(smem_u32(sm + tile + sw32_at(kTcRows, (uint32_t)r, (uint32_t)(cc * 8))), p, valid);
  }
}
template <typename TI>
__device__ __forceinline__ void tc_stage_gates(float* sU, const BwdArgs<TI>& a, const int* sRow, int b, int h) {
  const int cpr = a.dk / 4, pw = a.dk + 4;
  for (int idx = threadIdx.x; idx < kTcRows * cpr; idx += blockDim.x) {
    const int r = idx / cpr, cc = idx - r * cpr;
    const int tok = sRow[r];
    const float* p = tok >= 0 ? a.la + tok_off(a, b, h, tok, a.dk) + cc * 4 : a.la;
    cp_async16(smem_u32(sU + r * pw + cc * 4), p, tok >= 0);
  }
}
// n fp32 values (a multiple of 4) from src, or zeros when src is null.
__device__ __forceinline__ void tc_stage_f32(float* dst, const float* src, int n, const float* any) {
  for (int e = 4 * (int)threadIdx.x; e < n; e += 4 * (int)blockDim.x) cp_async16(smem_u32(dst + e), src ? src + e : any, src != nullptr);
}

// Segmented walks along a chunk's scan order: thread t takes channel i = t % dk and
// segment s = t / dk, the scan steps [st0, st1) of nseg nearly equal segments, as
// many as the block has threads for (at most 8).  A walk first needs the totals of the
// other segments (phase 1, one barrier), then runs over its own steps only.
constexpr int kMaxSegs = 8;
struct SegWalk {
  int i, s, nseg, st0, st1;
  bool active;
};
__device__ __forceinline__ SegWalk seg_walk(int dk) {
  SegWalk w;
  w.nseg = min(kMaxSegs, (int)blockDim.x / dk);
  const int len = (kTcRows + w.nseg - 1) / w.nseg;
  w.i = (int)threadIdx.x % dk;
  w.s = (int)threadIdx.x / dk;
  w.active = w.s < w.nseg;
  w.st0 = w.s * len;
  w.st1 = min(w.st0 + len, kTcRows);
  return w;
}
// Sums of the other segments' totals (sPart[s][i], 128 floats per segment): those
// before s in scan order and those after it, each added in a fixed order.
__device__ __forceinline__ void seg_offsets(const SegWalk& w, const float* sPart, float& before, float& after) {
  before = 0.f;
  after = 0.f;
  for (int s2 = 0; s2 < w.s; ++s2) before += sPart[s2 * kTcRows + w.i];
  for (int s2 = w.nseg - 1; s2 > w.s; --s2) after += sPart[s2 * kTcRows + w.i];
}
__device__ __forceinline__ int seg_row(int st, bool rev) { return rev ? (kTcRows - 1 - st) : st; }
// The same segmentation over channel pairs (p = t % (dk/2)): 6 to 8 segments of at
// most kPairSegMax steps for dk <= 80 and 256 threads.
constexpr int kPairSegMax = 22;  // ceil(128 / 6)
struct PairWalk {
  int p, s, nseg, st0, st1;
  bool active;
};
__device__ __forceinline__ PairWalk pair_walk(int dk) {
  const int np = dk / 2;
  PairWalk w;
  w.nseg = min(kMaxSegs, (int)blockDim.x / np);
  const int len = (kTcRows + w.nseg - 1) / w.nseg;
  w.p = (int)threadIdx.x % np;
  w.s = (int)threadIdx.x / np;
  w.active = w.s < w.nseg;
  w.st0 = w.s * len;
  w.st1 = min(w.st0 + len, kTcRows);
  return w;
}


// Exact sweep of a flagged chunk from fp32 tiles (alpha, k, v) staged in shared
// memory; q and dout rows are read from global memory one position at a time.
__device__ void tc_chunk_serial(const BwdArgs<__nv_bfloat16>& a, float* smem, int c, int b, int h, int f0) {
  constexpr int MC = kTcRows;
  const int pk = pitch_of(a.dk), pv = pitch_of(a.dv);
  float* sAl = smem;                 // [MC][pk] alpha
  float* sK = sAl + MC * pk;         // [MC][pk]
  float* sV = sK + MC * pk;          // [MC][pv]
  float* sGg = sV + MC * pv;         // [dk][pv] gradient of the state
  float* sW = sGg + a.dk * pv;       // [dk][pv] S_{r-1}
  stage<MC>(sAl, a.la, a.dk, a.g, f0, b, h, a.H);
  stage<MC>(sK, a.k, a.dk, a.g, f0, b, h, a.H);
  stage<MC>(sV, a.v, a.dv, a.g, f0, b, h, a.H);
  const int64_t cid = (int64_t)blockIdx.y * a.NC + c;
  const size_t st = (size_t)a.dk * a.dv;
  const float* sin = c > 0 ? a.sx + (cid - 1) * st : nullptr;
  const float* dd = a.dd + cid * st;
  for (int e = threadIdx.x; e < a.dk * a.dv; e += blockDim.x) {
    const int i = e / a.dv, j = e - i * a.dv;
    sGg[i * pv + j] = dd[e];
  }
  __syncthreads();
  for (int e = threadIdx.x; e < MC * a.dk; e += blockDim.x) {
    const int r = e / a.dk, i = e - r * a.dk;
    sAl[r * pk + i] = expf(sAl[r * pk + i]);
  }
  __syncthreads();
  for (int step = MC - 1; step >= 0; --step) {
    const int r = a.g.reverse ? (MC - 1 - step) : step;
    const int f = f0 + r;
    const bool real = f >= 0 && f < a.g.T;
    const int64_t ok = real ? row_off(a, b, h, f, a.dk) : 0;
    const int64_t ov = real ? row_off(a, b, h, f, a.dv) : 0;
    for (int e = threadIdx.x; e < a.dk * a.dv; e += blockDim.x) {
      const int i = e / a.dv, j = e - i * a.dv;
      float w = sin ? sin[e] : 0.f;
      for (int s2 = 0; s2 < step; ++s2) {
        const int r2 = a.g.reverse ? (MC - 1 - s2) : s2;
        w = fmaf(sAl[r2 * pk + i], w, sK[r2 * pk + i] * sV[r2 * pv + j]);
      }
      sW[i * pv + j] = w;
      if (real) {
        const float qi = __bfloat162float(a.q[ok + i]), oj = __bfloat162float(a.dout[ov + j]);
        sGg[i * pv + j] = fmaf(qi, oj, sGg[i * pv + j]);
      }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < a.dk; i += blockDim.x) {
      const float al = sAl[r * pk + i], ki = sK[r * pk + i];
      float gq = 0.f, gk = 0.f, gl = 0.f;
      for (int j = 0; j < a.dv; ++j) {
        const float sr = fmaf(al, sW[i * pv + j], ki * sV[r * pv + j]);
        if (real) gq = fmaf(__bfloat162float(a.dout[ov + j]), sr, gq);
        gk = fmaf(sGg[i * pv + j], sV[r * pv + j], gk);
        gl = fmaf(sGg[i * pv + j], sW[i * pv + j], gl);
      }
      if (real) {
        store1(a.dq + ok + i, gq);
        store1(a.dk_out + ok + i, gk);
        a.dla[ok + i] = al * gl;
      }
    }
    for (int j = threadIdx.x; j < a.dv; j += blockDim.x) {
      float gv = 0.f;
      for (int i = 0; i < a.dk; ++i) gv = fmaf(sK[r * pk + i], sGg[i * pv + j], gv);
      if (real) store1(a.dv_out + ov + j, gv);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < a.dk * a.dv; e += blockDim.x) {
      const int i = e / a.dv, j = e - i * a.dv;
      sGg[i * pv + j] *= sAl[r * pk + i];
    }
    __syncthreads();
  }
}

struct TcLayout {
  uint32_t oQ, oK, oV, oO, oA, oP, oG, oD, oU, oMisc, bytes;
  int nst;  // fp32 chunk states staged in the A/P area: S_in, D, and S_out when it fits
};
__host__ __device__ inline TcLayout tc_layout(int dk, int dv) {
  const uint32_t Kp = (uint32_t)(dk + 15) / 16 * 16, Np = (uint32_t)(dv + 15) / 16 * 16;
  TcLayout L;
  L.oQ = 0;
  L.oK = L.oQ + Kp / 16 * kTcRows * 32u;
  L.oV = L.oK + Kp / 16 * kTcRows * 32u;
  L.oO = L.oV + Np / 16 * kTcRows * 32u;
  L.oA = L.oO + Np / 16 * kTcRows * 32u;
  L.oP = L.oA + 8u * kTcRows * 32u;
  L.oG = L.oP + 8u * kTcRows * 32u;
  L.oD = L.oG + (Np / 16) * Kp * 32u;
  L.oU = L.oD + (Np / 16) * Kp * 32u;
  L.oMisc = (L.oU + (uint32_t)kTcRows * (uint32_t)(dk + 4) * 4u + 15u) / 16u * 16u;
  // gate totals, e^{totals}, carry (128 floats each), segment totals (8 x 128), row
  // tokens (128), barrier and TMEM address; alignment slack
  L.bytes = L.oMisc + 3u * 512u + 4096u + 512u + 64u + 1024u;
  L.nst = 3u * (uint32_t)dk * (uint32_t)dv * 4u <= 2u * 8u * kTcRows * 32u ? 3 : 2;
  return L;
}

__global__ void __launch_bounds__(kTcChunkNT, 1) gla_bwd_tc_chunk(const BwdArgs<__nv_bfloat16> a) {
  extern __shared__ __align__(1024) uint8_t smem_raw_tc[];
  // Swizzled operand tiles start on a 1024-byte boundary.
  uint8_t* smem_tc = smem_raw_tc + ((1024u - (smem_u32(smem_raw_tc) & 1023u)) & 1023u);
  constexpr int MC = kTcRows;
  const int c = blockIdx.x, bh = blockIdx.y;
  const int b = bh / a.H, h = bh % a.H;
  const TcLayout L = tc_layout(a.dk, a.dv);
  const uint32_t Kp = (uint32_t)(a.dk + 15) / 16 * 16, Np = (uint32_t)(a.dv + 15) / 16 * 16;
  const uint32_t sb = smem_u32(smem_tc);
  float* sU = reinterpret_cast<float*>(smem_tc + L.oU);   // [MC][dk+4]: log-gates, u, then db
  float* sTot = reinterpret_cast<float*>(smem_tc + L.oMisc);
  float* sGam = sTot + 128;
  float* sCarry = sGam + 128;
  float* sPart = sCarry + 128;                            // [8][128] segment totals
  int* sRow = reinterpret_cast<int*>(sPart + kMaxSegs * 128);  // [128] row tokens
  uint64_t* sBar = reinterpret_cast<uint64_t*>(sRow + 128);
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(sBar + 1);
  // fp32 chunk states, staged over the A and P tiles (written only after the first MMAs)
  float* sSin = reinterpret_cast<float*>(smem_tc + L.oA);
  const int dkv = a.dk * a.dv;
  float* sDs = sSin + dkv;
  float* sSo = sDs + dkv;
  const int pu = a.dk + 4;
  const int f0 = chunk_first_base_pos(a.g, c, MC);
  const int64_t cid = (int64_t)bh * a.NC + c;
  const bool rev = a.g.reverse;
  const size_t st = (size_t)dkv;

  if (a.flags[cid]) {
    tc_chunk_serial(a, reinterpret_cast<float*>(smem_tc), c, b, h, f0);
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0) {
    tmem_alloc(smem_u32(sTmem), 512);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(sBar), 1);
    fence_mbar_init();
  }
  tc_row_tokens(sRow, a.g, f0);
  __syncthreads();
  // ---- staging, all in flight together, in three groups waited for in the order of
  // use: log-gates (fp32); q, k (bf16, swizzled, zero past the channels and rows);
  // v, dout, S_in, D and (when it fits) S_out
  tc_stage_gates(sU, a, sRow, b, h);
  cp_async_commit();
  tc_stage_bf16(smem_tc, L.oQ, a.q, a.dk, (int)Kp, a, sRow, b, h);
  tc_stage_bf16(smem_tc, L.oK, a.k, a.dk, (int)Kp, a, sRow, b, h);
  cp_async_commit();
  tc_stage_bf16(smem_tc, L.oV, a.v, a.dv, (int)Np, a, sRow, b, h);
  tc_stage_bf16(smem_tc, L.oO, a.dout, a.dv, (int)Np, a, sRow, b, h);
  tc_stage_f32(sSin, c > 0 ? a.sx + (cid - 1) * st : nullptr, dkv, a.la);
  tc_stage_f32(sDs, a.dd + cid * st, dkv, a.la);
  if (L.nst == 3) tc_stage_f32(sSo, a.sx + cid * st, dkv, a.la);
  cp_async_commit();
  cp_async_wait_group<2>();
  __syncthreads();
  // ---- u: exclusive suffix sums of the log-gates in scan order, in place (segmented)
  const SegWalk w = seg_walk(a.dk);
  if (w.active) {
    float t = 0.f;
    for (int st2 = w.st0; st2 < w.st1; ++st2) t += sU[seg_row(st2, rev) * pu + w.i];
    sPart[w.s * MC + w.i] = t;
  }
  __syncthreads();
  if (w.active) {
    float before, acc;
    seg_offsets(w, sPart, before, acc);
#pragma unroll 4
    for (int st2 = w.st1 - 1; st2 >= w.st0; --st2) {
      float* p = sU + seg_row(st2, rev) * pu + w.i;
      const float l = *p;
      *p = acc;
      acc += l;
    }
    if (w.s == 0) {
      sTot[w.i] = acc;
      sGam[w.i] = expf(acc);
    }
  }
  cp_async_wait_group<1>();
  __syncthreads();
  {
    // Q~ = q e^{-u}, K^ = k e^{u} in place (8 channels per thread), padding stays 0
    const int cq = (int)Kp / 8;
    for (int idx = threadIdx.x; idx < MC * cq; idx += blockDim.x) {
      const int r = idx % MC, cc = idx / MC;
      if (cc * 8 >= a.dk) continue;
      uint4* pq = reinterpret_cast<uint4*>(smem_tc + L.oQ + sw32_at(MC, (uint32_t)r, (uint32_t)(cc * 8)));
      uint4* pk = reinterpret_cast<uint4*>(smem_tc + L.oK + sw32_at(MC, (uint32_t)r, (uint32_t)(cc * 8)));
      uint4 wq = *pq, wk = *pk;
      uint32_t* uq = reinterpret_cast<uint32_t*>(&wq);
      uint32_t* uk = reinterpret_cast<uint32_t*>(&wk);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float u0 = sU[r * pu + cc * 8 + 2 * e], u1 = sU[r * pu + cc * 8 + 2 * e + 1];
        const float2 xq = unpack_bf16x2(uq[e]), xk = unpack_bf16x2(uk[e]);
        uq[e] = pack_bf16x2(xq.x * __expf(-u0), xq.y * __expf(-u1));
        uk[e] = pack_bf16x2(xk.x * __expf(u0), xk.y * __expf(u1));
      }
      *pq = wq;
      *pk = wk;
    }
    cp_async_wait_group<0>();
    __syncthreads();
    // G[i][j] = e^{g_i} S_in[i][j] and D[i][j] as bf16 tiles, rows i < Kp, channels
    // j < Np, eight channels (one 16-byte tile row piece) per item; dv is a multiple of 8
    const int n8 = (int)Np / 8;
    for (int idx = threadIdx.x; idx < (int)Kp * n8; idx += blockDim.x) {
      const int i = idx / n8, j0 = 8 * (idx - i * n8);
      uint4 wg = make_uint4(0u, 0u, 0u, 0u), wd = wg;
      if (i < a.dk && j0 < a.dv) {
        const float4* ps = reinterpret_cast<const float4*>(sSin + i * a.dv + j0);
        const float4* pd = reinterpret_cast<const float4*>(sDs + i * a.dv + j0);
        const float4 s0 = ps[0], s1 = ps[1], d0 = pd[0], d1 = pd[1];
        const float gm = sGam[i];
        wg = make_uint4(pack_bf16x2(gm * s0.x, gm * s0.y), pack_bf16x2(gm * s0.z, gm * s0.w),
                        pack_bf16x2(gm * s1.x, gm * s1.y), pack_bf16x2(gm * s1.z, gm * s1.w));
        wd = make_uint4(pack_bf16x2(d0.x, d0.y), pack_bf16x2(d0.z, d0.w), pack_bf16x2(d1.x, d1.y),
                        pack_bf16x2(d1.z, d1.w));
      }
      *reinterpret_cast<uint4*>(smem_tc + L.oG + sw32_at(Kp, (uint32_t)i, (uint32_t)j0)) = wg;
      *reinterpret_cast<uint4*>(smem_tc + L.oD + sw32_at(Kp, (uint32_t)i, (uint32_t)j0)) = wd;
    }
    // carry[i] = sum_j D[i][j] S_out[i][j]: one warp per row, a fixed shuffle tree
    if (L.nst == 3) {
      for (int i = warp; i < a.dk; i += (int)(blockDim.x >> 5)) {
        float acc = 0.f;
        for (int j = lane; j < a.dv; j += 32) acc = fmaf(sDs[i * a.dv + j], sSo[i * a.dv + j], acc);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0) sCarry[i] = acc;
      }
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *sTmem;
  const uint32_t cA = 0, cP = 128, cDQ = 256, cDK = 256 + Kp, cDV = 256 + 2 * Kp;
  const uint32_t bar = smem_u32(sBar);
  bool ok = true;
  // ---- A = dO V^T, P = Q~ K^^T
  if (threadIdx.x == 0) {
    const uint32_t idS = idesc_bf16_f32(MC, MC, false, false);
    const OpSteps kO = km_steps(sb + L.oO, MC), kV = km_steps(sb + L.oV, MC);
    const OpSteps kQ = km_steps(sb + L.oQ, MC), kK = km_steps(sb + L.oK, MC);
    for (int kk = 0; kk < (int)Np / 16; ++kk) umma_ss(tbase + cA, kO.at(kk), kV.at(kk), idS, kk > 0 ? 1u : 0u);
    for (int kk = 0; kk < (int)Kp / 16; ++kk) umma_ss(tbase + cP, kQ.at(kk), kK.at(kk), idS, kk > 0 ? 1u : 0u);
    umma_commit(bar);
  }
  ok = __syncthreads_and(mbar_wait(bar, 0u));
  if (!ok && threadIdx.x == 0) report_status(GLA_ERR_TIMEOUT);
  tc_fence_after();
  // ---- mask and round: lane = row r (TMEM lane); the four warps of a lane quarter
  // split the 128 columns into quarters
  const int qd = warp & 3, hf = warp >> 2;  // hf: column quarter
  const int r = 32 * qd + lane;
  const uint32_t lane_base = (uint32_t)(32 * qd) << 16;
  if (ok) {
    for (int which = 0; which < 2; ++which) {
      const uint32_t col = which ? cP : cA;
      const uint32_t tile = which ? L.oP : L.oA;
      uint32_t xr[2][16];
      tc_ld16_issue(tbase + lane_base + col + (uint32_t)(32 * hf), xr[0]);
      tc_ld16_issue(tbase + lane_base + col + (uint32_t)(32 * hf + 16), xr[1]);
      tmem_ld_wait();
      tc_tie16(xr[0]);
      tc_tie16(xr[1]);
#pragma unroll
      for (int g = 0; g < 2; ++g) {
        const int s0 = 32 * hf + 16 * g;
        float x[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) x[e] = __uint_as_float(xr[g][e]);
        uint32_t wv[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int sa = s0 + 2 * e, sbb = sa + 1;
          const float x0 = (rev ? sa >= r : sa <= r) ? x[2 * e] : 0.f;
          const float x1 = (rev ? sbb >= r : sbb <= r) ? x[2 * e + 1] : 0.f;
          wv[e] = pack_bf16x2(x0, x1);
        }
        *reinterpret_cast<uint4*>(smem_tc + tile + sw32_at(MC, (uint32_t)r, (uint32_t)s0)) =
            make_uint4(wv[0], wv[1], wv[2], wv[3]);
        *reinterpret_cast<uint4*>(smem_tc + tile + sw32_at(MC, (uint32_t)r, (uint32_t)(s0 + 8))) =
            make_uint4(wv[4], wv[5], wv[6], wv[7]);
      }
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // ---- dQ~ = dO G^T + A K^,  dK^ = A^T Q~ + V D^T,  dV = P^T dO + K^ D
  if (threadIdx.x == 0 && ok) {
    const uint32_t idKK = idesc_bf16_f32(MC, (int)Kp, false, false);  // both K-major
    const uint32_t idKM = idesc_bf16_f32(MC, (int)Kp, false, true);   // B MN-major
    const uint32_t idMM = idesc_bf16_f32(MC, (int)Kp, true, true);    // both MN-major
    const uint32_t idVM = idesc_bf16_f32(MC, (int)Np, true, true);
    const uint32_t idVK = idesc_bf16_f32(MC, (int)Np, false, true);   // A K-major, B MN-major
    const OpSteps kO = km_steps(sb + L.oO, MC), kG = km_steps(sb + L.oG, Kp), kA = km_steps(sb + L.oA, MC);
    const OpSteps mK = mn_steps(sb + L.oK, MC), mA = mn_steps(sb + L.oA, MC), mQ = mn_steps(sb + L.oQ, MC);
    const OpSteps kV = km_steps(sb + L.oV, MC), kD = km_steps(sb + L.oD, Kp), mP = mn_steps(sb + L.oP, MC);
    const OpSteps mO = mn_steps(sb + L.oO, MC), kK = km_steps(sb + L.oK, MC), mD = mn_steps(sb + L.oD, Kp);
    for (int kk = 0; kk < (int)Np / 16; ++kk) umma_ss(tbase + cDQ, kO.at(kk), kG.at(kk), idKK, kk > 0 ? 1u : 0u);
    for (int kk = 0; kk < MC / 16; ++kk) umma_ss(tbase + cDQ, kA.at(kk), mK.at(kk), idKM, 1u);
    for (int kk = 0; kk < MC / 16; ++kk) umma_ss(tbase + cDK, mA.at(kk), mQ.at(kk), idMM, kk > 0 ? 1u : 0u);
    for (int kk = 0; kk < (int)Np / 16; ++kk) umma_ss(tbase + cDK, kV.at(kk), kD.at(kk), idKK, 1u);
    for (int kk = 0; kk < MC / 16; ++kk) umma_ss(tbase + cDV, mP.at(kk), mO.at(kk), idVM, kk > 0 ? 1u : 0u);
    for (int kk = 0; kk < (int)Kp / 16; ++kk) umma_ss(tbase + cDV, kK.at(kk), mD.at(kk), idVK, 1u);
    umma_commit(bar);
  }
  if (ok) {
    ok = __syncthreads_and(mbar_wait(bar, 1u));
    if (!ok && threadIdx.x == 0) report_status(GLA_ERR_TIMEOUT);
  }
  tc_fence_after();
  // ---- epilogue: row r, 16-channel groups g with g % 4 == hf
  const int tok = sRow[r];
  const bool real = tok >= 0;
  if (ok) {
    // q dq - k dk = Q~ dQ~ - K^ dK^, with Q~ and K^ the bf16 tiles of the MMAs.
    const int64_t ok_ = real ? tok_off(a, b, h, tok, a.dk) : 0;
    for (int g = hf; g < (int)Kp / 16; g += 4) {
      float xq[16], xk[16];
      tc_ld16(tbase + lane_base + cDQ + (uint32_t)(16 * g), xq);
      tc_ld16(tbase + lane_base + cDK + (uint32_t)(16 * g), xk);
      for (int half = 0; half < 2; ++half) {
        const int i0 = 16 * g + 8 * half;
        if (i0 >= a.dk) break;
        const uint4 wq = *reinterpret_cast<const uint4*>(smem_tc + L.oQ + sw32_at(MC, (uint32_t)r, (uint32_t)i0));
        const uint4 wk = *reinterpret_cast<const uint4*>(smem_tc + L.oK + sw32_at(MC, (uint32_t)r, (uint32_t)i0));
        const uint32_t* uq = reinterpret_cast<const uint32_t*>(&wq);
        const uint32_t* uk = reinterpret_cast<const uint32_t*>(&wk);
        uint32_t pq[4], pk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i = i0 + 2 * e;
          const float2 tq = unpack_bf16x2(uq[e]), tk = unpack_bf16x2(uk[e]);
          const float a0 = xq[8 * half + 2 * e], a1 = xq[8 * half + 2 * e + 1];
          const float b0 = xk[8 * half + 2 * e], b1 = xk[8 * half + 2 * e + 1];
          const float u0 = sU[r * pu + i], u1 = sU[r * pu + i + 1];
          pq[e] = pack_bf16x2(__expf(-u0) * a0, __expf(-u1) * a1);
          pk[e] = pack_bf16x2(__expf(u0) * b0, __expf(u1) * b1);
          sU[r * pu + i] = real ? tq.x * a0 - tk.x * b0 : 0.f;
          sU[r * pu + i + 1] = real ? tq.y * a1 - tk.y * b1 : 0.f;
        }
        if (real) {
          *reinterpret_cast<uint4*>(a.dq + ok_ + i0) = make_uint4(pq[0], pq[1], pq[2], pq[3]);
          *reinterpret_cast<uint4*>(a.dk_out + ok_ + i0) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
      }
    }
    const int64_t ov_ = real ? tok_off(a, b, h, tok, a.dv) : 0;
    for (int g = hf; g < (int)Np / 16; g += 4) {
      float xv[16];
      tc_ld16(tbase + lane_base + cDV + (uint32_t)(16 * g), xv);
      for (int half = 0; half < 2; ++half) {
        const int j0 = 16 * g + 8 * half;
        if (j0 >= a.dv || !real) break;
        *reinterpret_cast<uint4*>(a.dv_out + ov_ + j0) =
            make_uint4(pack_bf16x2(xv[8 * half], xv[8 * half + 1]), pack_bf16x2(xv[8 * half + 2], xv[8 * half + 3]),
                       pack_bf16x2(xv[8 * half + 4], xv[8 * half + 5]), pack_bf16x2(xv[8 * half + 6], xv[8 * half + 7]));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (!ok && threadIdx.x == 0) {
    // A wait ran out: let every MMA issued so far complete (bounded) before TMEM goes.
    umma_commit(bar);
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, 0u) && !mbar_try_wait(bar, 1u) && clock64() - t0 < kWaitCycles) {
    }
  }
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tbase, 512);
  if (!ok) return;
  if (L.nst != 3) {
    chunk_carry(a.dd + cid * st, a.sx + cid * st, a.dk, a.dv, sCarry);
    __syncthreads();
  }
  // ---- d log alpha_r = carry + sum over the chunk's rows at or after r of db
  // (segmented: segment totals, then each segment's walk from its end)
  if (w.active) {
    float t = 0.f;
    for (int st2 = w.st0; st2 < w.st1; ++st2) t += sU[seg_row(st2, rev) * pu + w.i];
    sPart[w.s * MC + w.i] = t;
  }
  __syncthreads();
  if (w.active) {
    float before, after;
    seg_offsets(w, sPart, before, after);
    float acc = sCarry[w.i] + after;
#pragma unroll 4
    for (int st2 = w.st1 - 1; st2 >= w.st0; --st2) {
      const int rr = seg_row(st2, rev);
      acc += sU[rr * pu + w.i];
      const int tk = sRow[rr];
      if (tk >= 0) a.dla[tok_off(a, b, h, tk, a.dk) + w.i] = acc;
    }
  }
}

// Kernel 1 on tensor cores (bf16 inputs, dk and dv at most 80): per 128-row chunk,
// K^T V and Qbar^T dO as M = 128 MMAs whose A operands are the k and q tiles read
// MN-major (M = key channels).  The tiles hold Kp channels; the MMA's A rows past Kp
// read whatever follows a tile (the next tile) and only reach accumulator rows past
// dk, which are never stored, so the tiles sit back to back and two CTAs fit per SM.
// Each thread (channel pair, segment) holds its log-gates in registers and gates Qbar
// and K^ during its two walks: no fp32 gate tile is staged.
struct TlLayout {
  uint32_t oK, oQ, oV, oO, oMisc, bytes;
};
__host__ __device__ inline TlLayout tl_layout(int dk, int dv) {
  const uint32_t Kp = (uint32_t)(dk + 15) / 16 * 16, Np = (uint32_t)(dv + 15) / 16 * 16;
  TlLayout L;
  L.oK = 0;
  L.oQ = Kp / 16 * kTcRows * 32u;
  L.oV = L.oQ + Kp / 16 * kTcRows * 32u;
  L.oO = L.oV + Np / 16 * kTcRows * 32u;
  const uint32_t end = L.oO + Np / 16 * kTcRows * 32u;
  const uint32_t reach = L.oQ + 8u * kTcRows * 32u;  // the q operand's last MMA read
  L.oMisc = end > reach ? end : reach;
  // segment totals (8 x 128 floats), row tokens (128), barrier, TMEM address; slack
  L.bytes = L.oMisc + 4096u + 512u + 64u + 1024u;
  return L;
}

__global__ void __launch_bounds__(NT, 2) gla_bwd_tc_local(const BwdArgs<__nv_bfloat16> a) {
  extern __shared__ __align__(1024) uint8_t smem_raw_tl[];
  uint8_t* sm = smem_raw_tl + ((1024u - (smem_u32(smem_raw_tl) & 1023u)) & 1023u);
  constexpr int MC = kTcRows;
  const int c = blockIdx.x, bh = blockIdx.y;
  const int b = bh / a.H, h = bh % a.H;
  const uint32_t Kp = (uint32_t)(a.dk + 15) / 16 * 16, Np = (uint32_t)(a.dv + 15) / 16 * 16;
  const TlLayout L = tl_layout(a.dk, a.dv);
  float* sPart = reinterpret_cast<float*>(sm + L.oMisc);  // [8][128] segment totals
  int* sRow = reinterpret_cast<int*>(sPart + kMaxSegs * 128);
  uint64_t* sBar = reinterpret_cast<uint64_t*>(sRow + 128);
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(sBar + 1);
  const uint32_t sb = smem_u32(sm);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool rev = a.g.reverse;
  const int f0 = chunk_first_base_pos(a.g, c, MC);
  const int64_t cid = (int64_t)bh * a.NC + c;
  if (warp == 0) {
    tmem_alloc(smem_u32(sTmem), 256);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(sBar), 1);
    fence_mbar_init();
  }
  tc_row_tokens(sRow, a.g, f0);
  __syncthreads();
  tc_stage_bf16(sm, L.oK, a.k, a.dk, (int)Kp, a, sRow, b, h);
  tc_stage_bf16(sm, L.oQ, a.q, a.dk, (int)Kp, a, sRow, b, h);
  tc_stage_bf16(sm, L.oV, a.v, a.dv, (int)Np, a, sRow, b, h);
  tc_stage_bf16(sm, L.oO, a.dout, a.dv, (int)Np, a, sRow, b, h);
  cp_async_commit();
  // This thread's log-gates (its channel pair, its segment's rows) into registers
  // while the tiles arrive; then the segment's totals.
  const PairWalk w = pair_walk(a.dk);
  float2 lg[kPairSegMax];
#pragma unroll
  for (int t = 0; t < kPairSegMax; ++t) {
    const int st2 = w.st0 + t;
    float2 x = make_float2(0.f, 0.f);
    if (w.active && st2 < w.st1) {
      const int tk = sRow[seg_row(st2, rev)];
      if (tk >= 0) x = *reinterpret_cast<const float2*>(a.la + tok_off(a, b, h, tk, a.dk) + 2 * w.p);
    }
    lg[t] = x;
  }
  if (w.active) {
    float2 t = make_float2(0.f, 0.f);
#pragma unroll
    for (int t2 = 0; t2 < kPairSegMax; ++t2) {
      t.x += lg[t2].x;
      t.y += lg[t2].y;
    }
    sPart[w.s * MC + 2 * w.p] = t.x;
    sPart[w.s * MC + 2 * w.p + 1] = t.y;
  }
  cp_async_wait_all();
  __syncthreads();
  int code = 0;
  if (w.active) {
    float2 before = make_float2(0.f, 0.f), after = make_float2(0.f, 0.f);
    for (int s2 = 0; s2 < w.s; ++s2) {
      before.x += sPart[s2 * MC + 2 * w.p];
      before.y += sPart[s2 * MC + 2 * w.p + 1];
    }
    for (int s2 = w.nseg - 1; s2 > w.s; --s2) {
      after.x += sPart[s2 * MC + 2 * w.p];
      after.y += sPart[s2 * MC + 2 * w.p + 1];
    }
    // Each walk loads its segment's pairs, gates them, then stores them all.
    uint32_t x[kPairSegMax];
    // tile offset of this thread's pair in scan step st2
    auto pair_at = [&](uint32_t tile, int st2) {
      return tile + sw32_at(MC, (uint32_t)seg_row(st2, rev), (uint32_t)(2 * w.p));
    };
    // Qbar = q e^{b}, b the inclusive prefix of the log-gates in scan order, built by
    // additions only (a -inf gate gives 0, not inf - inf)
#pragma unroll
    for (int t = 0; t < kPairSegMax; ++t) {
      const int st2 = w.st0 + t;
      if (st2 < w.st1) x[t] = *reinterpret_cast<const uint32_t*>(sm + pair_at(L.oQ, st2));
    }
    float2 acc = before;
#pragma unroll
    for (int t = 0; t < kPairSegMax; ++t) {
      if (w.st0 + t < w.st1) {
        acc.x += lg[t].x;
        acc.y += lg[t].y;
        const float2 xq = unpack_bf16x2(x[t]);
        x[t] = pack_bf16x2(xq.x * __expf(acc.x), xq.y * __expf(acc.y));
      }
    }
#pragma unroll
    for (int t = 0; t < kPairSegMax; ++t)
      if (w.st0 + t < w.st1) *reinterpret_cast<uint32_t*>(sm + pair_at(L.oQ, w.st0 + t)) = x[t];
    // K^ = k e^{u}, u the exclusive suffix (decays only shrink it); the range check
    // covers every u and the chunk total
#pragma unroll
    for (int t = 0; t < kPairSegMax; ++t) {
      const int st2 = w.st0 + t;
      if (st2 < w.st1) x[t] = *reinterpret_cast<const uint32_t*>(sm + pair_at(L.oK, st2));
    }
    acc = after;
    float lo = fminf(acc.x, acc.y), hi = fmaxf(acc.x, acc.y);
#pragma unroll
    for (int t = kPairSegMax - 1; t >= 0; --t) {
      if (w.st0 + t < w.st1) {
        const float2 xk = unpack_bf16x2(x[t]);
        x[t] = pack_bf16x2(xk.x * __expf(acc.x), xk.y * __expf(acc.y));
        acc.x += lg[t].x;
        acc.y += lg[t].y;
        lo = fminf(lo, fminf(acc.x, acc.y));
        hi = fmaxf(hi, fmaxf(acc.x, acc.y));
      }
    }
#pragma unroll
    for (int t = 0; t < kPairSegMax; ++t)
      if (w.st0 + t < w.st1) *reinterpret_cast<uint32_t*>(sm + pair_at(L.oK, w.st0 + t)) = x[t];
    if (w.s == 0) {
      a.gamma[cid * a.dk + 2 * w.p] = expf(acc.x);
      a.gamma[cid * a.dk + 2 * w.p + 1] = expf(acc.y);
    }
    if (!(lo >= -kRange) || !(hi <= kRange)) code |= 1;
    if (!(hi <= kRange)) code |= 2;
  }
  if (code & 2) report_status(GLA_ERR_RANGE);
  const int wide = __syncthreads_or(code != 0);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *sTmem;
  const uint32_t bar = smem_u32(sBar);
  if (threadIdx.x == 0) {
    const uint32_t id = idesc_bf16_f32(MC, (int)Np, true, true);
    const OpSteps mK = mn_steps(sb + L.oK, MC), mV = mn_steps(sb + L.oV, MC);
    const OpSteps mQ = mn_steps(sb + L.oQ, MC), mO = mn_steps(sb + L.oO, MC);
    for (int kk = 0; kk < MC / 16; ++kk) umma_ss(tbase, mK.at(kk), mV.at(kk), id, kk > 0 ? 1u : 0u);
    for (int kk = 0; kk < MC / 16; ++kk) umma_ss(tbase + 128, mQ.at(kk), mO.at(kk), id, kk > 0 ? 1u : 0u);
    umma_commit(bar);
  }
  const bool ok = __syncthreads_and(mbar_wait(bar, 0u));
  if (!ok && threadIdx.x == 0) report_status(GLA_ERR_TIMEOUT);
  tc_fence_after();
  // TMEM lane = key channel i; warps 0-3 write K^T V, warps 4-7 Qbar^T dO.
  if (ok) {
    const int i = 32 * (warp & 3) + lane;
    const uint32_t col = (warp >> 2) ? 128u : 0u;
    float* dst = ((warp >> 2) ? a.dd : a.sx) + cid * a.dk * a.dv + (size_t)i * a.dv;
    for (int g = 0; g < (int)Np / 16; ++g) {
      float x[16];
      tmem_ld16(tbase + ((uint32_t)(32 * (warp & 3)) << 16) + col + (uint32_t)(16 * g), x);
      if (i < a.dk)
        for (int q4 = 0; q4 < 4; ++q4)
          if (16 * g + 4 * q4 < a.dv)
            *reinterpret_cast<float4*>(dst + 16 * g + 4 * q4) =
                make_float4(x[4 * q4], x[4 * q4 + 1], x[4 * q4 + 2], x[4 * q4 + 3]);
    }
  }
  if (threadIdx.x == 0) a.flags[cid] = wide;
  tc_fence_before();
  __syncthreads();
  if (!ok && threadIdx.x == 0) {
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, 0u) && clock64() - t0 < kWaitCycles) {
    }
  }
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tbase, 256);
}

bool use_tc(const GlaShape& s, int bf16) { return bf16 && s.dk <= 80 && s.dv <= 80; }

size_t rup(size_t x, size_t m) { return (x + m - 1) / m * m; }

// 32-row chunks: the gradient kernel's shared memory then fits two blocks per SM (the
// phases of one block have few independent 4 x 8 blocks), which outweighs the longer
// chunk scans (c4: 13 % faster than 64-row chunks).
int chunk_rows(const GlaShape&) { return 32; }

template <int MC>
size_t smem_local(const GlaShape& s) {
  return ((size_t)MC * pitch_of(s.dk) * 3 + (size_t)MC * pitch_of(s.dv) * 2 + 128) * sizeof(float);
}

template <int MC>
size_t smem_chunk(const GlaShape& s) {
  const size_t pk = pitch_of(s.dk), pv = pitch_of(s.dv);
  const size_t tiles = MC * pk * 3 + MC * pv * 2 + 256;
  const size_t fact = MC * pk + s.dk * pv + 2 * (size_t)MC * (MC + 1);
  const size_t serial = 2 * (size_t)s.dk * pv;
  return (tiles + (fact > serial ? fact : serial)) * sizeof(float);
}

template <typename TI, int MC>
cudaError_t launch_bwd(const BwdArgs<TI>& a, const GlaShape& s, cudaStream_t st) {
  const size_t s1 = smem_local<MC>(s), s3 = smem_chunk<MC>(s);
  const bool two_rows = (MC / 2) * (s.dk / 8 + s.dv / 8) <= NT;
  auto chunk_kernel = two_rows ? gla_bwd_chunk<TI, MC, 2> : gla_bwd_chunk<TI, MC, 4>;
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(gla_bwd_local<TI, MC>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s1)) !=
      cudaSuccess)
    return e;
  if ((e = cudaFuncSetAttribute(chunk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s3)) != cudaSuccess)
    return e;
  const dim3 grid(a.NC, s.B * s.H);
  gla_bwd_local<TI, MC><<<grid, NT, s1, st>>>(a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  gla_bwd_scan<TI><<<dim3((s.dk * s.dv / 4 + 255) / 256, s.B * s.H), 256, 0, st>>>(a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  chunk_kernel<<<grid, NT, s3, st>>>(a);
  return cudaGetLastError();
}

// The tensor-core path: gla_bwd_tc_local, the chunk scans over 128-row chunks, then
// gla_bwd_tc_chunk.
cudaError_t launch_bwd_tc(const BwdArgs<__nv_bfloat16>& a, const GlaShape& s, cudaStream_t st) {
  const size_t s1 = tl_layout(s.dk, s.dv).bytes;
  const TcLayout L = tc_layout(s.dk, s.dv);
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(gla_bwd_tc_local, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s1)) !=
      cudaSuccess)
    return e;
  if ((e = cudaFuncSetAttribute(gla_bwd_tc_chunk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.bytes)) !=
      cudaSuccess)
    return e;
  const dim3 grid(a.NC, s.B * s.H);
  gla_bwd_tc_local<<<grid, NT, s1, st>>>(a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  gla_bwd_scan<__nv_bfloat16><<<dim3((s.dk * s.dv / 4 + 255) / 256, s.B * s.H), 256, 0, st>>>(a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  gla_bwd_tc_chunk<<<grid, kTcChunkNT, L.bytes, st>>>(a);
  return cudaGetLastError();
}

template <typename TI>
cudaError_t run_bwd(const void* q, const void* k, const void* v, const float* la, const void* dout, void* dq,
                    void* dk, void* dv, float* dla, const GlaShape& s, void* workspace, cudaStream_t st) {
  BwdArgs<TI> a;
  a.q = static_cast<const TI*>(q);
  a.k = static_cast<const TI*>(k);
  a.v = static_cast<const TI*>(v);
  a.la = la;
  a.dout = static_cast<const TI*>(dout);
  a.dq = static_cast<TI*>(dq);
  a.dk_out = static_cast<TI*>(dk);
  a.dv_out = static_cast<TI*>(dv);
  a.dla = dla;
  a.H = s.H;
  a.dk = s.dk;
  a.dv = s.dv;
  const bool tc = use_tc(s, sizeof(TI) == 2);
  const int MC = tc ? kTcRows : chunk_rows(s);
  a.NC = (s.T() + MC - 1) / MC;
  a.g = make_geom(s.Hg, s.Wg, s.dir);
  const size_t BH = (size_t)s.B * s.H;
  const size_t big = rup(BH * a.NC * s.dk * s.dv * 4, 256);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  a.sx = reinterpret_cast<float*>(ws);
  a.dd = reinterpret_cast<float*>(ws + big);
  a.gamma = reinterpret_cast<float*>(ws + 2 * big);
  a.flags = reinterpret_cast<int*>(ws + 2 * big + rup(BH * a.NC * s.dk * 4, 256));
  if constexpr (sizeof(TI) == 2) {
    if (tc) return launch_bwd_tc(a, s, st);
  }
  return MC == 64 ? launch_bwd<TI, 64>(a, s, st) : launch_bwd<TI, 32>(a, s, st);
}

}  // namespace

size_t gla_bwd_workspace_bytes(const GlaShape& s, int bf16) {
  const int MC = use_tc(s, bf16) ? kTcRows : chunk_rows(s);
  const size_t NC = (size_t)(s.T() + MC - 1) / MC;
  const size_t BH = (size_t)s.B * s.H;
  return rup(BH * NC * s.dk * s.dv * 4, 256) * 2 + rup(BH * NC * s.dk * 4, 256) + rup(BH * NC * 4, 256);
}

cudaError_t gla_bwd_launch(const void* q, const void* k, const void* v, const float* la, const void* dout, void* dq,
                           void* dk, void* dv, float* dla, const GlaShape& s, int bf16, void* workspace,
                           cudaStream_t st) {
  return bf16 ? run_bwd<__nv_bfloat16>(q, k, v, la, dout, dq, dk, dv, dla, s, workspace, st)
              : run_bwd<float>(q, k, v, la, dout, dq, dk, dv, dla, s, workspace, st);
}

}  // namespace dig
