// gla_tc.cu -- chunk-wise GLA forward with bf16 q/k/v on sm_100a tensor cores.
//
// The recurrence S_t = Diag(alpha_t) S_{t-1} + k_t^T v_t, o_t = q_t S_t (DiG:
// gated linear attention) is evaluated chunk-wise (DiG paper notes, "硬件友好的
// 效率设计": the sequence is cut into chunks computed in on-chip memory, cost
// O(T M D + T D^2)).  For a chunk of M = 128 scan positions with incoming state
// S_in, let u_r be the sum of the log-gates scanned AFTER row r inside the chunk
// (an exclusive suffix sum, per key channel) and g the chunk total.  Then, exactly:
//     gamma   = exp(g)                            (per key channel)
//     Q~_r    = q_r * exp(-u_r),   K^_s = k_s * exp(u_s)
//     O       = ((Q~ K^T) masked to scanned-before-or-same) V  +  Q~ (Diag(gamma) S_in)
//     S_out   = Diag(gamma) S_in + K^T V
// because exp(-u_t) exp(u_s) = prod of alpha over the positions after s up to t.
// Suffix sums avoid differences of large cumulative sums.  exp(-u) overflows when
// a chunk's gates decay by more than e^80 inside the chunk; such chunks (flagged by
// pass 1) take an exact token-by-token path in pass 3 from the fp32 incoming state,
// so every log_alpha <= 0, including -inf (a full reset), is handled exactly.
// Three passes:
//   (1) gla_tc_chunk_state: per chunk, S_loc = K^T V (tcgen05), gamma and the
//                           out-of-range flag.
//   (2) gla_tc_prefix:      per (b, h, key, value) element, the scan over chunks
//                           S_in(c+1) = G_c + S_loc(c), G_c = Diag(gamma_c) S_in(c);
//                           G_c is written as a ready-to-use bf16 MMA operand image
//                           (and S_in itself, fp32, for flagged chunks).
//   (3) gla_tc_output:      per chunk, O = mask(Q~ K^T) V + Q~ G_c (tcgen05).
// The scan direction never moves data: rows are gathered in the direction's
// base order (raster or column-major) and reversed directions flip the mask and
// the cumulative sum.
#include <math.h>

#include "dev_common.cuh"
#include "internal.h"

namespace dig {

// Zero-initialised device status word for this module (declared in dev_common.cuh).
__device__ int g_device_status = 0;

namespace {

constexpr int MC = kChunkTC;          // chunk length = MMA M = TMEM lanes used
constexpr int NT = 128;               // one thread per tile row / TMEM lane
constexpr uint32_t PART = MC * 128u;  // one 64-element, 128-row swizzled part: 16 KB
constexpr float kMaxGateRange = 80.0f;

struct TcArgs {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const float* la;
  __nv_bfloat16* out;
  float* s_locT;   // [BH][NC][dv][dk]  chunk-local states, transposed (fp32)
  float* gamma;    // [BH][NC][dk]      exp(total log-gate of the chunk)
  int* flags;      // [BH][NC]          1: gate range too wide for the factorised form
  uint8_t* g_img;  // [BH][NC][img]     bf16 image of G^T as a K-major swizzled operand
  int H, dk, dv, NC;
  int PK, PV, Np;  // 64-wide parts for dk / dv, dv rounded up to 16
  ScanGeom g;
};

__device__ __forceinline__ uint32_t g_img_bytes(int PK, int Np) { return (uint32_t)PK * (uint32_t)Np * 128u; }

// Stage tile rows r = 0..MC-1 (base positions f0 + r) of head h, batch b of a
// [B][T][H][d] bf16 tensor into `parts` swizzled 64-element parts.  Channels >= d
// and rows outside the sequence are zero-filled.
__device__ __forceinline__ void stage_bf16(uint32_t tile, const __nv_bfloat16* base, int d, int parts,
                                           const ScanGeom& g, int f0, int b, int h, int H) {
  const int cpr = parts * 8;
  for (int idx = threadIdx.x; idx < MC * cpr; idx += NT) {
    const int r = idx / cpr;
    const int cc = idx - r * cpr;
    const int ch = cc * 8;
    const int f = f0 + r;
    const bool valid = (f >= 0) && (f < g.T) && (ch < d);
    const __nv_bfloat16* src = base;
    if (valid) src = base + (((int64_t)b * g.T + base_pos_to_token(g, f)) * H + h) * d + ch;
    cp_async16(tile + (uint32_t)(cc >> 3) * PART + sw128((uint32_t)r, (uint32_t)(cc & 7) * 16u), src, valid);
  }
}

// Stage the fp32 log-gate rows into a plain row-major tile with a pitch of dk+4
// floats (conflict-free row-per-thread reads).  Padding rows are zero.
__device__ __forceinline__ void stage_la(uint32_t dst, const float* la, int dk, const ScanGeom& g, int f0,
                                         int b, int h, int H) {
  const int cpr = dk / 4;
  const uint32_t pitch = (uint32_t)(dk + 4) * 4u;
  for (int idx = threadIdx.x; idx < MC * cpr; idx += NT) {
    const int r = idx / cpr;
    const int cc = idx - r * cpr;
    const int f = f0 + r;
    const bool valid = (f >= 0) && (f < g.T);
    const float* src = la;
    if (valid) src = la + (((int64_t)b * g.T + base_pos_to_token(g, f)) * H + h) * dk + cc * 4;
    cp_async16(dst + (uint32_t)r * pitch + (uint32_t)cc * 16u, src, valid);
  }
}

// Threads i < dk: exclusive suffix sums u_r of the log-gate along the scan order,
// in place (u_r = sum of the log-gates scanned after row r); the chunk total goes
// to sBL[i].  Returns a bit set: kWide if some |u_r| exceeds the range whose
// exponential stays comfortably inside fp32 / bf16 (the chunk then takes the exact
// serial path), kGrowth if the gates GROW the state beyond that range (log_alpha
// > 0), which no fp32 evaluation can represent.
constexpr int kWide = 1, kGrowth = 2;
__device__ __forceinline__ int chunk_suffix(float* sLA, float* sBL, int dk, int reverse) {
  const int i = threadIdx.x;
  int code = 0;
  if (i < dk) {
    const int pw = dk + 4;
    float acc = 0.f, lo = 0.f, hi = 0.f;
    for (int s = 0; s < MC; ++s) {
      const int r = reverse ? s : (MC - 1 - s);  // walk the scan order backwards
      const float la = sLA[r * pw + i];
      sLA[r * pw + i] = acc;
      lo = fminf(lo, acc);
      hi = fmaxf(hi, acc);
      acc += la;
    }
    sBL[i] = acc;
    hi = fmaxf(hi, acc);
    if (!(lo >= -kMaxGateRange) || !(hi <= kMaxGateRange)) code |= kWide;
    if (!(hi <= kMaxGateRange)) code |= kGrowth;
  }
  return code;
}

// Row r (this thread): Q~ = q * exp(-u) and/or K^ = k * exp(u), in place in the
// swizzled bf16 tiles.  Padding channels stay zero.
template <bool DO_Q, bool DO_K>
__device__ __forceinline__ void gate_row(uint8_t* smem, uint32_t offQ, uint32_t offK, const float* sLA, int dk,
                                         int r) {
  const float* urow = sLA + r * (dk + 4);
  for (int c0 = 0; c0 < dk; c0 += 8) {
    const uint32_t o = (uint32_t)(c0 >> 6) * PART + sw128((uint32_t)r, (uint32_t)(c0 & 63) * 2u);
    const float4 u0 = *reinterpret_cast<const float4*>(urow + c0);
    const float4 u1 = *reinterpret_cast<const float4*>(urow + c0 + 4);
    const float e[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
    if (DO_Q) {
      uint4* p = reinterpret_cast<uint4*>(smem + offQ + o);
      uint4 w = *p;
      uint32_t* u = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 x = unpack_bf16x2(u[j]);
        u[j] = pack_bf16x2(x.x * __expf(-e[2 * j]), x.y * __expf(-e[2 * j + 1]));
      }
      *p = w;
    }
    if (DO_K) {
      uint4* p = reinterpret_cast<uint4*>(smem + offK + o);
      uint4 w = *p;
      uint32_t* u = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 x = unpack_bf16x2(u[j]);
        u[j] = pack_bf16x2(x.x * __expf(e[2 * j]), x.y * __expf(e[2 * j + 1]));
      }
      *p = w;
    }
  }
}

// bf16 element (row r, channel i) of a swizzled tile.
__device__ __forceinline__ float tile_at(const uint8_t* tile, int r, int i) {
  const uint32_t o = (uint32_t)(i >> 6) * PART + sw128((uint32_t)r, (uint32_t)(i & 63) * 2u);
  return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(tile + o));
}

// Exact token-by-token recurrence for one chunk, used when the chunk's gates
// decay too fast for the factorised form.  Thread j < dv keeps value column j of
// the fp32 state in registers, starting from S_in (stored [dv][dk] at `s_in`);
// sLA holds the raw log-gates of the chunk.
__device__ void chunk_serial(const uint8_t* sQ, const uint8_t* sK, const uint8_t* sV, float* sLA, const float* s_in,
                             const TcArgs& a, int f0, int b, int h) {
  const int pw = a.dk + 4;
  for (int e = threadIdx.x; e < MC * a.dk; e += NT) {
    const int r = e / a.dk, i = e - r * a.dk;
    sLA[r * pw + i] = __expf(sLA[r * pw + i]);  // alpha; exp(-inf) = 0 is a full reset
  }
  const int j = threadIdx.x;
  const bool own = j < a.dv;
  float st[128];
#pragma unroll
  for (int i = 0; i < 128; ++i) st[i] = (own && i < a.dk) ? s_in[(int64_t)j * a.dk + i] : 0.f;
  __syncthreads();
  for (int s = 0; s < MC; ++s) {
    const int r = a.g.reverse ? (MC - 1 - s) : s;
    const int f = f0 + r;
    if (f < 0 || f >= a.g.T) continue;  // padding rows (uniform across the block)
    if (own) {
      const float vj = tile_at(sV, r, j);
      const float* al = sLA + r * pw;
      float acc = 0.f;
#pragma unroll
      for (int i = 0; i < 128; ++i) {
        if (i < a.dk) {
          st[i] = fmaf(al[i], st[i], tile_at(sK, r, i) * vj);
          acc = fmaf(tile_at(sQ, r, i), st[i], acc);
        }
      }
      a.out[(((int64_t)b * a.g.T + base_pos_to_token(a.g, f)) * a.H + h) * a.dv + j] = __float2bfloat16_rn(acc);
    }
  }
}

__device__ __forceinline__ uint32_t align1024(uint32_t a) { return (a + 1023u) & ~1023u; }

// ---------------------------------------------------------------------------
// Pass 1: chunk-local state S_loc = K^T V and gamma.
// smem: sK (2 parts: the MMA's M = 128 spans key channels 0..127), sV (PV parts),
//       sLA (MC x (dk+4) fp32), sBL (dk fp32), mbarrier, TMEM base.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(NT, 1) gla_tc_chunk_state(const TcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t base_u32 = align1024(raw_u32);
  uint8_t* smem = smem_raw + (base_u32 - raw_u32);

  const int c = blockIdx.x;
  const int bh = blockIdx.y;
  const int b = bh / a.H, h = bh % a.H;
  const int tid = threadIdx.x, warp = tid >> 5;

  const uint32_t oK = 0;
  const uint32_t oV = oK + 2 * PART;
  const uint32_t oLA = oV + (uint32_t)a.PV * PART;
  const uint32_t oBL = oLA + (uint32_t)MC * (uint32_t)(a.dk + 4) * 4u;
  const uint32_t oBar = (oBL + (uint32_t)a.dk * 4u + 15u) & ~15u;
  const uint32_t oTm = oBar + 8;
  float* sLA = reinterpret_cast<float*>(smem + oLA);
  float* sBL = reinterpret_cast<float*>(smem + oBL);
  volatile uint32_t* sTm = reinterpret_cast<volatile uint32_t*>(smem + oTm);

  if (warp == 0) {
    tmem_alloc(base_u32 + oTm, 128);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(base_u32 + oBar, 1);
    fence_mbar_init();
  }

  const int f0 = chunk_first_base_pos(a.g, c, MC);
  stage_bf16(base_u32 + oK, a.k, a.dk, 2, a.g, f0, b, h, a.H);
  stage_bf16(base_u32 + oV, a.v, a.dv, a.PV, a.g, f0, b, h, a.H);
  stage_la(base_u32 + oLA, a.la, a.dk, a.g, f0, b, h, a.H);
  cp_async_commit();
  cp_async_wait_all();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *sTm;

  const int code = chunk_suffix(sLA, sBL, a.dk, a.g.reverse);
  if (code & kGrowth) report_status(GLA_ERR_RANGE);
  const int wide = __syncthreads_or(code != 0);
  gate_row<false, true>(smem, 0, oK, sLA, a.dk, tid);
  fence_proxy_async_smem();
  __syncthreads();

  if (tid == 0) {
    tc_fence_after();
    const uint32_t idesc = idesc_bf16_f32(MC, a.Np, true, true);
#pragma unroll 1
    for (int kk = 0; kk < MC / 16; ++kk)
      umma_ss(tbase, desc_mnmajor(base_u32 + oK, PART, kk), desc_mnmajor(base_u32 + oV, PART, kk), idesc,
              kk > 0 ? 1u : 0u);
    umma_commit(base_u32 + oBar);
  }
  const bool ok = mbar_wait(base_u32 + oBar, 0);
  tc_fence_after();
  if (!ok) report_status(GLA_ERR_TIMEOUT);

  // Epilogue: lane i holds row i of S_loc (key channel i).
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
  const int64_t chunk_id = (int64_t)bh * a.NC + c;
  float* dst = a.s_locT + chunk_id * a.dv * a.dk;
  for (int cb = 0; cb < a.Np; cb += 16) {
    float s[16];
    tmem_ld16(tbase + lane_base + (uint32_t)cb, s);
    if (ok && tid < a.dk) {
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (cb + j < a.dv) dst[(int64_t)(cb + j) * a.dk + tid] = s[j];
    }
  }
  if (tid < a.dk) a.gamma[chunk_id * a.dk + tid] = __expf(sBL[tid]);
  if (tid == 0) a.flags[chunk_id] = wide;

  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tbase, 128);
}

// ---------------------------------------------------------------------------
// Pass 2: scan over chunks, one thread per entry of the G^T image (Np rows j x
// PK*64 columns i, zero outside dv x dk).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) gla_tc_prefix(const TcArgs a) {
  const int bh = blockIdx.y;
  const int W = a.PK * 64;
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= a.Np * W) return;
  const int j = e / W, i = e - j * W;
  const bool valid = (j < a.dv) && (i < a.dk);
  const uint32_t img = g_img_bytes(a.PK, a.Np);
  const uint32_t off = (uint32_t)(i >> 6) * (uint32_t)a.Np * 128u + sw128((uint32_t)j, (uint32_t)(i & 63) * 2u);
  const int64_t first = (int64_t)bh * a.NC;
  float S = 0.f;
#pragma unroll 4
  for (int c = 0; c < a.NC; ++c) {
    const int64_t cid = first + c;
    const float gm = valid ? a.gamma[cid * a.dk + i] : 0.f;
    const float sl = valid ? a.s_locT[(cid * a.dv + j) * a.dk + i] : 0.f;
    const float G = gm * S;
    *reinterpret_cast<__nv_bfloat16*>(a.g_img + (size_t)cid * img + off) = __float2bfloat16_rn(G);
    if (valid && a.flags[cid]) a.s_locT[(cid * a.dv + j) * a.dk + i] = S;  // exact S_in for pass 3
    S = G + sl;
  }
}

// ---------------------------------------------------------------------------
// Pass 3: outputs.  smem: sQ, sK (PK parts), sV (PV parts), sP (2 parts: K = 128
// keys), sG (PK parts of Np rows), sLA, sBL, mbarrier, TMEM base.
// TMEM: columns [0,128) scores, [128, 128+Np) output accumulator.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(NT, 1) gla_tc_output(const TcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t base_u32 = align1024(raw_u32);
  uint8_t* smem = smem_raw + (base_u32 - raw_u32);

  const int c = blockIdx.x;
  const int bh = blockIdx.y;
  const int b = bh / a.H, h = bh % a.H;
  const int tid = threadIdx.x, warp = tid >> 5;

  const uint32_t gpart = (uint32_t)a.Np * 128u;
  const uint32_t la_bytes = (uint32_t)MC * (uint32_t)(a.dk + 4) * 4u;
  const uint32_t oQ = 0;
  const uint32_t oK = oQ + (uint32_t)a.PK * PART;
  const uint32_t oV = oK + (uint32_t)a.PK * PART;
  const uint32_t oG = oV + (uint32_t)a.PV * PART;
  // Scratch: the log-gate tile lives here until the gates are applied; the bf16
  // score tile P (2 parts, K = 128 keys) reuses it after the score MMA.
  const uint32_t oLA = oG + (uint32_t)a.PK * gpart;
  const uint32_t oP = oLA;
  const uint32_t oBL = oLA + (la_bytes > 2 * PART ? la_bytes : 2 * PART);
  const uint32_t oBar = (oBL + (uint32_t)a.dk * 4u + 15u) & ~15u;
  const uint32_t oTm = oBar + 8;
  float* sLA = reinterpret_cast<float*>(smem + oLA);
  float* sBL = reinterpret_cast<float*>(smem + oBL);
  volatile uint32_t* sTm = reinterpret_cast<volatile uint32_t*>(smem + oTm);

  if (warp == 0) {
    tmem_alloc(base_u32 + oTm, 256);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(base_u32 + oBar, 1);
    fence_mbar_init();
  }

  const int f0 = chunk_first_base_pos(a.g, c, MC);
  stage_bf16(base_u32 + oQ, a.q, a.dk, a.PK, a.g, f0, b, h, a.H);
  stage_bf16(base_u32 + oK, a.k, a.dk, a.PK, a.g, f0, b, h, a.H);
  stage_bf16(base_u32 + oV, a.v, a.dv, a.PV, a.g, f0, b, h, a.H);
  stage_la(base_u32 + oLA, a.la, a.dk, a.g, f0, b, h, a.H);
  {
    const uint8_t* src = a.g_img + ((size_t)bh * a.NC + c) * g_img_bytes(a.PK, a.Np);
    const int n16 = (int)(g_img_bytes(a.PK, a.Np) / 16u);
    for (int idx = tid; idx < n16; idx += NT) cp_async16(base_u32 + oG + (uint32_t)idx * 16u, src + idx * 16, true);
  }
  cp_async_commit();
  cp_async_wait_all();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *sTm;
  const uint32_t tS = tbase, tO = tbase + 128u;

  const int64_t cid = (int64_t)bh * a.NC + c;
  if (a.flags[cid]) {
    // Exact serial path; S_in (fp32, [dv][dk]) was left in the S_loc slot by pass 2.
    chunk_serial(smem + oQ, smem + oK, smem + oV, sLA, a.s_locT + cid * a.dv * a.dk, a, f0, b, h);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, 256);
    return;
  }
  chunk_suffix(sLA, sBL, a.dk, a.g.reverse);
  __syncthreads();
  gate_row<true, true>(smem, oQ, oK, sLA, a.dk, tid);
  fence_proxy_async_smem();
  __syncthreads();

  const int nk = (a.dk + 15) / 16;  // K steps over key channels
  if (tid == 0) {
    tc_fence_after();
    const uint32_t idesc = idesc_bf16_f32(MC, MC, false, false);
#pragma unroll 1
    for (int kk = 0; kk < nk; ++kk)
      umma_ss(tS, desc_kmajor(base_u32 + oQ, PART, kk), desc_kmajor(base_u32 + oK, PART, kk), idesc,
              kk > 0 ? 1u : 0u);
    umma_commit(base_u32 + oBar);
  }
  bool ok = mbar_wait(base_u32 + oBar, 0);
  tc_fence_after();

  // Scores of row r -> mask to keys scanned no later than r -> bf16 P (K-major).
  const int r = tid;
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
  for (int cb = 0; cb < MC; cb += 32) {
    float sc[32];
    tmem_ld32(tS + lane_base + (uint32_t)cb, sc);
    uint32_t pk[16];
#pragma unroll
    for (int j = 0; j < 32; j += 2) {
      const int s0 = cb + j, s1 = cb + j + 1;
      const bool k0 = a.g.reverse ? (s0 >= r) : (s0 <= r);
      const bool k1 = a.g.reverse ? (s1 >= r) : (s1 <= r);
      pk[j >> 1] = pack_bf16x2(k0 ? sc[j] : 0.f, k1 ? sc[j + 1] : 0.f);
    }
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) {
      const int s = cb + q4 * 8;
      const uint32_t o = oP + (uint32_t)(s >> 6) * PART + sw128((uint32_t)r, (uint32_t)(s & 63) * 2u);
      *reinterpret_cast<uint4*>(smem + o) = make_uint4(pk[q4 * 4], pk[q4 * 4 + 1], pk[q4 * 4 + 2], pk[q4 * 4 + 3]);
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();

  if (tid == 0 && ok) {
    tc_fence_after();
    const uint32_t id_pv = idesc_bf16_f32(MC, a.Np, false, true);
#pragma unroll 1
    for (int kk = 0; kk < MC / 16; ++kk)
      umma_ss(tO, desc_kmajor(base_u32 + oP, PART, kk), desc_mnmajor(base_u32 + oV, PART, kk), id_pv,
              kk > 0 ? 1u : 0u);
    const uint32_t id_qg = idesc_bf16_f32(MC, a.Np, false, false);
#pragma unroll 1
    for (int kk = 0; kk < nk; ++kk)
      umma_ss(tO, desc_kmajor(base_u32 + oQ, PART, kk), desc_kmajor(base_u32 + oG, gpart, kk), id_qg, 1u);
    umma_commit(base_u32 + oBar);
  }
  if (ok) ok = mbar_wait(base_u32 + oBar, 1);
  tc_fence_after();
  if (!ok) report_status(GLA_ERR_TIMEOUT);

  // Epilogue: row r -> out[b][token(f0 + r)][h][:]
  const int f = f0 + r;
  const bool valid = ok && (f >= 0) && (f < a.g.T);
  __nv_bfloat16* orow = a.out;
  if (valid) orow = a.out + (((int64_t)b * a.g.T + base_pos_to_token(a.g, f)) * a.H + h) * a.dv;
  for (int cb = 0; cb < a.Np; cb += 16) {
    float o[16];
    tmem_ld16(tO + lane_base + (uint32_t)cb, o);
    if (valid) {
#pragma unroll
      for (int j = 0; j < 16; j += 8) {
        if (cb + j < a.dv) {
          const uint4 w = make_uint4(pack_bf16x2(o[j], o[j + 1]), pack_bf16x2(o[j + 2], o[j + 3]),
                                     pack_bf16x2(o[j + 4], o[j + 5]), pack_bf16x2(o[j + 6], o[j + 7]));
          *reinterpret_cast<uint4*>(orow + cb + j) = w;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tbase, 256);
}

struct TcLayout {
  int NC, PK, PV, Np;
  size_t s_loc_bytes, gamma_bytes, flag_bytes, img_bytes;
  size_t smem_state, smem_out;
};

size_t round_up(size_t x, size_t m) { return (x + m - 1) / m * m; }

TcLayout tc_layout(const GlaShape& s) {
  TcLayout L;
  const int T = s.T();
  L.NC = (T + MC - 1) / MC;
  L.PK = (s.dk + 63) / 64;
  L.PV = (s.dv + 63) / 64;
  L.Np = (s.dv + 15) / 16 * 16;
  const size_t BH = (size_t)s.B * s.H;
  L.s_loc_bytes = round_up(BH * L.NC * s.dv * s.dk * sizeof(float), 256);
  L.gamma_bytes = round_up(BH * L.NC * s.dk * sizeof(float), 256);
  L.flag_bytes = round_up(BH * L.NC * sizeof(int), 256);
  L.img_bytes = round_up(BH * L.NC * (size_t)L.PK * L.Np * 128, 256);
  const size_t la = (size_t)MC * (s.dk + 4) * 4 + (size_t)s.dk * 4 + 16 + 16;
  L.smem_state = 1024 + (size_t)(2 + L.PV) * PART + la;
  const size_t la_tile = (size_t)MC * (s.dk + 4) * 4;
  L.smem_out = 1024 + (size_t)(2 * L.PK + L.PV) * PART + (size_t)L.PK * L.Np * 128 +
               (la_tile > 2 * PART ? la_tile : 2 * PART) + (size_t)s.dk * 4 + 16 + 16;
  return L;
}

}  // namespace

size_t gla_tc_workspace_bytes(const GlaShape& s) {
  const TcLayout L = tc_layout(s);
  return L.s_loc_bytes + L.gamma_bytes + L.flag_bytes + L.img_bytes;
}

cudaError_t gla_tc_forward(const void* q, const void* k, const void* v, const float* la, void* out,
                           const GlaShape& s, void* workspace, cudaStream_t st) {
  const TcLayout L = tc_layout(s);
  TcArgs a;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.k = static_cast<const __nv_bfloat16*>(k);
  a.v = static_cast<const __nv_bfloat16*>(v);
  a.la = la;
  a.out = static_cast<__nv_bfloat16*>(out);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  a.s_locT = reinterpret_cast<float*>(ws);
  a.gamma = reinterpret_cast<float*>(ws + L.s_loc_bytes);
  a.flags = reinterpret_cast<int*>(ws + L.s_loc_bytes + L.gamma_bytes);
  a.g_img = ws + L.s_loc_bytes + L.gamma_bytes + L.flag_bytes;
  a.H = s.H;
  a.dk = s.dk;
  a.dv = s.dv;
  a.NC = L.NC;
  a.PK = L.PK;
  a.PV = L.PV;
  a.Np = L.Np;
  a.g = make_geom(s.Hg, s.Wg, s.dir);

  cudaError_t e;
  e = cudaFuncSetAttribute(gla_tc_chunk_state, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.smem_state);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(gla_tc_output, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.smem_out);
  if (e != cudaSuccess) return e;

  const dim3 grid_chunks(L.NC, s.B * s.H);
  gla_tc_chunk_state<<<grid_chunks, NT, L.smem_state, st>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int entries = L.Np * L.PK * 64;
  gla_tc_prefix<<<dim3((entries + 255) / 256, s.B * s.H), 256, 0, st>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  gla_tc_output<<<grid_chunks, NT, L.smem_out, st>>>(a);
  return cudaGetLastError();
}

}  // namespace dig
