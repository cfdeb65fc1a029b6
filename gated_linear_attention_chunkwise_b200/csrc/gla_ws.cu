// gla_ws.cu -- warp-specialised chunk-wise GLA forward, bf16 q/k/v, sm_100a.
//
// Recurrence (DiG: gated linear attention): S_t = Diag(alpha_t) S_{t-1} + k_t^T v_t,
// o_t = q_t S_t, evaluated chunk-wise in on-chip memory (DiG paper notes,
// "硬件友好的效率设计": chunks of M tokens computed in SRAM, O(T M D + T D^2)).
//
// One CTA per (head, segment of G chunks of 128 scan positions), in ticket order.
//   pass 1  (chunks in reverse scan order)  u_s = log-gates scanned after s up to the
//           segment end; K^ = k exp(u) (<= 1 for decaying gates); S_seg += K^T V.
//   look-back  publish (exp(segment gate sum), S_seg); fold earlier segments of the
//           same head until an inclusive state is found: S_in; publish the inclusive
//           state Diag(gamma_seg) S_in + S_seg; S_in becomes the running state.
//   pass 2  (scan order; rows still in L2)  u = in-chunk suffix, gamma = exp(chunk sum):
//           G = Diag(gamma) S;  O = mask(Q~ K^T) V + Q~ G;  S = G + K^T V
//           with Q~ = q exp(-u), K^ = k exp(u); O stored in bf16 at canonical positions.
// Chunks whose gates decay by more than e^80 inside the chunk are evaluated token by
// token from the running state instead (exact).
//
// Roles (14 warps, 448 threads), connected by mbarriers:
//   warp 0      producer: TMA loads of each chunk's q, k, v (32-byte-swizzled 16-channel
//               boxes, the UMMA operand layout) and log-gates into a ring of stages;
//   warp 1      MMA issuer (tcgen05, one thread) and TMEM owner;
//   warps 2-5   suffix sums of the log-gates, one thread per key channel;
//   warps 6-9   gates applied in place (K^, Q~), one thread per row;
//   warps 10-13 TMEM-side work, one thread per TMEM lane: G = Diag(gamma) S, score
//               masking to bf16 P, output epilogue, look-back, serial path.
// TMEM (512 columns): scores [0,128) -- overwritten by the bf16 P matrix (two keys per
// column, the A operand of P V) --, O buffer 0 [128,256), running state [256,384),
// segment aggregate [384,512) -- reused as O buffer 1 once the look-back is done.
// A stage is free once the MMAs that read it complete, so loads run ahead of the
// output epilogue.
//
// Chunks follow the direction's base order (raster rows, or grid columns for T->B /
// B->T) and are always cut in forward order; reversed scans visit them backwards and
// walk each chunk's rows backwards.  Each chunk is one TMA box per tensor: 128
// consecutive raster positions; 128/Hgrid whole columns when Hgrid divides 128;
// otherwise one column cut into pieces of at most 128 rows.  Rows past the grid are
// zero-filled by the TMA and contribute nothing.
#include <math.h>
#include <string.h>

#include <cuda.h>

#include "dev_common.cuh"
#include "internal.h"

namespace dig {

namespace {

constexpr int MC = kChunkTC;
constexpr int NT = 448;
constexpr int kWarpProd = 0, kWarpMma = 1, kWarpSuf = 2, kWarpGate = 6, kWarpEpi = 10;
constexpr uint32_t ATOM32 = MC * 32u;    // one 16-channel block of a 32B-swizzled 128-row tile
constexpr float kMaxGateRange = 80.0f;
constexpr uint32_t kColS = 0, kColO0 = 128, kColState = 256, kColSeg = 384;
constexpr uint32_t kLayoutSW32 = 6;
constexpr int kMaxStages = 2;

// mbarrier indices (8 bytes each)
enum {
  kBarFull = 0,                          // [S]  tiles landed
  kBarSuf = kBarFull + kMaxStages,       // [S]  suffix sums done (128 arrivals)
  kBarGate = kBarSuf + kMaxStages,       // [S]  gates applied (128 arrivals)
  kBarEmpty = kBarGate + kMaxStages,     // [S]  stage free (MMA commit, or the serial path)
  kBarScFull = kBarEmpty + kMaxStages,   // score MMA done
  kBarScEmpty,                           // scores read (128 arrivals)
  kBarPReady,                            // P and G written (128 arrivals)
  kBarBatch0,                            // [2] output MMAs done
  kBarOEmpty0 = kBarBatch0 + 2,          // [2] output buffer read (128 arrivals)
  kBarSegDone = kBarOEmpty0 + 2,         // pass-1 MMAs done
  kBarDrain,                             // all MMAs of the CTA done (teardown)
  kNumBars
};

struct WsArgs {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const float* la;
  __nv_bfloat16* out;
  float* agg_S;   // [BH][NS][dv/4][dk][4]  segment aggregates (quads of value columns)
  float* agg_g;   // [BH][NS][dk]           exp(segment log-gate sums)
  float* incl_S;  // [BH][NS][dv/4][dk][4]  state after the segment
  int* flags;     // [BH][NS]               0 nothing, 1 aggregate, 2 inclusive
  int* ticket;
  int H, BH, dk, dv, NC, NS, G;
  int Kp, Np, nstage;
  int mode, rpc, ppr;  // chunk geometry: 0 raster, 1 whole columns (rpc per chunk), 2 column pieces (ppr per column)
  uint32_t stage_bytes, oK, oV, oQ, oLA, oG, oBL, oWide, oGam, oRed, oMisc, oBar, oTm;
  ScanGeom g;
};

struct TensorMaps {
  CUtensorMap q, k, v, la;
};

// ---------------------------------------------------------------------------
// Helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t sw32_off(uint32_t r, uint32_t ch) {
  return (ch >> 4) * ATOM32 + r * 32u + (((((ch >> 3) & 1u) ^ (r >> 2)) & 1u) << 4) + (ch & 7u) * 2u;
}
__device__ __forceinline__ uint32_t g_off(uint32_t i, uint32_t jcol, uint32_t Kp) {
  return (jcol >> 4) * (Kp * 32u) + i * 32u + (((((jcol >> 3) & 1u) ^ (i >> 2)) & 1u) << 4) + (jcol & 7u) * 2u;
}
__device__ __forceinline__ uint64_t desc_sw32(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return umma_desc(saddr, lbo, sbo, kLayoutSW32);
}
__device__ __forceinline__ uint32_t ld_acquire(const int* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release(int* p, int v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void named_sync(uint32_t id, uint32_t n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
// Group-wide AND over a named barrier: every thread of the group gets the same
// answer, so a group either continues or leaves together (no thread is left
// waiting at a later named barrier).
__device__ __forceinline__ bool group_and(uint32_t id, uint32_t n, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_cnt(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15]))
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 16-column TMEM load without the wait: the registers hold the columns only after
// tmem_ld_cols' wait (several loads then share one round trip).
__device__ __forceinline__ void tmem_ld16_issue(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}
// Orders every later use of r after the preceding tcgen05.wait::ld.
__device__ __forceinline__ void reg_tie16(uint32_t (&r)[16]) {
  asm volatile(""
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                 "+r"(r[15]));
}
// Columns [0, n) of this warp's lanes from taddr (n <= 16 P, multiple of 16), one wait.
template <int P>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, int n, uint32_t (&r)[P][16]) {
#pragma unroll
  for (int q = 0; q < P; ++q)
    if (16 * q < n) tmem_ld16_issue(taddr + (uint32_t)(16 * q), r[q]);
  tmem_ld_wait();
#pragma unroll
  for (int q = 0; q < P; ++q) reg_tie16(r[q]);
}
__device__ __forceinline__ void tmem_st16u(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}
// D (+)= A * B with A read from TMEM (lane = row, two bf16 of K per column) and B
// described in shared memory.
__device__ __forceinline__ void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ uint32_t pack_u2(uint32_t x, uint32_t y) {
  return pack_bf16x2(__uint_as_float(x), __uint_as_float(y));
}

__device__ __forceinline__ void tma_load_5d(uint32_t dst, const CUtensorMap* map, int c0, int c1, int c2, int c3,
                                            int c4, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5, %6}], "
      "[%7];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4), "r"(bar)
      : "memory");
}

// Bounded wait on an mbarrier phase that also gives up when another role has
// aborted the CTA.  Returns false on timeout / abort (the caller stops its role).
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (*abort_flag) return false;
    if (clock64() - t0 > kWaitCycles) {
      report_status(GLA_ERR_TIMEOUT);
      *abort_flag = 1;
      return false;
    }
  }
  return true;
}

// Spin (one thread) until flags[idx] != 0; 0 on timeout.
__device__ int wait_flag(const int* flags, int64_t idx) {
  uint32_t f = ld_acquire(flags + idx);
  if (f) return (int)f;
  const long long t0 = clock64();
  while ((f = ld_acquire(flags + idx)) == 0) {
    if (clock64() - t0 > kWaitCycles) {
      report_status(GLA_ERR_TIMEOUT);
      return 0;
    }
    __nanosleep(64);
  }
  return (int)f;
}

// Forward chunk index of scan-order chunk c.
__device__ __forceinline__ int fwd_chunk(const WsArgs& a, int c) { return a.g.reverse ? a.NC - 1 - c : c; }

// Raster token of tile row r of forward chunk cf, or -1 for a padding row.
__device__ __forceinline__ int row_token(const WsArgs& a, int cf, int r) {
  if (a.mode == 0) {
    const int f = cf * MC + r;
    return f < a.g.T ? f : -1;
  }
  if (a.mode == 1) {
    const int xl = r / a.g.Hg;
    const int x = cf * a.rpc + xl, y = r - xl * a.g.Hg;
    return x < a.g.Wg ? y * a.g.Wg + x : -1;
  }
  const int x = cf / a.ppr, y = (cf - x * a.ppr) * MC + r;
  return y < a.g.Hg ? y * a.g.Wg + x : -1;
}

// TMA coordinates (run position, run index) of forward chunk cf's box.
__device__ __forceinline__ void chunk_box(const WsArgs& a, int cf, int& y, int& x) {
  if (a.mode == 0) {
    y = cf * MC;
    x = 0;
  } else if (a.mode == 1) {
    y = 0;
    x = cf * a.rpc;
  } else {
    x = cf / a.ppr;
    y = (cf - x * a.ppr) * MC;
  }
}

__device__ __forceinline__ int job_chunk(int j, int c0, int n) { return j < n ? c0 + n - 1 - j : c0 + (j - n); }

// ---------------------------------------------------------------------------
// Producer
// ---------------------------------------------------------------------------
__device__ void tma_job(const WsArgs& a, const TensorMaps& tm, uint32_t st, uint32_t bar, int cf, bool with_q, int b,
                        int h) {
  const uint32_t bytes = (uint32_t)(with_q ? 2 : 1) * (uint32_t)a.Kp * 256u + (uint32_t)a.Np * 256u +
                         (uint32_t)MC * (uint32_t)(a.dk + 4) * 4u;
  mbar_expect_tx(bar, bytes);
  int y, x;
  chunk_box(a, cf, y, x);
  for (int cb = 0; cb < (a.Kp >> 4); ++cb) {
    tma_load_5d(st + a.oK + (uint32_t)cb * ATOM32, &tm.k, cb * 16, h, y, x, b, bar);
    if (with_q) tma_load_5d(st + a.oQ + (uint32_t)cb * ATOM32, &tm.q, cb * 16, h, y, x, b, bar);
  }
  for (int cb = 0; cb < (a.Np >> 4); ++cb) tma_load_5d(st + a.oV + (uint32_t)cb * ATOM32, &tm.v, cb * 16, h, y, x, b, bar);
  tma_load_5d(st + a.oLA, &tm.la, 0, h, y, x, b, bar);
}

// ---------------------------------------------------------------------------
// Serial path (wide chunks), run by the 128 TMEM-side threads: lane i owns state
// row i; 16 value columns at a time, outputs reduced over lanes with shuffles.
// q, k are still the raw (unscaled) swizzled tiles.
// ---------------------------------------------------------------------------
__device__ void chunk_serial(const WsArgs& a, const uint8_t* st, float* red, uint32_t tstate, uint32_t lane_base,
                             int i, int cf, int b, int h) {
  const int lane = threadIdx.x & 31, ew = (threadIdx.x >> 5) - kWarpEpi;  // 0..3
  for (int cb = 0; cb < (a.Np >> 4); ++cb) {
    float s[16];
    tmem_ld16(tstate + lane_base + (uint32_t)(cb * 16), s);
    if (i >= a.dk)
#pragma unroll
      for (int q = 0; q < 16; ++q) s[q] = 0.f;
    for (int step = 0; step < MC; ++step) {
      const int r = a.g.reverse ? (MC - 1 - step) : step;
      const int t = row_token(a, cf, r);
      if (t < 0) continue;  // padding row: uniform
      float alpha = 1.f, kq = 0.f, qi = 0.f;
      if (i < a.dk) {
        alpha = __expf(__ldg(a.la + (((int64_t)b * a.g.T + t) * a.H + h) * a.dk + i));
        kq = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(st + a.oK + sw32_off((uint32_t)r, (uint32_t)i)));
        qi = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(st + a.oQ + sw32_off((uint32_t)r, (uint32_t)i)));
      }
      float vv[16];
      {
        const uint4 w0 = *reinterpret_cast<const uint4*>(st + a.oV + sw32_off((uint32_t)r, (uint32_t)(cb * 16)));
        const uint4 w1 = *reinterpret_cast<const uint4*>(st + a.oV + sw32_off((uint32_t)r, (uint32_t)(cb * 16 + 8)));
        const uint32_t u[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float2 p = unpack_bf16x2(u[q]);
          vv[2 * q] = p.x;
          vv[2 * q + 1] = p.y;
        }
      }
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        s[q] = fmaf(alpha, s[q], kq * vv[q]);
        float x = qi * s[q];
        x += __shfl_xor_sync(0xffffffffu, x, 16);
        x += __shfl_xor_sync(0xffffffffu, x, 8);
        x += __shfl_xor_sync(0xffffffffu, x, 4);
        x += __shfl_xor_sync(0xffffffffu, x, 2);
        x += __shfl_xor_sync(0xffffffffu, x, 1);
        if (lane == 0) red[ew * 16 + q] = x;
      }
      named_sync(2, 128);
      const int e = threadIdx.x - 32 * kWarpEpi;
      if (e < 16 && cb * 16 + e < a.dv)
        a.out[(((int64_t)b * a.g.T + t) * a.H + h) * a.dv + cb * 16 + e] =
            __float2bfloat16_rn(red[e] + red[16 + e] + red[32 + e] + red[48 + e]);
      named_sync(2, 128);
    }
    tmem_st16(tstate + lane_base + (uint32_t)(cb * 16), s);
  }
  tmem_st_wait();
}

__device__ __forceinline__ uint32_t align1024(uint32_t x) { return (x + 1023u) & ~1023u; }

// ---------------------------------------------------------------------------
// The kernel
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(NT, 1) gla_ws_fwd(const WsArgs a, const __grid_constant__ TensorMaps tm) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t sbase = align1024(raw_u32);
  uint8_t* smem = smem_raw + (sbase - raw_u32);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  float* sBL = reinterpret_cast<float*>(smem + a.oBL);      // [S][128] chunk gate sums
  volatile int* sWide = reinterpret_cast<volatile int*>(smem + a.oWide);  // [S] + [S][4] per-warp flags
  float* sGam = reinterpret_cast<float*>(smem + a.oGam);    // [128] exp(segment gate sum)
  float* red = reinterpret_cast<float*>(smem + a.oRed);     // serial-path reduction [4][16]
  volatile int* sMisc = reinterpret_cast<volatile int*>(smem + a.oMisc);  // [0] item [1] abort [2] flag
  const uint32_t bars = sbase + a.oBar;
  auto BAR = [&](int idx) -> uint32_t { return bars + 8u * (uint32_t)idx; };
  volatile int* abort_flag = sMisc + 1;

  if (warp == kWarpMma) {
    tmem_alloc(sbase + a.oTm, 512);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int s = 0; s < a.nstage; ++s) {
      mbar_init(BAR(kBarFull + s), 1);
      mbar_init(BAR(kBarSuf + s), 128);
      mbar_init(BAR(kBarGate + s), 128);
      mbar_init(BAR(kBarEmpty + s), 1);
    }
    mbar_init(BAR(kBarScFull), 1);
    mbar_init(BAR(kBarScEmpty), 128);
    mbar_init(BAR(kBarPReady), 128);
    mbar_init(BAR(kBarBatch0), 1);
    mbar_init(BAR(kBarBatch0 + 1), 1);
    mbar_init(BAR(kBarOEmpty0), 128);
    mbar_init(BAR(kBarOEmpty0 + 1), 128);
    mbar_init(BAR(kBarSegDone), 1);
    mbar_init(BAR(kBarDrain), 1);
    fence_mbar_init();
    sMisc[0] = atomicAdd(a.ticket, 1);
    sMisc[1] = 0;  // abort
    sMisc[3] = 0;  // load jobs issued
    sMisc[4] = 0;  // load jobs consumed
  }
  for (int x = tid; x < kMaxStages * 128; x += NT) sBL[x] = 0.f;  // rows >= dk: gamma = 1
  for (int x = tid; x < 128; x += NT) sGam[x] = 1.f;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *reinterpret_cast<volatile uint32_t*>(smem + a.oTm);
  const int item = sMisc[0];
  const int seg = item / a.BH, bh = item - seg * a.BH;
  const int b = bh / a.H, h = bh - b * a.H;
  const int c0 = seg * a.G;
  const int n = min(a.G, a.NC - c0);
  const int64_t seg_id = (int64_t)bh * a.NS + seg;
  const int njob = 2 * n;
  const int S = a.nstage;

  if (warp == kWarpProd) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      for (int j = 0; j < njob; ++j) {
        const int s = j % S, k = j / S;
        if (k > 0 && !wait_bar(BAR(kBarEmpty + s), (uint32_t)((k - 1) & 1), abort_flag)) break;
        const uint32_t st = sbase + (uint32_t)s * a.stage_bytes;
        tma_job(a, tm, st, BAR(kBarFull + s), fwd_chunk(a, job_chunk(j, c0, n)), j >= n, b, h);
        sMisc[3] = j + 1;
      }
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int kb = 0;
      for (int j = 0; j < njob; ++j) {
        const int s = j % S, k = j / S;
        if (!wait_bar(BAR(kBarGate + s), (uint32_t)(k & 1), abort_flag)) break;
        tc_fence_after();
        const uint32_t st = sbase + (uint32_t)s * a.stage_bytes;
        if (j < n) {
          const uint32_t id = idesc_bf16_f32(MC, a.Np, true, true);
#pragma unroll 1
          for (int kk = 0; kk < MC / 16; ++kk)
            umma_ss(tbase + kColSeg, desc_sw32(st + a.oK + (uint32_t)kk * 512u, ATOM32, 256u),
                    desc_sw32(st + a.oV + (uint32_t)kk * 512u, ATOM32, 256u), id, (j > 0 || kk > 0) ? 1u : 0u);
          umma_commit(BAR(kBarEmpty + s));
          if (j == n - 1) umma_commit(BAR(kBarSegDone));
          continue;
        }
        if (sWide[s]) continue;  // evaluated serially by the TMEM-side warps, which free the stage
        if (kb > 0 && !wait_bar(BAR(kBarScEmpty), (uint32_t)((kb - 1) & 1), abort_flag)) break;
        tc_fence_after();
        {
          const uint32_t id = idesc_bf16_f32(MC, MC, false, false);
#pragma unroll 1
          for (int kk = 0; kk < (a.Kp >> 4); ++kk)
            umma_ss(tbase + kColS, desc_sw32(st + a.oQ + (uint32_t)kk * ATOM32, 16u, 256u),
                    desc_sw32(st + a.oK + (uint32_t)kk * ATOM32, 16u, 256u), id, kk > 0 ? 1u : 0u);
          umma_commit(BAR(kBarScFull));
        }
        if (!wait_bar(BAR(kBarPReady), (uint32_t)(kb & 1), abort_flag)) break;
        const int ob = kb & 1;
        if (kb >= 2 && !wait_bar(BAR(kBarOEmpty0 + ob), (uint32_t)(((kb >> 1) - 1) & 1), abort_flag)) break;
        tc_fence_after();
        {
          const uint32_t tO = tbase + (ob ? kColSeg : kColO0);
          const uint32_t id_pv = idesc_bf16_f32(MC, a.Np, false, true);
#pragma unroll 1
          for (int kk = 0; kk < MC / 16; ++kk)  // P is bf16 in the score columns
            umma_ts(tO, tbase + kColS + (uint32_t)(kk * 8), desc_sw32(st + a.oV + (uint32_t)kk * 512u, ATOM32, 256u),
                    id_pv, kk > 0 ? 1u : 0u);
#pragma unroll 1
          for (int kk = 0; kk < (a.Kp >> 4); ++kk)
            umma_ss(tO, desc_sw32(st + a.oQ + (uint32_t)kk * ATOM32, 16u, 256u),
                    desc_sw32(sbase + a.oG + (uint32_t)kk * 512u, (uint32_t)a.Kp * 32u, 256u), id_pv, 1u);
          const uint32_t id_s = idesc_bf16_f32(MC, a.Np, true, true);
#pragma unroll 1
          for (int kk = 0; kk < MC / 16; ++kk)
            umma_ss(tbase + kColState, desc_sw32(st + a.oK + (uint32_t)kk * 512u, ATOM32, 256u),
                    desc_sw32(st + a.oV + (uint32_t)kk * 512u, ATOM32, 256u), id_s, 1u);
          umma_commit(BAR(kBarBatch0 + ob));
          umma_commit(BAR(kBarEmpty + s));
        }
        ++kb;
      }
      // Every MMA of this CTA completes before TMEM is released (bounded).
      umma_commit(BAR(kBarDrain));
      const long long t0 = clock64();
      while (!mbar_try_wait(BAR(kBarDrain), 0u) && clock64() - t0 < kWaitCycles) {
      }
    }
  } else if (warp < kWarpGate) {
    // ------------------------------------------------------------ suffix sums
    const int i = tid - 32 * kWarpSuf;  // key channel
    const int sw = warp - kWarpSuf;
    float off = 0.f, pos_seg = 0.f;
    for (int j = 0; j < njob; ++j) {
      const int s = j % S, k = j / S;
      if (!group_and(1, 128, wait_bar(BAR(kBarFull + s), (uint32_t)(k & 1), abort_flag))) break;
      if (i == 0) sMisc[4] = j + 1;
      float* sLA = reinterpret_cast<float*>(smem + (uint32_t)s * a.stage_bytes + a.oLA);
      const bool pass1 = j < n;
      int wide = 0;
      if (i < a.dk) {
        const int pw = a.dk + 4;
        float* ptr = sLA + (a.g.reverse ? 0 : (MC - 1)) * pw + i;  // last scanned row first
        const int step = a.g.reverse ? pw : -pw;
        const float base = pass1 ? off : 0.f;
        float acc = 0.f, ab = 0.f, po = 0.f;
        // Sixteen loads are issued before their stores so that they overlap.
#pragma unroll 1
        for (int p0 = 0; p0 < MC; p0 += 16) {
          float x[16];
#pragma unroll
          for (int q = 0; q < 16; ++q) x[q] = ptr[q * step];
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            ptr[q * step] = acc + base;
            acc += x[q];
            ab += fabsf(x[q]);
            po += fmaxf(x[q], 0.f);
          }
          ptr += 16 * step;
        }
        sBL[s * 128 + i] = acc;
        if (pass1) {
          off += acc;
          pos_seg += po;
          if (j == n - 1) {
            if (!(pos_seg <= kMaxGateRange)) report_status(GLA_ERR_RANGE);
            sGam[i] = __expf(off);
          }
        } else {
          wide = !(ab <= kMaxGateRange);
        }
      }
      const int any = __any_sync(0xffffffffu, wide);
      if (lane == 0) sWide[kMaxStages + s * 4 + sw] = any;
      named_sync(1, 128);
      if (i == 0)
        sWide[s] = sWide[kMaxStages + s * 4 + 0] | sWide[kMaxStages + s * 4 + 1] | sWide[kMaxStages + s * 4 + 2] |
                   sWide[kMaxStages + s * 4 + 3];
      mbar_arrive(BAR(kBarSuf + s));
    }
  } else if (warp < kWarpEpi) {
    // ------------------------------------------------------------ gates (row r)
    const int r = tid - 32 * kWarpGate;
    for (int j = 0; j < njob; ++j) {
      const int s = j % S, k = j / S;
      if (!wait_bar(BAR(kBarSuf + s), (uint32_t)(k & 1), abort_flag)) break;
      const bool pass1 = j < n;
      uint8_t* st = smem + (uint32_t)s * a.stage_bytes;
      if (pass1 || !sWide[s]) {
        const float* urow = reinterpret_cast<const float*>(st + a.oLA) + r * (a.dk + 4);
        // Three 8-channel groups per round: all loads first, then gates, then stores.
        for (int cbase = 0; cbase < a.dk; cbase += 24) {
          float4 u[3][2];
          uint4 kw[3], qw[3];
#pragma unroll
          for (int g3 = 0; g3 < 3; ++g3) {
            const int c = cbase + 8 * g3;
            if (c < a.dk) {
              const uint32_t o = sw32_off((uint32_t)r, (uint32_t)c);
              u[g3][0] = *reinterpret_cast<const float4*>(urow + c);
              u[g3][1] = *reinterpret_cast<const float4*>(urow + c + 4);
              kw[g3] = *reinterpret_cast<const uint4*>(st + a.oK + o);
              if (!pass1) qw[g3] = *reinterpret_cast<const uint4*>(st + a.oQ + o);
            }
          }
#pragma unroll
          for (int g3 = 0; g3 < 3; ++g3) {
            const int c = cbase + 8 * g3;
            if (c < a.dk) {
              const uint32_t o = sw32_off((uint32_t)r, (uint32_t)c);
              const float e[8] = {u[g3][0].x, u[g3][0].y, u[g3][0].z, u[g3][0].w,
                                  u[g3][1].x, u[g3][1].y, u[g3][1].z, u[g3][1].w};
              uint32_t* uk = reinterpret_cast<uint32_t*>(&kw[g3]);
#pragma unroll
              for (int jj = 0; jj < 4; ++jj) {
                const float2 xx = unpack_bf16x2(uk[jj]);
                uk[jj] = pack_bf16x2(xx.x * __expf(e[2 * jj]), xx.y * __expf(e[2 * jj + 1]));
              }
              *reinterpret_cast<uint4*>(st + a.oK + o) = kw[g3];
              if (!pass1) {
                uint32_t* uq = reinterpret_cast<uint32_t*>(&qw[g3]);
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                  const float2 xx = unpack_bf16x2(uq[jj]);
                  uq[jj] = pack_bf16x2(xx.x * __expf(-e[2 * jj]), xx.y * __expf(-e[2 * jj + 1]));
                }
                *reinterpret_cast<uint4*>(st + a.oQ + o) = qw[g3];
              }
            }
          }
        }
        fence_proxy_async_smem();
      }
      mbar_arrive(BAR(kBarGate + s));
    }
  } else {
    // ------------------------------------------------------------ TMEM-side work
    const int i = 32 * (warp & 3) + lane;  // TMEM lane = row / key channel
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    const int e = tid - 32 * kWarpEpi;
    int kb = 0;
    bool prev_pending = false;
    int prev_cf = 0;
    bool ok = true;

    // Epilogue of the previous output buffer: O -> bf16 -> out[b][token][h][:].
    auto finish_prev = [&]() -> bool {
      if (!prev_pending) return true;
      const int ob = (kb - 1) & 1;
      if (!group_and(2, 128, wait_bar(BAR(kBarBatch0 + ob), (uint32_t)(((kb - 1) >> 1) & 1), abort_flag)))
        return false;
      tc_fence_after();
      const int t = row_token(a, prev_cf, i);
      const bool valid = t >= 0;
      __nv_bfloat16* orow = a.out;
      if (valid) orow = a.out + (((int64_t)b * a.g.T + t) * a.H + h) * a.dv;
      const uint32_t tO = tbase + (ob ? kColSeg : kColO0) + lane_base;
      for (int c0 = 0; c0 < a.Np; c0 += 32) {
        uint32_t o[2][16];
        tmem_ld_cols<2>(tO + (uint32_t)c0, a.Np - c0, o);
        if (valid) {
#pragma unroll
          for (int q = 0; q < 2; ++q)
#pragma unroll
            for (int hh = 0; hh < 16; hh += 8)
              if (c0 + 16 * q + hh < a.dv)
                *reinterpret_cast<uint4*>(orow + c0 + 16 * q + hh) =
                    make_uint4(pack_u2(o[q][hh], o[q][hh + 1]), pack_u2(o[q][hh + 2], o[q][hh + 3]),
                               pack_u2(o[q][hh + 4], o[q][hh + 5]), pack_u2(o[q][hh + 6], o[q][hh + 7]));
        }
      }
      tc_fence_before();
      mbar_arrive(BAR(kBarOEmpty0 + ob));
      prev_pending = false;
      return true;
    };

    // ---- end of pass 1: publish the segment aggregate and look back ----
    // (this group takes no part in pass 1 itself)
    if (!group_and(2, 128, wait_bar(BAR(kBarSegDone), 0u, abort_flag))) ok = false;
    if (ok) {
      tc_fence_after();
      const int DQ = a.dv >> 2;
      const uint32_t tSeg = tbase + kColSeg + lane_base, tSt = tbase + kColState + lane_base;
      const float gs = sGam[i];
      if (i < a.dk) a.agg_g[seg_id * a.dk + i] = gs;
      for (int c0 = 0; c0 < a.Np; c0 += 64) {
        uint32_t t[4][16];
        tmem_ld_cols<4>(tSeg + (uint32_t)c0, a.Np - c0, t);
        if (i < a.dk) {
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            const int jq = c0 / 4 + q;
            if (jq < DQ)
              *reinterpret_cast<float4*>(a.agg_S + ((seg_id * DQ + jq) * a.dk + i) * 4) =
                  make_float4(__uint_as_float(t[q >> 2][4 * (q & 3)]), __uint_as_float(t[q >> 2][4 * (q & 3) + 1]),
                              __uint_as_float(t[q >> 2][4 * (q & 3) + 2]), __uint_as_float(t[q >> 2][4 * (q & 3) + 3]));
          }
        }
      }
      __threadfence();
      named_sync(2, 128);
      if (e == 0) st_release(a.flags + seg_id, 1);
      {
        float z[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) z[q] = 0.f;
        for (int cb = 0; cb < a.Np; cb += 16) tmem_st16(tSt + (uint32_t)cb, z);
        tmem_st_wait();
      }
      float gam = 1.f;
      for (int p = seg - 1; p >= 0; --p) {
        const int64_t pid = (int64_t)bh * a.NS + p;
        if (e == 0) sMisc[2] = wait_flag(a.flags, pid);
        named_sync(2, 128);
        const int fl = sMisc[2];
        named_sync(2, 128);
        if (fl == 0) break;  // timed out (recorded)
        const float* src = (fl == 2 ? a.incl_S : a.agg_S);
        // 32 columns of the predecessor's rows are loaded before the TMEM round trip.
        for (int c0 = 0; c0 < a.Np; c0 += 32) {
          float4 x[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const int jq = c0 / 4 + q;
            x[q] = (i < a.dk && jq < DQ)
                       ? __ldcg(reinterpret_cast<const float4*>(src + ((pid * DQ + jq) * a.dk + i) * 4))
                       : make_float4(0.f, 0.f, 0.f, 0.f);
          }
          uint32_t t[2][16];
          tmem_ld_cols<2>(tSt + (uint32_t)c0, a.Np - c0, t);
#pragma unroll
          for (int c4 = 0; c4 < 2; ++c4) {
            if (c0 + 16 * c4 < a.Np) {
              float t16[16];
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                t16[4 * q] = fmaf(gam, x[4 * c4 + q].x, __uint_as_float(t[c4][4 * q]));
                t16[4 * q + 1] = fmaf(gam, x[4 * c4 + q].y, __uint_as_float(t[c4][4 * q + 1]));
                t16[4 * q + 2] = fmaf(gam, x[4 * c4 + q].z, __uint_as_float(t[c4][4 * q + 2]));
                t16[4 * q + 3] = fmaf(gam, x[4 * c4 + q].w, __uint_as_float(t[c4][4 * q + 3]));
              }
              tmem_st16(tSt + (uint32_t)(c0 + 16 * c4), t16);
            }
          }
        }
        tmem_st_wait();
        if (fl == 1 && i < a.dk) gam *= __ldcg(a.agg_g + pid * a.dk + i);
        if (fl == 2) break;
      }
      // Inclusive state of this segment: Diag(gamma_seg) S_in + aggregate.
      for (int c0 = 0; c0 < a.Np; c0 += 32) {
        uint32_t sin[2][16], sg[2][16];
        tmem_ld_cols<2>(tSt + (uint32_t)c0, a.Np - c0, sin);
        tmem_ld_cols<2>(tSeg + (uint32_t)c0, a.Np - c0, sg);
        if (i < a.dk) {
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const int jq = c0 / 4 + q;
            const int pc = q >> 2, o4 = 4 * (q & 3);
            if (jq < DQ)
              *reinterpret_cast<float4*>(a.incl_S + ((seg_id * DQ + jq) * a.dk + i) * 4) = make_float4(
                  fmaf(gs, __uint_as_float(sin[pc][o4]), __uint_as_float(sg[pc][o4])),
                  fmaf(gs, __uint_as_float(sin[pc][o4 + 1]), __uint_as_float(sg[pc][o4 + 1])),
                  fmaf(gs, __uint_as_float(sin[pc][o4 + 2]), __uint_as_float(sg[pc][o4 + 2])),
                  fmaf(gs, __uint_as_float(sin[pc][o4 + 3]), __uint_as_float(sg[pc][o4 + 3])));
          }
        }
      }
      __threadfence();
      tc_fence_before();
      named_sync(2, 128);
      if (e == 0) st_release(a.flags + seg_id, 2);
      tc_fence_after();
    }

    for (int j = n; j < njob && ok; ++j) {
      const int s = j % S, k = j / S;
      // The previous chunk's epilogue releases its stage; it must not wait behind this
      // chunk's gates (with one stage, those need that very stage).
      if (j > n && !finish_prev()) {
        ok = false;
        break;
      }
      if (!group_and(2, 128, wait_bar(BAR(kBarGate + s), (uint32_t)(k & 1), abort_flag))) {
        ok = false;
        break;
      }
      uint8_t* st = smem + (uint32_t)s * a.stage_bytes;
      const int cf = fwd_chunk(a, job_chunk(j, c0, n));

      // ---- pass 2 ----
      if (sWide[s]) {
        chunk_serial(a, st, red, tbase + kColState, lane_base, i, cf, b, h);
        tc_fence_before();
        named_sync(2, 128);
        if (e == 0) mbar_arrive(BAR(kBarEmpty + s));
        continue;
      }
      // G = Diag(gamma) S (state -> state, bf16 copy into the G tile)
      {
        const float gm = __expf(sBL[s * 128 + i]);
        const uint32_t tSt = tbase + kColState + lane_base;
        for (int c0 = 0; c0 < a.Np; c0 += 32) {
          uint32_t t[2][16];
          tmem_ld_cols<2>(tSt + (uint32_t)c0, a.Np - c0, t);
#pragma unroll
          for (int c4 = 0; c4 < 2; ++c4) {
            const int cb = c0 + 16 * c4;
            if (cb < a.Np) {
              float t16[16];
#pragma unroll
              for (int q = 0; q < 16; ++q) t16[q] = __uint_as_float(t[c4][q]) * gm;
              tmem_st16(tSt + (uint32_t)cb, t16);
              if (i < a.Kp) {
                const uint4 w0 = make_uint4(pack_bf16x2(t16[0], t16[1]), pack_bf16x2(t16[2], t16[3]),
                                            pack_bf16x2(t16[4], t16[5]), pack_bf16x2(t16[6], t16[7]));
                const uint4 w1 = make_uint4(pack_bf16x2(t16[8], t16[9]), pack_bf16x2(t16[10], t16[11]),
                                            pack_bf16x2(t16[12], t16[13]), pack_bf16x2(t16[14], t16[15]));
                *reinterpret_cast<uint4*>(smem + a.oG + g_off((uint32_t)i, (uint32_t)cb, (uint32_t)a.Kp)) = w0;
                *reinterpret_cast<uint4*>(smem + a.oG + g_off((uint32_t)i, (uint32_t)cb + 8u, (uint32_t)a.Kp)) = w1;
              }
            }
          }
        }
        tmem_st_wait();
      }
      // scores -> mask (keys scanned no later than the row) -> bf16 P in TMEM
      if (!group_and(2, 128, wait_bar(BAR(kBarScFull), (uint32_t)(kb & 1), abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      {
        const int rlo = 32 * (warp & 3), rhi = rlo + 31;
#pragma unroll 1
        for (int cb = 0; cb < MC; cb += 32) {
          const bool none = a.g.reverse ? (cb + 31 < rlo) : (cb > rhi);
          const bool all = a.g.reverse ? (cb >= rhi) : (cb + 31 <= rlo);
          uint32_t sc[2][16];
          if (!none) tmem_ld_cols<2>(tbase + kColS + lane_base + (uint32_t)cb, 32, sc);
          uint32_t pk[16];
          if (none) {
#pragma unroll
            for (int q = 0; q < 16; ++q) pk[q] = 0u;
          } else if (all) {
#pragma unroll
            for (int q = 0; q < 32; q += 2) pk[q >> 1] = pack_u2(sc[q >> 4][q & 15], sc[q >> 4][(q & 15) + 1]);
          } else {
#pragma unroll
            for (int q = 0; q < 32; q += 2) {
              const int s0 = cb + q, s1 = cb + q + 1;
              const bool k0 = a.g.reverse ? (s0 >= i) : (s0 <= i);
              const bool k1 = a.g.reverse ? (s1 >= i) : (s1 <= i);
              const float v0 = __uint_as_float(sc[q >> 4][q & 15]);
              const float v1 = __uint_as_float(sc[q >> 4][(q & 15) + 1]);
              pk[q >> 1] = pack_bf16x2(k0 ? v0 : 0.f, k1 ? v1 : 0.f);
            }
          }
          // bf16 pairs of keys overwrite score columns this thread has already read.
          tmem_st16u(tbase + kColS + lane_base + (uint32_t)(cb >> 1), pk);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(BAR(kBarScEmpty));
      mbar_arrive(BAR(kBarPReady));
      prev_pending = true;
      prev_cf = cf;
      ++kb;
    }
    if (ok) finish_prev();
  }

  // ---------------------------------------------------------------- teardown
  __syncthreads();
  if (*abort_flag && tid == 0) {
    // Let loads still in flight land before the shared memory is released.
    for (int jj = sMisc[4]; jj < sMisc[3]; ++jj) {
      const long long t0 = clock64();
      while (!mbar_try_wait(BAR(kBarFull + jj % S), (uint32_t)((jj / S) & 1)) && clock64() - t0 < kWaitCycles) {
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) tmem_dealloc(tbase, 512);
}

struct WsLayout {
  int NC, NS, G, Kp, Np, nstage, mode, rpc, ppr;
  uint32_t stage_bytes, oK, oV, oQ, oLA, oG, oBL, oWide, oGam, oRed, oMisc, oBar, oTm;
  size_t smem;
  size_t flag_bytes, agg_bytes, aggg_bytes;
};

constexpr int kSegChunks = 4;
constexpr size_t kMaxSmem = 227 * 1024;

uint32_t al1024(uint32_t x) { return (x + 1023u) & ~1023u; }
size_t al256(size_t x) { return (x + 255) / 256 * 256; }

WsLayout ws_layout(const GlaShape& s) {
  WsLayout L;
  // Chunk geometry (see the kernel's header comment).
  L.rpc = 1;
  L.ppr = 1;
  if (s.dir < 2) {
    L.mode = 0;
    L.NC = (s.T() + MC - 1) / MC;
  } else if (MC % s.Hg == 0) {
    L.mode = 1;
    L.rpc = MC / s.Hg;
    L.NC = (s.Wg + L.rpc - 1) / L.rpc;
  } else {
    L.mode = 2;
    L.ppr = (s.Hg + MC - 1) / MC;
    L.NC = s.Wg * L.ppr;
  }
  L.G = kSegChunks;
  L.NS = (L.NC + L.G - 1) / L.G;
  L.Kp = (s.dk + 15) / 16 * 16;
  L.Np = (s.dv + 15) / 16 * 16;
  L.oK = 0;
  L.oV = L.oK + (uint32_t)(L.Kp / 16) * ATOM32;
  L.oQ = L.oV + (uint32_t)(L.Np / 16) * ATOM32;
  L.oLA = al1024(L.oQ + (uint32_t)(L.Kp / 16) * ATOM32);
  const uint32_t la = (uint32_t)MC * (uint32_t)(s.dk + 4) * 4u;
  // The state MMA's A operand (K^ transposed, MN-major, M = 128 key channels) reads 8
  // channel blocks from oK; the stage is at least that large.
  L.stage_bytes = al1024(L.oLA + la > 8 * ATOM32 ? L.oLA + la : 8 * ATOM32);
  const uint32_t gtile = al1024((uint32_t)L.Kp * (uint32_t)L.Np * 2u);
  const uint32_t fixed = gtile + kMaxStages * 512 + 256 + 512 + 256 + 64 + 8 * kNumBars + 16;
  L.nstage = (1024 + 2 * (size_t)L.stage_bytes + fixed <= kMaxSmem) ? 2 : 1;
  L.oG = (uint32_t)L.nstage * L.stage_bytes;
  L.oBL = L.oG + gtile;
  L.oWide = L.oBL + kMaxStages * 512;
  L.oGam = L.oWide + 256;
  L.oRed = L.oGam + 512;
  L.oMisc = L.oRed + 256;
  L.oBar = L.oMisc + 64;
  L.oTm = L.oBar + 8 * kNumBars;
  L.smem = 1024 + (size_t)L.oTm + 16;
  if (L.smem < 120 * 1024) L.smem = 120 * 1024;  // one CTA per SM: it owns all 512 TMEM columns
  const size_t BH = (size_t)s.B * s.H;
  L.flag_bytes = al256((BH * L.NS + 1) * sizeof(int));
  L.agg_bytes = al256(BH * L.NS * s.dk * s.dv * sizeof(float));
  L.aggg_bytes = al256(BH * L.NS * s.dk * sizeof(float));
  return L;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
    else
      cudaGetLastError();
  }
  return fn;
}

// 5-D map over a [B][T][H][d] tensor viewed as (d, H, run position, run, B):
// raster scans have one run of T positions, column scans Wg runs of Hg.
bool encode_map(CUtensorMap* m, const void* base, bool f32, int d, int box0, CUtensorMapSwizzle sw, const GlaShape& s,
                bool column, int box_rows, int box_runs) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t e = f32 ? 4 : 2;
  const cuuint64_t T = (cuuint64_t)s.T(), H = (cuuint64_t)s.H;
  cuuint64_t dims[5], strides[4];
  dims[0] = (cuuint64_t)d;
  dims[1] = H;
  if (!column) {
    dims[2] = T;
    dims[3] = 1;
    strides[1] = H * d * e;
    strides[2] = T * H * d * e;
  } else {
    dims[2] = (cuuint64_t)s.Hg;
    dims[3] = (cuuint64_t)s.Wg;
    strides[1] = (cuuint64_t)s.Wg * H * d * e;
    strides[2] = H * d * e;
  }
  dims[4] = (cuuint64_t)s.B;
  strides[0] = (cuuint64_t)d * e;
  strides[3] = T * H * d * e;
  const cuuint32_t box[5] = {(cuuint32_t)box0, 1, (cuuint32_t)box_rows, (cuuint32_t)box_runs, 1};
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base),
            dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

size_t gla_ws_workspace_bytes(const GlaShape& s) {
  const WsLayout L = ws_layout(s);
  return L.flag_bytes + 2 * L.agg_bytes + L.aggg_bytes;
}

cudaError_t gla_ws_forward(const void* q, const void* k, const void* v, const float* la, void* out, const GlaShape& s,
                           void* workspace, cudaStream_t st) {
  const WsLayout L = ws_layout(s);
  if (L.smem > kMaxSmem) return cudaErrorInvalidValue;
  WsArgs a;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.k = static_cast<const __nv_bfloat16*>(k);
  a.v = static_cast<const __nv_bfloat16*>(v);
  a.la = la;
  a.out = static_cast<__nv_bfloat16*>(out);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const size_t BH = (size_t)s.B * s.H;
  a.flags = reinterpret_cast<int*>(ws);
  a.ticket = a.flags + BH * L.NS;
  a.agg_S = reinterpret_cast<float*>(ws + L.flag_bytes);
  a.incl_S = reinterpret_cast<float*>(ws + L.flag_bytes + L.agg_bytes);
  a.agg_g = reinterpret_cast<float*>(ws + L.flag_bytes + 2 * L.agg_bytes);
  a.H = s.H;
  a.BH = s.B * s.H;
  a.dk = s.dk;
  a.dv = s.dv;
  a.NC = L.NC;
  a.NS = L.NS;
  a.G = L.G;
  a.Kp = L.Kp;
  a.Np = L.Np;
  a.nstage = L.nstage;
  a.stage_bytes = L.stage_bytes;
  a.oK = L.oK;
  a.oV = L.oV;
  a.oQ = L.oQ;
  a.oLA = L.oLA;
  a.oG = L.oG;
  a.oBL = L.oBL;
  a.oWide = L.oWide;
  a.oGam = L.oGam;
  a.oRed = L.oRed;
  a.oMisc = L.oMisc;
  a.oBar = L.oBar;
  a.oTm = L.oTm;
  a.g = make_geom(s.Hg, s.Wg, s.dir);

  const bool column = s.dir >= 2;
  a.mode = L.mode;
  a.rpc = L.rpc;
  a.ppr = L.ppr;
  const int box_rows = L.mode == 1 ? s.Hg : MC, box_runs = L.mode == 1 ? L.rpc : 1;
  TensorMaps tm;
  memset(&tm, 0, sizeof(tm));
  // 16-channel boxes with the 32-byte swizzle land directly in the operand layout;
  // the kernel's expected transaction bytes assume exactly these boxes.
  if (!(encode_map(&tm.q, q, false, s.dk, 16, CU_TENSOR_MAP_SWIZZLE_32B, s, column, box_rows, box_runs) &&
        encode_map(&tm.k, k, false, s.dk, 16, CU_TENSOR_MAP_SWIZZLE_32B, s, column, box_rows, box_runs) &&
        encode_map(&tm.v, v, false, s.dv, 16, CU_TENSOR_MAP_SWIZZLE_32B, s, column, box_rows, box_runs) &&
        encode_map(&tm.la, la, true, s.dk, s.dk + 4, CU_TENSOR_MAP_SWIZZLE_NONE, s, column, box_rows, box_runs)))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaMemsetAsync(ws, 0, L.flag_bytes, st);  // flags and the ticket counter
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(gla_ws_fwd, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.smem);
  if (e != cudaSuccess) return e;
  gla_ws_fwd<<<(unsigned)(BH * L.NS), NT, L.smem, st>>>(a, tm);
  return cudaGetLastError();
}

}  // namespace dig
