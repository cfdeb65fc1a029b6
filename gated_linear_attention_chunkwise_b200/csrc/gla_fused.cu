// gla_fused.cu -- single-kernel chunk-wise GLA forward, bf16 q/k/v, sm_100a.
//
// Recurrence (DiG: gated linear attention): S_t = Diag(alpha_t) S_{t-1} + k_t^T v_t,
// o_t = q_t S_t, evaluated chunk-wise in on-chip memory (DiG paper notes,
// "硬件友好的效率设计": chunks of M tokens computed in SRAM, O(T M D + T D^2)).
//
// Work item = (head, segment of `G` consecutive 128-position chunks), taken in
// ticket order (all heads' segment 0, then segment 1, ...).  Per item:
//   pass 1  chunks of the segment in reverse scan order: with u_s the sum of the
//           log-gates scanned after s up to the segment end, K^_s = k_s exp(u_s)
//           (<= 1 for decaying gates) and the segment aggregate
//               S_seg = sum_s K^_s^T v_s,   gamma_seg = exp(sum of the segment's log-gates)
//           accumulates in TMEM (tcgen05, fp32).
//   look-back  publish (gamma_seg, S_seg); walk back over predecessor segments
//           of the same head (decoupled look-back: aggregates until an inclusive
//           state is found) to get S_in, the state before the segment; publish
//           the inclusive state Diag(gamma_seg) S_in + S_seg.  S_in goes straight
//           into TMEM as the running state.
//   pass 2  chunks in scan order (their rows are still in L2 from pass 1): with
//           u_r the in-chunk suffix, Q~ = q exp(-u), K^ = k exp(u), gamma = exp(chunk sum):
//               G = Diag(gamma) S                (threads, TMEM -> TMEM, bf16 copy to smem)
//               O = mask(Q~ K^T) V + Q~ G         (tcgen05; mask = scanned before or same)
//               S = G + K^T V                    (tcgen05, accumulates onto G in TMEM)
//           and O is stored in bf16 at each token's canonical position.
// A chunk whose gates decay by more than e^80 inside it cannot use exp(-u); it is
// evaluated token by token from the TMEM state (exact, slower).
//
// Suffix sums run as (key channel x part of the chunk) tasks over all threads;
// each part's offset (the sum of the later parts) is added when the gates are
// applied.  q, k, v arrive as whole rows; the threads apply the gates in registers
// and write the operands back in place in the swizzled UMMA layout.
//
// Shared memory: NSTAGE stages of {k, v, q: 32-byte-swizzled tiles of 128 rows x
// (d rounded up to 16) bf16; log-gate tile fp32 with a row pitch of dk+4, later
// reused for the bf16 score tile P}, plus the bf16 G tile.  Tiles are loaded by TMA
// (5-D tensor maps over [B][scan runs][run position][H][d], one elected thread,
// mbarrier completion), double-buffered across chunks; column scans of grids whose
// height is not a multiple of 8 use per-thread cp.async instead.
// TMEM: 512 columns -- scores [0,128), output [128,256), running state [256,384),
// segment aggregate [384,512); lane = tile row (scores, output) or key channel (states).
#include <math.h>
#include <string.h>

#include <cuda.h>

#include "dev_common.cuh"
#include "internal.h"

namespace dig {

namespace {

constexpr int MC = kChunkTC;             // chunk length = tcgen05 M
constexpr int NT = 256;                  // 8 warps: two groups of four cover all 128 TMEM lanes
constexpr uint32_t ATOM32 = MC * 32u;    // one 16-channel column block of a 32B-swizzled tile (4 KB)
constexpr uint32_t PART128 = MC * 128u;  // one 64-key part of the 128B-swizzled P tile (16 KB)
constexpr float kMaxGateRange = 80.0f;
constexpr uint32_t kColS = 0, kColO = 128, kColState = 256, kColSeg = 384;
constexpr uint32_t kLayoutSW32 = 6;

struct FusedArgs {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const float* la;
  __nv_bfloat16* out;
  float* agg_S;   // [BH][NS][dv/4][dk][4]  segment aggregates (quads of value columns)
  float* agg_g;   // [BH][NS][dk]           exp(segment log-gate sums)
  float* incl_S;  // [BH][NS][dv/4][dk][4]  state after the segment
  int* flags;     // [BH][NS]          0 nothing, 1 aggregate published, 2 inclusive published
  int* ticket;    // work-item counter
  int H, BH, dk, dv, NC, NS, G;
  int Kp, Np, nstage, box_rows;
  uint32_t stage_bytes, oK, oV, oQ, oLA, oG, oBL, oGam, oRed, oQT, oSeg, oBar, oTm;
  ScanGeom g;
};

struct TensorMaps {
  CUtensorMap q, k, v, la;
};

// ---------------------------------------------------------------------------
// Small helpers
// ---------------------------------------------------------------------------
// Byte offset of (row r, channel ch) in a 128-row tile stored as 16-channel
// column blocks of 32-byte rows with the 32-byte swizzle (16B chunk ^= bit 2 of the row).
__device__ __forceinline__ uint32_t sw32_off(uint32_t r, uint32_t ch) {
  return (ch >> 4) * ATOM32 + r * 32u + (((((ch >> 3) & 1u) ^ (r >> 2)) & 1u) << 4) + (ch & 7u) * 2u;
}

// Byte offset of G[i][j] in the G tile: rows i (key channel, the MMA's K) of 32
// bytes, 16-column blocks of Kp rows, 32-byte swizzle.
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

__device__ __forceinline__ float4 tmem_ld4(uint32_t taddr) {
  uint32_t r0, r1, r2, r3;
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(taddr));
  tmem_ld_wait();
  return make_float4(__uint_as_float(r0), __uint_as_float(r1), __uint_as_float(r2), __uint_as_float(r3));
}
__device__ __forceinline__ void tmem_st4(uint32_t taddr, float4 v) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1,%2,%3,%4};" ::"r"(taddr), "r"(__float_as_uint(v.x)),
               "r"(__float_as_uint(v.y)), "r"(__float_as_uint(v.z)), "r"(__float_as_uint(v.w))
               : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

// 5-D tiled TMA load into shared memory, completion counted on `bar`.
__device__ __forceinline__ void tma_load_5d(uint32_t dst, const CUtensorMap* map, int c0, int c1, int c2, int c3,
                                            int c4, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5, %6}], "
      "[%7];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4), "r"(bar)
      : "memory");
}

// ---------------------------------------------------------------------------
// Staging
// ---------------------------------------------------------------------------
// Base position f -> (position in run, run index) for the tensor maps' dims 2, 3.
__device__ __forceinline__ void run_coords(const ScanGeom& g, int f, int& y, int& x) {
  if (!g.column_base) {
    y = f;
    x = 0;
  } else {
    x = (f >= 0) ? f / g.Hg : -((-f + g.Hg - 1) / g.Hg);  // floor division
    y = f - x * g.Hg;
  }
}

// TMA: one thread issues every box of a job; the stage barrier counts the bytes.
// q, k, v arrive as whole rows of Kp (Np) channels -- 2*Kp bytes per row, channels
// >= d zero-filled -- and are permuted into the swizzled operand layout by the
// threads afterwards; the log-gate rows arrive with a pitch of dk+4 floats.
__device__ void issue_job_tma(const FusedArgs& a, const TensorMaps& tm, uint32_t st, uint32_t bar, int f0, bool with_q,
                              int b, int h) {
  const int R = a.box_rows;
  const int nbox = MC / R;
  const uint32_t bytes = (uint32_t)(with_q ? 2 : 1) * (uint32_t)a.Kp * 256u + (uint32_t)a.Np * 256u +
                         (uint32_t)MC * (uint32_t)(a.dk + 4) * 4u;
  mbar_expect_tx(bar, bytes);
  for (int m = 0; m < nbox; ++m) {
    int y, x;
    run_coords(a.g, f0 + m * R, y, x);
    const uint32_t r0 = (uint32_t)(m * R);
    tma_load_5d(st + a.oK + r0 * (uint32_t)a.Kp * 2u, &tm.k, 0, h, y, x, b, bar);
    if (with_q) tma_load_5d(st + a.oQ + r0 * (uint32_t)a.Kp * 2u, &tm.q, 0, h, y, x, b, bar);
    tma_load_5d(st + a.oV + r0 * (uint32_t)a.Np * 2u, &tm.v, 0, h, y, x, b, bar);
    tma_load_5d(st + a.oLA + r0 * (uint32_t)(a.dk + 4) * 4u, &tm.la, 0, h, y, x, b, bar);
  }
}

// cp.async fallback (column scans of grids whose height is not a multiple of 8):
// the same whole-row layout as the TMA path.
__device__ __forceinline__ void stage_rows_bf16(uint32_t tile, const __nv_bfloat16* base, int d, int W,
                                                const ScanGeom& g, int f0, int b, int h, int H) {
  const int cpr = W >> 3;
  for (int idx = threadIdx.x; idx < MC * cpr; idx += NT) {
    const int r = idx / cpr;
    const int cc = idx - r * cpr;
    const int f = f0 + r;
    const bool valid = (f >= 0) && (f < g.T) && (cc * 8 < d);
    const __nv_bfloat16* src = base;
    if (valid) src = base + (((int64_t)b * g.T + base_pos_to_token(g, f)) * H + h) * d + cc * 8;
    cp_async16(tile + (uint32_t)idx * 16u, src, valid);
  }
}

__device__ __forceinline__ void stage_la(uint32_t dst, const float* la, int dk, const ScanGeom& g, int f0, int b,
                                         int h, int H) {
  const int cpr = (dk + 4) >> 2;
  const uint32_t pitch = (uint32_t)(dk + 4) * 4u;
  for (int idx = threadIdx.x; idx < MC * cpr; idx += NT) {
    const int r = idx / cpr;
    const int cc = idx - r * cpr;
    const int f = f0 + r;
    const bool valid = (f >= 0) && (f < g.T) && (cc * 4 < dk);
    const float* src = la;
    if (valid) src = la + (((int64_t)b * g.T + base_pos_to_token(g, f)) * H + h) * dk + cc * 4;
    cp_async16(dst + (uint32_t)r * pitch + (uint32_t)cc * 16u, src, valid);
  }
}

// Load job j of an item: jobs [0, n) are pass 1 (reverse scan order), jobs
// [n, 2n) pass 2 (scan order).  Pass 1 needs no q.
__device__ __forceinline__ int job_chunk(int j, int c0, int n) { return j < n ? c0 + n - 1 - j : c0 + (j - n); }

template <bool TMA>
__device__ void issue_job(const FusedArgs& a, const TensorMaps& tm, uint32_t sbase, uint32_t bars, int j, int c0,
                          int n, int b, int h) {
  if (TMA) {
    if (j < 2 * n && threadIdx.x == 0) {
      const int s = j % a.nstage;
      const int f0 = chunk_first_base_pos(a.g, job_chunk(j, c0, n), MC);
      issue_job_tma(a, tm, sbase + (uint32_t)s * a.stage_bytes, bars + 8u * (uint32_t)s, f0, j >= n, b, h);
    }
  } else {
    if (j < 2 * n) {
      const uint32_t st = sbase + (uint32_t)(j % a.nstage) * a.stage_bytes;
      const int f0 = chunk_first_base_pos(a.g, job_chunk(j, c0, n), MC);
      stage_rows_bf16(st + a.oK, a.k, a.dk, a.Kp, a.g, f0, b, h, a.H);
      stage_rows_bf16(st + a.oV, a.v, a.dv, a.Np, a.g, f0, b, h, a.H);
      if (j >= n) stage_rows_bf16(st + a.oQ, a.q, a.dk, a.Kp, a.g, f0, b, h, a.H);
      stage_la(st + a.oLA, a.la, a.dk, a.g, f0, b, h, a.H);
    }
    cp_async_commit();  // one group per job slot (possibly empty) keeps the count uniform
  }
}

// Suffix sums of one chunk's log-gates as (channel, part) tasks over all threads:
// the 128 scan positions are cut into `np` parts (np*dk <= 256), and in place
// sLA[r][i] becomes the sum of the log-gates scanned after row r within its part.
// Scratch rows of 128 floats: part sums at row p, sums of |log-gate| at np+p and
// of the positive parts at 2np+p.
__device__ __forceinline__ void suffix_tasks(float* sLA, const FusedArgs& a, float* sScr, int np, int plen) {
  const int pw = a.dk + 4;
  const int task = threadIdx.x;
  if (task < np * a.dk) {
    const int i = task % a.dk, part = task / a.dk;
    const int p_hi = min(MC, (part + 1) * plen) - 1;  // last scan position of the part
    const int p_lo = part * plen;
    // walk scan positions p_hi down to p_lo: row r = p (forward) or 127 - p (reverse)
    float* ptr = sLA + (a.g.reverse ? (MC - 1 - p_hi) : p_hi) * pw + i;
    const int step = a.g.reverse ? pw : -pw;
    float acc = 0.f, ab = 0.f, po = 0.f;
#pragma unroll 4
    for (int p = p_hi; p >= p_lo; --p) {
      const float x = *ptr;
      *ptr = acc;
      acc += x;
      ab += fabsf(x);
      po += fmaxf(x, 0.f);
      ptr += step;
    }
    sScr[part * 128 + i] = acc;
    sScr[(np + part) * 128 + i] = ab;
    sScr[(2 * np + part) * 128 + i] = po;
  }
}

// Threads i < dk, after suffix_tasks: sQT[p][i] = offset of part p (sum over the
// later parts), sBL[i] = chunk sum, scratch row 3np = chunk sum of |log-gate|,
// row 3np+1 = chunk sum of the positive log-gates.
__device__ __forceinline__ void suffix_offsets(float* sQT, float* sBL, const FusedArgs& a, float* sScr, int np) {
  for (int i = threadIdx.x; i < a.dk; i += NT) {
    float off = 0.f, ab = 0.f, po = 0.f;
    for (int p = np - 1; p >= 0; --p) {
      sQT[p * 128 + i] = off;
      off += sScr[p * 128 + i];
      ab += sScr[(np + p) * 128 + i];
      po += sScr[(2 * np + p) * 128 + i];
    }
    sBL[i] = off;
    sScr[(3 * np) * 128 + i] = ab;
    sScr[(3 * np + 1) * 128 + i] = po;
  }
}

// In-place permutation of a whole-row tile (row r at r*2W bytes) into the
// 32-byte-swizzled operand layout.  Each thread owns 16-byte chunks c = tid + 256 t.
constexpr int kMaxChunksPerThread = 8;  // 128 rows x 16 chunks / 256 threads

template <int MODE>  // 0: copy (v), 1: K^ = k exp(u), 2: Q~ = q exp(-u)
__device__ __forceinline__ void load_rows(const uint8_t* tile, int W, uint4 (&reg)[kMaxChunksPerThread],
                                          const FusedArgs& a, const float* sLA, const float* sQT, const float* sOff,
                                          int plen) {
  const int cpr = W >> 3;
  const int total = MC * cpr;
#pragma unroll
  for (int t = 0; t < kMaxChunksPerThread; ++t) {
    const int c = threadIdx.x + NT * t;
    if (c < total) {
      uint4 w = *reinterpret_cast<const uint4*>(tile + (uint32_t)c * 16u);
      if (MODE != 0) {
        const int r = c / cpr, ch = (c - r * cpr) * 8;
        if (ch < a.dk) {
          const int p = a.g.reverse ? (MC - 1 - r) : r;
          const float* qoff = sQT + (p / plen) * 128 + ch;
          const float* urow = sLA + r * (a.dk + 4) + ch;
          const float4 u0 = *reinterpret_cast<const float4*>(urow);
          const float4 u1 = *reinterpret_cast<const float4*>(urow + 4);
          const float4 o0 = *reinterpret_cast<const float4*>(qoff);
          const float4 o1 = *reinterpret_cast<const float4*>(qoff + 4);
          float e[8] = {u0.x + o0.x, u0.y + o0.y, u0.z + o0.z, u0.w + o0.w,
                        u1.x + o1.x, u1.y + o1.y, u1.z + o1.z, u1.w + o1.w};
          if (sOff) {
            const float4 f0 = *reinterpret_cast<const float4*>(sOff + ch);
            const float4 f1 = *reinterpret_cast<const float4*>(sOff + ch + 4);
            e[0] += f0.x;
            e[1] += f0.y;
            e[2] += f0.z;
            e[3] += f0.w;
            e[4] += f1.x;
            e[5] += f1.y;
            e[6] += f1.z;
            e[7] += f1.w;
          }
          uint32_t* u = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) {
            const float2 x = unpack_bf16x2(u[jj]);
            const float s0 = MODE == 1 ? e[2 * jj] : -e[2 * jj];
            const float s1 = MODE == 1 ? e[2 * jj + 1] : -e[2 * jj + 1];
            u[jj] = pack_bf16x2(x.x * __expf(s0), x.y * __expf(s1));
          }
        }
      }
      reg[t] = w;
    }
  }
}

__device__ __forceinline__ void store_swizzled(uint8_t* tile, int W, const uint4 (&reg)[kMaxChunksPerThread]) {
  const int cpr = W >> 3;
  const int total = MC * cpr;
#pragma unroll
  for (int t = 0; t < kMaxChunksPerThread; ++t) {
    const int c = threadIdx.x + NT * t;
    if (c < total) {
      const int r = c / cpr, cc = c - r * cpr;
      *reinterpret_cast<uint4*>(tile + sw32_off((uint32_t)r, (uint32_t)cc * 8u)) = reg[t];
    }
  }
}

__device__ __forceinline__ int wait_mma(uint32_t bar, uint32_t& phase) {
  const bool ok = mbar_wait(bar, phase);
  phase ^= 1u;
  tc_fence_after();
  if (!ok) report_status(GLA_ERR_TIMEOUT);
  return ok ? 0 : 1;
}

// Spin (thread 0) until flags[idx] >= 1; returns the flag, or 0 on timeout.
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

// Exact token-by-token evaluation of one chunk from the TMEM running state, for
// chunks whose gates decay too fast for the factorised form (q, k still whole
// rows, v already swizzled).  Thread (lane i, group w) owns state row i, columns
// [64w, 64w+64).  The output is reduced over
// key channels with warp shuffles and a small shared buffer.
__device__ void chunk_serial(const FusedArgs& a, const uint8_t* st, float* red, uint32_t tstate, int f0, int b,
                             int h) {
  const int i = threadIdx.x & (MC - 1);
  const int grp = threadIdx.x >> 7;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
  const int col0 = grp * 64;
  float s[64];
#pragma unroll
  for (int blk = 0; blk < 4; ++blk) {
    float t16[16];
    tmem_ld16(tstate + lane_base + (uint32_t)(col0 + blk * 16), t16);
#pragma unroll
    for (int j = 0; j < 16; ++j) s[blk * 16 + j] = (i < a.dk && col0 + blk * 16 + j < a.dv) ? t16[j] : 0.f;
  }
  const uint8_t* sQ = st + a.oQ;
  const uint8_t* sK = st + a.oK;
  const uint8_t* sV = st + a.oV;
  for (int step = 0; step < MC; ++step) {
    const int r = a.g.reverse ? (MC - 1 - step) : step;
    const int f = f0 + r;
    if (f < 0 || f >= a.g.T) continue;  // padding row: uniform across the block
    const int t = base_pos_to_token(a.g, f);
    float alpha = 1.f, kq = 0.f, qi = 0.f;
    if (i < a.dk) {
      alpha = __expf(__ldg(a.la + (((int64_t)b * a.g.T + t) * a.H + h) * a.dk + i));
      kq = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sK + ((uint32_t)r * (uint32_t)a.Kp + i) * 2u));
      qi = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sQ + ((uint32_t)r * (uint32_t)a.Kp + i) * 2u));
    }
#pragma unroll
    for (int j = 0; j < 64; ++j) {
      const int col = col0 + j;
      float vj = 0.f;
      if (col < a.dv)
        vj = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sV + sw32_off((uint32_t)r, (uint32_t)col)));
      s[j] = fmaf(alpha, s[j], kq * vj);
      float x = qi * s[j];
      x += __shfl_xor_sync(0xffffffffu, x, 16);
      x += __shfl_xor_sync(0xffffffffu, x, 8);
      x += __shfl_xor_sync(0xffffffffu, x, 4);
      x += __shfl_xor_sync(0xffffffffu, x, 2);
      x += __shfl_xor_sync(0xffffffffu, x, 1);
      if (lane == 0) red[warp * 64 + j] = x;
    }
    __syncthreads();
    if (threadIdx.x < a.dv) {
      const int col = threadIdx.x;
      const int g2 = col >> 6, jj = col & 63;
      const float o = red[(g2 * 4 + 0) * 64 + jj] + red[(g2 * 4 + 1) * 64 + jj] + red[(g2 * 4 + 2) * 64 + jj] +
                      red[(g2 * 4 + 3) * 64 + jj];
      a.out[(((int64_t)b * a.g.T + t) * a.H + h) * a.dv + col] = __float2bfloat16_rn(o);
    }
    __syncthreads();
  }
#pragma unroll
  for (int blk = 0; blk < 4; ++blk) {
    float t16[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) t16[j] = s[blk * 16 + j];
    tmem_st16(tstate + lane_base + (uint32_t)(col0 + blk * 16), t16);
  }
  tmem_st_wait();
}

__device__ __forceinline__ uint32_t align1024(uint32_t x) { return (x + 1023u) & ~1023u; }

// ---------------------------------------------------------------------------
// The kernel
// ---------------------------------------------------------------------------
template <bool TMA>
__global__ void __launch_bounds__(NT, 1) gla_fused_fwd(const FusedArgs a, const __grid_constant__ TensorMaps tm) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t sbase = align1024(raw_u32);
  uint8_t* smem = smem_raw + (sbase - raw_u32);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int lane_row = tid & (MC - 1);  // TMEM lane of this thread (tile row / key channel)
  const int grp = tid >> 7;             // 0: warps 0-3, 1: warps 4-7 (split columns)
  const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
  float* sBL = reinterpret_cast<float*>(smem + a.oBL);
  float* sGam = reinterpret_cast<float*>(smem + a.oGam);
  float* red = reinterpret_cast<float*>(smem + a.oRed);   // suffix scratch / serial-path reduction
  float* sQT = reinterpret_cast<float*>(smem + a.oQT);    // [4][128] quarter offsets
  float* sOff = reinterpret_cast<float*>(smem + a.oSeg);  // [128] pass-1 segment offset
  float* sPos = sOff + 128;                               // [128] pass-1 positive log-gate mass
  volatile int* sInt = reinterpret_cast<volatile int*>(smem + a.oTm + 8);  // [0] item, [1] flag
  const uint32_t bar_mma = sbase + a.oBar;
  const uint32_t bar_ld = sbase + a.oBar + 8;  // one per stage (TMA)

  if (warp == 0) {
    tmem_alloc(sbase + a.oTm, 512);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(bar_mma, 1);
    for (int s = 0; s < a.nstage; ++s) mbar_init(bar_ld + 8u * (uint32_t)s, 1);
    fence_mbar_init();
    sInt[0] = atomicAdd(a.ticket, 1);
  }
  for (int i = tid; i < 128; i += NT) {
    sBL[i] = 0.f;  // rows dk..127 of the state get gamma = exp(0) = 1 (their state stays zero)
    sGam[i] = 1.f;
    sOff[i] = 0.f;
    sPos[i] = 0.f;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *reinterpret_cast<volatile uint32_t*>(smem + a.oTm);
  const int item = sInt[0];
  const int seg = item / a.BH, bh = item - seg * a.BH;
  const int b = bh / a.H, h = bh - b * a.H;
  const int c0 = seg * a.G;
  const int n = min(a.G, a.NC - c0);
  const int64_t seg_id = (int64_t)bh * a.NS + seg;
  const int col0 = grp * 64;  // state / aggregate columns owned by this thread
  uint32_t phase = 0;

  // Suffix parts: np parts of plen scan positions, np * dk <= 256 tasks.
  const int np = max(1, min(8, NT / a.dk));
  const int plen = (MC + np - 1) / np;

  for (int j = 0; j < a.nstage; ++j) issue_job<TMA>(a, tm, sbase, bar_ld, j, c0, n, b, h);

  int aborted = 0, jstop = 2 * n;  // 1: a load never arrived, 2: an MMA never completed
  for (int j = 0; j < 2 * n; ++j) {
    const int s_idx = j % a.nstage;
    int fail = 0;
    if (TMA) {
      fail = mbar_wait(bar_ld + 8u * (uint32_t)s_idx, (uint32_t)((j / a.nstage) & 1)) ? 0 : 1;
    } else {
      if (a.nstage == 2)
        asm volatile("cp.async.wait_group 1;" ::: "memory");
      else
        asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    if (__syncthreads_or(fail)) {  // a load never arrived: record it and stop this CTA
      if (tid == 0) report_status(GLA_ERR_TIMEOUT);
      aborted = 1;
      jstop = j;
      break;
    }
    const uint32_t st_u32 = sbase + (uint32_t)s_idx * a.stage_bytes;
    uint8_t* st = smem + (st_u32 - sbase);
    float* sLA = reinterpret_cast<float*>(st + a.oLA);
    const int c = job_chunk(j, c0, n);
    const int f0 = chunk_first_base_pos(a.g, c, MC);

    // v: whole rows -> swizzled (copy); suffix sums of the log-gates meanwhile.
    uint4 regA[kMaxChunksPerThread], regB[kMaxChunksPerThread];
    load_rows<0>(st + a.oV, a.Np, regA, a, sLA, sQT, nullptr, plen);
    suffix_tasks(sLA, a, red, np, plen);
    __syncthreads();
    store_swizzled(st + a.oV, a.Np, regA);
    suffix_offsets(sQT, sBL, a, red, np);
    __syncthreads();

    if (j < n) {
      // ---------------- pass 1: segment aggregate --------------------------
      load_rows<1>(st + a.oK, a.Kp, regA, a, sLA, sQT, sOff, plen);
      __syncthreads();
      store_swizzled(st + a.oK, a.Kp, regA);
      fence_proxy_async_smem();
      __syncthreads();
      if (tid == 0) {
        tc_fence_after();
        const uint32_t id = idesc_bf16_f32(MC, a.Np, true, true);
#pragma unroll 1
        for (int kk = 0; kk < MC / 16; ++kk)
          umma_ss(tbase + kColSeg, desc_sw32(st_u32 + a.oK + (uint32_t)kk * 512u, ATOM32, 256u),
                  desc_sw32(st_u32 + a.oV + (uint32_t)kk * 512u, ATOM32, 256u), id, (j > 0 || kk > 0) ? 1u : 0u);
        umma_commit(bar_mma);
      }
      // The offset for the next (earlier) chunk includes this chunk's sum.
      for (int i = tid; i < a.dk; i += NT) {
        sOff[i] += sBL[i];
        sPos[i] += red[(3 * np + 1) * 128 + i];  // sum of the positive log-gates
      }
      fail |= wait_mma(bar_mma, phase);
    } else {
      if (j == n) {
        // ---------------- publish the aggregate, look back --------------------
        for (int i = tid; i < a.dk; i += NT) {
          if (!(sPos[i] <= kMaxGateRange)) report_status(GLA_ERR_RANGE);
          const float gseg = __expf(sOff[i]);
          a.agg_g[seg_id * a.dk + i] = gseg;
          sGam[i] = gseg;
        }
        // States travel as quads of value columns ([dv/4][dk][4]) so that lane i's
        // 16-byte accesses are contiguous across a warp; group g owns quads [q0, q1).
        const int i = lane_row;
        const int DQ = a.dv >> 2, hq = (DQ + 1) >> 1;
        const int q0 = grp * hq, q1 = min(DQ, q0 + hq);
        for (int jq = q0; jq < q1; ++jq) {
          const float4 x = tmem_ld4(tbase + kColSeg + lane_base + (uint32_t)(4 * jq));
          if (i < a.dk) *reinterpret_cast<float4*>(a.agg_S + ((seg_id * DQ + jq) * a.dk + i) * 4) = x;
        }
        __threadfence();
        __syncthreads();
        if (tid == 0) st_release(a.flags + seg_id, 1);

        float4 acc[16];
#pragma unroll
        for (int t = 0; t < 16; ++t) acc[t] = make_float4(0.f, 0.f, 0.f, 0.f);
        float gam = 1.f;
        for (int p = seg - 1; p >= 0; --p) {
          const int64_t pid = (int64_t)bh * a.NS + p;
          if (tid == 0) sInt[1] = wait_flag(a.flags, pid);
          __syncthreads();
          const int f = sInt[1];
          __syncthreads();
          if (f == 0) break;  // timed out (recorded in the device status)
          if (i < a.dk) {
            const float* src = (f == 2 ? a.incl_S : a.agg_S);
#pragma unroll
            for (int t = 0; t < 16; ++t) {
              if (q0 + t < q1) {
                const float4 x = __ldcg(reinterpret_cast<const float4*>(src + ((pid * DQ + q0 + t) * a.dk + i) * 4));
                acc[t].x = fmaf(gam, x.x, acc[t].x);
                acc[t].y = fmaf(gam, x.y, acc[t].y);
                acc[t].z = fmaf(gam, x.z, acc[t].z);
                acc[t].w = fmaf(gam, x.w, acc[t].w);
              }
            }
            if (f == 1) gam *= __ldcg(a.agg_g + pid * a.dk + i);
          }
          if (f == 2) break;
        }
        // acc = S_in (row i): the running state starts there; the inclusive state
        // after this segment is Diag(gamma_seg) S_in + S_seg.
        {
          const float gs = sGam[i];
#pragma unroll
          for (int t = 0; t < 16; ++t) {
            if (q0 + t < q1) {
              const uint32_t col = (uint32_t)(4 * (q0 + t));
              tmem_st4(tbase + kColState + lane_base + col, acc[t]);
              const float4 sg = tmem_ld4(tbase + kColSeg + lane_base + col);
              if (i < a.dk)
                *reinterpret_cast<float4*>(a.incl_S + ((seg_id * DQ + q0 + t) * a.dk + i) * 4) =
                    make_float4(fmaf(gs, acc[t].x, sg.x), fmaf(gs, acc[t].y, sg.y), fmaf(gs, acc[t].z, sg.z),
                                fmaf(gs, acc[t].w, sg.w));
            }
          }
        }
        tmem_st_wait();
        __threadfence();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) st_release(a.flags + seg_id, 2);
        tc_fence_after();
      }

      // ---------------- pass 2: outputs ---------------------------------------
      int wide = 0;
      for (int i = tid; i < a.dk; i += NT)
        if (!(red[(3 * np) * 128 + i] <= kMaxGateRange)) wide = 1;
      wide = __syncthreads_or(wide);
      if (wide) {
        chunk_serial(a, st, red, tbase + kColState, f0, b, h);
      } else {
        load_rows<1>(st + a.oK, a.Kp, regA, a, sLA, sQT, nullptr, plen);
        load_rows<2>(st + a.oQ, a.Kp, regB, a, sLA, sQT, nullptr, plen);
        __syncthreads();
        store_swizzled(st + a.oK, a.Kp, regA);
        store_swizzled(st + a.oQ, a.Kp, regB);
        fence_proxy_async_smem();
        __syncthreads();
        if (tid == 0) {
          tc_fence_after();
          const uint32_t id = idesc_bf16_f32(MC, MC, false, false);
          const int nk = a.Kp >> 4;
#pragma unroll 1
          for (int kk = 0; kk < nk; ++kk)
            umma_ss(tbase + kColS, desc_sw32(st_u32 + a.oQ + (uint32_t)kk * ATOM32, 16u, 256u),
                    desc_sw32(st_u32 + a.oK + (uint32_t)kk * ATOM32, 16u, 256u), id, kk > 0 ? 1u : 0u);
          umma_commit(bar_mma);
        }
        // While the score MMA runs: G = Diag(gamma) S, back into TMEM and (bf16) into smem.
        if ((warp & 3) * 32 < a.Kp) {  // lanes >= Kp hold no key channel
          const int i = lane_row;
          const float gm = __expf(sBL[i]);
          for (int blk = 0; blk < 4; ++blk) {
            const int cb = col0 + blk * 16;
            if (cb >= a.Np) break;  // uniform per warp group
            float t16[16];
            tmem_ld16(tbase + kColState + lane_base + (uint32_t)cb, t16);
#pragma unroll
            for (int q = 0; q < 16; ++q) t16[q] *= gm;
            tmem_st16(tbase + kColState + lane_base + (uint32_t)cb, t16);
            if (i < a.Kp) {
              uint4 w0 = make_uint4(pack_bf16x2(t16[0], t16[1]), pack_bf16x2(t16[2], t16[3]),
                                    pack_bf16x2(t16[4], t16[5]), pack_bf16x2(t16[6], t16[7]));
              uint4 w1 = make_uint4(pack_bf16x2(t16[8], t16[9]), pack_bf16x2(t16[10], t16[11]),
                                    pack_bf16x2(t16[12], t16[13]), pack_bf16x2(t16[14], t16[15]));
              *reinterpret_cast<uint4*>(smem + a.oG + g_off((uint32_t)i, (uint32_t)cb, (uint32_t)a.Kp)) = w0;
              *reinterpret_cast<uint4*>(smem + a.oG + g_off((uint32_t)i, (uint32_t)cb + 8u, (uint32_t)a.Kp)) = w1;
            }
          }
          tmem_st_wait();
          fence_proxy_async_smem();
        }
        fail |= wait_mma(bar_mma, phase);

        // Scores -> mask -> bf16 P (this group: keys [64 grp, 64 grp + 64)), in the log-gate area.
        // 32-key blocks that a whole warp keeps (or drops) entirely skip the compares.
        {
          const int r = lane_row;
          const int rlo = (warp & 3) * 32, rhi = rlo + 31;
#pragma unroll 1
          for (int half = 0; half < 2; ++half) {
            const int cb = col0 + half * 32;
            const bool none = a.g.reverse ? (cb + 31 < rlo) : (cb > rhi);
            const bool all = a.g.reverse ? (cb >= rhi) : (cb + 31 <= rlo);
            uint32_t pk[16];
            if (none) {
#pragma unroll
              for (int q = 0; q < 16; ++q) pk[q] = 0u;
            } else {
              float sc[32];
              tmem_ld32(tbase + kColS + lane_base + (uint32_t)cb, sc);
              if (all) {
#pragma unroll
                for (int q = 0; q < 32; q += 2) pk[q >> 1] = pack_bf16x2(sc[q], sc[q + 1]);
              } else {
#pragma unroll
                for (int q = 0; q < 32; q += 2) {
                  const int s0 = cb + q, s1 = cb + q + 1;
                  const bool k0 = a.g.reverse ? (s0 >= r) : (s0 <= r);
                  const bool k1 = a.g.reverse ? (s1 >= r) : (s1 <= r);
                  pk[q >> 1] = pack_bf16x2(k0 ? sc[q] : 0.f, k1 ? sc[q + 1] : 0.f);
                }
              }
            }
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              const int s = cb + q4 * 8;
              const uint32_t o = a.oLA + (uint32_t)(s >> 6) * PART128 + sw128((uint32_t)r, (uint32_t)(s & 63) * 2u);
              *reinterpret_cast<uint4*>(st + o) =
                  make_uint4(pk[q4 * 4], pk[q4 * 4 + 1], pk[q4 * 4 + 2], pk[q4 * 4 + 3]);
            }
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
          tc_fence_after();
          const uint32_t id_pv = idesc_bf16_f32(MC, a.Np, false, true);
#pragma unroll 1
          for (int kk = 0; kk < MC / 16; ++kk)
            umma_ss(tbase + kColO, desc_kmajor(st_u32 + a.oLA, PART128, kk),
                    desc_sw32(st_u32 + a.oV + (uint32_t)kk * 512u, ATOM32, 256u), id_pv, kk > 0 ? 1u : 0u);
          const uint32_t id_qg = idesc_bf16_f32(MC, a.Np, false, true);
          const int nk = a.Kp >> 4;
#pragma unroll 1
          for (int kk = 0; kk < nk; ++kk)
            umma_ss(tbase + kColO, desc_sw32(st_u32 + a.oQ + (uint32_t)kk * ATOM32, 16u, 256u),
                    desc_sw32(sbase + a.oG + (uint32_t)kk * 512u, (uint32_t)a.Kp * 32u, 256u), id_qg, 1u);
          const uint32_t id_s = idesc_bf16_f32(MC, a.Np, true, true);
#pragma unroll 1
          for (int kk = 0; kk < MC / 16; ++kk)
            umma_ss(tbase + kColState, desc_sw32(st_u32 + a.oK + (uint32_t)kk * 512u, ATOM32, 256u),
                    desc_sw32(st_u32 + a.oV + (uint32_t)kk * 512u, ATOM32, 256u), id_s, 1u);
          umma_commit(bar_mma);
        }
        fail |= wait_mma(bar_mma, phase);

        // Epilogue: output row r -> out[b][token][h][:], 16-column blocks split between the groups.
        {
          const int r = lane_row;
          const int f = f0 + r;
          const bool valid = (f >= 0) && (f < a.g.T);
          __nv_bfloat16* orow = a.out;
          if (valid) orow = a.out + (((int64_t)b * a.g.T + base_pos_to_token(a.g, f)) * a.H + h) * a.dv;
          for (int blk = grp; blk < (a.Np >> 4); blk += 2) {
            const int cb = blk * 16;
            float o[16];
            tmem_ld16(tbase + kColO + lane_base + (uint32_t)cb, o);
            if (valid) {
#pragma unroll
              for (int q = 0; q < 16; q += 8) {
                if (cb + q < a.dv) {
                  *reinterpret_cast<uint4*>(orow + cb + q) =
                      make_uint4(pack_bf16x2(o[q], o[q + 1]), pack_bf16x2(o[q + 2], o[q + 3]),
                                 pack_bf16x2(o[q + 4], o[q + 5]), pack_bf16x2(o[q + 6], o[q + 7]));
                }
              }
            }
          }
        }
      }
    }
    // Stage j % nstage is free (all MMAs on it have completed): load job j + nstage into it.
    fence_proxy_async_smem();
    tc_fence_before();
    if (__syncthreads_or(fail)) {  // an MMA never completed (recorded): stop this CTA
      aborted = 2;
      jstop = j + 1;
      break;
    }
    tc_fence_after();
    issue_job<TMA>(a, tm, sbase, bar_ld, j + a.nstage, c0, n, b, h);
  }

  if (aborted) {
    // Give copies and MMAs still in flight a bounded chance to land before the
    // shared memory and TMEM are released.
    if (TMA)
      for (int jj = jstop; jj < min(2 * n, jstop + a.nstage); ++jj)
        mbar_wait(bar_ld + 8u * (uint32_t)(jj % a.nstage), (uint32_t)((jj / a.nstage) & 1));
    if (aborted == 2) mbar_wait(bar_mma, phase ^ 1u);
  }
  if (!TMA) asm volatile("cp.async.wait_group 0;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tbase, 512);
}

struct FusedLayout {
  int NC, NS, G, Kp, Np, nstage;
  uint32_t stage_bytes, oK, oV, oQ, oLA, oG, oBL, oGam, oRed, oQT, oSeg, oBar, oTm;
  size_t smem;
  size_t flag_bytes, agg_bytes, aggg_bytes;
};

constexpr int kSegChunks = 4;
constexpr size_t kMaxSmem = 227 * 1024;

uint32_t al1024(uint32_t x) { return (x + 1023u) & ~1023u; }
size_t al256(size_t x) { return (x + 255) / 256 * 256; }

FusedLayout fused_layout(const GlaShape& s) {
  FusedLayout L;
  L.NC = (s.T() + MC - 1) / MC;
  L.G = kSegChunks;
  L.NS = (L.NC + L.G - 1) / L.G;
  L.Kp = (s.dk + 15) / 16 * 16;
  L.Np = (s.dv + 15) / 16 * 16;
  L.oK = 0;
  L.oV = L.oK + (uint32_t)(L.Kp / 16) * ATOM32;
  L.oQ = L.oV + (uint32_t)(L.Np / 16) * ATOM32;
  L.oLA = al1024(L.oQ + (uint32_t)(L.Kp / 16) * ATOM32);
  const uint32_t la = (uint32_t)MC * (uint32_t)(s.dk + 4) * 4u;
  L.stage_bytes = al1024(L.oLA + (la > 2 * PART128 ? la : 2 * PART128));
  // G tile, gate sums (BL, Gam), scratch (3np+2 rows of 128 floats, at least the 4
  // the serial path uses), part offsets (np x 128), segment offset / positive mass
  // (2 x 128), barriers and TMEM base.
  const int np = s.dk >= 256 ? 1 : (256 / s.dk > 8 ? 8 : 256 / s.dk);
  const uint32_t red_rows = (uint32_t)(3 * np + 2 > 4 ? 3 * np + 2 : 4);
  const uint32_t fixed =
      al1024((uint32_t)L.Kp * (uint32_t)L.Np * 2u) + 512 + 512 + red_rows * 512 + (uint32_t)np * 512 + 1024 + 64;
  L.nstage = (1024 + 2 * (size_t)L.stage_bytes + fixed <= kMaxSmem) ? 2 : 1;
  L.oG = (uint32_t)L.nstage * L.stage_bytes;
  L.oBL = L.oG + al1024((uint32_t)L.Kp * (uint32_t)L.Np * 2u);
  L.oGam = L.oBL + 512;
  L.oRed = L.oGam + 512;
  L.oQT = L.oRed + red_rows * 512;
  L.oSeg = L.oQT + (uint32_t)np * 512;
  L.oBar = L.oSeg + 1024;
  L.oTm = L.oBar + 32;
  L.smem = 1024 + (size_t)L.oTm + 32;
  if (L.smem < 120 * 1024) L.smem = 120 * 1024;  // one CTA per SM: it owns all 512 TMEM columns
  const size_t BH = (size_t)s.B * s.H;
  L.flag_bytes = al256((BH * L.NS + 1) * sizeof(int));
  L.agg_bytes = al256(BH * L.NS * s.dk * s.dv * sizeof(float));
  L.aggg_bytes = al256(BH * L.NS * s.dk * sizeof(float));
  return L;
}

// ---- tensor maps (driver entry point, looked up once) ----
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
                bool column, int box_rows) {
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
    strides[1] = H * d * e;      // next position of the run
    strides[2] = T * H * d * e;  // (a single run)
  } else {
    dims[2] = (cuuint64_t)s.Hg;
    dims[3] = (cuuint64_t)s.Wg;
    strides[1] = (cuuint64_t)s.Wg * H * d * e;  // next row of the grid
    strides[2] = H * d * e;                     // next column
  }
  dims[4] = (cuuint64_t)s.B;
  strides[0] = (cuuint64_t)d * e;
  strides[3] = T * H * d * e;
  const cuuint32_t box[5] = {(cuuint32_t)box0, 1, (cuuint32_t)box_rows, 1, 1};
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  const CUresult r = fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5,
                        const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int gcd_int(int x, int y) {
  while (y) {
    const int t = x % y;
    x = y;
    y = t;
  }
  return x;
}

}  // namespace

size_t gla_fused_workspace_bytes(const GlaShape& s) {
  const FusedLayout L = fused_layout(s);
  return L.flag_bytes + 2 * L.agg_bytes + L.aggg_bytes;
}

cudaError_t gla_fused_forward(const void* q, const void* k, const void* v, const float* la, void* out,
                              const GlaShape& s, void* workspace, cudaStream_t st) {
  const FusedLayout L = fused_layout(s);
  if (L.smem > kMaxSmem) return cudaErrorInvalidValue;
  FusedArgs a;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.k = static_cast<const __nv_bfloat16*>(k);
  a.v = static_cast<const __nv_bfloat16*>(v);
  a.la = la;
  a.out = static_cast<__nv_bfloat16*>(out);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  a.flags = reinterpret_cast<int*>(ws);
  const size_t BH = (size_t)s.B * s.H;
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
  a.oGam = L.oGam;
  a.oRed = L.oRed;
  a.oQT = L.oQT;
  a.oSeg = L.oSeg;
  a.oBar = L.oBar;
  a.oTm = L.oTm;
  a.g = make_geom(s.Hg, s.Wg, s.dir);

  // TMA boxes must cover whole 8-row swizzle atoms: raster scans load 128-row boxes;
  // column scans load boxes of gcd(Hgrid, 128) rows, used when that is >= 8.
  const bool column = s.dir >= 2;
  a.box_rows = column ? gcd_int(s.Hg, MC) : MC;
  TensorMaps tm;
  memset(&tm, 0, sizeof(tm));
  bool use_tma = a.box_rows >= 8;
  if (use_tma) {
    // Whole rows: Kp (Np) channels per box row, channels >= d read as zero.  The
    // kernel's expected transaction bytes assume exactly these boxes.
    use_tma = encode_map(&tm.q, q, false, s.dk, L.Kp, CU_TENSOR_MAP_SWIZZLE_NONE, s, column, a.box_rows) &&
              encode_map(&tm.k, k, false, s.dk, L.Kp, CU_TENSOR_MAP_SWIZZLE_NONE, s, column, a.box_rows) &&
              encode_map(&tm.v, v, false, s.dv, L.Np, CU_TENSOR_MAP_SWIZZLE_NONE, s, column, a.box_rows) &&
              encode_map(&tm.la, la, true, s.dk, s.dk + 4, CU_TENSOR_MAP_SWIZZLE_NONE, s, column, a.box_rows);
  }

  cudaError_t e = cudaMemsetAsync(ws, 0, L.flag_bytes, st);  // flags and the ticket counter
  if (e != cudaSuccess) return e;
  if (use_tma) {
    e = cudaFuncSetAttribute(gla_fused_fwd<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.smem);
    if (e != cudaSuccess) return e;
    gla_fused_fwd<true><<<(unsigned)(BH * L.NS), NT, L.smem, st>>>(a, tm);
  } else {
    e = cudaFuncSetAttribute(gla_fused_fwd<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.smem);
    if (e != cudaSuccess) return e;
    gla_fused_fwd<false><<<(unsigned)(BH * L.NS), NT, L.smem, st>>>(a, tm);
  }
  return cudaGetLastError();
}

}  // namespace dig
