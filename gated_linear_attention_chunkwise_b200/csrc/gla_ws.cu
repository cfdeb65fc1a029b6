// gla_ws.cu -- warp-specialised chunk-wise GLA forward, bf16 q/k/v, sm_100a.
//
// Recurrence (DiG: gated linear attention): S_t = Diag(alpha_t) S_{t-1} + k_t^T v_t,
// o_t = q_t S_t, evaluated chunk-wise in on-chip memory (DiG paper notes,
// "硬件友好的效率设计": chunks of M tokens computed in SRAM, O(T M D + T D^2)).
//
// Work items are (head, segment of G chunks of 128 scan positions), taken in ticket
// order by persistent CTAs.  Per item:
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
// Roles (16 warps, 512 threads), connected by mbarriers:
//   warp 0      producer: takes tickets and posts jobs (pass 1 of the next item, then
//               pass 2 of the current one); TMA loads of each chunk's q, k, v
//               (32-byte-swizzled 16-channel boxes, the UMMA operand layout) and
//               log-gates into a ring of stages;
//   warp 1      MMA issuer (tcgen05, one thread) and TMEM owner; per pass-2 chunk
//               S = Q~ K^T, then Q~ G and K^T V, then P V;
//   warps 2-3   suffix sums of the log-gates, two row quarters per warp in parallel
//               (lane = pair of key channels), and each quarter's offset;
//   warps 4-7   gate group, warp = quarter of the chunk's rows: the gates applied in
//               place (K^, Q~; lane = row), then the score masking to bf16 P;
//   warps 8-11  output group, one thread per TMEM lane: G = Diag(gamma) S, output
//               epilogue, serial path;
//   warps 12-15 look-back group, one thread per TMEM lane.
// TMEM (512 columns): scores [0,128) -- overwritten by the bf16 P matrix (two keys per
// column, the A operand of P V) --, O (two buffers when dv <= 96), and two buffers
// that each hold an item's segment aggregate, then its incoming state, then its
// running state.  A stage is released in two parts: its log-gate, q and k tiles once
// the K^T V MMAs complete (the next job's loads into them start while P V still runs),
// its v tile once P V completes.
//
// Chunks follow the direction's base order (raster rows, or grid columns for T->B /
// B->T) and are always cut in forward order; reversed scans visit them backwards and
// walk each chunk's rows backwards.  A chunk is: 128
// consecutive raster positions; 128/Hgrid whole columns when Hgrid divides 128;
// otherwise one column cut into pieces of at most 128 rows.  Rows past the grid are
// zero-filled by the TMA and contribute nothing.  The operand tiles arrive as 16-channel
// 32-byte-swizzled atoms; raster scans load all full atoms of a tile with one box.
// All gate sums are kept in log2 units (times log2 e), so a gate is one ex2.
#include <math.h>
#include <string.h>

#include <cuda.h>

#include "dev_common.cuh"
#include "internal.h"

namespace dig {

namespace {

constexpr int MC = kChunkTC;
constexpr int NT = 512;
constexpr int kWarpProd = 0, kWarpMma = 1, kWarpSuf = 2, kWarpGate = 4, kWarpEpi = 8, kWarpLb = 12;
constexpr uint32_t ATOM32 = MC * 32u;    // one 16-channel block of a 32B-swizzled 128-row tile
constexpr float kMaxGateRange = 80.0f;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kMaxGateRange2 = kMaxGateRange * kLog2e;  // the same bound on log2-scaled sums
constexpr uint32_t kColS = 0;
constexpr uint32_t kLayoutSW32 = 6;
constexpr int kMaxStages = 2;

// mbarrier indices (8 bytes each)
enum {
  kBarFull = 0,                       // [S]  log-gate tile landed (or an end-of-stream job posted)
  kBarOps = kBarFull + kMaxStages,    // [S]  q, k tiles landed
  kBarOpsV = kBarOps + kMaxStages,    // [S]  v tile landed
  kBarSufDone = kBarOpsV + kMaxStages, // [S]  suffix sums and quarter offsets done (64 arrivals)
  kBarGate = kBarSufDone + kMaxStages,  // [S]  gates applied (128 arrivals)
  kBarEmpty = kBarGate + kMaxStages,  // [S]  log-gate, q, k tiles free (MMA commit, or the serial path)
  kBarEmptyV = kBarEmpty + kMaxStages, // [S] v tile free
  kBarMail = kBarEmptyV + kMaxStages, // pass-2 job handed to the output group
  kBarScFull,                         // score MMA done
  kBarScEmpty,                        // pass-2 job taken by the output group (128 arrivals)
  kBarPReady,                         // P written by the gate warps (128 arrivals)
  kBarGReady,                         // state scaled and G written (128 arrivals)
  kBarBatch,                          // [2] output and state MMAs done, per O buffer
  kBarOFree = kBarBatch + 2,          // [2] O buffer read (128 arrivals)
  kBarSegDone = kBarOFree + 2,        // [3] pass-1 MMAs of an item done (or end of stream)
  kBarSinReady = kBarSegDone + 3,     // [3] look-back done: incoming state in the buffer
  kBarSegFree = kBarSinReady + 3,     // [3] pass 2 done with the buffer
  kBarDrain = kBarSegFree + 3,        // all MMAs of the CTA done (teardown)
  kNumBars
};

// Jobs posted by the producer, one per stage use.
enum { kJobP1 = 1, kJobP2 = 2, kJobEnd = 3 };

struct WsArgs {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const float* la;
  const __nv_bfloat16* glog;  // gate logits [B][T][H][dk] when set: log_alpha = logsigmoid(g) / gate_norm
  float inv_gate_norm;        // 1 / gate_norm
  __nv_bfloat16* out;
  float* agg_S;   // [BH][NS][dv/4][dk][4]  segment aggregates (quads of value columns)
  float* agg_g;   // [BH][NS][dk]           exp(segment log-gate sums)
  float* incl_S;  // [BH][NS][dv/4][dk][4]  state after the segment
  int* flags;     // [BH][NS]               0 nothing, 1 aggregate, 2 inclusive
  int* ticket;
  int H, BH, dk, dv, NC, NS, G, items;
  int skip;  // items left out (test hook; 0 normally)
  int Kp, Np, nstage, nO, nbuf;
  int nak, nav;  // full 16-channel atoms of q/k and v loaded by one box each (raster scans; else 0)
  uint32_t colO0, colO1, colSeg0, colSeg1, colSeg2;
  int mode, rpc, ppr;  // chunk geometry: 0 raster, 1 whole columns (rpc per chunk), 2 column pieces (ppr per column)
  uint32_t stage_bytes, oK, oV, oQ, oLA, oG, oBL, oWide, oGam, oRed, oTot, oOff, oMisc, oJob, oMail, oItem, oBar, oTm;
  ScanGeom g;
  __device__ __forceinline__ uint32_t col_seg(int buf) const {
    return buf == 0 ? colSeg0 : (buf == 1 ? colSeg1 : colSeg2);
  }
  __device__ __forceinline__ uint32_t col_o(int ob) const { return ob ? colO1 : colO0; }
};

// One work item: a segment of G chunks of one (batch, head).
struct Item {
  int seg, bh, b, h, c0, n;
  int64_t seg_id;
};
__device__ __forceinline__ Item decode_item(const WsArgs& a, int item) {
  Item it;
  it.seg = item / a.BH;
  it.bh = item - it.seg * a.BH;
  it.b = it.bh / a.H;
  it.h = it.bh - it.b * a.H;
  it.c0 = it.seg * a.G;
  it.n = min(a.G, a.NC - it.c0);
  it.seg_id = (int64_t)it.bh * a.NS + it.seg;
  return it;
}

struct TensorMaps {
  CUtensorMap q, k, v, la;  // operand tiles (16-channel boxes, 32-byte swizzle) and log-gate tiles
  // Raster scans: all full 16-channel atoms of an operand tile in one box (the
  // channel atoms are a box dimension); the rest, if any, come from q, k, v.
  CUtensorMap qa, ka, va;
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
// Group-wide OR over a named barrier.
__device__ __forceinline__ bool group_or(uint32_t id, uint32_t n, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
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
// 2^x (hardware approximation); the gate sums are kept in log2 units.
__device__ __forceinline__ float exp2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float lg2_approx(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// log2(alpha) for a gate logit g: logsigmoid(g) / gate_norm in log2 units,
//   logsigmoid(g) = min(g, 0) - ln(1 + e^{-|g|}),
// so log2 alpha = (min(g, 0) log2 e - log2(1 + 2^{-|g| log2 e})) / gate_norm; the
// exponential never exceeds 1.
__device__ __forceinline__ float log2_gate(float g, float inv_norm) {
  return (fminf(g, 0.f) * kLog2e - lg2_approx(1.f + exp2_approx(-fabsf(g) * kLog2e))) * inv_norm;
}

// Lane-wise product of two packed bf16 pairs, rounded to bf16.
__device__ __forceinline__ uint32_t mul_bf16x2(uint32_t x, uint32_t y) {
  __nv_bfloat162 r = __hmul2(*reinterpret_cast<__nv_bfloat162*>(&x), *reinterpret_cast<__nv_bfloat162*>(&y));
  return *reinterpret_cast<uint32_t*>(&r);
}
__device__ __forceinline__ uint32_t pack_u2(uint32_t x, uint32_t y) {
  return pack_bf16x2(__uint_as_float(x), __uint_as_float(y));
}

// TMA tile load with an L2 eviction-priority policy (from createpolicy).
__device__ __forceinline__ void tma_load_5d(uint32_t dst, const CUtensorMap* map, int c0, int c1, int c2, int c3,
                                            int c4, uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1, {%2, %3, "
      "%4, %5, %6}], [%7], %8;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4), "r"(bar), "l"(policy)
      : "memory");
}
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
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

// Rows of forward chunk cf's tile that hold tokens: always a prefix [0, n) of the tile
// (the end of the sequence, the columns past Wg, or the end of a column piece).
__device__ __forceinline__ int chunk_valid_rows(const WsArgs& a, int cf) {
  int n;
  if (a.mode == 0) {
    n = a.g.T - cf * MC;
  } else if (a.mode == 1) {
    n = (a.g.Wg - cf * a.rpc) * a.g.Hg;
  } else {
    const int x = cf / a.ppr;
    n = a.g.Hg - (cf - x * a.ppr) * MC;
  }
  return n < MC ? n : MC;
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

// ---------------------------------------------------------------------------
// Producer
// ---------------------------------------------------------------------------
// The log-gate tile is issued first, on its own barrier, so that the suffix sums can
// start while the operand tiles are still arriving.
__device__ void tma_job(const WsArgs& a, const TensorMaps& tm, uint32_t st, uint32_t bar_la, uint32_t bar_ops, int cf,
                        bool with_q, int b, int h) {
  int y, x;
  chunk_box(a, cf, y, x);
  // Pass 1 marks its tiles' lines evict-last: pass 2 reads them again about one item
  // later.  Pass 2 is the last use of every tile and marks its lines first to go.
  const uint64_t pol = with_q ? l2_policy_evict_first() : l2_policy_evict_last();
  mbar_expect_tx(bar_la, (uint32_t)MC * (uint32_t)(a.dk + 4) * 4u);
  tma_load_5d(st + a.oLA, &tm.la, 0, h, y, x, b, bar_la, pol);
  mbar_expect_tx(bar_ops, (uint32_t)(with_q ? 2 : 1) * (uint32_t)a.Kp * 256u);
  if (a.nak) {  // (channel, row, atom, head, batch)
    tma_load_5d(st + a.oK, &tm.ka, 0, y, 0, h, b, bar_ops, pol);
    if (with_q) tma_load_5d(st + a.oQ, &tm.qa, 0, y, 0, h, b, bar_ops, pol);
  }
  for (int cb = a.nak; cb < (a.Kp >> 4); ++cb) {
    tma_load_5d(st + a.oK + (uint32_t)cb * ATOM32, &tm.k, cb * 16, h, y, x, b, bar_ops, pol);
    if (with_q) tma_load_5d(st + a.oQ + (uint32_t)cb * ATOM32, &tm.q, cb * 16, h, y, x, b, bar_ops, pol);
  }
}
// The chunk's v tile (its own barrier: the v part of a stage is released last).
__device__ void tma_job_v(const WsArgs& a, const TensorMaps& tm, uint32_t st, uint32_t bar_v, int cf, bool pass2,
                          int b, int h) {
  int y, x;
  chunk_box(a, cf, y, x);
  const uint64_t pol = pass2 ? l2_policy_evict_first() : l2_policy_evict_last();
  mbar_expect_tx(bar_v, (uint32_t)a.Np * 256u);
  if (a.nav) tma_load_5d(st + a.oV, &tm.va, 0, y, 0, h, b, bar_v, pol);
  for (int cb = a.nav; cb < (a.Np >> 4); ++cb)
    tma_load_5d(st + a.oV + (uint32_t)cb * ATOM32, &tm.v, cb * 16, h, y, x, b, bar_v, pol);
}

// ---------------------------------------------------------------------------
// Serial path (wide chunks), run by the 128 TMEM-side threads: lane i owns state
// row i; 16 value columns at a time, outputs reduced over lanes with shuffles.
// The stage's q, k tiles may already be gated, so raw q, k come from global memory.
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
    // alpha, k and q of the next row are fetched one step ahead.
    auto fetch = [&](int step, float& al, float& kq, float& qi) -> int {
      const int r = a.g.reverse ? (MC - 1 - step) : step;
      const int t = row_token(a, cf, r);
      al = 1.f;
      kq = 0.f;
      qi = 0.f;
      if (t >= 0 && i < a.dk) {
        const int64_t o = (((int64_t)b * a.g.T + t) * a.H + h) * a.dk + i;
        if (a.glog) {
          const float gg = __bfloat162float(a.glog[o]);
          al = expf((fminf(gg, 0.f) - log1pf(expf(-fabsf(gg)))) * a.inv_gate_norm);
        } else {
          al = __expf(__ldg(a.la + o));
        }
        kq = __bfloat162float(a.k[o]);
        qi = __bfloat162float(a.q[o]);
      }
      return t;
    };
    float n_al, n_kq, n_qi;
    int n_t = fetch(0, n_al, n_kq, n_qi);
    for (int step = 0; step < MC; ++step) {
      const int r = a.g.reverse ? (MC - 1 - step) : step;
      const int t = n_t;
      const float alpha = n_al, kq = n_kq, qi = n_qi;
      if (step + 1 < MC) n_t = fetch(step + 1, n_al, n_kq, n_qi);
      if (t < 0) continue;  // padding row: uniform
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

// Adds coef * src[pid] (an aggregate or inclusive state in the quad layout) to the
// state rows this thread owns in TMEM (tSt), 32 columns per global round trip; also
// returns coef * gamma[pid] when want_gam (the coefficient for the next predecessor).
__device__ __forceinline__ float fold_state(const WsArgs& a, const float* src, int64_t pid, float coef, uint32_t tSt,
                                            int i, bool want_gam) {
  const int DQ = a.dv >> 2;
  const float g = (want_gam && i < a.dk) ? __ldcg(a.agg_g + pid * a.dk + i) : 1.f;
#pragma unroll 1
  for (int c0 = 0; c0 < a.Np; c0 += 32) {
    float4 x[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int jq = c0 / 4 + q;
      x[q] = (i < a.dk && jq < DQ) ? __ldcg(reinterpret_cast<const float4*>(src + ((pid * DQ + jq) * a.dk + i) * 4))
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int c4 = 0; c4 < 2; ++c4) {
      const int cb = c0 + 16 * c4;
      if (cb < a.Np) {
        uint32_t t[1][16];
        tmem_ld_cols<1>(tSt + (uint32_t)cb, 16, t);
        float t16[16];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          t16[4 * q] = fmaf(coef, x[4 * c4 + q].x, __uint_as_float(t[0][4 * q]));
          t16[4 * q + 1] = fmaf(coef, x[4 * c4 + q].y, __uint_as_float(t[0][4 * q + 1]));
          t16[4 * q + 2] = fmaf(coef, x[4 * c4 + q].z, __uint_as_float(t[0][4 * q + 2]));
          t16[4 * q + 3] = fmaf(coef, x[4 * c4 + q].w, __uint_as_float(t[0][4 * q + 3]));
        }
        tmem_st16(tSt + (uint32_t)cb, t16);
      }
    }
  }
  tmem_st_wait();
  return coef * g;
}

// Look-back of one item, run by the 128 look-back threads (lane i = key channel).
// tSeg holds the item's segment aggregate when called and its incoming state on
// return.  Steps: publish the aggregate and exp(segment gate sum) (flag 1); fold
// earlier segments of the same head, nearest first, into the incoming state until an
// inclusive state is found (decoupled look-back); publish this segment's inclusive
// state Diag(gamma_seg) S_in + aggregate (flag 2), handing S_in to pass 2 (sin_item,
// bar_sin) just before that flag's fence.  Predecessor flags are read 32 at a time by
// one warp; sLb is a small shared scratch.
__device__ __forceinline__ void lookback(const WsArgs& a, int seg, int bh, int64_t seg_id, uint32_t tSeg, int i, int e,
                                         float gs, volatile int* sLb, uint32_t bar_sin, volatile int* sin_item,
                                         int item) {
  const int DQ = a.dv >> 2;
  const int lane = e & 31;
  if (i < a.dk) a.agg_g[seg_id * a.dk + i] = gs;
#pragma unroll 1
  for (int c0 = 0; c0 < a.Np; c0 += 32) {
    uint32_t t[2][16];
    tmem_ld_cols<2>(tSeg + (uint32_t)c0, a.Np - c0, t);
    if (i < a.dk) {
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int jq = c0 / 4 + q;
        if (jq < DQ)
          *reinterpret_cast<float4*>(a.agg_S + ((seg_id * DQ + jq) * a.dk + i) * 4) =
              make_float4(__uint_as_float(t[q >> 2][4 * (q & 3)]), __uint_as_float(t[q >> 2][4 * (q & 3) + 1]),
                          __uint_as_float(t[q >> 2][4 * (q & 3) + 2]), __uint_as_float(t[q >> 2][4 * (q & 3) + 3]));
      }
    }
    // The columns now accumulate the incoming state.
    float z[16];
#pragma unroll
    for (int q = 0; q < 16; ++q) z[q] = 0.f;
    tmem_st16(tSeg + (uint32_t)c0, z);
    if (c0 + 16 < a.Np) tmem_st16(tSeg + (uint32_t)(c0 + 16), z);
  }
  tmem_st_wait();
  named_sync(3, 128);
  // The flag is released by a thread of the last warp: the first warp scans the
  // predecessors' flags meanwhile, without waiting for this fence.
  if (e == 127) {
    __threadfence();
    st_release(a.flags + seg_id, 1);
  }
  float coef = 1.f;
  int base = seg - 1;  // nearest predecessor not folded yet
  while (base >= 0) {
    if (e < 32) {
      // Wait until the window [base-31, base] shows an inclusive state (or the start of
      // the sequence) with aggregates everywhere before it, or 32 aggregates.
      int nagg = -1, incl = 0;
      const long long t0 = clock64();
      for (;;) {
        const int p = base - lane;
        const int fl = p >= 0 ? (int)ld_acquire(a.flags + (int64_t)bh * a.NS + p) : 2;
        const uint32_t m2 = __ballot_sync(0xffffffffu, fl == 2);
        const uint32_t m0 = __ballot_sync(0xffffffffu, fl == 0);
        const int first2 = m2 ? __ffs(m2) - 1 : 32;
        const uint32_t before = first2 == 32 ? 0xffffffffu : ((1u << first2) - 1u);
        if ((m0 & before) == 0) {
          nagg = first2;
          incl = first2 < 32 && base - first2 >= 0;
          break;
        }
        if (clock64() - t0 > kWaitCycles) {
          if (lane == 0) report_status(GLA_ERR_TIMEOUT);
          break;
        }
        __nanosleep(32);
      }
      if (lane == 0) {
        sLb[0] = nagg;
        sLb[1] = incl;
      }
    }
    named_sync(3, 128);
    const int nagg = sLb[0], incl = sLb[1];
    named_sync(3, 128);
    if (nagg < 0) break;  // timed out (recorded)
    for (int m = 0; m < nagg; ++m) {
      const int64_t pid = (int64_t)bh * a.NS + base - m;
      coef = fold_state(a, a.agg_S, pid, coef, tSeg, i, true);
    }
    if (incl) {
      fold_state(a, a.incl_S, (int64_t)bh * a.NS + base - nagg, coef, tSeg, i, false);
      break;
    }
    base -= nagg;
  }
  // Inclusive state of this segment: Diag(gamma_seg) S_in + aggregate (re-read from
  // the copy this thread published above).
#pragma unroll 1
  for (int c0 = 0; c0 < a.Np; c0 += 32) {
    float4 g[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int jq = c0 / 4 + q;
      g[q] = (i < a.dk && jq < DQ) ? __ldcg(reinterpret_cast<const float4*>(a.agg_S + ((seg_id * DQ + jq) * a.dk + i) * 4))
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    uint32_t sin[2][16];
    tmem_ld_cols<2>(tSeg + (uint32_t)c0, a.Np - c0, sin);
    if (i < a.dk) {
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int jq = c0 / 4 + q;
        if (jq < DQ) {
          const uint32_t* v = &sin[q >> 2][4 * (q & 3)];
          *reinterpret_cast<float4*>(a.incl_S + ((seg_id * DQ + jq) * a.dk + i) * 4) =
              make_float4(fmaf(gs, __uint_as_float(v[0]), g[q].x), fmaf(gs, __uint_as_float(v[1]), g[q].y),
                          fmaf(gs, __uint_as_float(v[2]), g[q].z), fmaf(gs, __uint_as_float(v[3]), g[q].w));
        }
      }
    }
  }
  tc_fence_before();
  named_sync(3, 128);
  if (e == 0) {
    // TMEM is no longer read here: pass 2 may take the incoming state now.
    *sin_item = item;
    mbar_arrive(bar_sin);
    __threadfence();
    st_release(a.flags + seg_id, 2);
  }
}

__device__ __forceinline__ uint32_t align1024(uint32_t x) { return (x + 1023u) & ~1023u; }

// ---------------------------------------------------------------------------
// The kernel (persistent: each CTA takes items from a ticket counter until none
// are left).  The producer posts, per item, its pass-1 jobs and then the pass-2
// jobs of the previous item; the look-back group works on an item while pass 1 of
// the next one and pass 2 of the previous one proceed.  Item k uses aggregate buffer
// k % 2, which holds its aggregate after pass 1, its incoming state after the
// look-back and its running state during pass 2.
// ---------------------------------------------------------------------------
// kGlogit: the gates arrive as bf16 logits (a.glog) and the suffix warps turn them into
// log2 gates; a separate instance so that the fp32-gate kernel carries none of that code.
template <bool kGlogit>
__global__ void __launch_bounds__(NT, 1) gla_ws_fwd(const __grid_constant__ WsArgs a, const __grid_constant__ TensorMaps tm) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t sbase = align1024(raw_u32);
  uint8_t* smem = smem_raw + (sbase - raw_u32);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  float* sBL = reinterpret_cast<float*>(smem + a.oBL);      // [S][128] chunk gate sums
  volatile int* sWide = reinterpret_cast<volatile int*>(smem + a.oWide);  // [S] chunk evaluated serially
  float* sGam = reinterpret_cast<float*>(smem + a.oGam);    // [3][128] exp(segment gate sum)
  float* red = reinterpret_cast<float*>(smem + a.oRed);     // serial-path reduction [4][16]
  float* sTot = reinterpret_cast<float*>(smem + a.oTot);    // [4][128] log-gate sums of the row quarters
  float* sOff = reinterpret_cast<float*>(smem + a.oOff);    // [S][4][128] log-gate sums after each quarter
  // [0] first item [1] abort [3] jobs posted [5] end item index [6..7] look-back scan result
  volatile int* sMisc = reinterpret_cast<volatile int*>(smem + a.oMisc);
  volatile int* sJob = reinterpret_cast<volatile int*>(smem + a.oJob);    // [S][4] kind, item, j, buf
  volatile int* sMail = reinterpret_cast<volatile int*>(smem + a.oMail);  // [4]    stage, wide, item, j
  volatile int* sItem = reinterpret_cast<volatile int*>(smem + a.oItem);  // [3] item per buffer, [3] same for pass 2
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
      mbar_init(BAR(kBarOps + s), 1);
      mbar_init(BAR(kBarOpsV + s), 1);
      mbar_init(BAR(kBarEmptyV + s), 1);
      mbar_init(BAR(kBarSufDone + s), 64);
      mbar_init(BAR(kBarGate + s), 128);
      mbar_init(BAR(kBarEmpty + s), 1);
    }
    mbar_init(BAR(kBarMail), 1);
    mbar_init(BAR(kBarScFull), 1);
    mbar_init(BAR(kBarScEmpty), 128);
    mbar_init(BAR(kBarPReady), 128);
    mbar_init(BAR(kBarGReady), 128);
    for (int q = 0; q < 2; ++q) {
      mbar_init(BAR(kBarBatch + q), 1);
      mbar_init(BAR(kBarOFree + q), 128);
    }
    for (int q = 0; q < 3; ++q) {
      mbar_init(BAR(kBarSegDone + q), 1);
      mbar_init(BAR(kBarSinReady + q), 1);
      mbar_init(BAR(kBarSegFree + q), 1);
    }
    mbar_init(BAR(kBarDrain), 1);
    fence_mbar_init();
    sMisc[0] = atomicAdd(a.ticket, 1) + a.skip;
    sMisc[1] = 0;
    sMisc[3] = 0;
    sMisc[4] = 0;
    sMisc[5] = 0x7fffffff;
  }
  for (int x = tid; x < kMaxStages * 128; x += NT) sBL[x] = 0.f;  // rows >= dk: gamma = 1
  for (int x = tid; x < 3 * 128; x += NT) sGam[x] = 1.f;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *reinterpret_cast<volatile uint32_t*>(smem + a.oTm);
  const int S = a.nstage;
  const bool has_work = sMisc[0] < a.items;

  if (!has_work) {
    // every ticket was taken by earlier CTAs
  } else if (warp == kWarpProd) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      // Warm the TMA descriptor cache with every tensor map this kernel loads through.
      const CUtensorMap* maps[7] = {&tm.la, &tm.k, &tm.q, &tm.v, &tm.ka, &tm.qa, &tm.va};
#pragma unroll
      for (int m = 0; m < 7; ++m)
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(maps[m])) : "memory");
      int jc = 0;
      auto post = [&](int kind, int item, int j, int buf) -> bool {
        const int s = jc % S, use = jc / S;
        if (use > 0 && !wait_bar(BAR(kBarEmpty + s), (uint32_t)((use - 1) & 1), abort_flag)) return false;
        sJob[4 * s] = kind;
        sJob[4 * s + 1] = item;
        sJob[4 * s + 2] = j;
        sJob[4 * s + 3] = buf;
        if (kind == kJobEnd) {
          mbar_arrive(BAR(kBarFull + s));
          mbar_arrive(BAR(kBarOps + s));
          mbar_arrive(BAR(kBarOpsV + s));
          sMisc[3] = jc + 1;
        } else {
          const Item it = decode_item(a, item);
          const int c = kind == kJobP1 ? it.c0 + it.n - 1 - j : it.c0 + j;  // pass 1 walks backwards
          tma_job(a, tm, sbase + (uint32_t)s * a.stage_bytes, BAR(kBarFull + s), BAR(kBarOps + s), fwd_chunk(a, c),
                  kind == kJobP2, it.b, it.h);
          sMisc[3] = jc + 1;  // log-gate, q, k loads of this job issued
          if (use > 0 && !wait_bar(BAR(kBarEmptyV + s), (uint32_t)((use - 1) & 1), abort_flag)) return false;
          tma_job_v(a, tm, sbase + (uint32_t)s * a.stage_bytes, BAR(kBarOpsV + s), fwd_chunk(a, c), kind == kJobP2,
                    it.b, it.h);
        }
        sMisc[4] = ++jc;  // v load issued too
        return true;
      };
      auto post_p1 = [&](int item, int k) -> bool {
        const int buf = k % a.nbuf;
        // sItem[buf] is rewritten once the look-back of item k - nbuf has read it.
        if (k >= a.nbuf && !wait_bar(BAR(kBarSinReady + buf), (uint32_t)(((k / a.nbuf) - 1) & 1), abort_flag))
          return false;
        sItem[buf] = item;
        const int n = decode_item(a, item).n;
        for (int j = 0; j < n; ++j)
          if (!post(kJobP1, item, j, buf)) return false;
        return true;
      };
      auto post_p2 = [&](int item, int k) -> bool {
        const int n = decode_item(a, item).n;
        for (int j = 0; j < n; ++j)
          if (!post(kJobP2, item, j, k % a.nbuf)) return false;
        return true;
      };
      // Pass 1 runs nbuf - 1 items ahead of pass 2.
      int ring[4];
      int have = 0;  // items claimed (their pass 1 posted)
      bool ok = true, more = true;
      auto claim = [&]() {
        const int t = have == 0 ? sMisc[0] : atomicAdd(a.ticket, 1) + a.skip;
        if (t >= a.items) {
          more = false;
          return;
        }
        ring[have & 3] = t;
        ok = post_p1(t, have);
        ++have;
      };
      claim();
      for (int l = 1; l < a.nbuf - 1 && ok && more; ++l) claim();
      for (int k = 0; ok && k < have; ++k) {
        if (more) claim();
        if (ok) ok = post_p2(ring[k & 3], k);
      }
      if (ok) post(kJobEnd, -1, 0, 0);
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    // Pass-2 order per chunk: S, then Q~ G and K^T V (while the gate warps mask S into
    // P), then P V; the stage's q/k/log-gate part is released after K^T V, its v part
    // after P V.
    if (lane == 0) {
      int kb = 0, jb = 0, km = 0;  // non-serial pass-2 jobs, pass-2 jobs, items through pass 1
      bool ok = true;
      // Operand descriptors of stage 0 (stage s: + s * dstage); a K step adds a constant
      // to the start-address field.  Loops are unrolled to their maximum trip count so
      // that each MMA costs little more than its issue.
      const uint64_t dQ = desc_sw32(sbase + a.oQ, 16u, 256u);      // K-major, step ATOM32
      const uint64_t dK = desc_sw32(sbase + a.oK, 16u, 256u);      // K-major, step ATOM32
      const uint64_t dKt = desc_sw32(sbase + a.oK, ATOM32, 256u);  // MN-major (K^ transposed), step 512 B
      const uint64_t dV = desc_sw32(sbase + a.oV, ATOM32, 256u);   // MN-major, step 512 B
      const uint64_t dG = desc_sw32(sbase + a.oG, (uint32_t)a.Kp * 32u, 256u);
      const uint64_t dstage = (uint64_t)(a.stage_bytes >> 4);
      constexpr uint64_t kStepK = ATOM32 >> 4, kStepMN = 512u >> 4;
      const int nk = a.Kp >> 4;
      const uint32_t id_s = idesc_bf16_f32(MC, MC, false, false);
      const uint32_t id_pv = idesc_bf16_f32(MC, a.Np, false, true);
      const uint32_t id_kv = idesc_bf16_f32(MC, a.Np, true, true);
      for (int jc = 0; ok; ++jc) {
        const int s = jc % S, use = jc / S;
        if (!wait_bar(BAR(kBarGate + s), (uint32_t)(use & 1), abort_flag)) break;
        tc_fence_after();
        const int kind = sJob[4 * s], item = sJob[4 * s + 1], j = sJob[4 * s + 2], buf = sJob[4 * s + 3];
        if (kind == kJobEnd) {
          sMisc[5] = km;  // the look-back and output groups stop at item km
          mbar_arrive(BAR(kBarSegDone + km % a.nbuf));
          break;
        }
        const uint64_t so = (uint64_t)s * dstage;
        const uint32_t tS = tbase + a.col_seg(buf);
        if (kind == kJobP1) {
          // The buffer is free once pass 2 of item km - 2 is done with it.
          if (j == 0 && km >= a.nbuf &&
              !wait_bar(BAR(kBarSegFree + buf), (uint32_t)(((km / a.nbuf) - 1) & 1), abort_flag))
            break;
          if (!wait_bar(BAR(kBarOpsV + s), (uint32_t)(use & 1), abort_flag)) break;
          tc_fence_after();
          umma_ss(tS, dKt + so, dV + so, id_kv, j > 0 ? 1u : 0u);
#pragma unroll
          for (int kk = 1; kk < MC / 16; ++kk) umma_ss(tS, dKt + so + kk * kStepMN, dV + so + kk * kStepMN, id_kv, 1u);
          umma_commit(BAR(kBarEmpty + s));
          umma_commit(BAR(kBarEmptyV + s));
          if (j == decode_item(a, item).n - 1) {
            umma_commit(BAR(kBarSegDone + buf));
            ++km;
          }
          continue;
        }
        // pass 2: hand the job to the output group once it has taken the previous one
        if (jb > 0 && !wait_bar(BAR(kBarScEmpty), (uint32_t)((jb - 1) & 1), abort_flag)) break;
        tc_fence_after();
        const int wide = sWide[s];
        sMail[0] = s;
        sMail[1] = wide | ((use & 1) << 1);  // + the stage use's parity (v barrier)
        sMail[2] = item;
        sMail[3] = j;
        mbar_arrive(BAR(kBarMail));
        ++jb;
        if (wide) continue;  // evaluated serially by the output group, which frees the stage
        // The score columns still hold the previous chunk's P, the TMEM A operand of its
        // P V, and S overwrites them: a later MMA's writes are not ordered after an
        // earlier MMA's operand reads, so S waits for that P V to complete.
        if (kb > 0 &&
            !wait_bar(BAR(kBarBatch + (kb - 1) % a.nO), (uint32_t)(((kb - 1) / a.nO) & 1), abort_flag))
          break;
        tc_fence_after();
        // S = Q~ K^T (masked into P by the gate warps meanwhile)
        umma_ss(tbase + kColS, dQ + so, dK + so, id_s, 0u);
#pragma unroll
        for (int kk = 1; kk < 8; ++kk)
          if (kk < nk) umma_ss(tbase + kColS, dQ + so + kk * kStepK, dK + so + kk * kStepK, id_s, 1u);
        umma_commit(BAR(kBarScFull));
        // O = Q~ G and S += K^T V once the output group has scaled the state into G,
        // then O += P V: the stage is free when these complete.
        const int ob = kb % a.nO;
        if (!wait_bar(BAR(kBarGReady), (uint32_t)(kb & 1), abort_flag)) break;
        if (kb >= a.nO && !wait_bar(BAR(kBarOFree + ob), (uint32_t)(((kb / a.nO) - 1) & 1), abort_flag)) break;
        tc_fence_after();
        const uint32_t tO = tbase + a.col_o(ob);
        umma_ss(tO, dQ + so, dG, id_pv, 0u);
#pragma unroll
        for (int kk = 1; kk < 8; ++kk)
          if (kk < nk) umma_ss(tO, dQ + so + kk * kStepK, dG + kk * kStepMN, id_pv, 1u);
#pragma unroll
        if (!wait_bar(BAR(kBarOpsV + s), (uint32_t)(use & 1), abort_flag)) break;
        tc_fence_after();
        for (int kk = 0; kk < MC / 16; ++kk) umma_ss(tS, dKt + so + kk * kStepMN, dV + so + kk * kStepMN, id_kv, 1u);
        umma_commit(BAR(kBarEmpty + s));  // q, k and the log-gate tile are no longer read
        if (!wait_bar(BAR(kBarPReady), (uint32_t)(kb & 1), abort_flag)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < MC / 16; ++kk)  // P is bf16 in the score columns
          umma_ts(tO, tbase + kColS + (uint32_t)(kk * 8), dV + so + kk * kStepMN, id_pv, 1u);
        umma_commit(BAR(kBarBatch + ob));
        umma_commit(BAR(kBarEmptyV + s));
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
    // Warp sw walks row quarters 2sw and 2sw+1 of every chunk; lane = pair of key
    // channels (lanes 0..3 also take pairs 32..35 and beyond).  Per quarter: exclusive
    // suffix sums of the log-gates over its 32 rows in scan order, in place; the
    // quarter totals go to sTot.  All gate sums from here on are in log2 units (times
    // log2 e).  After the pair barrier each warp turns them into the
    // offsets of its quarters (totals of the later quarters, + the later chunks of the
    // segment in pass 1), so that the gate warps add one offset per channel.
    const int sw = warp - kWarpSuf;
    const int pw = a.dk + 4;         // log-gate row pitch in floats
    const int np = (a.dk + 1) >> 1;  // key-channel pairs
    const bool act0 = lane < np, act1 = lane + 32 < np;
    float2 cy0 = make_float2(0.f, 0.f), cy1 = cy0;  // pass 1: later chunks of the segment
    int ks = 0;                                     // items through pass 1
    for (int jc = 0;; ++jc) {
      const int s = jc % S, use = jc / S;
      if (!group_and(1, 64, wait_bar(BAR(kBarFull + s), (uint32_t)(use & 1), abort_flag))) break;
      const int kind = sJob[4 * s];
      if (kind == kJobEnd) {
        mbar_arrive(BAR(kBarSufDone + s));
        break;
      }
      const int j = sJob[4 * s + 2], buf = sJob[4 * s + 3];
      const bool pass1 = kind == kJobP1;
      const bool last1 = pass1 && j == decode_item(a, sJob[4 * s + 1]).n - 1;
      // sGam[buf] is rewritten once the look-back of item ks - nbuf has read it.
      if (last1 && ks >= a.nbuf &&
          !group_and(1, 64, wait_bar(BAR(kBarSinReady + buf), (uint32_t)(((ks / a.nbuf) - 1) & 1), abort_flag)))
        break;
      if (pass1 && j == 0) cy0 = cy1 = make_float2(0.f, 0.f);
      float* lag = reinterpret_cast<float*>(smem + (uint32_t)s * a.stage_bytes + a.oLA);
      {
        // The two quarters' walks are interleaved (independent chains).
        const int dr = a.g.reverse ? (pw >> 1) : -(pw >> 1);  // in float2
        float2* pa = reinterpret_cast<float2*>(lag + (a.g.reverse ? 64 * sw : 64 * sw + 31) * pw) + lane;
        float2* pb = pa + 16 * pw;  // the other quarter: 32 rows on
        // Gate logits arrive as bf16 at the start of each fp32 row (the box is padded to
        // the row pitch), one packed pair per lane: a row's logits are read before the
        // same row's sums overwrite them, and rows never overlap.
        const uint32_t* ua =
            reinterpret_cast<const uint32_t*>(lag + (a.g.reverse ? 64 * sw : 64 * sw + 31) * pw) + lane;
        const uint32_t* ub = ua + 32 * pw;  // the other quarter: 32 rows on
        const int du = 2 * dr;  // 4-byte words per row step
        const float mul = kGlogit ? 1.f : kLog2e;  // logits are converted straight to log2 units
        // Rows past the chunk's tokens hold the box's zero fill: a zero logit is not a
        // neutral gate (logsigmoid(0) < 0), so those rows get gate 0 explicitly.
        int nvalid = MC;
        if (kGlogit) {
          const Item itj = decode_item(a, sJob[4 * s + 1]);
          const int cj = pass1 ? itj.c0 + itj.n - 1 - j : itj.c0 + j;  // pass 1 walks its chunks backwards
          nvalid = chunk_valid_rows(a, fwd_chunk(a, cj));
        }
        const int row_a0 = a.g.reverse ? 64 * sw : 64 * sw + 31, row_step = a.g.reverse ? 1 : -1;
        auto gate2 = [&](uint32_t w) {
          const float2 g = unpack_bf16x2(w);
          return make_float2(log2_gate(g.x, a.inv_gate_norm), log2_gate(g.y, a.inv_gate_norm));
        };
        float2 a0 = make_float2(0.f, 0.f), a1 = a0, b0 = a0, b1 = a0;
#pragma unroll 1
        for (int h8 = 0; h8 < 4; ++h8) {
          float2 xa[8], xb[8], ya[8], yb[8];
          if (kGlogit) {
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const float2 z = make_float2(0.f, 0.f);
              const int ra = row_a0 + row_step * (8 * h8 + q);  // row of quarter a; quarter b is 32 on
              const bool va = ra < nvalid, vb = ra + 32 < nvalid;
              xa[q] = act0 && va ? gate2(ua[q * du]) : z;
              xb[q] = act0 && vb ? gate2(ub[q * du]) : z;
              ya[q] = act1 && va ? gate2(ua[q * du + 32]) : z;
              yb[q] = act1 && vb ? gate2(ub[q * du + 32]) : z;
            }
            ua += 8 * du;
            ub += 8 * du;
          } else {
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              xa[q] = act0 ? pa[q * dr] : make_float2(0.f, 0.f);
              xb[q] = act0 ? pb[q * dr] : make_float2(0.f, 0.f);
              ya[q] = act1 ? pa[q * dr + 32] : make_float2(0.f, 0.f);
              yb[q] = act1 ? pb[q * dr + 32] : make_float2(0.f, 0.f);
            }
          }
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            if (act0) {
              pa[q * dr] = a0;
              pb[q * dr] = b0;
            }
            if (act1) {
              pa[q * dr + 32] = a1;
              pb[q * dr + 32] = b1;
            }
            a0.x = fmaf(xa[q].x, mul, a0.x);
            a0.y = fmaf(xa[q].y, mul, a0.y);
            b0.x = fmaf(xb[q].x, mul, b0.x);
            b0.y = fmaf(xb[q].y, mul, b0.y);
            a1.x = fmaf(ya[q].x, mul, a1.x);
            a1.y = fmaf(ya[q].y, mul, a1.y);
            b1.x = fmaf(yb[q].x, mul, b1.x);
            b1.y = fmaf(yb[q].y, mul, b1.y);
          }
          pa += 8 * dr;
          pb += 8 * dr;
        }
        float2* ta = reinterpret_cast<float2*>(sTot + (2 * sw) * 128);
        float2* tb = reinterpret_cast<float2*>(sTot + (2 * sw + 1) * 128);
        ta[lane] = a0;
        ta[lane + 32] = a1;
        tb[lane] = b0;
        tb[lane + 32] = b1;
      }
      named_sync(1, 64);
      // Offsets of this warp's quarters and the chunk totals, for pairs lane and lane + 32.
      {
        const float2* tot = reinterpret_cast<const float2*>(sTot);
        float2 t0[4], t1[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          t0[q] = tot[q * 64 + lane];
          t1[q] = tot[q * 64 + lane + 32];
        }
        const float2 z = make_float2(0.f, 0.f);
#pragma unroll
        for (int e2 = 0; e2 < 2; ++e2) {
          const int qq = 2 * sw + e2;
          float2 o0 = pass1 ? cy0 : z, o1 = pass1 ? cy1 : z;
#pragma unroll
          for (int q = 0; q < 4; ++q)
            if (a.g.reverse ? q < qq : q > qq) {
              o0.x += t0[q].x;
              o0.y += t0[q].y;
              o1.x += t1[q].x;
              o1.y += t1[q].y;
            }
          float2* off = reinterpret_cast<float2*>(sOff + (s * 4 + qq) * 128);
          off[lane] = o0;
          off[lane + 32] = o1;
        }
        float2 c0 = z, c1 = z;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          c0.x += t0[q].x;
          c0.y += t0[q].y;
          c1.x += t1[q].x;
          c1.y += t1[q].y;
        }
        if (sw == 0) {
          float2* bl = reinterpret_cast<float2*>(sBL + s * 128);  // chunk gate sums; channels >= dk stay 0
          if (act0) bl[lane] = c0;
          if (act1) bl[lane + 32] = c1;
        }
        if (pass1) {
          cy0.x += c0.x;
          cy0.y += c0.y;
          cy1.x += c1.x;
          cy1.y += c1.y;
          if (last1 && sw == 0) {
            // exp(segment gate sum) of growth gates must stay finite
            bool bad = false;
            if (act0) {
              bad |= !(cy0.x <= kMaxGateRange2) || !(cy0.y <= kMaxGateRange2);
              sGam[buf * 128 + 2 * lane] = exp2_approx(cy0.x);
              sGam[buf * 128 + 2 * lane + 1] = exp2_approx(cy0.y);
            }
            if (act1) {
              bad |= !(cy1.x <= kMaxGateRange2) || !(cy1.y <= kMaxGateRange2);
              sGam[buf * 128 + 2 * lane + 64] = exp2_approx(cy1.x);
              sGam[buf * 128 + 2 * lane + 65] = exp2_approx(cy1.y);
            }
            if (bad) report_status(GLA_ERR_RANGE);
          }
          if (last1) ++ks;
        }
      }
      // (sTot is rewritten for the next chunk only after the group barrier at its start,
      // so both warps have read it by then.)
      mbar_arrive(BAR(kBarSufDone + s));
    }
  } else if (warp < kWarpEpi) {
    // ------------------------------------------------------------ gates
    // Gate warp gq owns rows 32gq..32gq+31 of every chunk (its TMEM subpartition):
    // u = the in-place local suffix sum + the offset of its quarter; K^ = k exp(u) and,
    // in pass 2, Q~ = q exp(-u), in place (lane = row); then the score masking.  A
    // chunk whose |u| exceeds the fp32-safe range anywhere is evaluated serially instead
    // (flagged here; the serial path reads the raw q and k from global memory).
    const int gq = warp - kWarpGate;
    const int pw = a.dk + 4;  // log-gate row pitch in floats
    int kbg = 0;              // non-serial pass-2 jobs masked so far
    for (int jc = 0;; ++jc) {
      const int s = jc % S, use = jc / S;
      if (!group_and(4, 128, wait_bar(BAR(kBarSufDone + s), (uint32_t)(use & 1), abort_flag))) break;
      const int kind = sJob[4 * s];
      if (kind == kJobEnd) {
        mbar_arrive(BAR(kBarGate + s));
        break;
      }
      const bool pass1 = kind == kJobP1;
      uint8_t* st = smem + (uint32_t)s * a.stage_bytes;
      const float* lag = reinterpret_cast<const float*>(st + a.oLA);
      // lane = row; q, k, v landed
      if (!group_and(4, 128, wait_bar(BAR(kBarOps + s), (uint32_t)(use & 1), abort_flag))) break;
      float umax = 0.f;  // pass 1: largest u; pass 2: largest |u|
      {
        const int r = 32 * gq + lane;
        const float* urow = lag + r * pw;
        const float* offq = sOff + (s * 4 + gq) * 128;
        // exp(u) = 2^(u log2 e) is rounded to bf16 pairs and applied with packed bf16
        // multiplies, exp(-u) as its reciprocal.
#pragma unroll 1
        for (int cc = 0; cc < a.dk; cc += 8) {
          const uint32_t o = sw32_off((uint32_t)r, (uint32_t)cc);
          const float4 u0 = *reinterpret_cast<const float4*>(urow + cc);
          const float4 u1 = *reinterpret_cast<const float4*>(urow + cc + 4);
          const float4 f0 = *reinterpret_cast<const float4*>(offq + cc);
          const float4 f1 = *reinterpret_cast<const float4*>(offq + cc + 4);
          uint4 kw = *reinterpret_cast<const uint4*>(st + a.oK + o);
          uint4 qw = make_uint4(0u, 0u, 0u, 0u);
          if (!pass1) qw = *reinterpret_cast<const uint4*>(st + a.oQ + o);
          const float ev[8] = {u0.x + f0.x, u0.y + f0.y, u0.z + f0.z, u0.w + f0.w,
                               u1.x + f1.x, u1.y + f1.y, u1.z + f1.z, u1.w + f1.w};
          uint32_t* uk = reinterpret_cast<uint32_t*>(&kw);
          uint32_t* uq = reinterpret_cast<uint32_t*>(&qw);
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) {
            const float a0 = ev[2 * jj], a1 = ev[2 * jj + 1];
            umax = fmaxf(umax, pass1 ? fmaxf(a0, a1) : fmaxf(fabsf(a0), fabsf(a1)));
            const float p0 = exp2_approx(a0), p1 = exp2_approx(a1);
            uk[jj] = mul_bf16x2(uk[jj], pack_bf16x2(p0, p1));
            if (!pass1) uq[jj] = mul_bf16x2(uq[jj], pack_bf16x2(__fdividef(1.f, p0), __fdividef(1.f, p1)));
          }
          *reinterpret_cast<uint4*>(st + a.oK + o) = kw;
          if (!pass1) *reinterpret_cast<uint4*>(st + a.oQ + o) = qw;
        }
      }
      fence_proxy_async_smem();
      // NaN compares false: a NaN or infinite u also counts as out of range.
      bool bad = !(umax <= kMaxGateRange2);
      if (!pass1 && gq == 0)
        for (int cc = lane; cc < a.dk; cc += 32) bad |= !(sBL[s * 128 + cc] <= kMaxGateRange2);  // exp(chunk sum)
      if (pass1) {
        if (bad) report_status(GLA_ERR_RANGE);  // exp(u) of growth gates overflows
        mbar_arrive(BAR(kBarGate + s));
        continue;
      }
      const bool wide = group_or(4, 128, bad);
      if (gq == 0 && lane == 0) sWide[s] = wide;
      mbar_arrive(BAR(kBarGate + s));
      if (wide) continue;
      // scores -> mask (keys scanned no later than the row) -> bf16 P in TMEM.
      // Warp gq owns TMEM lanes (rows) 32gq..32gq+31.
      if (!group_and(4, 128, wait_bar(BAR(kBarScFull), (uint32_t)(kbg & 1), abort_flag))) break;
      ++kbg;
      tc_fence_after();
      const int i = 32 * gq + lane;
      const uint32_t lane_base = (uint32_t)(32 * gq) << 16;
      {
        const int rlo = 32 * gq, rhi = rlo + 31;
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
      mbar_arrive(BAR(kBarPReady));
    }
  } else if (warp < kWarpLb) {
    // ------------------------------------------------------------ output group (pass 2)
    // Per chunk j (its scores are masked by the gate warps): once the MMAs of chunk j-1
    // have completed (O(j-1) written, state updated), G = Diag(gamma_j) S for chunk j's
    // Q~ G and K^T V; then the epilogue of chunk j-1 while chunk j's MMAs run.  A
    // chunk flagged serial is evaluated here token by token instead.
    const int i = 32 * (warp & 3) + lane;  // TMEM lane = row / key channel
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    const int e = tid - 32 * kWarpEpi;
    int kb = 0, jb = 0;
    bool ok = true;

    // MMAs of non-serial job pkb complete (output and state update).
    auto wait_batch = [&](int pkb) -> bool {
      if (!group_and(2, 128, wait_bar(BAR(kBarBatch + pkb % a.nO), (uint32_t)((pkb / a.nO) & 1), abort_flag)))
        return false;
      tc_fence_after();
      return true;
    };
    // Epilogue of non-serial job pkb (after wait_batch): O -> bf16 -> out[b][token][h][:],
    // then the O buffer is released.
    auto epilogue = [&](int ib, int ih, int cf, int pkb) {
      const int ob = pkb % a.nO;
      const int t = row_token(a, cf, i);
      const bool valid = t >= 0;
      __nv_bfloat16* orow = a.out;
      if (valid) orow = a.out + (((int64_t)ib * a.g.T + t) * a.H + ih) * a.dv;
      const uint32_t tO = tbase + a.col_o(ob) + lane_base;
#pragma unroll 1
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
      mbar_arrive(BAR(kBarOFree + ob));
    };

    for (int k = 0; ok; ++k) {
      const int buf = k % a.nbuf;
      if (!group_and(2, 128, wait_bar(BAR(kBarSinReady + buf), (uint32_t)((k / a.nbuf) & 1), abort_flag))) break;
      if (k >= sMisc[5]) break;  // end of the job stream
      tc_fence_after();
      const Item it = decode_item(a, sItem[3 + buf]);
      const uint32_t tSt = tbase + a.col_seg(buf) + lane_base;  // running state
      bool pending = false;  // epilogue of the last non-serial chunk still to do
      int p_cf = 0, p_kb = 0;
      // j == n only finishes the last chunk.
      for (int j = 0; j <= it.n; ++j) {
        const bool last = j == it.n;
        bool wide = false;
        int s = 0, cf = 0;
        uint32_t vpar = 0;
        if (!last) {
          if (!group_and(2, 128, wait_bar(BAR(kBarMail), (uint32_t)(jb & 1), abort_flag))) {
            ok = false;
            break;
          }
          s = sMail[0];
          wide = (sMail[1] & 1) != 0;
          vpar = (uint32_t)((sMail[1] >> 1) & 1);
          ++jb;
          cf = fwd_chunk(a, it.c0 + j);
          mbar_arrive(BAR(kBarScEmpty));  // the job is taken (the gate warps mask its scores)
        }
        // The previous chunk's MMAs complete: they updated the state and wrote its O.
        if (pending && !wait_batch(p_kb)) {
          ok = false;
          break;
        }
        uint8_t* st = smem + (uint32_t)s * a.stage_bytes;
        if (!last && !wide) {
          // G = Diag(gamma) S (state -> state, bf16 copy into the G tile)
          {
            const float gm = exp2_approx(sBL[s * 128 + i]);  // sums in log2 units
#pragma unroll 1
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
          fence_proxy_async_smem();  // the G tile is read by the tensor core
          tc_fence_before();
          mbar_arrive(BAR(kBarGReady));
        }
        // The previous chunk's epilogue runs while this chunk's state MMAs do.
        if (pending) epilogue(it.b, it.h, p_cf, p_kb);
        pending = false;
        if (last) break;
        if (wide) {
          if (!group_and(2, 128, wait_bar(BAR(kBarOpsV + s), vpar, abort_flag))) {
            ok = false;
            break;
          }
          chunk_serial(a, st, red, tbase + a.col_seg(buf), lane_base, i, cf, it.b, it.h);
          tc_fence_before();
          named_sync(2, 128);
          if (e == 0) {
            mbar_arrive(BAR(kBarEmpty + s));
            mbar_arrive(BAR(kBarEmptyV + s));
          }
          continue;
        }
        pending = true;
        p_cf = cf;
        p_kb = kb;
        ++kb;
      }
      if (!ok) break;
      // pass 2 is done with the buffer
      named_sync(2, 128);
      if (e == 0) mbar_arrive(BAR(kBarSegFree + buf));
    }
  } else {
    // ------------------------------------------------------------ look-back group
    const int i = 32 * (warp & 3) + lane;  // TMEM lane = key channel
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    const int e = tid - 32 * kWarpLb;
    for (int k = 0;; ++k) {
      const int buf = k % a.nbuf;
      if (!group_and(3, 128, wait_bar(BAR(kBarSegDone + buf), (uint32_t)((k / a.nbuf) & 1), abort_flag))) break;
      if (k >= sMisc[5]) {  // end of the job stream: pass it on to the output group
        if (e == 0) mbar_arrive(BAR(kBarSinReady + buf));
        break;
      }
      tc_fence_after();
      const int item = sItem[buf];
      const Item it = decode_item(a, item);
      lookback(a, it.seg, it.bh, it.seg_id, tbase + a.col_seg(buf) + lane_base, i, e, sGam[buf * 128 + i], sMisc + 6,
               BAR(kBarSinReady + buf), sItem + 3 + buf, item);
    }
  }

  // ---------------------------------------------------------------- teardown
  __syncthreads();
  if (*abort_flag && tid == 0) {
    // Let loads still in flight land before the shared memory is released: only the
    // last S posted jobs can still have any (earlier stages were reposted).
    for (int bb = 0; bb < 3; ++bb) {
      const int posted = bb == 2 ? sMisc[4] : sMisc[3];
      const int bar = bb == 0 ? kBarFull : (bb == 1 ? kBarOps : kBarOpsV);
      for (int jj = max(posted - S, 0); jj < posted; ++jj) {
        const long long t0 = clock64();
        while (!mbar_try_wait(BAR(bar + jj % S), (uint32_t)((jj / S) & 1)) && clock64() - t0 < kWaitCycles) {
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) tmem_dealloc(tbase, 512);
}

struct WsLayout {
  int NC, NS, G, Kp, Np, nstage, mode, rpc, ppr;
  uint32_t stage_bytes, oK, oV, oQ, oLA, oG, oBL, oWide, oGam, oRed, oTot, oOff, oMisc, oJob, oMail, oItem, oBar, oTm;
  int nO, nbuf;
  uint32_t colO0, colO1, colSeg0, colSeg1, colSeg2;
  size_t smem;
  size_t flag_bytes, agg_bytes, aggg_bytes;
};

constexpr int kSegChunks = 3;
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
  const uint32_t fixed = gtile + kMaxStages * 512 + 256 + 1536 + 256 + 2048 * (1 + kMaxStages) + 64 + 16 * kMaxStages + 16 + 32 +
                         8 * kNumBars + 16;
  L.nstage = (1024 + 2 * (size_t)L.stage_bytes + fixed <= kMaxSmem) ? 2 : 1;
  L.oG = (uint32_t)L.nstage * L.stage_bytes;
  L.oBL = L.oG + gtile;
  L.oWide = L.oBL + kMaxStages * 512;
  L.oGam = L.oWide + 256;
  L.oRed = L.oGam + 1536;
  L.oTot = L.oRed + 256;
  L.oOff = L.oTot + 2048;
  L.oMisc = L.oOff + 2048 * kMaxStages;
  L.oJob = L.oMisc + 64;
  L.oMail = L.oJob + 16 * kMaxStages;
  L.oItem = L.oMail + 16;
  L.oBar = L.oItem + 32;
  L.oTm = L.oBar + 8 * kNumBars;
  L.smem = 1024 + (size_t)L.oTm + 16;
  if (L.smem < 120 * 1024) L.smem = 120 * 1024;  // one CTA per SM: it owns all 512 TMEM columns
  // TMEM columns: scores / P [0,128), O, then the aggregate / state buffers: two O
  // buffers and two aggregate buffers when dv <= 96, else one O and two aggregates.
  L.nbuf = 2;
  if (L.Np <= 96) {
    L.nO = 2;
    L.colO0 = 128;
    L.colO1 = 224;
    L.colSeg0 = 320;
    L.colSeg1 = L.colSeg2 = 416;
  } else {
    L.nO = 1;
    L.colO0 = L.colO1 = 128;
    L.colSeg0 = 256;
    L.colSeg1 = L.colSeg2 = 384;
  }
  const size_t BH = (size_t)s.B * s.H;
  L.flag_bytes = al256((BH * L.NS + 1) * sizeof(int));
  L.agg_bytes = al256(BH * L.NS * s.dk * s.dv * sizeof(float));
  L.aggg_bytes = al256(BH * L.NS * s.dk * sizeof(float));
  return L;
}

// 5-D map over a [B][T][H][d] tensor viewed as (d, H, run position, run, B):
// raster scans have one run of T positions, column scans Wg runs of Hg.
bool encode_map(CUtensorMap* m, const void* base, bool f32, int d, int box0, CUtensorMapSwizzle sw, const GlaShape& s,
                bool column, int box_rows, int box_runs) {
  EncodeTiledFn fn = tensor_map_encoder();
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

// Raster 5-D map over a [B][T][H][d] bf16 tensor viewed as (16 channels, token,
// 16-channel atom, head, batch): a box of (16, 128, natoms, 1, 1) lands as natoms
// consecutive 32-byte-swizzled atoms of 128 rows.  natoms * 16 <= d keeps every
// element of the box inside the head's channels.
bool encode_atoms_map(CUtensorMap* m, const void* base, int d, int natoms, const GlaShape& s) {
  EncodeTiledFn fn = tensor_map_encoder();
  if (!fn) return false;
  const cuuint64_t T = (cuuint64_t)s.T(), H = (cuuint64_t)s.H;
  const cuuint64_t dims[5] = {16, T, (cuuint64_t)natoms, H, (cuuint64_t)s.B};
  const cuuint64_t strides[4] = {H * d * 2, 32, (cuuint64_t)d * 2, T * H * d * 2};
  const cuuint32_t box[5] = {16, (cuuint32_t)MC, (cuuint32_t)natoms, 1, 1};
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

size_t gla_ws_workspace_bytes(const GlaShape& s) {
  const WsLayout L = ws_layout(s);
  return L.flag_bytes + 2 * L.agg_bytes + L.aggg_bytes;
}

namespace {
// glog != nullptr: the gates are bf16 logits g and log_alpha = logsigmoid(g) / gate_norm
// (la unused); the logit tile's TMA box is padded to the fp32 tile's row pitch.
cudaError_t ws_forward(const void* q, const void* k, const void* v, const float* la, const void* glog,
                       float gate_norm, void* out, const GlaShape& s, void* workspace, cudaStream_t st) {
  const WsLayout L = ws_layout(s);
  if (L.smem > kMaxSmem) return cudaErrorInvalidValue;
  if (glog && 2 * (s.dk + 4) > 256) return cudaErrorInvalidValue;  // TMA box of at most 256 elements
  WsArgs a;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.k = static_cast<const __nv_bfloat16*>(k);
  a.v = static_cast<const __nv_bfloat16*>(v);
  a.la = la;
  a.glog = static_cast<const __nv_bfloat16*>(glog);
  a.inv_gate_norm = glog ? 1.f / gate_norm : 1.f;
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
  a.oTot = L.oTot;
  a.oOff = L.oOff;
  a.oMisc = L.oMisc;
  a.oJob = L.oJob;
  a.oMail = L.oMail;
  a.oItem = L.oItem;
  a.oBar = L.oBar;
  a.nO = L.nO;
  a.colO0 = L.colO0;
  a.colO1 = L.colO1;
  a.colSeg0 = L.colSeg0;
  a.colSeg1 = L.colSeg1;
  a.colSeg2 = L.colSeg2;
  a.nbuf = L.nbuf;
  a.items = (int)(BH * L.NS);
  a.skip = take_test_skip_items();
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
        (glog ? encode_map(&tm.la, glog, false, s.dk, 2 * (s.dk + 4), CU_TENSOR_MAP_SWIZZLE_NONE, s, column, box_rows,
                           box_runs)
              : encode_map(&tm.la, la, true, s.dk, s.dk + 4, CU_TENSOR_MAP_SWIZZLE_NONE, s, column, box_rows,
                           box_runs))))
    return cudaErrorInvalidValue;
  a.nak = a.nav = 0;
  if (L.mode == 0) {
    a.nak = s.dk / 16;
    a.nav = s.dv / 16;
    if ((a.nak && !(encode_atoms_map(&tm.qa, q, s.dk, a.nak, s) && encode_atoms_map(&tm.ka, k, s.dk, a.nak, s))) ||
        (a.nav && !encode_atoms_map(&tm.va, v, s.dv, a.nav, s)))
      return cudaErrorInvalidValue;
  }
  cudaError_t e = cudaMemsetAsync(ws, 0, L.flag_bytes, st);  // flags and the ticket counter
  if (e != cudaSuccess) return e;
  auto kernel = glog ? gla_ws_fwd<true> : gla_ws_fwd<false>;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const size_t grid = (size_t)a.items < (size_t)sms ? (size_t)a.items : (size_t)sms;
  kernel<<<(unsigned)grid, NT, L.smem, st>>>(a, tm);
  return cudaGetLastError();
}
}  // namespace

cudaError_t gla_ws_forward(const void* q, const void* k, const void* v, const float* la, void* out, const GlaShape& s,
                           void* workspace, cudaStream_t st) {
  return ws_forward(q, k, v, la, nullptr, 1.f, out, s, workspace, st);
}

cudaError_t gla_ws_forward_glogit(const void* q, const void* k, const void* v, const void* g, float gate_norm, void* out,
                                  const GlaShape& s, void* workspace, cudaStream_t st) {
  return ws_forward(q, k, v, nullptr, g, gate_norm, out, s, workspace, st);
}

}  // namespace dig
