// dev_common.cuh -- sm_100a device helpers for the DiG GLA library:
// mbarriers, cp.async staging, tcgen05 (TMEM alloc / MMA / load), UMMA shared
// memory descriptors, the 128-byte swizzle, the scan-order index map and the
// device status word.  Everything here is written against the public PTX ISA.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "dig_gla.h"

namespace dig {

// ---------------------------------------------------------------------------
// Device status word: the first error a kernel detects (bounded wait expired,
// gate range outside the supported domain) is recorded here; the host reads and
// clears it with dig_gla_device_status().
// ---------------------------------------------------------------------------
extern __device__ int g_device_status;

__device__ __forceinline__ void report_status(int code) { atomicCAS(&g_device_status, 0, code); }

// Upper bound, in SM clock cycles, for any wait on hardware progress (an MMA
// commit).  ~1 s at 2 GHz: far beyond any legitimate wait, small enough that a
// broken wait returns control instead of hanging the GPU.
constexpr long long kWaitCycles = 2000000000LL;

// ---------------------------------------------------------------------------
// Shared memory addresses and proxies
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Make this thread's generic-proxy shared memory writes visible to the async
// proxy (tensor core operand reads).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ uint32_t mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok;
}
// Wait for the phase with the given parity to complete; false if the cycle
// budget ran out first (the caller records an error and stops).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitCycles) return false;
  }
  return true;
}

// ---------------------------------------------------------------------------
// cp.async (16-byte, L2 only) with zero fill
// ---------------------------------------------------------------------------
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const uint32_t n = valid ? 16u : 0u;  // src-size 0 writes 16 zero bytes
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// ---------------------------------------------------------------------------
// 128-byte swizzle (the layout UMMA calls SWIZZLE_128B): rows of 128 bytes,
// 8-row atoms of 1024 bytes; the 16-byte chunk c of row r sits at chunk c ^ (r & 7).
// `tile` must be 1024-byte aligned.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t sw128(uint32_t row, uint32_t byte_in_row) {
  return row * 128u + ((((byte_in_row >> 4) ^ (row & 7u)) & 7u) << 4) + (byte_in_row & 15u);
}

// ---------------------------------------------------------------------------
// UMMA shared memory matrix descriptor (sm_100 format):
//   [0,14) start address >> 4, [16,30) leading byte offset >> 4,
//   [32,46) stride byte offset >> 4, [46,48) version = 1, [61,64) layout type.
// ---------------------------------------------------------------------------
constexpr uint32_t kLayoutSW128 = 2;

__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes,
                                              uint32_t layout) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1u << 46;
  d |= (uint64_t)(layout & 7u) << 61;
  return d;
}

// K-major operand in 128-byte-swizzled 64-element parts of `rows` rows each:
// K step kk (16 bf16) lives in part kk/4 at byte offset 32*(kk%4) of each row.
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t tile, uint32_t part_bytes, int kk) {
  const uint32_t a = tile + (uint32_t)(kk >> 2) * part_bytes + (uint32_t)(kk & 3) * 32u;
  return umma_desc(a, 16u, 1024u, kLayoutSW128);
}

// MN-major operand stored as [K rows][MN] in 128-byte-swizzled 64-element MN
// parts (`part_bytes` apart): K step kk (16 rows) starts 16*128 bytes further.
__device__ __forceinline__ uint64_t desc_mnmajor(uint32_t tile, uint32_t part_bytes, int kk) {
  const uint32_t a = tile + (uint32_t)kk * 2048u;
  return umma_desc(a, part_bytes, 1024u, kLayoutSW128);
}

// Instruction descriptor, kind::f16 with bf16 A/B and fp32 accumulation.
//   [4,6) D format (1 = f32), [7,10) A format (1 = bf16), [10,13) B format,
//   bit 15 A MN-major, bit 16 B MN-major, [17,23) N >> 3, [24,29) M >> 4.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool a_mn, bool b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// ---------------------------------------------------------------------------
// tcgen05
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem] * B[smem]
__device__ __forceinline__ void umma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on `bar` when all previously issued MMAs of this thread complete.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Each thread of the warp reads 32 consecutive fp32 columns of its own TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  tmem_ld_wait();
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
// 16 columns variant.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  tmem_ld_wait();
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// ---------------------------------------------------------------------------
// bf16 packing
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);  // round to nearest even
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ float2 unpack_bf16x2(uint32_t u) {
  __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&u);
  return __bfloat1622float2(h);
}

// ---------------------------------------------------------------------------
// Scan geometry.  The four SREM orders are handled as a "base" order (raster
// for L->R / R->L, column-major for T->B / B->T) and a reversal flag.  A forward
// position f in [0, T) of the base order maps to the raster token id:
//   raster base: t = f;  column base: t = (f mod Hg) * Wg + f / Hg.
// Reverse directions visit base positions T-1, T-2, ..., 0.
// ---------------------------------------------------------------------------
struct ScanGeom {
  int T, Hg, Wg;
  int column_base;  // 1 for T->B / B->T
  int reverse;      // 1 for R->L / B->T
  int zigzag;       // 0: one of the four SREM orders; 1 + j: zigzag scheme j (codes 4 + j)
};

__host__ __device__ __forceinline__ ScanGeom make_geom(int Hg, int Wg, int dir) {
  ScanGeom g;
  g.T = Hg * Wg;
  g.Hg = Hg;
  g.Wg = Wg;
  g.zigzag = dir >= 4 ? dir - 3 : 0;
  g.column_base = (dir == 2 || dir == 3) ? 1 : 0;
  g.reverse = (dir == 1 || dir == 3) ? 1 : 0;
  return g;
}

// Zigzag scheme j (ZigMa notes, "Zigzag 扫描方案": the scan turns back at the end of
// every line): lines are rows for j < 4, columns for j >= 4; bit 1 of j visits the
// lines last to first, bit 0 walks the first line from its end; every line reverses
// the direction of the one before.  Token visited at scan position p.
__device__ __forceinline__ int zigzag_token(const ScanGeom& g, int p) {
  const int j = g.zigzag - 1;
  const bool cols = j >= 4;
  const int len = cols ? g.Hg : g.Wg, nl = cols ? g.Wg : g.Hg;
  const int k = p / len, i = p - k * len;
  const int line = (j & 2) ? nl - 1 - k : k;
  const bool back = ((k & 1) != 0) != ((j & 1) != 0);
  const int at = back ? len - 1 - i : i;
  return cols ? at * g.Wg + line : line * g.Wg + at;
}

__device__ __forceinline__ int base_pos_to_token(const ScanGeom& g, int f) {
  if (!g.column_base) return f;
  const int x = f / g.Hg;
  const int y = f - x * g.Hg;
  return y * g.Wg + x;
}

// Token visited at scan position p.
__device__ __forceinline__ int scan_pos_to_token(const ScanGeom& g, int p) {
  if (g.zigzag) return zigzag_token(g, p);
  const int f = g.reverse ? (g.T - 1 - p) : p;
  return base_pos_to_token(g, f);
}

// First base position covered by chunk c (chunks of `mc` scan positions).  The
// tile's rows are base positions f0 .. f0+mc-1; rows outside [0, T) are padding.
__device__ __forceinline__ int chunk_first_base_pos(const ScanGeom& g, int c, int mc) {
  return g.reverse ? (g.T - mc * (c + 1)) : (mc * c);
}

}  // namespace dig
