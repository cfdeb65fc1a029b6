// api.cu -- the extern "C" entry points declared in include/dig_gla.h.
//
// Each entry point validates its arguments on the host (returning a status code
// before anything is enqueued), checks that the current device is an sm_100
// part, and enqueues the kernels on the caller's stream.  Scratch memory for the
// GLA passes comes from the stream-ordered allocator and is released on the same
// stream, so calls never synchronise.
#include <stdint.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "dev_common.cuh"
#include "dig_gla.h"
#include "internal.h"

namespace dig {

// Scan order codes: 0..3 the SREM orders, 4..11 the zigzag schemes.
constexpr int kDirLast = 11;

// First error a kernel recorded on this device (GLA_OK while none).
__device__ int g_device_status = 0;

namespace {

std::mutex g_mu;
int g_arch_ok[64];  // per device: 0 unknown, 1 sm_100, -1 other

}  // namespace

int check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return GLA_ERR_CUDA;
  if (dev < 0 || dev >= 64) return GLA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_arch_ok[dev] == 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return GLA_ERR_CUDA;
    g_arch_ok[dev] = (major == 10 && minor == 0) ? 1 : -1;
  }
  return g_arch_ok[dev] == 1 ? GLA_OK : GLA_ERR_UNSUPPORTED;
}

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + nb && b0 < a0 + na;
}

}  // namespace

int validate_gla(const void* q, const void* k, const void* v, const void* la, const void* out, int B, int H,
                 int Hg, int Wg, int dk, int dv, int dir, size_t elt) {
  if (!q || !k || !v || !la || !out) return GLA_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || Hg <= 0 || Wg <= 0 || dk <= 0 || dv <= 0) return GLA_ERR_INVALID_ARG;
  if (dir < 0 || dir > kDirLast) return GLA_ERR_INVALID_ARG;
  if (dk % 8 || dv % 8 || dk > 128 || dv > 128) return GLA_ERR_UNSUPPORTED;
  const int64_t T = (int64_t)Hg * Wg;
  if (T > (int64_t)1 << 30) return GLA_ERR_UNSUPPORTED;
  if ((int64_t)B * H > 65535) return GLA_ERR_UNSUPPORTED;
  const int64_t rows = (int64_t)B * T * H;
  if (rows > ((int64_t)1 << 40) / 128) return GLA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(la) || !aligned16(out))
    return GLA_ERR_ALIGNMENT;
  const size_t nq = (size_t)rows * dk * elt, nv = (size_t)rows * dv * elt, nl = (size_t)rows * dk * 4;
  const size_t no = (size_t)rows * dv * elt;
  if (overlaps(out, no, q, nq) || overlaps(out, no, k, nq) || overlaps(out, no, v, nv) || overlaps(out, no, la, nl))
    return GLA_ERR_INVALID_ARG;
  return GLA_OK;
}

// The backward's extra tensors: dout is read like v; dq, dk, dv, dlog_alpha are
// written and may overlap nothing (validate_gla has checked q, k, v, log_alpha and dq).
int validate_gla_bwd(const void* q, const void* k, const void* v, const void* la, const void* dout, const void* dq,
                     const void* dk_out, const void* dv_out, const void* dla, int B, int H, int Hg, int Wg, int dk,
                     int dv, int dir, size_t elt) {
  int rc = validate_gla(q, k, v, la, dq, B, H, Hg, Wg, dk, dv, dir, elt);
  if (rc != GLA_OK) return rc;
  if (!dout || !dk_out || !dv_out || !dla) return GLA_ERR_INVALID_ARG;
  if (!aligned16(dout) || !aligned16(dk_out) || !aligned16(dv_out) || !aligned16(dla)) return GLA_ERR_ALIGNMENT;
  const size_t rows = (size_t)B * Hg * Wg * H;
  const size_t nk = rows * dk * elt, nv = rows * dv * elt, nl = rows * dk * 4;
  const void* in[5] = {q, k, v, la, dout};
  const size_t nin[5] = {nk, nk, nv, nl, nv};
  const void* outs[4] = {dq, dk_out, dv_out, dla};
  const size_t nout[4] = {nk, nk, nv, nl};
  for (int o = 0; o < 4; ++o) {
    for (int i = 0; i < 5; ++i)
      if (overlaps(outs[o], nout[o], in[i], nin[i])) return GLA_ERR_INVALID_ARG;
    for (int o2 = o + 1; o2 < 4; ++o2)
      if (overlaps(outs[o], nout[o], outs[o2], nout[o2])) return GLA_ERR_INVALID_ARG;
  }
  return GLA_OK;
}

// The normalised variant: q, k, v, out as the forward's (no log_alpha: the gate comes
// from q and k); eps positive; dv at most 120, leaving room for the ones column.
int validate_gla_norm(const void* q, const void* k, const void* v, const void* out, int B, int H, int Hg, int Wg,
                      int dk, int dv, int dir, float eps, size_t elt) {
  if (!q || !k || !v || !out) return GLA_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || Hg <= 0 || Wg <= 0 || dk <= 0 || dv <= 0) return GLA_ERR_INVALID_ARG;
  if (dir < 0 || dir > kDirLast || !(eps > 0.f)) return GLA_ERR_INVALID_ARG;
  if (dk % 8 || dv % 8 || dk > 128 || dv > 120) return GLA_ERR_UNSUPPORTED;
  const int64_t T = (int64_t)Hg * Wg;
  if (T > (int64_t)1 << 30 || (int64_t)B * H > 65535) return GLA_ERR_UNSUPPORTED;
  const int64_t rows = (int64_t)B * T * H;
  if (rows > ((int64_t)1 << 40) / 128) return GLA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return GLA_ERR_ALIGNMENT;
  const size_t nq = (size_t)rows * dk * elt, nv = (size_t)rows * dv * elt;
  if (overlaps(out, nv, q, nq) || overlaps(out, nv, k, nq) || overlaps(out, nv, v, nv)) return GLA_ERR_INVALID_ARG;
  return GLA_OK;
}

// The gate-logit forward: q, k, v, g (bf16, g shaped like q), out; dk at most 120
// (the logit tile's padded TMA box); the four SREM orders; gate_norm positive.
int validate_gla_glogit(const void* q, const void* k, const void* v, const void* g, const void* out, int B, int H,
                        int Hg, int Wg, int dk, int dv, int dir, float gate_norm) {
  if (!g) return GLA_ERR_INVALID_ARG;
  int rc = validate_gla_norm(q, k, v, out, B, H, Hg, Wg, dk, dv, dir > 3 ? 0 : dir, 1.f, 2);
  if (rc != GLA_OK) return rc;
  if (dir > 3) return GLA_ERR_UNSUPPORTED;
  if (!(gate_norm > 0.f)) return GLA_ERR_INVALID_ARG;
  if (dk > 120 || dv > 128) return GLA_ERR_UNSUPPORTED;
  if (!aligned16(g)) return GLA_ERR_ALIGNMENT;
  const size_t rows = (size_t)B * Hg * Wg * H;
  if (overlaps(out, rows * dv * 2, g, rows * dk * 2)) return GLA_ERR_INVALID_ARG;
  return GLA_OK;
}

namespace {

int validate_grid(const void* x, const void* y, int B, int Hg, int Wg, int C, int dtype, size_t* row_bytes) {
  if (!x || !y) return GLA_ERR_INVALID_ARG;
  if (B <= 0 || Hg <= 0 || Wg <= 0 || C <= 0) return GLA_ERR_INVALID_ARG;
  if (dtype != GLA_BF16 && dtype != GLA_F32) return GLA_ERR_INVALID_ARG;
  const size_t elt = dtype == GLA_BF16 ? 2 : 4;
  const size_t rb = (size_t)C * elt;
  if (rb % 16) return GLA_ERR_ALIGNMENT;
  if (!aligned16(x) || !aligned16(y)) return GLA_ERR_ALIGNMENT;
  const int64_t T = (int64_t)Hg * Wg;
  if (T > (int64_t)1 << 30 || (int64_t)B * T > ((int64_t)1 << 40) / (int64_t)rb) return GLA_ERR_UNSUPPORTED;
  if ((int64_t)B * ((Hg + 15) / 16) > 65535 || (Wg + 3) / 4 > 65535) return GLA_ERR_UNSUPPORTED;
  const size_t n = (size_t)B * T * rb;
  if (overlaps(x, n, y, n)) return GLA_ERR_INVALID_ARG;
  *row_bytes = rb;
  return GLA_OK;
}

// Per-device memory pool for the GLA scratch: stream-ordered like the default pool, but
// it keeps its memory across stream synchronisations (the default pool returns it at
// every synchronisation, so the next call would map it again on the host).
// dig_gla_release() trims it.
cudaMemPool_t g_pool[64];

cudaMemPool_t workspace_pool(int dev) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_pool[dev]) {
    cudaMemPoolProps props;
    memset(&props, 0, sizeof(props));
    props.allocType = cudaMemAllocationTypePinned;
    props.handleTypes = cudaMemHandleTypeNone;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaMemPool_t p = nullptr;
    if (cudaMemPoolCreate(&p, &props) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    uint64_t keep = UINT64_MAX;
    cudaMemPoolSetAttribute(p, cudaMemPoolAttrReleaseThreshold, &keep);
    g_pool[dev] = p;
  }
  return g_pool[dev];
}

int run_with_workspace(size_t bytes, cudaStream_t st, cudaError_t (*fn)(void*, void*), void* ctx) {
  void* ws = nullptr;
  if (bytes) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return GLA_ERR_CUDA;
    cudaMemPool_t pool = workspace_pool(dev);
    const cudaError_t e = pool ? cudaMallocFromPoolAsync(&ws, bytes, pool, st) : cudaMallocAsync(&ws, bytes, st);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return GLA_ERR_NOMEM;
    }
  }
  const cudaError_t e = fn(ws, ctx);
  if (ws) cudaFreeAsync(ws, st);
  return e == cudaSuccess ? GLA_OK : GLA_ERR_CUDA;
}

}  // namespace

EncodeTiledFn tensor_map_encoder() {
  static const EncodeTiledFn fn = []() -> EncodeTiledFn {  // initialised once, thread-safe
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<EncodeTiledFn>(p);
    cudaGetLastError();
    return nullptr;
  }();
  return fn;
}

cudaError_t read_and_clear_device_status(int* status, cudaStream_t st) {
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return e;
  int v = 0, zero = 0;
  e = cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int));
  if (e != cudaSuccess) return e;
  e = cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int));
  if (e != cudaSuccess) return e;
  *status = v;
  return cudaSuccess;
}

std::atomic<int> g_test_skip{0};
int take_test_skip_items() { return g_test_skip.exchange(0); }

}  // namespace dig

using dig::GlaShape;

namespace {
struct GlaCall {
  const void *q, *k, *v;
  const float* la;
  void* out;
  GlaShape s;
  cudaStream_t st;
};
// ---- zigzag orders (codes 4..11) ------------------------------------------------
// They run as the ZigMa notes write a layer ("异构逐层扫描": arrange the tokens into
// the scheme's order, scan, arrange the result back): the token rows of every input
// are gathered into scan order, the left-to-right scan runs over them as one line of
// T tokens, and the output rows are scattered back to canonical positions.  The four
// SREM orders need no copies: their order lives in the kernels' address math.
size_t rup256(size_t x) { return (x + 255) / 256 * 256; }
GlaShape line_shape(const GlaShape& s) { return GlaShape{s.B, s.H, 1, s.T(), s.dk, s.dv, 0}; }
size_t rows_of(const GlaShape& s) { return (size_t)s.B * s.T() * s.H; }

// Scratch of the arranged copies: n_k tensors of width dk and n_v of width dv in the
// call's element type, and n_l fp32 tensors of width dk.
size_t arranged_bytes(const GlaShape& s, size_t elt, int n_k, int n_v, int n_l) {
  const size_t r = rows_of(s);
  return n_k * rup256(r * s.dk * elt) + n_v * rup256(r * s.dv * elt) + n_l * rup256(r * s.dk * 4);
}

// Gathers (inverse 0) or scatters (inverse 1) whole token rows [B][T][H*d].
cudaError_t arrange(const void* x, void* y, const GlaShape& s, size_t row_bytes, int inverse, cudaStream_t st) {
  return dig::srem_reorient_launch(x, y, s.dir, inverse, s.B, s.Hg, s.Wg, row_bytes, st);
}

cudaError_t fwd_line(const GlaCall& c, size_t elt, void* ws,
                     cudaError_t (*fwd)(const GlaCall&, void*)) {
  if (c.s.dir < 4) return fwd(c, ws);
  const GlaShape& s = c.s;
  const size_t r = rows_of(s);
  uint8_t* p = static_cast<uint8_t*>(ws);
  void* q2 = p;
  p += rup256(r * s.dk * elt);
  void* k2 = p;
  p += rup256(r * s.dk * elt);
  void* v2 = p;
  p += rup256(r * s.dv * elt);
  void* o2 = p;
  p += rup256(r * s.dv * elt);
  float* l2 = reinterpret_cast<float*>(p);
  p += rup256(r * s.dk * 4);
  const size_t rk = (size_t)s.H * s.dk * elt, rv = (size_t)s.H * s.dv * elt, rl = (size_t)s.H * s.dk * 4;
  cudaError_t e;
  if ((e = arrange(c.q, q2, s, rk, 0, c.st)) != cudaSuccess || (e = arrange(c.k, k2, s, rk, 0, c.st)) != cudaSuccess ||
      (e = arrange(c.v, v2, s, rv, 0, c.st)) != cudaSuccess || (e = arrange(c.la, l2, s, rl, 0, c.st)) != cudaSuccess)
    return e;
  const GlaCall c2{q2, k2, v2, l2, o2, line_shape(s), c.st};
  if ((e = fwd(c2, p)) != cudaSuccess) return e;
  return arrange(o2, c.out, s, rv, 1, c.st);
}

cudaError_t tc_fwd(const GlaCall& c, void* ws) { return dig::gla_ws_forward(c.q, c.k, c.v, c.la, c.out, c.s, ws, c.st); }
cudaError_t f32_fwd(const GlaCall& c, void* ws) {
  return dig::gla_f32_forward(static_cast<const float*>(c.q), static_cast<const float*>(c.k),
                              static_cast<const float*>(c.v), c.la, static_cast<float*>(c.out), c.s, ws, c.st);
}
cudaError_t run_tc(void* ws, void* ctx) { return fwd_line(*static_cast<const GlaCall*>(ctx), 2, ws, tc_fwd); }
cudaError_t run_f32(void* ws, void* ctx) { return fwd_line(*static_cast<const GlaCall*>(ctx), 4, ws, f32_fwd); }
size_t tc_ws_bytes(const GlaShape& s) {
  return s.dir < 4 ? dig::gla_ws_workspace_bytes(s)
                   : arranged_bytes(s, 2, 2, 2, 1) + dig::gla_ws_workspace_bytes(line_shape(s));
}
size_t f32_ws_bytes(const GlaShape& s) {
  return s.dir < 4 ? dig::gla_f32_workspace_bytes(s)
                   : arranged_bytes(s, 4, 2, 2, 1) + dig::gla_f32_workspace_bytes(line_shape(s));
}
struct BwdCall {
  const void *q, *k, *v;
  const float* la;
  const void* dout;
  void *dq, *dk, *dv;
  float* dla;
  GlaShape s;
  int bf16;
  cudaStream_t st;
};
cudaError_t run_bwd(void* ws, void* ctx) {
  const BwdCall* c = static_cast<const BwdCall*>(ctx);
  const GlaShape& s = c->s;
  if (s.dir < 4)
    return dig::gla_bwd_launch(c->q, c->k, c->v, c->la, c->dout, c->dq, c->dk, c->dv, c->dla, s, c->bf16, ws, c->st);
  // zigzag: arrange the five inputs, differentiate the line, scatter the four gradients
  const size_t elt = c->bf16 ? 2 : 4;
  const size_t r = rows_of(s);
  const size_t nk = rup256(r * s.dk * elt), nv = rup256(r * s.dv * elt), nl = rup256(r * s.dk * 4);
  uint8_t* p = static_cast<uint8_t*>(ws);
  void *q2 = p, *k2 = p + nk, *dq2 = p + 2 * nk, *dk2 = p + 3 * nk;
  p += 4 * nk;
  void *v2 = p, *do2 = p + nv, *dv2 = p + 2 * nv;
  p += 3 * nv;
  float* l2 = reinterpret_cast<float*>(p);
  float* dl2 = reinterpret_cast<float*>(p + nl);
  p += 2 * nl;
  const size_t rk = (size_t)s.H * s.dk * elt, rv = (size_t)s.H * s.dv * elt, rl = (size_t)s.H * s.dk * 4;
  cudaError_t e;
  if ((e = arrange(c->q, q2, s, rk, 0, c->st)) != cudaSuccess || (e = arrange(c->k, k2, s, rk, 0, c->st)) != cudaSuccess ||
      (e = arrange(c->v, v2, s, rv, 0, c->st)) != cudaSuccess || (e = arrange(c->la, l2, s, rl, 0, c->st)) != cudaSuccess ||
      (e = arrange(c->dout, do2, s, rv, 0, c->st)) != cudaSuccess)
    return e;
  if ((e = dig::gla_bwd_launch(q2, k2, v2, l2, do2, dq2, dk2, dv2, dl2, line_shape(s), c->bf16, p, c->st)) !=
      cudaSuccess)
    return e;
  if ((e = arrange(dq2, c->dq, s, rk, 1, c->st)) != cudaSuccess || (e = arrange(dk2, c->dk, s, rk, 1, c->st)) != cudaSuccess ||
      (e = arrange(dv2, c->dv, s, rv, 1, c->st)) != cudaSuccess)
    return e;
  return arrange(dl2, c->dla, s, rl, 1, c->st);
}
size_t bwd_ws_bytes(const GlaShape& s, int bf16) {
  return s.dir < 4 ? dig::gla_bwd_workspace_bytes(s, bf16)
                   : arranged_bytes(s, bf16 ? 2 : 4, 4, 3, 2) + dig::gla_bwd_workspace_bytes(line_shape(s), bf16);
}
int gla_bwd_common(const void* q, const void* k, const void* v, const float* la, const void* dout, int B, int H,
                   int Hgrid, int Wgrid, int dk, int dv, int dir, void* dq, void* dk_out, void* dv_out, float* dla,
                   int bf16, cudaStream_t stream) {
  int rc = dig::validate_gla_bwd(q, k, v, la, dout, dq, dk_out, dv_out, dla, B, H, Hgrid, Wgrid, dk, dv, dir,
                                 bf16 ? 2 : 4);
  if (rc != GLA_OK) return rc;
  if ((rc = dig::check_device()) != GLA_OK) return rc;
  BwdCall c{q, k, v, la, dout, dq, dk_out, dv_out, dla, GlaShape{B, H, Hgrid, Wgrid, dk, dv, dir}, bf16, stream};
  return dig::run_with_workspace(bwd_ws_bytes(c.s, bf16), stream, run_bwd, &c);
}
// ---- gate logits in place of log_alpha ------------------------------------------
struct GlogitCall {
  const void *q, *k, *v, *g;
  float gate_norm;
  void* out;
  GlaShape s;
  cudaStream_t st;
};
cudaError_t run_glogit(void* ws, void* ctx) {
  const GlogitCall* c = static_cast<const GlogitCall*>(ctx);
  return dig::gla_ws_forward_glogit(c->q, c->k, c->v, c->g, c->gate_norm, c->out, c->s, ws, c->st);
}

// ---- the normalised variant ----------------------------------------------------
struct NormCall {
  const void *q, *k, *v;
  void* out;
  GlaShape s;
  float eps;
  int bf16;
  cudaStream_t st;
};
int norm_width(int dv) { return dv + 8; }  // v, a column of ones, zero padding to a multiple of 8
size_t norm_ws_bytes(const GlaShape& s) {
  const size_t r = rows_of(s);
  const GlaShape sa{s.B, s.H, s.Hg, s.Wg, s.dk, norm_width(s.dv), s.dir};
  return 3 * rup256(r * s.dk * 4) + 2 * rup256(r * sa.dv * 4) + f32_ws_bytes(sa);
}
cudaError_t run_norm(void* ws, void* ctx) {
  const NormCall* c = static_cast<const NormCall*>(ctx);
  const GlaShape& s = c->s;
  const int dva = norm_width(s.dv);
  const GlaShape sa{s.B, s.H, s.Hg, s.Wg, s.dk, dva, s.dir};
  const size_t r = rows_of(s);
  uint8_t* p = static_cast<uint8_t*>(ws);
  float* fq = reinterpret_cast<float*>(p);
  p += rup256(r * s.dk * 4);
  float* fk = reinterpret_cast<float*>(p);
  p += rup256(r * s.dk * 4);
  float* la = reinterpret_cast<float*>(p);
  p += rup256(r * s.dk * 4);
  float* va = reinterpret_cast<float*>(p);
  p += rup256(r * dva * 4);
  float* oa = reinterpret_cast<float*>(p);
  p += rup256(r * dva * 4);
  cudaError_t e;
  if ((e = dig::gla_norm_prep_launch(c->q, c->k, c->v, fq, fk, la, va, (int64_t)r, s.dk, s.dv, dva, c->bf16, c->st)) !=
      cudaSuccess)
    return e;
  const GlaCall g{fq, fk, va, la, oa, sa, c->st};
  if ((e = fwd_line(g, 4, p, f32_fwd)) != cudaSuccess) return e;
  return dig::gla_norm_post_launch(oa, c->out, (int64_t)r, s.dv, dva, c->eps, c->bf16, c->st);
}
int gla_norm_common(const void* q, const void* k, const void* v, int B, int H, int Hgrid, int Wgrid, int dk, int dv,
                    int dir, float eps, void* out, int bf16, cudaStream_t stream) {
  int rc = dig::validate_gla_norm(q, k, v, out, B, H, Hgrid, Wgrid, dk, dv, dir, eps, bf16 ? 2 : 4);
  if (rc != GLA_OK) return rc;
  if ((rc = dig::check_device()) != GLA_OK) return rc;
  NormCall c{q, k, v, out, GlaShape{B, H, Hgrid, Wgrid, dk, dv, dir}, eps, bf16, stream};
  return dig::run_with_workspace(norm_ws_bytes(c.s), stream, run_norm, &c);
}
}  // namespace

extern "C" {

int gla_fwd_glogit(const void* q, const void* k, const void* v, const void* g, int B, int H, int Hgrid, int Wgrid,
                   int dk, int dv, int dir, float gate_norm, void* out, cudaStream_t stream) {
  int rc = dig::validate_gla_glogit(q, k, v, g, out, B, H, Hgrid, Wgrid, dk, dv, dir, gate_norm);
  if (rc != GLA_OK) return rc;
  if ((rc = dig::check_device()) != GLA_OK) return rc;
  GlogitCall c{q, k, v, g, gate_norm, out, GlaShape{B, H, Hgrid, Wgrid, dk, dv, dir}, stream};
  return dig::run_with_workspace(dig::gla_ws_workspace_bytes(c.s), stream, run_glogit, &c);
}

int gla_norm_fwd(const void* q, const void* k, const void* v, int B, int H, int Hgrid, int Wgrid, int dk, int dv,
                 int dir, float eps, void* out, cudaStream_t stream) {
  return gla_norm_common(q, k, v, B, H, Hgrid, Wgrid, dk, dv, dir, eps, out, 1, stream);
}

int gla_norm_fwd_f32(const float* q, const float* k, const float* v, int B, int H, int Hgrid, int Wgrid, int dk,
                     int dv, int dir, float eps, float* out, cudaStream_t stream) {
  return gla_norm_common(q, k, v, B, H, Hgrid, Wgrid, dk, dv, dir, eps, out, 0, stream);
}

int gla_bwd(const void* q, const void* k, const void* v, const float* log_alpha, const void* dout, int B, int H,
            int Hgrid, int Wgrid, int dk, int dv, int dir, void* dq, void* dk_out, void* dv_out, float* dlog_alpha,
            cudaStream_t stream) {
  return gla_bwd_common(q, k, v, log_alpha, dout, B, H, Hgrid, Wgrid, dk, dv, dir, dq, dk_out, dv_out, dlog_alpha, 1,
                        stream);
}

int gla_bwd_f32(const float* q, const float* k, const float* v, const float* log_alpha, const float* dout, int B,
                int H, int Hgrid, int Wgrid, int dk, int dv, int dir, float* dq, float* dk_out, float* dv_out,
                float* dlog_alpha, cudaStream_t stream) {
  return gla_bwd_common(q, k, v, log_alpha, dout, B, H, Hgrid, Wgrid, dk, dv, dir, dq, dk_out, dv_out, dlog_alpha, 0,
                        stream);
}

int gla_fwd(const void* q, const void* k, const void* v, const float* log_alpha, int B, int H, int Hgrid, int Wgrid,
            int dk, int dv, int dir, void* out, cudaStream_t stream) {
  int rc = dig::validate_gla(q, k, v, log_alpha, out, B, H, Hgrid, Wgrid, dk, dv, dir, 2);
  if (rc != GLA_OK) return rc;
  if ((rc = dig::check_device()) != GLA_OK) return rc;
  GlaCall c{q, k, v, log_alpha, out, GlaShape{B, H, Hgrid, Wgrid, dk, dv, dir}, stream};
  return dig::run_with_workspace(tc_ws_bytes(c.s), stream, run_tc, &c);
}

int gla_fwd_f32(const float* q, const float* k, const float* v, const float* log_alpha, int B, int H, int Hgrid,
                int Wgrid, int dk, int dv, int dir, float* out, cudaStream_t stream) {
  int rc = dig::validate_gla(q, k, v, log_alpha, out, B, H, Hgrid, Wgrid, dk, dv, dir, 4);
  if (rc != GLA_OK) return rc;
  if ((rc = dig::check_device()) != GLA_OK) return rc;
  GlaCall c{q, k, v, log_alpha, out, GlaShape{B, H, Hgrid, Wgrid, dk, dv, dir}, stream};
  return dig::run_with_workspace(f32_ws_bytes(c.s), stream, run_f32, &c);
}

int srem_reorient(const void* x, int dir, int inverse, int B, int Hgrid, int Wgrid, int C, int dtype, void* y,
                  cudaStream_t stream) {
  size_t rb = 0;
  int rc = dig::validate_grid(x, y, B, Hgrid, Wgrid, C, dtype, &rb);
  if (rc != GLA_OK) return rc;
  if (dir < 0 || dir > dig::kDirLast || (inverse != 0 && inverse != 1)) return GLA_ERR_INVALID_ARG;
  if ((rc = dig::check_device()) != GLA_OK) return rc;
  return dig::srem_reorient_launch(x, y, dir, inverse, B, Hgrid, Wgrid, rb, stream) == cudaSuccess ? GLA_OK
                                                                                                   : GLA_ERR_CUDA;
}

int dwconv3x3(const void* x, const float* w, int B, int Hgrid, int Wgrid, int C, int dtype, void* y,
              cudaStream_t stream) {
  size_t rb = 0;
  int rc = dig::validate_grid(x, y, B, Hgrid, Wgrid, C, dtype, &rb);
  if (rc != GLA_OK) return rc;
  if (!w) return GLA_ERR_INVALID_ARG;
  if (!dig::aligned16(w)) return GLA_ERR_ALIGNMENT;
  if ((rc = dig::check_device()) != GLA_OK) return rc;
  return dig::dwconv3x3_launch(x, w, y, B, Hgrid, Wgrid, C, dtype, stream) == cudaSuccess ? GLA_OK : GLA_ERR_CUDA;
}

int dig_gla_device_status(cudaStream_t stream) {
  int rc = dig::check_device();
  if (rc != GLA_OK) return rc;
  int v = 0;
  if (dig::read_and_clear_device_status(&v, stream) != cudaSuccess) return GLA_ERR_CUDA;
  return v;
}

const char* dig_gla_status_string(int status) {
  switch (status) {
    case GLA_OK: return "GLA_OK";
    case GLA_ERR_INVALID_ARG: return "GLA_ERR_INVALID_ARG";
    case GLA_ERR_UNSUPPORTED: return "GLA_ERR_UNSUPPORTED";
    case GLA_ERR_ALIGNMENT: return "GLA_ERR_ALIGNMENT";
    case GLA_ERR_CUDA: return "GLA_ERR_CUDA";
    case GLA_ERR_TIMEOUT: return "GLA_ERR_TIMEOUT";
    case GLA_ERR_NOMEM: return "GLA_ERR_NOMEM";
    case GLA_ERR_RANGE: return "GLA_ERR_RANGE";
    default: return "GLA_ERR_UNKNOWN";
  }
}

void dig_gla_test_skip_items(int n) { dig::g_test_skip.store(n > 0 ? n : 0); }

void dig_gla_release(void) {
  {
    std::lock_guard<std::mutex> lk(dig::g_mu);
    memset(dig::g_arch_ok, 0, sizeof(dig::g_arch_ok));
    for (cudaMemPool_t& p : dig::g_pool) {
      // Allocations still in flight keep their memory until they are freed; the
      // pool itself goes once they are.  The next call creates a new one.
      if (p) cudaMemPoolDestroy(p);
      p = nullptr;
    }
  }
  cudaGetLastError();
  dig::noalloc_forget();
}

}  // extern "C"
