/*
 * dig_gla.h -- C ABI of the DiG gated-linear-attention hot path on NVIDIA B200
 * (sm_100a): the chunk-wise GLA forward over one of the four SREM scan orders,
 * the SREM reorientation of the token grid, and SREM's 3x3 depthwise conv.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All tensor arguments are DEVICE pointers to dense, contiguous buffers owned
 *    by the caller.  The library keeps no reference to them after the call.
 *  - Token grids are Hgrid x Wgrid patches, T = Hgrid*Wgrid, and token t is the
 *    raster index t = y*Wgrid + x.  Sequence tensors are token-major with heads
 *    interleaved: q, k, log_alpha are [B][T][H][dk]; v and out are [B][T][H][dv]
 *    (the layout a fused q/k/v projection writes).  Grid tensors for the conv and
 *    the reorientation are channels-last [B][Hgrid][Wgrid][C] (== [B][T][C]).
 *  - Scan directions (DiG paper notes, "空间重定向与增强模块 (SREM)": four scan
 *    orders -- left-to-right, right-to-left, top-to-bottom, bottom-to-top --
 *    produced by transposing the 2D token matrix and flipping the sequence),
 *    numbered in the order the notes list them:
 *      GLA_DIR_L2R = 0: raster order t = p
 *      GLA_DIR_R2L = 1: reversed raster order t = T-1-p
 *      GLA_DIR_T2B = 2: column-major order t = (p mod Hgrid)*Wgrid + p div Hgrid
 *      GLA_DIR_B2T = 3: reversed column-major order
 *    Codes 4..11 are the eight zigzag orders S_0..S_7 of the ZigMa notes ("Zigzag
 *    扫描方案": the scan turns back at the end of every line, so neighbours in the
 *    sequence are neighbours in the grid), code GLA_DIR_ZIGZAG0 + j for scheme j:
 *    lines are the grid's rows for j < 4 and its columns for j >= 4; bit 1 of j
 *    visits the lines last to first; bit 0 walks the first line from its end; each
 *    line then reverses the direction of the one before.  The GLA entry points run
 *    them as the notes write a layer: the token rows are gathered into the scan order
 *    (srem_reorient), scanned left to right as one line of T tokens, and the results
 *    scattered back, so a zigzag call also moves every input and output through HBM
 *    once more and needs that much more workspace.  gla_fwd_f32_noalloc takes codes
 *    0..3 only.
 *  - Every call is asynchronous on `stream` (0 = the legacy default stream) and
 *    never synchronises it.  Argument errors are returned synchronously before
 *    anything is launched; a launch failure returns GLA_ERR_CUDA.  Conditions a
 *    kernel detects while running (a bounded wait that expired, growth gates that
 *    overflow fp32) are recorded in a per-device status word that
 *    dig_gla_device_status() reads and clears.
 *  - Pointers must be 16-byte aligned.  There is no CPU fallback: a call on a
 *    device other than sm_100 returns GLA_ERR_UNSUPPORTED.
 */
#ifndef DIG_GLA_H_
#define DIG_GLA_H_

#include <cuda_runtime_api.h>
#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  GLA_OK = 0,
  GLA_ERR_INVALID_ARG = -1, /* null pointer, non-positive size, bad enum, aliasing */
  GLA_ERR_UNSUPPORTED = -2, /* a size or device this build does not handle */
  GLA_ERR_ALIGNMENT = -3,   /* a pointer or a row pitch that is not 16-byte aligned */
  GLA_ERR_CUDA = -4,        /* a CUDA runtime call failed (see cudaGetLastError) */
  GLA_ERR_TIMEOUT = -5,     /* a kernel gave up a bounded wait (device status only) */
  GLA_ERR_NOMEM = -6,       /* the stream-ordered workspace could not be allocated */
  GLA_ERR_RANGE = -7        /* growth gates (log_alpha > 0) overflowed fp32 inside a chunk
                               (device status only; the output is not valid) */
} gla_status_t;

enum { GLA_DIR_L2R = 0, GLA_DIR_R2L = 1, GLA_DIR_T2B = 2, GLA_DIR_B2T = 3, GLA_DIR_ZIGZAG0 = 4 };
enum { GLA_BF16 = 0, GLA_F32 = 1 };

/*
 * gla_fwd -- chunk-wise gated linear attention forward, bf16 inputs.
 *
 * Computes, for every batch b and head h, the recurrence over the scan order of
 * direction `dir` (DiG: "gated linear attention", S_t = Diag(alpha_t) S_{t-1} +
 * k_t^T v_t, o_t = q_t S_t; chunk-wise parallel form, DiG paper notes "硬件友好的
 * 效率设计": the sequence is cut into chunks processed in on-chip memory):
 *     S_0 = 0 (dk x dv),  alpha_{t,i} = exp(log_alpha[b][t][h][i])
 *     S  <- Diag(alpha_t) S + k_t^T v_t      (gate per key channel, broadcast over dv)
 *     out[b][t][h][:] = q_t S                (read after the update)
 * The output of token t is written at t (canonical position) for every dir.
 * No feature map, normaliser or 1/sqrt(dk) is applied: pre-scale q, k, v.
 *
 *   q, k       [B][T][H][dk] bf16        log_alpha [B][T][H][dk] fp32
 *   v          [B][T][H][dv] bf16        out       [B][T][H][dv] bf16 (written)
 *   dk, dv     multiples of 8 in [8, 128]
 *   dir        GLA_DIR_* (0..3), or GLA_DIR_ZIGZAG0 + j (j = 0..7)
 * Arithmetic: tensor-core products of bf16 operands with fp32 accumulation; the
 * chunk state and all gate arithmetic are fp32; out is rounded to nearest even.
 * Gates: any log_alpha <= 0 is handled, -inf (a full reset of the channel)
 * included.  Chunks of 128 positions whose gates decay by more than e^80 inside
 * the chunk are evaluated token by token (exact, slower).  Growth gates
 * (log_alpha > 0) whose product exceeds e^80 inside a chunk cannot be represented
 * in fp32: GLA_ERR_RANGE is recorded in the device status.
 * Workspace: stream-ordered, from a per-device pool of the library (cudaMallocFromPoolAsync;
 * the pool keeps its memory across synchronisations), freed on the same stream.
 * `out` must not overlap any input.
 */
int gla_fwd(const void* q, const void* k, const void* v, const float* log_alpha, int B, int H, int Hgrid,
            int Wgrid, int dk, int dv, int dir, void* out, cudaStream_t stream);

/*
 * gla_fwd_glogit -- gla_fwd with the forget gate given as bf16 logits g instead of
 * fp32 log_alpha: log_alpha = logsigmoid(g) / gate_norm, computed inside the kernel
 * from the bf16 tile (the gate definition of the GLA configurations, gate_norm = 16),
 * so log_alpha is never written or read in fp32: the gate costs 2 bytes per key
 * channel per token instead of 4.
 *   g          [B][T][H][dk] bf16 (the layout of q)
 *   gate_norm  > 0
 *   dk, dv     multiples of 8 in [8, 120]; dir 0..3 (the SREM orders)
 * Everything else -- shapes, arithmetic, output, errors, workspace -- as gla_fwd.
 * The logsigmoid is evaluated with the hardware base-2 exponential and logarithm
 * (relative error about 2^-22) in the suffix-sum warps; the token-serial fallback
 * uses expf / log1pf.  No output may overlap an input.
 */
int gla_fwd_glogit(const void* q, const void* k, const void* v, const void* g, int B, int H, int Hgrid, int Wgrid,
                   int dk, int dv, int dir, float gate_norm, void* out, cudaStream_t stream);

/*
 * gla_fwd_f32 -- the same recurrence with fp32 q, k, v and out (all arithmetic
 * fp32, no tensor-core rounding).  Same shapes, directions and errors as gla_fwd.
 */
int gla_fwd_f32(const float* q, const float* k, const float* v, const float* log_alpha, int B, int H,
                int Hgrid, int Wgrid, int dk, int dv, int dir, float* out, cudaStream_t stream);

/*
 * gla_fwd_f32_noalloc -- gla_fwd_f32 without any device allocation.  The paper
 * has no counterpart: this is a library convenience.
 *
 * For callers that cannot call cudaMalloc / cudaMallocAsync while they run the
 * GLA: a host framework that owns every device allocation through its own pool
 * and forbids foreign ones, a real-time or embedded program that allocates
 * everything at start-up because allocating may block or synchronise the device,
 * or work recorded into a CUDA graph that must not contain memory nodes.  The
 * caller passes the inputs and the output exactly as for gla_fwd_f32 (same
 * shapes, directions, arithmetic and result); the scratch lives in a fixed
 * array of DIG_GLA_NOALLOC_SCRATCH_BYTES (8 MiB) of device memory inside the
 * library, which every GPU that loads the library holds until the process exits.
 *
 *   - Capacity: with n = B*H*ceil(T/64) and rup(x) = x rounded up to a multiple
 *     of 256, the call needs
 *         2*rup(n*dk*dv*4) + rup(n*dk*4) + rup(n*4)
 *     bytes of scratch, at most DIG_GLA_NOALLOC_SCRATCH_BYTES; a larger problem
 *     returns GLA_ERR_UNSUPPORTED and launches nothing.  (B=2, H=6, T=256, d=64
 *     needs about 1.6 MB; B=H=1, dk=dv=128 fits up to T=4032.)
 *   - First call per device: it looks up the array's device address with
 *     cudaGetSymbolAddress (with that device current) and caches it.  Make this
 *     first call before any stream capture.  Call dig_gla_release() before a
 *     cudaDeviceReset: a new context places the array at a new address.
 *   - Sharing: every call uses the same array, which keeps the last call's
 *     contents; nothing in it needs to start at zero.  Calls that overlap on the
 *     GPU (concurrent streams, or host threads launching at the same time) race on
 *     the array and corrupt each other's results: serialise them.
 *   - Allocates nothing and frees nothing, on the host or the device.
 */
#define DIG_GLA_NOALLOC_SCRATCH_BYTES (8u << 20)
int gla_fwd_f32_noalloc(const float* q, const float* k, const float* v, const float* log_alpha, int B, int H,
                        int Hgrid, int Wgrid, int dk, int dv, int dir, float* out, cudaStream_t stream);

/*
 * gla_bwd -- gradients of the chunk-wise GLA forward, bf16 q, k, v, dout.
 *
 * DiG is trained like DiT (DiG paper notes, "损失函数 / 训练策略"), so every GLA
 * layer is differentiated; the notes' complexity claim for the chunk-wise form
 * ("硬件友好的效率设计") covers training.  Given dout = dL/dout for
 * out = gla_fwd(q, k, v, log_alpha, ..., dir), writes the exact gradients of L
 * (through the same recurrence, the same scan order and S_0 = 0):
 *   dq, dk        [B][T][H][dk] bf16        dv [B][T][H][dv] bf16
 *   dlog_alpha    [B][T][H][dk] fp32        (d L / d log_alpha, not d alpha)
 * from q, k [B][T][H][dk] bf16, v and dout [B][T][H][dv] bf16 and log_alpha
 * [B][T][H][dk] fp32, all at canonical token positions.
 * Arithmetic: for dk, dv <= 80, chunks of M = 128 scan positions whose products run
 * on tensor cores from bf16 operands (the gated q and k, the masked dout v^T and
 * q k^T scores, the carried state and its gradient, each rounded to bf16) with fp32
 * accumulation; gate sums, scans over chunks and d log_alpha in fp32.  Wider heads:
 * chunks of M = 32 with every product in fp32 on CUDA cores.  dq, dk, dv rounded to
 * nearest even on the store.  A chunk whose gates decay by more than e^80 inside it
 * (a full reset, -inf) is differentiated token by token in fp32 (exact, slower).
 * Growth gates whose product exceeds e^80 inside a chunk record GLA_ERR_RANGE.
 * Shapes, dims, directions and errors as gla_fwd; no output may overlap an input or
 * another output.  Workspace: 2 * B*H*ceil(T/M) * dk*dv fp32 values plus per-chunk
 * gates (130 MB for B=2, H=16, T=12544, d=72), stream-ordered from the library's
 * pool as gla_fwd's; zigzag orders add copies of the nine tensors in scan order.
 */
int gla_bwd(const void* q, const void* k, const void* v, const float* log_alpha, const void* dout, int B, int H,
            int Hgrid, int Wgrid, int dk, int dv, int dir, void* dq, void* dk_out, void* dv_out, float* dlog_alpha,
            cudaStream_t stream);

/*
 * gla_bwd_f32 -- gla_bwd with fp32 q, k, v, dout, dq, dk, dv: every product and sum
 * in fp32 on CUDA cores (chunks of M = 32), no rounding on the store.
 */
int gla_bwd_f32(const float* q, const float* k, const float* v, const float* log_alpha, const float* dout, int B,
                int H, int Hgrid, int Wgrid, int dk, int dv, int dir, float* dq, float* dk_out, float* dv_out,
                float* dlog_alpha, cudaStream_t stream);

/*
 * gla_norm_fwd -- the normalised variant of the diffusers draft (page 4,
 * `gated_linear_attention`), bf16 q, k, v, out.
 *
 * Per (batch, head), over the scan order of `dir`, from S = 0 (dk x dv), z = 0 (dk):
 *   phi(x) = elu(x) + 1 (x + 1 above zero, e^x otherwise), g_t = sigmoid(q_t * k_t)
 *   per key channel (of the raw q and k), S <- Diag(g_t) S + phi(k_t)^T v_t,
 *   z <- g_t * z + phi(k_t),  out_t = (phi(q_t) S) / max(phi(q_t) . z, eps).
 * q, k [B][T][H][dk] bf16; v, out [B][T][H][dv] bf16; dk multiple of 8 in [8, 128],
 * dv multiple of 8 in [8, 120]; eps > 0 (the draft uses 1e-6); dir as gla_fwd.
 * Arithmetic: fp32 throughout (features, gates and the chunk-wise recurrence, whose
 * denominator is a ones column appended to v); out rounded to nearest even.
 * Workspace: about (3*dk + 2*(dv+8)) fp32 values per token-head plus the fp32
 * forward's.  `out` must not overlap an input.  Errors as gla_fwd.
 */
int gla_norm_fwd(const void* q, const void* k, const void* v, int B, int H, int Hgrid, int Wgrid, int dk, int dv,
                 int dir, float eps, void* out, cudaStream_t stream);

/* gla_norm_fwd_f32 -- the same with fp32 q, k, v, out. */
int gla_norm_fwd_f32(const float* q, const float* k, const float* v, int B, int H, int Hgrid, int Wgrid, int dk,
                     int dv, int dir, float eps, float* out, cudaStream_t stream);

/*
 * srem_reorient -- SREM's change of scan direction as an explicit row gather
 * (DiG paper notes, SREM: the block ends by transposing the 2D token matrix and
 * flipping the sequence, both O(T) operations; DiG Block step (5)).
 *   inverse = 0:  y[b][p][:] = x[b][order_dir(p)][:]   (canonical -> scan order)
 *   inverse = 1:  y[b][order_dir(p)][:] = x[b][p][:]   (scan order -> canonical)
 * where order_dir(p) is the raster token visited at scan position p (dir 0..11).
 *   x, y   [B][T][C] elements of `dtype` (GLA_BF16 or GLA_F32); C*sizeof(elt)
 *          must be a multiple of 16 bytes.  Bit-exact copy.  y must not overlap x.
 */
int srem_reorient(const void* x, int dir, int inverse, int B, int Hgrid, int Wgrid, int C, int dtype, void* y,
                  cudaStream_t stream);

/*
 * dwconv3x3 -- SREM's 3x3 depthwise convolution on the 2D token grid (DiG paper
 * notes, SREM and DiG Block step (4): DWConv2d after reshaping the sequence to
 * 2D, identity-initialised):
 *   y[b][r][c][ch] = sum_{i,j in {-1,0,1}} w[ch][i+1][j+1] * x[b][r+i][c+j][ch]
 * with zero padding outside the grid (cross-correlation, no kernel flip, no bias).
 *   x, y   [B][Hgrid][Wgrid][C] of `dtype` (GLA_BF16 or GLA_F32), channels-last;
 *          C*sizeof(elt) must be a multiple of 16 bytes.  y must not overlap x.
 *   w      [C][3][3] fp32.
 * Accumulation is fp32; a bf16 result is rounded to nearest even.
 */
int dwconv3x3(const void* x, const float* w, int B, int Hgrid, int Wgrid, int C, int dtype, void* y,
              cudaStream_t stream);

/*
 * dig_gla_device_status -- synchronises `stream`, then returns and clears the
 * current device's status word: GLA_OK, or the first GLA_ERR_TIMEOUT /
 * GLA_ERR_RANGE a kernel recorded since the last call.  Returns GLA_ERR_CUDA if
 * the synchronisation itself fails.
 */
int dig_gla_device_status(cudaStream_t stream);

/* Human-readable name of a gla_status_t value (static storage). */
const char* dig_gla_status_string(int status);

/*
 * dig_gla_release -- forgets cached host-side state (device checks, the device
 * addresses of gla_fwd_f32_noalloc's scratch array) and destroys the library's
 * per-device memory pools, returning their memory to the device.  The GLA scratch
 * comes from such a pool, which keeps its memory across stream synchronisations so
 * that repeated calls do not map it again; scratch of calls still in flight stays
 * allocated until they complete.  Call it before cudaDeviceReset (the cached pools
 * and addresses belong to the context being destroyed); later calls set up anew.
 */
void dig_gla_release(void);

/*
 * dig_gla_test_skip_items -- test hook for gla_fwd's bounded waits (bf16 path only).
 * The next gla_fwd call of this process starts its work-item counter at n instead of
 * 0, so its first n items (segments of 3 chunks, taken segment-major over B*H) are
 * never processed and never publish their look-back flags; the waits of later
 * segments on those flags run out after about a second of GPU time.  That call
 * returns GLA_OK, dig_gla_device_status then reports GLA_ERR_TIMEOUT, and its output
 * is unspecified; the CUDA context stays usable and later calls are unaffected.
 * n <= 0 clears a pending request.
 */
void dig_gla_test_skip_items(int n);

#ifdef __cplusplus
}
#endif

#endif /* DIG_GLA_H_ */
