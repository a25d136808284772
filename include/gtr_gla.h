/*
 * gtr_gla.h -- C ABI of the B200 (sm_100a) Key-only gated linear attention
 * token mixer of GTR.
 *
 * Operator (GTR article "端侧实时感知新标杆！通用线性骨干网络GTR开源",
 * shuwu5.cn/article/3124, 方法详解 §1 "骨干架构：Key-only 门控递归与四向交替扫描";
 * the page's formulas were lost in extraction, the surviving prose fixes this
 * reading): for every batch entry b and head h, scanning the grid_h x grid_w
 * token grid in one direction,
 *
 *     S_s = diag(exp(g_s)) S_{s-1} + k_s^T v_s          (dk x dv state, S_-1 = 0)
 *     o_s = q_s S_s
 *     y_s = o_s / sqrt(mean(o_s^2) + 1e-5) * w * SiLU(z_s)
 *
 * with the value-side decay fixed to 1 and the key-side forget gate
 *
 *     g = logsigmoid(x W_down W_up + bias) / tau          (low-rank projection)
 *
 * computed by gtr_gate_fwd.  gtr_gla_fwd evaluates the recurrence chunk by
 * chunk in three stages (方法详解 §4 "硬件感知分块推理算子": chunk summaries on
 * tensor cores, a light sequential pass over chunk-boundary states, chunk
 * outputs with the output gate fused into the epilogue).
 *
 * Scan orders (方法详解 §1, four alternating directions, grid order restored
 * after the scan).  Sequence position s visits grid index t = row*grid_w + col:
 *     GTR_LR: t = s                                   (row-major raster)
 *     GTR_RL: t = T-1-s                               (LR reversed)
 *     GTR_TB: t = (s mod grid_h)*grid_w + s/grid_h    (down each column, columns left to right)
 *     GTR_BT: TB reversed
 *     GTR_ROTATE_BATCH: batch entry b uses direction (b mod 4) of the four above.
 * Output y is stored at the grid index its token came from, so every tensor
 * stays in grid order.
 *
 * Conventions shared by every entry point
 *   - Tensors are caller-owned DEVICE pointers, C-contiguous, in grid order:
 *       q, k, g      : [B, T, H, dk]     (T = grid_h * grid_w)
 *       v, z, out    : [B, T, H, dv]
 *       x            : [B, T, d_model]
 *     q, k, v, z and out share one element type `dtype` (gtr_dtype_t); the gate
 *     tensor g is always fp32.  Every tensor pointer must be 16-byte aligned.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Calls are asynchronous on it, never synchronise and launch no
 *     work on any other stream.
 *   - Errors are returned as a gtr_status_t; nothing is thrown and no device
 *     trap is raised.  All argument checks run before any launch; a rejected
 *     call launches nothing.  A launch failure maps to GTR_ERR_CUDA.
 *   - Sizes of zero (B, H, grid_h or grid_w == 0) are an empty problem:
 *     GTR_OK, nothing launched, pointers unused.  Negative sizes are invalid.
 */
#ifndef GTR_GLA_H
#define GTR_GLA_H

#include <stddef.h>

#if defined(__GNUC__) || defined(__clang__)
#define GTR_API __attribute__((visibility("default")))
#else
#define GTR_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GTR_OK = 0,
    GTR_ERR_INVALID_ARG = -1,   /* null pointer, negative size, bad enum, overflow */
    GTR_ERR_UNSUPPORTED = -2,   /* valid but not implemented (head dim, chunk, rank) */
    GTR_ERR_ALIGNMENT = -3,     /* a tensor pointer is not 16-byte aligned */
    GTR_ERR_NO_MEMORY = -4,     /* workspace could not be obtained */
    GTR_ERR_CUDA = -5,          /* a CUDA runtime call or launch failed */
    GTR_ERR_DEVICE_CHECK = -6   /* a device-side check recorded a failure */
} gtr_status_t;

typedef enum { GTR_F32 = 0, GTR_F16 = 1, GTR_BF16 = 2 } gtr_dtype_t;

typedef enum { GTR_LR = 0, GTR_RL = 1, GTR_TB = 2, GTR_BT = 3, GTR_ROTATE_BATCH = 4 } gtr_dir_t;

/* Kernel families gtr_gla_fwd can run (see gtr_gla_set_path). */
typedef enum {
    GTR_PATH_AUTO = 0,  /* tensor-core path where supported, else SIMT */
    GTR_PATH_SIMT = 1,  /* exact fp32 CUDA-core path, every dtype and head dim */
    GTR_PATH_TC = 2     /* tcgen05/TMEM path: 16-bit dtypes, chunk 64, dk = dv = 64 or 128 */
} gtr_path_t;

#define GTR_ABI_VERSION 1

/* ABI version of the loaded library (GTR_ABI_VERSION). */
GTR_API int gtr_abi_version(void);

/* Static text for a status code; never NULL. */
GTR_API const char *gtr_status_string(int status);

/*
 * Gate projection (GTR article 方法详解 §1, low-rank forget gate with
 * temperature):  g[n, j] = logsigmoid(sum_r (x[n,:] . w_down[:,r]) w_up[r,j]
 *                                      + bias[j]) / tau,    j < H*dk.
 *   x       [B*T, d_model] in x_dtype (gtr_dtype_t)
 *   w_down  [d_model, rank] fp32, w_up [rank, H*dk] fp32, bias [H*dk] fp32 or
 *           NULL (zero), g_out [B*T, H*dk] fp32 = the [B, T, H, dk] gate of
 *           gtr_gla_fwd.  logsigmoid uses the overflow-free form
 *           min(u,0) - log1p(exp(-|u|)), so g <= 0 always.
 *   Limits: 1 <= rank <= 64, d_model <= 4096, H*dk <= 4096, tau > 0 finite.
 *   For 16-bit x with the tensor-core shapes (see gtr_gate_pack) it packs the
 *   weights into a buffer cached per (device, stream) -- allocated with
 *   cudaMalloc by the first such call on a stream, which must not happen
 *   during stream capture -- and runs gtr_gate_fwd_packed.
 */
GTR_API gtr_status_t gtr_gate_fwd(const void *x, int x_dtype, const float *w_down, const float *w_up,
                          const float *bias, float *g_out, int B, int T, int d_model, int rank,
                          int H, int dk, float tau, void *stream);

/*
 * Packed gate weights for the tensor-core gate kernel.  The weights of a
 * model are fixed while it runs, so their preparation (splitting W_down and
 * W_up into the power-of-two-scaled multi-term 16-bit operand tiles the
 * kernel multiplies, in its shared-memory byte layout) can be done once and
 * reused by every gtr_gate_fwd_packed call.
 *   gtr_gate_packed_bytes: size of a packed weight buffer.
 *   gtr_gate_pack: w_down [d_model, 16] and w_up [16, H*dk] fp32 (as in
 *     gtr_gate_fwd) -> `packed`, a caller-owned device buffer of at least
 *     gtr_gate_packed_bytes() bytes, 16-byte aligned, written asynchronously
 *     on `stream`.  x_dtype (GTR_F16 or GTR_BF16) is the type of the x it
 *     will multiply.  Shapes: rank 16, d_model a multiple of 64 up to 384,
 *     H*dk a multiple of 64 up to 448; others return GTR_ERR_UNSUPPORTED.
 *   gtr_gate_fwd_packed: gtr_gate_fwd with packed weights (made for the same
 *     x_dtype, d_model, rank, H, dk); additionally B*T < 2^31.
 *   Errors: GTR_ERR_INVALID_ARG (NULL pointer, bad sizes), GTR_ERR_UNSUPPORTED
 *   (shape), GTR_ERR_NO_MEMORY (packed_bytes too small), GTR_ERR_ALIGNMENT,
 *   GTR_ERR_CUDA (launch or tensor-map failure).
 */
GTR_API size_t gtr_gate_packed_bytes(void);
GTR_API gtr_status_t gtr_gate_pack(const float *w_down, const float *w_up, int x_dtype, int d_model,
                           int rank, int H, int dk, void *packed, size_t packed_bytes,
                           void *stream);
GTR_API gtr_status_t gtr_gate_fwd_packed(const void *x, int x_dtype, const void *packed,
                                 const float *bias, float *g_out, int B, int T, int d_model,
                                 int rank, int H, int dk, float tau, void *stream);

/*
 * Key-only GLA forward with the fused RMSNorm x SiLU output gate (GTR article
 * 方法详解 §1 and §4; see the top of this file for the exact definition).
 *   q, k [B,T,H,dk], v, outgate (= z), out [B,T,H,dv] in `dtype`; g [B,T,H,dk]
 *   fp32 (log forget gate, expected <= 0; values > 0 are computed as given);
 *   rms_w [dv] fp32 or NULL (all ones), shared by all heads.
 *   dk, dv in {16, 32, 64, 128}; chunk (the chunk length C) in {16, 32, 64,
 *   128}; the result does not depend on C beyond rounding.  T = grid_h*grid_w
 *   must fit in an int.  `out` must not alias any input.
 *   Kernels: tcgen05 tensor-core kernels for 16-bit dtypes with chunk 64 and
 *   dk = dv = 64 or 128 (segments of chunks walked with the state on chip,
 *   one fp32 state per segment in the workspace); the exact fp32 CUDA-core
 *   kernels otherwise.
 *   Workspace: fp32 segment states taken from a library-owned buffer cached
 *   per (device, stream) and grown on demand with cudaMalloc (so the first call
 *   for a shape must not happen during stream capture), or from the buffer
 *   registered with gtr_gla_set_workspace.  Calls on one stream are ordered;
 *   calls that share a registered workspace on different streams race.
 */
GTR_API gtr_status_t gtr_gla_fwd(const void *q, const void *k, const void *v, const float *g,
                         const void *outgate, const float *rms_w, void *out, int B, int H,
                         int grid_h, int grid_w, int dk, int dv, int dir, int chunk, int dtype,
                         void *stream);

/*
 * gtr_gla_fwd for callers that cannot allocate device memory while they run
 * (the paper has no counterpart to this entry point).  Examples: a plugin
 * inside an inference engine that forbids allocation once execution starts, a
 * real-time loop whose memory footprint is fixed at start-up, or a process
 * under a hard memory cap.  cudaMalloc can block on the device and fail when
 * memory runs out, so such callers cannot use the workspace gtr_gla_fwd grows
 * on demand.  Same arguments and result as gtr_gla_fwd; this call allocates
 * nothing and calls no allocating routine.
 *   Scratch: a static device array of GTR_NOALLOC_SCRATCH_BYTES (8 MiB) that
 *   a GPU holds from the library's first call on it until the process exits
 *   (the CUDA runtime loads the library's device code onto a GPU lazily, at
 *   its first kernel launch or symbol lookup there, and the array comes with
 *   it).  A caller that must not allocate later should therefore make one
 *   call on each device at start-up, before memory fills up and before any
 *   stream capture; if the array cannot be placed the call returns
 *   GTR_ERR_NO_MEMORY.  The
 *   boundary states need B*H*nseg*(dk*dv + dk)*4 bytes; when the usual segment
 *   plan needs more, longer segments are used (same result up to rounding).
 *   If even one segment per sequence does not fit, i.e.
 *   B*H*(dk*dv + dk)*4 + 256 > 8 MiB, the call returns GTR_ERR_NO_MEMORY and
 *   launches nothing.
 *   The first call on a device also looks up the array's device address
 *   (once per device, with that device current).
 *   All calls share the one array and it keeps the last call's contents;
 *   nothing in it needs to start at zero (every element is written before it
 *   is read within a call).  Calls whose work overlaps on the GPU (other
 *   streams, or other host threads) race on the array and give wrong results:
 *   order them.
 */
#define GTR_NOALLOC_SCRATCH_BYTES (8u << 20)
GTR_API gtr_status_t gtr_gla_fwd_noalloc(const void *q, const void *k, const void *v,
                                         const float *g, const void *outgate, const float *rms_w,
                                         void *out, int B, int H, int grid_h, int grid_w, int dk,
                                         int dv, int dir, int chunk, int dtype, void *stream);

/*
 * gtr_gla_fwd that also records caller-created cudaEvent_t handles (any may be
 * NULL) on `stream`: ev[0] before the summary kernel, ev[1] after it, ev[2]
 * after the state scan, ev[3] after the output kernel.  For profiling only.
 */
GTR_API gtr_status_t gtr_gla_fwd_timed(const void *q, const void *k, const void *v, const float *g,
                               const void *outgate, const float *rms_w, void *out, int B, int H,
                               int grid_h, int grid_w, int dk, int dv, int dir, int chunk,
                               int dtype, void *stream, void *const *ev);

/*
 * Gate projection and GLA forward of one token mixer in one call:
 *     g_out = logsigmoid(x W_down W_up + bias) / tau        (as gtr_gate_fwd_packed)
 *     out   = gtr_gla_fwd(q, k, v, g_out, outgate, rms_w)
 * (GTR article 方法详解 §1, the low-rank key-side gate, and §4).
 *   x [B, T, d_model] in x_dtype; `packed`: W_down and W_up from gtr_gate_pack
 *   for this x_dtype, d_model, rank, H, dk (so the shapes gtr_gate_pack takes);
 *   bias [H*dk] fp32 or NULL; tau > 0.  q, k, v, outgate, rms_w, out, the sizes,
 *   dir, chunk and dtype as in gtr_gla_fwd; g_out [B, T, H, dk] fp32 receives g
 *   (the output stage reads it back; it must not alias another argument).
 *   Where gtr_gla_fwd takes its tensor-core path with dk = dv = 64 (chunk 64,
 *   16-bit dtype) the gate is split at its rank-16 bottleneck: one kernel writes
 *   x W_down ([B*T, 16] fp32, 64 bytes per token, in the workspace, which
 *   therefore grows by B*T*64 bytes), and the summary kernel forms g chunk by
 *   chunk from it, so the gate costs no pass of its own over g.  g_out and
 *   out equal those of gtr_gate_fwd_packed followed by gtr_gla_fwd up to
 *   rounding.  Other shapes run exactly those two calls.
 *   Errors as gtr_gate_fwd_packed and gtr_gla_fwd; B*T must be below 2^31.
 */
GTR_API gtr_status_t gtr_gla_fwd_gated(const void *x, int x_dtype, const void *packed,
                                       const float *bias, int d_model, int rank, float tau,
                                       const void *q, const void *k, const void *v,
                                       const void *outgate, const float *rms_w, float *g_out,
                                       void *out, int B, int H, int grid_h, int grid_w, int dk,
                                       int dv, int dir, int chunk, int dtype, void *stream);

/*
 * gtr_gla_fwd_gated that also records caller-created cudaEvent_t handles (any
 * may be NULL) on `stream`: ev[0] before the gate kernel, ev[1] after it, ev[2]
 * after the summary kernel, ev[3] after the state scan, ev[4] after the output
 * kernel.  For profiling only.
 */
GTR_API gtr_status_t gtr_gla_fwd_gated_timed(const void *x, int x_dtype, const void *packed,
                                             const float *bias, int d_model, int rank, float tau,
                                             const void *q, const void *k, const void *v,
                                             const void *outgate, const float *rms_w,
                                             float *g_out, void *out, int B, int H, int grid_h,
                                             int grid_w, int dk, int dv, int dir, int chunk,
                                             int dtype, void *stream, void *const *ev);

/*
 * The token mixer's projections on either side of the GLA (GTR article
 * 方法详解 §1: q, k, v and the output gate z are linear maps of the block input
 * x, and the mixer output is mapped back to the model width).  Plain dense
 * GEMMs with fp32 accumulation on the library's tcgen05 GEMM kernel (128 x 128
 * output tiles, operands staged by TMA, accumulators in tensor memory).  Row
 * pitches or column blocks that are not multiples of 8 elements go to cuBLAS,
 * which the library then loads with dlopen (GTR_ERR_UNSUPPORTED if it cannot
 * be loaded; make such a first call on a device outside stream capture).
 * 16-bit dtype only
 * (GTR_F16 or GTR_BF16; GTR_F32 is GTR_ERR_UNSUPPORTED); every pointer a
 * device pointer, 16-byte aligned, row-major.
 *   gtr_mixer_in_proj: x [B*T, d_model], w_in [d_model, 2 H dk + 2 H dv] whose
 *     column blocks are W_q | W_k | W_v | W_z -> q = x W_q, k = x W_k ([B, T, H,
 *     dk]), v = x W_v, z = x W_z ([B, T, H, dv]), rounded to dtype.  When dk ==
 *     dv and H dk is a multiple of 128 the four products are one launch with
 *     four outputs, else one launch each.
 *   gtr_mixer_out_proj: out [N, d_out] = y [N, d_in] w_out [d_in, d_out].
 *   Sizes of zero are an empty problem (GTR_OK, nothing launched).
 */
GTR_API gtr_status_t gtr_mixer_in_proj(const void *x, const void *w_in, void *q, void *k, void *v,
                                       void *z, int B, int T, int d_model, int H, int dk, int dv,
                                       int dtype, void *stream);
GTR_API gtr_status_t gtr_mixer_out_proj(const void *y, const void *w_out, void *out, long long N,
                                        int d_in, int d_out, int dtype, void *stream);

/*
 * The Spatial SwiGLU feed-forward block of a GTR layer (GTR article, 方法详解
 * §2, Spatial SwiGLU): the channel expansion u = x W_in holds a gate branch and
 * a value branch; the value branch, laid out as the 2-D token grid, is mixed by
 * a depthwise convolution with zero padding (output grid = input grid); the
 * result is multiplied by SiLU of the gate branch and projected back:
 *     h[b,y,x,c] = SiLU(u[b,y,x,c]) * (bias[c] + sum_{i,j} conv_w[i,j,c] * u[b,y+i-1,x+j-1,C+c]),
 *     y_out = h W_out.
 * The pages leave the kernel size blank; ksize must be 3 (other odd sizes are
 * GTR_ERR_UNSUPPORTED, even or non-positive ones GTR_ERR_INVALID_ARG).
 * Tokens are in grid order, t = row * grid_w + column.  dtype GTR_F16 or
 * GTR_BF16 for every activation and projection weight (GTR_F32 is
 * GTR_ERR_UNSUPPORTED); C (the hidden width) a multiple of 8, else
 * GTR_ERR_UNSUPPORTED.  Every pointer is a device pointer, 16-byte aligned
 * (GTR_ERR_ALIGNMENT otherwise), owned by the caller; the call launches on
 * `stream` and returns without synchronising.  Sizes of zero are an empty
 * problem (GTR_OK, nothing launched).
 *   gtr_sswiglu_mix: u [B, T, 2C] (gate channels [0, C), value channels [C, 2C)),
 *     conv_w [3, 3, C] fp32 (tap (i, j) = kernel row i, column j), conv_b [C]
 *     fp32 or NULL (no bias) -> h [B, T, C], fp32 arithmetic, rounded once to
 *     dtype.  One kernel; an h that overlaps u is GTR_ERR_INVALID_ARG.
 *   gtr_sswiglu_fwd: x [B*T, d_model], w_in [d_model, 2C], w_out [C, d_model]
 *     -> y [B*T, d_model]; u [B*T, 2C] and h [B*T, C] are caller-provided
 *     scratch that receive the expansion and the hidden activation.  The two
 *     projections run on the GEMM of gtr_mixer_in_proj (fp32 accumulation,
 *     the same cuBLAS fallback).  C = 0 writes y = 0.
 */
GTR_API gtr_status_t gtr_sswiglu_mix(const void *u, const float *conv_w, const float *conv_b, void *h,
                                     int B, int grid_h, int grid_w, int C, int ksize, int dtype,
                                     void *stream);
GTR_API gtr_status_t gtr_sswiglu_fwd(const void *x, const void *w_in, const float *conv_w,
                                     const float *conv_b, const void *w_out, void *u, void *h, void *y,
                                     int B, int grid_h, int grid_w, int d_model, int C, int ksize,
                                     int dtype, void *stream);

/*
 * A stack of GTR blocks (GTR article, 方法详解 §1: the single-scale backbone of
 * 12 blocks, each built around the Key-only GLA, block i scanning in direction
 * LR, RL, TB, BT for i mod 4 = 0, 1, 2, 3; 方法详解 §2: the Spatial SwiGLU
 * feed-forward half).  The pages leave the wiring blank; each block here is
 *     a = RMSNorm(x) * norm_mixer
 *     x += GLA(a W_q, a W_k, a W_v, gate(a), a W_z) W_o     (gla_norm on the GLA output)
 *     c = RMSNorm(x) * norm_ffn
 *     x += S-SwiGLU(c)                                      (as gtr_sswiglu_fwd, 3x3 taps)
 * with RMSNorm's epsilon 1e-5, gate(a) = logsigmoid(a W_down W_up + bias)/tau
 * at rank 16, and no normalisation after the last block.
 *
 * x [B, grid_h*grid_w, d_model] fp32 (grid order) is the residual stream,
 * updated in place.  Every other activation is kept in `dtype` (GTR_F16 or
 * GTR_BF16; GTR_F32 is GTR_ERR_UNSUPPORTED) in the caller's workspace of
 * gtr_stack_workspace_bytes bytes (GTR_ERR_NO_MEMORY if smaller), 16-byte
 * aligned.  blocks is a HOST array of nblocks entries whose members are
 * device pointers owned by the caller; 16-bit members are in `dtype`, the
 * others fp32; gate_packed is gtr_gate_pack's output for that block's W_down
 * [d_model, 16] and W_up [16, H dk] with x_dtype = dtype.  dirs is a host array
 * of nblocks directions (GTR_LR .. GTR_BT) or NULL for the rotation above.
 * The GLA stage takes gtr_gla_fwd's workspace for `stream` (grown at its first
 * use on that stream), so capture a stack into a CUDA graph only after one
 * uncaptured call on the capturing stream.  Shapes: d_model a multiple of 64
 * up to 384 and H dk a multiple of 64 up to 448 (the packed gate), dk, dv in
 * {16, 32, 64, 128}, hidden a multiple of 8, chunk in {16, 32, 64, 128}; every
 * stage's shape check runs before the first launch (GTR_ERR_UNSUPPORTED or
 * GTR_ERR_INVALID_ARG, nothing launched), as do the pointer and alignment
 * checks.  A CUDA error in a later stage returns GTR_ERR_CUDA with x partly
 * updated.  nblocks = 0 or an empty grid is GTR_OK with nothing launched.
 * Launches on `stream` and returns without synchronising.
 */
typedef struct gtr_block_weights {
  const float *norm_mixer; /* [d_model] RMSNorm weight before the token mixer */
  const void *w_in;        /* [d_model, 2 H dk + 2 H dv]: W_q | W_k | W_v | W_z */
  const void *gate_packed; /* gtr_gate_pack output (W_down, W_up of this block) */
  const float *gate_bias;  /* [H dk] or NULL */
  const float *gla_norm;   /* [dv] RMSNorm weight of the GLA output, or NULL (ones) */
  const void *w_o;         /* [H dv, d_model] */
  const float *norm_ffn;   /* [d_model] RMSNorm weight before the S-SwiGLU half */
  const void *w_e;         /* [d_model, 2 hidden]: gate channels, then value channels */
  const float *conv_w;     /* [3, 3, hidden] depthwise taps */
  const float *conv_b;     /* [hidden] or NULL */
  const void *w_p;         /* [hidden, d_model] */
} gtr_block_weights;

/* Workspace bytes of gtr_stack_fwd (0 for negative sizes). */
GTR_API size_t gtr_stack_workspace_bytes(int B, int grid_h, int grid_w, int d_model, int H, int dk, int dv,
                                         int hidden);
GTR_API gtr_status_t gtr_stack_fwd(float *x, const gtr_block_weights *blocks, int nblocks, const int *dirs,
                                   int B, int grid_h, int grid_w, int d_model, int H, int dk, int dv,
                                   int hidden, float tau, int chunk, int dtype, void *workspace,
                                   size_t workspace_bytes, void *stream);

/*
 * Chunk-boundary states, for testing the first two stages on their own: the
 * state each chunk of `chunk` scan positions ends with,
 *   states [B, H, ceil(T/chunk), dk, dv] fp32, entry c = S after scan position
 *   min((c+1)*chunk, T) - 1 (GTR article 方法详解 §4, boundary states).
 * Runs the summary and scan stages with one chunk per segment on `stream`.
 */
GTR_API gtr_status_t gtr_gla_chunk_states(const void *k, const void *v, const float *g, float *states,
                                  int B, int H, int grid_h, int grid_w, int dk, int dv, int dir,
                                  int chunk, int dtype, void *stream);

/* Bytes of workspace gtr_gla_fwd needs for this problem on the current device
 * (0 for an empty problem, (size_t)-1 for invalid arguments). */
GTR_API size_t gtr_gla_workspace_bytes(int B, int H, int grid_h, int grid_w, int dk, int dv, int chunk,
                               int dtype);

/* The segment plan gtr_gla_fwd would use for this problem on the current
 * device.  A segment is the run of consecutive chunks one block of the summary
 * and output kernels walks through; segment s of n covers chunks
 * [s*nc/n, (s+1)*nc/n) of the sequence's nc chunks (an even split).
 * gtr_gla_segment_chunks: chunks in the longest segment; gtr_gla_segment_count:
 * segments per sequence.  0 for an empty problem, or a negative status. */
GTR_API int gtr_gla_segment_count(int B, int H, int grid_h, int grid_w, int dk, int dv, int chunk,
                                  int dtype);
GTR_API int gtr_gla_segment_chunks(int B, int H, int grid_h, int grid_w, int dk, int dv, int chunk,
                                   int dtype);

/* Register a caller-owned device buffer as the workspace of the current device
 * (ptr 256-byte aligned).  NULL releases it: calls go back to the
 * library-owned buffers.  The caller keeps ownership and must keep the buffer
 * alive while calls that use it are in flight. */
GTR_API gtr_status_t gtr_gla_set_workspace(void *ptr, size_t bytes);

/* Select the kernel family (gtr_path_t) of later gtr_gla_fwd calls in this
 * process; GTR_ERR_UNSUPPORTED later if a forced path cannot run a shape. */
GTR_API gtr_status_t gtr_gla_set_path(int path);

/* The kernel family gtr_gla_fwd would use for this problem under the current
 * setting (GTR_PATH_SIMT or GTR_PATH_TC), or a negative status. */
GTR_API int gtr_gla_path_for(int B, int H, int grid_h, int grid_w, int dk, int dv, int chunk, int dtype);

/*
 * Device-side status of the current device: synchronises `stream`, returns
 * GTR_OK if no kernel recorded a failed check since the last call, else
 * GTR_ERR_DEVICE_CHECK, and clears the record.  If `counters` is not NULL it
 * receives {status bits, chunks that took the exact-decay path of the
 * tensor-core kernels} accumulated since the last call.
 */
GTR_API gtr_status_t gtr_last_device_status(void *stream, unsigned long long *counters);

#ifdef __cplusplus
}
#endif

#endif /* GTR_GLA_H */
