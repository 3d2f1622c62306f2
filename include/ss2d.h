/*
 * ss2d.h -- C ABI of libss2d: VMamba's 2D selective scan (SS2D) on NVIDIA B200 (sm_100a).
 *
 * SS2D ("VMamba: Visual State Space Model", section "2D Selective Scan (SS2D)
 * for visual data", Fig. 2) has three steps:
 *   CrossScan  -- unfold a (B, D, H, W) map into K = 4 sequences of length
 *                 L = H*W: row-major (k=0), column-major (k=1, step l = w*H + h)
 *                 and the two reversed (k=2 reverses k=0, k=3 reverses k=1);
 *   S6         -- one selective scan per sequence (channel c = k*D + d uses the
 *                 B/C group k): dt = softplus(delta + delta_bias),
 *                 h = exp(dt*A[c,n]) * h + dt * B[n,l] * u,
 *                 y = sum_n C[n,l] * h[n] + D[c] * u, with h = 0 at l = 0
 *                 ("vision mamba-yolov8", section "2. Vmamba module code",
 *                 selective_scan_ref);
 *   CrossMerge -- put the four outputs back in image order and sum them,
 *                 computed as (y0 + y2) + (y1 + y3) in fp32 and rounded once.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All tensor pointers are DEVICE pointers, owned by the caller, fully
 *    contiguous (row-major) in the layouts stated per argument.  The library
 *    never allocates, frees or synchronises; every kernel is enqueued on
 *    `stream` (a cudaStream_t; NULL means the legacy default stream).
 *  - Element types: u/x, delta, B, C (and the gradients of those) have
 *    desc->in_dtype; outputs y/out have desc->out_dtype.  A, D, delta_bias,
 *    dA, dD, ddelta_bias and chunk states are always fp32.  The state h and all
 *    accumulation are fp32 whatever the I/O type.
 *  - Optional pointers (D, delta_bias, chunk_states, and their gradients) may
 *    be NULL; a NULL D means no skip term, a NULL delta_bias means zero bias.
 *  - Errors: arguments are validated on the host BEFORE anything is launched;
 *    a bad argument returns its status and enqueues nothing.  A failed launch
 *    returns SS2D_ERR_LAUNCH.  No exception or abort crosses the ABI.  NaN/Inf
 *    in the data propagate and are not checked.
 *  - Gradients are written, not accumulated into what the caller's buffer held.
 *  - Pointers must be 16-byte aligned (what cudaMalloc and the PyTorch caching
 *    allocator return for tensors that start at the beginning of their storage).
 */
#ifndef SS2D_H
#define SS2D_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SS2D_API __attribute__((visibility("default")))
#else
#define SS2D_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* forward declaration of the CUDA runtime's stream type, so this header needs no CUDA include */
struct CUstream_st;
typedef struct CUstream_st *ss2d_stream_t;

typedef enum {
    SS2D_OK = 0,
    SS2D_ERR_NULL = 1,      /* a required pointer is NULL */
    SS2D_ERR_SHAPE = 2,     /* a size is <= 0, too large, or inconsistent (e.g. d_state > 16) */
    SS2D_ERR_DTYPE = 3,     /* unsupported dtype or dtype combination */
    SS2D_ERR_ALIGN = 4,     /* a pointer is not 16-byte aligned */
    SS2D_ERR_WORKSPACE = 5, /* workspace NULL or smaller than ss2d_workspace_bytes() */
    SS2D_ERR_LAUNCH = 6,    /* the CUDA launch failed (see ss2d_last_cuda_error()) */
    SS2D_ERR_TIMEOUT = 7,   /* reserved: a bounded device-side wait gave up */
    SS2D_ERR_DEVICE = 8     /* no usable CUDA device, or not an sm_100 device */
} ss2d_status_t;

typedef enum { SS2D_F32 = 0, SS2D_BF16 = 1 } ss2d_dtype_t;

/* Problem description.  K = 4 paths is fixed; channels of the sequence view = 4*dim;
 * sequence length L = height*width.  A 1-D problem is height = 1, width = L. */
typedef struct {
    int64_t batch;          /* B >= 1 */
    int64_t dim;            /* D >= 1: channels of the image; the sequence view has 4*D */
    int64_t height;         /* H >= 1 */
    int64_t width;          /* W >= 1 */
    int64_t d_state;        /* N, 1 <= N <= 16 */
    ss2d_dtype_t in_dtype;  /* type of u/x, delta, B, C */
    ss2d_dtype_t out_dtype; /* type of the output y / out */
} ss2d_desc_t;

/* Operation ids for ss2d_workspace_bytes(). */
typedef enum {
    SS2D_OP_SELECTIVE_SCAN_BWD = 1,
    SS2D_OP_FORWARD = 2,
    SS2D_OP_BACKWARD = 3,
    SS2D_OP_BIMAMBA_FORWARD = 4,
    SS2D_OP_BIMAMBA_BACKWARD = 5,
    SS2D_OP_FORWARD_TABLE = 6,
    SS2D_OP_BACKWARD_TABLE = 7,
    SS2D_OP_FORWARD_PROJ = 8,
    SS2D_OP_BACKWARD_PROJ = 9,
    SS2D_OP_FORWARD_PROJ_CONV = 10,
    SS2D_OP_BACKWARD_PROJ_CONV = 11
} ss2d_op_t;

/* Path sets that ss2d_path_tables generates (paths 2 and 3 are always 0 and 1 walked backwards). */
typedef enum {
    SS2D_PATHS_CROSS = 0,    /* row-major, column-major (l = w*H + h): the cross scan of ss2d_forward */
    SS2D_PATHS_DIAGONAL = 1  /* the two diagonal orders of SS2D._get_diagonal_indices (see ss2d_path_tables) */
} ss2d_paths_t;

/* Chunk length (steps) at which the forward saves scan states for the backward. */
#define SS2D_CHUNK_LEN 16

/* ----------------------------------------------------------------- steps -- */

/*
 * CrossScan (Fig. 2 of the VMamba page, "cross scan"):
 *   xs[b, k, d, l] = x[b, d, pixel_k(l)]
 * x  : (B, D, H, W)  desc->in_dtype
 * xs : (B, 4, D, L)  desc->in_dtype   (bit-exact copy, no arithmetic)
 */
SS2D_API ss2d_status_t ss2d_cross_scan(const ss2d_desc_t *desc, const void *x, void *xs,
                              ss2d_stream_t stream);

/*
 * CrossMerge (Fig. 2 of the VMamba page, "cross merge"):
 *   y[b, d, p] = round_out((t0[p] + t2[p]) + (t1[p] + t3[p])),  t_k[pixel_k(l)] = ys[b, k, d, l]
 * ys : (B, 4, D, L)  desc->in_dtype  (pass in_dtype = F32 to merge fp32 per-path outputs)
 * y  : (B, D, H, W)  desc->out_dtype
 * The sum is fp32 in that order, rounded once (so merge(scan(x)) == 4x exactly).
 */
SS2D_API ss2d_status_t ss2d_cross_merge(const ss2d_desc_t *desc, const void *ys, void *y,
                               ss2d_stream_t stream);

/*
 * S6 selective scan forward over the 4*D sequences ("vision mamba-yolov8",
 * section "2. Vmamba module code": selective_scan_ref and the forward of
 * SelectiveScanFn).  Channel c = k*D + d uses B/C group k.
 * u, delta     : (B, 4D, L)   in_dtype, delta[b, c, l] is step l of path k (sequence order)
 * A            : (4D, N)      fp32
 * Bm, Cm       : (B, 4, N, L) in_dtype
 * D, delta_bias: (4D)         fp32 or NULL
 * delta_softplus: nonzero -> dt = softplus(delta + bias), else dt = delta + bias
 * out          : (B, 4D, L)   out_dtype
 * chunk_states : (B, 4D, ceil(L / SS2D_CHUNK_LEN), N) fp32 or NULL.  Entry j holds
 *                h after step min((j+1)*SS2D_CHUNK_LEN, L) - 1; the last entry is
 *                the final state (the pages' last_state).
 */
SS2D_API ss2d_status_t ss2d_selective_scan_fwd(const ss2d_desc_t *desc, const void *u, const void *delta,
                                      const float *A, const void *Bm, const void *Cm,
                                      const float *D, const float *delta_bias, int delta_softplus,
                                      void *out, float *chunk_states, ss2d_stream_t stream);

/*
 * S6 selective scan backward (the pages print only the call: the backward of
 * SelectiveScanFn returns du, ddelta, dA, dB, dC, dD, ddelta_bias; the
 * gradients are the analytic derivatives of the forward recurrence).
 * Inputs as for ss2d_selective_scan_fwd, plus
 * dout         : (B, 4D, L) out_dtype
 * chunk_states : as written by the forward, or NULL (then recomputed internally)
 * du, ddelta   : (B, 4D, L)   in_dtype
 * dA           : (4D, N)      fp32, summed over batch and steps
 * dBm, dCm     : (B, 4, N, L) in_dtype, summed over the D channels of group k
 * dD, ddelta_bias: (4D) fp32; must be non-NULL exactly when D / delta_bias are
 * workspace    : device buffer of ss2d_workspace_bytes(desc, SS2D_OP_SELECTIVE_SCAN_BWD)
 *                bytes (16-byte aligned); contents on entry are ignored.
 * Reductions are deterministic (fixed-order partial sums, no float atomics).
 */
SS2D_API ss2d_status_t ss2d_selective_scan_bwd(const ss2d_desc_t *desc, const void *u, const void *delta,
                                      const float *A, const void *Bm, const void *Cm,
                                      const float *D, const float *delta_bias, int delta_softplus,
                                      const void *dout, const float *chunk_states,
                                      void *du, void *ddelta, float *dA, void *dBm, void *dCm,
                                      float *dD, float *ddelta_bias,
                                      void *workspace, size_t workspace_bytes,
                                      ss2d_stream_t stream);

/*
 * The same forward with the rest of selective_scan_fn's signature ("vision
 * mamba-yolov8", section "2. Vmamba module code": the z and return_last_state
 * arguments of SelectiveScanFn.forward and selective_scan_ref).
 * z            : (B, 4D, L) in_dtype, or NULL.  When given, the output is gated after
 *                the D*u term: out = (C.h + D u) * silu(z), silu(z) = z * sigmoid(z),
 *                computed in fp32 and rounded once to out_dtype.
 * last_state   : (B, 4D, N) fp32, or NULL: the state after the last step (h at l = L-1).
 *                It carries no gradient (the pages leave it out of the backward).
 * Other arguments, layouts and errors as for ss2d_selective_scan_fwd;
 * ss2d_selective_scan_fwd(...) is this call with z = last_state = NULL.
 */
SS2D_API ss2d_status_t ss2d_selective_scan_fwd_ex(const ss2d_desc_t *desc, const void *u, const void *delta,
                                                  const float *A, const void *Bm, const void *Cm,
                                                  const float *D, const void *z, const float *delta_bias,
                                                  int delta_softplus, void *out, float *last_state,
                                                  float *chunk_states, ss2d_stream_t stream);

/*
 * Backward of ss2d_selective_scan_fwd_ex (the backward of SelectiveScanFn with z).
 * z            : the forward's gate, or NULL.  dout is then the gradient of the gated
 *                output: dout * silu(z) drives the scan's backward, and
 *                dz = dout * silu'(z) * (C.h + D u), with C.h rebuilt from the
 *                recomputed states (the caller does not keep the ungated output).
 * dz           : (B, 4D, L) in_dtype; must be non-NULL exactly when z is.
 * Other arguments, layouts, workspace (SS2D_OP_SELECTIVE_SCAN_BWD) and errors as for
 * ss2d_selective_scan_bwd, which is this call with z = dz = NULL.
 */
SS2D_API ss2d_status_t ss2d_selective_scan_bwd_ex(const ss2d_desc_t *desc, const void *u, const void *delta,
                                                  const float *A, const void *Bm, const void *Cm,
                                                  const float *D, const void *z, const float *delta_bias,
                                                  int delta_softplus, const void *dout,
                                                  const float *chunk_states, void *du, void *ddelta, float *dA,
                                                  void *dBm, void *dCm, float *dD, float *ddelta_bias, void *dz,
                                                  void *workspace, size_t workspace_bytes,
                                                  ss2d_stream_t stream);

/* --------------------------------------------------------- fused SS2D -- */

/*
 * Fused SS2D forward: CrossScan -> S6 -> CrossMerge without the (B,4,D,L)
 * intermediates.  The traversal of each path is folded into the kernels' load
 * and store indexing.
 * x            : (B, D, H, W)  in_dtype
 * delta        : (B, 4D, L)    in_dtype (sequence order of each path)
 * A, Bm, Cm, D, delta_bias, delta_softplus: as for ss2d_selective_scan_fwd
 * y            : (B, D, H, W)  out_dtype
 * chunk_states : as for ss2d_selective_scan_fwd (per path sequence), or NULL
 * workspace    : ss2d_workspace_bytes(desc, SS2D_OP_FORWARD) bytes (may be 0 -> NULL ok)
 */
SS2D_API ss2d_status_t ss2d_forward(const ss2d_desc_t *desc, const void *x, const void *delta,
                           const float *A, const void *Bm, const void *Cm, const float *D,
                           const float *delta_bias, int delta_softplus, void *y,
                           float *chunk_states, void *workspace, size_t workspace_bytes,
                           ss2d_stream_t stream);

/*
 * Fused SS2D backward: g = CrossScan(dy) folded into the loads, S6 backward,
 * dx = CrossMerge(du) folded into the stores.
 * x, delta, A, Bm, Cm, D, delta_bias, delta_softplus, chunk_states: as for ss2d_forward
 * dy           : (B, D, H, W) out_dtype
 * dx           : (B, D, H, W) in_dtype
 * ddelta       : (B, 4D, L)   in_dtype
 * dA, dBm, dCm, dD, ddelta_bias: as for ss2d_selective_scan_bwd
 * workspace    : ss2d_workspace_bytes(desc, SS2D_OP_BACKWARD) bytes
 */
SS2D_API ss2d_status_t ss2d_backward(const ss2d_desc_t *desc, const void *x, const void *delta,
                            const float *A, const void *Bm, const void *Cm, const float *D,
                            const float *delta_bias, int delta_softplus, const void *dy,
                            const float *chunk_states, void *dx, void *ddelta, float *dA,
                            void *dBm, void *dCm, float *dD, float *ddelta_bias,
                            void *workspace, size_t workspace_bytes, ss2d_stream_t stream);

/* ------------------------------------------------ producer projections -- */

/*
 * Fused SS2D forward with its producer: the scan's delta, B and C are made from x by
 * per-path projections, as MambaInnerFn.forward makes them ("vision mamba-yolov8",
 * section 2): x_dbl = x_proj(u_k), delta = dt_proj.weight @ x_dbl[:R], B and C the next N
 * and the last N rows of x_dbl; dt_proj.bias is the delta bias.  For dt_rank <= 8 delta is
 * never written: the scan computes dt = softplus(W_dt . x_dbl[:R] + bias) at every step;
 * for larger ranks delta is materialised in the workspace (R multiply-adds per step would
 * cost the scan more than reading it).  B and C are read from x_dbl in both cases.
 * dt_rank          : R, 1 <= R <= 32 (ceil(d_model / 16) for d_model <= 512)
 * x                : (B, D, H, W)  in_dtype
 * x_proj_weight    : (4, R + 2N, D) fp32, one projection per path
 * dt_proj_weight   : (4, D, R)     fp32
 * dt_proj_bias     : (4D)          fp32 or NULL
 * A, D, delta_softplus, y, chunk_states: as for ss2d_forward
 * x_dbl            : (B, 4, R + 2N, L) in_dtype, written (each path's step order): the saved
 *                    activation a backward needs
 * workspace        : ss2d_workspace_bytes(desc, SS2D_OP_FORWARD_PROJ) bytes
 * Errors: SS2D_ERR_SHAPE for dt_rank outside [1, 32]; otherwise as for ss2d_forward.
 */
SS2D_API ss2d_status_t ss2d_forward_proj(const ss2d_desc_t *desc, int dt_rank, const void *x,
                                         const float *x_proj_weight, const float *dt_proj_weight,
                                         const float *dt_proj_bias, const float *A, const float *D,
                                         int delta_softplus, void *y, void *x_dbl, float *chunk_states,
                                         void *workspace, size_t workspace_bytes, ss2d_stream_t stream);

/*
 * Backward of ss2d_forward_proj: the gradients MambaInnerFn.backward ("vision mamba-yolov8",
 * section 2) takes through the scan and then through the producer.  With ddelta, dB, dC the
 * scan's gradients (as ss2d_backward gives them), per path k and token l:
 *   dx_dbl[:R]        = dt_proj.weight^T ddelta,   dx_dbl[R:] = (dB, dC)
 *   ddt_proj_weight   = sum over batch and tokens of ddelta (x) x_dbl[:R]
 *   dx_proj_weight    = sum over batch and tokens of dx_dbl (x) u_k
 *   dx                = the scan's du plus x_proj.weight^T dx_dbl, each merged along its path
 * ddt_proj_bias is the scan's delta-bias gradient; dA and dD the scan's.  delta is made again
 * from x_dbl (in in_dtype), B and C are read from x_dbl.  The sums over tokens and batch run
 * in a fixed order (deterministic), in fp32.
 * dt_rank, x, x_proj_weight, dt_proj_weight, dt_proj_bias, A, D, delta_softplus: as for
 *                    ss2d_forward_proj
 * x_dbl            : (B, 4, R + 2N, L) in_dtype, as ss2d_forward_proj wrote it
 * chunk_states     : as ss2d_forward_proj wrote them, or NULL (recomputed)
 * dy               : (B, D, H, W) out_dtype
 * dx               : (B, D, H, W) in_dtype, written
 * dx_proj_weight   : (4, R + 2N, D) fp32, written;  ddt_proj_weight: (4, D, R) fp32, written
 * ddt_proj_bias    : (4D) fp32, written; NULL exactly when dt_proj_bias is NULL
 * dA (4D, N) fp32, dD (4D) fp32 (NULL exactly when D is NULL): written
 * workspace        : ss2d_workspace_bytes(desc, SS2D_OP_BACKWARD_PROJ) bytes (sized for the
 *                    largest dt_rank, 32)
 * Errors: SS2D_ERR_SHAPE for dt_rank outside [1, 32]; otherwise as for ss2d_backward.
 */
SS2D_API ss2d_status_t ss2d_backward_proj(const ss2d_desc_t *desc, int dt_rank, const void *x,
                                          const float *x_proj_weight, const float *dt_proj_weight,
                                          const float *dt_proj_bias, const float *A, const float *D,
                                          int delta_softplus, const void *x_dbl, const float *chunk_states,
                                          const void *dy, void *dx, float *dx_proj_weight,
                                          float *ddt_proj_weight, float *ddt_proj_bias, float *dA, float *dD,
                                          void *workspace, size_t workspace_bytes, ss2d_stream_t stream);

/*
 * The producer with its causal depthwise conv: MambaInnerFn.forward ("vision mamba-yolov8",
 * section 2) passes its input through causal_conv1d_fwd(x, weight, bias, True) (a depthwise conv
 * of width d_conv over the current and previous steps, then SiLU) before x_proj.  As the Visual
 * Mamba page's SS2D runs one Mamba block per scan direction, every path k convolves x read along
 * its own step order with its own weights:
 *   u_k[d, l] = silu(conv_bias[k*D + d] + sum_j conv_weight[k, d, j] x_k[d, l - (d_conv-1) + j])
 * (x_k = 0 before step 0), then the producer of ss2d_forward_proj on u_k (x_proj, dt_proj, B and
 * C from x_dbl), the S6 scan of every path on u_k, and CrossMerge.
 * d_conv           : 1..4
 * conv_weight      : (4, D, d_conv) fp32;  conv_bias: (4D) fp32 or NULL
 * other arguments  : as for ss2d_forward_proj (x_dbl written, in each path's step order)
 * workspace        : ss2d_workspace_bytes(desc, SS2D_OP_FORWARD_PROJ_CONV) bytes
 * Errors: SS2D_ERR_SHAPE for dt_rank outside [1, 32] or d_conv outside [1, 4]; otherwise as for
 * ss2d_forward_proj.
 */
SS2D_API ss2d_status_t ss2d_forward_proj_conv(const ss2d_desc_t *desc, int dt_rank, int d_conv, const void *x,
                                              const float *conv_weight, const float *conv_bias,
                                              const float *x_proj_weight, const float *dt_proj_weight,
                                              const float *dt_proj_bias, const float *A, const float *D,
                                              int delta_softplus, void *y, void *x_dbl, float *chunk_states,
                                              void *workspace, size_t workspace_bytes, ss2d_stream_t stream);

/*
 * Backward of ss2d_forward_proj_conv (MambaInnerFn.backward with causal_conv1d_bwd): the scan's
 * gradients, the producer's as in ss2d_backward_proj, then the conv's: dpre = du * silu'(pre),
 * dconv_weight[k, d, j] = sum over batch and steps of dpre[l] x_k[l - (d_conv-1) + j],
 * dconv_bias = sum of dpre, and dx = the per-path sum_j w[k, d, j] dpre[m + (d_conv-1) - j] merged
 * along the paths.  u is made again from x; the sums run in a fixed order (deterministic), in fp32.
 * x_dbl, chunk_states: as ss2d_forward_proj_conv wrote them (chunk_states may be NULL)
 * dy (B, D, H, W) out_dtype;  dx (B, D, H, W) in_dtype, written
 * dconv_weight (4, D, d_conv), dconv_bias (4D; NULL exactly when conv_bias is NULL), and the
 * other gradients as for ss2d_backward_proj: fp32, written
 * workspace        : ss2d_workspace_bytes(desc, SS2D_OP_BACKWARD_PROJ_CONV) bytes (sized for dt
 *                    rank 32 and d_conv 4)
 * Errors: as for ss2d_forward_proj_conv and ss2d_backward_proj.
 */
SS2D_API ss2d_status_t ss2d_backward_proj_conv(const ss2d_desc_t *desc, int dt_rank, int d_conv, const void *x,
                                               const float *conv_weight, const float *conv_bias,
                                               const float *x_proj_weight, const float *dt_proj_weight,
                                               const float *dt_proj_bias, const float *A, const float *D,
                                               int delta_softplus, const void *x_dbl, const float *chunk_states,
                                               const void *dy, void *dx, float *dconv_weight, float *dconv_bias,
                                               float *dx_proj_weight, float *ddt_proj_weight, float *ddt_proj_bias,
                                               float *dA, float *dD, void *workspace, size_t workspace_bytes,
                                               ss2d_stream_t stream);

/* ------------------------------------------------------------ path sets -- */

/*
 * Fill a path table for a path set, on the device.  The table is int32 (4, L), L = H*W:
 *   rows 0, 1: fwd_k[l] = pixel p = h*W + w visited at step l of path k;
 *   rows 2, 3: inv_k[p] = the step at which path k visits pixel p.
 * Paths 2 and 3 are paths 0 and 1 walked backwards.  SS2D_PATHS_DIAGONAL follows
 * SS2D._get_diagonal_indices of "Visual Mamba实战从零开始搭建图像分类模型附PyTorch代码"
 * (section 3): anti-diagonals s = h + w in turn, h ascending within each, with w = s - h
 * (path 0) or w = (W-1) - (s - h) (path 1).
 * tables : device, 16-byte aligned, 4*L int32, written.  L must be below 2^31.
 * Errors: SS2D_ERR_SHAPE for an unknown path set or L >= 2^31.
 */
SS2D_API ss2d_status_t ss2d_path_tables(const ss2d_desc_t *desc, int paths, int32_t *tables, ss2d_stream_t stream);

/*
 * CrossScan and CrossMerge over the path set of a table (as ss2d_path_tables writes it,
 * or the caller's own: every entry is bounds-checked; an entry outside [0, L) reads as
 * zero, so a table that is not made of permutations gives wrong values, never a bad access).
 *   ss2d_cross_scan_table : xs[b, k, d, l] = x[b, d, fwd_k[l]] (k = 2, 3: fwd_{k-2}[L-1-l])
 *   ss2d_cross_merge_table: y[b, d, p] = round_out((t0 + t2) + (t1 + t3)), t_k = path k's
 *                           value at pixel p, summed in fp32
 * Layouts and dtypes as ss2d_cross_scan / ss2d_cross_merge.
 */
SS2D_API ss2d_status_t ss2d_cross_scan_table(const ss2d_desc_t *desc, const int32_t *tables, const void *x,
                                             void *xs, ss2d_stream_t stream);
SS2D_API ss2d_status_t ss2d_cross_merge_table(const ss2d_desc_t *desc, const int32_t *tables, const void *ys,
                                              void *y, ss2d_stream_t stream);

/*
 * Fused SS2D forward and backward over the path set of a table.  Arguments, layouts and
 * results are those of ss2d_forward / ss2d_backward with path k walking the table's order
 * (delta, B, C, chunk states in each path's own step order).  The scan reads x along
 * paths 0 and 1 from two path-order copies that the call makes in its workspace, as the
 * cross path set reads x and its transpose.
 * workspace: ss2d_workspace_bytes(desc, SS2D_OP_FORWARD_TABLE / SS2D_OP_BACKWARD_TABLE) bytes.
 */
SS2D_API ss2d_status_t ss2d_forward_table(const ss2d_desc_t *desc, const int32_t *tables, const void *x,
                                          const void *delta, const float *A, const void *Bm, const void *Cm,
                                          const float *D, const float *delta_bias, int delta_softplus, void *y,
                                          float *chunk_states, void *workspace, size_t workspace_bytes,
                                          ss2d_stream_t stream);
SS2D_API ss2d_status_t ss2d_backward_table(const ss2d_desc_t *desc, const int32_t *tables, const void *x,
                                           const void *delta, const float *A, const void *Bm, const void *Cm,
                                           const float *D, const float *delta_bias, int delta_softplus,
                                           const void *dy, const float *chunk_states, void *dx, void *ddelta,
                                           float *dA, void *dBm, void *dCm, float *dD, float *ddelta_bias,
                                           void *workspace, size_t workspace_bytes, ss2d_stream_t stream);

/* ------------------------------------------------- bidirectional scan -- */

/*
 * Bidirectional selective scan of bimamba_inner_ref ("vision mamba-yolov8",
 * section "2. Vmamba module code"): one scan over the sequence with A, one over
 * the reversed sequence with A_b (x, delta, B, C, z reversed with it; D and
 * delta_bias shared), the second output reversed back and added:
 *   y = S6(x, delta, A, B, C, D, z) + flip(S6(flip x, flip delta, A_b, flip B, flip C, D, flip z))
 * Both directions are one launch; the reverse one reads its inputs backwards and
 * writes at natural positions, and a merge adds the two in fp32 (gated by silu(z),
 * which both directions share position by position) and rounds once.
 * desc         : batch B, dim D, height 1, width L (a sequence), d_state N
 * x, delta     : (B, D, L)  in_dtype
 * A            : (2, D, N)  fp32: A, then A_b
 * Bm, Cm       : (B, N, L)  in_dtype, shared by the two directions
 * D, delta_bias: (D)        fp32 or NULL
 * z            : (B, D, L)  in_dtype or NULL (output gate silu(z))
 * y            : (B, D, L)  out_dtype
 * chunk_states : (B, 2D, ceil(L / SS2D_CHUNK_LEN), N) fp32 or NULL, per direction in its own
 *                step order (direction 1 counts steps from the end of the sequence)
 * workspace    : ss2d_workspace_bytes(desc, SS2D_OP_BIMAMBA_FORWARD) bytes
 * Errors: as for ss2d_forward; height != 1 is SS2D_ERR_SHAPE.
 */
SS2D_API ss2d_status_t ss2d_bimamba_forward(const ss2d_desc_t *desc, const void *x, const void *delta,
                                            const float *A, const void *Bm, const void *Cm, const float *D,
                                            const void *z, const float *delta_bias, int delta_softplus, void *y,
                                            float *chunk_states, void *workspace, size_t workspace_bytes,
                                            ss2d_stream_t stream);

/*
 * Gradients of ss2d_bimamba_forward.
 * dy           : (B, D, L) out_dtype
 * chunk_states : as written by ss2d_bimamba_forward, or NULL (recomputed)
 * dx, ddelta   : (B, D, L) in_dtype (both directions' contributions added)
 * dA           : (2, D, N) fp32: dA, then dA_b
 * dBm, dCm     : (B, N, L) in_dtype
 * dD, ddelta_bias: (D) fp32, non-NULL exactly when D / delta_bias are
 * dz           : (B, D, L) in_dtype, non-NULL exactly when z is
 * workspace    : ss2d_workspace_bytes(desc, SS2D_OP_BIMAMBA_BACKWARD) bytes
 * Reductions are deterministic (fixed-order partial sums, no float atomics).
 */
SS2D_API ss2d_status_t ss2d_bimamba_backward(const ss2d_desc_t *desc, const void *x, const void *delta,
                                             const float *A, const void *Bm, const void *Cm, const float *D,
                                             const void *z, const float *delta_bias, int delta_softplus,
                                             const void *dy, const float *chunk_states, void *dx, void *ddelta,
                                             float *dA, void *dBm, void *dCm, float *dD, float *ddelta_bias,
                                             void *dz, void *workspace, size_t workspace_bytes,
                                             ss2d_stream_t stream);

/*
 * S6 selective scan forward that allocates nothing and takes no workspace.
 * The pages have no counterpart: this is an addition of this library.
 *
 * Some callers cannot allocate device memory when they call: a serving loop
 * whose memory plan is fixed at start-up, or a host program that links only
 * this C library and has no device allocator to provide a workspace.  Arguments,
 * layouts and results are those of ss2d_selective_scan_fwd; unlike it, when a
 * problem has too few sequences to fill the GPU (fewer than ~76k), the scan
 * splits every sequence into up to 32 segments, keeping the per-segment
 * summaries (B * 4D * segments * 2N fp32) in a 16 MiB static device buffer
 * inside the library.
 *  - A problem whose summaries exceed 16 MiB returns SS2D_ERR_SHAPE before any
 *    launch (ss2d_last_cuda_error() says how many bytes it needed).
 *  - Every GPU that loads the library holds the 16 MiB buffer until exit.
 *  - The first call on each device looks up the buffer's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before any stream capture on the device.
 *  - All calls on a device share the buffer: calls that can overlap on the GPU
 *    (other streams, unordered host threads) race and give wrong results.  Each
 *    call writes every entry before reading it, so nothing needs clearing.
 */
SS2D_API ss2d_status_t ss2d_selective_scan_fwd_noalloc(const ss2d_desc_t *desc, const void *u, const void *delta,
                                                       const float *A, const void *Bm, const void *Cm,
                                                       const float *D, const float *delta_bias, int delta_softplus,
                                                       void *out, float *chunk_states, ss2d_stream_t stream);

/* ------------------------------------------------------------- helpers -- */

/* Bytes of workspace an operation needs for this problem (0 if none).
 * Returns (size_t)-1 for an invalid desc or op. */
SS2D_API size_t ss2d_workspace_bytes(const ss2d_desc_t *desc, int op);

/* Number of fp32 elements of the chunk_states buffer: B * 4D * ceil(L/SS2D_CHUNK_LEN) * N. */
SS2D_API size_t ss2d_chunk_states_elems(const ss2d_desc_t *desc);

/* Static, human-readable name of a status code. */
SS2D_API const char *ss2d_status_string(ss2d_status_t status);

/* Message of the last CUDA error this library saw on the calling thread ("" if none). */
SS2D_API const char *ss2d_last_cuda_error(void);

/* Kernels this library has launched since load (all threads); used to count launches. */
SS2D_API uint64_t ss2d_launch_count(void);

/* Tracing hook.  While set, the i-th kernel this library enqueues from the calling thread
 * is followed by cudaEventRecord(events[i], stream) for i < count (events are cudaEvent_t
 * handles the caller created; the library never creates, waits on or destroys them).  The
 * index restarts at 0 on every call of this function; pass (NULL, 0) to stop.  Used to time
 * the kernels of one entry point individually on their own stream. */
SS2D_API void ss2d_set_trace_events(void *const *events, int count);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
SS2D_API int ss2d_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SS2D_H */
