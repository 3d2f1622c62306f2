// kernels.h -- internal launch interface between the C ABI layer (api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/ss2d.h"

namespace ss2d {

struct LaunchShape {
    int64_t B, D, H, W, L, N;
};

// counts every kernel this library enqueues (exported as ss2d_launch_count) and, when the
// tracing hook is set, records the caller's event after it on `stream`
void note_launch(cudaStream_t stream);

cudaError_t launch_cross_scan(const LaunchShape &s, ss2d_dtype_t dt, const void *x, void *xs,
                              cudaStream_t stream);
// x (B, D, H, W) -> xT (B, D, W, H), bit-exact
cudaError_t launch_transpose(const LaunchShape &s, ss2d_dtype_t dt, const void *x, void *xT, cudaStream_t stream);
cudaError_t launch_cross_merge(const LaunchShape &s, ss2d_dtype_t din, ss2d_dtype_t dout, const void *ys,
                               void *y, cudaStream_t stream);

// ---------------------------------------------------------------- forward --

// How the scan kernels find a sequence's inputs:
//  kModeSeq   -- (B, 4D, L) sequences, each path's data in its own sequence order;
//  kModeImg   -- u read from the image along SS2D path k (fused CrossScan);
//  kModeBidir -- a 1D sequence and its reverse (K = 2 directions) reading the same
//                x, delta, B, C in natural order, the reverse direction backwards.
//  kModeImgProj -- kModeImg with the producer fused in: B, C and the low-rank dt rows come from
//                the per-path x_proj output, dt = softplus(W_dt . x_dbl[:R] + bias) in-kernel;
//  kModeImgProjWide -- B, C from the x_proj output, delta materialised (ranks above
//                kProjRNarrow, where R multiply-adds per step cost more than reading delta).
enum ScanMode { kModeSeq = 0, kModeImg = 1, kModeBidir = 2, kModeImgProj = 3, kModeImgProjWide = 4 };
constexpr int kProjRNarrow = 8;  // dt ranks up to this use the narrow (smaller) projection kernels
constexpr int kProjRMax = 32;    // largest dt_rank the fused projection takes

struct ScanFwdArgs {
    const void *u;       // (B, 4D, L) sequences, or (B, D, H, W) image when from_image
    const void *uT = nullptr;  // (B, D, W, H) transposed image, read by the column paths when from_image
    const void *delta;   // (B, 4D, L)
    const float *A;      // (4D, N)
    const void *Bm;      // (B, 4, N, L)
    const void *Cm;      // (B, 4, N, L)
    const float *Dv;     // (4D) or null
    const float *bias;   // (4D) or null
    int softplus;
    void *out;           // (B, 4D, L)
    float *chunk_states; // (B, 4D, ceil(L/SS2D_CHUNK_LEN), N) or null
    const void *z = nullptr;      // (B, 4D, L) output gate, out *= silu(z); sequences only
    float *last_state = nullptr;  // (B, 4D, N) state after the last step, or null
    bool from_image;     // read u along path k from the image (fused CrossScan)
    bool bidir = false;  // kModeBidir: x (B, D, L), delta (B, D, L), B/C (B, 1, N, L), A (2D, N),
                         // D/bias (D); out = per-direction outputs (B, 2, D, L) fp32 at natural positions
    const void *xdbl = nullptr;  // kModeImgProj (with from_image): x_proj outputs (B, 4, R+2N, L) in_dtype
    const float *Wdt = nullptr;  // kModeImgProj: dt_proj weight (4D, R)
    int R = 0;                   // kModeImgProj: dt rank
    ss2d_dtype_t in_dtype, out_dtype;
    int max_segments = 32;  // 1 = never split a sequence (no workspace needed)
};

// Number of sequence segments the forward scan is split into (1 = single pass).
int scan_fwd_segments(const LaunchShape &s, int paths = 4);
// Workspace bytes for the forward scan's segment summaries.
size_t scan_fwd_workspace_bytes(const LaunchShape &s, int paths = 4);
cudaError_t launch_scan_fwd(const LaunchShape &s, const ScanFwdArgs &a, void *workspace, cudaStream_t stream);

// --------------------------------------------------------------- backward --

// Path sets as tables (int32 (4, L): fwd0, fwd1, inv0, inv1; paths 2/3 are 0/1 backwards).
cudaError_t launch_path_tables(int kind, int64_t H, int64_t W, int32_t *tab, cudaStream_t stream);
// c0[b, d, l] = x[b, d, fwd0[l]], c1[b, d, l] = x[b, d, fwd1[l]]
cudaError_t launch_path_copies(const LaunchShape &s, ss2d_dtype_t dt, const void *x, const int32_t *tab, void *c0,
                               void *c1, cudaStream_t stream);
cudaError_t launch_cross_scan_table(const LaunchShape &s, ss2d_dtype_t dt, const void *x, const int32_t *tab,
                                    void *xs, cudaStream_t stream);
cudaError_t launch_cross_merge_table(const LaunchShape &s, ss2d_dtype_t din, ss2d_dtype_t dout, const void *ys,
                                     const int32_t *tab, void *y, cudaStream_t stream);

// delta[b, k*D + d, l] = sum_r Wdt[k*D + d, r] xdbl[b, k, r, l], in_dtype
cudaError_t launch_dtproj(const LaunchShape &s, ss2d_dtype_t dt, const void *xdbl, const float *Wdt, int R, int RN,
                          void *delta, cudaStream_t stream);
// Per-path x_proj: xdbl[b, k, c, l] = sum_d W[k, c, d] u_k[d, l] (u_0/u_2 from x, u_1/u_3 from xT),
// in each path's step order, RN = R + 2N <= 64 rows.
cudaError_t launch_xproj(const LaunchShape &s, ss2d_dtype_t dt, const void *x, const void *xT, const float *W,
                         int RN, void *xdbl, cudaStream_t stream);

// Producer backward (proj_bwd.cu).  dx_dbl is fp32 (B, 4, RN, L) in each path's step order.
constexpr int64_t kProjTokenChunk = 1024;  // tokens one CTA of a weight-gradient reduction sums
int64_t proj_bwd_chunks(const LaunchShape &s);
// dx_dbl[b, k, r, l] = sum_d Wdt[k*D + d, r] ddelta[b, k*D + d, l] for r < R
cudaError_t launch_proj_bwd_dtlow(const LaunchShape &s, ss2d_dtype_t dt, const void *ddelta, const float *Wdt, int R,
                                  int RN, float *dxdbl, cudaStream_t stream);
// dx_dbl[b, k, off + r, l] = src[b, k, r, l], r < rows
cudaError_t launch_proj_bwd_copy_rows(const LaunchShape &s, ss2d_dtype_t dt, const void *src, int rows, int RN,
                                      int off, float *dxdbl, cudaStream_t stream);
// du_seq[b, k*D + d, l] += sum_c Wx[k, c, d] dx_dbl[b, k, c, l]
cudaError_t launch_proj_bwd_du(const LaunchShape &s, const float *dxdbl, const float *Wx, int RN, float *du_seq,
                               cudaStream_t stream);
// dWdt[k*D + d, r] = sum_{b,l} ddelta[b, k*D + d, l] xdbl[b, k, r, l]; part holds
// 4 * B * proj_bwd_chunks(s) * D * R floats
cudaError_t launch_proj_bwd_dwdt(const LaunchShape &s, ss2d_dtype_t dt, const void *ddelta, const void *xdbl, int R,
                                 int RN, float *part, float *dWdt, cudaStream_t stream);
// dWx[k, c, d] = sum_{b,l} dx_dbl[b, k, c, l] u_k[b, d, l]; part holds 4 * B * proj_bwd_chunks(s) * RN * D floats
cudaError_t launch_proj_bwd_dwx(const LaunchShape &s, ss2d_dtype_t dt, const float *dxdbl, const void *x,
                                const void *xT, int RN, float *part, float *dWx, cudaStream_t stream);

// Causal depthwise conv with SiLU along every path (conv.cu): u[b, k*D + d, l] =
// silu(bias[k*D + d] + sum_j w[k, d, j] x_k[d, l - (W-1) + j]), x_k = x (k = 0, 2) or xT (k = 1, 3)
// read along path k; u in dt.  W = d_conv, 1..4; bias may be null.
cudaError_t launch_path_conv_fwd(const LaunchShape &s, ss2d_dtype_t dt, const void *x, const void *xT,
                                 const float *w, const float *bias, int W, void *u, cudaStream_t stream);
// Its backward from du (fp32 (B, 4D, L), d loss / d u along the paths): dxs (fp32 (B, 4D, L), the
// gradient of x read along each path, merged by the caller), dw (4, D, W) and dbias (4D, or null),
// summed in a fixed order.  part holds path_conv_partial_floats(s, W) floats.
size_t path_conv_partial_floats(const LaunchShape &s, int W);
cudaError_t launch_path_conv_bwd(const LaunchShape &s, ss2d_dtype_t dt, const void *x, const void *xT,
                                 const float *w, const float *bias, int W, const float *du, float *dxs, float *dw,
                                 float *dbias, float *part, cudaStream_t stream);
// d x_proj.weight for per-path sequences u (B, 4D, L) instead of the image read along the paths
cudaError_t launch_proj_bwd_dwx_seq(const LaunchShape &s, ss2d_dtype_t dt, const float *dxdbl, const void *u, int RN,
                                    float *part, float *dWx, cudaStream_t stream);
// Per-path x_proj of sequences: xdbl[b, k, c, l] = sum_d W[k, c, d] u[b, k*D + d, l], RN <= 64
cudaError_t launch_xproj_seq(const LaunchShape &s, ss2d_dtype_t dt, const void *u, const float *W, int RN,
                             void *xdbl, cudaStream_t stream);

// Bidirectional scan: out[b, d, m] = (two[b, 0, d, m] + two[b, 1, d, m]) * (z ? silu(z[b, d, m]) : 1),
// two (B, 2, D, L) fp32, z (B, D, L) z_dtype or null, out (B, D, L) out_dtype.
cudaError_t launch_bidir_sum(const float *two, const void *z, ss2d_dtype_t z_dtype, void *out,
                             ss2d_dtype_t out_dtype, int64_t B, int64_t D, int64_t L, cudaStream_t stream);

struct ScanBwdArgs {
    const void *u;       // (B, 4D, L) sequences, or (B, D, H, W) image when from_image
    const void *uT = nullptr;  // transposed image (recomputing chunk states from the image needs it)
    const void *delta;
    const float *A;
    const void *Bm;
    const void *Cm;
    const float *Dv;
    const float *bias;
    int softplus;
    const void *dout;          // (B, 4D, L), or (B, D, H, W) image when from_image
    const void *doutT = nullptr;  // transposed dout image (column paths when from_image)
    const float *chunk_states; // or null
    void *du;                  // (B, 4D, L) in_dtype, or fp32 when from_image (merged afterwards)
    void *ddelta;
    float *dA;
    void *dBm;
    void *dCm;
    float *dD;
    float *dbias;
    const void *z = nullptr;  // (B, 4D, L) output gate of the forward; sequences only
    void *dz = nullptr;       // (B, 4D, L) in_dtype, written when z is given
    bool from_image;
    bool bidir = false;       // kModeBidir: du, ddelta, dz are per-direction fp32 (B, 2, D, L) at natural
                              // positions; dA (2D, N); dB/dC (B, 1, N, L); dD/dbias (D)
    bool du_f32 = false;      // sequence form: du written in fp32 whatever in_dtype
    ss2d_dtype_t in_dtype, out_dtype;
};

size_t scan_bwd_workspace_bytes(const LaunchShape &s, int paths = 4);

// Helpers of the C-ABI layer (api.cu) for entry points defined in other files.
ss2d_status_t check_scan_fwd_args(const ss2d_desc_t *desc, const void *u, const void *delta, const float *A,
                                  const void *Bm, const void *Cm, const float *D, const float *delta_bias,
                                  const void *out, const float *chunk_states);
ss2d_status_t device_usable();
ss2d_status_t status_from_cuda(cudaError_t e);
void set_error_message(const char *fmt, ...);
cudaError_t launch_scan_bwd(const LaunchShape &s, const ScanBwdArgs &a, void *workspace, size_t ws_bytes,
                            cudaStream_t stream);

}  // namespace ss2d
