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
    ss2d_dtype_t in_dtype, out_dtype;
    int max_segments = 32;  // 1 = never split a sequence (no workspace needed)
};

// Number of sequence segments the forward scan is split into (1 = single pass).
int scan_fwd_segments(const LaunchShape &s);
// Workspace bytes for the forward scan's segment summaries.
size_t scan_fwd_workspace_bytes(const LaunchShape &s);
cudaError_t launch_scan_fwd(const LaunchShape &s, const ScanFwdArgs &a, void *workspace, cudaStream_t stream);

// --------------------------------------------------------------- backward --

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
    ss2d_dtype_t in_dtype, out_dtype;
};

size_t scan_bwd_workspace_bytes(const LaunchShape &s);

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
