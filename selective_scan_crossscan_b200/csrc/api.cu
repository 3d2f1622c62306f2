// api.cu -- the C ABI of libss2d (declared in include/ss2d.h): argument
// validation on the host, workspace layout, and dispatch to the kernels.
#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "common.cuh"
#include "kernels.h"

namespace ss2d {

static std::atomic<uint64_t> g_launches{0};
static thread_local void *const *g_trace_events = nullptr;
static thread_local int g_trace_count = 0;
static thread_local int g_trace_next = 0;

void note_launch(cudaStream_t stream) {
    g_launches.fetch_add(1, std::memory_order_relaxed);
    if (g_trace_events && g_trace_next < g_trace_count)
        cudaEventRecord(static_cast<cudaEvent_t>(g_trace_events[g_trace_next++]), stream);
}

static thread_local char g_last_error[256] = "";

static ss2d_status_t from_cuda(cudaError_t e) {
    if (e == cudaSuccess) return SS2D_OK;
    std::snprintf(g_last_error, sizeof(g_last_error), "%s: %s", cudaGetErrorName(e), cudaGetErrorString(e));
    return SS2D_ERR_LAUNCH;
}

static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static ss2d_status_t check_desc(const ss2d_desc_t *d) {
    if (!d) return SS2D_ERR_NULL;
    if (d->batch < 1 || d->dim < 1 || d->height < 1 || d->width < 1) return SS2D_ERR_SHAPE;
    if (d->d_state < 1 || d->d_state > 16) return SS2D_ERR_SHAPE;
    if ((d->in_dtype != SS2D_F32 && d->in_dtype != SS2D_BF16) ||
        (d->out_dtype != SS2D_F32 && d->out_dtype != SS2D_BF16))
        return SS2D_ERR_DTYPE;
    // grid limits: the batch is a grid dimension (<= 65535); keep element counts in int64 range
    if (d->batch > 65535) return SS2D_ERR_SHAPE;
    const double elems = (double)d->batch * 4.0 * (double)d->dim * (double)d->height * (double)d->width *
                         (double)d->d_state;
    if (elems > 9.0e15) return SS2D_ERR_SHAPE;
    if ((double)d->batch * (double)d->dim * ceil_div(d->height, 32) * ceil_div(d->width, 32) > 2147483647.0)
        return SS2D_ERR_SHAPE;
    return SS2D_OK;
}

static LaunchShape shape_of(const ss2d_desc_t *d) {
    LaunchShape s;
    s.B = d->batch;
    s.D = d->dim;
    s.H = d->height;
    s.W = d->width;
    s.L = d->height * d->width;
    s.N = d->d_state;
    return s;
}

// one cached compute-capability check per device
static ss2d_status_t check_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) {
        cudaGetLastError();
        std::snprintf(g_last_error, sizeof(g_last_error), "no CUDA device");
        return SS2D_ERR_DEVICE;
    }
    static std::atomic<int> ok[64];
    if (dev < 64 && ok[dev].load() == 1) return SS2D_OK;
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
        cudaGetLastError();
        return SS2D_ERR_DEVICE;
    }
    if (major != 10) {
        std::snprintf(g_last_error, sizeof(g_last_error), "device %d is compute capability %d.x, need 10.0 (sm_100a)",
                      dev, major);
        return SS2D_ERR_DEVICE;
    }
    if (dev < 64) ok[dev].store(1);
    return SS2D_OK;
}

#define SS2D_TRY(expr)                         \
    do {                                       \
        ss2d_status_t _st = (expr);            \
        if (_st != SS2D_OK) return _st;        \
    } while (0)

static ss2d_status_t need(const void *p) {
    if (!p) return SS2D_ERR_NULL;
    if (!aligned16(p)) return SS2D_ERR_ALIGN;
    return SS2D_OK;
}
static ss2d_status_t optional(const void *p) { return (p && !aligned16(p)) ? SS2D_ERR_ALIGN : SS2D_OK; }

// workspace layouts ---------------------------------------------------------

static size_t round64(size_t n) { return (n + 63) / 64 * 64; }

static size_t elem_size(ss2d_dtype_t t) { return t == SS2D_F32 ? 4 : 2; }

// fused forward workspace: [fp32 per-path outputs (B,4D,L)] [transposed image (B,D,W,H)] [segment summaries]
static size_t fwd_ws_bytes(const LaunchShape &s, ss2d_dtype_t in) {
    return round64((size_t)s.B * kPaths * s.D * s.L * sizeof(float)) +
           round64((size_t)s.B * s.D * s.L * elem_size(in)) + round64(scan_fwd_workspace_bytes(s));
}
// fused backward workspace: [fp32 per-path du (B,4D,L)] [transposed x] [transposed dy] [scan backward workspace]
static size_t bwd_fused_ws_bytes(const LaunchShape &s, ss2d_dtype_t in, ss2d_dtype_t out) {
    return round64((size_t)s.B * kPaths * s.D * s.L * sizeof(float)) +
           round64((size_t)s.B * s.D * s.L * elem_size(in)) + round64((size_t)s.B * s.D * s.L * elem_size(out)) +
           round64(scan_bwd_workspace_bytes(s));
}

// bidirectional forward workspace: [fp32 per-direction outputs (B,2,D,L)] [segment summaries]
static size_t bidir_fwd_ws_bytes(const LaunchShape &s) {
    return round64((size_t)s.B * 2 * s.D * s.L * sizeof(float)) + round64(scan_fwd_workspace_bytes(s, 2));
}
// bidirectional backward workspace: [fp32 per-direction du, ddelta, dz (B,2,D,L) each] [scan backward workspace]
static size_t bidir_bwd_ws_bytes(const LaunchShape &s) {
    return 3 * round64((size_t)s.B * 2 * s.D * s.L * sizeof(float)) + round64(scan_bwd_workspace_bytes(s, 2));
}

// table forward workspace: [fp32 per-path outputs (B,4D,L)] [x in path-0 order] [x in path-1 order] [segments]
static size_t table_fwd_ws_bytes(const LaunchShape &s, ss2d_dtype_t in) {
    const size_t img = round64((size_t)s.B * s.D * s.L * elem_size(in));
    return round64((size_t)s.B * kPaths * s.D * s.L * sizeof(float)) + 2 * img + round64(scan_fwd_workspace_bytes(s));
}
// table backward workspace: [fp32 per-path du] [x copies 0, 1] [dy copies 0, 1] [scan backward workspace]
static size_t table_bwd_ws_bytes(const LaunchShape &s, ss2d_dtype_t in, ss2d_dtype_t out) {
    return round64((size_t)s.B * kPaths * s.D * s.L * sizeof(float)) +
           2 * round64((size_t)s.B * s.D * s.L * elem_size(in)) + 2 * round64((size_t)s.B * s.D * s.L * elem_size(out)) +
           round64(scan_bwd_workspace_bytes(s));
}
// producer backward workspace (sized for the largest dt rank):
// [fp32 per-path du (B,4D,L)] [transposed x] [transposed dy] [delta] [ddelta] [B, C, dB, dC (B,4,N,L) each]
// [fp32 dx_dbl (B,4,RN,L)] [fp32 weight-gradient partials] [scan backward workspace]
static size_t proj_bwd_ws_bytes(const LaunchShape &s, ss2d_dtype_t in, ss2d_dtype_t out) {
    const size_t seq = (size_t)s.B * kPaths * s.D * s.L, img = (size_t)s.B * s.D * s.L;
    const size_t bc = (size_t)s.B * kPaths * s.N * s.L, rn = (size_t)kProjRMax + 2 * s.N;
    return round64(seq * sizeof(float)) + round64(img * elem_size(in)) + round64(img * elem_size(out)) +
           2 * round64(seq * elem_size(in)) + 4 * round64(bc * elem_size(in)) +
           round64((size_t)s.B * kPaths * rn * s.L * sizeof(float)) +
           round64((size_t)kPaths * s.B * proj_bwd_chunks(s) * rn * s.D * sizeof(float)) +
           round64(scan_bwd_workspace_bytes(s));
}
// producer-with-conv forward workspace: [transposed x] [u (B,4D,L)] [delta] [B, C (B,4,N,L)]
// [fp32 per-path outputs (B,4D,L)] [segment summaries]
static size_t conv_fwd_ws_bytes(const LaunchShape &s, ss2d_dtype_t in) {
    const size_t seq = (size_t)s.B * kPaths * s.D * s.L, img = (size_t)s.B * s.D * s.L;
    const size_t bc = (size_t)s.B * kPaths * s.N * s.L;
    return round64(img * elem_size(in)) + 2 * round64(seq * elem_size(in)) + 2 * round64(bc * elem_size(in)) +
           round64(seq * sizeof(float)) + round64(scan_fwd_workspace_bytes(s));
}
// producer-with-conv backward workspace: [transposed x] [u] [dy along the paths] [delta] [ddelta]
// [B, C, dB, dC] [fp32 du (B,4D,L)] [fp32 dx along the paths] [fp32 dx_dbl] [partials] [scan backward]
// (sized for dt rank 32 and d_conv 4)
static size_t conv_bwd_ws_bytes(const LaunchShape &s, ss2d_dtype_t in, ss2d_dtype_t out) {
    const size_t seq = (size_t)s.B * kPaths * s.D * s.L, img = (size_t)s.B * s.D * s.L;
    const size_t bc = (size_t)s.B * kPaths * s.N * s.L, rn = (size_t)kProjRMax + 2 * s.N;
    const size_t part = std::max((size_t)kPaths * s.B * proj_bwd_chunks(s) * rn * s.D, path_conv_partial_floats(s, 4));
    return round64(img * elem_size(in)) + round64(seq * elem_size(in)) + round64(seq * elem_size(out)) +
           2 * round64(seq * elem_size(in)) + 4 * round64(bc * elem_size(in)) + 2 * round64(seq * sizeof(float)) +
           round64((size_t)s.B * kPaths * rn * s.L * sizeof(float)) + round64(part * sizeof(float)) +
           round64(scan_bwd_workspace_bytes(s));
}
static ss2d_status_t check_table_shape(const ss2d_desc_t *desc) {
    return desc->height * desc->width < ((int64_t)1 << 31) ? SS2D_OK : SS2D_ERR_SHAPE;
}

}  // namespace ss2d

using namespace ss2d;

extern "C" {

int ss2d_version(void) { return 100; }  // 0.1.0

uint64_t ss2d_launch_count(void) { return g_launches.load(); }

void ss2d_set_trace_events(void *const *events, int count) {
    g_trace_events = (events && count > 0) ? events : nullptr;
    g_trace_count = g_trace_events ? count : 0;
    g_trace_next = 0;
}

const char *ss2d_last_cuda_error(void) { return g_last_error; }

const char *ss2d_status_string(ss2d_status_t s) {
    switch (s) {
        case SS2D_OK: return "SS2D_OK";
        case SS2D_ERR_NULL: return "SS2D_ERR_NULL: a required pointer is NULL";
        case SS2D_ERR_SHAPE: return "SS2D_ERR_SHAPE: invalid or unsupported sizes";
        case SS2D_ERR_DTYPE: return "SS2D_ERR_DTYPE: unsupported dtype";
        case SS2D_ERR_ALIGN: return "SS2D_ERR_ALIGN: pointer not 16-byte aligned";
        case SS2D_ERR_WORKSPACE: return "SS2D_ERR_WORKSPACE: workspace missing or too small";
        case SS2D_ERR_LAUNCH: return "SS2D_ERR_LAUNCH: CUDA launch failed";
        case SS2D_ERR_TIMEOUT: return "SS2D_ERR_TIMEOUT: device-side wait gave up";
        case SS2D_ERR_DEVICE: return "SS2D_ERR_DEVICE: no usable sm_100 device";
    }
    return "SS2D: unknown status";
}

size_t ss2d_chunk_states_elems(const ss2d_desc_t *desc) {
    if (check_desc(desc) != SS2D_OK) return 0;
    const LaunchShape s = shape_of(desc);
    return (size_t)s.B * kPaths * s.D * ceil_div(s.L, SS2D_CHUNK_LEN) * s.N;
}

size_t ss2d_workspace_bytes(const ss2d_desc_t *desc, int op) {
    if (check_desc(desc) != SS2D_OK) return (size_t)-1;
    const LaunchShape s = shape_of(desc);
    switch (op) {
        case SS2D_OP_SELECTIVE_SCAN_BWD: return scan_bwd_workspace_bytes(s);
        case SS2D_OP_FORWARD: return fwd_ws_bytes(s, desc->in_dtype);
        case SS2D_OP_BACKWARD: return bwd_fused_ws_bytes(s, desc->in_dtype, desc->out_dtype);
        case SS2D_OP_BIMAMBA_FORWARD: return bidir_fwd_ws_bytes(s);
        case SS2D_OP_BIMAMBA_BACKWARD: return bidir_bwd_ws_bytes(s);
        case SS2D_OP_FORWARD_TABLE: return table_fwd_ws_bytes(s, desc->in_dtype);
        case SS2D_OP_FORWARD_PROJ:
            return fwd_ws_bytes(s, desc->in_dtype) + round64((size_t)s.B * kPaths * s.D * s.L * elem_size(desc->in_dtype));
        case SS2D_OP_BACKWARD_TABLE: return table_bwd_ws_bytes(s, desc->in_dtype, desc->out_dtype);
        case SS2D_OP_BACKWARD_PROJ: return proj_bwd_ws_bytes(s, desc->in_dtype, desc->out_dtype);
        case SS2D_OP_FORWARD_PROJ_CONV: return conv_fwd_ws_bytes(s, desc->in_dtype);
        case SS2D_OP_BACKWARD_PROJ_CONV: return conv_bwd_ws_bytes(s, desc->in_dtype, desc->out_dtype);
        default: return (size_t)-1;
    }
}

ss2d_status_t ss2d_cross_scan(const ss2d_desc_t *desc, const void *x, void *xs, ss2d_stream_t stream) {
    SS2D_TRY(check_desc(desc));
    SS2D_TRY(need(x));
    SS2D_TRY(need(xs));
    SS2D_TRY(check_device());
    return from_cuda(launch_cross_scan(shape_of(desc), desc->in_dtype, x, xs, (cudaStream_t)stream));
}

ss2d_status_t ss2d_cross_merge(const ss2d_desc_t *desc, const void *ys, void *y, ss2d_stream_t stream) {
    SS2D_TRY(check_desc(desc));
    SS2D_TRY(need(ys));
    SS2D_TRY(need(y));
    SS2D_TRY(check_device());
    return from_cuda(
        launch_cross_merge(shape_of(desc), desc->in_dtype, desc->out_dtype, ys, y, (cudaStream_t)stream));
}

static ss2d_status_t check_scan_inputs(const void *u, const void *delta, const float *A, const void *Bm,
                                       const void *Cm, const float *D, const float *delta_bias) {
    SS2D_TRY(need(u));
    SS2D_TRY(need(delta));
    SS2D_TRY(need(A));
    SS2D_TRY(need(Bm));
    SS2D_TRY(need(Cm));
    SS2D_TRY(optional(D));
    SS2D_TRY(optional(delta_bias));
    return SS2D_OK;
}

ss2d_status_t ss2d_selective_scan_fwd_ex(const ss2d_desc_t *desc, const void *u, const void *delta, const float *A,
                                         const void *Bm, const void *Cm, const float *D, const void *z,
                                         const float *delta_bias, int delta_softplus, void *out,
                                         float *last_state, float *chunk_states, ss2d_stream_t stream) {
    SS2D_TRY(check_desc(desc));
    SS2D_TRY(check_scan_inputs(u, delta, A, Bm, Cm, D, delta_bias));
    SS2D_TRY(optional(z));
    SS2D_TRY(need(out));
    SS2D_TRY(optional(last_state));
    SS2D_TRY(optional(chunk_states));
    const LaunchShape s = shape_of(desc);
    SS2D_TRY(check_device());
    ScanFwdArgs a;
    a.u = u;
    a.delta = delta;
    a.A = A;
    a.Bm = Bm;
    a.Cm = Cm;
    a.Dv = D;
    a.bias = delta_bias;
    a.softplus = delta_softplus != 0;
    a.out = out;
    a.chunk_states = chunk_states;
    a.z = z;
    a.last_state = last_state;
    a.from_image = false;
    a.in_dtype = desc->in_dtype;
    a.out_dtype = desc->out_dtype;
    a.max_segments = 1;  // this entry point takes no workspace: one pass per sequence
    return from_cuda(launch_scan_fwd(s, a, nullptr, (cudaStream_t)stream));
}

ss2d_status_t ss2d_selective_scan_fwd(const ss2d_desc_t *desc, const void *u, const void *delta, const float *A,
                                      const void *Bm, const void *Cm, const float *D, const float *delta_bias,
                                      int delta_softplus, void *out, float *chunk_states, ss2d_stream_t stream) {
    return ss2d_selective_scan_fwd_ex(desc, u, delta, A, Bm, Cm, D, nullptr, delta_bias, delta_softplus, out,
                                      nullptr, chunk_states, stream);
}

ss2d_status_t ss2d_selective_scan_bwd_ex(const ss2d_desc_t *desc, const void *u, const void *delta, const float *A,
                                         const void *Bm, const void *Cm, const float *D, const void *z,
                                         const float *delta_bias, int delta_softplus, const void *dout,
                                         const float *chunk_states, void *du, void *ddelta, float *dA, void *dBm,
                                         void *dCm, float *dD, float *ddelta_bias, void *dz, void *workspace,
                                         size_t workspace_bytes, ss2d_stream_t stream) {
    SS2D_TRY(check_desc(desc));
    SS2D_TRY(check_scan_inputs(u, delta, A, Bm, Cm, D, delta_bias));
    SS2D_TRY(optional(z));
    SS2D_TRY(need(dout));
    SS2D_TRY(optional(chunk_states));
    SS2D_TRY(need(du));
    SS2D_TRY(need(ddelta));
    SS2D_TRY(need(dA));
    SS2D_TRY(need(dBm));
    SS2D_TRY(need(dCm));
    if ((D == nullptr) != (dD == nullptr)) return SS2D_ERR_NULL;
    if ((delta_bias == nullptr) != (ddelta_bias == nullptr)) return SS2D_ERR_NULL;
    if ((z == nullptr) != (dz == nullptr)) return SS2D_ERR_NULL;
    SS2D_TRY(optional(dD));
    SS2D_TRY(optional(ddelta_bias));
    SS2D_TRY(optional(dz));
    const LaunchShape s = shape_of(desc);
    const size_t ws = scan_bwd_workspace_bytes(s);
    if (ws > 0 && (!workspace || workspace_bytes < ws)) return SS2D_ERR_WORKSPACE;
    SS2D_TRY(optional(workspace));
    SS2D_TRY(check_device());
    ScanBwdArgs a;
    a.u = u;
    a.delta = delta;
    a.A = A;
    a.Bm = Bm;
    a.Cm = Cm;
    a.Dv = D;
    a.bias = delta_bias;
    a.softplus = delta_softplus != 0;
    a.dout = dout;
    a.chunk_states = chunk_states;
    a.du = du;
    a.ddelta = ddelta;
    a.dA = dA;
    a.dBm = dBm;
    a.dCm = dCm;
    a.dD = dD;
    a.dbias = ddelta_bias;
    a.z = z;
    a.dz = dz;
    a.from_image = false;
    a.in_dtype = desc->in_dtype;
    a.out_dtype = desc->out_dtype;
    return from_cuda(launch_scan_bwd(s, a, workspace, workspace_bytes, (cudaStream_t)stream));
}

ss2d_status_t ss2d_selective_scan_bwd(const ss2d_desc_t *desc, const void *u, const void *delta, const float *A,
                                      const void *Bm, const void *Cm, const float *D, const float *delta_bias,
                                      int delta_softplus, const void *dout, const float *chunk_states, void *du,
                                      void *ddelta, float *dA, void *dBm, void *dCm, float *dD,
                                      float *ddelta_bias, void *workspace, size_t workspace_bytes,
                                      ss2d_stream_t stream) {
    return ss2d_selective_scan_bwd_ex(desc, u, delta, A, Bm, Cm, D, nullptr, delta_bias, delta_softplus, dout,
                                      chunk_states, du, ddelta, dA, dBm, dCm, dD, ddelta_bias, nullptr, workspace,
                                      workspace_bytes, stream);
}

ss2d_status_t ss2d_forward_proj(const ss2d_desc_t *desc, int dt_rank, const void *x, const float *x_proj_weight,
                                const float *dt_proj_weight, const float *dt_proj_bias, const float *A,
                                const float *D, int delta_softplus, void *y, void *x_dbl, float *chunk_states,
                                void *workspace, size_t workspace_bytes, ss2d_stream_t stream) {
    SS2D_TRY(check_desc(desc));
    if (dt_rank < 1 || dt_rank > kProjRMax) return SS2D_ERR_SHAPE;
    SS2D_TRY(need(x));
    SS2D_TRY(need(x_proj_weight));
    SS2D_TRY(need(dt_proj_weight));
    SS2D_TRY(optional(dt_proj_bias));
    SS2D_TRY(need(A));
    SS2D_TRY(optional(D));
    SS2D_TRY(need(y));
    SS2D_TRY(need(x_dbl));
    SS2D_TRY(optional(chunk_states));
    const LaunchShape s = shape_of(desc);
    const size_t delta_bytes = round64((size_t)s.B * kPaths * s.D * s.L * elem_size(desc->in_dtype));
    const size_t ws = fwd_ws_bytes(s, desc->in_dtype) + delta_bytes;
    if (!workspace || workspace_bytes < ws) return SS2D_ERR_WORKSPACE;
    SS2D_TRY(optional(workspace));
    SS2D_TRY(check_device());
    unsigned char *w = static_cast<unsigned char *>(workspace);
    void *delta = w;  // used for ranks above kProjRNarrow only
    w += delta_bytes;
    float *ys = reinterpret_cast<float *>(w);
    w += round64((size_t)s.B * kPaths * s.D * s.L * sizeof(float));
    void *xT = w;
    w += round64((size_t)s.B * s.D * s.L * elem_size(desc->in_dtype));
    void *seg = w;
    cudaStream_t st = (cudaStream_t)stream;
    SS2D_TRY(from_cuda(launch_transpose(s, desc->in_dtype, x, xT, st)));
    const int RN = dt_rank + 2 * (int)s.N;
    SS2D_TRY(from_cuda(launch_xproj(s, desc->in_dtype, x, xT, x_proj_weight, RN, x_dbl, st)));
    const bool materialise = dt_rank > kProjRNarrow;
    if (materialise) SS2D_TRY(from_cuda(launch_dtproj(s, desc->in_dtype, x_dbl, dt_proj_weight, dt_rank, RN, delta, st)));
    ScanFwdArgs a;
    a.u = x;
    a.uT = xT;
    a.delta = materialise ? delta : nullptr;
    a.A = A;
    a.Bm = nullptr;
    a.Cm = nullptr;
    a.Dv = D;
    a.bias = dt_proj_bias;
    a.softplus = delta_softplus != 0;
    a.out = ys;
    a.chunk_states = chunk_states;
    a.from_image = true;
    a.xdbl = x_dbl;
    a.Wdt = dt_proj_weight;
    a.R = dt_rank;
    a.in_dtype = desc->in_dtype;
    a.out_dtype = SS2D_F32;
    SS2D_TRY(from_cuda(launch_scan_fwd(s, a, seg, st)));
    return from_cuda(launch_cross_merge(s, SS2D_F32, desc->out_dtype, ys, y, st));
}

ss2d_status_t ss2d_backward_proj(const ss2d_desc_t *desc, int dt_rank, const void *x, const float *x_proj_weight,
                                 const float *dt_proj_weight, const float *dt_proj_bias, const float *A,
                                 const float *D, int delta_softplus, const void *x_dbl, const float *chunk_states,
                                 const void *dy, void *dx, float *dx_proj_weight, float *ddt_proj_weight,
                                 float *ddt_proj_bias, float *dA, float *dD, void *workspace, size_t workspace_bytes,
                                 ss2d_stream_t stream) {
    SS2D_TRY(check_desc(desc));
    if (dt_rank < 1 || dt_rank > kProjRMax) return SS2D_ERR_SHAPE;
    SS2D_TRY(need(x));
    SS2D_TRY(need(x_proj_weight));
    SS2D_TRY(need(dt_proj_weight));
    SS2D_TRY(optional(dt_proj_bias));
    SS2D_TRY(need(A));
    SS2D_TRY(optional(D));
    SS2D_TRY(need(x_dbl));
    SS2D_TRY(optional(chunk_states));
    SS2D_TRY(need(dy));
    SS2D_TRY(need(dx));
    SS2D_TRY(need(dx_proj_weight));
    SS2D_TRY(need(ddt_proj_weight));
    SS2D_TRY(need(dA));
    if ((D == nullptr) != (dD == nullptr)) return SS2D_ERR_NULL;
    if ((dt_proj_bias == nullptr) != (ddt_proj_bias == nullptr)) return SS2D_ERR_NULL;
    SS2D_TRY(optional(dD));
    SS2D_TRY(optional(ddt_proj_bias));
    const LaunchShape s = shape_of(desc);
    const ss2d_dtype_t in = desc->in_dtype;
    if (!workspace || workspace_bytes < proj_bwd_ws_bytes(s, in, desc->out_dtype)) return SS2D_ERR_WORKSPACE;
    SS2D_TRY(optional(workspace));
    SS2D_TRY(check_device());
    const int R = dt_rank, RN = R + 2 * (int)s.N;
    const size_t seq = (size_t)s.B * kPaths * s.D * s.L, img = (size_t)s.B * s.D * s.L;
    const size_t bc = (size_t)s.B * kPaths * s.N * s.L, es = elem_size(in);
    unsigned char *w = static_cast<unsigned char *>(workspace);
    auto take = [&w](size_t bytes) {
        void *p = w;
        w += round64(bytes);
        return p;
    };
    float *du_seq = static_cast<float *>(take(seq * sizeof(float)));
    void *xT = take(img * es);
    void *dyT = take(img * elem_size(desc->out_dtype));
    void *delta = take(seq * es);
    void *ddelta = take(seq * es);
    void *Bm = take(bc * es);
    void *Cm = take(bc * es);
    void *dBm = take(bc * es);
    void *dCm = take(bc * es);
    float *dxdbl = static_cast<float *>(take((size_t)s.B * kPaths * (kProjRMax + 2 * s.N) * s.L * sizeof(float)));
    float *part = static_cast<float *>(
        take((size_t)kPaths * s.B * proj_bwd_chunks(s) * (kProjRMax + 2 * s.N) * s.D * sizeof(float)));
    void *inner = w;
    cudaStream_t st = (cudaStream_t)stream;
    SS2D_TRY(from_cuda(launch_transpose(s, in, x, xT, st)));
    SS2D_TRY(from_cuda(launch_transpose(s, desc->out_dtype, dy, dyT, st)));
    SS2D_TRY(from_cuda(launch_dtproj(s, in, x_dbl, dt_proj_weight, R, RN, delta, st)));
    // B and C: rows [R, R+N) and [R+N, R+2N) of every (b, k) block of x_dbl
    const size_t row = (size_t)s.N * s.L * es, pitch = (size_t)RN * s.L * es, blocks = (size_t)s.B * kPaths;
    const unsigned char *xd = static_cast<const unsigned char *>(x_dbl);
    SS2D_TRY(from_cuda(cudaMemcpy2DAsync(Bm, row, xd + (size_t)R * s.L * es, pitch, row, blocks,
                                         cudaMemcpyDeviceToDevice, st)));
    SS2D_TRY(from_cuda(cudaMemcpy2DAsync(Cm, row, xd + (size_t)(R + s.N) * s.L * es, pitch, row, blocks,
                                         cudaMemcpyDeviceToDevice, st)));
    ScanBwdArgs a;
    a.u = x;
    a.uT = xT;
    a.doutT = dyT;
    a.delta = delta;
    a.A = A;
    a.Bm = Bm;
    a.Cm = Cm;
    a.Dv = D;
    a.bias = dt_proj_bias;
    a.softplus = delta_softplus != 0;
    a.dout = dy;
    a.chunk_states = chunk_states;
    a.du = du_seq;
    a.ddelta = ddelta;
    a.dA = dA;
    a.dBm = dBm;
    a.dCm = dCm;
    a.dD = dD;
    a.dbias = ddt_proj_bias;
    a.from_image = true;
    a.in_dtype = in;
    a.out_dtype = desc->out_dtype;
    SS2D_TRY(from_cuda(launch_scan_bwd(s, a, inner, scan_bwd_workspace_bytes(s), st)));
    SS2D_TRY(from_cuda(launch_proj_bwd_dtlow(s, in, ddelta, dt_proj_weight, R, RN, dxdbl, st)));
    SS2D_TRY(from_cuda(launch_proj_bwd_copy_rows(s, in, dBm, (int)s.N, RN, R, dxdbl, st)));
    SS2D_TRY(from_cuda(launch_proj_bwd_copy_rows(s, in, dCm, (int)s.N, RN, R + (int)s.N, dxdbl, st)));
    SS2D_TRY(from_cuda(launch_proj_bwd_dwdt(s, in, ddelta, x_dbl, R, RN, part, ddt_proj_weight, st)));
    SS2D_TRY(from_cuda(launch_proj_bwd_dwx(s, in, dxdbl, x, xT, RN, part, dx_proj_weight, st)));
    SS2D_TRY(from_cuda(launch_proj_bwd_du(s, dxdbl, x_proj_weight, RN, du_seq, st)));
    return from_cuda(launch_cross_merge(s, SS2D_F32, in, du_seq, dx, st));
}

ss2d_status_t ss2d_forward_proj_conv(const ss2d_desc_t *desc, int dt_rank, int d_conv, const void *x,
                                     const float *conv_weight, const float *conv_bias, const float *x_proj_weight,
                                     const float *dt_proj_weight, const float *dt_proj_bias, const float *A,
                                     const float *D, int delta_softplus, void *y, void *x_dbl, float *chunk_states,
                                     void *workspace, size_t workspace_bytes, ss2d_stream_t stream) {
    SS2D_TRY(check_desc(desc));
    if (dt_rank < 1 || dt_rank > kProjRMax || d_conv < 1 || d_conv > 4) return SS2D_ERR_SHAPE;
    SS2D_TRY(need(x));
    SS2D_TRY(need(conv_weight));
    SS2D_TRY(optional(conv_bias));
    SS2D_TRY(need(x_proj_weight));
    SS2D_TRY(need(dt_proj_weight));
    SS2D_TRY(optional(dt_proj_bias));
    SS2D_TRY(need(A));
    SS2D_TRY(optional(D));
    SS2D_TRY(need(y));
    SS2D_TRY(need(x_dbl));
    SS2D_TRY(optional(chunk_states));
    const LaunchShape s = shape_of(desc);
    const ss2d_dtype_t in = desc->in_dtype;
    if (!workspace || workspace_bytes < conv_fwd_ws_bytes(s, in)) return SS2D_ERR_WORKSPACE;
    SS2D_TRY(optional(workspace));
    SS2D_TRY(check_device());
    const int R = dt_rank, RN = R + 2 * (int)s.N;
    const size_t seq = (size_t)s.B * kPaths * s.D * s.L, img = (size_t)s.B * s.D * s.L;
    const size_t bc = (size_t)s.B * kPaths * s.N * s.L, es = elem_size(in);
    unsigned char *w = static_cast<unsigned char *>(workspace);
    auto take = [&w](size_t bytes) {
        void *p = w;
        w += round64(bytes);
        return p;
    };
    void *xT = take(img * es);
    void *u = take(seq * es);
    void *delta = take(seq * es);
    void *Bm = take(bc * es);
    void *Cm = take(bc * es);
    float *ys = static_cast<float *>(take(seq * sizeof(float)));
    void *seg = w;
    cudaStream_t st = (cudaStream_t)stream;
    SS2D_TRY(from_cuda(launch_transpose(s, in, x, xT, st)));
    SS2D_TRY(from_cuda(launch_path_conv_fwd(s, in, x, xT, conv_weight, conv_bias, d_conv, u, st)));
    SS2D_TRY(from_cuda(launch_xproj_seq(s, in, u, x_proj_weight, RN, x_dbl, st)));
    SS2D_TRY(from_cuda(launch_dtproj(s, in, x_dbl, dt_proj_weight, R, RN, delta, st)));
    const size_t row = (size_t)s.N * s.L * es, pitch = (size_t)RN * s.L * es, blocks = (size_t)s.B * kPaths;
    const unsigned char *xd = static_cast<const unsigned char *>(x_dbl);
    SS2D_TRY(from_cuda(cudaMemcpy2DAsync(Bm, row, xd + (size_t)R * s.L * es, pitch, row, blocks,
                                         cudaMemcpyDeviceToDevice, st)));
    SS2D_TRY(from_cuda(cudaMemcpy2DAsync(Cm, row, xd + (size_t)(R + s.N) * s.L * es, pitch, row, blocks,
                                         cudaMemcpyDeviceToDevice, st)));
    ScanFwdArgs a;
    a.u = u;
    a.delta = delta;
    a.A = A;
    a.Bm = Bm;
    a.Cm = Cm;
    a.Dv = D;
    a.bias = dt_proj_bias;
    a.softplus = delta_softplus != 0;
    a.out = ys;
    a.chunk_states = chunk_states;
    a.from_image = false;
    a.in_dtype = in;
    a.out_dtype = SS2D_F32;
    SS2D_TRY(from_cuda(launch_scan_fwd(s, a, seg, st)));
    return from_cuda(launch_cross_merge(s, SS2D_F32, desc->out_dtype, ys, y, st));
}

ss2d_status_t ss2d_backward_proj_conv(const ss2d_desc_t *desc, int dt_rank, int d_conv, const void *x,
                                      const float *conv_weight, const float *conv_bias, const float *x_proj_weight,
                                      const float *dt_proj_weight, const float *dt_proj_bias, const float *A,
                                      const float *D, int delta_softplus, const void *x_dbl,
                                      const float *chunk_states, const void *dy, void *dx, float *dconv_weight,
                                      float *dconv_bias, float *dx_proj_weight, float *ddt_proj_weight,
                                      float *ddt_proj_bias, float *dA, float *dD, void *workspace,
                                      size_t workspace_bytes, ss2d_stream_t stream) {
    SS2D_TRY(check_desc(desc));
    if (dt_rank < 1 || dt_rank > kProjRMax || d_conv < 1 || d_conv > 4) return SS2D_ERR_SHAPE;
    SS2D_TRY(need(x));
    SS2D_TRY(need(conv_weight));
    SS2D_TRY(optional(conv_bias));
    SS2D_TRY(need(x_proj_weight));
    SS2D_TRY(need(dt_proj_weight));
    SS2D_TRY(optional(dt_proj_bias));
    SS2D_TRY(need(A));
    SS2D_TRY(optional(D));
    SS2D_TRY(need(x_dbl));
    SS2D_TRY(optional(chunk_states));
    SS2D_TRY(need(dy));
    SS2D_TRY(need(dx));
    SS2D_TRY(need(dconv_weight));
    SS2D_TRY(need(dx_proj_weight));
    SS2D_TRY(need(ddt_proj_weight));
    SS2D_TRY(need(dA));
    if ((D == nullptr) != (dD == nullptr)) return SS2D_ERR_NULL;
    if ((dt_proj_bias == nullptr) != (ddt_proj_bias == nullptr)) return SS2D_ERR_NULL;
    if ((conv_bias == nullptr) != (dconv_bias == nullptr)) return SS2D_ERR_NULL;
    SS2D_TRY(optional(dD));
    SS2D_TRY(optional(ddt_proj_bias));
    SS2D_TRY(optional(dconv_bias));
    const LaunchShape s = shape_of(desc);
    const ss2d_dtype_t in = desc->in_dtype, out = desc->out_dtype;
    if (!workspace || workspace_bytes < conv_bwd_ws_bytes(s, in, out)) return SS2D_ERR_WORKSPACE;
    SS2D_TRY(optional(workspace));
    SS2D_TRY(check_device());
    const int R = dt_rank, RN = R + 2 * (int)s.N;
    const size_t seq = (size_t)s.B * kPaths * s.D * s.L, img = (size_t)s.B * s.D * s.L;
    const size_t bc = (size_t)s.B * kPaths * s.N * s.L, es = elem_size(in), rn = (size_t)kProjRMax + 2 * s.N;
    unsigned char *w = static_cast<unsigned char *>(workspace);
    auto take = [&w](size_t bytes) {
        void *p = w;
        w += round64(bytes);
        return p;
    };
    void *xT = take(img * es);
    void *u = take(seq * es);
    void *g = take(seq * elem_size(out));
    void *delta = take(seq * es);
    void *ddelta = take(seq * es);
    void *Bm = take(bc * es);
    void *Cm = take(bc * es);
    void *dBm = take(bc * es);
    void *dCm = take(bc * es);
    float *du = static_cast<float *>(take(seq * sizeof(float)));
    float *dxs = static_cast<float *>(take(seq * sizeof(float)));
    float *dxdbl = static_cast<float *>(take((size_t)s.B * kPaths * rn * s.L * sizeof(float)));
    const size_t part_floats =
        std::max((size_t)kPaths * s.B * proj_bwd_chunks(s) * rn * s.D, path_conv_partial_floats(s, 4));
    float *part = static_cast<float *>(take(part_floats * sizeof(float)));
    void *inner = w;
    cudaStream_t st = (cudaStream_t)stream;
    SS2D_TRY(from_cuda(launch_transpose(s, in, x, xT, st)));
    SS2D_TRY(from_cuda(launch_path_conv_fwd(s, in, x, xT, conv_weight, conv_bias, d_conv, u, st)));
    SS2D_TRY(from_cuda(launch_cross_scan(s, out, dy, g, st)));
    SS2D_TRY(from_cuda(launch_dtproj(s, in, x_dbl, dt_proj_weight, R, RN, delta, st)));
    const size_t row = (size_t)s.N * s.L * es, pitch = (size_t)RN * s.L * es, blocks = (size_t)s.B * kPaths;
    const unsigned char *xd = static_cast<const unsigned char *>(x_dbl);
    SS2D_TRY(from_cuda(cudaMemcpy2DAsync(Bm, row, xd + (size_t)R * s.L * es, pitch, row, blocks,
                                         cudaMemcpyDeviceToDevice, st)));
    SS2D_TRY(from_cuda(cudaMemcpy2DAsync(Cm, row, xd + (size_t)(R + s.N) * s.L * es, pitch, row, blocks,
                                         cudaMemcpyDeviceToDevice, st)));
    ScanBwdArgs a;
    a.u = u;
    a.delta = delta;
    a.A = A;
    a.Bm = Bm;
    a.Cm = Cm;
    a.Dv = D;
    a.bias = dt_proj_bias;
    a.softplus = delta_softplus != 0;
    a.dout = g;
    a.chunk_states = chunk_states;
    a.du = du;
    a.ddelta = ddelta;
    a.dA = dA;
    a.dBm = dBm;
    a.dCm = dCm;
    a.dD = dD;
    a.dbias = ddt_proj_bias;
    a.from_image = false;
    a.du_f32 = true;
    a.in_dtype = in;
    a.out_dtype = out;
    SS2D_TRY(from_cuda(launch_scan_bwd(s, a, inner, scan_bwd_workspace_bytes(s), st)));
    SS2D_TRY(from_cuda(launch_proj_bwd_dtlow(s, in, ddelta, dt_proj_weight, R, RN, dxdbl, st)));
    SS2D_TRY(from_cuda(launch_proj_bwd_copy_rows(s, in, dBm, (int)s.N, RN, R, dxdbl, st)));
    SS2D_TRY(from_cuda(launch_proj_bwd_copy_rows(s, in, dCm, (int)s.N, RN, R + (int)s.N, dxdbl, st)));
    SS2D_TRY(from_cuda(launch_proj_bwd_dwdt(s, in, ddelta, x_dbl, R, RN, part, ddt_proj_weight, st)));
    SS2D_TRY(from_cuda(launch_proj_bwd_dwx_seq(s, in, dxdbl, u, RN, part, dx_proj_weight, st)));
    SS2D_TRY(from_cuda(launch_proj_bwd_du(s, dxdbl, x_proj_weight, RN, du, st)));
    SS2D_TRY(from_cuda(launch_path_conv_bwd(s, in, x, xT, conv_weight, conv_bias, d_conv, du, dxs, dconv_weight,
                                            dconv_bias, part, st)));
    return from_cuda(launch_cross_merge(s, SS2D_F32, in, dxs, dx, st));
}

ss2d_status_t ss2d_path_tables(const ss2d_desc_t *desc, int paths, int32_t *tables, ss2d_stream_t stream) {
    SS2D_TRY(check_desc(desc));
    SS2D_TRY(check_table_shape(desc));
    if (paths != SS2D_PATHS_CROSS && paths != SS2D_PATHS_DIAGONAL) return SS2D_ERR_SHAPE;
    SS2D_TRY(need(tables));
    SS2D_TRY(check_device());
    return from_cuda(launch_path_tables(paths, desc->height, desc->width, tables, (cudaStream_t)stream));
}

ss2d_status_t ss2d_cross_scan_table(const ss2d_desc_t *desc, const int32_t *tables, const void *x, void *xs,
                                    ss2d_stream_t stream) {
    SS2D_TRY(check_desc(desc));
    SS2D_TRY(check_table_shape(desc));
    SS2D_TRY(need(tables));
    SS2D_TRY(need(x));
    SS2D_TRY(need(xs));
    SS2D_TRY(check_device());
    return from_cuda(launch_cross_scan_table(shape_of(desc), desc->in_dtype, x, tables, xs, (cudaStream_t)stream));
}

ss2d_status_t ss2d_cross_merge_table(const ss2d_desc_t *desc, const int32_t *tables, const void *ys, void *y,
                                     ss2d_stream_t stream) {
    SS2D_TRY(check_desc(desc));
    SS2D_TRY(check_table_shape(desc));
    SS2D_TRY(need(tables));
    SS2D_TRY(need(ys));
    SS2D_TRY(need(y));
    SS2D_TRY(check_device());
    return from_cuda(launch_cross_merge_table(shape_of(desc), desc->in_dtype, desc->out_dtype, ys, tables, y,
                                              (cudaStream_t)stream));
}

ss2d_status_t ss2d_forward_table(const ss2d_desc_t *desc, const int32_t *tables, const void *x, const void *delta,
                                 const float *A, const void *Bm, const void *Cm, const float *D,
                                 const float *delta_bias, int delta_softplus, void *y, float *chunk_states,
                                 void *workspace, size_t workspace_bytes, ss2d_stream_t stream) {
    SS2D_TRY(check_desc(desc));
    SS2D_TRY(check_table_shape(desc));
    SS2D_TRY(need(tables));
    SS2D_TRY(check_scan_inputs(x, delta, A, Bm, Cm, D, delta_bias));
    SS2D_TRY(need(y));
    SS2D_TRY(optional(chunk_states));
    const LaunchShape s = shape_of(desc);
    if (!workspace || workspace_bytes < table_fwd_ws_bytes(s, desc->in_dtype)) return SS2D_ERR_WORKSPACE;
    SS2D_TRY(optional(workspace));
    SS2D_TRY(check_device());
    const size_t img = round64((size_t)s.B * s.D * s.L * elem_size(desc->in_dtype));
    unsigned char *w = static_cast<unsigned char *>(workspace);
    float *ys = reinterpret_cast<float *>(w);
    w += round64((size_t)s.B * kPaths * s.D * s.L * sizeof(float));
    void *c0 = w;
    void *c1 = w + img;
    void *seg = w + 2 * img;
    cudaStream_t st = (cudaStream_t)stream;
    SS2D_TRY(from_cuda(launch_path_copies(s, desc->in_dtype, x, tables, c0, c1, st)));
    ScanFwdArgs a;
    a.u = c0;   // path 0 (and 2, backwards)
    a.uT = c1;  // path 1 (and 3, backwards)
    a.delta = delta;
    a.A = A;
    a.Bm = Bm;
    a.Cm = Cm;
    a.Dv = D;
    a.bias = delta_bias;
    a.softplus = delta_softplus != 0;
    a.out = ys;
    a.chunk_states = chunk_states;
    a.from_image = true;
    a.in_dtype = desc->in_dtype;
    a.out_dtype = SS2D_F32;
    SS2D_TRY(from_cuda(launch_scan_fwd(s, a, seg, st)));
    return from_cuda(launch_cross_merge_table(s, SS2D_F32, desc->out_dtype, ys, tables, y, st));
}

ss2d_status_t ss2d_backward_table(const ss2d_desc_t *desc, const int32_t *tables, const void *x, const void *delta,
                                  const float *A, const void *Bm, const void *Cm, const float *D,
                                  const float *delta_bias, int delta_softplus, const void *dy,
                                  const float *chunk_states, void *dx, void *ddelta, float *dA, void *dBm, void *dCm,
                                  float *dD, float *ddelta_bias, void *workspace, size_t workspace_bytes,
                                  ss2d_stream_t stream) {
    SS2D_TRY(check_desc(desc));
    SS2D_TRY(check_table_shape(desc));
    SS2D_TRY(need(tables));
    SS2D_TRY(check_scan_inputs(x, delta, A, Bm, Cm, D, delta_bias));
    SS2D_TRY(need(dy));
    SS2D_TRY(optional(chunk_states));
    SS2D_TRY(need(dx));
    SS2D_TRY(need(ddelta));
    SS2D_TRY(need(dA));
    SS2D_TRY(need(dBm));
    SS2D_TRY(need(dCm));
    if ((D == nullptr) != (dD == nullptr)) return SS2D_ERR_NULL;
    if ((delta_bias == nullptr) != (ddelta_bias == nullptr)) return SS2D_ERR_NULL;
    SS2D_TRY(optional(dD));
    SS2D_TRY(optional(ddelta_bias));
    const LaunchShape s = shape_of(desc);
    if (!workspace || workspace_bytes < table_bwd_ws_bytes(s, desc->in_dtype, desc->out_dtype))
        return SS2D_ERR_WORKSPACE;
    SS2D_TRY(optional(workspace));
    SS2D_TRY(check_device());
    const size_t ximg = round64((size_t)s.B * s.D * s.L * elem_size(desc->in_dtype));
    const size_t gimg = round64((size_t)s.B * s.D * s.L * elem_size(desc->out_dtype));
    unsigned char *w = static_cast<unsigned char *>(workspace);
    float *du_seq = reinterpret_cast<float *>(w);
    w += round64((size_t)s.B * kPaths * s.D * s.L * sizeof(float));
    void *x0 = w, *x1 = w + ximg;
    w += 2 * ximg;
    void *g0 = w, *g1 = w + gimg;
    w += 2 * gimg;
    void *inner = w;
    cudaStream_t st = (cudaStream_t)stream;
    SS2D_TRY(from_cuda(launch_path_copies(s, desc->in_dtype, x, tables, x0, x1, st)));
    SS2D_TRY(from_cuda(launch_path_copies(s, desc->out_dtype, dy, tables, g0, g1, st)));
    ScanBwdArgs a;
    a.u = x0;
    a.uT = x1;
    a.dout = g0;
    a.doutT = g1;
    a.delta = delta;
    a.A = A;
    a.Bm = Bm;
    a.Cm = Cm;
    a.Dv = D;
    a.bias = delta_bias;
    a.softplus = delta_softplus != 0;
    a.chunk_states = chunk_states;
    a.du = du_seq;
    a.ddelta = ddelta;
    a.dA = dA;
    a.dBm = dBm;
    a.dCm = dCm;
    a.dD = dD;
    a.dbias = ddelta_bias;
    a.from_image = true;
    a.in_dtype = desc->in_dtype;
    a.out_dtype = desc->out_dtype;
    SS2D_TRY(from_cuda(launch_scan_bwd(s, a, inner, scan_bwd_workspace_bytes(s), st)));
    return from_cuda(launch_cross_merge_table(s, SS2D_F32, desc->in_dtype, du_seq, tables, dx, st));
}

ss2d_status_t ss2d_bimamba_forward(const ss2d_desc_t *desc, const void *x, const void *delta, const float *A,
                                   const void *Bm, const void *Cm, const float *D, const void *z,
                                   const float *delta_bias, int delta_softplus, void *y, float *chunk_states,
                                   void *workspace, size_t workspace_bytes, ss2d_stream_t stream) {
    SS2D_TRY(check_desc(desc));
    if (desc->height != 1) return SS2D_ERR_SHAPE;
    SS2D_TRY(check_scan_inputs(x, delta, A, Bm, Cm, D, delta_bias));
    SS2D_TRY(optional(z));
    SS2D_TRY(need(y));
    SS2D_TRY(optional(chunk_states));
    const LaunchShape s = shape_of(desc);
    const size_t ws = bidir_fwd_ws_bytes(s);
    if (!workspace || workspace_bytes < ws) return SS2D_ERR_WORKSPACE;
    SS2D_TRY(optional(workspace));
    SS2D_TRY(check_device());
    float *ys = static_cast<float *>(workspace);
    void *seg = static_cast<unsigned char *>(workspace) + round64((size_t)s.B * 2 * s.D * s.L * sizeof(float));
    ScanFwdArgs a;
    a.u = x;
    a.delta = delta;
    a.A = A;
    a.Bm = Bm;
    a.Cm = Cm;
    a.Dv = D;
    a.bias = delta_bias;
    a.softplus = delta_softplus != 0;
    a.out = ys;
    a.chunk_states = chunk_states;
    a.from_image = false;
    a.bidir = true;
    a.in_dtype = desc->in_dtype;
    a.out_dtype = SS2D_F32;
    cudaStream_t st = (cudaStream_t)stream;
    SS2D_TRY(from_cuda(launch_scan_fwd(s, a, seg, st)));
    return from_cuda(launch_bidir_sum(ys, z, desc->in_dtype, y, desc->out_dtype, s.B, s.D, s.L, st));
}

ss2d_status_t ss2d_bimamba_backward(const ss2d_desc_t *desc, const void *x, const void *delta, const float *A,
                                    const void *Bm, const void *Cm, const float *D, const void *z,
                                    const float *delta_bias, int delta_softplus, const void *dy,
                                    const float *chunk_states, void *dx, void *ddelta, float *dA, void *dBm,
                                    void *dCm, float *dD, float *ddelta_bias, void *dz, void *workspace,
                                    size_t workspace_bytes, ss2d_stream_t stream) {
    SS2D_TRY(check_desc(desc));
    if (desc->height != 1) return SS2D_ERR_SHAPE;
    SS2D_TRY(check_scan_inputs(x, delta, A, Bm, Cm, D, delta_bias));
    SS2D_TRY(optional(z));
    SS2D_TRY(need(dy));
    SS2D_TRY(optional(chunk_states));
    SS2D_TRY(need(dx));
    SS2D_TRY(need(ddelta));
    SS2D_TRY(need(dA));
    SS2D_TRY(need(dBm));
    SS2D_TRY(need(dCm));
    if ((D == nullptr) != (dD == nullptr)) return SS2D_ERR_NULL;
    if ((delta_bias == nullptr) != (ddelta_bias == nullptr)) return SS2D_ERR_NULL;
    if ((z == nullptr) != (dz == nullptr)) return SS2D_ERR_NULL;
    SS2D_TRY(optional(dD));
    SS2D_TRY(optional(ddelta_bias));
    SS2D_TRY(optional(dz));
    const LaunchShape s = shape_of(desc);
    const size_t ws = bidir_bwd_ws_bytes(s);
    if (!workspace || workspace_bytes < ws) return SS2D_ERR_WORKSPACE;
    SS2D_TRY(optional(workspace));
    SS2D_TRY(check_device());
    const size_t half = round64((size_t)s.B * 2 * s.D * s.L * sizeof(float));
    unsigned char *w = static_cast<unsigned char *>(workspace);
    float *du2 = reinterpret_cast<float *>(w);
    float *dd2 = reinterpret_cast<float *>(w + half);
    float *dz2 = reinterpret_cast<float *>(w + 2 * half);
    ScanBwdArgs a;
    a.u = x;
    a.delta = delta;
    a.A = A;
    a.Bm = Bm;
    a.Cm = Cm;
    a.Dv = D;
    a.bias = delta_bias;
    a.softplus = delta_softplus != 0;
    a.dout = dy;
    a.chunk_states = chunk_states;
    a.du = du2;
    a.ddelta = dd2;
    a.dA = dA;
    a.dBm = dBm;
    a.dCm = dCm;
    a.dD = dD;
    a.dbias = ddelta_bias;
    a.z = z;
    a.dz = z ? dz2 : nullptr;
    a.from_image = false;
    a.bidir = true;
    a.in_dtype = desc->in_dtype;
    a.out_dtype = desc->out_dtype;
    cudaStream_t st = (cudaStream_t)stream;
    SS2D_TRY(from_cuda(launch_scan_bwd(s, a, w + 3 * half, workspace_bytes - 3 * half, st)));
    SS2D_TRY(from_cuda(launch_bidir_sum(du2, nullptr, SS2D_F32, dx, desc->in_dtype, s.B, s.D, s.L, st)));
    SS2D_TRY(from_cuda(launch_bidir_sum(dd2, nullptr, SS2D_F32, ddelta, desc->in_dtype, s.B, s.D, s.L, st)));
    if (z) SS2D_TRY(from_cuda(launch_bidir_sum(dz2, nullptr, SS2D_F32, dz, desc->in_dtype, s.B, s.D, s.L, st)));
    return SS2D_OK;
}

ss2d_status_t ss2d_forward(const ss2d_desc_t *desc, const void *x, const void *delta, const float *A,
                           const void *Bm, const void *Cm, const float *D, const float *delta_bias,
                           int delta_softplus, void *y, float *chunk_states, void *workspace,
                           size_t workspace_bytes, ss2d_stream_t stream) {
    SS2D_TRY(check_desc(desc));
    SS2D_TRY(check_scan_inputs(x, delta, A, Bm, Cm, D, delta_bias));
    SS2D_TRY(need(y));
    SS2D_TRY(optional(chunk_states));
    const LaunchShape s = shape_of(desc);
    const size_t ws = fwd_ws_bytes(s, desc->in_dtype);
    if (ws > 0 && (!workspace || workspace_bytes < ws)) return SS2D_ERR_WORKSPACE;
    SS2D_TRY(optional(workspace));
    SS2D_TRY(check_device());
    unsigned char *w = static_cast<unsigned char *>(workspace);
    float *ys = reinterpret_cast<float *>(w);
    w += round64((size_t)s.B * kPaths * s.D * s.L * sizeof(float));
    void *xT = w;
    w += round64((size_t)s.B * s.D * s.L * elem_size(desc->in_dtype));
    void *seg = w;
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e = launch_transpose(s, desc->in_dtype, x, xT, st);
    if (e != cudaSuccess) return from_cuda(e);
    ScanFwdArgs a;
    a.u = x;
    a.uT = xT;
    a.delta = delta;
    a.A = A;
    a.Bm = Bm;
    a.Cm = Cm;
    a.Dv = D;
    a.bias = delta_bias;
    a.softplus = delta_softplus != 0;
    a.out = ys;
    a.chunk_states = chunk_states;
    a.from_image = true;
    a.in_dtype = desc->in_dtype;
    a.out_dtype = SS2D_F32;
    e = launch_scan_fwd(s, a, seg, st);
    if (e != cudaSuccess) return from_cuda(e);
    return from_cuda(launch_cross_merge(s, SS2D_F32, desc->out_dtype, ys, y, st));
}

ss2d_status_t ss2d_backward(const ss2d_desc_t *desc, const void *x, const void *delta, const float *A,
                            const void *Bm, const void *Cm, const float *D, const float *delta_bias,
                            int delta_softplus, const void *dy, const float *chunk_states, void *dx, void *ddelta,
                            float *dA, void *dBm, void *dCm, float *dD, float *ddelta_bias, void *workspace,
                            size_t workspace_bytes, ss2d_stream_t stream) {
    SS2D_TRY(check_desc(desc));
    SS2D_TRY(check_scan_inputs(x, delta, A, Bm, Cm, D, delta_bias));
    SS2D_TRY(need(dy));
    SS2D_TRY(optional(chunk_states));
    SS2D_TRY(need(dx));
    SS2D_TRY(need(ddelta));
    SS2D_TRY(need(dA));
    SS2D_TRY(need(dBm));
    SS2D_TRY(need(dCm));
    if ((D == nullptr) != (dD == nullptr)) return SS2D_ERR_NULL;
    if ((delta_bias == nullptr) != (ddelta_bias == nullptr)) return SS2D_ERR_NULL;
    SS2D_TRY(optional(dD));
    SS2D_TRY(optional(ddelta_bias));
    const LaunchShape s = shape_of(desc);
    const size_t ws = bwd_fused_ws_bytes(s, desc->in_dtype, desc->out_dtype);
    if (ws > 0 && (!workspace || workspace_bytes < ws)) return SS2D_ERR_WORKSPACE;
    SS2D_TRY(optional(workspace));
    SS2D_TRY(check_device());
    unsigned char *w = static_cast<unsigned char *>(workspace);
    float *du_seq = reinterpret_cast<float *>(w);
    w += round64((size_t)s.B * kPaths * s.D * s.L * sizeof(float));
    void *xT = w;
    w += round64((size_t)s.B * s.D * s.L * elem_size(desc->in_dtype));
    void *dyT = w;
    w += round64((size_t)s.B * s.D * s.L * elem_size(desc->out_dtype));
    void *inner = w;
    cudaStream_t st = (cudaStream_t)stream;
    // the column-major paths read x and dy from transposed copies, so every load is a contiguous row
    cudaError_t e = launch_transpose(s, desc->in_dtype, x, xT, st);
    if (e != cudaSuccess) return from_cuda(e);
    e = launch_transpose(s, desc->out_dtype, dy, dyT, st);
    if (e != cudaSuccess) return from_cuda(e);
    ScanBwdArgs a;
    a.u = x;
    a.uT = xT;
    a.doutT = dyT;
    a.delta = delta;
    a.A = A;
    a.Bm = Bm;
    a.Cm = Cm;
    a.Dv = D;
    a.bias = delta_bias;
    a.softplus = delta_softplus != 0;
    a.dout = dy;
    a.chunk_states = chunk_states;
    a.du = du_seq;
    a.ddelta = ddelta;
    a.dA = dA;
    a.dBm = dBm;
    a.dCm = dCm;
    a.dD = dD;
    a.dbias = ddelta_bias;
    a.from_image = true;
    a.in_dtype = desc->in_dtype;
    a.out_dtype = desc->out_dtype;
    e = launch_scan_bwd(s, a, inner, scan_bwd_workspace_bytes(s), st);
    if (e != cudaSuccess) return from_cuda(e);
    return from_cuda(launch_cross_merge(s, SS2D_F32, desc->in_dtype, du_seq, dx, st));
}

}  // extern "C"

namespace ss2d {

// the argument checks of ss2d_selective_scan_fwd, for entry points defined elsewhere
ss2d_status_t check_scan_fwd_args(const ss2d_desc_t *desc, const void *u, const void *delta, const float *A,
                                  const void *Bm, const void *Cm, const float *D, const float *delta_bias,
                                  const void *out, const float *chunk_states) {
    SS2D_TRY(check_desc(desc));
    SS2D_TRY(check_scan_inputs(u, delta, A, Bm, Cm, D, delta_bias));
    SS2D_TRY(need(out));
    SS2D_TRY(optional(chunk_states));
    return SS2D_OK;
}

ss2d_status_t device_usable() { return check_device(); }

ss2d_status_t status_from_cuda(cudaError_t e) { return from_cuda(e); }

void set_error_message(const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    std::vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
    va_end(ap);
}

}  // namespace ss2d
