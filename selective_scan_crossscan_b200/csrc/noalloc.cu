// noalloc.cu -- an S6 selective-scan forward that needs no workspace from the caller.
//
// Some callers cannot allocate device memory when they call us: a serving loop
// whose memory plan is fixed at start-up, or a host program that links only this
// C library and has no device allocator of its own to hand us a workspace.  This
// entry point is ss2d_selective_scan_fwd with one difference: when a problem has
// too few sequences to fill the GPU, it cuts each sequence into segments (a
// summary pass, then an output pass that starts every segment from the carry of
// the segments before it).  The segment summaries it needs live in the static
// device buffer below instead of in caller-provided memory.
//
// The buffer is a file-scope __device__ array, so every GPU that loads this
// library holds it (16 MiB) until the process exits.  All calls on a device share
// it: calls that may run at the same time on the GPU (different streams, or
// different host threads without ordering) race on it and give wrong results.
// Each call writes every summary entry before reading it, so nothing has to be
// cleared between calls; the buffer simply keeps the last call's contents.
#include <cstdio>
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace ss2d {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB of segment summaries

static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchBytes / sizeof(float)];

// Host code cannot use g_noalloc_scratch's name as a device address; its device
// address is looked up once per device (with that device current) and cached.
static std::mutex g_scratch_mutex;
static void *g_scratch_ptr[64] = {};

static cudaError_t scratch_address(void **out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_ptr[dev]) {
        void *ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = ptr;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

}  // namespace ss2d

using namespace ss2d;

extern "C" {

ss2d_status_t ss2d_selective_scan_fwd_noalloc(const ss2d_desc_t *desc, const void *u, const void *delta,
                                              const float *A, const void *Bm, const void *Cm, const float *D,
                                              const float *delta_bias, int delta_softplus, void *out,
                                              float *chunk_states, ss2d_stream_t stream) {
    // the same argument checks as ss2d_selective_scan_fwd, then the scratch limit
    ss2d_status_t st = check_scan_fwd_args(desc, u, delta, A, Bm, Cm, D, delta_bias, out, chunk_states);
    if (st != SS2D_OK) return st;
    LaunchShape s;
    s.B = desc->batch;
    s.D = desc->dim;
    s.H = desc->height;
    s.W = desc->width;
    s.L = desc->height * desc->width;
    s.N = desc->d_state;
    const size_t need = scan_fwd_workspace_bytes(s);
    if (need > kNoAllocScratchBytes) {
        set_error_message("ss2d_selective_scan_fwd_noalloc: this problem needs %zu bytes of segment summaries; "
                          "the static scratch holds %zu",
                          need, kNoAllocScratchBytes);
        return SS2D_ERR_SHAPE;
    }
    st = device_usable();
    if (st != SS2D_OK) return st;
    void *scratch = nullptr;
    if (need > 0) {
        const cudaError_t e = scratch_address(&scratch);
        if (e != cudaSuccess) return status_from_cuda(e);
    }
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
    a.from_image = false;
    a.in_dtype = desc->in_dtype;
    a.out_dtype = desc->out_dtype;
    a.max_segments = 32;
    return status_from_cuda(launch_scan_fwd(s, a, scratch, (cudaStream_t)stream));
}

}  // extern "C"
