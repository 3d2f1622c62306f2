// scan_fwd.cu -- S6 selective-scan forward engine.
//
// Arithmetic ("vision mamba-yolov8", section "2. Vmamba module code",
// selective_scan_ref): dt = softplus(delta + bias); per state n
// h = exp(dt*A[c,n]) * h + dt*B[n,l]*u; y = sum_n C[n,l]*h + D[c]*u; h = 0 at
// the start; channel c = k*D + d uses the B/C group k.
//
// Design (B200, sm_100a).  The work is one exponential per state update, so
// the engine is bound by the SFU (MUFU.EX2: 16 per clock per SM) and by issue
// slots, not by HBM.  Each thread owns one whole (b, c) sequence with all N
// states in registers and walks it in order: per state update that is one
// FMUL (dt * A*log2e), one MUFU.EX2, one FMUL (dt*u * B) and two FFMAs -- no
// cross-thread scan arithmetic at all.  A CTA holds 64 channels of one (b, k),
// so B[., l] and C[., l] are the same for all its threads: they are staged in
// shared memory as [step][state] and read as broadcast 16-byte loads.  u and
// delta are staged per 32-step chunk with coalesced loads.
//
// When a problem has too few sequences to fill the GPU, each sequence is cut
// into segments: a summary pass computes, per segment, the state reached
// from zero and the decay product exp(A * sum dt); the output pass starts
// each segment from the carry combined over the segments before it.
//
// The fused SS2D forward reads u straight from the (B, D, H, W) image along
// path k (CrossScan folded into the loads).
#include "common.cuh"
#include "kernels.h"

namespace ss2d {

constexpr int kTD = 64;  // channels (= threads) per CTA
constexpr int kLC = 32;  // steps staged per chunk
constexpr int kStateChunk = SS2D_CHUNK_LEN;

struct FwdParams {
    const void *u;
    const void *delta;
    const float *A;
    const void *Bm;
    const void *Cm;
    const float *Dv;
    const float *bias;
    void *out;
    float *chunk_states;
    float *seg;  // (B, 4D, nseg, 2, N): decay product and end state of each segment
    int64_t B, D, H, W, L;
    int N;
    int softplus;
    int nseg;
    int64_t seglen;
    int64_t nchunks;
};

// PASS 0: single pass.  PASS 1: segment summaries only.  PASS 2: outputs with carries.
template <int NS, typename Tin, typename Tout, bool IMG, int PASS>
__global__ void __launch_bounds__(kTD) scan_fwd_kernel(const FwdParams p) {
    __shared__ float us[kTD][kLC + 1];
    __shared__ float ds[kTD][kLC + 1];
    __shared__ __align__(16) float Bs[kLC][NS];
    __shared__ __align__(16) float Cs[kLC][NS];

    const int t = threadIdx.x;
    const int k = blockIdx.y;
    const int64_t b = blockIdx.z / p.nseg;
    const int s = blockIdx.z % p.nseg;
    const int64_t D = p.D, L = p.L, C4 = kPaths * p.D;
    const int64_t d0 = (int64_t)blockIdx.x * kTD;
    const int nch = (int)min((int64_t)kTD, D - d0);
    const bool active = t < nch;
    const int64_t c = k * D + d0 + t;
    const int N = p.N;
    const int64_t lbeg = (int64_t)s * p.seglen;
    const int64_t lend = min(L, lbeg + p.seglen);

    float A2[NS], h[NS];
#pragma unroll
    for (int n = 0; n < NS; ++n) {
        A2[n] = (active && n < N) ? p.A[c * N + n] * kLog2e : 0.f;
        h[n] = 0.f;
    }
    const float Dc = (active && p.Dv) ? p.Dv[c] : 0.f;
    const float bias = (active && p.bias) ? p.bias[c] : 0.f;

    if (PASS == 2 && active) {
        // carry into this segment: fold the summaries of the segments before it
        const float *sg = p.seg + (b * C4 + c) * (int64_t)p.nseg * 2 * N;
        for (int s2 = 0; s2 < s; ++s2) {
#pragma unroll
            for (int n = 0; n < NS; ++n)
                if (n < N) h[n] = fmaf(sg[(s2 * 2 + 0) * N + n], h[n], sg[(s2 * 2 + 1) * N + n]);
        }
    }
    float dtsum = 0.f;

    const Tin *delta = static_cast<const Tin *>(p.delta);
    const Tin *u = static_cast<const Tin *>(p.u);
    const Tin *Bk = static_cast<const Tin *>(p.Bm) + (b * kPaths + k) * N * L;
    const Tin *Ck = static_cast<const Tin *>(p.Cm) + (b * kPaths + k) * N * L;
    Tout *out = static_cast<Tout *>(p.out);

    for (int64_t l0 = lbeg; l0 < lend; l0 += kLC) {
        const int len = (int)min((int64_t)kLC, lend - l0);
        __syncthreads();  // previous chunk fully consumed
        for (int idx = t; idx < kTD * kLC; idx += kTD) {
            const int ch = idx / kLC, i = idx % kLC;
            float uv = 0.f, dv = 0.f;
            if (ch < nch && i < len) {
                const int64_t l = l0 + i;
                const int64_t cc = k * D + d0 + ch;
                dv = ld(delta + (b * C4 + cc) * L + l);
                if (IMG)
                    uv = ld(u + (b * D + d0 + ch) * L + path_pixel(k, l, p.H, p.W));
                else
                    uv = ld(u + (b * C4 + cc) * L + l);
            }
            us[ch][i] = uv;
            ds[ch][i] = dv;
        }
        for (int idx = t; idx < NS * kLC; idx += kTD) {
            const int n = idx / kLC, i = idx % kLC;
            float bv = 0.f, cv = 0.f;
            if (n < N && i < len) {
                bv = ld(Bk + n * L + l0 + i);
                cv = ld(Ck + n * L + l0 + i);
            }
            Bs[i][n] = bv;
            Cs[i][n] = cv;
        }
        __syncthreads();

        if (active) {
            for (int i = 0; i < len; ++i) {
                const float uv = us[t][i];
                const float tt = ds[t][i] + bias;
                const float dt = p.softplus ? softplus_f(tt) : tt;
                const float dtu = dt * uv;
                float y = 0.f;
#pragma unroll
                for (int n4 = 0; n4 < NS / 4; ++n4) {
                    const float4 bq = *reinterpret_cast<const float4 *>(&Bs[i][4 * n4]);
                    const float4 cq = *reinterpret_cast<const float4 *>(&Cs[i][4 * n4]);
                    const float bb[4] = {bq.x, bq.y, bq.z, bq.w};
                    const float cc[4] = {cq.x, cq.y, cq.z, cq.w};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int n = 4 * n4 + j;
                        const float a = ex2_sfu(dt * A2[n]);
                        h[n] = fmaf(a, h[n], dtu * bb[j]);
                        y = fmaf(cc[j], h[n], y);
                    }
                }
                if (PASS == 1) {
                    dtsum += dt;
                } else {
                    us[t][i] = fmaf(Dc, uv, y);
                    const int64_t l = l0 + i;
                    if (p.chunk_states && (((l + 1) % kStateChunk) == 0 || l + 1 == L)) {
                        float *cs = p.chunk_states + ((b * C4 + c) * p.nchunks + l / kStateChunk) * N;
#pragma unroll
                        for (int n = 0; n < NS; ++n)
                            if (n < N) cs[n] = h[n];
                    }
                }
            }
        }
        if (PASS != 1 && p.out) {
            __syncthreads();
            for (int idx = t; idx < kTD * kLC; idx += kTD) {
                const int ch = idx / kLC, i = idx % kLC;
                if (ch < nch && i < len) st(out + (b * C4 + k * D + d0 + ch) * L + l0 + i, us[ch][i]);
            }
        }
    }

    if (PASS == 1 && active) {
        float *sg = p.seg + ((b * C4 + c) * (int64_t)p.nseg + s) * 2 * N;
#pragma unroll
        for (int n = 0; n < NS; ++n)
            if (n < N) {
                sg[n] = ex2_sfu(A2[n] * dtsum);
                sg[N + n] = h[n];
            }
    }
}

// Segment plan: how many segments each sequence is cut into, and their length
// (a multiple of the state-chunk length).  One segment means a single pass.
static void seg_plan(const LaunchShape &s, int max_segments, int *nseg_out, int64_t *seglen_out) {
    // aim for at least ~512 resident sequences (threads) per SM on 148 SMs
    const int64_t seqs = s.B * kPaths * s.D;
    const int64_t target = 148LL * 512;
    *nseg_out = 1;
    *seglen_out = s.L;
    if (seqs >= target || s.L <= 2 * kStateChunk) return;
    int64_t nseg = ceil_div(target, seqs);
    const int64_t max_seg = ceil_div(s.L, kStateChunk);
    if (nseg > max_seg) nseg = max_seg;
    if (nseg > max_segments) nseg = max_segments;
    if (nseg <= 1) return;
    const int64_t seglen = ceil_div(ceil_div(s.L, nseg), kStateChunk) * kStateChunk;
    *seglen_out = seglen;
    *nseg_out = (int)ceil_div(s.L, seglen);
}

int scan_fwd_segments(const LaunchShape &s) {
    int nseg;
    int64_t seglen;
    seg_plan(s, 32, &nseg, &seglen);
    return nseg;
}

size_t scan_fwd_workspace_bytes(const LaunchShape &s) {
    const int nseg = scan_fwd_segments(s);
    if (nseg <= 1) return 0;
    return (size_t)s.B * kPaths * s.D * nseg * 2 * s.N * sizeof(float);
}

template <int NS, typename Tin, typename Tout, bool IMG>
static cudaError_t launch_ns(const LaunchShape &s, const FwdParams &p, cudaStream_t stream) {
    dim3 grid((unsigned)ceil_div(s.D, kTD), kPaths, (unsigned)(s.B * p.nseg));
    if (p.nseg == 1) {
        scan_fwd_kernel<NS, Tin, Tout, IMG, 0><<<grid, kTD, 0, stream>>>(p);
        note_launch(stream);
    } else {
        scan_fwd_kernel<NS, Tin, Tout, IMG, 1><<<grid, kTD, 0, stream>>>(p);
        note_launch(stream);
        scan_fwd_kernel<NS, Tin, Tout, IMG, 2><<<grid, kTD, 0, stream>>>(p);
        note_launch(stream);
    }
    return cudaGetLastError();
}

template <typename Tin, typename Tout, bool IMG>
static cudaError_t launch_types(const LaunchShape &s, const FwdParams &p, cudaStream_t stream) {
    if (s.N <= 4) return launch_ns<4, Tin, Tout, IMG>(s, p, stream);
    if (s.N <= 8) return launch_ns<8, Tin, Tout, IMG>(s, p, stream);
    return launch_ns<16, Tin, Tout, IMG>(s, p, stream);
}

template <bool IMG>
static cudaError_t launch_img(const LaunchShape &s, const FwdParams &p, ss2d_dtype_t din, ss2d_dtype_t dout,
                              cudaStream_t stream) {
    if (din == SS2D_F32 && dout == SS2D_F32) return launch_types<float, float, IMG>(s, p, stream);
    if (din == SS2D_F32) return launch_types<float, __nv_bfloat16, IMG>(s, p, stream);
    if (dout == SS2D_F32) return launch_types<__nv_bfloat16, float, IMG>(s, p, stream);
    return launch_types<__nv_bfloat16, __nv_bfloat16, IMG>(s, p, stream);
}

cudaError_t launch_scan_fwd(const LaunchShape &s, const ScanFwdArgs &a, void *workspace, cudaStream_t stream) {
    FwdParams p;
    p.u = a.u;
    p.delta = a.delta;
    p.A = a.A;
    p.Bm = a.Bm;
    p.Cm = a.Cm;
    p.Dv = a.Dv;
    p.bias = a.bias;
    p.out = a.out;
    p.chunk_states = a.chunk_states;
    p.seg = static_cast<float *>(workspace);
    p.B = s.B;
    p.D = s.D;
    p.H = s.H;
    p.W = s.W;
    p.L = s.L;
    p.N = (int)s.N;
    p.softplus = a.softplus;
    seg_plan(s, a.max_segments, &p.nseg, &p.seglen);
    p.nchunks = ceil_div(s.L, kStateChunk);
    if (a.from_image) return launch_img<true>(s, p, a.in_dtype, a.out_dtype, stream);
    return launch_img<false>(s, p, a.in_dtype, a.out_dtype, stream);
}

}  // namespace ss2d
