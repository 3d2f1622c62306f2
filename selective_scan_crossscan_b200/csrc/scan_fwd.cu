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
// cross-thread scan arithmetic at all.
//
//  * A CTA is one warp: 32 channels of one (b, k).  The headline problem
//    (98,304 sequences) then fits the GPU in a single wave (~21 warps per SM),
//    so no SM idles while a second, nearly empty wave runs.
//  * u and delta are read by each thread along its own sequence, four steps at
//    a time (16-byte loads for fp32, 8-byte for bf16), one group ahead of use.
//  * B[., l] and C[., l] are the same for all 32 threads (group k of batch b):
//    they are staged in shared memory in 32-step chunks with cp.async, double
//    buffered, and read as broadcast vector loads.
//  * The fused SS2D forward reads u from the image along path k: row-major
//    paths from x (k=2 backwards), column-major paths from a transposed copy
//    of x (k=3 backwards), so every load stays sequential.
//
// When a problem has too few sequences to fill the GPU, each sequence is cut
// into segments: a summary pass computes, per segment, the state reached
// from zero and the decay product exp(A * sum dt); the output pass starts
// each segment from the carry combined over the segments before it.
#include "common.cuh"
#include "kernels.h"

namespace ss2d {

constexpr int kWarp = 32;   // threads (= channels) per CTA
constexpr int kLC = 32;     // steps of B/C per staged chunk
constexpr int kG = 4;       // steps per register group
constexpr int kStateChunk = SS2D_CHUNK_LEN;

// Resident CTAs (warps) per SM the forward kernel is compiled for; 21 puts the
// headline problem's 3,072 warps in one wave on 148 SMs, fewer leaves more registers.
#ifndef SS2D_FWD_MIN_BLOCKS
#define SS2D_FWD_MIN_BLOCKS 12
#endif

struct FwdParams {
    const void *u;       // (B, 4D, L) sequences, or image x (B, D, H, W)
    const void *uT;      // transposed image (B, D, W, H) for the column paths (image mode)
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

// Four steps l0..l0+3 of a sequence stored forwards (rev = false) or backwards
// (step l at index L-1-l).  VEC: one aligned vector load; else scalar loads
// with bounds (steps at or past lend read as 0).
template <bool VEC, typename T>
__device__ __forceinline__ void load_group(const T *row, bool rev, int64_t L, int64_t l0, int64_t lend, float v[4]) {
    if (VEC) {
        if (!rev) {
            ld4(row + l0, v);
        } else {
            float w[4];
            ld4(row + (L - 4 - l0), w);
            v[0] = w[3];
            v[1] = w[2];
            v[2] = w[1];
            v[3] = w[0];
        }
    } else {
#pragma unroll
        for (int j = 0; j < kG; ++j) {
            const int64_t l = l0 + j;
            v[j] = (l < lend) ? ld(row + (rev ? (L - 1 - l) : l)) : 0.f;
        }
    }
}

template <typename T>
__device__ __forceinline__ void cp_async_bytes(T *smem_dst, const T *gsrc, int bytes) {
    const unsigned dst = (unsigned)__cvta_generic_to_shared(smem_dst);
    if (bytes == 16)
        asm volatile("cp.async.ca.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(gsrc));
    else if (bytes == 8)
        asm volatile("cp.async.ca.shared.global [%0], [%1], 8;\n" ::"r"(dst), "l"(gsrc));
    else
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(dst), "l"(gsrc));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

// Stage B/C steps [l0, l0+len) of group (b, k) into smem buffers [NS][kLC].
// VEC: 4-element cp.async copies (len is a multiple of 4); else plain loads.
template <int NS, bool VEC, typename Tin>
__device__ __forceinline__ void stage_bc(Tin (*Bs)[kLC], Tin (*Cs)[kLC], const Tin *Bk, const Tin *Ck, int N,
                                         int64_t L, int64_t l0, int len) {
    const int t = threadIdx.x;
    if (VEC) {
        const int q = kLC / 4;
        for (int idx = t; idx < NS * q; idx += kWarp) {
            const int n = idx / q, i4 = (idx % q) * 4;
            if (n < N && i4 < len) {
                cp_async_bytes(&Bs[n][i4], Bk + (int64_t)n * L + l0 + i4, 4 * (int)sizeof(Tin));
                cp_async_bytes(&Cs[n][i4], Ck + (int64_t)n * L + l0 + i4, 4 * (int)sizeof(Tin));
            }
        }
    } else {
        for (int idx = t; idx < NS * kLC; idx += kWarp) {
            const int n = idx / kLC, i = idx % kLC;
            const bool ok = n < N && i < len;
            Bs[n][i] = ok ? Bk[(int64_t)n * L + l0 + i] : Tin(0.f);
            Cs[n][i] = ok ? Ck[(int64_t)n * L + l0 + i] : Tin(0.f);
        }
    }
}

// PASS 0: single pass.  PASS 1: segment summaries only.  PASS 2: outputs with carries.
// SEQ sequences per thread: lane t of the CTA owns channels d0 + t + 32*s, s < SEQ, so
// the B/C loads are shared by SEQ sequences and the independent chains interleave.
template <int NS, int SEQ, typename Tin, typename Tout, bool IMG, int PASS, bool VEC>
__global__ void __launch_bounds__(kWarp, SS2D_FWD_MIN_BLOCKS) scan_fwd_kernel(const FwdParams p) {
    __shared__ __align__(16) Tin Bs[2][NS][kLC];
    __shared__ __align__(16) Tin Cs[2][NS][kLC];
    __shared__ float2 A2s[SEQ][NS][kWarp];  // (A[c,n]*log2 e) twice per lane's channel (kept out of registers)

    const int t = threadIdx.x;
    const int k = blockIdx.y;
    const int64_t b = blockIdx.z / p.nseg;
    const int sg_i = blockIdx.z % p.nseg;
    const int64_t D = p.D, L = p.L, C4 = kPaths * p.D;
    const int64_t d0 = (int64_t)blockIdx.x * (kWarp * SEQ) + t;  // channel of sequence 0
    const int N = p.N;
    const int64_t lbeg = (int64_t)sg_i * p.seglen;
    const int64_t lend = min(L, lbeg + p.seglen);

    bool active[SEQ];
    int64_t c[SEQ];
    float h[SEQ][NS], Dc[SEQ], bias[SEQ], dtsum[SEQ];
#pragma unroll
    for (int q = 0; q < SEQ; ++q) {
        const int64_t d = d0 + kWarp * q;
        active[q] = d < D;
        c[q] = k * D + (active[q] ? d : 0);
        Dc[q] = (active[q] && p.Dv) ? p.Dv[c[q]] : 0.f;
        bias[q] = (active[q] && p.bias) ? p.bias[c[q]] : 0.f;
        dtsum[q] = 0.f;
#pragma unroll
        for (int n = 0; n < NS; ++n) {
            const float a2 = (active[q] && n < N) ? p.A[c[q] * N + n] * kLog2e : 0.f;
            A2s[q][n][t] = make_float2(a2, a2);
            h[q][n] = 0.f;
        }
        if (PASS == 2 && active[q]) {
            // carry into this segment: fold the summaries of the segments before it
            const float *sg = p.seg + (b * C4 + c[q]) * (int64_t)p.nseg * 2 * N;
            for (int s2 = 0; s2 < sg_i; ++s2) {
#pragma unroll
                for (int n = 0; n < NS; ++n)
                    if (n < N) h[q][n] = fmaf(sg[(s2 * 2 + 0) * N + n], h[q][n], sg[(s2 * 2 + 1) * N + n]);
            }
        }
    }
    __syncwarp();

    // sequence 0's rows; sequence q sits 32*q rows further in every (.., channel, L) tensor
    const int64_t qstride = (int64_t)kWarp * L;
    const Tin *urow;
    bool urev;
    if (IMG) {
        const Tin *img = static_cast<const Tin *>((k & 1) ? p.uT : p.u);
        urow = img + (b * D + (active[0] ? d0 : 0)) * L;
        urev = k >= 2;
    } else {
        urow = static_cast<const Tin *>(p.u) + (b * C4 + c[0]) * L;
        urev = false;
    }
    const Tin *drow = static_cast<const Tin *>(p.delta) + (b * C4 + c[0]) * L;
    const Tin *Bk = static_cast<const Tin *>(p.Bm) + (b * kPaths + k) * N * L;
    const Tin *Ck = static_cast<const Tin *>(p.Cm) + (b * kPaths + k) * N * L;
    Tout *orow = p.out ? static_cast<Tout *>(p.out) + (b * C4 + c[0]) * L : nullptr;

    const int64_t nloc = lend - lbeg;
    const int nchunk = (int)ceil_div(nloc, kLC);

    // rows n >= N of the B/C buffers are never copied: zero them once so padded
    // states stay at h = 0 and contribute nothing
    if (VEC && N < NS) {
        Tin *bz = &Bs[0][0][0], *cz = &Cs[0][0][0];
        for (int i = t; i < 2 * NS * kLC; i += kWarp) {
            bz[i] = Tin(0.f);
            cz[i] = Tin(0.f);
        }
        __syncwarp();
    }

    float ucur[SEQ][kG], dcur[SEQ][kG];
#pragma unroll
    for (int q = 0; q < SEQ; ++q)
        if (active[q]) {
            load_group<VEC>(urow + q * qstride, urev, L, lbeg, lend, ucur[q]);
            load_group<VEC>(drow + q * qstride, false, L, lbeg, lend, dcur[q]);
        }
    stage_bc<NS, VEC>(Bs[0], Cs[0], Bk, Ck, N, L, lbeg, (int)min((int64_t)kLC, nloc));
    cp_async_commit();

    for (int ch = 0; ch < nchunk; ++ch) {
        const int64_t cbeg = lbeg + (int64_t)ch * kLC;
        const int clen = (int)min((int64_t)kLC, lend - cbeg);
        const int buf = ch & 1;
        if (ch + 1 < nchunk) {
            const int64_t nbeg = cbeg + kLC;
            stage_bc<NS, VEC>(Bs[buf ^ 1], Cs[buf ^ 1], Bk, Ck, N, L, nbeg, (int)min((int64_t)kLC, lend - nbeg));
            cp_async_commit();
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncwarp();

        for (int g = 0; g < clen; g += kG) {
            const int64_t l0 = cbeg + g;
            const int nvalid = (int)min((int64_t)kG, lend - l0);
            float unx[SEQ][kG], dnx[SEQ][kG];
            const bool more = l0 + kG < lend;
#pragma unroll
            for (int q = 0; q < SEQ; ++q)
                if (more && active[q]) {
                    load_group<VEC>(urow + q * qstride, urev, L, l0 + kG, lend, unx[q]);
                    load_group<VEC>(drow + q * qstride, false, L, l0 + kG, lend, dnx[q]);
                }

            // per sequence: step sizes, dt*u and the skip term, steps (0,1) and (2,3) packed (f32x2)
            float2 dt01[SEQ], dt23[SEQ], dtu01[SEQ], dtu23[SEQ], y01[SEQ], y23[SEQ];
#pragma unroll
            for (int q = 0; q < SEQ; ++q) {
                const float2 t01 = make_float2(dcur[q][0] + bias[q], dcur[q][1] + bias[q]);
                const float2 t23 = make_float2(dcur[q][2] + bias[q], dcur[q][3] + bias[q]);
                dt01[q] = p.softplus ? softplus_f2(t01) : t01;
                dt23[q] = p.softplus ? softplus_f2(t23) : t23;
                if (!VEC && nvalid < kG) {
                    // steps past the end keep h unchanged: dt = 0 gives decay 1 and input 0
                    if (nvalid < 2) dt01[q].y = 0.f;
                    if (nvalid < 3) dt23[q].x = 0.f;
                    dt23[q].y = 0.f;
                }
                const float2 u01 = make_float2(ucur[q][0], ucur[q][1]);
                const float2 u23 = make_float2(ucur[q][2], ucur[q][3]);
                dtu01[q] = __fmul2_rn(dt01[q], u01);
                dtu23[q] = __fmul2_rn(dt23[q], u23);
                // skip term first: u is not needed during the state loop
                y01[q] = __fmul2_rn(make_float2(Dc[q], Dc[q]), u01);
                y23[q] = __fmul2_rn(make_float2(Dc[q], Dc[q]), u23);
            }
#pragma unroll
            for (int n = 0; n < NS; ++n) {
                float bq[kG], cq[kG];
                if (VEC) {
                    ld4(&Bs[buf][n][g], bq);
                    ld4(&Cs[buf][n][g], cq);
                } else {
#pragma unroll
                    for (int j = 0; j < kG; ++j) {
                        bq[j] = (g + j < kLC) ? ld(&Bs[buf][n][g + j]) : 0.f;
                        cq[j] = (g + j < kLC) ? ld(&Cs[buf][n][g + j]) : 0.f;
                    }
                }
                const float2 b01v = make_float2(bq[0], bq[1]), b23v = make_float2(bq[2], bq[3]);
                const float2 c01v = make_float2(cq[0], cq[1]), c23v = make_float2(cq[2], cq[3]);
#pragma unroll
                for (int q = 0; q < SEQ; ++q) {
                    const float2 a2 = A2s[q][n][t];
                    const float2 x01 = __fmul2_rn(dt01[q], a2), x23 = __fmul2_rn(dt23[q], a2);
                    const float2 b01 = __fmul2_rn(dtu01[q], b01v), b23 = __fmul2_rn(dtu23[q], b23v);
                    const float h0 = fmaf(ex2_sfu(x01.x), h[q][n], b01.x);
                    const float h1 = fmaf(ex2_sfu(x01.y), h0, b01.y);
                    const float h2 = fmaf(ex2_sfu(x23.x), h1, b23.x);
                    const float h3 = fmaf(ex2_sfu(x23.y), h2, b23.y);
                    h[q][n] = h3;
                    y01[q] = __ffma2_rn(c01v, make_float2(h0, h1), y01[q]);
                    y23[q] = __ffma2_rn(c23v, make_float2(h2, h3), y23[q]);
                }
            }
#pragma unroll
            for (int q = 0; q < SEQ; ++q) {
                if (!active[q]) continue;
                if (PASS == 1) {
                    dtsum[q] += (dt01[q].x + dt01[q].y) + (dt23[q].x + dt23[q].y);
                } else {
                    const float y[kG] = {y01[q].x, y01[q].y, y23[q].x, y23[q].y};
                    if (orow) {
                        Tout *o = orow + q * qstride;
                        if (VEC) {
                            st4(o + l0, y);
                        } else {
#pragma unroll
                            for (int j = 0; j < kG; ++j)
                                if (j < nvalid) st(o + l0 + j, y[j]);
                        }
                    }
                    const int64_t llast = l0 + nvalid - 1;
                    if (p.chunk_states && (((llast + 1) % kStateChunk) == 0 || llast + 1 == L)) {
                        float *cs = p.chunk_states + ((b * C4 + c[q]) * p.nchunks + llast / kStateChunk) * N;
#pragma unroll
                        for (int n = 0; n < NS; ++n)
                            if (n < N) cs[n] = h[q][n];
                    }
                }
            }
            if (more) {
#pragma unroll
                for (int q = 0; q < SEQ; ++q)
#pragma unroll
                    for (int j = 0; j < kG; ++j) {
                        ucur[q][j] = unx[q][j];
                        dcur[q][j] = dnx[q][j];
                    }
            }
        }
        __syncwarp();  // every lane is done with this buffer before it is refilled
    }

    if (PASS == 1) {
#pragma unroll
        for (int q = 0; q < SEQ; ++q) {
            if (!active[q]) continue;
            float *sg = p.seg + ((b * C4 + c[q]) * (int64_t)p.nseg + sg_i) * 2 * N;
#pragma unroll
            for (int n = 0; n < NS; ++n)
                if (n < N) {
                    sg[n] = ex2_sfu(A2s[q][n][t].x * dtsum[q]);
                    sg[N + n] = h[q][n];
                }
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

// sequences per thread (see scan_fwd_kernel)
#ifndef SS2D_FWD_SEQ
#define SS2D_FWD_SEQ 1
#endif

template <int NS, typename Tin, typename Tout, bool IMG, bool VEC>
static cudaError_t launch_ns(const FwdParams &p, cudaStream_t stream) {
    constexpr int SEQ = SS2D_FWD_SEQ;
    dim3 grid((unsigned)ceil_div(p.D, kWarp * SEQ), kPaths, (unsigned)(p.B * p.nseg));
    if (p.nseg == 1) {
        scan_fwd_kernel<NS, SEQ, Tin, Tout, IMG, 0, VEC><<<grid, kWarp, 0, stream>>>(p);
        note_launch(stream);
    } else {
        scan_fwd_kernel<NS, SEQ, Tin, Tout, IMG, 1, VEC><<<grid, kWarp, 0, stream>>>(p);
        note_launch(stream);
        scan_fwd_kernel<NS, SEQ, Tin, Tout, IMG, 2, VEC><<<grid, kWarp, 0, stream>>>(p);
        note_launch(stream);
    }
    return cudaGetLastError();
}

template <typename Tin, typename Tout, bool IMG, bool VEC>
static cudaError_t launch_types(const FwdParams &p, cudaStream_t stream) {
    if (p.N <= 4) return launch_ns<4, Tin, Tout, IMG, VEC>(p, stream);
    if (p.N <= 8) return launch_ns<8, Tin, Tout, IMG, VEC>(p, stream);
    return launch_ns<16, Tin, Tout, IMG, VEC>(p, stream);
}

template <bool IMG, bool VEC>
static cudaError_t launch_img(const FwdParams &p, ss2d_dtype_t din, ss2d_dtype_t dout, cudaStream_t stream) {
    if (din == SS2D_F32 && dout == SS2D_F32) return launch_types<float, float, IMG, VEC>(p, stream);
    if (din == SS2D_F32) return launch_types<float, __nv_bfloat16, IMG, VEC>(p, stream);
    if (dout == SS2D_F32) return launch_types<__nv_bfloat16, float, IMG, VEC>(p, stream);
    return launch_types<__nv_bfloat16, __nv_bfloat16, IMG, VEC>(p, stream);
}

cudaError_t launch_scan_fwd(const LaunchShape &s, const ScanFwdArgs &a, void *workspace, cudaStream_t stream) {
    FwdParams p;
    p.u = a.u;
    p.uT = a.uT;
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
    // 4-step vector loads need every row start and step group 4-element aligned
    const bool vec = (s.L % 4) == 0;
    if (a.from_image)
        return vec ? launch_img<true, true>(p, a.in_dtype, a.out_dtype, stream)
                   : launch_img<true, false>(p, a.in_dtype, a.out_dtype, stream);
    return vec ? launch_img<false, true>(p, a.in_dtype, a.out_dtype, stream)
               : launch_img<false, false>(p, a.in_dtype, a.out_dtype, stream);
}

}  // namespace ss2d
