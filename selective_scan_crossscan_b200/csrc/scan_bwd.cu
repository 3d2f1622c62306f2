// scan_bwd.cu -- S6 selective-scan backward engine.
//
// The pages print only the interface of the CUDA backward (SelectiveScanFn.
// backward in "vision mamba-yolov8", section "2. Vmamba module code": it
// returns du, ddelta, dA, dB, dC, dD, ddelta_bias).  The arithmetic is the
// derivative of the forward recurrence h_l = a_l h_{l-1} + dt_l B_l u_l,
// a_l = exp(dt_l A), y_l = C_l . h_l + D u_l, walked backwards with the
// adjoint lambda_l = dLoss/dh_l = C_l g_l + a_{l+1} lambda_{l+1}:
//   dC[n,l] += g_l h_l[n]
//   ddt_l    = sum_n lambda[n] (A[n] a_l[n] h_{l-1}[n] + B[n,l] u_l)
//   dA[n]   += lambda[n] dt_l a_l[n] h_{l-1}[n]
//   dB[n,l] += lambda[n] dt_l u_l
//   du_l     = g_l D + sum_n lambda[n] dt_l B[n,l]
//   ddelta_l = ddt_l * sigmoid(delta_l + bias)   (softplus) or ddt_l
// and a_l h_{l-1} = h_l - dt_l B_l u_l, so the terms need h_l, not h_{l-1}.
//
// Design: one thread per (b, c) sequence with all N states in registers, as
// in the forward.  A CTA is one warp: 32 channels of one (b, k).  The
// sequence is walked backwards in 32-step halves of the forward's 64-step
// state chunks.  Per half: the states are recomputed forward from the chunk
// state, keeping a checkpoint every 4 steps in shared memory; then, for each
// 4-step block from last to first, the block's states are recomputed into
// registers and the adjoint walks back through them.  dB/dC sum over the
// channels of the group: each step's 2N contributions are transposed through
// shared memory and summed by the lanes (fixed order), one CTA partial per
// (b, k, tile); a second kernel sums the partials over tiles (and dA, dD,
// ddelta_bias over the batch) in a fixed order -- no float atomics.
#include "common.cuh"
#include "kernels.h"

namespace ss2d {

constexpr int kBT = 32;    // channels (= threads) per CTA
constexpr int kBH = 32;    // steps per staged half chunk
constexpr int kSub = 4;    // steps per register block
constexpr int kNCk = kBH / kSub;
constexpr int kChunk = SS2D_CHUNK_LEN;  // 64, the forward's state-chunk length
static_assert(kChunk == 2 * kBH, "backward walks each state chunk as two halves");

struct BwdParams {
    const void *u;
    const void *delta;
    const float *A;
    const void *Bm;
    const void *Cm;
    const float *Dv;
    const float *bias;
    const void *dout;
    const float *cs;   // (B, 4D, nchunks, N)
    void *du;
    void *ddelta;
    float *part_bc;    // (B, 4, ntiles, 2N, L)
    float *part_p;     // (B, 4D, N + 2): dA (N), dD, ddelta_bias partials
    int64_t B, D, H, W, L;
    int N;
    int softplus;
    int64_t nchunks;
    int ntiles;
};

template <int NS>
struct BwdSmem {
    float us[kBT][kBH + 1];
    float ds[kBT][kBH + 1];   // delta, overwritten by ddelta
    float gs[kBT][kBH + 1];   // dout, overwritten by du
    float Bs[kBH][NS];
    float Cs[kBH][NS];
    float ck[kBT][kNCk * NS + 4];     // checkpoints, padded rows
    float red[kBT][2 * NS + 1];       // per-step transpose for the channel sum
    float bct[kBH][2 * NS];           // channel sums of the half: [step][dB n | dC n]
};

template <int NS, typename Tin, typename Tg, bool IMG>
__device__ __forceinline__ void stage_half(BwdSmem<NS> &sm, const BwdParams &p, int64_t b, int k, int64_t d0,
                                           int nch, int64_t l0, int len) {
    const int t = threadIdx.x;
    const int64_t D = p.D, L = p.L, C4 = kPaths * p.D;
    const Tin *u = static_cast<const Tin *>(p.u);
    const Tin *delta = static_cast<const Tin *>(p.delta);
    const Tg *g = static_cast<const Tg *>(p.dout);
    for (int idx = t; idx < kBT * kBH; idx += kBT) {
        const int ch = idx / kBH, i = idx % kBH;
        float uv = 0.f, dv = 0.f, gv = 0.f;
        if (ch < nch && i < len) {
            const int64_t l = l0 + i;
            const int64_t cc = k * D + d0 + ch;
            dv = ld(delta + (b * C4 + cc) * L + l);
            if (IMG) {
                const int64_t pix = (b * D + d0 + ch) * L + path_pixel(k, l, p.H, p.W);
                uv = ld(u + pix);
                gv = ld(g + pix);
            } else {
                uv = ld(u + (b * C4 + cc) * L + l);
                gv = ld(g + (b * C4 + cc) * L + l);
            }
        }
        sm.us[ch][i] = uv;
        sm.ds[ch][i] = dv;
        sm.gs[ch][i] = gv;
    }
    const Tin *Bk = static_cast<const Tin *>(p.Bm) + (b * kPaths + k) * p.N * L;
    const Tin *Ck = static_cast<const Tin *>(p.Cm) + (b * kPaths + k) * p.N * L;
    for (int idx = t; idx < NS * kBH; idx += kBT) {
        const int n = idx / kBH, i = idx % kBH;
        float bv = 0.f, cv = 0.f;
        if (n < p.N && i < len) {
            bv = ld(Bk + n * L + l0 + i);
            cv = ld(Ck + n * L + l0 + i);
        }
        sm.Bs[i][n] = bv;
        sm.Cs[i][n] = cv;
    }
}

template <int NS, typename Tin, typename Tg, typename Tdu, bool IMG>
__global__ void __launch_bounds__(kBT) scan_bwd_kernel(const BwdParams p) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    BwdSmem<NS> &sm = *reinterpret_cast<BwdSmem<NS> *>(smem_raw);

    const int t = threadIdx.x;
    const int k = blockIdx.y;
    const int64_t b = blockIdx.z;
    const int64_t D = p.D, L = p.L, C4 = kPaths * p.D;
    const int64_t d0 = (int64_t)blockIdx.x * kBT;
    const int nch = (int)min((int64_t)kBT, D - d0);
    const bool active = t < nch;
    const int64_t c = k * D + d0 + t;
    const int N = p.N;

    float A2[NS], lam[NS], dA[NS];
#pragma unroll
    for (int n = 0; n < NS; ++n) {
        A2[n] = (active && n < N) ? p.A[c * N + n] * kLog2e : 0.f;
        lam[n] = 0.f;
        dA[n] = 0.f;
    }
    const float An_scale = kLn2;  // A = A2 * ln2
    const float Dc = (active && p.Dv) ? p.Dv[c] : 0.f;
    const float bias = (active && p.bias) ? p.bias[c] : 0.f;
    float dD = 0.f, dbias = 0.f;

    Tdu *du_out = static_cast<Tdu *>(p.du);
    Tin *dd_out = static_cast<Tin *>(p.ddelta);
    float *pbc = p.part_bc + ((b * kPaths + k) * p.ntiles + blockIdx.x) * (int64_t)(2 * N) * L;

    for (int64_t J = p.nchunks - 1; J >= 0; --J) {
        const int64_t cbeg = J * kChunk;
        const int clen = (int)min((int64_t)kChunk, L - cbeg);
        float hJ[NS];
        {
            const float *src = (J > 0 && active) ? p.cs + ((b * C4 + c) * p.nchunks + (J - 1)) * N : nullptr;
#pragma unroll
            for (int n = 0; n < NS; ++n) hJ[n] = (src && n < N) ? src[n] : 0.f;
        }
        const int nhalf = clen > kBH ? 2 : 1;
        float hmid[NS];
        if (nhalf == 2) {
            // state after the first half: run it forward once
            __syncthreads();
            stage_half<NS, Tin, Tg, IMG>(sm, p, b, k, d0, nch, cbeg, kBH);
            __syncthreads();
#pragma unroll
            for (int n = 0; n < NS; ++n) hmid[n] = hJ[n];
            if (active) {
                for (int i = 0; i < kBH; ++i) {
                    const float tt = sm.ds[t][i] + bias;
                    const float dt = p.softplus ? softplus_f(tt) : tt;
                    const float dtu = dt * sm.us[t][i];
#pragma unroll
                    for (int n = 0; n < NS; ++n)
                        hmid[n] = fmaf(ex2_sfu(dt * A2[n]), hmid[n], dtu * sm.Bs[i][n]);
                }
            }
        }
        for (int half = nhalf - 1; half >= 0; --half) {
            const int64_t l0 = cbeg + half * kBH;
            const int len = (int)min((int64_t)kBH, L - l0);
            __syncthreads();
            stage_half<NS, Tin, Tg, IMG>(sm, p, b, k, d0, nch, l0, len);
            __syncthreads();
            const int nsub = (len + kSub - 1) / kSub;

            // level 1: checkpoints every kSub steps
            if (active) {
                float h[NS];
#pragma unroll
                for (int n = 0; n < NS; ++n) h[n] = (half == 1) ? hmid[n] : hJ[n];
                for (int q = 0; q < nsub; ++q) {
#pragma unroll
                    for (int n = 0; n < NS; ++n) sm.ck[t][q * NS + n] = h[n];
                    for (int i = q * kSub; i < min(len, q * kSub + kSub); ++i) {
                        const float tt = sm.ds[t][i] + bias;
                        const float dt = p.softplus ? softplus_f(tt) : tt;
                        const float dtu = dt * sm.us[t][i];
#pragma unroll
                        for (int n = 0; n < NS; ++n) h[n] = fmaf(ex2_sfu(dt * A2[n]), h[n], dtu * sm.Bs[i][n]);
                    }
                }
            }

            // level 2 + adjoint walk, 4-step blocks from last to first
            for (int q = nsub - 1; q >= 0; --q) {
                const int i0 = q * kSub;
                const int cnt = min(kSub, len - i0);
                float hist[kSub][NS];
                if (active) {
                    float h[NS];
#pragma unroll
                    for (int n = 0; n < NS; ++n) h[n] = sm.ck[t][q * NS + n];
#pragma unroll
                    for (int j = 0; j < kSub; ++j) {
                        if (j < cnt) {
                            const int i = i0 + j;
                            const float tt = sm.ds[t][i] + bias;
                            const float dt = p.softplus ? softplus_f(tt) : tt;
                            const float dtu = dt * sm.us[t][i];
#pragma unroll
                            for (int n = 0; n < NS; ++n) {
                                // the same rounded dt*u*B as the adjoint subtracts below
                                h[n] = fmaf(ex2_sfu(dt * A2[n]), h[n], __fmul_rn(dtu, sm.Bs[i][n]));
                                hist[j][n] = h[n];
                            }
                        }
                    }
                }
#pragma unroll
                for (int j = kSub - 1; j >= 0; --j) {
                    if (j >= cnt) continue;  // uniform across the warp
                    const int i = i0 + j;
                    float ddt = 0.f;
                    if (active) {
                        const float uv = sm.us[t][i];
                        const float g = sm.gs[t][i];
                        const float tt = sm.ds[t][i] + bias;
                        const float dt = p.softplus ? softplus_f(tt) : tt;
                        const float dtu = dt * uv;
                        float dul = g * Dc;
                        dD = fmaf(g, uv, dD);
#pragma unroll
                        for (int n = 0; n < NS; ++n) {
                            const float Bn = sm.Bs[i][n];
                            const float Cn = sm.Cs[i][n];
                            const float a = ex2_sfu(dt * A2[n]);
                            lam[n] = fmaf(Cn, g, lam[n]);
                            // a_l * h_{l-1}, exactly 0 when h_{l-1} = 0
                            const float ah = __fsub_rn(hist[j][n], __fmul_rn(dtu, Bn));
                            ddt = fmaf(lam[n], fmaf(A2[n] * An_scale, ah, Bn * uv), ddt);
                            dA[n] = fmaf(lam[n] * dt, ah, dA[n]);
                            dul = fmaf(lam[n] * dt, Bn, dul);
                            sm.red[t][n] = lam[n] * dtu;          // dB contribution
                            sm.red[t][NS + n] = g * hist[j][n];    // dC contribution
                            lam[n] *= a;
                        }
                        const float dd = p.softplus ? ddt * sigmoid_f(tt) : ddt;
                        dbias += dd;
                        sm.ds[t][i] = dd;
                        sm.gs[t][i] = dul;
                    } else {
#pragma unroll
                        for (int n = 0; n < 2 * NS; ++n) sm.red[t][n] = 0.f;
                    }
                    __syncwarp();
                    // lane v < 2N sums contribution v over the 32 channels, in lane order
                    if (t < 2 * NS) {
                        float s = 0.f;
#pragma unroll 8
                        for (int r = 0; r < kBT; ++r) s += sm.red[r][t];
                        sm.bct[i][t] = s;
                    }
                    __syncwarp();
                }
            }
            __syncthreads();
            // write du, ddelta and the dB/dC partial of this half
            for (int idx = t; idx < kBT * kBH; idx += kBT) {
                const int ch = idx / kBH, i = idx % kBH;
                if (ch < nch && i < len) {
                    const int64_t cc = k * D + d0 + ch;
                    st(du_out + (b * C4 + cc) * L + l0 + i, sm.gs[ch][i]);
                    st(dd_out + (b * C4 + cc) * L + l0 + i, sm.ds[ch][i]);
                }
            }
            for (int idx = t; idx < 2 * N * kBH; idx += kBT) {
                const int v = idx / kBH, i = idx % kBH;
                const int col = v < N ? v : NS + (v - N);
                if (i < len) pbc[(int64_t)v * L + l0 + i] = sm.bct[i][col];
            }
        }
    }

    if (active) {
        float *pp = p.part_p + (b * C4 + c) * (N + 2);
#pragma unroll
        for (int n = 0; n < NS; ++n)
            if (n < N) pp[n] = dA[n];
        pp[N] = dD;
        pp[N + 1] = dbias;
    }
}

// dB/dC = sum over tiles of the partials (fixed order); dA/dD/ddelta_bias = sum over the batch.
template <typename Tin>
__global__ void bwd_reduce_bc_kernel(const float *__restrict__ part_bc, Tin *__restrict__ dB, Tin *__restrict__ dC,
                                     int64_t B, int N, int64_t L, int ntiles) {
    const int64_t total = B * kPaths * N * L;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t l = e % L;
        const int64_t n = (e / L) % N;
        const int64_t bk = e / (L * N);
        float sb = 0.f, sc = 0.f;
        for (int tl = 0; tl < ntiles; ++tl) {
            const float *pt = part_bc + ((bk * ntiles + tl) * 2 * N) * L;
            sb += pt[n * L + l];
            sc += pt[(N + n) * L + l];
        }
        st(dB + e, sb);
        st(dC + e, sc);
    }
}

__global__ void bwd_reduce_params_kernel(const float *__restrict__ part_p, float *__restrict__ dA, float *__restrict__ dD,
                                         float *__restrict__ dbias, int64_t B, int64_t C4, int N) {
    const int64_t total = C4 * (N + 2);
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t c = e / (N + 2);
        const int v = (int)(e % (N + 2));
        float s = 0.f;
        for (int64_t b = 0; b < B; ++b) s += part_p[(b * C4 + c) * (N + 2) + v];
        if (v < N) dA[c * N + v] = s;
        else if (v == N) { if (dD) dD[c] = s; }
        else if (dbias) dbias[c] = s;
    }
}

// ---------------------------------------------------------------- launch --

static int bwd_tiles(const LaunchShape &s) { return (int)ceil_div(s.D, kBT); }

size_t scan_bwd_workspace_bytes(const LaunchShape &s) {
    const size_t nchunks = (size_t)ceil_div(s.L, kChunk);
    size_t bytes = 0;
    auto add = [&](size_t n) { bytes += (n + 63) / 64 * 64; };
    add((size_t)s.B * kPaths * bwd_tiles(s) * 2 * s.N * s.L * sizeof(float));  // part_bc
    add((size_t)s.B * kPaths * s.D * (s.N + 2) * sizeof(float));               // part_p
    add((size_t)s.B * kPaths * s.D * nchunks * s.N * sizeof(float));            // recomputed chunk states
    add(scan_fwd_workspace_bytes(s));                                           // forward segment summaries
    return bytes;
}

template <int NS, typename Tin, typename Tg, typename Tdu, bool IMG>
static cudaError_t launch_bwd_t(const LaunchShape &s, const BwdParams &p, cudaStream_t stream) {
    const size_t smem = sizeof(BwdSmem<NS>);
    auto kern = scan_bwd_kernel<NS, Tin, Tg, Tdu, IMG>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)bwd_tiles(s), kPaths, (unsigned)s.B);
    kern<<<grid, kBT, smem, stream>>>(p);
    note_launch(stream);
    return cudaGetLastError();
}

template <typename Tin, typename Tg, typename Tdu, bool IMG>
static cudaError_t launch_bwd_ns(const LaunchShape &s, const BwdParams &p, cudaStream_t stream) {
    if (s.N <= 4) return launch_bwd_t<4, Tin, Tg, Tdu, IMG>(s, p, stream);
    if (s.N <= 8) return launch_bwd_t<8, Tin, Tg, Tdu, IMG>(s, p, stream);
    return launch_bwd_t<16, Tin, Tg, Tdu, IMG>(s, p, stream);
}

template <typename Tin, typename Tg, bool IMG>
static cudaError_t launch_bwd_du(const LaunchShape &s, const BwdParams &p, cudaStream_t stream) {
    // the fused backward keeps du in fp32 for the merge that follows
    if (IMG) return launch_bwd_ns<Tin, Tg, float, IMG>(s, p, stream);
    return launch_bwd_ns<Tin, Tg, Tin, IMG>(s, p, stream);
}

template <bool IMG>
static cudaError_t launch_bwd_types(const LaunchShape &s, const BwdParams &p, ss2d_dtype_t din, ss2d_dtype_t dg,
                                    cudaStream_t stream) {
    if (din == SS2D_F32 && dg == SS2D_F32) return launch_bwd_du<float, float, IMG>(s, p, stream);
    if (din == SS2D_F32) return launch_bwd_du<float, __nv_bfloat16, IMG>(s, p, stream);
    if (dg == SS2D_F32) return launch_bwd_du<__nv_bfloat16, float, IMG>(s, p, stream);
    return launch_bwd_du<__nv_bfloat16, __nv_bfloat16, IMG>(s, p, stream);
}

cudaError_t launch_scan_bwd(const LaunchShape &s, const ScanBwdArgs &a, void *workspace, size_t ws_bytes,
                            cudaStream_t stream) {
    (void)ws_bytes;
    const int64_t nchunks = ceil_div(s.L, kChunk);
    unsigned char *ws = static_cast<unsigned char *>(workspace);
    size_t off = 0;
    auto take = [&](size_t n) {
        void *ptr = ws + off;
        off += (n + 63) / 64 * 64;
        return ptr;
    };
    float *part_bc = (float *)take((size_t)s.B * kPaths * bwd_tiles(s) * 2 * s.N * s.L * sizeof(float));
    float *part_p = (float *)take((size_t)s.B * kPaths * s.D * (s.N + 2) * sizeof(float));
    float *cs_ws = (float *)take((size_t)s.B * kPaths * s.D * nchunks * s.N * sizeof(float));
    void *fwd_ws = take(scan_fwd_workspace_bytes(s));

    const float *cs = a.chunk_states;
    cudaError_t e;
    if (!cs) {
        // recompute the forward's chunk states (no outputs written)
        ScanFwdArgs f;
        f.u = a.u;
        f.uT = a.uT;
        f.delta = a.delta;
        f.A = a.A;
        f.Bm = a.Bm;
        f.Cm = a.Cm;
        f.Dv = a.Dv;
        f.bias = a.bias;
        f.softplus = a.softplus;
        f.out = nullptr;
        f.chunk_states = cs_ws;
        f.from_image = a.from_image;
        f.in_dtype = a.in_dtype;
        f.out_dtype = SS2D_F32;
        e = launch_scan_fwd(s, f, fwd_ws, stream);
        if (e != cudaSuccess) return e;
        cs = cs_ws;
    }

    BwdParams p;
    p.u = a.u;
    p.delta = a.delta;
    p.A = a.A;
    p.Bm = a.Bm;
    p.Cm = a.Cm;
    p.Dv = a.Dv;
    p.bias = a.bias;
    p.dout = a.dout;
    p.cs = cs;
    p.du = a.du;
    p.ddelta = a.ddelta;
    p.part_bc = part_bc;
    p.part_p = part_p;
    p.B = s.B;
    p.D = s.D;
    p.H = s.H;
    p.W = s.W;
    p.L = s.L;
    p.N = (int)s.N;
    p.softplus = a.softplus;
    p.nchunks = nchunks;
    p.ntiles = bwd_tiles(s);
    e = a.from_image ? launch_bwd_types<true>(s, p, a.in_dtype, a.out_dtype, stream)
                     : launch_bwd_types<false>(s, p, a.in_dtype, a.out_dtype, stream);
    if (e != cudaSuccess) return e;

    const int threads = 256;
    const int64_t nbc = s.B * kPaths * s.N * s.L;
    const int64_t nblk = ceil_div(nbc, threads);
    const int blocks_bc = (int)(nblk < 148 * 16 ? nblk : 148 * 16);
    if (a.in_dtype == SS2D_F32)
        bwd_reduce_bc_kernel<float><<<blocks_bc, threads, 0, stream>>>(part_bc, (float *)a.dBm, (float *)a.dCm, s.B,
                                                                     (int)s.N, s.L, p.ntiles);
    else
        bwd_reduce_bc_kernel<__nv_bfloat16><<<blocks_bc, threads, 0, stream>>>(
            part_bc, (__nv_bfloat16 *)a.dBm, (__nv_bfloat16 *)a.dCm, s.B, (int)s.N, s.L, p.ntiles);
    note_launch(stream);
    const int64_t np = kPaths * s.D * (s.N + 2);
    bwd_reduce_params_kernel<<<(int)ceil_div(np, threads), threads, 0, stream>>>(part_p, a.dA, a.dD, a.dbias, s.B,
                                                                                kPaths * s.D, (int)s.N);
    note_launch(stream);
    return cudaGetLastError();
}

}  // namespace ss2d
