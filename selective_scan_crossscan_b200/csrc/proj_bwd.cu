// proj_bwd.cu -- contractions of the producer's backward.
//
// MambaInnerFn.backward ("vision mamba-yolov8", section 2) turns the scan's ddelta, dB and
// dC into the producer's gradients.  Per SS2D path k, over the tokens l of that path:
//     dx_dbl[:R]      = dt_proj.weight^T @ ddelta                (R x D) . (D x L)
//     dx_dbl[R:]      = (dB, dC)
//     d dt_proj.weight = sum over tokens of ddelta (x) x_dbl[:R]  (D x R)
//     d x_proj.weight  = sum over tokens of dx_dbl (x) u_k       (R+2N x D)
//     du_k           += x_proj.weight^T @ dx_dbl                (D x R+2N) . (R+2N x L)
// u_k is x along path k (x or its transpose, paths 2 and 3 backwards).
//
// pp_gemm_kernel does the per-token contractions: a CTA computes a 64 x 64 tile (output rows
// x tokens) of one (b, k) with 256 threads holding 4 x 4 outputs each, streaming the
// contraction dimension through shared memory 16 at a time.  tr_gemm_kernel does the sums over
// tokens: a CTA computes a 64 x 64 tile of a weight gradient over one chunk of one batch
// item's tokens and writes it as a partial; reduce_partials_kernel adds the partials of every
// (batch item, chunk) in a fixed order, so the result is deterministic.  All arithmetic is
// fp32 on the FMA pipe.
#include "common.cuh"
#include "kernels.h"

namespace ss2d {

constexpr int kGT = 64;       // tile edge
constexpr int kGK = 16;       // contraction slice per shared-memory pass
constexpr int kGThreads = 256;

// out[g, m, l] (+)= sum_j M(k, m, j) in[g, j, l], g = b * 4 + k, M(k, m, j) = Mw[k*msk + m*sm + j*sj]
template <typename Tin, typename Tout, bool ACC>
__global__ void __launch_bounds__(kGThreads) pp_gemm_kernel(const Tin *__restrict__ in, int64_t in_gstride,
                                                            const float *__restrict__ Mw, int64_t msk, int64_t sm,
                                                            int64_t sj, Tout *__restrict__ out, int64_t out_gstride,
                                                            int Mrows, int J, int64_t L, int nmt, int64_t nlt) {
    __shared__ __align__(16) float As[kGK][kGT + 4];  // [j][m]
    __shared__ __align__(16) float Bs[kGK][kGT + 4];  // [j][l]
    const int t = threadIdx.x, tx = t % 16, ty = t / 16;
    // one flat grid: output-row tiles fastest (they share the input tile, read once through L2), then tokens, then g
    const int64_t bid = blockIdx.x, rest = bid / nmt, g = rest / nlt, k = g % kPaths;
    const int64_t m0 = (bid % nmt) * kGT, l0 = (rest % nlt) * kGT;
    const Tin *src = in + g * in_gstride;
    float acc[4][4] = {};
    for (int j0 = 0; j0 < J; j0 += kGK) {
        __syncthreads();
        for (int e = t; e < kGK * kGT; e += kGThreads) {
            const int jj = e / kGT, mm = e % kGT;
            const int64_t m = m0 + mm, j = j0 + jj, l = l0 + mm;
            As[jj][mm] = (m < Mrows && j < J) ? Mw[k * msk + m * sm + j * sj] : 0.f;
            Bs[jj][mm] = (j < J && l < L) ? ld(src + j * L + l) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int jj = 0; jj < kGK; ++jj) {
            const float4 a = *reinterpret_cast<const float4 *>(&As[jj][4 * ty]);
            const float4 b = *reinterpret_cast<const float4 *>(&Bs[jj][4 * tx]);
            const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int q = 0; q < 4; ++q) acc[i][q] = fmaf(av[i], bv[q], acc[i][q]);
        }
    }
    Tout *dst = out + g * out_gstride;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int64_t m = m0 + 4 * ty + i;
        if (m >= Mrows) continue;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int64_t l = l0 + 4 * tx + q;
            if (l < L) {
                Tout *o = dst + m * L + l;
                st(o, ACC ? ld(o) + acc[i][q] : acc[i][q]);
            }
        }
    }
}

// part[((k * B + b) * nlc + lc), m, n] = sum over l in chunk lc of A(b, k, m, l) * Bop(b, k, n, l),
// A(b, k, m, l) = A[b*a_bs + k*a_ks + m*L + l], Bop(b, k, n, l) = Bp[k][b*b_bs + n*L + (rev_k ? L-1-l : l)]
struct TrArgs {
    const void *A;
    int64_t a_bs, a_ks;
    const void *Bp[kPaths];
    int64_t b_bs;
    int rev_mask;
    int M, N;
    int64_t B, L;
    int64_t lchunk;
    int nlc;
    int nmt, nnt;  // tiles of M and of N
    float *part;
};

template <typename TA, typename TB>
__global__ void __launch_bounds__(kGThreads) tr_gemm_kernel(const TrArgs p) {
    __shared__ __align__(16) float As[kGK][kGT + 4];  // [token][m]
    __shared__ __align__(16) float Bs[kGK][kGT + 4];  // [token][n]
    const int t = threadIdx.x, tx = t % 16, ty = t / 16;
    // one flat grid: N tiles fastest, then M tiles, then (path, batch item, token chunk)
    const int64_t bid = blockIdx.x, r1 = bid / p.nnt, z = r1 / p.nmt;
    const int64_t k = z % kPaths, rest = z / kPaths, b = rest / p.nlc, lc = rest % p.nlc;
    const int64_t n0 = (bid % p.nnt) * kGT, m0 = (r1 % p.nmt) * kGT;
    const int64_t lb = lc * p.lchunk, le = min(p.L, lb + p.lchunk);
    const TA *A = static_cast<const TA *>(p.A) + b * p.a_bs + k * p.a_ks;
    const void *bk = k == 0 ? p.Bp[0] : k == 1 ? p.Bp[1] : k == 2 ? p.Bp[2] : p.Bp[3];  // no local copy of p.Bp
    const TB *Bo = static_cast<const TB *>(bk) + b * p.b_bs;
    const bool rev = (p.rev_mask >> k) & 1;
    float acc[4][4] = {};
    for (int64_t t0 = lb; t0 < le; t0 += kGK) {
        __syncthreads();
        for (int e = t; e < kGK * kGT; e += kGThreads) {
            const int rr = e / kGK, tt = e % kGK;  // row of the tile, token of the slice (tokens fastest)
            const int64_t l = t0 + tt, m = m0 + rr, n = n0 + rr;
            const bool ok = l < le;
            As[tt][rr] = (ok && m < p.M) ? ld(A + m * p.L + l) : 0.f;
            Bs[tt][rr] = (ok && n < p.N) ? ld(Bo + n * p.L + (rev ? p.L - 1 - l : l)) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int tt = 0; tt < kGK; ++tt) {
            const float4 a = *reinterpret_cast<const float4 *>(&As[tt][4 * ty]);
            const float4 bq = *reinterpret_cast<const float4 *>(&Bs[tt][4 * tx]);
            const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {bq.x, bq.y, bq.z, bq.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int q = 0; q < 4; ++q) acc[i][q] = fmaf(av[i], bv[q], acc[i][q]);
        }
    }
    float *dst = p.part + ((k * p.B + b) * p.nlc + lc) * (int64_t)p.M * p.N;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int64_t m = m0 + 4 * ty + i;
        if (m >= p.M) continue;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int64_t n = n0 + 4 * tx + q;
            if (n < p.N) dst[m * p.N + n] = acc[i][q];
        }
    }
}

// out[k, m, n] = sum over (b, lc) of part[(k * B + b) * nlc + lc][m][n], in that order
__global__ void reduce_partials_kernel(const float *__restrict__ part, float *__restrict__ out, int64_t nparts,
                                       int64_t MN) {
    const int64_t total = kPaths * MN;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t k = e / MN, mn = e - k * MN;
        const float *src = part + k * nparts * MN + mn;
        float s = 0.f;
        for (int64_t i = 0; i < nparts; ++i) s += src[i * MN];
        out[e] = s;
    }
}

// dst[g, off + r, l] = src[g, r, l] for r < rows (fp32 destination)
template <typename Tin>
__global__ void copy_rows_kernel(const Tin *__restrict__ src, float *__restrict__ dst, int64_t G, int rows,
                                 int dst_rows, int off, int64_t L) {
    const int64_t total = G * rows * L;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t g = e / (rows * L), rem = e - g * rows * L;
        dst[(g * dst_rows + off) * L + rem] = ld(src + e);
    }
}

// ------------------------------------------------------------------ launchers --

static int grid_cap(int64_t items, int threads) {
    const int64_t want = ceil_div(items, threads);
    return (int)(want < 148 * 16 ? (want > 0 ? want : 1) : 148 * 16);
}

template <typename Tin, typename Tout, bool ACC>
static cudaError_t pp_gemm_t(const void *in, int64_t in_gs, const float *Mw, int64_t msk, int64_t sm, int64_t sj, void *out,
                      int64_t out_gs, int Mrows, int J, int64_t L, int64_t groups, cudaStream_t stream) {
    const int nmt = (int)ceil_div(Mrows, kGT);
    const int64_t nlt = ceil_div(L, kGT), blocks = nmt * nlt * groups;
    if (blocks > INT32_MAX) return cudaErrorInvalidConfiguration;
    pp_gemm_kernel<Tin, Tout, ACC><<<(unsigned)blocks, kGThreads, 0, stream>>>(
        static_cast<const Tin *>(in), in_gs, Mw, msk, sm, sj, static_cast<Tout *>(out), out_gs, Mrows, J, L, nmt, nlt);
    return cudaSuccess;
}

// dx_dbl[:R] (fp32, group stride RN*L) = dt_proj.weight^T @ ddelta (in dtype, group stride D*L)
cudaError_t launch_proj_bwd_dtlow(const LaunchShape &s, ss2d_dtype_t dt, const void *ddelta, const float *Wdt, int R,
                                  int RN, float *dxdbl, cudaStream_t stream) {
    // M(k, m = r, j = d) = Wdt[(k*D + d)*R + r]
    const cudaError_t e =
        dt == SS2D_F32
            ? pp_gemm_t<float, float, false>(ddelta, s.D * s.L, Wdt, s.D * R, 1, R, dxdbl, (int64_t)RN * s.L, R,
                                             (int)s.D, s.L, s.B * kPaths, stream)
            : pp_gemm_t<__nv_bfloat16, float, false>(ddelta, s.D * s.L, Wdt, s.D * R, 1, R, dxdbl, (int64_t)RN * s.L,
                                                     R, (int)s.D, s.L, s.B * kPaths, stream);
    if (e != cudaSuccess) return e;
    note_launch(stream);
    return cudaGetLastError();
}

// du_seq (fp32, (B, 4D, L)) += x_proj.weight^T @ dx_dbl (fp32, group stride RN*L)
cudaError_t launch_proj_bwd_du(const LaunchShape &s, const float *dxdbl, const float *Wx, int RN, float *du_seq,
                               cudaStream_t stream) {
    // M(k, m = d, j = c) = Wx[(k*RN + c)*D + d]
    const cudaError_t e = pp_gemm_t<float, float, true>(dxdbl, (int64_t)RN * s.L, Wx, (int64_t)RN * s.D, 1, s.D, du_seq,
                                                        s.D * s.L, (int)s.D, RN, s.L, s.B * kPaths, stream);
    if (e != cudaSuccess) return e;
    note_launch(stream);
    return cudaGetLastError();
}

cudaError_t launch_proj_bwd_copy_rows(const LaunchShape &s, ss2d_dtype_t dt, const void *src, int rows, int RN,
                                      int off, float *dxdbl, cudaStream_t stream) {
    const int64_t G = s.B * kPaths;
    const int grid = grid_cap(G * rows * s.L, 256);
    if (dt == SS2D_F32)
        copy_rows_kernel<float><<<grid, 256, 0, stream>>>(static_cast<const float *>(src), dxdbl, G, rows, RN, off, s.L);
    else
        copy_rows_kernel<__nv_bfloat16><<<grid, 256, 0, stream>>>(static_cast<const __nv_bfloat16 *>(src), dxdbl, G,
                                                                  rows, RN, off, s.L);
    note_launch(stream);
    return cudaGetLastError();
}

int64_t proj_bwd_chunks(const LaunchShape &s) { return ceil_div(s.L, kProjTokenChunk); }

template <typename TA, typename TB>
static cudaError_t token_reduce_t(const LaunchShape &s, TrArgs p, float *out, cudaStream_t stream) {
    p.B = s.B;
    p.L = s.L;
    p.lchunk = kProjTokenChunk;
    p.nlc = (int)proj_bwd_chunks(s);
    p.nmt = (int)ceil_div(p.M, kGT);
    p.nnt = (int)ceil_div(p.N, kGT);
    const int64_t blocks = (int64_t)p.nmt * p.nnt * kPaths * s.B * p.nlc;
    if (blocks > INT32_MAX) return cudaErrorInvalidConfiguration;
    tr_gemm_kernel<TA, TB><<<(unsigned)blocks, kGThreads, 0, stream>>>(p);
    note_launch(stream);
    const int64_t MN = (int64_t)p.M * p.N;
    reduce_partials_kernel<<<grid_cap(kPaths * MN, 256), 256, 0, stream>>>(p.part, out, s.B * p.nlc, MN);
    note_launch(stream);
    return cudaGetLastError();
}

// d dt_proj.weight (4, D, R) = sum over tokens of ddelta (x) x_dbl[:R]
cudaError_t launch_proj_bwd_dwdt(const LaunchShape &s, ss2d_dtype_t dt, const void *ddelta, const void *xdbl, int R,
                                 int RN, float *part, float *dWdt, cudaStream_t stream) {
    TrArgs p{};
    p.A = ddelta;
    p.a_bs = kPaths * s.D * s.L;
    p.a_ks = s.D * s.L;
    const size_t es = dt == SS2D_F32 ? 4 : 2;
    for (int k = 0; k < kPaths; ++k)
        p.Bp[k] = static_cast<const unsigned char *>(xdbl) + (size_t)k * RN * s.L * es;
    p.b_bs = (int64_t)kPaths * RN * s.L;
    p.rev_mask = 0;
    p.M = (int)s.D;
    p.N = R;
    p.part = part;
    if (dt == SS2D_F32) return token_reduce_t<float, float>(s, p, dWdt, stream);
    return token_reduce_t<__nv_bfloat16, __nv_bfloat16>(s, p, dWdt, stream);
}

// d x_proj.weight (4, RN, D) = sum over tokens of dx_dbl (x) u_k, u_k = x / xT along path k
cudaError_t launch_proj_bwd_dwx(const LaunchShape &s, ss2d_dtype_t dt, const float *dxdbl, const void *x,
                                const void *xT, int RN, float *part, float *dWx, cudaStream_t stream) {
    TrArgs p{};
    p.A = dxdbl;
    p.a_bs = (int64_t)kPaths * RN * s.L;
    p.a_ks = (int64_t)RN * s.L;
    p.Bp[0] = x;
    p.Bp[1] = xT;
    p.Bp[2] = x;
    p.Bp[3] = xT;
    p.b_bs = s.D * s.L;
    p.rev_mask = 0b1100;  // paths 2 and 3 walk their base order backwards
    p.M = RN;
    p.N = (int)s.D;
    p.part = part;
    if (dt == SS2D_F32) return token_reduce_t<float, float>(s, p, dWx, stream);
    return token_reduce_t<float, __nv_bfloat16>(s, p, dWx, stream);
}

}  // namespace ss2d
