// conv.cu -- the causal depthwise conv with SiLU in front of the producer, along every path.
//
// MambaInnerFn.forward ("vision mamba-yolov8", section 2) passes its input through
// causal_conv1d_fwd(x, weight, bias, True) before x_proj: a depthwise conv of width W over the
// sequence, reading the current and the W-1 previous steps, then SiLU.  The Visual Mamba page's
// SS2D runs one Mamba block per scan direction, so here every path k has its own weights and
// convolves x read along its own step order:
//     pre_k[d, l] = bias[k, d] + sum_j w[k, d, j] x_k[d, l - (W-1) + j]     (x_k = 0 before step 0)
//     u_k[d, l]   = silu(pre_k[d, l])
// x_k is x (k = 0) or its transpose (k = 1) read forwards, or backwards (k = 2, 3).
// The backward (causal_conv1d_bwd with SiLU) takes du = d loss / d u along the paths:
//     dpre = du * silu'(pre),  silu'(p) = s (1 + p (1 - s)),  s = sigmoid(p)
//     dx_k[d, m] = sum_j w[k, d, j] dpre[m + (W-1) - j]
//     dw[k, d, j] = sum over batch and steps of dpre[l] x_k[l - (W-1) + j],  dbias = sum of dpre
// A CTA takes 256 steps of one (b, k, d) row, one per thread; the backward keeps the tile's dpre
// and the W-1 steps after it in shared memory, reduces its weight and bias terms in a fixed
// tree order, and a second kernel adds the per-(batch item, tile) partials in a fixed order.
// The work is a few multiply-adds per element: bound by HBM.
#include "common.cuh"
#include "kernels.h"

namespace ss2d {

constexpr int kConvTok = 256;  // steps per CTA, one per thread
constexpr int kConvWMax = 4;

// step m of path k in a row of x (or xT): 0 before the first step
template <typename Tin>
__device__ __forceinline__ float path_x(const Tin *row, bool rev, int64_t L, int64_t m) {
    return m < 0 ? 0.f : ld(row + (rev ? L - 1 - m : m));
}

template <typename Tin, int W>
__global__ void __launch_bounds__(kConvTok) path_conv_fwd_kernel(const Tin *__restrict__ x, const Tin *__restrict__ xT,
                                                                 const float *__restrict__ w,
                                                                 const float *__restrict__ bias, Tin *__restrict__ u,
                                                                 int64_t D, int64_t L, int64_t nlt) {
    const int64_t bid = blockIdx.x, row = bid / nlt;  // row = (b * 4 + k) * D + d
    const int64_t l = (bid % nlt) * kConvTok + threadIdx.x;
    if (l >= L) return;
    const int64_t d = row % D, bk = row / D, k = bk % kPaths, b = bk / kPaths;
    const Tin *xr = ((k & 1) ? xT : x) + (b * D + d) * L;
    const bool rev = k >= 2;
    const float *wk = w + (k * D + d) * W;
    float pre = bias ? bias[k * D + d] : 0.f;
#pragma unroll
    for (int j = 0; j < W; ++j) pre = fmaf(wk[j], path_x(xr, rev, L, l - (W - 1) + j), pre);
    st(u + row * L + l, silu_f(pre));
}

template <typename Tin, int W>
__global__ void __launch_bounds__(kConvTok) path_conv_bwd_kernel(const Tin *__restrict__ x, const Tin *__restrict__ xT,
                                                                 const float *__restrict__ w,
                                                                 const float *__restrict__ bias,
                                                                 const float *__restrict__ du, float *__restrict__ dxs,
                                                                 float *__restrict__ part, int64_t D, int64_t L,
                                                                 int64_t nlt) {
    __shared__ float dp[kConvTok + kConvWMax];      // dpre of the tile's steps and of the W-1 after it
    __shared__ float red[kConvTok / 32][W + 1];     // per-warp sums of the weight and bias terms
    const int t = threadIdx.x;
    const int64_t bid = blockIdx.x, row = bid / nlt, tile = bid % nlt;
    const int64_t l0 = tile * kConvTok, l = l0 + t;
    const int64_t d = row % D, bk = row / D, k = bk % kPaths, b = bk / kPaths;
    const Tin *xr = ((k & 1) ? xT : x) + (b * D + d) * L;
    const bool rev = k >= 2;
    const float *wk = w + (k * D + d) * W;
    const float b0 = bias ? bias[k * D + d] : 0.f;
    const float *dur = du + row * L;
    auto dpre_of = [&](const float (&xin)[W], int64_t m) {
        float pre = b0;
#pragma unroll
        for (int j = 0; j < W; ++j) pre = fmaf(wk[j], xin[j], pre);
        const float sg = sigmoid_f(pre);
        return dur[m] * sg * fmaf(pre, 1.f - sg, 1.f);
    };
    float xin[W];
#pragma unroll
    for (int j = 0; j < W; ++j) xin[j] = l < L ? path_x(xr, rev, L, l - (W - 1) + j) : 0.f;
    const float dpl = l < L ? dpre_of(xin, l) : 0.f;
    dp[t] = dpl;
    if (t < W - 1) {
        const int64_t m = l0 + kConvTok + t;
        float xh[W];
#pragma unroll
        for (int j = 0; j < W; ++j) xh[j] = m < L ? path_x(xr, rev, L, m - (W - 1) + j) : 0.f;
        dp[kConvTok + t] = m < L ? dpre_of(xh, m) : 0.f;
    }
    __syncthreads();
    if (l < L) {
        float acc = 0.f;
#pragma unroll
        for (int j = 0; j < W; ++j) acc = fmaf(wk[j], dp[t + (W - 1) - j], acc);
        dxs[row * L + l] = acc;
    }
    // weight and bias terms of this tile: a fixed shuffle tree per warp, then the warps in order
    float v[W + 1];
#pragma unroll
    for (int j = 0; j < W; ++j) v[j] = dpl * xin[j];
    v[W] = dpl;
#pragma unroll
    for (int j = 0; j <= W; ++j)
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v[j] += __shfl_xor_sync(0xffffffffu, v[j], o);
    if (t % 32 == 0)
#pragma unroll
        for (int j = 0; j <= W; ++j) red[t / 32][j] = v[j];
    __syncthreads();
    if (t <= W) {
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < kConvTok / 32; ++i) s += red[i][t];
        part[(row * nlt + tile) * (W + 1) + t] = s;
    }
}

// dw[k, d, j] (j < W) and dbias[k, d] (j = W) = sum over b, then tiles, of the partials
__global__ void path_conv_reduce_kernel(const float *__restrict__ part, float *__restrict__ dw,
                                        float *__restrict__ dbias, int64_t B, int64_t D, int64_t nlt, int W) {
    const int64_t total = kPaths * D * (W + 1);
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t kd = e / (W + 1);
        const int j = (int)(e % (W + 1));
        const int64_t k = kd / D, d = kd % D;
        float s = 0.f;
        for (int64_t b = 0; b < B; ++b) {
            const float *src = part + (((b * kPaths + k) * D + d) * nlt) * (W + 1) + j;
            for (int64_t tl = 0; tl < nlt; ++tl) s += src[tl * (W + 1)];
        }
        if (j < W)
            dw[kd * W + j] = s;
        else if (dbias)
            dbias[kd] = s;
    }
}

// ------------------------------------------------------------------ launchers --

size_t path_conv_partial_floats(const LaunchShape &s, int W) {
    return (size_t)s.B * kPaths * s.D * ceil_div(s.L, kConvTok) * (W + 1);
}

template <typename Tin, int W>
static cudaError_t conv_fwd_t(const LaunchShape &s, const void *x, const void *xT, const float *w, const float *bias,
                              void *u, cudaStream_t stream) {
    const int64_t nlt = ceil_div(s.L, kConvTok), blocks = s.B * kPaths * s.D * nlt;
    if (blocks > INT32_MAX) return cudaErrorInvalidConfiguration;
    path_conv_fwd_kernel<Tin, W><<<(unsigned)blocks, kConvTok, 0, stream>>>(
        static_cast<const Tin *>(x), static_cast<const Tin *>(xT), w, bias, static_cast<Tin *>(u), s.D, s.L, nlt);
    return cudaSuccess;
}

template <typename Tin>
static cudaError_t conv_fwd_w(const LaunchShape &s, int W, const void *x, const void *xT, const float *w,
                              const float *bias, void *u, cudaStream_t stream) {
    switch (W) {
        case 1: return conv_fwd_t<Tin, 1>(s, x, xT, w, bias, u, stream);
        case 2: return conv_fwd_t<Tin, 2>(s, x, xT, w, bias, u, stream);
        case 3: return conv_fwd_t<Tin, 3>(s, x, xT, w, bias, u, stream);
        case 4: return conv_fwd_t<Tin, 4>(s, x, xT, w, bias, u, stream);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_path_conv_fwd(const LaunchShape &s, ss2d_dtype_t dt, const void *x, const void *xT,
                                 const float *w, const float *bias, int W, void *u, cudaStream_t stream) {
    const cudaError_t e = dt == SS2D_F32 ? conv_fwd_w<float>(s, W, x, xT, w, bias, u, stream)
                                         : conv_fwd_w<__nv_bfloat16>(s, W, x, xT, w, bias, u, stream);
    if (e != cudaSuccess) return e;
    note_launch(stream);
    return cudaGetLastError();
}

template <typename Tin, int W>
static cudaError_t conv_bwd_t(const LaunchShape &s, const void *x, const void *xT, const float *w, const float *bias,
                              const float *du, float *dxs, float *part, cudaStream_t stream) {
    const int64_t nlt = ceil_div(s.L, kConvTok), blocks = s.B * kPaths * s.D * nlt;
    if (blocks > INT32_MAX) return cudaErrorInvalidConfiguration;
    path_conv_bwd_kernel<Tin, W><<<(unsigned)blocks, kConvTok, 0, stream>>>(
        static_cast<const Tin *>(x), static_cast<const Tin *>(xT), w, bias, du, dxs, part, s.D, s.L, nlt);
    return cudaSuccess;
}

template <typename Tin>
static cudaError_t conv_bwd_w(const LaunchShape &s, int W, const void *x, const void *xT, const float *w,
                              const float *bias, const float *du, float *dxs, float *part, cudaStream_t stream) {
    switch (W) {
        case 1: return conv_bwd_t<Tin, 1>(s, x, xT, w, bias, du, dxs, part, stream);
        case 2: return conv_bwd_t<Tin, 2>(s, x, xT, w, bias, du, dxs, part, stream);
        case 3: return conv_bwd_t<Tin, 3>(s, x, xT, w, bias, du, dxs, part, stream);
        case 4: return conv_bwd_t<Tin, 4>(s, x, xT, w, bias, du, dxs, part, stream);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_path_conv_bwd(const LaunchShape &s, ss2d_dtype_t dt, const void *x, const void *xT,
                                 const float *w, const float *bias, int W, const float *du, float *dxs, float *dw,
                                 float *dbias, float *part, cudaStream_t stream) {
    cudaError_t e = dt == SS2D_F32 ? conv_bwd_w<float>(s, W, x, xT, w, bias, du, dxs, part, stream)
                                   : conv_bwd_w<__nv_bfloat16>(s, W, x, xT, w, bias, du, dxs, part, stream);
    if (e != cudaSuccess) return e;
    note_launch(stream);
    const int64_t total = kPaths * s.D * (W + 1);
    const int64_t want = ceil_div(total, 256);
    path_conv_reduce_kernel<<<(unsigned)(want < 148 * 8 ? want : 148 * 8), 256, 0, stream>>>(
        part, dw, dbias, s.B, s.D, ceil_div(s.L, kConvTok), W);
    note_launch(stream);
    return cudaGetLastError();
}

}  // namespace ss2d
