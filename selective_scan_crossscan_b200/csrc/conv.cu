// conv.cu -- the causal depthwise conv with SiLU in front of the producer, along every path.
//
// MambaInnerFn.forward ("vision mamba-yolov8", section 2) passes its input through
// causal_conv1d_fwd(x, weight, bias, True) before x_proj: a depthwise conv of width W over the
// sequence, reading the current and the W-1 previous steps, then SiLU.  The SS2D of "Visual
// Mamba实战从零开始搭建图像分类模型附PyTorch代码" (section 3) runs one Mamba block per scan direction,
// so here every path k has its own weights and convolves x read along its own step order:
//     pre_k[d, l] = bias[k, d] + sum_j w[k, d, j] x_k[d, l - (W-1) + j]     (x_k = 0 before step 0)
//     u_k[d, l]   = silu(pre_k[d, l])
// x_k is x (k = 0) or its transpose (k = 1) read forwards, or backwards (k = 2, 3).
// The backward (causal_conv1d_bwd with SiLU) takes du = d loss / d u along the paths:
//     dpre = du * silu'(pre),  silu'(p) = s (1 + p (1 - s)),  s = sigmoid(p)
//     dx_k[d, m] = sum_j w[k, d, j] dpre[m + (W-1) - j]
//     dw[k, d, j] = sum over batch and steps of dpre[l] x_k[l - (W-1) + j],  dbias = sum of dpre
// A CTA takes 1024 steps of one (b, k, d) row, four consecutive ones per thread (the row is
// decoded once per thread in 32-bit arithmetic); the backward keeps the tile's dpre and the
// W-1 steps after it in shared memory, reduces its weight and bias terms in a fixed tree
// order, and a second kernel adds the per-(batch item, tile) partials in a fixed order.
// The work is a few multiply-adds per element: bound by HBM.
#include "common.cuh"
#include "kernels.h"

namespace ss2d {

constexpr int kConvThreads = 256;
constexpr int kConvPer = 4;                            // consecutive steps per thread
constexpr int kConvTok = kConvThreads * kConvPer;      // steps per CTA
constexpr int kConvWMax = 4;

// step m of path k in a row of x (or xT): 0 before the first step
template <typename Tin>
__device__ __forceinline__ float path_x(const Tin *row, bool rev, int64_t L, int64_t m) {
    return m < 0 ? 0.f : ld(row + (rev ? L - 1 - m : m));
}

// four consecutive elements as floats / from floats (16 bytes fp32, 8 bytes bf16; aligned)
__device__ __forceinline__ float4 ld4v(const float *p) { return *reinterpret_cast<const float4 *>(p); }
__device__ __forceinline__ float4 ld4v(const __nv_bfloat16 *p) {
    const uint2 v = *reinterpret_cast<const uint2 *>(p);
    return make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xffff0000u), __uint_as_float(v.y << 16),
                       __uint_as_float(v.y & 0xffff0000u));
}
__device__ __forceinline__ void st4v(float *p, float4 v) { *reinterpret_cast<float4 *>(p) = v; }
__device__ __forceinline__ void st4v(__nv_bfloat16 *p, float4 v) {
    const __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
    *reinterpret_cast<uint2 *>(p) = make_uint2(*reinterpret_cast<const uint32_t *>(&lo),
                                               *reinterpret_cast<const uint32_t *>(&hi));
}

// The CTA's row (b, k, d) and tile, decoded once in 32-bit arithmetic (the launcher checks the
// row count fits), and the row's x (or xT) base, direction, weights and bias.
template <typename Tin, int W>
struct ConvRow {
    int64_t row, l0;
    const Tin *xr;
    bool rev;
    float w[W], b0;
    __device__ __forceinline__ ConvRow(const Tin *x, const Tin *xT, const float *wt, const float *bias, uint32_t D,
                                       uint32_t nlt, int64_t L) {
        const uint32_t bid = blockIdx.x, r = bid / nlt, d = r % D, bk = r / D, k = bk % kPaths, b = bk / kPaths;
        row = r;
        l0 = (int64_t)(bid - r * nlt) * kConvTok;
        xr = ((k & 1) ? xT : x) + ((int64_t)b * D + d) * L;
        rev = k >= 2;
#pragma unroll
        for (int j = 0; j < W; ++j) w[j] = wt[((int64_t)k * D + d) * W + j];
        b0 = bias ? bias[(int64_t)k * D + d] : 0.f;
    }
    // x_k at steps l - (W-1) .. l + kConvPer - 1: the windows of kConvPer consecutive outputs.
    // VEC (L % 4 == 0, l % 4 == 0): two aligned quads of the row, steps l-4..l-1 and l..l+3, read
    // backwards on the reversed paths (row positions L-l..L+3-l and L-4-l..L-1-l).
    template <bool VEC>
    __device__ __forceinline__ void window(int64_t l, int64_t L, float (&xv)[kConvPer + W - 1]) const {
        if (VEC) {
            static_assert(kConvPer == 4, "quads");
            float cat[8];  // x_k[l - 4 + j]
            const float4 hi = ld4v(xr + (rev ? L - 4 - l : l));
            const float4 lo = l >= 4 ? ld4v(xr + (rev ? L - l : l - 4)) : make_float4(0.f, 0.f, 0.f, 0.f);
            if (rev) {
                cat[0] = lo.w; cat[1] = lo.z; cat[2] = lo.y; cat[3] = lo.x;
                cat[4] = hi.w; cat[5] = hi.z; cat[6] = hi.y; cat[7] = hi.x;
            } else {
                cat[0] = lo.x; cat[1] = lo.y; cat[2] = lo.z; cat[3] = lo.w;
                cat[4] = hi.x; cat[5] = hi.y; cat[6] = hi.z; cat[7] = hi.w;
            }
#pragma unroll
            for (int i = 0; i < kConvPer + W - 1; ++i) xv[i] = cat[4 - (W - 1) + i];
        } else {
#pragma unroll
            for (int i = 0; i < kConvPer + W - 1; ++i) {
                const int64_t m = l - (W - 1) + i;
                xv[i] = m < L ? path_x(xr, rev, L, m) : 0.f;
            }
        }
    }
    __device__ __forceinline__ float pre(const float (&xv)[kConvPer + W - 1], int q) const {
        float p = b0;
#pragma unroll
        for (int j = 0; j < W; ++j) p = fmaf(w[j], xv[q + j], p);
        return p;
    }
};

template <typename Tin, int W, bool VEC>
__global__ void __launch_bounds__(kConvThreads) path_conv_fwd_kernel(const Tin *__restrict__ x, const Tin *__restrict__ xT,
                                                                     const float *__restrict__ w,
                                                                     const float *__restrict__ bias,
                                                                     Tin *__restrict__ u, uint32_t D, int64_t L,
                                                                     uint32_t nlt) {
    const ConvRow<Tin, W> cr(x, xT, w, bias, D, nlt, L);
    const int64_t l = cr.l0 + kConvPer * threadIdx.x;
    if (l >= L) return;
    float xv[kConvPer + W - 1];
    cr.template window<VEC>(l, L, xv);
    Tin *o = u + cr.row * L + l;
    if (VEC) {
        st4v(o, make_float4(silu_f(cr.pre(xv, 0)), silu_f(cr.pre(xv, 1)), silu_f(cr.pre(xv, 2)),
                            silu_f(cr.pre(xv, 3))));
        return;
    }
#pragma unroll
    for (int q = 0; q < kConvPer; ++q)
        if (l + q < L) st(o + q, silu_f(cr.pre(xv, q)));
}

template <typename Tin, int W, bool VEC>
__global__ void __launch_bounds__(kConvThreads) path_conv_bwd_kernel(const Tin *__restrict__ x, const Tin *__restrict__ xT,
                                                                     const float *__restrict__ w,
                                                                     const float *__restrict__ bias,
                                                                     const float *__restrict__ du,
                                                                     float *__restrict__ dxs, float *__restrict__ part,
                                                                     uint32_t D, int64_t L, uint32_t nlt) {
    __shared__ float dp[kConvTok + kConvWMax];          // dpre of the tile's steps and of the W-1 after it
    __shared__ float red[kConvThreads / 32][W + 1];     // per-warp sums of the weight and bias terms
    const int t = threadIdx.x;
    const ConvRow<Tin, W> cr(x, xT, w, bias, D, nlt, L);
    const int64_t l = cr.l0 + kConvPer * t;
    const float *dur = du + cr.row * L;
    auto dpre_of = [&](float p, int64_t m) {
        const float sg = sigmoid_f(p);
        return dur[m] * sg * fmaf(p, 1.f - sg, 1.f);
    };
    float xv[kConvPer + W - 1];
    float dpl[kConvPer];
    if (VEC) {
        if (l < L) {
            cr.template window<true>(l, L, xv);
            const float4 g4 = ld4v(dur + l);
            const float gv[4] = {g4.x, g4.y, g4.z, g4.w};
#pragma unroll
            for (int q = 0; q < kConvPer; ++q) {
                const float p = cr.pre(xv, q), sg = sigmoid_f(p);
                dpl[q] = gv[q] * sg * fmaf(p, 1.f - sg, 1.f);
            }
        } else {
#pragma unroll
            for (int i = 0; i < kConvPer + W - 1; ++i) xv[i] = 0.f;
#pragma unroll
            for (int q = 0; q < kConvPer; ++q) dpl[q] = 0.f;
        }
    } else {
        cr.template window<false>(l, L, xv);
#pragma unroll
        for (int q = 0; q < kConvPer; ++q) dpl[q] = l + q < L ? dpre_of(cr.pre(xv, q), l + q) : 0.f;
    }
#pragma unroll
    for (int q = 0; q < kConvPer; ++q) dp[kConvPer * t + q] = dpl[q];
    if (t < W - 1) {  // the halo: dpre of the W-1 steps after the tile
        const int64_t m = cr.l0 + kConvTok + t;
        float p = cr.b0;
#pragma unroll
        for (int j = 0; j < W; ++j) p = fmaf(cr.w[j], m < L ? path_x(cr.xr, cr.rev, L, m - (W - 1) + j) : 0.f, p);
        dp[kConvTok + t] = m < L ? dpre_of(p, m) : 0.f;
    }
    __syncthreads();
    if (VEC && l < L) {
        float a[kConvPer];
#pragma unroll
        for (int q = 0; q < kConvPer; ++q) {
            a[q] = 0.f;
#pragma unroll
            for (int j = 0; j < W; ++j) a[q] = fmaf(cr.w[j], dp[kConvPer * t + q + (W - 1) - j], a[q]);
        }
        st4v(dxs + cr.row * L + l, make_float4(a[0], a[1], a[2], a[3]));
    } else if (!VEC) {
#pragma unroll
        for (int q = 0; q < kConvPer; ++q) {
            if (l + q >= L) break;
            float acc = 0.f;
#pragma unroll
            for (int j = 0; j < W; ++j) acc = fmaf(cr.w[j], dp[kConvPer * t + q + (W - 1) - j], acc);
            dxs[cr.row * L + l + q] = acc;
        }
    }
    // weight and bias terms: this thread's steps in order, a fixed shuffle tree per warp, then the
    // warps in order
    float v[W + 1];
#pragma unroll
    for (int j = 0; j <= W; ++j) v[j] = 0.f;
#pragma unroll
    for (int q = 0; q < kConvPer; ++q) {
#pragma unroll
        for (int j = 0; j < W; ++j) v[j] = fmaf(dpl[q], xv[q + j], v[j]);
        v[W] += dpl[q];
    }
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
        for (int i = 0; i < kConvThreads / 32; ++i) s += red[i][t];
        part[(int64_t)blockIdx.x * (W + 1) + t] = s;
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
    if (blocks > INT32_MAX) return cudaErrorInvalidConfiguration;  // also keeps the 32-bit row decode exact
    // quads of 4 steps are aligned (16 bytes fp32, 8 bytes bf16) when L % 4 == 0
    auto kern = s.L % 4 == 0 ? path_conv_fwd_kernel<Tin, W, true> : path_conv_fwd_kernel<Tin, W, false>;
    kern<<<(unsigned)blocks, kConvThreads, 0, stream>>>(static_cast<const Tin *>(x), static_cast<const Tin *>(xT), w,
                                                        bias, static_cast<Tin *>(u), (uint32_t)s.D, s.L,
                                                        (uint32_t)nlt);
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
    if (blocks > INT32_MAX) return cudaErrorInvalidConfiguration;  // also keeps the 32-bit row decode exact
    auto kern = s.L % 4 == 0 ? path_conv_bwd_kernel<Tin, W, true> : path_conv_bwd_kernel<Tin, W, false>;
    kern<<<(unsigned)blocks, kConvThreads, 0, stream>>>(static_cast<const Tin *>(x), static_cast<const Tin *>(xT), w,
                                                        bias, du, dxs, part, (uint32_t)s.D, s.L, (uint32_t)nlt);
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
