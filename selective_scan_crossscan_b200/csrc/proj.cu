// proj.cu -- the producer of the scan's inputs: the per-path x_proj contraction.
//
// MambaInnerFn.forward ("vision mamba-yolov8", section 2) makes the scan's inputs
// from its input sequence: x_dbl = x_proj(u), R + 2N outputs per token, whose first
// R rows go through dt_proj to become delta and whose next N and last N rows are B
// and C.  SS2D gives every path k its own x_proj, applied to u_k = x read along path
// k.  This kernel computes
//     x_dbl[b, k, c, l] = sum_d W[k, c, d] * u_k[d, l]
// and stores it in each path's own step order.  dt_proj and the softplus are not done
// here: the scan applies them per step, so delta (B, 4D, L) is never written.
//
// Paths k and k + 2 walk the same base order backwards (the cross scan's structure):
// base 0 is x itself, base 1 its transpose.  A CTA takes a tile of consecutive tokens of
// one base order of one batch item and computes both paths' R + 2N rows for them,
// streaming D through shared memory 16 channels at a time, double-buffered.  Half of the threads work for
// path k, half for path k + 2; each owns TOK tokens and keeps their R + 2N accumulators in
// registers as output pairs, so one packed FFMA2 (x, x) * (w_c, w_c+1) updates two outputs
// and a 128-bit broadcast shared load feeds two of them.  Path k + 2's outputs go to step
// L-1-l, so its stores run backwards through memory but stay contiguous across the warp.
//
// The contraction is skinny (R + 2N = 38 outputs per token for VMamba-T): about 10
// multiply-adds per byte of u, so it runs on the fp32 FMA pipe in fp32 (exact products for
// the 1e-4 fp32 parity), bound by the FMA rate rather than by HBM.
#include "common.cuh"
#include "kernels.h"

namespace ss2d {

#ifndef SS2D_PROJ_MIN_BLOCKS
#define SS2D_PROJ_MIN_BLOCKS 2  // resident CTAs per SM the producer's registers are held to
#endif

constexpr int kProjKc = 16;        // channels per shared-memory chunk
constexpr int kProjThreads = 256;  // 128 per path of the pair

__device__ __forceinline__ void cp_async4(float *dst, const float *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"((unsigned)__cvta_generic_to_shared(dst)), "l"(src));
}
__device__ __forceinline__ void cp_async16(float *dst, const float *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"((unsigned)__cvta_generic_to_shared(dst)),
                 "l"(src));
}

// RNB: R + 2N rounded up to the accumulators kept (a multiple of 4); TOK: tokens per thread.
// The token chunk is double-buffered in shared memory: fp32 inputs are copied with cp.async
// (16-byte pieces when every row of the tile is 16-byte aligned, ALIGNED) while the previous
// chunk is consumed; bf16 inputs are converted through registers.  The next weight chunk is
// loaded into registers during the current chunk and stored after it.
template <typename Tin, int RNB, int TOK, bool ALIGNED>
__global__ void __launch_bounds__(kProjThreads, SS2D_PROJ_MIN_BLOCKS) xproj_kernel(const Tin *__restrict__ x, const Tin *__restrict__ xT,
                                                             const float *__restrict__ W, Tin *__restrict__ xdbl,
                                                             int64_t D, int64_t L, int RN) {
    constexpr int kTile = (kProjThreads / 2) * TOK;  // tokens per CTA
    constexpr int kWPer = (2 * RNB * kProjKc + kProjThreads - 1) / kProjThreads;  // weights staged per thread
    constexpr bool kAsync = sizeof(Tin) == 4;
    __shared__ __align__(16) float Xs[2][kProjKc][kTile + 4];
    __shared__ __align__(16) float Ws[2][2][kProjKc][RNB];
    const int t = threadIdx.x, half = t / (kProjThreads / 2), tp = t % (kProjThreads / 2);
    const int j = blockIdx.y;  // base order: 0 = x (paths 0, 2), 1 = xT (paths 1, 3)
    const int64_t b = blockIdx.z, l0 = (int64_t)blockIdx.x * kTile;
    const Tin *X = (j ? xT : x) + b * D * L;
    const int64_t nchunk = (D + kProjKc - 1) / kProjKc;

    // chunk copies: X rows d0 .. d0+15 of the tile, and the two paths' weights for them
    auto stage_x = [&](int buf, int64_t d0) {
        if (kAsync && ALIGNED) {
            for (int e = t; e < kProjKc * (kTile / 4); e += kProjThreads) {
                const int kk = e / (kTile / 4), l4 = (e % (kTile / 4)) * 4;
                const int64_t d = d0 + kk, l = l0 + l4;
                if (d < D && l + 3 < L)
                    cp_async16(&Xs[buf][kk][l4], reinterpret_cast<const float *>(X) + d * L + l);
                else
                    for (int q = 0; q < 4; ++q)
                        Xs[buf][kk][l4 + q] = (d < D && l + q < L) ? ld(X + d * L + l + q) : 0.f;
            }
        } else {
            for (int e = t; e < kProjKc * kTile; e += kProjThreads) {
                const int kk = e / kTile, ll = e % kTile;
                const int64_t d = d0 + kk, l = l0 + ll;
                if (kAsync && d < D && l < L)
                    cp_async4(&Xs[buf][kk][ll], reinterpret_cast<const float *>(X) + d * L + l);
                else
                    Xs[buf][kk][ll] = (d < D && l < L) ? ld(X + d * L + l) : 0.f;
            }
        }
        asm volatile("cp.async.commit_group;\n" ::);
    };
    auto load_w = [&](float (&wr)[kWPer], int64_t d0) {
#pragma unroll
        for (int i = 0; i < kWPer; ++i) {
            const int e = t + i * kProjThreads;
            const int h = e / (RNB * kProjKc), rem = e % (RNB * kProjKc);
            const int c = rem / kProjKc, kk = rem % kProjKc;
            const int64_t d = d0 + kk;
            wr[i] = (e < 2 * RNB * kProjKc && c < RN && d < D) ? W[((int64_t)(j + 2 * h) * RN + c) * D + d] : 0.f;
        }
    };
    auto store_w = [&](const float (&wr)[kWPer], int buf) {
#pragma unroll
        for (int i = 0; i < kWPer; ++i) {
            const int e = t + i * kProjThreads;
            if (e < 2 * RNB * kProjKc) {
                const int h = e / (RNB * kProjKc), rem = e % (RNB * kProjKc);
                Ws[buf][h][rem % kProjKc][rem / kProjKc] = wr[i];
            }
        }
    };

    float2 acc[TOK][RNB / 2];
#pragma unroll
    for (int q = 0; q < TOK; ++q)
#pragma unroll
        for (int c = 0; c < RNB / 2; ++c) acc[q][c] = make_float2(0.f, 0.f);

    float wr[kWPer];
    stage_x(0, 0);
    load_w(wr, 0);
    store_w(wr, 0);
    for (int64_t ch = 0; ch < nchunk; ++ch) {
        const int buf = (int)(ch & 1);
        const bool more = ch + 1 < nchunk;
        if (more) {
            stage_x(buf ^ 1, (ch + 1) * kProjKc);  // the previous readers of buf^1 passed the last barrier
            load_w(wr, (ch + 1) * kProjKc);
            asm volatile("cp.async.wait_group 1;\n" ::);
        } else {
            asm volatile("cp.async.wait_group 0;\n" ::);
        }
        __syncthreads();  // chunk ch (copies and weights) is in shared memory for every thread
#pragma unroll 2
        for (int kk = 0; kk < kProjKc; ++kk) {
            float2 xv[TOK];
            if (TOK == 2) {
                const float2 v = *reinterpret_cast<const float2 *>(&Xs[buf][kk][2 * tp]);
                xv[0] = make_float2(v.x, v.x);
                xv[TOK - 1] = make_float2(v.y, v.y);
            } else {
                const float v = Xs[buf][kk][tp];
                xv[0] = make_float2(v, v);
            }
#pragma unroll
            for (int c = 0; c < RNB; c += 4) {
                const float4 w = *reinterpret_cast<const float4 *>(&Ws[buf][half][kk][c]);
                const float2 w01 = make_float2(w.x, w.y), w23 = make_float2(w.z, w.w);
#pragma unroll
                for (int q = 0; q < TOK; ++q) {
                    acc[q][c / 2] = __ffma2_rn(xv[q], w01, acc[q][c / 2]);
                    acc[q][c / 2 + 1] = __ffma2_rn(xv[q], w23, acc[q][c / 2 + 1]);
                }
            }
        }
        if (more) store_w(wr, buf ^ 1);  // buf^1's weights were last read before the barrier above
        __syncthreads();                 // chunk ch is consumed before its buffers are refilled
    }
    const int k = j + 2 * half;
    Tin *o = xdbl + ((b * kPaths + k) * RN) * L;
#pragma unroll
    for (int q = 0; q < TOK; ++q) {
        const int64_t l = l0 + TOK * tp + q;
        if (l < L) {
            const int64_t pos = half ? L - 1 - l : l;
#pragma unroll
            for (int c = 0; c < RNB / 2; ++c) {
                if (2 * c < RN) st(o + (int64_t)(2 * c) * L + pos, acc[q][c].x);
                if (2 * c + 1 < RN) st(o + (int64_t)(2 * c + 1) * L + pos, acc[q][c].y);
            }
        }
    }
}

template <typename Tin, int RNB, int TOK>
static void launch_xproj_t(const LaunchShape &s, const void *x, const void *xT, const float *W, int RN, void *xdbl,
                           cudaStream_t stream) {
    constexpr int kTile = (kProjThreads / 2) * TOK;
    dim3 grid((unsigned)ceil_div(s.L, kTile), 2, (unsigned)s.B);
    // 16-byte copies need every row start aligned: L % 4 == 0 and 16-byte aligned bases
    const bool aligned = s.L % 4 == 0 &&
                         ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(xT)) & 15) == 0;
    if (aligned)
        xproj_kernel<Tin, RNB, TOK, true><<<grid, kProjThreads, 0, stream>>>(
            static_cast<const Tin *>(x), static_cast<const Tin *>(xT), W, static_cast<Tin *>(xdbl), s.D, s.L, RN);
    else
        xproj_kernel<Tin, RNB, TOK, false><<<grid, kProjThreads, 0, stream>>>(
            static_cast<const Tin *>(x), static_cast<const Tin *>(xT), W, static_cast<Tin *>(xdbl), s.D, s.L, RN);
}

cudaError_t launch_xproj(const LaunchShape &s, ss2d_dtype_t dt, const void *x, const void *xT, const float *W,
                         int RN, void *xdbl, cudaStream_t stream) {
    // RN = R + 2N: up to 40 (dt rank <= 8) with two tokens per thread, else up to 64 with one;
    // weight rows past RN are staged as zeros and their accumulators never stored
    using bf = __nv_bfloat16;
    if (RN <= 40) {
        if (dt == SS2D_F32)
            launch_xproj_t<float, 40, 2>(s, x, xT, W, RN, xdbl, stream);
        else
            launch_xproj_t<bf, 40, 2>(s, x, xT, W, RN, xdbl, stream);
    } else {
        if (dt == SS2D_F32)
            launch_xproj_t<float, 64, 1>(s, x, xT, W, RN, xdbl, stream);
        else
            launch_xproj_t<bf, 64, 1>(s, x, xT, W, RN, xdbl, stream);
    }
    note_launch(stream);
    return cudaGetLastError();
}

}  // namespace ss2d
