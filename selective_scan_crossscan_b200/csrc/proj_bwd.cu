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
// The two contractions with R on one side are narrow (R <= 32) and bound by reading ddelta
// once: rows_kernel gives each thread one token and its R sums; dwdt_kernel gives each
// thread one channel's R sums over a quarter of a staged token tile.  xseq_kernel (x_proj of the
// per-path sequences the conv makes) streams the channels through a cp.async ring into an all-rows
// x 128-token tile.  chan_kernel stages both
// operands of a 64-channel x 128-token tile whole (the contraction is R + 2N <= 64 long); it
// also makes delta from x_dbl[:R] (dt_proj) for the backward and for wide ranks.
// tr_gemm_kernel (d x_proj.weight) holds all R + 2N (<= 64) rows of a 128-column tile per CTA
// and streams tokens through a 3-stage cp.async ring, 4 tokens per step.  The sums over tokens
// are written per (batch item, token chunk) as partials that reduce_partials_kernel adds in
// a fixed order, so every gradient is deterministic.  All arithmetic is fp32 on the FMA pipe.
#include "common.cuh"
#include "kernels.h"

namespace ss2d {

constexpr int kTS = 32;     // tokens per pipeline stage
constexpr int kStages = 3;  // cp.async ring depth

__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"((unsigned)__cvta_generic_to_shared(dst)),
                 "l"(src));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

// copy / zero four consecutive elements (16 bytes fp32, 8 bytes bf16)
__device__ __forceinline__ void cp_async_quad(float *dst, const float *src) { cp_async16(dst, src); }
__device__ __forceinline__ void cp_async_quad(__nv_bfloat16 *dst, const __nv_bfloat16 *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;\n" ::"r"((unsigned)__cvta_generic_to_shared(dst)),
                 "l"(src));
}
__device__ __forceinline__ void zero_quad(float *dst) {
    *reinterpret_cast<float4 *>(dst) = make_float4(0.f, 0.f, 0.f, 0.f);
}
__device__ __forceinline__ void zero_quad(__nv_bfloat16 *dst) { *reinterpret_cast<uint2 *>(dst) = make_uint2(0u, 0u); }

// four consecutive outputs (16 bytes fp32, 8 bytes bf16, aligned)
__device__ __forceinline__ void store4(float *p, float4 v) { *reinterpret_cast<float4 *>(p) = v; }
__device__ __forceinline__ void store4(__nv_bfloat16 *p, float4 v) {
    const __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
    *reinterpret_cast<uint2 *>(p) = make_uint2(*reinterpret_cast<const uint32_t *>(&lo),
                                               *reinterpret_cast<const uint32_t *>(&hi));
}

// four consecutive elements of a shared-memory row as floats (fp32: one 16-byte load; bf16: 8 bytes)
__device__ __forceinline__ float4 ld4(const float *p) { return *reinterpret_cast<const float4 *>(p); }
__device__ __forceinline__ float4 ld4(const __nv_bfloat16 *p) {
    const uint2 v = *reinterpret_cast<const uint2 *>(p);
    return make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xffff0000u), __uint_as_float(v.y << 16),
                       __uint_as_float(v.y & 0xffff0000u));
}

// shared-memory row pitch in elements: 16-byte aligned, and 4 words apart (mod 32) so that eight
// consecutive rows read at one column fill distinct banks
template <typename T>
__host__ __device__ constexpr int row_pitch() { return sizeof(T) == 4 ? kTS + 4 : kTS + 8; }

// ------------------------------------------------------------ narrow: R sums --

constexpr int kNarrowTok = 256;  // tokens (one per thread) of a dtlow_kernel CTA
constexpr int kNarrowD = 64;     // channels per staged slice of dt_proj.weight

// out[g, r, l] = sum_d M(k, r, d) in[g, d, l] for r < R, g = b * 4 + k, M(k, r, d) =
// Wm[k*w_ks + r*w_rs + d*w_ds]; in has D rows per group, out out_gs elements per group.  A thread
// owns one token and its RB (R rounded up to 8) sums; M sits in shared memory 64 channels at a time.
// Used for dx_dbl[:R] = dt_proj.weight^T ddelta and for x_proj of per-path sequences.
template <typename Tin, typename Tout, int RB>
__global__ void __launch_bounds__(kNarrowTok) rows_kernel(const Tin *__restrict__ in, const float *__restrict__ Wm,
                                                          int64_t w_ks, int64_t w_rs, int64_t w_ds,
                                                          Tout *__restrict__ out, int64_t out_gs, int64_t D,
                                                          int64_t L, int R, int64_t nlt) {
    __shared__ __align__(16) float Ws[kNarrowD][RB];
    const int64_t bid = blockIdx.x, g = bid / nlt, k = g % kPaths;
    const int64_t l = (bid % nlt) * kNarrowTok + threadIdx.x;
    const bool live = l < L;
    const Tin *src = in + g * D * L + (live ? l : L - 1);  // dead threads re-read the last token
    float acc[RB];
#pragma unroll
    for (int r = 0; r < RB; ++r) acc[r] = 0.f;
    for (int64_t d0 = 0; d0 < D; d0 += kNarrowD) {
        const int n = (int)(D - d0 < kNarrowD ? D - d0 : kNarrowD);
        __syncthreads();
        for (int e = threadIdx.x; e < kNarrowD * RB; e += kNarrowTok) {
            const int i = e / RB, r = e % RB;
            Ws[i][r] = (i < n && r < R) ? Wm[k * w_ks + r * w_rs + (d0 + i) * w_ds] : 0.f;
        }
        __syncthreads();
        const Tin *sp = src + d0 * L;
#pragma unroll 8
        for (int i = 0; i < n; ++i) {
            const float v = ld(sp + i * L);
#pragma unroll
            for (int q = 0; q < RB / 4; ++q) {
                const float4 w = *reinterpret_cast<const float4 *>(&Ws[i][4 * q]);
                acc[4 * q + 0] = fmaf(w.x, v, acc[4 * q + 0]);
                acc[4 * q + 1] = fmaf(w.y, v, acc[4 * q + 1]);
                acc[4 * q + 2] = fmaf(w.z, v, acc[4 * q + 2]);
                acc[4 * q + 3] = fmaf(w.w, v, acc[4 * q + 3]);
            }
        }
    }
    if (!live) return;
#pragma unroll
    for (int r = 0; r < RB; ++r)
        if (r < R) st(out + g * out_gs + r * L + l, acc[r]);
}

constexpr int kDwD = 64;  // channels per dwdt_kernel CTA (4 threads each)

template <typename Tin, int RB>
constexpr size_t dwdt_smem_bytes() { return (size_t)kStages * (kDwD + RB) * row_pitch<Tin>() * sizeof(Tin); }

// part[(k*B + b)*nlc + lc][d][r] = sum over the chunk's tokens of ddelta[g, d, l] x_dbl[g, r, l].
// ddelta and x_dbl's dt rows stream through a 3-stage cp.async ring of 32-token tiles in their
// global [row][token] layout (plain loads when L % 4 != 0).  Thread (dl, q) sums channel dl over
// tokens 8q..8q+7 of each tile, one quad at a time: 1 + RB quad loads feed 4*RB FMAs.
template <typename Tin, int RB, bool VEC>
__global__ void __launch_bounds__(256, 2) dwdt_kernel(const Tin *__restrict__ ddelta, const Tin *__restrict__ xdbl,
                                                      float *__restrict__ part, int64_t B, int64_t D, int64_t L,
                                                      int R, int RN, int64_t lchunk, int nlc, int ndt) {
    constexpr int P = row_pitch<Tin>(), CS = kDwD * kTS / 4, CX = RB * kTS / 4;
    extern __shared__ __align__(16) unsigned char dw_smem[];
    Tin *S = reinterpret_cast<Tin *>(dw_smem);      // [kStages][kDwD][P]
    Tin *X = S + (size_t)kStages * kDwD * P;        // [kStages][RB][P]
    const int t = threadIdx.x, dl = t / 4, q = t % 4;
    // one flat grid: channel tiles fastest (they share the x_dbl tile), then (path, batch item, chunk)
    const int64_t bid = blockIdx.x, z = bid / ndt, k = z % kPaths, rest = z / kPaths, b = rest / nlc,
                  lc = rest % nlc;
    const int64_t d0 = (bid % ndt) * kDwD, g = b * kPaths + k;
    const int64_t lb = lc * lchunk, le = L < lb + lchunk ? L : lb + lchunk;
    const Tin *s_src = ddelta + g * D * L;
    const Tin *x_src = xdbl + g * RN * L;
    const int nst = (int)ceil_div(le - lb, kTS);
    auto issue = [&](int st_) {
        const int buf = st_ % kStages;
        const int64_t t0 = lb + (int64_t)st_ * kTS;
        const int nv = (int)(le - t0 < kTS ? le - t0 : kTS);
        Tin *ss = S + (size_t)buf * kDwD * P, *xs = X + (size_t)buf * RB * P;
        if (VEC) {
            for (int c = t; c < CS + CX; c += 256) {
                const bool sx = c < CS;
                const int cc = sx ? c : c - CS, r = cc / (kTS / 4), j = 4 * (cc % (kTS / 4));
                Tin *dst = (sx ? ss : xs) + r * P + j;
                const bool ok = j < nv && (sx ? d0 + r < D : r < R);
                if (ok) cp_async_quad(dst, (sx ? s_src + (d0 + r) * L : x_src + r * L) + t0 + j);
                else zero_quad(dst);
            }
        } else {
            for (int e = t; e < (kDwD + RB) * kTS; e += 256) {
                const int r = e / kTS, j = e % kTS;
                const bool sx = r < kDwD;
                const int rr = sx ? r : r - kDwD;
                const bool ok = j < nv && (sx ? d0 + rr < D : rr < R);
                const float v = ok ? ld((sx ? s_src + (d0 + rr) * L : x_src + rr * L) + t0 + j) : 0.f;
                st((sx ? ss : xs) + rr * P + j, v);
            }
        }
    };
    float acc[RB];
#pragma unroll
    for (int r = 0; r < RB; ++r) acc[r] = 0.f;
#pragma unroll
    for (int st_ = 0; st_ < kStages - 1; ++st_) {
        if (st_ < nst) issue(st_);
        cp_async_commit();
    }
    for (int st_ = 0; st_ < nst; ++st_) {
        cp_async_wait<kStages - 2>();
        __syncthreads();  // tile st_ visible to all; every thread is done with tile st_ - 1's buffer
        if (st_ + kStages - 1 < nst) issue(st_ + kStages - 1);
        cp_async_commit();
        const Tin *ss = S + (size_t)(st_ % kStages) * kDwD * P + dl * P, *xs = X + (size_t)(st_ % kStages) * RB * P;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int tq = 8 * q + 4 * h;
            const float4 sv = ld4(ss + tq);
#pragma unroll
            for (int r = 0; r < RB; ++r) {
                const float4 xv = ld4(xs + r * P + tq);
                float a = acc[r];
                a = fmaf(sv.x, xv.x, a);
                a = fmaf(sv.y, xv.y, a);
                a = fmaf(sv.z, xv.z, a);
                acc[r] = fmaf(sv.w, xv.w, a);
            }
        }
    }
    // the 4 threads of a channel are adjacent lanes: fold them in a fixed order
#pragma unroll
    for (int r = 0; r < RB; ++r) {
        acc[r] += __shfl_xor_sync(0xffffffffu, acc[r], 1);
        acc[r] += __shfl_xor_sync(0xffffffffu, acc[r], 2);
    }
    const int64_t d = d0 + dl;
    if (q != 0 || d >= D) return;
    float *dst = part + ((k * B + b) * nlc + lc) * D * R + d * R;
#pragma unroll
    for (int r = 0; r < RB; ++r)
        if (r < R) dst[r] = acc[r];
}

// -------------------------------------------------- x_proj of per-path sequences --

constexpr int kXsL = 128;  // tokens per CTA (32 lanes x 4)
constexpr int kXsK = 16;   // channels per pipeline stage

template <typename Tin, int TY>
constexpr size_t xseq_smem_bytes() {
    return (size_t)kStages * (8 * TY * (kXsK + 4) * sizeof(float) +
                              kXsK * (sizeof(Tin) == 4 ? kXsL + 4 : kXsL + 8) * sizeof(Tin));
}

// xdbl[g, c, l] = sum_d W[k, c, d] u[g, d, l] for c < RN (g = b * 4 + k): all RN rows of a 128-token
// tile per CTA, the channels streamed 16 at a time through a 3-stage cp.async ring (plain loads
// when L or D is not a multiple of 4).  Warp ty holds rows ty + 8i (i < TY), lane tx tokens
// 4tx..4tx+3 as two packed pairs: one 16-byte token load and TY broadcast weight loads feed 2*TY
// FFMA2 per channel.
template <typename Tin, int TY, bool VEC>
__global__ void __launch_bounds__(256) xseq_kernel(const Tin *__restrict__ u, const float *__restrict__ W,
                                                   Tin *__restrict__ xdbl, int64_t D, int64_t L, int RN,
                                                   int64_t nlt) {
    constexpr int TM = 8 * TY, PA = kXsK + 4, PB = sizeof(Tin) == 4 ? kXsL + 4 : kXsL + 8;
    extern __shared__ __align__(16) unsigned char xs_smem[];
    float *As = reinterpret_cast<float *>(xs_smem);                                        // [kStages][TM][PA]
    Tin *Bs = reinterpret_cast<Tin *>(xs_smem + (size_t)kStages * TM * PA * sizeof(float));  // [kStages][kXsK][PB]
    const int t = threadIdx.x, ty = t / 32, tx = t % 32;
    const int64_t bid = blockIdx.x, g = bid / nlt, k = g % kPaths, l0 = (bid % nlt) * kXsL;
    const Tin *src = u + g * D * L + l0;
    const float *Wk = W + k * RN * D;
    const int nst = (int)ceil_div(D, kXsK);
    auto issue = [&](int st_) {
        const int buf = st_ % kStages;
        const int64_t d0 = (int64_t)st_ * kXsK;
        float *as = As + (size_t)buf * TM * PA;
        Tin *bs = Bs + (size_t)buf * kXsK * PB;
        if (VEC) {  // D % 4 == 0 and L % 4 == 0: every quad is wholly inside or outside
            for (int c = t; c < TM * (kXsK / 4); c += 256) {
                const int r = c / (kXsK / 4), j = 4 * (c % (kXsK / 4));
                float *dst = as + r * PA + j;
                if (r < RN && d0 + j < D) cp_async16(dst, Wk + r * D + d0 + j);
                else zero_quad(dst);
            }
            for (int c = t; c < kXsK * (kXsL / 4); c += 256) {
                const int r = c / (kXsL / 4), j = 4 * (c % (kXsL / 4));
                Tin *dst = bs + r * PB + j;
                if (d0 + r < D && l0 + j < L) cp_async_quad(dst, src + (d0 + r) * L + j);
                else zero_quad(dst);
            }
        } else {
            for (int e = t; e < TM * kXsK; e += 256) {
                const int r = e / kXsK, j = e % kXsK;
                as[r * PA + j] = (r < RN && d0 + j < D) ? Wk[r * D + d0 + j] : 0.f;
            }
            for (int e = t; e < kXsK * kXsL; e += 256) {
                const int r = e / kXsL, j = e % kXsL;
                st(bs + r * PB + j, (d0 + r < D && l0 + j < L) ? ld(src + (d0 + r) * L + j) : 0.f);
            }
        }
    };
    float2 acc[TY][2];
#pragma unroll
    for (int i = 0; i < TY; ++i) acc[i][0] = acc[i][1] = make_float2(0.f, 0.f);
#pragma unroll
    for (int st_ = 0; st_ < kStages - 1; ++st_) {
        if (st_ < nst) issue(st_);
        cp_async_commit();
    }
    for (int st_ = 0; st_ < nst; ++st_) {
        cp_async_wait<kStages - 2>();
        __syncthreads();  // stage st_ visible to all; every thread is done with stage st_ - 1's buffer
        if (st_ + kStages - 1 < nst) issue(st_ + kStages - 1);
        cp_async_commit();
        const float *as = As + (size_t)(st_ % kStages) * TM * PA + ty * PA;
        const Tin *bs = Bs + (size_t)(st_ % kStages) * kXsK * PB + 4 * tx;
#pragma unroll
        for (int dd = 0; dd < kXsK; ++dd) {
            const float4 b = ld4(bs + dd * PB);
            const float2 b01 = make_float2(b.x, b.y), b23 = make_float2(b.z, b.w);
#pragma unroll
            for (int i = 0; i < TY; ++i) {
                const float a = as[8 * i * PA + dd];
                acc[i][0] = __ffma2_rn(make_float2(a, a), b01, acc[i][0]);
                acc[i][1] = __ffma2_rn(make_float2(a, a), b23, acc[i][1]);
            }
        }
    }
    const int64_t l = l0 + 4 * tx;
    if (l >= L) return;
    Tin *o = xdbl + g * RN * L + l;
#pragma unroll
    for (int i = 0; i < TY; ++i) {
        const int c = ty + 8 * i;
        if (c >= RN) continue;
        const float v[4] = {acc[i][0].x, acc[i][0].y, acc[i][1].x, acc[i][1].y};
        if (VEC) {  // the quad is inside the row and 16-byte (fp32) / 8-byte (bf16) aligned
            store4(o + (int64_t)c * L, make_float4(v[0], v[1], v[2], v[3]));
        } else {
#pragma unroll
            for (int q = 0; q < 4; ++q)
                if (l + q < L) st(o + (int64_t)c * L + q, v[q]);
        }
    }
}

// ------------------------------------------------ short contractions (du, delta) --

constexpr int kChM = 64;   // channels per chan_kernel tile (8 thread rows x 8)
constexpr int kChL = 128;  // tokens per tile (32 thread columns x 4)

// out[g, d, l] (+)= sum_{c < C} M(k, d, c) in[g, c, l] over a 64-channel x 128-token tile, with
// M(k, d, c) = Wm[k*w_ks + d*w_ds + c*w_cs], in in_gs elements per group (rows of L), out D rows of L
// per group.  The contraction is short (C <= 64), so both operands (and, when ACC, the out tile
// itself) are staged whole and summed after one barrier; thread (ty, tx) holds channels ty + 8i
// and tokens 4tx..4tx+3, so a warp's write covers 128 contiguous elements of one row.  Token rows
// are copied with 16-byte cp.async when VEC (L % 4 == 0) and fp32, else with plain loads.
//   du:    du_seq += x_proj.weight^T dx_dbl   (fp32, ACC; M(k, d, c) = Wx[(k*RN + c)*D + d])
//   delta: delta   = dt_proj.weight x_dbl[:R] (in dtype; M(k, d, c) = Wdt[(k*D + d)*R + c])
template <typename Tin, typename Tout, bool ACC, bool VEC>
__global__ void __launch_bounds__(256) chan_kernel(const Tin *__restrict__ in, int64_t in_gs,
                                                   const float *__restrict__ Wm, int64_t w_ks, int64_t w_ds,
                                                   int64_t w_cs, Tout *__restrict__ out, int64_t D, int64_t L, int C,
                                                   int nmt, int64_t nlt) {
    static_assert(!ACC || sizeof(Tout) == 4, "accumulation is in fp32");
    constexpr int AS = kChM + 4, BS = kChL + 4;
    constexpr bool kAsyncIn = VEC && sizeof(Tin) == 4;
    extern __shared__ __align__(16) float chan_smem[];
    float *As = chan_smem;      // [C][AS]    M(k, d0 + ., c)
    float *Bs = As + C * AS;    // [C][BS]    in[g, c, l0 + .]
    float *Us = Bs + C * BS;    // [kChM][BS] out[g, d0 + ., l0 + .] (ACC and VEC only)
    const int t = threadIdx.x, ty = t / 32, tx = t % 32;
    // one flat grid: channel tiles fastest (they share the input tile, read once through L2)
    const int64_t bid = blockIdx.x, rest = bid / nmt, g = rest / nlt, k = g % kPaths;
    const int64_t d0 = (bid % nmt) * kChM, l0 = (rest % nlt) * kChL;
    const Tin *src = in + g * in_gs + l0;
    Tout *o0 = out + g * D * L + l0;
    // weights contiguous along the channels (w_ds = 1) and 16-byte aligned quads: cp.async too
    const bool async_w = VEC && w_ds == 1 && D % 4 == 0 && w_cs % 4 == 0 && w_ks % 4 == 0;
    if (async_w) {
        for (int e = t; e < C * (kChM / 4); e += 256) {
            const int c = e / (kChM / 4), j = 4 * (e % (kChM / 4));
            float *dst = As + c * AS + j;
            if (d0 + j < D) cp_async16(dst, Wm + k * w_ks + d0 + j + c * w_cs);
            else zero_quad(dst);
        }
    } else {
        for (int e = t; e < C * kChM; e += 256) {
            const int c = e / kChM, dd = e % kChM;
            As[c * AS + dd] = d0 + dd < D ? Wm[k * w_ks + (d0 + dd) * w_ds + c * w_cs] : 0.f;
        }
    }
    if (kAsyncIn || (ACC && VEC) || async_w) {
        const int cb = kAsyncIn ? C * (kChL / 4) : 0, cu = (ACC && VEC) ? kChM * (kChL / 4) : 0;
        for (int c = t; c < cb + cu; c += 256) {
            if (c < cb) {
                const int r = c / (kChL / 4), j = 4 * (c % (kChL / 4));
                float *dst = Bs + r * BS + j;
                if (l0 + j < L) cp_async16(dst, reinterpret_cast<const float *>(src) + r * L + j);
                else zero_quad(dst);
            } else {
                const int cc = c - cb, r = cc / (kChL / 4), j = 4 * (cc % (kChL / 4));
                if (d0 + r < D && l0 + j < L) cp_async16(Us + r * BS + j, o0 + (d0 + r) * L + j);
            }
        }
        cp_async_commit();
    }
    if (!kAsyncIn)
        for (int e = t; e < C * kChL; e += 256) {
            const int c = e / kChL, ll = e % kChL;
            Bs[c * BS + ll] = l0 + ll < L ? ld(src + c * L + ll) : 0.f;
        }
    if (kAsyncIn || (ACC && VEC) || async_w) cp_async_wait<0>();
    __syncthreads();
    float acc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[i][q] = 0.f;
#pragma unroll 4
    for (int c = 0; c < C; ++c) {
        const float4 bq = *reinterpret_cast<const float4 *>(&Bs[c * BS + 4 * tx]);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float a = As[c * AS + ty + 8 * i];
            acc[i][0] = fmaf(a, bq.x, acc[i][0]);
            acc[i][1] = fmaf(a, bq.y, acc[i][1]);
            acc[i][2] = fmaf(a, bq.z, acc[i][2]);
            acc[i][3] = fmaf(a, bq.w, acc[i][3]);
        }
    }
    const int64_t l = 4 * tx;  // within the tile
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int64_t d = d0 + ty + 8 * i;
        if (d >= D || l0 + l >= L) continue;
        Tout *o = o0 + d * L + l;
        if (VEC) {  // the whole quad is inside the row (L % 4 == 0)
            float4 v = make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
            if (ACC) {
                const float4 u = *reinterpret_cast<const float4 *>(&Us[(ty + 8 * i) * BS + l]);
                v = make_float4(u.x + v.x, u.y + v.y, u.z + v.z, u.w + v.w);
            }
            store4(o, v);
        } else {
#pragma unroll
            for (int q = 0; q < 4; ++q)
                if (l0 + l + q < L) st(o + q, ACC ? ld(o + q) + acc[i][q] : acc[i][q]);
        }
    }
}

// ------------------------------------------------- token sums of outer products --

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
    int nnt;  // tiles of N
    float *part;
};

constexpr int kTN = 128;  // tile columns: 32 lanes x 4, spaced 32 apart

template <typename TB, int TY>
constexpr size_t tr_smem_bytes() {
    return (size_t)kStages * (8 * TY * row_pitch<float>() * sizeof(float) + kTN * row_pitch<TB>() * sizeof(TB));
}

// CTA tile TM = 8*TY rows (all of M) x 128 columns over one token chunk, 256 threads: warp ty holds
// rows ty + 8i (i < TY), lane tx columns tx + 32q (q < 4).  Both operands sit in shared memory as
// [row][token] (their global layout), filled by 16-byte cp.async through a 3-stage ring when
// VEC (L % 4 == 0; every chunk of 4 tokens is then wholly inside or outside the range), else by
// plain loads.  Each step takes 4 tokens: TY row quads (broadcast in the warp) and 4 column quads
// feed 16*TY FMAs.  A reversed path (rev) holds its tokens backwards in the row.
template <typename TB, int TY, bool VEC>
__global__ void __launch_bounds__(256, 2) tr_gemm_kernel(const TrArgs p) {
    constexpr int TM = 8 * TY, PA = row_pitch<float>(), PB = row_pitch<TB>();
    constexpr int CA = TM * kTS / 4, CB = kTN * kTS / 4;  // 4-token chunks per stage
    extern __shared__ __align__(16) unsigned char tr_smem[];
    float *As = reinterpret_cast<float *>(tr_smem);                                   // [kStages][TM][PA]
    TB *Bs = reinterpret_cast<TB *>(tr_smem + (size_t)kStages * TM * PA * sizeof(float));  // [kStages][kTN][PB]
    const int t = threadIdx.x, ty = t / 32, tx = t % 32;
    // one flat grid: N tiles fastest, then (path, batch item, token chunk)
    const int64_t bid = blockIdx.x, z = bid / p.nnt;
    const int64_t k = z % kPaths, rest = z / kPaths, b = rest / p.nlc, lc = rest % p.nlc;
    const int64_t n0 = (bid % p.nnt) * kTN;
    const int64_t lb = lc * p.lchunk, le = p.L < lb + p.lchunk ? p.L : lb + p.lchunk;
    const float *A = static_cast<const float *>(p.A) + b * p.a_bs + k * p.a_ks;
    const void *bk = k == 0 ? p.Bp[0] : k == 1 ? p.Bp[1] : k == 2 ? p.Bp[2] : p.Bp[3];  // no local copy of p.Bp
    const TB *Bo = static_cast<const TB *>(bk) + b * p.b_bs;
    const bool rev = (p.rev_mask >> k) & 1;
    const int nst = (int)ceil_div(le - lb, kTS);

    // stage s: tokens t0 = lb + s*kTS .. min(t0 + kTS, le); slot j of a B row holds token
    // t0 + j, or t0 + kTS - 1 - j when rev.  Slots past the range hold zeros.
    auto issue = [&](int s) {
        const int buf = s % kStages;
        const int64_t t0 = lb + (int64_t)s * kTS;
        const int nv = (int)(le - t0 < kTS ? le - t0 : kTS);
        float *as = As + (size_t)buf * TM * PA;
        TB *bs = Bs + (size_t)buf * kTN * PB;
        if (VEC) {
            for (int c = t; c < CA; c += 256) {
                const int r = c / (kTS / 4), j = 4 * (c % (kTS / 4));
                float *dst = as + r * PA + j;
                if (r < p.M && j < nv) cp_async16(dst, A + r * p.L + t0 + j);
                else *reinterpret_cast<float4 *>(dst) = make_float4(0.f, 0.f, 0.f, 0.f);
            }
            for (int c = t; c < CB; c += 256) {
                const int r = c / (kTS / 4), j = 4 * (c % (kTS / 4));
                TB *dst = bs + r * PB + j;
                const int tok = rev ? kTS - 4 - j : j;  // first token of the slot quad, counted from t0
                if (n0 + r < p.N && tok < nv) {
                    const TB *src = Bo + (n0 + r) * p.L + (rev ? p.L - t0 - kTS + j : t0 + j);
                    cp_async_quad(dst, src);
                } else {
                    zero_quad(dst);
                }
            }
        } else {
            for (int e = t; e < TM * kTS; e += 256) {
                const int r = e / kTS, j = e % kTS;
                as[r * PA + j] = (r < p.M && j < nv) ? A[r * p.L + t0 + j] : 0.f;
            }
            for (int e = t; e < kTN * kTS; e += 256) {
                const int r = e / kTS, j = e % kTS, tok = rev ? kTS - 1 - j : j;
                const float v = (n0 + r < p.N && tok < nv) ? ld(Bo + (n0 + r) * p.L + (rev ? p.L - 1 - t0 - tok : t0 + tok))
                                                          : 0.f;
                st(bs + r * PB + j, v);
            }
        }
    };
    float acc[TY][4];
#pragma unroll
    for (int i = 0; i < TY; ++i)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[i][q] = 0.f;
#pragma unroll
    for (int s = 0; s < kStages - 1; ++s) {
        if (s < nst) issue(s);
        cp_async_commit();
    }
    for (int s = 0; s < nst; ++s) {
        cp_async_wait<kStages - 2>();
        __syncthreads();  // stage s visible to all; every thread is done with stage s - 1's buffer
        if (s + kStages - 1 < nst) issue(s + kStages - 1);
        cp_async_commit();
        const float *as = As + (size_t)(s % kStages) * TM * PA + ty * PA;
        const TB *bs = Bs + (size_t)(s % kStages) * kTN * PB + tx * PB;
#pragma unroll 2
        for (int tt = 0; tt < kTS; tt += 4) {
            float4 av[TY];
#pragma unroll
            for (int i = 0; i < TY; ++i) av[i] = ld4(as + 8 * i * PA + tt);
            const int jb = rev ? kTS - 4 - tt : tt;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float4 bq = ld4(bs + 32 * q * PB + jb);
                if (rev) bq = make_float4(bq.w, bq.z, bq.y, bq.x);
#pragma unroll
                for (int i = 0; i < TY; ++i) {
                    float a = acc[i][q];
                    a = fmaf(av[i].x, bq.x, a);
                    a = fmaf(av[i].y, bq.y, a);
                    a = fmaf(av[i].z, bq.z, a);
                    acc[i][q] = fmaf(av[i].w, bq.w, a);
                }
            }
        }
    }
    float *dst = p.part + ((k * p.B + b) * p.nlc + lc) * (int64_t)p.M * p.N;
#pragma unroll
    for (int i = 0; i < TY; ++i) {
        const int64_t m = ty + 8 * i;
        if (m >= p.M) continue;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int64_t n = n0 + tx + 32 * q;
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
        int64_t i = 0;
        for (; i + 8 <= nparts; i += 8) {  // eight loads in flight, added in the same order
            float v[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) v[j] = src[(i + j) * MN];
#pragma unroll
            for (int j = 0; j < 8; ++j) s += v[j];
        }
        for (; i < nparts; ++i) s += src[i * MN];
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

template <typename Tin, typename Tout, int RB>
static cudaError_t rows_t(const LaunchShape &s, const void *in, const float *Wm, int64_t w_ks, int64_t w_rs,
                          int64_t w_ds, void *out, int64_t out_gs, int R, cudaStream_t stream) {
    const int64_t nlt = ceil_div(s.L, kNarrowTok), blocks = nlt * s.B * kPaths;
    if (blocks > INT32_MAX) return cudaErrorInvalidConfiguration;
    rows_kernel<Tin, Tout, RB><<<(unsigned)blocks, kNarrowTok, 0, stream>>>(
        static_cast<const Tin *>(in), Wm, w_ks, w_rs, w_ds, static_cast<Tout *>(out), out_gs, s.D, s.L, R, nlt);
    return cudaSuccess;
}

template <typename Tin, typename Tout>
static cudaError_t rows_r(const LaunchShape &s, const void *in, const float *Wm, int64_t w_ks, int64_t w_rs,
                          int64_t w_ds, void *out, int64_t out_gs, int R, cudaStream_t stream) {
    switch ((R + 7) / 8) {  // R rounded up to 8 sums per thread, R <= 64
        case 1: return rows_t<Tin, Tout, 8>(s, in, Wm, w_ks, w_rs, w_ds, out, out_gs, R, stream);
        case 2: return rows_t<Tin, Tout, 16>(s, in, Wm, w_ks, w_rs, w_ds, out, out_gs, R, stream);
        case 3: return rows_t<Tin, Tout, 24>(s, in, Wm, w_ks, w_rs, w_ds, out, out_gs, R, stream);
        case 4: return rows_t<Tin, Tout, 32>(s, in, Wm, w_ks, w_rs, w_ds, out, out_gs, R, stream);
        case 5: return rows_t<Tin, Tout, 40>(s, in, Wm, w_ks, w_rs, w_ds, out, out_gs, R, stream);
        case 6: return rows_t<Tin, Tout, 48>(s, in, Wm, w_ks, w_rs, w_ds, out, out_gs, R, stream);
        case 7: return rows_t<Tin, Tout, 56>(s, in, Wm, w_ks, w_rs, w_ds, out, out_gs, R, stream);
        case 8: return rows_t<Tin, Tout, 64>(s, in, Wm, w_ks, w_rs, w_ds, out, out_gs, R, stream);
        default: return cudaErrorInvalidValue;
    }
}

// dx_dbl[:R] (fp32, group stride RN*L) = dt_proj.weight^T @ ddelta (in dtype, group stride D*L)
cudaError_t launch_proj_bwd_dtlow(const LaunchShape &s, ss2d_dtype_t dt, const void *ddelta, const float *Wdt, int R,
                                  int RN, float *dxdbl, cudaStream_t stream) {
    if (R < 1 || R > kProjRMax) return cudaErrorInvalidValue;
    // M(k, r, d) = Wdt[(k*D + d)*R + r]
    const cudaError_t e =
        dt == SS2D_F32
            ? rows_r<float, float>(s, ddelta, Wdt, s.D * R, 1, R, dxdbl, (int64_t)RN * s.L, R, stream)
            : rows_r<__nv_bfloat16, float>(s, ddelta, Wdt, s.D * R, 1, R, dxdbl, (int64_t)RN * s.L, R, stream);
    if (e != cudaSuccess) return e;
    note_launch(stream);
    return cudaGetLastError();
}

template <typename Tin, int TY>
static cudaError_t xseq_t(const LaunchShape &s, const void *u, const float *W, int RN, void *xdbl,
                          cudaStream_t stream) {
    const int64_t nlt = ceil_div(s.L, kXsL), blocks = nlt * s.B * kPaths;
    if (blocks > INT32_MAX) return cudaErrorInvalidConfiguration;
    const bool vec = s.L % 4 == 0 && s.D % 4 == 0;  // token and weight quads 16-byte (8-byte bf16) aligned
    auto kern = vec ? xseq_kernel<Tin, TY, true> : xseq_kernel<Tin, TY, false>;
    constexpr size_t smem = xseq_smem_bytes<Tin, TY>();  // at most 3 * (64 * 20 + 16 * 132) * 4 = 40,704 bytes
    kern<<<(unsigned)blocks, 256, smem, stream>>>(static_cast<const Tin *>(u), W, static_cast<Tin *>(xdbl), s.D,
                                                  s.L, RN, nlt);
    return cudaSuccess;
}

template <typename Tin>
static cudaError_t xseq_ty(const LaunchShape &s, const void *u, const float *W, int RN, void *xdbl,
                           cudaStream_t stream) {
    switch ((RN + 7) / 8) {  // rows R + 2N, 3..64, in one tile of 8 * TY rows
        case 1: return xseq_t<Tin, 1>(s, u, W, RN, xdbl, stream);
        case 2: return xseq_t<Tin, 2>(s, u, W, RN, xdbl, stream);
        case 3: return xseq_t<Tin, 3>(s, u, W, RN, xdbl, stream);
        case 4: return xseq_t<Tin, 4>(s, u, W, RN, xdbl, stream);
        case 5: return xseq_t<Tin, 5>(s, u, W, RN, xdbl, stream);
        case 6: return xseq_t<Tin, 6>(s, u, W, RN, xdbl, stream);
        case 7: return xseq_t<Tin, 7>(s, u, W, RN, xdbl, stream);
        case 8: return xseq_t<Tin, 8>(s, u, W, RN, xdbl, stream);
        default: return cudaErrorInvalidValue;
    }
}

// x_proj of per-path sequences: xdbl[b, k, c, l] = sum_d W[k, c, d] u[b, k*D + d, l] (in dtype)
cudaError_t launch_xproj_seq(const LaunchShape &s, ss2d_dtype_t dt, const void *u, const float *W, int RN, void *xdbl,
                             cudaStream_t stream) {
    if (RN < 1 || RN > kProjRMax + 2 * 16) return cudaErrorInvalidValue;
    const cudaError_t e = dt == SS2D_F32 ? xseq_ty<float>(s, u, W, RN, xdbl, stream)
                                         : xseq_ty<__nv_bfloat16>(s, u, W, RN, xdbl, stream);
    if (e != cudaSuccess) return e;
    note_launch(stream);
    return cudaGetLastError();
}

constexpr int kRNMax = kProjRMax + 2 * 16;  // rows of x_dbl: dt rank <= 32, d_state <= 16

static size_t chan_smem_bytes(int C, bool acc) {
    return ((size_t)C * ((kChM + 4) + (kChL + 4)) + (acc ? kChM * (kChL + 4) : 0)) * sizeof(float);
}

template <typename Tin, typename Tout, bool ACC>
static cudaError_t chan_t(const LaunchShape &s, const void *in, int64_t in_gs, const float *Wm, int64_t w_ks,
                          int64_t w_ds, int64_t w_cs, void *out, int C, cudaStream_t stream) {
    if (C < 1 || C > kRNMax) return cudaErrorInvalidValue;
    const bool vec = s.L % 4 == 0;  // token rows, and the out rows, 16-byte (fp32) / 8-byte (bf16) aligned
    auto kern = vec ? chan_kernel<Tin, Tout, ACC, true> : chan_kernel<Tin, Tout, ACC, false>;
    // up to (64 * 200 + 64 * 132) * 4 = 84,992 bytes: opt in on the current device (cheap, right on any device)
    const cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)chan_smem_bytes(kRNMax, ACC));
    if (e != cudaSuccess) return e;
    const int nmt = (int)ceil_div(s.D, kChM);
    const int64_t nlt = ceil_div(s.L, kChL), blocks = nmt * nlt * s.B * kPaths;
    if (blocks > INT32_MAX) return cudaErrorInvalidConfiguration;
    kern<<<(unsigned)blocks, 256, chan_smem_bytes(C, ACC), stream>>>(static_cast<const Tin *>(in), in_gs, Wm, w_ks,
                                                                     w_ds, w_cs, static_cast<Tout *>(out), s.D, s.L,
                                                                     C, nmt, nlt);
    return cudaSuccess;
}

// du_seq (fp32, (B, 4D, L)) += x_proj.weight^T @ dx_dbl (fp32, group stride RN*L); du_seq 16-byte aligned
cudaError_t launch_proj_bwd_du(const LaunchShape &s, const float *dxdbl, const float *Wx, int RN, float *du_seq,
                               cudaStream_t stream) {
    // M(k, d, c) = Wx[(k*RN + c)*D + d]
    const cudaError_t e = chan_t<float, float, true>(s, dxdbl, (int64_t)RN * s.L, Wx, (int64_t)RN * s.D, 1, s.D,
                                                     du_seq, RN, stream);
    if (e != cudaSuccess) return e;
    note_launch(stream);
    return cudaGetLastError();
}

// delta[b, k*D + d, l] = sum_r Wdt[k*D + d, r] xdbl[b, k, r, l] (in dtype): dt_proj for ranks where
// the scan would spend more on R multiply-adds per step than on reading delta, and for the backward
cudaError_t launch_dtproj(const LaunchShape &s, ss2d_dtype_t dt, const void *xdbl, const float *Wdt, int R, int RN,
                          void *delta, cudaStream_t stream) {
    if (R < 1 || R > kProjRMax) return cudaErrorInvalidValue;
    // M(k, d, c) = Wdt[(k*D + d)*R + c]
    const cudaError_t e =
        dt == SS2D_F32 ? chan_t<float, float, false>(s, xdbl, (int64_t)RN * s.L, Wdt, s.D * R, R, 1, delta, R, stream)
                       : chan_t<__nv_bfloat16, __nv_bfloat16, false>(s, xdbl, (int64_t)RN * s.L, Wdt, s.D * R, R, 1,
                                                                     delta, R, stream);
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

static void reduce_partials(const LaunchShape &s, const float *part, float *out, int64_t MN, cudaStream_t stream) {
    reduce_partials_kernel<<<grid_cap(kPaths * MN, 256), 256, 0, stream>>>(part, out, s.B * proj_bwd_chunks(s), MN);
    note_launch(stream);
}

template <typename Tin, int RB>
static cudaError_t dwdt_t(const LaunchShape &s, const void *ddelta, const void *xdbl, int R, int RN, float *part,
                          cudaStream_t stream) {
    const int nlc = (int)proj_bwd_chunks(s), ndt = (int)ceil_div(s.D, kDwD);
    const int64_t blocks = (int64_t)ndt * kPaths * s.B * nlc;
    if (blocks > INT32_MAX) return cudaErrorInvalidConfiguration;
    constexpr size_t smem = dwdt_smem_bytes<Tin, RB>();  // at most 3 * 96 * 36 * 4 = 41,472 bytes
    auto kern = s.L % 4 == 0 ? dwdt_kernel<Tin, RB, true> : dwdt_kernel<Tin, RB, false>;
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)blocks, 256, smem, stream>>>(static_cast<const Tin *>(ddelta), static_cast<const Tin *>(xdbl),
                                                  part, s.B, s.D, s.L, R, RN, kProjTokenChunk, nlc, ndt);
    return cudaSuccess;
}

template <typename Tin>
static cudaError_t dwdt_r(const LaunchShape &s, const void *ddelta, const void *xdbl, int R, int RN, float *part,
                          cudaStream_t stream) {
    if (R <= 8) return dwdt_t<Tin, 8>(s, ddelta, xdbl, R, RN, part, stream);
    if (R <= 16) return dwdt_t<Tin, 16>(s, ddelta, xdbl, R, RN, part, stream);
    if (R <= 24) return dwdt_t<Tin, 24>(s, ddelta, xdbl, R, RN, part, stream);
    return dwdt_t<Tin, 32>(s, ddelta, xdbl, R, RN, part, stream);
}

// d dt_proj.weight (4, D, R) = sum over tokens of ddelta (x) x_dbl[:R]
cudaError_t launch_proj_bwd_dwdt(const LaunchShape &s, ss2d_dtype_t dt, const void *ddelta, const void *xdbl, int R,
                                 int RN, float *part, float *dWdt, cudaStream_t stream) {
    if (R < 1 || R > kProjRMax) return cudaErrorInvalidValue;
    const cudaError_t e = dt == SS2D_F32 ? dwdt_r<float>(s, ddelta, xdbl, R, RN, part, stream)
                                         : dwdt_r<__nv_bfloat16>(s, ddelta, xdbl, R, RN, part, stream);
    if (e != cudaSuccess) return e;
    note_launch(stream);
    reduce_partials(s, part, dWdt, s.D * R, stream);
    return cudaGetLastError();
}

template <typename TB, int TY>
static cudaError_t dwx_t(const LaunchShape &s, TrArgs p, cudaStream_t stream) {
    const int64_t blocks = (int64_t)p.nnt * kPaths * s.B * p.nlc;
    if (blocks > INT32_MAX) return cudaErrorInvalidConfiguration;
    constexpr size_t smem = tr_smem_bytes<TB, TY>();  // at most 3 * (64 + 128) * 36 * 4 = 82,944 bytes
    const bool vec = s.L % 4 == 0;  // token quads then start 16-byte (fp32) / 8-byte (bf16) aligned
    auto kern = vec ? tr_gemm_kernel<TB, TY, true> : tr_gemm_kernel<TB, TY, false>;
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)blocks, 256, smem, stream>>>(p);
    return cudaSuccess;
}

template <typename TB>
static cudaError_t dwx_ty(const LaunchShape &s, TrArgs p, cudaStream_t stream) {
    switch ((int)ceil_div(p.M, 8)) {  // rows R + 2N, 3..64, in one tile of 8 * TY rows
        case 1: return dwx_t<TB, 1>(s, p, stream);
        case 2: return dwx_t<TB, 2>(s, p, stream);
        case 3: return dwx_t<TB, 3>(s, p, stream);
        case 4: return dwx_t<TB, 4>(s, p, stream);
        case 5: return dwx_t<TB, 5>(s, p, stream);
        case 6: return dwx_t<TB, 6>(s, p, stream);
        case 7: return dwx_t<TB, 7>(s, p, stream);
        case 8: return dwx_t<TB, 8>(s, p, stream);
        default: return cudaErrorInvalidValue;
    }
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
    p.B = s.B;
    p.L = s.L;
    p.lchunk = kProjTokenChunk;
    p.nlc = (int)proj_bwd_chunks(s);
    p.nnt = (int)ceil_div(p.N, kTN);
    p.part = part;
    const cudaError_t e = dt == SS2D_F32 ? dwx_ty<float>(s, p, stream) : dwx_ty<__nv_bfloat16>(s, p, stream);
    if (e != cudaSuccess) return e;
    note_launch(stream);
    reduce_partials(s, part, dWx, (int64_t)RN * s.D, stream);
    return cudaGetLastError();
}


// d x_proj.weight (4, RN, D) = sum over tokens of dx_dbl (x) u_k for per-path sequences u (B, 4D, L)
cudaError_t launch_proj_bwd_dwx_seq(const LaunchShape &s, ss2d_dtype_t dt, const float *dxdbl, const void *u, int RN,
                                    float *part, float *dWx, cudaStream_t stream) {
    TrArgs p{};
    p.A = dxdbl;
    p.a_bs = (int64_t)kPaths * RN * s.L;
    p.a_ks = (int64_t)RN * s.L;
    const size_t es = dt == SS2D_F32 ? 4 : 2;
    for (int k = 0; k < kPaths; ++k) p.Bp[k] = static_cast<const unsigned char *>(u) + (size_t)k * s.D * s.L * es;
    p.b_bs = (int64_t)kPaths * s.D * s.L;
    p.rev_mask = 0;
    p.M = RN;
    p.N = (int)s.D;
    p.B = s.B;
    p.L = s.L;
    p.lchunk = kProjTokenChunk;
    p.nlc = (int)proj_bwd_chunks(s);
    p.nnt = (int)ceil_div(p.N, kTN);
    p.part = part;
    const cudaError_t e = dt == SS2D_F32 ? dwx_ty<float>(s, p, stream) : dwx_ty<__nv_bfloat16>(s, p, stream);
    if (e != cudaSuccess) return e;
    note_launch(stream);
    reduce_partials(s, part, dWx, (int64_t)RN * s.D, stream);
    return cudaGetLastError();
}

}  // namespace ss2d
