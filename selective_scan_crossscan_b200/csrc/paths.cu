// paths.cu -- path sets given as tables: CrossScan, CrossMerge and the path-order copies
// that let the fused kernels run any four paths.
//
// A path set is two pixel orders over the H x W grid, paths 0 and 1; paths 2 and 3
// walk them backwards (the structure of the VMamba page's cross scan, Fig. 2).  The
// table holds, as int32 (4, L): fwd0[l], fwd1[l] = pixel visited at step l, then
// inv0[p], inv1[p] = step at which pixel p is visited.  Two sets are generated here:
//  * cross:    row-major, column-major (l = w*H + h);
//  * diagonal: the two diagonal scans of "Visual Mamba实战从零开始搭建图像分类模型附PyTorch
//              代码" (section 3, SS2D._get_diagonal_indices): anti-diagonals s = i + j in
//              turn, rows ascending within each, j = s - i (path 0) or j = (W-1) - (s - i)
//              (path 1).
// Any table a caller supplies is bounds-checked entry by entry: an entry outside [0, L)
// reads as zero and is never used as a store address.
//
// The fused path keeps the image-mode scan unchanged: path 0 reads a copy of x in path-0
// order, path 1 a copy in path-1 order (the cross set's copies are x itself and its
// transpose), paths 2/3 the same copies backwards.  Copies and merges stage one (b, d)
// plane in shared memory so that both the global reads and the global writes are
// contiguous; planes too large for shared memory (96 KB) gather through L2 instead.
#include "common.cuh"
#include "kernels.h"

namespace ss2d {

constexpr int kPathThreads = 256;
constexpr size_t kPlaneSmemMax = 96 * 1024;  // bytes of shared memory a staged plane may use

// first step of anti-diagonal s: the lengths min(t + 1, H, W, H + W - 1 - t) of the ones before it
__device__ __forceinline__ int64_t diag_start(int64_t s, int64_t H, int64_t W) {
    int64_t acc = 0;
    for (int64_t t = 0; t < s; ++t) acc += min(min(t + 1, H), min(W, H + W - 1 - t));
    return acc;
}

__device__ __forceinline__ int64_t diag_step(int64_t i, int64_t s, int64_t H, int64_t W) {
    return diag_start(s, H, W) + (i - max((int64_t)0, s - W + 1));
}

__global__ void path_tables_kernel(int kind, int64_t H, int64_t W, int32_t *tab) {
    const int64_t L = H * W;
    const int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (p >= L) return;
    const int64_t i = p / W, j = p - (p / W) * W;
    int64_t l0, l1;
    if (kind == SS2D_PATHS_DIAGONAL) {
        l0 = diag_step(i, i + j, H, W);            // j = s - i
        l1 = diag_step(i, i + (W - 1 - j), H, W);  // j = (W-1) - (s - i)
    } else {
        l0 = p;
        l1 = j * H + i;
    }
    if (l0 >= 0 && l0 < L) {
        tab[l0] = (int32_t)p;
        tab[2 * L + p] = (int32_t)l0;
    }
    if (l1 >= 0 && l1 < L) {
        tab[L + l1] = (int32_t)p;
        tab[3 * L + p] = (int32_t)l1;
    }
}

__device__ __forceinline__ bool in_range(int32_t v, int64_t L) { return v >= 0 && (int64_t)v < L; }

// KOUT = 2: the path-order copies c0[l] = x[fwd0[l]], c1[l] = x[fwd1[l]] of every plane.
// KOUT = 4: CrossScan xs[b, k, d, l] along the four paths (2 and 3 backwards).
template <typename T, int KOUT, bool SMEM, bool VEC4>
__global__ void __launch_bounds__(kPathThreads) path_gather_kernel(const T *__restrict__ x,
                                                                   const int32_t *__restrict__ tab,
                                                                   T *__restrict__ out0, T *__restrict__ out1,
                                                                   int64_t B, int64_t D, int64_t L) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    T *row = reinterpret_cast<T *>(smem_raw);
    const int32_t *f0 = tab, *f1 = tab + L;
    for (int64_t plane = blockIdx.x; plane < B * D; plane += gridDim.x) {
        const T *src = x + plane * L;
        if (SMEM) {
            __syncthreads();  // the previous plane's reads are done
            if (VEC4) {
                for (int64_t l = 4 * threadIdx.x; l < L; l += 4 * blockDim.x) {
                    float v[4];
                    ld4(src + l, v);
                    st4(row + l, v);
                }
            } else {
                for (int64_t l = threadIdx.x; l < L; l += blockDim.x) row[l] = src[l];
            }
            __syncthreads();
        }
        const T *rd = SMEM ? row : src;
        const T zero = T(0.f);
        if (KOUT == 2 && VEC4) {  // four steps per thread, 16-byte table loads, 4-element stores
            for (int64_t l = 4 * threadIdx.x; l < L; l += 4 * blockDim.x) {
                const int4 p0 = *reinterpret_cast<const int4 *>(f0 + l);
                const int4 p1 = *reinterpret_cast<const int4 *>(f1 + l);
                const float a[4] = {in_range(p0.x, L) ? ld(rd + p0.x) : 0.f, in_range(p0.y, L) ? ld(rd + p0.y) : 0.f,
                                    in_range(p0.z, L) ? ld(rd + p0.z) : 0.f, in_range(p0.w, L) ? ld(rd + p0.w) : 0.f};
                const float c[4] = {in_range(p1.x, L) ? ld(rd + p1.x) : 0.f, in_range(p1.y, L) ? ld(rd + p1.y) : 0.f,
                                    in_range(p1.z, L) ? ld(rd + p1.z) : 0.f, in_range(p1.w, L) ? ld(rd + p1.w) : 0.f};
                st4(out0 + plane * L + l, a);
                st4(out1 + plane * L + l, c);
            }
        } else if (KOUT == 2) {
            for (int64_t l = threadIdx.x; l < L; l += blockDim.x) {
                const int32_t p0 = f0[l], p1 = f1[l];
                out0[plane * L + l] = in_range(p0, L) ? rd[p0] : zero;
                out1[plane * L + l] = in_range(p1, L) ? rd[p1] : zero;
            }
        } else {
            const int64_t b = plane / D, d = plane - (plane / D) * D;
            T *o = out0 + (b * kPaths * D + d) * L;  // xs[b, 0, d, :]; path k is k*D*L further
            for (int64_t l = threadIdx.x; l < L; l += blockDim.x) {
                const int32_t p0 = f0[l], p1 = f1[l], q0 = f0[L - 1 - l], q1 = f1[L - 1 - l];
                o[l] = in_range(p0, L) ? rd[p0] : zero;
                o[D * L + l] = in_range(p1, L) ? rd[p1] : zero;
                o[2 * D * L + l] = in_range(q0, L) ? rd[q0] : zero;
                o[3 * D * L + l] = in_range(q1, L) ? rd[q1] : zero;
            }
        }
    }
}

// CrossMerge over a table: y[b, d, p] = (t0 + t2) + (t1 + t3) in fp32, one rounding, where t_k
// is path k's output for pixel p.  SMEM: walk paths 0/2 in their own order (reading the ys rows
// front to back and back to front, so every global read is sequential) and scatter t0 + t2 into
// a shared plane, then add t1 + t3 the same way along paths 1/3, then write the plane out
// contiguously.  Along a path consecutive steps are pixels W-1 or W+1 apart, so the scattered
// shared accesses spread over the banks.  Otherwise gather each pixel's values through the
// inverse rows of the table.
template <typename Tin, typename Tout, bool SMEM, bool VEC4>
__global__ void __launch_bounds__(kPathThreads) path_merge_kernel(const Tin *__restrict__ ys,
                                                                  const int32_t *__restrict__ tab,
                                                                  Tout *__restrict__ y, int64_t B, int64_t D,
                                                                  int64_t L) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    float *acc = reinterpret_cast<float *>(smem_raw);  // [L]
    const int32_t *f0 = tab, *f1 = tab + L, *i0 = tab + 2 * L, *i1 = tab + 3 * L;
    for (int64_t plane = blockIdx.x; plane < B * D; plane += gridDim.x) {
        const int64_t b = plane / D, d = plane - (plane / D) * D;
        const Tin *r0 = ys + (b * kPaths * D + d) * L;  // ys[b, k, d, :] is k*D*L further
        const Tin *r1 = r0 + D * L, *r2 = r0 + 2 * D * L, *r3 = r0 + 3 * D * L;
        if (SMEM) {
            __syncthreads();  // the previous plane has been written out
            for (int64_t p = threadIdx.x; p < L; p += blockDim.x) acc[p] = 0.f;
            __syncthreads();
            if (VEC4) {  // L % 4 == 0: four steps per thread, 16-byte row and table loads
                for (int64_t l = 4 * threadIdx.x; l < L; l += 4 * blockDim.x) {
                    float u[4], w[4];
                    ld4(r0 + l, u);
                    ld4(r2 + (L - 4 - l), w);  // steps L-1-l .. L-4-l of path 2, backwards
                    const int4 a = *reinterpret_cast<const int4 *>(f0 + l);
                    if (in_range(a.x, L)) acc[a.x] = u[0] + w[3];
                    if (in_range(a.y, L)) acc[a.y] = u[1] + w[2];
                    if (in_range(a.z, L)) acc[a.z] = u[2] + w[1];
                    if (in_range(a.w, L)) acc[a.w] = u[3] + w[0];
                }
                __syncthreads();
                for (int64_t l = 4 * threadIdx.x; l < L; l += 4 * blockDim.x) {
                    float u[4], w[4];
                    ld4(r1 + l, u);
                    ld4(r3 + (L - 4 - l), w);
                    const int4 c = *reinterpret_cast<const int4 *>(f1 + l);
                    if (in_range(c.x, L)) acc[c.x] = acc[c.x] + (u[0] + w[3]);
                    if (in_range(c.y, L)) acc[c.y] = acc[c.y] + (u[1] + w[2]);
                    if (in_range(c.z, L)) acc[c.z] = acc[c.z] + (u[2] + w[1]);
                    if (in_range(c.w, L)) acc[c.w] = acc[c.w] + (u[3] + w[0]);
                }
                __syncthreads();
                for (int64_t p = 4 * threadIdx.x; p < L; p += 4 * blockDim.x) {
                    const float v[4] = {acc[p], acc[p + 1], acc[p + 2], acc[p + 3]};
                    st4(y + plane * L + p, v);
                }
            } else {
                for (int64_t l = threadIdx.x; l < L; l += blockDim.x) {
                    const int32_t a = f0[l];
                    if (in_range(a, L)) acc[a] = ld(r0 + l) + ld(r2 + (L - 1 - l));
                }
                __syncthreads();
                for (int64_t l = threadIdx.x; l < L; l += blockDim.x) {
                    const int32_t c = f1[l];
                    if (in_range(c, L)) acc[c] = acc[c] + (ld(r1 + l) + ld(r3 + (L - 1 - l)));
                }
                __syncthreads();
                for (int64_t p = threadIdx.x; p < L; p += blockDim.x) st(y + plane * L + p, acc[p]);
            }
        } else {
            for (int64_t p = threadIdx.x; p < L; p += blockDim.x) {
                const int32_t a = i0[p], c = i1[p];
                float v = 0.f;
                if (in_range(a, L) && in_range(c, L))
                    v = (ld(r0 + a) + ld(r2 + (L - 1 - a))) + (ld(r1 + c) + ld(r3 + (L - 1 - c)));
                st(y + plane * L + p, v);
            }
        }
    }
}

// A CTA works on one plane at a time: as many threads as the plane has items (steps, or
// 4-step vectors), rounded up to whole warps, at most kPathThreads; enough CTAs to keep
// 2048 threads on each of the 148 SMs.
static int plane_threads(int64_t items) {
    const int64_t t = (items + 31) / 32 * 32;
    return (int)(t < 32 ? 32 : (t > kPathThreads ? kPathThreads : t));
}

static int plane_grid(int64_t planes, int threads) {
    const int64_t cap = 148LL * (2048 / threads);
    return (int)(planes < cap ? (planes > 0 ? planes : 1) : cap);
}

cudaError_t launch_path_tables(int kind, int64_t H, int64_t W, int32_t *tab, cudaStream_t stream) {
    const int64_t L = H * W;
    path_tables_kernel<<<(unsigned)ceil_div(L, kPathThreads), kPathThreads, 0, stream>>>(kind, H, W, tab);
    note_launch(stream);
    return cudaGetLastError();
}

template <typename T, int KOUT>
static cudaError_t launch_gather_t(const LaunchShape &s, const void *x, const int32_t *tab, void *out0, void *out1,
                                   cudaStream_t stream) {
    const size_t smem = (size_t)s.L * sizeof(T);
    if (smem <= kPlaneSmemMax) {
        // 4-step vectors need L % 4 == 0 and aligned rows, tables and outputs (the 4-path form
        // keeps scalar stores)
        const uintptr_t bases = reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(tab) |
                                reinterpret_cast<uintptr_t>(out0) | reinterpret_cast<uintptr_t>(out1);
        const bool vec = KOUT == 2 && s.L % 4 == 0 && (bases & 15) == 0;
        const int threads = plane_threads(vec ? s.L / 4 : s.L);
        auto kern = vec ? path_gather_kernel<T, KOUT, true, true> : path_gather_kernel<T, KOUT, true, false>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<plane_grid(s.B * s.D, threads), threads, smem, stream>>>(
            static_cast<const T *>(x), tab, static_cast<T *>(out0), static_cast<T *>(out1), s.B, s.D, s.L);
    } else {
        path_gather_kernel<T, KOUT, false, false><<<plane_grid(s.B * s.D, kPathThreads), kPathThreads, 0, stream>>>(
            static_cast<const T *>(x), tab, static_cast<T *>(out0), static_cast<T *>(out1), s.B, s.D, s.L);
    }
    note_launch(stream);
    return cudaGetLastError();
}

cudaError_t launch_path_copies(const LaunchShape &s, ss2d_dtype_t dt, const void *x, const int32_t *tab, void *c0,
                               void *c1, cudaStream_t stream) {
    if (dt == SS2D_F32) return launch_gather_t<float, 2>(s, x, tab, c0, c1, stream);
    return launch_gather_t<__nv_bfloat16, 2>(s, x, tab, c0, c1, stream);
}

cudaError_t launch_cross_scan_table(const LaunchShape &s, ss2d_dtype_t dt, const void *x, const int32_t *tab,
                                    void *xs, cudaStream_t stream) {
    if (dt == SS2D_F32) return launch_gather_t<float, 4>(s, x, tab, xs, nullptr, stream);
    return launch_gather_t<__nv_bfloat16, 4>(s, x, tab, xs, nullptr, stream);
}

template <typename Tin, typename Tout>
static cudaError_t launch_merge_t(const LaunchShape &s, const void *ys, const int32_t *tab, void *y,
                                  cudaStream_t stream) {
    const size_t smem = (size_t)s.L * sizeof(float);
    if (smem <= kPlaneSmemMax) {
        // 4-step vectors need 16-byte aligned rows, tables and outputs: L % 4 == 0 and aligned bases
        const bool vec = s.L % 4 == 0 && ((reinterpret_cast<uintptr_t>(ys) | reinterpret_cast<uintptr_t>(tab) |
                                           reinterpret_cast<uintptr_t>(y)) & 15) == 0;
        const int threads = plane_threads(vec ? s.L / 4 : s.L);
        auto kern = vec ? path_merge_kernel<Tin, Tout, true, true> : path_merge_kernel<Tin, Tout, true, false>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<plane_grid(s.B * s.D, threads), threads, smem, stream>>>(static_cast<const Tin *>(ys), tab,
                                                                         static_cast<Tout *>(y), s.B, s.D, s.L);
    } else {
        path_merge_kernel<Tin, Tout, false, false><<<plane_grid(s.B * s.D, kPathThreads), kPathThreads, 0, stream>>>(
            static_cast<const Tin *>(ys), tab, static_cast<Tout *>(y), s.B, s.D, s.L);
    }
    note_launch(stream);
    return cudaGetLastError();
}

cudaError_t launch_cross_merge_table(const LaunchShape &s, ss2d_dtype_t din, ss2d_dtype_t dout, const void *ys,
                                     const int32_t *tab, void *y, cudaStream_t stream) {
    using bf = __nv_bfloat16;
    if (din == SS2D_F32 && dout == SS2D_F32) return launch_merge_t<float, float>(s, ys, tab, y, stream);
    if (din == SS2D_F32) return launch_merge_t<float, bf>(s, ys, tab, y, stream);
    if (dout == SS2D_F32) return launch_merge_t<bf, float>(s, ys, tab, y, stream);
    return launch_merge_t<bf, bf>(s, ys, tab, y, stream);
}

}  // namespace ss2d
