// cross.cu -- CrossScan and CrossMerge (VMamba, "2D Selective Scan (SS2D) for
// visual data", Fig. 2: unfold the map along four paths / merge the four
// per-path outputs back into the map by summation).
//
// Both are pure data movement bounded by HBM.  A CTA owns a 32x32 pixel tile
// of one (b, d) plane.  Row-major paths (k=0 forward, k=2 backward) are read
// or written with lanes along w; column-major paths (k=1, k=3, step
// l = w*H + h) with lanes along h, the tile being transposed through shared
// memory, so every global access of a warp touches consecutive addresses.
#include "common.cuh"
#include "kernels.h"

namespace ss2d {

constexpr int kTile = 32;
constexpr int kRows = 8;  // blockDim = (32, 8)

template <typename T>
__global__ void __launch_bounds__(kTile * kRows)
cross_scan_kernel(const T *__restrict__ x, T *__restrict__ xs, int64_t Dn, int64_t H, int64_t W,
                  int64_t tiles_w, int64_t tiles_h) {
    __shared__ T tile[kTile][kTile + 1];
    int64_t blk = blockIdx.x;
    const int64_t tw = blk % tiles_w;
    blk /= tiles_w;
    const int64_t th = blk % tiles_h;
    const int64_t bd = blk / tiles_h;  // b * D + d
    const int64_t b = bd / Dn, d = bd - b * Dn;
    const int64_t L = H * W;
    const int64_t h0 = th * kTile, w0 = tw * kTile;
    const T *plane = x + bd * L;
    T *out0 = xs + ((b * kPaths + 0) * Dn + d) * L;
    T *out1 = xs + ((b * kPaths + 1) * Dn + d) * L;
    T *out2 = xs + ((b * kPaths + 2) * Dn + d) * L;
    T *out3 = xs + ((b * kPaths + 3) * Dn + d) * L;
    const int tx = threadIdx.x, ty = threadIdx.y;

#pragma unroll
    for (int j = 0; j < kTile / kRows; ++j) {
        const int hh = ty + kRows * j;
        const int64_t h = h0 + hh, w = w0 + tx;
        if (h < H && w < W) {
            const int64_t p = h * W + w;
            const T v = plane[p];
            tile[hh][tx] = v;
            out0[p] = v;          // row-major: step l = p
            out2[L - 1 - p] = v;  // reversed row-major
        }
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < kTile / kRows; ++j) {
        const int ww = ty + kRows * j;
        const int64_t h = h0 + tx, w = w0 + ww;
        if (h < H && w < W) {
            const T v = tile[tx][ww];
            const int64_t l = w * H + h;  // column-major step
            out1[l] = v;
            out3[L - 1 - l] = v;
        }
    }
}

template <typename Tin, typename Tout>
__global__ void __launch_bounds__(kTile * kRows)
cross_merge_kernel(const Tin *__restrict__ ys, Tout *__restrict__ y, int64_t Dn, int64_t H, int64_t W,
                   int64_t tiles_w, int64_t tiles_h) {
    __shared__ float t13[kTile][kTile + 1];  // (t1 + t3) at (hh, ww)
    int64_t blk = blockIdx.x;
    const int64_t tw = blk % tiles_w;
    blk /= tiles_w;
    const int64_t th = blk % tiles_h;
    const int64_t bd = blk / tiles_h;
    const int64_t b = bd / Dn, d = bd - b * Dn;
    const int64_t L = H * W;
    const int64_t h0 = th * kTile, w0 = tw * kTile;
    const Tin *in0 = ys + ((b * kPaths + 0) * Dn + d) * L;
    const Tin *in1 = ys + ((b * kPaths + 1) * Dn + d) * L;
    const Tin *in2 = ys + ((b * kPaths + 2) * Dn + d) * L;
    const Tin *in3 = ys + ((b * kPaths + 3) * Dn + d) * L;
    Tout *plane = y + bd * L;
    const int tx = threadIdx.x, ty = threadIdx.y;

#pragma unroll
    for (int j = 0; j < kTile / kRows; ++j) {
        const int ww = ty + kRows * j;
        const int64_t h = h0 + tx, w = w0 + ww;
        if (h < H && w < W) {
            const int64_t l = w * H + h;
            t13[tx][ww] = ld(in1 + l) + ld(in3 + (L - 1 - l));
        }
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < kTile / kRows; ++j) {
        const int hh = ty + kRows * j;
        const int64_t h = h0 + hh, w = w0 + tx;
        if (h < H && w < W) {
            const int64_t p = h * W + w;
            const float t02 = ld(in0 + p) + ld(in2 + (L - 1 - p));
            st(plane + p, t02 + t13[hh][tx]);
        }
    }
}

static dim3 tile_grid(int64_t planes, int64_t H, int64_t W, int64_t *tw, int64_t *th) {
    *tw = ceil_div(W, kTile);
    *th = ceil_div(H, kTile);
    return dim3((unsigned)(planes * *tw * *th));
}

cudaError_t launch_cross_scan(const LaunchShape &s, ss2d_dtype_t dt, const void *x, void *xs,
                              cudaStream_t stream) {
    int64_t tw, th;
    dim3 grid = tile_grid(s.B * s.D, s.H, s.W, &tw, &th);
    dim3 block(kTile, kRows);
    if (dt == SS2D_F32)
        cross_scan_kernel<float><<<grid, block, 0, stream>>>((const float *)x, (float *)xs, s.D, s.H, s.W, tw, th);
    else
        cross_scan_kernel<__nv_bfloat16><<<grid, block, 0, stream>>>(
            (const __nv_bfloat16 *)x, (__nv_bfloat16 *)xs, s.D, s.H, s.W, tw, th);
    note_launch(stream);
    return cudaGetLastError();
}

// x (B, D, H, W) -> xT (B, D, W, H): the column-major paths of the fused
// forward then read their sequence contiguously (row k=1 of xT is path 1).
template <typename T>
__global__ void __launch_bounds__(kTile * kRows)
transpose_kernel(const T *__restrict__ x, T *__restrict__ xT, int64_t H, int64_t W, int64_t tiles_w,
                 int64_t tiles_h) {
    __shared__ T tile[kTile][kTile + 1];
    int64_t blk = blockIdx.x;
    const int64_t tw = blk % tiles_w;
    blk /= tiles_w;
    const int64_t th = blk % tiles_h;
    const int64_t bd = blk / tiles_h;
    const int64_t L = H * W;
    const int64_t h0 = th * kTile, w0 = tw * kTile;
    const T *plane = x + bd * L;
    T *tplane = xT + bd * L;
    const int tx = threadIdx.x, ty = threadIdx.y;
#pragma unroll
    for (int j = 0; j < kTile / kRows; ++j) {
        const int hh = ty + kRows * j;
        const int64_t h = h0 + hh, w = w0 + tx;
        if (h < H && w < W) tile[hh][tx] = plane[h * W + w];
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < kTile / kRows; ++j) {
        const int ww = ty + kRows * j;
        const int64_t h = h0 + tx, w = w0 + ww;
        if (h < H && w < W) tplane[w * H + h] = tile[tx][ww];
    }
}

// x -> xT with 4-element vector accesses (H % 4 == 0 and W % 4 == 0): 256 threads per
// 32x32 tile, 16-byte row loads (8-byte for bf16) and 16-byte column stores through
// a padded shared tile.  bf16 values pass through fp32 unchanged (exact).
template <typename T>
__global__ void __launch_bounds__(256)
transpose_vec_kernel(const T *__restrict__ x, T *__restrict__ xT, int64_t H, int64_t W, int64_t tiles_w,
                     int64_t tiles_h) {
    __shared__ float tile[kTile][kTile + 1];
    int64_t blk = blockIdx.x;
    const int64_t tw = blk % tiles_w;
    blk /= tiles_w;
    const int64_t th = blk % tiles_h;
    const int64_t bd = blk / tiles_h;
    const int64_t L = H * W;
    const int64_t h0 = th * kTile, w0 = tw * kTile;
    const int t = threadIdx.x;
    {
        const int row = t >> 3, wq = t & 7;
        const int64_t h = h0 + row, w = w0 + 4 * wq;
        if (h < H && w < W) {
            float v[4];
            ld4(x + bd * L + h * W + w, v);
#pragma unroll
            for (int e = 0; e < 4; ++e) tile[row][4 * wq + e] = v[e];
        }
    }
    __syncthreads();
    {
        const int col = t >> 3, hq = t & 7;
        const int64_t w = w0 + col, h = h0 + 4 * hq;
        if (w < W && h < H) {
            float v[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) v[e] = tile[4 * hq + e][col];
            st4(xT + bd * L + w * H + h, v);
        }
    }
}

// CrossMerge with 4-element vector accesses, for H % 4 == 0 and W % 4 == 0 (then
// every 4-pixel run of a row or a column, and its mirror in a reversed path, is
// aligned).  256 threads per 32x32 tile; each thread handles 4 pixels.
template <typename Tin, typename Tout>
__global__ void __launch_bounds__(256)
cross_merge_vec_kernel(const Tin *__restrict__ ys, Tout *__restrict__ y, int64_t Dn, int64_t H, int64_t W,
                       int64_t tiles_w, int64_t tiles_h) {
    __shared__ float t13[kTile][kTile + 1];  // (t1 + t3) at [w - w0][h - h0]
    int64_t blk = blockIdx.x;
    const int64_t tw = blk % tiles_w;
    blk /= tiles_w;
    const int64_t th = blk % tiles_h;
    const int64_t bd = blk / tiles_h;
    const int64_t b = bd / Dn, d = bd - b * Dn;
    const int64_t L = H * W;
    const int64_t h0 = th * kTile, w0 = tw * kTile;
    const Tin *in0 = ys + ((b * kPaths + 0) * Dn + d) * L;
    const Tin *in1 = ys + ((b * kPaths + 1) * Dn + d) * L;
    const Tin *in2 = ys + ((b * kPaths + 2) * Dn + d) * L;
    const Tin *in3 = ys + ((b * kPaths + 3) * Dn + d) * L;
    const int t = threadIdx.x;
    {
        const int col = t >> 3, hq = t & 7;
        const int64_t w = w0 + col, h = h0 + 4 * hq;
        if (w < W && h < H) {
            const int64_t l = w * H + h;  // steps l..l+3 of the column path
            float v1[4], v3[4];
            ld4(in1 + l, v1);
            ld4(in3 + (L - 4 - l), v3);  // reversed: step l+e sits at L-1-l-e
#pragma unroll
            for (int e = 0; e < 4; ++e) t13[col][4 * hq + e] = v1[e] + v3[3 - e];
        }
    }
    __syncthreads();
    {
        const int row = t >> 3, wq = t & 7;
        const int64_t h = h0 + row, w = w0 + 4 * wq;
        if (h < H && w < W) {
            const int64_t p = h * W + w;
            float v0[4], v2[4], out[4];
            ld4(in0 + p, v0);
            ld4(in2 + (L - 4 - p), v2);
#pragma unroll
            for (int e = 0; e < 4; ++e) out[e] = (v0[e] + v2[3 - e]) + t13[4 * wq + e][row];
            st4(y + bd * L + p, out);
        }
    }
}

// Small planes (L <= kSmallPlane): a tile would leave most threads idle, so a CTA
// handles whole planes instead.  Transpose: the CTA's planes are one contiguous
// block in both x and xT; it is staged in shared memory and written back in
// output order, so both global passes are fully coalesced.
constexpr int kSmallPlane = 1024;
constexpr int kSmallElems = 4096;  // elements staged per CTA

template <typename T>
__global__ void __launch_bounds__(256)
transpose_small_kernel(const T *__restrict__ x, T *__restrict__ xT, int64_t planes, int H, int W) {
    __shared__ T buf[kSmallElems];
    const int L = H * W;
    const int ppb = kSmallElems / L;
    const int64_t p0 = (int64_t)blockIdx.x * ppb;
    const int np = (int)min((int64_t)ppb, planes - p0);
    const int n = np * L;
    const T *src = x + p0 * L;
    T *dst = xT + p0 * L;
    for (int i = threadIdx.x; i < n; i += blockDim.x) buf[i] = src[i];
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const int q = i / L, m = i - q * L;  // output position m = w*H + h of plane q
        const int w = m / H, h = m - w * H;
        dst[i] = buf[q * L + h * W + w];
    }
}

// CrossMerge for small planes: one thread per output pixel; the four per-path
// planes of a (b, d) span at most 4 KB each, so the column-order gathers stay in cache.
template <typename Tin, typename Tout>
__global__ void __launch_bounds__(256)
cross_merge_small_kernel(const Tin *__restrict__ ys, Tout *__restrict__ y, int64_t Dn, int H, int W,
                         int64_t total) {
    const int64_t L = (int64_t)H * W;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t bd = e / L;
        const int p = (int)(e - bd * L);
        const int64_t b = bd / Dn, d = bd - b * Dn;
        const int h = p / W, w = p - h * W;
        const int64_t lc = (int64_t)w * H + h;
        const Tin *base = ys + (b * kPaths * Dn + d) * L;
        const int64_t stride = Dn * L;  // between paths
        const float t02 = ld(base + p) + ld(base + 2 * stride + (L - 1 - p));
        const float t13 = ld(base + stride + lc) + ld(base + 3 * stride + (L - 1 - lc));
        st(y + e, t02 + t13);
    }
}

cudaError_t launch_transpose(const LaunchShape &s, ss2d_dtype_t dt, const void *x, void *xT, cudaStream_t stream) {
    if (s.L <= kSmallPlane) {
        const int64_t planes = s.B * s.D;
        const int ppb = kSmallElems / (int)s.L;
        const unsigned grid = (unsigned)ceil_div(planes, ppb);
        if (dt == SS2D_F32)
            transpose_small_kernel<float><<<grid, 256, 0, stream>>>((const float *)x, (float *)xT, planes, (int)s.H,
                                                                    (int)s.W);
        else
            transpose_small_kernel<__nv_bfloat16><<<grid, 256, 0, stream>>>(
                (const __nv_bfloat16 *)x, (__nv_bfloat16 *)xT, planes, (int)s.H, (int)s.W);
        note_launch(stream);
        return cudaGetLastError();
    }
    int64_t tw, th;
    dim3 grid = tile_grid(s.B * s.D, s.H, s.W, &tw, &th);
    if ((s.H % 4) == 0 && (s.W % 4) == 0) {
        if (dt == SS2D_F32)
            transpose_vec_kernel<float><<<grid, 256, 0, stream>>>((const float *)x, (float *)xT, s.H, s.W, tw, th);
        else
            transpose_vec_kernel<__nv_bfloat16><<<grid, 256, 0, stream>>>((const __nv_bfloat16 *)x,
                                                                        (__nv_bfloat16 *)xT, s.H, s.W, tw, th);
        note_launch(stream);
        return cudaGetLastError();
    }
    dim3 block(kTile, kRows);
    if (dt == SS2D_F32)
        transpose_kernel<float><<<grid, block, 0, stream>>>((const float *)x, (float *)xT, s.H, s.W, tw, th);
    else
        transpose_kernel<__nv_bfloat16><<<grid, block, 0, stream>>>((const __nv_bfloat16 *)x,
                                                                    (__nv_bfloat16 *)xT, s.H, s.W, tw, th);
    note_launch(stream);
    return cudaGetLastError();
}

cudaError_t launch_cross_merge(const LaunchShape &s, ss2d_dtype_t din, ss2d_dtype_t dout, const void *ys,
                               void *y, cudaStream_t stream) {
    int64_t tw, th;
    dim3 grid = tile_grid(s.B * s.D, s.H, s.W, &tw, &th);
    dim3 block(kTile, kRows);
    const bool vec = (s.H % 4) == 0 && (s.W % 4) == 0;
    const bool small = s.L <= kSmallPlane && !vec;
    const int64_t total = s.B * s.D * s.L;
    const int64_t small_blocks = ceil_div(total, 256);
    const unsigned small_grid = (unsigned)(small_blocks < 148 * 32 ? small_blocks : 148 * 32);
#define SS2D_MERGE(TI, TO)                                                                                      \
    do {                                                                                                        \
        if (small)                                                                                              \
            cross_merge_small_kernel<TI, TO><<<small_grid, 256, 0, stream>>>((const TI *)ys, (TO *)y, s.D,       \
                                                                            (int)s.H, (int)s.W, total);         \
        else if (vec)                                                                                           \
            cross_merge_vec_kernel<TI, TO><<<grid, 256, 0, stream>>>((const TI *)ys, (TO *)y, s.D, s.H, s.W, tw, \
                                                                      th);                                      \
        else                                                                                                    \
            cross_merge_kernel<TI, TO><<<grid, block, 0, stream>>>((const TI *)ys, (TO *)y, s.D, s.H, s.W, tw,  \
                                                                    th);                                        \
    } while (0)
    if (din == SS2D_F32 && dout == SS2D_F32) SS2D_MERGE(float, float);
    else if (din == SS2D_F32) SS2D_MERGE(float, __nv_bfloat16);
    else if (dout == SS2D_F32) SS2D_MERGE(__nv_bfloat16, float);
    else SS2D_MERGE(__nv_bfloat16, __nv_bfloat16);
#undef SS2D_MERGE
    note_launch(stream);
    return cudaGetLastError();
}

}  // namespace ss2d
