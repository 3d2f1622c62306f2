// bidir.cu -- the sum of the two directions of the bidirectional scan.
//
// bimamba_inner_ref ("vision mamba-yolov8", section "2. Vmamba module code") adds
// the forward scan's output and the reverse scan's output flipped back.  The scan
// kernels store the reverse direction at its natural positions already, so the
// merge is an elementwise sum of the two (B, 2, D, L) fp32 halves in a fixed order,
// times silu(z) when the scan is gated (both directions are gated by the same z
// at the same position, so gating the sum is the same), rounded once.  The
// backward uses the same kernel, ungated, for dx, ddelta and dz.
#include "common.cuh"
#include "kernels.h"

namespace ss2d {

// out[b, d, m] = round((two[b, 0, d, m] + two[b, 1, d, m]) * (GATE ? silu(z[b, d, m]) : 1))
template <typename Tz, typename Tout, bool GATE, bool VEC>
__global__ void bidir_sum_kernel(const float *__restrict__ two, const Tz *__restrict__ z, Tout *__restrict__ out,
                                 int64_t B, int64_t DL) {
    const int64_t total = B * DL;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x * (VEC ? 4 : 1);
    for (int64_t e = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * (VEC ? 4 : 1); e < total; e += stride) {
        const int64_t b = e / DL, r = e - b * DL;
        const float *t0 = two + b * 2 * DL + r;
        const float *t1 = t0 + DL;
        if (VEC) {  // DL % 4 == 0: four elements of one row
            float a[4], c[4], v[4];
            ld4(t0, a);
            ld4(t1, c);
            float zv[4];
            if (GATE) ld4(z + e, zv);
#pragma unroll
            for (int j = 0; j < 4; ++j) v[j] = GATE ? (a[j] + c[j]) * silu_f(zv[j]) : a[j] + c[j];
            st4(out + e, v);
        } else {
            const float v = *t0 + *t1;
            st(out + e, GATE ? v * silu_f(ld(z + e)) : v);
        }
    }
}

template <typename Tz, typename Tout, bool GATE>
static cudaError_t launch_sum_t(const float *two, const void *z, void *out, int64_t B, int64_t DL,
                                cudaStream_t stream) {
    const bool vec = DL % 4 == 0;
    const int threads = 256;
    const int64_t items = vec ? B * DL / 4 : B * DL;
    const int64_t want = ceil_div(items, threads);
    const int blocks = (int)(want < 148 * 16 ? (want > 0 ? want : 1) : 148 * 16);
    if (vec)
        bidir_sum_kernel<Tz, Tout, GATE, true><<<blocks, threads, 0, stream>>>(
            two, static_cast<const Tz *>(z), static_cast<Tout *>(out), B, DL);
    else
        bidir_sum_kernel<Tz, Tout, GATE, false><<<blocks, threads, 0, stream>>>(
            two, static_cast<const Tz *>(z), static_cast<Tout *>(out), B, DL);
    note_launch(stream);
    return cudaGetLastError();
}

cudaError_t launch_bidir_sum(const float *two, const void *z, ss2d_dtype_t z_dtype, void *out,
                             ss2d_dtype_t out_dtype, int64_t B, int64_t D, int64_t L, cudaStream_t stream) {
    const int64_t DL = D * L;
    using bf = __nv_bfloat16;
    if (!z) {
        if (out_dtype == SS2D_F32) return launch_sum_t<float, float, false>(two, z, out, B, DL, stream);
        return launch_sum_t<float, bf, false>(two, z, out, B, DL, stream);
    }
    if (z_dtype == SS2D_F32) {
        if (out_dtype == SS2D_F32) return launch_sum_t<float, float, true>(two, z, out, B, DL, stream);
        return launch_sum_t<float, bf, true>(two, z, out, B, DL, stream);
    }
    if (out_dtype == SS2D_F32) return launch_sum_t<bf, float, true>(two, z, out, B, DL, stream);
    return launch_sum_t<bf, bf, true>(two, z, out, B, DL, stream);
}

}  // namespace ss2d
