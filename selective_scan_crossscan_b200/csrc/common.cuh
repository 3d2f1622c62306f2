// common.cuh -- device helpers shared by the SS2D kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ss2d {

constexpr int kPaths = 4;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// ------------------------------------------------------------- element I/O --

template <typename T>
struct Elem;

template <>
struct Elem<float> {
    static __device__ __forceinline__ float load(const float *p) { return *p; }
    static __device__ __forceinline__ void store(float *p, float v) { *p = v; }
};

template <>
struct Elem<__nv_bfloat16> {
    static __device__ __forceinline__ float load(const __nv_bfloat16 *p) { return __bfloat162float(*p); }
    static __device__ __forceinline__ void store(__nv_bfloat16 *p, float v) { *p = __float2bfloat16_rn(v); }
};

template <typename T>
__device__ __forceinline__ float ld(const T *p) { return Elem<T>::load(p); }
template <typename T>
__device__ __forceinline__ void st(T *p, float v) { Elem<T>::store(p, v); }

// ---------------------------------------------- 4-element vector I/O --
// (16-byte accesses for fp32, 8-byte for bf16; the address must be aligned to them)

__device__ __forceinline__ void ld4(const float *p, float v[4]) {
    const float4 q = *reinterpret_cast<const float4 *>(p);
    v[0] = q.x;
    v[1] = q.y;
    v[2] = q.z;
    v[3] = q.w;
}
__device__ __forceinline__ void ld4(const __nv_bfloat16 *p, float v[4]) {
    const uint2 q = *reinterpret_cast<const uint2 *>(p);
    v[0] = __uint_as_float(q.x << 16);
    v[1] = __uint_as_float(q.x & 0xffff0000u);
    v[2] = __uint_as_float(q.y << 16);
    v[3] = __uint_as_float(q.y & 0xffff0000u);
}
__device__ __forceinline__ void st4(float *p, const float v[4]) {
    *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
}
__device__ __forceinline__ void st4(__nv_bfloat16 *p, const float v[4]) {
    const __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]);
    const __nv_bfloat162 b = __floats2bfloat162_rn(v[2], v[3]);
    uint2 q;
    q.x = *reinterpret_cast<const uint32_t *>(&a);
    q.y = *reinterpret_cast<const uint32_t *>(&b);
    *reinterpret_cast<uint2 *>(p) = q;
}

// ------------------------------------------------------------- path maps --

// Pixel index h*W + w visited at step l of path k.  k=0 row-major, k=1
// column-major (l = w*H + h), k=2 / k=3 the same orders walked backwards
// (VMamba, "2D Selective Scan (SS2D) for visual data", Fig. 2).
__device__ __forceinline__ int64_t path_pixel(int k, int64_t l, int64_t H, int64_t W) {
    const int64_t L = H * W;
    const int64_t m = (k >= 2) ? (L - 1 - l) : l;
    if ((k & 1) == 0) return m;
    const int64_t w = m / H;
    const int64_t h = m - w * H;
    return h * W + w;
}

// ------------------------------------------------------------------ math --

// 2^x on the SFU (MUFU.EX2); flushes subnormal results to zero.
__device__ __forceinline__ float ex2_sfu(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// log2(x) on the SFU.
__device__ __forceinline__ float lg2_sfu(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// softplus(t) = log(1 + e^t) in fp32.
//  t > 20        : t (the neglected e^-t is below 2.1e-9);
//  e^t < 1/16    : log1p(e) by its alternating Taylor series to e^7/7
//                  (relative truncation error below e^7/8 < 6e-10);
//  otherwise     : log(1 + e) with 1 + e >= 1.0625, so lg2's absolute error
//                  of ~1e-7 stays a relative error of a few 1e-6.
__device__ __forceinline__ float softplus_f(float t) {
    if (t > 20.f) return t;
    const float e = ex2_sfu(t * kLog2e);
    if (e < 0.0625f) {
        float p = 1.f / 7.f;
        p = fmaf(p, -e, 1.f / 6.f);
        p = fmaf(p, -e, 1.f / 5.f);
        p = fmaf(p, -e, 1.f / 4.f);
        p = fmaf(p, -e, 1.f / 3.f);
        p = fmaf(p, -e, 1.f / 2.f);
        p = fmaf(p, -e, 1.f);
        return e * p;
    }
    return lg2_sfu(1.f + e) * kLn2;
}

// d softplus / dt = sigmoid(t)
__device__ __forceinline__ float sigmoid_f(float t) {
    return 1.f / (1.f + ex2_sfu(-t * kLog2e));
}

__host__ __device__ __forceinline__ int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

}  // namespace ss2d
