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
// 1 / x from the special-function unit (about 1 ulp; no IEEE special-case path)
__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

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

// softplus(t) = log(1 + e^t) = max(t, 0) + log1p(z), z = e^{-|t|} in (0, 1].
// One SFU exponential, then log1p(z) = z * q(z) with q a degree-7 polynomial
// fitted to log1p(z)/z on [0, 1] (Chebyshev least squares; fit_softplus_poly.py
// prints these coefficients): relative error of z*q(z) below 3.6e-7 in fp32.
// Branch-free, so lanes with different t never diverge.
constexpr float kL1pC0 = 0.99999981021784778f;
constexpr float kL1pC1 = -0.49997449384836073f;
constexpr float kL1pC2 = 0.33276176571522004f;
constexpr float kL1pC3 = -0.24499611724605175f;
constexpr float kL1pC4 = 0.17757023992469328f;
constexpr float kL1pC5 = -0.10785367917432163f;
constexpr float kL1pC6 = 0.04421419233997316f;
constexpr float kL1pC7 = -0.0085746762053331097f;

__device__ __forceinline__ float softplus_f(float t) {
    const float z = ex2_sfu(-fabsf(t) * kLog2e);
    float q = kL1pC7;
    q = fmaf(q, z, kL1pC6);
    q = fmaf(q, z, kL1pC5);
    q = fmaf(q, z, kL1pC4);
    q = fmaf(q, z, kL1pC3);
    q = fmaf(q, z, kL1pC2);
    q = fmaf(q, z, kL1pC1);
    q = fmaf(q, z, kL1pC0);
    return fmaxf(t, 0.f) + z * q;
}

// the same for two values at once on the packed fp32 pipe (sm_100 f32x2)
__device__ __forceinline__ float2 softplus_f2(float2 t) {
    const float2 z = make_float2(ex2_sfu(-fabsf(t.x) * kLog2e), ex2_sfu(-fabsf(t.y) * kLog2e));
    float2 q = make_float2(kL1pC7, kL1pC7);
    q = __ffma2_rn(q, z, make_float2(kL1pC6, kL1pC6));
    q = __ffma2_rn(q, z, make_float2(kL1pC5, kL1pC5));
    q = __ffma2_rn(q, z, make_float2(kL1pC4, kL1pC4));
    q = __ffma2_rn(q, z, make_float2(kL1pC3, kL1pC3));
    q = __ffma2_rn(q, z, make_float2(kL1pC2, kL1pC2));
    q = __ffma2_rn(q, z, make_float2(kL1pC1, kL1pC1));
    q = __ffma2_rn(q, z, make_float2(kL1pC0, kL1pC0));
    return __ffma2_rn(z, q, make_float2(fmaxf(t.x, 0.f), fmaxf(t.y, 0.f)));
}

// 2^x for two values on the FMA pipe (packed f32x2), to take exponentials off the
// SFU: Cody-Waite split x = j + f with j = rint(x) (magic-number rounding) and
// f in [-1/2, 1/2], 2^f by a degree-5 polynomial fitted to 2^f on [-1/2, 1/2]
// (Chebyshev least squares weighted for relative error; maximum relative error
// 2.2e-7 in fp32, about that of the SFU's approximation), then j added to the
// exponent field.  Arguments are clamped below at -125 (results under 2^-125
// are returned as ~2^-125 instead of flushing to zero: both are negligible
// against O(1) terms).
constexpr float kEx2C0 = 1.0000001192092896f;
constexpr float kEx2C1 = 0.6931469440460205f;
constexpr float kEx2C2 = 0.24022121727466583f;
constexpr float kEx2C3 = 0.05550742521882057f;
constexpr float kEx2C4 = 0.009675459936261177f;
constexpr float kEx2C5 = 0.0013266970636323094f;
constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23

__device__ __forceinline__ float2 ex2_poly2(float2 x) {
    x = make_float2(fmaxf(x.x, -125.f), fmaxf(x.y, -125.f));
    const float2 t = __fadd2_rn(x, make_float2(kRoundMagic, kRoundMagic));      // low bits hold rint(x)
    const float2 j = __fadd2_rn(t, make_float2(-kRoundMagic, -kRoundMagic));    // rint(x) as a float
    const float2 f = __ffma2_rn(j, make_float2(-1.f, -1.f), x);                  // x - rint(x), exact
    float2 q = make_float2(kEx2C5, kEx2C5);
    q = __ffma2_rn(q, f, make_float2(kEx2C4, kEx2C4));
    q = __ffma2_rn(q, f, make_float2(kEx2C3, kEx2C3));
    q = __ffma2_rn(q, f, make_float2(kEx2C2, kEx2C2));
    q = __ffma2_rn(q, f, make_float2(kEx2C1, kEx2C1));
    q = __ffma2_rn(q, f, make_float2(kEx2C0, kEx2C0));
    // t's bit pattern is 0x4B400000 + rint(x); shifted by 23 only rint(x) lands in the exponent field
    return make_float2(__int_as_float(__float_as_int(q.x) + (__float_as_int(t.x) << 23)),
                       __int_as_float(__float_as_int(q.y) + (__float_as_int(t.y) << 23)));
}

// sigmoid(t) = 1 / (1 + e^{-t}) (= d softplus / dt); for t -> -inf, e^{-t} -> inf and the result -> 0
__device__ __forceinline__ float sigmoid_f(float t) { return rcp_approx(1.f + ex2_sfu(-t * kLog2e)); }

// silu(z) = z * sigmoid(z), the output gate of the selective scan
__device__ __forceinline__ float silu_f(float z) { return z * sigmoid_f(z); }

__host__ __device__ __forceinline__ int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

}  // namespace ss2d
