// Device helpers shared by the routed-scan kernels: element loads/stores for
// the two I/O types, the discretization functions and the gate.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace vscan {

constexpr unsigned FULL_MASK = 0xffffffffu;

// Bits of the caller's device status word (vscan_args.status), OR-ed in by the
// kernels instead of trapping.
constexpr int DEV_STATUS_VALUE = 1;    // a value check failed
constexpr int DEV_STATUS_TIMEOUT = 2;  // a pipeline wait gave up (the output is invalid)
constexpr float LOG2E = 1.4426950408889634f;

// ---- element I/O -----------------------------------------------------------
template <typename T>
__device__ __forceinline__ float load_elem(const T* p);

template <>
__device__ __forceinline__ float load_elem<float>(const float* p) { return __ldg(p); }

template <>
__device__ __forceinline__ float load_elem<__nv_bfloat16>(const __nv_bfloat16* p)
{
    return __bfloat162float(__ldg(p));
}

template <typename T>
__device__ __forceinline__ void store_elem(T* p, float v);

template <>
__device__ __forceinline__ void store_elem<float>(float* p, float v) { *p = v; }

template <>
__device__ __forceinline__ void store_elem<__nv_bfloat16>(__nv_bfloat16* p, float v)
{
    *p = __float2bfloat16_rn(v);
}

__device__ __forceinline__ float to_float(float v) { return v; }
__device__ __forceinline__ float to_float(__nv_bfloat16 v) { return __bfloat162float(v); }

// Four consecutive elements starting at a 4-element-aligned address.
template <typename T>
__device__ __forceinline__ float4 load4(const T* p);

template <>
__device__ __forceinline__ float4 load4<float>(const float* p)
{
    return __ldg(reinterpret_cast<const float4*>(p));
}

template <>
__device__ __forceinline__ float4 load4<__nv_bfloat16>(const __nv_bfloat16* p)
{
    const uint2 raw = __ldg(reinterpret_cast<const uint2*>(p));
    float4 r;
    r.x = __uint_as_float(raw.x << 16);
    r.y = __uint_as_float(raw.x & 0xffff0000u);
    r.z = __uint_as_float(raw.y << 16);
    r.w = __uint_as_float(raw.y & 0xffff0000u);
    return r;
}

template <typename T>
__device__ __forceinline__ void store4(T* p, float4 v);

template <>
__device__ __forceinline__ void store4<float>(float* p, float4 v)
{
    *reinterpret_cast<float4*>(p) = v;
}

template <>
__device__ __forceinline__ void store4<__nv_bfloat16>(__nv_bfloat16* p, float4 v)
{
    __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y);
    __nv_bfloat162 b = __floats2bfloat162_rn(v.z, v.w);
    uint2 raw;
    raw.x = *reinterpret_cast<uint32_t*>(&a);
    raw.y = *reinterpret_cast<uint32_t*>(&b);
    *reinterpret_cast<uint2*>(p) = raw;
}

// Optional steps of the scan, as kernel template flags: the zero-order-hold
// write term, the fused causal convolution of u, (pooled routes) a masked
// token set addressed by grid position, and (streaming kernel) saving the state
// at every chunk boundary for the backward pass.
enum ScanFlags : int { FL_ZOH = 1, FL_CONV = 2, FL_MASK = 4, FL_CKPT = 8 };

// ---- discretization ---------------------------------------------------------
// 2^x on the special-function unit (PTX ex2.approx.ftz.f32). The retention
// exp(Delta * A) is evaluated as 2^(Delta * A * log2 e), with A pre-scaled.
__device__ __forceinline__ float fast_exp2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// 2^x for a pair of x <= 0 on the FMA pipe instead of the SFU, so that a kernel
// bound by the SFU's 16 results per clock and SM can move part of its
// retentions to the 128-lane FP32 pipe. Range reduction of Cody and Waite
// ("Software Manual for the Elementary Functions", 1980): k = round(x) by the
// 1.5 * 2^23 shifter, f = x - k in [-1/2, 1/2], 2^f = 1 + f q(f) with q a
// degree-5 least-squares fit of (2^f - 1)/f made by fit_exp2.py (relative
// error 1e-7 in float32; 2^0 = 1 exactly), and 2^k added to the exponent
// field. x is clamped at -126, where 2^x is below every normal float (the SFU
// form flushes it to 0; this one returns 2^-126).
__device__ __forceinline__ float2 exp2_fma2(float2 x)
{
    x.x = fmaxf(x.x, -126.f);
    x.y = fmaxf(x.y, -126.f);
    const float2 j = __fadd2_rn(x, make_float2(12582912.f, 12582912.f));
    const float2 k = __fadd2_rn(j, make_float2(-12582912.f, -12582912.f));
    const float2 f = __ffma2_rn(k, make_float2(-1.f, -1.f), x);
    float2 q = make_float2(1.537070493e-04f, 1.537070493e-04f);
    q = __ffma2_rn(q, f, make_float2(1.339984825e-03f, 1.339984825e-03f));
    q = __ffma2_rn(q, f, make_float2(9.618373588e-03f, 9.618373588e-03f));
    q = __ffma2_rn(q, f, make_float2(5.550329015e-02f, 5.550329015e-02f));
    q = __ffma2_rn(q, f, make_float2(2.402264774e-01f, 2.402264774e-01f));
    q = __ffma2_rn(q, f, make_float2(6.931471825e-01f, 6.931471825e-01f));
    const float2 p = __ffma2_rn(q, f, make_float2(1.f, 1.f));
    // the low bits of j hold k (two's complement); k << 23 lands in the exponent
    return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(j.x) << 23)),
                       __int_as_float(__float_as_int(p.y) + (__float_as_int(j.y) << 23)));
}

__device__ __forceinline__ float fast_rcp(float x)
{
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

constexpr float LN2 = 0.69314718055994531f;

// softplus(x) = log(1 + e^x) ("Vision Mamba ...", sec. 3), evaluated as
//     max(x, 0) + ln 2 * t * P(t),   t = 2^(-|x| log2 e) in (0, 1],
// i.e. max(x, 0) + log(1 + e^-|x|) with log2(1 + t) = t * P(t). P is a degree-8
// least-squares fit of log2(1 + t) / t on [0, 1] made by fit_log2p1.py
// (relative error 1.4e-7 in float32). One SFU op.
__device__ __forceinline__ float softplus_f(float x)
{
    const float t = fast_exp2(-fabsf(x) * LOG2E);
    float p = 7.366087753e-03f;
    p = fmaf(p, t, -4.182628542e-02f);
    p = fmaf(p, t, 1.116363406e-01f);
    p = fmaf(p, t, -1.960704774e-01f);
    p = fmaf(p, t, 2.751406133e-01f);
    p = fmaf(p, t, -3.582780361e-01f);
    p = fmaf(p, t, 4.806761742e-01f);
    p = fmaf(p, t, -7.213394046e-01f);
    p = fmaf(p, t, 1.442695022e+00f);
    return fmaxf(x, 0.f) + LN2 * (t * p);
}

// softplus of a pair: softplus_f's operations, in the same order and rounding,
// with the polynomial on packed f32x2 instructions.
__device__ __forceinline__ float2 softplus2(float2 x)
{
    const float2 t = make_float2(fast_exp2(-fabsf(x.x) * LOG2E), fast_exp2(-fabsf(x.y) * LOG2E));
    float2 p = make_float2(7.366087753e-03f, 7.366087753e-03f);
    p = __ffma2_rn(p, t, make_float2(-4.182628542e-02f, -4.182628542e-02f));
    p = __ffma2_rn(p, t, make_float2(1.116363406e-01f, 1.116363406e-01f));
    p = __ffma2_rn(p, t, make_float2(-1.960704774e-01f, -1.960704774e-01f));
    p = __ffma2_rn(p, t, make_float2(2.751406133e-01f, 2.751406133e-01f));
    p = __ffma2_rn(p, t, make_float2(-3.582780361e-01f, -3.582780361e-01f));
    p = __ffma2_rn(p, t, make_float2(4.806761742e-01f, 4.806761742e-01f));
    p = __ffma2_rn(p, t, make_float2(-7.213394046e-01f, -7.213394046e-01f));
    p = __ffma2_rn(p, t, make_float2(1.442695022e+00f, 1.442695022e+00f));
    const float2 tp = __fmul2_rn(t, p);
    return make_float2(fmaxf(x.x, 0.f) + LN2 * tp.x, fmaxf(x.y, 0.f) + LN2 * tp.y);
}

// SiLU(z) = z * sigma(z) = z / (1 + e^-z), signed and unbounded ("Vision
// Mamba ...", sec. 5). Two SFU ops (2^x and the reciprocal); for z below about
// -88, e^-z overflows to +inf and the result is a signed zero.
__device__ __forceinline__ float silu_f(float z)
{
    return z * fast_rcp(1.0f + fast_exp2(-z * LOG2E));
}

// Zero-order-hold gain ("Norm or Direction? ...", Eq. 2): for the diagonal A of
// the scan, Bbar = (Delta A)^-1 (e^(Delta A) - 1) Delta B = phi(x) * Delta * B with
//     phi(x) = (e^x - 1) / x,   x = Delta * A.
// e = e^x is the retention the caller already has and rx = 1 / x. For |x| < 0.5
// phi is a degree-6 least-squares polynomial with phi(0) = 1 made by
// fit_expm1x.py (relative error 8e-8 in float32), which avoids the
// cancellation in e - 1; elsewhere (e - 1) * rx. x = 0 (A = 0 or Delta = 0)
// gives exactly 1, the Delta*B*u write.
__device__ __forceinline__ float zoh_phi(float x, float e, float rx)
{
    float q = 1.986203570e-04f;
    q = fmaf(q, x, 1.399721252e-03f);
    q = fmaf(q, x, 8.333531208e-03f);
    q = fmaf(q, x, 4.166532308e-02f);
    q = fmaf(q, x, 1.666666418e-01f);
    q = fmaf(q, x, 5.000000596e-01f);
    q = fmaf(q, x, 1.0f);
    return fabsf(x) < 0.5f ? q : (e - 1.0f) * rx;
}

}  // namespace vscan
