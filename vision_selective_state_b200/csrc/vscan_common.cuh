// Device helpers shared by the routed-scan kernels: element loads/stores for
// the two I/O types, the discretization functions and the gate.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace vscan {

constexpr unsigned FULL_MASK = 0xffffffffu;
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
