// Opt-in value checks of the scan's inputs (VSCAN_FLAG_CHECK_VALUES).
//
// The scalar reference scan of "EfficientVMamba: Atrous Selective Scan for
// Light Weight Visual Mamba" (sec. 2, "Update an independent state inside each
// group") refuses non-finite inputs, an unstable state matrix (A > 0) and
// negative time scales. This kernel tests the same conditions on the device
// and records a failure by OR-ing DEV_STATUS_VALUE into a status word; it never
// traps, and the scan that follows runs regardless.
//   - every element of u, raw Delta, B, C, z, A, D, bias and the convolution
//     weights is finite;
//   - every A is <= 0;
//   - with softplus off, every time scale raw Delta + bias of every direction
//     that reads it is >= 0.
#pragma once

#include "vscan_common.cuh"

namespace vscan {

constexpr int CHECK_MAX_SEGS = 12;

// One array to check: ptr[0 .. n), in bf16 or float32.
struct CheckSeg {
    const void* ptr;
    long long n;
    int bf16;      // 1: bfloat16 elements, 0: float32
    int nonpos;    // 1: values must also be <= 0 (A)
    int vec;       // 1: ptr is 16-byte aligned and n a multiple of 16 bytes
};

struct CheckParams {
    CheckSeg seg[CHECK_MAX_SEGS];
    int nseg;
    int* status;
    // softplus off: Delta = raw + bias >= 0 (segment index dseg is raw Delta)
    int dt_check;
    const void* delta;
    int delta_bf16;
    const float* bias;   // [Kp][D] or nullptr (bias 0)
    long long plane;     // elements of one raw-Delta plane (batch * tokens * D)
    int D, Ki, Kp;
};

__device__ __forceinline__ bool finite_bits(uint32_t f32bits) { return (f32bits & 0x7f800000u) != 0x7f800000u; }

__device__ __forceinline__ bool elem_ok(float v, int nonpos)
{
    return finite_bits(__float_as_uint(v)) && (!nonpos || v <= 0.f);
}

// blockIdx.y: segment (or, for the last row when dt_check, the time-scale test).
__global__ void __launch_bounds__(256) check_values_kernel(const CheckParams p)
{
    const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long nthr = (long long)gridDim.x * blockDim.x;
    bool bad = false;
    if ((int)blockIdx.y < p.nseg) {
        const CheckSeg sg = p.seg[blockIdx.y];
        if (sg.vec) {
            const long long nv = sg.n / (sg.bf16 ? 8 : 4);
            const uint4* v = static_cast<const uint4*>(sg.ptr);
            for (long long i = tid; i < nv; i += nthr) {
                const uint4 w = __ldg(v + i);
                const uint32_t q[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    if (sg.bf16) {
                        bad |= !elem_ok(__uint_as_float(q[e] << 16), sg.nonpos);
                        bad |= !elem_ok(__uint_as_float(q[e] & 0xffff0000u), sg.nonpos);
                    } else {
                        bad |= !elem_ok(__uint_as_float(q[e]), sg.nonpos);
                    }
                }
            }
        } else {
            for (long long i = tid; i < sg.n; i += nthr) {
                const float x = sg.bf16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(sg.ptr)[i])
                                        : static_cast<const float*>(sg.ptr)[i];
                bad |= !elem_ok(x, sg.nonpos);
            }
        }
    } else if (p.dt_check) {
        const long long n = p.plane * p.Ki;
        for (long long i = tid; i < n; i += nthr) {
            const int kin = (int)(i / p.plane);
            const int d = (int)(i % p.D);
            const float raw = p.delta_bf16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(p.delta)[i])
                                           : static_cast<const float*>(p.delta)[i];
            // per-direction inputs: plane k meets bias plane k (or the shared one);
            // shared inputs meet every direction's bias
            const int k0 = (p.Ki > 1) ? (p.Kp > 1 ? kin : 0) : 0;
            const int k1 = (p.Ki > 1) ? k0 + 1 : p.Kp;
            for (int kk = k0; kk < k1; ++kk) {
                const float bsum = raw + (p.bias ? __ldg(p.bias + (long long)kk * p.D + d) : 0.f);
                bad |= !(bsum >= 0.f);
            }
        }
    }
    if (__any_sync(FULL_MASK, bad) && (threadIdx.x & 31) == 0) atomicOr(p.status, DEV_STATUS_VALUE);
}

}  // namespace vscan
