// Launch parameters of the forward scan kernels and the 16-byte cp.async
// helpers they share (streaming, pipelined and resident kernels; the backward
// scan uses the copies).
#pragma once

#include "vscan_route.cuh"

namespace vscan {

struct ScanParams {
    RouteGeom g;
    int batch, D, N;
    const void* u;
    const void* delta;
    const void* B;
    const void* C;
    const void* z;
    void* y;
    const float* A;
    const float* Dskip;
    const float* bias;
    long long in_dir;  // elements between directions of u / delta (0: shared)
    long long bc_dir;  // elements between directions of B / C (0: shared)
    int a_dir;         // elements between directions of A (0 or D*N)
    int v_dir;         // elements between directions of Dskip / bias (0 or D)
    int softplus;
    float merge_scale;
    int k_base;        // first direction of this launch (direction = k_base + blockIdx.z*KC + local)
    float* scratch;    // PARK: [K][batch][tokens][D] float32
    const float* conv_w;  // FL_CONV: [Kp][D][4]
    const float* conv_b;  // FL_CONV: [Kp][D] (nullable)
    float* ckpt;          // nullable: [K][batch][ceil(L/16)][D][16], the state entering every
                          // 16-step chunk (saved for the backward pass)
    int* status;          // nullable device word: bits DEV_STATUS_* OR-ed in by the kernels
};

// ---- cp.async (16-byte, L2 only) ------------------------------------------------
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, bool valid)
{
    const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    const int n = valid ? 16 : 0;  // 0: fill the 16 bytes with zeros, read nothing
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem), "r"(n));
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }

template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

}  // namespace vscan
