// Streaming routed selective scan: BIDIR, CROSS4 and ATROUS2 routes.
//
// Work decomposition. One CTA covers one image b and a tile of 8 channels for
// all K directions of the route: warp k runs direction k. Inside a warp,
// lane = 4*c + g owns channel c of the tile and the four states 4g..4g+3, so the
// N = 16 states of a channel sit on 4 adjacent lanes and the read-out sum over
// n is a 4-lane reduction.
//
// Data movement. Each warp walks its direction's sequence in chunks of 16
// steps. For every chunk it gathers the route's tokens with cp.async straight
// into a shared-memory stage: the 8-channel segments of u, raw Delta and z
// (channels-last rows, so every gathered token is one contiguous 16- or
// 32-byte piece) and the B and C rows, with zero fill for ATROUS2 padding.
// NSTAGE chunks are in flight, so the gather latency is hidden behind the
// recurrence of the chunks before it. Once a stage lands, the warp discretizes
// it once per (step, channel) and runs the recurrence:
//
// Per step and state ("Vision Mamba ...", sec. 4; "EfficientVMamba", sec. 2):
//     dA = 2^(Delta * A * log2 e)          (one SFU op)
//     h  = dA * h + (Delta * u) * B        (FMUL + FFMA)
//     y += C * h                           (FFMA)
//
// Merge. ATROUS2 gives every pixel one owner ("EfficientVMamba", sec. 3), so
// each direction gates and stores its own outputs. BIDIR and CROSS4 add the
// K aligned outputs of every token ("Vision Mamba ...", sec. 5; SS2D): the
// direction that visits a token in the latest 16-step chunk (ties: larger k)
// is its finalizer. Every other direction parks its contribution in the fp32
// workspace; after the CTA barrier that closes the chunk, the finalizer adds
// the parked values to its own, scales, gates with SiLU(z) and stores. All
// directions of a token live in the same CTA, so no atomics and no second pass
// over y are needed.
#pragma once

#include "vscan_common.cuh"
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
    float* scratch;    // merge routes: [K][batch][tokens][D] float32
};

constexpr int ST_TOK = 16;   // steps per chunk
constexpr int ST_CH = 8;     // channels per warp
constexpr int NSTAGE = 4;    // chunks in flight per warp

// ---- cp.async (sm_80+ form, 16- and 4-byte) ------------------------------------
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, bool valid)
{
    const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    const int n = valid ? 16 : 0;  // 0: fill the 16 bytes with zeros, read nothing
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem), "r"(n));
}

__device__ __forceinline__ void cp_async4(void* smem, const void* gmem, bool valid)
{
    const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    const int n = valid ? 4 : 0;
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(s), "l"(gmem), "r"(n));
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }

template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

// Raw gathered chunk, in the I/O type.
template <typename T>
struct __align__(16) RawStage {
    T u[ST_TOK][ST_CH];
    T d[ST_TOK][ST_CH];
    T z[ST_TOK][ST_CH];
    T B[ST_TOK][16];
    T C[ST_TOK][16];
    int pos[ST_TOK];  // token index, -1 pad, -2 past the end
};

// Discretized chunk (float32), written once per chunk by the warp.
struct __align__(16) PrepStage {
    float4 B[ST_TOK][4];
    float4 C[ST_TOK][4];
    float dsp[ST_TOK][ST_CH];  // Delta after bias + softplus
    float du[ST_TOK][ST_CH];   // Delta * u
    float uu[ST_TOK][ST_CH];   // u (skip term)
};

template <typename T>
struct WarpSmem {
    RawStage<T> raw[NSTAGE];
    PrepStage prep;
};

template <typename T>
constexpr size_t stream_smem_bytes(int K) { return K * sizeof(WarpSmem<T>); }

// Direction that adds up token p: the one visiting p in the latest chunk.
template <int RK>
__device__ __forceinline__ int finalizer(const RouteGeom& g, int p)
{
    int best_k = 0;
    int best_c = visit_step<RK>(g, 0, p) / ST_TOK;
#pragma unroll
    for (int kk = 1; kk < (RK == RK_CROSS4 ? 4 : 2); ++kk) {
        const int c = visit_step<RK>(g, kk, p) / ST_TOK;
        if (c >= best_c) {
            best_c = c;
            best_k = kk;
        }
    }
    return best_k;
}

template <int RK, typename T, bool N16>
__global__ void __launch_bounds__(128) stream_scan_kernel(const ScanParams p)
{
    constexpr bool MERGE = (RK == RK_BIDIR || RK == RK_CROSS4);
    constexpr int K = (RK == RK_BIDIR) ? 2 : 4;
    constexpr bool F32 = sizeof(T) == 4;
    extern __shared__ __align__(16) unsigned char smem_raw[];

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int k = warp;
    WarpSmem<T>& sm = reinterpret_cast<WarpSmem<T>*>(smem_raw)[warp];
    PrepStage& pr = sm.prep;

    const int b = blockIdx.y;
    const int c0 = blockIdx.x * ST_CH;
    const int D = p.D, N = p.N, L = p.g.L, tokens = p.g.tokens;

    // Compute role: channel cc, states 4*grp .. 4*grp+3.
    const int cc = lane >> 2, grp = lane & 3;
    const int d = c0 + cc;
    const bool dvalid = d < D;
    float a2[4];
#pragma unroll
    for (int s = 0; s < 4; ++s) {
        const int n = 4 * grp + s;
        a2[s] = (dvalid && n < N) ? __ldg(p.A + (long long)k * p.a_dir + (long long)d * N + n) * LOG2E : 0.f;
    }
    const float Dd = (dvalid && p.Dskip) ? __ldg(p.Dskip + k * p.v_dir + d) : 0.f;

    // Prep role: channel ce of the tile, steps (lane >> 3) + 4i.
    const int ce = lane & 7;
    const bool evalid = c0 + ce < D;
    const float bias_e = (evalid && p.bias) ? __ldg(p.bias + k * p.v_dir + c0 + ce) : 0.f;

    const long long img = (long long)b * tokens;
    const T* u_base = static_cast<const T*>(p.u) + k * p.in_dir + img * D + c0;
    const T* d_base = static_cast<const T*>(p.delta) + k * p.in_dir + img * D + c0;
    const T* z_base = p.z ? static_cast<const T*>(p.z) + img * D + c0 : nullptr;
    const T* B_base = static_cast<const T*>(p.B) + k * p.bc_dir + img * N;
    const T* C_base = static_cast<const T*>(p.C) + k * p.bc_dir + img * N;
    T* y_base = static_cast<T*>(p.y) + img * D;

    // Gather one chunk into raw stage s. Every lane issues the same number of
    // cp.async operations and one commit, so group counting stays uniform.
    auto issue = [&](int chunk, int s) {
        RawStage<T>& st = sm.raw[s];
        const int t = chunk * ST_TOK + (lane & 15);
        const int mypos = (t < L) ? route_token<RK>(p.g, k, t) : -2;
        if (lane < 16) st.pos[lane] = mypos;
        if (F32) {
            // u, Delta, z: 16 steps x 32 bytes; lane -> (step lane>>1, 4-channel half lane&1)
            const int j = lane >> 1, hf = lane & 1;
            const int pj = __shfl_sync(FULL_MASK, mypos, j);
            const bool ok = pj >= 0 && (c0 + 4 * hf) < D;
            const long long off = (long long)(ok ? pj : 0) * D + 4 * hf;
            cp_async16(&st.u[j][4 * hf], u_base + off, ok);
            cp_async16(&st.d[j][4 * hf], d_base + off, ok);
            if (z_base) cp_async16(&st.z[j][4 * hf], z_base + off, ok);
        } else {
            // 16 steps x 16 bytes: lanes 0-15 take u (and z), lanes 16-31 take Delta
            const int j = lane & 15;
            const int pj = __shfl_sync(FULL_MASK, mypos, j);
            const bool ok = pj >= 0;
            const long long off = (long long)(ok ? pj : 0) * D;
            if (lane < 16) {
                cp_async16(&st.u[j][0], u_base + off, ok);
                if (z_base) cp_async16(&st.z[j][0], z_base + off, ok);
            } else {
                cp_async16(&st.d[j][0], d_base + off, ok);
            }
        }
        if (N16) {
            if (F32) {
                // 16 steps x 4 quads x 16 bytes per tensor: f = lane + 32i -> (step f>>2, quad f&3)
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const int f = lane + 32 * i;
                    const int pj = __shfl_sync(FULL_MASK, mypos, f >> 2);
                    const bool ok = pj >= 0;
                    const long long off = (long long)(ok ? pj : 0) * 16 + 4 * (f & 3);
                    cp_async16(&st.B[f >> 2][4 * (f & 3)], B_base + off, ok);
                    cp_async16(&st.C[f >> 2][4 * (f & 3)], C_base + off, ok);
                }
            } else {
                // 16 steps x 2 halves x 16 bytes: lane -> (step lane>>1, half lane&1)
                const int j = lane >> 1, hf = lane & 1;
                const int pj = __shfl_sync(FULL_MASK, mypos, j);
                const bool ok = pj >= 0;
                const long long off = (long long)(ok ? pj : 0) * 16 + 8 * hf;
                cp_async16(&st.B[j][8 * hf], B_base + off, ok);
                cp_async16(&st.C[j][8 * hf], C_base + off, ok);
            }
        } else {
            // Any N <= 16: element loads (the 16-byte path needs 16-float rows).
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int e = lane + 32 * i;
                const int n = e & 15, j = e >> 4;
                const int pj = __shfl_sync(FULL_MASK, mypos, j);
                T vb = T(0.f), vc = T(0.f);
                if (pj >= 0 && n < N) {
                    vb = B_base[(long long)pj * N + n];
                    vc = C_base[(long long)pj * N + n];
                }
                st.B[j][n] = vb;
                st.C[j][n] = vc;
            }
        }
        cp_async_commit();
    };

    // Discretize a landed raw stage into the prep buffers (once per step and channel).
    auto prepare = [&](const RawStage<T>& st) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int j = (lane >> 3) + 4 * i;
            const int pj = st.pos[j];
            float uu = to_float(st.u[j][ce]);
            const float x = to_float(st.d[j][ce]) + bias_e;
            float dsp = p.softplus ? softplus_f(x) : x;
            if (pj == -2 || !evalid) {  // past the end: a no-op step
                dsp = 0.f;
                uu = 0.f;
            }
            pr.dsp[j][ce] = dsp;
            pr.du[j][ce] = dsp * uu;
            pr.uu[j][ce] = uu;
        }
        // B and C to float32: 16 steps x 16 states each, lane -> 8 values per tensor
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int f = lane + 32 * i;  // (step f>>2, quad f&3)
            const int j = f >> 2, q = f & 3;
            pr.B[j][q] = make_float4(to_float(st.B[j][4 * q]), to_float(st.B[j][4 * q + 1]),
                                     to_float(st.B[j][4 * q + 2]), to_float(st.B[j][4 * q + 3]));
            pr.C[j][q] = make_float4(to_float(st.C[j][4 * q]), to_float(st.C[j][4 * q + 1]),
                                     to_float(st.C[j][4 * q + 2]), to_float(st.C[j][4 * q + 3]));
        }
    };

    float h[4] = {0.f, 0.f, 0.f, 0.f};
    const int nchunks = (L + ST_TOK - 1) / ST_TOK;

#pragma unroll
    for (int s = 0; s < NSTAGE - 1; ++s) {
        if (s < nchunks) issue(s, s);
        else cp_async_commit();
    }

    for (int chunk = 0; chunk < nchunks; ++chunk) {
        const int ahead = chunk + NSTAGE - 1;
        if (ahead < nchunks) issue(ahead, ahead % NSTAGE);
        else cp_async_commit();
        cp_async_wait<NSTAGE - 1>();
        __syncwarp();
        const RawStage<T>& st = sm.raw[chunk % NSTAGE];
        prepare(st);
        __syncwarp();

        // ---- recurrence over the 16 steps ----------------------------------------
        float yv[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            float yp[4];
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                const int j = 4 * q + jj;
                const float dsp = pr.dsp[j][cc];
                const float du = pr.du[j][cc];
                const float4 Bv = pr.B[j][grp];
                const float4 Cv = pr.C[j][grp];
                const float e0 = fast_exp2(dsp * a2[0]);
                const float e1 = fast_exp2(dsp * a2[1]);
                const float e2 = fast_exp2(dsp * a2[2]);
                const float e3 = fast_exp2(dsp * a2[3]);
                h[0] = fmaf(e0, h[0], du * Bv.x);
                h[1] = fmaf(e1, h[1], du * Bv.y);
                h[2] = fmaf(e2, h[2], du * Bv.z);
                h[3] = fmaf(e3, h[3], du * Bv.w);
                float acc = Cv.x * h[0];
                acc = fmaf(Cv.y, h[1], acc);
                acc = fmaf(Cv.z, h[2], acc);
                acc = fmaf(Cv.w, h[3], acc);
                yp[jj] = acc;
            }
            // Reduce-scatter over the 4 state-group lanes: lane grp keeps step 4q+grp.
            const bool hi = grp & 2;
            float a0 = hi ? yp[2] : yp[0];
            float a1 = hi ? yp[3] : yp[1];
            const float s0 = hi ? yp[0] : yp[2];
            const float s1 = hi ? yp[1] : yp[3];
            a0 += __shfl_xor_sync(FULL_MASK, s0, 2);
            a1 += __shfl_xor_sync(FULL_MASK, s1, 2);
            const bool odd = grp & 1;
            float keep = odd ? a1 : a0;
            const float send = odd ? a0 : a1;
            keep += __shfl_xor_sync(FULL_MASK, send, 1);
            yv[q] = fmaf(Dd, pr.uu[4 * q + grp][cc], keep);
        }

        // ---- merge, gate and store ------------------------------------------------
        if (!MERGE) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int j = 4 * q + grp;
                const int pj = st.pos[j];
                if (pj >= 0 && dvalid) {
                    float o = yv[q] * p.merge_scale;
                    if (z_base) o *= silu_f(to_float(st.z[j][cc]));
                    store_elem<T>(y_base + (long long)pj * D + d, o);
                }
            }
        } else {
            bool mine[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int pj = st.pos[4 * q + grp];
                mine[q] = false;
                if (pj >= 0 && dvalid) {
                    if (finalizer<RK>(p.g, pj) == k) {
                        mine[q] = true;
                    } else {
                        p.scratch[(((long long)k * p.batch + b) * tokens + pj) * D + d] = yv[q];
                    }
                }
            }
            __syncthreads();
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                if (mine[q]) {
                    const int j = 4 * q + grp;
                    const int pj = st.pos[j];
                    float acc = yv[q];
#pragma unroll
                    for (int kk = 0; kk < K; ++kk) {
                        if (kk == k) continue;
                        acc += p.scratch[(((long long)kk * p.batch + b) * tokens + pj) * D + d];
                    }
                    float o = acc * p.merge_scale;
                    if (z_base) o *= silu_f(to_float(st.z[j][cc]));
                    store_elem<T>(y_base + (long long)pj * D + d, o);
                }
            }
        }
        __syncwarp();
    }
    cp_async_wait<0>();
}

}  // namespace vscan
