// Streaming routed selective scan: BIDIR, CROSS4 and ATROUS2 routes.
//
// Work decomposition. One CTA covers one image b and a tile of 8 channels for
// all K directions of the route: warp k runs direction k. Inside a warp,
// lane = 4*c + g owns channel c of the tile and the four states 4g..4g+3, so the
// N = 16 states of a channel sit on 4 adjacent lanes and the read-out sum over
// n is a 4-lane reduction. Each warp walks its direction's sequence in chunks
// of 16 steps: the chunk's route tokens are gathered from HBM into registers
// one chunk ahead (channels-last rows, so every gathered token is a contiguous
// channel segment), then discretized once per (token, channel) into shared
// memory, then consumed by the recurrence.
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

constexpr int ST_TOK = 16;  // steps per staged chunk
constexpr int ST_CH = 8;    // channels per warp

struct __align__(16) StreamStage {
    float4 B[ST_TOK][4];        // B[t][4q..4q+3]
    float4 C[ST_TOK][4];
    float dsp[ST_TOK][ST_CH];   // Delta after bias + softplus
    float du[ST_TOK][ST_CH];    // Delta * u
    float uu[ST_TOK][ST_CH];    // u (skip term)
    int pos[ST_TOK];            // token index, -1 pad, -2 past the end
};

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
    extern __shared__ __align__(16) unsigned char smem_raw[];
    StreamStage* stages = reinterpret_cast<StreamStage*>(smem_raw);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int k = warp;
    StreamStage& st = stages[warp];

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

    // Staging role: channel ce of the tile, steps (lane >> 3) + 4i.
    const int ce = lane & 7;
    const int ds = c0 + ce;
    const bool svalid = ds < D;
    const float bias_s = (svalid && p.bias) ? __ldg(p.bias + k * p.v_dir + ds) : 0.f;

    const long long img = (long long)b * tokens;
    const T* u_base = static_cast<const T*>(p.u) + k * p.in_dir + img * D;
    const T* d_base = static_cast<const T*>(p.delta) + k * p.in_dir + img * D;
    const T* B_base = static_cast<const T*>(p.B) + k * p.bc_dir + img * N;
    const T* C_base = static_cast<const T*>(p.C) + k * p.bc_dir + img * N;
    const T* z_base = p.z ? static_cast<const T*>(p.z) + img * D : nullptr;
    T* y_base = static_cast<T*>(p.y) + img * D;

    float h[4] = {0.f, 0.f, 0.f, 0.f};

    // Registers holding the next chunk while the current one is computed.
    float ru[4], rd[4];
    float rb[8], rc[8];
    int rpos = -2;

    auto load_chunk = [&](int chunk) {
        const int t = chunk * ST_TOK + (lane & 15);
        rpos = (t < L) ? route_token<RK>(p.g, k, t) : -2;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int j = (lane >> 3) + 4 * i;
            const int pj = __shfl_sync(FULL_MASK, rpos, j);
            if (pj >= 0 && svalid) {
                ru[i] = load_elem<T>(u_base + (long long)pj * D + ds);
                rd[i] = load_elem<T>(d_base + (long long)pj * D + ds);
            } else {
                ru[i] = 0.f;
                rd[i] = 0.f;
            }
        }
        if (N16) {
            if (sizeof(T) == 4) {
                // 16 steps x 4 float4 per tensor: lane takes (step f>>2, quad f&3), f = lane + 32i
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const int f = lane + 32 * i;
                    const int pj = __shfl_sync(FULL_MASK, rpos, f >> 2);
                    float4 vb = make_float4(0.f, 0.f, 0.f, 0.f), vc = vb;
                    if (pj >= 0) {
                        vb = load4<T>(B_base + (long long)pj * 16 + 4 * (f & 3));
                        vc = load4<T>(C_base + (long long)pj * 16 + 4 * (f & 3));
                    }
                    rb[4 * i + 0] = vb.x; rb[4 * i + 1] = vb.y; rb[4 * i + 2] = vb.z; rb[4 * i + 3] = vb.w;
                    rc[4 * i + 0] = vc.x; rc[4 * i + 1] = vc.y; rc[4 * i + 2] = vc.z; rc[4 * i + 3] = vc.w;
                }
            } else {
                // 16 steps x 2 halves of 8 bf16: lane takes (step lane>>1, half lane&1)
                const int pj = __shfl_sync(FULL_MASK, rpos, lane >> 1);
                float4 b0 = make_float4(0.f, 0.f, 0.f, 0.f), b1 = b0, q0 = b0, q1 = b0;
                if (pj >= 0) {
                    const T* pb = B_base + (long long)pj * 16 + 8 * (lane & 1);
                    const T* pc = C_base + (long long)pj * 16 + 8 * (lane & 1);
                    b0 = load4<T>(pb); b1 = load4<T>(pb + 4);
                    q0 = load4<T>(pc); q1 = load4<T>(pc + 4);
                }
                rb[0] = b0.x; rb[1] = b0.y; rb[2] = b0.z; rb[3] = b0.w;
                rb[4] = b1.x; rb[5] = b1.y; rb[6] = b1.z; rb[7] = b1.w;
                rc[0] = q0.x; rc[1] = q0.y; rc[2] = q0.z; rc[3] = q0.w;
                rc[4] = q1.x; rc[5] = q1.y; rc[6] = q1.z; rc[7] = q1.w;
            }
        } else {
            // Any N <= 16: 16 steps x 16 state slots, lane takes slot e = lane + 32i.
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int e = lane + 32 * i;
                const int n = e & 15;
                const int pj = __shfl_sync(FULL_MASK, rpos, e >> 4);
                float vb = 0.f, vc = 0.f;
                if (pj >= 0 && n < N) {
                    vb = load_elem<T>(B_base + (long long)pj * N + n);
                    vc = load_elem<T>(C_base + (long long)pj * N + n);
                }
                rb[i] = vb;
                rc[i] = vc;
            }
        }
    };

    auto commit_chunk = [&]() {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int j = (lane >> 3) + 4 * i;
            const int pj = __shfl_sync(FULL_MASK, rpos, j);
            const float x = rd[i] + bias_s;
            float dsp = p.softplus ? softplus_f(x) : x;
            float uu = ru[i];
            if (pj == -2 || !svalid) {  // past the end: a no-op step
                dsp = 0.f;
                uu = 0.f;
            }
            st.dsp[j][ce] = dsp;
            st.du[j][ce] = dsp * uu;
            st.uu[j][ce] = uu;
        }
        if (N16) {
            if (sizeof(T) == 4) {
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const int f = lane + 32 * i;
                    st.B[f >> 2][f & 3] = make_float4(rb[4 * i], rb[4 * i + 1], rb[4 * i + 2], rb[4 * i + 3]);
                    st.C[f >> 2][f & 3] = make_float4(rc[4 * i], rc[4 * i + 1], rc[4 * i + 2], rc[4 * i + 3]);
                }
            } else {
                const int j = lane >> 1, q = 2 * (lane & 1);
                st.B[j][q] = make_float4(rb[0], rb[1], rb[2], rb[3]);
                st.B[j][q + 1] = make_float4(rb[4], rb[5], rb[6], rb[7]);
                st.C[j][q] = make_float4(rc[0], rc[1], rc[2], rc[3]);
                st.C[j][q + 1] = make_float4(rc[4], rc[5], rc[6], rc[7]);
            }
        } else {
            float* sb = reinterpret_cast<float*>(&st.B[0][0]);
            float* sc = reinterpret_cast<float*>(&st.C[0][0]);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int e = lane + 32 * i;
                sb[e] = rb[i];
                sc[e] = rc[i];
            }
        }
        if (lane < 16) st.pos[lane] = rpos;
    };

    const int nchunks = (L + ST_TOK - 1) / ST_TOK;
    load_chunk(0);
    commit_chunk();
    __syncwarp();

    for (int chunk = 0; chunk < nchunks; ++chunk) {
        const bool more = chunk + 1 < nchunks;
        if (more) load_chunk(chunk + 1);

        // ---- recurrence over the 16 staged steps -----------------------------
        float yv[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            float yp[4];
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                const int j = 4 * q + jj;
                const float dsp = st.dsp[j][cc];
                const float du = st.du[j][cc];
                const float4 Bv = st.B[j][grp];
                const float4 Cv = st.C[j][grp];
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
            yv[q] = fmaf(Dd, st.uu[4 * q + grp][cc], keep);
        }

        // ---- merge, gate and store --------------------------------------------
        if (!MERGE) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int pj = st.pos[4 * q + grp];
                if (pj >= 0 && dvalid) {
                    float o = yv[q] * p.merge_scale;
                    if (z_base) o *= silu_f(load_elem<T>(z_base + (long long)pj * D + d));
                    store_elem<T>(y_base + (long long)pj * D + d, o);
                }
            }
        } else {
            bool mine[4];
            int pos4[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int pj = st.pos[4 * q + grp];
                pos4[q] = pj;
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
                    const int pj = pos4[q];
                    float acc = yv[q];
#pragma unroll
                    for (int kk = 0; kk < K; ++kk) {
                        if (kk == k) continue;
                        acc += p.scratch[(((long long)kk * p.batch + b) * tokens + pj) * D + d];
                    }
                    float o = acc * p.merge_scale;
                    if (z_base) o *= silu_f(load_elem<T>(z_base + (long long)pj * D + d));
                    store_elem<T>(y_base + (long long)pj * D + d, o);
                }
            }
        }

        __syncwarp();
        if (more) commit_chunk();
        __syncwarp();
    }
}

}  // namespace vscan
