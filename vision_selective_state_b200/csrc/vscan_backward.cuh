// Backward pass of the routed selective scan (gradients of vscan_forward).
//
// Reverse-mode differentiation of the forward steps ("Vision Mamba ...",
// sec. 3-5; "EfficientVMamba ...", sec. 1-3; "Fast Vision Mamba ...",
// Methodology), for the released Delta*B*u write term. With x = Delta and
// a = exp(x A), the recurrence h_t = a_t h_{t-1} + x_t B_t u_t, y_t = C_t.h_t +
// D u_t has the adjoint g_t = dL/dh_t = C_t dy_t + a_{t+1} g_{t+1}, and
//     dC_t = dy_t h_t,   dB_t = g_t x_t u_t,   du_t = D dy_t + sum_n g_t x_t B_t,
//     dx_t = sum_n g_t (A a_t h_{t-1} + B_t u_t),   dA += g_t x_t a_t h_{t-1},
//     dD += dy_t u_t,    draw_t = dx_t sigmoid(raw_t + bias).
//
// Kernels (launched by vscan_backward):
//   gate_grad_kernel     dz and the gradient gy of the merged pre-gate value
//                        (merge scale folded in), from dy, z and the pre-gate
//                        forward output.
//   bwd_pool_kernel      pooled routes: means of u, raw Delta, B, C and sums of
//                        gy over each pooled index, so the scan below runs on the
//                        pooled sequence exactly as the forward does.
//   bwd_scan_kernel      one warp per (channel tile of 8, image, direction);
//                        lane 4c + g holds channel c, states 4g..4g+3. Pass 1
//                        runs the recurrence forward and saves the state at
//                        every 16-step chunk boundary; pass 2 walks the chunks
//                        backwards, recomputes the chunk's states from its
//                        checkpoint and runs the adjoint recurrence. Token
//                        gradients are summed over channels (B, C: one shuffle
//                        reduce-scatter per step) or state groups (u, Delta:
//                        shuffles) and added with float atomics (directions,
//                        channel tiles and images meet there); dA, D and bias
//                        gradients stay in registers until the end.
//   bwd_scan_split_kernel  the same with each tile's 16 states split over a CTA
//                        of two warps, for grids with few warps per SM.
//   bwd_unpool_kernel    pooled routes: every member token receives its pooled
//                        index's gradient divided by the member count.
#pragma once

#include "vscan_common.cuh"
#include "vscan_route.cuh"
#include "vscan_params.cuh"

namespace vscan {

struct BwdParams {
    RouteGeom g;       // route of the scan (pooled routes: BIDIR over the Lp pooled steps)
    int batch, D, N;
    const void* u;     // [Ki][batch][tokens][D] (TI)
    const void* delta; // [Ki][batch][tokens][D] raw step (TI)
    const void* B;     // [Ki][batch][tokens][N] (TI)
    const void* C;     // [Ki][batch][tokens][N] (TI)
    long long in_dir, bc_dir;
    int a_dir, v_dir;
    const float* A;
    const float* Dskip;
    const float* bias;
    int softplus;
    const float* gy;   // [batch][tokens][D]: dL / d(merged pre-gate value)
    float* ckpt;       // [K][batch][nchunks][D][16]
    int ckpt_ready;    // 1: the forward pass already saved the checkpoints (skip pass 1)
    float* du;         // [Ki][batch][tokens][D]
    float* ddelta;     // [Ki][batch][tokens][D]
    float* dB;         // [Ki][batch][tokens][N]
    float* dC;         // [Ki][batch][tokens][N]
    float* dA;         // [Kp][D][N]
    float* dD;         // [Kp][D]
    float* dbias;      // [Kp][D]
};

constexpr int BW_TOK = 16;  // steps per chunk
constexpr int BW_CH = 8;    // channels per warp

// d softplus(x) / dx = sigma(x) = 1 / (1 + e^-x), on the SFU (2^x and the
// reciprocal): 0 for x below about -88, where e^-x overflows, and 1 for large x.
__device__ __forceinline__ float sigmoid_f(float x) { return fast_rcp(1.0f + fast_exp2(-x * LOG2E)); }

// dz = dy * pre * sigmoid(z) * (1 + z (1 - sigmoid(z))) and gy = dy * s * SiLU(z),
// where pre = s * (merged scan output) is the forward output without the gate.
template <typename T>
__global__ void gate_grad_kernel(const T* __restrict__ dy, const T* __restrict__ z,
                                 const T* __restrict__ pre, float scale, long long n,
                                 float* __restrict__ gy, float* __restrict__ dz)
{
    for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n;
         e += (long long)gridDim.x * blockDim.x) {
        const float d = to_float(dy[e]);
        if (z) {
            const float zz = to_float(z[e]);
            const float sg = 1.0f / (1.0f + __expf(-zz));
            gy[e] = d * scale * zz * sg;
            if (dz) dz[e] = d * to_float(pre[e]) * sg * (1.0f + zz * (1.0f - sg));
        } else {
            gy[e] = d * scale;
        }
    }
}

// Pooled routes: pu, praw [Ki][batch][Lp][D] and pB, pC [Ki][batch][Lp][N] are
// the means over the members of each pooled index, pg [batch][Lp][D] the sum
// of gy over them. The gate's gradient is formed here, per member token (as
// gate_grad_kernel does for the grid routes), so gy never goes through HBM:
// gy = dy * s * SiLU(z) and dz = dy * pre * sigmoid(z) * (1 + z (1 - sigmoid(z))),
// pre the forward output without the gate. Grid (Lp, batch); threads stride over
// channels and states.
template <typename T>
__global__ void bwd_pool_kernel(RouteGeom g, int batch, int D, int N, int Ki, const T* u, const T* delta,
                                const T* B, const T* C, long long in_dir, long long bc_dir, const T* dy,
                                const T* z, const T* pre, float scale, float* dz, float* pu, float* praw,
                                float* pB, float* pC, float* pg)
{
    const int i = blockIdx.x, b = blockIdx.y, Lp = g.L;
    const int cnt = (g.kind == RK_POOL_W) ? g.w : g.h;
    const float inv = 1.0f / (float)cnt;
    const long long img = (long long)b * g.tokens;
    auto member = [&](int j) { return (long long)((g.kind == RK_POOL_W) ? i * g.w + j : j * g.w + i); };
    for (int k = 0; k < Ki; ++k) {
        for (int d = threadIdx.x; d < D; d += blockDim.x) {
            float su = 0.f, sr = 0.f, sg = 0.f;
            constexpr int U = 8;  // members per round, all loads issued before the sums
            for (int j0 = 0; j0 < cnt; j0 += U) {
                float vu[U], vr[U], vd[U], vz[U], vp[U];
#pragma unroll
                for (int v = 0; v < U; ++v) {
                    const bool in = j0 + v < cnt;
                    const long long o = (img + member(in ? j0 + v : 0)) * D + d;
                    vu[v] = in ? to_float(u[k * in_dir + o]) : 0.f;
                    vr[v] = in ? to_float(delta[k * in_dir + o]) : 0.f;
                    const bool gate = in && k == 0;
                    vd[v] = gate ? to_float(dy[o]) : 0.f;
                    vz[v] = (gate && z) ? to_float(z[o]) : 0.f;
                    vp[v] = (gate && z && dz) ? to_float(pre[o]) : 0.f;
                }
#pragma unroll
                for (int v = 0; v < U; ++v) {
                    su += vu[v];
                    sr += vr[v];
                    if (k == 0) {
                        if (z) {
                            const float sgm = 1.0f / (1.0f + __expf(-vz[v]));
                            sg += vd[v] * scale * vz[v] * sgm;
                            if (dz && j0 + v < cnt)
                                dz[(img + member(j0 + v)) * D + d] = vd[v] * vp[v] * sgm * (1.0f + vz[v] * (1.0f - sgm));
                        } else {
                            sg += vd[v] * scale;
                        }
                    }
                }
            }
            const long long po = (((long long)k * batch + b) * Lp + i) * D + d;
            pu[po] = su * inv;
            praw[po] = sr * inv;
            if (k == 0) pg[((long long)b * Lp + i) * D + d] = sg;
        }
        for (int n = threadIdx.x; n < N; n += blockDim.x) {
            float sb = 0.f, sc = 0.f;
            constexpr int U = 8;
            for (int j0 = 0; j0 < cnt; j0 += U) {
                float vb[U], vc[U];
#pragma unroll
                for (int v = 0; v < U; ++v) {
                    const bool in = j0 + v < cnt;
                    const long long o = (img + member(in ? j0 + v : 0)) * N + n;
                    vb[v] = in ? to_float(B[k * bc_dir + o]) : 0.f;
                    vc[v] = in ? to_float(C[k * bc_dir + o]) : 0.f;
                }
#pragma unroll
                for (int v = 0; v < U; ++v) {
                    sb += vb[v];
                    sc += vc[v];
                }
            }
            const long long po = (((long long)k * batch + b) * Lp + i) * N + n;
            pB[po] = sb * inv;
            pC[po] = sc * inv;
        }
    }
}

// Pooled routes: token gradients from the pooled ones (the mean's adjoint).
// Grid (x, batch), 8 warps per CTA: each warp writes whole token rows (u and
// raw Delta gradients in 16-byte pieces, D a multiple of 4), striding over the
// image's tokens, so the stores stream at full width.
__global__ void __launch_bounds__(256) bwd_unpool_kernel(RouteGeom g, int batch, int D, int N, int Ki,
                                                         const float* dpu, const float* dpraw, const float* dpB,
                                                         const float* dpC, float* du, float* ddelta, float* dB,
                                                         float* dC)
{
    const int b = blockIdx.y, Lp = g.L, lane = threadIdx.x & 31;
    const int nw = gridDim.x * (blockDim.x >> 5);
    const float inv = 1.0f / (float)((g.kind == RK_POOL_W) ? g.w : g.h);
    const int Q = D / 4;
    constexpr int U = 2;  // token rows per warp per round, loads first
    for (int t0 = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t0 < g.tokens; t0 += U * nw) {
        int tk[U], ix[U];
#pragma unroll
        for (int v = 0; v < U; ++v) {
            tk[v] = t0 + v * nw;
            const int r = tk[v] / g.w, c = tk[v] - r * g.w;
            ix[v] = tk[v] < g.tokens ? ((g.kind == RK_POOL_W) ? r : c) : -1;
        }
        for (int k = 0; k < Ki; ++k) {
            for (int q = lane; q < Q; q += 32) {
                float4 vu[U], vd[U];
#pragma unroll
                for (int v = 0; v < U; ++v) {
                    const long long po = (((long long)k * batch + b) * Lp + max(ix[v], 0)) * D + 4 * q;
                    vu[v] = du ? *reinterpret_cast<const float4*>(dpu + po) : make_float4(0.f, 0.f, 0.f, 0.f);
                    vd[v] = ddelta ? *reinterpret_cast<const float4*>(dpraw + po) : make_float4(0.f, 0.f, 0.f, 0.f);
                }
#pragma unroll
                for (int v = 0; v < U; ++v) {
                    if (ix[v] < 0) continue;
                    const long long to = (((long long)k * batch + b) * g.tokens + tk[v]) * D + 4 * q;
                    if (du) *reinterpret_cast<float4*>(du + to) = make_float4(vu[v].x * inv, vu[v].y * inv, vu[v].z * inv, vu[v].w * inv);
                    if (ddelta)
                        *reinterpret_cast<float4*>(ddelta + to) =
                            make_float4(vd[v].x * inv, vd[v].y * inv, vd[v].z * inv, vd[v].w * inv);
                }
            }
            if (lane < N) {
#pragma unroll
                for (int v = 0; v < U; ++v) {
                    if (ix[v] < 0) continue;
                    const long long to = ((long long)k * batch + b) * g.tokens + tk[v];
                    const long long po = ((long long)k * batch + b) * Lp + ix[v];
                    if (dB) dB[to * N + lane] = dpB[po * N + lane] * inv;
                    if (dC) dC[to * N + lane] = dpC[po * N + lane] * inv;
                }
            }
        }
    }
}

// Raw rows of one 16-step chunk as gathered by cp.async (ASYNC builds): the
// next chunk's rows land here while the current chunk's adjoint runs.
template <typename TI>
struct __align__(16) BwdRaw {
    TI d[BW_TOK][BW_CH];
    TI u[BW_TOK][BW_CH];
    float gy[BW_TOK][BW_CH];
    TI B[BW_TOK][16];
    TI C[BW_TOK][16];
    int pos[BW_TOK];
};

// One 16-step chunk of one direction, staged in shared memory (B and C rows are
// read as 16-byte quads).
struct __align__(16) BwdStage {
    int pos[BW_TOK];           // token, -1 pad, -2 past the end
    float x[BW_TOK][BW_CH];    // discretized step Delta
    float sig[BW_TOK][BW_CH];  // d Delta / d raw
    float u[BW_TOK][BW_CH];
    float gy[BW_TOK][BW_CH];
    float B[BW_TOK][16];
    float C[BW_TOK][16];
};

// Per-chunk gradient partials of bwd_scan_kernel, added to global memory after
// the chunk (dB and dC are summed over the channels with shuffles at every step).
struct BwdReduceUX {
    float u[BW_TOK][BW_CH];  // du per (step, channel), state groups already summed
    float x[BW_TOK][BW_CH];  // d raw Delta per (step, channel)
};

// Warps per SM the one-warp backward scan is compiled for: capped registers per
// thread and small shared memory (the kernel is latency-bound, so on large grids
// resident warps matter more than scheduling room).
constexpr int BW_MIN_WARPS = 16;

// ASYNC (d_state 16): pass 2 gathers chunk c - 1 with cp.async while the
// adjoint of chunk c runs, so a chunk's rows are waited for only once they have
// had a whole chunk of compute to arrive.
template <int RK, typename TI, bool ASYNC>
__global__ void __launch_bounds__(32, BW_MIN_WARPS) bwd_scan_kernel(const BwdParams p)
{
    __shared__ BwdStage st;
    __shared__ __align__(16) BwdReduceUX rd;
    __shared__ BwdRaw<TI> raw[ASYNC ? 2 : 1];
    const int lane = threadIdx.x;
    const int cc = lane >> 2, grp = lane & 3;
    const int c0 = blockIdx.x * BW_CH, b = blockIdx.y, k = blockIdx.z;
    const int D = p.D, N = p.N, L = p.g.L, tokens = p.g.tokens;
    const int d = c0 + cc;
    const bool dvalid = d < D;
    const int ki = p.in_dir ? k : 0;
    const long long img = (long long)b * tokens;
    const int nch = (L + BW_TOK - 1) / BW_TOK;
    // this lane's four states as two pairs (packed f32x2 arithmetic)
    float2 a2[2], An[2];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        const int n = 4 * grp + 2 * q;
        const float* Ar = p.A + (long long)k * p.a_dir + (long long)d * N + n;
        An[q] = make_float2((dvalid && n < N) ? __ldg(Ar) : 0.f, (dvalid && n + 1 < N) ? __ldg(Ar + 1) : 0.f);
        a2[q] = make_float2(An[q].x * LOG2E, An[q].y * LOG2E);
    }
    const float Dd = (dvalid && p.Dskip) ? __ldg(p.Dskip + k * p.v_dir + d) : 0.f;
    const float* gyb = p.gy + img * D;
    const TI* ub = static_cast<const TI*>(p.u) + ki * p.in_dir + img * D;
    const TI* rb = static_cast<const TI*>(p.delta) + ki * p.in_dir + img * D;
    const TI* Bb = static_cast<const TI*>(p.B) + ki * p.bc_dir + img * N;
    const TI* Cb = static_cast<const TI*>(p.C) + ki * p.bc_dir + img * N;
    float* ck = p.ckpt + (((long long)k * p.batch + b) * nch) * D * 16;

    // Stage chunk c: positions, Delta and its derivative, u, gy, B, C. Every
    // global load of the chunk is issued before any of them is used, so a chunk
    // costs one memory latency, not one per element.
    constexpr int NE = BW_TOK * BW_CH / 32;  // (step, channel) elements per lane: 4
    constexpr int NS = BW_TOK * 16 / 32;     // (step, state) elements per lane: 8
    // the channel of every staged (step, channel) element of a lane is lane % 8
    const float bias_l = (c0 + (lane % BW_CH) < D && p.bias) ? __ldg(p.bias + k * p.v_dir + c0 + (lane % BW_CH)) : 0.f;
    auto stage = [&](int c, bool with_grad) {
        __syncwarp();
        if (lane < BW_TOK) {
            const int t = c * BW_TOK + lane;
            st.pos[lane] = (t < L) ? route_token<RK>(p.g, k, t) : -2;
        }
        __syncwarp();
        float vr[NE], vu[NE], vg[NE], vb[NS], vc[NS];
#pragma unroll
        for (int r = 0; r < NE; ++r) {  // element e = lane + 32 r: step e / 8, channel e % 8 (= lane % 8)
            const int e = lane + 32 * r;
            const int j = e / BW_CH, dd = c0 + e % BW_CH;
            const int q = st.pos[j];
            const bool ok = q >= 0 && dd < D;
            vr[r] = ok ? to_float(rb[(long long)q * D + dd]) : 0.f;
            vu[r] = ok ? to_float(ub[(long long)q * D + dd]) : 0.f;
            vg[r] = (ok && with_grad) ? gyb[(long long)q * D + dd] : 0.f;
        }
#pragma unroll
        for (int r = 0; r < NS; ++r) {  // element e = lane + 32 r: step e / 16, state e % 16
            const int e = lane + 32 * r;
            const int j = e >> 4, n = e & 15;
            const int q = st.pos[j];
            const bool ok = q >= 0 && n < N;
            vb[r] = ok ? to_float(Bb[(long long)q * N + n]) : 0.f;
            vc[r] = ok ? to_float(Cb[(long long)q * N + n]) : 0.f;
        }
#pragma unroll
        for (int r = 0; r < NE; ++r) {
            const int e = lane + 32 * r;
            const int j = e / BW_CH, ch = e % BW_CH, dd = c0 + ch;
            const float xr = vr[r] + bias_l;
            float x = xr, sg = 1.f;
            if (p.softplus) {
                x = softplus_f(xr);
                sg = sigmoid_f(xr);
            }
            const bool live = st.pos[j] != -2 && dd < D;
            st.x[j][ch] = live ? x : 0.f;
            st.sig[j][ch] = sg;
            st.u[j][ch] = vu[r];
            st.gy[j][ch] = vg[r];
        }
#pragma unroll
        for (int r = 0; r < NS; ++r) {
            const int e = lane + 32 * r;
            st.B[e >> 4][e & 15] = vb[r];
            st.C[e >> 4][e & 15] = vc[r];
        }
        __syncwarp();
    };

    // ASYNC: gather chunk c's rows into raw[buf] (16-byte cp.async, zero fill for
    // padding, past-the-end steps and channels beyond D), one commit group.
    auto issue = [&](int c, int buf) {
        BwdRaw<TI>& rw = raw[buf];
        int q = -2;
        if (lane < BW_TOK) {
            const int t = c * BW_TOK + lane;
            q = (t < L) ? route_token<RK>(p.g, k, t) : -2;
            rw.pos[lane] = q;
        }
        constexpr int EL = 16 / (int)sizeof(TI);      // elements per 16-byte piece
        constexpr int PR = BW_CH / EL;                 // pieces per u / Delta row
        constexpr int PB = 16 / EL;                    // pieces per B / C row
        constexpr int NPC = BW_TOK * (2 * PR + 2 + 2 * PB);  // + gy rows of 2 pieces
#pragma unroll
        for (int it = 0; it < (NPC + 31) / 32; ++it) {
            const int f = lane + 32 * it;
            int tsr, row, pc;  // 0 Delta, 1 u (PR pieces), 2 gy (2), 3 B, 4 C (PB)
            if (f < 2 * BW_TOK * PR) {
                tsr = f / (BW_TOK * PR);
                const int r = f - tsr * BW_TOK * PR;
                row = r / PR;
                pc = r - row * PR;
            } else if (f < 2 * BW_TOK * PR + 2 * BW_TOK) {
                tsr = 2;
                const int r = f - 2 * BW_TOK * PR;
                row = r >> 1;
                pc = r & 1;
            } else {
                const int r = f - 2 * BW_TOK * PR - 2 * BW_TOK;
                tsr = 3 + r / (BW_TOK * PB);
                const int r2 = r - (tsr - 3) * BW_TOK * PB;
                row = r2 / PB;
                pc = r2 - row * PB;
            }
            const int qj = __shfl_sync(FULL_MASK, q, row & (BW_TOK - 1));
            if (f < NPC) {
                const long long tok = qj >= 0 ? qj : 0;
                if (tsr < 2) {
                    const bool ok = qj >= 0 && c0 + pc * EL < D;
                    const TI* src = (tsr == 0 ? rb : ub) + (ok ? tok * D + c0 + pc * EL : 0);
                    cp_async16(tsr == 0 ? &rw.d[row][pc * EL] : &rw.u[row][pc * EL], src, ok);
                } else if (tsr == 2) {
                    const bool ok = qj >= 0 && c0 + 4 * pc < D;
                    cp_async16(&rw.gy[row][4 * pc], gyb + (ok ? tok * D + c0 + 4 * pc : 0), ok);
                } else {
                    const bool ok = qj >= 0;
                    const TI* src = (tsr == 3 ? Bb : Cb) + (ok ? tok * 16 + pc * EL : 0);
                    cp_async16(tsr == 3 ? &rw.B[row][pc * EL] : &rw.C[row][pc * EL], src, ok);
                }
            }
        }
        cp_async_commit();
    };
    // ASYNC: wait for raw[buf] and discretize it into st (as stage() does).
    auto convert = [&](int buf) {
        cp_async_wait<0>();
        __syncwarp();
        const BwdRaw<TI>& rw = raw[buf];
        if (lane < BW_TOK) st.pos[lane] = rw.pos[lane];
#pragma unroll
        for (int r = 0; r < NE; ++r) {
            const int e = lane + 32 * r;
            const int j = e / BW_CH, ch = e % BW_CH, dd = c0 + ch;
            const float xr = to_float(rw.d[j][ch]) + bias_l;
            float x = xr, sg = 1.f;
            if (p.softplus) {
                x = softplus_f(xr);
                sg = sigmoid_f(xr);
            }
            const bool live = rw.pos[j] != -2 && dd < D;
            st.x[j][ch] = live ? x : 0.f;
            st.sig[j][ch] = sg;
            st.u[j][ch] = to_float(rw.u[j][ch]);
            st.gy[j][ch] = rw.gy[j][ch];
        }
#pragma unroll
        for (int r = 0; r < NS; ++r) {
            const int e = lane + 32 * r;
            st.B[e >> 4][e & 15] = to_float(rw.B[e >> 4][e & 15]);
            st.C[e >> 4][e & 15] = to_float(rw.C[e >> 4][e & 15]);
        }
        __syncwarp();
    };

    // ---- pass 1: forward recurrence, state saved at every chunk boundary --------
    // one step of the recurrence for a pair of states: h = 2^(x A log2 e) h + (x B) u
    auto step2 = [&](float2 hp, float x, float uu, float2 Bq, float2 a2q) {
        const float2 xx = make_float2(x, x);
        const float2 xa = __fmul2_rn(xx, a2q);
        const float2 e = make_float2(fast_exp2(xa.x), fast_exp2(xa.y));
        return __ffma2_rn(e, hp, __fmul2_rn(__fmul2_rn(xx, Bq), make_float2(uu, uu)));
    };
    float2 h[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
    for (int c = 0; c < (p.ckpt_ready ? 0 : nch); ++c) {
        if (dvalid) {
#pragma unroll
            for (int q = 0; q < 2; ++q)
                *reinterpret_cast<float2*>(&ck[((long long)c * D + d) * 16 + 4 * grp + 2 * q]) = h[q];
        }
        stage(c, false);
#pragma unroll 4
        for (int j = 0; j < BW_TOK; ++j) {
            const float x = st.x[j][cc], uu = st.u[j][cc];
            const float4 Bv = *reinterpret_cast<const float4*>(&st.B[j][4 * grp]);
            h[0] = step2(h[0], x, uu, make_float2(Bv.x, Bv.y), a2[0]);
            h[1] = step2(h[1], x, uu, make_float2(Bv.z, Bv.w), a2[1]);
        }
    }
    __syncwarp();

    // ---- pass 2: adjoint recurrence, chunks in reverse ------------------------------
    float2 gs[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
    float2 dAs[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
    float dDs = 0.f, dbs = 0.f;
    // dB and dC partials per (step, channel, state) of two steps: B at [slot][channel][16],
    // C BC_C floats further (16 words past a multiple of 32, so a half-warp reading
    // both tensors at one channel hits 32 distinct banks). They live in the raw
    // buffer the current chunk was converted from, which is idle until the chunk after
    // next is gathered into it.
    constexpr int BC_C = 2 * BW_CH * 16 + 16;
    static_assert((BC_C + 2 * BW_CH * 16) * sizeof(float) <= sizeof(BwdRaw<TI>), "partials fit a raw buffer");
    if constexpr (ASYNC) issue(nch - 1, 0);
    for (int c = nch - 1; c >= 0; --c) {
        float* bcs;
        if constexpr (ASYNC) {
            const int buf = (nch - 1 - c) & 1;
            convert(buf);
            if (c > 0) issue(c - 1, buf ^ 1);  // lands while this chunk's adjoint runs
            bcs = reinterpret_cast<float*>(&raw[buf]);
        } else {
            stage(c, true);
            bcs = reinterpret_cast<float*>(&raw[0]);
        }
        float2 hs[BW_TOK + 1][2];  // hs[0] = state entering the chunk, hs[j + 1] after step j
#pragma unroll
        for (int q = 0; q < 2; ++q)
            hs[0][q] = dvalid ? *reinterpret_cast<const float2*>(&ck[((long long)c * D + d) * 16 + 4 * grp + 2 * q])
                              : make_float2(0.f, 0.f);
#pragma unroll
        for (int j = 0; j < BW_TOK; ++j) {
            const float x = st.x[j][cc], uu = st.u[j][cc];
            const float4 Bv = *reinterpret_cast<const float4*>(&st.B[j][4 * grp]);
            hs[j + 1][0] = step2(hs[j][0], x, uu, make_float2(Bv.x, Bv.y), a2[0]);
            hs[j + 1][1] = step2(hs[j][1], x, uu, make_float2(Bv.z, Bv.w), a2[1]);
        }
#pragma unroll
        for (int j = BW_TOK - 1; j >= 0; --j) {
            const int q = st.pos[j];
            if (q == -2) continue;  // past the end of the sequence (uniform over the warp)
            const float x = st.x[j][cc], uu = st.u[j][cc], dy = st.gy[j][cc];
            const float2 xx = make_float2(x, x), uu2 = make_float2(uu, uu), dy2 = make_float2(dy, dy);
            const float4 Bv = *reinterpret_cast<const float4*>(&st.B[j][4 * grp]);
            const float4 Cv = *reinterpret_cast<const float4*>(&st.C[j][4 * grp]);
            const float2 Bp[2] = {make_float2(Bv.x, Bv.y), make_float2(Bv.z, Bv.w)};
            const float2 Cp[2] = {make_float2(Cv.x, Cv.y), make_float2(Cv.z, Cv.w)};
            float2 dut2 = make_float2(0.f, 0.f), dxt2 = make_float2(0.f, 0.f), dB2[2], dC2[2];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const float2 xa = __fmul2_rn(xx, a2[q]);
                const float2 a = make_float2(fast_exp2(xa.x), fast_exp2(xa.y));
                gs[q] = __ffma2_rn(Cp[q], dy2, gs[q]);                   // g += C dy
                dC2[q] = __fmul2_rn(dy2, hs[j + 1][q]);                  // dC = dy h
                const float2 gx = __fmul2_rn(gs[q], xx);
                dB2[q] = __fmul2_rn(gx, uu2);                             // dB = g x u
                dut2 = __ffma2_rn(gx, Bp[q], dut2);                       // du += g x B
                const float2 t = __ffma2_rn(__fmul2_rn(An[q], a), hs[j][q], __fmul2_rn(Bp[q], uu2));
                dxt2 = __ffma2_rn(gs[q], t, dxt2);                        // dx += g (A a h' + B u)
                dAs[q] = __ffma2_rn(__fmul2_rn(gx, a), hs[j][q], dAs[q]); // dA += g x a h'
                gs[q] = __fmul2_rn(gs[q], a);                             // carried to step j - 1
            }
            float dut = dut2.x + dut2.y, dxt = dxt2.x + dxt2.y;
            const float dBv[4] = {dB2[0].x, dB2[0].y, dB2[1].x, dB2[1].y};
            const float dCv[4] = {dC2[0].x, dC2[0].y, dC2[1].x, dC2[1].y};
            // sums over the four state groups of a channel (u, Delta)
            dut += __shfl_xor_sync(FULL_MASK, dut, 1);
            dut += __shfl_xor_sync(FULL_MASK, dut, 2);
            dxt += __shfl_xor_sync(FULL_MASK, dxt, 1);
            dxt += __shfl_xor_sync(FULL_MASK, dxt, 2);
            const float draw = dxt * st.sig[j][cc];
            if (grp == 0) {
                if (dvalid) {
                    dbs += draw;
                    dDs = fmaf(dy, uu, dDs);
                }
                rd.u[j][cc] = fmaf(Dd, dy, dut);
                rd.x[j][cc] = draw;
            }
            // dB and dC of steps j + 1 and j, summed over the 8 channels once both are in
            // (slot = step & 1; a step past the end is skipped, and so is every later one)
            *reinterpret_cast<float4*>(&bcs[((j & 1) * BW_CH + cc) * 16 + 4 * grp]) =
                make_float4(dBv[0], dBv[1], dBv[2], dBv[3]);
            *reinterpret_cast<float4*>(&bcs[BC_C + ((j & 1) * BW_CH + cc) * 16 + 4 * grp]) =
                make_float4(dCv[0], dCv[1], dCv[2], dCv[3]);
            if ((j & 1) == 0) {
                __syncwarp();
                // this lane's share: slot lane >> 4, states s_n and s_n + 1, tensor lane & 1
                const int s_sl = lane >> 4, s_n = 4 * ((lane >> 2) & 3) + 2 * ((lane >> 1) & 1);
                const bool s_tz = lane & 1;
                float* const s_dst = s_tz ? p.dC : p.dB;
                const float* src = bcs + (s_tz ? BC_C : 0) + s_sl * BW_CH * 16 + s_n;
                float2 acc = *reinterpret_cast<const float2*>(src);
#pragma unroll
                for (int ch = 1; ch < BW_CH; ++ch) acc = __fadd2_rn(acc, *reinterpret_cast<const float2*>(src + ch * 16));
                const int qs = st.pos[j + s_sl];
                if (qs >= 0 && s_dst) {
                    float* o = s_dst + ki * p.bc_dir + (img + qs) * N + s_n;
                    if (s_n < N) atomicAdd(o, acc.x);
                    if (s_n + 1 < N) atomicAdd(o + 1, acc.y);
                }
                __syncwarp();
            }
        }
        // add the chunk's token gradients: one atomic per (step, channel), every lane
        // taking its share
        __syncwarp();
#pragma unroll
        for (int r = 0; r < BW_TOK * BW_CH / 32; ++r) {
            const int e = lane + 32 * r;
            const int j = e / BW_CH, ch = e % BW_CH, dd = c0 + ch;
            const int q = st.pos[j];
            if (q < 0 || dd >= D) continue;
            const long long o = ki * p.in_dir + (img + q) * D + dd;
            if constexpr (RK == RK_ATROUS2) {
                // one owner per pixel and channel: no other warp writes this element
                if (p.du) p.du[o] = rd.u[j][ch];
                if (p.ddelta) p.ddelta[o] = rd.x[j][ch];
            } else {
                if (p.du) atomicAdd(p.du + o, rd.u[j][ch]);
                if (p.ddelta) atomicAdd(p.ddelta + o, rd.x[j][ch]);
            }
        }
        __syncwarp();
    }
    if (dvalid) {
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            const int n = 4 * grp + s;
            const float v = (s & 1) ? dAs[s >> 1].y : dAs[s >> 1].x;
            if (n < N && p.dA) atomicAdd(p.dA + (long long)k * p.a_dir + (long long)d * N + n, v);
        }
        if (grp == 0) {
            if (p.dD) atomicAdd(p.dD + k * p.v_dir + d, dDs);
            if (p.dbias) atomicAdd(p.dbias + k * p.v_dir + d, dbs);
        }
    }
}

// The adjoint scan with a tile's 16 states split over two warps, for grids that
// leave SMs short of warps with one warp per tile (at most 8 tiles per SM): a CTA of two warps covers one
// (8-channel tile, image, direction); warp h holds states 8h..8h+7, lane 4c + g
// channel c and the state pair 8h + 2g, 8h + 2g + 1. Each warp's per-step chain is
// one state pair instead of two, and twice as many warps share the SMs. The
// chunk's rows are staged once for both warps. The du and dDelta partials of the
// two state halves meet in shared memory after the chunk; dB and dC are summed
// over the 8 channels inside each warp (4 shuffles per step), so the atomics per
// step equal the one-warp kernel's.
constexpr int BWS_THREADS = 64;
constexpr int BWS_MIN_BLOCKS = 12;  // 24 warps per SM: at most 85 registers per thread

struct __align__(16) BwdSplitPart {
    float u[2][BW_TOK][BW_CH];  // du partial of each state half, per (step, channel)
    float x[2][BW_TOK][BW_CH];  // dDelta partial likewise
};

template <int RK, typename TI, bool ASYNC>
__global__ void __launch_bounds__(BWS_THREADS, BWS_MIN_BLOCKS) bwd_scan_split_kernel(const BwdParams p)
{
    __shared__ BwdStage st;
    __shared__ BwdSplitPart part;
    __shared__ BwdRaw<TI> raw[ASYNC ? 2 : 1];
    const int tid = threadIdx.x, h = tid >> 5, lane = tid & 31;
    const int cc = lane >> 2, grp = lane & 3;
    const int n0 = 8 * h + 2 * grp;  // this lane's state pair
    const int c0 = blockIdx.x * BW_CH, b = blockIdx.y, k = blockIdx.z;
    const int D = p.D, N = p.N, L = p.g.L, tokens = p.g.tokens;
    const int d = c0 + cc;
    const bool dvalid = d < D;
    const int ki = p.in_dir ? k : 0;
    const long long img = (long long)b * tokens;
    const int nch = (L + BW_TOK - 1) / BW_TOK;
    float2 An, a2;
    {
        const float* Ar = p.A + (long long)k * p.a_dir + (long long)d * N + n0;
        An = make_float2((dvalid && n0 < N) ? __ldg(Ar) : 0.f, (dvalid && n0 + 1 < N) ? __ldg(Ar + 1) : 0.f);
        a2 = make_float2(An.x * LOG2E, An.y * LOG2E);
    }
    // (step, channel) items of the staging and of the after-chunk sums: e = tid + 64 r,
    // step e / 8, channel e % 8 = tid % 8 for every r
    const int ce = tid & (BW_CH - 1);
    const bool cev = c0 + ce < D;
    const float Dd_e = (cev && p.Dskip) ? __ldg(p.Dskip + k * p.v_dir + c0 + ce) : 0.f;
    const float bias_e = (cev && p.bias) ? __ldg(p.bias + k * p.v_dir + c0 + ce) : 0.f;
    const float* gyb = p.gy + img * D;
    const TI* ub = static_cast<const TI*>(p.u) + ki * p.in_dir + img * D;
    const TI* rb = static_cast<const TI*>(p.delta) + ki * p.in_dir + img * D;
    const TI* Bb = static_cast<const TI*>(p.B) + ki * p.bc_dir + img * N;
    const TI* Cb = static_cast<const TI*>(p.C) + ki * p.bc_dir + img * N;
    float* ck = p.ckpt + (((long long)k * p.batch + b) * nch) * D * 16;
    constexpr int NE = BW_TOK * BW_CH / BWS_THREADS;  // (step, channel) items per thread: 2
    constexpr int NS = BW_TOK * 16 / BWS_THREADS;     // (step, state) items per thread: 4

    // discretized step (0 past the end and beyond D) and its derivative of one
    // (step, channel) item
    auto disc = [&](float raw_d, bool live, float& x, float& sg) {
        const float xr = raw_d + bias_e;
        x = xr;
        sg = 1.f;
        if (p.softplus) {
            x = softplus_f(xr);
            sg = sigmoid_f(xr);
        }
        if (!live) x = 0.f;
    };

    // Stage chunk c with plain loads, every load of a thread issued before any use.
    auto stage = [&](int c, bool with_grad) {
        __syncthreads();  // every thread is done with st and part
        if (tid < BW_TOK) {
            const int t = c * BW_TOK + tid;
            st.pos[tid] = (t < L) ? route_token<RK>(p.g, k, t) : -2;
        }
        __syncthreads();
        float vr[NE], vu[NE], vg[NE], vb[NS], vc[NS];
#pragma unroll
        for (int r = 0; r < NE; ++r) {
            const int j = (tid + BWS_THREADS * r) / BW_CH, dd = c0 + ce;
            const int q = st.pos[j];
            const bool ok = q >= 0 && dd < D;
            vr[r] = ok ? to_float(rb[(long long)q * D + dd]) : 0.f;
            vu[r] = ok ? to_float(ub[(long long)q * D + dd]) : 0.f;
            vg[r] = (ok && with_grad) ? gyb[(long long)q * D + dd] : 0.f;
        }
#pragma unroll
        for (int r = 0; r < NS; ++r) {
            const int e = tid + BWS_THREADS * r;
            const int j = e >> 4, n = e & 15;
            const int q = st.pos[j];
            const bool ok = q >= 0 && n < N;
            vb[r] = ok ? to_float(Bb[(long long)q * N + n]) : 0.f;
            vc[r] = ok ? to_float(Cb[(long long)q * N + n]) : 0.f;
        }
#pragma unroll
        for (int r = 0; r < NE; ++r) {
            const int j = (tid + BWS_THREADS * r) / BW_CH;
            float x, sg;
            disc(vr[r], st.pos[j] != -2 && cev, x, sg);
            st.x[j][ce] = x;
            st.sig[j][ce] = sg;
            st.u[j][ce] = vu[r];
            st.gy[j][ce] = vg[r];
        }
#pragma unroll
        for (int r = 0; r < NS; ++r) {
            const int e = tid + BWS_THREADS * r;
            st.B[e >> 4][e & 15] = vb[r];
            st.C[e >> 4][e & 15] = vc[r];
        }
        __syncthreads();
    };

    // ASYNC: gather chunk c's rows into raw[buf] (16-byte cp.async, zero fill for
    // padding, past-the-end steps and channels beyond D), one commit group per thread.
    auto issue = [&](int c, int buf) {
        BwdRaw<TI>& rw = raw[buf];
        int q = -2;
        if (lane < BW_TOK) {  // both warps compute the chunk's positions for their shuffles
            const int t = c * BW_TOK + lane;
            q = (t < L) ? route_token<RK>(p.g, k, t) : -2;
            if (h == 0) rw.pos[lane] = q;
        }
        constexpr int EL = 16 / (int)sizeof(TI);             // elements per 16-byte piece
        constexpr int PR = BW_CH / EL;                        // pieces per u / Delta row
        constexpr int PB = 16 / EL;                           // pieces per B / C row
        constexpr int NPC = BW_TOK * (2 * PR + 2 + 2 * PB);   // + gy rows of 2 pieces
#pragma unroll
        for (int it = 0; it < (NPC + BWS_THREADS - 1) / BWS_THREADS; ++it) {
            const int f = tid + BWS_THREADS * it;
            int tsr, row, pc;  // 0 Delta, 1 u (PR pieces), 2 gy (2), 3 B, 4 C (PB)
            if (f < 2 * BW_TOK * PR) {
                tsr = f / (BW_TOK * PR);
                const int r = f - tsr * BW_TOK * PR;
                row = r / PR;
                pc = r - row * PR;
            } else if (f < 2 * BW_TOK * PR + 2 * BW_TOK) {
                tsr = 2;
                const int r = f - 2 * BW_TOK * PR;
                row = r >> 1;
                pc = r & 1;
            } else {
                const int r = f - 2 * BW_TOK * PR - 2 * BW_TOK;
                tsr = 3 + r / (BW_TOK * PB);
                const int r2 = r - (tsr - 3) * BW_TOK * PB;
                row = r2 / PB;
                pc = r2 - row * PB;
            }
            const int qj = __shfl_sync(FULL_MASK, q, row & (BW_TOK - 1));
            if (f < NPC) {
                const long long tok = qj >= 0 ? qj : 0;
                if (tsr < 2) {
                    const bool ok = qj >= 0 && c0 + pc * EL < D;
                    const TI* src = (tsr == 0 ? rb : ub) + (ok ? tok * D + c0 + pc * EL : 0);
                    cp_async16(tsr == 0 ? &rw.d[row][pc * EL] : &rw.u[row][pc * EL], src, ok);
                } else if (tsr == 2) {
                    const bool ok = qj >= 0 && c0 + 4 * pc < D;
                    cp_async16(&rw.gy[row][4 * pc], gyb + (ok ? tok * D + c0 + 4 * pc : 0), ok);
                } else {
                    const bool ok = qj >= 0;
                    const TI* src = (tsr == 3 ? Bb : Cb) + (ok ? tok * 16 + pc * EL : 0);
                    cp_async16(tsr == 3 ? &rw.B[row][pc * EL] : &rw.C[row][pc * EL], src, ok);
                }
            }
        }
        cp_async_commit();
    };
    // ASYNC: wait for raw[buf] and discretize it into st.
    auto convert = [&](int buf) {
        cp_async_wait<0>();
        __syncthreads();  // all copies of raw[buf] landed; every thread is done with st and part
        const BwdRaw<TI>& rw = raw[buf];
        if (tid < BW_TOK) st.pos[tid] = rw.pos[tid];
#pragma unroll
        for (int r = 0; r < NE; ++r) {
            const int j = (tid + BWS_THREADS * r) / BW_CH;
            float x, sg;
            disc(to_float(rw.d[j][ce]), rw.pos[j] != -2 && cev, x, sg);
            st.x[j][ce] = x;
            st.sig[j][ce] = sg;
            st.u[j][ce] = to_float(rw.u[j][ce]);
            st.gy[j][ce] = rw.gy[j][ce];
        }
#pragma unroll
        for (int r = 0; r < NS; ++r) {
            const int e = tid + BWS_THREADS * r;
            st.B[e >> 4][e & 15] = to_float(rw.B[e >> 4][e & 15]);
            st.C[e >> 4][e & 15] = to_float(rw.C[e >> 4][e & 15]);
        }
        __syncthreads();
    };

    // one step of the recurrence for the lane's pair: h = 2^(x A log2 e) h + (x B) u
    auto step2 = [&](float2 hp, float x, float uu, float2 Bq) {
        const float2 xx = make_float2(x, x);
        const float2 xa = __fmul2_rn(xx, a2);
        const float2 e = make_float2(fast_exp2(xa.x), fast_exp2(xa.y));
        return __ffma2_rn(e, hp, __fmul2_rn(__fmul2_rn(xx, Bq), make_float2(uu, uu)));
    };

    // ---- pass 1: forward recurrence, state saved at every chunk boundary --------
    float2 hh = make_float2(0.f, 0.f);
    for (int c = 0; c < (p.ckpt_ready ? 0 : nch); ++c) {
        if (dvalid) *reinterpret_cast<float2*>(&ck[((long long)c * D + d) * 16 + n0]) = hh;
        stage(c, false);
#pragma unroll 4
        for (int j = 0; j < BW_TOK; ++j)
            hh = step2(hh, st.x[j][cc], st.u[j][cc], *reinterpret_cast<const float2*>(&st.B[j][n0]));
    }

    // ---- pass 2: adjoint recurrence, chunks in reverse ------------------------------
    float2 gs = make_float2(0.f, 0.f), dAs = make_float2(0.f, 0.f);
    float dDs = 0.f, dbs = 0.f;  // channel ce, summed over this thread's items
    const bool b4 = cc & 4, b2 = cc & 2, b1 = cc & 1;
    if constexpr (ASYNC) issue(nch - 1, 0);
    for (int c = nch - 1; c >= 0; --c) {
        if constexpr (ASYNC) {
            const int buf = (nch - 1 - c) & 1;
            convert(buf);
            if (c > 0) issue(c - 1, buf ^ 1);  // lands while this chunk's adjoint runs
        } else {
            stage(c, true);
        }
        float2 hs[BW_TOK + 1];  // hs[0] = state entering the chunk, hs[j + 1] after step j
        hs[0] = dvalid ? *reinterpret_cast<const float2*>(&ck[((long long)c * D + d) * 16 + n0]) : make_float2(0.f, 0.f);
#pragma unroll
        for (int j = 0; j < BW_TOK; ++j)
            hs[j + 1] = step2(hs[j], st.x[j][cc], st.u[j][cc], *reinterpret_cast<const float2*>(&st.B[j][n0]));
#pragma unroll
        for (int j = BW_TOK - 1; j >= 0; --j) {
            const int q = st.pos[j];
            if (q == -2) continue;  // past the end of the sequence (uniform over the CTA)
            const float x = st.x[j][cc], uu = st.u[j][cc], dy = st.gy[j][cc];
            const float2 xx = make_float2(x, x), uu2 = make_float2(uu, uu), dy2 = make_float2(dy, dy);
            const float2 Bp = *reinterpret_cast<const float2*>(&st.B[j][n0]);
            const float2 Cp = *reinterpret_cast<const float2*>(&st.C[j][n0]);
            const float2 xa = __fmul2_rn(xx, a2);
            const float2 a = make_float2(fast_exp2(xa.x), fast_exp2(xa.y));
            gs = __ffma2_rn(Cp, dy2, gs);                              // g += C dy
            const float2 dC2 = __fmul2_rn(dy2, hs[j + 1]);             // dC = dy h
            const float2 gx = __fmul2_rn(gs, xx);
            const float2 dB2 = __fmul2_rn(gx, uu2);                    // dB = g x u
            const float2 dut2 = __fmul2_rn(gx, Bp);                    // du = g x B
            const float2 t = __ffma2_rn(__fmul2_rn(An, a), hs[j], __fmul2_rn(Bp, uu2));
            const float2 dxt2 = __fmul2_rn(gs, t);                     // dx = g (A a h' + B u)
            dAs = __ffma2_rn(__fmul2_rn(gx, a), hs[j], dAs);           // dA += g x a h'
            gs = __fmul2_rn(gs, a);                                    // carried to step j - 1
            // du and dDelta over the warp's 8 states of the channel (lanes 4c .. 4c + 3)
            float dut = dut2.x + dut2.y, dxt = dxt2.x + dxt2.y;
            dut += __shfl_xor_sync(FULL_MASK, dut, 1);
            dut += __shfl_xor_sync(FULL_MASK, dut, 2);
            dxt += __shfl_xor_sync(FULL_MASK, dxt, 1);
            dxt += __shfl_xor_sync(FULL_MASK, dxt, 2);
            if (grp == 0) {
                part.u[h][j][cc] = dut;
                part.x[h][j][cc] = dxt;
            }
            // dB and dC of the step summed over the 8 channels (lane bits 4, 3, 2): lane
            // 4c + g ends with tensor c >> 2 (0: B, 1: C) at state n0 + ((c >> 1) & 1);
            // lanes 4c + g and 4(c ^ 1) + g hold the same sum and the even c adds it.
            const float o0 = b4 ? dC2.x : dB2.x, o1 = b4 ? dC2.y : dB2.y;
            const float s0 = b4 ? dB2.x : dC2.x, s1 = b4 ? dB2.y : dC2.y;
            const float v0 = o0 + __shfl_xor_sync(FULL_MASK, s0, 16);
            const float v1 = o1 + __shfl_xor_sync(FULL_MASK, s1, 16);
            float w = (b2 ? v1 : v0) + __shfl_xor_sync(FULL_MASK, b2 ? v0 : v1, 8);
            w += __shfl_xor_sync(FULL_MASK, w, 4);
            const int n = n0 + (b2 ? 1 : 0);
            float* dst = b4 ? p.dC : p.dB;
            if (!b1 && q >= 0 && n < N && dst) atomicAdd(dst + ki * p.bc_dir + (img + q) * N + n, w);
        }
        __syncthreads();  // both state halves' partials are in part
        // the chunk's token gradients: one store or atomic per (step, channel)
#pragma unroll
        for (int r = 0; r < NE; ++r) {
            const int j = (tid + BWS_THREADS * r) / BW_CH;
            const int q = st.pos[j];
            if (q == -2 || !cev) continue;
            const float gyv = st.gy[j][ce];
            const float draw = (part.x[0][j][ce] + part.x[1][j][ce]) * st.sig[j][ce];
            dbs += draw;
            dDs = fmaf(gyv, st.u[j][ce], dDs);
            if (q < 0) continue;
            const float duv = fmaf(Dd_e, gyv, part.u[0][j][ce] + part.u[1][j][ce]);
            const long long o = ki * p.in_dir + (img + q) * D + c0 + ce;
            if constexpr (RK == RK_ATROUS2) {
                // one owner per pixel and channel: no other CTA writes this element
                if (p.du) p.du[o] = duv;
                if (p.ddelta) p.ddelta[o] = draw;
            } else {
                if (p.du) atomicAdd(p.du + o, duv);
                if (p.ddelta) atomicAdd(p.ddelta + o, draw);
            }
        }
    }
    if (dvalid) {
        if (n0 < N && p.dA) atomicAdd(p.dA + (long long)k * p.a_dir + (long long)d * N + n0, dAs.x);
        if (n0 + 1 < N && p.dA) atomicAdd(p.dA + (long long)k * p.a_dir + (long long)d * N + n0 + 1, dAs.y);
    }
    // D and bias gradients: lanes l, l ^ 8, l ^ 16, l ^ 24 of a warp share channel ce
    dDs += __shfl_xor_sync(FULL_MASK, dDs, 8);
    dDs += __shfl_xor_sync(FULL_MASK, dDs, 16);
    dbs += __shfl_xor_sync(FULL_MASK, dbs, 8);
    dbs += __shfl_xor_sync(FULL_MASK, dbs, 16);
    if (lane < BW_CH && cev) {
        if (p.dD) atomicAdd(p.dD + k * p.v_dir + c0 + ce, dDs);
        if (p.dbias) atomicAdd(p.dbias + k * p.v_dir + c0 + ce, dbs);
    }
}

}  // namespace vscan
