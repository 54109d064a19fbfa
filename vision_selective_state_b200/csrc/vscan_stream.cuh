// Streaming routed selective scan: BIDIR, CROSS4 and ATROUS2 routes.
//
// One CTA covers one image b, a tile of CH = 8 or 16 channels and KC directions
// of the route, and runs them as a software pipeline over chunks of TOK = 16
// steps (32 for the long BIDIR sequences) with two kinds of warps:
//
//   consumer warps (SS * CH / 8 per direction) run only the recurrence, each for 8
//     channels of the tile. Lane 4*c + g
//     owns channel c of the tile and states 4g..4g+3, so the 16 states of a
//     channel sit on 4 adjacent lanes and the read-out sum over n is a 4-lane
//     reduction; with SS = 2 (float32 atrous launches with few CTAs per SM) two
//     warps share the 8 channels, warp h holding states 8h + 2g, 8h + 2g + 1, and
//     the epilogue adds their two partial read-outs. Per step and state ("Vision Mamba ...", sec. 4;
//     "EfficientVMamba", sec. 2), two states per packed f32x2 instruction:
//         dA = 2^(Delta * A * log2 e)        (one SFU op)
//         h  = dA * h + (Delta * u) * B      (FMUL + FFMA)
//         y += C * h                         (FFMA)
//
//   producer warps (PW per direction, each owning TOK/PW steps of every chunk)
//     do everything that happens once per (step, channel): they gather the
//     route's tokens for chunk tau+1+LOOK with
//     cp.async into a shared-memory ring (zero fill for ATROUS2 padding;
//     channels-last rows make every gathered token one contiguous segment),
//     discretizes chunk tau+1 (Delta = softplus(raw + bias), Delta*u, B and C
//     as float32), and finishes chunk tau-1.
//
// All warps meet at one CTA barrier per chunk, so the gather of chunk tau+1+LOOK,
// the discretization of tau+1, the recurrence of tau and the epilogue of tau-1
// overlap.
//
// How a direction's output y_k (including its skip term D*u) becomes y
// (merge: "Vision Mamba ...", sec. 5; "EfficientVMamba", sec. 3; SS2D):
//   MODE_OWNER    ATROUS2: every pixel has one owner; y = s * y_k * SiLU(z).
//   MODE_PARK     all KC = K directions in one CTA (BIDIR, CROSS4): the
//                 direction that visits a token in the latest chunk (ties:
//                 larger k) adds it up. The others park y_k in the fp32
//                 workspace; one barrier later the finalizer adds the parked
//                 values to its own, scales, gates and stores.
// Neither mode uses atomics or a separate pass over y.
//
// Optional steps (template flags FL):
//   FL_ZOH   the write term uses the zero-order-hold gain phi(Delta A) (zoh_phi)
//            instead of Delta*B*u ("Norm or Direction? ...", Eq. 2).
//   FL_CKPT  the consumer also stores its state entering every chunk (ckpt),
//            for the backward pass.
//   FL_CONV  (BIDIR) u holds the convolution input x; the producer applies the
//            direction's kernel-four causal Conv1d + SiLU along the route
//            ("Vision Mamba ...", "Inside the released Vim block"), reading the
//            three previous steps from the previous chunk's token slot.
#pragma once

#include "vscan_common.cuh"
#include "vscan_params.cuh"
#include "vscan_route.cuh"

namespace vscan {

enum StreamMode : int { MODE_OWNER = 0, MODE_PARK = 1 };

constexpr int ST_TOK = 16;  // steps per chunk (default; the checkpointing run always uses 16)
constexpr int ST_CH = 8;    // channels per consumer warp (a CTA covers CH = 8 or 16 channels)
constexpr int ST_LOOK = 3;  // chunks between a gather and its discretization

// Gathered per-token rows of one direction's chunk, in the I/O type.
template <typename T, int CH, int TOK>
struct __align__(16) TokStage {
    T u[TOK][CH];
    T d[TOK][CH];
    T z[TOK][CH];
    int pos[TOK];  // token index, -1 pad, -2 past the end
    int fin[TOK];  // MODE_PARK: 1 if this direction adds up the token
};

// Gathered B and C rows of one direction's chunk, in the I/O type.
template <typename T, int TOK>
struct __align__(16) BCStage {
    T B[TOK][16];
    T C[TOK][16];
};

// Discretized chunk of one direction: with BCF (bf16 I/O) float32 copies of B
// and C, with ZOH the reciprocal of Delta.
template <bool ON, int TOK> struct PrepBC {};
template <int TOK> struct PrepBC<true, TOK> {
    float4 B[TOK][4];
    float4 C[TOK][4];
};
template <bool ON, int CH, int TOK> struct PrepRD {};
template <int CH, int TOK> struct PrepRD<true, CH, TOK> {
    float rd[TOK][CH];  // 1 / Delta (inf for Delta = 0, where zoh_phi does not use it)
};

template <bool BCF, bool ZOH, int CH, int TOK>
struct __align__(16) PrepStage : PrepBC<BCF, TOK>, PrepRD<ZOH, CH, TOK> {
    float2 dd[TOK][CH];  // {Delta after bias + softplus (0 past the end), Delta * u}
};

// FL_CONV: the convolved u of the last three chunks of each direction, for the
// skip term D*u of the epilogue.
template <bool ON, int KC, int CH, int TOK> struct ConvRing {};
template <int KC, int CH, int TOK> struct ConvRing<true, KC, CH, TOK> {
    float uc[KC][3][TOK][CH];
};

// SS: consumer warps sharing a channel's 16 states (1: lane 4c + g holds states
// 4g..4g+3 of channel c; 2: warp h of the pair holds states 8h..8h+7, lane 4c + g
// the pair 8h + 2g, 8h + 2g + 1, and the epilogue adds the two partial read-outs).
template <typename T, int KC, int MODE, int PW = 1, int CH = ST_CH, int TOK = ST_TOK, int SS = 1>
struct StreamShape {
    static constexpr bool F32 = sizeof(T) == 4;
    static constexpr bool PARK = MODE == MODE_PARK;
    // token slot of chunk c lives from its gather (tau = c-1-LOOK) to its last
    // epilogue use (tau = c+1, or c+2 when parking)
    // chunks between a gather and its discretization: 3 for 16-step chunks, 1 for 32
    static constexpr int LOOK = TOK >= 32 ? 1 : ST_LOOK;
    static constexpr int NR = LOOK + (PARK ? 4 : 3);
    // B/C slot: until discretized at tau = c-1 (bf16) or consumed at tau = c (f32)
    static constexpr int NBC = LOOK + (F32 ? 2 : 1);
    static constexpr int NY = PARK ? 3 : 2;  // output ring
    static constexpr int CW = SS * CH / ST_CH;           // consumer warps per direction
    static constexpr int THREADS = 32 * KC * (CW + PW);  // CW consumers and PW producers per direction
    static constexpr int SPW = TOK / PW;                 // steps of a chunk per producer warp
    static constexpr int RPL = SPW * CH / 32;            // (step, channel) items per producer lane
    static constexpr int NBCV = SPW / 8;                 // bf16 B/C quads converted per producer lane
    static_assert(PW == 1 || PW == 2, "one or two producer warps per direction");
    static_assert(CH == 8 || CH == 16, "8 or 16 channels per CTA");
    static_assert(TOK == 16 || TOK == 32, "16- or 32-step chunks");
    static_assert(SS == 1 || SS == 2, "one or two consumer warps per channel");
};

template <typename T, int KC, int MODE, int FL = 0, int CH = ST_CH, int TOK = ST_TOK, int SS = 1>
struct StreamSmem : ConvRing<(FL & FL_CONV) != 0, KC, CH, TOK> {
    using S = StreamShape<T, KC, MODE, 1, CH, TOK, SS>;
    TokStage<T, CH, TOK> tok[KC][S::NR];
    BCStage<T, TOK> bc[KC][S::NBC];
    PrepStage<!S::F32, (FL & FL_ZOH) != 0, CH, TOK> prep[KC][2];
    float yout[KC][S::NY][SS][TOK][CH];  // read-outs (SS partial planes) of the last NY chunks
};

template <typename T, int KC, int MODE, int FL = 0, int CH = ST_CH, int TOK = ST_TOK, int SS = 1>
constexpr size_t stream_smem_bytes() { return sizeof(StreamSmem<T, KC, MODE, FL, CH, TOK, SS>); }

// Direction that adds up token p: the one visiting p in the latest chunk.
template <int RK, int TOK>
__device__ __forceinline__ int finalizer(const RouteGeom& g, int p)
{
    int best_k = 0;
    int best_c = visit_step<RK>(g, 0, p) / TOK;
#pragma unroll
    for (int kk = 1; kk < (RK == RK_CROSS4 ? 4 : 2); ++kk) {
        const int c = visit_step<RK>(g, kk, p) / TOK;
        if (c >= best_c) {
            best_c = c;
            best_k = kk;
        }
    }
    return best_k;
}

template <int RK, typename T, bool N16, int KC, int MODE, int PW, int FL, int CH, int TOK, int SS = 1>
__global__ void __launch_bounds__(StreamShape<T, KC, MODE, PW, CH, TOK, SS>::THREADS) stream_scan_kernel(const ScanParams p)
{
    using S = StreamShape<T, KC, MODE, PW, CH, TOK, SS>;
    constexpr int LOOK = S::LOOK;
    constexpr int SPW = S::SPW, RPL = S::RPL, CW = S::CW, NBCV = S::NBCV;
    constexpr int RSTEP = 32 / CH;  // rows between a producer lane's items
    constexpr bool ZOH = (FL & FL_ZOH) != 0;
    constexpr bool CONV = (FL & FL_CONV) != 0;
    constexpr bool CKPT = (FL & FL_CKPT) != 0;
    static_assert(!CONV || RK == RK_BIDIR, "the fused convolution is defined for the bidirectional route");
    static_assert(!CONV || PW == 1, "the convolution reads steps gathered by the same producer warp");
    constexpr int NR = S::NR, NBC = S::NBC, NY = S::NY;
    constexpr bool PARK = S::PARK;
    constexpr bool F32 = S::F32;
    constexpr int KR = (RK == RK_BIDIR) ? 2 : 4;  // directions of the route
    extern __shared__ __align__(16) unsigned char smem_raw[];
    StreamSmem<T, KC, MODE, FL, CH, TOK, SS>& sm = *reinterpret_cast<StreamSmem<T, KC, MODE, FL, CH, TOK, SS>*>(smem_raw);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int b = blockIdx.y;
    const int c0 = blockIdx.x * CH;
    const int D = p.D, N = p.N, L = p.g.L, tokens = p.g.tokens;
    const int nchunks = (L + TOK - 1) / TOK;
    const int last_tau = nchunks + (PARK ? 1 : 0);
    const long long img = (long long)b * tokens;

    if (warp < KC * CW) {
        // =============================== consumer =================================
        const int kl = warp / CW;
        const int k = p.k_base + blockIdx.z * KC + kl;
        const int sub = warp % CW;                 // consumer warp of this direction
        const int half = SS == 2 ? (sub & 1) : 0;  // SS = 2: which 8 states of the channel
        const int cc = (sub / SS) * ST_CH + (lane >> 2), grp = lane & 3;  // channel of the tile
        const int d = c0 + cc;
        const bool dvalid = d < D;
        constexpr int NP = 2 / SS;  // state pairs per lane
        const int n0 = SS == 1 ? 4 * grp : 8 * half + 2 * grp;  // this lane's first state
        float2 a2p[NP];
        float ia[2 * NP];  // ZOH: 1 / A per state (0 for A = 0, where x = Delta A = 0 selects the polynomial)
#pragma unroll
        for (int q = 0; q < NP; ++q) {
            float av[2];
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const int n = n0 + 2 * q + i;
                av[i] = (dvalid && n < N) ? __ldg(p.A + (long long)k * p.a_dir + (long long)d * N + n) * LOG2E : 0.f;
                ia[2 * q + i] = (av[i] != 0.f) ? LOG2E / av[i] : 0.f;
            }
            a2p[q] = make_float2(av[0], av[1]);
        }
        float2 hp[NP];
#pragma unroll
        for (int q = 0; q < NP; ++q) hp[q] = make_float2(0.f, 0.f);
        __syncthreads();  // prologue: chunk 0 discretized

        float* ck = (CKPT && dvalid)
                        ? p.ckpt + (((long long)k * p.batch + b) * nchunks * D + d) * 16 + n0 : nullptr;
        for (int tau = 0; tau <= last_tau; ++tau) {
            if (tau < nchunks) {
                if constexpr (CKPT) {  // state entering chunk tau
                    if (ck) {
                        if constexpr (NP == 2)
                            *reinterpret_cast<float4*>(ck + (long long)tau * D * 16) = make_float4(hp[0].x, hp[0].y, hp[1].x, hp[1].y);
                        else
                            *reinterpret_cast<float2*>(ck + (long long)tau * D * 16) = hp[0];
                    }
                }
                const auto& pr = sm.prep[kl][tau & 1];
                const BCStage<T, TOK>& bcs = sm.bc[kl][tau % NBC];
                float* yo = &sm.yout[kl][tau % NY][half][0][0];
                // Software pipeline over the chunk's TOK steps: the loads, the SFU
                // exponentials and the input terms of step j + 2 are issued before
                // the state update of step j, which is the only serial dependency.
                float2 ep[TOK][NP], wp[TOK][NP], cp[TOK][NP];
                auto front = [&](int j) {
                    const float2 dd = pr.dd[j][cc];
                    float2 Bq[NP], Cq[NP];
                    if constexpr (F32) {
                        if constexpr (NP == 2) {
                            const float4 Bv = *reinterpret_cast<const float4*>(&bcs.B[j][n0]);
                            const float4 Cv = *reinterpret_cast<const float4*>(&bcs.C[j][n0]);
                            Bq[0] = make_float2(Bv.x, Bv.y); Bq[1] = make_float2(Bv.z, Bv.w);
                            Cq[0] = make_float2(Cv.x, Cv.y); Cq[1] = make_float2(Cv.z, Cv.w);
                        } else {
                            Bq[0] = *reinterpret_cast<const float2*>(&bcs.B[j][n0]);
                            Cq[0] = *reinterpret_cast<const float2*>(&bcs.C[j][n0]);
                        }
                    } else {
                        const float4 Bv = pr.B[j][n0 >> 2], Cv = pr.C[j][n0 >> 2];
                        if constexpr (NP == 2) {
                            Bq[0] = make_float2(Bv.x, Bv.y); Bq[1] = make_float2(Bv.z, Bv.w);
                            Cq[0] = make_float2(Cv.x, Cv.y); Cq[1] = make_float2(Cv.z, Cv.w);
                        } else {
                            const bool hi = n0 & 2;
                            Bq[0] = hi ? make_float2(Bv.z, Bv.w) : make_float2(Bv.x, Bv.y);
                            Cq[0] = hi ? make_float2(Cv.z, Cv.w) : make_float2(Cv.x, Cv.y);
                        }
                    }
                    const float2 dsp2 = make_float2(dd.x, dd.x);
                    const float2 du2 = make_float2(dd.y, dd.y);
                    float2 xq[NP];
#pragma unroll
                    for (int q = 0; q < NP; ++q) {
                        xq[q] = __fmul2_rn(dsp2, a2p[q]);
                        ep[j][q] = make_float2(fast_exp2(xq[q].x), fast_exp2(xq[q].y));
                        wp[j][q] = __fmul2_rn(du2, Bq[q]);
                        cp[j][q] = Cq[q];
                    }
                    if constexpr (ZOH) {
                        const float rd = pr.rd[j][cc];
#pragma unroll
                        for (int q = 0; q < NP; ++q) {
                            const float g0 = zoh_phi(xq[q].x * LN2, ep[j][q].x, rd * ia[2 * q]);
                            const float g1 = zoh_phi(xq[q].y * LN2, ep[j][q].y, rd * ia[2 * q + 1]);
                            wp[j][q] = __fmul2_rn(wp[j][q], make_float2(g0, g1));
                        }
                    }
                };
                front(0);
                front(1);
                float yv[TOK / 4];
#pragma unroll
                for (int q = 0; q < TOK / 4; ++q) {
                    float yp[4];
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        const int j = 4 * q + jj;
                        if (j + 2 < TOK) front(j + 2);
#pragma unroll
                        for (int r = 0; r < NP; ++r) hp[r] = __ffma2_rn(ep[j][r], hp[r], wp[j][r]);
                        float2 acc = __fmul2_rn(cp[j][0], hp[0]);
#pragma unroll
                        for (int r = 1; r < NP; ++r) acc = __ffma2_rn(cp[j][r], hp[r], acc);
                        yp[jj] = acc.x + acc.y;
                    }
                    // Reduce-scatter over the 4 state-group lanes: lane grp keeps step 4q+grp.
                    const bool hi = grp & 2;
                    float x0 = hi ? yp[2] : yp[0];
                    float x1 = hi ? yp[3] : yp[1];
                    const float s0 = hi ? yp[0] : yp[2];
                    const float s1 = hi ? yp[1] : yp[3];
                    x0 += __shfl_xor_sync(FULL_MASK, s0, 2);
                    x1 += __shfl_xor_sync(FULL_MASK, s1, 2);
                    const bool odd = grp & 1;
                    float keep = odd ? x1 : x0;
                    const float send = odd ? x0 : x1;
                    keep += __shfl_xor_sync(FULL_MASK, send, 1);
                    yv[q] = keep;
                }
                // stores after every load of the chunk, so none of them waits on a store
#pragma unroll
                for (int q = 0; q < TOK / 4; ++q) yo[(4 * q + grp) * CH + cc] = yv[q];
            }
            __syncthreads();
        }
        return;
    }

    // ================================= producer ===================================
    const int kl = (warp - KC * CW) / PW;
    const int j0 = ((warp - KC * CW) % PW) * SPW;   // first step of a chunk this warp owns
    const int k = p.k_base + blockIdx.z * KC + kl;  // direction this producer serves
    const int ce = lane % CH;  // channel of the tile this lane discretizes / stores
    const int jl = j0 + lane / CH;  // first row of this lane's items; then every RSTEP rows
    const int dch = c0 + ce;
    const bool evalid = dch < D;
    const float bias_k = (evalid && p.bias) ? __ldg(p.bias + k * p.v_dir + dch) : 0.f;
    const float Dk = (evalid && p.Dskip) ? __ldg(p.Dskip + k * p.v_dir + dch) : 0.f;
    float kw[4] = {0.f, 0.f, 0.f, 0.f};  // FL_CONV: the direction's kernel and bias for channel dch
    float kb = 0.f;
    if constexpr (CONV) {
        if (evalid) {
#pragma unroll
            for (int i = 0; i < 4; ++i) kw[i] = __ldg(p.conv_w + ((long long)k * p.v_dir + dch) * 4 + i);
            kb = p.conv_b ? __ldg(p.conv_b + k * p.v_dir + dch) : 0.f;
        }
    }
    const T* z_base = p.z ? static_cast<const T*>(p.z) + img * D + c0 : nullptr;
    T* y_base = static_cast<T*>(p.y) + img * D + dch;  // + token * D (fits in int32)
    // parked contributions of direction kk for this image and channel: + token * D
    auto park = [&](int kk) { return p.scratch + ((long long)kk * p.batch + b) * tokens * D + dch; };

    // Gather this warp's steps of chunk `chunk` into token slot chunk % NR and
    // B/C slot chunk % NBC.
    auto issue = [&](int chunk) {
        if (chunk < nchunks) {
            auto& st = sm.tok[kl][chunk % NR];
            BCStage<T, TOK>& sb = sm.bc[kl][chunk % NBC];
            const T* u_base = static_cast<const T*>(p.u) + k * p.in_dir + img * D + c0;
            const T* d_base = static_cast<const T*>(p.delta) + k * p.in_dir + img * D + c0;
            const T* B_base = static_cast<const T*>(p.B) + k * p.bc_dir + img * N;
            const T* C_base = static_cast<const T*>(p.C) + k * p.bc_dir + img * N;
            // lane i < SPW computes the route position of step j0 + i
            const int t = chunk * TOK + j0 + (lane & (SPW - 1));
            const int mypos = (t < L) ? route_token<RK>(p.g, k, t) : -2;
            if (lane < SPW) {
                st.pos[j0 + lane] = mypos;
                if constexpr (PARK) st.fin[j0 + lane] = (mypos >= 0 && finalizer<RK, TOK>(p.g, mypos) == k) ? 1 : 0;
            }
            if constexpr (CH == ST_CH && TOK == 16) {
                // 8-channel tiles of 16 steps: one 16- or 32-byte row piece per lane and tensor
                if (F32 && PW == 1) {
                    // u, Delta, z: 16 steps x 32 bytes; lane -> (step lane>>1, 4-channel half lane&1)
                    const int j = lane >> 1, hf = lane & 1;
                    const int pj = __shfl_sync(FULL_MASK, mypos, j);
                    const bool ok = pj >= 0 && (c0 + 4 * hf) < D;
                    const long long off = (long long)(ok ? pj : 0) * D + 4 * hf;
                    cp_async16(&st.u[j][4 * hf], u_base + off, ok);
                    cp_async16(&st.d[j][4 * hf], d_base + off, ok);
                    if (z_base) cp_async16(&st.z[j][4 * hf], z_base + off, ok);
                } else if (F32) {
                    // 8 steps x 32 bytes per tensor: lanes 0-15 take u and z, lanes 16-31 take Delta;
                    // lane -> (step (lane&15)>>1, 4-channel half lane&1)
                    const int i = (lane & 15) >> 1, hf = lane & 1, j = j0 + i;
                    const int pj = __shfl_sync(FULL_MASK, mypos, i);
                    const bool ok = pj >= 0 && (c0 + 4 * hf) < D;
                    const long long off = (long long)(ok ? pj : 0) * D + 4 * hf;
                    if (lane < 16) {
                        cp_async16(&st.u[j][4 * hf], u_base + off, ok);
                        if (z_base) cp_async16(&st.z[j][4 * hf], z_base + off, ok);
                    } else {
                        cp_async16(&st.d[j][4 * hf], d_base + off, ok);
                    }
                } else {
                    // SPW steps x 16 bytes per tensor: lane -> (tensor lane / SPW, step lane % SPW)
                    const int i = lane & (SPW - 1), j = j0 + i, which = lane / SPW;
                    const int pj = __shfl_sync(FULL_MASK, mypos, i);
                    const bool ok = pj >= 0;
                    const long long off = (long long)(ok ? pj : 0) * D;
                    if (PW == 1) {
                        if (lane < 16) {
                            cp_async16(&st.u[j][0], u_base + off, ok);
                            if (z_base) cp_async16(&st.z[j][0], z_base + off, ok);
                        } else {
                            cp_async16(&st.d[j][0], d_base + off, ok);
                        }
                    } else if (which == 0) {
                        cp_async16(&st.u[j][0], u_base + off, ok);
                    } else if (which == 1) {
                        cp_async16(&st.d[j][0], d_base + off, ok);
                    } else if (which == 2 && z_base) {
                        cp_async16(&st.z[j][0], z_base + off, ok);
                    }
                }
            } else
            {
                // u, Delta, z: SPW steps x CH channels per tensor, in 16-byte pieces;
                // copy f -> (tensor, step, piece). Every lane runs every round (the
                // position shuffle needs the whole warp); copies past the count skip.
                constexpr int EL = 16 / sizeof(T);          // channels per piece
                constexpr int PCS = CH / EL;                // pieces per step and tensor
                constexpr int NT = 3 * SPW * PCS;           // copies of the three tensors
#pragma unroll
                for (int it = 0; it < (NT + 31) / 32; ++it) {
                    const int f = lane + 32 * it;
                    const int tsr = f / (SPW * PCS), rem = f % (SPW * PCS);
                    const int i = rem / PCS, cel = (rem % PCS) * EL;
                    const int pj = __shfl_sync(FULL_MASK, mypos, i);
                    if (f < NT && (tsr < 2 || z_base)) {
                        const bool ok = pj >= 0 && (c0 + cel) < D;
                        const long long off = (long long)(ok ? pj : 0) * D + cel;
                        T* dst = tsr == 0 ? &st.u[j0 + i][cel] : (tsr == 1 ? &st.d[j0 + i][cel] : &st.z[j0 + i][cel]);
                        const T* src = (tsr == 0 ? u_base : (tsr == 1 ? d_base : z_base)) + off;
                        cp_async16(dst, src, ok);
                    }
                }
            }
            if (N16) {
                if (F32) {
                    // SPW steps x 4 quads x 16 bytes per tensor: f = lane + 32i -> (step f>>2, quad f&3)
#pragma unroll
                    for (int i = 0; i < SPW / 8; ++i) {
                        const int f = lane + 32 * i;
                        const int pj = __shfl_sync(FULL_MASK, mypos, f >> 2);
                        const bool ok = pj >= 0;
                        const long long off = (long long)(ok ? pj : 0) * 16 + 4 * (f & 3);
                        cp_async16(&sb.B[j0 + (f >> 2)][4 * (f & 3)], B_base + off, ok);
                        cp_async16(&sb.C[j0 + (f >> 2)][4 * (f & 3)], C_base + off, ok);
                    }
                } else if (PW == 1 && SPW == 16) {
                    // 16 steps x 2 halves x 16 bytes: lane -> (step lane>>1, half lane&1)
                    const int j = lane >> 1, hf = lane & 1;
                    const int pj = __shfl_sync(FULL_MASK, mypos, j);
                    const bool ok = pj >= 0;
                    const long long off = (long long)(ok ? pj : 0) * 16 + 8 * hf;
                    cp_async16(&sb.B[j][8 * hf], B_base + off, ok);
                    cp_async16(&sb.C[j][8 * hf], C_base + off, ok);
                } else if (SPW == 8) {
                    // 8 steps x 2 halves x 16 bytes per tensor: lanes 0-15 take B, 16-31 take C
                    const int i = (lane & 15) >> 1, hf = lane & 1;
                    const int pj = __shfl_sync(FULL_MASK, mypos, i);
                    const bool ok = pj >= 0;
                    const long long off = (long long)(ok ? pj : 0) * 16 + 8 * hf;
                    if (lane < 16) cp_async16(&sb.B[j0 + i][8 * hf], B_base + off, ok);
                    else cp_async16(&sb.C[j0 + i][8 * hf], C_base + off, ok);
                } else {
                    // SPW steps x 2 halves x 16 bytes per tensor: copy f -> (tensor, step, half)
#pragma unroll
                    for (int it = 0; it < (4 * SPW + 31) / 32; ++it) {
                        const int f = lane + 32 * it;
                        const int tsr = f / (2 * SPW), i = (f % (2 * SPW)) >> 1, hf = f & 1;
                        const int pj = __shfl_sync(FULL_MASK, mypos, i);
                        if (f < 4 * SPW) {
                            const bool ok = pj >= 0;
                            const long long off = (long long)(ok ? pj : 0) * 16 + 8 * hf;
                            if (tsr == 0) cp_async16(&sb.B[j0 + i][8 * hf], B_base + off, ok);
                            else cp_async16(&sb.C[j0 + i][8 * hf], C_base + off, ok);
                        }
                    }
                }
            } else {
                // Any N <= 16: element loads (the 16-byte path needs rows of 16 states).
#pragma unroll
                for (int i = 0; i < SPW / 2; ++i) {
                    const int e = lane + 32 * i;
                    const int n = e & 15, j = j0 + (e >> 4);
                    const int pj = __shfl_sync(FULL_MASK, mypos, e >> 4);
                    T vb = T(0.f), vc = T(0.f);
                    if (pj >= 0 && n < N) {
                        vb = B_base[(long long)pj * N + n];
                        vc = C_base[(long long)pj * N + n];
                    }
                    sb.B[j][n] = vb;
                    sb.C[j][n] = vc;
                }
            }
        }
        cp_async_commit();  // one group per chunk, possibly empty
    };

    // Discretize chunk c: once per (step, channel); loads first, then math, then stores.
    auto prepare = [&](int c) {
        const auto& st = sm.tok[kl][c % NR];
        auto& pr = sm.prep[kl][c & 1];
        float xd[RPL], xu[RPL];
        bool live[RPL];
#pragma unroll
        for (int r = 0; r < RPL; ++r) {
            const int j = jl + RSTEP * r;
            xd[r] = to_float(st.d[j][ce]);
            xu[r] = to_float(st.u[j][ce]);
            live[r] = st.pos[j] != -2 && evalid;  // past the end: a no-op step
        }
        if constexpr (CONV) {
            // u = SiLU(kb + sum_i kw[i] x[t - 3 + i]) along the route: steps before
            // the chunk come from the previous chunk's slot, before step 0 they are 0
            const auto& prev = sm.tok[kl][(c + NR - 1) % NR];
#pragma unroll
            for (int r = 0; r < RPL; ++r) {
                const int j = jl + RSTEP * r;
                float acc = kb;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int jj = j - 3 + i;
                    float xv;
                    if (jj >= 0) xv = (i == 3) ? xu[r] : to_float(st.u[jj][ce]);
                    else xv = (c > 0) ? to_float(prev.u[TOK + jj][ce]) : 0.f;
                    acc = fmaf(kw[i], xv, acc);
                }
                xu[r] = silu_f(acc);
                sm.uc[kl][c % 3][j][ce] = xu[r];
            }
        }
        float4 cb[NBCV], cv[NBCV];
        if constexpr (!F32) {
            const BCStage<T, TOK>& sb = sm.bc[kl][c % NBC];
#pragma unroll
            for (int r = 0; r < NBCV; ++r) {
                const int f = lane + 32 * r;  // (step j0 + f>>2, quad f&3)
                const int j = j0 + (f >> 2), q = f & 3;
                cb[r] = make_float4(to_float(sb.B[j][4 * q]), to_float(sb.B[j][4 * q + 1]),
                                    to_float(sb.B[j][4 * q + 2]), to_float(sb.B[j][4 * q + 3]));
                cv[r] = make_float4(to_float(sb.C[j][4 * q]), to_float(sb.C[j][4 * q + 1]),
                                    to_float(sb.C[j][4 * q + 2]), to_float(sb.C[j][4 * q + 3]));
            }
        }
        float2 out[RPL];
#pragma unroll
        for (int r = 0; r < RPL; ++r) {
            const float x = xd[r] + bias_k;
            const float dsp = live[r] ? (p.softplus ? softplus_f(x) : x) : 0.f;
            out[r] = make_float2(dsp, live[r] ? dsp * xu[r] : 0.f);
        }
#pragma unroll
        for (int r = 0; r < RPL; ++r) pr.dd[jl + RSTEP * r][ce] = out[r];
        if constexpr (ZOH) {
#pragma unroll
            for (int r = 0; r < RPL; ++r) pr.rd[jl + RSTEP * r][ce] = fast_rcp(out[r].x);
        }
        if constexpr (!F32) {
#pragma unroll
            for (int r = 0; r < NBCV; ++r) {
                const int f = lane + 32 * r;
                pr.B[j0 + (f >> 2)][f & 3] = cb[r];
                pr.C[j0 + (f >> 2)][f & 3] = cv[r];
            }
        }
    };

    // Epilogue of chunk c: add the skip term, then store (one owner) or park / keep.
    auto finish_a = [&](int c) {
        const auto& st = sm.tok[kl][c % NR];
        float* yo = &sm.yout[kl][c % NY][0][0][0];  // SS = 2: the second partial plane follows
        int pj[RPL], fin[RPL];
        float yk[RPL], zz[RPL];
#pragma unroll
        for (int r = 0; r < RPL; ++r) {
            const int j = jl + RSTEP * r;
            pj[r] = evalid ? st.pos[j] : -1;
            fin[r] = PARK ? st.fin[j] : 1;
            float uj;
            if constexpr (CONV) uj = sm.uc[kl][c % 3][j][ce];
            else uj = to_float(st.u[j][ce]);
            const float ys = SS == 2 ? yo[j * CH + ce] + yo[(SS - 1) * TOK * CH + j * CH + ce] : yo[j * CH + ce];
            yk[r] = fmaf(Dk, uj, ys);
            zz[r] = z_base ? to_float(st.z[j][ce]) : 0.f;
        }
        // every row computes its value; only the stores are predicated
        float o[RPL];
#pragma unroll
        for (int r = 0; r < RPL; ++r) {
            o[r] = yk[r];
            if constexpr (MODE == MODE_OWNER) {
                o[r] *= p.merge_scale;
                if (z_base) o[r] *= silu_f(zz[r]);
            }
        }
#pragma unroll
        for (int r = 0; r < RPL; ++r) {
            const int j = jl + RSTEP * r;
            if constexpr (MODE == MODE_OWNER) {
                if (pj[r] >= 0) store_elem<T>(y_base + pj[r] * D, o[r]);
            } else {
                if (pj[r] >= 0 && fin[r]) yo[j * CH + ce] = o[r];
                if (pj[r] >= 0 && !fin[r]) park(k)[pj[r] * D] = o[r];
            }
        }
    };

    // MODE_PARK, second half (chunk c, one barrier after finish_a): the finalizer
    // adds the parked contributions, scales, gates and stores. The parked values
    // are loaded at the top of the iteration (fetch_b) and used at its end.
    float parked[RPL];
    auto fetch_b = [&](int c) {
        const auto& st = sm.tok[kl][c % NR];
#pragma unroll
        for (int r = 0; r < RPL; ++r) {
            const int j = jl + RSTEP * r;
            const int pj = st.pos[j];
            float acc = 0.f;
            if (evalid && pj >= 0 && st.fin[j]) {
#pragma unroll
                for (int kk = 0; kk < KR; ++kk) {
                    if (kk == k) continue;
                    acc += park(kk)[pj * D];
                }
            }
            parked[r] = acc;
        }
    };
    auto finish_b = [&](int c) {
        const auto& st = sm.tok[kl][c % NR];
        const float* yo = &sm.yout[kl][c % NY][0][0][0];  // the finalizer's value, kept by finish_a
#pragma unroll
        for (int r = 0; r < RPL; ++r) {
            const int j = jl + RSTEP * r;
            const int pj = st.pos[j];
            if (!evalid || pj < 0 || !st.fin[j]) continue;
            float o = (yo[j * CH + ce] + parked[r]) * p.merge_scale;
            if (z_base) o *= silu_f(to_float(st.z[j][ce]));
            store_elem<T>(y_base + pj * D, o);
        }
    };

    // Prologue: gathers for chunks 0..LOOK in flight, chunk 0 discretized.
#pragma unroll
    for (int c = 0; c <= LOOK; ++c) issue(c);
    cp_async_wait<LOOK>();
    __syncwarp();
    if (nchunks > 0) prepare(0);
    __syncthreads();

    for (int tau = 0; tau <= last_tau; ++tau) {
        const bool do_b = PARK && tau >= 2 && tau - 2 < nchunks;
        if (do_b) fetch_b(tau - 2);
        issue(tau + 1 + LOOK);
        if (tau + 1 < nchunks) {
            cp_async_wait<LOOK>();  // chunk tau+1 has landed (this lane's copies)
            __syncwarp();              // ... and every lane's
            prepare(tau + 1);
        }
        if (tau >= 1 && tau - 1 < nchunks) finish_a(tau - 1);
        if (do_b) finish_b(tau - 2);
        __syncthreads();
    }
    cp_async_wait<0>();
}

}  // namespace vscan
