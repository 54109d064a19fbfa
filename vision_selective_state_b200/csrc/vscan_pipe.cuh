// Pipelined routed selective scan for the routes whose directions all visit
// every token: BIDIR (Vim, two directions) and CROSS4 (SS2D, four).
//
// One CTA covers one image b, a tile of CT channels and all KR directions of the
// route, with one producer warp and one consumer warp per direction.
//
//   producer   gathers every direction's chunks of TOK steps with 16-byte
//              cp.async into a ring of NS slots per direction (channels-last
//              rows make every gathered token one contiguous channel segment;
//              z only where the direction finalizes the token) and signals the
//              slot's "full" mbarrier with cp.async.mbarrier.arrive, so a slot
//              is ready exactly when its copies have landed. It refills a slot
//              after the consumer has released it on the slot's "empty"
//              mbarrier. It never waits for the consumers otherwise, so the
//              gathers of up to NS chunks are in flight ahead of the scan.
//
//   consumer   (one warp per direction) LPC lanes per channel, lane
//              cl * LPC + g owning channel cl of the tile and states
//              g * SPL .. g * SPL + SPL - 1 (SPL = 16 / LPC). Per chunk:
//                - discretize once per (step, channel) ("Vision Mamba ...",
//                  sec. 3; "EfficientVMamba", sec. 2), two items per packed
//                  softplus:
//                      Delta = softplus(raw + bias),  Delta * u
//                  and, for bf16 I/O, widen the chunk's B and C to float32;
//                - the recurrence and read-out per step and state (sec. 4),
//                  two states per packed f32x2 instruction:
//                      dA = 2^(Delta * A * log2 e)   (SFU, or MP states per lane
//                                                     on the FMA pipe)
//                      h  = dA * h + (Delta * u) * B
//                      y  = sum_n C * h              (butterfly reduce-scatter
//                                                     over the LPC lanes)
//                - the merge ("Vision Mamba ...", sec. 5; SS2D): y_k + D * u
//                  of every step goes to shared memory; the direction that
//                  visits a token in the latest chunk (ties: larger k) is its
//                  finalizer and adds the other directions' values, from
//                  shared memory when they were made in the same chunk, else
//                  from their parking plane in the workspace (prefetched one
//                  chunk ahead with cp.async); it applies merge_scale and
//                  SiLU(z) and stores y. A non-finalizer parks its value only
//                  when the finalizer meets the token in a later chunk.
//              The consumers of a CTA stay in step: two named barriers per
//              chunk (all values of the chunk in shared memory; all parked
//              values of the chunk written).
//
// FL_CKPT (16-step chunks): each consumer also stores its states entering every
// chunk into p.ckpt ([K][batch][chunks][D][16]) for the backward pass.
//
// No wait can hang: every mbarrier wait gives up after a bounded number of
// polls, records DEV_STATUS_TIMEOUT in the caller's status word (if any) and
// carries on without waiting again, so the kernel always terminates (with an
// invalid y). Addresses never depend on loaded data, so a broken pipeline
// computes garbage but stays in bounds.
#pragma once

#include "vscan_common.cuh"
#include "vscan_route.cuh"
#include "vscan_params.cuh"

namespace vscan {

// ---- mbarrier, cp.async and named-barrier helpers --------------------------------
__device__ __forceinline__ unsigned smem_u32(const void* p)
{
    return static_cast<unsigned>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar)
{
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ bool mbar_test(uint64_t* bar, unsigned parity)
{
    unsigned ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Polls of a pipeline wait before it gives up (each poll may suspend the
// thread for a short, hardware-defined time).
constexpr int PIPE_WAIT_POLLS = 1 << 18;

// Wait until the phase with the given parity of an mbarrier has completed.
// After PIPE_WAIT_POLLS polls it records the timeout and returns false; the
// caller keeps that as its `live` flag and a warp whose pipeline is no longer
// live skips every later wait, so a broken pipeline costs one timeout, not one
// per chunk.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, unsigned parity, int* status, bool live)
{
    if (!live) return false;
    for (int i = 0; i < PIPE_WAIT_POLLS; ++i)
        if (mbar_test(bar, parity)) return true;
    if (status) atomicOr(status, DEV_STATUS_TIMEOUT);
    return false;
}

// Arrive on bar once all cp.async copies this thread issued before have landed
// (the arrival is counted in the barrier's expected count).
__device__ __forceinline__ void cp_async_mbar_arrive(uint64_t* bar)
{
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;\n" ::: "memory"); }

__device__ __forceinline__ void named_sync(int id, int nthreads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ---- shape and shared-memory layout --------------------------------------------
template <int RK, typename T, int LPC, int TOK, int NS>
struct PipeShape {
    static constexpr int KR = (RK == RK_BIDIR) ? 2 : 4;  // directions, one consumer warp each
    static constexpr int CT = 32 / LPC;                  // channels of the tile
    static constexpr int SPL = 16 / LPC;                 // states per lane
    static constexpr int THREADS = 32 * (KR + 1);        // consumers + one producer warp
    static constexpr bool F32 = sizeof(T) == 4;
    static constexpr int EPI = TOK / LPC;                // (step, channel) items per lane per chunk
    static constexpr int EL = 16 / (int)sizeof(T);       // elements per 16-byte piece
    static constexpr int PC = CT / EL;                   // pieces per gathered row of u / Delta / z
    static constexpr int BCP = 16 / EL;                  // pieces per row of B (and of C)
    static constexpr int PPR = 3 * PC + 2 * BCP;         // pieces per step and direction
    static constexpr int PARTS = 32 / TOK;               // producer lanes per step
    static_assert(LPC == 1 || LPC == 2 || LPC == 4, "1, 2 or 4 lanes per channel");
    static_assert(RK == RK_BIDIR || RK == RK_CROSS4, "routes whose directions all visit every token");
    static_assert(PC >= 1, "a tile row must be at least 16 bytes");
    static_assert(TOK == 16 || TOK == 32, "16- or 32-step chunks");
    static_assert(TOK % LPC == 0, "whole groups of LPC steps per chunk");
    static_assert(NS >= 2, "at least two slots per direction");
};

// Gathered rows of one direction's chunk, in the I/O type, with the chunk's
// merge plan. meta[j] for step j: x = token (-2 past the end), y = 1 if this
// direction finalizes it, z = (finalizer) byte o = where the o-th other
// direction's value is: its row in that direction's current chunk, or 0xFF =
// parked in an earlier chunk; (non-finalizer) 1 if the value must be parked.
template <typename T, int CT, int TOK>
struct __align__(16) PipeSlot {
    int4 meta[TOK];
    T u[TOK][CT];
    T d[TOK][CT];
    T z[TOK][CT];
    T B[TOK][16];
    T C[TOK][16];
};

template <int KR, int CT, int TOK, bool F32>
struct __align__(16) PipeWarpSmem {
    float2 dd[TOK][CT];           // {Delta, Delta * u}
    float yk[TOK][CT];            // y_k + D * u of the chunk (read by same-chunk finalizers)
    float stg[KR - 1][TOK][CT];   // parked values of the other directions (earlier chunks)
    float4 bcf[F32 ? 1 : TOK][8]; // bf16 I/O: the chunk's B (quads 0-3) and C (4-7) in float32
};

template <int RK, typename T, int LPC, int TOK, int NS>
struct PipeSmem {
    using S = PipeShape<RK, T, LPC, TOK, NS>;
    uint64_t full[S::KR][NS];
    uint64_t empty[S::KR][NS];
    PipeSlot<T, S::CT, TOK> slot[S::KR][NS];
    PipeWarpSmem<S::KR, S::CT, TOK, S::F32> w[S::KR];
};

template <int RK, typename T, int LPC, int TOK, int NS>
constexpr size_t pipe_smem_bytes() { return sizeof(PipeSmem<RK, T, LPC, TOK, NS>); }

// Sum over the LPC lanes of a channel of the per-step partial read-outs v[0..LPC)
// of LPC consecutive steps, scattered so that lane g of the group keeps step g.
template <int LPC>
__device__ __forceinline__ float reduce_scatter(const float (&v)[LPC], int g)
{
    if constexpr (LPC == 1) {
        return v[0];
    } else {
        float cur[LPC];
#pragma unroll
        for (int i = 0; i < LPC; ++i) cur[i] = v[i];
#pragma unroll
        for (int s = LPC / 2; s >= 1; s /= 2) {
            const bool hi = (g & s) != 0;
#pragma unroll
            for (int i = 0; i < s; ++i) {
                const float keep = hi ? cur[i + s] : cur[i];
                const float send = hi ? cur[i] : cur[i + s];
                cur[i] = keep + __shfl_xor_sync(FULL_MASK, send, s);
            }
        }
        return cur[0];
    }
}

// Route position, finalizer and merge sources of step j of chunk c (direction k).
template <int RK, int KR, int TOK>
__device__ __forceinline__ int4 pipe_meta(const RouteGeom& g, int k, int c, int j)
{
    const int t = c * TOK + j;
    if (t >= g.L) return make_int4(-2, 0, 0, 0);
    const int p = route_token<RK>(g, k, t);
    int vs[KR];
#pragma unroll
    for (int kk = 0; kk < KR; ++kk) vs[kk] = visit_step<RK>(g, kk, p);
    // the finalizer and its chunk (kept alongside: indexing vs by a runtime value
    // would put the array in local memory)
    int fk = 0, fc = vs[0] / TOK;
#pragma unroll
    for (int kk = 1; kk < KR; ++kk) {
        const int ck = vs[kk] / TOK;
        if (ck >= fc) {
            fc = ck;
            fk = kk;
        }
    }
    if (fk == k) {
        // byte o: the o-th other direction (constant array indices; the shift is
        // the only runtime part)
        int src = 0, o = 0;
#pragma unroll
        for (int kk = 0; kk < KR; ++kk) {
            if (kk == k) continue;
            const int row = (vs[kk] / TOK == c) ? vs[kk] - c * TOK : 0xFF;
            src |= row << (8 * o);
            ++o;
        }
        return make_int4(p, 1, src, 0);
    }
    return make_int4(p, 0, (fc != c) ? 1 : 0, 0);
}

template <int RK, typename T, int LPC, int TOK, int NS, int MP, int MINB, int FL = 0>
__global__ void __launch_bounds__(PipeShape<RK, T, LPC, TOK, NS>::THREADS, MINB) pipe_scan_kernel(const ScanParams p)
{
    constexpr bool CKPT = (FL & FL_CKPT) != 0;
    static_assert((FL & ~FL_CKPT) == 0, "the pipelined kernel takes no optional step but checkpoints");
    static_assert(!CKPT || TOK == 16, "checkpoints every 16 steps (the adjoint scan's chunks)");
    using S = PipeShape<RK, T, LPC, TOK, NS>;
    constexpr int KR = S::KR, CT = S::CT, SPL = S::SPL, EPI = S::EPI, PC = S::PC, EL = S::EL;
    constexpr bool F32 = S::F32;
    constexpr int NCONS = 32 * KR;            // threads in the consumers' named barriers
    static_assert(MP % 2 == 0 && MP <= SPL, "FMA-pipe retentions come in pairs");
    extern __shared__ __align__(16) unsigned char smem_raw[];
    PipeSmem<RK, T, LPC, TOK, NS>& sm = *reinterpret_cast<PipeSmem<RK, T, LPC, TOK, NS>*>(smem_raw);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int b = blockIdx.y;
    const int c0 = blockIdx.x * CT;
    const int D = p.D, L = p.g.L, tokens = p.g.tokens;
    const int nchunks = (L + TOK - 1) / TOK;
    const long long img = (long long)b * tokens;

    if (threadIdx.x == 0) {
        for (int k = 0; k < KR; ++k)
            for (int s = 0; s < NS; ++s) {
                mbar_init(&sm.full[k][s], 64);   // per producer lane: its copies landed, its plan written
                mbar_init(&sm.empty[k][s], 1);   // lane 0 of the consumer releases
            }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    if (warp == KR) {
        // ================================ producer ==================================
        const int r = lane % TOK, part = lane / TOK;
        bool live = true;
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % NS;
            for (int k = 0; k < KR; ++k) {
                if (c >= NS) live = mbar_wait(&sm.empty[k][s], ((c / NS) - 1) & 1, p.status, live);
                PipeSlot<T, CT, TOK>& st = sm.slot[k][s];
                // lane -> (step r, part q of the step's 16-byte pieces): the lane's
                // own plan gives the token, so no piece needs another lane's data
                const int4 plan = pipe_meta<RK, KR, TOK>(p.g, k, c, r);
                if (part == 0) st.meta[r] = plan;
                const bool v = plan.x >= 0;
                const long long tok = v ? plan.x : 0;
                const T* u_row = static_cast<const T*>(p.u) + k * p.in_dir + (img + tok) * D + c0;
                const T* d_row = static_cast<const T*>(p.delta) + k * p.in_dir + (img + tok) * D + c0;
                const T* z_row = p.z ? static_cast<const T*>(p.z) + (img + tok) * D + c0 : u_row;
                const bool zc = v && plan.y && p.z;
                const T* B_row = static_cast<const T*>(p.B) + k * p.bc_dir + (img + tok) * 16;
                const T* C_row = static_cast<const T*>(p.C) + k * p.bc_dir + (img + tok) * 16;
#pragma unroll
                for (int i = 0; i < S::PPR; ++i) {
                    if (S::PARTS > 1 && i % S::PARTS != part) continue;
                    if (i < 3 * PC) {  // u, Delta, z: PC pieces each
                        const int t = i / PC, q = i % PC;
                        const bool ok = (t == 2 ? zc : v) && (c0 + q * EL) < D;
                        const T* src = (t == 0 ? u_row : (t == 1 ? d_row : z_row)) + (ok ? q * EL : 0);
                        T* dst = (t == 0 ? &st.u[r][0] : (t == 1 ? &st.d[r][0] : &st.z[r][0])) + q * EL;
                        cp_async16(dst, src, ok);
                    } else {  // B, C: BCP pieces each
                        const int t = (i - 3 * PC) / S::BCP, q = (i - 3 * PC) % S::BCP;
                        const T* src = (t == 0 ? B_row : C_row) + (v ? q * EL : 0);
                        T* dst = (t == 0 ? &st.B[r][0] : &st.C[r][0]) + q * EL;
                        cp_async16(dst, src, v);
                    }
                }
                cp_async_mbar_arrive(&sm.full[k][s]);
                mbar_arrive(&sm.full[k][s]);  // releases this lane's plan store
            }
        }
        cp_async_wait_all();
        return;
    }

    // ================================== consumer ====================================
    const int k = warp;
    const int cl = lane / LPC, g = lane % LPC;
    const int d = c0 + cl;
    const bool dvalid = d < D;
    PipeWarpSmem<KR, CT, TOK, F32>& ws = sm.w[k];
    float2 a2[SPL / 2];
#pragma unroll
    for (int i = 0; i < SPL / 2; ++i) {
        const int n = g * SPL + 2 * i;
        const float* Ar = p.A + (long long)k * p.a_dir + (long long)(dvalid ? d : 0) * 16;
        a2[i] = dvalid ? make_float2(__ldg(Ar + n) * LOG2E, __ldg(Ar + n + 1) * LOG2E) : make_float2(0.f, 0.f);
    }
    const float bias_k = (dvalid && p.bias) ? __ldg(p.bias + k * p.v_dir + d) : 0.f;
    const float Dk = (dvalid && p.Dskip) ? __ldg(p.Dskip + k * p.v_dir + d) : 0.f;
    float2 h[SPL / 2];
#pragma unroll
    for (int i = 0; i < SPL / 2; ++i) h[i] = make_float2(0.f, 0.f);
    T* y_base = static_cast<T*>(p.y) + img * D + d;
    float* park_k = p.scratch + ((long long)k * p.batch + b) * tokens * D + d;
    // FL_CKPT: this lane's SPL states of chunk c go to ck + c * D * 16
    float* ck = (CKPT && dvalid) ? p.ckpt + (((long long)k * p.batch + b) * nchunks * D + d) * 16 + g * SPL : nullptr;

    bool live = nchunks > 0 && mbar_wait(&sm.full[k][0], 0, p.status, true);
    for (int c = 0; c < nchunks; ++c) {
        const int s = c % NS;
        const int t0 = c * TOK;
        const PipeSlot<T, CT, TOK>& st = sm.slot[k][s];

        // ---- discretize once per (step, channel); widen B and C (bf16). Every
        // load comes before the first store: a store to the warp's buffers would
        // otherwise hold back each later load (the compiler cannot tell the slot
        // and the buffers apart), making one long chain of the chunk's items.
        static_assert(EPI % 2 == 0, "items come in pairs");
        float dr[EPI], ur[EPI];
#pragma unroll
        for (int i = 0; i < EPI; ++i) {
            const int j = g + LPC * i;
            dr[i] = to_float(st.d[j][cl]) + bias_k;
            ur[i] = to_float(st.u[j][cl]);
        }
        constexpr int NBC = F32 ? 1 : TOK / 4;
        uint2 bcr[NBC];
        if constexpr (!F32) {
#pragma unroll
            for (int i = 0; i < NBC; ++i) {
                const int q = lane & 7, j = (lane >> 3) + 4 * i;
                bcr[i] = *reinterpret_cast<const uint2*>(q < 4 ? &st.B[j][4 * q] : &st.C[j][4 * (q - 4)]);
            }
        }
#pragma unroll
        for (int i = 0; i < EPI; i += 2) {
            const int j0 = g + LPC * i, j1 = j0 + LPC;
            const float2 x = make_float2(dr[i], dr[i + 1]);
            const float2 sq = p.softplus ? softplus2(x) : x;
            const float d0 = (dvalid && t0 + j0 < L) ? sq.x : 0.f, d1 = (dvalid && t0 + j1 < L) ? sq.y : 0.f;
            ws.dd[j0][cl] = make_float2(d0, d0 * ur[i]);
            ws.dd[j1][cl] = make_float2(d1, d1 * ur[i + 1]);
        }
        if constexpr (!F32) {
#pragma unroll
            for (int i = 0; i < NBC; ++i) {
                const int q = lane & 7, j = (lane >> 3) + 4 * i;
                const uint2 raw = bcr[i];
                ws.bcf[j][q] = make_float4(__uint_as_float(raw.x << 16), __uint_as_float(raw.x & 0xffff0000u),
                                           __uint_as_float(raw.y << 16), __uint_as_float(raw.y & 0xffff0000u));
            }
        }
        __syncwarp();

        if constexpr (CKPT) {  // the state entering chunk c
            if (ck) {
#pragma unroll
                for (int i = 0; i < SPL / 2; ++i)
                    *reinterpret_cast<float2*>(ck + (long long)c * D * 16 + 2 * i) = h[i];
            }
        }

        // ---- recurrence and read-out. The chunk's sums stay in registers until the
        // loop ends: a shared-memory store inside it would order every later
        // step's loads behind it (the compiler cannot tell the slot and the
        // output buffers apart), and the steps could no longer overlap.
        float yv[EPI];
#pragma unroll
        for (int gq = 0; gq < EPI; ++gq) {
            float yp[LPC];
#pragma unroll
            for (int jj = 0; jj < LPC; ++jj) {
                const int j = gq * LPC + jj;
                const float2 dd = ws.dd[j][cl];
                const float2 ds = make_float2(dd.x, dd.x), du = make_float2(dd.y, dd.y);
                // this lane's SPL states of B and C, in pairs
                float2 Bp[SPL / 2], Cp[SPL / 2];
                if constexpr (F32 && SPL == 2) {
                    Bp[0] = *reinterpret_cast<const float2*>(&st.B[j][g * SPL]);
                    Cp[0] = *reinterpret_cast<const float2*>(&st.C[j][g * SPL]);
                } else {
                    const float4* Bq;
                    const float4* Cq;
                    if constexpr (F32) {
                        Bq = reinterpret_cast<const float4*>(&st.B[j][g * SPL]);
                        Cq = reinterpret_cast<const float4*>(&st.C[j][g * SPL]);
                    } else {
                        Bq = &ws.bcf[j][g * SPL / 4];
                        Cq = &ws.bcf[j][4 + g * SPL / 4];
                    }
#pragma unroll
                    for (int q = 0; q < SPL / 4; ++q) {
                        const float4 Bv = Bq[q], Cv = Cq[q];
                        Bp[2 * q] = make_float2(Bv.x, Bv.y);
                        Bp[2 * q + 1] = make_float2(Bv.z, Bv.w);
                        Cp[2 * q] = make_float2(Cv.x, Cv.y);
                        Cp[2 * q + 1] = make_float2(Cv.z, Cv.w);
                    }
                }
                float2 acc = make_float2(0.f, 0.f);
#pragma unroll
                for (int q = 0; q < SPL / 2; ++q) {
                    const float2 x = __fmul2_rn(ds, a2[q]);
                    const float2 e = (q < MP / 2) ? exp2_fma2(x) : make_float2(fast_exp2(x.x), fast_exp2(x.y));
                    h[q] = __ffma2_rn(e, h[q], __fmul2_rn(du, Bp[q]));
                    acc = __ffma2_rn(Cp[q], h[q], acc);
                }
                yp[jj] = acc.x + acc.y;
            }
            yv[gq] = reduce_scatter<LPC>(yp, g);  // this lane now holds step gq * LPC + g
        }
        // y_k + D * u of every step into shared memory (read by same-chunk finalizers)
        float uy[EPI];
#pragma unroll
        for (int i = 0; i < EPI; ++i) uy[i] = to_float(st.u[g + LPC * i][cl]);
#pragma unroll
        for (int i = 0; i < EPI; ++i) {
            yv[i] = fmaf(Dk, uy[i], yv[i]);
            ws.yk[g + LPC * i][cl] = yv[i];
        }
        named_sync(1, NCONS);
        cp_async_wait_all();  // this lane's prefetched parked values
        __syncwarp();

        // ---- merge, part 2: finalize (add the other directions, scale, gate, store) or park.
        // Loads first, then the arithmetic, then predicated stores; the two guards
        // are warp-uniform (whole chunks finalize or park, but for the few where
        // the directions cross).
        int4 mt[EPI];
        bool fin[EPI], park[EPI];
        bool any_fin = false, any_park = false;
#pragma unroll
        for (int i = 0; i < EPI; ++i) {
            mt[i] = st.meta[g + LPC * i];
            const bool ok = mt[i].x >= 0 && dvalid;
            fin[i] = ok && mt[i].y;
            park[i] = ok && !mt[i].y && mt[i].z;
            any_fin |= fin[i];
            any_park |= park[i];
        }
        if (__any_sync(FULL_MASK, any_fin)) {
            // a non-finalizer's plan holds 0 or 1 in byte 0 and zeros above: every
            // address below stays inside the buffers
            float acc[EPI], zg[EPI];
#pragma unroll
            for (int i = 0; i < EPI; ++i) {
                const int j = g + LPC * i;
                acc[i] = yv[i];
#pragma unroll
                for (int o = 0; o < KR - 1; ++o) {
                    const int kk = o < k ? o : o + 1;
                    const int row = (mt[i].z >> (8 * o)) & 0xFF;
                    const float* src = row == 0xFF ? &ws.stg[o][j][cl] : &sm.w[kk].yk[row & (TOK - 1)][cl];
                    acc[i] += *src;
                }
                zg[i] = p.z ? to_float(st.z[j][cl]) : 0.f;
            }
#pragma unroll
            for (int i = 0; i < EPI; ++i) {
                float out = acc[i] * p.merge_scale;
                if (p.z) out *= silu_f(zg[i]);
                if (fin[i]) store_elem<T>(y_base + (long long)mt[i].x * D, out);
            }
        }
        if (__any_sync(FULL_MASK, any_park)) {
#pragma unroll
            for (int i = 0; i < EPI; ++i)
                if (park[i]) park_k[(long long)mt[i].x * D] = yv[i];
        }
        // the slot (u, z and the plan were its last readers) goes back to the producer
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.empty[k][s]);
        named_sync(2, NCONS);

        // ---- next chunk: wait for its slot, prefetch the parked values its
        // finalizations need
        if (c + 1 < nchunks) {
            const int s1 = (c + 1) % NS;
            live = mbar_wait(&sm.full[k][s1], ((c + 1) / NS) & 1, p.status, live);
            const PipeSlot<T, CT, TOK>& nx = sm.slot[k][s1];
            constexpr int PF = TOK * (KR - 1) * (CT / 4);  // 16-byte pieces of float32 rows
#pragma unroll
            for (int it = 0; it < (PF + 31) / 32; ++it) {
                const int f = lane + 32 * it;
                if (f < PF) {
                    const int j = f / ((KR - 1) * (CT / 4));
                    const int r = f - j * (KR - 1) * (CT / 4);
                    const int o = r / (CT / 4), q = r - o * (CT / 4);
                    const int4 m = nx.meta[j];
                    const bool ok = m.x >= 0 && m.y && ((m.z >> (8 * o)) & 0xFF) == 0xFF && (c0 + 4 * q) < D;
                    const int kk = o < k ? o : o + 1;
                    const float* src = p.scratch + ((long long)kk * p.batch + b) * tokens * D + c0 + 4 * q +
                                       (ok ? (long long)m.x * D : 0);
                    cp_async16(&ws.stg[o][j][4 * q], src, ok);
                }
            }
            asm volatile("cp.async.commit_group;\n" ::: "memory");
        }
    }
    cp_async_wait_all();
}

}  // namespace vscan
