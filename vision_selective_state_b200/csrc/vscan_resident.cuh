// Resident chunked routed selective scan, for grids whose channel tile fits on
// chip (e.g. Vim-Tiny's 197 tokens): more parallelism per sequence at the cost
// of a second pass over each chunk.
//
// The CTA stages the whole token array of one image and a tile of CH channels
// in shared memory, with the step Delta = softplus(raw Delta + bias)
// discretized once per token and channel. With f32 I/O and N = 16 every row of
// the tile is whole 16-byte pieces and the staging is one round trip: a cp.async
// per piece (u, raw Delta, z, B, C), all in flight together, then the softplus in
// place; the per-channel parameters are loaded before it so their latency hides
// under it. Other cases stage element by element through registers. The launch
// takes CH = 4 instead of 8 for BIDIR when 8-channel tiles would give fewer CTAs
// than SMs: the launch is a chain of dependent steps per warp, so spreading the
// warps over more SMs shortens it. Each direction's sequence is cut into NC chunks; lane
// (chunk j, group g) of a channel runs its chunk sequentially for states
// 4g..4g+3:
//   pass 1  from a zero state: P = prod_t dA_t and H = the chunk's end state,
//           i.e. the chunk as one affine map h -> P (.) h + H;
//   combine an inclusive warp-shuffle scan of the affine pairs over the chunk
//           lanes, (P1, H1) then (P2, H2) -> (P1 P2, P2 H1 + H2), gives every
//           chunk the state entering it;
//   pass 2  from that state: recurrence and read-out, y summed over the four
//           group lanes, written to a per-direction output plane in shared
//           memory at the token's grid position.
// A CTA barrier then merges the planes (sum; ATROUS2 has one owner per token
// and a single plane), scales, gates with SiLU(z) and stores.
//
// The recurrence, discretization and merge follow "Vision Mamba ...", sec. 3-5,
// and "EfficientVMamba ...", sec. 1-3, exactly as the streaming kernel does;
// "Fast Vision Mamba ..." cites the log-depth parallel scan this realizes.
//
// Optional steps (template flags FL): FL_ZOH, the zero-order-hold write term;
// FL_CONV (BIDIR), u holds the convolution input x and each direction's
// kernel-four causal Conv1d + SiLU is applied along its route after staging,
// into one convolved plane per direction.
#pragma once

#include "vscan_common.cuh"
#include "vscan_route.cuh"
#include "vscan_params.cuh"

namespace vscan {

template <int RK>
struct ResidentShape {
    static constexpr int K = (RK == RK_BIDIR) ? 2 : 4;
    static constexpr int CH = (K == 2) ? 8 : 4;               // widest channel tile per CTA
    static constexpr int PLANES = (RK == RK_ATROUS2) ? 1 : K;  // output planes
};

// Shared-memory bytes of the resident kernel with a tile of ch channels (0: the
// route's widest tile), or 0 if the route is not supported. Ki: input planes
// (u, B, C); Kd: planes of the discretized step (K when the inputs or the bias
// differ per direction, else 1). The z plane is counted whether or not a gate
// is given.
inline size_t resident_smem_bytes(int kind, int tokens, int Ki, int Kd, bool conv = false, int ch = 0)
{
    int CH, PLANES;
    switch (kind) {
    case RK_BIDIR: CH = 8; PLANES = 2; break;
    case RK_CROSS4: CH = 4; PLANES = 4; break;
    case RK_ATROUS2: CH = 4; PLANES = 1; break;
    default: return 0;
    }
    if (conv && kind != RK_BIDIR) return 0;
    if (ch > 0) CH = ch;
    const size_t per_token = (size_t)Ki * (CH + 32) + (size_t)Kd * CH + (size_t)PLANES * CH + CH +
                             (conv ? (size_t)2 * CH : 0);
    return per_token * tokens * sizeof(float);
}

// CH: channels per CTA (a multiple of the channels one warp covers, 8 / NC).
template <int RK, typename T, int NC, int FL, int CH>
__global__ void __launch_bounds__(64 * NC * CH / ResidentShape<RK>::CH) resident_scan_kernel(const ScanParams p)
{
    using S = ResidentShape<RK>;
    constexpr bool ZOH = (FL & FL_ZOH) != 0;
    constexpr bool CONV = (FL & FL_CONV) != 0;
    static_assert(!CONV || RK == RK_BIDIR, "the fused convolution is defined for the bidirectional route");
    constexpr int K = S::K, PLANES = S::PLANES;
    constexpr int LPC = 4 * NC;        // lanes per channel
    constexpr int CPW = 32 / LPC;      // channels per warp
    constexpr int WPD = CH / CPW;      // warps per direction
    static_assert(CPW >= 1 && CH % CPW == 0 && CH <= S::CH, "chunk count must be 2, 4 or 8; CH a multiple of 8 / NC");
    static_assert(CH % 4 == 0 || sizeof(T) != 4, "");

    extern __shared__ __align__(16) float rsm[];
    const int tokens = p.g.tokens, L = p.g.L, D = p.D, N = p.N;
    const int Ki = p.in_dir ? K : 1;
    const int Kd = (p.in_dir || p.v_dir) ? K : 1;
    float* su = rsm;                                  // [Ki][tokens][CH]  u
    float* sp = su + (size_t)Ki * tokens * CH;        // [Kd][tokens][CH]  softplus(raw delta + bias)
    float* sB = sp + (size_t)Kd * tokens * CH;        // [Ki][tokens][16]
    float* sC = sB + (size_t)Ki * tokens * 16;        // [Ki][tokens][16]
    float* sY = sC + (size_t)Ki * tokens * 16;        // [PLANES][tokens][CH]
    float* sZ = sY + (size_t)PLANES * tokens * CH;    // [tokens][CH] gate input (f32 staging path)
    float* sX = sZ + (size_t)tokens * CH;             // FL_CONV: [2][tokens][CH] convolved u

    const int tid = threadIdx.x;
    constexpr int nthreads = K * WPD * 32;
    const int b = blockIdx.y;
    const int c0 = blockIdx.x * CH;
    const long long img = (long long)b * tokens;
    const T* zb = p.z ? static_cast<const T*>(p.z) + img * D : nullptr;

    // ---- roles and per-channel parameters, loaded before the staging so that their
    //      latency overlaps it
    const int warp = tid >> 5, lane = tid & 31;
    const int k = warp / WPD;
    const int wi = warp - k * WPD;
    const int cl = lane / LPC;
    const int r = lane - cl * LPC;
    const int j = r >> 2;          // chunk
    const int grp = r & 3;         // states 4*grp .. 4*grp+3
    const int c = wi * CPW + cl;   // channel within the tile
    const int d = c0 + c;
    const bool dvalid = d < D;
    const int ki = Ki > 1 ? k : 0;
    float a2[4];
#pragma unroll
    for (int s = 0; s < 4; ++s) {
        const int n = 4 * grp + s;
        a2[s] = (dvalid && n < N) ? __ldg(p.A + (long long)k * p.a_dir + (long long)d * N + n) * LOG2E : 0.f;
    }
    const float Dd = (dvalid && p.Dskip) ? __ldg(p.Dskip + k * p.v_dir + d) : 0.f;
    const float bias = (dvalid && p.bias) ? __ldg(p.bias + k * p.v_dir + d) : 0.f;

    // ---- stage the tile: u, the discretized step (once per token and channel), B, C
    //      (and z on the f32 path)
    constexpr bool F32 = sizeof(T) == 4;
    if (F32 && N == 16) {
        // Every row a whole number of 16-byte pieces (channels are a multiple of 4 and
        // every tensor 16-byte aligned): one cp.async per piece, all in flight at once,
        // then Delta = softplus(raw + bias) in place.
        constexpr int Q = CH / 4;  // pieces per token row of the tile
        const int n_u = Ki * tokens * Q, n_d = Kd * tokens * Q, n_z = zb ? tokens * Q : 0;
        for (int e = tid; e < n_u + n_d + n_z; e += nthreads) {
            const int which = e < n_u ? 0 : (e < n_u + n_d ? 1 : 2);
            const int ee = e - (which == 0 ? 0 : (which == 1 ? n_u : n_u + n_d));
            const int kk = ee / (tokens * Q);
            const int rem = ee - kk * tokens * Q;
            const int tok = rem / Q, q = rem - tok * Q;
            const int dq = c0 + 4 * q;
            const bool ok = dq < D;
            const float* base = static_cast<const float*>(which == 0 ? p.u : (which == 1 ? p.delta : p.z));
            const long long o = (which == 2 ? 0 : kk * p.in_dir) + (img + tok) * D + dq;
            float* dst = (which == 0 ? su : (which == 1 ? sp : sZ)) + ((size_t)kk * tokens + tok) * CH + 4 * q;
            cp_async16(dst, ok ? base + o : base, ok);
        }
        const int n_bc = Ki * tokens * 4;
        for (int e = tid; e < 2 * n_bc; e += nthreads) {
            const bool isC = e >= n_bc;
            const int ee = isC ? e - n_bc : e;  // (plane, token, piece) = piece index in [Ki][tokens][4]
            const int kk = ee / (tokens * 4);
            const long long o = kk * p.bc_dir + (img + (ee - kk * tokens * 4) / 4) * 16 + 4 * (ee & 3);
            cp_async16((isC ? sC : sB) + 4 * (size_t)ee, static_cast<const float*>(isC ? p.C : p.B) + o, true);
        }
        cp_async_commit();
        // this thread's channel in the in-place pass (nthreads is a multiple of CH)
        const int cs = tid % CH;
        float bsp[K];
#pragma unroll
        for (int kd = 0; kd < K; ++kd)
            bsp[kd] = (kd < Kd && c0 + cs < D && p.bias) ? __ldg(p.bias + kd * p.v_dir + c0 + cs) : 0.f;
        cp_async_wait<0>();
        __syncthreads();
#pragma unroll
        for (int kd = 0; kd < K; ++kd) {
            if (kd < Kd) {
                float* spk = sp + (size_t)kd * tokens * CH;
                for (int e = tid; e < tokens * CH; e += nthreads) {
                    const float x = spk[e] + bsp[kd];
                    spk[e] = p.softplus ? softplus_f(x) : x;
                }
            }
        }
    } else {
        constexpr int BATCH = 4;  // independent loads in flight per thread while staging
        const int n_u = Ki * tokens * CH, n_d = Kd * tokens * CH;
        for (int base = tid; base < n_u + n_d; base += BATCH * nthreads) {
            float v[BATCH];
#pragma unroll
            for (int rr = 0; rr < BATCH; ++rr) {
                const int e = base + rr * nthreads;
                v[rr] = 0.f;
                if (e < n_u + n_d) {
                    const bool is_u = e < n_u;
                    const int ee = is_u ? e : e - n_u;
                    const int kk = ee / (tokens * CH);
                    const int rem = ee - kk * tokens * CH;
                    const int tok = rem / CH, cc = rem - tok * CH;
                    const int dd = c0 + cc;
                    if (dd < D) {
                        const int kx = is_u ? kk : (Ki > 1 ? kk : 0);
                        const long long o = kx * p.in_dir + (img + tok) * D + dd;
                        v[rr] = load_elem<T>(static_cast<const T*>(is_u ? p.u : p.delta) + o);
                    }
                }
            }
#pragma unroll
            for (int rr = 0; rr < BATCH; ++rr) {
                const int e = base + rr * nthreads;
                if (e < n_u) {
                    su[e] = v[rr];
                } else if (e < n_u + n_d) {
                    const int ee = e - n_u;
                    const int kd = ee / (tokens * CH);
                    const int cc = (ee - kd * tokens * CH) % CH;
                    const int dd = c0 + cc;
                    const float bb = (dd < D && p.bias) ? __ldg(p.bias + kd * p.v_dir + dd) : 0.f;
                    const float x = v[rr] + bb;
                    sp[ee] = p.softplus ? softplus_f(x) : x;
                }
            }
        }
        const int n_bc = Ki * tokens * 16;
        for (int base = tid; base < n_bc; base += BATCH * nthreads) {
            float vb[BATCH], vc[BATCH];
#pragma unroll
            for (int rr = 0; rr < BATCH; ++rr) {
                const int e = base + rr * nthreads;
                vb[rr] = 0.f;
                vc[rr] = 0.f;
                if (e < n_bc) {
                    const int kk = e / (tokens * 16);
                    const int rem = e - kk * tokens * 16;
                    const int tok = rem >> 4, n = rem & 15;
                    if (n < N) {
                        const long long o = kk * p.bc_dir + (img + tok) * N + n;
                        vb[rr] = load_elem<T>(static_cast<const T*>(p.B) + o);
                        vc[rr] = load_elem<T>(static_cast<const T*>(p.C) + o);
                    }
                }
            }
#pragma unroll
            for (int rr = 0; rr < BATCH; ++rr) {
                const int e = base + rr * nthreads;
                if (e < n_bc) {
                    sB[e] = vb[rr];
                    sC[e] = vc[rr];
                }
            }
        }
    }
    __syncthreads();

    // ---- FL_CONV: u_k = SiLU(conv_k(x)) along each direction's route -------------
    if constexpr (CONV) {
        // BIDIR: direction 0 visits token t at step t, direction 1 at step tokens-1-t,
        // so the causal taps of token t are x[t-3+i] (forward) and x[t+3-i] (backward).
        for (int e = tid; e < 2 * tokens * CH; e += nthreads) {
            const int kd = e / (tokens * CH);
            const int rem = e - kd * tokens * CH;
            const int tok = rem / CH, c = rem - tok * CH;
            const int d = c0 + c;
            float acc = 0.f;
            if (d < D) {
                const float* xk = su + (size_t)(Ki > 1 ? kd : 0) * tokens * CH;
                const long long o = (long long)kd * p.v_dir + d;
                acc = p.conv_b ? __ldg(p.conv_b + o) : 0.f;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int tt = kd == 0 ? tok - 3 + i : tok + 3 - i;
                    if (tt >= 0 && tt < tokens) acc = fmaf(__ldg(p.conv_w + o * 4 + i), xk[(size_t)tt * CH + c], acc);
                }
            }
            sX[e] = silu_f(acc);
        }
        __syncthreads();
    }

    // ---- per-warp views of the staged tile ------------------------------------
    const float dsp_pad = p.softplus ? softplus_f(bias) : bias;  // ATROUS2 padding step
    const float* suk = CONV ? sX + (size_t)k * tokens * CH : su + (size_t)ki * tokens * CH;
    float ia[4];  // ZOH: 1 / A per state (0 for A = 0)
#pragma unroll
    for (int s = 0; s < 4; ++s) ia[s] = (a2[s] != 0.f) ? LOG2E / a2[s] : 0.f;
    const float* spk = sp + (size_t)(Kd > 1 ? k : 0) * tokens * CH;
    const float4* sBk = reinterpret_cast<const float4*>(sB + (size_t)ki * tokens * 16);
    const float4* sCk = reinterpret_cast<const float4*>(sC + (size_t)ki * tokens * 16);
    float* sYk = sY + (size_t)(PLANES == 1 ? 0 : k) * tokens * CH;

    const int Lc = (L + NC - 1) / NC;
    const int t0 = j * Lc;

    // One step: discretized delta, delta*u, u, and this lane's B/C quads.
    auto step = [&](int t, float& dsp, float& du, float& uu, float4& Bv, float4& Cv, int& pos) {
        pos = (t < L) ? route_token<RK>(p.g, k, t) : -2;
        dsp = 0.f; du = 0.f; uu = 0.f;
        Bv = make_float4(0.f, 0.f, 0.f, 0.f);
        Cv = Bv;
        if (pos >= 0) {
            uu = suk[(size_t)pos * CH + c];
            dsp = spk[(size_t)pos * CH + c];
            Bv = sBk[(size_t)pos * 4 + grp];
            Cv = sCk[(size_t)pos * 4 + grp];
            du = dsp * uu;
        } else if (pos == -1) {
            dsp = dsp_pad;
        }
    };

    // ---- pass 1: each chunk as an affine map -------------------------------------
    float P[4] = {1.f, 1.f, 1.f, 1.f}, H[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
    for (int i = 0; i < Lc; ++i) {
        float dsp, du, uu;
        float4 Bv, Cv;
        int pos;
        step(t0 + i, dsp, du, uu, Bv, Cv, pos);
        const float bv[4] = {Bv.x, Bv.y, Bv.z, Bv.w};
        const float rd = ZOH ? fast_rcp(dsp) : 0.f;
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            const float e = fast_exp2(dsp * a2[s]);
            float w = du * bv[s];
            if constexpr (ZOH) w *= zoh_phi(dsp * a2[s] * LN2, e, rd * ia[s]);
            P[s] *= e;
            H[s] = fmaf(e, H[s], w);
        }
    }

    // ---- combine: inclusive shuffle scan of (P, H) over the chunk lanes ----------
#pragma unroll
    for (int off = 1; off < NC; off <<= 1) {
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            const float Pp = __shfl_up_sync(FULL_MASK, P[s], 4 * off, LPC);
            const float Hp = __shfl_up_sync(FULL_MASK, H[s], 4 * off, LPC);
            if (j >= off) {
                H[s] = fmaf(P[s], Hp, H[s]);
                P[s] *= Pp;
            }
        }
    }
    float h[4];
#pragma unroll
    for (int s = 0; s < 4; ++s) {
        const float hin = __shfl_up_sync(FULL_MASK, H[s], 4, LPC);
        h[s] = (j > 0) ? hin : 0.f;
    }

    // ---- pass 2: recurrence from the entering state, read-out ---------------------
#pragma unroll 4
    for (int i = 0; i < Lc; ++i) {
        float dsp, du, uu;
        float4 Bv, Cv;
        int pos;
        step(t0 + i, dsp, du, uu, Bv, Cv, pos);
        const float bv[4] = {Bv.x, Bv.y, Bv.z, Bv.w};
        const float cv[4] = {Cv.x, Cv.y, Cv.z, Cv.w};
        const float rd = ZOH ? fast_rcp(dsp) : 0.f;
        float acc = 0.f;
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            const float e = fast_exp2(dsp * a2[s]);
            float w = du * bv[s];
            if constexpr (ZOH) w *= zoh_phi(dsp * a2[s] * LN2, e, rd * ia[s]);
            h[s] = fmaf(e, h[s], w);
            acc = fmaf(cv[s], h[s], acc);
        }
        acc += __shfl_xor_sync(FULL_MASK, acc, 1);
        acc += __shfl_xor_sync(FULL_MASK, acc, 2);
        if (grp == 0 && pos >= 0) sYk[(size_t)pos * CH + c] = fmaf(Dd, uu, acc);
    }
    __syncthreads();

    // ---- merge the directions, gate, store ----------------------------------------
    const bool z_staged = F32 && N == 16;
    T* yb = static_cast<T*>(p.y) + img * D;
    for (int e = tid; e < tokens * CH; e += nthreads) {
        const int tok = e / CH, cc = e - tok * CH;
        const int dd = c0 + cc;
        if (dd >= D) continue;
        float acc = 0.f;
#pragma unroll
        for (int pl = 0; pl < PLANES; ++pl) acc += sY[(size_t)pl * tokens * CH + e];
        float o = acc * p.merge_scale;
        if (zb) o *= silu_f(z_staged ? sZ[e] : load_elem<T>(zb + (long long)tok * D + dd));
        store_elem<T>(yb + (long long)tok * D + dd, o);
    }
}

}  // namespace vscan
