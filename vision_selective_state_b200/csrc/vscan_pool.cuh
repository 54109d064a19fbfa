// Pooled route (FastVim): POOL_W and POOL_H.
//
// "Fast Vision Mamba: Pooling Spatial Dimensions for Accelerated Processing",
// Methodology: reshape the tokens to (h, w), mean-pool one spatial axis, run the
// forward and backward selective scans on the pooled tokens only, repeat the
// outputs along the pooled axis. The gate uses the un-pooled z of each token.
//
// Two kernels:
//   pool_bc_kernel    mean-pools B and C (shared by all channels) into the
//                     workspace: [Ki][batch][Lp][N] float32 each.
//   pool_scan_kernel  one CTA per (image, 32-channel tile): pools u and raw
//                     Delta of the tile into shared memory (HBM stream), runs
//                     both scan directions on the Lp pooled steps, then streams
//                     the repeated, gated output over every grid token.
// The pooled-route memory traffic is the compulsory one: u, Delta and z read
// once, y written once; B and C are read once by the small pre-pass.
//
// Optional steps (template flags FL, as for the streaming kernel):
//   FL_ZOH   zero-order-hold write term (zoh_phi).
//   FL_CONV  u holds the convolution input x. Each direction's kernel-four causal
//            Conv1d + SiLU runs over the full token sequence before pooling
//            ("Fast Vision Mamba ...", Methodology: Conv1D, then mean-pool one
//            axis; "Vision Mamba ...", "Inside the released Vim block": the
//            backward branch convolves the reversed sequence). The sequence is
//            the row-major (POOL_W) or column-major (POOL_H) token order, so the
//            members of one pooled index are consecutive in it.
//   FL_MASK  masked token set (FastMaskVim, "Fast Vision Mamba ...", Innovation
//            and Methodology: sparse indexing, mask-aware aggregation, row sums
//            normalized by the nominal width). The token arrays hold n_tok
//            visible tokens with their grid positions pos[]; pooling adds every
//            visible token into its row (column) with shared-memory (u, Delta)
//            and global (B, C; pool_bc_masked_kernel) float atomics, and the sums
//            are divided by the nominal w (h). The repeat writes each visible
//            token from its row (column). Positions outside the grid are skipped
//            and their y written as 0.
#pragma once

#include "vscan_common.cuh"
#include "vscan_route.cuh"

namespace vscan {

struct PoolParams {
    RouteGeom g;
    int batch, D, N, Ki;
    const void* u;
    const void* delta;
    const void* B;
    const void* C;
    const void* z;
    void* y;
    const float* A;
    const float* Dskip;
    const float* bias;
    long long in_dir;
    long long bc_dir;
    int a_dir;
    int v_dir;
    int softplus;
    float merge_scale;
    float* pB;  // [Ki][batch][Lp][N]
    float* pC;  // [Ki][batch][Lp][N]
    const float* conv_w;  // FL_CONV: [Kp][D][4]
    const float* conv_b;  // FL_CONV: [Kp][D] (nullable)
    const int* pos;       // FL_MASK: [batch][n_tok] grid positions
    int n_tok;            // tokens per image in the token arrays (h*w when dense)
};

// FL_MASK: pooled index of grid position q, or -1 outside the grid.
__device__ __forceinline__ int pool_index(const RouteGeom& g, int q)
{
    if (q < 0 || q >= g.h * g.w) return -1;
    const int r = q / g.w;
    return (g.kind == RK_POOL_W) ? r : q - r * g.w;
}

// FL_MASK: sums of B and C over the visible tokens of every pooled index, added
// into the zeroed workspace ([Ki][batch][Lp][N]) with global float atomics; the
// scan divides them by the nominal width. Grid (splits, batch, Ki), 256
// threads: thread (range r = tid >> 4, state n = tid & 15) walks a contiguous
// range of PB_RUN tokens, sums consecutive tokens of one pooled index in
// registers (one row of a sorted mask) and adds each run once.
constexpr int PB_RUN = 16;
template <typename T>
__global__ void __launch_bounds__(256) pool_bc_masked_kernel(const PoolParams p)
{
    const int b = blockIdx.y, k = blockIdx.z, N = p.N;
    const int n = threadIdx.x & 15;
    const long long r = (long long)blockIdx.x * 16 + (threadIdx.x >> 4);
    const long long tb = r * PB_RUN;
    if (n >= N || tb >= p.n_tok) return;
    const int te = (int)min((long long)p.n_tok, tb + PB_RUN);
    const int* pb = p.pos + (long long)b * p.n_tok;
    const T* Bb = static_cast<const T*>(p.B) + k * p.bc_dir + (long long)b * p.n_tok * N + n;
    const T* Cb = static_cast<const T*>(p.C) + k * p.bc_dir + (long long)b * p.n_tok * N + n;
    float* oB = p.pB + ((long long)k * p.batch + b) * p.g.L * N + n;
    float* oC = p.pC + ((long long)k * p.batch + b) * p.g.L * N + n;
    int cur = -1;
    float sb = 0.f, sc = 0.f;
    constexpr int U = 8;
    for (int t0 = (int)tb; t0 < te; t0 += U) {
        int ix[U];
        float vb[U], vc[U];
#pragma unroll
        for (int v = 0; v < U; ++v) {  // loads first
            const int t = t0 + v;
            const bool in = t < te;
            ix[v] = in ? __ldg(pb + t) : -1;
            vb[v] = in ? load_elem<T>(Bb + (long long)t * N) : 0.f;
            vc[v] = in ? load_elem<T>(Cb + (long long)t * N) : 0.f;
        }
#pragma unroll
        for (int v = 0; v < U; ++v) {
            const int i = pool_index(p.g, ix[v]);
            if (i < 0) continue;
            if (i != cur) {
                if (cur >= 0) {
                    atomicAdd(oB + (long long)cur * N, sb);
                    atomicAdd(oC + (long long)cur * N, sc);
                }
                cur = i;
                sb = 0.f;
                sc = 0.f;
            }
            sb += vb[v];
            sc += vc[v];
        }
    }
    if (cur >= 0) {
        atomicAdd(oB + (long long)cur * N, sb);
        atomicAdd(oC + (long long)cur * N, sc);
    }
}

constexpr int PL_CH = 32;       // channels per CTA
constexpr int PL_THREADS = 256;

// Token of the grid that is the j-th member of pooled index i.
__device__ __forceinline__ int pool_member(const RouteGeom& g, int i, int j)
{
    return (g.kind == RK_POOL_W) ? i * g.w + j : j * g.w + i;
}

template <typename T>
__global__ void __launch_bounds__(128) pool_bc_kernel(const PoolParams p)
{
    __shared__ float part_b[8][16];
    __shared__ float part_c[8][16];
    const int i = blockIdx.x, b = blockIdx.y, k = blockIdx.z;
    const int n = threadIdx.x & 15, jl = threadIdx.x >> 4;
    const int N = p.N;
    const int cnt = (p.g.kind == RK_POOL_W) ? p.g.w : p.g.h;
    const long long img = (long long)b * p.g.tokens;
    const T* Bb = static_cast<const T*>(p.B) + k * p.bc_dir + img * N;
    const T* Cb = static_cast<const T*>(p.C) + k * p.bc_dir + img * N;
    float sb = 0.f, sc = 0.f;
    if (n < N) {
        for (int j = jl; j < cnt; j += 8) {
            const long long tok = pool_member(p.g, i, j);
            sb += load_elem<T>(Bb + tok * N + n);
            sc += load_elem<T>(Cb + tok * N + n);
        }
    }
    part_b[jl][n] = sb;
    part_c[jl][n] = sc;
    __syncthreads();
    if (jl == 0 && n < N) {
        float tb = 0.f, tc = 0.f;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            tb += part_b[q][n];
            tc += part_c[q][n];
        }
        const float inv = 1.0f / (float)cnt;
        const long long o = (((long long)k * p.batch + b) * p.g.L + i) * N + n;
        p.pB[o] = tb * inv;
        p.pC[o] = tc * inv;
    }
}

// Dynamic shared memory (floats): pd[Ki][Lp][32] (pooled raw Delta),
// pu[Ku][Lp][32] (pooled u; Ku = 2 with the convolution, whose output differs
// per direction, else Ki), Y[2][Lp][32] (per-direction outputs).
inline size_t pool_scan_smem_bytes(int Ki, int Lp, bool conv = false)
{
    const int Ku = conv ? 2 : Ki;
    return sizeof(float) * (size_t)(Ki + Ku + 2) * Lp * PL_CH;
}

// Three CTAs per SM (80 registers) where shared memory allows them; two for the
// convolution and the mask (128 registers), whose phase 1 holds more state.
template <typename T, int FL>
__global__ void __launch_bounds__(PL_THREADS, (FL & (FL_CONV | FL_MASK)) ? 2 : 3) pool_scan_kernel(const PoolParams p)
{
    constexpr bool ZOH = (FL & FL_ZOH) != 0;
    constexpr bool CONV = (FL & FL_CONV) != 0;
    constexpr bool MASK = (FL & FL_MASK) != 0;
    static_assert(!(CONV && MASK), "no convolution order is defined on a masked token set");
    extern __shared__ __align__(16) float psm[];
    const int Lp = p.g.L;
    const int Ki = p.Ki;
    const int Ku = CONV ? 2 : Ki;
    float* pd = psm;                          // [Ki][Lp][32]
    float* pu = psm + (size_t)Ki * Lp * PL_CH;  // [Ku][Lp][32]
    float* Y = pu + (size_t)Ku * Lp * PL_CH;    // [2][Lp][32]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int b = blockIdx.y;
    const int c0 = blockIdx.x * PL_CH;
    const int D = p.D, N = p.N;
    const int tokens = p.n_tok;
    const long long img = (long long)b * tokens;
    const int cnt = (p.g.kind == RK_POOL_W) ? p.g.w : p.g.h;
    const float inv_cnt = 1.0f / (float)cnt;

    // ---- phase 1 (FL_CONV): convolve along the token sequence, then pool -------
    if constexpr (CONV) {
        const int jl = lane >> 3;   // run of consecutive members 0..3
        const int q = lane & 7;     // channel quad of the tile
        const int ch = c0 + 4 * q;
        const bool cval = ch < D;
        const long long g_tok = (long long)p.g.h * p.g.w;
        const int run = (cnt + 3) / 4;
        const int jb = jl * run, je = min(cnt, jb + run);
        for (int k = 0; k < Ki; ++k) {
            // directions whose convolution reads this input plane
            const int dlo = (Ki == 1) ? 0 : k, dhi = (Ki == 1) ? 1 : k;
            float kw[2][4][4], kb[2][4];  // [direction][tap][channel of the quad]
#pragma unroll
            for (int dd = 0; dd < 2; ++dd)
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    const int dr = dd == 0 ? dlo : dhi;
                    const long long o = (long long)dr * p.v_dir + ch + cc;
#pragma unroll
                    for (int i = 0; i < 4; ++i) kw[dd][i][cc] = cval ? __ldg(p.conv_w + o * 4 + i) : 0.f;
                    kb[dd][cc] = (cval && p.conv_b) ? __ldg(p.conv_b + o) : 0.f;
                }
            const T* xb = static_cast<const T*>(p.u) + k * p.in_dir + img * D + ch;
            const T* db = static_cast<const T*>(p.delta) + k * p.in_dir + img * D + ch;
            // Sequence position sq <-> token: POOL_W walks the tokens in order
            // (sq = token); POOL_H walks the columns (sq = col * h + row). The
            // loads of a run advance one position at a time, so the token index
            // is carried along instead of divided out.
            const bool colmajor = p.g.kind == RK_POOL_H;
            auto xat = [&](int tok, bool in) {
                return (cval && in) ? load4<T>(xb + (long long)tok * D) : make_float4(0.f, 0.f, 0.f, 0.f);
            };
            for (int i = warp; i < Lp; i += PL_THREADS / 32) {
                float4 au0 = make_float4(0.f, 0.f, 0.f, 0.f), au1 = au0, ad = au0;
                // position of the first window entry, s0 - 3, as (sequence index, row, col)
                int sq = i * cnt + jb - 3;
                int row, col;
                if (colmajor) { col = (sq + 3) / p.g.h; row = (sq + 3) - col * p.g.h - 3; }
                else { row = (sq + 3) / p.g.w; col = (sq + 3) - row * p.g.w - 3; }
                // normalize a negative offset within the row (POOL_W) or column (POOL_H)
                if (colmajor) { while (row < 0) { row += p.g.h; --col; } }
                else { while (col < 0) { col += p.g.w; --row; } }
                auto advance = [&]() {
                    ++sq;
                    if (colmajor) { if (++row == p.g.h) { row = 0; ++col; } }
                    else { if (++col == p.g.w) { col = 0; ++row; } }
                };
                // x at s-3 .. s+6 for a group of four members s .. s+3
                float4 win[10];
#pragma unroll
                for (int m = 0; m < 6; ++m) {
                    win[m] = xat(row * p.g.w + col, sq >= 0 && sq < g_tok);
                    advance();
                }
                for (int j = jb; j < je; j += 4) {
                    // loads first: the next four window entries and four raw Deltas
                    float4 dl[4];
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        win[6 + v] = xat(row * p.g.w + col, sq < g_tok);
                        advance();
                        dl[v] = (cval && j + v < je) ? load4<T>(db + (long long)pool_member(p.g, i, j + v) * D)
                                                     : make_float4(0.f, 0.f, 0.f, 0.f);
                    }
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        if (j + v >= je) break;
                        ad.x += dl[v].x; ad.y += dl[v].y; ad.z += dl[v].z; ad.w += dl[v].w;
                        const float* wv = reinterpret_cast<const float*>(win + v);  // x[s + v - 3 ..]
                        float f[4], bk[4];
#pragma unroll
                        for (int cc = 0; cc < 4; ++cc) {
                            float a0 = kb[0][cc], a1 = kb[1][cc];
#pragma unroll
                            for (int t = 0; t < 4; ++t) {
                                a0 = fmaf(kw[0][t][cc], wv[4 * t + cc], a0);        // x[s - 3 + t]
                                a1 = fmaf(kw[1][t][cc], wv[4 * (6 - t) + cc], a1);  // x[s + 3 - t]
                            }
                            f[cc] = silu_f(a0);
                            bk[cc] = silu_f(a1);
                        }
                        if (Ki == 1 || k == 0) { au0.x += f[0]; au0.y += f[1]; au0.z += f[2]; au0.w += f[3]; }
                        if (Ki == 1 || k == 1) { au1.x += bk[0]; au1.y += bk[1]; au1.z += bk[2]; au1.w += bk[3]; }
                    }
#pragma unroll
                    for (int m = 0; m < 6; ++m) win[m] = win[m + 4];
                }
#pragma unroll
                for (int m = 8; m <= 16; m <<= 1) {
                    au0.x += __shfl_xor_sync(FULL_MASK, au0.x, m);
                    au0.y += __shfl_xor_sync(FULL_MASK, au0.y, m);
                    au0.z += __shfl_xor_sync(FULL_MASK, au0.z, m);
                    au0.w += __shfl_xor_sync(FULL_MASK, au0.w, m);
                    au1.x += __shfl_xor_sync(FULL_MASK, au1.x, m);
                    au1.y += __shfl_xor_sync(FULL_MASK, au1.y, m);
                    au1.z += __shfl_xor_sync(FULL_MASK, au1.z, m);
                    au1.w += __shfl_xor_sync(FULL_MASK, au1.w, m);
                    ad.x += __shfl_xor_sync(FULL_MASK, ad.x, m);
                    ad.y += __shfl_xor_sync(FULL_MASK, ad.y, m);
                    ad.z += __shfl_xor_sync(FULL_MASK, ad.z, m);
                    ad.w += __shfl_xor_sync(FULL_MASK, ad.w, m);
                }
                if (jl == 0) {
                    float* dd_ = pd + ((size_t)k * Lp + i) * PL_CH + 4 * q;
                    dd_[0] = ad.x * inv_cnt; dd_[1] = ad.y * inv_cnt; dd_[2] = ad.z * inv_cnt; dd_[3] = ad.w * inv_cnt;
                    if (Ki == 1 || k == 0) {
                        float* u0 = pu + ((size_t)0 * Lp + i) * PL_CH + 4 * q;
                        u0[0] = au0.x * inv_cnt; u0[1] = au0.y * inv_cnt; u0[2] = au0.z * inv_cnt; u0[3] = au0.w * inv_cnt;
                    }
                    if (Ki == 1 || k == 1) {
                        float* u1 = pu + ((size_t)1 * Lp + i) * PL_CH + 4 * q;
                        u1[0] = au1.x * inv_cnt; u1[1] = au1.y * inv_cnt; u1[2] = au1.z * inv_cnt; u1[3] = au1.w * inv_cnt;
                    }
                }
            }
        }
    }

    // ---- phase 1 (FL_MASK): add every visible token into its pooled index -----
    if constexpr (MASK) {
        for (int e = tid; e < (Ki + Ku) * Lp * PL_CH; e += PL_THREADS) psm[e] = 0.f;
        __syncthreads();
        const int q = lane & 7;        // channel quad of the tile
        const int ch = c0 + 4 * q;
        if (ch < D) {
            const int* pb = p.pos + (long long)b * tokens;
            for (int k = 0; k < Ki; ++k) {
                const T* ub = static_cast<const T*>(p.u) + k * p.in_dir + img * D + ch;
                const T* db = static_cast<const T*>(p.delta) + k * p.in_dir + img * D + ch;
                // Lane group g (tid >> 3, 32 groups) adds the contiguous token range
                // [g*tokens/32, (g+1)*tokens/32): the four groups of a warp are far
                // apart, so their atomics rarely meet, and consecutive tokens of one
                // row (the usual sorted mask) are summed in registers and added once.
                constexpr int G = PL_THREADS / 8, U = 8;
                const int g = tid >> 3;
                const int tb = (int)((long long)tokens * g / G), te = (int)((long long)tokens * (g + 1) / G);
                int cur = -1;
                float4 su = make_float4(0.f, 0.f, 0.f, 0.f), sd = su;
                auto flush = [&]() {
                    if (cur < 0) return;
                    float* du_ = pu + ((size_t)k * Lp + cur) * PL_CH + 4 * q;
                    float* dd_ = pd + ((size_t)k * Lp + cur) * PL_CH + 4 * q;
                    atomicAdd(du_ + 0, su.x); atomicAdd(du_ + 1, su.y); atomicAdd(du_ + 2, su.z); atomicAdd(du_ + 3, su.w);
                    atomicAdd(dd_ + 0, sd.x); atomicAdd(dd_ + 1, sd.y); atomicAdd(dd_ + 2, sd.z); atomicAdd(dd_ + 3, sd.w);
                };
                for (int t0 = tb; t0 < te; t0 += U) {
                    int ix[U];
                    float4 u4[U], d4[U];
#pragma unroll
                    for (int v = 0; v < U; ++v) {  // loads first
                        const int t = t0 + v;
                        const bool in = t < te;
                        ix[v] = in ? __ldg(pb + t) : -1;
                        u4[v] = in ? load4<T>(ub + (long long)t * D) : make_float4(0.f, 0.f, 0.f, 0.f);
                        d4[v] = in ? load4<T>(db + (long long)t * D) : make_float4(0.f, 0.f, 0.f, 0.f);
                    }
#pragma unroll
                    for (int v = 0; v < U; ++v) {
                        const int i = pool_index(p.g, ix[v]);
                        if (i < 0) continue;
                        if (i != cur) {
                            flush();
                            cur = i;
                            su = make_float4(0.f, 0.f, 0.f, 0.f);
                            sd = su;
                        }
                        su.x += u4[v].x; su.y += u4[v].y; su.z += u4[v].z; su.w += u4[v].w;
                        sd.x += d4[v].x; sd.y += d4[v].y; sd.z += d4[v].z; sd.w += d4[v].w;
                    }
                }
                flush();
            }
        }
        __syncthreads();
        for (int e = tid; e < (Ki + Ku) * Lp * PL_CH; e += PL_THREADS) psm[e] *= inv_cnt;
    }

    // ---- phase 1: mean-pool u and raw Delta of the channel tile ---------------
    if constexpr (!CONV && !MASK) {
        const int jl = lane >> 3;   // token sub-lane 0..3
        const int q = lane & 7;     // channel quad of the tile
        const int ch = c0 + 4 * q;
        const bool cval = ch < D;
        for (int k = 0; k < Ki; ++k) {
            const T* ub = static_cast<const T*>(p.u) + k * p.in_dir + img * D + ch;
            const T* db = static_cast<const T*>(p.delta) + k * p.in_dir + img * D + ch;
            for (int i = warp; i < Lp; i += PL_THREADS / 32) {
                float4 au = make_float4(0.f, 0.f, 0.f, 0.f), ad = au;
                if (cval) {
                    int j = jl;
                    for (; j + 12 < cnt; j += 16) {
                        float4 u4[4], d4[4];
#pragma unroll
                        for (int r = 0; r < 4; ++r) {
                            const long long tok = pool_member(p.g, i, j + 4 * r);
                            u4[r] = load4<T>(ub + tok * D);
                            d4[r] = load4<T>(db + tok * D);
                        }
#pragma unroll
                        for (int r = 0; r < 4; ++r) {
                            au.x += u4[r].x; au.y += u4[r].y; au.z += u4[r].z; au.w += u4[r].w;
                            ad.x += d4[r].x; ad.y += d4[r].y; ad.z += d4[r].z; ad.w += d4[r].w;
                        }
                    }
                    for (; j < cnt; j += 4) {
                        const long long tok = pool_member(p.g, i, j);
                        const float4 u1 = load4<T>(ub + tok * D);
                        const float4 d1 = load4<T>(db + tok * D);
                        au.x += u1.x; au.y += u1.y; au.z += u1.z; au.w += u1.w;
                        ad.x += d1.x; ad.y += d1.y; ad.z += d1.z; ad.w += d1.w;
                    }
                }
#pragma unroll
                for (int m = 8; m <= 16; m <<= 1) {
                    au.x += __shfl_xor_sync(FULL_MASK, au.x, m);
                    au.y += __shfl_xor_sync(FULL_MASK, au.y, m);
                    au.z += __shfl_xor_sync(FULL_MASK, au.z, m);
                    au.w += __shfl_xor_sync(FULL_MASK, au.w, m);
                    ad.x += __shfl_xor_sync(FULL_MASK, ad.x, m);
                    ad.y += __shfl_xor_sync(FULL_MASK, ad.y, m);
                    ad.z += __shfl_xor_sync(FULL_MASK, ad.z, m);
                    ad.w += __shfl_xor_sync(FULL_MASK, ad.w, m);
                }
                if (jl == 0) {
                    float* du_ = pu + ((size_t)k * Lp + i) * PL_CH + 4 * q;
                    float* dd_ = pd + ((size_t)k * Lp + i) * PL_CH + 4 * q;
                    du_[0] = au.x * inv_cnt; du_[1] = au.y * inv_cnt; du_[2] = au.z * inv_cnt; du_[3] = au.w * inv_cnt;
                    dd_[0] = ad.x * inv_cnt; dd_[1] = ad.y * inv_cnt; dd_[2] = ad.z * inv_cnt; dd_[3] = ad.w * inv_cnt;
                }
            }
        }
    }
    __syncthreads();

    // ---- phase 2: both directions over the Lp pooled steps ----------------------
    {
        const int kd = warp >> 2;          // direction 0 (forward) / 1 (backward)
        const int cg = warp & 3;           // 8-channel group of the tile
        const int ki = (Ki > 1) ? kd : 0;  // input plane
        const int cc = lane >> 2, grp = lane & 3;
        const int c = 8 * cg + cc;
        const int d = c0 + c;
        const bool dvalid = d < D;
        float a2[4];
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            const int n = 4 * grp + s;
            a2[s] = (dvalid && n < N) ? __ldg(p.A + (long long)kd * p.a_dir + (long long)d * N + n) * LOG2E : 0.f;
        }
        const float Dd = (dvalid && p.Dskip) ? __ldg(p.Dskip + kd * p.v_dir + d) : 0.f;
        const float bias = (dvalid && p.bias) ? __ldg(p.bias + kd * p.v_dir + d) : 0.f;
        const float* pBk = p.pB + ((long long)ki * p.batch + b) * Lp * N;
        const float* pCk = p.pC + ((long long)ki * p.batch + b) * Lp * N;
        const float* pdk = pd + (size_t)ki * Lp * PL_CH;
        const float* puk = pu + (size_t)(CONV ? kd : ki) * Lp * PL_CH;
        float ia[4];  // ZOH: 1 / A per state (0 for A = 0)
#pragma unroll
        for (int s = 0; s < 4; ++s) ia[s] = (a2[s] != 0.f) ? LOG2E / a2[s] : 0.f;
        float* Yk = Y + (size_t)kd * Lp * PL_CH;
        float h[4] = {0.f, 0.f, 0.f, 0.f};
        // B and C of the lane's four states as 16-byte quads (N = 16), else per state
        const bool quad = N == 16;
        for (int t0 = 0; t0 < Lp; t0 += 4) {
            // the four steps' loads first (a step past the end re-reads step
            // Lp - 1 and is not applied): the pooled B and C come from L2, and a
            // load per step behind the previous step's update would cost one L2
            // round trip per step
            float xs[4], us[4];
            float4 bq[4], cq[4];
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                const int t = min(t0 + jj, Lp - 1);
                const int i = kd == 0 ? t : Lp - 1 - t;
                xs[jj] = pdk[(size_t)i * PL_CH + c];
                us[jj] = puk[(size_t)i * PL_CH + c];
                if (quad) {
                    bq[jj] = __ldg(reinterpret_cast<const float4*>(pBk + (size_t)i * 16 + 4 * grp));
                    cq[jj] = __ldg(reinterpret_cast<const float4*>(pCk + (size_t)i * 16 + 4 * grp));
                } else {
                    float bb[4], cc4[4];
#pragma unroll
                    for (int s = 0; s < 4; ++s) {
                        const int n = 4 * grp + s;
                        bb[s] = n < N ? __ldg(pBk + (size_t)i * N + n) : 0.f;
                        cc4[s] = n < N ? __ldg(pCk + (size_t)i * N + n) : 0.f;
                    }
                    bq[jj] = make_float4(bb[0], bb[1], bb[2], bb[3]);
                    cq[jj] = make_float4(cc4[0], cc4[1], cc4[2], cc4[3]);
                }
            }
            float yp[4];
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                const bool live = t0 + jj < Lp;
                // Delta = softplus(mean raw Delta + bias): the bias and
                // softplus act on the pooled token.
                const float x = xs[jj] + bias;
                const float dsp = p.softplus ? softplus_f(x) : x;
                const float du = dsp * us[jj];
                float bv[4] = {bq[jj].x, bq[jj].y, bq[jj].z, bq[jj].w};
                float cv[4] = {cq[jj].x, cq[jj].y, cq[jj].z, cq[jj].w};
                if constexpr (MASK) {
#pragma unroll
                    for (int s = 0; s < 4; ++s) { bv[s] *= inv_cnt; cv[s] *= inv_cnt; }  // sums -> means
                }
                const float rd = ZOH ? fast_rcp(dsp) : 0.f;
                float acc = 0.f;
#pragma unroll
                for (int s = 0; s < 4; ++s) {
                    const float e = fast_exp2(dsp * a2[s]);
                    float w = du * bv[s];
                    if constexpr (ZOH) w *= zoh_phi(dsp * a2[s] * LN2, e, rd * ia[s]);
                    const float hn = fmaf(e, h[s], w);
                    h[s] = live ? hn : h[s];
                    acc = fmaf(cv[s], h[s], acc);
                }
                yp[jj] = live ? acc : 0.f;
            }
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
            const int t = t0 + grp;
            if (t < Lp) {
                const int i = kd == 0 ? t : Lp - 1 - t;
                Yk[(size_t)i * PL_CH + c] = fmaf(Dd, puk[(size_t)i * PL_CH + c], keep);
            }
        }
    }
    __syncthreads();

    // ---- phase 3: repeat over the pooled axis, merge, gate, store ---------------
    // Eight tokens per thread per round, loads first, so that each thread keeps
    // 128 bytes of z in flight.
    {
        constexpr int U = 8;
        const int q = tid & 7;        // channel quad
        const int tl = tid >> 3;      // token lane 0..31
        const int ch = c0 + 4 * q;
        if (ch < D) {
            const float* Y0 = Y;
            const float* Y1 = Y + (size_t)Lp * PL_CH;
            const T* zb = p.z ? static_cast<const T*>(p.z) + img * D + ch : nullptr;
            T* yb = static_cast<T*>(p.y) + img * D + ch;
            const float scale = p.merge_scale;
            for (int tok0 = tl; tok0 < tokens; tok0 += 32 * U) {
                float4 zz[U];
                int mp[U];  // FL_MASK: grid positions, loaded with z
#pragma unroll
                for (int v = 0; v < U; ++v) {
                    const int tok = tok0 + 32 * v;
                    zz[v] = (zb && tok < tokens) ? load4<T>(zb + (long long)tok * D) : make_float4(0.f, 0.f, 0.f, 0.f);
                    if constexpr (MASK) mp[v] = tok < tokens ? __ldg(p.pos + (long long)b * tokens + tok) : -1;
                }
#pragma unroll
                for (int v = 0; v < U; ++v) {
                    const int tok = tok0 + 32 * v;
                    if (tok >= tokens) break;
                    int i;
                    if constexpr (MASK) {
                        i = pool_index(p.g, mp[v]);
                        if (i < 0) {  // outside the grid: written as 0
                            store4<T>(yb + (long long)tok * D, make_float4(0.f, 0.f, 0.f, 0.f));
                            continue;
                        }
                    } else {
                        const int r = tok / p.g.w;
                        const int col = tok - r * p.g.w;
                        i = (p.g.kind == RK_POOL_W) ? r : col;
                    }
                    const float4 f = *reinterpret_cast<const float4*>(Y0 + (size_t)i * PL_CH + 4 * q);
                    const float4 g = *reinterpret_cast<const float4*>(Y1 + (size_t)i * PL_CH + 4 * q);
                    float4 o = make_float4((f.x + g.x) * scale, (f.y + g.y) * scale,
                                           (f.z + g.z) * scale, (f.w + g.w) * scale);
                    if (zb) {
                        o.x *= silu_f(zz[v].x); o.y *= silu_f(zz[v].y);
                        o.z *= silu_f(zz[v].z); o.w *= silu_f(zz[v].w);
                    }
                    store4<T>(yb + (long long)tok * D, o);
                }
            }
        }
    }
}

}  // namespace vscan
