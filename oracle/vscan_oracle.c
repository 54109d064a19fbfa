/*
 * vscan_oracle.c -- plain fp64 CPU oracle for the routed visual selective scan.
 *
 * TEST INFRASTRUCTURE ONLY. This file is the slow, obviously-correct statement
 * of what the routed selective scan computes. It is used by the tests, by
 * __graft_entry__.smoke() and by the cpu_baseline / reference legs of bench.py,
 * and by nothing else. It shares no code, header, table or helper with the
 * CUDA library under vision_selective_state_b200/csrc, and it never calls it.
 *
 * Every step follows the pages it cites, in their order and notation:
 *
 *   [Vim]   "Vision Mamba: Bidirectional State Space Models for Images"
 *           (abhik.ai review): sec. 3 "Choose the state update from the current
 *           content", sec. 4 "Keep a running state, then read it", sec. 5 "Align
 *           the backward scan before combining", and the prose section "Two
 *           scans meet at the same token".
 *   [EVM]   "EfficientVMamba: Atrous Selective Scan for Light Weight Visual
 *           Mamba" (abhik.ai review): sec. 1 "Gather spatial residues into
 *           ordered streams", sec. 2 "Update an independent state inside each
 *           group", sec. 3 "Invert the routing, then crop the padding", and the
 *           prose section "Merge restores coordinates instead of adding
 *           directions".
 *   [FVim]  "Fast Vision Mamba: Pooling Spatial Dimensions for Accelerated
 *           Processing" (gptget.net summary): "Methodology" list.
 *   [NoD]   "Norm or Direction? Decoding Vision Mambas for High-Resolution
 *           Vision": sec. 3 Background, Eq. 1-2 and "2D Selective Scan (SS2D)".
 *
 * Readings taken where the pages are silent or ambiguous (each one is listed
 * with its reason in the design notes at the repository root):
 *   - merge of several directions: summed, then multiplied by merge_scale
 *     (1 = sum as in SS2D and Vim's Algorithm 1; 0.5 = the released Vim average);
 *   - atrous padding slots carry u = rawDelta = B = C = 0, so Delta is
 *     softplus(bias) and the state still decays across them;
 *   - pooled route: u, rawDelta, B and C are mean-pooled over the pooled axis
 *     before the bias and softplus; the whole scan (including D*u) runs on the
 *     pooled tokens; the result is repeated over the pooled axis and then gated
 *     with the un-pooled z of every grid token;
 *   - input write is Delta*B*u (the released convention) unless the zero-order
 *     hold flag asks for the exact integral of [NoD] Eq. 2;
 *   - softplus is the exact log(1 + e^x), evaluated without a threshold;
 *   - fused convolution: u holds the convolution input; each direction applies
 *     its own kernel-four causal Conv1d + SiLU along its own sequence order
 *     (BIDIR: the route; pooled routes: the row-major (POOL_W) or column-major
 *     (POOL_H) token order, reversed for the backward direction) before any
 *     pooling; the skip term D*u uses the convolved (and pooled) u.
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Route kinds. The numbering is part of the oracle's own interface. */
#define OR_BIDIR 0   /* [Vim] forward + whole-sequence reverse               */
#define OR_CROSS4 1  /* [NoD] SS2D: row fwd, row rev, column fwd, column rev  */
#define OR_ATROUS2 2 /* [EVM] p=2 residue groups, right/bottom zero padding   */
#define OR_POOL_W 3  /* [FVim] mean over columns -> length h, fwd + bwd      */
#define OR_POOL_H 4  /* [FVim] mean over rows    -> length w, fwd + bwd      */

#define OR_OK 0
#define OR_EINVAL -1
#define OR_ENOMEM -6
#define OR_EOWNER -9 /* a real pixel was written by zero or by two atrous streams */

/* ------------------------------------------------------------------------- */
/* Geometry: number of directions K, sequence length L per direction and the  */
/* number of tokens per image in the token array (grid + optional CLS).        */
/* ------------------------------------------------------------------------- */
int oracle_geometry(int kind, int h, int w, int cls_pos, int* K, int* L, int* tokens)
{
    if (h <= 0 || w <= 0) return OR_EINVAL;
    int hw = h * w;
    switch (kind) {
    case OR_BIDIR:
        /* [Vim] "Insert the class token": CLS sits at floor(P/2) of the P
         * patches, giving P + 1 tokens; both scans run over all of them. */
        if (cls_pos != -1 && cls_pos != hw / 2) return OR_EINVAL;
        *K = 2;
        *tokens = hw + (cls_pos >= 0 ? 1 : 0);
        *L = *tokens;
        return OR_OK;
    case OR_CROSS4:
        if (cls_pos != -1) return OR_EINVAL;
        *K = 4; *L = hw; *tokens = hw;
        return OR_OK;
    case OR_ATROUS2:
        if (cls_pos != -1) return OR_EINVAL;
        /* [EVM] sec. 1: four lists of ceil(H/2) x ceil(W/2). */
        *K = 4; *L = ((h + 1) / 2) * ((w + 1) / 2); *tokens = hw;
        return OR_OK;
    case OR_POOL_W:
        if (cls_pos != -1) return OR_EINVAL;
        *K = 2; *L = h; *tokens = hw;
        return OR_OK;
    case OR_POOL_H:
        if (cls_pos != -1) return OR_EINVAL;
        *K = 2; *L = w; *tokens = hw;
        return OR_OK;
    default:
        return OR_EINVAL;
    }
}

/*
 * Route coordinates, written as explicit coordinate loops.
 * out[k*L + t] = index (into the token array, or into the pooled sequence for
 * the pooled routes) visited by step t of direction k, or -1 for a padding slot.
 */
int oracle_route(int kind, int h, int w, int cls_pos, int64_t* out)
{
    int K, L, tokens;
    int rc = oracle_geometry(kind, h, w, cls_pos, &K, &L, &tokens);
    if (rc != OR_OK) return rc;

    if (kind == OR_BIDIR || kind == OR_POOL_W || kind == OR_POOL_H) {
        /* [Vim] "Two scans meet at the same token": the forward scan takes the
         * sequence in order, the backward scan the entire reversed sequence. */
        for (int t = 0; t < L; ++t) {
            out[0 * L + t] = t;
            out[1 * L + t] = L - 1 - t;
        }
        return OR_OK;
    }

    if (kind == OR_CROSS4) {
        /* [NoD] SS2D: the four traversals are the row-major order, its reverse,
         * the column-major order and its reverse. Tokens are stored row-major
         * (columns fastest), as the Vim patch flattening fixes. */
        int64_t* row = out + 0 * (int64_t)L;
        int64_t* col = out + 2 * (int64_t)L;
        int t = 0;
        for (int r = 0; r < h; ++r)
            for (int c = 0; c < w; ++c) row[t++] = (int64_t)r * w + c;
        t = 0;
        for (int c = 0; c < w; ++c)
            for (int r = 0; r < h; ++r) col[t++] = (int64_t)r * w + c;
        for (int s = 0; s < L; ++s) {
            out[1 * (int64_t)L + s] = row[L - 1 - s];
            out[3 * (int64_t)L + s] = col[L - 1 - s];
        }
        return OR_OK;
    }

    /* OR_ATROUS2. [EVM] sec. 1: O_k[t] = X[2 r_t + m_k, 2 c_t + n_k] with
     * offsets (m_k, n_k) = (0,0), (1,0), (0,1), (1,1) in (row, column); groups
     * 0 and 2 walk their residue sub-grid row-major, groups 1 and 3 walk it
     * column-major; coordinates beyond the H x W map are right/bottom padding. */
    const int dy[4] = {0, 1, 0, 1};
    const int dx[4] = {0, 0, 1, 1};
    int rows = (h + 1) / 2, cols = (w + 1) / 2;
    for (int k = 0; k < 4; ++k) {
        int t = 0;
        if (k == 0 || k == 2) {
            for (int a = 0; a < rows; ++a)
                for (int b = 0; b < cols; ++b) {
                    int y = 2 * a + dy[k], x = 2 * b + dx[k];
                    out[(int64_t)k * L + t++] = (y < h && x < w) ? (int64_t)y * w + x : -1;
                }
        } else {
            for (int a = 0; a < cols; ++a)
                for (int b = 0; b < rows; ++b) {
                    int y = 2 * b + dy[k], x = 2 * a + dx[k];
                    out[(int64_t)k * L + t++] = (y < h && x < w) ? (int64_t)y * w + x : -1;
                }
        }
    }
    return OR_OK;
}

/* softplus(x) = log(1 + e^x), evaluated as max(x, 0) + log1p(e^-|x|), which is
 * the same real function written so that no term overflows. [Vim] sec. 3. */
static double softplus(double x)
{
    return (x > 0.0 ? x : 0.0) + log1p(exp(-fabs(x)));
}

/* SiLU(z) = z * sigma(z), sigma(z) = 1 / (1 + e^-z). [Vim] sec. 5 and the
 * prose under "Inside the released Vim block". */
static double silu(double z)
{
    return z / (1.0 + exp(-z));
}

/*
 * One selective scan over one sequence of one channel, [Vim] sec. 4 and
 * [EVM] sec. 2:
 *     h_t = exp(dt_t * A) (.) h_{t-1} + dt_t * B_t * u_t,   h_{-1} = 0
 *     y_t = sum_n C_{t,n} h_{t,n} + D * u_t
 * dt is the already-discretized step (after bias and softplus).
 * B and C are [L][N]; A is [N]; u, dt, y are [L]. h is caller scratch [N].
 *
 * zoh != 0 replaces the write term by the exact zero-order-hold input
 * integral of [NoD] Eq. (2) (also the "discretization detail" paragraph of
 * [Vim] sec. 4): for the diagonal A of the scan,
 *     Bbar_n = (dt A_n)^-1 (exp(dt A_n) - 1) dt B_n = expm1(dt A_n) / A_n * B_n,
 * whose limit for A_n = 0 is dt B_n.
 */
void oracle_scan_sequence(int L, int N, const double* u, const double* dt, const double* A,
                          const double* B, const double* C, double D, int zoh, double* h,
                          double* y)
{
    for (int n = 0; n < N; ++n) h[n] = 0.0;
    for (int t = 0; t < L; ++t) {
        double read = 0.0;
        for (int n = 0; n < N; ++n) {
            double retention = exp(dt[t] * A[n]);
            double gain = dt[t];
            if (zoh && A[n] != 0.0) gain = expm1(dt[t] * A[n]) / A[n];
            double write = gain * B[(int64_t)t * N + n] * u[t];
            h[n] = retention * h[n] + write;
            read += C[(int64_t)t * N + n] * h[n];
        }
        y[t] = read + D * u[t];
    }
}

/*
 * Causal depthwise convolution of kernel size 4 followed by SiLU, at step s of
 * a sequence seq[0..]: SiLU(cb + sum_i cw[i] * seq[s - 3 + i]), with seq[<0] = 0
 * ([Vim] "Inside the released Vim block": kernel-four causal Conv1d, then SiLU;
 * "CPU backend substitutions": a grouped conv1d with left padding, then SiLU).
 */
static double causal_conv_silu(const double* seq, int64_t s, const double* cw, double cb)
{
    double acc = cb;
    for (int i = 0; i < 4; ++i) {
        int64_t j = s - 3 + i;
        if (j >= 0) acc += cw[i] * seq[j];
    }
    return silu(acc);
}

/*
 * Routed forward pass.
 *
 * Layouts (row-major, element strides):
 *   u, delta : [Ki][batch][tokens][D]   delta is the raw step, before bias/softplus
 *   B, C     : [Ki][batch][tokens][N]
 *   A        : [Kp][D][N]
 *   Dskip    : [Kp][D]      (nullable: no skip term)
 *   bias     : [Kp][D]      (nullable: no bias)
 *   z        : [batch][tokens][D] (nullable: no gate); the gate is shared by all
 *              directions ([Vim] "Inside the released Vim block").
 *   y        : [batch][tokens][D]   output
 *   conv_w   : [Kp][D][4]   (nullable: no convolution) -- with it, u holds the
 *              convolution's input x and every direction k runs
 *              u_k = SiLU(conv_k(x)) along its own sequence order before the
 *              scan ([Vim] "Inside the released Vim block": each branch has its
 *              own kernel-four causal Conv1d, the backward one on the reversed
 *              sequence; it crosses row boundaries as the sequence does). BIDIR
 *              convolves along the route; POOL_W / POOL_H convolve along the
 *              row-major / column-major token order (forward and reversed) and
 *              then pool the convolved values ([FVim] Methodology: Conv1D, then
 *              mean-pool one axis). ATROUS2 and CROSS4 take no convolution
 *              (OR_EINVAL): their pages convolve on the 2-D grid before routing.
 *   conv_b   : [Kp][D]      (nullable: zero)
 *   zoh      : 0 = dt * B * u write term; 1 = zero-order hold (oracle_scan_sequence)
 * Ki = K when per_dir_inputs, else 1; Kp = K when per_dir_params, else 1.
 * Every (batch, channel) pair is independent; channels and batches are
 * processed by OpenMP threads (nthreads <= 0: the OpenMP default).
 */
int oracle_forward(int kind, int h, int w, int cls_pos, int batch, int D, int N,
                   const double* u, const double* delta, const double* A,
                   const double* B, const double* C, const double* Dskip,
                   const double* bias, const double* z, int delta_softplus,
                   double merge_scale, int per_dir_inputs, int per_dir_params,
                   const double* conv_w, const double* conv_b, int zoh,
                   double* y, int nthreads)
{
    int K, L, tokens;
    int rc = oracle_geometry(kind, h, w, cls_pos, &K, &L, &tokens);
    if (rc != OR_OK) return rc;
    if (batch < 0 || D <= 0 || N <= 0) return OR_EINVAL;
    if (conv_w && (kind == OR_ATROUS2 || kind == OR_CROSS4)) return OR_EINVAL;
    if (batch == 0) return OR_OK;

    int64_t* route = (int64_t*)malloc(sizeof(int64_t) * (size_t)K * L);
    if (!route) return OR_ENOMEM;
    rc = oracle_route(kind, h, w, cls_pos, route);
    if (rc != OR_OK) { free(route); return rc; }

    const int pooled = (kind == OR_POOL_W || kind == OR_POOL_H);
    const int64_t in_dir = per_dir_inputs ? (int64_t)batch * tokens * D : 0;
    const int64_t bc_dir = per_dir_inputs ? (int64_t)batch * tokens * N : 0;
    const int64_t a_dir = per_dir_params ? (int64_t)D * N : 0;
    const int64_t v_dir = per_dir_params ? (int64_t)D : 0;

    int failed = 0; /* bit 0: scratch allocation failed; bit 1: atrous owner check failed */
    int64_t pairs = (int64_t)batch * D;
    int nt = nthreads > 0 ? nthreads : omp_get_max_threads();

#pragma omp parallel num_threads(nt) reduction(| : failed)
    {
        /* per-thread scratch */
        double* su = (double*)malloc(sizeof(double) * L);
        double* sdt = (double*)malloc(sizeof(double) * L);
        double* sB = (double*)malloc(sizeof(double) * (size_t)L * N);
        double* sC = (double*)malloc(sizeof(double) * (size_t)L * N);
        double* sy = (double*)malloc(sizeof(double) * L);
        double* hs = (double*)malloc(sizeof(double) * N);
        double* acc = (double*)malloc(sizeof(double) * (pooled ? L : tokens));
        int* owners = (int*)malloc(sizeof(int) * tokens);
        double* xs = (double*)malloc(sizeof(double) * tokens); /* sequence-ordered conv input */
        double* cu = (double*)malloc(sizeof(double) * tokens); /* conv output per token */
        int bad = (!su || !sdt || !sB || !sC || !sy || !hs || !acc || !owners || !xs || !cu);
        if (bad) failed |= 1;

#pragma omp for schedule(static)
        for (int64_t pr = 0; pr < pairs; ++pr) {
            if (bad) continue;
            int bi = (int)(pr / D);
            int d = (int)(pr % D);

            for (int i = 0; i < (pooled ? L : tokens); ++i) acc[i] = 0.0;
            for (int i = 0; i < tokens; ++i) owners[i] = 0;

            for (int k = 0; k < K; ++k) {
                const double* uk = u + k * in_dir + (int64_t)bi * tokens * D;
                const double* dk = delta + k * in_dir + (int64_t)bi * tokens * D;
                const double* Bk = B + k * bc_dir + (int64_t)bi * tokens * N;
                const double* Ck = C + k * bc_dir + (int64_t)bi * tokens * N;
                const double* Ak = A + k * a_dir + (int64_t)d * N;
                double Dk = Dskip ? Dskip[k * v_dir + d] : 0.0;
                double bk = bias ? bias[k * v_dir + d] : 0.0;
                const double* cw = conv_w ? conv_w + (k * v_dir + d) * 4 : 0;
                double cb = (conv_w && conv_b) ? conv_b[k * v_dir + d] : 0.0;

                if (conv_w && !pooled) {
                    /* BIDIR: the convolution runs along this direction's route. */
                    for (int t = 0; t < L; ++t) {
                        int64_t q = route[(int64_t)k * L + t];
                        xs[t] = q >= 0 ? uk[q * D + d] : 0.0;
                    }
                }
                if (conv_w && pooled) {
                    /* Token order of the convolution: row-major for POOL_W,
                     * column-major for POOL_H; direction 1 runs it reversed. */
                    int64_t g = (int64_t)h * w;
                    for (int64_t s = 0; s < g; ++s) {
                        int64_t q = k == 0 ? s : g - 1 - s;
                        int64_t tok = (kind == OR_POOL_W) ? q : (q % h) * w + q / h;
                        xs[s] = uk[tok * D + d];
                    }
                    for (int64_t s = 0; s < g; ++s) {
                        int64_t q = k == 0 ? s : g - 1 - s;
                        int64_t tok = (kind == OR_POOL_W) ? q : (q % h) * w + q / h;
                        cu[tok] = causal_conv_silu(xs, s, cw, cb);
                    }
                }

                /* Gather: one sequence step per route step. */
                for (int t = 0; t < L; ++t) {
                    int64_t q = route[(int64_t)k * L + t];
                    double uu = 0.0, dd = 0.0;
                    if (!pooled) {
                        if (q >= 0) { /* a real token */
                            uu = conv_w ? causal_conv_silu(xs, t, cw, cb) : uk[q * D + d];
                            dd = dk[q * D + d];
                            for (int n = 0; n < N; ++n) {
                                sB[(int64_t)t * N + n] = Bk[q * N + n];
                                sC[(int64_t)t * N + n] = Ck[q * N + n];
                            }
                        } else { /* [EVM] sec. 1: padding supplies zeros */
                            for (int n = 0; n < N; ++n) {
                                sB[(int64_t)t * N + n] = 0.0;
                                sC[(int64_t)t * N + n] = 0.0;
                            }
                        }
                    } else {
                        /* [FVim] Methodology: mean-pool one spatial axis. For
                         * POOL_W pooled token q is grid row q averaged over its
                         * w columns; for POOL_H it is column q averaged over
                         * its h rows. */
                        int cnt = (kind == OR_POOL_W) ? w : h;
                        double su_ = 0.0, sd_ = 0.0;
                        for (int n = 0; n < N; ++n) {
                            sB[(int64_t)t * N + n] = 0.0;
                            sC[(int64_t)t * N + n] = 0.0;
                        }
                        for (int j = 0; j < cnt; ++j) {
                            int64_t tok = (kind == OR_POOL_W) ? q * w + j : (int64_t)j * w + q;
                            su_ += conv_w ? cu[tok] : uk[tok * D + d];
                            sd_ += dk[tok * D + d];
                            for (int n = 0; n < N; ++n) {
                                sB[(int64_t)t * N + n] += Bk[tok * N + n];
                                sC[(int64_t)t * N + n] += Ck[tok * N + n];
                            }
                        }
                        uu = su_ / cnt;
                        dd = sd_ / cnt;
                        for (int n = 0; n < N; ++n) {
                            sB[(int64_t)t * N + n] /= cnt;
                            sC[(int64_t)t * N + n] /= cnt;
                        }
                    }
                    /* Discretization, [Vim] sec. 3 and sec. 4: bias, then softplus. */
                    double x = dd + bk;
                    su[t] = uu;
                    sdt[t] = delta_softplus ? softplus(x) : x;
                }

                oracle_scan_sequence(L, N, su, sdt, Ak, sB, sC, Dk, zoh, hs, sy);

                /* Scatter back to the original coordinates. */
                for (int t = 0; t < L; ++t) {
                    int64_t q = route[(int64_t)k * L + t];
                    if (q < 0) continue; /* [EVM] sec. 3: crop padding */
                    if (kind == OR_ATROUS2) {
                        /* [EVM] sec. 3: one owner per coordinate, assignment. */
                        acc[q] = sy[t];
                        owners[q] += 1;
                    } else {
                        /* [Vim] sec. 5 / [NoD] SS2D: aligned outputs are added. */
                        acc[q] += sy[t];
                    }
                }
            }

            if (kind == OR_ATROUS2) {
                for (int i = 0; i < tokens; ++i)
                    if (owners[i] != 1) failed |= 2;
            }

            /* Merge scale, repeat (pooled routes), then the shared SiLU gate. */
            double* yb = y + (int64_t)bi * tokens * D;
            const double* zb = z ? z + (int64_t)bi * tokens * D : 0;
            for (int i = 0; i < tokens; ++i) {
                double v;
                if (!pooled) {
                    v = acc[i];
                } else {
                    int r = i / w, c = i % w;
                    v = acc[kind == OR_POOL_W ? r : c];
                }
                v *= merge_scale;
                if (zb) v *= silu(zb[(int64_t)i * D + d]);
                yb[(int64_t)i * D + d] = v;
            }
        }
        free(su); free(sdt); free(sB); free(sC); free(sy); free(hs); free(acc); free(owners);
        free(xs); free(cu);
    }
    free(route);
    if (failed & 1) return OR_ENOMEM;
    if (failed & 2) return OR_EOWNER;
    return OR_OK;
}

/*
 * Pooled route on a masked (sparse) token set, [FVim] "Innovation" and
 * "Methodology": FastMaskVim keeps only the visible tokens, addresses them by
 * their grid position (sparse indexing) and forms each pooled token as the sum
 * of the visible tokens of that grid row (POOL_W) or column (POOL_H) divided by
 * the nominal width w (or height h), not by the number of visible tokens. The
 * pooled scan is the one of oracle_forward; its output is repeated onto every
 * visible token of the row (column) and gated with that token's z.
 *
 * Layouts: pos [batch][n_tok] grid positions (row * w + col) in [0, h*w);
 * u, delta [Ki][batch][n_tok][D]; B, C [Ki][batch][n_tok][N]; z, y
 * [batch][n_tok][D]; A, Dskip, bias as in oracle_forward. A row (column) with
 * no visible token pools to zeros. Returns OR_EINVAL for a position outside
 * the grid.
 */
int oracle_forward_masked(int kind, int h, int w, int batch, int n_tok, const int32_t* pos,
                          int D, int N, const double* u, const double* delta, const double* A,
                          const double* B, const double* C, const double* Dskip,
                          const double* bias, const double* z, int delta_softplus,
                          double merge_scale, int per_dir_inputs, int per_dir_params, int zoh,
                          double* y, int nthreads)
{
    if (kind != OR_POOL_W && kind != OR_POOL_H) return OR_EINVAL;
    if (h < 1 || w < 1 || batch < 0 || n_tok < 0 || D <= 0 || N <= 0) return OR_EINVAL;
    for (int64_t i = 0; i < (int64_t)batch * n_tok; ++i)
        if (pos[i] < 0 || (int64_t)pos[i] >= (int64_t)h * w) return OR_EINVAL;
    if (batch == 0 || n_tok == 0) return OR_OK;

    const int K = 2;
    const int L = (kind == OR_POOL_W) ? h : w;      /* pooled sequence length */
    const double nominal = (kind == OR_POOL_W) ? w : h;
    const int64_t in_dir = per_dir_inputs ? (int64_t)batch * n_tok * D : 0;
    const int64_t bc_dir = per_dir_inputs ? (int64_t)batch * n_tok * N : 0;
    const int64_t a_dir = per_dir_params ? (int64_t)D * N : 0;
    const int64_t v_dir = per_dir_params ? (int64_t)D : 0;
    int failed = 0;
    int64_t pairs = (int64_t)batch * D;
    int nt = nthreads > 0 ? nthreads : omp_get_max_threads();

#pragma omp parallel num_threads(nt) reduction(| : failed)
    {
        double* pu = (double*)malloc(sizeof(double) * L);
        double* pd = (double*)malloc(sizeof(double) * L);
        double* pB = (double*)malloc(sizeof(double) * (size_t)L * N);
        double* pC = (double*)malloc(sizeof(double) * (size_t)L * N);
        double* su = (double*)malloc(sizeof(double) * L);
        double* sdt = (double*)malloc(sizeof(double) * L);
        double* sB = (double*)malloc(sizeof(double) * (size_t)L * N);
        double* sC = (double*)malloc(sizeof(double) * (size_t)L * N);
        double* sy = (double*)malloc(sizeof(double) * L);
        double* hs = (double*)malloc(sizeof(double) * N);
        double* acc = (double*)malloc(sizeof(double) * L);
        int bad = (!pu || !pd || !pB || !pC || !su || !sdt || !sB || !sC || !sy || !hs || !acc);
        if (bad) failed |= 1;

#pragma omp for schedule(static)
        for (int64_t pr = 0; pr < pairs; ++pr) {
            if (bad) continue;
            int bi = (int)(pr / D);
            int d = (int)(pr % D);
            const int32_t* pb = pos + (int64_t)bi * n_tok;
            for (int i = 0; i < L; ++i) acc[i] = 0.0;
            for (int k = 0; k < K; ++k) {
                const double* uk = u + k * in_dir + (int64_t)bi * n_tok * D;
                const double* dk = delta + k * in_dir + (int64_t)bi * n_tok * D;
                const double* Bk = B + k * bc_dir + (int64_t)bi * n_tok * N;
                const double* Ck = C + k * bc_dir + (int64_t)bi * n_tok * N;
                const double* Ak = A + k * a_dir + (int64_t)d * N;
                double Dk = Dskip ? Dskip[k * v_dir + d] : 0.0;
                double bk = bias ? bias[k * v_dir + d] : 0.0;
                /* mask-aware aggregation: sum the visible tokens of each row
                 * (column), then divide by the nominal width (height) */
                for (int i = 0; i < L; ++i) {
                    pu[i] = 0.0; pd[i] = 0.0;
                    for (int n = 0; n < N; ++n) { pB[(int64_t)i * N + n] = 0.0; pC[(int64_t)i * N + n] = 0.0; }
                }
                for (int t = 0; t < n_tok; ++t) {
                    int row = pb[t] / w, col = pb[t] % w;
                    int i = (kind == OR_POOL_W) ? row : col;
                    pu[i] += uk[(int64_t)t * D + d];
                    pd[i] += dk[(int64_t)t * D + d];
                    for (int n = 0; n < N; ++n) {
                        pB[(int64_t)i * N + n] += Bk[(int64_t)t * N + n];
                        pC[(int64_t)i * N + n] += Ck[(int64_t)t * N + n];
                    }
                }
                /* direction 0 walks the pooled sequence forward, 1 reversed */
                for (int t = 0; t < L; ++t) {
                    int i = (k == 0) ? t : L - 1 - t;
                    su[t] = pu[i] / nominal;
                    double x = pd[i] / nominal + bk;
                    sdt[t] = delta_softplus ? softplus(x) : x;
                    for (int n = 0; n < N; ++n) {
                        sB[(int64_t)t * N + n] = pB[(int64_t)i * N + n] / nominal;
                        sC[(int64_t)t * N + n] = pC[(int64_t)i * N + n] / nominal;
                    }
                }
                oracle_scan_sequence(L, N, su, sdt, Ak, sB, sC, Dk, zoh, hs, sy);
                for (int t = 0; t < L; ++t) acc[(k == 0) ? t : L - 1 - t] += sy[t];
            }
            /* repeat onto the visible tokens, merge scale, gate */
            double* yb = y + (int64_t)bi * n_tok * D;
            const double* zb = z ? z + (int64_t)bi * n_tok * D : 0;
            for (int t = 0; t < n_tok; ++t) {
                int row = pb[t] / w, col = pb[t] % w;
                double v = acc[(kind == OR_POOL_W) ? row : col] * merge_scale;
                if (zb) v *= silu(zb[(int64_t)t * D + d]);
                yb[(int64_t)t * D + d] = v;
            }
        }
        free(pu); free(pd); free(pB); free(pC); free(su); free(sdt); free(sB); free(sC);
        free(sy); free(hs); free(acc);
    }
    if (failed & 1) return OR_ENOMEM;
    return OR_OK;
}

/*
 * Gradient of oracle_forward by reverse-mode differentiation of its own loops:
 * the gate, the merge (sum, or one owner for ATROUS2), the repeat and mean of
 * the pooled routes, the recurrence run backwards in time, and the
 * discretization. The released Delta*B*u write term only; no convolution.
 * Steps of the recurrence ([Vim] sec. 4): with x = Delta, a = exp(x A),
 *     h_t = a_t h_{t-1} + x_t B_t u_t,   y_t = C_t . h_t + D u_t,
 * the adjoint g_t = dL/dh_t satisfies g_t = C_t dy_t + a_{t+1} g_{t+1}, and
 *     dC_t = dy_t h_t,  dB_t = g_t x_t u_t,  du_t = D dy_t + sum_n g_t x_t B_t,
 *     dx_t = sum_n g_t (A a_t h_{t-1} + B_t u_t),  dA += g_t x_t a_t h_{t-1},
 *     dD += dy_t u_t,  draw_t = dx_t * sigmoid(raw_t + bias) (softplus' = sigmoid).
 *
 * dy: [batch][tokens][D]. Outputs (all overwritten; any may be NULL):
 *   du, ddelta [Ki][batch][tokens][D] (ddelta: w.r.t. the raw step),
 *   dB, dC [Ki][batch][tokens][N], dA [Kp][D][N], dDskip [Kp][D],
 *   dbias [Kp][D], dz [batch][tokens][D].
 */
int oracle_backward(int kind, int h, int w, int cls_pos, int batch, int D, int N,
                    const double* u, const double* delta, const double* A, const double* B,
                    const double* C, const double* Dskip, const double* bias, const double* z,
                    int delta_softplus, double merge_scale, int per_dir_inputs, int per_dir_params,
                    const double* dy, double* du, double* ddelta, double* dA, double* dB,
                    double* dC, double* dDskip, double* dbias, double* dz, int nthreads)
{
    int K, L, tokens;
    int rc = oracle_geometry(kind, h, w, cls_pos, &K, &L, &tokens);
    if (rc != OR_OK) return rc;
    if (batch < 0 || D <= 0 || N <= 0) return OR_EINVAL;
    const int pooled = (kind == OR_POOL_W || kind == OR_POOL_H);
    const int Ki = per_dir_inputs ? K : 1, Kp = per_dir_params ? K : 1;
    const int64_t in_dir = per_dir_inputs ? (int64_t)batch * tokens * D : 0;
    const int64_t bc_dir = per_dir_inputs ? (int64_t)batch * tokens * N : 0;
    const int64_t a_dir = per_dir_params ? (int64_t)D * N : 0;
    const int64_t v_dir = per_dir_params ? (int64_t)D : 0;
    if (du) memset(du, 0, sizeof(double) * (size_t)Ki * batch * tokens * D);
    if (ddelta) memset(ddelta, 0, sizeof(double) * (size_t)Ki * batch * tokens * D);
    if (dB) memset(dB, 0, sizeof(double) * (size_t)Ki * batch * tokens * N);
    if (dC) memset(dC, 0, sizeof(double) * (size_t)Ki * batch * tokens * N);
    if (dA) memset(dA, 0, sizeof(double) * (size_t)Kp * D * N);
    if (dDskip) memset(dDskip, 0, sizeof(double) * (size_t)Kp * D);
    if (dbias) memset(dbias, 0, sizeof(double) * (size_t)Kp * D);
    if (batch == 0) return OR_OK;

    int64_t* route = (int64_t*)malloc(sizeof(int64_t) * (size_t)K * L);
    if (!route) return OR_ENOMEM;
    rc = oracle_route(kind, h, w, cls_pos, route);
    if (rc != OR_OK) { free(route); return rc; }
    const int cnt = pooled ? ((kind == OR_POOL_W) ? w : h) : 1;
    int failed = 0;
    int nt = nthreads > 0 ? nthreads : omp_get_max_threads();

    /* one image per thread: its token gradients are private; the parameter
     * gradients are summed into thread-local arrays and added at the end */
#pragma omp parallel num_threads(nt) reduction(| : failed)
    {
        double* su = (double*)malloc(sizeof(double) * L);
        double* sraw = (double*)malloc(sizeof(double) * L);
        double* sx = (double*)malloc(sizeof(double) * L);
        double* sB = (double*)malloc(sizeof(double) * (size_t)L * N);
        double* sC = (double*)malloc(sizeof(double) * (size_t)L * N);
        double* hs = (double*)malloc(sizeof(double) * (size_t)(L + 1) * N); /* h_{-1} .. h_{L-1} */
        double* ys = (double*)malloc(sizeof(double) * (size_t)K * L);
        double* acc = (double*)malloc(sizeof(double) * tokens);
        double* gacc = (double*)malloc(sizeof(double) * tokens);
        double* dys = (double*)malloc(sizeof(double) * L);
        double* g = (double*)malloc(sizeof(double) * N);
        double* lA = (double*)calloc((size_t)Kp * D * N, sizeof(double));
        double* lD = (double*)calloc((size_t)Kp * D, sizeof(double));
        double* lb = (double*)calloc((size_t)Kp * D, sizeof(double));
        int bad = (!su || !sraw || !sx || !sB || !sC || !hs || !ys || !acc || !gacc || !dys || !g ||
                   !lA || !lD || !lb);
        if (bad) failed |= 1;

#pragma omp for schedule(static)
        for (int bi = 0; bi < batch; ++bi) {
            if (bad) continue;
            for (int d = 0; d < D; ++d) {
                /* gather direction kk's sequence from input plane pl */
                #define GATHER(pl, kk)                                                          \
                    do {                                                                        \
                        const double* uk = u + (pl) * in_dir + (int64_t)bi * tokens * D;         \
                        const double* dk = delta + (pl) * in_dir + (int64_t)bi * tokens * D;     \
                        const double* Bk = B + (pl) * bc_dir + (int64_t)bi * tokens * N;         \
                        const double* Ck = C + (pl) * bc_dir + (int64_t)bi * tokens * N;         \
                        for (int t = 0; t < L; ++t) {                                           \
                            int64_t q = route[(int64_t)(kk) * L + t];                           \
                            su[t] = 0.0; sraw[t] = 0.0;                                         \
                            for (int n = 0; n < N; ++n) { sB[(int64_t)t * N + n] = 0.0; sC[(int64_t)t * N + n] = 0.0; } \
                            if (!pooled) {                                                      \
                                if (q < 0) continue;                                            \
                                su[t] = uk[q * D + d]; sraw[t] = dk[q * D + d];                 \
                                for (int n = 0; n < N; ++n) {                                   \
                                    sB[(int64_t)t * N + n] = Bk[q * N + n];                     \
                                    sC[(int64_t)t * N + n] = Ck[q * N + n];                     \
                                }                                                               \
                            } else {                                                            \
                                for (int j = 0; j < cnt; ++j) {                                 \
                                    int64_t tok = (kind == OR_POOL_W) ? q * w + j : (int64_t)j * w + q; \
                                    su[t] += uk[tok * D + d] / cnt; sraw[t] += dk[tok * D + d] / cnt; \
                                    for (int n = 0; n < N; ++n) {                               \
                                        sB[(int64_t)t * N + n] += Bk[tok * N + n] / cnt;        \
                                        sC[(int64_t)t * N + n] += Ck[tok * N + n] / cnt;        \
                                    }                                                           \
                                }                                                               \
                            }                                                                   \
                        }                                                                       \
                    } while (0)

                /* forward: per-direction outputs and the merged pre-gate value */
                for (int i = 0; i < tokens; ++i) acc[i] = 0.0;
                for (int k = 0; k < K; ++k) {
                    GATHER(per_dir_inputs ? k : 0, k);
                    const double* Ak = A + k * a_dir + (int64_t)d * N;
                    double Dk = Dskip ? Dskip[k * v_dir + d] : 0.0;
                    double bk = bias ? bias[k * v_dir + d] : 0.0;
                    for (int n = 0; n < N; ++n) hs[n] = 0.0;
                    for (int t = 0; t < L; ++t) {
                        double xr = sraw[t] + bk;
                        double x = delta_softplus ? softplus(xr) : xr;
                        double read = 0.0;
                        for (int n = 0; n < N; ++n) {
                            double hn = exp(x * Ak[n]) * hs[(int64_t)t * N + n] + x * sB[(int64_t)t * N + n] * su[t];
                            hs[(int64_t)(t + 1) * N + n] = hn;
                            read += sC[(int64_t)t * N + n] * hn;
                        }
                        ys[(int64_t)k * L + t] = read + Dk * su[t];
                    }
                    for (int t = 0; t < L; ++t) {
                        int64_t q = route[(int64_t)k * L + t];
                        if (q < 0) continue;
                        if (kind == OR_ATROUS2) acc[q] = ys[(int64_t)k * L + t];
                        else acc[q] += ys[(int64_t)k * L + t];
                    }
                }
                /* gate and merge scale: Y = s * acc_repeated * silu(z) */
                const double* zb = z ? z + (int64_t)bi * tokens * D : 0;
                const double* dyb = dy + (int64_t)bi * tokens * D;
                for (int i = 0; i < tokens; ++i) gacc[i] = 0.0;
                for (int p = 0; p < tokens; ++p) {
                    int pi = p;
                    if (pooled) { int r = p / w, c = p % w; pi = (kind == OR_POOL_W) ? r : c; }
                    double pre = merge_scale * acc[pi];
                    double dyp = dyb[(int64_t)p * D + d];
                    if (zb) {
                        double zz = zb[(int64_t)p * D + d];
                        double sg = 1.0 / (1.0 + exp(-zz));
                        if (dz) dz[((int64_t)bi * tokens + p) * D + d] = dyp * pre * sg * (1.0 + zz * (1.0 - sg));
                        gacc[pi] += dyp * merge_scale * zz * sg;
                    } else {
                        gacc[pi] += dyp * merge_scale;
                    }
                }
                /* backward through each direction's recurrence */
                for (int k = 0; k < K; ++k) {
                    int ki = per_dir_inputs ? k : 0, kp = per_dir_params ? k : 0;
                    GATHER(ki, k);
                    const double* Ak = A + k * a_dir + (int64_t)d * N;
                    double Dk = Dskip ? Dskip[k * v_dir + d] : 0.0;
                    double bk = bias ? bias[k * v_dir + d] : 0.0;
                    /* recompute the states h_t of this direction */
                    for (int n = 0; n < N; ++n) hs[n] = 0.0;
                    for (int t = 0; t < L; ++t) {
                        double xr = sraw[t] + bk;
                        sx[t] = delta_softplus ? softplus(xr) : xr;
                        for (int n = 0; n < N; ++n)
                            hs[(int64_t)(t + 1) * N + n] = exp(sx[t] * Ak[n]) * hs[(int64_t)t * N + n] +
                                                           sx[t] * sB[(int64_t)t * N + n] * su[t];
                    }
                    for (int t = 0; t < L; ++t) {
                        int64_t q = route[(int64_t)k * L + t];
                        dys[t] = q >= 0 ? gacc[q] : 0.0;
                    }
                    for (int n = 0; n < N; ++n) g[n] = 0.0;
                    for (int t = L - 1; t >= 0; --t) {
                        double dyt = dys[t], dut = Dk * dyt, dxt = 0.0;
                        lD[kp * D + d] += dyt * su[t];
                        for (int n = 0; n < N; ++n) {
                            double ht = hs[(int64_t)(t + 1) * N + n], hp = hs[(int64_t)t * N + n];
                            double a = exp(sx[t] * Ak[n]);
                            g[n] += sC[(int64_t)t * N + n] * dyt;
                            double dCt = dyt * ht;
                            double dBt = g[n] * sx[t] * su[t];
                            dut += g[n] * sx[t] * sB[(int64_t)t * N + n];
                            dxt += g[n] * (Ak[n] * a * hp + sB[(int64_t)t * N + n] * su[t]);
                            lA[(kp * D + d) * N + n] += g[n] * sx[t] * a * hp;
                            g[n] *= a;
                            /* scatter the token gradients of B and C */
                            int64_t q = route[(int64_t)k * L + t];
                            if (q < 0) continue;
                            double* dBk = dB ? dB + ki * bc_dir + (int64_t)bi * tokens * N : 0;
                            double* dCk = dC ? dC + ki * bc_dir + (int64_t)bi * tokens * N : 0;
                            if (!pooled) {
                                if (dBk) dBk[q * N + n] += dBt;
                                if (dCk) dCk[q * N + n] += dCt;
                            } else {
                                for (int j = 0; j < cnt; ++j) {
                                    int64_t tok = (kind == OR_POOL_W) ? q * w + j : (int64_t)j * w + q;
                                    if (dBk) dBk[tok * N + n] += dBt / cnt;
                                    if (dCk) dCk[tok * N + n] += dCt / cnt;
                                }
                            }
                        }
                        double xr = sraw[t] + bk;
                        double draw = delta_softplus ? dxt / (1.0 + exp(-xr)) : dxt;
                        lb[kp * D + d] += draw;
                        int64_t q = route[(int64_t)k * L + t];
                        if (q < 0) continue; /* padding: only the bias gradient */
                        double* duk = du ? du + ki * in_dir + (int64_t)bi * tokens * D : 0;
                        double* ddk = ddelta ? ddelta + ki * in_dir + (int64_t)bi * tokens * D : 0;
                        if (!pooled) {
                            if (duk) duk[q * D + d] += dut;
                            if (ddk) ddk[q * D + d] += draw;
                        } else {
                            for (int j = 0; j < cnt; ++j) {
                                int64_t tok = (kind == OR_POOL_W) ? q * w + j : (int64_t)j * w + q;
                                if (duk) duk[tok * D + d] += dut / cnt;
                                if (ddk) ddk[tok * D + d] += draw / cnt;
                            }
                        }
                    }
                }
                #undef GATHER
            }
        }
#pragma omp critical
        {
            if (!bad) {
                if (dA) for (int64_t i = 0; i < (int64_t)Kp * D * N; ++i) dA[i] += lA[i];
                if (dDskip) for (int64_t i = 0; i < (int64_t)Kp * D; ++i) dDskip[i] += lD[i];
                if (dbias) for (int64_t i = 0; i < (int64_t)Kp * D; ++i) dbias[i] += lb[i];
            }
        }
        free(su); free(sraw); free(sx); free(sB); free(sC); free(hs); free(ys); free(acc); free(gacc);
        free(dys); free(g); free(lA); free(lD); free(lb);
    }
    free(route);
    if (failed & 1) return OR_ENOMEM;
    return OR_OK;
}

/* Number of OpenMP threads oracle_forward uses when nthreads <= 0. */
int oracle_default_threads(void)
{
    return omp_get_max_threads();
}
