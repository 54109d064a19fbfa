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

/* Number of OpenMP threads oracle_forward uses when nthreads <= 0. */
int oracle_default_threads(void)
{
    return omp_get_max_threads();
}
