// Route geometry and index arithmetic of the routed selective scan.
//
// One definition, used by the scan kernels (inline, per token) and by the map
// kernel behind vscan_route_indices(), so the maps a caller can inspect are the
// ones the kernels walk.
//
// Token arrays are row-major over the h x w grid (columns fastest: "Vision
// Mamba: Bidirectional State Space Models for Images", sec. 1), with the CLS
// token already inserted for the bidirectional route (sec. 2).
#pragma once

#include <stdint.h>

namespace vscan {

enum RouteKind : int {
    RK_BIDIR = 0,
    RK_CROSS4 = 1,
    RK_ATROUS2 = 2,
    RK_POOL_W = 3,
    RK_POOL_H = 4,
};

struct RouteGeom {
    int kind;
    int h, w;      // grid
    int cls_pos;   // BIDIR: CLS index or -1
    int K;         // directions
    int L;         // steps per direction
    int tokens;    // tokens per image in the token array
    int rows, cols;  // ATROUS2: residue sub-grid (ceil(h/2), ceil(w/2)); else h, w
};

// Fill a RouteGeom; returns false for an invalid combination.
inline bool make_geom(int kind, int h, int w, int cls_pos, RouteGeom* g)
{
    if (h < 1 || w < 1) return false;
    const long long hw = (long long)h * w;
    if (hw > (1LL << 24)) return false;
    g->kind = kind; g->h = h; g->w = w; g->cls_pos = cls_pos;
    g->rows = h; g->cols = w;
    switch (kind) {
    case RK_BIDIR:
        if (cls_pos != -1 && cls_pos != (int)(hw / 2)) return false;
        g->K = 2; g->tokens = (int)hw + (cls_pos >= 0 ? 1 : 0); g->L = g->tokens;
        return true;
    case RK_CROSS4:
        if (cls_pos != -1) return false;
        g->K = 4; g->tokens = (int)hw; g->L = (int)hw;
        return true;
    case RK_ATROUS2:
        if (cls_pos != -1) return false;
        g->K = 4; g->tokens = (int)hw;
        g->rows = (h + 1) / 2; g->cols = (w + 1) / 2;
        g->L = g->rows * g->cols;
        return true;
    case RK_POOL_W:
        if (cls_pos != -1) return false;
        g->K = 2; g->tokens = (int)hw; g->L = h;
        return true;
    case RK_POOL_H:
        if (cls_pos != -1) return false;
        g->K = 2; g->tokens = (int)hw; g->L = w;
        return true;
    default:
        return false;
    }
}

// Token visited at step t (0 <= t < L) of direction k: an index into the token
// array (pooled routes: into the pooled sequence), or -1 for an ATROUS2 pad.
template <int RK>
__host__ __device__ __forceinline__ int route_token(const RouteGeom& g, int k, int t)
{
    if (RK == RK_BIDIR || RK == RK_POOL_W || RK == RK_POOL_H) {
        // Forward, and the whole sequence reversed ("Two scans meet at the
        // same token"): the backward stream's step t holds token L-1-t.
        return (k == 0) ? t : g.L - 1 - t;
    } else if (RK == RK_CROSS4) {
        // SS2D ("Norm or Direction?", sec. 3): k0 row-major, k1 its reverse,
        // k2 column-major (step s = c*h + r), k3 its reverse.
        const int s = (k & 1) ? g.L - 1 - t : t;
        if (k < 2) return s;
        const int c = s / g.h;
        const int r = s - c * g.h;
        return r * g.w + c;
    } else {  // RK_ATROUS2
        // "EfficientVMamba", sec. 1: O_k[t] = X[2 r_t + m_k, 2 c_t + n_k],
        // (m_k, n_k) = (0,0), (1,0), (0,1), (1,1); odd k walk column-major.
        const int m = k & 1, n = k >> 1;
        int r, c;
        if (k & 1) {
            c = t / g.rows;
            r = t - c * g.rows;
        } else {
            r = t / g.cols;
            c = t - r * g.cols;
        }
        const int y = 2 * r + m, x = 2 * c + n;
        return (y < g.h && x < g.w) ? y * g.w + x : -1;
    }
}

__host__ __device__ __forceinline__ int route_token_any(const RouteGeom& g, int k, int t)
{
    switch (g.kind) {
    case RK_BIDIR: return route_token<RK_BIDIR>(g, k, t);
    case RK_CROSS4: return route_token<RK_CROSS4>(g, k, t);
    case RK_ATROUS2: return route_token<RK_ATROUS2>(g, k, t);
    case RK_POOL_W: return route_token<RK_POOL_W>(g, k, t);
    default: return route_token<RK_POOL_H>(g, k, t);
    }
}

// Step at which direction k visits token p (inverse of route_token) for the
// routes whose directions all visit every token (BIDIR, CROSS4).
template <int RK>
__host__ __device__ __forceinline__ int visit_step(const RouteGeom& g, int k, int p)
{
    if (RK == RK_BIDIR) {
        return (k == 0) ? p : g.L - 1 - p;
    } else {  // RK_CROSS4
        if (k < 2) return (k == 0) ? p : g.L - 1 - p;
        const int r = p / g.w;
        const int c = p - r * g.w;
        const int s = c * g.h + r;
        return (k == 2) ? s : g.L - 1 - s;
    }
}

}  // namespace vscan
