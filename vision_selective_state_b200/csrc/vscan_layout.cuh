// Copies of token rows between strided layouts: vscan_forward packs strided
// input tensors densely into its workspace before a scan and copies the packed
// output back out after it, so every scan kernel reads the dense channels-last
// rows its gathers are built for.
#pragma once

#include <stdint.h>

namespace vscan {

// Image m (0 <= m < nimg) has ntok rows of R elements of type E: source row t
// at src + m * s_img + t * s_tok, destination row at dst + m * d_img + t * d_tok
// (strides in elements of E). Grid (x, y): blocks along the rows, images along
// y (striding by gridDim.y); one warp per row, lanes along its elements.
template <typename E>
__global__ void __launch_bounds__(256) copy_rows_kernel(const E* __restrict__ src, long long s_img, long long s_tok,
                                                        E* __restrict__ dst, long long d_img, long long d_tok,
                                                        int nimg, int ntok, int R)
{
    const int warps = blockDim.x >> 5, lane = threadIdx.x & 31;
    for (int m = blockIdx.y; m < nimg; m += gridDim.y) {
        const E* sm = src + (long long)m * s_img;
        E* dm = dst + (long long)m * d_img;
        for (int t = blockIdx.x * warps + (threadIdx.x >> 5); t < ntok; t += gridDim.x * warps) {
            const E* sr = sm + (long long)t * s_tok;
            E* dr = dm + (long long)t * d_tok;
            for (int i = lane; i < R; i += 32) dr[i] = sr[i];
        }
    }
}

}  // namespace vscan
