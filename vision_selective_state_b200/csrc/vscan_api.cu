// C ABI of the routed selective scan (declared in include/vscan.h).
//
// Host side only: argument checks, workspace sizing, kernel selection and
// launch, and the host-buffer (end-to-end) entry point. Every check runs before
// the first CUDA call, so a rejected call launches nothing.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <string>

#include "vscan.h"
#include "vscan_backward.cuh"
#include <nvtx3/nvToolsExt.h>

#include "vscan_check.cuh"
#include "vscan_layout.cuh"
#include "vscan_pipe.cuh"
#include "vscan_pool.cuh"
#include "vscan_resident.cuh"
#include "vscan_route.cuh"
#include "vscan_stream.cuh"

struct vscan_route {
    vscan::RouteGeom g;
};

namespace {

constexpr int32_t kAbiVersion = 5;

// A named NVTX range for the duration of a public call, so a profiler's
// timeline groups each call's copies and kernels (a no-op unless a tool is
// attached; NVTX v3 is header-only).
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};
constexpr int32_t kKnownFlags = VSCAN_FLAG_ZOH | VSCAN_FLAG_CHECK_VALUES;
constexpr size_t kMaxSmem = 200 * 1024;  // dynamic shared memory the kernels may ask for
thread_local std::string g_last_error;

vscan_status fail(vscan_status s, const char* fmt, ...)
{
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return s;
}

vscan_status cuda_fail(cudaError_t e, const char* what)
{
    return fail(VSCAN_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorString(e), cudaGetErrorName(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t round256(size_t n) { return (n + 255) & ~size_t(255); }

size_t elem_bytes(int32_t dtype) { return dtype == VSCAN_BF16 ? 2 : 4; }

bool is_pool(int kind) { return kind == vscan::RK_POOL_W || kind == vscan::RK_POOL_H; }

// Tokens per image in the token arrays: the visible ones of a masked set, else
// the route's (grid, plus CLS for BIDIR).
int tokens_of(const vscan_route* r, const vscan_args* a) { return a->token_pos ? a->n_tokens : r->g.tokens; }

// Strides of the token arrays in elements, with 0 resolved to the dense value.
long long tok_stride_of(const vscan_args* a) { return a->tok_stride ? a->tok_stride : a->channels; }
long long batch_stride_of(const vscan_route* r, const vscan_args* a)
{
    return a->batch_stride ? a->batch_stride : (long long)tokens_of(r, a) * tok_stride_of(a);
}
long long bc_tok_stride_of(const vscan_args* a) { return a->bc_tok_stride ? a->bc_tok_stride : a->d_state; }
long long bc_batch_stride_of(const vscan_route* r, const vscan_args* a)
{
    return a->bc_batch_stride ? a->bc_batch_stride : (long long)tokens_of(r, a) * bc_tok_stride_of(a);
}
// u, delta, z, y (main) or B, C not laid out densely
bool strided_main(const vscan_route* r, const vscan_args* a)
{
    return tok_stride_of(a) != a->channels || batch_stride_of(r, a) != (long long)tokens_of(r, a) * a->channels;
}
bool strided_bc(const vscan_route* r, const vscan_args* a)
{
    return bc_tok_stride_of(a) != a->d_state ||
           bc_batch_stride_of(r, a) != (long long)tokens_of(r, a) * a->d_state;
}

size_t resident_bytes(const vscan_route* r, const vscan_args* a)
{
    const int Ki = a->per_dir_inputs ? r->g.K : 1;
    const int Kd = (a->per_dir_inputs || a->per_dir_params) ? r->g.K : 1;
    return vscan::resident_smem_bytes(r->g.kind, r->g.tokens, Ki, Kd, a->conv_w != nullptr);
}

// Checks that do not depend on where the tensors live.
vscan_status check_shape(const vscan_route* r, const vscan_args* a)
{
    if (!r) return fail(VSCAN_ERR_INVALID_ARGUMENT, "route is NULL");
    if (!a) return fail(VSCAN_ERR_INVALID_ARGUMENT, "args is NULL");
    if (a->flags & ~kKnownFlags)
        return fail(VSCAN_ERR_INVALID_ARGUMENT, "unknown bits in args.flags 0x%x", (unsigned)a->flags);
    if ((a->flags & VSCAN_FLAG_CHECK_VALUES) && !a->status)
        return fail(VSCAN_ERR_INVALID_ARGUMENT, "VSCAN_FLAG_CHECK_VALUES needs a device status word (args.status)");
    if ((reinterpret_cast<uintptr_t>(a->status) & 3u) != 0)
        return fail(VSCAN_ERR_ALIGNMENT, "status is not 4-byte aligned");
    if (a->conv_b && !a->conv_w) return fail(VSCAN_ERR_INVALID_ARGUMENT, "conv_b given without conv_w");
    if (a->reserved2 != 0) return fail(VSCAN_ERR_INVALID_ARGUMENT, "args.reserved2 must be 0");
    if (a->token_pos) {
        if (!is_pool(r->g.kind))
            return fail(VSCAN_ERR_UNSUPPORTED, "a masked token set (token_pos) needs POOL_W or POOL_H");
        if (a->conv_w)
            return fail(VSCAN_ERR_UNSUPPORTED, "no convolution order is defined on a masked token set");
        if (a->n_tokens < 0) return fail(VSCAN_ERR_INVALID_ARGUMENT, "n_tokens %d < 0", a->n_tokens);
    } else if (a->n_tokens != 0) {
        return fail(VSCAN_ERR_INVALID_ARGUMENT, "n_tokens is set without token_pos");
    }
    if (a->conv_w && (r->g.kind == vscan::RK_CROSS4 || r->g.kind == vscan::RK_ATROUS2))
        return fail(VSCAN_ERR_UNSUPPORTED, "the fused convolution is defined for BIDIR and the pooled routes");
    if (a->dtype != VSCAN_F32 && a->dtype != VSCAN_BF16)
        return fail(VSCAN_ERR_INVALID_ARGUMENT, "unknown dtype %d", a->dtype);
    if (a->batch < 0) return fail(VSCAN_ERR_INVALID_ARGUMENT, "batch %d < 0", a->batch);
    if (a->channels < 1) return fail(VSCAN_ERR_INVALID_ARGUMENT, "channels %d < 1", a->channels);
    if (a->d_state < 1) return fail(VSCAN_ERR_INVALID_ARGUMENT, "d_state %d < 1", a->d_state);
    if (a->d_state > 16) return fail(VSCAN_ERR_UNSUPPORTED, "d_state %d > 16", a->d_state);
    const int vec = a->dtype == VSCAN_F32 ? 4 : 8;
    if (a->channels % vec != 0)
        return fail(VSCAN_ERR_ALIGNMENT, "channels %d is not a multiple of %d (16-byte rows)", a->channels, vec);
    if (a->per_dir_inputs != 0 && a->per_dir_inputs != 1)
        return fail(VSCAN_ERR_INVALID_ARGUMENT, "per_dir_inputs must be 0 or 1");
    if (a->per_dir_params != 0 && a->per_dir_params != 1)
        return fail(VSCAN_ERR_INVALID_ARGUMENT, "per_dir_params must be 0 or 1");
    if (a->delta_softplus != 0 && a->delta_softplus != 1)
        return fail(VSCAN_ERR_INVALID_ARGUMENT, "delta_softplus must be 0 or 1");
    if (!std::isfinite(a->merge_scale)) return fail(VSCAN_ERR_INVALID_ARGUMENT, "merge_scale is not finite");
    if (a->seq_chunks != 0 && a->seq_chunks != 1 && a->seq_chunks != 2 && a->seq_chunks != 4 &&
        a->seq_chunks != 8)
        return fail(VSCAN_ERR_INVALID_ARGUMENT, "seq_chunks %d is not 0, 1, 2, 4 or 8", a->seq_chunks);
    if (a->batch > 65535) return fail(VSCAN_ERR_UNSUPPORTED, "batch %d > 65535", a->batch);
    if ((long long)tokens_of(r, a) * a->channels >= (1LL << 31))
        return fail(VSCAN_ERR_UNSUPPORTED, "tokens x channels of one image must be below 2^31");
    if (a->tok_stride < 0 || a->batch_stride < 0 || a->bc_tok_stride < 0 || a->bc_batch_stride < 0)
        return fail(VSCAN_ERR_INVALID_ARGUMENT, "strides must be >= 0 (0 = dense)");
    if (tok_stride_of(a) < a->channels || tok_stride_of(a) % vec != 0)
        return fail(VSCAN_ERR_ALIGNMENT, "tok_stride %lld must be >= channels and a multiple of %d",
                    (long long)a->tok_stride, vec);
    if (batch_stride_of(r, a) < (long long)tokens_of(r, a) * tok_stride_of(a) || batch_stride_of(r, a) % vec != 0)
        return fail(VSCAN_ERR_ALIGNMENT, "batch_stride %lld must be >= tokens x tok_stride and a multiple of %d",
                    (long long)a->batch_stride, vec);
    if (bc_tok_stride_of(a) < a->d_state)
        return fail(VSCAN_ERR_INVALID_ARGUMENT, "bc_tok_stride %lld < d_state", (long long)a->bc_tok_stride);
    if (bc_batch_stride_of(r, a) < (long long)tokens_of(r, a) * bc_tok_stride_of(a))
        return fail(VSCAN_ERR_INVALID_ARGUMENT, "bc_batch_stride %lld < tokens x bc_tok_stride",
                    (long long)a->bc_batch_stride);
    if (is_pool(r->g.kind)) {
        const int Ki = a->per_dir_inputs ? 2 : 1;
        if (vscan::pool_scan_smem_bytes(Ki, r->g.L, a->conv_w != nullptr) > kMaxSmem)
            return fail(VSCAN_ERR_UNSUPPORTED, "pooled length %d too long for the on-chip tile", r->g.L);
    } else if (a->seq_chunks > 1) {
        if (resident_bytes(r, a) > kMaxSmem)
            return fail(VSCAN_ERR_UNSUPPORTED, "seq_chunks > 1 needs the token tile on chip; %d tokens do not fit",
                        r->g.tokens);
    }
    return VSCAN_OK;
}

// SMs of the current device (148 on B200), read once per process.
int num_sms()
{
    static int n = [] {
        int dev = 0, v = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
            v = 148;
        return v;
    }();
    return n;
}

// Chunks per sequence for the streaming routes: 1 = streaming kernel, 2/4/8 =
// resident chunked kernel. The library picks the resident kernel when the tile
// fits on chip and the streaming kernel would leave most SMs idle.
int choose_chunks(const vscan_route* r, const vscan_args* a)
{
    if (is_pool(r->g.kind)) return 1;
    if (a->seq_chunks >= 1) return a->seq_chunks;
    if (resident_bytes(r, a) > kMaxSmem) return 1;
    const long long stream_warps = (long long)a->batch * ((a->channels + vscan::ST_CH - 1) / vscan::ST_CH) * r->g.K;
    if (stream_warps >= 4LL * 148) return 1;
    return r->g.L >= 128 ? 8 : (r->g.L >= 32 ? 4 : 2);
}

vscan_status check_pointers(const vscan_args* a, bool device)
{
    if (a->batch == 0) return VSCAN_OK;
    const char* names[] = {"u", "delta", "B", "C", "y", "A"};
    const void* ptrs[] = {a->u, a->delta, a->B, a->C, a->y, a->A};
    for (int i = 0; i < 6; ++i)
        if (!ptrs[i]) return fail(VSCAN_ERR_INVALID_ARGUMENT, "%s is NULL", names[i]);
    if (device) {
        const char* vn[] = {"u", "delta", "B", "C", "z", "y"};
        const void* vp[] = {a->u, a->delta, a->B, a->C, a->z, a->y};
        for (int i = 0; i < 6; ++i)
            if (vp[i] && !aligned16(vp[i]))
                return fail(VSCAN_ERR_ALIGNMENT, "%s is not 16-byte aligned", vn[i]);
    }
    return VSCAN_OK;
}

uint64_t workspace_need(const vscan_route* r, const vscan_args* a)
{
    const vscan::RouteGeom& g = r->g;
    if (a->batch == 0) return 0;
    if (g.kind == vscan::RK_BIDIR || g.kind == vscan::RK_CROSS4)  // one parking plane per direction
        return round256((uint64_t)g.K * a->batch * g.tokens * a->channels * sizeof(float));
    if (is_pool(g.kind)) {
        const int Ki = a->per_dir_inputs ? 2 : 1;
        return 2 * round256((uint64_t)Ki * a->batch * g.L * a->d_state * sizeof(float));
    }
    return 0;
}

// BIDIR sequences at least this long run 32-step chunks (bf16 I/O, no options).
constexpr int kLongChunkMinL = 2048;

// Raise a kernel's dynamic shared-memory limit once per device (the attribute
// stays set for the process), not on every launch: one flag per instantiation
// of the calling template and device ordinal.
template <typename Kernel>
cudaError_t set_smem_once(Kernel* fn, int bytes, int* done_by_device, int max_devices)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < max_devices && __atomic_load_n(&done_by_device[dev], __ATOMIC_ACQUIRE) >= bytes)
        return cudaSuccess;
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && dev >= 0 && dev < max_devices)
        __atomic_store_n(&done_by_device[dev], bytes, __ATOMIC_RELEASE);
    return e;
}

constexpr int kAttrDevices = 64;

// float32 atrous launches whose per-warp chains dominate take the two-warp state
// split: at most 4 CTAs per SM (b1 56x56: 42.1 -> 36.5 us), or 8 with the ZOH term's
// longer per-state work (b8: 125 -> 109 us); the plain b8 launch (5.2 CTAs per SM)
// measured 3 % slower split (61.1 against 63.1 us) and keeps one consumer warp.
bool atrous_split(long long ctas, bool zoh) { return ctas <= (zoh ? 8LL : 4LL) * num_sms(); }

template <int RK, typename T, bool N16, int KC, int MODE, int PW, int FL, int TOK = vscan::ST_TOK,
          int CH = vscan::ST_CH, int SS = 1>
cudaError_t launch_stream_mode(vscan::ScanParams p, int k_base, int grid_z, cudaStream_t s)
{
    static_assert(!(FL & vscan::FL_CKPT) || TOK == vscan::BW_TOK, "checkpoints every BW_TOK steps");
    const size_t smem = vscan::stream_smem_bytes<T, KC, MODE, FL, CH, TOK, SS>();
    static int attr_done[kAttrDevices] = {};
    cudaError_t e = set_smem_once(vscan::stream_scan_kernel<RK, T, N16, KC, MODE, PW, FL, CH, TOK, SS>, (int)smem,
                                  attr_done, kAttrDevices);
    if (e != cudaSuccess) return e;
    p.k_base = k_base;
    const dim3 grid((p.D + CH - 1) / CH, p.batch, grid_z);
    vscan::stream_scan_kernel<RK, T, N16, KC, MODE, PW, FL, CH, TOK, SS>
        <<<grid, vscan::StreamShape<T, KC, MODE, PW, CH, TOK, SS>::THREADS, smem, s>>>(p);
    return cudaGetLastError();
}

// ATROUS2: every pixel has one owner; float32 I/O runs one direction per CTA
//   (grid.z = 4), bf16 I/O all four directions per CTA.
// BIDIR, CROSS4: all directions of an image tile in one CTA, merged by parking.
template <int RK, typename T, bool N16, int FL>
cudaError_t launch_stream_n(const vscan::ScanParams& p, cudaStream_t s)
{
    using namespace vscan;
    if constexpr (RK == RK_ATROUS2) {
        if constexpr (sizeof(T) == 4) {
            // few CTAs per SM: each channel's states split over two consumer warps and
            // each chunk's steps over two producer warps, so every warp runs a chain
            // half as long per chunk
            if (atrous_split((long long)p.batch * ((p.D + ST_CH - 1) / ST_CH) * 4, (FL & FL_ZOH) != 0))
                return launch_stream_mode<RK, T, N16, 1, MODE_OWNER, 2, FL, ST_TOK, ST_CH, 2>(p, 0, 4, s);
            return launch_stream_mode<RK, T, N16, 1, MODE_OWNER, 1, FL>(p, 0, 4, s);
        }
        else return launch_stream_mode<RK, T, N16, 4, MODE_OWNER, 1, FL>(p, 0, 1, s);
    } else if constexpr (RK == RK_BIDIR) {
        // two producer warps per direction (measured faster on Vim-Small); the fused
        // convolution reads steps gathered by one producer warp and keeps one.
        constexpr int PW = (FL & FL_CONV) ? 1 : 2;
        // 32-step chunks halve the barriers per token: measured 3-9 % faster for bf16
        // sequences of 4097 steps, but slower for float32, for short sequences and with
        // the ZOH or convolution options (which stay at 16, as does the checkpointing run
        // the backward scan's 16-step chunks read).
        if constexpr (FL == 0 && sizeof(T) == 2) {
            if (p.g.L >= kLongChunkMinL) return launch_stream_mode<RK, T, N16, 2, MODE_PARK, PW, FL, 32>(p, 0, 1, s);
        }
        return launch_stream_mode<RK, T, N16, 2, MODE_PARK, PW, FL>(p, 0, 1, s);
    } else {
        return launch_stream_mode<RK, T, N16, 4, MODE_PARK, 1, FL>(p, 0, 1, s);
    }
}

template <int RK, typename T, int FL>
cudaError_t launch_stream_fl(const vscan::ScanParams& p, cudaStream_t s)
{
    return p.N == 16 ? launch_stream_n<RK, T, true, FL>(p, s) : launch_stream_n<RK, T, false, FL>(p, s);
}

// fl: OR of vscan::FL_ZOH and vscan::FL_CONV (the latter for BIDIR only).
template <int RK, typename T>
cudaError_t launch_stream(const vscan::ScanParams& p, int fl, cudaStream_t s)
{
    using namespace vscan;
    if (fl & FL_CKPT) return launch_stream_fl<RK, T, FL_CKPT>(p, s);  // backward's forward run (plain scan)
    if constexpr (RK == RK_BIDIR) {
        switch (fl) {
        case FL_ZOH: return launch_stream_fl<RK, T, FL_ZOH>(p, s);
        case FL_CONV: return launch_stream_fl<RK, T, FL_CONV>(p, s);
        case FL_ZOH | FL_CONV: return launch_stream_fl<RK, T, FL_ZOH | FL_CONV>(p, s);
        default: return launch_stream_fl<RK, T, 0>(p, s);
        }
    } else {
        return (fl & FL_ZOH) ? launch_stream_fl<RK, T, FL_ZOH>(p, s) : launch_stream_fl<RK, T, 0>(p, s);
    }
}

// The mbarrier-pipelined kernel (BIDIR, CROSS4; d_state 16; no optional step,
// or the checkpoints of the backward's forward run).
template <int RK, typename T, int LPC, int TOK, int NS, int MP, int MINB, int FL>
cudaError_t launch_pipe_cfg(const vscan::ScanParams& p, cudaStream_t s)
{
    using Sh = vscan::PipeShape<RK, T, LPC, TOK, NS>;
    const size_t smem = vscan::pipe_smem_bytes<RK, T, LPC, TOK, NS>();
    static int attr_done[kAttrDevices] = {};
    cudaError_t e = set_smem_once(vscan::pipe_scan_kernel<RK, T, LPC, TOK, NS, MP, MINB, FL>, (int)smem,
                                  attr_done, kAttrDevices);
    if (e != cudaSuccess) return e;
    const dim3 grid((p.D + Sh::CT - 1) / Sh::CT, p.batch);
    vscan::pipe_scan_kernel<RK, T, LPC, TOK, NS, MP, MINB, FL><<<grid, Sh::THREADS, smem, s>>>(p);
    return cudaGetLastError();
}

// Launch shape per route, measured on B200 (Vim-Small b64 bf16, SS2D b16 bf16):
// BIDIR two lanes per channel (16-channel tiles), 16-step chunks, two slots,
// launch bounds for 8 CTAs per SM (80 registers; shared memory then also fits
// 8, where three slots fit 7 and measured 6 % slower); CROSS4 four lanes per
// channel (8-channel tiles: about ten consumer warps per SM on the SS2D grid),
// 32-step chunks with two slots. The checkpointing run of the backward pass
// takes 16-step chunks (the adjoint scan's spacing).
template <int RK, typename T, int FL>
cudaError_t launch_pipe(const vscan::ScanParams& p, cudaStream_t s)
{
    constexpr bool CK = (FL & vscan::FL_CKPT) != 0;
    if constexpr (RK == vscan::RK_BIDIR) return launch_pipe_cfg<RK, T, 2, 16, 2, 0, 8, FL>(p, s);
    else if constexpr (CK) return launch_pipe_cfg<RK, T, 4, 16, 3, 0, 4, FL>(p, s);
    else return launch_pipe_cfg<RK, T, 4, 32, 2, 0, 3, FL>(p, s);
}

// BIDIR and CROSS4 forwards with d_state 16 and none of the optional steps (the
// backward's checkpointing run included) take the pipelined kernel when they
// stream (the resident chunked kernel keeps the small grids).
bool use_pipe(const vscan_route* r, const vscan_args* a, int fl)
{
    return (r->g.kind == vscan::RK_BIDIR || r->g.kind == vscan::RK_CROSS4) && (fl & ~vscan::FL_CKPT) == 0 &&
           a->d_state == 16;
}

template <int RK, typename T, int NC, int FL, int CH>
cudaError_t launch_resident_ch(const vscan::ScanParams& p, cudaStream_t s)
{
    constexpr int threads = vscan::ResidentShape<RK>::K * CH * NC * 4;  // one channel-direction per 32 / (4 NC) lanes
    const int Ki = p.in_dir ? p.g.K : 1;
    const int Kd = (p.in_dir || p.v_dir) ? p.g.K : 1;
    const size_t smem = vscan::resident_smem_bytes(RK, p.g.tokens, Ki, Kd, (FL & vscan::FL_CONV) != 0, CH);
    static int attr_done[kAttrDevices] = {};
    cudaError_t e = set_smem_once(vscan::resident_scan_kernel<RK, T, NC, FL, CH>, (int)kMaxSmem, attr_done,
                                  kAttrDevices);
    if (e != cudaSuccess) return e;
    const dim3 grid((p.D + CH - 1) / CH, p.batch);
    vscan::resident_scan_kernel<RK, T, NC, FL, CH><<<grid, threads, smem, s>>>(p);
    return cudaGetLastError();
}

// BIDIR takes 4-channel tiles when 8-channel ones would give fewer CTAs than SMs
// (Vim-Tiny at batch 1: 96 CTAs instead of 48), so that twice as many SMs share the
// latency-bound chains.
template <int RK, typename T, int NC, int FL>
cudaError_t launch_resident_nc(const vscan::ScanParams& p, cudaStream_t s)
{
    constexpr int CH = vscan::ResidentShape<RK>::CH;
    if constexpr (CH == 8 && NC >= 2) {
        if ((long long)p.batch * ((p.D + CH - 1) / CH) < num_sms()) return launch_resident_ch<RK, T, NC, FL, 4>(p, s);
    }
    return launch_resident_ch<RK, T, NC, FL, CH>(p, s);
}

template <int RK, typename T, int FL>
cudaError_t launch_resident_fl(const vscan::ScanParams& p, int nc, cudaStream_t s)
{
    switch (nc) {
    case 2: return launch_resident_nc<RK, T, 2, FL>(p, s);
    case 4: return launch_resident_nc<RK, T, 4, FL>(p, s);
    default: return launch_resident_nc<RK, T, 8, FL>(p, s);
    }
}

template <int RK, typename T>
cudaError_t launch_resident(const vscan::ScanParams& p, int nc, int fl, cudaStream_t s)
{
    using namespace vscan;
    if constexpr (RK == RK_BIDIR) {
        switch (fl) {
        case FL_ZOH: return launch_resident_fl<RK, T, FL_ZOH>(p, nc, s);
        case FL_CONV: return launch_resident_fl<RK, T, FL_CONV>(p, nc, s);
        case FL_ZOH | FL_CONV: return launch_resident_fl<RK, T, FL_ZOH | FL_CONV>(p, nc, s);
        default: return launch_resident_fl<RK, T, 0>(p, nc, s);
        }
    } else {
        return (fl & FL_ZOH) ? launch_resident_fl<RK, T, FL_ZOH>(p, nc, s) : launch_resident_fl<RK, T, 0>(p, nc, s);
    }
}

// The pooled route's two launches; a failure names the step that failed.
template <typename T, int FL>
vscan_status launch_pool_fl(const vscan::PoolParams& p, cudaStream_t s, size_t ws_bytes)
{
    if constexpr ((FL & vscan::FL_MASK) != 0) {
        // B and C sums are added into the zeroed workspace (pB and pC)
        cudaError_t e = cudaMemsetAsync(p.pB, 0, ws_bytes, s);
        if (e != cudaSuccess) return cuda_fail(e, "zeroing the pooled B/C sums");
        if (p.n_tok > 0) {
            constexpr int per_cta = 16 * vscan::PB_RUN;  // tokens of one CTA
            const dim3 g1((unsigned)((p.n_tok + per_cta - 1) / per_cta), p.batch, p.Ki);
            vscan::pool_bc_masked_kernel<T><<<g1, 256, 0, s>>>(p);
            e = cudaGetLastError();
            if (e != cudaSuccess) return cuda_fail(e, "launching pool_bc_masked_kernel");
        }
    } else {
        const dim3 g1(p.g.L, p.batch, p.Ki);
        vscan::pool_bc_kernel<T><<<g1, 128, 0, s>>>(p);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(e, "launching pool_bc_kernel");
    }
    const size_t smem = vscan::pool_scan_smem_bytes(p.Ki, p.g.L, (FL & vscan::FL_CONV) != 0);
    static int attr_done[kAttrDevices] = {};
    cudaError_t e = set_smem_once(vscan::pool_scan_kernel<T, FL>, (int)kMaxSmem, attr_done, kAttrDevices);
    if (e != cudaSuccess) return cuda_fail(e, "setting pool_scan_kernel's shared-memory limit");
    const dim3 g2((p.D + vscan::PL_CH - 1) / vscan::PL_CH, p.batch);
    vscan::pool_scan_kernel<T, FL><<<g2, vscan::PL_THREADS, smem, s>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "launching pool_scan_kernel");
    return VSCAN_OK;
}

template <typename T>
vscan_status launch_pool(const vscan::PoolParams& p, int fl, cudaStream_t s, size_t ws_bytes)
{
    using namespace vscan;
    switch (fl) {
    case FL_ZOH: return launch_pool_fl<T, FL_ZOH>(p, s, ws_bytes);
    case FL_CONV: return launch_pool_fl<T, FL_CONV>(p, s, ws_bytes);
    case FL_ZOH | FL_CONV: return launch_pool_fl<T, FL_ZOH | FL_CONV>(p, s, ws_bytes);
    case FL_MASK: return launch_pool_fl<T, FL_MASK>(p, s, ws_bytes);
    case FL_MASK | FL_ZOH: return launch_pool_fl<T, FL_MASK | FL_ZOH>(p, s, ws_bytes);
    default: return launch_pool_fl<T, 0>(p, s, ws_bytes);
    }
}

template <typename T>
vscan_status dispatch(const vscan_route* r, const vscan_args* a, cudaStream_t s, float* ckpt = nullptr)
{
    const vscan::RouteGeom& g = r->g;
    const long long plane = (long long)a->batch * tokens_of(r, a);
    const int fl = ((a->flags & VSCAN_FLAG_ZOH) ? vscan::FL_ZOH : 0) | (a->conv_w ? vscan::FL_CONV : 0) |
                   (a->token_pos ? vscan::FL_MASK : 0) | (ckpt ? vscan::FL_CKPT : 0);
    if (is_pool(g.kind)) {
        vscan::PoolParams p{};
        p.g = g;
        p.batch = a->batch; p.D = a->channels; p.N = a->d_state;
        p.Ki = a->per_dir_inputs ? 2 : 1;
        p.u = a->u; p.delta = a->delta; p.B = a->B; p.C = a->C; p.z = a->z; p.y = a->y;
        p.A = a->A; p.Dskip = a->Dskip; p.bias = a->delta_bias;
        p.in_dir = a->per_dir_inputs ? plane * a->channels : 0;
        p.bc_dir = a->per_dir_inputs ? plane * a->d_state : 0;
        p.a_dir = a->per_dir_params ? a->channels * a->d_state : 0;
        p.v_dir = a->per_dir_params ? a->channels : 0;
        p.softplus = a->delta_softplus;
        p.merge_scale = a->merge_scale;
        const uint64_t half = workspace_need(r, a) / 2;
        p.pB = static_cast<float*>(a->workspace);
        p.pC = reinterpret_cast<float*>(static_cast<char*>(a->workspace) + half);
        p.conv_w = a->conv_w; p.conv_b = a->conv_b;
        p.pos = a->token_pos;
        p.n_tok = tokens_of(r, a);
        const vscan_status st = launch_pool<T>(p, fl, s, workspace_need(r, a));
        if (st != VSCAN_OK) return st;
    } else {
        vscan::ScanParams p{};
        p.g = g;
        p.batch = a->batch; p.D = a->channels; p.N = a->d_state;
        p.u = a->u; p.delta = a->delta; p.B = a->B; p.C = a->C; p.z = a->z; p.y = a->y;
        p.A = a->A; p.Dskip = a->Dskip; p.bias = a->delta_bias;
        p.in_dir = a->per_dir_inputs ? plane * a->channels : 0;
        p.bc_dir = a->per_dir_inputs ? plane * a->d_state : 0;
        p.a_dir = a->per_dir_params ? a->channels * a->d_state : 0;
        p.v_dir = a->per_dir_params ? a->channels : 0;
        p.softplus = a->delta_softplus;
        p.merge_scale = a->merge_scale;
        p.scratch = static_cast<float*>(a->workspace);
        p.conv_w = a->conv_w; p.conv_b = a->conv_b;
        p.ckpt = ckpt;
        p.status = a->status;
        const int nc = ckpt ? 1 : choose_chunks(r, a);  // checkpoints come from the streaming kernel
        if (nc == 1 && use_pipe(r, a, fl)) {
            cudaError_t e;
            if (ckpt)
                e = g.kind == vscan::RK_BIDIR ? launch_pipe<vscan::RK_BIDIR, T, vscan::FL_CKPT>(p, s)
                                              : launch_pipe<vscan::RK_CROSS4, T, vscan::FL_CKPT>(p, s);
            else
                e = g.kind == vscan::RK_BIDIR ? launch_pipe<vscan::RK_BIDIR, T, 0>(p, s)
                                              : launch_pipe<vscan::RK_CROSS4, T, 0>(p, s);
            if (e != cudaSuccess) return cuda_fail(e, "launching pipe_scan_kernel");
        } else if (nc > 1) {
            cudaError_t e;
            switch (g.kind) {
            case vscan::RK_BIDIR: e = launch_resident<vscan::RK_BIDIR, T>(p, nc, fl, s); break;
            case vscan::RK_CROSS4: e = launch_resident<vscan::RK_CROSS4, T>(p, nc, fl, s); break;
            default: e = launch_resident<vscan::RK_ATROUS2, T>(p, nc, fl, s); break;
            }
            if (e != cudaSuccess) return cuda_fail(e, "configuring the resident scan kernel");
        } else {
            cudaError_t e;
            switch (g.kind) {
            case vscan::RK_BIDIR: e = launch_stream<vscan::RK_BIDIR, T>(p, fl, s); break;
            case vscan::RK_CROSS4: e = launch_stream<vscan::RK_CROSS4, T>(p, fl, s); break;
            default: e = launch_stream<vscan::RK_ATROUS2, T>(p, fl, s); break;
            }
            if (e != cudaSuccess) return cuda_fail(e, "configuring the streaming scan kernel");
        }
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
    return VSCAN_OK;
}

// VSCAN_FLAG_CHECK_VALUES: one bandwidth-bound pass over every input.
vscan_status launch_value_checks(const vscan_route* r, const vscan_args* a, cudaStream_t s)
{
    vscan::CheckParams c{};
    const int K = r->g.K;
    const long long Ki = a->per_dir_inputs ? K : 1, Kp = a->per_dir_params ? K : 1;
    const long long plane = (long long)a->batch * tokens_of(r, a);
    const int bf = a->dtype == VSCAN_BF16;
    auto add = [&](const void* ptr, long long n, int is_bf16, int nonpos, int vec) {
        if (ptr && n > 0) c.seg[c.nseg++] = vscan::CheckSeg{ptr, n, is_bf16, nonpos, vec};
    };
    add(a->u, Ki * plane * a->channels, bf, 0, 1);
    add(a->delta, Ki * plane * a->channels, bf, 0, 1);
    add(a->B, Ki * plane * a->d_state, bf, 0, 0);
    add(a->C, Ki * plane * a->d_state, bf, 0, 0);
    add(a->z, plane * a->channels, bf, 0, 1);
    add(a->A, Kp * a->channels * a->d_state, 0, 1, 0);
    add(a->Dskip, Kp * a->channels, 0, 0, 0);
    add(a->delta_bias, Kp * a->channels, 0, 0, 0);
    add(a->conv_w, Kp * a->channels * 4, 0, 0, 0);
    add(a->conv_b, Kp * a->channels, 0, 0, 0);
    c.status = a->status;
    c.dt_check = a->delta_softplus ? 0 : 1;
    c.delta = a->delta;
    c.delta_bf16 = bf;
    c.bias = a->delta_bias;
    c.plane = plane * a->channels;
    c.D = a->channels;
    c.Ki = (int)Ki;
    c.Kp = (int)Kp;
    const dim3 grid((unsigned)(4 * num_sms()), (unsigned)(c.nseg + c.dt_check));
    vscan::check_values_kernel<<<grid, 256, 0, s>>>(c);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "launching check_values_kernel");
    return VSCAN_OK;
}

// Packed copies of strided tensors, placed in the workspace after the path's
// own scratch (offsets from its start; main: u, delta, z and y are packed; bc:
// B and C are).
struct PackLayout {
    bool main, bc;
    uint64_t u, d, z, y, B, C, total;
};

uint64_t pack_layout(const vscan_route* r, const vscan_args* a, PackLayout* L)
{
    *L = PackLayout{};
    const bool mn = strided_main(r, a), bc = strided_bc(r, a);
    if (!mn && !bc) return 0;
    const int Ki = a->per_dir_inputs ? r->g.K : 1;
    const uint64_t eb = a->dtype == VSCAN_F32 ? 4 : 2;
    const uint64_t plane = (uint64_t)a->batch * tokens_of(r, a);
    uint64_t off = round256(workspace_need(r, a));
    auto take = [&](uint64_t bytes) { const uint64_t o = off; off += round256(bytes); return o; };
    L->main = mn;
    L->bc = bc;
    if (mn) {
        L->u = take(Ki * plane * a->channels * eb);
        L->d = take(Ki * plane * a->channels * eb);
        if (a->z) L->z = take(plane * a->channels * eb);
        L->y = take(plane * a->channels * eb);
    }
    if (bc) {
        L->B = take(Ki * plane * a->d_state * eb);
        L->C = take(Ki * plane * a->d_state * eb);
    }
    L->total = off;
    return off;
}

// Workspace bytes vscan_forward needs: the path's scratch, plus the packed copies
// of strided tensors.
uint64_t forward_workspace_need(const vscan_route* r, const vscan_args* a)
{
    PackLayout L;
    const uint64_t packed = pack_layout(r, a, &L);
    return packed ? packed : workspace_need(r, a);
}

// Copy nimg images of ntok rows of `row` elements between strided layouts (strides
// in elements of size eb); 16-byte pieces where rows, strides and both bases allow.
vscan_status copy_rows(const void* src, long long s_img, long long s_tok, void* dst, long long d_img,
                       long long d_tok, int nimg, int ntok, int row, int eb, cudaStream_t s)
{
    if (nimg == 0 || ntok == 0) return VSCAN_OK;
    const long long bytes = (long long)row * eb;
    const bool v16 = bytes % 16 == 0 && (s_img * eb) % 16 == 0 && (s_tok * eb) % 16 == 0 &&
                     (d_img * eb) % 16 == 0 && (d_tok * eb) % 16 == 0 && aligned16(src) && aligned16(dst);
    const dim3 grid((unsigned)std::min(1024, (ntok + 7) / 8), (unsigned)std::min(nimg, 65535));
    if (v16) {
        const long long k = 16 / eb;
        vscan::copy_rows_kernel<uint4><<<grid, 256, 0, s>>>(static_cast<const uint4*>(src), s_img / k, s_tok / k,
                                                            static_cast<uint4*>(dst), d_img / k, d_tok / k, nimg,
                                                            ntok, (int)(bytes / 16));
    } else if (eb == 4) {
        vscan::copy_rows_kernel<uint32_t><<<grid, 256, 0, s>>>(static_cast<const uint32_t*>(src), s_img, s_tok,
                                                               static_cast<uint32_t*>(dst), d_img, d_tok, nimg,
                                                               ntok, row);
    } else {
        vscan::copy_rows_kernel<uint16_t><<<grid, 256, 0, s>>>(static_cast<const uint16_t*>(src), s_img, s_tok,
                                                               static_cast<uint16_t*>(dst), d_img, d_tok, nimg,
                                                               ntok, row);
    }
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? VSCAN_OK : cuda_fail(e, "launching copy_rows_kernel");
}

vscan_status forward_dense(const vscan_route* r, const vscan_args* a, cudaStream_t s, float* ckpt)
{
    if (a->flags & VSCAN_FLAG_CHECK_VALUES) {
        const vscan_status st = launch_value_checks(r, a, s);
        if (st != VSCAN_OK) return st;
    }
    return a->dtype == VSCAN_F32 ? dispatch<float>(r, a, s, ckpt) : dispatch<__nv_bfloat16>(r, a, s, ckpt);
}

vscan_status forward_device(const vscan_route* r, const vscan_args* a, cudaStream_t s, float* ckpt = nullptr)
{
    PackLayout L;
    const uint64_t packed = pack_layout(r, a, &L);
    const uint64_t need = packed ? packed : workspace_need(r, a);
    if (need > 0) {
        if (!a->workspace || a->workspace_bytes < need)
            return fail(VSCAN_ERR_WORKSPACE, "workspace of %llu bytes needed, %llu given",
                        (unsigned long long)need, (unsigned long long)(a->workspace ? a->workspace_bytes : 0));
        if (!aligned16(a->workspace)) return fail(VSCAN_ERR_ALIGNMENT, "workspace is not 16-byte aligned");
    }
    if (a->batch == 0) return VSCAN_OK;
    if (!packed) return forward_dense(r, a, s, ckpt);

    // strided tensors: pack them densely, scan, copy y out
    char* ws = static_cast<char*>(a->workspace);
    vscan_args b = *a;
    b.tok_stride = b.batch_stride = b.bc_tok_stride = b.bc_batch_stride = 0;
    b.workspace_bytes = workspace_need(r, a);
    const int Ki = a->per_dir_inputs ? r->g.K : 1, T = tokens_of(r, a), D = a->channels, N = a->d_state;
    const int eb = a->dtype == VSCAN_F32 ? 4 : 2;
    const long long ts = tok_stride_of(a), bs = batch_stride_of(r, a);
    const long long bts = bc_tok_stride_of(a), bbs = bc_batch_stride_of(r, a);
    vscan_status st = VSCAN_OK;
    if (L.main) {
        b.u = ws + L.u;
        b.delta = ws + L.d;
        st = copy_rows(a->u, bs, ts, ws + L.u, (long long)T * D, D, Ki * a->batch, T, D, eb, s);
        if (st == VSCAN_OK) st = copy_rows(a->delta, bs, ts, ws + L.d, (long long)T * D, D, Ki * a->batch, T, D, eb, s);
        if (st == VSCAN_OK && a->z) {
            b.z = ws + L.z;
            st = copy_rows(a->z, bs, ts, ws + L.z, (long long)T * D, D, a->batch, T, D, eb, s);
        }
        b.y = ws + L.y;
    }
    if (st == VSCAN_OK && L.bc) {
        b.B = ws + L.B;
        b.C = ws + L.C;
        st = copy_rows(a->B, bbs, bts, ws + L.B, (long long)T * N, N, Ki * a->batch, T, N, eb, s);
        if (st == VSCAN_OK) st = copy_rows(a->C, bbs, bts, ws + L.C, (long long)T * N, N, Ki * a->batch, T, N, eb, s);
    }
    if (st == VSCAN_OK) st = forward_dense(r, &b, s, ckpt);
    if (st == VSCAN_OK && L.main) st = copy_rows(ws + L.y, (long long)T * D, D, a->y, bs, ts, a->batch, T, D, eb, s);
    return st;
}

// Entry points that take dense tensors only.
vscan_status require_dense(const vscan_route* r, const vscan_args* a, const char* what)
{
    if (strided_main(r, a) || strided_bc(r, a))
        return fail(VSCAN_ERR_UNSUPPORTED, "%s takes dense tensors only (strides 0 or the dense values)", what);
    return VSCAN_OK;
}

int forward_flags(const vscan_args* a)
{
    return ((a->flags & VSCAN_FLAG_ZOH) ? vscan::FL_ZOH : 0) | (a->conv_w ? vscan::FL_CONV : 0) |
           (a->token_pos ? vscan::FL_MASK : 0);
}

__global__ void route_map_kernel(vscan::RouteGeom g, int32_t* out)
{
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx < (long long)g.K * g.L) {
        const int k = (int)(idx / g.L);
        const int t = (int)(idx - (long long)k * g.L);
        out[idx] = vscan::route_token_any(g, k, t);
    }
}

struct HostLayout {
    size_t u, delta, B, C, z, y, A, Dskip, bias, conv_w, conv_b, pos, ws, total;
};

HostLayout host_layout(const vscan_route* r, const vscan_args* a)
{
    const vscan::RouteGeom& g = r->g;
    const size_t eb = elem_bytes(a->dtype);
    const size_t Ki = a->per_dir_inputs ? g.K : 1;
    const size_t Kp = a->per_dir_params ? g.K : 1;
    const size_t plane = (size_t)a->batch * tokens_of(r, a);
    HostLayout L{};
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t o = off; off += round256(bytes); return o; };
    L.u = take(Ki * plane * a->channels * eb);
    L.delta = take(Ki * plane * a->channels * eb);
    L.B = take(Ki * plane * a->d_state * eb);
    L.C = take(Ki * plane * a->d_state * eb);
    L.z = take(a->z ? plane * a->channels * eb : 0);
    L.y = take(plane * a->channels * eb);
    L.A = take(Kp * a->channels * a->d_state * sizeof(float));
    L.Dskip = take(a->Dskip ? Kp * a->channels * sizeof(float) : 0);
    L.bias = take(a->delta_bias ? Kp * a->channels * sizeof(float) : 0);
    L.conv_w = take(a->conv_w ? Kp * a->channels * 4 * sizeof(float) : 0);
    L.conv_b = take(a->conv_b ? Kp * a->channels * sizeof(float) : 0);
    L.pos = take(a->token_pos ? plane * sizeof(int32_t) : 0);
    L.ws = take(workspace_need(r, a));
    L.total = off;
    return L;
}

// ---- fixed scratch for vscan_forward_pooled_noalloc ---------------------------------
// The pooled routes need scratch only for the pooled B and C
// (2 x Ki x batch x L x N floats). This array holds it for callers that cannot
// allocate device memory; every GPU that loads the library keeps it until exit.
constexpr size_t kStaticScratchBytes = size_t(4) << 20;  // 4 MiB
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// Device address of g_static_scratch, resolved once per device: in host code the
// symbol is only a host-side stand-in and must never be passed to a kernel.
constexpr int kMaxDevices = 64;
std::mutex g_static_mutex;
void* g_static_addr[kMaxDevices] = {};

vscan_status static_scratch_address(void** out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(VSCAN_ERR_UNSUPPORTED, "device ordinal %d >= %d", dev, kMaxDevices);
    std::lock_guard<std::mutex> lock(g_static_mutex);
    if (!g_static_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_static_scratch);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress of the fixed scratch");
        g_static_addr[dev] = p;
    }
    *out = g_static_addr[dev];
    return VSCAN_OK;
}

// ---- backward ----------------------------------------------------------------------
// the streaming kernel saves its state every ST_TOK steps for the adjoint scan's BW_TOK chunks
static_assert(vscan::ST_TOK == vscan::BW_TOK, "checkpoint spacing of the forward and backward scans");
struct BwdLayout {
    size_t fwd_ws, pre, gy, ckpt, pu, praw, pB, pC, pg, dpu, dpraw, dpB, dpC, total;
};

BwdLayout bwd_layout(const vscan_route* r, const vscan_args* a)
{
    const vscan::RouteGeom& g = r->g;
    const size_t eb = elem_bytes(a->dtype);
    const size_t Ki = a->per_dir_inputs ? g.K : 1;
    const size_t b = a->batch, T = g.tokens, D = a->channels, N = a->d_state, L = g.L;
    const size_t nch = (L + vscan::BW_TOK - 1) / vscan::BW_TOK;
    BwdLayout Lo{};
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t o = off; off += round256(bytes); return o; };
    Lo.fwd_ws = take(workspace_need(r, a));
    Lo.pre = take(b * T * D * eb);
    Lo.gy = take(is_pool(g.kind) ? 0 : b * T * D * sizeof(float));  // pooled routes sum gy while pooling
    Lo.ckpt = take((size_t)g.K * b * nch * D * 16 * sizeof(float));
    if (is_pool(g.kind)) {
        Lo.pu = take(Ki * b * L * D * sizeof(float));
        Lo.praw = take(Ki * b * L * D * sizeof(float));
        Lo.pB = take(Ki * b * L * N * sizeof(float));
        Lo.pC = take(Ki * b * L * N * sizeof(float));
        Lo.pg = take(b * L * D * sizeof(float));
        Lo.dpu = take(Ki * b * L * D * sizeof(float));
        Lo.dpraw = take(Ki * b * L * D * sizeof(float));
        Lo.dpB = take(Ki * b * L * N * sizeof(float));
        Lo.dpC = take(Ki * b * L * N * sizeof(float));
    }
    Lo.total = off;
    return Lo;
}

vscan_status check_backward(const vscan_route* r, const vscan_args* a)
{
    vscan_status st = check_shape(r, a);
    if (st != VSCAN_OK) return st;
    if (a->conv_w) return fail(VSCAN_ERR_UNSUPPORTED, "the backward pass does not take the fused convolution");
    if (a->flags & VSCAN_FLAG_ZOH) return fail(VSCAN_ERR_UNSUPPORTED, "the backward pass is for the Delta*B*u write term");
    if (a->token_pos) return fail(VSCAN_ERR_UNSUPPORTED, "the backward pass does not take a masked token set");
    st = require_dense(r, a, "vscan_backward");
    if (st != VSCAN_OK) return st;
    return VSCAN_OK;
}

// The adjoint scan. Grids of at most 8 tiles (8 channels, one image, one direction)
// per SM split every tile's states over a CTA of two warps: twice the warps, each with
// half the per-step chain (measured 7-13 % faster than one warp per tile on Vim-Tiny
// b1 and b8, the atrous b8 and SS2D b8 grids). Larger grids take one warp per tile,
// built for 16 resident warps per SM, where the split's extra instructions cost more
// than its latency hiding gains (SS2D b16 2.24 against 2.17 ms, Vim-Small b64 17.6
// against 16.9 ms).
bool bwd_split(long long tiles) { return tiles <= 8LL * num_sms(); }

// Tiles of the adjoint scan's grid: channel tiles x images x directions (2 for the
// pooled routes, whose pooled sequence is scanned as a bidirectional route).
long long bwd_tiles(const vscan_route* r, const vscan_args* a)
{
    return (long long)((a->channels + vscan::BW_CH - 1) / vscan::BW_CH) * a->batch * r->g.K;
}

template <int RK, typename T, bool ASYNC>
void launch_bwd_scan_async(const vscan::BwdParams& p, dim3 grid, cudaStream_t s)
{
    if (bwd_split((long long)grid.x * grid.y * grid.z))
        vscan::bwd_scan_split_kernel<RK, T, ASYNC><<<grid, vscan::BWS_THREADS, 0, s>>>(p);
    else
        vscan::bwd_scan_kernel<RK, T, ASYNC><<<grid, 32, 0, s>>>(p);
}

// d_state 16 takes the build that gathers the next chunk with cp.async while the
// current one runs (16-byte rows of B and C); other state counts load per element.
template <int RK, typename T>
void launch_bwd_scan(const vscan::BwdParams& p, dim3 grid, cudaStream_t s)
{
    if (p.N == 16) launch_bwd_scan_async<RK, T, true>(p, grid, s);
    else launch_bwd_scan_async<RK, T, false>(p, grid, s);
}

template <typename T>
vscan_status backward_device(const vscan_route* r, const vscan_args* a, const void* dy, const vscan_grads* gr,
                             cudaStream_t s)
{
    const vscan::RouteGeom& g = r->g;
    const BwdLayout Lo = bwd_layout(r, a);
    char* ws = static_cast<char*>(gr->workspace);
    const int K = g.K, Ki = a->per_dir_inputs ? K : 1, Kp = a->per_dir_params ? K : 1;
    const long long b = a->batch, TK = g.tokens, D = a->channels, N = a->d_state, L = g.L;
    const bool pooled = is_pool(g.kind);

    struct Zero { void* p; size_t bytes; };
    // token gradients are accumulated with atomics on the grid routes; the pooled
    // routes write them in full (bwd_unpool_kernel) and zero their pooled copies
    const Zero zeros[] = {
        {pooled ? nullptr : gr->du, (size_t)Ki * b * TK * D * 4},
        {pooled ? nullptr : gr->ddelta, (size_t)Ki * b * TK * D * 4},
        {pooled ? nullptr : gr->dB, (size_t)Ki * b * TK * N * 4},
        {pooled ? nullptr : gr->dC, (size_t)Ki * b * TK * N * 4},
        {gr->dA, (size_t)Kp * D * N * 4}, {gr->dDskip, (size_t)Kp * D * 4}, {gr->dbias, (size_t)Kp * D * 4},
        {pooled ? ws + Lo.dpu : nullptr, Lo.dpraw - Lo.dpu}, {pooled ? ws + Lo.dpraw : nullptr, Lo.dpB - Lo.dpraw},
        {pooled ? ws + Lo.dpB : nullptr, Lo.dpC - Lo.dpB}, {pooled ? ws + Lo.dpC : nullptr, Lo.total - Lo.dpC},
    };
    for (const Zero& z : zeros) {
        if (!z.p || z.bytes == 0) continue;
        cudaError_t e = cudaMemsetAsync(z.p, 0, z.bytes, s);
        if (e != cudaSuccess) return cuda_fail(e, "zeroing a gradient");
    }
    // forward without the gate: pre = s * merged scan output
    vscan_args fa = *a;
    fa.z = nullptr;
    fa.y = ws + Lo.pre;
    fa.workspace = ws + Lo.fwd_ws;
    fa.workspace_bytes = Lo.pre - Lo.fwd_ws;
    // grid routes: the forward's streaming kernel also saves the state at every
    // chunk boundary, so the adjoint scan needs no forward pass of its own
    float* ckpt = reinterpret_cast<float*>(ws + Lo.ckpt);
    vscan_status st = forward_device(r, &fa, s, pooled ? nullptr : ckpt);
    if (st != VSCAN_OK) return st;
    // gradient of the gate and of the merged value (the pooled routes form it inside
    // their pooling kernel, member by member)
    float* gy = reinterpret_cast<float*>(ws + Lo.gy);
    if (!pooled) {
        const long long n = b * TK * D;
        const unsigned blocks = (unsigned)std::min<long long>((n + 255) / 256, 148LL * 16);
        vscan::gate_grad_kernel<T><<<blocks, 256, 0, s>>>(static_cast<const T*>(dy), static_cast<const T*>(a->z),
                                                          static_cast<const T*>(fa.y), a->merge_scale, n, gy, gr->dz);
    }
    vscan::BwdParams p{};
    p.batch = a->batch; p.D = a->channels; p.N = a->d_state;
    p.a_dir = a->per_dir_params ? a->channels * a->d_state : 0;
    p.v_dir = a->per_dir_params ? a->channels : 0;
    p.A = a->A; p.Dskip = a->Dskip; p.bias = a->delta_bias; p.softplus = a->delta_softplus;
    p.ckpt = ckpt;
    p.ckpt_ready = pooled ? 0 : 1;
    p.dA = gr->dA; p.dD = gr->dDskip; p.dbias = gr->dbias;
    const dim3 grid((unsigned)((D + vscan::BW_CH - 1) / vscan::BW_CH), (unsigned)b, (unsigned)K);
    if (!pooled) {
        p.g = g;
        p.u = a->u; p.delta = a->delta; p.B = a->B; p.C = a->C;
        p.in_dir = a->per_dir_inputs ? b * TK * D : 0;
        p.bc_dir = a->per_dir_inputs ? b * TK * N : 0;
        p.gy = gy;
        p.du = gr->du; p.ddelta = gr->ddelta; p.dB = gr->dB; p.dC = gr->dC;
        switch (g.kind) {
        case vscan::RK_BIDIR: launch_bwd_scan<vscan::RK_BIDIR, T>(p, grid, s); break;
        case vscan::RK_CROSS4: launch_bwd_scan<vscan::RK_CROSS4, T>(p, grid, s); break;
        default: launch_bwd_scan<vscan::RK_ATROUS2, T>(p, grid, s); break;
        }
    } else {
        float* pu = reinterpret_cast<float*>(ws + Lo.pu);
        float* praw = reinterpret_cast<float*>(ws + Lo.praw);
        float* pB = reinterpret_cast<float*>(ws + Lo.pB);
        float* pC = reinterpret_cast<float*>(ws + Lo.pC);
        float* pg = reinterpret_cast<float*>(ws + Lo.pg);
        const long long in_dir = a->per_dir_inputs ? b * TK * D : 0, bc_dir = a->per_dir_inputs ? b * TK * N : 0;
        vscan::bwd_pool_kernel<T><<<dim3((unsigned)L, (unsigned)b), 256, 0, s>>>(
            g, (int)b, (int)D, (int)N, Ki, static_cast<const T*>(a->u), static_cast<const T*>(a->delta),
            static_cast<const T*>(a->B), static_cast<const T*>(a->C), in_dir, bc_dir, static_cast<const T*>(dy),
            static_cast<const T*>(a->z), static_cast<const T*>(fa.y), a->merge_scale, gr->dz, pu, praw, pB, pC, pg);
        // the pooled sequence scanned forward and reversed: a bidirectional route of length L
        vscan::make_geom(vscan::RK_BIDIR, 1, (int)L, -1, &p.g);
        p.u = pu; p.delta = praw; p.B = pB; p.C = pC;
        p.in_dir = a->per_dir_inputs ? b * L * D : 0;
        p.bc_dir = a->per_dir_inputs ? b * L * N : 0;
        p.gy = pg;
        p.du = reinterpret_cast<float*>(ws + Lo.dpu);
        p.ddelta = reinterpret_cast<float*>(ws + Lo.dpraw);
        p.dB = reinterpret_cast<float*>(ws + Lo.dpB);
        p.dC = reinterpret_cast<float*>(ws + Lo.dpC);
        launch_bwd_scan<vscan::RK_BIDIR, float>(p, grid, s);
        // 8 token rows per CTA at a time, about 16 CTAs per SM over the batch
        const unsigned ux = (unsigned)std::max(1LL, std::min<long long>((TK + 7) / 8, 16LL * 148 / std::max(1LL, (long long)b)));
        vscan::bwd_unpool_kernel<<<dim3(ux, (unsigned)b), 256, 0, s>>>(
            g, (int)b, (int)D, (int)N, Ki, p.du, p.ddelta, p.dB, p.dC, gr->du, gr->ddelta, gr->dB, gr->dC);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "backward kernel launch");
    return VSCAN_OK;
}

}  // namespace

extern "C" {

vscan_status vscan_create_route(vscan_route** out, int32_t kind, int32_t h, int32_t w, int32_t cls_pos)
{
    if (!out) return fail(VSCAN_ERR_INVALID_ARGUMENT, "out is NULL");
    *out = nullptr;
    if (kind < vscan::RK_BIDIR || kind > vscan::RK_POOL_H)
        return fail(VSCAN_ERR_INVALID_ARGUMENT, "unknown route kind %d", kind);
    if (h < 1 || w < 1) return fail(VSCAN_ERR_INVALID_ARGUMENT, "grid %dx%d is empty", h, w);
    if ((long long)h * w > (1LL << 24))
        return fail(VSCAN_ERR_INVALID_ARGUMENT, "grid %dx%d has more than 2^24 tokens", h, w);
    vscan::RouteGeom g{};
    if (!vscan::make_geom(kind, h, w, cls_pos, &g)) {
        if (kind == vscan::RK_BIDIR)
            return fail(VSCAN_ERR_SHAPE, "cls_pos %d must be -1 or floor(h*w/2) = %lld", cls_pos,
                        (long long)h * w / 2);
        return fail(VSCAN_ERR_SHAPE, "cls_pos %d must be -1 for route kind %d", cls_pos, kind);
    }
    vscan_route* r = new (std::nothrow) vscan_route;
    if (!r) return fail(VSCAN_ERR_INVALID_ARGUMENT, "out of host memory");
    r->g = g;
    *out = r;
    return VSCAN_OK;
}

vscan_status vscan_destroy(vscan_route* route)
{
    delete route;
    return VSCAN_OK;
}

vscan_status vscan_route_info(const vscan_route* r, int32_t* K, int32_t* seq_len, int32_t* tokens,
                              int32_t* padded_h, int32_t* padded_w)
{
    if (!r) return fail(VSCAN_ERR_INVALID_ARGUMENT, "route is NULL");
    if (K) *K = r->g.K;
    if (seq_len) *seq_len = r->g.L;
    if (tokens) *tokens = r->g.tokens;
    const bool atrous = r->g.kind == vscan::RK_ATROUS2;
    if (padded_h) *padded_h = atrous ? 2 * r->g.rows : r->g.h;
    if (padded_w) *padded_w = atrous ? 2 * r->g.cols : r->g.w;
    return VSCAN_OK;
}

vscan_status vscan_route_indices(const vscan_route* r, int32_t* dev_out, void* stream)
{
    if (!r) return fail(VSCAN_ERR_INVALID_ARGUMENT, "route is NULL");
    if (!dev_out) return fail(VSCAN_ERR_INVALID_ARGUMENT, "dev_out is NULL");
    const long long n = (long long)r->g.K * r->g.L;
    const int threads = 256;
    const unsigned blocks = (unsigned)((n + threads - 1) / threads);
    route_map_kernel<<<blocks, threads, 0, static_cast<cudaStream_t>(stream)>>>(r->g, dev_out);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "route map kernel launch");
    return VSCAN_OK;
}

vscan_status vscan_workspace_size(const vscan_route* r, const vscan_args* a, uint64_t* bytes)
{
    if (!bytes) return fail(VSCAN_ERR_INVALID_ARGUMENT, "bytes is NULL");
    vscan_status st = check_shape(r, a);
    if (st != VSCAN_OK) return st;
    *bytes = forward_workspace_need(r, a);
    return VSCAN_OK;
}

vscan_status vscan_forward(const vscan_route* r, const vscan_args* a, void* stream)
{
    NvtxRange range("vscan_forward");
    vscan_status st = check_shape(r, a);
    if (st != VSCAN_OK) return st;
    st = check_pointers(a, true);
    if (st != VSCAN_OK) return st;
    return forward_device(r, a, static_cast<cudaStream_t>(stream));
}

vscan_status vscan_plan_info(const vscan_route* r, const vscan_args* a, int32_t* kernels)
{
    if (!kernels) return fail(VSCAN_ERR_INVALID_ARGUMENT, "kernels is NULL");
    vscan_status st = check_shape(r, a);
    if (st != VSCAN_OK) return st;
    if (a->batch == 0) {
        *kernels = 0;
    } else {
        *kernels = (is_pool(r->g.kind) ? 2 : 1) + ((a->flags & VSCAN_FLAG_CHECK_VALUES) ? 1 : 0);
        if (strided_main(r, a)) *kernels += 3 + (a->z ? 1 : 0);  // pack u, delta (z), copy y out
        if (strided_bc(r, a)) *kernels += 2;                      // pack B, C
    }
    return VSCAN_OK;
}

vscan_status vscan_plan_kernel(const vscan_route* r, const vscan_args* a, const char** name)
{
    if (!name) return fail(VSCAN_ERR_INVALID_ARGUMENT, "name is NULL");
    vscan_status st = check_shape(r, a);
    if (st != VSCAN_OK) return st;
    static const char* const stream_names[] = {"stream_scan_kernel<BIDIR>", "stream_scan_kernel<CROSS4>",
                                               "stream_scan_kernel<ATROUS2>"};
    static const char* const resident_names[] = {"resident_scan_kernel<BIDIR>",
                                                 "resident_scan_kernel<CROSS4>",
                                                 "resident_scan_kernel<ATROUS2>"};
    static const char* const pipe_names[] = {"pipe_scan_kernel<BIDIR>", "pipe_scan_kernel<CROSS4>"};
    if (a->batch == 0) *name = "none";
    else if (is_pool(r->g.kind)) *name = "pool_scan_kernel";
    else if (choose_chunks(r, a) > 1) *name = resident_names[r->g.kind];
    else if (use_pipe(r, a, forward_flags(a))) *name = pipe_names[r->g.kind];
    else *name = stream_names[r->g.kind];
    return VSCAN_OK;
}

vscan_status vscan_host_buffer_size(const vscan_route* r, const vscan_args* a, uint64_t* bytes)
{
    if (!bytes) return fail(VSCAN_ERR_INVALID_ARGUMENT, "bytes is NULL");
    vscan_status st = check_shape(r, a);
    if (st != VSCAN_OK) return st;
    st = require_dense(r, a, "vscan_forward_host");
    if (st != VSCAN_OK) return st;
    *bytes = host_layout(r, a).total;
    return VSCAN_OK;
}

vscan_status vscan_forward_host(const vscan_route* r, const vscan_args* ha, void* device_buffer,
                                uint64_t device_buffer_bytes, void* stream)
{
    NvtxRange range("vscan_forward_host");
    vscan_status st = check_shape(r, ha);
    if (st != VSCAN_OK) return st;
    st = require_dense(r, ha, "vscan_forward_host");
    if (st != VSCAN_OK) return st;
    st = check_pointers(ha, false);
    if (st != VSCAN_OK) return st;
    if (ha->batch == 0) return VSCAN_OK;
    const HostLayout L = host_layout(r, ha);
    if (!device_buffer || device_buffer_bytes < L.total)
        return fail(VSCAN_ERR_WORKSPACE, "device buffer of %llu bytes needed, %llu given",
                    (unsigned long long)L.total, (unsigned long long)(device_buffer ? device_buffer_bytes : 0));
    if ((reinterpret_cast<uintptr_t>(device_buffer) & 255u) != 0)
        return fail(VSCAN_ERR_ALIGNMENT, "device buffer is not 256-byte aligned");

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    char* base = static_cast<char*>(device_buffer);
    const vscan::RouteGeom& g = r->g;
    const size_t eb = elem_bytes(ha->dtype);
    const size_t Ki = ha->per_dir_inputs ? g.K : 1;
    const size_t Kp = ha->per_dir_params ? g.K : 1;
    const size_t plane = (size_t)ha->batch * tokens_of(r, ha);

    vscan_args da = *ha;
    da.u = base + L.u;
    da.delta = base + L.delta;
    da.B = base + L.B;
    da.C = base + L.C;
    da.z = ha->z ? base + L.z : nullptr;
    da.y = base + L.y;
    da.A = reinterpret_cast<const float*>(base + L.A);
    da.Dskip = ha->Dskip ? reinterpret_cast<const float*>(base + L.Dskip) : nullptr;
    da.delta_bias = ha->delta_bias ? reinterpret_cast<const float*>(base + L.bias) : nullptr;
    da.conv_w = ha->conv_w ? reinterpret_cast<const float*>(base + L.conv_w) : nullptr;
    da.conv_b = ha->conv_b ? reinterpret_cast<const float*>(base + L.conv_b) : nullptr;
    da.token_pos = ha->token_pos ? reinterpret_cast<const int32_t*>(base + L.pos) : nullptr;
    da.workspace = base + L.ws;
    da.workspace_bytes = workspace_need(r, ha);

    struct Copy { void* dst; const void* src; size_t bytes; };
    const Copy in[] = {
        {const_cast<void*>(da.u), ha->u, Ki * plane * ha->channels * eb},
        {const_cast<void*>(da.delta), ha->delta, Ki * plane * ha->channels * eb},
        {const_cast<void*>(da.B), ha->B, Ki * plane * ha->d_state * eb},
        {const_cast<void*>(da.C), ha->C, Ki * plane * ha->d_state * eb},
        {const_cast<void*>(da.z), ha->z, ha->z ? plane * ha->channels * eb : 0},
        {const_cast<float*>(da.A), ha->A, Kp * ha->channels * ha->d_state * sizeof(float)},
        {const_cast<float*>(da.Dskip), ha->Dskip, ha->Dskip ? Kp * ha->channels * sizeof(float) : 0},
        {const_cast<float*>(da.delta_bias), ha->delta_bias, ha->delta_bias ? Kp * ha->channels * sizeof(float) : 0},
        {const_cast<float*>(da.conv_w), ha->conv_w, ha->conv_w ? Kp * ha->channels * 4 * sizeof(float) : 0},
        {const_cast<float*>(da.conv_b), ha->conv_b, ha->conv_b ? Kp * ha->channels * sizeof(float) : 0},
        {const_cast<int32_t*>(da.token_pos), ha->token_pos, ha->token_pos ? plane * sizeof(int32_t) : 0},
    };
    for (const Copy& c : in) {
        if (c.bytes == 0) continue;
        cudaError_t e = cudaMemcpyAsync(c.dst, c.src, c.bytes, cudaMemcpyHostToDevice, s);
        if (e != cudaSuccess) return cuda_fail(e, "host-to-device copy");
    }
    st = forward_device(r, &da, s);
    if (st != VSCAN_OK) return st;
    cudaError_t e = cudaMemcpyAsync(ha->y, da.y, plane * ha->channels * eb, cudaMemcpyDeviceToHost, s);
    if (e != cudaSuccess) return cuda_fail(e, "device-to-host copy");
    return VSCAN_OK;
}

vscan_status vscan_backward_workspace_size(const vscan_route* r, const vscan_args* a, uint64_t* bytes)
{
    if (!bytes) return fail(VSCAN_ERR_INVALID_ARGUMENT, "bytes is NULL");
    vscan_status st = check_backward(r, a);
    if (st != VSCAN_OK) return st;
    *bytes = a->batch == 0 ? 0 : bwd_layout(r, a).total;
    return VSCAN_OK;
}

vscan_status vscan_backward_plan_kernel(const vscan_route* r, const vscan_args* a, const char** name)
{
    if (!name) return fail(VSCAN_ERR_INVALID_ARGUMENT, "name is NULL");
    vscan_status st = check_backward(r, a);
    if (st != VSCAN_OK) return st;
    static const char* const split_names[] = {"bwd_scan_split_kernel<BIDIR>", "bwd_scan_split_kernel<CROSS4>",
                                              "bwd_scan_split_kernel<ATROUS2>"};
    static const char* const warp_names[] = {"bwd_scan_kernel<BIDIR>", "bwd_scan_kernel<CROSS4>",
                                             "bwd_scan_kernel<ATROUS2>"};
    if (a->batch == 0) {
        *name = "none";
        return VSCAN_OK;
    }
    const int kind = is_pool(r->g.kind) ? (int)vscan::RK_BIDIR : r->g.kind;
    *name = bwd_split(bwd_tiles(r, a)) ? split_names[kind] : warp_names[kind];
    return VSCAN_OK;
}

vscan_status vscan_backward(const vscan_route* r, const vscan_args* a, const void* dy, const vscan_grads* gr,
                            void* stream)
{
    NvtxRange range("vscan_backward");
    vscan_status st = check_backward(r, a);
    if (st != VSCAN_OK) return st;
    if (!gr) return fail(VSCAN_ERR_INVALID_ARGUMENT, "grads is NULL");
    if (a->batch == 0) return VSCAN_OK;
    if (!dy) return fail(VSCAN_ERR_INVALID_ARGUMENT, "dy is NULL");
    if (!aligned16(dy)) return fail(VSCAN_ERR_ALIGNMENT, "dy is not 16-byte aligned");
    if (gr->dz && !a->z) return fail(VSCAN_ERR_INVALID_ARGUMENT, "dz requested without z");
    if ((gr->du && !aligned16(gr->du)) || (gr->ddelta && !aligned16(gr->ddelta)))
        return fail(VSCAN_ERR_ALIGNMENT, "du and ddelta must be 16-byte aligned");
    vscan_args chk = *a;
    chk.y = const_cast<void*>(dy);  // y is not used by the backward pass
    st = check_pointers(&chk, true);
    if (st != VSCAN_OK) return st;
    const uint64_t need = bwd_layout(r, a).total;
    if (!gr->workspace || gr->workspace_bytes < need)
        return fail(VSCAN_ERR_WORKSPACE, "backward workspace of %llu bytes needed, %llu given",
                    (unsigned long long)need, (unsigned long long)(gr->workspace ? gr->workspace_bytes : 0));
    if ((reinterpret_cast<uintptr_t>(gr->workspace) & 255u) != 0)
        return fail(VSCAN_ERR_ALIGNMENT, "backward workspace is not 256-byte aligned");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    return a->dtype == VSCAN_F32 ? backward_device<float>(r, a, dy, gr, s)
                                 : backward_device<__nv_bfloat16>(r, a, dy, gr, s);
}

vscan_status vscan_forward_pooled_noalloc(const vscan_route* r, const vscan_args* a, void* stream)
{
    NvtxRange range("vscan_forward_pooled_noalloc");
    vscan_status st = check_shape(r, a);
    if (st != VSCAN_OK) return st;
    st = require_dense(r, a, "vscan_forward_pooled_noalloc");
    if (st != VSCAN_OK) return st;
    st = check_pointers(a, true);
    if (st != VSCAN_OK) return st;
    if (!is_pool(r->g.kind))
        return fail(VSCAN_ERR_UNSUPPORTED, "vscan_forward_pooled_noalloc takes POOL_W or POOL_H routes only");
    const uint64_t need = workspace_need(r, a);
    if (need > kStaticScratchBytes)
        return fail(VSCAN_ERR_UNSUPPORTED,
                    "pooled B/C need %llu bytes of scratch; the fixed scratch holds %llu "
                    "(2 x planes x batch x pooled length x d_state floats)",
                    (unsigned long long)need, (unsigned long long)kStaticScratchBytes);
    if (a->batch == 0) return VSCAN_OK;
    void* scratch = nullptr;
    st = static_scratch_address(&scratch);
    if (st != VSCAN_OK) return st;
    vscan_args b = *a;
    b.workspace = scratch;
    b.workspace_bytes = kStaticScratchBytes;
    return forward_device(r, &b, static_cast<cudaStream_t>(stream));
}

vscan_status vscan_status_from_device_word(int32_t word)
{
    if (word & vscan::DEV_STATUS_TIMEOUT)
        return fail(VSCAN_ERR_DEVICE_TIMEOUT, "a kernel's pipeline wait gave up (device word 0x%x); y is invalid",
                    (unsigned)word);
    if (word & vscan::DEV_STATUS_VALUE)
        return fail(VSCAN_ERR_VALUE,
                    "value check failed (device word 0x%x): a non-finite input, A > 0, or a negative time scale",
                    (unsigned)word);
    if (word != 0) return fail(VSCAN_ERR_INVALID_ARGUMENT, "unknown bits in device word 0x%x", (unsigned)word);
    return VSCAN_OK;
}

const char* vscan_last_error(void) { return g_last_error.c_str(); }

const char* vscan_status_string(int32_t status)
{
    switch (status) {
    case VSCAN_OK: return "VSCAN_OK";
    case VSCAN_ERR_INVALID_ARGUMENT: return "VSCAN_ERR_INVALID_ARGUMENT";
    case VSCAN_ERR_SHAPE: return "VSCAN_ERR_SHAPE";
    case VSCAN_ERR_ALIGNMENT: return "VSCAN_ERR_ALIGNMENT";
    case VSCAN_ERR_UNSUPPORTED: return "VSCAN_ERR_UNSUPPORTED";
    case VSCAN_ERR_CUDA: return "VSCAN_ERR_CUDA";
    case VSCAN_ERR_WORKSPACE: return "VSCAN_ERR_WORKSPACE";
    case VSCAN_ERR_VALUE: return "VSCAN_ERR_VALUE";
    case VSCAN_ERR_DEVICE_TIMEOUT: return "VSCAN_ERR_DEVICE_TIMEOUT";
    default: return "VSCAN_UNKNOWN_STATUS";
    }
}

int32_t vscan_abi_version(void) { return kAbiVersion; }

}  // extern "C"
