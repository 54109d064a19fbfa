/*
 * vscan.h -- C ABI of the routed visual selective scan library (libvscan.so).
 *
 * The library computes, on one NVIDIA B200 (sm_100a), the Mamba S6 selective
 * scan run over image-token sequences under a spatial routing, fused with the
 * gather, the discretization, the read-out, the SiLU gate and the
 * direction-merging scatter:
 *
 *   for every image b, channel d and direction k of the route:
 *     (u_t, rawDelta_t, B_t, C_t) = tokens gathered in the route's order
 *     Delta_t = softplus(rawDelta_t + bias_d)
 *     h_t     = exp(Delta_t * A_d) (.) h_{t-1} + Delta_t * B_t * u_t,  h_{-1} = 0
 *     y_t     = sum_n C_{t,n} h_{t,n} + D_d * u_t
 *   then y is scattered back to the grid, the directions are summed and scaled
 *   by merge_scale, and the result is gated: Y = merge_scale * sum_k y_k * SiLU(z).
 *
 * Sources (page title and section):
 *   - "Vision Mamba: Bidirectional State Space Models for Images": sec. 3-4
 *     (discretization, recurrence, read-out, released Delta*B*u write), sec. 5
 *     and "Two scans meet at the same token" (bidirectional route, flip back,
 *     shared SiLU gate), sec. 2 (middle CLS at floor(P/2)).
 *   - "EfficientVMamba: Atrous Selective Scan for Light Weight Visual Mamba":
 *     sec. 1-3 (p = 2 atrous groups, right/bottom zero padding, merge by
 *     inverse permutation and crop).
 *   - "Norm or Direction? Decoding Vision Mambas for High-Resolution Vision":
 *     sec. 3, Eq. 1-2 and "2D Selective Scan (SS2D)" (four traversals, summed).
 *   - "Fast Vision Mamba: Pooling Spatial Dimensions for Accelerated
 *     Processing": Methodology (mean-pool one axis, scan forward and backward,
 *     repeat the outputs over the pooled axis).
 *
 * Conventions for every function below:
 *   - Return value: VSCAN_OK (0) or a negative vscan_status. Nothing throws
 *     across the ABI. After a non-OK status, vscan_last_error() returns a
 *     message for the calling thread.
 *   - Argument checks happen on the host before any CUDA call; a rejected call
 *     launches nothing and changes no memory.
 *   - "device pointer" means memory the caller allocated on the current CUDA
 *     device; "stream" is a cudaStream_t passed as void* (NULL = legacy default
 *     stream). Work is enqueued on that stream; no function synchronizes it
 *     unless its comment says so.
 *   - The library owns only the vscan_route objects it creates. Every tensor,
 *     the workspace and every host buffer are owned by the caller.
 */
#ifndef VSCAN_H
#define VSCAN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum vscan_status {
    VSCAN_OK = 0,
    VSCAN_ERR_INVALID_ARGUMENT = -1, /* null pointer, bad enum, non-positive size */
    VSCAN_ERR_SHAPE = -2,            /* size combination the route cannot take     */
    VSCAN_ERR_ALIGNMENT = -3,        /* pointer or channel count not 16-byte aligned */
    VSCAN_ERR_UNSUPPORTED = -4,      /* valid but not implemented (e.g. N > 16)    */
    VSCAN_ERR_CUDA = -5,             /* a CUDA runtime call failed                 */
    VSCAN_ERR_WORKSPACE = -6,        /* workspace missing or smaller than required */
    VSCAN_ERR_VALUE = -7,            /* device value check failed (see
                                        VSCAN_FLAG_CHECK_VALUES); from
                                        vscan_status_from_device_word only        */
    VSCAN_ERR_DEVICE_TIMEOUT = -8    /* a kernel's internal pipeline wait gave up;
                                        y is invalid; from
                                        vscan_status_from_device_word only        */
} vscan_status;

/* Spatial routings. The token array of one image is row-major over the h x w
 * grid (columns fastest), with the CLS token inserted at cls_pos for BIDIR. */
typedef enum vscan_route_kind {
    /* Vim: forward over the assembled sequence (grid + optional middle CLS) and
     * backward over the whole reversed sequence; outputs aligned and added.
     * "Vision Mamba ...", sec. 2 and 5. K = 2, L = h*w (+1 with CLS). */
    VSCAN_ROUTE_BIDIR = 0,
    /* VMamba SS2D: k0 row-major, k1 row-major reversed, k2 column-major,
     * k3 column-major reversed; the four outputs are summed at the original
     * coordinates. "Norm or Direction? ...", sec. 3. K = 4, L = h*w. */
    VSCAN_ROUTE_CROSS4 = 1,
    /* EfficientVMamba p = 2: group k takes grid coordinates
     * (2 r + m_k, 2 c + n_k), (m_k, n_k) = (0,0), (1,0), (0,1), (1,1); groups 0
     * and 2 row-major, 1 and 3 column-major, on the grid zero-padded
     * right/bottom to even size; each real pixel has one owner (no summation)
     * and padding outputs are cropped. "EfficientVMamba ...", sec. 1-3.
     * K = 4, L = ceil(h/2) * ceil(w/2). */
    VSCAN_ROUTE_ATROUS2 = 2,
    /* FastVim: u, rawDelta, B, C mean-pooled over the columns of every grid
     * row (length h), scanned forward and backward, summed, repeated over the
     * columns and gated with the un-pooled z. "Fast Vision Mamba ...",
     * Methodology. K = 2, L = h. */
    VSCAN_ROUTE_POOL_W = 3,
    /* FastVim alternate axis: mean over the rows of every column, L = w. */
    VSCAN_ROUTE_POOL_H = 4
} vscan_route_kind;

typedef enum vscan_dtype {
    VSCAN_F32 = 0, /* IEEE float32 */
    VSCAN_BF16 = 1 /* bfloat16; state and accumulation stay float32 */
} vscan_dtype;

/* Bits of vscan_args.flags. */
typedef enum vscan_flag {
    /* Exact zero-order-hold write term instead of Delta*B*u: for the diagonal A
     * of the scan, Bbar = (Delta A)^-1 (exp(Delta A) - 1) Delta B =
     * expm1(Delta A_n) / A_n * B_n, equal to Delta B_n for A_n = 0.
     * "Norm or Direction? ...", sec. 3, Eq. 2; "Vision Mamba ...", sec. 4 (the
     * released kernels keep Delta*B*u, the default). */
    VSCAN_FLAG_ZOH = 1,
    /* Opt-in value checks on the device before the scan, the conditions under
     * which the scalar reference scan of "EfficientVMamba ...", sec. 2 ("Update
     * an independent state inside each group") refuses its inputs: a
     * non-finite value in any input or parameter, an unstable A (A > 0), or,
     * with delta_softplus = 0, a negative time scale (raw Delta + bias < 0).
     * A failure sets bit 1 of *args->status (which must then be non-NULL); the
     * scan still runs. Costs one read of every input (bandwidth-bound). */
    VSCAN_FLAG_CHECK_VALUES = 2
} vscan_flag;

/* Opaque, immutable route description (host memory only). */
typedef struct vscan_route vscan_route;

/*
 * Arguments of one forward pass. All tensors are row-major with the channel
 * (or state) axis contiguous; u, delta, z and y may step between tokens and
 * images by tok_stride and batch_stride elements, B and C by bc_tok_stride and
 * bc_batch_stride (0 = dense). "tokens" is the route's token count per image
 * (vscan_route_info), Ki = K if per_dir_inputs else 1, Kp = K if
 * per_dir_params else 1. The shapes below are the dense case.
 */
typedef struct vscan_args {
    int32_t batch;          /* images, >= 0 (0 = nothing to do)                      */
    int32_t channels;       /* D (expanded width); multiple of 4 (f32) or 8 (bf16)   */
    int32_t d_state;        /* N, 1..16                                              */
    int32_t dtype;          /* vscan_dtype of u, delta, B, C, z and y                */
    const void* u;          /* device, [Ki][batch][tokens][D]                        */
    const void* delta;      /* device, [Ki][batch][tokens][D], raw step before bias  */
    const void* B;          /* device, [Ki][batch][tokens][N]                        */
    const void* C;          /* device, [Ki][batch][tokens][N]                        */
    const void* z;          /* device, [batch][tokens][D], or NULL for no gate       */
    void* y;                /* device, [batch][tokens][D], written (not accumulated) */
    const float* A;         /* device, [Kp][D][N] float32 (negative for stability)   */
    const float* Dskip;     /* device, [Kp][D] float32, or NULL for no skip term     */
    const float* delta_bias;/* device, [Kp][D] float32, or NULL for no bias          */
    int32_t per_dir_inputs; /* 0: u, delta, B, C shared by all directions; 1: per k  */
    int32_t per_dir_params; /* 0: A, Dskip, delta_bias shared; 1: leading K axis     */
    int32_t delta_softplus; /* 1: Delta = softplus(raw + bias); 0: Delta = raw + bias */
    float merge_scale;      /* scales the merged output: 1 = sum, 0.5 = Vim average  */
    void* workspace;        /* device scratch of >= vscan_workspace_size() bytes     */
    uint64_t workspace_bytes;
    int32_t seq_chunks;     /* 0 = library choice; 1 = one sequential pass per
                               direction (streaming kernel); 2, 4 or 8 = split each
                               sequence into that many chunks joined by a prefix
                               scan of affine pairs (BIDIR, CROSS4 and ATROUS2 when
                               the image's token tile fits on chip, else
                               VSCAN_ERR_UNSUPPORTED); ignored by the pooled routes */
    int32_t flags;          /* OR of vscan_flag bits; other bits are rejected        */
    const float* conv_w;    /* device, [Kp][D][4] float32, or NULL: no convolution.
                               With it, u holds the convolution INPUT x and every
                               direction k uses u_k = SiLU(conv_b + sum_i
                               conv_w[i] * x[t - 3 + i]) along its own sequence
                               order (x before the first step = 0) as the scan
                               input, in the write term and in the skip term
                               ("Vision Mamba ...", "Inside the released Vim
                               block": each branch's kernel-four causal Conv1d,
                               then SiLU; the backward branch on the reversed
                               sequence). BIDIR: along the route. POOL_W / POOL_H:
                               along the row-major / column-major token order
                               (reversed for k = 1), before pooling ("Fast Vision
                               Mamba ...", Methodology). CROSS4 and ATROUS2:
                               VSCAN_ERR_UNSUPPORTED (their pages convolve on the
                               2-D grid before routing).                          */
    const float* conv_b;    /* device, [Kp][D] float32, or NULL for no conv bias    */
    const int32_t* token_pos;/* device, [batch][n_tokens] int32, or NULL (dense grid).
                               POOL_W / POOL_H on a masked or irregular token set
                               (FastMaskVim: "Fast Vision Mamba ...", Innovation
                               and Methodology): the token arrays hold n_tokens
                               visible tokens per image instead of h*w, and
                               token_pos gives each one's grid position
                               row * w + col in [0, h*w). Every pooled token is the
                               sum of the visible tokens of its row (POOL_W) or
                               column (POOL_H) divided by the nominal w (h); the
                               pooled output goes back to every visible token of
                               that row (column). A position outside the grid is
                               ignored and its y written as 0 (not checked on the
                               host). Other routes, or together with conv_w:
                               VSCAN_ERR_UNSUPPORTED.                             */
    int32_t n_tokens;       /* visible tokens per image with token_pos, else 0     */
    int32_t reserved2;      /* must be 0                                            */
    int32_t* status;        /* device int32 or NULL (also with vscan_forward_host).
                               When given, kernels OR bits into it and never trap:
                               1 = a value check failed (VSCAN_FLAG_CHECK_VALUES),
                               2 = an internal pipeline wait gave up (y invalid).
                               The caller zeroes it, synchronizes the stream and
                               decodes it with vscan_status_from_device_word.
                               Required with VSCAN_FLAG_CHECK_VALUES.             */
    /* Strides in elements (0 = dense). Token t of image b of direction plane k
     * of u and delta sits at (k * batch + b) * batch_stride + t * tok_stride;
     * z and y use the same strides with k = 0; B and C use the bc_ strides.
     * tok_stride >= channels, a multiple of 4 (f32) or 8 (bf16);
     * batch_stride >= tokens * tok_stride, the same multiple; bc_tok_stride >=
     * d_state; bc_batch_stride >= tokens * bc_tok_stride. Strided tensors are
     * packed into the workspace by a copy kernel before the scan (y: written
     * there and copied out after it), one more read and write of each: an
     * addition of this library for callers holding views of larger buffers
     * (the pages' tensors are dense). vscan_forward only; vscan_forward_host,
     * vscan_backward and vscan_forward_pooled_noalloc return
     * VSCAN_ERR_UNSUPPORTED for non-dense strides.                          */
    int64_t tok_stride;
    int64_t batch_stride;
    int64_t bc_tok_stride;
    int64_t bc_batch_stride;
} vscan_args;

/*
 * Describe a route. Host only: no CUDA call, no device memory.
 *   kind    : vscan_route_kind.
 *   h, w    : grid rows and columns, >= 1.
 *   cls_pos : BIDIR only: index of the CLS token in the token array, which
 *             must be floor(h*w/2) ("Vision Mamba ...", sec. 2), or -1 for no
 *             CLS; every other route requires -1.
 * On success *out receives a route to be released with vscan_destroy.
 * Errors: VSCAN_ERR_INVALID_ARGUMENT (null out, bad kind, h or w < 1, a
 * sequence longer than 2^24 tokens), VSCAN_ERR_SHAPE (cls_pos not allowed).
 */
vscan_status vscan_create_route(vscan_route** out, int32_t kind, int32_t h, int32_t w,
                                int32_t cls_pos);

/* Release a route. NULL is a no-op. Always returns VSCAN_OK. */
vscan_status vscan_destroy(vscan_route* route);

/*
 * Geometry of a route (host only). Any output pointer may be NULL.
 *   K        : directions (2 or 4).
 *   seq_len  : steps per direction.
 *   tokens   : tokens per image in the token array (h*w, +1 with CLS).
 *   padded_h, padded_w : working grid (ATROUS2: rounded up to even; else h, w).
 */
vscan_status vscan_route_info(const vscan_route* route, int32_t* K, int32_t* seq_len,
                              int32_t* tokens, int32_t* padded_h, int32_t* padded_w);

/*
 * Write the route's index maps into a device buffer of K * seq_len int32:
 * out[k * seq_len + t] = token index visited at step t of direction k (for
 * the pooled routes: the pooled-sequence index), or -1 for an ATROUS2 padding
 * slot. The maps are produced on the GPU by the same index functions the scan
 * kernels evaluate. Enqueued on stream.
 */
vscan_status vscan_route_indices(const vscan_route* route, int32_t* dev_out, void* stream);

/*
 * Device scratch bytes vscan_forward needs for these arguments (host only).
 * BIDIR and CROSS4 park per-direction partial outputs until the last
 * direction of a token adds them up ([K][batch][tokens][D] float32); POOL_W
 * and POOL_H hold the pooled B and C; ATROUS2 needs none (one owner per pixel).
 */
vscan_status vscan_workspace_size(const vscan_route* route, const vscan_args* args,
                                  uint64_t* bytes);

/*
 * Number of kernel launches vscan_forward makes for these arguments (host
 * only): 1 for BIDIR, CROSS4 and ATROUS2 (pipelined, streaming or resident
 * chunked scan), 2 for the pooled routes (B/C pooling, then the fused
 * pool-scan-repeat), plus 1 with VSCAN_FLAG_CHECK_VALUES; 0 for an empty
 * batch.
 */
vscan_status vscan_plan_info(const vscan_route* route, const vscan_args* args, int32_t* kernels);

/*
 * Name of the kernel that runs the scan for these arguments (host only), as
 * a static NUL-terminated string owned by the library: "pipe_scan_kernel<R>"
 * (mbarrier-pipelined scan, R = BIDIR or CROSS4, d_state 16 without the
 * optional steps), "stream_scan_kernel<R>" (streaming scan),
 * "resident_scan_kernel<R>" (chunked parallel scan of a shared-memory-resident
 * tile; R = BIDIR, CROSS4 or ATROUS2), "pool_scan_kernel" (pooled routes) or
 * "none" (empty batch). Same argument checks and errors as vscan_plan_info;
 * *name is untouched on error.
 */
vscan_status vscan_plan_kernel(const vscan_route* route, const vscan_args* args, const char** name);

/*
 * Run the fused routed scan on the device. Enqueued on stream; allocates
 * nothing; never synchronizes. The output y is fully overwritten. Concurrent
 * calls on different streams must use different workspaces.
 * Errors: INVALID_ARGUMENT / SHAPE / ALIGNMENT / UNSUPPORTED for bad
 * arguments (nothing launched), WORKSPACE if the workspace is too small,
 * CUDA if a launch failed (message from the CUDA runtime).
 */
vscan_status vscan_forward(const vscan_route* route, const vscan_args* args, void* stream);

/*
 * Pooled-route forward pass that allocates nothing and needs no workspace.
 * (An addition of this library; the pages have no counterpart.)
 *
 * For callers that cannot allocate device memory: a plugin whose host runtime
 * owns all device memory, or a latency-bound loop that must not call
 * cudaMalloc (which can synchronize the device and fail under memory pressure).
 * The only scratch of the pooled routes, the pooled B and C, is placed in a
 * fixed 4 MiB array inside the library instead of the caller's workspace; the
 * caller still passes every input and the output, as for vscan_forward, and
 * args->workspace is ignored.
 *   - Routes: VSCAN_ROUTE_POOL_W and VSCAN_ROUTE_POOL_H only (else
 *     VSCAN_ERR_UNSUPPORTED).
 *   - Limit: 2 * Ki * batch * pooled_length * d_state * 4 bytes must not
 *     exceed 4 MiB (e.g. batch 32, length 128, N 16 uses 512 KiB); larger
 *     calls return VSCAN_ERR_UNSUPPORTED with the sizes in vscan_last_error().
 *   - Every GPU that loads the library holds the 4 MiB until the process exits.
 *   - The first call on a device, with that device current, resolves the
 *     array's device address (cudaGetSymbolAddress) and keeps it; make that
 *     first call before any stream capture.
 *   - All calls share the one array and it keeps the last call's contents.
 *     On a dense grid every element the call reads is first written by the
 *     same call. With a masked token set (token_pos) the pooled sums are
 *     accumulated into the array, so the call first clears the bytes it uses
 *     with an asynchronous memset on the caller's stream (no allocation).
 *     Calls that overlap on the GPU (different streams, no ordering between
 *     them) race on the array: order them.
 * Errors and the other conventions are those of vscan_forward.
 */
vscan_status vscan_forward_pooled_noalloc(const vscan_route* route, const vscan_args* args, void* stream);

/*
 * Bytes of device memory vscan_forward_host needs in its device_buffer for
 * these arguments (host only): device copies of every input and of y, plus
 * the workspace, each rounded up to 256 bytes.
 */
vscan_status vscan_host_buffer_size(const vscan_route* route, const vscan_args* host_args,
                                    uint64_t* bytes);

/*
 * End-to-end call with HOST tensors. host_args holds host pointers (page-locked
 * memory gives asynchronous copies) with the same layouts as vscan_forward;
 * its workspace fields are ignored. The call enqueues on stream: host-to-device
 * copies of the inputs into device_buffer, the forward pass, and the
 * device-to-host copy of y into host_args->y. The caller synchronizes the
 * stream before reading y. device_buffer is caller-owned device memory of at
 * least vscan_host_buffer_size() bytes.
 */
vscan_status vscan_forward_host(const vscan_route* route, const vscan_args* host_args,
                                void* device_buffer, uint64_t device_buffer_bytes, void* stream);

/*
 * Gradients of vscan_forward, all float32 and written (not accumulated):
 * the reverse-mode derivative of the forward steps ("Vision Mamba ...",
 * sec. 3-5; "EfficientVMamba ...", sec. 1-3; "Fast Vision Mamba ...",
 * Methodology) for the Delta*B*u write term. Any pointer may be NULL when that
 * gradient is not wanted (its work is then skipped where possible).
 */
typedef struct vscan_grads {
    float* du;        /* device, [Ki][batch][tokens][D], 16-byte aligned        */
    float* ddelta;    /* device, [Ki][batch][tokens][D], w.r.t. the raw step,
                         16-byte aligned                                        */
    float* dB;        /* device, [Ki][batch][tokens][N]                         */
    float* dC;        /* device, [Ki][batch][tokens][N]                         */
    float* dA;        /* device, [Kp][D][N]                                     */
    float* dDskip;    /* device, [Kp][D] (w.r.t. D even when args->Dskip is NULL)  */
    float* dbias;     /* device, [Kp][D] (w.r.t. the bias, also when it is NULL) */
    float* dz;        /* device, [batch][tokens][D]; needs args->z              */
    void* workspace;  /* device scratch of >= vscan_backward_workspace_size()   */
    uint64_t workspace_bytes;
} vscan_grads;

/*
 * Device scratch bytes vscan_backward needs for these arguments (host only):
 * the pre-gate forward output, the forward's own workspace, the gradient of the
 * merged value (grid routes), the state at every 16-step chunk boundary of every
 * sequence ([K][batch][ceil(L/16)][D][16] float32), and for the pooled routes the
 * pooled inputs and their gradients.
 */
vscan_status vscan_backward_workspace_size(const vscan_route* route, const vscan_args* args,
                                           uint64_t* bytes);

/*
 * Name of the kernel that runs vscan_backward's adjoint scan for these arguments
 * (host only), as a static NUL-terminated string owned by the library:
 * "bwd_scan_split_kernel<R>" (each tile of 8 channels, one image and one
 * direction on a CTA of two warps that split its 16 states; grids of at most 8
 * tiles per SM) or "bwd_scan_kernel<R>" (one warp per tile), R = BIDIR, CROSS4 or
 * ATROUS2, BIDIR for the pooled routes (their pooled sequence is scanned as a
 * bidirectional route); "none" for an empty batch. Same argument checks and errors
 * as vscan_backward_workspace_size; *name is untouched on error.
 */
vscan_status vscan_backward_plan_kernel(const vscan_route* route, const vscan_args* args, const char** name);

/*
 * Backward pass. args are the forward's arguments (args->y and args->workspace
 * are not used); dy is dL/dy, [batch][tokens][D] in args->dtype, device. The
 * call enqueues on stream: zeroing of the requested gradients, the pre-gate
 * forward pass, the gate's gradient (for the pooled routes inside the pooling of
 * the inputs and the merged value's gradient), and the reverse-time adjoint scan
 * of every direction (checkpointed every 16 steps), then the gradients. Token gradients
 * shared by several directions, channel tiles or images are summed with float
 * atomics, so their low-order bits can vary from run to run.
 * Errors: as vscan_forward; VSCAN_ERR_UNSUPPORTED with the fused convolution,
 * the zero-order-hold flag or a masked token set; VSCAN_ERR_WORKSPACE if
 * grads->workspace is too small; VSCAN_ERR_INVALID_ARGUMENT for dy or grads
 * NULL, or dz requested without args->z.
 */
vscan_status vscan_backward(const vscan_route* route, const vscan_args* args, const void* dy,
                            const vscan_grads* grads, void* stream);

/*
 * Decode a device status word (vscan_args.status) after the stream has been
 * synchronized: VSCAN_OK for 0, VSCAN_ERR_DEVICE_TIMEOUT if bit 2 is set, else
 * VSCAN_ERR_VALUE if bit 1 is set. Host only; sets vscan_last_error() to a
 * description when the result is not VSCAN_OK.
 */
vscan_status vscan_status_from_device_word(int32_t word);

/* Message for the last non-OK status on this thread ("" if none). */
const char* vscan_last_error(void);

/* Static name of a status code. */
const char* vscan_status_string(int32_t status);

/* Library ABI version; changes whenever vscan_args changes layout (2: flags,
 * conv_w and conv_b; 3: token_pos and n_tokens; 4: status; 5: strides). */
int32_t vscan_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* VSCAN_H */
