"""Routed visual selective scan on NVIDIA B200: Python binding of libvscan.so.

The binding only marshals PyTorch tensors (device memory and streams) into the
C ABI declared in include/vscan.h; every step of the scan runs in the CUDA
kernels of the library. Tensors are channels-last:

    u, delta, z, y : [batch, tokens, D]   (leading K axis for per-direction u/delta)
    B, C           : [batch, tokens, N]   (leading K axis for per-direction B/C)
    A              : [D, N] float32        ([K, D, N] per direction)
    Dskip, bias    : [D] float32           ([K, D] per direction)
    conv_w, conv_b : [D, 4], [D] float32   ([K, D, 4], [K, D] per direction), optional:
                     fuse each direction's causal kernel-four Conv1d + SiLU into u
                     (u then holds the convolution input); BIDIR and pooled routes
    zoh=True       : zero-order-hold write term instead of Delta*B*u
    token_pos      : [batch, n] int32, optional (POOL_W / POOL_H): a masked token set
                     (FastMaskVim); u, delta, B, C, z, y then hold the n visible tokens
                     and token_pos their grid positions row * w + col

u, delta, B, C, z and y share one dtype: torch.float32 or torch.bfloat16.
"""
import ctypes

import torch

from ._abi import BF16, F32, FLAG_CHECK_VALUES, FLAG_ZOH, ROUTES, VscanArgs, VscanError, VscanGrads, check, lib

__all__ = ["Route", "forward", "backward", "forward_host", "workspace_size", "host_buffer_size",
           "status_from_device_word", "VscanError", "ROUTES"]


class Route:
    """An immutable route description (vscan_create_route / vscan_destroy)."""

    def __init__(self, kind, h, w, cls_pos=-1):
        self.kind_name = kind if isinstance(kind, str) else {v: k for k, v in ROUTES.items()}[kind]
        self.kind = ROUTES[kind] if isinstance(kind, str) else int(kind)
        self.h, self.w, self.cls_pos = int(h), int(w), int(cls_pos)
        handle = ctypes.c_void_p()
        check(lib.vscan_create_route(ctypes.byref(handle), self.kind, self.h, self.w, self.cls_pos))
        self._handle = handle
        # bound here: at interpreter exit the module global may be gone before __del__ runs
        self._destroy = lib.vscan_destroy
        vals = [ctypes.c_int32() for _ in range(5)]
        check(lib.vscan_route_info(self._handle, *[ctypes.byref(v) for v in vals]))
        self.K, self.seq_len, self.tokens, self.padded_h, self.padded_w = (v.value for v in vals)

    @property
    def handle(self):
        if self._handle is None:
            raise ValueError("route was closed")
        return self._handle

    def close(self):
        if getattr(self, "_handle", None) is not None:
            self._destroy(self._handle)
            self._handle = None

    def __del__(self):
        self.close()

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def indices(self, device="cuda", stream=None):
        """[K, seq_len] int32 maps computed on the GPU by the kernels' index functions."""
        out = torch.empty((self.K, self.seq_len), dtype=torch.int32, device=device)
        s = _stream(stream, out.device)
        check(lib.vscan_route_indices(self.handle, ctypes.c_void_p(out.data_ptr()), s))
        return out


def _stream(stream, device):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t):
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError(f"unsupported dtype {t.dtype} (float32 or bfloat16)")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _layout(t, per_dir):
    """(token stride, image stride) in elements of a [(K,) batch, tokens, rows] tensor whose
    last axis is contiguous; with a direction axis its planes must follow one another."""
    if t.dim() < 3 or (t.stride(-1) != 1 and t.shape[-1] > 1):
        raise ValueError("the channel (state) axis must be contiguous")
    # a size-1 axis has no meaningful stride: take the dense value
    ts = t.stride(-2) if t.shape[-2] > 1 else t.shape[-1]
    bs = t.stride(-3) if t.shape[-3] > 1 else t.shape[-2] * ts
    if per_dir and t.shape[0] > 1 and t.stride(0) != t.shape[1] * bs:
        raise ValueError("direction planes must be spaced batch x image stride apart")
    return ts, bs


def _strides(u, delta, z, y, B, C, per_dir_inputs):
    """The ABI's strides: one layout for u, delta, z, y and one for B, C."""
    ts, bs = _layout(u, per_dir_inputs)
    for name, t, pd in (("delta", delta, per_dir_inputs), ("z", z, False), ("y", y, False)):
        if t is not None and _layout(t, pd) != (ts, bs):
            raise ValueError(f"{name} must have u's token and image strides {(ts, bs)}")
    bts, bbs = _layout(B, per_dir_inputs)
    if _layout(C, per_dir_inputs) != (bts, bbs):
        raise ValueError(f"C must have B's token and image strides {(bts, bbs)}")
    return ts, bs, bts, bbs


def _args(route, u, delta, A, B, C, Dskip, delta_bias, z, y, delta_softplus, merge_scale,
          per_dir_inputs, per_dir_params, workspace, seq_chunks, conv_w=None, conv_b=None,
          zoh=False, token_pos=None, status=None, check_values=False):
    for name, t in (("A", A), ("Dskip", Dskip), ("delta_bias", delta_bias), ("conv_w", conv_w),
                    ("conv_b", conv_b)):
        if t is not None and not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    for name, t in (("A", A), ("Dskip", Dskip), ("delta_bias", delta_bias), ("conv_w", conv_w),
                    ("conv_b", conv_b)):
        if t is not None and t.dtype != torch.float32:
            raise TypeError(f"{name} must be float32")
    lead = 1 if per_dir_inputs else 0
    batch, tokens, D = u.shape[lead:]
    N = B.shape[-1]
    if token_pos is not None:
        if token_pos.dtype != torch.int32 or not token_pos.is_contiguous():
            raise TypeError("token_pos must be a contiguous int32 tensor")
        if tuple(token_pos.shape) != (batch, tokens):
            raise ValueError(f"token_pos shape {tuple(token_pos.shape)} != {(batch, tokens)}")
    elif tokens != route.tokens:
        raise ValueError(f"u has {tokens} tokens per image, the route has {route.tokens}")
    code = _dtype_code(u)
    for name, t in (("delta", delta), ("B", B), ("C", C), ("z", z), ("y", y)):
        if t is not None and t.dtype != u.dtype:
            raise TypeError(f"{name} dtype {t.dtype} != u dtype {u.dtype}")
    a = VscanArgs()
    a.batch, a.channels, a.d_state, a.dtype = batch, D, N, code
    a.u, a.delta, a.B, a.C, a.z, a.y = (_ptr(u), _ptr(delta), _ptr(B), _ptr(C), _ptr(z), _ptr(y))
    a.A, a.Dskip, a.delta_bias = _ptr(A), _ptr(Dskip), _ptr(delta_bias)
    a.per_dir_inputs, a.per_dir_params = int(bool(per_dir_inputs)), int(bool(per_dir_params))
    a.delta_softplus = int(bool(delta_softplus))
    a.merge_scale = float(merge_scale)
    if workspace is not None:
        a.workspace, a.workspace_bytes = _ptr(workspace), workspace.numel() * workspace.element_size()
    a.seq_chunks = int(seq_chunks)
    a.flags = (FLAG_ZOH if zoh else 0) | (FLAG_CHECK_VALUES if check_values else 0)
    if status is not None:
        if status.dtype != torch.int32 or status.numel() < 1 or not status.is_cuda:
            raise TypeError("status must be a CUDA int32 tensor")
        a.status = _ptr(status)
    a.conv_w, a.conv_b = _ptr(conv_w), _ptr(conv_b)
    a.token_pos = _ptr(token_pos)
    a.n_tokens = tokens if token_pos is not None else 0
    a.tok_stride, a.batch_stride, a.bc_tok_stride, a.bc_batch_stride = _strides(u, delta, z, y, B, C,
                                                                                per_dir_inputs)
    return a


def workspace_size(route, u, B, *, per_dir_inputs=False, per_dir_params=False, z=None, token_pos=None, **_):
    """Bytes of device scratch vscan_forward needs (host-only query); u's and B's strides
    (and whether z is given) count when the tensors are not dense, and a masked token set
    (token_pos) sets the tokens per image."""
    lead = 1 if per_dir_inputs else 0
    a = VscanArgs()
    a.batch, _, a.channels = u.shape[lead:]
    a.d_state = B.shape[-1]
    a.dtype = _dtype_code(u)
    a.per_dir_inputs, a.per_dir_params = int(bool(per_dir_inputs)), int(bool(per_dir_params))
    a.delta_softplus, a.merge_scale = 1, 1.0
    a.z = ctypes.c_void_p(1) if z is not None else None  # only nullness matters here
    if token_pos is not None:
        a.token_pos = ctypes.c_void_p(1)
        a.n_tokens = u.shape[lead + 1]
    a.tok_stride, a.batch_stride = _layout(u, per_dir_inputs)
    a.bc_tok_stride, a.bc_batch_stride = _layout(B, per_dir_inputs)
    n = ctypes.c_uint64()
    check(lib.vscan_workspace_size(route.handle, ctypes.byref(a), ctypes.byref(n)))
    return n.value


def forward(route, u, delta, A, B, C, Dskip=None, delta_bias=None, z=None, *, delta_softplus=True,
            merge_scale=1.0, per_dir_inputs=False, per_dir_params=False, out=None, workspace=None,
            seq_chunks=0, conv_w=None, conv_b=None, zoh=False, token_pos=None, stream=None,
            status=None, check_values=False):
    """Routed selective scan on the GPU (vscan_forward). Returns y [batch, tokens, D].

    status: optional CUDA int32 tensor (one element, zeroed by the caller) into which the
    kernels OR device-side findings; decode it with status_from_device_word after
    synchronizing. check_values=True (needs status) first checks every input on the device:
    non-finite values, A > 0, and (delta_softplus=False) a negative time scale.
    """
    lead = 1 if per_dir_inputs else 0
    if out is None:  # in u's layout (the ABI has one layout for u, delta, z and y)
        ts, bs = _layout(u, per_dir_inputs)
        out = torch.empty_strided(u.shape[lead:], (bs, ts, 1), dtype=u.dtype, device=u.device)
    if token_pos is not None and token_pos.shape[-1] == 0:
        return out  # an empty token set: nothing to compute (and no data pointers to pass)
    if workspace is None:
        need = workspace_size(route, u, B, per_dir_inputs=per_dir_inputs, per_dir_params=per_dir_params, z=z,
                              token_pos=token_pos)
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=u.device)
    a = _args(route, u, delta, A, B, C, Dskip, delta_bias, z, out, delta_softplus, merge_scale,
              per_dir_inputs, per_dir_params, workspace, seq_chunks, conv_w, conv_b, zoh, token_pos,
              status, check_values)
    check(lib.vscan_forward(route.handle, ctypes.byref(a), _stream(stream, u.device)))
    return out


def status_from_device_word(word):
    """vscan_status_from_device_word: 0 (VSCAN_OK) or the negative status a device word encodes."""
    return int(lib.vscan_status_from_device_word(int(word)))


def host_buffer_size(route, u, B, *, z=True, Dskip=True, delta_bias=True, per_dir_inputs=False,
                     per_dir_params=False, conv_w=False, conv_b=False, token_pos=False):
    """Bytes of device memory forward_host needs (host-only query)."""
    lead = 1 if per_dir_inputs else 0
    a = VscanArgs()
    a.batch, _, a.channels = u.shape[lead:]
    a.d_state = B.shape[-1]
    a.dtype = _dtype_code(u)
    a.per_dir_inputs, a.per_dir_params = int(bool(per_dir_inputs)), int(bool(per_dir_params))
    a.delta_softplus, a.merge_scale = 1, 1.0
    # only nullness matters for the size query
    a.z = ctypes.c_void_p(1) if z else None
    a.Dskip = ctypes.c_void_p(1) if Dskip else None
    a.delta_bias = ctypes.c_void_p(1) if delta_bias else None
    a.conv_w = ctypes.c_void_p(1) if conv_w else None
    a.conv_b = ctypes.c_void_p(1) if conv_b else None
    if token_pos:
        a.token_pos = ctypes.c_void_p(1)
        a.n_tokens = u.shape[lead + 1]
    n = ctypes.c_uint64()
    check(lib.vscan_host_buffer_size(route.handle, ctypes.byref(a), ctypes.byref(n)))
    return n.value


def forward_host(route, u, delta, A, B, C, Dskip=None, delta_bias=None, z=None, *, out,
                 device_buffer, delta_softplus=True, merge_scale=1.0, per_dir_inputs=False,
                 per_dir_params=False, conv_w=None, conv_b=None, zoh=False, token_pos=None, stream=None):
    """End-to-end call with host (CPU, ideally pinned) tensors (vscan_forward_host).

    Enqueues the host-to-device copies, the scan and the copy of y into `out`
    (a host tensor) on the stream; synchronize the stream before reading `out`.
    """
    for t in (u, delta, A, B, C, Dskip, delta_bias, z, out, conv_w, conv_b, token_pos):
        if t is not None and t.is_cuda:
            raise ValueError("forward_host takes host tensors")
    a = _args(route, u, delta, A, B, C, Dskip, delta_bias, z, out, delta_softplus, merge_scale,
              per_dir_inputs, per_dir_params, None, 0, conv_w, conv_b, zoh, token_pos)
    nbytes = device_buffer.numel() * device_buffer.element_size()
    check(lib.vscan_forward_host(route.handle, ctypes.byref(a), ctypes.c_void_p(device_buffer.data_ptr()),
                                 nbytes, _stream(stream, device_buffer.device)))
    return out


class Plan:
    """A forward call with its arguments marshalled once (for repeated launches).

    Holds references to every tensor it points at; run() is one vscan_forward call.
    """

    def __init__(self, route, u, delta, A, B, C, Dskip=None, delta_bias=None, z=None, *, out,
                 workspace, delta_softplus=True, merge_scale=1.0, per_dir_inputs=False,
                 per_dir_params=False, seq_chunks=0, conv_w=None, conv_b=None, zoh=False,
                 token_pos=None):
        self.route = route
        self._keep = (u, delta, A, B, C, Dskip, delta_bias, z, out, workspace, conv_w, conv_b, token_pos)
        self.out = out
        self.args = _args(route, u, delta, A, B, C, Dskip, delta_bias, z, out, delta_softplus,
                          merge_scale, per_dir_inputs, per_dir_params, workspace, seq_chunks,
                          conv_w, conv_b, zoh, token_pos)
        self._ref = ctypes.byref(self.args)

    def run(self, stream):
        """Enqueue the forward pass on a torch.cuda.Stream."""
        check(lib.vscan_forward(self.route.handle, self._ref, ctypes.c_void_p(stream.cuda_stream)))

    def kernels(self):
        """Number of kernel launches one run() makes (vscan_plan_info)."""
        n = ctypes.c_int32()
        check(lib.vscan_plan_info(self.route.handle, self._ref, ctypes.byref(n)))
        return n.value

    def kernel_name(self):
        """Name of the kernel that runs the scan (vscan_plan_kernel)."""
        name = ctypes.c_char_p()
        check(lib.vscan_plan_kernel(self.route.handle, self._ref, ctypes.byref(name)))
        return name.value.decode()


__all__.append("Plan")


class HostPlan:
    """An end-to-end forward_host call with its arguments marshalled once."""

    def __init__(self, route, u, delta, A, B, C, Dskip=None, delta_bias=None, z=None, *, out,
                 device_buffer, delta_softplus=True, merge_scale=1.0, per_dir_inputs=False,
                 per_dir_params=False, conv_w=None, conv_b=None, zoh=False, token_pos=None):
        for t in (u, delta, A, B, C, Dskip, delta_bias, z, out, conv_w, conv_b, token_pos):
            if t is not None and t.is_cuda:
                raise ValueError("HostPlan takes host tensors")
        self.route = route
        self._keep = (u, delta, A, B, C, Dskip, delta_bias, z, out, device_buffer, conv_w, conv_b, token_pos)
        self.out = out
        self.args = _args(route, u, delta, A, B, C, Dskip, delta_bias, z, out, delta_softplus,
                          merge_scale, per_dir_inputs, per_dir_params, None, 0, conv_w, conv_b, zoh,
                          token_pos)
        self._ref = ctypes.byref(self.args)
        self._buf = ctypes.c_void_p(device_buffer.data_ptr())
        self._nbytes = device_buffer.numel() * device_buffer.element_size()

    def run(self, stream):
        check(lib.vscan_forward_host(self.route.handle, self._ref, self._buf, self._nbytes,
                                     ctypes.c_void_p(stream.cuda_stream)))


__all__.append("HostPlan")


def backward(route, u, delta, A, B, C, Dskip=None, delta_bias=None, z=None, *, dy, delta_softplus=True,
             merge_scale=1.0, per_dir_inputs=False, per_dir_params=False, want=None, stream=None):
    """Gradients of forward() (vscan_backward), float32 tensors in a dict.

    dy: dL/dy, [batch, tokens, D] in the dtype of u. Keys: du, ddelta (w.r.t. the raw
    step), dB, dC, dA, dDskip, dbias and dz (with z). `want` limits the keys computed.
    """
    lead = 1 if per_dir_inputs else 0
    dev = u.device
    K = route.K
    Kp = K if per_dir_params else 1
    D = u.shape[-1]
    shapes = dict(du=u.shape, ddelta=u.shape, dB=B.shape, dC=C.shape, dA=A.shape,
                  dDskip=(Kp, D) if per_dir_params else (D,), dbias=(Kp, D) if per_dir_params else (D,))
    if z is not None:
        shapes["dz"] = z.shape
    keys = list(shapes) if want is None else [k for k in want if k in shapes]
    out = {k: torch.empty(shapes[k], dtype=torch.float32, device=dev) for k in keys}
    a = _args(route, u, delta, A, B, C, Dskip, delta_bias, z, u[0] if lead else u, delta_softplus, merge_scale,
              per_dir_inputs, per_dir_params, None, 0)
    a.y = None
    n = ctypes.c_uint64()
    check(lib.vscan_backward_workspace_size(route.handle, ctypes.byref(a), ctypes.byref(n)))
    ws = torch.empty(max(n.value, 256), dtype=torch.uint8, device=dev)
    g = VscanGrads()
    for k, t in out.items():
        setattr(g, k, ctypes.c_void_p(t.data_ptr()))
    g.workspace, g.workspace_bytes = ctypes.c_void_p(ws.data_ptr()), ws.numel()
    if not dy.is_contiguous() or dy.dtype != u.dtype:
        raise TypeError("dy must be contiguous with the dtype of u")
    check(lib.vscan_backward(route.handle, ctypes.byref(a), ctypes.c_void_p(dy.data_ptr()), ctypes.byref(g),
                             _stream(stream, dev)))
    out["_workspace"] = ws  # keeps the scratch alive until the caller synchronizes
    return out


class BackwardPlan:
    """A backward call with its arguments, gradients and scratch marshalled once."""

    def __init__(self, route, u, delta, A, B, C, Dskip=None, delta_bias=None, z=None, *, dy,
                 delta_softplus=True, merge_scale=1.0, per_dir_inputs=False, per_dir_params=False):
        self.route = route
        dev = u.device
        K = route.K
        Kp = K if per_dir_params else 1
        D = u.shape[-1]
        shapes = dict(du=u.shape, ddelta=u.shape, dB=B.shape, dC=C.shape, dA=A.shape,
                      dDskip=(Kp, D) if per_dir_params else (D,), dbias=(Kp, D) if per_dir_params else (D,))
        if z is not None:
            shapes["dz"] = z.shape
        self.grads = {k: torch.empty(v, dtype=torch.float32, device=dev) for k, v in shapes.items()}
        lead = 1 if per_dir_inputs else 0
        self.args = _args(route, u, delta, A, B, C, Dskip, delta_bias, z, u[0] if lead else u, delta_softplus,
                          merge_scale, per_dir_inputs, per_dir_params, None, 0)
        self.args.y = None
        n = ctypes.c_uint64()
        check(lib.vscan_backward_workspace_size(route.handle, ctypes.byref(self.args), ctypes.byref(n)))
        self.workspace = torch.empty(max(n.value, 256), dtype=torch.uint8, device=dev)
        self.g = VscanGrads()
        for k, t in self.grads.items():
            setattr(self.g, k, ctypes.c_void_p(t.data_ptr()))
        self.g.workspace, self.g.workspace_bytes = ctypes.c_void_p(self.workspace.data_ptr()), n.value
        self._keep = (u, delta, A, B, C, Dskip, delta_bias, z, dy)
        self._dy = ctypes.c_void_p(dy.data_ptr())
        self._ra, self._rg = ctypes.byref(self.args), ctypes.byref(self.g)

    def kernels(self):
        """Kernel launches of one run(): the pre-gate forward, then the gate gradient and the
        adjoint scan (grid routes) or pooling with the gate gradient, the adjoint scan and
        unpooling (pooled routes)."""
        n = ctypes.c_int32()
        check(lib.vscan_plan_info(self.route.handle, ctypes.byref(self.args), ctypes.byref(n)))
        return n.value + (3 if self.route.kind_name in ("pool_w", "pool_h") else 2)

    def kernel_name(self):
        """Name of the kernel that runs the adjoint scan (vscan_backward_plan_kernel)."""
        name = ctypes.c_char_p()
        check(lib.vscan_backward_plan_kernel(self.route.handle, self._ra, ctypes.byref(name)))
        return name.value.decode()

    def run(self, stream):
        """Enqueue the backward pass on a torch.cuda.Stream."""
        check(lib.vscan_backward(self.route.handle, self._ra, self._dy, self._rg, ctypes.c_void_p(stream.cuda_stream)))


__all__.append("BackwardPlan")
