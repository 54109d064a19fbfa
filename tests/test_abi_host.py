"""Host-side checks of the C ABI: no GPU needed, no kernel launched.

Every call here either is host-only by contract (route creation, geometry,
workspace sizing) or fails argument validation, which the library performs
before its first CUDA call. No call with plausible-looking fake device pointers
is ever allowed to pass validation.
"""
import ctypes
import os
import re

import pytest
import torch

from conftest import ROOT, read_golden

import oracle as O

abi = pytest.importorskip("vision_selective_state_b200._abi")
vs = pytest.importorskip("vision_selective_state_b200")

HEADER = os.path.join(ROOT, "include", "vscan.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(vscan_[a-z_]+)\s*\(", text)))


def test_library_exports_every_declared_function():
    names = declared_functions()
    assert len(names) >= 10
    lib = ctypes.CDLL(abi.LIB_PATH)
    for name in names:
        assert hasattr(lib, name), name


def test_struct_layout_matches_the_header():
    # int32 x4, 6 pointers, 3 pointers, int32 x3, float, pointer, uint64, int32 x2, 3 pointers, int32 x2,
    # pointer, int64 x4
    assert ctypes.sizeof(abi.VscanArgs) == 16 + 48 + 24 + 12 + 4 + 8 + 8 + 8 + 24 + 8 + 8 + 32
    assert abi.VscanArgs.flags.offset == 124 and abi.VscanArgs.conv_w.offset == 128
    assert abi.VscanArgs.token_pos.offset == 144 and abi.VscanArgs.n_tokens.offset == 152
    assert abi.VscanArgs.status.offset == 160
    assert (abi.VscanArgs.tok_stride.offset, abi.VscanArgs.batch_stride.offset,
            abi.VscanArgs.bc_tok_stride.offset, abi.VscanArgs.bc_batch_stride.offset) == (168, 176, 184, 192)
    assert abi.lib.vscan_abi_version() == abi.ABI_VERSION == 5


def test_status_strings():
    for code, name in abi.STATUS.items():
        assert abi.lib.vscan_status_string(code).decode() == name


@pytest.mark.parametrize("kind", ["bidir", "cross4", "atrous2", "pool_w", "pool_h"])
@pytest.mark.parametrize("h,w", [(1, 1), (3, 5), (14, 14), (55, 57), (56, 56), (128, 128)])
def test_route_geometry_matches_the_oracle(kind, h, w):
    cls = (h * w) // 2 if kind == "bidir" else -1
    r = vs.Route(kind, h, w, cls)
    K, L, T = O.geometry(kind, h, w, cls)
    assert (r.K, r.seq_len, r.tokens) == (K, L, T)
    if kind == "atrous2":
        assert (r.padded_h, r.padded_w) == (h + h % 2, w + w % 2)
    r.close()


def test_vim_sequence_lengths_fixture():
    for ln in read_golden("vim_sequence_lengths.txt"):
        h, w, cls, tokens = map(int, ln.split())
        r = vs.Route("bidir", h, w, cls)
        assert (r.K, r.seq_len, r.tokens) == (2, tokens, tokens)


@pytest.mark.parametrize("kind,h,w,cls,status", [
    ("bidir", 14, 14, 97, -2), ("bidir", 0, 4, -1, -1), ("cross4", 4, 4, 8, -2),
    ("atrous2", 3, -1, -1, -1), ("pool_w", 4, 4, 0, -2), (7, 4, 4, -1, -1),
])
def test_invalid_routes_are_rejected(kind, h, w, cls, status):
    handle = ctypes.c_void_p()
    code = abi.ROUTES[kind] if isinstance(kind, str) else kind
    got = abi.lib.vscan_create_route(ctypes.byref(handle), code, h, w, cls)
    assert got == status
    assert handle.value is None
    assert abi.lib.vscan_last_error().decode()


def _args(**kw):
    a = abi.VscanArgs()
    a.batch, a.channels, a.d_state, a.dtype = 2, 16, 16, abi.F32
    a.delta_softplus, a.merge_scale = 1, 1.0
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def test_workspace_sizes():
    n = ctypes.c_uint64()
    for kind, expect in (("atrous2", 0), ("bidir", 2 * 2 * 197 * 16 * 4), ("cross4", 4 * 2 * 36 * 16 * 4)):
        h, w, cls = (14, 14, 98) if kind == "bidir" else (6, 6, -1)
        r = vs.Route(kind, h, w, cls)
        assert abi.lib.vscan_workspace_size(r.handle, ctypes.byref(_args()), ctypes.byref(n)) == 0
        assert n.value == (expect + 255) // 256 * 256
    r = vs.Route("pool_w", 8, 8)
    assert abi.lib.vscan_workspace_size(r.handle, ctypes.byref(_args()), ctypes.byref(n)) == 0
    assert n.value == 2 * ((2 * 8 * 16 * 4 + 255) // 256 * 256)


@pytest.mark.parametrize("field,value,status", [
    ("channels", 6, -3), ("channels", 0, -1), ("d_state", 17, -4), ("d_state", 0, -1),
    ("dtype", 5, -1), ("batch", -1, -1), ("flags", 2, -1), ("flags", -1, -1), ("seq_chunks", 9, -1),
    ("seq_chunks", 3, -1), ("seq_chunks", -1, -1),
    ("per_dir_inputs", 2, -1), ("merge_scale", float("nan"), -1),
])
def test_bad_arguments_fail_before_any_cuda_call(field, value, status):
    r = vs.Route("atrous2", 5, 5)
    a = _args(**{field: value})
    assert abi.lib.vscan_forward(r.handle, ctypes.byref(a), None) == status
    n = ctypes.c_uint64()
    assert abi.lib.vscan_workspace_size(r.handle, ctypes.byref(a), ctypes.byref(n)) == status


def test_null_and_misaligned_pointers_are_rejected():
    r = vs.Route("atrous2", 5, 5)
    assert abi.lib.vscan_forward(r.handle, ctypes.byref(_args()), None) == -1  # u is NULL
    fake = dict(u=0x1000, delta=0x2000, B=0x3000, C=0x4000, y=0x5000, A=0x6000)
    a = _args(**dict(fake, delta=0x2004))
    assert abi.lib.vscan_forward(r.handle, ctypes.byref(a), None) == -3
    rb = vs.Route("bidir", 5, 5, 12)
    a = _args(**fake)  # BIDIR needs a workspace; none given
    assert abi.lib.vscan_forward(rb.handle, ctypes.byref(a), None) == -6
    a = _args(**fake, workspace=0x7000, workspace_bytes=64)
    assert abi.lib.vscan_forward(rb.handle, ctypes.byref(a), None) == -6
    assert "workspace" in abi.lib.vscan_last_error().decode()
    hb = _args(**fake)
    n = ctypes.c_uint64()
    assert abi.lib.vscan_host_buffer_size(rb.handle, ctypes.byref(hb), ctypes.byref(n)) == 0
    assert abi.lib.vscan_forward_host(rb.handle, ctypes.byref(hb), None, 0, None) == -6


def test_plan_info_counts_launches():
    n = ctypes.c_int32()
    for kind, h, w, cls, chunks, expect in (("atrous2", 56, 56, -1, 0, 1), ("cross4", 56, 56, -1, 0, 1),
                                            ("bidir", 64, 64, 2048, 1, 1), ("bidir", 14, 14, 98, 4, 1),
                                            ("pool_w", 8, 8, -1, 0, 2)):
        r = vs.Route(kind, h, w, cls)
        assert abi.lib.vscan_plan_info(r.handle, ctypes.byref(_args(seq_chunks=chunks)), ctypes.byref(n)) == 0
        assert n.value == expect, kind
    r = vs.Route("atrous2", 4, 4)
    assert abi.lib.vscan_plan_info(r.handle, ctypes.byref(_args(batch=0)), ctypes.byref(n)) == 0 and n.value == 0


def test_plan_kernel_names_the_scan_kernel():
    name = ctypes.c_char_p()
    for kind, h, w, cls, batch, D, chunks, expect in (
            ("atrous2", 56, 56, -1, 8, 192, 0, "stream_scan_kernel<ATROUS2>"),
            ("cross4", 56, 56, -1, 16, 192, 0, "pipe_scan_kernel<CROSS4>"),
            ("bidir", 64, 64, 2048, 64, 768, 0, "pipe_scan_kernel<BIDIR>"),
            ("bidir", 14, 14, 98, 1, 384, 0, "resident_scan_kernel<BIDIR>"),  # few sequences
            ("cross4", 14, 14, -1, 1, 64, 4, "resident_scan_kernel<CROSS4>"),
            ("atrous2", 9, 13, -1, 1, 64, 2, "resident_scan_kernel<ATROUS2>"),
            ("atrous2", 9, 13, -1, 1, 64, 1, "stream_scan_kernel<ATROUS2>"),
            ("pool_w", 8, 8, -1, 2, 64, 0, "pool_scan_kernel"),
            ("pool_h", 8, 8, -1, 2, 64, 0, "pool_scan_kernel"),
            ("atrous2", 4, 4, -1, 0, 64, 0, "none")):
        r = vs.Route(kind, h, w, cls)
        a = _args(batch=batch, channels=D, seq_chunks=chunks)
        assert abi.lib.vscan_plan_kernel(r.handle, ctypes.byref(a), ctypes.byref(name)) == 0
        assert name.value.decode() == expect, (kind, h, w, batch, chunks)
    r = vs.Route("atrous2", 4, 4)
    assert abi.lib.vscan_plan_kernel(r.handle, ctypes.byref(_args()), None) == -1
    assert abi.lib.vscan_plan_kernel(r.handle, ctypes.byref(_args(d_state=0)), ctypes.byref(name)) != 0


def test_backward_plan_kernel_names_the_adjoint_scan_kernel():
    """Grids of at most 8 adjoint tiles (8 channels x image x direction) per SM take the
    two-warp state split (148 SMs are assumed without a GPU)."""
    name = ctypes.c_char_p()
    for kind, h, w, cls, batch, D, expect in (
            ("atrous2", 56, 56, -1, 8, 192, "bwd_scan_split_kernel<ATROUS2>"),    # 768 tiles
            ("cross4", 56, 56, -1, 16, 192, "bwd_scan_kernel<CROSS4>"),           # 1536
            ("cross4", 56, 56, -1, 8, 192, "bwd_scan_split_kernel<CROSS4>"),      # 768
            ("bidir", 14, 14, 98, 1, 384, "bwd_scan_split_kernel<BIDIR>"),        # 96
            ("bidir", 64, 64, 2048, 64, 768, "bwd_scan_kernel<BIDIR>"),           # 12288
            ("pool_w", 128, 128, -1, 32, 384, "bwd_scan_kernel<BIDIR>"),          # 3072, pooled as BIDIR
            ("pool_h", 8, 8, -1, 2, 64, "bwd_scan_split_kernel<BIDIR>"),          # 32
            ("atrous2", 5, 5, -1, 296, 8, "bwd_scan_split_kernel<ATROUS2>"),      # 1184 = 8 x 148
            ("atrous2", 5, 5, -1, 297, 8, "bwd_scan_kernel<ATROUS2>"),            # 1188
            ("atrous2", 4, 4, -1, 0, 64, "none")):
        r = vs.Route(kind, h, w, cls)
        a = _args(batch=batch, channels=D)
        assert abi.lib.vscan_backward_plan_kernel(r.handle, ctypes.byref(a), ctypes.byref(name)) == 0
        assert name.value.decode() == expect, (kind, h, w, batch, D)
    r = vs.Route("bidir", 4, 4)
    assert abi.lib.vscan_backward_plan_kernel(r.handle, ctypes.byref(_args()), None) == -1
    assert abi.lib.vscan_backward_plan_kernel(r.handle, ctypes.byref(_args(d_state=0)), ctypes.byref(name)) != 0


def test_chunked_scan_needs_the_tile_on_chip():
    big = vs.Route("cross4", 56, 56)
    assert abi.lib.vscan_forward(big.handle, ctypes.byref(_args(seq_chunks=4)), None) == -4
    small = vs.Route("cross4", 14, 14)
    # passes the shape checks, then stops at the NULL tensors
    assert abi.lib.vscan_forward(small.handle, ctypes.byref(_args(seq_chunks=4)), None) == -1


def test_noalloc_pooled_forward_rejects_before_any_cuda_call():
    fake = dict(u=0x1000, delta=0x2000, B=0x3000, C=0x4000, y=0x5000, A=0x6000)
    r = vs.Route("cross4", 8, 8)  # not a pooled route
    assert abi.lib.vscan_forward_pooled_noalloc(r.handle, ctypes.byref(_args(**fake)), None) == -4
    # 2 planes x 256 images x 256 pooled steps x 16 states x 4 bytes = 8 MiB > 4 MiB
    big = vs.Route("pool_w", 256, 2)
    a = _args(**fake, batch=256)
    assert abi.lib.vscan_forward_pooled_noalloc(big.handle, ctypes.byref(a), None) == -4
    assert "fixed scratch" in abi.lib.vscan_last_error().decode()


def test_pooled_route_length_limit():
    r = vs.Route("pool_w", 4000, 2)
    assert abi.lib.vscan_forward(r.handle, ctypes.byref(_args()), None) == -4


def test_convolution_is_refused_on_grid_routes_and_conv_b_needs_conv_w():
    fake = dict(u=0x1000, delta=0x2000, B=0x3000, C=0x4000, y=0x5000, A=0x6000)
    for kind in ("cross4", "atrous2"):
        r = vs.Route(kind, 4, 4)
        assert abi.lib.vscan_forward(r.handle, ctypes.byref(_args(**fake, conv_w=0x7000)), None) == -4
        assert "BIDIR and the pooled routes" in abi.lib.vscan_last_error().decode()
    r = vs.Route("bidir", 4, 4)
    assert abi.lib.vscan_forward(r.handle, ctypes.byref(_args(**fake, conv_b=0x7000)), None) == -1
    # accepted on BIDIR and the pooled routes: the next failure is the missing workspace
    for kind in ("bidir", "pool_w", "pool_h"):
        r = vs.Route(kind, 4, 4)
        assert abi.lib.vscan_forward(r.handle, ctypes.byref(_args(**fake, conv_w=0x7000)), None) == -6


def test_zoh_flag_is_accepted_and_unknown_flags_are_not():
    fake = dict(u=0x1000, delta=0x2000, B=0x3000, C=0x4000, y=0x5000, A=0x6000)
    r = vs.Route("atrous2", 4, 4)
    assert abi.lib.vscan_forward(r.handle, ctypes.byref(_args(**fake, flags=abi.FLAG_ZOH)), None) != -1
    assert abi.lib.vscan_forward(r.handle, ctypes.byref(_args(**fake, flags=4)), None) == -1


def test_value_check_flag_needs_an_aligned_status_word():
    fake = dict(u=0x1000, delta=0x2000, B=0x3000, C=0x4000, y=0x5000, A=0x6000)
    r = vs.Route("cross4", 4, 4)
    chk = abi.FLAG_CHECK_VALUES
    assert abi.lib.vscan_forward(r.handle, ctypes.byref(_args(**fake, flags=chk)), None) == -1
    assert "status" in abi.lib.vscan_last_error().decode()
    assert abi.lib.vscan_forward(r.handle, ctypes.byref(_args(**fake, flags=chk, status=0x7002)), None) == -3
    # accepted: the next failure is the missing workspace
    assert abi.lib.vscan_forward(r.handle, ctypes.byref(_args(**fake, flags=chk, status=0x7000)), None) == -6
    assert abi.lib.vscan_forward(r.handle, ctypes.byref(_args(**fake, flags=chk | abi.FLAG_ZOH,
                                                              status=0x7000)), None) == -6
    n = ctypes.c_int32()
    assert abi.lib.vscan_plan_info(r.handle, ctypes.byref(_args(**fake, flags=chk, status=0x7000)),
                                   ctypes.byref(n)) == 0
    assert n.value == 2


def test_device_status_words_decode_on_the_host():
    assert abi.lib.vscan_status_from_device_word(0) == 0
    assert abi.lib.vscan_status_from_device_word(1) == -7
    assert "value check" in abi.lib.vscan_last_error().decode()
    assert abi.lib.vscan_status_from_device_word(2) == -8
    assert abi.lib.vscan_status_from_device_word(3) == -8
    assert abi.lib.vscan_status_from_device_word(8) == -1


def test_plan_kernel_names_the_pipelined_kernel():
    fake = dict(u=0x1000, delta=0x2000, B=0x3000, C=0x4000, y=0x5000, A=0x6000)
    name = ctypes.c_char_p()
    for kind, expect in (("bidir", "pipe_scan_kernel<BIDIR>"), ("cross4", "pipe_scan_kernel<CROSS4>"),
                         ("atrous2", "stream_scan_kernel<ATROUS2>")):
        r = vs.Route(kind, 8, 8)
        for extra, exp in ((dict(seq_chunks=1), expect),
                           (dict(seq_chunks=1, flags=abi.FLAG_ZOH), f"stream_scan_kernel<{kind.upper()}>"),
                           (dict(seq_chunks=1, d_state=8), f"stream_scan_kernel<{kind.upper()}>")):
            assert abi.lib.vscan_plan_kernel(r.handle, ctypes.byref(_args(**{**fake, **extra})),
                                             ctypes.byref(name)) == 0
            assert name.value.decode() == exp, (kind, extra)


def test_host_buffer_holds_the_convolution_parameters():
    r = vs.Route("bidir", 6, 6, 18)
    n0, n1 = ctypes.c_uint64(), ctypes.c_uint64()
    assert abi.lib.vscan_host_buffer_size(r.handle, ctypes.byref(_args()), ctypes.byref(n0)) == 0
    a = _args(conv_w=1, conv_b=1)
    assert abi.lib.vscan_host_buffer_size(r.handle, ctypes.byref(a), ctypes.byref(n1)) == 0
    assert n1.value - n0.value == 2 * 256  # [D][4] and [D] floats, 256-byte rounded (D = 16)


def test_masked_token_sets_are_checked_on_the_host():
    fake = dict(u=0x1000, delta=0x2000, B=0x3000, C=0x4000, y=0x5000, A=0x6000)
    for kind in ("bidir", "cross4", "atrous2"):
        r = vs.Route(kind, 4, 4, 8 if kind == "bidir" else -1)
        assert abi.lib.vscan_forward(r.handle, ctypes.byref(_args(**fake, token_pos=0x7000, n_tokens=3)), None) == -4
    r = vs.Route("pool_w", 4, 4)
    assert abi.lib.vscan_forward(r.handle, ctypes.byref(_args(**fake, n_tokens=3)), None) == -1
    assert abi.lib.vscan_forward(r.handle, ctypes.byref(_args(**fake, token_pos=0x7000, n_tokens=-1)), None) == -1
    assert abi.lib.vscan_forward(r.handle, ctypes.byref(_args(**fake, token_pos=0x7000, n_tokens=3,
                                                              conv_w=0x8000)), None) == -4
    assert abi.lib.vscan_forward(r.handle, ctypes.byref(_args(**fake, reserved2=1)), None) == -1
    # accepted: the next failure is the missing workspace
    assert abi.lib.vscan_forward(r.handle, ctypes.byref(_args(**fake, token_pos=0x7000, n_tokens=3)), None) == -6
    # the host buffer holds the visible tokens and their positions, not the grid
    n_dense, n_mask = ctypes.c_uint64(), ctypes.c_uint64()
    big = vs.Route("pool_w", 64, 64)
    assert abi.lib.vscan_host_buffer_size(big.handle, ctypes.byref(_args()), ctypes.byref(n_dense)) == 0
    a = _args(token_pos=1, n_tokens=1024)
    assert abi.lib.vscan_host_buffer_size(big.handle, ctypes.byref(a), ctypes.byref(n_mask)) == 0
    assert n_mask.value < n_dense.value


def test_backward_argument_checks_run_before_any_cuda_call():
    fake = dict(u=0x1000, delta=0x2000, B=0x3000, C=0x4000, y=0x5000, A=0x6000)
    r = vs.Route("bidir", 4, 4)
    n = ctypes.c_uint64()
    for extra in (dict(conv_w=0x7000), dict(flags=abi.FLAG_ZOH)):
        assert abi.lib.vscan_backward_workspace_size(r.handle, ctypes.byref(_args(**fake, **extra)),
                                                     ctypes.byref(n)) == -4
    pw = vs.Route("pool_w", 4, 4)
    assert abi.lib.vscan_backward_workspace_size(pw.handle, ctypes.byref(_args(**fake, token_pos=0x7000, n_tokens=3)),
                                                 ctypes.byref(n)) == -4
    # size: forward workspace + pre-gate output + gy + checkpoints (batch 2, 16 tokens, D 16, N 16)
    assert abi.lib.vscan_backward_workspace_size(r.handle, ctypes.byref(_args(**fake)), ctypes.byref(n)) == 0
    fwd = 2 * 2 * 16 * 16 * 4
    assert n.value == fwd + 2 * 16 * 16 * 4 + 2 * 16 * 16 * 4 + 2 * 2 * 1 * 16 * 16 * 4
    g = abi.VscanGrads()
    assert abi.lib.vscan_backward(r.handle, ctypes.byref(_args(**fake)), None, ctypes.byref(g), None) == -1
    assert abi.lib.vscan_backward(r.handle, ctypes.byref(_args(**fake)), ctypes.c_void_p(0x8000), None, None) == -1
    g.dz = 0x9000  # dz without z
    assert abi.lib.vscan_backward(r.handle, ctypes.byref(_args(**fake)), ctypes.c_void_p(0x8000),
                                  ctypes.byref(g), None) == -1
    g.dz = None  # workspace missing
    assert abi.lib.vscan_backward(r.handle, ctypes.byref(_args(**fake)), ctypes.c_void_p(0x8000),
                                  ctypes.byref(g), None) == -6


@pytest.mark.parametrize("field,value,status", [
    ("tok_stride", -4, -1), ("tok_stride", 8, -3), ("tok_stride", 18, -3), ("batch_stride", 16, -3),
    ("batch_stride", 17 * 16 + 2, -3), ("bc_tok_stride", 8, -1), ("bc_batch_stride", 16, -1)])
def test_stride_checks(field, value, status):
    r = vs.Route("bidir", 4, 4, 8)  # 17 tokens; channels 16, d_state 16, float32 (multiples of 4)
    n = ctypes.c_uint64()
    assert abi.lib.vscan_workspace_size(r.handle, ctypes.byref(_args(**{field: value})), ctypes.byref(n)) == status


def test_workspace_counts_packed_copies():
    r = vs.Route("bidir", 4, 4, 8)
    r256 = lambda x: (x + 255) // 256 * 256
    path = r256(2 * 2 * 17 * 16 * 4)          # parking planes: K x batch x tokens x D float32
    plane = r256(2 * 17 * 16 * 4)             # one packed batch x tokens x 16 float32 tensor
    n = ctypes.c_uint64()

    def ws(**kw):
        assert abi.lib.vscan_workspace_size(r.handle, ctypes.byref(_args(**kw)), ctypes.byref(n)) == 0
        return n.value
    assert ws() == path
    assert ws(tok_stride=16, batch_stride=17 * 16, bc_tok_stride=16, bc_batch_stride=17 * 16) == path  # dense
    assert ws(tok_stride=32) == path + 3 * plane             # u, delta, y
    assert ws(tok_stride=32, z=0x7000) == path + 4 * plane   # and z
    assert ws(batch_stride=18 * 16) == path + 3 * plane      # padding between images only
    assert ws(bc_tok_stride=20) == path + 2 * plane          # B, C
    assert ws(tok_stride=32, bc_batch_stride=20 * 16) == path + 5 * plane


def test_plan_info_counts_pack_launches():
    r = vs.Route("bidir", 64, 64, 2048)
    n = ctypes.c_int32()

    def launches(**kw):
        assert abi.lib.vscan_plan_info(r.handle, ctypes.byref(_args(seq_chunks=1, **kw)), ctypes.byref(n)) == 0
        return n.value
    assert launches() == 1
    assert launches(tok_stride=32) == 4                 # pack u, delta; scan; copy y out
    assert launches(tok_stride=32, z=0x7000) == 5
    assert launches(bc_tok_stride=32) == 3
    assert launches(tok_stride=32, bc_tok_stride=32) == 6


def test_dense_only_entry_points_reject_strides():
    fake = dict(u=0x1000, delta=0x2000, B=0x3000, C=0x4000, y=0x5000, A=0x6000)
    n = ctypes.c_uint64()
    for route in ("bidir", "pool_w"):
        r = vs.Route(route, 4, 4, 8 if route == "bidir" else -1)
        for kw in (dict(tok_stride=32), dict(bc_batch_stride=32 * 16)):
            a = _args(**fake, **kw)
            assert abi.lib.vscan_host_buffer_size(r.handle, ctypes.byref(a), ctypes.byref(n)) == -4
            assert "dense" in abi.lib.vscan_last_error().decode()
            assert abi.lib.vscan_backward_workspace_size(r.handle, ctypes.byref(a), ctypes.byref(n)) == -4
            if route == "pool_w":
                assert abi.lib.vscan_forward_pooled_noalloc(r.handle, ctypes.byref(a), None) == -4


def test_binding_reads_strides_from_views():
    u = torch.zeros(3, 17, 24)[:, :, :16]
    B = torch.zeros(3, 20, 18)[:, :17, :16]
    assert vs._layout(u, False) == (24, 17 * 24)
    assert vs._strides(u, u, None, u, B, B, False) == (24, 17 * 24, 18, 20 * 18)
    dense = torch.zeros(3, 17, 16)
    with pytest.raises(ValueError, match="delta"):
        vs._strides(u, dense, None, u, B, B, False)
    with pytest.raises(ValueError, match="contiguous"):
        vs._layout(torch.zeros(3, 17, 16).transpose(1, 2), False)
    planes = torch.zeros(2, 3, 18, 16)[:, :, :17, :]      # per-direction planes, batch x image stride apart
    assert vs._layout(planes, True) == (16, 18 * 16)
    with pytest.raises(ValueError, match="planes"):
        vs._layout(torch.zeros(2, 4, 17, 16)[:, :3], True)
