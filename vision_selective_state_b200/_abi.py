"""ctypes view of the C ABI in include/vscan.h (libvscan.so, built in-tree).

Argument marshalling only: no arithmetic of the scan happens in Python. Loading
fails loudly when the library has not been built; there is no fallback path.
"""
import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libvscan.so")

OK = 0
STATUS = {
    0: "VSCAN_OK",
    -1: "VSCAN_ERR_INVALID_ARGUMENT",
    -2: "VSCAN_ERR_SHAPE",
    -3: "VSCAN_ERR_ALIGNMENT",
    -4: "VSCAN_ERR_UNSUPPORTED",
    -5: "VSCAN_ERR_CUDA",
    -6: "VSCAN_ERR_WORKSPACE",
    -7: "VSCAN_ERR_VALUE",
    -8: "VSCAN_ERR_DEVICE_TIMEOUT",
}
ROUTES = {"bidir": 0, "cross4": 1, "atrous2": 2, "pool_w": 3, "pool_h": 4}
F32, BF16 = 0, 1
ABI_VERSION = 5
FLAG_ZOH = 1
FLAG_CHECK_VALUES = 2


class VscanArgs(ctypes.Structure):
    """Mirror of struct vscan_args (include/vscan.h)."""

    _fields_ = [
        ("batch", ctypes.c_int32),
        ("channels", ctypes.c_int32),
        ("d_state", ctypes.c_int32),
        ("dtype", ctypes.c_int32),
        ("u", ctypes.c_void_p),
        ("delta", ctypes.c_void_p),
        ("B", ctypes.c_void_p),
        ("C", ctypes.c_void_p),
        ("z", ctypes.c_void_p),
        ("y", ctypes.c_void_p),
        ("A", ctypes.c_void_p),
        ("Dskip", ctypes.c_void_p),
        ("delta_bias", ctypes.c_void_p),
        ("per_dir_inputs", ctypes.c_int32),
        ("per_dir_params", ctypes.c_int32),
        ("delta_softplus", ctypes.c_int32),
        ("merge_scale", ctypes.c_float),
        ("workspace", ctypes.c_void_p),
        ("workspace_bytes", ctypes.c_uint64),
        ("seq_chunks", ctypes.c_int32),
        ("flags", ctypes.c_int32),
        ("conv_w", ctypes.c_void_p),
        ("conv_b", ctypes.c_void_p),
        ("token_pos", ctypes.c_void_p),
        ("n_tokens", ctypes.c_int32),
        ("reserved2", ctypes.c_int32),
        ("status", ctypes.c_void_p),
        ("tok_stride", ctypes.c_int64),
        ("batch_stride", ctypes.c_int64),
        ("bc_tok_stride", ctypes.c_int64),
        ("bc_batch_stride", ctypes.c_int64),
    ]


class VscanGrads(ctypes.Structure):
    """Mirror of struct vscan_grads (include/vscan.h)."""

    _fields_ = [(name, ctypes.c_void_p) for name in
                ("du", "ddelta", "dB", "dC", "dA", "dDskip", "dbias", "dz", "workspace")] + [
        ("workspace_bytes", ctypes.c_uint64)]


class VscanError(RuntimeError):
    def __init__(self, status, message):
        self.status = status
        super().__init__(f"{STATUS.get(status, status)}: {message}")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -c 'import __graft_entry__ as g; g.build()'` "
            "(or python vision_selective_state_b200/build.py). There is no CPU fallback.")
    lib = ctypes.CDLL(LIB_PATH)
    i32, p, u64 = ctypes.c_int32, ctypes.c_void_p, ctypes.c_uint64
    pa = ctypes.POINTER(VscanArgs)
    sigs = {
        "vscan_create_route": ([ctypes.POINTER(p), i32, i32, i32, i32], i32),
        "vscan_destroy": ([p], i32),
        "vscan_route_info": ([p] + [ctypes.POINTER(i32)] * 5, i32),
        "vscan_route_indices": ([p, p, p], i32),
        "vscan_workspace_size": ([p, pa, ctypes.POINTER(u64)], i32),
        "vscan_forward": ([p, pa, p], i32),
        "vscan_plan_info": ([p, pa, ctypes.POINTER(i32)], i32),
        "vscan_plan_kernel": ([p, pa, ctypes.POINTER(ctypes.c_char_p)], i32),
        "vscan_forward_pooled_noalloc": ([p, pa, p], i32),
        "vscan_host_buffer_size": ([p, pa, ctypes.POINTER(u64)], i32),
        "vscan_forward_host": ([p, pa, p, u64, p], i32),
        "vscan_backward_workspace_size": ([p, pa, ctypes.POINTER(u64)], i32),
        "vscan_backward_plan_kernel": ([p, pa, ctypes.POINTER(ctypes.c_char_p)], i32),
        "vscan_backward": ([p, pa, p, ctypes.POINTER(VscanGrads), p], i32),
        "vscan_last_error": ([], ctypes.c_char_p),
        "vscan_status_string": ([i32], ctypes.c_char_p),
        "vscan_status_from_device_word": ([i32], i32),
        "vscan_abi_version": ([], i32),
    }
    for name, (argtypes, restype) in sigs.items():
        fn = getattr(lib, name)
        fn.argtypes = argtypes
        fn.restype = restype
    if lib.vscan_abi_version() != ABI_VERSION:
        raise ImportError(f"libvscan.so ABI {lib.vscan_abi_version()} != binding ABI {ABI_VERSION}")
    return lib


lib = _load()


def check(status):
    if status != OK:
        raise VscanError(status, lib.vscan_last_error().decode())
    return status
