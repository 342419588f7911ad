"""ctypes binding of libmoe.so (include/moe.h): argument marshalling only.

Every step of the layer runs in the library's CUDA kernels. If the library is
missing or cannot be loaded, every entry point raises: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe.so")
# the same library built with MOE_DEBUG (device bounds checks); tests only
DEBUG_LIB_PATH = os.path.join(_PKG, "libmoe_debug.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED = 2
MOE_ERR_WORKSPACE = 3
MOE_ERR_CUDA = 4
MOE_ERR_DEVICE_TIMEOUT = 5
MOE_ERR_SCRATCH_LIMIT = 6
MOE_ERR_DEVICE_BOUNDS = 7
MOE_NO_ALLOC_WORKSPACE_BYTES = 64 << 20
MOE_F32 = 0
MOE_BF16 = 1
MOE_GATE_RENORM, MOE_GATE_RAW, MOE_GATE_SIGMOID = 0, 1, 2
MOE_WEIGHTS_DTYPE, MOE_WEIGHTS_FP8, MOE_WEIGHTS_FP8_W8A8, MOE_WEIGHTS_MXFP4 = 0, 1, 2, 3
MOE_NUM_KERNELS = 7
KERNEL_NAMES = ("router_logits", "route", "scan", "scatter", "gate_up_swiglu", "down_scale", "combine")

EXPORTED = ("moe_workspace_size", "moe_capacity", "moe_forward", "moe_forward_host_io",
            "moe_workspace_layout", "moe_get_device_status", "moe_status_string",
            "moe_forward_no_alloc", "moe_quantize_fp8", "moe_dequantize_fp8",
            "moe_quantize_mxfp4", "moe_dequantize_mxfp4")


class moe_dims(ctypes.Structure):
    _fields_ = [
        ("T", ctypes.c_int64),
        ("d", ctypes.c_int32),
        ("d_e", ctypes.c_int32),
        ("d_s", ctypes.c_int32),
        ("dtype", ctypes.c_int32),
        ("gate_mode", ctypes.c_int32),
        ("router_bias", ctypes.c_void_p),
        ("workspace", ctypes.c_void_p),
        ("workspace_bytes", ctypes.c_size_t),
        ("stream", ctypes.c_void_p),
        ("events", ctypes.c_void_p),
        ("selection_bias", ctypes.c_void_p),
        ("n_group", ctypes.c_int32),
        ("topk_group", ctypes.c_int32),
        ("weight_format", ctypes.c_int32),
        ("weight_scales", ctypes.c_void_p),
        ("wait_timeout_ns", ctypes.c_uint64),
        ("weight_block_scales", ctypes.c_void_p),
    ]


class moe_workspace_layout_t(ctypes.Structure):
    _fields_ = [
        ("logits", ctypes.c_size_t),
        ("topk_idx", ctypes.c_size_t),
        ("gates", ctypes.c_size_t),
        ("slot_pos", ctypes.c_size_t),
        ("probsum", ctypes.c_size_t),
        ("tile_start", ctypes.c_size_t),
        ("xp", ctypes.c_size_t),
        ("h", ctypes.c_size_t),
        ("yrows", ctypes.c_size_t),
        ("rows_max", ctypes.c_int64),
        ("capacity", ctypes.c_int64),
        ("xscale", ctypes.c_size_t),
        ("hq", ctypes.c_size_t),
        ("hscale", ctypes.c_size_t),
        ("status", ctypes.c_size_t),
    ]


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


_lib = None
_debug_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libmoe.so once and declare its signatures. Raises if it is absent."""
    global _lib
    if _lib is None:
        _lib = _open(path)
    return _lib


def load_debug() -> ctypes.CDLL:
    """The MOE_DEBUG build (libmoe_debug.so), loaded once beside the release one."""
    global _debug_lib
    if _debug_lib is None:
        _debug_lib = _open(DEBUG_LIB_PATH)
    return _debug_lib


def _open(path: str) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise RuntimeError(f"{os.path.basename(path)} not found at {path}; build it with "
                           "`python -m sparse_mixture_experts_aux_b200.build`")
    lib = ctypes.CDLL(path)
    P = ctypes.POINTER
    vp, i32, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.moe_workspace_size.argtypes = [P(moe_dims), i32, i32, f32]
    lib.moe_workspace_size.restype = ctypes.c_size_t
    lib.moe_capacity.argtypes = [ctypes.c_int64, i32, i32, f32]
    lib.moe_capacity.restype = ctypes.c_int64
    lib.moe_forward.argtypes = [P(moe_dims), vp, vp, vp, vp, vp, vp, i32, i32, f32, vp, vp, vp]
    lib.moe_forward.restype = i32
    lib.moe_forward_host_io.argtypes = [P(moe_dims), vp, vp, vp, vp, vp, vp, vp, i32, i32, f32,
                                        vp, vp, vp, vp, vp, vp]
    lib.moe_forward_host_io.restype = i32
    lib.moe_forward_no_alloc.argtypes = [P(moe_dims), vp, vp, vp, vp, vp, vp, i32, i32, f32, vp, vp,
                                         vp]
    lib.moe_forward_no_alloc.restype = i32
    lib.moe_workspace_layout.argtypes = [P(moe_dims), i32, i32, f32, P(moe_workspace_layout_t)]
    lib.moe_workspace_layout.restype = i32
    lib.moe_get_device_status.argtypes = []
    lib.moe_get_device_status.restype = i32
    lib.moe_status_string.argtypes = [i32]
    lib.moe_status_string.restype = ctypes.c_char_p
    lib.moe_quantize_fp8.argtypes = [vp, i32, ctypes.c_int64, i32, vp, vp, vp]
    lib.moe_quantize_fp8.restype = i32
    lib.moe_dequantize_fp8.argtypes = [vp, vp, ctypes.c_int64, i32, vp, vp]
    lib.moe_dequantize_fp8.restype = i32
    lib.moe_quantize_mxfp4.argtypes = [vp, i32, ctypes.c_int64, i32, vp, vp, vp, vp]
    lib.moe_quantize_mxfp4.restype = i32
    lib.moe_dequantize_mxfp4.argtypes = [vp, vp, vp, ctypes.c_int64, i32, vp, vp]
    lib.moe_dequantize_mxfp4.restype = i32
    return lib


def status_string(status: int) -> str:
    return load().moe_status_string(int(status)).decode()


def _ref(dims):
    return ctypes.byref(dims) if dims is not None else None


def _ptr(t) -> int:
    if t is None:
        return 0
    if isinstance(t, int):
        return t
    return t.data_ptr()


def make_dims(T: int, d: int, d_e: int, d_s: int = 0, dtype: int = MOE_BF16, router_bias=None,
              workspace=None, workspace_bytes: int = 0, stream: int = 0, events=None,
              gate_mode: int = 0, wait_timeout_ns: int = 0, selection_bias=None,
              n_group: int = 0, topk_group: int = 0, weight_format: int = MOE_WEIGHTS_DTYPE,
              weight_scales=None, weight_block_scales=None) -> moe_dims:
    """Fill a moe_dims. `events` is a ctypes array of cudaEvent_t handles or None."""
    dims = moe_dims()
    dims.T, dims.d, dims.d_e, dims.d_s = int(T), int(d), int(d_e), int(d_s)
    dims.dtype, dims.gate_mode = int(dtype), int(gate_mode)
    dims.router_bias = _ptr(router_bias) or None
    dims.workspace = _ptr(workspace) or None
    dims.workspace_bytes = int(workspace_bytes)
    dims.stream = int(stream) or None
    dims.events = ctypes.cast(events, ctypes.c_void_p) if events is not None else None
    dims.wait_timeout_ns = int(wait_timeout_ns)
    dims.selection_bias = _ptr(selection_bias) or None
    dims.n_group, dims.topk_group = int(n_group), int(topk_group)
    dims.weight_format = int(weight_format)
    dims.weight_scales = _ptr(weight_scales) or None
    dims.weight_block_scales = _ptr(weight_block_scales) or None
    return dims


def moe_workspace_size(dims: moe_dims, E: int, k: int, capacity_factor: float) -> int:
    return int(load().moe_workspace_size(ctypes.byref(dims), E, k, capacity_factor))


def moe_capacity(T: int, E: int, k: int, capacity_factor: float) -> int:
    return int(load().moe_capacity(T, E, k, capacity_factor))


def moe_workspace_layout(dims: moe_dims, E: int, k: int, capacity_factor: float) -> moe_workspace_layout_t:
    out = moe_workspace_layout_t()
    st = load().moe_workspace_layout(ctypes.byref(dims), E, k, capacity_factor, ctypes.byref(out))
    if st != MOE_OK:
        raise MoeError(st, "moe_workspace_layout")
    return out


def moe_forward(dims: moe_dims, x, W_r, W_g, W_u, W_d, W_shared, E: int, k: int,
                capacity_factor: float, y, aux, counts, check: bool = True) -> int:
    st = load().moe_forward(_ref(dims), _ptr(x), _ptr(W_r), _ptr(W_g), _ptr(W_u),
                            _ptr(W_d), _ptr(W_shared), E, k, capacity_factor, _ptr(y), _ptr(aux),
                            _ptr(counts))
    if check and st != MOE_OK:
        raise MoeError(st, "moe_forward")
    return st


def moe_forward_host_io(dims: moe_dims, x_host, x_dev, W_r, W_g, W_u, W_d, W_shared, E: int,
                        k: int, capacity_factor: float, y_dev, y_host, aux_dev, aux_host,
                        counts_dev, counts_host, check: bool = True) -> int:
    st = load().moe_forward_host_io(_ref(dims), _ptr(x_host), _ptr(x_dev), _ptr(W_r),
                                    _ptr(W_g), _ptr(W_u), _ptr(W_d), _ptr(W_shared), E, k,
                                    capacity_factor, _ptr(y_dev), _ptr(y_host), _ptr(aux_dev),
                                    _ptr(aux_host), _ptr(counts_dev), _ptr(counts_host))
    if check and st != MOE_OK:
        raise MoeError(st, "moe_forward_host_io")
    return st


def moe_forward_no_alloc(dims: moe_dims, x, W_r, W_g, W_u, W_d, W_shared, E: int, k: int,
                         capacity_factor: float, y, aux, counts, check: bool = True) -> int:
    """moe_forward on the library's static scratch; dims.workspace is ignored."""
    st = load().moe_forward_no_alloc(_ref(dims), _ptr(x), _ptr(W_r), _ptr(W_g), _ptr(W_u),
                                     _ptr(W_d), _ptr(W_shared), E, k, capacity_factor, _ptr(y),
                                     _ptr(aux), _ptr(counts))
    if check and st != MOE_OK:
        raise MoeError(st, "moe_forward_no_alloc")
    return st


def moe_get_device_status() -> int:
    return int(load().moe_get_device_status())


def moe_quantize_fp8(w, dtype: int, rows: int, cols: int, codes, scales, stream: int = 0) -> int:
    """Raw call: returns the status code."""
    return int(load().moe_quantize_fp8(_ptr(w) or None, int(dtype), int(rows), int(cols),
                                       _ptr(codes) or None, _ptr(scales) or None, int(stream) or None))


def moe_dequantize_fp8(codes, scales, rows: int, cols: int, out, stream: int = 0) -> int:
    """Raw call: returns the status code."""
    return int(load().moe_dequantize_fp8(_ptr(codes) or None, _ptr(scales) or None, int(rows),
                                         int(cols), _ptr(out) or None, int(stream) or None))


def moe_quantize_mxfp4(w, dtype: int, rows: int, cols: int, codes, block_scales, row_factors,
                       stream: int = 0) -> int:
    """Raw call: returns the status code."""
    return int(load().moe_quantize_mxfp4(_ptr(w) or None, int(dtype), int(rows), int(cols),
                                         _ptr(codes) or None, _ptr(block_scales) or None,
                                         _ptr(row_factors) or None, int(stream) or None))


def moe_dequantize_mxfp4(codes, block_scales, row_factors, rows: int, cols: int, out,
                         stream: int = 0) -> int:
    """Raw call: returns the status code."""
    return int(load().moe_dequantize_mxfp4(_ptr(codes) or None, _ptr(block_scales) or None,
                                           _ptr(row_factors) or None, int(rows), int(cols),
                                           _ptr(out) or None, int(stream) or None))
