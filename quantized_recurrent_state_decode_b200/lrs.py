"""Python binding of liblrs (include/lrs.h): the same entry points, with
argument marshalling only.

Every function forwards to the C function of the same name. Tensors are
passed by their data pointer (torch tensors, or plain integers holding device
or host addresses); a `stream` of None means torch's current CUDA stream. A
status other than LRS_OK raises LrsError carrying the status and the
library's message. There is no fallback: if liblrs.so cannot be loaded, every
call raises.
"""
import ctypes
import os

LRS_OK = 0
LRS_ERR_INVALID_ARG = 1
LRS_ERR_ALIGNMENT = 2
LRS_ERR_UNSUPPORTED = 3
LRS_ERR_OOM = 4
LRS_ERR_CUDA = 5
LRS_ERR_DEVICE_TIMEOUT = 6
LRS_ERR_DEVICE_LAYOUT = 7
LRS_ERR_DEVICE_RANGE = 8
LRS_ERR_DEVICE_BOUNDS = 9

LRS_ROUND_RTN, LRS_ROUND_SR, LRS_ROUND_BDR = 0, 1, 2
LRS_UPDATE_GATED, LRS_UPDATE_DELTA = 0, 1
LRS_GATE_SCALAR, LRS_GATE_PER_KEY = 0, 1

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "liblrs.so")


class LrsError(RuntimeError):
    def __init__(self, status, message):
        super().__init__("%s (status %d)" % (message, status))
        self.status = status


class lrs_shape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("heads", ctypes.c_int32), ("d_k", ctypes.c_int32),
                ("d_v", ctypes.c_int32), ("group", ctypes.c_int32),
                ("update_kind", ctypes.c_int32), ("gate_kind", ctypes.c_int32)]


class lrs_state(ctypes.Structure):
    _fields_ = [("shape", lrs_shape), ("state_codes", ctypes.c_void_p),
                ("scales", ctypes.c_void_p), ("prec_map", ctypes.c_void_p),
                ("head_offsets", ctypes.c_void_p), ("batch_stride_bytes", ctypes.c_int64),
                ("code_bytes", ctypes.c_int64), ("scale_count", ctypes.c_int64),
                ("priv", ctypes.c_void_p)]


_lib = None

_P = ctypes.c_void_p
_SIGS = {
    "lrs_layout_query": [ctypes.POINTER(lrs_shape), _P, _P, _P, _P],
    "lrs_state_alloc": [ctypes.POINTER(lrs_shape), _P, ctypes.POINTER(lrs_state)],
    "lrs_layout_query_groups": [ctypes.POINTER(lrs_shape), _P, _P, _P, _P],
    "lrs_state_alloc_groups": [ctypes.POINTER(lrs_shape), _P, ctypes.POINTER(lrs_state)],
    "lrs_state_free": [ctypes.POINTER(lrs_state)],
    "lrs_decode_step": [ctypes.POINTER(lrs_state), _P, _P, _P, _P, _P, _P, _P, _P, _P,
                        ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int32, _P],
    "lrs_decode_step_bf16": [ctypes.POINTER(lrs_state), _P, _P, _P, _P, _P, _P, _P, _P, _P,
                             ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int32, _P],
    "lrs_chunk_step": [ctypes.POINTER(lrs_state), _P, _P, _P, ctypes.c_int32, _P, _P, _P, _P, _P,
                       _P, ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int32, _P],
    "lrs_lrb_step": [ctypes.POINTER(lrs_state), _P, _P, _P, ctypes.c_int32, _P, _P, _P, _P, _P, _P,
                     _P, _P, ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int32, _P],
    "lrs_decode_step_host": [ctypes.POINTER(lrs_state), _P, _P, _P, _P, _P, _P,
                             ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int32, _P],
    "lrs_decode_step_host_noalloc": [ctypes.POINTER(lrs_state), _P, _P, _P, _P, _P, _P, _P,
                                     ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int32, _P],
    "lrs_state_import_fp32": [ctypes.POINTER(lrs_state), _P, _P],
    "lrs_state_export_fp32": [ctypes.POINTER(lrs_state), _P, _P],
    "lrs_state_export_codes": [ctypes.POINTER(lrs_state), _P, _P],
    "lrs_state_import_codes": [ctypes.POINTER(lrs_state), _P, _P, _P],
    "lrs_state_copy_raw": [ctypes.POINTER(lrs_state), _P, _P, ctypes.c_int32, _P],
    "lrs_fp32_decode_step": [ctypes.POINTER(lrs_shape), _P, _P, _P, _P, _P, _P, _P, _P],
    "lrs_decay_head_means": [_P, ctypes.c_int64, ctypes.c_int32, ctypes.c_int64, _P, _P],
    "lrs_precision_map": [ctypes.c_int32, _P, ctypes.c_int32, _P],
    "lrs_sync": [_P],
    "lrs_debug_inject_timeout": [ctypes.c_int32, ctypes.c_int32],
    "lrs_debug_inject_timeout_after": [ctypes.c_int32, ctypes.c_int32],
}


def use_library(path):
    """Load another build of the library (e.g. the bounds-checked
    liblrs_checked.so) instead of liblrs.so; only before the first call."""
    global LIB_PATH
    if _lib is not None:
        raise RuntimeError("the library is already loaded from %s" % LIB_PATH)
    LIB_PATH = path


def lib():
    """The loaded liblrs.so (raises if it is missing: there is no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError("liblrs.so is not built (run quantized_recurrent_state_decode_b200"
                              ".build.build()): %s" % LIB_PATH)
        L = ctypes.CDLL(LIB_PATH)
        for name, args in _SIGS.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = ctypes.c_int
        L.lrs_last_error.restype = ctypes.c_char_p
        L.lrs_last_error.argtypes = []
        L.lrs_status_string.restype = ctypes.c_char_p
        L.lrs_status_string.argtypes = [ctypes.c_int]
        L.lrs_version.restype = ctypes.c_int32
        L.lrs_version.argtypes = []
        _lib = L
    return _lib


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, "data_ptr"):
        return x.data_ptr()
    if hasattr(x, "ctypes"):          # numpy array (host memory)
        return x.ctypes.data
    raise TypeError("cannot pass %r as a pointer" % type(x))


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(status):
    if status != LRS_OK:
        raise LrsError(status, lib().lrs_last_error().decode())


def shape(batch, heads, d_k, d_v, group, update_kind, gate_kind):
    return lrs_shape(batch, heads, d_k, d_v, group, update_kind, gate_kind)


def lrs_version():
    return lib().lrs_version()


def lrs_status_string(status):
    return lib().lrs_status_string(status).decode()


def lrs_last_error():
    return lib().lrs_last_error().decode()


def lrs_layout_query(shp, prec_map_host):
    """-> (head_offsets list, batch_stride_bytes, scale_count). Host only."""
    import numpy as np
    pm = np.ascontiguousarray(prec_map_host, dtype=np.uint8)
    offs = np.zeros(shp.heads, np.int64)
    stride = ctypes.c_int64()
    count = ctypes.c_int64()
    _check(lib().lrs_layout_query(ctypes.byref(shp), pm.ctypes.data, offs.ctypes.data,
                                  ctypes.addressof(stride), ctypes.addressof(count)))
    return offs, stride.value, count.value


def lrs_layout_query_groups(shp, prec_map_host):
    """prec_map_host [H][G] -> (head_offsets, batch_stride_bytes, scale_count). Host only."""
    import numpy as np
    pm = np.ascontiguousarray(prec_map_host, dtype=np.uint8)
    offs = np.zeros(shp.heads, np.int64)
    stride = ctypes.c_int64()
    count = ctypes.c_int64()
    _check(lib().lrs_layout_query_groups(ctypes.byref(shp), pm.ctypes.data, offs.ctypes.data,
                                         ctypes.addressof(stride), ctypes.addressof(count)))
    return offs, stride.value, count.value


def lrs_state_alloc(shp, prec_map_host):
    """prec_map_host [H]: one width per head; [H][G]: one per (head, scale group)
    (lrs_state_alloc_groups)."""
    import numpy as np
    pm = np.ascontiguousarray(prec_map_host, dtype=np.uint8)
    st = lrs_state()
    if pm.ndim == 2:
        if pm.shape != (shp.heads, shp.d_k // shp.group):
            raise ValueError("prec_map must be [H] or [H][d_k/group]")
        _check(lib().lrs_state_alloc_groups(ctypes.byref(shp), pm.ctypes.data, ctypes.byref(st)))
    else:
        _check(lib().lrs_state_alloc(ctypes.byref(shp), pm.ctypes.data, ctypes.byref(st)))
    return st


def lrs_state_free(st):
    _check(lib().lrs_state_free(ctypes.byref(st)))


def lrs_decode_step(st, state_codes, scales, prec_map, q, k, v, gates, beta, out, seed, step,
                    mode, stream=None):
    _check(lib().lrs_decode_step(ctypes.byref(st), _ptr(state_codes), _ptr(scales),
                                 _ptr(prec_map), _ptr(q), _ptr(k), _ptr(v), _ptr(gates),
                                 _ptr(beta), _ptr(out), seed, step, mode, _stream(stream)))


def lrs_decode_step_bf16(st, state_codes, scales, prec_map, q, k, v, gates, beta, out, seed,
                         step, mode, stream=None):
    """q, k, v, out: bfloat16 device buffers (torch.bfloat16 tensors or addresses)."""
    _check(lib().lrs_decode_step_bf16(ctypes.byref(st), _ptr(state_codes), _ptr(scales),
                                      _ptr(prec_map), _ptr(q), _ptr(k), _ptr(v), _ptr(gates),
                                      _ptr(beta), _ptr(out), seed, step, mode, _stream(stream)))


def lrs_chunk_step(st, state_codes, scales, prec_map, T, q, k, v, gates, beta, out, seed, step,
                   mode, stream=None):
    """T tokens per tile, one requantization at the end; inputs [T][B][H][...]."""
    _check(lib().lrs_chunk_step(ctypes.byref(st), _ptr(state_codes), _ptr(scales), _ptr(prec_map),
                                T, _ptr(q), _ptr(k), _ptr(v), _ptr(gates), _ptr(beta), _ptr(out),
                                seed, step, mode, _stream(stream)))


def lrs_lrb_step(st, state_codes, scales, prec_map, rank, U, V, q, k, v, gates, beta, out, seed,
                 step, mode, stream=None):
    """Decode step with a Low-Rank Bypass buffer U [B][H][rank][d_k], V [B][H][rank][d_v]."""
    _check(lib().lrs_lrb_step(ctypes.byref(st), _ptr(state_codes), _ptr(scales), _ptr(prec_map),
                              rank, _ptr(U), _ptr(V), _ptr(q), _ptr(k), _ptr(v), _ptr(gates),
                              _ptr(beta), _ptr(out), seed, step, mode, _stream(stream)))


def lrs_decode_step_host(st, q_host, k_host, v_host, gates_host, beta_host, out_host, seed, step,
                         mode, stream=None):
    _check(lib().lrs_decode_step_host(ctypes.byref(st), _ptr(q_host), _ptr(k_host),
                                      _ptr(v_host), _ptr(gates_host), _ptr(beta_host),
                                      _ptr(out_host), seed, step, mode, _stream(stream)))


def lrs_decode_step_host_noalloc(st, q_host, k_host, v_host, gates_host, beta_host, out_host,
                                 device_error_host, seed, step, mode, stream=None):
    _check(lib().lrs_decode_step_host_noalloc(
        ctypes.byref(st), _ptr(q_host), _ptr(k_host), _ptr(v_host), _ptr(gates_host),
        _ptr(beta_host), _ptr(out_host), _ptr(device_error_host), seed, step, mode,
        _stream(stream)))


def lrs_state_import_fp32(st, S, stream=None):
    _check(lib().lrs_state_import_fp32(ctypes.byref(st), _ptr(S), _stream(stream)))


def lrs_state_export_fp32(st, S, stream=None):
    _check(lib().lrs_state_export_fp32(ctypes.byref(st), _ptr(S), _stream(stream)))


def lrs_state_export_codes(st, codes, stream=None):
    _check(lib().lrs_state_export_codes(ctypes.byref(st), _ptr(codes), _stream(stream)))


def lrs_state_import_codes(st, codes, scales, stream=None):
    _check(lib().lrs_state_import_codes(ctypes.byref(st), _ptr(codes), _ptr(scales),
                                        _stream(stream)))


def lrs_state_copy_raw(st, codes_host, scales_host, to_host, stream=None):
    _check(lib().lrs_state_copy_raw(ctypes.byref(st), _ptr(codes_host), _ptr(scales_host),
                                    1 if to_host else 0, _stream(stream)))


def lrs_fp32_decode_step(shp, S, q, k, v, gates, beta, out, stream=None):
    _check(lib().lrs_fp32_decode_step(ctypes.byref(shp), _ptr(S), _ptr(q), _ptr(k), _ptr(v),
                                      _ptr(gates), _ptr(beta), _ptr(out), _stream(stream)))


def lrs_decay_head_means(decay, outer, heads, inner, means, stream=None):
    _check(lib().lrs_decay_head_means(_ptr(decay), outer, heads, inner, _ptr(means),
                                      _stream(stream)))


def lrs_precision_map(means_host, n_int8):
    import numpy as np
    m = np.ascontiguousarray(means_host, dtype=np.float64)
    pm = np.zeros(m.shape[0], np.uint8)
    _check(lib().lrs_precision_map(m.shape[0], m.ctypes.data, n_int8, pm.ctypes.data))
    return pm


def lrs_sync(stream=None):
    _check(lib().lrs_sync(_stream(stream)))


def lrs_debug_inject_timeout(enable, timeout_us=1000):
    _check(lib().lrs_debug_inject_timeout(1 if enable else 0, timeout_us))


def lrs_debug_inject_timeout_after(items_copied, timeout_us=1000):
    _check(lib().lrs_debug_inject_timeout_after(items_copied, timeout_us))
