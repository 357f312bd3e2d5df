"""numpy front end of the CPU oracle (oracle/lrs_oracle.c).

TEST INFRASTRUCTURE ONLY: imported by tests/, by the package's smoke check and
by the benchmark's CPU-baseline leg. The product library never imports it.

All arrays are C-contiguous numpy arrays in the oracle's logical layout
(one int8 code per element; see lrs_oracle.h). Functions that update the state
do so in place, like the library they are compared with.
"""
import ctypes
import os

import numpy as np

from . import build as _build

ROUND_RTN, ROUND_SR, ROUND_BDR = 0, 1, 2
UPDATE_GATED, UPDATE_DELTA = 0, 1
GATE_SCALAR, GATE_PER_KEY = 0, 1

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i32, i64, u32, u64 = ctypes.c_int, ctypes.c_int64, ctypes.c_uint32, ctypes.c_uint64
        L.orc_splitmix64.argtypes = [u64]
        L.orc_splitmix64.restype = u64
        L.orc_hash.argtypes = [u64, u64, u32, u32, u32, u32]
        L.orc_hash.restype = u64
        L.orc_uniform.argtypes = [u64]
        L.orc_uniform.restype = ctypes.c_float
        L.orc_step.argtypes = [i32, P, P, i32, i32, i32, i32, i32, i32, P, P, P, P, P, P, P, P,
                               P, u64, u64, i32]
        L.orc_step.restype = i32
        L.orc_chunk_step.argtypes = [i32, P, P, i32, i32, i32, i32, i32, i32, P, P, P, i32, P, P,
                                     P, P, P, P, u64, u64, i32]
        L.orc_chunk_step.restype = i32
        L.orc_step_pg.argtypes = L.orc_step.argtypes
        L.orc_step_pg.restype = i32
        L.orc_chunk_step_pg.argtypes = L.orc_chunk_step.argtypes
        L.orc_chunk_step_pg.restype = i32
        L.orc_lrb_step.argtypes = [i32, P, P, i32, i32, i32, i32, i32, i32, P, P, P, i32, P, P,
                                   P, P, P, P, P, P, u64, u64, P]
        L.orc_lrb_step.restype = i32
        L.orc_lrb_step_pg.argtypes = L.orc_lrb_step.argtypes
        L.orc_lrb_step_pg.restype = i32
        L.orc_bdr_additive_step.argtypes = [i32, i32, i32, i32, i32, P, P, P, P, P, P, P]
        L.orc_bdr_additive_step.restype = i32
        L.orc_bf16_rne.argtypes = [ctypes.c_float]
        L.orc_bf16_rne.restype = ctypes.c_uint16
        L.orc_bf16_rne_array.argtypes = [i64, P, P]
        L.orc_bf16_rne_array.restype = None
        L.orc_fp32_step.argtypes = [i32, i32, i32, i32, i32, P, P, P, P, P, P, P, i32]
        L.orc_fp32_step.restype = i32
        L.orc_import.argtypes = [i32, P, i32, i32, i32, P, P, P, P]
        L.orc_import.restype = i32
        L.orc_import_pg.argtypes = L.orc_import.argtypes
        L.orc_import_pg.restype = i32
        L.orc_dequant.argtypes = [i32, i32, i32, i32, P, P, P]
        L.orc_dequant.restype = i32
        L.orc_decay_means.argtypes = [i64, i32, i64, P, P]
        L.orc_decay_means.restype = None
        L.orc_precision_map.argtypes = [i32, P, i32, P]
        L.orc_precision_map.restype = i32
        _lib = L
    return _lib


def _p(a):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _f32(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float32)


def _per_group(prec_map, d_k, group, per_head_fn, per_group_fn):
    """prec_map [H] selects the per-head entry point, [H][d_k/group] the
    per-(head, group) one."""
    if prec_map.ndim == 1:
        return per_head_fn
    if prec_map.ndim != 2 or prec_map.shape[1] != d_k // group:
        raise ValueError("prec_map must be [H] or [H][d_k/group]")
    return per_group_fn


def splitmix64(z):
    return int(lib().orc_splitmix64(z & (2**64 - 1)))


def hash64(seed, step, b, h, i, j):
    return int(lib().orc_hash(seed, step, b, h, i, j))


def uniform(r):
    return float(lib().orc_uniform(r))


def default_threads():
    return os.cpu_count() or 1


def step(codes, scales, q, k, v, gates, beta, prec_map, tile_b, tile_h, *, group,
         update_kind, gate_kind, mode, seed=0, step=0, nthreads=1):
    """One quantized decode step for ntiles tiles; codes/scales updated in place.

    codes int8 [n][d_k][d_v]; scales f32 [n][G][d_v]; q, k [n][d_k]; v [n][d_v];
    gates [n][d_k] or [n]; beta [n] or None; prec_map u8 [H]; tile_b, tile_h [n].
    Returns out f32 [n][d_v].
    """
    n, d_k, d_v = codes.shape
    assert codes.dtype == np.int8 and scales.dtype == np.float32
    q, k, v, gates, beta = map(_f32, (q, k, v, gates, beta))
    prec_map = np.ascontiguousarray(prec_map, dtype=np.uint8)
    tile_b = np.ascontiguousarray(tile_b, dtype=np.int32)
    tile_h = np.ascontiguousarray(tile_h, dtype=np.int32)
    out = np.zeros((n, d_v), np.float32)
    fn = _per_group(prec_map, d_k, group, lib().orc_step, lib().orc_step_pg)
    rc = fn(n, _p(tile_b), _p(tile_h), d_k, d_v, group, update_kind, gate_kind, mode,
                        _p(prec_map), _p(codes), _p(scales), _p(q), _p(k), _p(v), _p(gates),
                        _p(beta), _p(out), seed, step, nthreads)
    if rc != 0:
        raise ValueError("orc_step rejected its arguments (%d)" % rc)
    return out


def chunk_step(codes, scales, q, k, v, gates, beta, prec_map, tile_b, tile_h, *, group,
               update_kind, gate_kind, mode, seed=0, step=0, nthreads=1):
    """T tokens per tile applied to the fp32 state, one requantization at the end.

    q, k [T][n][d_k]; v [T][n][d_v]; gates [T][n][d_k] or [T][n]; beta [T][n]
    or None; codes/scales as in step(), updated in place. Returns out f32
    [T][n][d_v].
    """
    n, d_k, d_v = codes.shape
    assert codes.dtype == np.int8 and scales.dtype == np.float32
    q, k, v, gates, beta = map(_f32, (q, k, v, gates, beta))
    T = q.shape[0]
    assert q.shape == (T, n, d_k) and k.shape == (T, n, d_k) and v.shape == (T, n, d_v)
    prec_map = np.ascontiguousarray(prec_map, dtype=np.uint8)
    tile_b = np.ascontiguousarray(tile_b, dtype=np.int32)
    tile_h = np.ascontiguousarray(tile_h, dtype=np.int32)
    out = np.zeros((T, n, d_v), np.float32)
    fn = _per_group(prec_map, d_k, group, lib().orc_chunk_step, lib().orc_chunk_step_pg)
    rc = fn(n, _p(tile_b), _p(tile_h), d_k, d_v, group, update_kind,
                              gate_kind, mode, _p(prec_map), _p(codes), _p(scales), T, _p(q),
                              _p(k), _p(v), _p(gates), _p(beta), _p(out), seed, step, nthreads)
    if rc != 0:
        raise ValueError("orc_chunk_step rejected its arguments (%d)" % rc)
    return out


def lrb_step(codes, scales, U, V, q, k, v, gates, beta, prec_map, tile_b, tile_h, *, group,
             update_kind, gate_kind, mode, rank, seed=0, step=0, want_x=False):
    """Decode step with Low-Rank Bypass; codes, scales, U [n][rank][d_k] and V
    [n][rank][d_v] (float32) updated in place. prec_map is [H] (per head) or
    [H][d_k/group] (per head and scale group). Returns out [n][d_v] (and the
    values before rounding [n][d_k][d_v] with want_x)."""
    n, d_k, d_v = codes.shape
    assert codes.dtype == np.int8 and scales.dtype == np.float32
    assert U.dtype == np.float32 and V.dtype == np.float32
    assert U.shape == (n, rank, d_k) and V.shape == (n, rank, d_v)
    q, k, v, gates, beta = map(_f32, (q, k, v, gates, beta))
    prec_map = np.ascontiguousarray(prec_map, dtype=np.uint8)
    tile_b = np.ascontiguousarray(tile_b, dtype=np.int32)
    tile_h = np.ascontiguousarray(tile_h, dtype=np.int32)
    out = np.zeros((n, d_v), np.float32)
    x = np.zeros((n, d_k, d_v), np.float32) if want_x else None
    fn = _per_group(prec_map, d_k, group, lib().orc_lrb_step, lib().orc_lrb_step_pg)
    rc = fn(n, _p(tile_b), _p(tile_h), d_k, d_v, group, update_kind, gate_kind, mode,
            _p(prec_map), _p(codes), _p(scales), rank, _p(U), _p(V), _p(q), _p(k), _p(v),
            _p(gates), _p(beta), _p(out), seed, step, _p(x))
    if rc != 0:
        raise ValueError("orc_lrb_step rejected its arguments (%d)" % rc)
    return (out, x) if want_x else out


def bf16_rne(x):
    """float32 array -> uint16 bfloat16 patterns, nearest with ties to even."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.zeros(x.shape, np.uint16)
    lib().orc_bf16_rne_array(x.size, _p(x), _p(out))
    return out


def bf16_to_f32(u):
    """uint16 bfloat16 patterns -> the float32 values they denote (exact)."""
    u = np.ascontiguousarray(u, dtype=np.uint16)
    return (u.astype(np.uint32) << 16).view(np.float32)


def fp32_step(S, q, k, v, gates, beta, *, update_kind, gate_kind, nthreads=1):
    """The same recurrence on an fp32 state S [n][d_k][d_v] (updated in place)."""
    n, d_k, d_v = S.shape
    assert S.dtype == np.float32
    q, k, v, gates, beta = map(_f32, (q, k, v, gates, beta))
    out = np.zeros((n, d_v), np.float32)
    rc = lib().orc_fp32_step(n, d_k, d_v, update_kind, gate_kind, _p(S), _p(q), _p(k), _p(v),
                             _p(gates), _p(beta), _p(out), nthreads)
    if rc != 0:
        raise ValueError("orc_fp32_step rejected its arguments (%d)" % rc)
    return out


def bdr_additive_step(codes, scales, q, k, v, gates, *, group, qmax):
    """Study of the other BDR reading (update = the additive term k_i w_j):
    one gated step with per-key gates, one width for all tiles; codes and
    scales updated in place. Returns out f32 [n][d_v]. Not a library step."""
    n, d_k, d_v = codes.shape
    assert codes.dtype == np.int8 and scales.dtype == np.float32
    q, k, v, gates = map(_f32, (q, k, v, gates))
    out = np.zeros((n, d_v), np.float32)
    rc = lib().orc_bdr_additive_step(n, d_k, d_v, group, qmax, _p(codes), _p(scales), _p(q),
                                     _p(k), _p(v), _p(gates), _p(out))
    if rc != 0:
        raise ValueError("orc_bdr_additive_step rejected its arguments (%d)" % rc)
    return out


def import_fp32(S0, prec_map, tile_h, *, group):
    """Round-to-nearest quantization of S0 [n][d_k][d_v] -> (codes, scales)."""
    S0 = _f32(S0)
    n, d_k, d_v = S0.shape
    prec_map = np.ascontiguousarray(prec_map, dtype=np.uint8)
    tile_h = np.ascontiguousarray(tile_h, dtype=np.int32)
    codes = np.zeros((n, d_k, d_v), np.int8)
    scales = np.zeros((n, d_k // group, d_v), np.float32)
    fn = _per_group(prec_map, d_k, group, lib().orc_import, lib().orc_import_pg)
    rc = fn(n, _p(tile_h), d_k, d_v, group, _p(prec_map), _p(S0), _p(codes),
                          _p(scales))
    if rc != 0:
        raise ValueError("orc_import rejected its arguments (%d)" % rc)
    return codes, scales


def dequant(codes, scales, *, group):
    n, d_k, d_v = codes.shape
    S = np.zeros((n, d_k, d_v), np.float32)
    rc = lib().orc_dequant(n, d_k, d_v, group, _p(np.ascontiguousarray(codes)),
                           _p(np.ascontiguousarray(scales, dtype=np.float32)), _p(S))
    if rc != 0:
        raise ValueError("orc_dequant rejected its arguments (%d)" % rc)
    return S


def decay_means(decay):
    """decay f32 [outer][H][inner] -> f64 [H]."""
    decay = _f32(decay)
    outer, H, inner = decay.shape
    means = np.zeros(H, np.float64)
    lib().orc_decay_means(outer, H, inner, _p(decay), _p(means))
    return means


def precision_map(means, n_int8):
    means = np.ascontiguousarray(means, dtype=np.float64)
    H = means.shape[0]
    pm = np.zeros(H, np.uint8)
    rc = lib().orc_precision_map(H, _p(means), n_int8, _p(pm))
    if rc != 0:
        raise ValueError("orc_precision_map rejected its arguments (%d)" % rc)
    return pm
