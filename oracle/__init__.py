"""Oracle for the fused ShortConv K/V step -- TEST INFRASTRUCTURE ONLY.

A thin ctypes/numpy front end over ``sconv_kv_oracle.c`` (plain double
precision loops, one step of the method per function; see that file's header
for the passages each step follows and the readings taken where the pages are
silent).  Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's
CPU-baseline leg may import this package.  It never touches the GPU and
shares nothing with the CUDA library.

Arrays are numpy: bf16 tensors travel as their uint16 bit patterns.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None

_u16p = ctypes.POINTER(ctypes.c_uint16)
_i32p = ctypes.POINTER(ctypes.c_int32)
_i64p = ctypes.POINTER(ctypes.c_int64)
_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)
_i64 = ctypes.c_int64
_int = ctypes.c_int

ERRORS = {
    0: "ok",
    -1: "bad argument",
    -2: "slot out of range",
    -3: "duplicate slot",
    -4: "state index out of range",
    -5: "cu_seqlens is not a partition of the tokens",
    -6: "out of memory",
}


class OracleError(RuntimeError):
    def __init__(self, code):
        super().__init__(f"oracle returned {code}: {ERRORS.get(code, '?')}")
        self.code = code


def load(path=None):
    """Load (building first if needed) the oracle library."""
    global _lib
    if path is None and _lib is not None:
        return _lib
    if path is None:
        if _build.needs_build():
            _build.build()
        path = _build.LIB
    lib = ctypes.CDLL(path)
    lib.oracle_conv.argtypes = [_u16p, _i64, _i64, _u16p, _i64, _u16p, _int,
                                _int, _f64p]
    lib.oracle_conv.restype = None
    lib.oracle_rmsnorm.argtypes = [_f64p, _i64, _int, _int, _f32p,
                                   ctypes.c_double, _f64p]
    lib.oracle_rmsnorm.restype = None
    lib.oracle_scatter.argtypes = [_f64p, _i64, _int, _int, _i64p, _i64, _i64,
                                   _i64, _i64, _i64, _u16p]
    lib.oracle_scatter.restype = _int
    lib.oracle_state_update.argtypes = [_u16p, _i64, _i64, _u16p, _i64, _int,
                                        _int]
    lib.oracle_state_update.restype = None
    common_tail = [_u16p, _i32p, _i64, _i64p, _u16p, _u16p, _i64, _i64, _i64,
                   _i64, _i64, _f64p, _f64p]
    lib.oracle_prefill_varlen.argtypes = (
        [_u16p, _u16p, _i64, _i64, _i32p, _int, _u16p, _u16p, _f32p, _f32p,
         ctypes.c_double, _int, _int, _int] + common_tail)
    lib.oracle_prefill_varlen.restype = _int
    lib.oracle_decode.argtypes = (
        [_u16p, _u16p, _i64, _int, _u16p, _u16p, _f32p, _f32p,
         ctypes.c_double, _int, _int, _int] + common_tail)
    lib.oracle_decode.restype = _int
    lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
    lib.oracle_bf16_to_double.restype = ctypes.c_double
    lib.oracle_double_to_bf16.argtypes = [ctypes.c_double]
    lib.oracle_double_to_bf16.restype = ctypes.c_uint16
    lib.oracle_round_bf16_array.argtypes = [_f64p, _i64, _u16p]
    lib.oracle_round_bf16_array.restype = None
    _u8p = ctypes.POINTER(ctypes.c_uint8)
    lib.oracle_double_to_e4m3.argtypes = [ctypes.c_double]
    lib.oracle_double_to_e4m3.restype = ctypes.c_uint8
    lib.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
    lib.oracle_e4m3_to_double.restype = ctypes.c_double
    lib.oracle_e4m3_array.argtypes = [_f64p, _i64, _u8p]
    lib.oracle_e4m3_array.restype = None
    lib.oracle_mx_block.argtypes = [_f32p, _int, _u8p, _u8p]
    lib.oracle_mx_block.restype = None
    lib.oracle_prefill_varlen_mxfp8.argtypes = (
        [_u16p, _u16p, _i64, _i64, _i32p, _int, _u16p, _u16p, _f32p, _f32p,
         ctypes.c_double, _int, _int, _int, _u16p, _i32p, _i64, _i64p,
         _u8p, _u8p, _u8p, _u8p, _i64, _i64, _i64, _i64, _i64, _f64p, _f64p])
    lib.oracle_prefill_varlen_mxfp8.restype = _int
    # layout variants: per-head gamma stride, ring-buffer state positions
    lib.oracle_rmsnorm_strided.argtypes = [_f64p, _i64, _int, _int, _f32p, _i64,
                                           ctypes.c_double, _f64p]
    lib.oracle_rmsnorm_strided.restype = None
    lib.oracle_state_update_ring.argtypes = [_u16p, _i64, _i64, _u16p, _i64, _int, _int, _i64]
    lib.oracle_state_update_ring.restype = None
    lib.oracle_prefill_varlen_opts.argtypes = (
        [_u16p, _u16p, _i64, _i64, _i32p, _int, _u16p, _u16p, _f32p, _f32p, _i64,
         ctypes.c_double, _int, _int, _int, _u16p, _i32p, _i64p, _i64, _i64p, _u16p, _u16p,
         _i64, _i64, _i64, _i64, _i64, _f64p, _f64p])
    lib.oracle_prefill_varlen_opts.restype = _int
    lib.oracle_decode_opts.argtypes = (
        [_u16p, _u16p, _i64, _int, _u16p, _u16p, _f32p, _f32p, _i64, ctypes.c_double, _int,
         _int, _int, _u16p, _i32p, _i64p, _i64, _i64p, _u16p, _u16p, _i64, _i64, _i64, _i64,
         _i64, _f64p, _f64p])
    lib.oracle_decode_opts.restype = _int
    lib.oracle_prefill_varlen_mxfp8_opts.argtypes = (
        [_u16p, _u16p, _i64, _i64, _i32p, _int, _u16p, _u16p, _f32p, _f32p, _i64,
         ctypes.c_double, _int, _int, _int, _u16p, _i32p, _i64p, _i64, _i64p,
         _u8p, _u8p, _u8p, _u8p, _i64, _i64, _i64, _i64, _i64, _f64p, _f64p])
    lib.oracle_prefill_varlen_mxfp8_opts.restype = _int
    if path == _build.LIB:
        _lib = lib
    return lib


def _p(a, ptype):
    if a is None:
        return ctypes.cast(None, ptype)
    assert a.flags["C_CONTIGUOUS"], "oracle wants C-contiguous arrays"
    return a.ctypes.data_as(ptype)


def _u16(a):
    a = np.asarray(a)
    if a.dtype != np.uint16:
        raise TypeError(f"expected uint16 bf16 bit patterns, got {a.dtype}")
    return np.ascontiguousarray(a)


# ---------------------------------------------------------------- bf16 bits

def bf16_bits_to_f64(bits):
    """Exact widening of bf16 bit patterns to float64."""
    bits = np.asarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def round_to_bf16_bits(x, lib=None):
    """Round float64 values to bf16 (nearest, ties to even), one rounding."""
    lib = lib or load()
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.uint16)
    lib.oracle_round_bf16_array(_p(x, _f64p), x.size, _p(out, _u16p))
    return out


# ---------------------------------------------------------------- stages

def conv(x, state, w, lib=None):
    """Step a1+a2 for one tensor of one sequence.

    x: uint16 [L, C]; state: uint16 [W-1, C] (old rows, oldest first);
    w: uint16 [W, C].  Returns float64 y [L, C].
    """
    lib = lib or load()
    x, w = _u16(x), _u16(w)
    W, C = w.shape
    L = x.shape[0]
    state = _u16(state) if W > 1 else np.zeros((1, C), np.uint16)
    y = np.empty((L, C), np.float64)
    lib.oracle_conv(_p(x, _u16p), C, L, _p(state, _u16p), C, _p(w, _u16p),
                    W, C, _p(y, _f64p))
    return y


def rmsnorm(y, num_heads, gamma, eps, lib=None):
    """Step a3: y float64 [L, H*D] -> z float64 [L, H*D]."""
    lib = lib or load()
    y = np.ascontiguousarray(y, dtype=np.float64)
    gamma = np.ascontiguousarray(gamma, dtype=np.float32)
    L = y.shape[0]
    D = gamma.shape[-1]
    z = np.empty_like(y)
    lib.oracle_rmsnorm_strided(_p(y, _f64p), L, num_heads, D, _p(gamma, _f32p),
                               D if gamma.ndim == 2 else 0, float(eps), _p(z, _f64p))
    return z


def scatter(z, num_heads, D, slots, cache, page_size, lib=None):
    """Step a4 into a contiguous [num_pages, page_size, H, D] uint16 cache
    (modified in place).  Returns the oracle status code."""
    lib = lib or load()
    z = np.ascontiguousarray(z, dtype=np.float64)
    slots = np.ascontiguousarray(slots, dtype=np.int64)
    assert cache.flags["C_CONTIGUOUS"] and cache.dtype == np.uint16
    num_pages = cache.shape[0]
    return lib.oracle_scatter(
        _p(z, _f64p), z.shape[0], num_heads, D, _p(slots, _i64p),
        num_pages * page_size, page_size, page_size * num_heads * D,
        num_heads * D, D, _p(cache, _u16p))


def state_update(x, state, lib=None):
    """Step a5 for one tensor of one sequence; returns the new state rows."""
    lib = lib or load()
    x = _u16(x)
    s = _u16(state).copy()
    n, C = s.shape
    lib.oracle_state_update(_p(x, _u16p), C, x.shape[0], _p(s, _u16p), C, C,
                            n + 1)
    return s


def _gammas(gamma_k, gamma_v, H):
    """float32 gammas and their head stride: [D] (shared by every head,
    stride 0) or [H, D] (one per head, stride D)."""
    gk = np.ascontiguousarray(gamma_k, dtype=np.float32)
    gv = np.ascontiguousarray(gamma_v, dtype=np.float32)
    assert gk.shape == gv.shape and gk.ndim in (1, 2)
    if gk.ndim == 2:
        assert gk.shape[0] == H
        return gk, gv, gk.shape[1]
    return gk, gv, 0


def _positions(state_positions):
    return None if state_positions is None else np.ascontiguousarray(state_positions, np.int64)


def state_update_ring(x, state, pos0, lib=None):
    """Step a5 with a ring-buffer state (position p in row p mod (W-1)) for
    one tensor of one sequence that has seen pos0 tokens; returns the new
    state rows."""
    lib = lib or load()
    x = _u16(x)
    s = _u16(state).copy()
    n, C = s.shape
    lib.oracle_state_update_ring(_p(x, _u16p), C, x.shape[0], _p(s, _u16p), C, C, n + 1,
                                 int(pos0))
    return s


# ---------------------------------------------------------------- whole step

def prefill_varlen(k, v, cu_seqlens, conv_w_k, conv_w_v, gamma_k, gamma_v,
                   eps, conv_state, slot_mapping, k_cache, v_cache,
                   state_indices=None, want_z=True, check=True, lib=None,
                   state_positions=None):
    """The whole step (a1..a5) over a varlen batch.

    k, v: uint16 [T, H, D] (or [T, C]); cu_seqlens int32 [S+1];
    conv_w_*: uint16 [W, C]; gamma_*: float32 [D] (shared by every head) or
    [H, D] (per head); conv_state: uint16 [pool, W-1, 2C], oldest row first,
    or, with state_positions (int64 [S], tokens each sequence has seen), a
    ring in which position p lives in row p mod (W-1); slot_mapping int64
    [T]; caches uint16 [num_pages, page_size, H, D].  Inputs are not
    modified: returns dict(k_cache, v_cache, conv_state, z_k, z_v, status)
    with fresh arrays.
    """
    lib = lib or load()
    k, v = _u16(k), _u16(v)
    T = k.shape[0]
    num_pages, page_size, H, D = k_cache.shape
    C = H * D
    k2, v2 = k.reshape(T, C), v.reshape(T, C)
    wk, wv = _u16(conv_w_k), _u16(conv_w_v)
    W = wk.shape[0]
    gk, gv, ghs = _gammas(gamma_k, gamma_v, H)
    pos = _positions(state_positions)
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    S = cu.shape[0] - 1
    st = _u16(conv_state).copy()
    pool = st.shape[0]
    sm = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    kc, vc = _u16(k_cache).copy(), _u16(v_cache).copy()
    si = None if state_indices is None else np.ascontiguousarray(
        state_indices, dtype=np.int32)
    zk = np.zeros((T, C), np.float64) if want_z else None
    zv = np.zeros((T, C), np.float64) if want_z else None
    rc = lib.oracle_prefill_varlen_opts(
        _p(k2, _u16p), _p(v2, _u16p), C, T, _p(cu, _i32p), S,
        _p(wk, _u16p), _p(wv, _u16p), _p(gk, _f32p), _p(gv, _f32p), ghs,
        float(eps), W, H, D, _p(st if W > 1 else None, _u16p),
        _p(si, _i32p), _p(pos, _i64p), pool, _p(sm, _i64p), _p(kc, _u16p), _p(vc, _u16p),
        num_pages, page_size, page_size * C, C, D, _p(zk, _f64p),
        _p(zv, _f64p))
    if check and rc != 0:
        raise OracleError(rc)
    return dict(k_cache=kc, v_cache=vc, conv_state=st, z_k=zk, z_v=zv,
                status=rc)


def decode(k, v, conv_w_k, conv_w_v, gamma_k, gamma_v, eps, conv_state,
           slot_mapping, k_cache, v_cache, state_indices=None, want_z=True,
           check=True, lib=None, state_positions=None):
    """One decode step: one new token per sequence (k, v: [B, H, D])."""
    B = np.asarray(k).shape[0]
    cu = np.arange(B + 1, dtype=np.int32)
    return prefill_varlen(k, v, cu, conv_w_k, conv_w_v, gamma_k, gamma_v, eps,
                          conv_state, slot_mapping, k_cache, v_cache,
                          state_indices=state_indices, want_z=want_z,
                          check=check, lib=lib, state_positions=state_positions)


def decode_direct(k, v, conv_w_k, conv_w_v, gamma_k, gamma_v, eps,
                  conv_state, slot_mapping, k_cache, v_cache,
                  state_indices=None, lib=None, state_positions=None):
    """Decode through the C entry point oracle_decode (same semantics as
    decode(); kept so both entry points are exercised)."""
    lib = lib or load()
    k, v = _u16(k), _u16(v)
    B = k.shape[0]
    num_pages, page_size, H, D = k_cache.shape
    C = H * D
    k2, v2 = k.reshape(B, C), v.reshape(B, C)
    wk, wv = _u16(conv_w_k), _u16(conv_w_v)
    W = wk.shape[0]
    gk, gv, ghs = _gammas(gamma_k, gamma_v, H)
    pos = _positions(state_positions)
    st = _u16(conv_state).copy()
    sm = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    kc, vc = _u16(k_cache).copy(), _u16(v_cache).copy()
    si = None if state_indices is None else np.ascontiguousarray(
        state_indices, dtype=np.int32)
    zk = np.zeros((B, C), np.float64)
    zv = np.zeros((B, C), np.float64)
    rc = lib.oracle_decode_opts(
        _p(k2, _u16p), _p(v2, _u16p), C, B, _p(wk, _u16p), _p(wv, _u16p),
        _p(gk, _f32p), _p(gv, _f32p), ghs, float(eps), W, H, D,
        _p(st if W > 1 else None, _u16p), _p(si, _i32p), _p(pos, _i64p), st.shape[0],
        _p(sm, _i64p), _p(kc, _u16p), _p(vc, _u16p), num_pages, page_size,
        page_size * C, C, D, _p(zk, _f64p), _p(zv, _f64p))
    if rc != 0:
        raise OracleError(rc)
    return dict(k_cache=kc, v_cache=vc, conv_state=st, z_k=zk, z_v=zv,
                status=rc)


# ---------------------------------------------------------------- MXFP8 store

def e4m3_from_f64(x, lib=None):
    """FP8 E4M3 codes (nearest even, saturating at +-448) of float64 values."""
    lib = lib or load()
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(x.shape, np.uint8)
    lib.oracle_e4m3_array(_p(x, _f64p), x.size,
                          out.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)))
    return out


def e4m3_to_f64(codes, lib=None):
    lib = lib or load()
    c = np.asarray(codes, dtype=np.uint8)
    return np.array([lib.oracle_e4m3_to_double(int(t)) for t in c.reshape(-1)],
                    dtype=np.float64).reshape(c.shape)


def mx_block(values_f32, lib=None):
    """Quantise one block of float32 values -> (codes uint8[n], scale uint8)."""
    lib = lib or load()
    v = np.ascontiguousarray(values_f32, dtype=np.float32)
    codes = np.zeros(v.shape[0], np.uint8)
    scale = np.zeros(1, np.uint8)
    _u8p = ctypes.POINTER(ctypes.c_uint8)
    lib.oracle_mx_block(_p(v, _f32p), v.shape[0], codes.ctypes.data_as(_u8p),
                        scale.ctypes.data_as(_u8p))
    return codes, int(scale[0])


def prefill_varlen_mxfp8(k, v, cu_seqlens, conv_w_k, conv_w_v, gamma_k, gamma_v,
                         eps, conv_state, slot_mapping, num_pages, page_size,
                         state_indices=None, check=True, lib=None, state_positions=None):
    """The step with the MXFP8 store into dense caches: data uint8
    [num_pages, page_size, H, D], scales uint8 [num_pages, page_size, H, D/32]
    (fresh, zero-filled).  Returns dict(k_data, k_scale, v_data, v_scale,
    conv_state, z_k, z_v, status)."""
    lib = lib or load()
    k, v = _u16(k), _u16(v)
    T = k.shape[0]
    wk, wv = _u16(conv_w_k), _u16(conv_w_v)
    W, C = wk.shape
    D = np.asarray(gamma_k).shape[-1]
    H = C // D
    gk, gv, ghs = _gammas(gamma_k, gamma_v, H)
    pos = _positions(state_positions)
    k2, v2 = k.reshape(T, C), v.reshape(T, C)
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    S = cu.shape[0] - 1
    st = _u16(conv_state).copy()
    sm = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    si = None if state_indices is None else np.ascontiguousarray(state_indices, dtype=np.int32)
    kd = np.zeros((num_pages, page_size, H, D), np.uint8)
    vd = np.zeros_like(kd)
    ks = np.zeros((num_pages, page_size, H, D // 32), np.uint8)
    vs = np.zeros_like(ks)
    zk = np.zeros((T, C), np.float64)
    zv = np.zeros((T, C), np.float64)
    _u8p = ctypes.POINTER(ctypes.c_uint8)
    rc = lib.oracle_prefill_varlen_mxfp8_opts(
        _p(k2, _u16p), _p(v2, _u16p), C, T, _p(cu, _i32p), S, _p(wk, _u16p),
        _p(wv, _u16p), _p(gk, _f32p), _p(gv, _f32p), ghs, float(eps), W, H, D,
        _p(st if W > 1 else None, _u16p), _p(si, _i32p), _p(pos, _i64p), st.shape[0],
        _p(sm, _i64p), kd.ctypes.data_as(_u8p), ks.ctypes.data_as(_u8p),
        vd.ctypes.data_as(_u8p), vs.ctypes.data_as(_u8p), num_pages, page_size,
        page_size * C, C, D, _p(zk, _f64p), _p(zv, _f64p))
    if check and rc != 0:
        raise OracleError(rc)
    return dict(k_data=kd, k_scale=ks, v_data=vd, v_scale=vs, conv_state=st,
                z_k=zk, z_v=zv, status=rc)
