"""ctypes front end of ``libsconvkv.so`` (the fused ShortConv K/V step).

Argument marshalling only: every function takes torch tensors, passes their
device pointers, sizes and the current CUDA stream to the C ABI declared in
``include/sconv_kv.h``, and raises on a non-zero status.  All of the step's
work runs in the library's CUDA kernels; there is no CPU fallback, and if the
library is missing the import fails loudly.
"""
import ctypes
import os

import torch

from . import build as _build

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("SCONV_KV_LIB", _build.LIB)

# status codes and device flag bits (values fixed by include/sconv_kv.h)
OK = 0
ERR_NULL, ERR_SHAPE, ERR_ALIGN, ERR_UNSUPPORTED, ERR_CUDA, ERR_SCRATCH = -1, -2, -3, -4, -5, -6
NOALLOC_SCRATCH_BYTES = 64 << 20
FLAG_SLOT_RANGE, FLAG_STATE_INDEX, FLAG_CU_SEQLENS, FLAG_TIMEOUT = 1, 2, 4, 8
MAX_W = 8


class CacheLayout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in (
        "num_pages", "page_size", "num_kv_heads", "head_dim", "stride_page",
        "stride_slot", "stride_head", "bytes_per_cache")]


class Options(ctypes.Structure):
    """sconv_kv_options_t: per-head gamma stride and ring-state positions."""
    _fields_ = [("gamma_head_stride", ctypes.c_int64), ("state_positions", ctypes.c_void_p),
                ("wait_timeout_ns", ctypes.c_int64), ("withhold_first_copy", ctypes.c_int64),
                ("state_only_dependency", ctypes.c_int64), ("independent_state", ctypes.c_int64)]


class SconvKVError(RuntimeError):
    def __init__(self, code, where):
        msg = _lib.sconv_kv_strerror(code).decode()
        if code == ERR_CUDA:
            msg += ": " + _lib.sconv_kv_last_cuda_error().decode()
        super().__init__(f"{where} failed with status {code}: {msg}")
        self.code = code


def _load(path):
    if not os.path.exists(path):
        raise ImportError(
            f"CUDA library {path} is not built; run `python -m short_conv_kv_b200.build` "
            "(there is no CPU fallback)")
    lib = ctypes.CDLL(path)
    vp, i64, i32, f32, ip = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int,
                             ctypes.c_float, ctypes.c_void_p)
    lp = ctypes.POINTER(CacheLayout)
    lib.sconv_kv_cache_layout.argtypes = [i64, i64, i32, i32, lp]
    lib.sconv_kv_cache_layout.restype = i32
    lib.sconv_kv_prefill_varlen.argtypes = [
        vp, vp, i64, i64, vp, i32, vp, vp, vp, vp, f32, i32, i32, i32, vp, vp,
        i64, vp, vp, vp, lp, ip, vp]
    lib.sconv_kv_prefill_varlen.restype = i32
    lib.sconv_kv_decode.argtypes = [
        vp, vp, i64, i32, vp, vp, vp, vp, f32, i32, i32, i32, vp, vp, i64, vp,
        vp, vp, lp, ip, vp]
    lib.sconv_kv_decode.restype = i32
    lib.sconv_kv_prefill_varlen_mxfp8.argtypes = [
        vp, vp, i64, i64, vp, i32, vp, vp, vp, vp, f32, i32, i32, i32, vp, vp,
        i64, vp, vp, vp, vp, vp, lp, ip, vp]
    lib.sconv_kv_prefill_varlen_mxfp8.restype = i32
    lib.sconv_kv_decode_mxfp8.argtypes = [
        vp, vp, i64, i32, vp, vp, vp, vp, f32, i32, i32, i32, vp, vp, i64, vp,
        vp, vp, vp, vp, lp, ip, vp]
    lib.sconv_kv_decode_mxfp8.restype = i32
    op = ctypes.POINTER(Options)
    lib.sconv_kv_prefill_varlen_ex.argtypes = [
        vp, vp, i64, i64, vp, i32, vp, vp, vp, vp, f32, i32, i32, i32, vp, vp,
        i64, vp, vp, vp, lp, op, ip, vp]
    lib.sconv_kv_prefill_varlen_ex.restype = i32
    lib.sconv_kv_decode_ex.argtypes = [
        vp, vp, i64, i32, vp, vp, vp, vp, f32, i32, i32, i32, vp, vp, i64, vp,
        vp, vp, lp, op, ip, vp]
    lib.sconv_kv_decode_ex.restype = i32
    lib.sconv_kv_prefill_varlen_mxfp8_ex.argtypes = [
        vp, vp, i64, i64, vp, i32, vp, vp, vp, vp, f32, i32, i32, i32, vp, vp,
        i64, vp, vp, vp, vp, vp, lp, op, ip, vp]
    lib.sconv_kv_prefill_varlen_mxfp8_ex.restype = i32
    lib.sconv_kv_decode_mxfp8_ex.argtypes = [
        vp, vp, i64, i32, vp, vp, vp, vp, f32, i32, i32, i32, vp, vp, i64, vp,
        vp, vp, vp, vp, lp, op, ip, vp]
    lib.sconv_kv_decode_mxfp8_ex.restype = i32
    lib.sconv_kv_stage_conv.argtypes = [
        vp, vp, i64, i64, vp, i32, vp, vp, i32, i32, i32, vp, vp, i64, vp, ip, vp]
    lib.sconv_kv_stage_conv.restype = i32
    lib.sconv_kv_stage_rmsnorm.argtypes = [vp, i64, vp, vp, f32, i32, i32, vp, vp]
    lib.sconv_kv_stage_rmsnorm.restype = i32
    lib.sconv_kv_stage_scatter.argtypes = [vp, i64, i32, i32, vp, vp, vp, lp, vp, i32, i32,
                                           vp, i64, ip, vp]
    lib.sconv_kv_stage_scatter.restype = i32
    lib.sconv_kv_stage_state_update.argtypes = [
        vp, vp, i64, i64, vp, i32, i32, i32, i32, vp, vp, i64, ip, vp]
    lib.sconv_kv_stage_state_update.restype = i32
    lib.sconv_kv_unfused_step_noalloc.argtypes = [
        vp, vp, i64, i64, vp, i32, vp, vp, vp, vp, f32, i32, i32, i32, vp, vp,
        i64, vp, vp, vp, lp, ip, vp]
    lib.sconv_kv_unfused_step_noalloc.restype = i32
    lib.sconv_kv_strerror.argtypes = [i32]
    lib.sconv_kv_strerror.restype = ctypes.c_char_p
    lib.sconv_kv_last_cuda_error.argtypes = []
    lib.sconv_kv_last_cuda_error.restype = ctypes.c_char_p
    lib.sconv_kv_version.argtypes = []
    lib.sconv_kv_version.restype = i32
    return lib


_lib = _load(LIB_PATH)
lib = _lib


def strerror(code):
    return _lib.sconv_kv_strerror(int(code)).decode()


def version():
    return _lib.sconv_kv_version()


def cache_layout(num_pages, page_size, num_kv_heads, head_dim):
    """Dense [num_pages, page_size, Hkv, D] layout (sconv_kv_cache_layout)."""
    out = CacheLayout()
    rc = _lib.sconv_kv_cache_layout(int(num_pages), int(page_size),
                                    int(num_kv_heads), int(head_dim),
                                    ctypes.byref(out))
    if rc != OK:
        raise SconvKVError(rc, "sconv_kv_cache_layout")
    return out


def layout_of(cache):
    """Layout of a 4-D cache view [num_pages, page_size, Hkv, D] with unit
    dim stride (e.g. the k or v half of a combined per-page KV buffer)."""
    if cache.dim() != 4 or cache.stride(3) != 1:
        raise ValueError("cache must be [num_pages, page_size, Hkv, D] with dim stride 1")
    P, S, H, D = cache.shape
    lay = CacheLayout()
    lay.num_pages, lay.page_size, lay.num_kv_heads, lay.head_dim = P, S, H, D
    lay.stride_page, lay.stride_slot, lay.stride_head = cache.stride(0), cache.stride(1), cache.stride(2)
    lay.bytes_per_cache = cache.untyped_storage().nbytes()
    return lay


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _options(gamma_k, state_positions, wait_timeout_ns=None, withhold_first_copy=False,
             state_only_dependency=False, independent_state=False):
    """Options struct for the _ex entry points, or None for the defaults
    (gamma [D] shared by every head, linear state, 1 s wait limit, every
    CTA waiting for the previous kernel).  gamma [Hkv, D] selects per-head
    gammas; state_positions (int64 [S] on the device) a ring state;
    wait_timeout_ns the kernels' wait limit; state_only_dependency the
    caller's promise that the previous kernel on the stream writes none of
    this call's inputs but conv_state; independent_state (decode) the
    promise that it writes none of them but k and v (see
    include/sconv_kv.h)."""
    per_head = gamma_k is not None and gamma_k.dim() == 2
    if not per_head and state_positions is None and not wait_timeout_ns and \
            not withhold_first_copy and not state_only_dependency and not independent_state:
        return None
    if state_positions is not None and state_positions.dtype != torch.int64:
        raise TypeError("state_positions must be int64")
    o = Options()
    o.gamma_head_stride = gamma_k.shape[-1] if per_head else 0
    o.state_positions = _ptr(state_positions)
    o.wait_timeout_ns = int(wait_timeout_ns or 0)
    o.withhold_first_copy = 1 if withhold_first_copy else 0
    o.state_only_dependency = 1 if state_only_dependency else 0
    o.independent_state = 1 if independent_state else 0
    return o


def _rows(x, name):
    """(pointer, row_stride) of a [T, Hkv, D] or [T, Hkv*D] bf16 view whose
    channels are contiguous."""
    if x.dtype != torch.bfloat16:
        raise TypeError(f"{name} must be bfloat16")
    if x.dim() == 3:
        if x.stride(2) != 1 or x.stride(1) != x.shape[2]:
            raise ValueError(f"{name}: heads and head_dim must be contiguous")
    elif x.dim() != 2 or x.stride(1) != 1:
        raise ValueError(f"{name} must be [T, Hkv, D] or [T, Hkv*D]")
    C = x[0].numel() if x.shape[0] else x.shape[-1] * (x.shape[1] if x.dim() == 3 else 1)
    return x.data_ptr(), max(x.stride(0), C)


def prefill_varlen(k, v, cu_seqlens, conv_w_k, conv_w_v, gamma_k, gamma_v,
                   eps, conv_state, slot_mapping, k_cache, v_cache,
                   state_indices=None, err_flag=None, stream=None,
                   layout=None, state_positions=None, wait_timeout_ns=None,
                   withhold_first_copy=False, state_only_dependency=False):
    """Fused ShortConv K/V step over a packed varlen batch, on the GPU.

    k, v: bf16 [T, Hkv, D] (rows may be strided slices); cu_seqlens int32
    [S+1]; conv_w_*: bf16 [W, Hkv*D]; gamma_*: fp32 [D]; conv_state bf16
    [pool, W-1, 2*Hkv*D] (updated in place); slot_mapping int64 [T];
    k_cache / v_cache bf16 [num_pages, page_size, Hkv, D] (written in
    place); state_indices optional int32 [S]; err_flag optional int32 [1].
    """
    kp, rs = _rows(k, "k")
    vp, rs_v = _rows(v, "v")
    if rs != rs_v:
        raise ValueError("k and v must share the row stride")
    T = k.shape[0]
    W = conv_w_k.shape[0]
    H, D = k_cache.shape[2], k_cache.shape[3]
    lay = layout if layout is not None else layout_of(k_cache)
    if v_cache.stride() != k_cache.stride() or v_cache.shape != k_cache.shape:
        raise ValueError("k_cache and v_cache must have the same shape and strides")
    pool = conv_state.shape[0] if conv_state is not None else 0
    args = (kp, vp, rs, T, _ptr(cu_seqlens), cu_seqlens.shape[0] - 1,
            _ptr(conv_w_k), _ptr(conv_w_v), _ptr(gamma_k), _ptr(gamma_v),
            float(eps), W, H, D, _ptr(conv_state) if W > 1 else None,
            _ptr(state_indices), pool, _ptr(slot_mapping), _ptr(k_cache),
            _ptr(v_cache), ctypes.byref(lay))
    opts = _options(gamma_k, state_positions, wait_timeout_ns, withhold_first_copy,
                    state_only_dependency)
    if opts is None:
        rc = _lib.sconv_kv_prefill_varlen(*args, _ptr(err_flag), _stream(stream))
    else:
        rc = _lib.sconv_kv_prefill_varlen_ex(*args, ctypes.byref(opts), _ptr(err_flag),
                                             _stream(stream))
    if rc != OK:
        raise SconvKVError(rc, "sconv_kv_prefill_varlen")


def decode(k, v, conv_w_k, conv_w_v, gamma_k, gamma_v, eps, conv_state,
           slot_mapping, k_cache, v_cache, state_indices=None, err_flag=None,
           stream=None, layout=None, state_positions=None, wait_timeout_ns=None,
           withhold_first_copy=False, independent_state=False):
    """Fused ShortConv K/V decode step: one new token per sequence
    (k, v: bf16 [B, Hkv, D]); same other arguments as prefill_varlen."""
    kp, rs = _rows(k, "k")
    vp, rs_v = _rows(v, "v")
    if rs != rs_v:
        raise ValueError("k and v must share the row stride")
    B = k.shape[0]
    W = conv_w_k.shape[0]
    H, D = k_cache.shape[2], k_cache.shape[3]
    lay = layout if layout is not None else layout_of(k_cache)
    pool = conv_state.shape[0] if conv_state is not None else 0
    args = (kp, vp, rs, B, _ptr(conv_w_k), _ptr(conv_w_v), _ptr(gamma_k),
            _ptr(gamma_v), float(eps), W, H, D,
            _ptr(conv_state) if W > 1 else None, _ptr(state_indices), pool,
            _ptr(slot_mapping), _ptr(k_cache), _ptr(v_cache), ctypes.byref(lay))
    opts = _options(gamma_k, state_positions, wait_timeout_ns, withhold_first_copy,
                    independent_state=independent_state)
    if opts is None:
        rc = _lib.sconv_kv_decode(*args, _ptr(err_flag), _stream(stream))
    else:
        rc = _lib.sconv_kv_decode_ex(*args, ctypes.byref(opts), _ptr(err_flag), _stream(stream))
    if rc != OK:
        raise SconvKVError(rc, "sconv_kv_decode")


def _mx_layout(k_data, k_scale, v_data, v_scale):
    """Layout of MXFP8 caches: data uint8 [num_pages, page_size, Hkv, D]
    (unit dim stride), scales uint8 [num_pages, page_size, Hkv, D/32] whose
    strides are the data strides / 32."""
    for t, n in ((k_data, "k_data"), (v_data, "v_data"), (k_scale, "k_scale"), (v_scale, "v_scale")):
        if t.dtype != torch.uint8:
            raise TypeError(f"{n} must be uint8")
    lay = layout_of(k_data)
    if v_data.stride() != k_data.stride() or v_data.shape != k_data.shape:
        raise ValueError("k_data and v_data must have the same shape and strides")
    P, S, H, D = k_data.shape
    want = (P, S, H, D // 32)
    for sc in (k_scale, v_scale):
        if tuple(sc.shape) != want or sc.stride(3) != 1 or any(
                sc.stride(i) * 32 != k_data.stride(i) for i in range(3)):
            raise ValueError("scale caches must be [num_pages, page_size, Hkv, D/32] with "
                             "strides equal to the data strides / 32")
    return lay


def prefill_varlen_mxfp8(k, v, cu_seqlens, conv_w_k, conv_w_v, gamma_k, gamma_v,
                         eps, conv_state, slot_mapping, k_data, k_scale, v_data, v_scale,
                         state_indices=None, err_flag=None, stream=None, state_positions=None,
                         state_only_dependency=False):
    """The fused step with the block-scaled MXFP8 cache store (E4M3 codes in
    k_data/v_data, one E8M0 scale byte per 32 channels in k_scale/v_scale)."""
    kp, rs = _rows(k, "k")
    vp, rs_v = _rows(v, "v")
    if rs != rs_v:
        raise ValueError("k and v must share the row stride")
    lay = _mx_layout(k_data, k_scale, v_data, v_scale)
    W = conv_w_k.shape[0]
    H, D = k_data.shape[2], k_data.shape[3]
    pool = conv_state.shape[0] if conv_state is not None else 0
    args = (kp, vp, rs, k.shape[0], _ptr(cu_seqlens), cu_seqlens.shape[0] - 1,
            _ptr(conv_w_k), _ptr(conv_w_v), _ptr(gamma_k), _ptr(gamma_v), float(eps), W, H, D,
            _ptr(conv_state) if W > 1 else None, _ptr(state_indices), pool, _ptr(slot_mapping),
            _ptr(k_data), _ptr(k_scale), _ptr(v_data), _ptr(v_scale), ctypes.byref(lay))
    opts = _options(gamma_k, state_positions, state_only_dependency=state_only_dependency)
    if opts is None:
        rc = _lib.sconv_kv_prefill_varlen_mxfp8(*args, _ptr(err_flag), _stream(stream))
    else:
        rc = _lib.sconv_kv_prefill_varlen_mxfp8_ex(*args, ctypes.byref(opts), _ptr(err_flag),
                                                   _stream(stream))
    if rc != OK:
        raise SconvKVError(rc, "sconv_kv_prefill_varlen_mxfp8")


def decode_mxfp8(k, v, conv_w_k, conv_w_v, gamma_k, gamma_v, eps, conv_state,
                 slot_mapping, k_data, k_scale, v_data, v_scale, state_indices=None,
                 err_flag=None, stream=None, state_positions=None, independent_state=False):
    """Decode step with the MXFP8 cache store (one new token per sequence)."""
    kp, rs = _rows(k, "k")
    vp, rs_v = _rows(v, "v")
    if rs != rs_v:
        raise ValueError("k and v must share the row stride")
    lay = _mx_layout(k_data, k_scale, v_data, v_scale)
    W = conv_w_k.shape[0]
    H, D = k_data.shape[2], k_data.shape[3]
    pool = conv_state.shape[0] if conv_state is not None else 0
    args = (kp, vp, rs, k.shape[0], _ptr(conv_w_k), _ptr(conv_w_v), _ptr(gamma_k),
            _ptr(gamma_v), float(eps), W, H, D, _ptr(conv_state) if W > 1 else None,
            _ptr(state_indices), pool, _ptr(slot_mapping), _ptr(k_data), _ptr(k_scale),
            _ptr(v_data), _ptr(v_scale), ctypes.byref(lay))
    opts = _options(gamma_k, state_positions, independent_state=independent_state)
    if opts is None:
        rc = _lib.sconv_kv_decode_mxfp8(*args, _ptr(err_flag), _stream(stream))
    else:
        rc = _lib.sconv_kv_decode_mxfp8_ex(*args, ctypes.byref(opts), _ptr(err_flag),
                                           _stream(stream))
    if rc != OK:
        raise SconvKVError(rc, "sconv_kv_decode_mxfp8")


class PreparedCall:
    """A pre-marshalled C-ABI call (for tight launch loops and graph
    capture): the ctypes argument tuple is built once; `__call__` only
    invokes the C entry point and checks the status."""

    def __init__(self, fn_name, args, keep_alive=()):
        self._fn = getattr(_lib, fn_name)
        self._args = tuple(args)
        self._keep = keep_alive
        self._name = fn_name

    def __call__(self):
        rc = self._fn(*self._args)
        if rc != OK:
            raise SconvKVError(rc, self._name)


def prepare_prefill_varlen(k, v, cu_seqlens, conv_w_k, conv_w_v, gamma_k,
                           gamma_v, eps, conv_state, slot_mapping, k_cache,
                           v_cache, state_indices=None, err_flag=None,
                           stream=None, state_only_dependency=False):
    kp, rs = _rows(k, "k")
    vp, _ = _rows(v, "v")
    W = conv_w_k.shape[0]
    H, D = k_cache.shape[2], k_cache.shape[3]
    lay = layout_of(k_cache)
    pool = conv_state.shape[0] if conv_state is not None else 0
    head = (kp, vp, rs, k.shape[0], _ptr(cu_seqlens), cu_seqlens.shape[0] - 1,
            _ptr(conv_w_k), _ptr(conv_w_v), _ptr(gamma_k), _ptr(gamma_v),
            ctypes.c_float(eps), W, H, D,
            _ptr(conv_state) if W > 1 else None, _ptr(state_indices), pool,
            _ptr(slot_mapping), _ptr(k_cache), _ptr(v_cache), ctypes.byref(lay))
    opts = _options(gamma_k, None, state_only_dependency=state_only_dependency)
    if opts is None:
        return PreparedCall("sconv_kv_prefill_varlen", head + (_ptr(err_flag), _stream(stream)),
                            keep_alive=(lay,))
    return PreparedCall("sconv_kv_prefill_varlen_ex",
                        head + (ctypes.byref(opts), _ptr(err_flag), _stream(stream)),
                        keep_alive=(lay, opts))


def prepare_decode(k, v, conv_w_k, conv_w_v, gamma_k, gamma_v, eps,
                   conv_state, slot_mapping, k_cache, v_cache,
                   state_indices=None, err_flag=None, stream=None, state_positions=None,
                   independent_state=False):
    kp, rs = _rows(k, "k")
    vp, _ = _rows(v, "v")
    W = conv_w_k.shape[0]
    H, D = k_cache.shape[2], k_cache.shape[3]
    lay = layout_of(k_cache)
    pool = conv_state.shape[0] if conv_state is not None else 0
    opts = _options(gamma_k, state_positions, independent_state=independent_state)
    head = (kp, vp, rs, k.shape[0], _ptr(conv_w_k), _ptr(conv_w_v),
            _ptr(gamma_k), _ptr(gamma_v), ctypes.c_float(eps), W, H, D,
            _ptr(conv_state) if W > 1 else None, _ptr(state_indices), pool,
            _ptr(slot_mapping), _ptr(k_cache), _ptr(v_cache), ctypes.byref(lay))
    if opts is None:
        return PreparedCall("sconv_kv_decode", head + (_ptr(err_flag), _stream(stream)),
                            keep_alive=(lay,))
    return PreparedCall("sconv_kv_decode_ex",
                        head + (ctypes.byref(opts), _ptr(err_flag), _stream(stream)),
                        keep_alive=(lay, opts))


def prepare_prefill_varlen_mxfp8(k, v, cu_seqlens, conv_w_k, conv_w_v, gamma_k, gamma_v,
                                 eps, conv_state, slot_mapping, k_data, k_scale, v_data,
                                 v_scale, state_indices=None, err_flag=None, stream=None,
                                 state_only_dependency=False):
    kp, rs = _rows(k, "k")
    vp, _ = _rows(v, "v")
    lay = _mx_layout(k_data, k_scale, v_data, v_scale)
    W = conv_w_k.shape[0]
    H, D = k_data.shape[2], k_data.shape[3]
    pool = conv_state.shape[0] if conv_state is not None else 0
    head = (kp, vp, rs, k.shape[0], _ptr(cu_seqlens), cu_seqlens.shape[0] - 1,
            _ptr(conv_w_k), _ptr(conv_w_v), _ptr(gamma_k), _ptr(gamma_v),
            ctypes.c_float(eps), W, H, D, _ptr(conv_state) if W > 1 else None,
            _ptr(state_indices), pool, _ptr(slot_mapping), _ptr(k_data), _ptr(k_scale),
            _ptr(v_data), _ptr(v_scale), ctypes.byref(lay))
    opts = _options(gamma_k, None, state_only_dependency=state_only_dependency)
    if opts is None:
        return PreparedCall("sconv_kv_prefill_varlen_mxfp8",
                            head + (_ptr(err_flag), _stream(stream)), keep_alive=(lay,))
    return PreparedCall("sconv_kv_prefill_varlen_mxfp8_ex",
                        head + (ctypes.byref(opts), _ptr(err_flag), _stream(stream)),
                        keep_alive=(lay, opts))


def prepare_decode_mxfp8(k, v, conv_w_k, conv_w_v, gamma_k, gamma_v, eps, conv_state,
                         slot_mapping, k_data, k_scale, v_data, v_scale, state_indices=None,
                         err_flag=None, stream=None, independent_state=False):
    kp, rs = _rows(k, "k")
    vp, _ = _rows(v, "v")
    lay = _mx_layout(k_data, k_scale, v_data, v_scale)
    W = conv_w_k.shape[0]
    H, D = k_data.shape[2], k_data.shape[3]
    pool = conv_state.shape[0] if conv_state is not None else 0
    head = (kp, vp, rs, k.shape[0], _ptr(conv_w_k), _ptr(conv_w_v), _ptr(gamma_k),
            _ptr(gamma_v), ctypes.c_float(eps), W, H, D,
            _ptr(conv_state) if W > 1 else None, _ptr(state_indices), pool,
            _ptr(slot_mapping), _ptr(k_data), _ptr(k_scale), _ptr(v_data), _ptr(v_scale),
            ctypes.byref(lay))
    opts = _options(gamma_k, None, independent_state=independent_state)
    if opts is None:
        return PreparedCall("sconv_kv_decode_mxfp8", head + (_ptr(err_flag), _stream(stream)),
                            keep_alive=(lay,))
    return PreparedCall("sconv_kv_decode_mxfp8_ex",
                        head + (ctypes.byref(opts), _ptr(err_flag), _stream(stream)),
                        keep_alive=(lay, opts))


# ---------------------------------------------------------------- unfused stages

def _check(rc, name):
    if rc != OK:
        raise SconvKVError(rc, name)


def stage_conv(k, v, cu_seqlens, conv_w_k, conv_w_v, conv_state, y, state_indices=None,
               err_flag=None, stream=None):
    """Pass 1 of the unfused chain: y (bf16 [T, 2*Hkv*D], K then V) = the
    causal conv of k and v; conv_state is only read."""
    kp, rs = _rows(k, "k")
    vp, rs_v = _rows(v, "v")
    if rs != rs_v:
        raise ValueError("k and v must share the row stride")
    W = conv_w_k.shape[0]
    H, D = (k.shape[1], k.shape[2]) if k.dim() == 3 else (None, None)
    if H is None:
        raise ValueError("k must be [T, Hkv, D] for the stage entry points")
    pool = conv_state.shape[0] if conv_state is not None else 0
    _check(_lib.sconv_kv_stage_conv(
        kp, vp, rs, k.shape[0], _ptr(cu_seqlens), cu_seqlens.shape[0] - 1, _ptr(conv_w_k),
        _ptr(conv_w_v), W, H, D, _ptr(conv_state) if W > 1 else None, _ptr(state_indices),
        pool, _ptr(y), _ptr(err_flag), _stream(stream)), "sconv_kv_stage_conv")


def stage_rmsnorm(y, gamma_k, gamma_v, eps, num_kv_heads, z, stream=None):
    """Pass 2: z = per-head RMSNorm of y times gamma (bf16 [T, 2*Hkv*D])."""
    D = gamma_k.shape[0]
    _check(_lib.sconv_kv_stage_rmsnorm(_ptr(y), y.shape[0], _ptr(gamma_k), _ptr(gamma_v),
                                       float(eps), int(num_kv_heads), D, _ptr(z),
                                       _stream(stream)), "sconv_kv_stage_rmsnorm")


def stage_scatter(z, slot_mapping, k_cache, v_cache, err_flag=None, stream=None,
                  cu_seqlens=None, W=1, state_indices=None, state_pool_size=0):
    """Pass 3: cache[slot_mapping[t]] = z[t] (K half / V half).  With
    cu_seqlens, the tokens of sequences the other stages skip (malformed
    cu_seqlens entry; for W > 1 a state index outside the pool) are not
    written."""
    lay = layout_of(k_cache)
    H, D = k_cache.shape[2], k_cache.shape[3]
    S = cu_seqlens.shape[0] - 1 if cu_seqlens is not None else 0
    _check(_lib.sconv_kv_stage_scatter(_ptr(z), z.shape[0], H, D, _ptr(slot_mapping),
                                       _ptr(k_cache), _ptr(v_cache), ctypes.byref(lay),
                                       _ptr(cu_seqlens), S, int(W), _ptr(state_indices),
                                       int(state_pool_size), _ptr(err_flag), _stream(stream)),
           "sconv_kv_stage_scatter")


def stage_state_update(k, v, cu_seqlens, W, conv_state, state_indices=None, err_flag=None,
                       stream=None):
    """Pass 4: conv_state <- last W-1 raw rows of (old state ++ rows), in place."""
    kp, rs = _rows(k, "k")
    vp, _ = _rows(v, "v")
    H, D = k.shape[1], k.shape[2]
    pool = conv_state.shape[0] if conv_state is not None else 0
    _check(_lib.sconv_kv_stage_state_update(
        kp, vp, rs, k.shape[0], _ptr(cu_seqlens), cu_seqlens.shape[0] - 1, int(W), H, D,
        _ptr(conv_state) if W > 1 else None, _ptr(state_indices), pool, _ptr(err_flag),
        _stream(stream)), "sconv_kv_stage_state_update")


def prepare_unfused(k, v, cu_seqlens, conv_w_k, conv_w_v, gamma_k, gamma_v, eps, conv_state,
                    slot_mapping, k_cache, v_cache, y, z, state_indices=None, err_flag=None,
                    stream=None):
    """The four stage calls of one step, pre-marshalled (conv, rmsnorm,
    scatter, state update, in that order on one stream)."""
    kp, rs = _rows(k, "k")
    vp, _ = _rows(v, "v")
    W = conv_w_k.shape[0]
    T, H, D = k.shape[0], k.shape[1], k.shape[2]
    S = cu_seqlens.shape[0] - 1
    pool = conv_state.shape[0] if conv_state is not None else 0
    st = _ptr(conv_state) if W > 1 else None
    lay = layout_of(k_cache)
    sp = _stream(stream)
    calls = [
        PreparedCall("sconv_kv_stage_conv", (kp, vp, rs, T, _ptr(cu_seqlens), S, _ptr(conv_w_k),
                                             _ptr(conv_w_v), W, H, D, st, _ptr(state_indices),
                                             pool, _ptr(y), _ptr(err_flag), sp)),
        PreparedCall("sconv_kv_stage_rmsnorm", (_ptr(y), T, _ptr(gamma_k), _ptr(gamma_v),
                                                ctypes.c_float(eps), H, D, _ptr(z), sp)),
        PreparedCall("sconv_kv_stage_scatter", (_ptr(z), T, H, D, _ptr(slot_mapping),
                                                _ptr(k_cache), _ptr(v_cache), ctypes.byref(lay),
                                                _ptr(cu_seqlens), S, W, _ptr(state_indices), pool,
                                                _ptr(err_flag), sp), keep_alive=(lay,)),
        PreparedCall("sconv_kv_stage_state_update", (kp, vp, rs, T, _ptr(cu_seqlens), S, W, H, D,
                                                     st, _ptr(state_indices), pool,
                                                     _ptr(err_flag), sp)),
    ]

    def run():
        for c in calls:
            c()
    return run


def unfused_step_noalloc(k, v, cu_seqlens, conv_w_k, conv_w_v, gamma_k, gamma_v, eps,
                         conv_state, slot_mapping, k_cache, v_cache, state_indices=None,
                         err_flag=None, stream=None):
    """The four unfused stages in one call, intermediates in the library's
    static scratch (no allocation); same arguments as prefill_varlen.
    Raises SconvKVError with code ERR_SCRATCH when the batch needs more than
    NOALLOC_SCRATCH_BYTES of scratch."""
    kp, rs = _rows(k, "k")
    vp, rs_v = _rows(v, "v")
    if rs != rs_v:
        raise ValueError("k and v must share the row stride")
    W = conv_w_k.shape[0]
    H, D = k_cache.shape[2], k_cache.shape[3]
    lay = layout_of(k_cache)
    pool = conv_state.shape[0] if conv_state is not None else 0
    _check(_lib.sconv_kv_unfused_step_noalloc(
        kp, vp, rs, k.shape[0], _ptr(cu_seqlens), cu_seqlens.shape[0] - 1, _ptr(conv_w_k),
        _ptr(conv_w_v), _ptr(gamma_k), _ptr(gamma_v), float(eps), W, H, D,
        _ptr(conv_state) if W > 1 else None, _ptr(state_indices), pool, _ptr(slot_mapping),
        _ptr(k_cache), _ptr(v_cache), ctypes.byref(lay), _ptr(err_flag), _stream(stream)),
        "sconv_kv_unfused_step_noalloc")
