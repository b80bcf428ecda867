"""The C-ABI library loads, exports every symbol include/*.h declares, and
rejects bad arguments before touching the GPU (CPU only: no kernel runs)."""
import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        names |= set(re.findall(r"SCONV_KV_API\s+[\w\s\*]*?\b(sconv_kv_\w+)\s*\(", text))
    return names


def test_header_declares_entry_points():
    names = declared_symbols()
    for must in ("sconv_kv_prefill_varlen", "sconv_kv_decode", "sconv_kv_cache_layout",
                 "sconv_kv_strerror"):
        assert must in names


def test_library_exports_all_declared():
    from short_conv_kv_b200 import binding
    lib = ctypes.CDLL(binding.LIB_PATH)
    missing = [n for n in declared_symbols() if not hasattr(lib, n)]
    assert not missing, missing


def test_strerror_and_version():
    from short_conv_kv_b200 import binding as b
    assert b.strerror(0) == "ok"
    for code in (-1, -2, -3, -4, -5):
        assert b.strerror(code) and b.strerror(code) != "unknown status"
    assert b.strerror(-99) == "unknown status"
    assert b.version() >= 100


def test_cache_layout():
    from short_conv_kv_b200 import binding as b
    lay = b.cache_layout(16, 16, 2, 64)
    assert (lay.stride_head, lay.stride_slot, lay.stride_page) == (64, 128, 2048)
    assert lay.bytes_per_cache == 16 * 2048 * 2
    with pytest.raises(b.SconvKVError) as e:
        b.cache_layout(4, 0, 2, 64)
    assert e.value.code == b.ERR_SHAPE
    assert b.lib.sconv_kv_cache_layout(1, 1, 1, 64, None) == b.ERR_NULL


def _call_prefill(b, **over):
    """Call the C entry point with fake (never dereferenced) device pointers;
    every case here is rejected on the host before any CUDA call, or is an
    empty call that enqueues nothing."""
    lay = b.cache_layout(16, 16, 2, 64)
    A = 0x10000  # 16-byte aligned fake address
    args = dict(k=A, v=A, row_stride=128, num_tokens=10, cu=A, num_seqs=1, wk=A, wv=A,
                gk=A, gv=A, eps=1e-6, W=4, H=2, D=64, state=A, sidx=None, pool=1,
                slots=A, kc=A, vc=A, layout=ctypes.byref(lay), err=None, stream=None)
    args.update(over)
    return b.lib.sconv_kv_prefill_varlen(*args.values())


def test_validation_codes_on_host():
    from short_conv_kv_b200 import binding as b
    assert _call_prefill(b, k=None) == b.ERR_NULL
    assert _call_prefill(b, cu=None) == b.ERR_NULL
    assert _call_prefill(b, state=None) == b.ERR_NULL          # W > 1 needs a state
    assert _call_prefill(b, layout=None) == b.ERR_NULL
    assert _call_prefill(b, W=0) == b.ERR_SHAPE
    assert _call_prefill(b, W=9) == b.ERR_SHAPE
    assert _call_prefill(b, D=96) == b.ERR_SHAPE
    assert _call_prefill(b, H=0) == b.ERR_SHAPE
    assert _call_prefill(b, row_stride=64) == b.ERR_SHAPE      # < Hkv*D
    assert _call_prefill(b, num_seqs=-1) == b.ERR_SHAPE
    assert _call_prefill(b, num_tokens=-1) == b.ERR_SHAPE
    assert _call_prefill(b, H=4) == b.ERR_SHAPE                # layout disagrees
    assert _call_prefill(b, k=0x10008) == b.ERR_ALIGN
    assert _call_prefill(b, kc=0x10002) == b.ERR_ALIGN
    assert _call_prefill(b, state=0x10004) == b.ERR_ALIGN
    assert _call_prefill(b, row_stride=132) == b.ERR_ALIGN
    lay = b.cache_layout(16, 16, 2, 64)
    lay.stride_slot = 132
    assert _call_prefill(b, layout=ctypes.byref(lay)) == b.ERR_ALIGN
    # empty calls enqueue nothing and succeed, whatever the pointers
    assert _call_prefill(b, num_tokens=0) == b.OK
    assert _call_prefill(b, num_seqs=0) == b.OK
    assert _call_prefill(b, num_tokens=0, k=None, v=None, slots=None, cu=None) == b.OK


def test_decode_validation_on_host():
    from short_conv_kv_b200 import binding as b
    lay = b.cache_layout(16, 16, 2, 64)
    A = 0x10000
    base = [A, A, 128, 4, A, A, A, A, 1e-6, 4, 2, 64, A, None, 4, A, A, A,
            ctypes.byref(lay), None, None]
    assert b.lib.sconv_kv_decode(*base[:3], 0, *base[4:]) == b.OK
    assert b.lib.sconv_kv_decode(*base[:3], -1, *base[4:]) == b.ERR_SHAPE
    bad = list(base)
    bad[9] = 0
    assert b.lib.sconv_kv_decode(*bad) == b.ERR_SHAPE
    bad = list(base)
    bad[0] = None
    assert b.lib.sconv_kv_decode(*bad) == b.ERR_NULL
    bad = list(base)
    bad[12] = None  # W = 4 needs a state
    assert b.lib.sconv_kv_decode(*bad) == b.ERR_NULL
    bad = list(base)
    bad[0], bad[1], bad[15] = None, None, None  # batch 0: pointers not examined
    assert b.lib.sconv_kv_decode(*bad[:3], 0, *bad[4:]) == b.OK


def test_binding_has_no_cpu_fallback():
    """The product module carries no CPU implementation of the step and does
    not import the oracle."""
    src = open(os.path.join(ROOT, "short_conv_kv_b200", "binding.py")).read()
    assert "oracle" not in src.replace("no CPU fallback", "")
    for name in ("rms_norm", "conv1d", "index_copy"):
        assert name not in src
