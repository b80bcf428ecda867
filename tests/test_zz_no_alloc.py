"""The no-alloc unfused step (sconv_kv_unfused_step_noalloc: y and z in the
library's static device scratch) against the unfused stage entry points with
caller-allocated intermediates.

Some callers cannot allocate device memory at the point where they run the
step (an allocator that is locked, or memory pools sized in advance), so
this entry point takes only inputs and outputs.  Every case is run twice in
a row through the one shared scratch buffer; caches, state and flags must be
bit-identical to the stage calls'.  Also: W=1 with head_dim 64 (no state
at all), a sequence with a bad state index (its cache slots stay untouched,
as in the fused step), and a batch too large for the scratch, refused on the
host before anything is enqueued."""
import numpy as np
import pytest
import torch

from short_conv_kv_b200 import workloads as wl
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield
    torch.cuda.synchronize()


def _run(b, path):
    """Caches, state and flag word after one step through `path`:
    'noalloc', 'stages' (the four stage calls) or 'fused'."""
    from short_conv_kv_b200 import binding as bd
    kc, vc = gu.dev(b.empty_cache()), gu.dev(b.empty_cache())
    st = gu.dev(b.conv_state.clone())
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    args = (gu.dev(b.k), gu.dev(b.v), gu.dev(b.cu_seqlens), gu.dev(b.conv_w_k),
            gu.dev(b.conv_w_v), gu.dev(b.gamma_k), gu.dev(b.gamma_v), b.eps, st,
            gu.dev(b.slot_mapping), kc, vc)
    si = gu.dev(b.state_indices)
    if path == "noalloc":
        bd.unfused_step_noalloc(*args, state_indices=si, err_flag=err)
    elif path == "stages":
        y = torch.empty(b.num_tokens, 2 * b.C, dtype=torch.bfloat16, device="cuda")
        z = torch.empty_like(y)
        bd.prepare_unfused(*args, y, z, state_indices=si, err_flag=err)()
    else:
        bd.prefill_varlen(*args, state_indices=si, err_flag=err)
    torch.cuda.synchronize()
    return wl.bits(kc.cpu()), wl.bits(vc.cpu()), wl.bits(st.cpu()), int(err.item())


def _same(b):
    for _ in range(2):  # two calls in a row through the one scratch buffer
        got = _run(b, "noalloc")
        ref = _run(b, "stages")
        for g, r in zip(got[:3], ref[:3]):
            assert np.array_equal(g, r)
        assert got[3] == ref[3]
    return got


def test_noalloc_matches_stage_calls_twice():
    batches = [
        wl.make_prefill([300, 1, 0, 77, 2], Hkv=8, D=128, W=4, seed=2701, state="normal",
                        page_size=16, spare_pages=3),
        wl.make_prefill([8192], Hkv=8, D=128, W=4, seed=2702, state="zero", page_size=64,
                        spare_pages=1),
    ]
    for b in batches:
        assert _same(b)[3] == 0


def test_noalloc_w1_head_dim_64():
    b = wl.make_prefill([129, 3, 64], Hkv=4, D=64, W=1, seed=2704, state="zero", page_size=16,
                        spare_pages=2)
    assert _same(b)[3] == 0


def test_noalloc_bad_state_index_leaves_slots_untouched():
    from short_conv_kv_b200 import binding as bd
    b = wl.make_prefill([40, 17, 90], Hkv=2, D=128, W=4, seed=2705, state="normal",
                        page_size=16, spare_pages=2, pool_size=4, state_indices=[3, 9, 0])
    kc, vc, st, err = _same(b)
    assert err & bd.FLAG_STATE_INDEX
    # the fused step skips the same sequence: the same slots stay untouched
    fk, fv, fst, ferr = _run(b, "fused")
    assert ferr & bd.FLAG_STATE_INDEX
    sent = np.uint16(wl.SENTINEL_BITS)
    for got, fused in ((kc, fk), (vc, fv)):
        g, f = got.reshape(-1, b.C), fused.reshape(-1, b.C)
        assert np.array_equal(np.all(g == sent, axis=1), np.all(f == sent, axis=1))
        bad = b.slot_mapping.numpy()[40:57]
        assert np.all(g[bad] == sent)
    assert np.array_equal(st, fst)


def test_noalloc_refuses_oversize_batch():
    from short_conv_kv_b200 import binding as bd
    H, D = 8, 128
    T = bd.NOALLOC_SCRATCH_BYTES // (2 * 2 * H * D * 2) + 1  # one token too many
    b = wl.make_prefill([T], Hkv=H, D=D, W=4, seed=2703, state="zero", page_size=64)
    kc = gu.dev(b.empty_cache())
    with pytest.raises(bd.SconvKVError) as e:
        bd.unfused_step_noalloc(gu.dev(b.k), gu.dev(b.v), gu.dev(b.cu_seqlens),
                                gu.dev(b.conv_w_k), gu.dev(b.conv_w_v), gu.dev(b.gamma_k),
                                gu.dev(b.gamma_v), b.eps, gu.dev(b.conv_state),
                                gu.dev(b.slot_mapping), kc, kc.clone())
    assert e.value.code == bd.ERR_SCRATCH
