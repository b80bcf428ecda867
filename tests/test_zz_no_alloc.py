"""The no-alloc unfused step (intermediates in the library's static
scratch) against the unfused stage entry points with caller-allocated
intermediates: two calls in a row on different batches, each bit-identical
in caches and state; and a batch too large for the scratch is refused on
the host before anything is enqueued."""
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


def _run(b, noalloc):
    from short_conv_kv_b200 import binding as bd
    kc, vc = gu.dev(b.empty_cache()), gu.dev(b.empty_cache())
    st = gu.dev(b.conv_state.clone())
    args = (gu.dev(b.k), gu.dev(b.v), gu.dev(b.cu_seqlens), gu.dev(b.conv_w_k),
            gu.dev(b.conv_w_v), gu.dev(b.gamma_k), gu.dev(b.gamma_v), b.eps, st,
            gu.dev(b.slot_mapping), kc, vc)
    if noalloc:
        bd.unfused_step_noalloc(*args, state_indices=gu.dev(b.state_indices))
    else:
        y = torch.empty(b.num_tokens, 2 * b.C, dtype=torch.bfloat16, device="cuda")
        z = torch.empty_like(y)
        bd.prepare_unfused(*args, y, z, state_indices=gu.dev(b.state_indices))()
    torch.cuda.synchronize()
    return kc, vc, st


def test_noalloc_matches_stage_calls_twice():
    batches = [
        wl.make_prefill([300, 1, 0, 77, 2], Hkv=8, D=128, W=4, seed=2701, state="normal",
                        page_size=16, spare_pages=3),
        wl.make_prefill([8192], Hkv=8, D=128, W=4, seed=2702, state="zero", page_size=64,
                        spare_pages=1),
    ]
    for b in batches:  # two calls in a row through the one scratch buffer
        got = _run(b, noalloc=True)
        ref = _run(b, noalloc=False)
        for g, r in zip(got, ref):
            assert np.array_equal(wl.bits(g.cpu()), wl.bits(r.cpu()))


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
