"""Failure detection without a GPU fault: the kernels' pipeline waits are
bounded.  With the first copy withheld (a wait on something nothing
completes) and a 100 us limit, every CTA's first wait runs out: the kernel
lets the copies it did issue land, sets SCONV_KV_FLAG_TIMEOUT and returns,
and the context stays usable for the next calls."""
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


def _timed_out(call):
    from short_conv_kv_b200 import binding as bd
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    call(err)
    torch.cuda.synchronize()
    return bool(int(err.item()) & bd.FLAG_TIMEOUT)


def test_prefill_wait_timeout_sets_flag_and_context_survives():
    from short_conv_kv_b200 import binding as bd
    b = wl.single()
    k, v, cu = gu.dev(b.k), gu.dev(b.v), gu.dev(b.cu_seqlens)
    w = [gu.dev(x) for x in (b.conv_w_k, b.conv_w_v, b.gamma_k, b.gamma_v)]
    sm = gu.dev(b.slot_mapping)

    def call(err):
        kc, vc = gu.dev(b.empty_cache()), gu.dev(b.empty_cache())
        st = gu.dev(b.conv_state.clone())
        bd.prefill_varlen(k, v, cu, *w, b.eps, st, sm, kc, vc, err_flag=err, wait_timeout_ns=100_000,
                          withhold_first_copy=True)

    assert _timed_out(call)
    # the next calls run normally and match the oracle
    gu.full_parity(wl.tiny())
    gu.full_parity(wl.make_prefill([300, 7], Hkv=8, D=128, W=4, seed=2901, state="normal",
                                   page_size=16, spare_pages=1))


@pytest.mark.parametrize("early", [False, True])
def test_decode_wait_timeout_sets_flag_and_context_survives(early):
    """(early: with the independent-state promise, whose CTAs request their
    state rows before the dependency wait.)"""
    from short_conv_kv_b200 import binding as bd
    s = wl.decode(seed=2910)
    k, v, sm = s.step_inputs(0)
    k, v, sm = gu.dev(k), gu.dev(v), gu.dev(sm)
    w = [gu.dev(x) for x in (s.conv_w_k, s.conv_w_v, s.gamma_k, s.gamma_v)]

    def call(err):
        kc, vc = gu.dev(s.empty_cache()), gu.dev(s.empty_cache())
        st = gu.dev(s.conv_state.clone())
        bd.decode(k, v, *w, s.eps, st, sm, kc, vc, err_flag=err, wait_timeout_ns=100_000,
                  withhold_first_copy=True, independent_state=early)

    assert _timed_out(call)
    # a normal decode step right after: state bit-exact, no flag
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = gu.dev(s.conv_state.clone())
    kc, vc = gu.dev(s.empty_cache()), gu.dev(s.empty_cache())
    bd.decode(k, v, *w, s.eps, st, sm, kc, vc, err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    exp = gu.expected_final_state(wl.bits(s.step_inputs(0)[0]).reshape(s.batch, -1),
                                  wl.bits(s.step_inputs(0)[1]).reshape(s.batch, -1),
                                  np.arange(s.batch + 1), wl.bits(s.conv_state), s.W)
    assert np.array_equal(wl.bits(st.cpu()), exp)
