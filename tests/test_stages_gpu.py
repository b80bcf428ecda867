"""GPU parity of the unfused stages (conv, rmsnorm, scatter, state update)
against the oracle's per-stage functions, and of the four-stage chain
against the oracle's whole step."""
import numpy as np
import pytest
import torch

import oracle
from short_conv_kv_b200 import workloads as wl
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield
    torch.cuda.synchronize()


def _bd():
    from short_conv_kv_b200 import binding
    return binding


def _state_rows(b, i):
    si = i if b.state_indices is None else int(b.state_indices[i])
    return wl.bits(b.conv_state)[si]  # [W-1, 2C]


def oracle_y(b):
    """Per-sequence oracle conv of K and V: float64 [T, 2C]."""
    C, W = b.C, b.W
    kb = wl.bits(b.k).reshape(-1, C)
    vb = wl.bits(b.v).reshape(-1, C)
    cu = b.cu_seqlens.numpy()
    y = np.zeros((b.num_tokens, 2 * C))
    for i in range(b.num_seqs):
        a, e = int(cu[i]), int(cu[i + 1])
        if e == a:
            continue
        st = _state_rows(b, i) if W > 1 else np.zeros((1, 2 * C), np.uint16)
        y[a:e, :C] = oracle.conv(kb[a:e], st[:, :C], wl.bits(b.conv_w_k))
        y[a:e, C:] = oracle.conv(vb[a:e], st[:, C:], wl.bits(b.conv_w_v))
    return y


def run_conv(b):
    bd = _bd()
    y = torch.empty(b.num_tokens, 2 * b.C, dtype=torch.bfloat16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    bd.stage_conv(gu.dev(b.k), gu.dev(b.v), gu.dev(b.cu_seqlens), gu.dev(b.conv_w_k),
                  gu.dev(b.conv_w_v), gu.dev(b.conv_state), y,
                  state_indices=gu.dev(b.state_indices), err_flag=err)
    torch.cuda.synchronize()
    return y, int(err.item())


@pytest.mark.parametrize("W", [1, 2, 4, 8])
def test_stage_conv(W):
    b = wl.make_prefill([300, 1, 0, 77, 2, 9], Hkv=4, D=128, W=W, seed=2600 + W, state="normal",
                        page_size=16, spare_pages=2)
    y, err = run_conv(b)
    assert err == 0
    gu.assert_close(wl.bits(y.cpu()), oracle_y(b), f"y W={W}")


def test_stage_conv_state_indices():
    b = wl.make_prefill([0, 1, 2, 3, 40, 1], Hkv=2, D=64, W=4, seed=2611, state="normal",
                        page_size=8, spare_pages=1, pool_size=9,
                        state_indices=[8, 3, 0, 7, 5, 1])
    y, err = run_conv(b)
    assert err == 0
    gu.assert_close(wl.bits(y.cpu()), oracle_y(b), "y state_indices")


@pytest.mark.parametrize("Hkv,D", [(2, 64), (8, 128), (3, 256)])
def test_stage_rmsnorm(Hkv, D):
    bd = _bd()
    g = torch.Generator().manual_seed(2620 + D)
    T, C = 203, Hkv * D
    y = (torch.randn(T, 2 * C, generator=g) * 2).to(torch.bfloat16)
    gk = 1 + 0.1 * torch.randn(D, generator=g)
    gv = 1 + 0.1 * torch.randn(D, generator=g)
    z = torch.empty_like(y, device="cuda")
    bd.stage_rmsnorm(gu.dev(y), gu.dev(gk), gu.dev(gv), 1e-6, Hkv, z)
    torch.cuda.synchronize()
    yd = gu.f64(wl.bits(y))
    ref = np.concatenate([oracle.rmsnorm(yd[:, :C], Hkv, gk.numpy(), 1e-6),
                          oracle.rmsnorm(yd[:, C:], Hkv, gv.numpy(), 1e-6)], axis=1)
    gu.assert_close(wl.bits(z.cpu()), ref, f"z Hkv={Hkv} D={D}")


def test_stage_scatter_bitwise():
    bd = _bd()
    b = wl.make_prefill([37, 64, 5], Hkv=2, D=64, W=4, seed=2630, state="zero", page_size=16,
                        spare_pages=3)
    g = torch.Generator().manual_seed(2631)
    z = torch.randn(b.num_tokens, 2 * b.C, generator=g).to(torch.bfloat16)
    sm = b.slot_mapping.clone()
    sm[4] = -1
    kc, vc = gu.dev(b.empty_cache()), gu.dev(b.empty_cache())
    bd.stage_scatter(gu.dev(z), gu.dev(sm), kc, vc)
    torch.cuda.synchronize()
    zd = gu.f64(wl.bits(z))
    for half, cache in ((slice(0, b.C), kc), (slice(b.C, 2 * b.C), vc)):
        ref = wl.bits(b.empty_cache()).copy()
        assert oracle.scatter(zd[:, half], b.Hkv, b.D, sm.numpy(), ref, b.page_size) == 0
        assert np.array_equal(wl.bits(cache.cpu()), ref)


def test_stage_scatter_flags_range():
    bd = _bd()
    b = wl.tiny()
    z = torch.zeros(b.num_tokens, 2 * b.C, dtype=torch.bfloat16, device="cuda")
    sm = b.slot_mapping.clone()
    sm[0] = b.num_pages * b.page_size  # one past the cache
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    kc, vc = gu.dev(b.empty_cache()), gu.dev(b.empty_cache())
    bd.stage_scatter(z, gu.dev(sm), kc, vc, err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) & bd.FLAG_SLOT_RANGE


@pytest.mark.parametrize("W", [2, 4, 8])
def test_stage_state_update(W):
    bd = _bd()
    b = wl.make_prefill([0, 1, 2, 3, 9, 50], Hkv=2, D=128, W=W, seed=2640 + W, state="normal",
                        page_size=16, spare_pages=1, pool_size=8,
                        state_indices=[7, 0, 3, 5, 1, 6])
    st = gu.dev(b.conv_state.clone())
    bd.stage_state_update(gu.dev(b.k), gu.dev(b.v), gu.dev(b.cu_seqlens), W, st,
                          state_indices=gu.dev(b.state_indices))
    torch.cuda.synchronize()
    exp = gu.expected_final_state(wl.bits(b.k).reshape(-1, b.C), wl.bits(b.v).reshape(-1, b.C),
                                  b.cu_seqlens.numpy(),
                                  wl.bits(b.conv_state), W, b.state_indices.numpy())
    assert np.array_equal(wl.bits(st.cpu()), exp)


@pytest.mark.parametrize("lengths,W", [([37, 64], 4), ([300, 1, 0, 77, 2], 2), ([8192], 4)])
def test_unfused_chain_matches_oracle(lengths, W):
    """Conv -> rmsnorm -> scatter -> state update equals the oracle's whole
    step within the stated bound (|err| <= max(2e-2, 1e-2*|z|)); y's bf16
    rounding between the passes makes the exact-rounding check inapplicable.
    Placement, untouched slots and the state are bit-exact."""
    bd = _bd()
    H, D = (8, 128) if lengths == [8192] else (4, 64)
    b = wl.make_prefill(lengths, Hkv=H, D=D, W=W, seed=2650 + W, state="normal", page_size=16,
                        spare_pages=2)
    kc, vc = gu.dev(b.empty_cache()), gu.dev(b.empty_cache())
    st = gu.dev(b.conv_state.clone())
    y = torch.empty(b.num_tokens, 2 * b.C, dtype=torch.bfloat16, device="cuda")
    z = torch.empty_like(y)
    run = bd.prepare_unfused(gu.dev(b.k), gu.dev(b.v), gu.dev(b.cu_seqlens), gu.dev(b.conv_w_k),
                             gu.dev(b.conv_w_v), gu.dev(b.gamma_k), gu.dev(b.gamma_v), b.eps, st,
                             gu.dev(b.slot_mapping), kc, vc, y, z)
    run()
    torch.cuda.synchronize()
    ref = gu.oracle_prefill(b)
    sm = b.slot_mapping.numpy()
    for which, cache, oc, zz in (("k", kc, ref["k_cache"], ref["z_k"]),
                                 ("v", vc, ref["v_cache"], ref["z_v"])):
        g = wl.bits(cache.cpu()).reshape(-1, b.C)
        o = oc.reshape(-1, b.C)
        written = np.zeros(g.shape[0], bool)
        written[sm[sm >= 0]] = True
        assert np.array_equal(g[~written], o[~written]), which
        got = gu.f64(g[sm])
        zz = np.asarray(zz).reshape(-1, b.C)
        err = np.abs(got - zz)
        assert (err <= np.maximum(gu.ABS_TOL, gu.REL_TOL * np.abs(zz))).all(), (which, err.max())
    assert np.array_equal(wl.bits(st.cpu()), ref["conv_state"])


def test_stage_scatter_skips_flagged_sequences():
    """Given cu_seqlens, scatter leaves the slots of a sequence with a bad
    state index (W > 1) untouched, as the fused step does; without it,
    every token is written."""
    bd = _bd()
    b = wl.make_prefill([20, 33, 11], Hkv=2, D=64, W=4, seed=2660, state="zero", page_size=16,
                        spare_pages=2, pool_size=3, state_indices=[0, 7, 2])
    g = torch.Generator().manual_seed(2661)
    z = gu.dev(torch.randn(b.num_tokens, 2 * b.C, generator=g).to(torch.bfloat16))
    sent = np.uint16(wl.SENTINEL_BITS)
    sm = b.slot_mapping.numpy()
    for with_seqs in (True, False):
        kc, vc = gu.dev(b.empty_cache()), gu.dev(b.empty_cache())
        kw = dict(cu_seqlens=gu.dev(b.cu_seqlens), W=b.W, state_indices=gu.dev(b.state_indices),
                  state_pool_size=3) if with_seqs else {}
        bd.stage_scatter(z, gu.dev(b.slot_mapping), kc, vc, **kw)
        torch.cuda.synchronize()
        for cache in (kc, vc):
            rows = wl.bits(cache.cpu()).reshape(-1, b.C)
            untouched = np.all(rows == sent, axis=1)
            assert untouched[sm[20:53]].all() == with_seqs
            assert not untouched[sm[:20]].any() and not untouched[sm[53:]].any()
