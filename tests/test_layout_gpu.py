"""GPU parity of the layout variants against the oracle: per-head gammas
[Hkv, D] and the ring-buffer conv_state (position p in row p mod (W-1)),
for prefill and decode, bf16 and MXFP8 stores."""
import ctypes

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


def _per_head(b, seed):
    g = torch.Generator().manual_seed(seed)
    gk = (1 + 0.3 * torch.randn(b.Hkv, b.D, generator=g)).float()
    gv = (1 + 0.3 * torch.randn(b.Hkv, b.D, generator=g)).float()
    return gk, gv


def _oracle(b, gk, gv, positions=None, state=None):
    return oracle.prefill_varlen(
        wl.bits(b.k), wl.bits(b.v), b.cu_seqlens.numpy(), wl.bits(b.conv_w_k),
        wl.bits(b.conv_w_v), gk.numpy(), gv.numpy(), b.eps,
        wl.bits(b.conv_state) if state is None else state, b.slot_mapping.numpy(),
        wl.bits(b.empty_cache()), wl.bits(b.empty_cache()),
        state_indices=None if b.state_indices is None else b.state_indices.numpy(),
        state_positions=positions)


def _gpu(b, gk, gv, positions=None, err=None):
    bd = _bd()
    kc, vc = gu.dev(b.empty_cache()), gu.dev(b.empty_cache())
    st = gu.dev(b.conv_state.clone())
    bd.prefill_varlen(gu.dev(b.k), gu.dev(b.v), gu.dev(b.cu_seqlens), gu.dev(b.conv_w_k),
                      gu.dev(b.conv_w_v), gu.dev(gk), gu.dev(gv), b.eps, st,
                      gu.dev(b.slot_mapping), kc, vc, state_indices=gu.dev(b.state_indices),
                      err_flag=err,
                      state_positions=None if positions is None else gu.dev(
                          torch.from_numpy(np.asarray(positions, np.int64))))
    torch.cuda.synchronize()
    return kc, vc, st


def _check(b, got, ref):
    kc, vc, st = got
    sm = b.slot_mapping.numpy()
    gu.check_cache(wl.bits(kc.cpu()), ref["k_cache"], sm, ref["z_k"], "k_cache")
    gu.check_cache(wl.bits(vc.cpu()), ref["v_cache"], sm, ref["z_v"], "v_cache")
    assert np.array_equal(wl.bits(st.cpu()), ref["conv_state"]), "conv_state"


# ------------------------------------------------------------ per-head gamma

@pytest.mark.parametrize("W,Hkv,D", [(4, 4, 128), (3, 2, 64), (8, 3, 64), (2, 2, 256)])
def test_per_head_gamma_prefill(W, Hkv, D):
    b = wl.make_prefill([300, 1, 0, 77, 9], Hkv=Hkv, D=D, W=W, seed=2800 + W, state="normal",
                        page_size=16, spare_pages=2)
    gk, gv = _per_head(b, 2810 + W)
    _check(b, _gpu(b, gk, gv), _oracle(b, gk, gv))


def test_per_head_gamma_decode():
    bd = _bd()
    s = wl.decode(seed=2820, batch=96, Hkv=8, D=128, W=4, pages_per_seq=2, page_size=16,
                  max_start=8)
    g = torch.Generator().manual_seed(2821)
    gk = (1 + 0.3 * torch.randn(s.Hkv, s.D, generator=g)).float()
    gv = (1 + 0.3 * torch.randn(s.Hkv, s.D, generator=g)).float()
    k, v, sm = s.step_inputs(0)
    kc, vc = gu.dev(s.empty_cache()), gu.dev(s.empty_cache())
    st = gu.dev(s.conv_state.clone())
    bd.decode(gu.dev(k), gu.dev(v), gu.dev(s.conv_w_k), gu.dev(s.conv_w_v), gu.dev(gk),
              gu.dev(gv), s.eps, st, gu.dev(sm), kc, vc)
    torch.cuda.synchronize()
    ref = oracle.decode(wl.bits(k), wl.bits(v), wl.bits(s.conv_w_k), wl.bits(s.conv_w_v),
                        gk.numpy(), gv.numpy(), s.eps, wl.bits(s.conv_state), sm.numpy(),
                        wl.bits(s.empty_cache()), wl.bits(s.empty_cache()))
    smn = sm.numpy()
    gu.check_cache(wl.bits(kc.cpu()), ref["k_cache"], smn, ref["z_k"], "k")
    gu.check_cache(wl.bits(vc.cpu()), ref["v_cache"], smn, ref["z_v"], "v")
    assert np.array_equal(wl.bits(st.cpu()), ref["conv_state"])


def test_per_head_gamma_mxfp8():
    bd = _bd()
    b = wl.make_prefill([120, 7, 33], Hkv=4, D=128, W=4, seed=2830, state="normal",
                        page_size=16, spare_pages=2)
    gk, gv = _per_head(b, 2831)
    kd, ks = gu.mx_caches(b.num_pages, b.page_size, b.Hkv, b.D)
    vd, vs = gu.mx_caches(b.num_pages, b.page_size, b.Hkv, b.D)
    st = gu.dev(b.conv_state.clone())
    bd.prefill_varlen_mxfp8(gu.dev(b.k), gu.dev(b.v), gu.dev(b.cu_seqlens), gu.dev(b.conv_w_k),
                            gu.dev(b.conv_w_v), gu.dev(gk), gu.dev(gv), b.eps, st,
                            gu.dev(b.slot_mapping), kd, ks, vd, vs)
    torch.cuda.synchronize()
    ref = _oracle(b, gk, gv)
    sm = b.slot_mapping.numpy()
    gu.check_mx(kd.cpu().numpy(), ks.cpu().numpy(), sm, ref["z_k"], "k mx")
    gu.check_mx(vd.cpu().numpy(), vs.cpu().numpy(), sm, ref["z_v"], "v mx")
    assert np.array_equal(wl.bits(st.cpu()), ref["conv_state"])


def test_gamma_head_stride_rejected():
    """A head stride other than 0 or head_dim is refused on the host."""
    bd = _bd()
    b = wl.tiny()
    kc, vc = gu.dev(b.empty_cache()), gu.dev(b.empty_cache())
    lay = bd.layout_of(kc)
    o = bd.Options()
    o.gamma_head_stride = 7
    rc = bd.lib.sconv_kv_prefill_varlen_ex(
        gu.dev(b.k).data_ptr(), gu.dev(b.v).data_ptr(), b.C, b.num_tokens,
        gu.dev(b.cu_seqlens).data_ptr(), b.num_seqs, gu.dev(b.conv_w_k).data_ptr(),
        gu.dev(b.conv_w_v).data_ptr(), gu.dev(b.gamma_k).data_ptr(),
        gu.dev(b.gamma_v).data_ptr(), b.eps, b.W, b.Hkv, b.D, gu.dev(b.conv_state).data_ptr(),
        None, b.conv_state.shape[0], gu.dev(b.slot_mapping).data_ptr(), kc.data_ptr(),
        vc.data_ptr(), ctypes.byref(lay), ctypes.byref(o), None, None)
    assert rc == bd.ERR_SHAPE


# ------------------------------------------------------------ ring state

@pytest.mark.parametrize("W", [2, 3, 4, 8])
def test_ring_prefill(W):
    lengths = [0, 1, 2, 3, 9, 40, 700]
    b = wl.make_prefill(lengths, Hkv=4, D=128, W=W, seed=2840 + W, state="normal",
                        page_size=16, spare_pages=2, pool_size=9,
                        state_indices=[8, 3, 0, 7, 5, 1, 6])
    pos = np.random.default_rng(2850 + W).integers(0, 100, size=len(lengths)).astype(np.int64)
    gk, gv = b.gamma_k, b.gamma_v
    _check(b, _gpu(b, gk, gv, positions=pos), _oracle(b, gk, gv, positions=pos))


def test_ring_decode_chain():
    """Eight decode steps with the ring state: each step against the
    oracle's ring decode; a step rewrites one state row per sequence."""
    bd = _bd()
    s = wl.decode(seed=2860, batch=64, Hkv=8, D=128, W=4, pages_per_seq=2, page_size=16,
                  max_start=8)
    pos = np.random.default_rng(2861).integers(0, 30, size=s.batch).astype(np.int64)
    st = gu.dev(s.conv_state.clone())
    st_ref = wl.bits(s.conv_state)
    kc, vc = gu.dev(s.empty_cache()), gu.dev(s.empty_cache())
    for step in range(8):
        k, v, sm = s.step_inputs(step)
        p = pos + step
        before = wl.bits(st.cpu())
        # the oracle writes into the GPU's previous caches, so slots written
        # by earlier steps compare bit for bit and this step's within bounds
        kc_prev, vc_prev = wl.bits(kc.cpu()), wl.bits(vc.cpu())
        bd.decode(gu.dev(k), gu.dev(v), gu.dev(s.conv_w_k), gu.dev(s.conv_w_v),
                  gu.dev(s.gamma_k), gu.dev(s.gamma_v), s.eps, st, gu.dev(sm), kc, vc,
                  state_positions=gu.dev(torch.from_numpy(p)))
        ref = oracle.decode(wl.bits(k), wl.bits(v), wl.bits(s.conv_w_k), wl.bits(s.conv_w_v),
                            s.gamma_k.numpy(), s.gamma_v.numpy(), s.eps, st_ref, sm.numpy(),
                            kc_prev, vc_prev, state_positions=p)
        torch.cuda.synchronize()
        got = wl.bits(st.cpu())
        assert np.array_equal(got, ref["conv_state"]), f"state step {step}"
        changed = (got != before).any(axis=2)  # [B, W-1]: rows that changed
        assert (changed.sum(axis=1) <= 1).all()
        smn = sm.numpy()
        gu.check_cache(wl.bits(kc.cpu()), ref["k_cache"], smn, ref["z_k"], f"k {step}")
        gu.check_cache(wl.bits(vc.cpu()), ref["v_cache"], smn, ref["z_v"], f"v {step}")
        st_ref = ref["conv_state"]


def test_ring_chunks_equal_linear_one_shot():
    """One sequence through the ring state in prefill chunks and decode
    steps writes the same cache bits as one linear-state call."""
    bd = _bd()
    b = wl.make_prefill([300], Hkv=8, D=128, W=4, seed=2870, state="zero", page_size=16,
                        spare_pages=2)
    k1, v1, s1 = _gpu(b, b.gamma_k, b.gamma_v)
    args = [gu.dev(x) for x in (b.conv_w_k, b.conv_w_v, b.gamma_k, b.gamma_v)]
    k, v, sm = gu.dev(b.k), gu.dev(b.v), gu.dev(b.slot_mapping)
    kc, vc = gu.dev(b.empty_cache()), gu.dev(b.empty_cache())
    st = gu.dev(b.conv_state.clone())
    cuts = [0, 1, 2, 50, 51, 52, 200, 300]
    for a, e in zip(cuts[:-1], cuts[1:]):
        p = gu.dev(torch.tensor([a], dtype=torch.int64))
        if e - a == 1:
            bd.decode(k[a:e], v[a:e], *args, b.eps, st, sm[a:e], kc, vc, state_positions=p)
        else:
            bd.prefill_varlen(k[a:e], v[a:e],
                              torch.tensor([0, e - a], dtype=torch.int32, device="cuda"),
                              *args, b.eps, st, sm[a:e], kc, vc, state_positions=p)
    torch.cuda.synchronize()
    # bit patterns (the unwritten-slot sentinel is a NaN)
    assert torch.equal(kc.view(torch.int16), k1.view(torch.int16))
    assert torch.equal(vc.view(torch.int16), v1.view(torch.int16))
    ring = wl.bits(st.cpu())[0]
    n = b.W - 1
    lin = np.stack([ring[(300 - n + j) % n] for j in range(n)])
    assert np.array_equal(lin, wl.bits(s1.cpu())[0])


def test_ring_negative_position_skips_and_flags():
    bd = _bd()
    b = wl.make_prefill([5, 6, 7], Hkv=2, D=64, W=4, seed=2880, state="normal", page_size=8,
                        spare_pages=1)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pos = np.array([3, -1, 0], np.int64)
    kc, vc, st = _gpu(b, b.gamma_k, b.gamma_v, positions=pos, err=err)
    assert int(err.item()) & bd.FLAG_STATE_INDEX
    assert np.array_equal(wl.bits(st.cpu())[1], wl.bits(b.conv_state)[1])  # untouched
    written = b.slot_mapping.numpy()[5:11]
    assert (wl.bits(kc.cpu()).reshape(-1, b.C)[written] == wl.SENTINEL_BITS).all()


def test_ring_decode_mxfp8():
    bd = _bd()
    s = wl.decode(seed=2890, batch=64, Hkv=8, D=128, W=4, pages_per_seq=2, page_size=16,
                  max_start=8)
    pos = np.random.default_rng(2891).integers(0, 30, size=s.batch).astype(np.int64)
    k, v, sm = s.step_inputs(0)
    st = gu.dev(s.conv_state.clone())
    kd, ks = gu.mx_caches(s.num_pages, s.page_size, s.Hkv, s.D)
    vd, vs = gu.mx_caches(s.num_pages, s.page_size, s.Hkv, s.D)
    bd.decode_mxfp8(gu.dev(k), gu.dev(v), gu.dev(s.conv_w_k), gu.dev(s.conv_w_v),
                    gu.dev(s.gamma_k), gu.dev(s.gamma_v), s.eps, st, gu.dev(sm), kd, ks, vd, vs,
                    state_positions=gu.dev(torch.from_numpy(pos)))
    torch.cuda.synchronize()
    small = np.zeros((s.batch, 1, s.Hkv, s.D), np.uint16)
    ref = oracle.decode(wl.bits(k), wl.bits(v), wl.bits(s.conv_w_k), wl.bits(s.conv_w_v),
                        s.gamma_k.numpy(), s.gamma_v.numpy(), s.eps, wl.bits(s.conv_state),
                        np.arange(s.batch, dtype=np.int64), small, small.copy(),
                        state_positions=pos)
    assert np.array_equal(wl.bits(st.cpu()), ref["conv_state"])
    C = s.C
    for which, d, sc, z in (("k", kd, ks, ref["z_k"]), ("v", vd, vs, ref["z_v"])):
        dd = d.view(-1, C)[gu.dev(sm)].cpu().numpy().reshape(s.batch, 1, s.Hkv, s.D)
        ss = sc.view(-1, C // 32)[gu.dev(sm)].cpu().numpy().reshape(s.batch, 1, s.Hkv, s.D // 32)
        gu.check_mx(dd, ss, np.arange(s.batch), z, which)
