"""GPU parity of the MXFP8 (block-scaled) cache store against the oracle:
block scales and E4M3 codes as the oracle decides them from the binary32
normalised values (adjacent codes only at near-ties), untouched slots kept,
conv_state bit-exact."""
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


def _binding():
    from short_conv_kv_b200 import binding
    return binding


def test_mx_tiny():
    gu.full_parity_mx(wl.tiny())


def test_mx_single_8192():
    gu.full_parity_mx(wl.single())


@pytest.mark.parametrize("i", range(7))
def test_mx_partial_last_chunks(i):
    """MXFP8 store (2-token groups) over ranges ending in a partial chunk of
    every length 1..7."""
    from tests.test_parity_gpu import tail_lengths
    T = tail_lengths()[i]
    gu.full_parity_mx(wl.make_prefill([T], Hkv=8, D=128, W=4, seed=2200 + i, state="normal",
                                      page_size=64, permute_pages=True))


@pytest.mark.parametrize("W", [1, 2, 4, 8])
def test_mx_every_w(W):
    b = wl.make_prefill([300, 1, 0, 77, 2], Hkv=4, D=128, W=W, seed=1600 + W,
                        state="normal", page_size=16, spare_pages=5)
    gu.full_parity_mx(b)


@pytest.mark.parametrize("Hkv,D", [(3, 64), (8, 256), (16, 128), (1, 64)])
def test_mx_head_shapes(Hkv, D):
    b = wl.make_prefill([90, 33, 5], Hkv=Hkv, D=D, W=4, seed=1700 + Hkv * D,
                        state="normal", page_size=16, spare_pages=3)
    gu.full_parity_mx(b)


def test_mx_zero_rows_take_smallest_scale():
    """All-zero K rows (and a zero state): y = 0, z = 0, so every block has
    the smallest scale (code 0) and every element encodes zero (the sign of
    a zero product with a negative tap may survive: 0x00 or 0x80)."""
    b = wl.make_prefill([40], Hkv=2, D=64, W=4, seed=1801, state="zero", page_size=16,
                        spare_pages=1)
    b.k = torch.zeros_like(b.k)
    kd, ks, vd, vs, st = gu.run_gpu_prefill_mx(b)
    sm = b.slot_mapping.numpy()
    assert not (kd.view(-1, b.C)[torch.from_numpy(sm).cuda()] & 0x7F).any()
    assert not ks.view(-1, b.C // 32)[torch.from_numpy(sm).cuda()].any()
    ref = gu.oracle_prefill(b)
    gu.check_mx(vd.cpu().numpy(), vs.cpu().numpy(), sm, ref["z_v"], "v mx")


def test_mx_varlen_subset_with_state_indices():
    lengths = [0, 1, 2, 3, 0, 6, 40, 1, 700]
    b = wl.make_prefill(lengths, Hkv=8, D=128, W=4, seed=1802, state="normal",
                        page_size=8, spare_pages=2, pool_size=12,
                        state_indices=[11, 3, 0, 7, 5, 9, 1, 2, 4])
    gu.full_parity_mx(b)


def test_mx_decode_steps():
    """Decode with the MXFP8 store: 6 steps over 256 sequences, each step
    against the oracle chain."""
    bd = _binding()
    s = wl.decode(seed=4300, batch=256, Hkv=8, D=128, W=4, pages_per_seq=2, page_size=16,
                  max_start=8)
    st = gu.dev(s.conv_state.clone())
    kd, ks = gu.mx_caches(s.num_pages, s.page_size, s.Hkv, s.D)
    vd, vs = gu.mx_caches(s.num_pages, s.page_size, s.Hkv, s.D)
    st_ref = wl.bits(s.conv_state)
    small = np.zeros((s.batch, 1, s.Hkv, s.D), np.uint16)
    all_slots = []
    for step in range(6):
        k, v, sm = s.step_inputs(step)
        bd.decode_mxfp8(gu.dev(k), gu.dev(v), gu.dev(s.conv_w_k), gu.dev(s.conv_w_v),
                        gu.dev(s.gamma_k), gu.dev(s.gamma_v), s.eps, st, gu.dev(sm),
                        kd, ks, vd, vs)
        ref = oracle.decode(wl.bits(k), wl.bits(v), wl.bits(s.conv_w_k), wl.bits(s.conv_w_v),
                            s.gamma_k.numpy(), s.gamma_v.numpy(), s.eps, st_ref,
                            np.arange(s.batch, dtype=np.int64), small, small.copy())
        st_ref = ref["conv_state"]
        torch.cuda.synchronize()
        all_slots.append(sm.numpy())
        # this step's slots, gathered on the device, against this step's z
        C = s.C
        for which, d, sc, z in (("k", kd, ks, ref["z_k"]), ("v", vd, vs, ref["z_v"])):
            dd = d.view(-1, C)[gu.dev(sm)].cpu().numpy().reshape(s.batch, 1, s.Hkv, s.D)
            ss = sc.view(-1, C // 32)[gu.dev(sm)].cpu().numpy().reshape(s.batch, 1, s.Hkv, s.D // 32)
            gu.check_mx(dd, ss, np.arange(s.batch), z, f"{which} step {step}")
        assert np.array_equal(wl.bits(st.cpu()), st_ref), f"state step {step}"
    used = np.concatenate(all_slots)
    mask = np.ones(s.num_pages * s.page_size, bool)
    mask[used] = False
    assert bool((kd.view(-1, s.C)[torch.from_numpy(mask).cuda()] == gu.MX_SENTINEL).all())


def test_mx_chunked_equals_one_shot_bitwise():
    bd = _binding()
    b = wl.make_prefill([500], Hkv=8, D=128, W=4, seed=1803, state="normal", page_size=16,
                        spare_pages=2)
    kd1, ks1, vd1, vs1, st1 = gu.run_gpu_prefill_mx(b)
    args = [gu.dev(x) for x in (b.conv_w_k, b.conv_w_v, b.gamma_k, b.gamma_v)]
    k, v, sm = gu.dev(b.k), gu.dev(b.v), gu.dev(b.slot_mapping)
    kd, ks = gu.mx_caches(b.num_pages, b.page_size, b.Hkv, b.D)
    vd, vs = gu.mx_caches(b.num_pages, b.page_size, b.Hkv, b.D)
    st = gu.dev(b.conv_state.clone())
    cuts = [0, 1, 3, 64, 65, 200, 499, 500]
    for a, e in zip(cuts[:-1], cuts[1:]):
        if e - a == 1:
            bd.decode_mxfp8(k[a:e], v[a:e], *args, b.eps, st, sm[a:e], kd, ks, vd, vs)
        else:
            bd.prefill_varlen_mxfp8(k[a:e], v[a:e],
                                    torch.tensor([0, e - a], dtype=torch.int32, device="cuda"),
                                    *args, b.eps, st, sm[a:e], kd, ks, vd, vs)
    torch.cuda.synchronize()
    for x, y in ((kd, kd1), (ks, ks1), (vd, vd1), (vs, vs1)):
        assert torch.equal(x, y)
    assert torch.equal(st.view(torch.int16), st1.view(torch.int16))


def test_mx_rejects_unaligned_layout():
    """Scale caches address a byte per 32 elements: strides must be
    multiples of 32 (checked on the host, nothing launched)."""
    bd = _binding()
    b = wl.tiny()
    kd, ks = gu.mx_caches(b.num_pages, b.page_size, b.Hkv, b.D)
    with pytest.raises(ValueError):
        bd.prefill_varlen_mxfp8(gu.dev(b.k), gu.dev(b.v), gu.dev(b.cu_seqlens),
                                gu.dev(b.conv_w_k), gu.dev(b.conv_w_v), gu.dev(b.gamma_k),
                                gu.dev(b.gamma_v), b.eps, gu.dev(b.conv_state),
                                gu.dev(b.slot_mapping), kd, ks[:, :, :, :1], kd.clone(), ks)


def test_mx_chunks_back_to_back_state_only_dependency():
    """Five chunks of one sequence (3,000 tokens each) through the MXFP8
    store, launched back to back with the state-only dependency and no
    synchronisation in between; each chunk against the oracle run on the
    state the previous chunk left, and the final state bit for bit."""
    b = _binding()
    n, L = 5, 3000
    chunks = [wl.make_prefill([L], Hkv=8, D=128, W=4, seed=1900 + c, state="zero", page_size=16,
                              spare_pages=0) for c in range(n)]
    base = chunks[0]
    for x in chunks:
        x.conv_w_k, x.conv_w_v, x.gamma_k, x.gamma_v = (base.conv_w_k, base.conv_w_v,
                                                        base.gamma_k, base.gamma_v)
    st = gu.dev(base.conv_state.clone())
    w = [gu.dev(t) for t in (base.conv_w_k, base.conv_w_v, base.gamma_k, base.gamma_v)]
    caches = [gu.mx_caches(x.num_pages, x.page_size, x.Hkv, x.D) + gu.mx_caches(
        x.num_pages, x.page_size, x.Hkv, x.D) for x in chunks]
    devs = [(gu.dev(x.k), gu.dev(x.v), gu.dev(x.cu_seqlens), gu.dev(x.slot_mapping)) for x in chunks]
    torch.cuda.synchronize()
    for (k, v, cu, sm), (kd, ks, vd, vs) in zip(devs, caches):
        b.prefill_varlen_mxfp8(k, v, cu, *w, base.eps, st, sm, kd, ks, vd, vs,
                               state_only_dependency=True)
    torch.cuda.synchronize()
    state = wl.bits(base.conv_state)
    for c, (x, (kd, ks, vd, vs)) in enumerate(zip(chunks, caches)):
        x.conv_state = wl.from_bits(state)
        ref = gu.oracle_prefill(x)
        sm = x.slot_mapping.numpy()
        gu.check_mx(kd.cpu().numpy(), ks.cpu().numpy(), sm, ref["z_k"], f"k mx chunk {c}")
        gu.check_mx(vd.cpu().numpy(), vs.cpu().numpy(), sm, ref["z_v"], f"v mx chunk {c}")
        state = ref["conv_state"]
    assert np.array_equal(wl.bits(st.cpu()), state)


def test_mx_decode_independent_state_alternating():
    """MXFP8 decode: two batches on disjoint state rows of one pool,
    launched alternately with the independent-state promise, 6 steps each,
    no synchronisation in between; every step against the oracle chain."""
    b = _binding()
    B, steps = 128, 6
    setups = [wl.decode(seed=7300 + j, batch=B, pages_per_seq=1, page_size=16, max_start=8)
              for j in range(2)]
    sA = setups[0]
    pool = torch.cat([s.conv_state for s in setups])
    st = gu.dev(pool.clone())
    idx = [gu.dev(torch.arange(j * B, (j + 1) * B, dtype=torch.int32)) for j in range(2)]
    w = [gu.dev(x) for x in (sA.conv_w_k, sA.conv_w_v, sA.gamma_k, sA.gamma_v)]
    caches = [[gu.mx_caches(s.num_pages, s.page_size, s.Hkv, s.D) + gu.mx_caches(
        s.num_pages, s.page_size, s.Hkv, s.D) for _ in range(steps)] for s in setups]
    inputs = [[s.step_inputs(t) for t in range(steps)] for s in setups]
    dev_in = [[tuple(gu.dev(x) for x in inp) for inp in seq] for seq in inputs]
    torch.cuda.synchronize()
    for t in range(steps):
        for j in range(2):
            k, v, sm = dev_in[j][t]
            b.decode_mxfp8(k, v, *w, sA.eps, st, sm, *caches[j][t], state_indices=idx[j],
                           independent_state=True)
    torch.cuda.synchronize()
    small = np.zeros((B, 1, sA.Hkv, sA.D), np.uint16)
    for j, s in enumerate(setups):
        ref_state = wl.bits(s.conv_state)
        for t in range(steps):
            k, v, sm = inputs[j][t]
            ref = oracle.decode(wl.bits(k), wl.bits(v), wl.bits(sA.conv_w_k), wl.bits(sA.conv_w_v),
                                sA.gamma_k.numpy(), sA.gamma_v.numpy(), sA.eps, ref_state,
                                np.arange(B, dtype=np.int64), small, small.copy())
            ref_state = ref["conv_state"]
            kd, ks, vd, vs = caches[j][t]
            smn = sm.numpy()
            gu.check_mx(kd.cpu().numpy(), ks.cpu().numpy(), smn, ref["z_k"], f"k {j} {t}")
            gu.check_mx(vd.cpu().numpy(), vs.cpu().numpy(), smn, ref["z_v"], f"v {j} {t}")
        got = wl.bits(st.cpu())[j * B:(j + 1) * B]
        assert np.array_equal(got, ref_state), f"state of batch {j}"
