"""GPU parity: the CUDA path (through the C ABI) against the oracle on the
same seeded inputs.  Placement, untouched slots and conv_state must match
bit for bit; normalised bf16 values within 2e-2 abs / 1e-2 rel of the
oracle's double-precision z."""
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
    torch.cuda.init()
    yield
    torch.cuda.synchronize()


def _binding():
    from short_conv_kv_b200 import binding
    return binding


def tail_lengths():
    """Single-sequence lengths that give every persistent CTA of the W <= 4
    prefill (two per SM, 8-row chunks) exactly k rows, k = 25..31: ranges
    ending in partial chunks of 1..7 rows, whose unrolled groups wholly
    past the end are skipped."""
    ctas = 2 * torch.cuda.get_device_properties(0).multi_processor_count
    return [ctas * k for k in range(25, 32)]


# ----------------------------------------------------------- named configs

def test_tiny_full():
    """2 sequences (37, 64 tokens), Hkv=2, D=64, W=4, paged 16x16 cache."""
    gu.full_parity(wl.tiny())


def test_single_8192_full():
    """One 8192-token sequence, Hkv=8, D=128, W=4, contiguous cache."""
    gu.full_parity(wl.single())


def test_short_launch_instance_threshold_full():
    """Around the token count where the host switches between the
    short-launch bf16 instance (at most 8 chunks of 8 rows per persistent
    CTA; 4-token head reductions) and the default one (2-token reductions):
    both calls equal the oracle, and the rows they share are bitwise equal
    (the batched reductions add the same lane sets in the same order)."""
    import dataclasses
    ctas = torch.cuda.get_device_properties(0).multi_processor_count * 2
    Ts = ctas * 8 * 8  # largest single-sequence launch of the short instance
    b = wl.make_prefill([Ts + 8], Hkv=2, D=128, W=4, seed=2190, state="normal",
                        page_size=64, permute_pages=True)
    short = dataclasses.replace(b, k=b.k[:Ts].clone(), v=b.v[:Ts].clone(),
                                cu_seqlens=torch.tensor([0, Ts], dtype=torch.int32),
                                slot_mapping=b.slot_mapping[:Ts].clone())
    gu.full_parity(b)
    gu.full_parity(short)
    kl, vl, _ = gu.run_gpu_prefill(b)
    ks, vs, _ = gu.run_gpu_prefill(short)
    rows = b.slot_mapping[:Ts].numpy()
    for a, c in ((kl, ks), (vl, vs)):
        la = wl.bits(a.cpu()).reshape(-1, 2 * 128)[rows]
        lc = wl.bits(c.cpu()).reshape(-1, 2 * 128)[rows]
        assert np.array_equal(la, lc)


@pytest.mark.parametrize("i", range(7))
def test_partial_last_chunks_full(i):
    """Ranges ending in a partial chunk of every length 1..7 (one sequence,
    W=4, N(0,1) state, permuted pages)."""
    T = tail_lengths()[i]
    gu.full_parity(wl.make_prefill([T], Hkv=8, D=128, W=4, seed=2100 + i, state="normal",
                                   page_size=64, permute_pages=True))


def _sample_tokens(cu, W, rng, n_random=2000, tile=32):
    """Tokens that exercise the halo (first W-1 of each sequence), sequence
    ends, tile edges, plus a random sample."""
    cu = np.asarray(cu)
    T = int(cu[-1])
    pick = set()
    for i in range(len(cu) - 1):
        a, b = int(cu[i]), int(cu[i + 1])
        pick.update(range(a, min(b, a + W)))
        pick.update(range(max(a, b - 2), b))
        for e in range(a + tile, b, tile * 17):
            pick.update((e - 1, e))
    pick.update(rng.integers(0, T, size=n_random).tolist())
    return np.array(sorted(t for t in pick if 0 <= t < T), dtype=np.int64)


def _check_sampled(b, kc, vc, st, tokens):
    """Sampled tokens (oracle decodes each from its window) + full state +
    untouched slots, for a batch too large for a whole-batch oracle run."""
    T, C = b.num_tokens, b.C
    kb, vb = wl.bits(b.k).reshape(T, C), wl.bits(b.v).reshape(T, C)
    cu = b.cu_seqlens.numpy()
    sb = wl.bits(b.conv_state)
    si = None if b.state_indices is None else b.state_indices.numpy()
    zk, zv = gu.sampled_oracle_z(kb, vb, cu, sb, tokens, b.W, wl.bits(b.conv_w_k),
                                 wl.bits(b.conv_w_v), b.gamma_k.numpy(), b.gamma_v.numpy(),
                                 b.eps, b.Hkv, b.D, state_indices=si)
    sm = b.slot_mapping.numpy()
    slots = torch.from_numpy(sm[tokens]).cuda()
    gk = wl.bits(kc.reshape(-1, C)[slots].cpu())
    gv = wl.bits(vc.reshape(-1, C)[slots].cpu())
    gu.assert_close(gk, zk, "k sampled")
    gu.assert_close(gv, zv, "v sampled")
    exp_state = gu.expected_final_state(kb, vb, cu, sb, b.W, si)
    assert np.array_equal(wl.bits(st.cpu()), exp_state)
    _check_untouched_device(kc, vc, b.slot_mapping)


def _check_untouched_device(kc, vc, slot_mapping):
    C = kc.shape[-1] * kc.shape[-2]
    mask = torch.ones(kc.shape[0] * kc.shape[1], dtype=torch.bool, device="cuda")
    sm = slot_mapping.cuda()
    mask[sm[sm >= 0]] = False
    for c in (kc, vc):
        rows = c.reshape(-1, C).view(torch.int16)[mask]
        assert bool((rows == wl.SENTINEL_BITS).all()), "untouched slot changed"
        written = c.reshape(-1, C).view(torch.int16)[~mask]
        assert not bool((written == wl.SENTINEL_BITS).any()), "written slot kept sentinel"


def test_varlen_32_sequences_sampled():
    """32 sequences, lengths U[512, 8192], N(0,1) state, permuted pages."""
    b = wl.varlen()
    kc, vc, st = gu.run_gpu_prefill(b)
    tokens = _sample_tokens(b.cu_seqlens.numpy(), b.W, np.random.default_rng(3))
    _check_sampled(b, kc, vc, st, tokens)


def test_many_sequences_1900_sampled():
    """1,900 sequences of 32..96 tokens, Hkv=8, D=128, W=4: cu_seqlens no
    longer fits in shared memory beside two CTAs per SM, so the CTAs read it
    from global memory (and all stay resident); sampled tokens of every
    sequence start, the full state, untouched slots against the oracle."""
    g = torch.Generator().manual_seed(3600)
    lengths = torch.randint(32, 97, (1900,), generator=g).tolist()
    b = wl.make_prefill(lengths, Hkv=8, D=128, W=4, seed=3601, state="normal",
                        page_size=64, permute_pages=True, spare_pages=64)
    kc, vc, st = gu.run_gpu_prefill(b)
    tokens = _sample_tokens(b.cu_seqlens.numpy(), b.W, np.random.default_rng(19), n_random=500)
    _check_sampled(b, kc, vc, st, tokens)


def test_varlen_subset_full():
    """Whole-batch oracle on 6 of the varlen workload's sequences (packed as
    their own batch with their own initial state rows)."""
    lengths = wl.varlen_lengths(3000)[:6]
    b = wl.make_prefill(lengths, Hkv=8, D=128, W=4, seed=3001, state="normal",
                        page_size=64, permute_pages=True, spare_pages=64)
    gu.full_parity(b)


def test_decode_1024_x_64_steps():
    """1024 sequences x 64 decode steps, state carried; every step compared
    with the oracle run as its own chain (cache values + state bits)."""
    b = _binding()
    s = wl.decode()
    C = s.C
    st_gpu = gu.dev(s.conv_state.clone())
    kc, vc = gu.dev(s.empty_cache()), gu.dev(s.empty_cache())
    wk, wv, gk, gv = (gu.dev(s.conv_w_k), gu.dev(s.conv_w_v), gu.dev(s.gamma_k),
                      gu.dev(s.gamma_v))
    import oracle
    st_ref = wl.bits(s.conv_state)
    small = np.zeros((s.batch, 1, s.Hkv, s.D), np.uint16)
    for step in range(64):
        k, v, sm = s.step_inputs(step)
        b.decode(gu.dev(k), gu.dev(v), wk, wv, gk, gv, s.eps, st_gpu, gu.dev(sm), kc, vc)
        ref = oracle.decode(wl.bits(k), wl.bits(v), wl.bits(s.conv_w_k), wl.bits(s.conv_w_v),
                            s.gamma_k.numpy(), s.gamma_v.numpy(), s.eps, st_ref,
                            np.arange(s.batch, dtype=np.int64), small, small.copy())
        st_ref = ref["conv_state"]
        torch.cuda.synchronize()
        slots = gu.dev(sm)
        gu.assert_close(wl.bits(kc.reshape(-1, C)[slots].cpu()), ref["z_k"], f"k step {step}")
        gu.assert_close(wl.bits(vc.reshape(-1, C)[slots].cpu()), ref["z_v"], f"v step {step}")
        assert np.array_equal(wl.bits(st_gpu.cpu()), st_ref), f"state step {step}"
    all_slots = torch.cat([s.step_inputs(i)[2] for i in range(64)])
    _check_untouched_device(kc, vc, all_slots)


def test_long_context_1m_chunked_sampled():
    """One 1,048,576-token sequence in 16 chunks of 65,536 with the state
    carried; sampled tokens of every chunk (incl. each chunk's first W-1,
    whose window reaches into the previous chunk) against the oracle."""
    b = _binding()
    s = wl.long_context()
    C, W = s.C, s.W
    st = gu.dev(s.initial_state())
    kc, vc = gu.dev(s.empty_cache()), gu.dev(s.empty_cache())
    wk, wv, gk, gv = (gu.dev(s.conv_w_k), gu.dev(s.conv_w_v), gu.dev(s.gamma_k),
                      gu.dev(s.gamma_v))
    rng = np.random.default_rng(5)
    prev_tail = wl.bits(s.initial_state())
    all_slots = []
    for c in range(s.num_chunks):
        k, v, sm, cu = s.chunk_inputs(c)
        b.prefill_varlen(gu.dev(k), gu.dev(v), gu.dev(cu), wk, wv, gk, gv, s.eps, st,
                         gu.dev(sm), kc, vc)
        torch.cuda.synchronize()
        L = k.shape[0]
        kb, vb = wl.bits(k).reshape(L, C), wl.bits(v).reshape(L, C)
        tokens = _sample_tokens(np.array([0, L]), W, rng, n_random=150)
        zk, zv = gu.sampled_oracle_z(kb, vb, np.array([0, L]), prev_tail, tokens, W,
                                     wl.bits(s.conv_w_k), wl.bits(s.conv_w_v),
                                     s.gamma_k.numpy(), s.gamma_v.numpy(), s.eps,
                                     s.Hkv, s.D)
        slots = gu.dev(sm[tokens])
        gu.assert_close(wl.bits(kc.reshape(-1, C)[slots].cpu()), zk, f"k chunk {c}")
        gu.assert_close(wl.bits(vc.reshape(-1, C)[slots].cpu()), zv, f"v chunk {c}")
        prev_tail = gu.expected_final_state(kb, vb, np.array([0, L]), prev_tail, W)
        assert np.array_equal(wl.bits(st.cpu()), prev_tail), f"state after chunk {c}"
        all_slots.append(sm)
    _check_untouched_device(kc, vc, torch.cat(all_slots))


@pytest.mark.parametrize("overlap", [True, False])
def test_chunks_back_to_back_sampled(overlap):
    """Six 65,536-token chunks of one sequence launched back to back on one
    stream with no synchronisation in between -- with the state-only
    dependency (only the CTA that reads the carried state waits for the
    previous launch) and without it.  Afterwards: sampled tokens of every
    chunk (incl. each chunk's first W-1, whose window reaches into the
    previous chunk, and every chunk's last rows) against the oracle, the
    final state bit for bit, untouched slots."""
    b = _binding()
    s = wl.long_context(seed=5300)
    n = 6
    C, W = s.C, s.W
    chunks = [s.chunk_inputs(c) for c in range(n)]
    dev_chunks = [tuple(gu.dev(x) for x in ch) for ch in chunks]
    st = gu.dev(s.initial_state())
    kc, vc = gu.dev(s.empty_cache()), gu.dev(s.empty_cache())
    wk, wv, gk, gv = (gu.dev(s.conv_w_k), gu.dev(s.conv_w_v), gu.dev(s.gamma_k),
                      gu.dev(s.gamma_v))
    torch.cuda.synchronize()
    for k, v, sm, cu in dev_chunks:
        b.prefill_varlen(k, v, cu, wk, wv, gk, gv, s.eps, st, sm, kc, vc,
                         state_only_dependency=overlap)
    torch.cuda.synchronize()
    rng = np.random.default_rng(53)
    prev_tail = wl.bits(s.initial_state())
    for c, (k, v, sm, cu) in enumerate(chunks):
        L = k.shape[0]
        kb, vb = wl.bits(k).reshape(L, C), wl.bits(v).reshape(L, C)
        tokens = _sample_tokens(np.array([0, L]), W, rng, n_random=150)
        zk, zv = gu.sampled_oracle_z(kb, vb, np.array([0, L]), prev_tail, tokens, W,
                                     wl.bits(s.conv_w_k), wl.bits(s.conv_w_v),
                                     s.gamma_k.numpy(), s.gamma_v.numpy(), s.eps, s.Hkv, s.D)
        slots = gu.dev(sm[tokens])
        gu.assert_close(wl.bits(kc.reshape(-1, C)[slots].cpu()), zk, f"k chunk {c}")
        gu.assert_close(wl.bits(vc.reshape(-1, C)[slots].cpu()), zv, f"v chunk {c}")
        prev_tail = gu.expected_final_state(kb, vb, np.array([0, L]), prev_tail, W)
    assert np.array_equal(wl.bits(st.cpu()), prev_tail), "state after the chain"
    _check_untouched_device(kc, vc, torch.cat([ch[2] for ch in chunks]))


def test_varlen_chunks_back_to_back_state_only_dependency():
    """Four continuation chunks of the same 8 sequences (state carried in a
    shuffled pool), launched back to back with the state-only dependency:
    here most CTAs hold a sequence start and wait; the rest stream at once.
    Each chunk against the oracle run on the state the previous chunk left."""
    b = _binding()
    n_seq, pool = 8, 11
    si = torch.tensor([3, 10, 0, 7, 5, 9, 1, 2], dtype=torch.int32)
    batches = [wl.make_prefill(list(np.random.default_rng(60 + c).integers(0, 700, n_seq)),
                               Hkv=4, D=128, W=4, seed=6100 + c, state="normal",
                               page_size=16, spare_pages=0, pool_size=pool,
                               state_indices=si) for c in range(4)]
    st0 = batches[0].conv_state.clone()
    st = gu.dev(st0)
    caches = [(gu.dev(x.empty_cache()), gu.dev(x.empty_cache())) for x in batches]
    w = [gu.dev(t) for t in (batches[0].conv_w_k, batches[0].conv_w_v, batches[0].gamma_k,
                             batches[0].gamma_v)]
    devs = [(gu.dev(x.k), gu.dev(x.v), gu.dev(x.cu_seqlens), gu.dev(x.slot_mapping))
            for x in batches]
    sid = gu.dev(si)
    torch.cuda.synchronize()
    for (k, v, cu, sm), (kc, vc) in zip(devs, caches):
        b.prefill_varlen(k, v, cu, *w, batches[0].eps, st, sm, kc, vc, state_indices=sid,
                         state_only_dependency=True)
    torch.cuda.synchronize()
    state = wl.bits(st0)
    for c, (x, (kc, vc)) in enumerate(zip(batches, caches)):
        x.conv_w_k, x.conv_w_v = batches[0].conv_w_k, batches[0].conv_w_v
        x.gamma_k, x.gamma_v = batches[0].gamma_k, batches[0].gamma_v
        x.conv_state = wl.from_bits(state)
        ref = gu.oracle_prefill(x)
        gu.check_cache(wl.bits(kc.cpu()), ref["k_cache"], x.slot_mapping.numpy(), ref["z_k"],
                       f"k chunk {c}")
        gu.check_cache(wl.bits(vc.cpu()), ref["v_cache"], x.slot_mapping.numpy(), ref["z_v"],
                       f"v chunk {c}")
        state = ref["conv_state"]
    assert np.array_equal(wl.bits(st.cpu()), state)


@pytest.mark.parametrize("W", [2, 4, 8])
def test_w_sweep_65536_sampled(W):
    """W in {2, 4, 8} at T=65,536, one chunk, zero state."""
    b = wl.make_prefill([65536], Hkv=8, D=128, W=W, seed=5100 + W, state="zero",
                        page_size=64, permute_pages=True, spare_pages=64)
    kc, vc, st = gu.run_gpu_prefill(b)
    tokens = _sample_tokens(b.cu_seqlens.numpy(), W, np.random.default_rng(W))
    _check_sampled(b, kc, vc, st, tokens)


# ----------------------------------------------------------- shapes and W

@pytest.mark.parametrize("W", [1, 2, 3, 4, 5, 6, 7, 8])
def test_every_w_full(W):
    b = wl.make_prefill([300, 1, 0, 77, 2], Hkv=4, D=128, W=W, seed=600 + W,
                        state="normal", page_size=16, spare_pages=5)
    gu.full_parity(b)


@pytest.mark.parametrize("Hkv,D", [(1, 64), (3, 64), (2, 128), (5, 128), (8, 256),
                                   (1, 256), (16, 128), (12, 64)])
def test_head_shapes_full(Hkv, D):
    """Partial warps (Hkv*D/4 not a multiple of 32), several CTAs per row
    (more than 256 channel groups), every head_dim."""
    b = wl.make_prefill([90, 33, 5], Hkv=Hkv, D=D, W=4, seed=700 + Hkv * D,
                        state="normal", page_size=16, spare_pages=3)
    gu.full_parity(b)


# ----------------------------------------------------------- edge cases

def test_short_and_empty_sequences_with_state():
    """L = 0, L < W-1 (window and new state mix old and new rows), L = W-1,
    and a state index permutation into a larger pool."""
    lengths = [0, 1, 2, 3, 0, 6, 40, 1]
    b = wl.make_prefill(lengths, Hkv=2, D=64, W=8, seed=801, state="normal",
                        page_size=8, spare_pages=2, pool_size=12,
                        state_indices=[11, 3, 0, 7, 5, 9, 1, 2])
    gu.full_parity(b)


def test_negative_slots_skip_tokens():
    b = wl.make_prefill([50, 70], Hkv=2, D=128, W=4, seed=802, state="normal",
                        page_size=16, spare_pages=2)
    sm = b.slot_mapping.clone()
    sm[::3] = -1
    b.slot_mapping = sm
    gu.full_parity(b)


def test_strided_rows_from_fused_qkv():
    """k and v as column slices of a fused [T, (Hq + 2 Hkv) * D] buffer."""
    b = wl.make_prefill([65, 40], Hkv=2, D=128, W=4, seed=803, state="normal",
                        page_size=16, spare_pages=1)
    T, C = b.num_tokens, b.C
    qkv = torch.zeros(T, 4 * C + C, dtype=torch.bfloat16)
    qkv[:, 4 * C - 2 * C:4 * C - C] = b.k.reshape(T, C)   # layout: q | k | v | pad
    qkv[:, 4 * C - C:4 * C] = b.v.reshape(T, C)
    qd = qkv.cuda()
    kview = qd[:, 2 * C:3 * C].view(T, b.Hkv, b.D)
    vview = qd[:, 3 * C:4 * C].view(T, b.Hkv, b.D)
    assert kview.stride(0) == 5 * C
    bd = _binding()
    kc, vc = gu.dev(b.empty_cache()), gu.dev(b.empty_cache())
    st = gu.dev(b.conv_state.clone())
    bd.prefill_varlen(kview, vview, gu.dev(b.cu_seqlens), gu.dev(b.conv_w_k),
                      gu.dev(b.conv_w_v), gu.dev(b.gamma_k), gu.dev(b.gamma_v), b.eps, st,
                      gu.dev(b.slot_mapping), kc, vc)
    torch.cuda.synchronize()
    ref = gu.oracle_prefill(b)
    gu.check_cache(wl.bits(kc.cpu()), ref["k_cache"], b.slot_mapping.numpy(), ref["z_k"])
    gu.check_cache(wl.bits(vc.cpu()), ref["v_cache"], b.slot_mapping.numpy(), ref["z_v"])
    assert np.array_equal(wl.bits(st.cpu()), ref["conv_state"])


def test_interleaved_kv_cache_layout():
    """K and V as the two halves of one [num_pages, 2, page_size, Hkv, D]
    buffer (stride_page != page_size * stride_slot: the page/offset path)."""
    b = wl.make_prefill([45, 20], Hkv=2, D=64, W=3, seed=804, state="normal",
                        page_size=8, spare_pages=3)
    buf = torch.full((b.num_pages, 2, b.page_size, b.Hkv, b.D), wl.SENTINEL_BITS,
                     dtype=torch.int16).view(torch.bfloat16).cuda()
    kc, vc = buf[:, 0], buf[:, 1]
    assert kc.stride(0) != kc.shape[1] * kc.stride(1)
    st = gu.dev(b.conv_state.clone())
    _binding().prefill_varlen(gu.dev(b.k), gu.dev(b.v), gu.dev(b.cu_seqlens),
                              gu.dev(b.conv_w_k), gu.dev(b.conv_w_v), gu.dev(b.gamma_k),
                              gu.dev(b.gamma_v), b.eps, st, gu.dev(b.slot_mapping), kc, vc)
    torch.cuda.synchronize()
    ref = gu.oracle_prefill(b)
    gu.check_cache(wl.bits(kc.contiguous().cpu()), ref["k_cache"], b.slot_mapping.numpy(),
                   ref["z_k"])
    gu.check_cache(wl.bits(vc.contiguous().cpu()), ref["v_cache"], b.slot_mapping.numpy(),
                   ref["z_v"])
    assert np.array_equal(wl.bits(st.cpu()), ref["conv_state"])


def test_many_sequences_global_search():
    """More sequences than fit the kernel's shared-memory cu_seqlens copy
    (the binary search then reads cu_seqlens from global memory)."""
    rng = np.random.default_rng(9)
    lengths = rng.integers(0, 12, size=2600).tolist()
    b = wl.make_prefill(lengths, Hkv=1, D=64, W=4, seed=805, state="normal",
                        page_size=16, spare_pages=4)
    gu.full_parity(b)


def test_out_of_range_slot_sets_flag_and_skips():
    b = wl.make_prefill([30, 30], Hkv=2, D=64, W=4, seed=806, state="normal",
                        page_size=16, spare_pages=2)
    sm = b.slot_mapping.clone()
    bad = [3, 40]
    sm[bad] = b.num_pages * b.page_size + 5
    b.slot_mapping = sm
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    kc, vc, st = gu.run_gpu_prefill(b, err=err)
    assert int(err.item()) == _binding().FLAG_SLOT_RANGE
    ok = sm.clone()
    ok[bad] = -1
    b.slot_mapping = ok
    ref = gu.oracle_prefill(b)
    gu.check_cache(wl.bits(kc.cpu()), ref["k_cache"], ok.numpy(), ref["z_k"])
    gu.check_cache(wl.bits(vc.cpu()), ref["v_cache"], ok.numpy(), ref["z_v"])
    assert np.array_equal(wl.bits(st.cpu()), ref["conv_state"])


def test_bad_state_index_sets_flag_and_skips_sequence():
    b = wl.make_prefill([20, 25, 9], Hkv=2, D=64, W=4, seed=807, state="normal",
                        page_size=16, spare_pages=2, pool_size=3, state_indices=[0, 7, 2])
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    kc, vc, st = gu.run_gpu_prefill(b, err=err)
    assert int(err.item()) == _binding().FLAG_STATE_INDEX
    # sequence 1 is skipped entirely: its slots untouched, no state written
    cu = b.cu_seqlens.numpy()
    skip = b.slot_mapping.clone()
    skip[cu[1]:cu[2]] = -1
    b2 = wl.make_prefill([20, 25, 9], Hkv=2, D=64, W=4, seed=807, state="normal",
                         page_size=16, spare_pages=2, pool_size=3, state_indices=[0, 1, 2])
    b2.slot_mapping = skip
    ref = gu.oracle_prefill(b2)
    expect_state = ref["conv_state"].copy()
    expect_state[1] = wl.bits(b.conv_state)[1]
    gu.check_cache(wl.bits(kc.cpu()), ref["k_cache"], skip.numpy(), ref["z_k"])
    gu.check_cache(wl.bits(vc.cpu()), ref["v_cache"], skip.numpy(), ref["z_v"])
    assert np.array_equal(wl.bits(st.cpu()), expect_state)


def test_bad_cu_seqlens_sets_flag():
    b = wl.make_prefill([10, 10], Hkv=2, D=64, W=4, seed=808, page_size=16,
                        spare_pages=2)
    b.cu_seqlens = torch.tensor([0, 12, 30], dtype=torch.int32)  # ends past T=20
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    gu.run_gpu_prefill(b, err=err)
    assert int(err.item()) & _binding().FLAG_CU_SEQLENS


def test_valid_call_leaves_flag_clear():
    b = wl.tiny()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    gu.run_gpu_prefill(b, err=err)
    assert int(err.item()) == 0


def test_empty_calls_are_noops():
    bd = _binding()
    b = wl.tiny()
    kc, vc = gu.dev(b.empty_cache()), gu.dev(b.empty_cache())
    st = gu.dev(b.conv_state.clone())
    e = torch.zeros(0, b.Hkv, b.D, dtype=torch.bfloat16, device="cuda")
    bd.prefill_varlen(e, e, torch.zeros(1, dtype=torch.int32, device="cuda"),
                      gu.dev(b.conv_w_k), gu.dev(b.conv_w_v), gu.dev(b.gamma_k),
                      gu.dev(b.gamma_v), b.eps, st,
                      torch.zeros(0, dtype=torch.int64, device="cuda"), kc, vc)
    bd.decode(e, e, gu.dev(b.conv_w_k), gu.dev(b.conv_w_v), gu.dev(b.gamma_k),
              gu.dev(b.gamma_v), b.eps, st, torch.zeros(0, dtype=torch.int64, device="cuda"),
              kc, vc)
    torch.cuda.synchronize()
    assert bool((kc.view(torch.int16) == wl.SENTINEL_BITS).all())
    assert torch.equal(st.cpu(), b.conv_state)


def test_decode_state_indices_and_skip():
    bd = _binding()
    s = wl.decode(seed=4100, batch=37, Hkv=3, D=64, W=5, pages_per_seq=2, page_size=16,
                  max_start=8)
    k, v, sm = s.step_inputs(0)
    sm = sm.clone()
    sm[5] = -1
    perm = torch.randperm(37, generator=torch.Generator().manual_seed(1)).to(torch.int32)
    pool = torch.cat([s.conv_state, s.conv_state[:4]])  # pool of 41 rows
    st = gu.dev(pool.clone())
    kc, vc = gu.dev(s.empty_cache()), gu.dev(s.empty_cache())
    bd.decode(gu.dev(k), gu.dev(v), gu.dev(s.conv_w_k), gu.dev(s.conv_w_v),
              gu.dev(s.gamma_k), gu.dev(s.gamma_v), s.eps, st, gu.dev(sm), kc, vc,
              state_indices=gu.dev(perm))
    torch.cuda.synchronize()
    import oracle
    ref = oracle.decode(wl.bits(k), wl.bits(v), wl.bits(s.conv_w_k), wl.bits(s.conv_w_v),
                        s.gamma_k.numpy(), s.gamma_v.numpy(), s.eps, wl.bits(pool),
                        sm.numpy(), wl.bits(s.empty_cache()), wl.bits(s.empty_cache()),
                        state_indices=perm.numpy())
    gu.check_cache(wl.bits(kc.cpu()), ref["k_cache"], sm.numpy(), ref["z_k"])
    gu.check_cache(wl.bits(vc.cpu()), ref["v_cache"], sm.numpy(), ref["z_v"])
    assert np.array_equal(wl.bits(st.cpu()), ref["conv_state"])


# ----------------------------------------------------------- invariants (GPU vs GPU)

def test_chunked_equals_one_shot_equals_decode_bitwise():
    """The GPU result does not depend on how a sequence is cut into calls:
    one-shot prefill, random chunks and token-by-token decode give the same
    cache bits and state bits."""
    bd = _binding()
    W, L = 4, 700
    b = wl.make_prefill([L], Hkv=8, D=128, W=W, seed=900, state="normal",
                        page_size=16, spare_pages=2)
    kc1, vc1, st1 = gu.run_gpu_prefill(b)
    args = [gu.dev(x) for x in (b.conv_w_k, b.conv_w_v, b.gamma_k, b.gamma_v)]
    k, v, sm = gu.dev(b.k), gu.dev(b.v), gu.dev(b.slot_mapping)
    for mode in ("chunks", "decode"):
        kc, vc = gu.dev(b.empty_cache()), gu.dev(b.empty_cache())
        st = gu.dev(b.conv_state.clone())
        if mode == "chunks":
            cuts = [0, 1, 2, 37, 64, 65, 300, 333, 699, 700]
            for a, e in zip(cuts[:-1], cuts[1:]):
                bd.prefill_varlen(k[a:e], v[a:e],
                                  torch.tensor([0, e - a], dtype=torch.int32, device="cuda"),
                                  *args, b.eps, st, sm[a:e], kc, vc)
        else:
            for t in range(L):
                bd.decode(k[t:t + 1], v[t:t + 1], *args, b.eps, st, sm[t:t + 1], kc, vc)
        torch.cuda.synchronize()
        assert torch.equal(kc.view(torch.int16), kc1.view(torch.int16)), mode
        assert torch.equal(vc.view(torch.int16), vc1.view(torch.int16)), mode
        assert torch.equal(st.view(torch.int16), st1.view(torch.int16)), mode


def test_deterministic():
    b = wl.make_prefill([500, 300], Hkv=8, D=128, W=4, seed=901, state="normal",
                        page_size=64, spare_pages=1)
    r1 = gu.run_gpu_prefill(b)
    r2 = gu.run_gpu_prefill(b)
    for x, y in zip(r1, r2):
        assert torch.equal(x.view(torch.int16), y.view(torch.int16))


def test_skewed_lengths_full():
    """One long sequence among many short ones (the even token split puts
    many CTAs inside the long one and several short sequences in one CTA)."""
    lengths = [4000] + [3, 16, 1, 0, 7] * 60
    b = wl.make_prefill(lengths, Hkv=4, D=128, W=4, seed=905, state="normal",
                        page_size=16, spare_pages=4)
    gu.full_parity(b)


@pytest.mark.parametrize("ring", [False, True])
def test_decode_independent_state_alternating_batches(ring):
    """Two decode batches with disjoint state rows in one pool, launched
    alternately with the independent-state promise (each call's previous
    kernel is the other batch's step, which writes none of this call's
    state rows), 8 steps each with no synchronisation in between.  Every
    step's cache rows and the final states against two oracle chains."""
    import oracle
    b = _binding()
    B, steps = 256, 8
    sA = wl.decode(seed=7100, batch=B, pages_per_seq=1, page_size=16, max_start=8)
    sB = wl.decode(seed=7200, batch=B, pages_per_seq=1, page_size=16, max_start=8)
    C = sA.C
    pool = torch.cat([sA.conv_state, sB.conv_state])
    st = gu.dev(pool.clone())
    idx = [gu.dev(torch.arange(B, dtype=torch.int32)),
           gu.dev(torch.arange(B, 2 * B, dtype=torch.int32))]
    setups = [sA, sB]
    w = [gu.dev(x) for x in (sA.conv_w_k, sA.conv_w_v, sA.gamma_k, sA.gamma_v)]
    caches = [(gu.dev(s.empty_cache()), gu.dev(s.empty_cache())) for s in setups]
    inputs = [[s.step_inputs(t) for t in range(steps)] for s in setups]
    dev_in = [[tuple(gu.dev(x) for x in inp) for inp in seq] for seq in inputs]
    pos = [[gu.dev(torch.from_numpy(s.start_len.astype(np.int64) + t)) for t in range(steps)]
           for s in setups]
    torch.cuda.synchronize()
    for t in range(steps):
        for j in range(2):
            k, v, sm = dev_in[j][t]
            b.decode(k, v, *w, sA.eps, st, sm, *caches[j], state_indices=idx[j],
                     state_positions=pos[j][t] if ring else None, independent_state=True)
    torch.cuda.synchronize()
    small = np.zeros((B, 1, sA.Hkv, sA.D), np.uint16)
    for j, s in enumerate(setups):
        ref_state = wl.bits(s.conv_state)
        kc, vc = caches[j]
        for t in range(steps):
            k, v, sm = inputs[j][t]
            ref = oracle.decode(wl.bits(k), wl.bits(v), wl.bits(sA.conv_w_k),
                                wl.bits(sA.conv_w_v), sA.gamma_k.numpy(), sA.gamma_v.numpy(),
                                sA.eps, ref_state, np.arange(B, dtype=np.int64), small,
                                small.copy(),
                                state_positions=(s.start_len.astype(np.int64) + t) if ring
                                else None)
            ref_state = ref["conv_state"]
            slots = gu.dev(sm)
            gu.assert_close(wl.bits(kc.reshape(-1, C)[slots].cpu()), ref["z_k"], f"k {j} {t}")
            gu.assert_close(wl.bits(vc.reshape(-1, C)[slots].cpu()), ref["z_v"], f"v {j} {t}")
        got = wl.bits(st.cpu())[j * B:(j + 1) * B]
        assert np.array_equal(got, ref_state), f"state of batch {j}"
