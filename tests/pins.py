"""Pins for the oracle: each check ties the oracle to something other than
itself (a brute-force restatement, a library routine, a closed form, an
invariant of the method).  Every check takes the oracle library handle so the
same checks can be run against deliberately broken copies of the oracle
(see test_oracle_mutants.py) to show that a plausible mistake is caught.

A check raises AssertionError on failure.
"""
import numpy as np
import torch

import oracle
from short_conv_kv_b200 import workloads as wl
from tests.brute import brute_step, to_floats


def _bits(t):
    return wl.bits(t)


def _run(lib, b, cache_k=None, cache_v=None, state=None, slots=None, cu=None,
         k=None, v=None, check=True):
    kc = _bits(b.empty_cache()) if cache_k is None else cache_k
    vc = _bits(b.empty_cache()) if cache_v is None else cache_v
    return oracle.prefill_varlen(
        _bits(b.k) if k is None else k, _bits(b.v) if v is None else v,
        b.cu_seqlens.numpy() if cu is None else cu,
        _bits(b.conv_w_k), _bits(b.conv_w_v), b.gamma_k.numpy(),
        b.gamma_v.numpy(), b.eps,
        _bits(b.conv_state) if state is None else state,
        b.slot_mapping.numpy() if slots is None else slots, kc, vc,
        state_indices=None if b.state_indices is None else b.state_indices.numpy(),
        check=check, lib=lib)


# ------------------------------------------------------------------ pins

def pin_bf16_rounding(lib):
    """One-step RNE to bf16, checked against exact binary arithmetic and
    against torch's float32->bf16 conversion (RNE) for float32 inputs."""
    r = lambda x: int(lib.oracle_double_to_bf16(float(x)))
    # exactly representable values map to themselves
    for bits in (0x3F80, 0xBF80, 0x0000, 0x8000, 0x7F7F, 0x0001, 0x4049):
        x = float(to_floats(np.array([bits], np.uint16))[0])
        assert r(x) == bits, (hex(bits), hex(r(x)))
    # ties go to even: 1 + 2^-8 is halfway between 1 and 1 + 2^-7
    assert r(1.0 + 2.0 ** -8) == 0x3F80
    assert r(1.0 + 3 * 2.0 ** -8) == 0x3F82  # halfway 1+2^-7 / 1+2^-6 -> even
    # just above a tie rounds up even when float32 would have hidden it
    assert r(1.0 + 2.0 ** -8 + 2.0 ** -30) == 0x3F81
    assert r(-(1.0 + 2.0 ** -8 + 2.0 ** -30)) == 0xBF81
    # overflow
    assert r(3.5e38) == 0x7F80 and r(-3.5e38) == 0xFF80
    # agreement with torch on random float32 values
    g = torch.Generator().manual_seed(11)
    x32 = (torch.randn(4096, generator=g) * torch.exp(torch.randn(4096, generator=g) * 8))
    ref = x32.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.round_to_bf16_bits(x32.double().numpy(), lib=lib)
    assert np.array_equal(ref, got)


def pin_brute_force(lib):
    """Tiny batches against the pure-Python brute force: sequences shorter
    and longer than W-1, nonzero state, several W and D, state indices."""
    cases = [
        dict(lengths=[5, 1, 0, 9], Hkv=2, D=8, W=4, state="normal"),
        dict(lengths=[2, 7], Hkv=1, D=16, W=8, state="normal"),
        dict(lengths=[6, 3], Hkv=3, D=4, W=1, state="zero"),
        dict(lengths=[4, 4, 1], Hkv=2, D=8, W=2, state="normal"),
        dict(lengths=[3, 11], Hkv=2, D=8, W=3, state="normal"),
    ]
    for n, cfg in enumerate(cases):
        b = wl.make_prefill(cfg["lengths"], Hkv=cfg["Hkv"], D=cfg["D"],
                            W=cfg["W"], seed=77 + n, state=cfg["state"],
                            page_size=4, spare_pages=3,
                            pool_size=len(cfg["lengths"]) + 2,
                            state_indices=list(range(len(cfg["lengths"]) + 1, 0, -1))[:len(cfg["lengths"])],
                            eps=1e-5)
        out = _run(lib, b)
        T, C = b.num_tokens, b.C
        zk, zv, placement, new_state = brute_step(
            _bits(b.k).reshape(T, C), _bits(b.v).reshape(T, C),
            b.cu_seqlens.numpy(), _bits(b.conv_w_k), _bits(b.conv_w_v),
            b.gamma_k.numpy(), b.gamma_v.numpy(), b.eps,
            _bits(b.conv_state), b.slot_mapping.numpy(),
            b.num_pages * b.page_size, state_indices=b.state_indices.numpy())
        assert np.allclose(out["z_k"], zk, rtol=1e-12, atol=1e-12), n
        assert np.allclose(out["z_v"], zv, rtol=1e-12, atol=1e-12), n
        assert np.array_equal(out["conv_state"], new_state), n
        # placement: every written slot holds the rounded value of its token
        for which, z in (("k_cache", zk), ("v_cache", zv)):
            cache = out[which].reshape(-1, C)
            rounded = oracle.round_to_bf16_bits(z, lib=lib)
            for s in range(cache.shape[0]):
                if s in placement:
                    assert np.array_equal(cache[s], rounded[placement[s]]), (n, s)
                else:
                    assert np.all(cache[s] == wl.SENTINEL_BITS), (n, s)


def pin_conv_is_correlation(lib):
    """Step a2 equals numpy's cross-correlation of (old state ++ x) with the
    taps in 'valid' mode, channel by channel."""
    g = torch.Generator().manual_seed(5)
    for W in (1, 2, 4, 8):
        L, C = 13, 6
        x = _bits(torch.randn(L, C, generator=g).to(torch.bfloat16))
        s = _bits(torch.randn(max(W - 1, 1), C, generator=g).to(torch.bfloat16))
        w = _bits(torch.randn(W, C, generator=g).to(torch.bfloat16))
        y = oracle.conv(x, s[:W - 1] if W > 1 else s, w, lib=lib)
        xf, sf, wf = to_floats(x), to_floats(s[:W - 1]), to_floats(w)
        for c in range(C):
            seq = np.concatenate([sf[:, c], xf[:, c]]) if W > 1 else xf[:, c]
            ref = np.correlate(seq, wf[:, c], mode="valid")
            assert ref.shape == (L,)
            assert np.allclose(y[:, c], ref, rtol=1e-13, atol=1e-13), (W, c)


def pin_impulse(lib):
    """Zero state, x = unit impulse at token t0 in channel c: the conv
    output reproduces the taps in reverse, y[t0+j, c] = w[W-1-j, c], and is
    zero elsewhere.  This fixes which tap meets the current token."""
    g = torch.Generator().manual_seed(9)
    for W in (2, 3, 4, 8):
        L, C, t0 = 20, 5, 6
        w = _bits(torch.randn(W, C, generator=g).to(torch.bfloat16))
        wf = to_floats(w)
        for c in range(C):
            xf = np.zeros((L, C))
            xf[t0, c] = 1.0
            x = oracle.round_to_bf16_bits(xf, lib=lib)
            y = oracle.conv(x, np.zeros((W - 1, C), np.uint16), w, lib=lib)
            exp = np.zeros((L, C))
            for j in range(W):
                exp[t0 + j, c] = wf[W - 1 - j, c]
            assert np.array_equal(y, exp), (W, c)


def pin_w1_is_rmsnorm(lib):
    """W = 1 with tap 1: the step is plain RMSNorm of each head times gamma;
    checked against torch.nn.functional.rms_norm in float64, including a
    small-magnitude input where eps matters."""
    for D, scale, eps in ((64, 1.0, 1e-6), (16, 1e-3, 1e-6), (8, 1.0, 0.25)):
        b = wl.make_prefill([7, 5], Hkv=3, D=D, W=1, seed=3 + D, k_std=scale,
                            eps=eps, page_size=4, spare_pages=1)
        ones = torch.ones(1, b.C).to(torch.bfloat16)
        b.conv_w_k = ones.clone()
        b.conv_w_v = ones.clone()
        out = _run(lib, b)
        for x, gam, z in ((b.k, b.gamma_k, out["z_k"]), (b.v, b.gamma_v, out["z_v"])):
            xd = x.double()
            ref = torch.nn.functional.rms_norm(xd, (D,), weight=gam.double(), eps=eps)
            assert np.allclose(z, ref.reshape(b.num_tokens, -1).numpy(),
                               rtol=1e-12, atol=1e-15), (D, scale, eps)


def pin_constant_row(lib):
    """Closed form: if every channel of a head carries the same y, RMSNorm
    gives y/sqrt(y^2+eps) * gamma[d]; with eps = 0 that is sign(y)*gamma."""
    D, H, W = 16, 2, 3
    C = H * D
    b = wl.make_prefill([6], Hkv=H, D=D, W=W, seed=1, eps=0.0, page_size=8)
    b.k = torch.full((6, H, D), 0.5).to(torch.bfloat16)
    b.v = torch.full((6, H, D), -2.0).to(torch.bfloat16)
    b.conv_w_k = torch.full((W, C), 0.25).to(torch.bfloat16)
    b.conv_w_v = torch.full((W, C), 0.125).to(torch.bfloat16)
    out = _run(lib, b)
    gk, gv = b.gamma_k.double().numpy(), b.gamma_v.double().numpy()
    # zero state: the first W-1 tokens see fewer nonzero rows, but y stays
    # constant over channels, so sign(y)*gamma holds at every token
    assert np.allclose(out["z_k"], np.tile(gk, (6, H)), rtol=1e-15, atol=0)
    assert np.allclose(out["z_v"], -np.tile(gv, (6, H)), rtol=1e-15, atol=0)
    # with eps > 0: y = 0.25*0.5*m (m = number of nonzero rows in window)
    b.eps = 0.01
    out = _run(lib, b)
    for p in range(6):
        m = min(p + 1, W)
        y = 0.25 * 0.5 * m
        exp = y / np.sqrt(y * y + 0.01) * gk
        assert np.allclose(out["z_k"][p], np.tile(exp, H), rtol=1e-14), p


def pin_chunking_invariance(lib):
    """One-shot prefill == random chunking with state carried ==
    token-by-token decode, bit for bit (z, cache bits, final state)."""
    rng = np.random.default_rng(1)
    for W in (1, 2, 4, 8):
        L = 41
        b = wl.make_prefill([L], Hkv=2, D=8, W=W, seed=50 + W, state="normal",
                            page_size=8, spare_pages=2)
        one = _run(lib, b)
        kb, vb = _bits(b.k), _bits(b.v)
        sm = b.slot_mapping.numpy()
        for mode in ("chunks", "tokens"):
            if mode == "tokens":
                cuts = list(range(0, L + 1))
            else:
                cuts = sorted(set([0, L] + list(rng.integers(0, L, size=6))))
            state = _bits(b.conv_state)
            kc, vc = _bits(b.empty_cache()), _bits(b.empty_cache())
            zk = np.zeros_like(one["z_k"])
            zv = np.zeros_like(one["z_v"])
            for a, e in zip(cuts[:-1], cuts[1:]):
                if mode == "tokens":
                    out = oracle.decode(
                        kb[a:e], vb[a:e], _bits(b.conv_w_k), _bits(b.conv_w_v),
                        b.gamma_k.numpy(), b.gamma_v.numpy(), b.eps, state,
                        sm[a:e], kc, vc, lib=lib)
                else:
                    out = oracle.prefill_varlen(
                        kb[a:e], vb[a:e], np.array([0, e - a], np.int32),
                        _bits(b.conv_w_k), _bits(b.conv_w_v),
                        b.gamma_k.numpy(), b.gamma_v.numpy(), b.eps, state,
                        sm[a:e], kc, vc, lib=lib)
                state, kc, vc = out["conv_state"], out["k_cache"], out["v_cache"]
                zk[a:e], zv[a:e] = out["z_k"], out["z_v"]
            assert np.array_equal(zk, one["z_k"]), (W, mode)
            assert np.array_equal(zv, one["z_v"]), (W, mode)
            assert np.array_equal(kc, one["k_cache"]), (W, mode)
            assert np.array_equal(vc, one["v_cache"]), (W, mode)
            assert np.array_equal(state, one["conv_state"]), (W, mode)


def pin_untouched_slots(lib):
    """Slots not named in slot_mapping (and tokens with slot -1) leave the
    cache's sentinel bits alone, in both caches."""
    b = wl.tiny()
    sm = b.slot_mapping.numpy().copy()
    sm[::5] = -1
    out = _run(lib, b, slots=sm)
    C = b.C
    written = set(int(s) for s in sm if s >= 0)
    for which in ("k_cache", "v_cache"):
        cache = out[which].reshape(-1, C)
        for s in range(cache.shape[0]):
            if s in written:
                assert not np.any(cache[s] == wl.SENTINEL_BITS), s
            else:
                assert np.all(cache[s] == wl.SENTINEL_BITS), s


def pin_state_update(lib):
    """The new state is a bit copy of the last W-1 raw rows of
    (old state ++ sequence), including L = 0 and L < W-1."""
    W = 5
    b = wl.make_prefill([0, 1, 3, 4, 9], Hkv=1, D=8, W=W, seed=8,
                        state="normal", page_size=4, spare_pages=1)
    out = _run(lib, b)
    kb, vb = _bits(b.k).reshape(b.num_tokens, -1), _bits(b.v).reshape(b.num_tokens, -1)
    old = _bits(b.conv_state)
    cu = b.cu_seqlens.numpy()
    C = b.C
    for i in range(5):
        a, e = cu[i], cu[i + 1]
        for half, x in enumerate((kb, vb)):
            rows = list(old[i, :, half * C:(half + 1) * C]) + list(x[a:e])
            exp = np.stack(rows[-(W - 1):])
            got = out["conv_state"][i, :, half * C:(half + 1) * C]
            assert np.array_equal(got, exp), (i, half)


def pin_scale_invariance(lib):
    """eps = 0: scaling every input row (and the state) by a power of two
    leaves z bit-identical; by another factor, equal to rounding.  Taps of
    zero give z = 0 when eps > 0."""
    b = wl.make_prefill([9, 4], Hkv=2, D=16, W=4, seed=4, eps=0.0,
                        state="normal", page_size=4, spare_pages=1)
    base = _run(lib, b)
    for alpha, exact in ((4.0, True), (0.125, True), (3.0, False)):
        k = _bits((b.k.float() * alpha).to(torch.bfloat16))
        v = _bits((b.v.float() * alpha).to(torch.bfloat16))
        st = _bits((b.conv_state.float() * alpha).to(torch.bfloat16))
        out = _run(lib, b, k=k, v=v, state=st)
        if exact:
            assert np.array_equal(out["z_k"], base["z_k"]), alpha
            assert np.array_equal(out["z_v"], base["z_v"]), alpha
        else:
            # bf16(3x) != 3*bf16(x) in general: compare against the same
            # rounded inputs scaled back is not possible, so only the
            # scale-free quantity (unit RMS per head) is checked
            for z, g in ((out["z_k"], b.gamma_k), (out["z_v"], b.gamma_v)):
                u = z.reshape(b.num_tokens, b.Hkv, b.D) / g.double().numpy()
                assert np.allclose(np.sqrt((u ** 2).mean(-1)), 1.0, rtol=1e-12)
    b.eps = 1e-6
    b.conv_w_k = torch.zeros_like(b.conv_w_k)
    b.conv_w_v = torch.zeros_like(b.conv_w_v)
    out = _run(lib, b)
    assert np.all(out["z_k"] == 0) and np.all(out["z_v"] == 0)


def pin_page_permutation(lib):
    """Reading the cache back through slot_mapping gives the same rows
    whatever page permutation placed them."""
    b1 = wl.make_prefill([30, 17], Hkv=2, D=8, W=4, seed=12, state="normal",
                         page_size=4, permute_pages=False, spare_pages=3)
    b2 = wl.make_prefill([30, 17], Hkv=2, D=8, W=4, seed=12, state="normal",
                         page_size=4, permute_pages=True, spare_pages=3)
    assert not np.array_equal(b1.slot_mapping.numpy(), b2.slot_mapping.numpy())
    o1, o2 = _run(lib, b1), _run(lib, b2)
    C = b1.C
    for which in ("k_cache", "v_cache"):
        g1 = o1[which].reshape(-1, C)[b1.slot_mapping.numpy()]
        g2 = o2[which].reshape(-1, C)[b2.slot_mapping.numpy()]
        assert np.array_equal(g1, g2)


def pin_errors(lib):
    """Refused inputs: duplicate slot, slot beyond the cache, state index
    beyond the pool, cu_seqlens that is not a partition."""
    b = wl.make_prefill([5, 4], Hkv=1, D=8, W=3, seed=2, page_size=4,
                        spare_pages=2)
    sm = b.slot_mapping.numpy().copy()
    sm[3] = sm[1]
    assert _run(lib, b, slots=sm, check=False)["status"] == -3
    sm = b.slot_mapping.numpy().copy()
    sm[2] = b.num_pages * b.page_size
    assert _run(lib, b, slots=sm, check=False)["status"] == -2
    assert _run(lib, b, cu=np.array([0, 6, 9], np.int32), check=False)["status"] == 0
    assert _run(lib, b, cu=np.array([0, 6, 8], np.int32), check=False)["status"] == -5
    assert _run(lib, b, cu=np.array([0, 7, 5], np.int32), check=False)["status"] == -5
    b.state_indices = torch.tensor([0, 2], dtype=torch.int32)
    assert _run(lib, b, check=False)["status"] == -4


def pin_decode_entry(lib):
    """The decode entry point equals the varlen step with one token per
    sequence, and decode with slot -1 still advances the state."""
    s = wl.decode(seed=44, batch=6, Hkv=2, D=8, W=4, pages_per_seq=2,
                  page_size=8, max_start=4)
    k, v, sm = s.step_inputs(0)
    args = (wl.bits(k), wl.bits(v), wl.bits(s.conv_w_k), wl.bits(s.conv_w_v),
            s.gamma_k.numpy(), s.gamma_v.numpy(), s.eps, wl.bits(s.conv_state))
    sm = sm.numpy().copy()
    sm[2] = -1
    a = oracle.decode(*args, sm, wl.bits(s.empty_cache()), wl.bits(s.empty_cache()), lib=lib)
    d = oracle.decode_direct(*args, sm, wl.bits(s.empty_cache()), wl.bits(s.empty_cache()), lib=lib)
    for key in ("k_cache", "v_cache", "conv_state", "z_k", "z_v"):
        assert np.array_equal(a[key], d[key]), key
    st = a["conv_state"]
    assert np.array_equal(st[2, -1, :s.C], wl.bits(k)[2].reshape(-1))
    assert np.array_equal(st[2, :-1], wl.bits(s.conv_state)[2, 1:])


ALL_PINS = [
    pin_bf16_rounding, pin_brute_force, pin_conv_is_correlation, pin_impulse,
    pin_w1_is_rmsnorm, pin_constant_row, pin_chunking_invariance,
    pin_untouched_slots, pin_state_update, pin_scale_invariance,
    pin_page_permutation, pin_errors, pin_decode_entry,
]


# ------------------------------------------------------------ MXFP8 store pins

def _e4m3_table():
    """All finite E4M3 values by code, built from the format's definition
    (sign, exponent bias 7, 3 mantissa bits, E=15/M=7 is NaN)."""
    vals = {}
    for c in range(256):
        E, M = (c >> 3) & 0xF, c & 7
        if E == 0xF and M == 7:
            continue
        mag = (M / 8.0) * 2.0 ** -6 if E == 0 else (1 + M / 8.0) * 2.0 ** (E - 7)
        vals[c] = -mag if c & 0x80 else mag
    return vals


def pin_e4m3_rounding(lib):
    """E4M3 rounding: nearest value of the code table with ties to the even
    code (brute force), torch's float8_e4m3fn conversion for in-range
    float32 inputs, saturation to +-448, subnormal ties, round trips."""
    table = _e4m3_table()
    pos = sorted((v, c) for c, v in table.items() if v > 0 or c == 0)
    rng = np.random.default_rng(3)
    xs = np.concatenate([rng.standard_normal(3000) * 30, rng.standard_normal(1000) * 1e-2,
                         np.array([v for v, _ in pos]),
                         np.array([(a[0] + b[0]) / 2 for a, b in zip(pos[:-1], pos[1:])])])
    got = oracle.e4m3_from_f64(xs, lib=lib)
    for x, g in zip(xs, got):
        a = abs(x)
        if a >= 448:
            exp = 0x7E
        else:
            best = min(pos, key=lambda vc: (abs(vc[0] - a), vc[1] & 1))
            exp = best[1]
        if x < 0 or (x == 0 and np.signbit(x)):
            exp |= 0x80
        assert int(g) == exp, (x, int(g), exp)
    x32 = (rng.standard_normal(4000) * 50).astype(np.float32)
    x32 = x32[np.abs(x32) < 448]
    ref = torch.from_numpy(x32).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e4m3_from_f64(x32.astype(np.float64), lib=lib), ref)
    assert int(oracle.e4m3_from_f64(np.array([1e9]), lib=lib)[0]) == 0x7E
    assert int(oracle.e4m3_from_f64(np.array([-500.0]), lib=lib)[0]) == 0xFE
    assert int(oracle.e4m3_from_f64(np.array([2.0 ** -10]), lib=lib)[0]) == 0x00  # tie -> even 0
    assert int(oracle.e4m3_from_f64(np.array([3 * 2.0 ** -10]), lib=lib)[0]) == 0x02  # tie -> even 2
    codes = np.array([c for c in table if c != 0x80], np.uint8)
    back = oracle.e4m3_from_f64(oracle.e4m3_to_f64(codes, lib=lib), lib=lib)
    assert np.array_equal(back, codes)


def pin_mx_block(lib):
    """Block scaling: the scale is 2^(floor(log2 amax) - 8) (checked against
    math.frexp), a power-of-two amax maps to 256 (code 0x78), a zero block
    takes the smallest scale, scaling the block by 2^j shifts the scale
    code by j and keeps the element codes, and every element is the E4M3
    rounding of v / 2^s."""
    import math
    rng = np.random.default_rng(4)
    for _ in range(200):
        v = (rng.standard_normal(32) * 10.0 ** rng.uniform(-3, 3)).astype(np.float32)
        codes, scale = oracle.mx_block(v, lib=lib)
        amax = float(np.max(np.abs(v.astype(np.float64))))
        m, e = math.frexp(amax)
        s = max(-127, min(127, (e - 1) - 8))
        assert scale == s + 127, (amax, scale, s)
        assert np.array_equal(codes, oracle.e4m3_from_f64(v.astype(np.float64) * 2.0 ** -s, lib=lib))
        for j in (-3, 2, 7):
            c2, s2 = oracle.mx_block((v.astype(np.float64) * 2.0 ** j).astype(np.float32), lib=lib)
            assert s2 == scale + j and np.array_equal(c2, codes)
    v = np.zeros(32, np.float32)
    v[5] = 2.0 ** 3
    v[6] = -2.0 ** 1
    codes, scale = oracle.mx_block(v, lib=lib)
    assert scale == (3 - 8) + 127 and codes[5] == 0x78 and codes[6] == (0x80 | 0x68)
    codes, scale = oracle.mx_block(np.zeros(32, np.float32), lib=lib)
    assert scale == 0 and not codes.any()
    # the largest element lands in [256, 448]: values in (448, 512) saturate
    v = np.full(32, 1.9, np.float32)
    codes, scale = oracle.mx_block(v, lib=lib)
    assert scale == (0 - 8) + 127 and np.all(codes == 0x7E)


def pin_mxfp8_step(lib):
    """The MXFP8 store writes, for every written slot, head and 32-channel
    block, exactly the block quantisation of the step's normalised values
    rounded to binary32, leaves unnamed slots zero, and updates the state
    like the bf16 step."""
    b = wl.make_prefill([20, 9], Hkv=2, D=64, W=4, seed=61, state="normal",
                        page_size=8, spare_pages=2)
    sm = b.slot_mapping.numpy().copy()
    sm[3] = -1
    out = oracle.prefill_varlen_mxfp8(
        _bits(b.k), _bits(b.v), b.cu_seqlens.numpy(), _bits(b.conv_w_k), _bits(b.conv_w_v),
        b.gamma_k.numpy(), b.gamma_v.numpy(), b.eps, _bits(b.conv_state), sm,
        b.num_pages, b.page_size, lib=lib)
    ref = _run(lib, b, slots=sm)
    assert np.array_equal(out["conv_state"], ref["conv_state"])
    assert np.array_equal(out["z_k"], ref["z_k"]) and np.array_equal(out["z_v"], ref["z_v"])
    H, D = b.Hkv, b.D
    for which in ("k", "v"):
        data = out[f"{which}_data"].reshape(-1, H, D)
        scl = out[f"{which}_scale"].reshape(-1, H, D // 32)
        z = out[f"z_{which}"].reshape(-1, H, D)
        written = np.zeros(data.shape[0], bool)
        for t, slot in enumerate(sm):
            if slot < 0:
                continue
            written[slot] = True
            for h in range(H):
                for blk in range(D // 32):
                    c, s = oracle.mx_block(z[t, h, blk * 32:(blk + 1) * 32].astype(np.float32), lib=lib)
                    assert np.array_equal(data[slot, h, blk * 32:(blk + 1) * 32], c)
                    assert scl[slot, h, blk] == s
        assert not data[~written].any() and not scl[~written].any()


ALL_PINS += [pin_e4m3_rounding, pin_mx_block, pin_mxfp8_step]


# ------------------------------------------------------------ layout variants

def pin_per_head_gamma(lib):
    """Per-head gammas [H, D]: z equals the z of unit gammas times
    Gamma[h, d] exactly (the oracle forms (y * r) * gamma, and y * r * 1.0
    is y * r), for K and V separately; gammas with identical rows equal the
    shared-gamma step bit for bit; the cache store and the state are the
    shared-gamma ones' when the gammas agree."""
    b = wl.make_prefill([19, 6], Hkv=3, D=64, W=4, seed=91, state="normal",
                        page_size=8, spare_pages=1)
    H, D = b.Hkv, b.D
    g = torch.Generator().manual_seed(92)
    Gk = (1 + 0.3 * torch.randn(H, D, generator=g)).numpy().astype(np.float32)
    Gv = (1 + 0.3 * torch.randn(H, D, generator=g)).numpy().astype(np.float32)
    ones = np.ones((H, D), np.float32)

    def run(gk, gv):
        return oracle.prefill_varlen(
            _bits(b.k), _bits(b.v), b.cu_seqlens.numpy(), _bits(b.conv_w_k),
            _bits(b.conv_w_v), gk, gv, b.eps, _bits(b.conv_state), b.slot_mapping.numpy(),
            _bits(b.empty_cache()), _bits(b.empty_cache()), lib=lib)

    per = run(Gk, Gv)
    unit = run(ones, ones)
    T = b.num_tokens
    for z, zu, G in ((per["z_k"], unit["z_k"], Gk), (per["z_v"], unit["z_v"], Gv)):
        want = (zu.reshape(T, H, D) * G[None].astype(np.float64)).reshape(T, H * D)
        assert np.array_equal(z, want)
    g0 = b.gamma_k.numpy().astype(np.float32)
    tiled = run(np.tile(g0, (H, 1)), np.tile(b.gamma_v.numpy().astype(np.float32), (H, 1)))
    shared = run(g0, b.gamma_v.numpy().astype(np.float32))
    for key in ("z_k", "z_v", "k_cache", "v_cache", "conv_state"):
        assert np.array_equal(tiled[key], shared[key]), key


def _ring_to_linear(ring, pos):
    """Rows of the W-1 positions in front of `pos`, oldest first, read from a
    ring in which position p lives in row p mod (W-1) (index permutation)."""
    n = ring.shape[0]
    return np.stack([ring[(pos - n + j) % n] for j in range(n)]) if n else ring.copy()


def pin_ring_state(lib):
    """Ring-buffer state (position p in row p mod (W-1)): for random rings
    and positions, and along chunked and decode chains, the normalised
    values equal those of the linear state obtained by reading the ring in
    position order, bit for bit; afterwards the ring read in the new
    position order equals the linear step's new state; and a call rewrites
    only the rows of its last min(L, W-1) positions."""
    for W, lengths, seed in ((4, [1, 2, 3, 7, 0], 93), (8, [1, 5, 9, 2], 94), (2, [3, 1], 95)):
        n = W - 1
        b = wl.make_prefill(lengths, Hkv=2, D=64, W=W, seed=seed, state="normal",
                            page_size=8, spare_pages=1)
        S = b.num_seqs
        rng = np.random.default_rng(seed)
        pos = rng.integers(0, 50, size=S).astype(np.int64)
        ring = _bits(b.conv_state)
        lin = np.stack([_ring_to_linear(ring[i], pos[i]) for i in range(S)])
        common = (_bits(b.k), _bits(b.v), b.cu_seqlens.numpy(), _bits(b.conv_w_k),
                  _bits(b.conv_w_v), b.gamma_k.numpy(), b.gamma_v.numpy(), b.eps)
        r_ring = oracle.prefill_varlen(*common, ring, b.slot_mapping.numpy(),
                                       _bits(b.empty_cache()), _bits(b.empty_cache()),
                                       state_positions=pos, lib=lib)
        r_lin = oracle.prefill_varlen(*common, lin, b.slot_mapping.numpy(),
                                      _bits(b.empty_cache()), _bits(b.empty_cache()), lib=lib)
        for key in ("z_k", "z_v", "k_cache", "v_cache"):
            assert np.array_equal(r_ring[key], r_lin[key]), (W, key)
        cu = b.cu_seqlens.numpy()
        for i in range(S):
            L = int(cu[i + 1] - cu[i])
            new = r_ring["conv_state"][i]
            assert np.array_equal(_ring_to_linear(new, pos[i] + L), r_lin["conv_state"][i]), (W, i)
            written = {int((pos[i] + q) % n) for q in range(max(0, L - n), L)}
            for row in range(n):
                if row not in written:
                    assert np.array_equal(new[row], ring[i][row]), (W, i, row)
    # a chain: one sequence fed in chunks and decode steps through a ring
    # equals the one-shot linear step
    b = wl.make_prefill([23], Hkv=2, D=64, W=4, seed=96, state="zero", page_size=8,
                        spare_pages=1)
    kb, vb = _bits(b.k), _bits(b.v)
    one = oracle.prefill_varlen(kb, vb, b.cu_seqlens.numpy(), _bits(b.conv_w_k),
                                _bits(b.conv_w_v), b.gamma_k.numpy(), b.gamma_v.numpy(), b.eps,
                                _bits(b.conv_state), b.slot_mapping.numpy(),
                                _bits(b.empty_cache()), _bits(b.empty_cache()), lib=lib)
    ring = _bits(b.conv_state)
    kc, vc = _bits(b.empty_cache()), _bits(b.empty_cache())
    p = 0
    for cut in (5, 1, 1, 7, 1, 8):
        sl = slice(p, p + cut)
        r = oracle.prefill_varlen(kb[sl], vb[sl], np.array([0, cut], np.int32),
                                  _bits(b.conv_w_k), _bits(b.conv_w_v), b.gamma_k.numpy(),
                                  b.gamma_v.numpy(), b.eps, ring, b.slot_mapping.numpy()[sl],
                                  kc, vc, state_positions=np.array([p], np.int64), lib=lib)
        assert np.array_equal(r["z_k"], one["z_k"][sl]) and np.array_equal(r["z_v"], one["z_v"][sl])
        ring, kc, vc = r["conv_state"], r["k_cache"], r["v_cache"]
        p += cut
    assert np.array_equal(kc, one["k_cache"]) and np.array_equal(vc, one["v_cache"])
    assert np.array_equal(_ring_to_linear(ring[0], p), one["conv_state"][0])


ALL_PINS += [pin_per_head_gamma, pin_ring_state]
