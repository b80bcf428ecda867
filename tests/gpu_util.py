"""Helpers for the GPU parity tests: move seeded inputs to the device, run
the C-ABI entry points, run the oracle on the same bytes, compare.

Comparison rules (the stated parity bar):
  - cache placement, untouched slots and conv_state: bit-exact;
  - normalised values: the GPU's bf16 against the oracle's unrounded
    double z, |err| <= max(2e-2, 1e-2*|z|) per element, and the GPU value
    is the correctly rounded one except at near-ties (see assert_close).
"""
import numpy as np
import torch

import oracle
from short_conv_kv_b200 import workloads as wl

ABS_TOL = 2e-2
REL_TOL = 1e-2
REL_FLOOR = 1e-2


def dev(t):
    return None if t is None else t.to("cuda", non_blocking=False)


def f64(bits):
    return oracle.bf16_bits_to_f64(bits)


def assert_close(got_bits, ref, what=""):
    """GPU bf16 bits vs oracle float64 z.

    Primary bar (the stated 2e-2 abs / 1e-2 rel tolerance, read per element
    as |err| <= max(2e-2, 1e-2*|z|): the values are stored in bf16, whose
    half-ulp exceeds 2e-2 once |z| >= 8, so an absolute bound alone would
    fail even for an exactly rounded store; the relative bound governs there).

    Secondary, stricter check: the GPU value equals the correctly rounded
    (RNE) oracle value, except where z lies within fp32 evaluation error of
    the midpoint between two bf16 neighbours (then either neighbour is
    acceptable).  The fp32 path's error is below ~1e-6*|z| + 3e-7, so the
    margin below is 20x that.
    """
    got_bits = np.asarray(got_bits, dtype=np.uint16)
    got = f64(got_bits)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    if got.size == 0:
        return dict(max_abs=0.0, max_rel=0.0, worst=0.0, mismatch=0.0)
    assert np.all(np.isfinite(got)), f"{what}: non-finite GPU values"
    err = np.abs(got - ref)
    bound = np.maximum(ABS_TOL, REL_TOL * np.abs(ref))
    worst = float((err / bound).max())
    big = np.abs(ref) >= REL_FLOOR
    max_rel = float((err[big] / np.abs(ref[big])).max()) if big.any() else 0.0
    assert worst <= 1.0, (f"{what}: error above max(2e-2, 1e-2*|z|): worst ratio {worst}, "
                          f"max abs {err.max()}, max rel {max_rel}")
    rounded = oracle.round_to_bf16_bits(ref)
    mism = got_bits != rounded
    if mism.any():
        g, r, z = got[mism], f64(rounded[mism]), ref[mism]
        mid = 0.5 * (g + r)
        margin = 1e-5 + 2e-5 * np.abs(z)
        far = np.abs(z - mid) > margin
        assert not far.any(), (f"{what}: {int(far.sum())} values differ from the correctly "
                               f"rounded oracle value away from a rounding tie; e.g. z={z[far][:4]}, "
                               f"gpu={g[far][:4]}, rne={r[far][:4]}")
    return dict(max_abs=float(err.max()), max_rel=max_rel, worst=worst,
                mismatch=float(mism.mean()))


def check_cache(gpu_cache_bits, oracle_cache_bits, slot_mapping, z, what=""):
    """Placement + untouched (bitwise, against the oracle's cache) and values
    (tolerance, against the oracle's z) for one cache."""
    C = gpu_cache_bits.shape[-1] * gpu_cache_bits.shape[-2]
    g = gpu_cache_bits.reshape(-1, C)
    o = oracle_cache_bits.reshape(-1, C)
    sm = np.asarray(slot_mapping)
    tok = np.nonzero(sm >= 0)[0]
    written = np.zeros(g.shape[0], bool)
    written[sm[tok]] = True
    assert np.array_equal(g[~written], o[~written]), f"{what}: untouched slots changed"
    return assert_close(g[sm[tok]], z[tok], what)


def run_gpu_prefill(b: wl.Batch, k_cache=None, v_cache=None, state=None, err=None):
    """Run sconv_kv_prefill_varlen on device copies of b; returns device
    caches and state."""
    from short_conv_kv_b200 import binding
    kc = dev(b.empty_cache()) if k_cache is None else k_cache
    vc = dev(b.empty_cache()) if v_cache is None else v_cache
    st = dev(b.conv_state.clone()) if state is None else state
    binding.prefill_varlen(
        dev(b.k), dev(b.v), dev(b.cu_seqlens), dev(b.conv_w_k), dev(b.conv_w_v),
        dev(b.gamma_k), dev(b.gamma_v), b.eps, st, dev(b.slot_mapping), kc, vc,
        state_indices=dev(b.state_indices), err_flag=err)
    torch.cuda.synchronize()
    return kc, vc, st


def oracle_prefill(b: wl.Batch, want_z=True):
    return oracle.prefill_varlen(
        wl.bits(b.k), wl.bits(b.v), b.cu_seqlens.numpy(), wl.bits(b.conv_w_k),
        wl.bits(b.conv_w_v), b.gamma_k.numpy(), b.gamma_v.numpy(), b.eps,
        wl.bits(b.conv_state), b.slot_mapping.numpy(), wl.bits(b.empty_cache()),
        wl.bits(b.empty_cache()),
        state_indices=None if b.state_indices is None else b.state_indices.numpy(),
        want_z=want_z)


def full_parity(b: wl.Batch):
    """Whole-batch GPU vs oracle comparison; returns error stats."""
    kc, vc, st = run_gpu_prefill(b)
    ref = oracle_prefill(b)
    T = b.num_tokens
    sk = check_cache(wl.bits(kc.cpu()), ref["k_cache"], b.slot_mapping.numpy(),
                     ref["z_k"], "k_cache")
    sv = check_cache(wl.bits(vc.cpu()), ref["v_cache"], b.slot_mapping.numpy(),
                     ref["z_v"], "v_cache")
    assert np.array_equal(wl.bits(st.cpu()), ref["conv_state"]), "conv_state differs"
    return sk, sv


def window_states(k_bits, v_bits, cu, state_bits, tokens, W, state_indices=None):
    """For sampled global token indices, the W-1 raw rows that precede each
    token in (old state ++ its sequence), as a [n, W-1, 2C] state block: the
    state the sequence would carry if the token were decoded on its own.
    Pure index gathering from the inputs."""
    T, C = k_bits.shape
    n = len(tokens)
    out = np.zeros((n, max(W - 1, 0), 2 * C), np.uint16)
    seq_of = np.searchsorted(cu, tokens, side="right") - 1
    for r, (t, i) in enumerate(zip(tokens, seq_of)):
        si = i if state_indices is None else state_indices[i]
        p = t - cu[i]
        for j in range(W - 1):
            q = p - (W - 1) + j
            if q >= 0:
                out[r, j, :C] = k_bits[cu[i] + q]
                out[r, j, C:] = v_bits[cu[i] + q]
            else:
                out[r, j] = state_bits[si, W - 1 + q]
    return out


def sampled_oracle_z(k_bits, v_bits, cu, state_bits, tokens, W, wk, wv, gk, gv,
                     eps, H, D, state_indices=None):
    """Oracle z for sampled tokens, each decoded on its own from its window
    state (one oracle decode call over all samples)."""
    tokens = np.asarray(tokens, dtype=np.int64)
    st = window_states(k_bits, v_bits, cu, state_bits, tokens, W, state_indices)
    n = len(tokens)
    kc = np.zeros((n, 1, H, D), np.uint16)
    out = oracle.decode(k_bits[tokens].reshape(n, H, D), v_bits[tokens].reshape(n, H, D),
                        wk, wv, gk, gv, eps, st, np.arange(n, dtype=np.int64),
                        kc, kc.copy())
    return out["z_k"], out["z_v"]


def expected_final_state(k_bits, v_bits, cu, state_bits, W, state_indices=None):
    """New conv_state by index arithmetic: the last W-1 rows of
    (old ++ sequence) for every sequence (a bit copy)."""
    st = state_bits.copy()
    C = k_bits.shape[1]
    for i in range(len(cu) - 1):
        si = i if state_indices is None else state_indices[i]
        L = cu[i + 1] - cu[i]
        if L == 0:
            continue
        old = state_bits[si].copy()
        for j in range(W - 1):
            q = L - (W - 1) + j
            if q >= 0:
                st[si, j, :C] = k_bits[cu[i] + q]
                st[si, j, C:] = v_bits[cu[i] + q]
            else:
                st[si, j] = old[W - 1 + q]
    return st


# ------------------------------------------------------------------ MXFP8 store

MX_SENTINEL = 0xFF


def check_mx(gpu_data, gpu_scale, slot_mapping, z, what=""):
    """GPU MXFP8 caches (uint8 data [P, S, H, D], scales [P, S, H, D/32])
    against the oracle's unrounded z [T, H*D] (double).

    Decisions are taken on z rounded to binary32 on both sides; the GPU's
    binary32 z may differ from the oracle's by a few ulps, so:
      - a block scale must equal the oracle's, or differ by one when the
        block's amax lies within 1e-5 (relative) of the power of two where
        the scale steps;
      - every element code must be the E4M3 rounding of z / 2^s under the
        GPU's scale s, except an adjacent code when z / 2^s lies within
        fp32 evaluation error of the midpoint between the two;
      - slots not in slot_mapping keep the sentinel bytes.
    """
    P, S, H, D = gpu_data.shape
    NB = D // 32
    gd = gpu_data.reshape(P * S, H, D)
    gs = gpu_scale.reshape(P * S, H, NB)
    sm = np.asarray(slot_mapping)
    tok = np.nonzero(sm >= 0)[0]
    written = np.zeros(P * S, bool)
    written[sm[tok]] = True
    assert np.all(gd[~written] == MX_SENTINEL), f"{what}: untouched data changed"
    assert np.all(gs[~written] == MX_SENTINEL), f"{what}: untouched scales changed"
    if tok.size == 0:
        return {}
    zf = np.asarray(z, np.float64)[tok].astype(np.float32).astype(np.float64).reshape(-1, H, NB, 32)
    g_codes = gd[sm[tok]].reshape(-1, H, NB, 32)
    s_g = gs[sm[tok]].astype(np.int64) - 127
    amax = np.abs(zf).max(axis=-1)
    _, e = np.frexp(amax)
    s_o = np.where(amax < 2.0 ** -126, -127, np.clip(e - 1 - 8, -127, 127))
    bad_scale = s_g != s_o
    if bad_scale.any():
        edge = 2.0 ** (np.maximum(s_g, s_o) + 8).astype(np.float64)
        near = (np.abs(s_g - s_o) == 1) & (np.abs(amax - edge) <= 1e-5 * edge)
        assert np.all(near[bad_scale]), (
            f"{what}: {int((bad_scale & ~near).sum())} block scales differ away from a "
            f"power-of-two boundary")
    u = zf * np.exp2(-s_g.astype(np.float64))[..., None]
    exp_codes = oracle.e4m3_from_f64(u)
    mism = g_codes != exp_codes
    if mism.any():
        gv = oracle.e4m3_to_f64(g_codes[mism])
        ev = oracle.e4m3_to_f64(exp_codes[mism])
        uu = u[mism]
        gc = g_codes[mism].astype(np.int64)
        ec = exp_codes[mism].astype(np.int64)
        adjacent = ((gc & 0x80) == (ec & 0x80)) & (np.abs((gc & 0x7F) - (ec & 0x7F)) == 1)
        tiny = (np.abs(gv) <= 2.0 ** -9) & (np.abs(ev) <= 2.0 ** -9)
        scale_mag = np.exp2(-np.broadcast_to(s_g[..., None], u.shape)[mism].astype(np.float64))
        margin = 2e-5 * np.abs(uu) + 1e-6 * scale_mag
        near_tie = np.abs(uu - 0.5 * (gv + ev)) <= margin
        ok = (adjacent | tiny) & near_tie
        assert ok.all(), (f"{what}: {int((~ok).sum())} element codes differ from the E4M3 "
                          f"rounding away from a tie; e.g. u={uu[~ok][:4]}, gpu={gv[~ok][:4]}, "
                          f"rne={ev[~ok][:4]}")
    return dict(scale_mismatch=float(bad_scale.mean()), code_mismatch=float(mism.mean()))


def mx_caches(num_pages, page_size, H, D, device="cuda"):
    """Sentinel-filled MXFP8 data and scale caches."""
    data = torch.full((num_pages, page_size, H, D), MX_SENTINEL, dtype=torch.uint8, device=device)
    scale = torch.full((num_pages, page_size, H, D // 32), MX_SENTINEL, dtype=torch.uint8,
                       device=device)
    return data, scale


def run_gpu_prefill_mx(b: wl.Batch, state=None, err=None):
    from short_conv_kv_b200 import binding
    kd, ks = mx_caches(b.num_pages, b.page_size, b.Hkv, b.D)
    vd, vs = mx_caches(b.num_pages, b.page_size, b.Hkv, b.D)
    st = dev(b.conv_state.clone()) if state is None else state
    binding.prefill_varlen_mxfp8(
        dev(b.k), dev(b.v), dev(b.cu_seqlens), dev(b.conv_w_k), dev(b.conv_w_v),
        dev(b.gamma_k), dev(b.gamma_v), b.eps, st, dev(b.slot_mapping), kd, ks, vd, vs,
        state_indices=dev(b.state_indices), err_flag=err)
    torch.cuda.synchronize()
    return kd, ks, vd, vs, st


def full_parity_mx(b: wl.Batch):
    kd, ks, vd, vs, st = run_gpu_prefill_mx(b)
    ref = oracle_prefill(b)
    sm = b.slot_mapping.numpy()
    rk = check_mx(kd.cpu().numpy(), ks.cpu().numpy(), sm, ref["z_k"], "k mx")
    rv = check_mx(vd.cpu().numpy(), vs.cpu().numpy(), sm, ref["z_v"], "v mx")
    assert np.array_equal(wl.bits(st.cpu()), ref["conv_state"]), "conv_state differs"
    return rk, rv
