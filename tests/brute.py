"""Brute-force restatement of the fused ShortConv K/V step, pure Python.

Used only to pin the oracle on tiny inputs.  It is written in a different
form from the oracle on purpose: the window is built by concatenating the
old state rows in front of the sequence's rows and sliding over that list,
sums are exact (math.fsum) before one rounding to float64, and the new state
is the tail of the concatenated list.  Sources: causal conv over tokens
(aib.vote news item, paragraph 1), current token plus previous W-1 states
(axbrief.com, SConv section), conv -> normalisation -> cache write
(aib.vote, paragraph 2), per-request state pool (Inkling-Small cookbook,
section 2).
"""
import math

import numpy as np


def to_floats(bits_array):
    a = np.asarray(bits_array, dtype=np.uint16)
    return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def brute_step(k, v, cu, wk, wv, gk, gv, eps, state, slots, num_slots,
               state_indices=None):
    """Inputs as numpy (bf16 as uint16 bits).  k, v: [T, C]; state:
    [pool, W-1, 2C].  Returns (zk, zv, placement, new_state): z* float64
    [T, C]; placement maps slot -> token; new_state uint16 like `state`."""
    kf, vf = to_floats(k), to_floats(v)
    T, C = kf.shape
    W = wk.shape[0]
    D = len(gk)
    H = C // D
    wkf, wvf = to_floats(wk), to_floats(wv)
    state = np.array(state, dtype=np.uint16, copy=True)
    new_state = state.copy()
    zk = np.zeros((T, C))
    zv = np.zeros((T, C))
    placement = {}
    S = len(cu) - 1
    n = W - 1
    for i in range(S):
        a, b = int(cu[i]), int(cu[i + 1])
        si = i if state_indices is None else int(state_indices[i])
        for half, (xf, xb, wf, g, z) in enumerate(
                ((kf, k, wkf, gk, zk), (vf, v, wvf, gv, zv))):
            c0 = half * C
            old_bits = [state[si, r, c0:c0 + C] for r in range(n)]
            padded = [to_floats(r) for r in old_bits] + [xf[t] for t in range(a, b)]
            for p in range(b - a):
                window = padded[p:p + W]           # W rows ending at token p
                y = [math.fsum(wf[j, c] * window[j][c] for j in range(W))
                     for c in range(C)]
                for h in range(H):
                    seg = y[h * D:(h + 1) * D]
                    ms = math.fsum(t * t for t in seg) / D
                    r = 1.0 / math.sqrt(ms + eps)
                    for d in range(D):
                        z[a + p, h * D + d] = seg[d] * r * float(g[d])
            # new state = the last n raw rows of (old ++ new)
            rows_bits = old_bits + [np.asarray(xb[t]) for t in range(a, b)]
            tail = rows_bits[len(rows_bits) - n:] if n > 0 else []
            for r in range(n):
                new_state[si, r, c0:c0 + C] = tail[r]
        for p in range(b - a):
            s = int(slots[a + p])
            if s >= 0:
                assert s < num_slots
                assert s not in placement, "duplicate slot"
                placement[s] = a + p
    return zk, zv, placement, new_state
