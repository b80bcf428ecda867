"""Write / check the oracle regression fixture ``tiny_oracle.json``.

The pages print no worked numeric example for the ShortConv step, so no
stored value here comes from them.  This fixture is written by this script,
which calls only the oracle, on the seeded tiny workload (2 sequences of 37
and 64 tokens, Hkv=2, D=64, W=4, zero state, 16 x 16-slot paged cache).  It
records SHA-256 digests of the oracle's bf16 caches and new state and a
sample of its unrounded normalised values, so an accidental change of the
oracle's arithmetic shows up as a failing test.  Regenerate only together
with a deliberate, justified change of the oracle:

    python -m tests.golden.make_golden
"""
import hashlib
import json
import os

import numpy as np

import oracle
from short_conv_kv_b200 import workloads as wl

HERE = os.path.dirname(os.path.abspath(__file__))
FIXTURE = os.path.join(HERE, "tiny_oracle.json")
SAMPLE = 64


def _compute(lib=None):
    b = wl.tiny()
    out = oracle.prefill_varlen(
        wl.bits(b.k), wl.bits(b.v), b.cu_seqlens.numpy(), wl.bits(b.conv_w_k),
        wl.bits(b.conv_w_v), b.gamma_k.numpy(), b.gamma_v.numpy(), b.eps,
        wl.bits(b.conv_state), b.slot_mapping.numpy(),
        wl.bits(b.empty_cache()), wl.bits(b.empty_cache()), lib=lib)
    rng = np.random.default_rng(0)
    idx = rng.integers(0, out["z_k"].size, size=SAMPLE)
    h = lambda a: hashlib.sha256(np.ascontiguousarray(a).tobytes()).hexdigest()
    return {
        "workload": "tiny: lengths [37, 64], Hkv=2, D=64, W=4, eps=1e-6, seed 1000",
        "k_cache_sha256": h(out["k_cache"]),
        "v_cache_sha256": h(out["v_cache"]),
        "conv_state_sha256": h(out["conv_state"]),
        "sample_index": idx.tolist(),
        "z_k_sample": [float(x).hex() for x in out["z_k"].reshape(-1)[idx]],
        "z_v_sample": [float(x).hex() for x in out["z_v"].reshape(-1)[idx]],
    }


def write():
    with open(FIXTURE, "w") as f:
        json.dump(_compute(), f, indent=1)
    return FIXTURE


def check(lib=None):
    with open(FIXTURE) as f:
        stored = json.load(f)
    now = _compute(lib)
    for key in ("k_cache_sha256", "v_cache_sha256", "conv_state_sha256",
                "sample_index", "z_k_sample", "z_v_sample"):
        assert stored[key] == now[key], key


if __name__ == "__main__":
    print(write())
