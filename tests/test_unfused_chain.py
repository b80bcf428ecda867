"""The bench's unfused torch-op chain (context for the fusion speed-up) must
compute the same step as the oracle, or its timing compares unlike work.
Stock torch ops run on the CPU too, so this needs no GPU."""
import numpy as np
import pytest
import torch

import bench
from short_conv_kv_b200 import workloads as wl
from tests import gpu_util as gu


def _run_chain(b):
    chain = bench.UnfusedChain(b.cu_seqlens.diff().tolist(), b.W, b.Hkv, b.D, "cpu")
    a = dict(k=b.k.clone(), v=b.v.clone(), conv_state=b.conv_state.clone(),
             conv_w_k=b.conv_w_k, conv_w_v=b.conv_w_v, gamma_k=b.gamma_k,
             gamma_v=b.gamma_v, eps=b.eps, slot_mapping=b.slot_mapping,
             k_cache=b.empty_cache(), v_cache=b.empty_cache())
    chain(a)
    return a


@pytest.mark.parametrize("lengths,W", [([37, 64], 4), ([5, 1, 2, 40], 2), ([9, 3], 1),
                                       ([1, 1, 1, 1], 4), ([2, 70, 1], 8)])
def test_unfused_chain_matches_oracle(lengths, W):
    b = wl.make_prefill(lengths, Hkv=2, D=64, W=W, seed=2400 + W + len(lengths),
                        state="normal", page_size=16, spare_pages=2)
    a = _run_chain(b)
    ref = gu.oracle_prefill(b)
    sm = b.slot_mapping.numpy()
    gu.check_cache(wl.bits(a["k_cache"]), ref["k_cache"], sm, ref["z_k"], "chain k")
    gu.check_cache(wl.bits(a["v_cache"]), ref["v_cache"], sm, ref["z_v"], "chain v")
    assert np.array_equal(wl.bits(a["conv_state"]), ref["conv_state"])


def test_unfused_chain_decode_shape():
    """One token per sequence (the decode workload's shape)."""
    b = wl.make_prefill([1] * 12, Hkv=2, D=128, W=4, seed=2450, state="normal",
                        page_size=16, spare_pages=1)
    a = _run_chain(b)
    ref = gu.oracle_prefill(b)
    sm = b.slot_mapping.numpy()
    gu.check_cache(wl.bits(a["k_cache"]), ref["k_cache"], sm, ref["z_k"], "chain k")
    assert np.array_equal(wl.bits(a["conv_state"]), ref["conv_state"])
