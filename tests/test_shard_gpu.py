"""The multi-GPU data path on one GPU: a varlen batch split by
shard.partition_sequences, each rank's shard.local_view (its rows of k/v
and slot_mapping, a rebased cu_seqlens, explicit state indices into the
shared pool) run through the CUDA entry point into one shared pool and
cache.  The union must equal the whole-batch oracle: the state and the
cache placement bit for bit, values within the stated tolerance.  With
several GPUs each view runs on its own rank; nothing crosses between
ranks, so running the views one after another on one GPU exercises the
same kernels on the same arguments."""
import numpy as np
import pytest
import torch

from short_conv_kv_b200 import shard, workloads as wl
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield
    torch.cuda.synchronize()


@pytest.mark.parametrize("world", [2, 3, 8])
def test_sharded_views_equal_whole_batch(world):
    from short_conv_kv_b200 import binding as bd
    lengths = [5, 700, 0, 333, 2, 41, 1290, 18, 77, 3, 512, 64]
    b = wl.make_prefill(lengths, Hkv=4, D=128, W=4, seed=3100 + world, state="normal",
                        page_size=16, spare_pages=3, pool_size=len(lengths) + 5,
                        state_indices=list(np.random.default_rng(world).permutation(
                            len(lengths) + 5)[:len(lengths)]))
    kc, vc = gu.dev(b.empty_cache()), gu.dev(b.empty_cache())
    st = gu.dev(b.conv_state.clone())
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    w = [gu.dev(t) for t in (b.conv_w_k, b.conv_w_v, b.gamma_k, b.gamma_v)]
    for part in shard.partition_sequences(lengths, world):
        local = shard.local_view(b, part)
        if local.num_seqs == 0:
            continue
        bd.prefill_varlen(gu.dev(local.k), gu.dev(local.v), gu.dev(local.cu_seqlens), *w,
                          local.eps, st, gu.dev(local.slot_mapping), kc, vc,
                          state_indices=gu.dev(local.state_indices), err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    ref = gu.oracle_prefill(b)
    sm = b.slot_mapping.numpy()
    gu.check_cache(wl.bits(kc.cpu()), ref["k_cache"], sm, ref["z_k"], "k_cache")
    gu.check_cache(wl.bits(vc.cpu()), ref["v_cache"], sm, ref["z_v"], "v_cache")
    assert np.array_equal(wl.bits(st.cpu()), ref["conv_state"])
