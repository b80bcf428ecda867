"""Child process of test_threads_gpu: several host threads call the library
at once, each on its own CUDA stream with its own buffers, in a fresh
process so that the first launch of every kernel instance (and the host
caches that go with it: SM count, shared-memory attribute, scratch
address) happens concurrently.  Every result is then checked against the
oracle.  Exit status 0 = all equal within the stated bounds."""
import sys
import threading

import numpy as np
import torch

import oracle
from short_conv_kv_b200 import binding
from short_conv_kv_b200 import workloads as wl
from tests import gpu_util as gu

# (W, Hkv, D, lengths): a different prefill instance per thread
PREFILL_CASES = [
    (2, 2, 64, [37, 64, 5]),
    (3, 3, 128, [300, 1]),
    (5, 1, 256, [129, 40]),
    (6, 4, 64, [17, 250]),
    (7, 2, 128, [64, 64, 3]),
    (8, 2, 256, [200]),
    (4, 8, 128, [513, 2, 77]),
]
DECODE_CASES = [(4, 4, 128, 96), (2, 2, 64, 40), (8, 1, 256, 33)]  # (W, Hkv, D, batch)
ROUNDS = 3


def run_prefill(i, case, out, barrier):
    W, H, D, lengths = case
    b = wl.make_prefill(lengths, Hkv=H, D=D, W=W, seed=7100 + i, state="normal",
                        page_size=16, spare_pages=2)
    args = [gu.dev(t) for t in (b.k, b.v, b.cu_seqlens, b.conv_w_k, b.conv_w_v,
                                b.gamma_k, b.gamma_v)]
    stream = torch.cuda.Stream()
    res = []
    barrier.wait()
    with torch.cuda.stream(stream):
        for _ in range(ROUNDS):
            kc, vc = gu.dev(b.empty_cache()), gu.dev(b.empty_cache())
            st = gu.dev(b.conv_state.clone())
            binding.prefill_varlen(*args[:7], b.eps, st, gu.dev(b.slot_mapping), kc, vc)
            res.append((kc, vc, st))
    stream.synchronize()
    out[("p", i)] = (b, [(wl.bits(kc.cpu()), wl.bits(vc.cpu()), wl.bits(st.cpu()))
                         for kc, vc, st in res])


def run_decode(i, case, out, barrier):
    W, H, D, B = case
    s = wl.decode(seed=7200 + i, batch=B, Hkv=H, D=D, W=W, pages_per_seq=2, page_size=16,
                  max_start=24)
    k, v, sm = s.step_inputs(0)
    stream = torch.cuda.Stream()
    res = []
    barrier.wait()
    with torch.cuda.stream(stream):
        for _ in range(ROUNDS):
            kc, vc = gu.dev(s.empty_cache()), gu.dev(s.empty_cache())
            st = gu.dev(s.conv_state.clone())
            binding.decode(gu.dev(k), gu.dev(v), gu.dev(s.conv_w_k), gu.dev(s.conv_w_v),
                           gu.dev(s.gamma_k), gu.dev(s.gamma_v), s.eps, st, gu.dev(sm), kc, vc)
            res.append((kc, vc, st))
    stream.synchronize()
    out[("d", i)] = (s, (k, v, sm), [(wl.bits(kc.cpu()), wl.bits(vc.cpu()), wl.bits(st.cpu()))
                                     for kc, vc, st in res])


def main():
    torch.cuda.init()
    out, errors = {}, []
    n = len(PREFILL_CASES) + len(DECODE_CASES)
    barrier = threading.Barrier(n)

    def guarded(fn, *a):
        try:
            fn(*a)
        except BaseException as e:  # reported after the join
            errors.append(repr(e))
            barrier.abort()

    threads = [threading.Thread(target=guarded, args=(run_prefill, i, c, out, barrier))
               for i, c in enumerate(PREFILL_CASES)]
    threads += [threading.Thread(target=guarded, args=(run_decode, i, c, out, barrier))
                for i, c in enumerate(DECODE_CASES)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=240)
    torch.cuda.synchronize()
    if errors or any(t.is_alive() for t in threads):
        print("thread errors:", errors, file=sys.stderr)
        return 1

    for i, _ in enumerate(PREFILL_CASES):
        b, runs = out[("p", i)]
        ref = gu.oracle_prefill(b)
        sm = b.slot_mapping.numpy()
        for kc, vc, st in runs:
            gu.check_cache(kc, ref["k_cache"], sm, ref["z_k"], f"prefill {i} k")
            gu.check_cache(vc, ref["v_cache"], sm, ref["z_v"], f"prefill {i} v")
            assert np.array_equal(st, ref["conv_state"]), f"prefill {i} state"
            # identical inputs, identical bits on every round
            assert np.array_equal(kc, runs[0][0]) and np.array_equal(vc, runs[0][1])
    for i, _ in enumerate(DECODE_CASES):
        s, (k, v, sm), runs = out[("d", i)]
        small = np.zeros((s.batch, 1, s.Hkv, s.D), np.uint16)
        ref = oracle.decode(wl.bits(k), wl.bits(v), wl.bits(s.conv_w_k), wl.bits(s.conv_w_v),
                            s.gamma_k.numpy(), s.gamma_v.numpy(), s.eps, wl.bits(s.conv_state),
                            np.arange(s.batch, dtype=np.int64), small, small.copy())
        slots = sm.numpy()
        for kc, vc, st in runs:
            gu.assert_close(kc.reshape(-1, s.C)[slots], ref["z_k"], f"decode {i} k")
            gu.assert_close(vc.reshape(-1, s.C)[slots], ref["z_v"], f"decode {i} v")
            assert np.array_equal(st, ref["conv_state"]), f"decode {i} state"
    print("threads ok")
    return 0


if __name__ == "__main__":
    sys.exit(main())
