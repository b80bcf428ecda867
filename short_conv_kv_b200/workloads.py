"""Seeded synthetic inputs for the fused ShortConv K/V step.

This module only draws random numbers and lays out index arrays; it holds
none of the step's arithmetic, so the CUDA path and the CPU oracle can both
be fed from it.  Everything is generated on the CPU with
``torch.Generator().manual_seed(seed)`` in a fixed order (k, v, conv_w_k,
conv_w_v, gamma_k, gamma_v, conv_state, lengths, page permutation), so the
two sides see the same bf16 bytes.

Value distributions follow the workloads described for the Inkling ShortConv
step: K and V ~ N(0, 1) rounded to bf16; conv taps ~ N(0, 1/W) rounded to
bf16; gamma = 1 + 0.1 * N(0, 1) in fp32; conv_state zero (fresh sequences)
or N(0, 1) (continuation chunks); slots from a seeded permutation of the
cache's pages, each sequence taking consecutive entries of it.
"""
from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np
import torch

SENTINEL_BITS = 0x7FC1  # a quiet-NaN bf16 payload used to mark unwritten cache


@dataclass
class Batch:
    """One call's worth of inputs (CPU tensors)."""
    W: int
    Hkv: int
    D: int
    eps: float
    k: torch.Tensor            # bf16 [T, Hkv, D]
    v: torch.Tensor            # bf16 [T, Hkv, D]
    cu_seqlens: torch.Tensor   # int32 [S+1]
    conv_w_k: torch.Tensor     # bf16 [W, C]
    conv_w_v: torch.Tensor     # bf16 [W, C]
    gamma_k: torch.Tensor      # fp32 [D]
    gamma_v: torch.Tensor      # fp32 [D]
    conv_state: torch.Tensor   # bf16 [pool, W-1, 2C]
    slot_mapping: torch.Tensor  # int64 [T]
    num_pages: int
    page_size: int
    state_indices: Optional[torch.Tensor] = None  # int32 [S] or None
    meta: dict = field(default_factory=dict)

    @property
    def C(self):
        return self.Hkv * self.D

    @property
    def num_tokens(self):
        return int(self.k.shape[0])

    @property
    def num_seqs(self):
        return int(self.cu_seqlens.shape[0] - 1)

    def empty_cache(self, sentinel=SENTINEL_BITS):
        """A [num_pages, page_size, Hkv, D] bf16 cache filled with a
        sentinel bit pattern, so untouched slots can be checked bitwise."""
        c = torch.full((self.num_pages, self.page_size, self.Hkv, self.D),
                       sentinel, dtype=torch.int16)
        return c.view(torch.bfloat16)


def _bf16_normal(gen, shape, std=1.0):
    x = torch.randn(*shape, generator=gen, dtype=torch.float32)
    if std != 1.0:
        x = x * std
    return x.to(torch.bfloat16)


def _weights(gen, W, Hkv, D):
    C = Hkv * D
    wk = _bf16_normal(gen, (W, C), std=(1.0 / W) ** 0.5)
    wv = _bf16_normal(gen, (W, C), std=(1.0 / W) ** 0.5)
    gk = 1.0 + 0.1 * torch.randn(D, generator=gen, dtype=torch.float32)
    gv = 1.0 + 0.1 * torch.randn(D, generator=gen, dtype=torch.float32)
    return wk, wv, gk, gv


def _state(gen, pool, W, C, init):
    if init == "zero":
        return torch.zeros(pool, W - 1, 2 * C, dtype=torch.bfloat16)
    if init == "normal":
        return _bf16_normal(gen, (pool, W - 1, 2 * C))
    raise ValueError(init)


def pages_for(length, page_size):
    return -(-int(length) // page_size)


def slots_from_pages(lengths, page_lists, page_size, starts=None):
    """Slot of position p of sequence i = page_lists[i][p // page_size] *
    page_size + p % page_size, for p in [start_i, start_i + length_i)."""
    out = []
    for i, (L, pl) in enumerate(zip(lengths, page_lists)):
        s0 = 0 if starts is None else int(starts[i])
        p = np.arange(s0, s0 + int(L), dtype=np.int64)
        pl = np.asarray(pl, dtype=np.int64)
        out.append(pl[p // page_size] * page_size + p % page_size)
    if not out:
        return torch.zeros(0, dtype=torch.int64)
    return torch.from_numpy(np.concatenate(out))


def make_prefill(lengths: List[int], *, Hkv, D, W, seed, eps=1e-6,
                 state="zero", page_size=64, permute_pages=True,
                 spare_pages=0, pool_size=None, state_indices=None,
                 k_std=1.0):
    """A varlen prefill batch.  Sequence i takes the next ceil(L_i/page_size)
    entries of the (optionally permuted) page list."""
    gen = torch.Generator().manual_seed(int(seed))
    C = Hkv * D
    T = int(sum(lengths))
    k = _bf16_normal(gen, (T, Hkv, D), std=k_std)
    v = _bf16_normal(gen, (T, Hkv, D), std=k_std)
    wk, wv, gk, gv = _weights(gen, W, Hkv, D)
    S = len(lengths)
    pool = S if pool_size is None else int(pool_size)
    st = _state(gen, pool, W, C, state)
    npages_used = sum(pages_for(L, page_size) for L in lengths)
    num_pages = npages_used + int(spare_pages)
    if permute_pages:
        perm = torch.randperm(num_pages, generator=gen).numpy()
    else:
        perm = np.arange(num_pages)
    page_lists, at = [], 0
    for L in lengths:
        n = pages_for(L, page_size)
        page_lists.append(perm[at:at + n])
        at += n
    slots = slots_from_pages(lengths, page_lists, page_size)
    cu = torch.zeros(S + 1, dtype=torch.int32)
    if S:
        cu[1:] = torch.cumsum(torch.tensor(lengths, dtype=torch.int64), 0).to(torch.int32)
    si = None if state_indices is None else torch.as_tensor(state_indices, dtype=torch.int32)
    return Batch(W=W, Hkv=Hkv, D=D, eps=eps, k=k, v=v, cu_seqlens=cu,
                 conv_w_k=wk, conv_w_v=wv, gamma_k=gk, gamma_v=gv,
                 conv_state=st, slot_mapping=slots, num_pages=num_pages,
                 page_size=page_size, state_indices=si,
                 meta=dict(lengths=list(map(int, lengths)), seed=int(seed),
                           page_lists=page_lists))


# ------------------------------------------------------------ named workloads

def tiny(seed=1000):
    """2 sequences (37 and 64 tokens), Hkv=2, D=64, W=4, zero state, a
    16-page x 16-slot cache with pages drawn from a seeded permutation."""
    return make_prefill([37, 64], Hkv=2, D=64, W=4, seed=seed, state="zero",
                        page_size=16, permute_pages=True, spare_pages=16 - 7)


def single(seed=2000, T=8192, W=4):
    """One sequence of T tokens, Hkv=8, D=128, zero state, contiguous cache
    (page_size 64, slot = position)."""
    return make_prefill([T], Hkv=8, D=128, W=W, seed=seed, state="zero",
                        page_size=64, permute_pages=False)


def varlen_lengths(seed, n=32, lo=512, hi=8192):
    g = torch.Generator().manual_seed(int(seed) + 7)
    return torch.randint(lo, hi + 1, (n,), generator=g).tolist()


def varlen(seed=3000, n=32, lo=512, hi=8192):
    """n sequences with lengths uniform in [lo, hi], Hkv=8, D=128, W=4,
    N(0,1) initial state (continuation chunks), page_size 64, permuted
    pages plus 64 spare pages."""
    lengths = varlen_lengths(seed, n, lo, hi)
    return make_prefill(lengths, Hkv=8, D=128, W=4, seed=seed, state="normal",
                        page_size=64, permute_pages=True, spare_pages=64)


@dataclass
class DecodeSetup:
    """Fixed part of a multi-step decode workload."""
    W: int
    Hkv: int
    D: int
    eps: float
    batch: int
    conv_w_k: torch.Tensor
    conv_w_v: torch.Tensor
    gamma_k: torch.Tensor
    gamma_v: torch.Tensor
    conv_state: torch.Tensor     # initial state [batch, W-1, 2C]
    num_pages: int
    page_size: int
    page_lists: np.ndarray       # [batch, pages_per_seq]
    start_len: np.ndarray        # [batch] tokens already in the cache
    seed: int

    @property
    def C(self):
        return self.Hkv * self.D

    def step_inputs(self, step):
        """(k, v, slot_mapping) of decode step `step` (seeded by seed+step)."""
        gen = torch.Generator().manual_seed(self.seed + 1 + int(step))
        k = _bf16_normal(gen, (self.batch, self.Hkv, self.D))
        v = _bf16_normal(gen, (self.batch, self.Hkv, self.D))
        pos = self.start_len.astype(np.int64) + int(step)
        pages = self.page_lists[np.arange(self.batch), pos // self.page_size]
        slots = pages.astype(np.int64) * self.page_size + pos % self.page_size
        return k, v, torch.from_numpy(slots)

    def empty_cache(self, sentinel=SENTINEL_BITS):
        c = torch.full((self.num_pages, self.page_size, self.Hkv, self.D),
                       sentinel, dtype=torch.int16)
        return c.view(torch.bfloat16)


def decode(seed=4000, batch=1024, Hkv=8, D=128, W=4, pages_per_seq=4,
           page_size=64, max_start=192, eps=1e-6, state="normal"):
    """batch sequences, one new token each per step; N(0,1) state; sequence
    i owns pages perm[4i:4i+4] of a (batch*4)-page cache and starts at a
    seeded length in [0, max_start)."""
    gen = torch.Generator().manual_seed(int(seed))
    wk, wv, gk, gv = _weights(gen, W, Hkv, D)
    st = _state(gen, batch, W, Hkv * D, state)
    num_pages = batch * pages_per_seq
    perm = torch.randperm(num_pages, generator=gen).numpy()
    start = torch.randint(0, max_start, (batch,), generator=gen).numpy()
    return DecodeSetup(W=W, Hkv=Hkv, D=D, eps=eps, batch=batch, conv_w_k=wk,
                       conv_w_v=wv, gamma_k=gk, gamma_v=gv, conv_state=st,
                       num_pages=num_pages, page_size=page_size,
                       page_lists=perm.reshape(batch, pages_per_seq),
                       start_len=start, seed=int(seed))


@dataclass
class LongSetup:
    """One long sequence processed in fixed-size chunks with the state
    carried between calls.  Chunk c's k/v come from generator seed+1+c so a
    chunk can be regenerated on its own."""
    W: int
    Hkv: int
    D: int
    eps: float
    total: int
    chunk: int
    conv_w_k: torch.Tensor
    conv_w_v: torch.Tensor
    gamma_k: torch.Tensor
    gamma_v: torch.Tensor
    num_pages: int
    page_size: int
    perm: np.ndarray
    seed: int

    @property
    def C(self):
        return self.Hkv * self.D

    @property
    def num_chunks(self):
        return -(-self.total // self.chunk)

    def chunk_inputs(self, c):
        """(k, v, slot_mapping, cu_seqlens) of chunk c."""
        t0 = c * self.chunk
        L = min(self.chunk, self.total - t0)
        gen = torch.Generator().manual_seed(self.seed + 1 + int(c))
        k = _bf16_normal(gen, (L, self.Hkv, self.D))
        v = _bf16_normal(gen, (L, self.Hkv, self.D))
        p = np.arange(t0, t0 + L, dtype=np.int64)
        slots = self.perm[p // self.page_size].astype(np.int64) * self.page_size + p % self.page_size
        cu = torch.tensor([0, L], dtype=torch.int32)
        return k, v, torch.from_numpy(slots), cu

    def initial_state(self):
        return torch.zeros(1, self.W - 1, 2 * self.C, dtype=torch.bfloat16)

    def empty_cache(self, sentinel=SENTINEL_BITS):
        c = torch.full((self.num_pages, self.page_size, self.Hkv, self.D),
                       sentinel, dtype=torch.int16)
        return c.view(torch.bfloat16)


def long_context(seed=5000, total=1 << 20, chunk=1 << 16, Hkv=8, D=128, W=4,
                 page_size=64, spare_pages=64, eps=1e-6):
    """One sequence of `total` tokens in `chunk`-token calls, zero initial
    state, seeded page permutation (+ spare pages)."""
    gen = torch.Generator().manual_seed(int(seed))
    wk, wv, gk, gv = _weights(gen, W, Hkv, D)
    num_pages = pages_for(total, page_size) + spare_pages
    perm = torch.randperm(num_pages, generator=gen).numpy()
    return LongSetup(W=W, Hkv=Hkv, D=D, eps=eps, total=total, chunk=chunk,
                     conv_w_k=wk, conv_w_v=wv, gamma_k=gk, gamma_v=gv,
                     num_pages=num_pages, page_size=page_size, perm=perm,
                     seed=int(seed))


# ------------------------------------------------------------ conversions

def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> numpy uint16 bit patterns (C-contiguous copy)."""
    assert t.dtype == torch.bfloat16
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16).copy()


def from_bits(a: np.ndarray) -> torch.Tensor:
    """numpy uint16 bit patterns -> bf16 tensor."""
    a = np.ascontiguousarray(a, dtype=np.uint16)
    return torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16)
