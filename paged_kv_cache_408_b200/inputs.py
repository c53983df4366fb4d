"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle checks.

This module only draws random numbers and lays them out in the documented
formats; it holds none of the attention, quantisation or allocation
arithmetic.  Every array is numpy, on the host:

* bf16 tensors are ``uint16`` bit patterns (float32 N(0,1) draws rounded to
  nearest-even bf16 by torch's own conversion);
* fp8 caches are ``uint8`` E4M3 codes produced by torch's
  ``float8_e4m3fn`` conversion of ``x / scale`` with a per-head scale
  ``amax / 448`` over that head's draws;
* caches are ``[num_blocks, Hkv, 16, D]``; block tables are int32
  ``[B, max_blocks]`` padded with -1; seq_lens int32 ``[B]``; slot mappings
  int64 ``[T]``.

Physical blocks are handed out from a seeded random permutation of the pool,
so logically adjacent blocks are scattered in memory, as in a pool that has
served many requests ("Production Serving: Continuous Batching and
PagedAttention", PagedAttention, the thing you build for memory: pages need
not be contiguous).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

BLOCK_SIZE = 16
FP8_MAX = 448.0


def _torch():
    import torch
    return torch


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 array -> bf16 bit patterns (uint16), nearest-even, via torch."""
    torch = _torch()
    t = torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bf16_values(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float32 values (exact widening, via torch)."""
    torch = _torch()
    t = torch.from_numpy(np.ascontiguousarray(bits, np.uint16).view(np.int16)).view(torch.bfloat16)
    return t.float().numpy()


def normal_bf16(rng: np.random.Generator, shape) -> np.ndarray:
    return bf16_bits(rng.standard_normal(shape, dtype=np.float32))


def fp8_cache_from_normal(rng: np.random.Generator, shape):
    """Draw N(0,1) values for a cache [nb, Hkv, 16, D]; choose per-head scale
    amax/448 and return (codes uint8, scale float32 [Hkv]) using torch's
    float8_e4m3fn conversion."""
    torch = _torch()
    x = rng.standard_normal(shape, dtype=np.float32)
    amax = np.abs(x).max(axis=(0, 2, 3))
    scale = (amax / FP8_MAX).astype(np.float32)
    scale[scale == 0] = 1.0
    xt = torch.from_numpy(x) / torch.from_numpy(scale).view(1, -1, 1, 1)
    codes = xt.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    return codes, scale


def blocks_for(n_tokens: int) -> int:
    return (n_tokens + BLOCK_SIZE - 1) // BLOCK_SIZE


def assign_block_tables(seq_lens, perm, max_blocks=None, reserve_extra_token=False):
    """Hand out blocks from ``perm`` in order to each sequence; returns
    (block_tables int32 [B, max_blocks] padded with -1, number of blocks used).
    ``reserve_extra_token`` sizes each table for len+1 tokens."""
    lens = np.asarray(seq_lens, np.int64)
    need = np.array([blocks_for(int(n) + (1 if reserve_extra_token else 0)) for n in lens], np.int64)
    mb = int(max_blocks) if max_blocks is not None else int(max(1, need.max(initial=1)))
    if need.sum() > len(perm):
        raise ValueError("pool too small for the requested sequences")
    bt = np.full((len(lens), mb), -1, np.int32)
    pos = 0
    for i, n in enumerate(need):
        bt[i, :n] = perm[pos:pos + n]
        pos += n
    return bt, int(pos)


@dataclass
class DecodeCase:
    """Inputs of one paged-decode call (plus, optionally, one write)."""
    name: str
    q: np.ndarray             # uint16 [B, Hq, D]
    k_cache: np.ndarray       # uint16 or uint8 [nb, Hkv, 16, D]
    v_cache: np.ndarray
    block_tables: np.ndarray  # int32 [B, max_blocks]
    seq_lens: np.ndarray      # int32 [B]
    scale: float
    k_scale: np.ndarray | None = None  # float32 [Hkv] for fp8
    v_scale: np.ndarray | None = None
    # optional write of new tokens before the decode
    new_k: np.ndarray | None = None    # uint16 [T, Hkv, D]
    new_v: np.ndarray | None = None
    slot_mapping: np.ndarray | None = None  # int64 [T]
    extra: dict = field(default_factory=dict)

    @property
    def B(self):
        return self.q.shape[0]

    @property
    def Hq(self):
        return self.q.shape[1]

    @property
    def Hkv(self):
        return self.k_cache.shape[1]

    @property
    def D(self):
        return self.k_cache.shape[3]

    @property
    def num_blocks(self):
        return self.k_cache.shape[0]

    @property
    def fp8(self):
        return self.k_cache.dtype == np.uint8


def new_token_slots(block_tables, positions):
    """Slot of the token at logical ``positions[b]`` of each sequence (the
    mapping a host allocator hands the write kernel)."""
    bt = np.asarray(block_tables)
    pos = np.asarray(positions, np.int64)
    phys = bt[np.arange(len(pos)), pos // BLOCK_SIZE].astype(np.int64)
    return phys * BLOCK_SIZE + pos % BLOCK_SIZE


def make_decode_case(seed, seq_lens, Hq, Hkv, D, num_blocks=None, fp8=False, pool_factor=1.1, name="decode",
                     with_write=False, max_blocks=None, fill_cache=True):
    """Generic decode case.  ``seq_lens`` are the lengths *after* the optional
    write of one new token per sequence (the write lands at position len-1)."""
    rng = np.random.default_rng(seed)
    lens = np.asarray(seq_lens, np.int32)
    need = int(sum(blocks_for(int(n)) for n in lens))
    nb = int(num_blocks) if num_blocks is not None else max(1, int(math.ceil(pool_factor * need)))
    perm = rng.permutation(nb).astype(np.int32)
    bt, _ = assign_block_tables(lens, perm, max_blocks=max_blocks)
    B = len(lens)
    q = normal_bf16(rng, (B, Hq, D))
    shape = (nb, Hkv, BLOCK_SIZE, D)
    ks = vs = None
    if fp8:
        kc, ks = fp8_cache_from_normal(rng, shape)
        vc, vs = fp8_cache_from_normal(rng, shape)
    elif fill_cache:
        kc = normal_bf16(rng, shape)
        vc = normal_bf16(rng, shape)
    else:
        kc = np.zeros(shape, np.uint16)
        vc = np.zeros(shape, np.uint16)
    case = DecodeCase(name, q, kc, vc, bt, lens, 1.0 / math.sqrt(D), ks, vs)
    if with_write:
        case.new_k = normal_bf16(rng, (B, Hkv, D))
        case.new_v = normal_bf16(rng, (B, Hkv, D))
        case.slot_mapping = new_token_slots(bt, np.maximum(lens.astype(np.int64) - 1, 0))
        case.slot_mapping[lens <= 0] = -1
    return case


# ------------------------------------------------------------------ workloads
# The five workloads: sizes, distributions and structure.

def tiny_decode(seed=0) -> DecodeCase:
    """4 sequences with 5/17/33/48 stored tokens, 4 q heads / 4 kv heads,
    head_dim 64, a 32-block pool handed out by a seeded permutation, q/K/V
    bf16 N(0,1), scale 1/8, plus one new token per sequence written through
    a slot mapping (post-write lengths 6/18/34/49)."""
    return make_decode_case(seed, [6, 18, 34, 49], 4, 4, 64, num_blocks=32, name="tiny 4 seqs, 4/4 heads, d64",
                            with_write=True)


def batch64_2k(seed=0, fixed_len=None) -> DecodeCase:
    """64 sequences, lengths uniform in [1, 2048] (or all ``fixed_len``),
    32 q heads / 8 kv heads, head_dim 128, bf16, pool 1.1x the blocks needed,
    permuted block tables."""
    rng = np.random.default_rng(10_000 + seed)
    lens = np.full(64, fixed_len, np.int32) if fixed_len else rng.integers(1, 2049, 64).astype(np.int32)
    return make_decode_case(seed, lens, 32, 8, 128, name="64 seqs x U[1,2048], 32/8 heads, d128, bf16",
                            with_write=True)


def long_context(seed=0, n_seqs=16, seq_len=32768, num_blocks=40960) -> DecodeCase:
    """16 sequences of 32768 tokens, 32/8 heads, head_dim 128, bf16, blocks
    scattered over a 40960-block pool."""
    return make_decode_case(seed, [seq_len] * n_seqs, 32, 8, 128, num_blocks=num_blocks,
                            name=f"{n_seqs} seqs x {seq_len}, 32/8 heads, d128, bf16")


def lognormal_lengths(rng, n, median=1024, sigma=1.0, cap=8192):
    x = rng.lognormal(math.log(median), sigma, n)
    return np.clip(np.round(x), 1, cap).astype(np.int32)


@dataclass
class PrefillCase:
    name: str
    q: np.ndarray            # uint16 [sum C, Hq, D]
    cu_q: np.ndarray         # int32 [n+1]
    prefix_lens: np.ndarray  # int32 [n]
    block_tables: np.ndarray  # int32 [n, max_blocks]
    k_cache: np.ndarray
    v_cache: np.ndarray
    scale: float
    new_k: np.ndarray        # uint16 [sum C, Hkv, D] -- the chunks' own K/V
    new_v: np.ndarray
    slot_mapping: np.ndarray  # int64 [sum C]
    k_scale: np.ndarray | None = None
    v_scale: np.ndarray | None = None

    @property
    def Hq(self):
        return self.q.shape[1]

    @property
    def Hkv(self):
        return self.k_cache.shape[1]

    @property
    def D(self):
        return self.k_cache.shape[3]

    @property
    def chunk_lens(self):
        return np.diff(self.cu_q)

    @property
    def max_q_len(self):
        return int(self.chunk_lens.max(initial=0))


def make_prefill_case(seed, chunk_lens, prefix_lens, Hq, Hkv, D, num_blocks=None, pool_factor=1.1,
                      name="prefill", fp8=False):
    """Chunks with the given lengths over existing prefixes.  The prefix
    tokens are already in the cache (random N(0,1) contents; with ``fp8`` as
    E4M3 codes with per-head scales amax/448); the chunks' own K/V come as
    new bf16 tokens with their slot mapping (write them first)."""
    rng = np.random.default_rng(seed)
    cl = np.asarray(chunk_lens, np.int32)
    pl = np.asarray(prefix_lens, np.int32)
    tot = (cl + pl).astype(np.int64)
    need = int(sum(blocks_for(int(n)) for n in tot))
    nb = int(num_blocks) if num_blocks is not None else max(1, int(math.ceil(pool_factor * need)))
    perm = rng.permutation(nb).astype(np.int32)
    bt, _ = assign_block_tables(tot, perm)
    cu = np.zeros(len(cl) + 1, np.int32)
    cu[1:] = np.cumsum(cl)
    total = int(cu[-1])
    q = normal_bf16(rng, (total, Hq, D))
    shape = (nb, Hkv, BLOCK_SIZE, D)
    ks = vs = None
    if fp8:
        kc, ks = fp8_cache_from_normal(rng, shape)
        vc, vs = fp8_cache_from_normal(rng, shape)
    else:
        kc = normal_bf16(rng, shape)
        vc = normal_bf16(rng, shape)
    nk = normal_bf16(rng, (total, Hkv, D))
    nv = normal_bf16(rng, (total, Hkv, D))
    pos = np.concatenate([np.arange(pl[c], pl[c] + cl[c], dtype=np.int64) for c in range(len(cl))]) \
        if total else np.zeros(0, np.int64)
    rows = np.repeat(np.arange(len(cl)), cl)
    slots = bt[rows, pos // BLOCK_SIZE].astype(np.int64) * BLOCK_SIZE + pos % BLOCK_SIZE
    return PrefillCase(name, q, cu, pl, bt, kc, vc, 1.0 / math.sqrt(D), nk, nv, slots, ks, vs)


def mixed_step(seed=0, n_decode=192, n_chunks=8, chunk=512):
    """192 decode sequences (lognormal lengths, median 1024, sigma 1, capped
    at 8192; block tables 512 entries wide, the cap) plus 8 prefill chunks
    of 512 tokens over prefixes uniform in [0, 4096]; 32/8 heads, head_dim
    128, bf16.  Returned as two separate cases (each with its own pool); the
    scheduler-driven mixed trace runs both halves on one pool."""
    rng = np.random.default_rng(20_000 + seed)
    dec_lens = lognormal_lengths(rng, n_decode)
    prefixes = rng.integers(0, 4097, n_chunks).astype(np.int32)
    dec = make_decode_case(seed, dec_lens, 32, 8, 128, name="mixed: 192 decode seqs", with_write=True,
                           max_blocks=blocks_for(8192))
    pre = make_prefill_case(seed + 1, [chunk] * n_chunks, prefixes, 32, 8, 128,
                            name="mixed: 8 chunks x 512 over U[0,4096] prefixes")
    return dec, pre


def mixed_step_prefill(seed=0, n_decode=192, n_chunks=8, chunk=512, fp8=False):
    """The prefill half of ``mixed_step(seed)`` alone (the same chunk
    prefixes), without drawing its decode half's cache; with ``fp8`` the
    same chunks over an E4M3 cache drawn from another seed."""
    rng = np.random.default_rng(20_000 + seed)
    lognormal_lengths(rng, n_decode)  # the decode lengths come first in mixed_step's draw order
    prefixes = rng.integers(0, 4097, n_chunks).astype(np.int32)
    if fp8:
        return make_prefill_case(seed + 543, [chunk] * n_chunks, prefixes, 32, 8, 128, fp8=True,
                                 name="8 chunks x 512 over U[0,4096] prefixes, fp8")
    return make_prefill_case(seed + 1, [chunk] * n_chunks, prefixes, 32, 8, 128,
                             name="mixed: 8 chunks x 512 over U[0,4096] prefixes")


def prefix_share(seed=0, n_seqs=256, prefix=2048, suffix_lo=16, suffix_hi=512, Hq=64, Hkv=8, D=128, fp8=True):
    """256 sequences sharing one 2048-token prefix (the same physical blocks)
    plus per-sequence suffixes uniform in [16, 512]; 64/8 heads, head_dim
    128; fp8 E4M3 cache with per-head fp32 scales (bf16 with ``fp8=False``).
    A prefix that is not a whole number of blocks shares its partial last
    block too (the block table entry), as a forked sequence does before its
    first write."""
    rng = np.random.default_rng(30_000 + seed)
    suf = rng.integers(suffix_lo, suffix_hi + 1, n_seqs).astype(np.int32)
    pre_blocks = blocks_for(prefix)
    suf_blocks = np.array([blocks_for(prefix + int(s)) - pre_blocks for s in suf])
    need = pre_blocks + int(suf_blocks.sum())
    nb = int(math.ceil(1.1 * need)) + 64
    perm = rng.permutation(nb).astype(np.int32)
    shared = perm[:pre_blocks]
    mb = pre_blocks + int(suf_blocks.max())
    bt = np.full((n_seqs, mb), -1, np.int32)
    pos = pre_blocks
    for i in range(n_seqs):
        bt[i, :pre_blocks] = shared
        bt[i, pre_blocks:pre_blocks + suf_blocks[i]] = perm[pos:pos + suf_blocks[i]]
        pos += suf_blocks[i]
    lens = (prefix + suf).astype(np.int32)
    q = normal_bf16(rng, (n_seqs, Hq, D))
    if fp8:
        kc, ks = fp8_cache_from_normal(rng, (nb, Hkv, BLOCK_SIZE, D))
        vc, vs = fp8_cache_from_normal(rng, (nb, Hkv, BLOCK_SIZE, D))
    else:
        kc = normal_bf16(rng, (nb, Hkv, BLOCK_SIZE, D))
        vc = normal_bf16(rng, (nb, Hkv, BLOCK_SIZE, D))
        ks = vs = None
    case = DecodeCase(f"{n_seqs} seqs sharing a {prefix}-token prefix, {Hq}/{Hkv} heads, d{D}, "
                      f"{'fp8' if fp8 else 'bf16'}", q, kc, vc, bt, lens, 1.0 / math.sqrt(D), ks, vs)
    case.extra["free_blocks"] = perm[pos:].copy()
    case.extra["shared_blocks"] = shared.copy()
    return case


# ------------------------------------------------------- trace randomness
def geometric_steps(rng, n, p=1.0 / 256):
    """Remaining decode steps of newly admitted sequences (mean 1/p)."""
    return rng.geometric(p, n).astype(np.int64)


def uniform_lengths(rng, n, lo=1, hi=2048):
    return rng.integers(lo, hi + 1, n).astype(np.int64)
