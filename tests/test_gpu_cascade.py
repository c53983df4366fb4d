"""GPU parity of cascade decode (pa_decode_cascade) against the fp64 oracle.

Cascade decode computes exactly what paged decode computes ("Production
Serving: Continuous Batching and PagedAttention", Step 6): softmax over every
cached token of each sequence.  Its inputs are batches whose rows all begin
with the same physical blocks (forked sequences, "Continuous batching and
PagedAttention", PagedAttention: KV cache memory); the shared blocks are
attended once per kv head on the tensor cores, the rest by the decode kernel,
and the pieces merged.  So the oracle is plain ``oracle.decode`` on the same
tables, and outputs must be within the decode tolerance (max-abs 1e-2,
mean-abs 1e-3)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_attn_close, cache_to_device, dev, dev_bf16, to_float
from paged_kv_cache_408_b200 import inputs as I
from paged_kv_cache_408_b200 import ops

pytestmark = pytest.mark.gpu


def run_cascade(c, kc, vc, prefix_blocks, ws=None, seq_lens=None, fill=0xFF):
    lens = c.seq_lens if seq_lens is None else seq_lens
    qd = dev_bf16(c.q)
    out = torch.empty_like(qd)
    B, Hq, _ = c.q.shape
    if ws is None:
        ws = ops.alloc_cascade_workspace(B, Hq, c.block_tables.shape[1], prefix_blocks, kc)
        ws.fill_(fill)  # the call needs no initialised workspace
    ks = vs = None
    if c.fp8:
        ks, vs = dev(c.k_scale, np.float32), dev(c.v_scale, np.float32)
    ops.decode_cascade(out, qd, kc, vc, dev(c.block_tables, np.int32), dev(lens, np.int32), c.scale,
                       prefix_blocks, ws, ks, vs)
    torch.cuda.synchronize()
    return to_float(out)


def oracle_of(c, rows=None, seq_lens=None):
    q, bt = c.q, c.block_tables
    lens = c.seq_lens if seq_lens is None else seq_lens
    if rows is not None:
        q, bt, lens = q[rows], bt[rows], np.asarray(lens)[rows]
    return oracle.decode(q, c.k_cache, c.v_cache, bt, lens, c.scale, c.k_scale, c.v_scale)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("fp8", [False, True])
def test_cascade_shapes(cuda_device, D, G, fp8):
    """37 sequences (ragged against the 128/G sequences of a query tile) over
    a 300-token shared prefix (18 full blocks and a shared partial one) with
    suffixes in [0, 200], some empty."""
    Hkv = 2
    c = I.prefix_share(7 + D + G + fp8, n_seqs=37, prefix=300, suffix_lo=0, suffix_hi=200, Hq=G * Hkv, Hkv=Hkv,
                       D=D, fp8=fp8)
    kc, vc = cache_to_device(c)
    ref = oracle_of(c)
    for pb in (18, 1, 7, 0):
        assert_attn_close(run_cascade(c, kc, vc, pb), ref, f"D{D} G{G} fp8={fp8} prefix_blocks={pb}")
    assert ops.get_last_device_error() == 0


@pytest.mark.parametrize("fp8", [False, True])
def test_cascade_with_no_suffix_and_whole_table_prefix(cuda_device, fp8):
    """Every key in the shared prefix: sequences of exactly 16*prefix_blocks
    tokens, and a prefix that is the whole block table."""
    c = I.prefix_share(3, n_seqs=20, prefix=128, suffix_lo=0, suffix_hi=0, Hq=32, Hkv=8, D=128, fp8=fp8)
    assert c.block_tables.shape[1] == 8 and (c.seq_lens == 128).all()
    kc, vc = cache_to_device(c)
    assert_attn_close(run_cascade(c, kc, vc, 8), oracle_of(c), "prefix = whole table")
    lens = c.seq_lens.copy()
    lens[::3] = 112  # shorter sequences that still cover 7 prefix blocks
    assert_attn_close(run_cascade(c, kc, vc, 7, seq_lens=lens), oracle_of(c, seq_lens=lens), "mixed lengths")
    assert ops.get_last_device_error() == 0


def test_cascade_single_sequence_and_long_prefix(cuda_device):
    """One sequence (one query row per kv head group) over a 5000-token prefix
    with a one-token suffix, and 3 sequences whose suffix spans many blocks."""
    c = I.prefix_share(4, n_seqs=1, prefix=5000, suffix_lo=1, suffix_hi=1, Hq=32, Hkv=8, D=128, fp8=False)
    kc, vc = cache_to_device(c)
    assert_attn_close(run_cascade(c, kc, vc, 5000 // 16), oracle_of(c), "1 seq")
    c = I.prefix_share(5, n_seqs=3, prefix=1024, suffix_lo=3000, suffix_hi=6000, Hq=64, Hkv=8, D=128, fp8=True)
    kc, vc = cache_to_device(c)
    assert_attn_close(run_cascade(c, kc, vc, 64), oracle_of(c), "long suffixes")
    assert ops.get_last_device_error() == 0


def test_cascade_workspace_reuse_across_batches(cuda_device):
    """One workspace, garbage-filled once, serves calls of several batch
    sizes and prefix lengths in turn."""
    c = I.prefix_share(6, n_seqs=40, prefix=512, suffix_lo=1, suffix_hi=300, Hq=32, Hkv=8, D=128, fp8=True)
    kc, vc = cache_to_device(c)
    n = max(ops.cascade_workspace_size(64, 32, c.block_tables.shape[1], pb, kc) for pb in (1, 16, 32))
    ws = torch.full((n,), 0xFF, dtype=torch.uint8, device=kc.device)
    ref = oracle_of(c)
    for rows, pb in (([*range(40)], 32), ([5], 32), ([3, 9, 1], 16), ([*range(0, 40, 2)], 1), ([*range(40)], 32)):
        rows = np.array(rows)
        sub = I.DecodeCase("sub", c.q[rows], c.k_cache, c.v_cache, c.block_tables[rows], c.seq_lens[rows], c.scale,
                           c.k_scale, c.v_scale)
        assert_attn_close(run_cascade(sub, kc, vc, pb, ws=ws), ref[rows], f"rows {rows.tolist()[:5]} pb {pb}")
    assert ops.get_last_device_error() == 0


def test_cascade_prefix_share_fp8_full_size_every_row(cuda_device):
    """256 sequences over one shared 2048-token prefix (128 blocks) with
    suffixes in [16, 512], 64/8 heads, fp8: every row against the oracle."""
    c = I.prefix_share(0)
    kc, vc = cache_to_device(c)
    got = run_cascade(c, kc, vc, 128)
    assert_attn_close(got, oracle_of(c), "256 x 2048 shared")
    assert ops.get_last_device_error() == 0


def test_cascade_flags_a_sequence_shorter_than_the_prefix(cuda_device):
    c = I.prefix_share(8, n_seqs=6, prefix=160, suffix_lo=5, suffix_hi=40, Hq=32, Hkv=8, D=128, fp8=False)
    kc, vc = cache_to_device(c)
    assert ops.get_last_device_error() == 0
    lens = c.seq_lens.copy()
    lens[2] = 100  # below 16 * 10 prefix tokens
    got = run_cascade(c, kc, vc, 10, seq_lens=lens)
    assert ops.get_last_device_error() & ops.DEVERR_BAD_LEN
    ok = np.array([0, 1, 3, 4, 5])
    assert_attn_close(got[ok], oracle_of(c, rows=ok), "unaffected rows")
