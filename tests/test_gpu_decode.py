"""GPU parity: slot-mapped write, block copy and paged decode (with split-K
and its merge) against the fp64 CPU oracle, through the C ABI.

Cache bytes and copies must be bit-exact; attention outputs must be within
max-abs 1e-2 and mean-abs 1e-3 of the oracle."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import (assert_attn_close, bf16_round, cache_to_device, dev, dev_bf16, dev_u8, host_bits,
                      run_decode, to_float)
from paged_kv_cache_408_b200 import inputs as I
from paged_kv_cache_408_b200 import ops

pytestmark = pytest.mark.gpu


def oracle_decode(case, kc_host=None, vc_host=None, seq_lens=None, rows=None):
    kc = case.k_cache if kc_host is None else kc_host
    vc = case.v_cache if vc_host is None else vc_host
    lens = case.seq_lens if seq_lens is None else seq_lens
    q, bt = case.q, case.block_tables
    if rows is not None:
        q, bt, lens = q[rows], bt[rows], np.asarray(lens)[rows]
    return oracle.decode(q, kc, vc, bt, lens, case.scale, case.k_scale, case.v_scale)


# ------------------------------------------------------------------- tiny
def test_tiny_write_is_bit_exact_and_decode_matches_before_and_after(cuda_device):
    c = I.tiny_decode(0)
    kc, vc = cache_to_device(c)
    pre_lens = c.seq_lens - 1  # 5, 17, 33, 48
    out = run_decode(c, kc, vc, seq_lens=pre_lens)
    assert_attn_close(to_float(out), oracle_decode(c, seq_lens=pre_lens), "pre-write")

    ops.write_kv(dev_bf16(c.new_k), dev_bf16(c.new_v), dev(c.slot_mapping, np.int64), kc, vc)
    kh, vh = c.k_cache.copy(), c.v_cache.copy()
    oracle.write_kv(c.new_k, c.new_v, c.slot_mapping, kh, vh)
    assert np.array_equal(host_bits(kc), kh) and np.array_equal(host_bits(vc), vh)

    out = run_decode(c, kc, vc)
    assert_attn_close(to_float(out), oracle_decode(c, kh, vh), "post-write")
    assert ops.get_last_device_error() == 0


# ------------------------------------------------------------ shape sweep
LENS = [1, 2, 15, 16, 17, 31, 33, 100, 255, 256, 257, 600, 1024, 1111]


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("fp8", [False, True])
def test_decode_shapes(cuda_device, D, G, fp8):
    Hkv = 2
    c = I.make_decode_case(100 + D + 10 * G + fp8, LENS, G * Hkv, Hkv, D, fp8=fp8)
    kc, vc = cache_to_device(c)
    ref = oracle_decode(c)
    for part in (0, 16, 48, 512, 2048):
        out = run_decode(c, kc, vc, partition_tokens=part)
        assert_attn_close(to_float(out), ref, f"D{D} G{G} fp8={fp8} P={part}")
    assert ops.get_last_device_error() == 0


def test_decode_zero_length_rows_are_zero(cuda_device):
    c = I.make_decode_case(7, [0, 5, 0, 300], 8, 2, 128)
    kc, vc = cache_to_device(c)
    for part in (0, 16):
        out = to_float(run_decode(c, kc, vc, partition_tokens=part))
        assert not out[0].any() and not out[2].any()
        assert_attn_close(out, oracle_decode(c), "zero-length rows")


@pytest.mark.parametrize("part", [16, 256, 1024])
def test_fixed_partitions_are_batch_invariant(cuda_device, part):
    """With fixed partitions a sequence's output is bitwise independent of
    what else is in the batch."""
    c = I.make_decode_case(8, [700, 33, 1500, 5, 260], 32, 8, 128)
    kc, vc = cache_to_device(c)
    full = host_bits(run_decode(c, kc, vc, partition_tokens=part))
    for rows in ([2], [4, 2, 0], [1, 3]):
        rows = np.array(rows)
        sub = host_bits(run_decode(c, kc, vc, seq_lens=c.seq_lens[rows], block_tables=c.block_tables[rows],
                                   q=c.q[rows], partition_tokens=part))
        assert np.array_equal(sub, full[rows])


# --------------------------------------------------------- fp8 write, copy
def test_fp8_write_is_bit_exact(cuda_device):
    rng = np.random.default_rng(5)
    nb, Hkv, D, T = 40, 8, 128, 300
    ks = rng.uniform(0.002, 0.05, Hkv).astype(np.float32)
    vs = rng.uniform(0.002, 0.05, Hkv).astype(np.float32)
    k = I.bf16_bits(rng.standard_normal((T, Hkv, D), dtype=np.float32) * 4)
    v = I.bf16_bits(rng.standard_normal((T, Hkv, D), dtype=np.float32) * 4)
    k[0, 0, :4] = I.bf16_bits(np.float32([1e30, -1e30, 0.0, -0.0]))  # saturation and signed zero
    slots = rng.permutation(nb * 16)[:T].astype(np.int64)
    slots[::17] = -1  # padding tokens
    kh = rng.integers(0, 255, (nb, Hkv, 16, D)).astype(np.uint8)
    vh = rng.integers(0, 255, (nb, Hkv, 16, D)).astype(np.uint8)
    kd, vd = dev_u8(kh), dev_u8(vh)
    ops.write_kv(dev_bf16(k), dev_bf16(v), dev(slots, np.int64), kd, vd, dev(ks, np.float32), dev(vs, np.float32))
    oracle.write_kv(k, v, slots, kh, vh, ks, vs)
    assert np.array_equal(host_bits(kd), kh) and np.array_equal(host_bits(vd), vh)


@pytest.mark.parametrize("fp8", [False, True])
def test_copy_blocks_is_bit_exact(cuda_device, fp8):
    rng = np.random.default_rng(6)
    shape = (50, 8, 16, 128)
    if fp8:
        kh, vh = rng.integers(0, 255, shape).astype(np.uint8), rng.integers(0, 255, shape).astype(np.uint8)
        kd, vd = dev_u8(kh), dev_u8(vh)
    else:
        kh, vh = I.normal_bf16(rng, shape), I.normal_bf16(rng, shape)
        kd, vd = dev_bf16(kh), dev_bf16(vh)
    perm = rng.permutation(50)
    pairs = np.stack([perm[:12], perm[12:24]], 1).astype(np.int32)
    ops.copy_blocks(kd, vd, dev(pairs, np.int32))
    oracle.copy_blocks(kh, vh, pairs)
    assert np.array_equal(host_bits(kd), kh) and np.array_equal(host_bits(vd), vh)


# ------------------------------------------------- full-size workloads
@pytest.mark.parametrize("part", [0, 512])
def test_batch64_2k_full_size_every_row(cuda_device, part):
    """64 sequences x U[1,2048] tokens, 32/8 heads, d128, bf16: the step's
    write, then every row of the decode against the oracle (balanced split
    and fixed 512-token partitions)."""
    c = I.batch64_2k(0)
    kc, vc = cache_to_device(c)
    ops.write_kv(dev_bf16(c.new_k), dev_bf16(c.new_v), dev(c.slot_mapping, np.int64), kc, vc)
    kh, vh = c.k_cache.copy(), c.v_cache.copy()
    oracle.write_kv(c.new_k, c.new_v, c.slot_mapping, kh, vh)
    assert np.array_equal(host_bits(kc), kh) and np.array_equal(host_bits(vc), vh)
    out = to_float(run_decode(c, kc, vc, partition_tokens=part))
    assert_attn_close(out, oracle_decode(c, kh, vh), "64 x U[1,2048]")
    assert ops.get_last_device_error() == 0


def test_long_context_split_k_every_row(cuda_device):
    """16 sequences x 32768 tokens over a 40960-block pool: split-K with
    every row merged from many pieces; every row against the oracle."""
    c = I.long_context(0)
    kc, vc = cache_to_device(c)
    out = to_float(run_decode(c, kc, vc))
    assert_attn_close(out, oracle_decode(c), "16 x 32768")
    assert ops.get_last_device_error() == 0


def test_prefix_share_fp8_every_row(cuda_device):
    """256 sequences sharing a 2048-token prefix plus U[16,512] suffixes,
    64/8 heads, fp8: plain decode (tensor-core GQA-8 path), every row."""
    c = I.prefix_share(0)
    kc, vc = cache_to_device(c)
    out = to_float(run_decode(c, kc, vc))
    assert_attn_close(out, oracle_decode(c), "256 seqs, shared 2048 prefix, fp8")
    assert ops.get_last_device_error() == 0


def test_mixed_step_decode_half_every_row(cuda_device):
    """The decode half of the mixed step: 192 sequences with lognormal
    lengths (median 1024, sigma 1, capped at 8192), 32/8 heads, d128, bf16,
    block tables 512 entries wide (the 8192-token cap); the step's write,
    then every row against the oracle."""
    dc, _ = I.mixed_step(0)
    assert dc.block_tables.shape[1] == 512 and dc.seq_lens.max() <= 8192
    kc, vc = cache_to_device(dc)
    ops.write_kv(dev_bf16(dc.new_k), dev_bf16(dc.new_v), dev(dc.slot_mapping, np.int64), kc, vc)
    kh, vh = dc.k_cache.copy(), dc.v_cache.copy()
    oracle.write_kv(dc.new_k, dc.new_v, dc.slot_mapping, kh, vh)
    assert np.array_equal(host_bits(kc), kh) and np.array_equal(host_bits(vc), vh)
    out = to_float(run_decode(dc, kc, vc))
    assert_attn_close(out, oracle_decode(dc, kh, vh), "192 lognormal")
    assert ops.get_last_device_error() == 0


# ------------------------------------------------ device-side bounds checks
def test_bad_block_id_is_flagged_not_faulted(cuda_device):
    c = I.make_decode_case(9, [40, 40], 8, 2, 128, num_blocks=10)
    kc, vc = cache_to_device(c)
    assert ops.get_last_device_error() == 0
    bt = c.block_tables.copy()
    bt[1, 1] = 10_000  # outside the pool
    out = to_float(run_decode(c, kc, vc, block_tables=bt))
    assert ops.get_last_device_error() & ops.DEVERR_BAD_BLOCK
    assert_attn_close(out[:1], oracle_decode(c, rows=np.array([0])), "unaffected row")


def test_bad_slot_and_bad_length_are_flagged(cuda_device):
    c = I.tiny_decode(1)
    kc, vc = cache_to_device(c)
    sm = c.slot_mapping.copy()
    sm[0] = 32 * 16 + 3  # past the last block
    ops.write_kv(dev_bf16(c.new_k), dev_bf16(c.new_v), dev(sm, np.int64), kc, vc)
    assert ops.get_last_device_error() & ops.DEVERR_BAD_SLOT
    lens = c.seq_lens.copy()
    lens[2] = 10_000  # longer than the block table
    run_decode(c, kc, vc, seq_lens=lens)
    assert ops.get_last_device_error() & ops.DEVERR_BAD_LEN


@pytest.mark.parametrize("part", [0, 256])
def test_workspace_reuse_across_calls_and_batch_sizes(cuda_device, part):
    """One workspace serves calls of any batch size in any order, and needs
    no initialisation: it starts filled with garbage (0xff bytes: NaN
    partials, piece counts of -1) and keeps the previous call's pieces, which
    a call must never read."""
    c = I.make_decode_case(15, [1000, 40, 2048, 513, 300], 32, 8, 128)
    kc, vc = cache_to_device(c)
    ws = ops.alloc_workspace(64, 32, 128, c.block_tables.shape[1], part, device=kc.device)
    ws.fill_(0xFF)
    ref = oracle_decode(c)
    for rows in ([0, 1, 2, 3, 4], [2], [3, 0], [4, 2, 1], [1], [0, 1, 2, 3, 4]):
        rows = np.array(rows)
        qd = dev_bf16(c.q[rows])
        out = torch.empty_like(qd)
        ops.decode(out, qd, kc, vc, dev(c.block_tables[rows], np.int32), dev(c.seq_lens[rows], np.int32), c.scale,
                   workspace=ws, partition_tokens=part)
        torch.cuda.synchronize()
        assert_attn_close(to_float(out), ref[rows], f"rows {rows.tolist()}")
    assert ops.get_last_device_error() == 0


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("mag", [0.0, 2.0 ** -80, 2.0 ** -40, 64.0, 1.0e5])
def test_fp8_gqa8_q_magnitudes(cuda_device, D, mag):
    """fp8 cache with GQA 8 runs on the tensor cores with q scaled by a power
    of two into f16 range: all-zero q (uniform softmax: the mean of V), q far
    below f16's normal range, large q, and q beyond f16's largest value (short
    sequences, so that the near one-hot softmax has no near ties).

    With large q the softmax is near one-hot and each output is close to one
    V row, of magnitude up to ~4, where rounding the output to bf16 alone
    costs up to 2^-9 relative (mean-abs ~1e-3 here, measured against the
    fp64 oracle with the kernel's arithmetic emulated exactly).  The
    reference is therefore the oracle rounded to bf16, the closest a bf16
    output can be; the tolerance is unchanged."""
    lens = [1, 17, 20] if mag > 1e4 else [1, 15, 16, 33, 200, 513]
    c = I.make_decode_case(300 + D, lens, 16, 2, D, fp8=True)
    rng = np.random.default_rng(301)
    c.q = I.bf16_bits(rng.standard_normal(c.q.shape).astype(np.float32) * np.float32(mag))
    kc, vc = cache_to_device(c)
    ref = bf16_round(oracle_decode(c))
    for part in (0, 16):
        out = to_float(run_decode(c, kc, vc, partition_tokens=part))
        assert_attn_close(out, ref, f"|q| x {mag:g}, D{D}, partition {part}")
    assert ops.get_last_device_error() == 0


@pytest.mark.parametrize("Hkv", [1, 3, 4])
def test_fp8_gqa8_kv_head_counts(cuda_device, Hkv):
    """fp8 with GQA 8 (tensor-core path) with one, an odd and an even number
    of kv heads, under every partition mode."""
    c = I.make_decode_case(320 + Hkv, [1, 16, 17, 100, 700, 1500], 8 * Hkv, Hkv, 128, fp8=True)
    kc, vc = cache_to_device(c)
    ref = oracle_decode(c)
    for part in (0, 32, 512):
        assert_attn_close(to_float(run_decode(c, kc, vc, partition_tokens=part)), ref, f"Hkv {Hkv} partition {part}")
    assert ops.get_last_device_error() == 0
