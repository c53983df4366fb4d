"""GPU parity of the tcgen05 chunked-prefill kernel against the fp64 oracle.

Each case writes the chunks' own K/V into the paged cache first (pa_write_kv),
then runs pa_prefill_chunk; outputs must be within max-abs 1e-2 and mean-abs
1e-3 of the oracle's causal attention over prefix + chunk."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_attn_close, assert_attn_close_bf16, dev, dev_bf16, dev_u8, host_bits, to_float
from paged_kv_cache_408_b200 import inputs as I
from paged_kv_cache_408_b200 import ops

pytestmark = pytest.mark.gpu


def run_prefill(pc, chunks=None):
    fp8 = pc.k_scale is not None
    if fp8:
        kc, vc = dev_u8(pc.k_cache), dev_u8(pc.v_cache)
        ks, vs = dev(pc.k_scale, np.float32), dev(pc.v_scale, np.float32)
    else:
        kc, vc = dev_bf16(pc.k_cache), dev_bf16(pc.v_cache)
        ks = vs = None
    ops.write_kv(dev_bf16(pc.new_k), dev_bf16(pc.new_v), dev(pc.slot_mapping, np.int64), kc, vc, ks, vs)
    q = dev_bf16(pc.q)
    out = torch.full_like(q, float("nan"))
    ops.prefill_chunk(out, q, dev(pc.cu_q, np.int32), dev(pc.prefix_lens, np.int32), dev(pc.block_tables, np.int32),
                      kc, vc, pc.scale, max(pc.max_q_len, 1), ks, vs)
    torch.cuda.synchronize()
    assert ops.get_last_device_error() == 0
    kh, vh = pc.k_cache.copy(), pc.v_cache.copy()
    oracle.write_kv(pc.new_k, pc.new_v, pc.slot_mapping, kh, vh, pc.k_scale, pc.v_scale)
    assert np.array_equal(host_bits(kc), kh) and np.array_equal(host_bits(vc), vh)
    return to_float(out), kh, vh


def oracle_prefill(pc, kh, vh, chunks=None):
    if chunks is None:
        return oracle.prefill(pc.q, pc.cu_q, pc.prefix_lens, pc.block_tables, kh, vh, pc.scale, pc.k_scale, pc.v_scale)
    rows = np.concatenate([np.arange(pc.cu_q[c], pc.cu_q[c + 1]) for c in chunks])
    lens = np.diff(pc.cu_q)[chunks]
    cu = np.zeros(len(chunks) + 1, np.int32)
    cu[1:] = np.cumsum(lens)
    ref = oracle.prefill(pc.q[rows], cu, pc.prefix_lens[chunks], pc.block_tables[chunks], kh, vh, pc.scale,
                         pc.k_scale, pc.v_scale)
    return rows, ref


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_prefill_shapes(cuda_device, D, G):
    # ragged chunk lengths (not multiples of the 128/G-row tile), prefixes that
    # are not block aligned, a 1-token chunk without prefix
    chunks = [1, 37, 128, 200, 65]
    prefixes = [0, 5, 300, 16, 1000]
    pc = I.make_prefill_case(300 + D + G, chunks, prefixes, 2 * G, 2, D)
    out, kh, vh = run_prefill(pc)
    assert_attn_close(out, oracle_prefill(pc, kh, vh), f"prefill D{D} G{G}")


def test_prefill_long_prefix_many_tiles(cuda_device):
    pc = I.make_prefill_case(41, [300, 7], [2500, 3333], 32, 8, 128)
    out, kh, vh = run_prefill(pc)
    assert_attn_close(out, oracle_prefill(pc, kh, vh), "long prefixes")


def test_prefill_empty_chunk_is_a_no_op(cuda_device):
    pc = I.make_prefill_case(42, [0, 20], [10, 33], 8, 2, 128)
    out, kh, vh = run_prefill(pc)
    assert_attn_close(out, oracle_prefill(pc, kh, vh), "empty chunk")


def test_mixed_step_prefill_full_size_every_chunk(cuda_device):
    """8 chunks of 512 tokens over prefixes uniform in [0, 4096], 32/8 heads,
    head_dim 128: the prefill part of the mixed decode + prefill step, every
    row of every chunk against the oracle."""
    _, pc = I.mixed_step(0)
    out, kh, vh = run_prefill(pc)
    assert_attn_close(out, oracle_prefill(pc, kh, vh), "8 x 512 over U[0,4096]")


# ------------------------------------------------------------ fp8 cache
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_prefill_fp8_shapes(cuda_device, D, G):
    """An E4M3 cache with per-head scales: the chunks' own K/V quantised on
    write (bit-exact against the oracle's encoder), then the tile loads
    widen the codes to f16 in shared memory and the MMAs take f16 operands;
    ragged chunks, unaligned prefixes, a 1-token chunk without prefix."""
    pc = I.make_prefill_case(500 + D + G, [1, 37, 128, 200, 65], [0, 5, 300, 16, 1000], 2 * G, 2, D, fp8=True)
    out, kh, vh = run_prefill(pc)
    assert_attn_close(out, oracle_prefill(pc, kh, vh), f"fp8 prefill D{D} G{G}")


def test_prefill_fp8_long_prefixes_and_q_magnitudes(cuda_device):
    """Long prefixes (many key tiles, both ring slots reused), and queries
    far from unit scale: the per-row power-of-two scaling into f16 range
    must keep them exact.  With |q| x 40 the softmax is near one-hot and the
    check allows the neighbouring bf16 value (gpu_util.assert_attn_close_bf16)."""
    pc = I.make_prefill_case(541, [300, 7, 129], [2500, 3333, 0], 32, 8, 128, fp8=True)
    out, kh, vh = run_prefill(pc)
    assert_attn_close(out, oracle_prefill(pc, kh, vh), "fp8 long prefixes")
    rng = np.random.default_rng(542)
    for mag in (2.0 ** -30, 40.0):
        pc.q = I.bf16_bits(rng.standard_normal(pc.q.shape).astype(np.float32) * np.float32(mag))
        out, kh, vh = run_prefill(pc)
        assert_attn_close_bf16(out, oracle_prefill(pc, kh, vh), f"fp8, |q| x {mag:g}")


def test_prefill_fp8_mixed_step_full_size(cuda_device):
    """8 chunks of 512 over prefixes uniform in [0, 4096], 32/8 heads, d128,
    an E4M3 cache: every row against the oracle."""
    _, pc0 = I.mixed_step(0)
    pc = I.make_prefill_case(543, pc0.chunk_lens, pc0.prefix_lens, 32, 8, 128, fp8=True)
    out, kh, vh = run_prefill(pc)
    assert_attn_close(out, oracle_prefill(pc, kh, vh), "fp8 8 x 512 over U[0,4096]")
