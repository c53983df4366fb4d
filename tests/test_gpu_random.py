"""GPU parity on randomly drawn small cases, several seeds: decode and chunked
prefill against the fp64 oracle over random head dims, GQA groups, kv-head
counts, cache formats, lengths (ragged against every tile size), prefixes
and split-K modes.  Each seed draws its shape from its own generator, so a
failure names a case that can be rerun alone."""
import numpy as np
import pytest

import oracle
from gpu_util import assert_attn_close, cache_to_device, run_decode, to_float
from paged_kv_cache_408_b200 import inputs as I
from paged_kv_cache_408_b200 import ops
from test_gpu_prefill import oracle_prefill, run_prefill

pytestmark = pytest.mark.gpu


def draw_heads(rng):
    D = int(rng.choice([64, 128]))
    G = int(rng.choice([1, 2, 4, 8]))
    Hkv = int(rng.integers(1, 4))
    return D, G, Hkv, bool(rng.integers(0, 2))


@pytest.mark.parametrize("seed", range(8))
def test_random_decode(cuda_device, seed):
    rng = np.random.default_rng(9100 + seed)
    D, G, Hkv, fp8 = draw_heads(rng)
    B = int(rng.integers(1, 40))
    lens = rng.integers(1, 1500, size=B).astype(np.int32)
    lens[rng.random(B) < 0.15] = int(rng.integers(1, 17))  # some rows within one block
    c = I.make_decode_case(9200 + seed, lens, G * Hkv, Hkv, D, fp8=fp8)
    kc, vc = cache_to_device(c)
    ref = oracle.decode(c.q, c.k_cache, c.v_cache, c.block_tables, c.seq_lens, c.scale, c.k_scale, c.v_scale)
    for part in (0, int(rng.choice([16, 64, 208, 512]))):  # fixed partitions: multiples of 16
        out = run_decode(c, kc, vc, partition_tokens=part)
        assert_attn_close(to_float(out), ref, f"seed {seed}: D{D} G{G} Hkv{Hkv} fp8={fp8} B{B} P={part}")
    assert ops.get_last_device_error() == 0


@pytest.mark.parametrize("seed", range(8))
def test_random_prefill(cuda_device, seed):
    rng = np.random.default_rng(9300 + seed)
    D, G, Hkv, fp8 = draw_heads(rng)
    n = int(rng.integers(1, 5))
    chunks = rng.integers(1, 260, size=n).astype(np.int32)
    prefixes = rng.integers(0, 900, size=n).astype(np.int32)
    prefixes[rng.random(n) < 0.3] = 0  # new prompts
    pc = I.make_prefill_case(9400 + seed, chunks, prefixes, G * Hkv, Hkv, D, fp8=fp8)
    out, kh, vh = run_prefill(pc)
    what = f"seed {seed}: D{D} G{G} Hkv{Hkv} fp8={fp8} chunks {chunks.tolist()} prefixes {prefixes.tolist()}"
    assert_attn_close(out, oracle_prefill(pc, kh, vh), what)
