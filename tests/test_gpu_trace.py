"""Multi-step trace replay on the GPU against the oracle.

Scheduler-planned steps of the synthetic continuous-batching traces run
through the C ABI exactly as the benchmark enqueues them (copy_blocks ->
write_kv -> decode or cascade decode with its merge -> chunked prefill, one
programmatic launch chain per step); the oracle replays the same plans.
After every step the whole K and V caches must be bit-exact (so every
copy-on-write copy ran before the write into its block, as "Continuous
batching and PagedAttention", PagedAttention: KV cache memory, requires),
and every decode and prefill output row within max-abs 1e-2 and mean-abs
1e-3 of the fp64 oracle."""
import numpy as np
import pytest

from paged_kv_cache_408_b200 import traces
from trace_util import replay

pytestmark = pytest.mark.gpu


def test_batch64_2k_trace_replay(cuda_device):
    """12 steps of the 64 x U[1,2048] trace (32/8 heads, d128, bf16):
    sequences retire after Geometric(1/256) steps and queued prompts are
    admitted, their K/V written in the step that admits them."""
    tr = traces.batch64_2k(3)
    stats = replay(tr, 12, seed=11)
    assert len(stats) == 12 and all(s["decode"] > 0 for s in stats)


def test_batch64_2k_trace_with_turnover(cuda_device):
    """A trace whose sequences end within a few steps, so that retirement,
    admission and block reuse happen in every step."""
    tr = traces.batch64_2k(4)
    for s in tr.sched.running:
        s.decode_left = int(tr.rng.integers(1, 6))
    stats = replay(tr, 10, seed=12)
    assert sum(s["retired"] for s in stats) >= 32 and sum(s["admitted"] for s in stats) >= 32


def test_prefix_share_fp8_trace_replay(cuda_device):
    """10 steps of the shared-prefix trace: 256 sequences over one 2048-token
    prefix, fp8 E4M3 cache, 64/8 heads; each step retires 32 sequences and
    forks 32 from survivors, so shared partly filled blocks are copied
    (copy_blocks) before the forked sequences' first fp8 writes, and decode
    takes the cascade over the shared prefix."""
    tr = traces.prefix_share_fp8(1)
    stats = replay(tr, 10, seed=13, expect_cascade=True)
    assert sum(s["copies"] for s in stats) > 0, "no copy-on-write copy in 10 steps"


def test_prefix_share_fp8_trace_replay_plain_decode(cuda_device):
    """The same trace with the cascade switched off: plain fp8 decode (the
    tensor-core GQA-8 path) over the forked tables."""
    tr = traces.prefix_share_fp8(2)
    stats = replay(tr, 4, seed=14, cascade=False, expect_cascade=False)
    assert sum(s["copies"] for s in stats) > 0


def test_mixed_trace_chained_steps(cuda_device):
    """The mixed continuous-batching step as the benchmark runs it: 192
    decode sequences (lognormal lengths, median 1024, capped at 8192, tables
    of 800 blocks) plus 8 prompts in prefill whose 512-token chunks attend
    their paged prefixes (U[0,4096] at step 0), under token budget 8192 --
    write -> decode -> merge -> prefill chained on one stream.  Three steps:
    every decode row and every chunk row against the oracle, caches
    bit-exact after each step."""
    tr = traces.mixed(5, headroom_steps=4)
    stats = replay(tr, 3, seed=15, attend_prefill=True)
    assert all(s["prefill_tokens"] > 0 and s["decode"] >= 192 for s in stats)
    assert stats[0]["prefill_tokens"] == 8 * 512
