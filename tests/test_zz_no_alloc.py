"""pa_decode_noalloc: paged decode for callers that cannot allocate device
memory (a plugin inside an engine whose pool already owns the GPU, or code
that must avoid the implicit synchronisation of cudaMalloc/cudaFree).

It uses the library's fixed device scratch instead of a caller workspace.
The GPU test calls it through the C ABI twice in a row, with different
batches, and checks each result against pa_decode with its own workspace.
This file is collected last on purpose."""
import ctypes as C

import numpy as np
import pytest
import torch

from gpu_util import MAX_ABS, MEAN_ABS, cache_to_device, dev, dev_bf16
from paged_kv_cache_408_b200 import inputs as I
from paged_kv_cache_408_b200 import ops

PA_ERR_WORKSPACE = -3


SCRATCH_BYTES = 16 << 20  # PA_DECODE_NOALLOC_SCRATCH_BYTES


def _call_noalloc(out, q, kc, vc, bt, lens, scale, partition_tokens, ks=None, vs=None):
    desc = ops.cache_desc(kc)
    ptr = (lambda t: None if t is None else C.c_void_p(t.data_ptr()))
    return ops.lib().pa_decode_noalloc(
        ptr(out), ptr(q), ptr(kc), ptr(vc), ptr(bt), ptr(lens), q.shape[0], bt.shape[1], q.shape[1], float(scale),
        ptr(ks), ptr(vs), int(partition_tokens), C.byref(desc), C.c_void_p(torch.cuda.current_stream().cuda_stream))


def _largest_batch_that_fits(Hq, D, max_blocks, part):
    """Largest num_seqs whose pa_decode workspace fits the fixed scratch
    (sizes from pa_decode_workspace_size, host only)."""
    B = 1
    while B < 2048 and ops.decode_workspace_size(B + 1, Hq, D, max_blocks, part) <= SCRATCH_BYTES:
        B += 1
    return B


def test_the_scratch_limit_is_exact():
    """A shape needing exactly up to 16 MiB passes the size check, one row
    more is rejected with PA_ERR_WORKSPACE before any device work (the
    pointers below are never dereferenced)."""
    B = _largest_batch_that_fits(32, 128, 128, 0)
    assert ops.decode_workspace_size(B, 32, 128, 128, 0) <= SCRATCH_BYTES < ops.decode_workspace_size(B + 1, 32, 128,
                                                                                                      128, 0)
    desc = ops.CacheDesc(4096, 8, 16, 128, 0)
    fake = C.c_void_p(0x10000)
    rc = ops.lib().pa_decode_noalloc(fake, fake, fake, fake, fake, fake, B + 1, 128, 32, 0.1, None, None, 0,
                                     C.byref(desc), None)
    assert rc == PA_ERR_WORKSPACE


def test_oversized_shape_is_rejected_before_any_device_work():
    # 2048 sequences x 32 heads x 2048 blocks needs far more than the 16 MiB scratch
    desc = ops.CacheDesc(4096, 8, 16, 128, 0)
    fake = C.c_void_p(0x10000)  # never dereferenced: the size check fails first
    rc = ops.lib().pa_decode_noalloc(fake, fake, fake, fake, fake, fake, 2048, 2048, 32, 0.1, None, None, 0,
                                     C.byref(desc), None)
    assert rc == PA_ERR_WORKSPACE


@pytest.mark.gpu
def test_noalloc_matches_decode_on_two_calls_in_a_row(cuda_device):
    cases = [(I.batch64_2k(3), 0), (I.make_decode_case(4, [1, 700, 33, 1500, 16, 257], 32, 8, 128), 256)]
    for c, part in cases:
        kc, vc = cache_to_device(c)
        q = dev_bf16(c.q)
        bt = dev(c.block_tables, np.int32)
        lens = dev(c.seq_lens, np.int32)
        ref = torch.empty_like(q)
        ws = ops.alloc_workspace(c.B, c.Hq, c.D, bt.shape[1], part, device=kc.device)
        ops.decode(ref, q, kc, vc, bt, lens, c.scale, workspace=ws, partition_tokens=part)
        got = torch.full_like(q, float("nan"))
        rc = _call_noalloc(got, q, kc, vc, bt, lens, c.scale, part)
        assert rc == 0, ops.status_string(rc)
        torch.cuda.synchronize()
        err = (got.float() - ref.float()).abs()
        assert torch.isfinite(got.float()).all()
        assert err.max().item() <= MAX_ABS and err.mean().item() <= MEAN_ABS, (err.max().item(), err.mean().item())
    assert ops.get_last_device_error() == 0


@pytest.mark.gpu
def test_noalloc_fp8_and_a_shape_at_the_end_of_the_scratch(cuda_device):
    """An fp8 cache (GQA 8, tensor-core path, with its per-head scales) and a
    bf16 batch whose split-K pieces fill the scratch up to its last bytes;
    each against pa_decode with a caller workspace, and the batch one row
    larger rejected."""
    c8 = I.make_decode_case(21, [1, 300, 2048, 17, 999], 64, 8, 128, fp8=True)
    B = _largest_batch_that_fits(32, 128, 128, 0)
    rng = np.random.default_rng(22)
    cb = I.make_decode_case(23, rng.integers(1, 2049, B), 32, 8, 128, max_blocks=128)
    assert ops.decode_workspace_size(B, 32, 128, 128, 0) > SCRATCH_BYTES - (256 << 10)
    for c in (c8, cb):
        kc, vc = cache_to_device(c)
        q = dev_bf16(c.q)
        bt = dev(c.block_tables, np.int32)
        lens = dev(c.seq_lens, np.int32)
        ks = vs = None
        if c.fp8:
            ks, vs = dev(c.k_scale, np.float32), dev(c.v_scale, np.float32)
        ref = torch.empty_like(q)
        ws = ops.alloc_workspace(c.B, c.Hq, c.D, bt.shape[1], 0, device=kc.device)
        ops.decode(ref, q, kc, vc, bt, lens, c.scale, ks, vs, workspace=ws)
        got = torch.full_like(q, float("nan"))
        rc = _call_noalloc(got, q, kc, vc, bt, lens, c.scale, 0, ks, vs)
        assert rc == 0, ops.status_string(rc)
        torch.cuda.synchronize()
        err = (got.float() - ref.float()).abs()
        assert torch.isfinite(got.float()).all()
        assert err.max().item() <= MAX_ABS and err.mean().item() <= MEAN_ABS, (err.max().item(), err.mean().item())
    q1 = torch.zeros((B + 1, 32, 128), dtype=torch.bfloat16, device=cuda_device)
    bt1 = torch.zeros((B + 1, 128), dtype=torch.int32, device=cuda_device)
    l1 = torch.ones(B + 1, dtype=torch.int32, device=cuda_device)
    kc, vc = cache_to_device(cb)
    assert _call_noalloc(torch.empty_like(q1), q1, kc, vc, bt1, l1, 0.1, 0) == PA_ERR_WORKSPACE
    assert ops.get_last_device_error() == 0
